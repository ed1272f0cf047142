// Host check of the attention kernels' CTA dispatch order (bucket_order):
// for every shape and lead, the grid visits each (key block, KV head) once,
// head h's first nb_max / 8 blocks come `lead` head-windows before its other
// blocks, and lead = 0 is plain head-major order; bucket_lead's choices on
// a few head sizes.  Prints "ok" or the first failure.
#include <cstdio>
#include <vector>

#include "common.cuh"
#include "launch.h"

int main() {
  const int nbs[] = {1, 2, 3, 7, 8, 9, 16, 100, 2049, 4097};
  for (int nb : nbs)
    for (int hkv = 1; hkv <= 16; hkv *= 2)
      for (int lead = 0; lead <= 3; ++lead) {
        std::vector<int> seen((size_t)nb * hkv, -1);
        const int big = nb / 8 > 1 ? nb / 8 : 1;
        for (int L = 0; L < nb * hkv; ++L) {
          const moba::BucketOrder o = moba::bucket_order(L, nb, hkv, lead);
          if (o.gb < 0 || o.gb >= nb || o.kvh < 0 || o.kvh >= hkv) {
            std::printf("out of range: nb %d hkv %d lead %d L %d -> (%d, %d)\n", nb, hkv, lead, L, o.gb, o.kvh);
            return 1;
          }
          int& s = seen[(size_t)o.kvh * nb + o.gb];
          if (s >= 0) {
            std::printf("visited twice: nb %d hkv %d lead %d (%d, %d)\n", nb, hkv, lead, o.gb, o.kvh);
            return 1;
          }
          s = L;
          if (lead == 0 && (o.kvh != L / nb || o.gb != L % nb)) {
            std::printf("lead 0 is not head-major: nb %d hkv %d L %d\n", nb, hkv, L);
            return 1;
          }
        }
        // A head's long blocks are all issued before its first short block.
        for (int h = 0; h < hkv; ++h) {
          int last_long = -1, first_short = 1 << 30;
          for (int gb = 0; gb < nb; ++gb) {
            const int L = seen[(size_t)h * nb + gb];
            if (gb < big) last_long = L > last_long ? L : last_long;
            else first_short = L < first_short ? L : first_short;
          }
          if (last_long > first_short) {
            std::printf("long after short: nb %d hkv %d lead %d head %d\n", nb, hkv, lead, h);
            return 1;
          }
        }
      }
  // The lead: as many head windows as let the extra heads' accumulators
  // share half of L2 with the current head's, at most 2.
  struct LeadCase { long long rows; int row_bytes, want; };
  const LeadCase lc[] = {
      {65536, 64 * 4 + 4, 2},        // 17 MB per head (N = 64K, d = 64)
      {16384, 128 * 4 + 4, 2},       // 8.5 MB (N = 16K, d = 128)
      {262144, 128 * 4 + 4, 0},      // 135 MB (N = 256K, d = 128)
      {122880 * 4, 128 * 4 + 4, 0},  // GQA 4:1, 254 MB per KV head
      {40000, 256 * 4, 0},           // 41 MB: one extra head would not fit
      {30000, 256 * 4, 1},           // 31 MB
      {0, 256, 0}};
  for (const LeadCase& c : lc)
    if (moba::bucket_lead(c.rows, c.row_bytes) != c.want) {
      std::printf("bucket_lead(%lld, %d) = %d, want %d\n", c.rows, c.row_bytes, moba::bucket_lead(c.rows, c.row_bytes),
                  c.want);
      return 1;
    }
  std::printf("ok\n");
  return 0;
}
