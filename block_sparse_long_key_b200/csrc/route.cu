// Router: block scores on the tcgen05 tensor cores, per-query top-k on the
// CUDA cores.
//
// "Optimizing Mixture of Block Attention", §"Architettura del Modello
// Statistico" 1 (router score s_j = q^T k~_j) and §"Definizione del Compito"
// (each query keeps the top-k blocks, k << n); the FlashMoBA "Flash TopK"
// stage 2 (§"Progettazione del Kernel FlashMoBA", "Tre Kernel Fusi" 1) scores
// tile by tile without materialising the N x n matrix; so does this kernel.
//
// Selection rule: a query at local position p (block b = p / B) scores the
// earlier blocks j < b only, keeps the topk-1 best (exact ties: lower j
// wins) and always keeps its own block b.  sel_idx rows are sorted
// ascending and padded with -1.
//
// One CTA owns 128 consecutive queries of one sequence and one query head.
// Their Q tile sits in tensor memory (thread t writes row t, the MMA's A
// operand); a stream of centroid chunks (NC blocks each, kCB = 2 buffers,
// TMA tile loads into 128-byte-swizzled K-major shared memory) is the B operand of
// tcgen05.mma (M = 128 queries, N = NC blocks, bf16 in, fp32 accumulate into
// tensor memory, three score tiles at d = 64, two at d = 128): a producer
// warp issues the loads and q.c_hi + q.c_lo, which carries ~16 mantissa bits
// of the fp32 centroid, while the four selecting warps work on earlier chunks
// (mbarrier hand-offs per score tile, no block-wide barrier per chunk).
// Thread t owns query row t, which is TMEM lane t: tcgen05.ld hands it that
// row's NC scores in registers.  Scores above the thread's running threshold
// (the worst of its current k-1 best) go to a small per-thread candidate
// buffer in shared memory (predicated stores); the whole warp flushes the
// buffers together.  The k-1 kept entries form a binary min-heap of 64-bit
// keys (order-preserving score bits << 32 | ~block index, so a larger key is
// a better block: higher score, then lower index) in shared memory
// ([slot][thread], bank-conflict free); admitting a candidate replaces the
// root and sifts it down a fixed log2(k) levels whatever the data, one level
// (two loads) per step (a sorted list would shift up to k-1 entries, and a
// warp pays for its slowest lane).  With four CTAs per SM the candidate
// stores and admissions are bound by shared-memory bandwidth.  At the
// end each thread sorts its row's kept block indices in registers and writes
// the row.
//
// At d = 64, tiles whose rows scan at least kTwoPassMinChunks chunks run two passes over
// the chunks.  The first keeps, per row, the ceil((k-1)/2) largest of its
// chunks' second-largest scores; the smallest of those is a lower bound lb of
// the row's (k-1)-th best score (at least k-1 scores reach it).  The second
// pass replays the same MMAs (bit-identical scores) and sends to the heap
// only scores >= lb, so the selection stays exact while the heap admits ~50
// instead of ~140 scores per row of 1024 candidates.
//
// Side outputs for the forward: mref = a lower bound of the query's largest
// attention logit, max(best kept score, q_i.k_i) / sqrt(d) (a block mean never
// exceeds the block max), the fixed softmax reference of the forward; the
// query's accumulator row (oacc, flag) is zeroed here.
#include "common.cuh"
#include "launch.h"
#include "tc.cuh"

namespace moba {
namespace {

constexpr int kTM = kRouteTile;  // query rows per CTA (= TMEM lanes)
constexpr int kSel = 128;        // selecting threads: thread t owns row t (warps 0-3)
constexpr int kThreads = kSel + 32;  // + one producer warp (chunk loads, MMAs)
constexpr uint64_t kKeyMax = ~0ull;  // heap padding: never the minimum
// An empty live slot: the key of score -inf (below every finite score), so
// the root's score reads back as -inf until k-1 blocks have been admitted.
constexpr uint64_t kKeyEmpty = (uint64_t)0x007fffffu << 32;
constexpr uint32_t kFull = 0xffffffffu;
constexpr int kGroup = 4;  // columns appended between buffer checks
constexpr int kBoundList = 16;  // chunk second-maxima kept for the bound: ceil((k-1)/2) <= 16
// Tiles whose rows scan fewer chunks route in one pass: the bound needs at
// least ceil((k-1)/2) chunks and saves little on short rows.  At d = 128 the
// replayed MMAs (twice the K steps) cost more than the admissions saved
// (N = 256K, k = 16: 4.76 ms in one pass against 6.44 ms in two), so only
// d = 64 tiles take two passes.
constexpr int kTwoPassMinChunks = 16;

template <int D, int NC, int LISTN>
struct RouteLayout {
  static constexpr int NB = D == 64 ? 3 : 2;              // score tiles in tensor memory
  static constexpr int kBuf = 6;                          // candidate buffer slots per thread
  static constexpr int KB = D / 64;                       // 128-byte K blocks
  static constexpr uint32_t C_OFF = 0;
  static constexpr uint32_t C_REGION = NC * 128;
  static constexpr uint32_t C_MAT = KB * C_REGION;       // hi or lo of one chunk
  static constexpr uint32_t C_BUF = 2 * C_MAT;           // hi + lo
  static constexpr int kCB = 2;                           // chunk buffers (loads in flight)
  static constexpr uint32_t HP_OFF = C_OFF + kCB * C_BUF;         // heap keys [LISTN][kSel] u64
  static constexpr uint32_t BK_OFF = HP_OFF + LISTN * kSel * 8;  // candidates [kBuf][kSel] (score bits, index)
  // mbarriers: score tile full [NB] (MMA done), score tile empty [NB] (read
  // by the four selecting warps), chunk landed [2], Q in tensor memory.
  static constexpr uint32_t MB_OFF = BK_OFF + kBuf * kSel * 8;
  static constexpr uint32_t HOLD_OFF = MB_OFF + 8 * (2 * NB + kCB + 1);
  static constexpr uint32_t BYTES = HOLD_OFF + 16;
  // Tensor memory: NB NC-column score tiles, then Q (D bf16 = D/2 columns).
  static constexpr uint32_t TM_Q = NB * NC;
  static constexpr uint32_t TMEM_COLS = 128;
  static_assert((LISTN & (LISTN - 1)) == 0, "heap is a complete tree of LISTN - 1 nodes");
  static_assert(C_REGION % 1024 == 0, "swizzle atoms must stay 1024-byte aligned");
  static_assert(TM_Q + D / 2 <= TMEM_COLS, "score tiles and Q fit the allocation");
};

__device__ __forceinline__ uint32_t order_bits(float v) {
  const uint32_t u = __float_as_uint(v);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float from_order_bits(uint32_t u) {
  return __uint_as_float((u & 0x80000000u) ? (u & 0x7fffffffu) : ~u);
}
// Larger key = better block: higher score, then lower index.
__device__ __forceinline__ uint64_t make_key(float x, int j) {
  return ((uint64_t)order_bits(x) << 32) | (uint64_t)(0xffffffffu - (uint32_t)j);
}

// Sorts N values held by one thread ascending (bitonic network; every index
// is a compile-time constant, so the values stay in registers).
template <int N>
__device__ __forceinline__ void sort_asc(uint32_t (&a)[N]) {
#pragma unroll
  for (int k = 2; k <= N; k <<= 1)
#pragma unroll
    for (int j = k >> 1; j > 0; j >>= 1)
#pragma unroll
      for (int i = 0; i < N; ++i) {
        const int l = i ^ j;
        if (l > i) {
          const uint32_t x = a[i], y = a[l];
          const bool up = (i & k) == 0;
          a[i] = up ? min(x, y) : max(x, y);
          a[l] = up ? max(x, y) : min(x, y);
        }
      }
}

template <int D, int NC, int LISTN>
__global__ void __launch_bounds__(kThreads, 4)
route_kernel(const bf16* __restrict__ q, const bf16* __restrict__ k, const __grid_constant__ CUtensorMap tm_hi,
             const __grid_constant__ CUtensorMap tm_lo, const int32_t* __restrict__ cu,
             const int32_t* __restrict__ blk_off, const int32_t* __restrict__ tile_off, int batch,
             int nb_max, int h_q, int h_kv, int block_size, int topk, int32_t* __restrict__ sel_idx,
             float* __restrict__ mref, int32_t* __restrict__ flag, float* __restrict__ oacc, float* __restrict__ lacc,
             const float* __restrict__ cent_norm_max, int32_t* __restrict__ status) {
  using Ly = RouteLayout<D, NC, LISTN>;
  // Sift depth of a complete tree with LISTN - 1 nodes (children of the
  // deepest internal node still lie below LISTN - 1).
  constexpr int kHeapDepth = LISTN == 64 ? 5 : (LISTN == 32 ? 4 : (LISTN == 16 ? 3 : 2));
  extern __shared__ unsigned char smem_raw[];
  // 1024-byte aligned base, derived from the shared array by pointer
  // arithmetic so that accesses through it stay shared-memory accesses.
  unsigned char* sm = smem_raw + (((smem_u32(smem_raw) + 1023u) & ~1023u) - smem_u32(smem_raw));
  const uint32_t sbase = smem_u32(sm);
  uint64_t* heap = reinterpret_cast<uint64_t*>(sm + Ly::HP_OFF);
  uint2* bk = reinterpret_cast<uint2*>(sm + Ly::BK_OFF);
  const uint32_t mb_full = sbase + Ly::MB_OFF, mb_empty = mb_full + 8 * Ly::NB;
  const uint32_t mb_c0 = mb_empty + 8 * Ly::NB, mb_q = mb_c0 + 8 * Ly::kCB;
  mark_path(status, kPathRouteTc);

  const int ntiles = __ldg(tile_off + batch);
  // Longest rows first, every head's together: a CTA's time grows with its
  // rows' position, so the grid ends on short tiles.
  const int h = (int)(blockIdx.x % (unsigned)h_q);
  const int tile = ntiles - 1 - (int)(blockIdx.x / (unsigned)h_q);
  if (tile < 0) return;
  const int kvh = h / (h_q / h_kv);
  const int s = upper_seq(tile_off, batch, tile);
  const int seq0 = __ldg(cu + s);
  const int L = __ldg(cu + s + 1) - seq0;
  const int p0 = (tile - __ldg(tile_off + s)) * kTM;
  const int nrows = min(kTM, L - p0);
  const int t0 = seq0 + p0;
  const int cbase = __ldg(blk_off + s);
  const int k1 = topk - 1;
  const int nscan = k1 > 0 ? (p0 + nrows - 1) / block_size : 0;  // blocks any row may score
  const int nchunks = (nscan + NC - 1) / NC;
  // Two passes over the chunks when the rows are long enough: the first only
  // computes a lower bound of each row's (k-1)-th best score, the second
  // replays the same MMAs (bit-identical scores) and admits into the heap
  // only the scores at or above that bound.  See pass_one below.
  const int k2 = (k1 + 1) / 2;
  const bool two_pass = D == 64 && LISTN == 32 && k1 >= 2 && nchunks >= kTwoPassMinChunks;
  const int nsteps = two_pass ? 2 * nchunks : nchunks;
  auto chunk_of = [&](int st) { return st < nchunks ? st : st - nchunks; };
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const size_t qstride = (size_t)h_q * D;

  // ---- loads: centroid chunks (hi, lo) into SW128 K-major layout by the
  // TMA (the producer thread): rows = global blocks of this KV head, boxes of
  // NC rows x 64 values; rows past `nscan` (the next sequence's or head's
  // blocks, or beyond the table: zero) are scored but never selected.
  const int crow0 = kvh * nb_max + cbase;
  // The screen pass (step < nchunks of a two-pass tile) needs only the hi halves.
  auto load_chunk = [&](int c, int buf, bool hi_only) {
    tc::mbar_arrive_expect_tx(mb_c0 + 8 * buf, (hi_only ? 1 : 2) * Ly::C_MAT);
#pragma unroll
    for (int r = 0; r < Ly::KB; ++r) {
      const uint32_t dst = sbase + Ly::C_OFF + buf * Ly::C_BUF + r * Ly::C_REGION;
      tc::tma_load_2d(dst, &tm_hi, r * 64, crow0 + c * NC, mb_c0 + 8 * buf);
      if (!hi_only) tc::tma_load_2d(dst + Ly::C_MAT, &tm_lo, r * 64, crow0 + c * NC, mb_c0 + 8 * buf);
    }
  };

  // ---- per-thread selection state; TMEM + barriers
  const bool sel_thread = tid < kSel;
  const bool row_ok = tid < nrows;
  const int my_b = row_ok ? (p0 + tid) / block_size : 0;
  // Min-heap of the kept keys: k1 live slots start empty (score -inf),
  // padding slots up to LISTN-1 hold kKeyMax and never surface.
  if (sel_thread)
    for (int sl = 0; sl < LISTN; ++sl) heap[sl * kSel + tid] = sl < k1 ? kKeyEmpty : kKeyMax;
  uint64_t root_key = kKeyEmpty;  // heap slot 0, the root: the worst kept key
  // Slots 1 and 2 (the root's children) live in registers as well, so an
  // admission touches shared memory from the third level on.
  uint64_t h1 = 1 < k1 ? kKeyEmpty : kKeyMax, h2 = 2 < k1 ? kKeyEmpty : kKeyMax;
  float tau = -INFINITY;          // its score
  float lb = -INFINITY;           // the first pass's lower bound (two-pass tiles)
  // Candidates pass when x > thr = max(tau, the float just below lb): x > tau
  // (strict: blocks arrive in ascending j, so a score equal to the root's,
  // which has a lower index, never wins) and x >= lb in one compare.
  float thr = -INFINITY;
  int cnt = 0;                    // buffered candidate keys
  if (tid == 0) {
    for (int i = 0; i < Ly::NB; ++i) {
      tc::mbar_init(mb_full + 8 * i, 1);
      tc::mbar_init(mb_empty + 8 * i, kSel / 32);
    }
    for (int b = 0; b < Ly::kCB; ++b) tc::mbar_init(mb_c0 + 8 * b, 1);
    tc::mbar_init(mb_q, kSel / 32);
    tc::mbar_init_fence();
  }
  if (nchunks > 0 && warp == 0) tc::tmem_alloc(sbase + Ly::HOLD_OFF, Ly::TMEM_COLS);

  // Zero this tile's accumulator rows (O and l) while the loads fly.
  constexpr int OS = oacc_stride(D);
  for (int i = tid; i < nrows * (OS / 4); i += kThreads) {
    const int r = i / (OS / 4), c = i % (OS / 4);
    const size_t row = (size_t)(t0 + r) * h_q + h;
    reinterpret_cast<float4*>(oacc + row * OS)[c] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
  if (tid < nrows) lacc[(size_t)(t0 + tid) * h_q + h] = 0.f;
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const bool producer = tid == kSel;  // lane 0 of the last warp
  auto screen_step = [&](int st) { return two_pass && st < nchunks; };
  if (producer)
    for (int b = 0; b < Ly::kCB && b < nsteps; ++b) load_chunk(chunk_of(b), b, screen_step(b));
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(sm + Ly::HOLD_OFF);
  constexpr uint32_t idesc = tc::idesc_bf16_f32(kTM, NC);
  const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
  float qn2 = 0.f;  // |q|^2 of the thread's row
  if (nchunks > 0 && sel_thread) {
    // Q row `tid` -> TMEM lane `tid`, columns TM_Q .. TM_Q + D/2 (bf16 pairs).
    const bf16* qrow = q + (size_t)(t0 + tid) * qstride + (size_t)h * D;
#pragma unroll
    for (int half = 0; half < D / 64; ++half) {
      uint32_t w[32];  // (the row's squared norm accumulates in qn2 on the way)
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        const uint4 u = row_ok ? __ldg(reinterpret_cast<const uint4*>(qrow + half * 64 + c * 8)) : make_uint4(0, 0, 0, 0);
        float f[8];
        bf16x8_to_f32(u, f);
#pragma unroll
        for (int i = 0; i < 8; ++i) qn2 = fmaf(f[i], f[i], qn2);
        w[4 * c] = u.x;
        w[4 * c + 1] = u.y;
        w[4 * c + 2] = u.z;
        w[4 * c + 3] = u.w;
      }
      tc::tmem_st32(tmem + lane_base + Ly::TM_Q + half * 32, w);
    }
    tc::tmem_st_wait();
    tc::fence_before_sync();
    __syncwarp();
    if (lane == 0) tc::mbar_arrive(mb_q);
  }

  // Admit a key above the root: replace the root and sift it down.
  // Admits `key` when `go` (branch-free: a thread with nothing to admit
  // walks the same instructions with every store switched off).
  auto admit = [&](uint64_t key, bool go) {
    // level 0: the root's children, in registers
    const bool left0 = h1 < h2;
    const uint64_t km0 = left0 ? h1 : h2;
    const bool up0 = go && km0 < key;
    const uint64_t root = up0 ? km0 : key;  // the new minimum
    int pos = up0 ? (left0 ? 1 : 2) : 0;
    bool done = !up0;
    // level 1: the children of register slot pos (slots 3 .. 6); what moves
    // up, or the key itself, goes into that register
    uint64_t r1 = key;
    {
      const int c1 = 2 * pos + 1;  // (pos 0: slots 1 and 2 of shared memory, stale and unused)
      const uint64_t k1v = heap[c1 * kSel + tid];
      const uint64_t k2v = heap[(c1 + 1) * kSel + tid];
      const bool left = k1v < k2v;
      const uint64_t km = left ? k1v : k2v;
      if (!done && km < key) {
        r1 = km;
        pos = left ? c1 : c1 + 1;
      } else {
        done = true;
      }
    }
    h1 = up0 && left0 ? r1 : h1;
    h2 = up0 && !left0 ? r1 : h2;
    // Deeper levels in shared memory, one level per step, two loads each:
    // with 16 selecting warps per SM the admissions are bound by
    // shared-memory bandwidth, not by the chain of dependent loads (loading
    // the four grandchildren with the children, two levels per step, costs
    // 50 % more loads and measured no faster).
#pragma unroll
    for (int lvl = 2; lvl < kHeapDepth; ++lvl) {
      const int c1 = 2 * pos + 1;
      const uint64_t k1v = heap[c1 * kSel + tid];
      const uint64_t k2v = heap[(c1 + 1) * kSel + tid];
      const bool left = k1v < k2v;
      const uint64_t km = left ? k1v : k2v;
      if (!done && km < key) {
        heap[pos * kSel + tid] = km;
        pos = left ? c1 : c1 + 1;
      } else {
        done = true;
      }
    }
    if (go) {
      if (pos >= 3) heap[pos * kSel + tid] = key;  // slots 0 .. 2 took it above
      root_key = root;
      tau = from_order_bits((uint32_t)(root >> 32));
      thr = fmaxf(tau, nextafterf(lb, -INFINITY));
    }
  };
  // One round: every thread with buffered keys admits its latest one (full
  // keys are compared, so the order of admission does not matter).  Rounds
  // run only while some thread's buffer is close to full, so most threads
  // have work in each of them.
  // Candidates wait in the buffer as (score bits, block index); the heap key
  // is built only for the one a round admits.
  auto flush_round = [&]() {
    const bool has = cnt > 0;
    cnt -= has ? 1 : 0;
    const uint2 e = bk[cnt * kSel + tid];  // slot 0 when empty: read, not used
    const uint64_t key = make_key(__uint_as_float(e.x), (int)e.y);
    admit(key, has && key > root_key);
  };

  // Lower bound of the row's (k-1)-th best score (first pass).  The row
  // keeps the k2 = ceil((k-1)/2) largest of its chunks' second-largest
  // scores; the k2-th of them, lb, is met or beaten by at least two scores in
  // each of k2 chunks, so at least k-1 scores of the row are >= lb: every
  // block of the row's top k-1 has a score >= lb, and a second pass that
  // admits only scores >= lb still selects exactly (the second pass replays
  // the same MMAs, so its scores are bit-identical).  On N(0, 1)-like scores
  // about 50 of 1024 scores pass it, against ~140 heap admissions for a plain
  // running threshold.

  const int wmin_b = __shfl_sync(kFull, my_b, 0);  // smallest own block of the warp's rows (lane 0's)

  // Selection on one chunk's scores: those above the row's threshold (and
  // the first pass's bound) go to the candidate buffer, which the warp
  // flushes into the heaps in rounds.
  auto select_scores = [&](uint32_t (&v)[NC], int c) {
    const int jbase = c * NC;
    if (jbase + NC > wmin_b) {  // blocks at or after a row's own block lie in this chunk
      const int lim = my_b - jbase;
#pragma unroll
      for (int col = 0; col < NC; ++col) v[col] = col < lim ? v[col] : 0xff800000u;  // -inf
    }
#pragma unroll
    for (int g = 0; g < NC / kGroup; ++g) {
      while (__any_sync(kFull, cnt > Ly::kBuf - kGroup)) flush_round();  // room for the next group
#pragma unroll
      for (int e = 0; e < kGroup; ++e) {
        const int col = g * kGroup + e;
        // Predicated store (slot cnt is free: cnt < kBuf here).  Only a few
        // per cent of the scores pass, and shared-memory bandwidth, shared
        // with the heap admissions, limits the selection: a lane that does
        // not store takes no bandwidth.
        if (__uint_as_float(v[col]) > thr) {
          bk[cnt * kSel + tid] = make_uint2(v[col], (uint32_t)(jbase + col));
          ++cnt;
        }
      }
    }
  };

  // Producer (one thread): chunk c's MMAs go into score tile c % NB once the
  // chunk has landed and the four selecting warps have read the tile's
  // previous contents; the load of chunk c + 1 reuses the shared-memory
  // buffer of chunk c - 1 once that chunk's MMAs are done.  Selecting warps:
  // wait for tile c % NB, read it into registers, release it, select.  No
  // block-wide barrier inside the loop, so the warps drift apart by up to NB
  // chunks.  Every wait is bounded and decided warp-wide; one that gives up
  // ends the loop, and the block agrees on the outcome afterwards.
  bool ok = true;
  if (producer && nsteps > 0) {
    ok = tc::mbar_wait(mb_q, 0);
    // step c of the (one or two) passes: chunk chunk_of(c)
    for (int c = 0; c < nsteps && ok; ++c) {
      const int buf = c % Ly::kCB, sc = c % Ly::NB;
      if (c >= 1 && c + Ly::kCB - 1 < nsteps) {
        // chunk c - 1's MMAs are done with its buffer: load chunk c + kCB - 1 there
        const int pc = c - 1;
        if (!(ok = tc::mbar_wait(mb_full + 8 * (pc % Ly::NB), (pc / Ly::NB) & 1))) break;
        load_chunk(chunk_of(c + Ly::kCB - 1), pc % Ly::kCB, screen_step(c + Ly::kCB - 1));
      }
      if (!(ok = tc::mbar_wait(mb_c0 + 8 * buf, (c / Ly::kCB) & 1))) break;
      if (c >= Ly::NB && !(ok = tc::mbar_wait(mb_empty + 8 * sc, ((c / Ly::NB) - 1) & 1))) break;
      tc::fence_after_sync();
      const uint32_t d_tmem = tmem + (uint32_t)(sc * NC);
      const uint32_t qa = tmem + Ly::TM_Q;  // lane 0, Q columns
      const uint32_t ca = sbase + Ly::C_OFF + buf * Ly::C_BUF;
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint32_t koff = (kk & 3) * 32;  // 16 bf16 per K step inside a 128-byte row
        tc::mma_bf16_ts(d_tmem, qa + kk * 8, tc::sw128_desc(ca + (kk >> 2) * Ly::C_REGION + koff), idesc, kk > 0);
      }
      if (!screen_step(c)) {
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t koff = (kk & 3) * 32;
          tc::mma_bf16_ts(d_tmem, qa + kk * 8, tc::sw128_desc(ca + Ly::C_MAT + (kk >> 2) * Ly::C_REGION + koff),
                          idesc, 1u);
        }
      }
      tc::mma_commit(mb_full + 8 * sc);
    }
  } else if (sel_thread) {
    // Waits for score tile c % NB, reads it into registers and releases it.
    auto take_tile = [&](int c, uint32_t (&v)[NC]) -> bool {
      const int sc = c % Ly::NB;
      const bool got = tc::mbar_wait(mb_full + 8 * sc, (c / Ly::NB) & 1);
      if (!__all_sync(kFull, got)) return false;
      tc::fence_after_sync();
      const uint32_t taddr = tmem + lane_base + (uint32_t)(sc * NC);
#pragma unroll
      for (int hf = 0; hf < NC / 32; ++hf)
        tc::tmem_ld32(taddr + hf * 32, *reinterpret_cast<uint32_t(*)[32]>(&v[hf * 32]));
      tc::tmem_ld_wait();
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(mb_empty + 8 * sc);
      return true;
    };
    int c = 0;
    if (two_pass) {
      // First pass: the bound.  Every chunk of NC blocks contributes its
      // second-largest score m2 (masked to the row's earlier blocks); the row
      // keeps the kBoundList largest m2 in a descending register list.
      float top2[kBoundList];
#pragma unroll
      for (int i = 0; i < kBoundList; ++i) top2[i] = -INFINITY;
      for (; c < nchunks; ++c) {
        uint32_t v[NC];
        if (!take_tile(c, v)) {
          ok = false;
          break;
        }
        const int jbase = c * NC;
        if (jbase + NC > wmin_b) {  // blocks at or after the row's own block count as -inf
          const int lim = my_b - jbase;
#pragma unroll
          for (int col = 0; col < NC; ++col) v[col] = col < lim ? v[col] : 0xff800000u;
        }
        // second-largest of the chunk: pairwise (hi, lo), then merged top-2 lists
        float hi[NC / 2], lo[NC / 2];
#pragma unroll
        for (int i = 0; i < NC / 2; ++i) {
          const float a = __uint_as_float(v[2 * i]), b = __uint_as_float(v[2 * i + 1]);
          hi[i] = fmaxf(a, b);
          lo[i] = fminf(a, b);
        }
#pragma unroll
        for (int w = NC / 4; w >= 1; w >>= 1)
#pragma unroll
          for (int i = 0; i < w; ++i) {
            const float h2 = fmaxf(hi[i], hi[i + w]);
            lo[i] = fmaxf(fminf(hi[i], hi[i + w]), fmaxf(lo[i], lo[i + w]));
            hi[i] = h2;
          }
        const float m2 = lo[0];
        // insert m2 into the descending list, dropping its smallest entry
#pragma unroll
        for (int i = kBoundList - 1; i >= 1; --i) top2[i] = fmaxf(top2[i], fminf(top2[i - 1], m2));
        top2[0] = fmaxf(top2[0], m2);
      }
      // the k2-th largest: the list is descending, so the least of its first k2
      lb = INFINITY;
#pragma unroll
      for (int i = 0; i < kBoundList; ++i) lb = i < k2 ? fminf(lb, top2[i]) : lb;
      // The screen scored q . c_hi; the exact score adds q . c_lo and its
      // fp32 rounding.  |q . c_lo| <= |q| |c_lo| <= 2^-9 (1 + 2^-9) |q| |c|
      // (c_lo is c - c_hi rounded to bf16), and the added accumulation steps
      // round far below 2^-14 |q| |c|: lowering the bound by
      // E = |q| max_j |c_j| (2^-9 + 2^-14), rounded down, keeps it below the
      // exact scores of the k - 1 blocks that reached it in the screen.
      const float err = sqrtf(qn2) * __ldg(cent_norm_max + kvh) * (0.001953125f + 0.00006103515625f) * 1.0001f;
      lb = __fsub_rd(lb, err);
      thr = fmaxf(tau, nextafterf(lb, -INFINITY));
    }
    // (Second) pass: selection into the heap.
    for (; ok && c < nsteps; ++c) {
      uint32_t v[NC];
      if (!take_tile(c, v)) {
        ok = false;
        break;
      }
      select_scores(v, chunk_of(c));
    }
    if (ok)
      while (__any_sync(kFull, cnt > 0)) flush_round();
  }
  tc::fence_before_sync();
  ok = __syncthreads_and(ok);
  if (!ok) {
    // A wait gave up: record it, give the MMAs and chunk loads in flight a
    // bounded chance to drain (a wait on a phase that is not pending returns
    // at once), release TMEM, leave outputs unwritten.
    if (tid == 0) set_status(status, kStatusTimeout);
    if (producer) {
      for (int i = 0; i < Ly::NB; ++i)
        for (int ph = 0; ph < 2; ++ph) tc::mbar_wait(mb_full + 8 * i, ph, 20000000ull);
      for (int b2 = 0; b2 < Ly::kCB; ++b2)
        for (int ph = 0; ph < 2; ++ph) tc::mbar_wait(mb_c0 + 8 * b2, ph, 20000000ull);
    }
    __syncthreads();
    if (nchunks > 0 && warp == 0) tc::tmem_dealloc(tmem, Ly::TMEM_COLS);
    return;
  }
  if (nchunks > 0 && warp == 0) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, Ly::TMEM_COLS);
  }

  // Each thread writes its own row: the kept keys (live heap slots holding a
  // real key) become block indices, sorted ascending in registers, followed
  // by the own block and -1 padding.
  float best_mine = -INFINITY;
  if (row_ok) {
    uint32_t ix[LISTN];
    uint64_t top = 0ull;
    int kept_n = 0;
#pragma unroll
    for (int sl = 0; sl < LISTN; ++sl) {
      const uint64_t key =
          sl >= k1 ? kKeyEmpty : (sl == 0 ? root_key : (sl == 1 ? h1 : (sl == 2 ? h2 : heap[sl * kSel + tid])));
      const bool real = key != kKeyEmpty;
      kept_n += real;
      ix[sl] = real ? 0xffffffffu - (uint32_t)key : 0x7fffffffu;  // block index; empty slots sort last
      top = real && key > top ? key : top;
    }
    if (top) best_mine = from_order_bits((uint32_t)(top >> 32));
    sort_asc<LISTN>(ix);
    int32_t* out = sel_idx + ((size_t)(t0 + tid) * h_q + h) * topk;
    auto val = [&](int i) -> int32_t { return i < kept_n ? (int32_t)ix[i] : (i == kept_n ? my_b : -1); };
    if ((topk & 3) == 0) {
#pragma unroll
      for (int i = 0; i < LISTN; i += 4)
        if (i < topk) *reinterpret_cast<int4*>(out + i) = make_int4(val(i), val(i + 1), val(i + 2), val(i + 3));
    } else {
#pragma unroll
      for (int i = 0; i < LISTN; ++i)
        if (i < topk) out[i] = val(i);
    }
  }

  if (row_ok) {
    const int t = t0 + tid;
    const size_t row = (size_t)t * h_q + h;
    const bf16* qrow = q + (size_t)t * qstride + (size_t)h * D;
    const bf16* krow = k + ((size_t)t * h_kv + kvh) * D;
    float dot = 0.f;
#pragma unroll 4
    for (int c8 = 0; c8 < D / 8; ++c8) {
      float fk[8], fq[8];
      bf16x8_to_f32(__ldg(reinterpret_cast<const uint4*>(krow + c8 * 8)), fk);
      bf16x8_to_f32(__ldg(reinterpret_cast<const uint4*>(qrow + c8 * 8)), fq);
#pragma unroll
      for (int i = 0; i < 8; ++i) dot = fmaf(fq[i], fk[i], dot);
    }
    mref[row] = fmaxf(best_mine, dot) * rsqrtf((float)D);
    flag[row] = 0;
  }
}

template <int D, int NC, int LISTN>
cudaError_t launch_route_t(const bf16* q, const bf16* k, const bf16* hi, const bf16* lo, const float* cnorm,
                           const SeqPlan& p, int h_q, int h_kv, int block_size, int topk, int32_t* sel, float* mref,
                           int32_t* flag, float* oacc, float* lacc, int32_t* status, cudaStream_t st) {
  const size_t smem = RouteLayout<D, NC, LISTN>::BYTES + 1024;
  auto kern = route_kernel<D, NC, LISTN>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int max_tiles = p.total_tokens / kTM + p.batch;
  if (max_tiles == 0 || p.nb_max == 0) return cudaSuccess;
  CUtensorMap tm_hi, tm_lo;  // the centroid tables as h_kv * nb_max rows of D
  const unsigned long long nrows = (unsigned long long)h_kv * p.nb_max;
  e = make_row_map(&tm_hi, hi, nrows, D, NC);
  if (e != cudaSuccess) return e;
  e = make_row_map(&tm_lo, lo, nrows, D, NC);
  if (e != cudaSuccess) return e;
  dim3 grid(max_tiles * h_q);
  kern<<<grid, kThreads, smem, st>>>(q, k, tm_hi, tm_lo, p.cu, p.blk_off, p.tile_off, p.batch, p.nb_max, h_q,
                                     h_kv, block_size, topk, sel, mref, flag, oacc, lacc, cnorm, status);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_route(const bf16* q, const bf16* k, const bf16* hi, const bf16* lo, const float* cnorm,
                         const SeqPlan& p, int h_q, int h_kv, int d, int block_size, int topk, int32_t* sel,
                         float* mref, int32_t* flag, float* oacc, float* lacc, int32_t* status, cudaStream_t st) {
  const int k1 = topk - 1;
#define MOBA_ROUTE(DD, NCC, LN) \
  return launch_route_t<DD, NCC, LN>(q, k, hi, lo, cnorm, p, h_q, h_kv, block_size, topk, sel, mref, flag, oacc, lacc, \
                                     status, st)
  if (d == 64) {
    if (k1 <= 32) MOBA_ROUTE(64, 32, 32);
    MOBA_ROUTE(64, 32, 64);
  } else {
    if (k1 <= 32) MOBA_ROUTE(128, 32, 32);
    MOBA_ROUTE(128, 32, 64);
  }
#undef MOBA_ROUTE
}

}  // namespace moba
