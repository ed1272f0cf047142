// Forward sparse attention on the tcgen05 tensor cores.
//
// "Optimizing Mixture of Block Attention", §"Definizione del Compito"
// (O = softmax(QK^T/sqrt(d)) V over the selected blocks only) and
// §"Progettazione del Kernel FlashMoBA", "Tre Kernel Fusi" 2 (gather the
// queries that chose a key block into dense tiles, dense GEMMs against the
// block, scatter the results).
//
// One CTA per (global key block j, KV head) walks the block's bucket in
// tiles of 128 gathered rows; thread t owns tile row t = TMEM lane t.  K_j
// and V_j arrive once, by TMA tile loads (64 channels x B tokens per box,
// 128-byte swizzle); rows of a partial last block are zeroed in shared
// memory before use.
//   1. Q rows are gathered by the TMA (tile::gather4, four rows per
//      instruction, 128-byte swizzle) into a K-major tile; completion is
//      counted in bytes on an mbarrier.
//   2. One thread issues S = Q K_j^T (M = 128, N = B, K = d).
//   3. Each thread reads its S row, applies the causal cut of the own block
//      and p = exp(z - M_i) against the row's fixed reference M_i (from the
//      router), sums l, checks the overflow bound and stores P as bf16.
//      The next tile's gather starts here: the Q tile is free once S is.
//   4. One thread issues O = P V_j (M = 128, N = d, K = B; V_j read
//      N-major) into the columns S used.
//   5. Each thread adds its row's l to the query's fp32 l; the O rows leave
//      through the (now free) P tile: each warp stages 32-column pieces of
//      its 32 rows there, then 8 lanes cover one 128-byte row piece per
//      16-byte vector reduction into the query's fp32 accumulator row (d
//      floats), so an instruction touches 4 rows, not 16 (one line each).
// The merge of a query's k blocks is therefore a plain sum; finalize divides
// by l.  Block sizes 16 .. 128: the P tile uses the 32-, 64- or 128-byte
// swizzle (two 128-byte regions at B = 128).  A CTA needs ~41 KB of shared
// memory and 64 TMEM columns at d = 64, B = 32, so five share an SM and
// overlap their phases.  Every mbarrier wait is bounded; a timeout sets
// MOBA_STATUS_TIMEOUT and the CTA winds down.
#include "common.cuh"
#include "launch.h"
#include "tc.cuh"

namespace moba {
namespace {

constexpr int kRows = 128;  // gathered rows per tile (= TMEM lanes)
constexpr int kThreads = 128;
constexpr float kOverflowLog2 = 90.f;  // ~62 in natural-log units

template <int D, int BLK>
struct FwdTcLayout {
  using PT = tc::KeyTile<BLK>;
  static constexpr int KB = D / 64;                          // 64-wide d chunks (128-byte rows)
  static constexpr uint32_t KV_REGION = BLK * 128;           // one d chunk of K_j or V_j
  static constexpr uint32_t Q_REGION = kRows * 128;          // one d chunk of the Q tile
  static constexpr uint32_t K_OFF = 0;
  static constexpr uint32_t V_OFF = K_OFF + KB * KV_REGION;
  static constexpr uint32_t Q_OFF = V_OFF + KB * KV_REGION;
  static constexpr uint32_t P_OFF = Q_OFF + KB * Q_REGION;
  // The P tile, grown to 16 KB where it is smaller, doubles as the staging
  // area of the O reductions (its first 16 KB: 32 rows x 128 bytes per warp).
  static constexpr uint32_t STG_BYTES = 16384;
  static constexpr uint32_t P_AREA = PT::BYTES < STG_BYTES ? STG_BYTES : PT::BYTES;
  static constexpr uint32_t MB_OFF = P_OFF + P_AREA;    // mbS, mbO, mbQ, mbKV
  static constexpr uint32_t HOLD_OFF = MB_OFF + 32;
  static constexpr uint32_t BYTES = HOLD_OFF + 16;
  static constexpr uint32_t KV_TX = 2 * KB * KV_REGION;      // bytes of one K_j + V_j load
  // Tensor memory: S (B columns), later overwritten by O (D columns).
  static constexpr uint32_t NCOLS = BLK > D ? BLK : D;
  static constexpr uint32_t TMEM_COLS = NCOLS <= 32 ? 32 : (NCOLS <= 64 ? 64 : (NCOLS <= 128 ? 128 : 256));
  static_assert(KV_REGION % 1024 == 0 && PT::REGION % 1024 == 0 && Q_REGION % 1024 == 0,
                "swizzle atoms stay aligned");
};

template <int D, int BLK>
__global__ void __launch_bounds__(kThreads)
fwd_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
              const __grid_constant__ CUtensorMap tm_v, const int32_t* __restrict__ cu,
              const int32_t* __restrict__ blk_off, int batch, int nb_max, int h_q, int h_kv, int lead,
              const int32_t* __restrict__ ptr, const int32_t* __restrict__ rows, const float* __restrict__ mref,
              float* __restrict__ oacc, float* __restrict__ lacc, int32_t* __restrict__ flag,
              int32_t* __restrict__ status) {
  using Ly = FwdTcLayout<D, BLK>;
  using PT = typename Ly::PT;
  constexpr int OS = oacc_stride(D);
  constexpr int CW = BLK < 32 ? BLK : 32;  // S columns per TMEM load
  extern __shared__ unsigned char smem_raw[];
  // 1024-byte aligned base, derived from the shared array by pointer
  // arithmetic so that accesses through it stay shared-memory accesses.
  unsigned char* sm = smem_raw + (((smem_u32(smem_raw) + 1023u) & ~1023u) - smem_u32(smem_raw));
  const uint32_t sbase = smem_u32(sm);
  const uint32_t mb_s = sbase + Ly::MB_OFF, mb_o = mb_s + 8, mb_q = mb_s + 16, mb_kv = mb_s + 24;
  mark_path(status, kPathFwdTc);

  const BucketOrder bo = bucket_order(blockIdx.x, nb_max, h_kv, lead);
  const int gb = bo.gb, kvh = bo.kvh;
  if (gb >= __ldg(blk_off + batch)) return;
  const int bucket = kvh * nb_max + gb;
  const int beg = __ldg(ptr + bucket), end = __ldg(ptr + bucket + 1);
  if (beg >= end) return;
  const int s = upper_seq(blk_off, batch, gb);
  const int t0 = __ldg(cu + s) + (gb - __ldg(blk_off + s)) * BLK;
  const int t1 = min(t0 + BLK, __ldg(cu + s + 1));
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const float scale_log2 = kLog2e * rsqrtf((float)D);
  const int ntiles = (end - beg + kRows - 1) / kRows;

  // Gather this warp's 32 rows of a tile with the TMA: lanes 0..7 each
  // issue one gather4 per 64-wide d chunk for rows 4l .. 4l+3 (row ids from
  // the lanes' `r_`; a missing row reads row 0, whose P is zero).
  auto gather = [&](int r_) {
    int ids[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int x = __shfl_sync(0xffffffffu, r_, 4 * (lane & 7) + u);
      ids[u] = x >= 0 ? x : 0;
    }
    if (lane == 0) tc::mbar_arrive_expect_tx(mb_q, 32 * D * 2);
    __syncwarp();
    if (lane < 8) {
#pragma unroll
      for (int c = 0; c < Ly::KB; ++c)
        tc::tma_gather4(sbase + Ly::Q_OFF + c * Ly::Q_REGION + (warp * 32 + 4 * lane) * 128, &tm_q, c * 64, ids[0],
                        ids[1], ids[2], ids[3], mb_q);
    }
  };
  auto meta_rid = [&](int tile) -> int {
    const int e = beg + tile * kRows + tid;
    return (tile < ntiles && e < end) ? __ldg(rows + e) : -1;
  };

  if (tid == 0) {
    tc::mbar_init(mb_s, 1);
    tc::mbar_init(mb_o, 1);
    tc::mbar_init(mb_q, kThreads / 32);
    tc::mbar_init(mb_kv, 1);
    tc::mbar_init_fence();
  }
  if (warp == 0) tc::tmem_alloc(sbase + Ly::HOLD_OFF, Ly::TMEM_COLS);
  int rid = meta_rid(0), nrid = -1;
  float mr_c = rid >= 0 ? __ldg(mref + rid) * kLog2e : 0.f, mr_n = 0.f;
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  // K_j, V_j -> SW128 K-major tiles (row = key, 64-wide d chunks as
  // regions): one TMA box of 64 channels x BLK tokens per chunk and tensor.
  if (tid == 0) {
    tc::mbar_arrive_expect_tx(mb_kv, Ly::KV_TX);
#pragma unroll
    for (int c = 0; c < Ly::KB; ++c) {
      tc::tma_load_3d(sbase + Ly::K_OFF + c * Ly::KV_REGION, &tm_k, c * 64, kvh, t0, mb_kv);
      tc::tma_load_3d(sbase + Ly::V_OFF + c * Ly::KV_REGION, &tm_v, c * 64, kvh, t0, mb_kv);
    }
  }
  gather(rid);
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(sm + Ly::HOLD_OFF);
  const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
  const uint32_t qa = sbase + Ly::Q_OFF;
  constexpr uint32_t id_s = tc::idesc_bf16_f32_major(kRows, BLK, 0, 0);  // S = Q K^T
  constexpr uint32_t id_o = tc::idesc_bf16_f32_major(kRows, D, 0, 1);    // O = P V

  // K_j / V_j have landed (decided block-wide); a partial block's tail rows
  // are cleared, ordered before the first MMA by the barrier of step A.
  bool ok = __syncthreads_and(tc::mbar_wait(mb_kv, 0));
  if (ok && t1 - t0 < BLK) {
    tc::zero_kv_tail_rows<D, BLK>(sm + Ly::K_OFF, sm + Ly::V_OFF, t1 - t0, tid, kThreads);
    tc::fence_proxy_async();
  }
  int it = 0;
  for (; ok && it < ntiles; ++it) {
    nrid = meta_rid(it + 1);
    // A. this tile's rows have landed
    const bool landed = tc::mbar_wait(mb_q, it & 1);
    tc::fence_before_sync();
    if (!__syncthreads_and(landed)) {
      ok = false;
      break;
    }
    // B. S = Q K_j^T
    if (tid == 0) {
      tc::fence_after_sync();
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint32_t ko = (kk >> 2) * Ly::Q_REGION + (kk & 3) * 32;
        const uint32_t kb = (kk >> 2) * Ly::KV_REGION + (kk & 3) * 32;
        tc::mma_bf16_ss(tmem, tc::smem_desc(qa + ko, 16, 1024, tc::kLayoutSW128),
                        tc::smem_desc(sbase + Ly::K_OFF + kb, 16, 1024, tc::kLayoutSW128), id_s, kk > 0);
      }
      tc::mma_commit(mb_s);
    }
    // C. P row; the Q tile is free: gather the next tile meanwhile
    if (!__syncthreads_and(tc::mbar_wait(mb_s, it & 1))) {
      ok = false;
      break;
    }
    tc::fence_after_sync();
    if (it + 1 < ntiles) gather(nrid);
    float l = 0.f, mx = -INFINITY;
    {
      // keys of this block the row may see: all of a block in its past, the
      // first (tok - t0 + 1) of its own block, none for a missing row
      const int tok = rid >= 0 ? rid / h_q : -1;
      const int nvis = max(0, min(tok + 1, t1) - t0);
#pragma unroll
      for (int h = 0; h < BLK / CW; ++h) {
        uint32_t sv[CW];
        if constexpr (CW == 32) tc::tmem_ld32(tmem + lane_base + h * CW, *reinterpret_cast<uint32_t(*)[32]>(sv));
        else tc::tmem_ld16(tmem + lane_base + h * CW, sv);
        tc::tmem_ld_wait();
        uint32_t pp[CW / 2];
#pragma unroll
        for (int c = 0; c < CW; c += 2) {
          float p2[2];
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            const int kk = h * CW + c + u;  // key index inside the block
            float p = 0.f;
            if (kk < nvis) {
              const float x = __uint_as_float(sv[c + u]) * scale_log2;
              p = fast_exp2(x - mr_c);
              mx = fmaxf(mx, x);
              l += p;
            }
            p2[u] = p;
          }
          pp[c / 2] = pack_bf16(p2[0], p2[1]);
        }
#pragma unroll
        for (int c = 0; c < CW / 8; ++c)
          *reinterpret_cast<uint4*>(sm + Ly::P_OFF + PT::offset(tid, h * (CW / 8) + c)) =
              make_uint4(pp[4 * c], pp[4 * c + 1], pp[4 * c + 2], pp[4 * c + 3]);
      }
    }
    mr_n = nrid >= 0 ? __ldg(mref + nrid) * kLog2e : 0.f;
    tc::fence_proxy_async();
    tc::fence_before_sync();
    __syncthreads();
    // D. O = P V_j into the score columns (K steps of 16 keys: 32 bytes of a
    // P row; 16 rows = 2048 bytes of V_j)
    if (tid == 0) {
      tc::fence_after_sync();
#pragma unroll
      for (int kk = 0; kk < BLK / 16; ++kk) {
        const uint32_t po = (uint32_t)((kk * 32) / PT::ROWB) * PT::REGION + (uint32_t)((kk * 32) % PT::ROWB);
        tc::mma_bf16_ss(tmem, tc::smem_desc(sbase + Ly::P_OFF + po, 16, PT::ATOM, PT::LAYOUT),
                        tc::smem_desc(sbase + Ly::V_OFF + kk * 2048, Ly::KV_REGION, 1024, tc::kLayoutSW128), id_o,
                        kk > 0);
      }
      tc::mma_commit(mb_o);
    }
    // E. add the O row and l to the accumulator
    if (!__syncthreads_and(tc::mbar_wait(mb_o, it & 1))) {
      ok = false;
      break;
    }
    tc::fence_after_sync();
    if (rid >= 0) {
      atomicAdd(lacc + rid, l);
      if (mx - mr_c > kOverflowLog2) flag[rid] = 1;
    }
    // O rows leave through the (now free) P tile: each warp stages 32-column
    // pieces of its 32 rows, then 8 lanes cover one 128-byte row piece per
    // 16-byte reduction (4 rows per instruction instead of one per lane).
    {
      unsigned char* stg = sm + Ly::P_OFF + warp * 4096;
#pragma unroll
      for (int h = 0; h < D / 32; ++h) {
        uint32_t ov[32];
        tc::tmem_ld32(tmem + lane_base + h * 32, ov);
        tc::tmem_ld_wait();
#pragma unroll
        for (int c = 0; c < 8; ++c)
          *reinterpret_cast<float4*>(stg + lane * 128 + ((c ^ (lane & 7)) << 4)) =
              make_float4(__uint_as_float(ov[4 * c]), __uint_as_float(ov[4 * c + 1]),
                          __uint_as_float(ov[4 * c + 2]), __uint_as_float(ov[4 * c + 3]));
        __syncwarp();
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int rl = i * 4 + (lane >> 3), c = lane & 7;
          const float4 val = *reinterpret_cast<const float4*>(stg + rl * 128 + ((c ^ (rl & 7)) << 4));
          const int row = __shfl_sync(0xffffffffu, rid, rl);
          if (row >= 0) red_add_v4(oacc + (size_t)row * OS + h * 32 + c * 4, val.x, val.y, val.z, val.w);
        }
        __syncwarp();
      }
    }
    tc::fence_before_sync();
    rid = nrid;
    mr_c = mr_n;
  }
  const int fail_it = it;
  tc::fence_before_sync();
  ok = __syncthreads_and(ok);
  if (!ok) {
    // A tensor-core or TMA completion never arrived: record it, give the
    // MMAs and copies in flight a bounded chance to drain (a wait on a phase
    // that is not pending returns at once), release TMEM.
    if (tid == 0) set_status(status, kStatusTimeout);
    tc::mbar_wait(mb_kv, 0, 100000000ull);
    tc::mbar_wait(mb_s, fail_it & 1, 100000000ull);
    tc::mbar_wait(mb_o, fail_it & 1, 100000000ull);
    tc::mbar_wait(mb_q, fail_it & 1, 100000000ull);
    tc::mbar_wait(mb_q, (fail_it + 1) & 1, 100000000ull);
    __syncthreads();
  }
  if (warp == 0) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, Ly::TMEM_COLS);
  }
}

}  // namespace

cudaError_t launch_fwd_tc(const CUtensorMap& tm_q, const CUtensorMap& tm_k, const CUtensorMap& tm_v,
                          const SeqPlan& p, const int32_t* ptr, const int32_t* rows, const float* mref, int h_q,
                          int h_kv, int d, int block_size, float* oacc, float* lacc, int32_t* flag,
                          int32_t* status, cudaStream_t st) {
#define MOBA_FWD_TC(DD, BB)                                                                                   \
  do {                                                                                                        \
    const size_t smem = FwdTcLayout<DD, BB>::BYTES + 1024;                                                    \
    auto kern = fwd_tc_kernel<DD, BB>;                                                                        \
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);      \
    if (e != cudaSuccess) return e;                                                                           \
    if (p.nb_max == 0) return cudaSuccess;                                                                    \
    const int lead = bucket_lead((long long)p.total_tokens * (h_q / h_kv), DD * 4 + 4);                     \
    kern<<<dim3(p.nb_max * h_kv), kThreads, smem, st>>>(tm_q, tm_k, tm_v, p.cu, p.blk_off, p.batch, p.nb_max, \
                                                       h_q, h_kv, lead, ptr, rows, mref, oacc, lacc, flag,    \
                                                       status);                                               \
    return cudaGetLastError();                                                                                \
  } while (0)
#define MOBA_FWD_TC_B(DD)                         \
  switch (block_size) {                           \
    case 16: MOBA_FWD_TC(DD, 16);                 \
    case 32: MOBA_FWD_TC(DD, 32);                 \
    case 64: MOBA_FWD_TC(DD, 64);                 \
    case 128: MOBA_FWD_TC(DD, 128);               \
  }
  if (d == 64) MOBA_FWD_TC_B(64);
  if (d == 128) MOBA_FWD_TC_B(128);
#undef MOBA_FWD_TC_B
#undef MOBA_FWD_TC
  return cudaErrorInvalidValue;
}

}  // namespace moba
