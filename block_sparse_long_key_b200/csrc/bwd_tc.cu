// Backward of the sparse attention on the tcgen05 tensor cores.
//
// "Optimizing Mixture of Block Attention", §"Progettazione del Kernel
// FlashMoBA", "Tre Kernel Fusi" 3 (backward parallel over key blocks, scores
// recomputed, partial dQ accumulated with atomic adds into a high-precision
// buffer) and §"Efficienza Backward Pass".  With the selection fixed:
// P = exp(S/sqrt(d) - LSE), dS = P (.) (dO V^T - D), dV_j += P^T dO,
// dK_j += dS^T Q / sqrt(d), dQ += dS K_j / sqrt(d).
//
// One CTA per (global key block j, KV head) walks the block's bucket of
// gathered (query, head) rows in tiles of 128; thread t owns tile row t,
// which is TMEM lane t.  Per tile:
//   1. Q and dO rows are gathered by the TMA (tile::gather4, four rows per
//      instruction, 128-byte swizzle) into K-major tiles; completion is
//      counted in bytes on an mbarrier.
//   2. One thread issues S = Q K_j^T and dP = dO V_j^T (M = 128 rows,
//      N = B keys, K = d) into tensor memory.
//   3. Each thread reads its row of S and dP (tcgen05.ld), forms P and dS in
//      fp32 and stores them as bf16 tiles in shared memory.
//   4. One thread issues dV_j^T += dO^T P and dK_j^T += Q^T dS (M = d, N = B,
//      K = 128 rows; the same Q / dO tiles read M-major) and dQ = dS K_j
//      (M = 128, N = d, K = B; K_j read N-major) into the columns S and dP
//      used.  dV_j^T and dK_j^T stay in tensor memory for the whole bucket.
//   5. Each thread reads its dQ row; the next tile's gather is issued (the
//      Q / dO tiles are free once the MMAs completed) and the rows are added
//      to the fp32 dQ accumulator with 16-byte vector reductions, staged
//      through the free P / dS tiles so that 8 lanes cover one 128-byte row
//      piece per instruction.
// The CTA is sequential; a small footprint (one gather stage, 128 TMEM
// columns at d = 64, B = 32) lets three CTAs share an SM so that their phases
// overlap.  K_j and V_j arrive once by TMA tile loads (a partial last
// block's tail rows are zeroed in shared memory).  Block sizes 16 .. 128: the
// P and dS tiles use the 32-, 64- or 128-byte swizzle (two 128-byte regions
// at B = 128, where S, dP, dV^T and dK^T take all 512 TMEM columns and one
// CTA runs per SM).  At the end dK_j and dV_j are written once (bf16).
// Every mbarrier wait is bounded; a timeout sets MOBA_STATUS_TIMEOUT and the
// CTA winds down.
#include "common.cuh"
#include "launch.h"
#include "tc.cuh"

namespace moba {
namespace {

constexpr int kRows = 128;  // gathered rows per tile (= TMEM lanes)
constexpr int kThreads = 128;

template <int D, int BLK>
struct BwdTcLayout {
  using PT = tc::KeyTile<BLK>;
  static constexpr int KB = D / 64;                          // 64-wide d chunks (128-byte rows)
  static constexpr uint32_t KV_REGION = BLK * 128;           // one d chunk of K_j or V_j
  static constexpr uint32_t QO_REGION = kRows * 128;         // one d chunk of a Q or dO tile
  static constexpr uint32_t K_OFF = 0;
  static constexpr uint32_t V_OFF = K_OFF + KB * KV_REGION;
  static constexpr uint32_t P_OFF = V_OFF + KB * KV_REGION;
  static constexpr uint32_t DS_OFF = P_OFF + PT::BYTES;
  // P and dS together, grown to 16 KB where smaller: the dQ rows are staged
  // there (32 rows x 128 bytes per warp) once the MMAs have read them.
  static constexpr uint32_t PD_AREA = 2 * PT::BYTES < 16384 ? 16384 : 2 * PT::BYTES;
  static constexpr uint32_t Q_OFF = P_OFF + PD_AREA;
  static constexpr uint32_t O_OFF = Q_OFF + KB * QO_REGION;
  static constexpr uint32_t MB_OFF = O_OFF + KB * QO_REGION;  // mbS, mbG, mbQ, mbKV
  static constexpr uint32_t HOLD_OFF = MB_OFF + 32;
  static constexpr uint32_t BYTES = HOLD_OFF + 16;
  static constexpr uint32_t KV_TX = 2 * KB * KV_REGION;      // bytes of one K_j + V_j load
  // Tensor memory columns: S and dP side by side, later overwritten by dQ
  // (D columns); then dV^T and dK^T (B each).
  static constexpr uint32_t S_COL = 0, DP_COL = BLK, DQ_COL = 0;
  static constexpr uint32_t DV_COL = (2 * BLK > D ? 2 * BLK : D), DK_COL = DV_COL + BLK;
  static constexpr uint32_t NCOLS = DK_COL + BLK;
  static constexpr uint32_t TMEM_COLS = NCOLS <= 128 ? 128 : (NCOLS <= 256 ? 256 : 512);
  static_assert(NCOLS <= 512, "tensor memory");
  static_assert(KV_REGION % 1024 == 0 && PT::REGION % 1024 == 0 && QO_REGION % 1024 == 0,
                "swizzle atoms stay aligned");
};

template <int D, int BLK>
__global__ void __launch_bounds__(kThreads)
bwd_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
              const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
              const float2* __restrict__ stat, const int32_t* __restrict__ cu, const int32_t* __restrict__ blk_off,
              int batch, int nb_max, int h_q, int h_kv, int lead, const int32_t* __restrict__ ptr,
              const int32_t* __restrict__ rows, float* __restrict__ dqacc, bf16* __restrict__ dk,
              bf16* __restrict__ dv, int32_t* __restrict__ status) {
  using Ly = BwdTcLayout<D, BLK>;
  using PT = typename Ly::PT;
  constexpr int CW = BLK < 32 ? BLK : 32;  // TMEM columns per load
  extern __shared__ unsigned char smem_raw[];
  // 1024-byte aligned base, derived from the shared array by pointer
  // arithmetic so that accesses through it stay shared-memory accesses.
  unsigned char* sm = smem_raw + (((smem_u32(smem_raw) + 1023u) & ~1023u) - smem_u32(smem_raw));
  const uint32_t sbase = smem_u32(sm);
  const uint32_t mb_s = sbase + Ly::MB_OFF, mb_g = mb_s + 8, mb_q = mb_s + 16, mb_kv = mb_s + 24;
  mark_path(status, kPathBwdTc);

  const BucketOrder bo = bucket_order(blockIdx.x, nb_max, h_kv, lead);
  const int gb = bo.gb, kvh = bo.kvh;
  if (gb >= __ldg(blk_off + batch)) return;
  const int bucket = kvh * nb_max + gb;
  const int beg = __ldg(ptr + bucket), end = __ldg(ptr + bucket + 1);
  const int s = upper_seq(blk_off, batch, gb);
  const int t0 = __ldg(cu + s) + (gb - __ldg(blk_off + s)) * BLK;
  const int t1 = min(t0 + BLK, __ldg(cu + s + 1));
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const size_t kv_stride = (size_t)h_kv * D;
  const float scale = rsqrtf((float)D);
  const float scale_log2 = kLog2e * scale;
  const int ntiles = (end - beg + kRows - 1) / kRows;

  // Gather this warp's 32 rows of a tile with the TMA: lanes 0..7 each
  // issue one gather4 per 64-wide d chunk and tensor for rows 4l .. 4l+3
  // (row ids from the lanes' `r_`; a missing row reads row 0, whose P and dS
  // are zero).
  auto gather = [&](int r_) {
    int ids[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int x = __shfl_sync(0xffffffffu, r_, 4 * (lane & 7) + u);
      ids[u] = x >= 0 ? x : 0;
    }
    if (lane == 0) tc::mbar_arrive_expect_tx(mb_q, 2 * 32 * D * 2);
    __syncwarp();
    if (lane < 8) {
      const uint32_t o = (warp * 32 + 4 * lane) * 128;
#pragma unroll
      for (int c = 0; c < Ly::KB; ++c) {
        tc::tma_gather4(sbase + Ly::Q_OFF + c * Ly::QO_REGION + o, &tm_q, c * 64, ids[0], ids[1], ids[2], ids[3],
                        mb_q);
        tc::tma_gather4(sbase + Ly::O_OFF + c * Ly::QO_REGION + o, &tm_do, c * 64, ids[0], ids[1], ids[2], ids[3],
                        mb_q);
      }
    }
  };
  // Row metadata (thread t: tile row t): row id, LSE and D.  The next
  // tile's row id is loaded at the top of a tile and its statistics after
  // the scores, so no load is waited for on the critical path.
  auto meta_rid = [&](int tile) -> int {
    const int e = beg + tile * kRows + tid;
    return (tile < ntiles && e < end) ? __ldg(rows + e) : -1;
  };

  if (tid == 0) {
    tc::mbar_init(mb_s, 1);
    tc::mbar_init(mb_g, 1);
    tc::mbar_init(mb_q, kThreads / 32);
    tc::mbar_init(mb_kv, 1);
    tc::mbar_init_fence();
  }
  if (warp == 0) tc::tmem_alloc(sbase + Ly::HOLD_OFF, Ly::TMEM_COLS);
  int rid = meta_rid(0), nrid = -1;
  const float2 st0 = rid >= 0 ? __ldg(stat + rid) : make_float2(0.f, 0.f);  // (LSE, D) of the row
  float lse_c = st0.x, dsum_c = st0.y;
  float lse_n = 0.f, dsum_n = 0.f;
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  // K_j, V_j -> SW128 K-major tiles (row = key, 64-wide d chunks as
  // regions): one TMA box of 64 channels x BLK tokens per chunk and tensor.
  if (ntiles > 0 && tid == 0) {
    tc::mbar_arrive_expect_tx(mb_kv, Ly::KV_TX);
#pragma unroll
    for (int c = 0; c < Ly::KB; ++c) {
      tc::tma_load_3d(sbase + Ly::K_OFF + c * Ly::KV_REGION, &tm_k, c * 64, kvh, t0, mb_kv);
      tc::tma_load_3d(sbase + Ly::V_OFF + c * Ly::KV_REGION, &tm_v, c * 64, kvh, t0, mb_kv);
    }
  }
  if (ntiles > 0) gather(rid);
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(sm + Ly::HOLD_OFF);
  const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
  const uint32_t qa = sbase + Ly::Q_OFF, oa = sbase + Ly::O_OFF;

  constexpr uint32_t id_s = tc::idesc_bf16_f32_major(kRows, BLK, 0, 0);  // S, dP
  constexpr uint32_t id_g = tc::idesc_bf16_f32_major(D, BLK, 1, 1);      // dV^T, dK^T
  constexpr uint32_t id_q = tc::idesc_bf16_f32_major(kRows, D, 0, 1);    // dQ
  // P / dS as the MN-major B operand of dV^T, dK^T: distance between the
  // 64-key groups (two at B = 128; one otherwise, where it is unused).
  constexpr uint32_t kPdLbo = PT::NREG > 1 ? PT::REGION : 16;

  // K_j / V_j have landed (decided block-wide); a partial block's tail rows
  // are cleared, ordered before the first MMA by the barrier of step A.
  bool ok = true;
  if (ntiles > 0) {
    ok = __syncthreads_and(tc::mbar_wait(mb_kv, 0));
    if (ok && t1 - t0 < BLK) {
      tc::zero_kv_tail_rows<D, BLK>(sm + Ly::K_OFF, sm + Ly::V_OFF, t1 - t0, tid, kThreads);
      tc::fence_proxy_async();
    }
  }
  int it = 0;
  for (; ok && it < ntiles; ++it) {
    nrid = meta_rid(it + 1);  // consumed by the gather at the end of this tile
    // A. this tile's rows have landed
    const bool landed = tc::mbar_wait(mb_q, it & 1);
    tc::fence_before_sync();
    if (!__syncthreads_and(landed)) {
      ok = false;
      break;
    }
    // B. S = Q K_j^T, dP = dO V_j^T
    if (tid == 0) {
      tc::fence_after_sync();
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint32_t ko = (kk >> 2) * Ly::QO_REGION + (kk & 3) * 32;
        const uint32_t kb = (kk >> 2) * Ly::KV_REGION + (kk & 3) * 32;
        tc::mma_bf16_ss(tmem + Ly::S_COL, tc::smem_desc(qa + ko, 16, 1024, tc::kLayoutSW128),
                        tc::smem_desc(sbase + Ly::K_OFF + kb, 16, 1024, tc::kLayoutSW128), id_s, kk > 0);
        tc::mma_bf16_ss(tmem + Ly::DP_COL, tc::smem_desc(oa + ko, 16, 1024, tc::kLayoutSW128),
                        tc::smem_desc(sbase + Ly::V_OFF + kb, 16, 1024, tc::kLayoutSW128), id_s, kk > 0);
      }
      tc::mma_commit(mb_s);
    }
    // C. P and dS rows
    if (!__syncthreads_and(tc::mbar_wait(mb_s, it & 1))) {
      ok = false;
      break;
    }
    tc::fence_after_sync();
    {
      const int tok = rid >= 0 ? rid / h_q : -1;
      const float lse2 = lse_c * kLog2e, dsm = dsum_c;
#pragma unroll
      for (int h = 0; h < BLK / CW; ++h) {
        uint32_t sv[CW], pv[CW];
        if constexpr (CW == 32) {
          tc::tmem_ld32(tmem + lane_base + Ly::S_COL + h * CW, *reinterpret_cast<uint32_t(*)[32]>(sv));
          tc::tmem_ld32(tmem + lane_base + Ly::DP_COL + h * CW, *reinterpret_cast<uint32_t(*)[32]>(pv));
        } else {
          tc::tmem_ld16(tmem + lane_base + Ly::S_COL + h * CW, sv);
          tc::tmem_ld16(tmem + lane_base + Ly::DP_COL + h * CW, pv);
        }
        tc::tmem_ld_wait();
        uint32_t pp[CW / 2], dd[CW / 2];
#pragma unroll
        for (int c = 0; c < CW; c += 2) {
          float p2[2], d2[2];
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            const int key_tok = t0 + h * CW + c + u;
            float p = 0.f;
            if (key_tok <= tok && key_tok < t1) p = fast_exp2(__uint_as_float(sv[c + u]) * scale_log2 - lse2);
            p2[u] = p;
            d2[u] = p * (__uint_as_float(pv[c + u]) - dsm);
          }
          pp[c / 2] = pack_bf16(p2[0], p2[1]);
          dd[c / 2] = pack_bf16(d2[0], d2[1]);
        }
#pragma unroll
        for (int c = 0; c < CW / 8; ++c) {
          const uint32_t o = PT::offset(tid, h * (CW / 8) + c);
          *reinterpret_cast<uint4*>(sm + Ly::P_OFF + o) =
              make_uint4(pp[4 * c], pp[4 * c + 1], pp[4 * c + 2], pp[4 * c + 3]);
          *reinterpret_cast<uint4*>(sm + Ly::DS_OFF + o) =
              make_uint4(dd[4 * c], dd[4 * c + 1], dd[4 * c + 2], dd[4 * c + 3]);
        }
      }
    }
    {
      const float2 st1 = nrid >= 0 ? __ldg(stat + nrid) : make_float2(0.f, 0.f);
      lse_n = st1.x;
      dsum_n = st1.y;
    }
    tc::fence_proxy_async();
    tc::fence_before_sync();
    __syncthreads();
    // D. dV^T += dO^T P, dK^T += Q^T dS, dQ = dS K_j
    if (tid == 0) {
      tc::fence_after_sync();
#pragma unroll
      for (int ks = 0; ks < kRows / 16; ++ks) {
        // 16 rows = two 8-row groups of the Q / dO tiles and of P / dS
        const uint32_t ro = ks * 2048;
        const uint32_t po = ks * 2 * PT::ATOM;
        const uint32_t acc = (it > 0 || ks > 0) ? 1u : 0u;
        tc::mma_bf16_ss(tmem + Ly::DV_COL, tc::smem_desc(oa + ro, Ly::QO_REGION, 1024, tc::kLayoutSW128),
                        tc::smem_desc(sbase + Ly::P_OFF + po, kPdLbo, PT::ATOM, PT::LAYOUT), id_g, acc);
        tc::mma_bf16_ss(tmem + Ly::DK_COL, tc::smem_desc(qa + ro, Ly::QO_REGION, 1024, tc::kLayoutSW128),
                        tc::smem_desc(sbase + Ly::DS_OFF + po, kPdLbo, PT::ATOM, PT::LAYOUT), id_g, acc);
      }
#pragma unroll
      for (int kk = 0; kk < BLK / 16; ++kk) {
        // K steps of 16 keys: 32 bytes along a dS row; two 8-key groups of K_j
        const uint32_t po = (uint32_t)((kk * 32) / PT::ROWB) * PT::REGION + (uint32_t)((kk * 32) % PT::ROWB);
        tc::mma_bf16_ss(tmem + Ly::DQ_COL, tc::smem_desc(sbase + Ly::DS_OFF + po, 16, PT::ATOM, PT::LAYOUT),
                        tc::smem_desc(sbase + Ly::K_OFF + kk * 2048, Ly::KV_REGION, 1024, tc::kLayoutSW128), id_q,
                        kk > 0);
      }
      tc::mma_commit(mb_g);
    }
    // E. the tiles are free once the MMAs completed: start the next gather,
    // then add this tile's dQ rows.
    if (!__syncthreads_and(tc::mbar_wait(mb_g, it & 1))) {
      ok = false;
      break;
    }
    tc::fence_after_sync();
    if (it + 1 < ntiles) gather(nrid);
    // dQ rows leave through the (now free) P / dS area: each warp stages
    // 32-column halves of its 32 rows, then 8 lanes cover one 128-byte row
    // piece per reduction instruction.
    unsigned char* stg = sm + Ly::P_OFF + warp * 4096;
#pragma unroll
    for (int h = 0; h < D / 32; ++h) {
      uint32_t qv[32];
      tc::tmem_ld32(tmem + lane_base + Ly::DQ_COL + h * 32, qv);
      tc::tmem_ld_wait();
#pragma unroll
      for (int c = 0; c < 8; ++c)
        *reinterpret_cast<float4*>(stg + lane * 128 + ((c ^ (lane & 7)) << 4)) =
            make_float4(__uint_as_float(qv[4 * c]) * scale, __uint_as_float(qv[4 * c + 1]) * scale,
                        __uint_as_float(qv[4 * c + 2]) * scale, __uint_as_float(qv[4 * c + 3]) * scale);
      __syncwarp();
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int rl = i * 4 + (lane >> 3), c = lane & 7;
        const float4 val = *reinterpret_cast<const float4*>(stg + rl * 128 + ((c ^ (rl & 7)) << 4));
        const int row = __shfl_sync(0xffffffffu, rid, rl);
        if (row >= 0) red_add_v4(dqacc + (size_t)row * D + h * 32 + c * 4, val.x, val.y, val.z, val.w);
      }
      __syncwarp();
    }
    tc::fence_before_sync();
    rid = nrid;
    lse_c = lse_n;
    dsum_c = dsum_n;
  }
  const int fail_it = it;
  tc::fence_before_sync();
  ok = __syncthreads_and(ok);
  if (!ok) {
    // A tensor-core or TMA completion never arrived: record it, give the
    // MMAs and copies in flight a bounded chance to drain (a wait on a phase
    // that is not pending returns at once), release TMEM, leave dK_j / dV_j
    // alone.
    if (tid == 0) set_status(status, kStatusTimeout);
    tc::mbar_wait(mb_kv, 0, 100000000ull);
    tc::mbar_wait(mb_s, fail_it & 1, 100000000ull);
    tc::mbar_wait(mb_g, fail_it & 1, 100000000ull);
    tc::mbar_wait(mb_q, fail_it & 1, 100000000ull);
    tc::mbar_wait(mb_q, (fail_it + 1) & 1, 100000000ull);
    __syncthreads();
    if (warp == 0) tc::tmem_dealloc(tmem, Ly::TMEM_COLS);
    return;
  }
  tc::fence_after_sync();
  // dV_j^T, dK_j^T: accumulator row m (a d index) sits in lane m for M = 128,
  // in lane (m % 16) + 32 (m / 16) for M = 64.
  const int m = D == 128 ? tid : (lane < 16 ? warp * 16 + lane : -1);
#pragma unroll
  for (int h = 0; h < BLK / CW; ++h) {
    uint32_t av[CW], bv[CW];
    if constexpr (CW == 32) {
      tc::tmem_ld32(tmem + lane_base + Ly::DV_COL + h * CW, *reinterpret_cast<uint32_t(*)[32]>(av));
      tc::tmem_ld32(tmem + lane_base + Ly::DK_COL + h * CW, *reinterpret_cast<uint32_t(*)[32]>(bv));
    } else {
      tc::tmem_ld16(tmem + lane_base + Ly::DV_COL + h * CW, av);
      tc::tmem_ld16(tmem + lane_base + Ly::DK_COL + h * CW, bv);
    }
    tc::tmem_ld_wait();
    if (m >= 0) {
#pragma unroll
      for (int c = 0; c < CW; ++c) {
        const int kt = t0 + h * CW + c;
        const float a = ntiles > 0 ? __uint_as_float(av[c]) : 0.f;
        const float b = ntiles > 0 ? __uint_as_float(bv[c]) * scale : 0.f;
        if (kt < t1) {
          const size_t o = (size_t)kt * kv_stride + (size_t)kvh * D + m;
          dv[o] = __float2bfloat16_rn(a);
          dk[o] = __float2bfloat16_rn(b);
        }
      }
    }
  }
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 0) tc::tmem_dealloc(tmem, Ly::TMEM_COLS);
}

}  // namespace

cudaError_t launch_bwd_tc(const CUtensorMap& tm_q, const CUtensorMap& tm_k, const CUtensorMap& tm_v,
                          const CUtensorMap& tm_do, const float2* stat, const SeqPlan& p, const int32_t* ptr,
                          const int32_t* rows, int h_q, int h_kv, int d, int block_size, float* dqacc, bf16* dk,
                          bf16* dv, int32_t* status, cudaStream_t st) {
#define MOBA_BWD_TC(DD, BB)                                                                                  \
  do {                                                                                                       \
    const size_t smem = BwdTcLayout<DD, BB>::BYTES + 1024;                                                   \
    auto kern = bwd_tc_kernel<DD, BB>;                                                                       \
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);     \
    if (e != cudaSuccess) return e;                                                                          \
    if (p.nb_max == 0) return cudaSuccess;                                                                   \
    const int lead = bucket_lead((long long)p.total_tokens * (h_q / h_kv), DD * 4);                          \
    kern<<<dim3(p.nb_max * h_kv), kThreads, smem, st>>>(tm_q, tm_k, tm_v, tm_do, stat, p.cu, p.blk_off,     \
                                                       p.batch, p.nb_max, h_q, h_kv, lead, ptr, rows, dqacc, \
                                                       dk, dv, status);                                      \
    return cudaGetLastError();                                                                               \
  } while (0)
#define MOBA_BWD_TC_B(DD)           \
  switch (block_size) {             \
    case 16: MOBA_BWD_TC(DD, 16);   \
    case 32: MOBA_BWD_TC(DD, 32);   \
    case 64: MOBA_BWD_TC(DD, 64);   \
    case 128: MOBA_BWD_TC(DD, 128); \
  }
  if (d == 64) MOBA_BWD_TC_B(64);
  if (d == 128) MOBA_BWD_TC_B(128);
#undef MOBA_BWD_TC_B
#undef MOBA_BWD_TC
  return cudaErrorInvalidValue;
}

}  // namespace moba
