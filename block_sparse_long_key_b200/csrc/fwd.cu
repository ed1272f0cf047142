// Forward sparse attention: gather-and-densify per key block.
//
// "Optimizing Mixture of Block Attention", §"Definizione del Compito"
// (O = softmax(QK^T/sqrt(d)) V over the selected blocks only) and
// §"Progettazione del Kernel FlashMoBA", "Tre Kernel Fusi" 2 ("Forward
// Pass: Gather-and-Densify": for each key block, find the queries that chose
// it from the varlen index, gather them into dense tiles in on-chip memory,
// run dense GEMMs against the block, scatter the results).
//
// Design on sm_100a: one CTA per (global key block, KV head).  The block's K
// and V (B x d, bf16) are loaded once into shared memory; each warp then
// gathers its own 16-row slices of the bucket (cp.async, double buffered) and
// runs S = Q K^T and O = P V on the tensor cores with P kept in registers.
// Own-block rows get the causal cut key_token <= query_token.
//
// Partial results are merged without a partial-output buffer: every query's
// softmax is taken against a fixed reference M_i (computed by the router as
// a lower bound of the query's largest logit), so the contributions of its k
// blocks are plain sums, exp(z - M_i) v and exp(z - M_i), added with fp32
// reductions into an accumulator row [O | l | pad] (32-byte aligned) that stays L2-resident
// while a head is processed (CTAs run block-major within one head).  fp32 keeps the
// full relative precision whatever the offset z - M_i, so M_i only has to be
// within ~60 of the true maximum; a row whose logits exceed M_i by more than
// 62 (possible only for keys far above their block mean) is flagged and
// recomputed exactly by the fallback kernel.
//
// finalize: O = acc / l, LSE = M_i + log l.  fallback: exact online softmax,
// one warp per flagged row (normally none).
#include <algorithm>

#include "common.cuh"
#include "launch.h"

namespace moba {
namespace {

constexpr int kWarps = 4;
constexpr int kThreads = kWarps * 32;
constexpr int kRows = 16;              // gathered query rows per warp tile
constexpr float kOverflowLog2 = 90.f;  // ~62 in natural-log units

template <int D, int BLK>
struct FwdSmem {
  bf16 k[BLK][D + 8];
  bf16 v[BLK][D + 8];
  bf16 q[kWarps][2][kRows][D + 8];      // per-warp gathered rows, double buffered
};

// One CTA per (global key block, KV head).  K_j, V_j are loaded once; then
// every warp independently walks its share of the bucket 16 rows at a time
// through a three-deep software pipeline: row ids two tiles ahead, the query
// gather (cp.async) and the row statistics one tile ahead, the tensor-core
// work (S = Q K^T, O = P V with P in registers) on the current tile.  Lanes
// 0..15 each carry one row's (id, M_i, causal limit) in registers and hand
// them to the MMA lanes by shuffles.  Partial O rows leave as 16-byte fp32
// vector reductions (lane pairs swap halves so each lane holds 4 consecutive
// columns), l as one fp32 add per row.  No CTA-wide barrier in the loop.
template <int D, int BLK>
__global__ void __launch_bounds__(kThreads)
fwd_attn_kernel(const bf16* __restrict__ q, const bf16* __restrict__ k, const bf16* __restrict__ v,
                const int32_t* __restrict__ cu, const int32_t* __restrict__ blk_off, int batch, int nb_max,
                int h_q, int h_kv, int lead, const int32_t* __restrict__ ptr, const int32_t* __restrict__ rows,
                const float* __restrict__ mref, float* __restrict__ oacc, float* __restrict__ lacc,
                int32_t* __restrict__ flag) {
  constexpr int KC = BLK < 64 ? BLK : 64;  // keys per register chunk
  constexpr int OS = oacc_stride(D);       // accumulator row: O (D); l in lacc
  constexpr unsigned FULL = 0xffffffffu;
  extern __shared__ __align__(128) unsigned char smem_raw[];
  FwdSmem<D, BLK>& sm = *reinterpret_cast<FwdSmem<D, BLK>*>(smem_raw);

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
  const size_t kv_stride = (size_t)h_kv * D;
  const float scale_log2 = kLog2e * rsqrtf((float)D);

  for (int i = tid; i < BLK * (D / 8); i += kThreads) {
    const int r = i / (D / 8), c = i % (D / 8);
    const bool ok = t0 + r < t1;
    const size_t off = ok ? (size_t)(t0 + r) * kv_stride + (size_t)kvh * D + c * 8 : 0;
    cp_async16_zfill(&sm.k[r][c * 8], k + off, ok);
    cp_async16_zfill(&sm.v[r][c * 8], v + off, ok);
  }
  cp_async_commit();

  // Tiles of this warp: warp, warp + kWarps, ...
  const int ntiles = (end - beg + kRows - 1) / kRows;
  auto load_id = [&](int tile) -> int {
    const int e = beg + tile * kRows + lane;
    return (tile < ntiles && lane < kRows && e < end) ? __ldg(rows + e) : -1;
  };
  auto issue_q = [&](int id, int buf) {
#pragma unroll
    for (int j = 0; j < kRows * (D / 8) / 32; ++j) {
      const int i = lane + 32 * j;
      const int r = i / (D / 8), c = i % (D / 8);
      const int row = __shfl_sync(FULL, id, r);
      const bool ok = row >= 0;
      const size_t off = ok ? (size_t)row * D + c * 8 : 0;   // q is [T, H_q, D]: row t*H_q + h
      cp_async16_zfill(&sm.q[warp][buf][r][c * 8], q + off, ok);
    }
  };
  // (M_i in log2 units, last visible key of this block) of the row in `id`.
  auto row_stats = [&](int id, float& mr, int& lim) {
    mr = 0.f;
    lim = -1;
    if (id >= 0) {
      mr = __ldg(mref + id) * kLog2e;
      lim = min(id / h_q, t1 - 1) - t0;   // own block: causal cut; earlier block: all keys
    }
  };

  int it = warp;
  int id0 = load_id(it), id1 = load_id(it + kWarps);
  float mr0_l = 0.f, mr1_l = 0.f;
  int lim0_l = -1, lim1_l = -1;
  if (it < ntiles) {
    issue_q(id0, 0);
    row_stats(id0, mr0_l, lim0_l);
  }
  cp_async_commit();
  cp_async_wait<0>();   // K, V and this warp's first rows
  __syncthreads();

  for (int li = 0; it < ntiles; ++li, it += kWarps) {
    const int buf = li & 1;
    const int id2 = load_id(it + 2 * kWarps);
    if (it + kWarps < ntiles) {
      issue_q(id1, buf ^ 1);
      row_stats(id1, mr1_l, lim1_l);
    }
    cp_async_commit();
    cp_async_wait<1>();
    __syncwarp();

    uint32_t qa[D / 16][4];
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk)
      ldsm_x4(qa[kk][0], qa[kk][1], qa[kk][2], qa[kk][3], &sm.q[warp][buf][lane & 15][kk * 16 + (lane >> 4) * 8]);
    const int r0 = lane >> 2, r1 = r0 + 8;
    const int lim0 = __shfl_sync(FULL, lim0_l, r0), lim1 = __shfl_sync(FULL, lim0_l, r1);
    const float mr0 = __shfl_sync(FULL, mr0_l, r0), mr1 = __shfl_sync(FULL, mr0_l, r1);
    const int row0 = __shfl_sync(FULL, id0, r0), row1 = __shfl_sync(FULL, id0, r1);

    float o[D / 8][4];
#pragma unroll
    for (int nt = 0; nt < D / 8; ++nt)
#pragma unroll
      for (int i = 0; i < 4; ++i) o[nt][i] = 0.f;
    float l0 = 0.f, l1 = 0.f, mx0 = -INFINITY, mx1 = -INFINITY;

#pragma unroll
    for (int kc = 0; kc < BLK / KC; ++kc) {
      float sacc[KC / 8][4];
#pragma unroll
      for (int nt = 0; nt < KC / 8; ++nt)
#pragma unroll
        for (int i = 0; i < 4; ++i) sacc[nt][i] = 0.f;
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
#pragma unroll
        for (int nt2 = 0; nt2 < KC / 16; ++nt2) {
          uint32_t b0, b1, b2, b3;
          ldsm_x4(b0, b1, b2, b3,
                  &sm.k[kc * KC + nt2 * 16 + (lane & 7) + ((lane >> 4) << 3)][kk * 16 + ((lane >> 3) & 1) * 8]);
          mma_bf16(sacc[2 * nt2], qa[kk], b0, b1);
          mma_bf16(sacc[2 * nt2 + 1], qa[kk], b2, b3);
        }
      }
      // causal cut + exp against the fixed reference
#pragma unroll
      for (int nt = 0; nt < KC / 8; ++nt) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int key = kc * KC + nt * 8 + (lane & 3) * 2 + (i & 1);
          const bool hi = i >= 2;
          const bool ok = key <= (hi ? lim1 : lim0);
          const float x = sacc[nt][i] * scale_log2;
          float p = 0.f;
          if (ok) {
            p = fast_exp2(x - (hi ? mr1 : mr0));
            if (hi) { mx1 = fmaxf(mx1, x); l1 += p; } else { mx0 = fmaxf(mx0, x); l0 += p; }
          }
          sacc[nt][i] = p;
        }
      }
      uint32_t pa[KC / 16][4];
#pragma unroll
      for (int ks = 0; ks < KC / 16; ++ks) {
        pa[ks][0] = pack_bf16(sacc[2 * ks][0], sacc[2 * ks][1]);
        pa[ks][1] = pack_bf16(sacc[2 * ks][2], sacc[2 * ks][3]);
        pa[ks][2] = pack_bf16(sacc[2 * ks + 1][0], sacc[2 * ks + 1][1]);
        pa[ks][3] = pack_bf16(sacc[2 * ks + 1][2], sacc[2 * ks + 1][3]);
      }
#pragma unroll
      for (int ks = 0; ks < KC / 16; ++ks) {
#pragma unroll
        for (int nt2 = 0; nt2 < D / 16; ++nt2) {
          uint32_t b0, b1, b2, b3;
          ldsm_x4_t(b0, b1, b2, b3,
                    &sm.v[kc * KC + ks * 16 + (lane & 7) + ((lane >> 3) & 1) * 8][nt2 * 16 + (lane >> 4) * 8]);
          mma_bf16(o[2 * nt2], pa[ks], b0, b1);
          mma_bf16(o[2 * nt2 + 1], pa[ks], b2, b3);
        }
      }
    }
#pragma unroll
    for (int off = 1; off <= 2; off <<= 1) {
      l0 += __shfl_xor_sync(FULL, l0, off);
      l1 += __shfl_xor_sync(FULL, l1, off);
      mx0 = fmaxf(mx0, __shfl_xor_sync(FULL, mx0, off));
      mx1 = fmaxf(mx1, __shfl_xor_sync(FULL, mx1, off));
    }
    // Lane pairs swap halves: even lanes take 4 columns of row r0, odd lanes
    // 4 columns of row r1, then one 16-byte reduction each.
    const int q4 = lane & 3;
    const bool even = (q4 & 1) == 0;
    const int rowx = even ? row0 : row1;
#pragma unroll
    for (int nt = 0; nt < D / 8; ++nt) {
      const float g0 = __shfl_xor_sync(FULL, even ? o[nt][2] : o[nt][0], 1);
      const float g1 = __shfl_xor_sync(FULL, even ? o[nt][3] : o[nt][1], 1);
      const int col = nt * 8 + (even ? q4 : q4 - 1) * 2;
      if (rowx >= 0) {
        if (even) red_add_v4(oacc + (size_t)rowx * OS + col, o[nt][0], o[nt][1], g0, g1);
        else red_add_v4(oacc + (size_t)rowx * OS + col, g0, g1, o[nt][2], o[nt][3]);
      }
    }
    if (q4 == 0) {
      if (row0 >= 0) {
        atomicAdd(lacc + row0, l0);
        if (mx0 - mr0 > kOverflowLog2) flag[row0] = 1;
      }
      if (row1 >= 0) {
        atomicAdd(lacc + row1, l1);
        if (mx1 - mr1 > kOverflowLog2) flag[row1] = 1;
      }
    }
    __syncwarp();   // everyone is done with q[buf] before it is refilled
    id0 = id1;
    id1 = id2;
    mr0_l = mr1_l;
    lim0_l = lim1_l;
  }
}

// O = acc / l (bf16), LSE = M + log l; flagged rows are queued instead.
// Accumulator rows are oacc_stride(D) floats of O; l is in its own array.
__global__ void __launch_bounds__(256)
fwd_finalize_kernel(const float* __restrict__ oacc, const float* __restrict__ lacc, const float* __restrict__ mref,
                    const int32_t* __restrict__ flag, long long nchunks, int d8, bf16* __restrict__ out,
                    float* __restrict__ lse, int32_t* __restrict__ flag_list) {
  const int os = oacc_stride(d8 * 8);
  for (long long i = blockIdx.x * 256LL + threadIdx.x; i < nchunks; i += (long long)gridDim.x * 256) {
    const long long row = i / d8;
    const int c = (int)(i % d8);
    if (__ldg(flag + row)) {
      if (c == 0) {
        const int slot = atomicAdd(flag_list, 1);
        flag_list[1 + slot] = (int32_t)row;
      }
      continue;
    }
    const float* acc = oacc + row * os;
    const float l = __ldg(lacc + row);
    const float inv = 1.f / l;
    const float4* src = reinterpret_cast<const float4*>(acc + c * 8);
    const float4 a = __ldg(src), b = __ldg(src + 1);
    float f[8] = {a.x * inv, a.y * inv, a.z * inv, a.w * inv, b.x * inv, b.y * inv, b.z * inv, b.w * inv};
    reinterpret_cast<uint4*>(out)[i] = f32_to_bf16x8(f);
    if (c == 0) lse[row] = __ldg(mref + row) + logf(l);
  }
}

// Exact recomputation of flagged rows: one warp per row, online softmax.
template <int D>
__global__ void __launch_bounds__(128)
fwd_fallback_kernel(const bf16* __restrict__ q, const bf16* __restrict__ k, const bf16* __restrict__ v,
                    const int32_t* __restrict__ cu, int batch, const int32_t* __restrict__ sel_idx,
                    const int32_t* __restrict__ flag_list, int h_q, int h_kv, int block_size, int topk,
                    bf16* __restrict__ out, float* __restrict__ lse) {
  constexpr int PL = D / 32;  // dims per lane
  const int lane = threadIdx.x & 31;
  const int n = __ldg(flag_list);
  const float scale = rsqrtf((float)D);
  for (int w = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; w < n; w += (gridDim.x * blockDim.x) >> 5) {
    const int row = __ldg(flag_list + 1 + w);
    const int t = row / h_q, h = row % h_q, kvh = h / (h_q / h_kv);
    const int s = upper_seq(cu, batch, t);
    const int seq0 = __ldg(cu + s), seq1 = __ldg(cu + s + 1);
    float qv[PL], o[PL];
#pragma unroll
    for (int i = 0; i < PL; ++i) {
      qv[i] = __bfloat162float(q[(size_t)row * D + lane * PL + i]);
      o[i] = 0.f;
    }
    float m = -INFINITY, l = 0.f;
    for (int sl = 0; sl < topk; ++sl) {
      const int j = __ldg(sel_idx + (size_t)row * topk + sl);
      if (j < 0 || j > (t - seq0) / block_size) continue;  // only blocks at or before the query's
      const int tb = seq0 + j * block_size;
      const int te = min(min(tb + block_size, seq1), t + 1);
      for (int tk = tb; tk < te; ++tk) {
        const size_t base = ((size_t)tk * h_kv + kvh) * D + lane * PL;
        float z = 0.f;
#pragma unroll
        for (int i = 0; i < PL; ++i) z = fmaf(qv[i], __bfloat162float(k[base + i]), z);
#pragma unroll
        for (int off = 16; off >= 1; off >>= 1) z += __shfl_xor_sync(0xffffffffu, z, off);
        z *= scale;
        const float mn = fmaxf(m, z);
        const float corr = expf(m - mn);
        const float p = expf(z - mn);
        l = l * corr + p;
#pragma unroll
        for (int i = 0; i < PL; ++i) o[i] = o[i] * corr + p * __bfloat162float(v[base + i]);
        m = mn;
      }
    }
#pragma unroll
    for (int i = 0; i < PL; ++i) out[(size_t)row * D + lane * PL + i] = __float2bfloat16_rn(o[i] / l);
    if (lane == 0) lse[row] = m + logf(l);
  }
}

template <int D, int BLK>
cudaError_t launch_fwd_t(const bf16* q, const bf16* k, const bf16* v, const SeqPlan& p, const int32_t* ptr,
                         const int32_t* rows, const float* mref, int h_q, int h_kv, float* oacc, float* lacc,
                         int32_t* flag, cudaStream_t st) {
  const size_t smem = sizeof(FwdSmem<D, BLK>);
  auto kern = fwd_attn_kernel<D, BLK>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  if (p.nb_max == 0) return cudaSuccess;
  dim3 grid(p.nb_max * h_kv);
  const int lead = bucket_lead((long long)p.total_tokens * (h_q / h_kv), D * 4 + 4);
  kern<<<grid, kThreads, smem, st>>>(q, k, v, p.cu, p.blk_off, p.batch, p.nb_max, h_q, h_kv, lead, ptr, rows, mref,
                                     oacc, lacc, flag);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_fwd_attn(const bf16* q, const bf16* k, const bf16* v, const SeqPlan& p, const int32_t* ptr,
                            const int32_t* rows, const float* mref, int h_q, int h_kv, int d, int block_size,
                            float* oacc, float* lacc, int32_t* flag, cudaStream_t st) {
#define MOBA_FWD(DD, BB) return launch_fwd_t<DD, BB>(q, k, v, p, ptr, rows, mref, h_q, h_kv, oacc, lacc, flag, st)
  if (d == 64) {
    switch (block_size) {
      case 16: MOBA_FWD(64, 16);
      case 32: MOBA_FWD(64, 32);
      case 64: MOBA_FWD(64, 64);
      case 128: MOBA_FWD(64, 128);
    }
  } else {
    switch (block_size) {
      case 16: MOBA_FWD(128, 16);
      case 32: MOBA_FWD(128, 32);
      case 64: MOBA_FWD(128, 64);
      case 128: MOBA_FWD(128, 128);
    }
  }
#undef MOBA_FWD
  return cudaErrorInvalidValue;
}

cudaError_t launch_fwd_finalize(const float* oacc, const float* lacc, const float* mref, const int32_t* flag, int nrows, int d,
                                bf16* out, float* lse, int32_t* flag_list, cudaStream_t st) {
  cudaError_t e = cudaMemsetAsync(flag_list, 0, sizeof(int32_t), st);
  if (e != cudaSuccess) return e;
  const long long nchunks = (long long)nrows * (d / 8);
  if (nchunks == 0) return cudaSuccess;
  const int grid = (int)std::min<long long>((nchunks + 255) / 256, 148LL * 32);
  fwd_finalize_kernel<<<grid, 256, 0, st>>>(oacc, lacc, mref, flag, nchunks, d / 8, out, lse, flag_list);
  return cudaGetLastError();
}

cudaError_t launch_fwd_fallback(const bf16* q, const bf16* k, const bf16* v, const SeqPlan& p,
                                const int32_t* sel_idx, const int32_t* flag_list, int h_q, int h_kv, int d,
                                int block_size, int topk, bf16* out, float* lse, cudaStream_t st) {
  if (d == 64)
    fwd_fallback_kernel<64><<<148, 128, 0, st>>>(q, k, v, p.cu, p.batch, sel_idx, flag_list, h_q, h_kv,
                                                 block_size, topk, out, lse);
  else
    fwd_fallback_kernel<128><<<148, 128, 0, st>>>(q, k, v, p.cu, p.batch, sel_idx, flag_list, h_q, h_kv,
                                                  block_size, topk, out, lse);
  return cudaGetLastError();
}

}  // namespace moba
