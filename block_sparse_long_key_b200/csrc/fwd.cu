// Forward helpers of the sparse attention (the attention itself runs in
// fwd_tc.cu on the tcgen05 tensor cores).
//
// "Optimizing Mixture of Block Attention", §"Definizione del Compito"
// (O = softmax(QK^T/sqrt(d)) V over the selected blocks only) and
// §"Progettazione del Kernel FlashMoBA", "Tre Kernel Fusi" 2 (the partial
// results of a query's k blocks are scattered and merged).
//
// Partial results are merged without a partial-output buffer: every query's
// softmax is taken against a fixed reference M_i (computed by the router as
// a lower bound of the query's largest logit), so the contributions of its k
// blocks are plain sums, exp(z - M_i) v and exp(z - M_i), added with fp32
// reductions into an accumulator (O rows of d floats, l in its own array).
// fp32 keeps the full relative precision whatever the offset z - M_i, so M_i
// only has to be within ~60 of the true maximum; a row whose logits exceed
// M_i by more than 62 (possible only for keys far above their block mean) is
// flagged by the attention kernel and recomputed exactly here.
//
//   fwd_finalize_kernel: O = acc / l (bf16), LSE = M_i + log l; flagged rows
//     are queued instead.
//   fwd_fallback_kernel: exact online softmax of the queued rows, one warp per
//     row (normally none).
#include <algorithm>

#include "common.cuh"
#include "launch.h"

namespace moba {
namespace {

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
                    bf16* __restrict__ out, float* __restrict__ lse, int32_t* __restrict__ status) {
  constexpr int PL = D / 32;  // dims per lane
  const int lane = threadIdx.x & 31;
  const int n = __ldg(flag_list);
  if (n > 0) mark_path(status, kPathExactRows);
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

}  // namespace

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
                                int block_size, int topk, bf16* out, float* lse, int32_t* status,
                                cudaStream_t st) {
  if (d == 64)
    fwd_fallback_kernel<64><<<148, 128, 0, st>>>(q, k, v, p.cu, p.batch, sel_idx, flag_list, h_q, h_kv,
                                                 block_size, topk, out, lse, status);
  else
    fwd_fallback_kernel<128><<<148, 128, 0, st>>>(q, k, v, p.cu, p.batch, sel_idx, flag_list, h_q, h_kv,
                                                  block_size, topk, out, lse, status);
  return cudaGetLastError();
}

}  // namespace moba
