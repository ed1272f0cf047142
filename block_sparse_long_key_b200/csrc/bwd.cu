// Backward helpers of the sparse attention (the attention itself runs in
// bwd_tc.cu on the tcgen05 tensor cores).
//
// "Optimizing Mixture of Block Attention", §"Progettazione del Kernel
// FlashMoBA", "Tre Kernel Fusi" 3 ("Backward Pass: Ricalcolo": the
// probabilities are recomputed per key block, partial dQ is accumulated with
// atomic adds into a high-precision global buffer).  With the selection
// fixed, P = exp(S/sqrt(d) - LSE) and D_i = dO_i . O_i.
//
//   bwd_pre_kernel: (LSE_i, D_i) per row, packed as one float2 so that the
//     attention kernel makes one 8-byte load per gathered row, and the fp32
//     dQ accumulator zeroed.
//   bwd_dq_kernel:  the fp32 dQ accumulator rounded to bf16.
#include <algorithm>

#include "common.cuh"
#include "launch.h"

namespace moba {
namespace {

// D_i = sum_c dO_ic O_ic (fp32) and dQ accumulator zeroing; D/8 lanes per row.
template <int D>
__global__ void __launch_bounds__(256)
bwd_pre_kernel(const bf16* __restrict__ out, const bf16* __restrict__ dout, const float* __restrict__ lse,
               long long nrows, float2* __restrict__ stat, float* __restrict__ dqacc) {
  constexpr int LPR = D / 8;
  const long long nthreads = (long long)gridDim.x * 256;
  const long long total = nrows * LPR;
  // Whole warps iterate together (the bound is rounded up to 32) so that the
  // row-sum shuffles always see every lane.
  const long long total_w = (total + 31) / 32 * 32;
  for (long long i = blockIdx.x * 256LL + threadIdx.x; i < total_w; i += nthreads) {
    const bool ok = i < total;
    float acc = 0.f;
    if (ok) {
      float a[8], b[8];
      bf16x8_to_f32(__ldg(reinterpret_cast<const uint4*>(out) + i), a);
      bf16x8_to_f32(__ldg(reinterpret_cast<const uint4*>(dout) + i), b);
#pragma unroll
      for (int j = 0; j < 8; ++j) acc = fmaf(a[j], b[j], acc);
    }
#pragma unroll
    for (int off = LPR / 2; off >= 1; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
    if (ok) {
      if (i % LPR == 0) stat[i / LPR] = make_float2(__ldg(lse + i / LPR), acc);
      float4* z = reinterpret_cast<float4*>(dqacc) + 2 * i;
      z[0] = make_float4(0.f, 0.f, 0.f, 0.f);
      z[1] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
  }
}

__global__ void __launch_bounds__(256)
bwd_dq_kernel(const float* __restrict__ dqacc, long long n8, bf16* __restrict__ dq) {
  for (long long i = blockIdx.x * 256LL + threadIdx.x; i < n8; i += (long long)gridDim.x * 256) {
    const float4* src = reinterpret_cast<const float4*>(dqacc) + 2 * i;
    const float4 a = __ldg(src), b = __ldg(src + 1);
    float f[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
    reinterpret_cast<uint4*>(dq)[i] = f32_to_bf16x8(f);
  }
}

}  // namespace

cudaError_t launch_bwd_pre(const bf16* out, const bf16* dout, const float* lse, int nrows, int d, float2* stat,
                           float* dqacc, cudaStream_t st) {
  const long long n = (long long)nrows * (d / 8);
  if (n == 0) return cudaSuccess;
  const int grid = (int)std::min<long long>((n + 255) / 256, 148LL * 32);
  if (d == 64)
    bwd_pre_kernel<64><<<grid, 256, 0, st>>>(out, dout, lse, nrows, stat, dqacc);
  else
    bwd_pre_kernel<128><<<grid, 256, 0, st>>>(out, dout, lse, nrows, stat, dqacc);
  return cudaGetLastError();
}

cudaError_t launch_bwd_dq(const float* dqacc, int n, bf16* dq, cudaStream_t st) {
  const long long n8 = n / 8;
  if (n8 == 0) return cudaSuccess;
  const int grid = (int)std::min<long long>((n8 + 255) / 256, 148LL * 32);
  bwd_dq_kernel<<<grid, 256, 0, st>>>(dqacc, n8, dq);
  return cudaGetLastError();
}

}  // namespace moba
