// Key-block centroids, optionally fused with the depthwise causal key
// convolution.
//
// "Optimizing Mixture of Block Attention":
//  * §"Architettura del Modello Statistico" 1: the router represents key
//    block j by its mean k~_j = (1/B) sum_{k in block j} k.
//  * §"Progettazione della Convoluzione delle Chiavi (Appendice B)", "Forma
//    Formale": k'_t = k_t + SiLU(sum_{l=0}^{W-1} W_l (.) k_{t-l}), one filter
//    per channel, causal (left zero padding at the sequence start).
//
// One CTA per (global block, KV head) reads the block's B key rows once with
// 16-byte vector loads (D/8 threads per row), writes k' (bf16, round to
// nearest even) when the conv is on, and the centroid of the (converted)
// keys as fp32 plus a bf16 hi/lo split (hi = bf16(c), lo = bf16(c - hi))
// that the tensor-core router uses to reach fp32-level score accuracy.
// HBM-bound: algorithmic bytes per block = B*D*2 read (+ B*D*2 written).
#include "common.cuh"
#include "launch.h"

namespace moba {
namespace {

constexpr int kThreads = 256;
constexpr int kMaxWidth = 8;

template <int D>
__global__ void __launch_bounds__(kThreads)
conv_centroid_kernel(const bf16* __restrict__ k, const float* __restrict__ conv_w, int width,
                     const int32_t* __restrict__ cu, const int32_t* __restrict__ blk_off, int batch,
                     int nb_max, int h_kv, int block_size, bf16* __restrict__ k_out,
                     float* __restrict__ cent, bf16* __restrict__ cent_hi, bf16* __restrict__ cent_lo) {
  constexpr int TPR = D / 8;            // threads per key row
  constexpr int RPP = kThreads / TPR;   // rows per pass
  __shared__ float s_part[RPP][D];

  const int gb = blockIdx.x;
  const int h = blockIdx.y;
  if (gb >= __ldg(blk_off + batch)) return;
  const int s = upper_seq(blk_off, batch, gb);
  const int j = gb - __ldg(blk_off + s);
  const int seq0 = __ldg(cu + s);
  const int t0 = seq0 + j * block_size;
  const int t1 = min(t0 + block_size, __ldg(cu + s + 1));
  const int nrows = t1 - t0;

  const int c8 = threadIdx.x % TPR;
  const int rr = threadIdx.x / TPR;
  const size_t row_stride = (size_t)h_kv * D;
  const bf16* kh = k + (size_t)h * D + c8 * 8;

  float acc[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) acc[i] = 0.f;

  if (width == 0) {
    for (int r = rr; r < nrows; r += RPP) {
      uint4 u = __ldg(reinterpret_cast<const uint4*>(kh + (size_t)(t0 + r) * row_stride));
      float f[8];
      bf16x8_to_f32(u, f);
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[i] += f[i];
    }
  } else {
    float w[kMaxWidth][8];
#pragma unroll
    for (int l = 0; l < kMaxWidth; ++l)
#pragma unroll
      for (int i = 0; i < 8; ++i)
        w[l][i] = l < width ? __ldg(conv_w + ((size_t)h * D + c8 * 8 + i) * width + l) : 0.f;
    bf16* ko = k_out + (size_t)h * D + c8 * 8;
    for (int r = rr; r < nrows; r += RPP) {
      const int t = t0 + r;
      float x[8], kt[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) x[i] = 0.f;
#pragma unroll
      for (int l = 0; l < kMaxWidth; ++l) {
        if (l < width && t - l >= seq0) {
          uint4 u = __ldg(reinterpret_cast<const uint4*>(kh + (size_t)(t - l) * row_stride));
          float f[8];
          bf16x8_to_f32(u, f);
          if (l == 0) {
#pragma unroll
            for (int i = 0; i < 8; ++i) kt[i] = f[i];
          }
#pragma unroll
          for (int i = 0; i < 8; ++i) x[i] = fmaf(w[l][i], f[i], x[i]);
        }
      }
      float y[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float silu = x[i] / (1.f + expf(-x[i]));
        y[i] = kt[i] + silu;
      }
      uint4 packed = f32_to_bf16x8(y);
      *reinterpret_cast<uint4*>(ko + (size_t)t * row_stride) = packed;
      float yr[8];
      bf16x8_to_f32(packed, yr);  // the centroid averages the stored bf16 keys
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[i] += yr[i];
    }
  }

#pragma unroll
  for (int i = 0; i < 8; ++i) s_part[rr][c8 * 8 + i] = acc[i];
  __syncthreads();
  if (threadIdx.x < D) {
    float sum = 0.f;
    for (int g = 0; g < RPP; ++g) sum += s_part[g][threadIdx.x];
    const float c = sum / (float)nrows;
    const size_t o = ((size_t)h * nb_max + gb) * D + threadIdx.x;
    cent[o] = c;
    const bf16 hi = __float2bfloat16_rn(c);
    cent_hi[o] = hi;
    cent_lo[o] = __float2bfloat16_rn(c - __bfloat162float(hi));
  }
}

}  // namespace

cudaError_t launch_conv_centroid(const bf16* k, const float* conv_w, int conv_width, const SeqPlan& p,
                                 int h_kv, int d, int block_size, bf16* k_out, float* cent,
                                 bf16* cent_hi, bf16* cent_lo, cudaStream_t st) {
  if (conv_width > kMaxWidth) return cudaErrorInvalidValue;
  dim3 grid(p.nb_max, h_kv);
  if (d == 64)
    conv_centroid_kernel<64><<<grid, kThreads, 0, st>>>(k, conv_w, conv_width, p.cu, p.blk_off, p.batch,
                                                        p.nb_max, h_kv, block_size, k_out, cent,
                                                        cent_hi, cent_lo);
  else
    conv_centroid_kernel<128><<<grid, kThreads, 0, st>>>(k, conv_w, conv_width, p.cu, p.blk_off, p.batch,
                                                         p.nb_max, h_kv, block_size, k_out, cent,
                                                         cent_hi, cent_lo);
  return cudaGetLastError();
}

}  // namespace moba
