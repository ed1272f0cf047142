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
// Eight threads per (global block, KV head), each owning 8 channels: a
// thread walks the block's rows in order with 16-byte loads (the 8 threads of
// a block read one 128/256-byte row segment together), keeps the previous
// W-1 rows of its channels in registers for the conv, writes k' and sums the
// (converted) keys itself, so no shared memory and no barrier are needed.
// The sum runs in ascending token order in fp32 and is divided by the block's
// token count.  HBM-bound: algorithmic bytes per block = B*D*2 read
// (+ B*D*2 written with conv) + centroid outputs.
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
  constexpr int TPB = D / 8;  // threads per block (8 channels each)
  const long long gtid = (long long)blockIdx.x * kThreads + threadIdx.x;
  const int c8 = (int)(gtid % TPB);
  const long long bidx = gtid / TPB;
  const int h = (int)(bidx / nb_max);
  const int gb = (int)(bidx % nb_max);
  if (h >= h_kv || gb >= __ldg(blk_off + batch)) return;
  const int s = upper_seq(blk_off, batch, gb);
  const int j = gb - __ldg(blk_off + s);
  const int seq0 = __ldg(cu + s);
  const int t0 = seq0 + j * block_size;
  const int t1 = min(t0 + block_size, __ldg(cu + s + 1));
  const size_t row_stride = (size_t)h_kv * D;
  const bf16* kh = k + (size_t)h * D + c8 * 8;

  float acc[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) acc[i] = 0.f;

  if (width == 0) {
#pragma unroll 4
    for (int t = t0; t < t1; ++t) {
      float f[8];
      bf16x8_to_f32(__ldg(reinterpret_cast<const uint4*>(kh + (size_t)t * row_stride)), f);
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
    // win[l] holds k_{t-1-l} (zero before the sequence start)
    float win[kMaxWidth - 1][8];
#pragma unroll
    for (int l = 0; l < kMaxWidth - 1; ++l) {
      const int tp = t0 - 1 - l;
      if (l + 1 < width && tp >= seq0) {
        bf16x8_to_f32(__ldg(reinterpret_cast<const uint4*>(kh + (size_t)tp * row_stride)), win[l]);
      } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) win[l][i] = 0.f;
      }
    }
    bf16* ko = k_out + (size_t)h * D + c8 * 8;
#pragma unroll 2
    for (int t = t0; t < t1; ++t) {
      float cur[8], x[8];
      bf16x8_to_f32(__ldg(reinterpret_cast<const uint4*>(kh + (size_t)t * row_stride)), cur);
#pragma unroll
      for (int i = 0; i < 8; ++i) x[i] = w[0][i] * cur[i];
#pragma unroll
      for (int l = 1; l < kMaxWidth; ++l)
#pragma unroll
        for (int i = 0; i < 8; ++i) x[i] = fmaf(w[l][i], win[l - 1][i], x[i]);
      float y[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) y[i] = cur[i] + x[i] / (1.f + expf(-x[i]));
      const uint4 packed = f32_to_bf16x8(y);
      *reinterpret_cast<uint4*>(ko + (size_t)t * row_stride) = packed;
      float yr[8];
      bf16x8_to_f32(packed, yr);  // the centroid averages the stored bf16 keys
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[i] += yr[i];
#pragma unroll
      for (int l = kMaxWidth - 2; l > 0; --l)
#pragma unroll
        for (int i = 0; i < 8; ++i) win[l][i] = win[l - 1][i];
#pragma unroll
      for (int i = 0; i < 8; ++i) win[0][i] = cur[i];
    }
  }

  const float inv = 1.f / (float)(t1 - t0);
  float c[8], lo[8];
  bf16 hb[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    c[i] = acc[i] * inv;
    hb[i] = __float2bfloat16_rn(c[i]);
    lo[i] = c[i] - __bfloat162float(hb[i]);
  }
  const size_t o = ((size_t)h * nb_max + gb) * D + c8 * 8;
  reinterpret_cast<float4*>(cent + o)[0] = make_float4(c[0], c[1], c[2], c[3]);
  reinterpret_cast<float4*>(cent + o)[1] = make_float4(c[4], c[5], c[6], c[7]);
  float hf[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) hf[i] = __bfloat162float(hb[i]);
  *reinterpret_cast<uint4*>(cent_hi + o) = f32_to_bf16x8(hf);
  *reinterpret_cast<uint4*>(cent_lo + o) = f32_to_bf16x8(lo);
}

}  // namespace

cudaError_t launch_conv_centroid(const bf16* k, const float* conv_w, int conv_width, const SeqPlan& p,
                                 int h_kv, int d, int block_size, bf16* k_out, float* cent,
                                 bf16* cent_hi, bf16* cent_lo, cudaStream_t st) {
  if (conv_width > kMaxWidth) return cudaErrorInvalidValue;
  const long long threads = (long long)p.nb_max * h_kv * (d / 8);
  const int grid = (int)((threads + kThreads - 1) / kThreads);
  if (grid == 0) return cudaSuccess;
  if (d == 64)
    conv_centroid_kernel<64><<<grid, kThreads, 0, st>>>(k, conv_w, conv_width, p.cu, p.blk_off, p.batch, p.nb_max,
                                                        h_kv, block_size, k_out, cent, cent_hi, cent_lo);
  else
    conv_centroid_kernel<128><<<grid, kThreads, 0, st>>>(k, conv_w, conv_width, p.cu, p.blk_off, p.batch, p.nb_max,
                                                         h_kv, block_size, k_out, cent, cent_hi, cent_lo);
  return cudaGetLastError();
}

}  // namespace moba
