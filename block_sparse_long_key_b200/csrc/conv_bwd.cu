// Backward of the depthwise causal key convolution.
//
// "Optimizing Mixture of Block Attention", §"Progettazione della
// Convoluzione delle Chiavi (Appendice B)", "Forma Formale":
// k'_t = k_t + SiLU(x_t), x_t = sum_{l<W} W_l (.) k_{t-l}.  With
// g_t = dK'_t (.) SiLU'(x_t), SiLU'(x) = s(x) (1 + x (1 - s(x))):
//   dK_t = dK'_t + sum_l W_l (.) g_{t+l}     (t + l inside the sequence)
//   dW_l = sum_t g_t (.) k_{t-l}
// (the bf16 rounding of k' is treated as the identity).
//
// One thread per (global block, KV head, 4 channels) walks u = t0 .. t1+W-2:
// it recomputes x_u from a register window of keys, forms g_u, adds W_l g_u
// to the pending outputs of t = u - l and emits dK_t once u = t + W - 1; its
// block's dW partial goes to a per-block buffer that a second kernel sums
// over blocks in a fixed order.  HBM-bound: K and dK' read once (plus a
// W-row halo), dK written once.
#include "common.cuh"
#include "launch.h"

namespace moba {
namespace {

constexpr int kThreads = 256;
constexpr int kCh = 4;  // channels per thread

__device__ __forceinline__ void load4(const bf16* p, float* f) {
  const uint2 u = __ldg(reinterpret_cast<const uint2*>(p));
  const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.x));
  const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.y));
  f[0] = a.x;
  f[1] = a.y;
  f[2] = b.x;
  f[3] = b.y;
}

template <int D, int W>
__global__ void __launch_bounds__(kThreads)
conv_bwd_kernel(const bf16* __restrict__ k, const float* __restrict__ conv_w, const bf16* __restrict__ dkc,
                const int32_t* __restrict__ cu, const int32_t* __restrict__ blk_off, int batch, int nb_max, int h_kv,
                int block_size, bf16* __restrict__ dk, float* __restrict__ dw_part) {
  constexpr int TPB = D / kCh;
  const long long gtid = (long long)blockIdx.x * kThreads + threadIdx.x;
  const int cc = (int)(gtid % TPB);
  const long long bidx = gtid / TPB;
  const int h = (int)(bidx / nb_max);
  const int gb = (int)(bidx % nb_max);
  if (h >= h_kv || gb >= __ldg(blk_off + batch)) return;
  const int s = upper_seq(blk_off, batch, gb);
  const int seq0 = __ldg(cu + s), seq1 = __ldg(cu + s + 1);
  const int t0 = seq0 + (gb - __ldg(blk_off + s)) * block_size;
  const int t1 = min(t0 + block_size, seq1);
  const size_t rs = (size_t)h_kv * D;
  const size_t coff = (size_t)h * D + cc * kCh;

  float w[W][kCh];
#pragma unroll
  for (int l = 0; l < W; ++l)
#pragma unroll
    for (int i = 0; i < kCh; ++i) w[l][i] = __ldg(conv_w + ((size_t)h * D + cc * kCh + i) * W + l);
  // kwin[l] = k_{u-l} (l >= 1 before the step), gwin / dwin / pend indexed
  // by the distance back from u.
  float kwin[W][kCh], dwin[W][kCh], pend[W][kCh], dwa[W][kCh];
#pragma unroll
  for (int l = 0; l < W; ++l)
#pragma unroll
    for (int i = 0; i < kCh; ++i) kwin[l][i] = dwin[l][i] = pend[l][i] = dwa[l][i] = 0.f;
#pragma unroll
  for (int l = 1; l < W; ++l)
    if (t0 - l >= seq0) load4(k + (size_t)(t0 - l) * rs + coff, kwin[l]);

#pragma unroll 2
  for (int u = t0; u <= t1 + W - 2; ++u) {
    float ku[kCh] = {0.f, 0.f, 0.f, 0.f}, du[kCh] = {0.f, 0.f, 0.f, 0.f}, g[kCh] = {0.f, 0.f, 0.f, 0.f};
    const bool in_seq = u < seq1;
    if (in_seq) {
      load4(k + (size_t)u * rs + coff, ku);
      load4(dkc + (size_t)u * rs + coff, du);
    }
#pragma unroll
    for (int i = 0; i < kCh; ++i) kwin[0][i] = ku[i];
    if (in_seq) {
#pragma unroll
      for (int i = 0; i < kCh; ++i) {
        float x = 0.f;
#pragma unroll
        for (int l = 0; l < W; ++l) x = fmaf(w[l][i], kwin[l][i], x);
        const float sg = 1.f / (1.f + expf(-x));
        g[i] = du[i] * sg * (1.f + x * (1.f - sg));
      }
    }
    if (u < t1) {
#pragma unroll
      for (int l = 0; l < W; ++l)
#pragma unroll
        for (int i = 0; i < kCh; ++i) dwa[l][i] = fmaf(g[i], kwin[l][i], dwa[l][i]);
    }
    // pending outputs: pend[l] belongs to t = u - l
#pragma unroll
    for (int i = 0; i < kCh; ++i) dwin[0][i] = du[i];
#pragma unroll
    for (int l = 0; l < W; ++l)
#pragma unroll
      for (int i = 0; i < kCh; ++i) pend[l][i] = fmaf(w[l][i], g[i], pend[l][i]);
    const int te = u - (W - 1);  // complete now
    if (te >= t0 && te < t1) {
      float o[kCh];
#pragma unroll
      for (int i = 0; i < kCh; ++i) o[i] = dwin[W - 1][i] + pend[W - 1][i];
      uint2 packed;
      packed.x = pack_bf16(o[0], o[1]);
      packed.y = pack_bf16(o[2], o[3]);
      *reinterpret_cast<uint2*>(dk + (size_t)te * rs + coff) = packed;
    }
    // shift every window by one token
#pragma unroll
    for (int l = W - 1; l > 0; --l)
#pragma unroll
      for (int i = 0; i < kCh; ++i) {
        kwin[l][i] = kwin[l - 1][i];
        dwin[l][i] = dwin[l - 1][i];
        pend[l][i] = pend[l - 1][i];
      }
#pragma unroll
    for (int i = 0; i < kCh; ++i) pend[0][i] = 0.f;
  }
  float* dst = dw_part + (((size_t)h * nb_max + gb) * D + cc * kCh) * W;
#pragma unroll
  for (int i = 0; i < kCh; ++i)
#pragma unroll
    for (int l = 0; l < W; ++l) dst[i * W + l] = dwa[l][i];
}

// dW[h][c][l] = sum over the blocks of head h: one warp per output, lane i
// sums blocks i, i+32, ..., then a fixed shuffle tree (deterministic).
__global__ void __launch_bounds__(kThreads)
conv_dw_reduce_kernel(const float* __restrict__ dw_part, const int32_t* __restrict__ blk_off, int batch, int nb_max,
                      int h_kv, int dwid, float* __restrict__ dw) {
  const int i = (blockIdx.x * kThreads + threadIdx.x) >> 5;  // over h_kv * dwid
  const int lane = threadIdx.x & 31;
  if (i >= h_kv * dwid) return;
  const int h = i / dwid, cl = i % dwid;
  const int nb = __ldg(blk_off + batch);
  const float* src = dw_part + (size_t)h * nb_max * dwid + cl;
  float acc = 0.f;
#pragma unroll 4
  for (int b = lane; b < nb; b += 32) acc += __ldg(src + (size_t)b * dwid);
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
  if (lane == 0) dw[i] = acc;
}

template <int D, int W>
cudaError_t launch_conv_bwd_t(const bf16* k, const float* conv_w, const bf16* dkc, const SeqPlan& p, int h_kv,
                              int block_size, bf16* dk, float* dw, float* dw_part, cudaStream_t st) {
  const long long threads = (long long)p.nb_max * h_kv * (D / kCh);
  const int grid = (int)((threads + kThreads - 1) / kThreads);
  if (grid == 0) return cudaSuccess;
  conv_bwd_kernel<D, W><<<grid, kThreads, 0, st>>>(k, conv_w, dkc, p.cu, p.blk_off, p.batch, p.nb_max, h_kv,
                                                   block_size, dk, dw_part);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const long long nthreads = (long long)h_kv * D * W * 32;
  conv_dw_reduce_kernel<<<(int)((nthreads + kThreads - 1) / kThreads), kThreads, 0, st>>>(dw_part, p.blk_off, p.batch,
                                                                                         p.nb_max, h_kv, D * W, dw);
  return cudaGetLastError();
}

template <int D>
cudaError_t launch_conv_bwd_d(const bf16* k, const float* conv_w, int width, const bf16* dkc, const SeqPlan& p,
                              int h_kv, int block_size, bf16* dk, float* dw, float* dw_part, cudaStream_t st) {
  switch (width) {
    case 1: return launch_conv_bwd_t<D, 1>(k, conv_w, dkc, p, h_kv, block_size, dk, dw, dw_part, st);
    case 2: return launch_conv_bwd_t<D, 2>(k, conv_w, dkc, p, h_kv, block_size, dk, dw, dw_part, st);
    case 3: return launch_conv_bwd_t<D, 3>(k, conv_w, dkc, p, h_kv, block_size, dk, dw, dw_part, st);
    case 4: return launch_conv_bwd_t<D, 4>(k, conv_w, dkc, p, h_kv, block_size, dk, dw, dw_part, st);
    case 5: return launch_conv_bwd_t<D, 5>(k, conv_w, dkc, p, h_kv, block_size, dk, dw, dw_part, st);
    case 6: return launch_conv_bwd_t<D, 6>(k, conv_w, dkc, p, h_kv, block_size, dk, dw, dw_part, st);
    case 7: return launch_conv_bwd_t<D, 7>(k, conv_w, dkc, p, h_kv, block_size, dk, dw, dw_part, st);
    case 8: return launch_conv_bwd_t<D, 8>(k, conv_w, dkc, p, h_kv, block_size, dk, dw, dw_part, st);
  }
  return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_conv_bwd(const bf16* k, const float* conv_w, int conv_width, const bf16* dk_conv, const SeqPlan& p,
                            int h_kv, int d, int block_size, bf16* dk, float* dw, float* dw_part, cudaStream_t st) {
  if (d == 64) return launch_conv_bwd_d<64>(k, conv_w, conv_width, dk_conv, p, h_kv, block_size, dk, dw, dw_part, st);
  return launch_conv_bwd_d<128>(k, conv_w, conv_width, dk_conv, p, h_kv, block_size, dk, dw, dw_part, st);
}

}  // namespace moba
