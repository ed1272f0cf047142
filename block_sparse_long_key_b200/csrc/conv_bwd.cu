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
// One CTA per (global block, group of KV heads), one thread per channel
// (256 channels: 4 heads at d = 64, 2 at d = 128).  The block's keys (with a
// W-1 row halo on both sides) and dK' (with the halo after it) are staged in
// shared memory by 16-byte cp.async copies of contiguous row segments, zero
// outside the sequence.  Each thread walks u = t0 .. t1+W-2 down its channel:
// it recomputes x_u from a register window of keys, forms g_u, adds W_l g_u
// to the pending outputs of t = u - l and emits dK_t into a shared output
// tile once u = t + W - 1; the tile leaves with 16-byte coalesced stores.
// Its block's dW partial goes to a per-block buffer that a second kernel sums
// over blocks in a fixed order (deterministic).  HBM-bound: K and dK' read
// once (plus the halo rows), dK written once.
#include "common.cuh"
#include "launch.h"

namespace moba {
namespace {

constexpr int kThreads = 256;  // channels per CTA

template <int D, int W, int BLK>
struct CbLayout {
  static constexpr int HG = kThreads / D;           // heads per CTA
  static constexpr int SEG = HG * D;                // channels (bf16) per staged row
  static constexpr int KROWS = BLK + 2 * (W - 1);   // keys t0-W+1 .. t0+BLK+W-2
  static constexpr int GROWS = BLK + W - 1;         // dK' t0 .. t0+BLK+W-2
  static constexpr uint32_t K_BYTES = KROWS * SEG * 2;
  static constexpr uint32_t G_BYTES = GROWS * SEG * 2;
  static constexpr uint32_t BYTES = K_BYTES + G_BYTES + BLK * SEG * 2;
};

template <int D, int W, int BLK>
__global__ void __launch_bounds__(kThreads)
conv_bwd_kernel(const bf16* __restrict__ k, const float* __restrict__ conv_w, const bf16* __restrict__ dkc,
                const int32_t* __restrict__ cu, const int32_t* __restrict__ blk_off, int batch, int nb_max, int h_kv,
                bf16* __restrict__ dk, float* __restrict__ dw_part) {
  using Ly = CbLayout<D, W, BLK>;
  extern __shared__ __align__(16) unsigned char smem[];
  bf16* ks = reinterpret_cast<bf16*>(smem);                                // [KROWS][SEG]
  bf16* gs = reinterpret_cast<bf16*>(smem + Ly::K_BYTES);                  // [GROWS][SEG]
  bf16* os = reinterpret_cast<bf16*>(smem + Ly::K_BYTES + Ly::G_BYTES);    // [BLK][SEG]

  const int gb = blockIdx.x;
  const int h0 = blockIdx.y * Ly::HG;
  if (gb >= __ldg(blk_off + batch)) return;
  const int s = upper_seq(blk_off, batch, gb);
  const int seq0 = __ldg(cu + s), seq1 = __ldg(cu + s + 1);
  const int t0 = seq0 + (gb - __ldg(blk_off + s)) * BLK;
  const int t1 = min(t0 + BLK, seq1);
  const int tid = threadIdx.x;
  const size_t rs = (size_t)h_kv * D;
  const int nh = min(Ly::HG, h_kv - h0);

  constexpr int CPR = Ly::SEG / 8;  // 16-byte chunks per staged row
  for (int i = tid; i < Ly::KROWS * CPR; i += kThreads) {
    const int r = i / CPR, c = i % CPR;
    const int t = t0 - (W - 1) + r;
    const bool ok = t >= seq0 && t < seq1 && c * 8 < nh * D;
    cp_async16_zfill(ks + r * Ly::SEG + c * 8, k + (ok ? (size_t)t * rs + (size_t)h0 * D + c * 8 : 0), ok);
  }
  for (int i = tid; i < Ly::GROWS * CPR; i += kThreads) {
    const int r = i / CPR, c = i % CPR;
    const int t = t0 + r;
    const bool ok = t < seq1 && c * 8 < nh * D;
    cp_async16_zfill(gs + r * Ly::SEG + c * 8, dkc + (ok ? (size_t)t * rs + (size_t)h0 * D + c * 8 : 0), ok);
  }
  cp_async_commit();
  const int ch = tid;
  const int h = h0 + ch / D, c = ch % D;
  float w[W];
#pragma unroll
  for (int l = 0; l < W; ++l) w[l] = h < h_kv ? __ldg(conv_w + ((size_t)h * D + c) * W + l) : 0.f;
  cp_async_wait<0>();
  __syncthreads();

  // kwin[l] = k_{u-l}; pend[l] accumulates sum_m W_m g_{t+m} for t = u - l;
  // dwa[l] = sum over the block's u of g_u k_{u-l}.
  float kwin[W], pend[W], dwa[W];
#pragma unroll
  for (int l = 0; l < W; ++l) {
    pend[l] = dwa[l] = 0.f;
    kwin[l] = l >= 1 ? __bfloat162float(ks[(W - 1 - l) * Ly::SEG + ch]) : 0.f;
  }
  const int n = t1 - t0;
#pragma unroll 2
  for (int r = 0; r < BLK + W - 1; ++r) {  // u = t0 + r
    kwin[0] = __bfloat162float(ks[(W - 1 + r) * Ly::SEG + ch]);
    float g = 0.f;
    if (t0 + r < seq1) {
      float x = 0.f;
#pragma unroll
      for (int l = 0; l < W; ++l) x = fmaf(w[l], kwin[l], x);
      const float sg = __frcp_rn(1.f + __expf(-x));
      g = __bfloat162float(gs[r * Ly::SEG + ch]) * sg * (1.f + x * (1.f - sg));
    }
    if (r < n) {
#pragma unroll
      for (int l = 0; l < W; ++l) dwa[l] = fmaf(g, kwin[l], dwa[l]);
    }
#pragma unroll
    for (int l = 0; l < W; ++l) pend[l] = fmaf(w[l], g, pend[l]);
    const int te = r - (W - 1);  // t = t0 + te is complete now
    if (te >= 0 && te < BLK)
      os[te * Ly::SEG + ch] = __float2bfloat16_rn(__bfloat162float(gs[te * Ly::SEG + ch]) + pend[W - 1]);
#pragma unroll
    for (int l = W - 1; l > 0; --l) {
      kwin[l] = kwin[l - 1];
      pend[l] = pend[l - 1];
    }
    pend[0] = 0.f;
  }
  __syncthreads();
  for (int i = tid; i < n * CPR; i += kThreads) {
    const int r = i / CPR, cc = i % CPR;
    if (cc * 8 < nh * D)
      *reinterpret_cast<uint4*>(dk + (size_t)(t0 + r) * rs + (size_t)h0 * D + cc * 8) =
          *reinterpret_cast<const uint4*>(os + r * Ly::SEG + cc * 8);
  }
  if (h < h_kv) {
    float* dst = dw_part + (((size_t)h * nb_max + gb) * D + c) * W;
#pragma unroll
    for (int l = 0; l < W; ++l) dst[l] = dwa[l];
  }
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
  if (p.nb_max == 0 || h_kv == 0) return cudaSuccess;
  const dim3 grid(p.nb_max, (h_kv + kThreads / D - 1) / (kThreads / D));
  cudaError_t e = cudaErrorInvalidValue;
#define MOBA_CB(BB)                                                                                        \
  {                                                                                                        \
    const size_t smem = CbLayout<D, W, BB>::BYTES;                                                         \
    auto kern = conv_bwd_kernel<D, W, BB>;                                                                 \
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);               \
    if (e != cudaSuccess) return e;                                                                        \
    kern<<<grid, kThreads, smem, st>>>(k, conv_w, dkc, p.cu, p.blk_off, p.batch, p.nb_max, h_kv, dk, dw_part); \
    e = cudaGetLastError();                                                                                \
    break;                                                                                                 \
  }
  switch (block_size) {
    case 16: MOBA_CB(16);
    case 32: MOBA_CB(32);
    case 64: MOBA_CB(64);
    case 128: MOBA_CB(128);
  }
#undef MOBA_CB
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
