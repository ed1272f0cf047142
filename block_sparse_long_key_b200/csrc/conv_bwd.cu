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
// over blocks in a fixed order (deterministic).  Traffic: K and dK' read
// once (plus the halo rows), dK written once; the walk itself (about 30
// instructions per element with the register rings below) sets the time.
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

  // Register rings indexed by the step's residue mod W, which is a
  // compile-time constant inside the unrolled inner loop, so no value moves
  // between registers as u advances: kr[(r - l) % W] = k_{u-l},
  // gr[r % W] = dK'_u, pr[(r - l) % W] accumulates sum_m W_m g_{t+m} for
  // t = u - l (the slot of t = u - (W - 1) is emitted at step r and taken by
  // t = u + 1 at the next); dwa[l] = sum over the block's u of g_u k_{u-l}.
  constexpr int R = BLK + W - 1;  // steps u = t0 + r, r < R
  float kr[W], gr[W], pr[W], dwa[W];
#pragma unroll
  for (int l = 0; l < W; ++l) kr[l] = gr[l] = pr[l] = dwa[l] = 0.f;
#pragma unroll
  for (int l = 1; l < W; ++l) kr[W - l] = __bfloat162float(ks[(W - 1 - l) * Ly::SEG + ch]);  // k_{t0-l}
  const int n = t1 - t0;
  for (int r0 = 0; r0 < R; r0 += W) {
#pragma unroll
    for (int i = 0; i < W; ++i) {
      const int r = r0 + i;
      if (r < R) {
        kr[i] = __bfloat162float(ks[(W - 1 + r) * Ly::SEG + ch]);
        gr[i] = __bfloat162float(gs[r * Ly::SEG + ch]);
        float g = 0.f;
        if (t0 + r < seq1) {
          float x = 0.f;
#pragma unroll
          for (int l = 0; l < W; ++l) x = fmaf(w[l], kr[(i - l + W) % W], x);
          const float sg = __fdividef(1.f, 1.f + __expf(-x));
          g = gr[i] * sg * (1.f + x * (1.f - sg));
        }
        if (r < n) {
#pragma unroll
          for (int l = 0; l < W; ++l) dwa[l] = fmaf(g, kr[(i - l + W) % W], dwa[l]);
        }
        // t = u takes its first term here: assigning it also drops what the
        // first W - 1 steps added to this slot for tokens before the block
        pr[i] = w[0] * g;
#pragma unroll
        for (int l = 1; l < W; ++l) pr[(i - l + W) % W] = fmaf(w[l], g, pr[(i - l + W) % W]);
        if (r >= W - 1) {  // t = u - (W - 1) is complete (slot (i + 1) % W)
          const int sl = (i + 1) % W;
          os[(r - (W - 1)) * Ly::SEG + ch] = __float2bfloat16_rn(gr[sl] + pr[sl]);
        }
      }
    }
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

// dW[h][c][l] = sum over the blocks of head h.  One CTA per (head, 32
// consecutive (channel, tap) entries): lane i of warp w sums entry i over
// blocks w, w + 32, ... (each warp load is one 128-byte row piece), then
// warp 0 adds the 32 warp sums in a fixed order (deterministic).
constexpr int kDwThreads = 1024;
__global__ void __launch_bounds__(kDwThreads)
conv_dw_reduce_kernel(const float* __restrict__ dw_part, const int32_t* __restrict__ blk_off, int batch, int nb_max,
                      int dwid, float* __restrict__ dw) {
  __shared__ float part[32][33];
  const int groups = (dwid + 31) / 32;
  const int h = blockIdx.x / groups, cl = (blockIdx.x % groups) * 32 + (threadIdx.x & 31);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nb = __ldg(blk_off + batch);
  const float* src = dw_part + (size_t)h * nb_max * dwid + cl;
  float acc = 0.f;
  if (cl < dwid) {
#pragma unroll 4
    for (int b = warp; b < nb; b += 32) acc += __ldg(src + (size_t)b * dwid);
  }
  part[warp][lane] = acc;
  __syncthreads();
  if (warp == 0 && cl < dwid) {
    float t = 0.f;
#pragma unroll
    for (int w2 = 0; w2 < 32; ++w2) t += part[w2][lane];
    dw[(size_t)h * dwid + cl] = t;
  }
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
  const int groups = (D * W + 31) / 32;
  conv_dw_reduce_kernel<<<h_kv * groups, kDwThreads, 0, st>>>(dw_part, p.blk_off, p.batch, p.nb_max, D * W, dw);
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
