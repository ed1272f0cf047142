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
// One CTA per (global key block, group of KV heads) with one thread per
// channel (256 channels: 4 heads at d = 64, 2 at d = 128).  The block's rows
// (plus the W-1 rows before it, zero outside the sequence) are staged in
// shared memory with 16-byte cp.async copies of whole contiguous row
// segments; each thread then walks its channel down the rows with the W taps
// and the last W-1 keys in registers, writes k' into a shared output tile
// (stored back with 16-byte coalesced stores) and sums the stored bf16 keys
// in ascending token order (fp32), dividing by the block's token count.
// HBM-bound: B*d*2 bytes read per (block, head), the same written with conv.
#include "common.cuh"
#include "launch.h"

namespace moba {
namespace {

constexpr int kThreads = 256;   // channels per CTA
constexpr int kMaxWidth = 8;
constexpr int kMaxBlock = 128;

template <int D, int W, int BLK>
struct CcLayout {
  static constexpr int HG = kThreads / D;           // heads per CTA
  static constexpr int SEG = HG * D;                // channels (bf16) per staged row
  static constexpr int PRE = W > 1 ? W - 1 : 0;     // rows staged before the block
  static constexpr int ROWS = BLK + PRE;
  static constexpr uint32_t IN_BYTES = ROWS * SEG * 2;
  static constexpr uint32_t OUT_BYTES = W > 0 ? BLK * SEG * 2 : 0;
  static constexpr uint32_t BYTES = IN_BYTES + OUT_BYTES;
};

template <int D, int W, int BLK>
__global__ void __launch_bounds__(kThreads)
conv_centroid_kernel(const bf16* __restrict__ k, const float* __restrict__ conv_w, const int32_t* __restrict__ cu,
                     const int32_t* __restrict__ blk_off, int batch, int nb_max, int h_kv, bf16* __restrict__ k_out,
                     float* __restrict__ cent, bf16* __restrict__ cent_hi, bf16* __restrict__ cent_lo,
                     float* __restrict__ cent_norm_max) {
  using Ly = CcLayout<D, W, BLK>;
  extern __shared__ __align__(16) unsigned char smem[];
  bf16* in = reinterpret_cast<bf16*>(smem);                    // [ROWS][SEG]
  bf16* outt = reinterpret_cast<bf16*>(smem + Ly::IN_BYTES);   // [BLK][SEG]

  const int gb = blockIdx.x;
  const int h0 = blockIdx.y * Ly::HG;
  if (gb >= __ldg(blk_off + batch)) return;
  const int s = upper_seq(blk_off, batch, gb);
  const int seq0 = __ldg(cu + s), seq1 = __ldg(cu + s + 1);
  const int t0 = seq0 + (gb - __ldg(blk_off + s)) * BLK;
  const int t1 = min(t0 + BLK, seq1);
  const int tid = threadIdx.x;
  const size_t row_stride = (size_t)h_kv * D;
  const int nh = min(Ly::HG, h_kv - h0);                       // heads of this CTA that exist

  // ---- stage rows t0-PRE .. t0+BLK-1 (zero outside [seq0, t1))
  constexpr int CPR = Ly::SEG / 8;                             // 16-byte chunks per staged row
  for (int i = tid; i < Ly::ROWS * CPR; i += kThreads) {
    const int r = i / CPR, c = i % CPR;
    const int t = t0 - Ly::PRE + r;
    const bool ok = t >= seq0 && t < t1 && c * 8 < nh * D;
    const size_t off = ok ? (size_t)t * row_stride + (size_t)h0 * D + c * 8 : 0;
    cp_async16_zfill(in + r * Ly::SEG + c * 8, k + off, ok);
  }
  cp_async_commit();
  const int ch = tid;                                          // channel within the segment
  const int h = h0 + ch / D, c = ch % D;
  float w[W > 0 ? W : 1];
#pragma unroll
  for (int l = 0; l < W; ++l) w[l] = h < h_kv ? __ldg(conv_w + ((size_t)h * D + c) * W + l) : 0.f;
  cp_async_wait<0>();
  __syncthreads();

  const int n = t1 - t0;
  float acc = 0.f;
  if constexpr (W == 0) {
    for (int r = 0; r < n; ++r) acc += __bfloat162float(in[r * Ly::SEG + ch]);
  } else {
    // Register ring indexed by the row's residue mod W (a compile-time
    // constant inside the unrolled inner loop, so no value moves as t
    // advances): kr[(r - l) % W] = k_{t-l} for t = t0 + r.
    float kr[W];
#pragma unroll
    for (int l = 0; l < W; ++l) kr[l] = 0.f;
#pragma unroll
    for (int l = 1; l < W; ++l) kr[W - l] = __bfloat162float(in[(Ly::PRE - l) * Ly::SEG + ch]);  // k_{t0-l}
    for (int r0 = 0; r0 < BLK; r0 += W) {
#pragma unroll
      for (int i = 0; i < W; ++i) {
        const int r = r0 + i;
        if (r < BLK) {
          kr[i] = __bfloat162float(in[(Ly::PRE + r) * Ly::SEG + ch]);
          float x = 0.f;
#pragma unroll
          for (int l = 0; l < W; ++l) x = fmaf(w[l], kr[(i - l + W) % W], x);
          const bf16 y = __float2bfloat16_rn(kr[i] + __fdividef(x, 1.f + __expf(-x)));  // k + SiLU(x)
          outt[r * Ly::SEG + ch] = y;
          if (r < n) acc += __bfloat162float(y);  // the centroid averages the stored bf16 keys
        }
      }
    }
    __syncthreads();
    for (int i = tid; i < n * CPR; i += kThreads) {
      const int r = i / CPR, cc = i % CPR;
      if (cc * 8 < nh * D)
        *reinterpret_cast<uint4*>(k_out + (size_t)(t0 + r) * row_stride + (size_t)h0 * D + cc * 8) =
            *reinterpret_cast<const uint4*>(outt + r * Ly::SEG + cc * 8);
    }
  }
  const float cv = h < h_kv ? acc / (float)n : 0.f;
  if (h < h_kv) {
    const bf16 hb = __float2bfloat16_rn(cv);
    const size_t o = ((size_t)h * nb_max + gb) * D + c;
    cent[o] = cv;
    cent_hi[o] = hb;
    cent_lo[o] = __float2bfloat16_rn(cv - __bfloat162float(hb));
  }
  if (cent_norm_max) {
    // Largest centroid norm of each KV head (the router's screen pass bounds
    // the part of a score it leaves out by it): a head's D channels are
    // D / 32 whole warps; their squares meet in shared memory.
    __shared__ float nrm2[Ly::HG];
    if (tid < Ly::HG) nrm2[tid] = 0.f;
    __syncthreads();
    float sq = cv * cv;
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, off);
    if ((tid & 31) == 0) atomicAdd(&nrm2[ch / D], sq);
    __syncthreads();
    if (tid < nh)  // non-negative floats order like their bit patterns
      atomicMax(reinterpret_cast<int*>(cent_norm_max) + h0 + tid, __float_as_int(sqrtf(nrm2[tid])));
  }
}

template <int D, int W>
cudaError_t launch_cc_w(const bf16* k, const float* conv_w, const SeqPlan& p, int h_kv, int block_size, bf16* k_out,
                        float* cent, bf16* cent_hi, bf16* cent_lo, float* cnorm, cudaStream_t st) {
  const dim3 grid(p.nb_max, (h_kv + kThreads / D - 1) / (kThreads / D));
#define MOBA_CC(BB)                                                                                      \
  {                                                                                                      \
    const size_t smem = CcLayout<D, W, BB>::BYTES;                                                       \
    auto kern = conv_centroid_kernel<D, W, BB>;                                                          \
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem); \
    if (e != cudaSuccess) return e;                                                                      \
    kern<<<grid, kThreads, smem, st>>>(k, conv_w, p.cu, p.blk_off, p.batch, p.nb_max, h_kv, k_out, cent,  \
                                       cent_hi, cent_lo, cnorm);                                         \
    return cudaGetLastError();                                                                           \
  }
  switch (block_size) {
    case 16: MOBA_CC(16);
    case 32: MOBA_CC(32);
    case 64: MOBA_CC(64);
    case 128: MOBA_CC(128);
  }
#undef MOBA_CC
  return cudaErrorInvalidValue;
}

template <int D>
cudaError_t launch_cc_d(const bf16* k, const float* conv_w, int conv_width, const SeqPlan& p, int h_kv,
                        int block_size, bf16* k_out, float* cent, bf16* cent_hi, bf16* cent_lo, float* cnorm,
                        cudaStream_t st) {
  switch (conv_width) {
    case 0: return launch_cc_w<D, 0>(k, conv_w, p, h_kv, block_size, k_out, cent, cent_hi, cent_lo, cnorm, st);
    case 1: return launch_cc_w<D, 1>(k, conv_w, p, h_kv, block_size, k_out, cent, cent_hi, cent_lo, cnorm, st);
    case 2: return launch_cc_w<D, 2>(k, conv_w, p, h_kv, block_size, k_out, cent, cent_hi, cent_lo, cnorm, st);
    case 3: return launch_cc_w<D, 3>(k, conv_w, p, h_kv, block_size, k_out, cent, cent_hi, cent_lo, cnorm, st);
    case 4: return launch_cc_w<D, 4>(k, conv_w, p, h_kv, block_size, k_out, cent, cent_hi, cent_lo, cnorm, st);
    case 5: return launch_cc_w<D, 5>(k, conv_w, p, h_kv, block_size, k_out, cent, cent_hi, cent_lo, cnorm, st);
    case 6: return launch_cc_w<D, 6>(k, conv_w, p, h_kv, block_size, k_out, cent, cent_hi, cent_lo, cnorm, st);
    case 7: return launch_cc_w<D, 7>(k, conv_w, p, h_kv, block_size, k_out, cent, cent_hi, cent_lo, cnorm, st);
    case 8: return launch_cc_w<D, 8>(k, conv_w, p, h_kv, block_size, k_out, cent, cent_hi, cent_lo, cnorm, st);
  }
  return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_conv_centroid(const bf16* k, const float* conv_w, int conv_width, const SeqPlan& p,
                                 int h_kv, int d, int block_size, bf16* k_out, float* cent,
                                 bf16* cent_hi, bf16* cent_lo, float* cent_norm_max, cudaStream_t st) {
  if (conv_width < 0 || conv_width > kMaxWidth || block_size > kMaxBlock) return cudaErrorInvalidValue;
  if (p.nb_max == 0 || h_kv == 0) return cudaSuccess;
  if (d == 64)
    return launch_cc_d<64>(k, conv_w, conv_width, p, h_kv, block_size, k_out, cent, cent_hi, cent_lo, cent_norm_max,
                           st);
  return launch_cc_d<128>(k, conv_w, conv_width, p, h_kv, block_size, k_out, cent, cent_hi, cent_lo, cent_norm_max,
                          st);
}

}  // namespace moba
