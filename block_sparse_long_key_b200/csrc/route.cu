// Router: block scores on tensor cores and per-query top-k in registers.
//
// "Optimizing Mixture of Block Attention", §"Architettura del Modello
// Statistico" 1 (router score s_j = q^T k~_j) and §"Definizione del Compito"
// (each query keeps the top-k blocks, k << n); the FlashMoBA "Flash TopK"
// stage 2 (§"Progettazione del Kernel FlashMoBA", "Tre Kernel Fusi" 1)
// computes these scores tile by tile without materialising the N x n matrix;
// this kernel does the same on sm_100a.
//
// Selection rule: a query at local position p (block b = p / B) scores the
// earlier blocks j < b only, keeps the topk-1 best (exact ties: lower j
// wins) and always keeps its own block b.  sel_idx rows are sorted
// ascending and padded with -1.
//
// A CTA owns 64 consecutive queries of one sequence and one query head.
// Centroid tiles of 64 blocks stream through shared memory (cp.async, double
// buffered); each warp forms a 16 x 64 score tile with bf16 mma (fp32
// accumulate) as q.c_hi + q.c_lo, which carries ~16 mantissa bits of the fp32
// centroid.  Two threads per query row then fold the tile into a running
// top-(k-1) list held in registers as 64-bit keys (order-preserving float
// bits << 32 | ~index): one compare per score, an insertion pass only when a
// score beats the current threshold.
//
// Side outputs for the forward: mref = a lower bound of the query's largest
// attention logit, max(best kept score, q_i.k_i) / sqrt(d) (a block mean never
// exceeds the block max), used as the fixed softmax reference; the query's
// accumulator row (oacc, lacc, flag) is zeroed here.
#include "common.cuh"
#include "launch.h"

namespace moba {
namespace {

constexpr int kTM = kRouteTile;  // query rows per CTA
constexpr int kNC = 64;          // blocks per centroid chunk
constexpr int kThreads = 128;
constexpr uint64_t kSentinel = ~0ull;

__device__ __forceinline__ uint32_t order_bits(float v) {
  uint32_t u = __float_as_uint(v);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float from_order_bits(uint32_t u) {
  return __uint_as_float((u & 0x80000000u) ? (u & 0x7fffffffu) : ~u);
}
__device__ __forceinline__ uint64_t make_key(float v, int j) {
  return ((uint64_t)order_bits(v) << 32) | (uint64_t)(0xffffffffu - (uint32_t)j);
}

template <int LISTN>
__device__ __forceinline__ void list_insert(uint64_t (&L)[LISTN], uint64_t key) {
  if (key <= L[LISTN - 1]) return;
  uint64_t x = key;
#pragma unroll
  for (int m = 0; m < LISTN; ++m) {
    const uint64_t a = L[m];
    L[m] = a > x ? a : x;
    x = a > x ? x : a;
  }
}

template <int D>
struct RouteSmem {
  bf16 q[kTM][D + 8];
  bf16 ch[2][kNC][D + 8];
  bf16 cl[2][kNC][D + 8];
  float s[kTM][kNC + 2];
};

template <int D, int LISTN>
__global__ void __launch_bounds__(kThreads)
route_kernel(const bf16* __restrict__ q, const bf16* __restrict__ k, const bf16* __restrict__ cent_hi,
             const bf16* __restrict__ cent_lo, const int32_t* __restrict__ cu,
             const int32_t* __restrict__ blk_off, const int32_t* __restrict__ tile_off, int batch,
             int nb_max, int h_q, int h_kv, int block_size, int topk, int32_t* __restrict__ sel_idx,
             float* __restrict__ mref, int32_t* __restrict__ flag, float* __restrict__ lacc,
             float* __restrict__ oacc) {
  extern __shared__ __align__(128) unsigned char smem_raw[];
  RouteSmem<D>& sm = *reinterpret_cast<RouteSmem<D>*>(smem_raw);

  const int ntiles = __ldg(tile_off + batch);
  const int tile = ntiles - 1 - (int)blockIdx.x;  // longest rows first
  if (tile < 0) return;
  const int h = blockIdx.y;
  const int kvh = h / (h_q / h_kv);
  const int s = upper_seq(tile_off, batch, tile);
  const int seq0 = __ldg(cu + s);
  const int L = __ldg(cu + s + 1) - seq0;
  const int p0 = (tile - __ldg(tile_off + s)) * kTM;
  const int nrows = min(kTM, L - p0);
  const int t0 = seq0 + p0;
  const int cbase = __ldg(blk_off + s);
  const int nscan = (p0 + nrows - 1) / block_size;  // blocks any row may score
  const int nchunks = (nscan + kNC - 1) / kNC;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const size_t qstride = (size_t)h_q * D;

  // Q tile (zero rows past the sequence end).
  for (int i = tid; i < kTM * (D / 8); i += kThreads) {
    const int r = i / (D / 8), c = i % (D / 8);
    const bool ok = r < nrows;
    cp_async16_zfill(&sm.q[r][c * 8], q + (ok ? (size_t)(t0 + r) * qstride + (size_t)h * D + c * 8 : 0), ok);
  }
  auto load_chunk = [&](int c, int buf) {
    const size_t head0 = ((size_t)kvh * nb_max + cbase) * D;
    for (int i = tid; i < kNC * (D / 8); i += kThreads) {
      const int n = i / (D / 8), cc = i % (D / 8);
      const int jb = c * kNC + n;
      const bool ok = jb < nscan;
      const size_t off = ok ? head0 + (size_t)jb * D + cc * 8 : 0;
      cp_async16_zfill(&sm.ch[buf][n][cc * 8], cent_hi + off, ok);
      cp_async16_zfill(&sm.cl[buf][n][cc * 8], cent_lo + off, ok);
    }
  };
  if (nchunks > 0) load_chunk(0, 0);
  cp_async_commit();

  // Zero this tile's accumulator rows while the loads fly.
  for (int i = tid; i < nrows * (D / 4); i += kThreads) {
    const int r = i / (D / 4), c = i % (D / 4);
    const size_t row = (size_t)(t0 + r) * h_q + h;
    reinterpret_cast<float4*>(oacc + row * D)[c] = make_float4(0.f, 0.f, 0.f, 0.f);
  }

  // Per-thread running list: row r = tid / 2, column parity = tid % 2.
  const int my_row = tid >> 1, parity = tid & 1;
  const int my_b = (p0 + my_row) / block_size;
  const int k1 = topk - 1;
  uint64_t list[LISTN];
#pragma unroll
  for (int m = 0; m < LISTN; ++m) list[m] = m < LISTN - k1 ? kSentinel : 0ull;

  uint32_t qa[D / 16][4];
  for (int c = 0; c < nchunks; ++c) {
    const int buf = c & 1;
    if (c + 1 < nchunks) load_chunk(c + 1, buf ^ 1);
    cp_async_commit();
    cp_async_wait<1>();
    __syncthreads();
    if (c == 0) {
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const int r = warp * 16 + (lane & 15), col = kk * 16 + (lane >> 4) * 8;
        ldsm_x4(qa[kk][0], qa[kk][1], qa[kk][2], qa[kk][3], &sm.q[r][col]);
      }
    }
    float acc[kNC / 8][4];
#pragma unroll
    for (int nt = 0; nt < kNC / 8; ++nt)
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[nt][i] = 0.f;
#pragma unroll
    for (int nt2 = 0; nt2 < kNC / 16; ++nt2) {
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const int n = nt2 * 16 + (lane & 7) + ((lane >> 4) << 3);
        const int col = kk * 16 + ((lane >> 3) & 1) * 8;
        uint32_t b0, b1, b2, b3;
        ldsm_x4(b0, b1, b2, b3, &sm.ch[buf][n][col]);
        mma_bf16(acc[2 * nt2], qa[kk], b0, b1);
        mma_bf16(acc[2 * nt2 + 1], qa[kk], b2, b3);
        ldsm_x4(b0, b1, b2, b3, &sm.cl[buf][n][col]);
        mma_bf16(acc[2 * nt2], qa[kk], b0, b1);
        mma_bf16(acc[2 * nt2 + 1], qa[kk], b2, b3);
      }
    }
#pragma unroll
    for (int nt = 0; nt < kNC / 8; ++nt) {
      const int r = warp * 16 + (lane >> 2), col = nt * 8 + (lane & 3) * 2;
      *reinterpret_cast<float2*>(&sm.s[r][col]) = make_float2(acc[nt][0], acc[nt][1]);
      *reinterpret_cast<float2*>(&sm.s[r + 8][col]) = make_float2(acc[nt][2], acc[nt][3]);
    }
    __syncthreads();
    if (k1 > 0 && my_row < nrows) {
      const int jlim = min(my_b - c * kNC, kNC);  // columns [0, jlim) are past blocks of my row
#pragma unroll 8
      for (int i = 0; i < kNC / 2; ++i) {
        const int col = 2 * i + parity;
        if (col < jlim) list_insert<LISTN>(list, make_key(sm.s[my_row][col], c * kNC + col));
      }
    }
  }
  cp_async_wait<0>();
  __syncthreads();

  // Merge the two half lists of each row (odd threads hand theirs over).
  // ch and cl are adjacent: together they hold the [kTM][LISTN] hand-over.
  uint64_t* xfer = reinterpret_cast<uint64_t*>(&sm.ch[0][0][0]);
  static_assert(sizeof(sm.ch) + sizeof(sm.cl) >= sizeof(uint64_t) * kTM * LISTN, "merge buffer");
  if (parity == 1) {
#pragma unroll
    for (int m = 0; m < LISTN; ++m) xfer[my_row * LISTN + m] = list[m];
  }
  __syncthreads();
  int32_t* idx_buf = reinterpret_cast<int32_t*>(&sm.s[0][0]);  // [kTM][LISTN + 1]
  static_assert(sizeof(sm.s) >= sizeof(int32_t) * kTM * (LISTN + 1), "index buffer");
  if (parity == 0 && my_row < nrows) {
    for (int m = 0; m < LISTN; ++m) {
      const uint64_t key = xfer[my_row * LISTN + m];
      if (key != kSentinel && key != 0ull) list_insert<LISTN>(list, key);
    }
    // Kept past blocks (unordered), best score for the softmax reference.
    int* mine = idx_buf + my_row * (LISTN + 1);
    int cnt = 0;
    float best = -INFINITY;
#pragma unroll
    for (int m = 0; m < LISTN; ++m) {
      const uint64_t key = list[m];
      if (key != kSentinel && key != 0ull) {
        mine[cnt++] = (int)(0xffffffffu - (uint32_t)(key & 0xffffffffu));
        best = fmaxf(best, from_order_bits((uint32_t)(key >> 32)));
      }
    }
    // Insertion sort ascending (at most 63 entries, once per query).
    for (int a = 1; a < cnt; ++a) {
      const int x = mine[a];
      int b2 = a - 1;
      while (b2 >= 0 && mine[b2] > x) {
        mine[b2 + 1] = mine[b2];
        --b2;
      }
      mine[b2 + 1] = x;
    }
    const int t = t0 + my_row;
    const size_t row = (size_t)t * h_q + h;
    int32_t* out = sel_idx + row * topk;
    for (int m = 0; m < topk; ++m) out[m] = m < cnt ? mine[m] : (m == cnt ? my_b : -1);
    // q_i . k_i for the diagonal logit (own key is always visible).
    const bf16* krow = k + ((size_t)t * h_kv + kvh) * D;
    float dot = 0.f;
#pragma unroll 4
    for (int c8 = 0; c8 < D / 8; ++c8) {
      float fk[8], fq[8];
      bf16x8_to_f32(__ldg(reinterpret_cast<const uint4*>(krow + c8 * 8)), fk);
      bf16x8_to_f32(*reinterpret_cast<const uint4*>(&sm.q[my_row][c8 * 8]), fq);
#pragma unroll
      for (int i = 0; i < 8; ++i) dot = fmaf(fq[i], fk[i], dot);
    }
    mref[row] = fmaxf(best, dot) * rsqrtf((float)D);
    flag[row] = 0;
    lacc[row] = 0.f;
  }
}

template <int D, int LISTN>
cudaError_t launch_route_t(const bf16* q, const bf16* k, const bf16* hi, const bf16* lo, const SeqPlan& p,
                           int h_q, int h_kv, int block_size, int topk, int32_t* sel, float* mref,
                           int32_t* flag, float* lacc, float* oacc, cudaStream_t st) {
  const size_t smem = sizeof(RouteSmem<D>);
  auto kern = route_kernel<D, LISTN>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int max_tiles = p.total_tokens / kTM + p.batch;
  if (max_tiles == 0) return cudaSuccess;
  dim3 grid(max_tiles, h_q);
  kern<<<grid, kThreads, smem, st>>>(q, k, hi, lo, p.cu, p.blk_off, p.tile_off, p.batch, p.nb_max, h_q, h_kv,
                                     block_size, topk, sel, mref, flag, lacc, oacc);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_route(const bf16* q, const bf16* k, const bf16* hi, const bf16* lo, const SeqPlan& p,
                         int h_q, int h_kv, int d, int block_size, int topk, int32_t* sel, float* mref,
                         int32_t* flag, float* lacc, float* oacc, cudaStream_t st) {
  const int k1 = topk - 1;
#define MOBA_ROUTE(DD, LN) \
  return launch_route_t<DD, LN>(q, k, hi, lo, p, h_q, h_kv, block_size, topk, sel, mref, flag, lacc, oacc, st)
  if (d == 64) {
    if (k1 <= 8) MOBA_ROUTE(64, 8);
    if (k1 <= 16) MOBA_ROUTE(64, 16);
    if (k1 <= 32) MOBA_ROUTE(64, 32);
    MOBA_ROUTE(64, 64);
  } else {
    if (k1 <= 8) MOBA_ROUTE(128, 8);
    if (k1 <= 16) MOBA_ROUTE(128, 16);
    if (k1 <= 32) MOBA_ROUTE(128, 32);
    MOBA_ROUTE(128, 64);
  }
#undef MOBA_ROUTE
}

}  // namespace moba
