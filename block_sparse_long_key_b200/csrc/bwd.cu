// Backward of the sparse attention: recompute per key block.
//
// "Optimizing Mixture of Block Attention", §"Progettazione del Kernel
// FlashMoBA", "Tre Kernel Fusi" 3 ("Backward Pass: Ricalcolo": parallel over
// key blocks, one thread block per key block, the same gather-and-densify
// pattern as the forward, attention scores recomputed instead of stored, and
// partial dQ accumulated with atomic adds into a high-precision global
// buffer) and §"Efficienza Backward Pass".
//
// With the selection fixed, P = exp(S/sqrt(d) - LSE), D_i = dO_i . O_i,
// dV_j += P^T dO, dS = P (.) (dO V^T - D), dK_j += dS^T Q / sqrt(d),
// dQ += dS K_j / sqrt(d) (fp32 reductions).
//
// One CTA per (global key block, KV head) owns dK_j and dV_j for the whole
// block (all query heads of the group land in the same bucket), so they are
// accumulated in registers and written once, without atomics.  The keys are
// the MMA M dimension: each warp holds 16 keys x 32 gathered rows, computes
// S^T = K Q^T and dP^T = V dO^T, and feeds P^T and dS^T straight from the
// accumulator registers into dV += P^T dO and dK += dS^T Q.  dS^T goes to
// shared memory once for dQ = dS K, which every warp shares by 16x32 output
// tiles and adds to the fp32 dQ buffer with 16-byte vector reductions (lane
// pairs exchange halves so each lane holds 4 consecutive columns of a row).
#include <algorithm>

#include "common.cuh"
#include "launch.h"

namespace moba {
namespace {

template <int D, int BLK>
struct BwdCfg {
  static constexpr int TR = BLK <= 64 ? 64 : 32;  // gathered rows per tile
  static constexpr int RW = TR / 32;              // row groups of 32
  static constexpr int KG = BLK / 16;             // key groups of 16
  static constexpr int NW = KG * RW;              // warps
  static constexpr int NT = NW * 32;
};

template <int D, int BLK>
struct BwdSmem {
  using C = BwdCfg<D, BLK>;
  bf16 k[BLK][D + 8];
  bf16 v[BLK][D + 8];
  bf16 q[2][C::TR][D + 8];
  bf16 dout[2][C::TR][D + 8];
  bf16 dst[BLK][C::TR + 8];
  int32_t row[2][C::TR];
  int32_t tok[2][C::TR];
  float lse2[2][C::TR];
  float dsum[2][C::TR];
};

template <int D, int BLK>
__global__ void __launch_bounds__(BwdCfg<D, BLK>::NT)
bwd_attn_kernel(const bf16* __restrict__ q, const bf16* __restrict__ k, const bf16* __restrict__ v,
                const bf16* __restrict__ dout, const float* __restrict__ lse, const float* __restrict__ dsum,
                const int32_t* __restrict__ cu, const int32_t* __restrict__ blk_off, int batch, int nb_max,
                int h_q, int h_kv, int lead, const int32_t* __restrict__ ptr, const int32_t* __restrict__ rows,
                float* __restrict__ dqacc, bf16* __restrict__ dk, bf16* __restrict__ dv) {
  using C = BwdCfg<D, BLK>;
  constexpr int TR = C::TR, KG = C::KG, NW = C::NW, NT = C::NT;
  extern __shared__ __align__(128) unsigned char smem_raw[];
  BwdSmem<D, BLK>& sm = *reinterpret_cast<BwdSmem<D, BLK>*>(smem_raw);

  const BucketOrder bo = bucket_order(blockIdx.x, nb_max, h_kv, lead);
  const int gb = bo.gb, kvh = bo.kvh;
  if (gb >= __ldg(blk_off + batch)) return;
  const int bucket = kvh * nb_max + gb;
  const int beg = __ldg(ptr + bucket), end = __ldg(ptr + bucket + 1);
  const int s = upper_seq(blk_off, batch, gb);
  const int t0 = __ldg(cu + s) + (gb - __ldg(blk_off + s)) * BLK;
  const int t1 = min(t0 + BLK, __ldg(cu + s + 1));
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int kg = warp % KG, rg = warp / KG;
  const size_t kv_stride = (size_t)h_kv * D;
  const float scale = rsqrtf((float)D);
  const float scale_log2 = kLog2e * scale;

  for (int i = tid; i < BLK * (D / 8); i += NT) {
    const int r = i / (D / 8), c = i % (D / 8);
    const bool ok = t0 + r < t1;
    const size_t off = ok ? (size_t)(t0 + r) * kv_stride + (size_t)kvh * D + c * 8 : 0;
    cp_async16_zfill(&sm.k[r][c * 8], k + off, ok);
    cp_async16_zfill(&sm.v[r][c * 8], v + off, ok);
  }
  auto load_meta = [&](int tile, int buf) {
    for (int i = tid; i < TR; i += NT) {
      const int e = beg + tile * TR + i;
      int r = -1, tk = -1;
      float l2 = 0.f, ds = 0.f;
      if (e < end) {
        r = __ldg(rows + e);
        tk = r / h_q;
        l2 = __ldg(lse + r) * kLog2e;
        ds = __ldg(dsum + r);
      }
      sm.row[buf][i] = r;
      sm.tok[buf][i] = tk;
      sm.lse2[buf][i] = l2;
      sm.dsum[buf][i] = ds;
    }
  };
  auto issue_rows = [&](int buf) {
    for (int i = tid; i < TR * (D / 8); i += NT) {
      const int r = i / (D / 8), c = i % (D / 8);
      const int row = sm.row[buf][r];
      const bool ok = row >= 0;
      const size_t off = ok ? (size_t)row * D + c * 8 : 0;   // [T, H_q, D]: row t*H_q + h
      cp_async16_zfill(&sm.q[buf][r][c * 8], q + off, ok);
      cp_async16_zfill(&sm.dout[buf][r][c * 8], dout + off, ok);
    }
  };

  float dva[D / 8][4], dka[D / 8][4];
#pragma unroll
  for (int nt = 0; nt < D / 8; ++nt)
#pragma unroll
    for (int i = 0; i < 4; ++i) dva[nt][i] = dka[nt][i] = 0.f;

  const int ntiles = (end - beg + TR - 1) / TR;
  if (ntiles > 0) load_meta(0, 0);
  __syncthreads();
  if (ntiles > 0) issue_rows(0);
  cp_async_commit();

  const int key_lo = kg * 16 + (lane >> 2);  // this thread's keys: key_lo, key_lo + 8
  for (int it = 0; it < ntiles; ++it) {
    const int buf = it & 1;
    if (it + 1 < ntiles) load_meta(it + 1, buf ^ 1);
    __syncthreads();
    if (it + 1 < ntiles) issue_rows(buf ^ 1);
    cp_async_commit();
    cp_async_wait<1>();
    __syncthreads();

    // S^T = K Q^T and dP^T = V dO^T for 16 keys x 32 rows.
    float st[4][4], dpt[4][4];
#pragma unroll
    for (int nt = 0; nt < 4; ++nt)
#pragma unroll
      for (int i = 0; i < 4; ++i) st[nt][i] = dpt[nt][i] = 0.f;
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      uint32_t ka[4], va[4];
      ldsm_x4(ka[0], ka[1], ka[2], ka[3], &sm.k[kg * 16 + (lane & 15)][kk * 16 + (lane >> 4) * 8]);
      ldsm_x4(va[0], va[1], va[2], va[3], &sm.v[kg * 16 + (lane & 15)][kk * 16 + (lane >> 4) * 8]);
#pragma unroll
      for (int nt2 = 0; nt2 < 2; ++nt2) {
        const int r = rg * 32 + nt2 * 16 + (lane & 7) + ((lane >> 4) << 3);
        const int col = kk * 16 + ((lane >> 3) & 1) * 8;
        uint32_t b0, b1, b2, b3;
        ldsm_x4(b0, b1, b2, b3, &sm.q[buf][r][col]);
        mma_bf16(st[2 * nt2], ka, b0, b1);
        mma_bf16(st[2 * nt2 + 1], ka, b2, b3);
        ldsm_x4(b0, b1, b2, b3, &sm.dout[buf][r][col]);
        mma_bf16(dpt[2 * nt2], va, b0, b1);
        mma_bf16(dpt[2 * nt2 + 1], va, b2, b3);
      }
    }
    // P^T and dS^T in place.
#pragma unroll
    for (int nt = 0; nt < 4; ++nt) {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int r = rg * 32 + nt * 8 + (lane & 3) * 2 + (i & 1);
        const int key_tok = t0 + key_lo + (i >= 2 ? 8 : 0);
        const int qt = sm.tok[buf][r];
        float p = 0.f;
        if (key_tok <= qt && key_tok < t1) p = fast_exp2(st[nt][i] * scale_log2 - sm.lse2[buf][r]);
        st[nt][i] = p;
        dpt[nt][i] = p * (dpt[nt][i] - sm.dsum[buf][r]);
      }
    }
    // dS^T -> shared memory (bf16) for the dQ product.
#pragma unroll
    for (int nt = 0; nt < 4; ++nt) {
      const int r = rg * 32 + nt * 8 + (lane & 3) * 2;
      *reinterpret_cast<uint32_t*>(&sm.dst[key_lo][r]) = pack_bf16(dpt[nt][0], dpt[nt][1]);
      *reinterpret_cast<uint32_t*>(&sm.dst[key_lo + 8][r]) = pack_bf16(dpt[nt][2], dpt[nt][3]);
    }
    // dV += P^T dO, dK += dS^T Q (rows are the reduction dimension).
#pragma unroll
    for (int ks = 0; ks < 2; ++ks) {
      uint32_t pa[4], da[4];
      pa[0] = pack_bf16(st[2 * ks][0], st[2 * ks][1]);
      pa[1] = pack_bf16(st[2 * ks][2], st[2 * ks][3]);
      pa[2] = pack_bf16(st[2 * ks + 1][0], st[2 * ks + 1][1]);
      pa[3] = pack_bf16(st[2 * ks + 1][2], st[2 * ks + 1][3]);
      da[0] = pack_bf16(dpt[2 * ks][0], dpt[2 * ks][1]);
      da[1] = pack_bf16(dpt[2 * ks][2], dpt[2 * ks][3]);
      da[2] = pack_bf16(dpt[2 * ks + 1][0], dpt[2 * ks + 1][1]);
      da[3] = pack_bf16(dpt[2 * ks + 1][2], dpt[2 * ks + 1][3]);
      const int r = rg * 32 + ks * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
#pragma unroll
      for (int nt2 = 0; nt2 < D / 16; ++nt2) {
        const int col = nt2 * 16 + (lane >> 4) * 8;
        uint32_t b0, b1, b2, b3;
        ldsm_x4_t(b0, b1, b2, b3, &sm.dout[buf][r][col]);
        mma_bf16(dva[2 * nt2], pa, b0, b1);
        mma_bf16(dva[2 * nt2 + 1], pa, b2, b3);
        ldsm_x4_t(b0, b1, b2, b3, &sm.q[buf][r][col]);
        mma_bf16(dka[2 * nt2], da, b0, b1);
        mma_bf16(dka[2 * nt2 + 1], da, b2, b3);
      }
    }
    __syncthreads();
    // dQ = dS K / sqrt(d): 16-row x 32-column output tiles shared by all warps.
    constexpr int MT = TR / 16, CT = D / 32;
    for (int u = warp; u < MT * CT; u += NW) {
      const int m0 = (u % MT) * 16, c0 = (u / MT) * 32;
      float acc[4][4];
#pragma unroll
      for (int nt = 0; nt < 4; ++nt)
#pragma unroll
        for (int i = 0; i < 4; ++i) acc[nt][i] = 0.f;
#pragma unroll
      for (int ks = 0; ks < BLK / 16; ++ks) {
        uint32_t a[4];
        ldsm_x4_t(a[0], a[1], a[2], a[3], &sm.dst[ks * 16 + (lane & 7) + (lane >> 4) * 8][m0 + ((lane >> 3) & 1) * 8]);
#pragma unroll
        for (int nt2 = 0; nt2 < 2; ++nt2) {
          uint32_t b0, b1, b2, b3;
          ldsm_x4_t(b0, b1, b2, b3,
                    &sm.k[ks * 16 + (lane & 7) + ((lane >> 3) & 1) * 8][c0 + nt2 * 16 + (lane >> 4) * 8]);
          mma_bf16(acc[2 * nt2], a, b0, b1);
          mma_bf16(acc[2 * nt2 + 1], a, b2, b3);
        }
      }
      // Lane pairs swap halves so that each lane owns 4 consecutive columns
      // of one row: one 16-byte reduction instead of two 8-byte ones.
      const int q4 = lane & 3;
      const bool even = (q4 & 1) == 0;
      const int rr = m0 + (lane >> 2) + (even ? 0 : 8);
      const int row = sm.row[buf][rr];
#pragma unroll
      for (int nt = 0; nt < 4; ++nt) {
        const float s0 = even ? acc[nt][2] : acc[nt][0];
        const float s1 = even ? acc[nt][3] : acc[nt][1];
        const float g0 = __shfl_xor_sync(0xffffffffu, s0, 1);
        const float g1 = __shfl_xor_sync(0xffffffffu, s1, 1);
        const int col = c0 + nt * 8 + (even ? q4 : q4 - 1) * 2;
        if (row >= 0) {
          if (even)
            red_add_v4(dqacc + (size_t)row * D + col, acc[nt][0] * scale, acc[nt][1] * scale, g0 * scale, g1 * scale);
          else
            red_add_v4(dqacc + (size_t)row * D + col, g0 * scale, g1 * scale, acc[nt][2] * scale, acc[nt][3] * scale);
        }
      }
    }
    __syncthreads();
  }
  cp_async_wait<0>();

  // Sum the row groups' partial dK/dV, then write bf16 once.
  if constexpr (C::RW == 2) {
    float* red = reinterpret_cast<float*>(&sm.q[0][0][0]);  // [2][BLK][D] fp32
    static_assert(sizeof(sm.q) + sizeof(sm.dout) >= 2 * sizeof(float) * BLK * D, "reduction buffer");
    __syncthreads();
    if (rg == 1) {
#pragma unroll
      for (int nt = 0; nt < D / 8; ++nt) {
        const int col = nt * 8 + (lane & 3) * 2;
        *reinterpret_cast<float2*>(&red[key_lo * D + col]) = make_float2(dva[nt][0], dva[nt][1]);
        *reinterpret_cast<float2*>(&red[(key_lo + 8) * D + col]) = make_float2(dva[nt][2], dva[nt][3]);
        *reinterpret_cast<float2*>(&red[(BLK + key_lo) * D + col]) = make_float2(dka[nt][0], dka[nt][1]);
        *reinterpret_cast<float2*>(&red[(BLK + key_lo + 8) * D + col]) = make_float2(dka[nt][2], dka[nt][3]);
      }
    }
    __syncthreads();
    if (rg == 1) return;
#pragma unroll
    for (int nt = 0; nt < D / 8; ++nt) {
      const int col = nt * 8 + (lane & 3) * 2;
      float2 a = *reinterpret_cast<float2*>(&red[key_lo * D + col]);
      float2 b = *reinterpret_cast<float2*>(&red[(key_lo + 8) * D + col]);
      float2 c = *reinterpret_cast<float2*>(&red[(BLK + key_lo) * D + col]);
      float2 d = *reinterpret_cast<float2*>(&red[(BLK + key_lo + 8) * D + col]);
      dva[nt][0] += a.x; dva[nt][1] += a.y; dva[nt][2] += b.x; dva[nt][3] += b.y;
      dka[nt][0] += c.x; dka[nt][1] += c.y; dka[nt][2] += d.x; dka[nt][3] += d.y;
    }
  }
  const int ta = t0 + key_lo, tb = ta + 8;
#pragma unroll
  for (int nt = 0; nt < D / 8; ++nt) {
    const int col = nt * 8 + (lane & 3) * 2;
    if (ta < t1) {
      const size_t o = (size_t)ta * kv_stride + (size_t)kvh * D + col;
      *reinterpret_cast<uint32_t*>(dv + o) = pack_bf16(dva[nt][0], dva[nt][1]);
      *reinterpret_cast<uint32_t*>(dk + o) = pack_bf16(dka[nt][0] * scale, dka[nt][1] * scale);
    }
    if (tb < t1) {
      const size_t o = (size_t)tb * kv_stride + (size_t)kvh * D + col;
      *reinterpret_cast<uint32_t*>(dv + o) = pack_bf16(dva[nt][2], dva[nt][3]);
      *reinterpret_cast<uint32_t*>(dk + o) = pack_bf16(dka[nt][2] * scale, dka[nt][3] * scale);
    }
  }
}

// D_i = sum_c dO_ic O_ic (fp32) and dQ accumulator zeroing; D/8 lanes per row.
template <int D>
__global__ void __launch_bounds__(256)
bwd_pre_kernel(const bf16* __restrict__ out, const bf16* __restrict__ dout, const float* __restrict__ lse,
               long long nrows, float* __restrict__ dsum, float2* __restrict__ stat, float* __restrict__ dqacc) {
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
      if (i % LPR == 0) {
        dsum[i / LPR] = acc;
        stat[i / LPR] = make_float2(__ldg(lse + i / LPR), acc);  // one 8-byte load per row downstream
      }
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

template <int D, int BLK>
cudaError_t launch_bwd_t(const bf16* q, const bf16* k, const bf16* v, const bf16* dout, const float* lse,
                         const float* dsum, const SeqPlan& p, const int32_t* ptr, const int32_t* rows, int h_q,
                         int h_kv, float* dqacc, bf16* dk, bf16* dv, cudaStream_t st) {
  const size_t smem = sizeof(BwdSmem<D, BLK>);
  auto kern = bwd_attn_kernel<D, BLK>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  if (p.nb_max == 0) return cudaSuccess;
  dim3 grid(p.nb_max * h_kv);
  const int lead = bucket_lead((long long)p.total_tokens * (h_q / h_kv), D * 4);
  kern<<<grid, BwdCfg<D, BLK>::NT, smem, st>>>(q, k, v, dout, lse, dsum, p.cu, p.blk_off, p.batch, p.nb_max, h_q,
                                               h_kv, lead, ptr, rows, dqacc, dk, dv);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_bwd_pre(const bf16* out, const bf16* dout, const float* lse, int nrows, int d, float* dsum,
                           float2* stat, float* dqacc, cudaStream_t st) {
  const long long n = (long long)nrows * (d / 8);
  if (n == 0) return cudaSuccess;
  const int grid = (int)std::min<long long>((n + 255) / 256, 148LL * 32);
  if (d == 64)
    bwd_pre_kernel<64><<<grid, 256, 0, st>>>(out, dout, lse, nrows, dsum, stat, dqacc);
  else
    bwd_pre_kernel<128><<<grid, 256, 0, st>>>(out, dout, lse, nrows, dsum, stat, dqacc);
  return cudaGetLastError();
}

cudaError_t launch_bwd_attn(const bf16* q, const bf16* k, const bf16* v, const bf16* dout, const float* lse,
                            const float* dsum, const SeqPlan& p, const int32_t* ptr, const int32_t* rows, int h_q,
                            int h_kv, int d, int block_size, float* dqacc, bf16* dk, bf16* dv, cudaStream_t st) {
#define MOBA_BWD(DD, BB) \
  return launch_bwd_t<DD, BB>(q, k, v, dout, lse, dsum, p, ptr, rows, h_q, h_kv, dqacc, dk, dv, st)
  if (d == 64) {
    switch (block_size) {
      case 16: MOBA_BWD(64, 16);
      case 32: MOBA_BWD(64, 32);
      case 64: MOBA_BWD(64, 64);
      case 128: MOBA_BWD(64, 128);
    }
  } else {
    switch (block_size) {
      case 16: MOBA_BWD(128, 16);
      case 32: MOBA_BWD(128, 32);
      case 64: MOBA_BWD(128, 64);
      case 128: MOBA_BWD(128, 128);
    }
  }
#undef MOBA_BWD
  return cudaErrorInvalidValue;
}

cudaError_t launch_bwd_dq(const float* dqacc, int n, bf16* dq, cudaStream_t st) {
  const long long n8 = n / 8;
  if (n8 == 0) return cudaSuccess;
  const int grid = (int)std::min<long long>((n8 + 255) / 256, 148LL * 32);
  bwd_dq_kernel<<<grid, 256, 0, st>>>(dqacc, n8, dq);
  return cudaGetLastError();
}

}  // namespace moba
