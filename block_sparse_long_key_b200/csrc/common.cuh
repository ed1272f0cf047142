// Device helpers shared by the MoBA kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace moba {

// Device status bits, OR-ed into the status word at the head of the
// workspace and reported by moba_check_status().
enum : int32_t {
  kStatusBadSeqlens = 1 << 0,   // cu_seqlens not monotone / not ending at T
  kStatusBadSelIdx = 1 << 1,    // sel_idx entry outside [-1, own block]
  kStatusIndexOverflow = 1 << 2, // CSR fill ran past its bucket
  kStatusTimeout = 1 << 3        // a bounded wait on the tensor cores gave up
};

__device__ __forceinline__ void set_status(int32_t* status, int32_t bit) {
  atomicOr(reinterpret_cast<int*>(status), bit);
}

// Kernel-path bits, OR-ed into the word after the status word (status[1])
// and reported by moba_check_path(): which kernel families ran.
enum : int32_t {
  kPathRouteTc = 1 << 0,    // route_kernel (tcgen05 scores)
  kPathFwdTc = 1 << 1,      // fwd_tc_kernel (tcgen05 forward attention)
  kPathBwdTc = 1 << 2,      // bwd_tc_kernel (tcgen05 backward attention)
  kPathExactRows = 1 << 3   // fwd_fallback_kernel recomputed at least one row
};

// Marks that the calling kernel ran: one atomic from the grid's first thread.
__device__ __forceinline__ void mark_path(int32_t* status, int32_t bit) {
  if (blockIdx.x == 0 && threadIdx.x == 0) atomicOr(reinterpret_cast<int*>(status + 1), bit);
}

// Largest s with off[s] <= x, for off[0..n] non-decreasing, off[0] <= x.
__device__ __forceinline__ int upper_seq(const int32_t* off, int n, int x) {
  int lo = 0, hi = n;  // answer in [0, n)
  while (hi - lo > 1) {
    int mid = (lo + hi) >> 1;
    if (__ldg(off + mid) <= x) lo = mid; else hi = mid;
  }
  return lo;
}

// Dispatch order of the attention kernels' CTAs, one per (key block, KV
// head), over a one-dimensional grid of nb_max * h_kv.  A block is a
// candidate for every later query, so a head's buckets shrink with the block
// index and its first blocks are its longest CTAs.  CTAs go head by head,
// which keeps the accumulator rows of the heads in flight resident in L2,
// except that the first nb_max / 8 blocks of head h are issued beside the
// short CTAs of head h - lead: long CTAs start `lead` head-windows early
// instead of trailing the grid on the last head.  lead = 0 is plain head-major
// order (for heads whose accumulator alone fills L2; see bucket_lead()).
struct BucketOrder {
  int gb, kvh;
};
__host__ __device__ __forceinline__ BucketOrder bucket_order(int L, int nb_max, int h_kv, int lead) {
  lead = lead < h_kv ? lead : h_kv;
  const int big = nb_max / 8 > 1 ? nb_max / 8 : 1;
  const int small = nb_max - big;
  BucketOrder o;
  if (L < lead * big) {  // the first heads' long CTAs
    o.kvh = L / big;
    o.gb = L % big;
    return o;
  }
  L -= lead * big;
  const int mid = (h_kv - lead) * nb_max;
  if (L < mid) {  // window s: long CTAs of head s + lead, then short ones of head s
    const int s = L / nb_max, r = L % nb_max;
    o.kvh = r < big ? s + lead : s;
    o.gb = r;
    return o;
  }
  L -= mid;  // the last heads' short CTAs (small > 0 whenever this is reached)
  o.kvh = h_kv - lead + L / small;
  o.gb = big + L % small;
  return o;
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// Zero-fill variant: copies src_bytes (0 or 16) and zero-fills the rest.
__device__ __forceinline__ void cp_async16_zfill(void* smem, const void* gmem, bool valid) {
  int n = valid ? 16 : 0;
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(smem_u32(smem)), "l"(gmem), "r"(n));
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;\n" ::"n"(N)); }

__device__ __forceinline__ void ldsm_x4(uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3, const void* p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(smem_u32(p)));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3, const void* p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(smem_u32(p)));
}

// D += A(16x16 bf16, row) * B(16x8 bf16, col), fp32 accumulate.
__device__ __forceinline__ void mma_bf16(float* c, const uint32_t* a, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

__device__ __forceinline__ void red_add_v4(float* gaddr, float a, float b, float c, float d) {
  asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};\n" ::"l"(gaddr), "f"(a), "f"(b), "f"(c), "f"(d)
               : "memory");
}



__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;\n" : "=f"(y) : "f"(x));
  return y;
}

// Unpack 8 bf16 held in a uint4 into fp32.
__device__ __forceinline__ void bf16x8_to_f32(const uint4& u, float* f) {
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float2 t = __bfloat1622float2(h[i]);
    f[2 * i] = t.x;
    f[2 * i + 1] = t.y;
  }
}

__device__ __forceinline__ uint4 f32_to_bf16x8(const float* f) {
  uint4 u;
  u.x = pack_bf16(f[0], f[1]);
  u.y = pack_bf16(f[2], f[3]);
  u.z = pack_bf16(f[4], f[5]);
  u.w = pack_bf16(f[6], f[7]);
  return u;
}

constexpr float kLog2e = 1.4426950408889634f;

}  // namespace moba
