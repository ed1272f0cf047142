// sm_100a tensor-core plumbing: tcgen05 MMA issue, TMEM allocation and loads,
// shared-memory matrix descriptors, mbarriers with bounded waits.
//
// Operand tiles live in shared memory in the K-major 128-byte-swizzled layout:
// rows of 64 bf16 (128 bytes), 8 rows per 1024-byte atom, the 16-byte chunk c
// of row r stored at chunk position c ^ (r % 8).  A tile with K > 64 is stored
// as K/64 such regions one after the other.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"

namespace moba {
namespace tc {

// Byte offset of the 16-byte chunk `c` (8 bf16) of row `r` in a SW128 K-major
// region whose rows are 128 bytes (64 bf16) wide.
__device__ __forceinline__ uint32_t sw128_offset(int r, int c) {
  return (uint32_t)((r >> 3) * 1024 + (r & 7) * 128 + ((c ^ (r & 7)) << 4));
}

// Shared-memory matrix descriptor: K-major, 128-byte swizzle, 8-row groups
// 1024 bytes apart (stride byte offset), descriptor version 1.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t smem_addr) {
  uint64_t d = 0;
  d |= (uint64_t)((smem_addr >> 4) & 0x3FFFu);  // start address
  d |= (uint64_t)1u << 16;                      // leading byte offset (unused for swizzled K-major)
  d |= (uint64_t)(1024u >> 4) << 32;            // stride byte offset
  d |= (uint64_t)1u << 46;                      // version
  d |= (uint64_t)2u << 61;                      // SWIZZLE_128B
  return d;
}

// Byte offset of the 16-byte chunk `c` (8 bf16) of row `r` in a SW64 region
// whose rows are 64 bytes (32 bf16) wide: 8 rows per 512-byte atom, chunk c
// stored at c ^ ((r / 2) % 4).
__device__ __forceinline__ uint32_t sw64_offset(int r, int c) {
  return (uint32_t)((r >> 3) * 512 + (r & 7) * 64 + ((c ^ ((r >> 1) & 3)) << 4));
}

// Byte offset of the 16-byte chunk `c` of row `r` in a SW32 region whose
// rows are 32 bytes (16 bf16) wide: 8 rows per 256-byte atom, chunk c stored
// at c ^ ((r / 4) % 2).
__device__ __forceinline__ uint32_t sw32_offset(int r, int c) {
  return (uint32_t)((r >> 3) * 256 + (r & 7) * 32 + ((c ^ ((r >> 2) & 1)) << 4));
}

constexpr uint32_t kLayoutSW128 = 2;
constexpr uint32_t kLayoutSW64 = 4;
constexpr uint32_t kLayoutSW32 = 6;

// General shared-memory matrix descriptor.  K-major swizzled operands use
// `sbo` = byte distance between 8-row groups (the leading offset is unused);
// MN-major ones use `lbo` = byte distance between swizzle-wide groups along
// M/N and `sbo` = byte distance between 8-row groups along K.
__device__ __forceinline__ uint64_t smem_desc(uint32_t smem_addr, uint32_t lbo, uint32_t sbo, uint32_t layout) {
  uint64_t d = 0;
  d |= (uint64_t)((smem_addr >> 4) & 0x3FFFu);
  d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
  d |= (uint64_t)1u << 46;
  d |= (uint64_t)layout << 61;
  return d;
}

// A tile of 128 rows x BLK keys (bf16; the P and dS tiles of the attention
// kernels), keys contiguous in a row.  Rows up to 128 bytes wide use one
// region with the widest swizzle that fits (32, 64 or 128 bytes); BLK = 128
// uses two 128-byte-swizzled regions of 64 keys each, one after the other.
template <int BLK>
struct KeyTile {
  static_assert(BLK == 16 || BLK == 32 || BLK == 64 || BLK == 128, "block size");
  static constexpr uint32_t ROWB = BLK * 2 < 128 ? BLK * 2 : 128;  // bytes per row and region
  static constexpr int NREG = BLK * 2 / (int)ROWB;
  static constexpr uint32_t ATOM = 8 * ROWB;                       // one 8-row group
  static constexpr uint32_t REGION = 128 * ROWB;
  static constexpr uint32_t BYTES = NREG * REGION;
  static constexpr uint32_t LAYOUT = BLK == 16 ? kLayoutSW32 : (BLK == 32 ? kLayoutSW64 : kLayoutSW128);
  // Byte offset of the 16-byte chunk c (keys 8c .. 8c+7) of row r.
  static __device__ __forceinline__ uint32_t offset(int r, int c) {
    constexpr int CPR = (int)ROWB / 16;  // chunks per region row
    const uint32_t reg = (uint32_t)(c / CPR) * REGION;
    const int cc = c % CPR;
    if constexpr (BLK == 16) return reg + sw32_offset(r, cc);
    else if constexpr (BLK == 32) return reg + sw64_offset(r, cc);
    else return reg + sw128_offset(r, cc);
  }
};

// Zeroes rows [n, BLK) of a key block's K_j and V_j tiles (BLK rows, SW128
// K-major, 64-wide d chunks as regions of BLK * 128 bytes): a partial last
// block, where the TMA brought the next sequence's tokens or its zero fill,
// so no value outside the block reaches an MMA.  Generic-proxy stores: the
// caller fences them (fence_proxy_async) before the tensor cores read.
template <int D, int BLK>
__device__ __forceinline__ void zero_kv_tail_rows(unsigned char* k_tile, unsigned char* v_tile, int n, int tid,
                                                  int nthreads) {
  constexpr int KB = D / 64;
  constexpr uint32_t KV_REGION = BLK * 128;
  for (int i = tid; i < (BLK - n) * KB * 8; i += nthreads) {
    const int r = n + i / (KB * 8), c = i % (KB * 8);
    const uint32_t o = (c >> 3) * KV_REGION + sw128_offset(r, c & 7);
    *reinterpret_cast<uint4*>(k_tile + o) = make_uint4(0, 0, 0, 0);
    *reinterpret_cast<uint4*>(v_tile + o) = make_uint4(0, 0, 0, 0);
  }
}

// Instruction descriptor with the operand majorness: a_mn / b_mn = 1 when A
// (M x K) / B (N x K) is stored M- / N-contiguous instead of K-contiguous.
__host__ __device__ constexpr uint32_t idesc_bf16_f32_major(int M, int N, int a_mn, int b_mn) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)a_mn << 15) | ((uint32_t)b_mn << 16) |
         ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// Instruction descriptor: kind::f16 with bf16 A and B, fp32 accumulator,
// both operands K-major, shape M x N.
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int M, int N) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

__device__ __forceinline__ void mma_bf16_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                            uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate));
}

// Same with the A operand (M rows -> TMEM lanes, K bf16 packed two per
// 32-bit column) in tensor memory.
__device__ __forceinline__ void mma_bf16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                            uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate));
}

__device__ __forceinline__ void mma_commit(uint32_t mbar_addr) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(mbar_addr)
               : "memory");
}

__device__ __forceinline__ void fence_before_sync() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void fence_after_sync() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
// Generic-proxy shared-memory writes (st.shared, cp.async) -> async proxy (MMA reads).
__device__ __forceinline__ void fence_proxy_async() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// One full warp: allocate `ncols` TMEM columns (power of two >= 32); the base
// address is written to shared memory at `holder`.
__device__ __forceinline__ void tmem_alloc(uint32_t holder_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(holder_smem), "r"(ncols)
               : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

// 32 lanes x 32 consecutive columns (fp32): thread t of the warp receives
// row (warp's lane base + t), columns col .. col+31.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&v)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];\n"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
        "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15]),
        "=r"(v[16]), "=r"(v[17]), "=r"(v[18]), "=r"(v[19]), "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]),
        "=r"(v[24]), "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]), "=r"(v[31])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// 32 lanes x 16 consecutive columns (fp32).
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t* v) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];\n"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
        "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
      : "r"(taddr));
}

// 32 lanes x 32 consecutive columns: thread t writes its lane's columns.
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&v)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};\n" ::"r"(taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]),
      "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15]), "r"(v[16]),
      "r"(v[17]), "r"(v[18]), "r"(v[19]), "r"(v[20]), "r"(v[21]), "r"(v[22]), "r"(v[23]), "r"(v[24]),
      "r"(v[25]), "r"(v[26]), "r"(v[27]), "r"(v[28]), "r"(v[29]), "r"(v[30]), "r"(v[31])
      : "memory");
}
__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ void mbar_init(uint32_t addr, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(addr), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_init_fence() { asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory"); }

__device__ __forceinline__ uint64_t globaltimer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
  return t;
}

// Waits for phase `parity` of the mbarrier to complete.  Gives up after
// `limit_ns` of wall time and returns false (the caller records the failure
// and winds down instead of spinning forever).
__device__ __forceinline__ bool mbar_wait(uint32_t addr, uint32_t parity, uint64_t limit_ns = 2000000000ull) {
  uint32_t done = 0;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(done) : "r"(addr), "r"(parity) : "memory");
  if (done) return true;
  const uint64_t t0 = globaltimer();
  while (true) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}\n"
        : "=r"(done) : "r"(addr), "r"(parity) : "memory");
    if (done) return true;
    if (globaltimer() - t0 > limit_ns) return false;
  }
}

// One plain arrival (no transaction bytes).
__device__ __forceinline__ void mbar_arrive(uint32_t addr) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(addr) : "memory");
}

// Registers `bytes` of expected async transactions with one arrival.
__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t addr, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(addr), "r"(bytes) : "memory");
}

// TMA 2-D tile load: the box at (x, y) of `tmap` into shared memory at
// `dst` (128-byte aligned; a 1024-byte aligned tile gets the SW128 layout),
// completion counted in bytes on `mbar`.  No cluster multicast.
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const void* tmap, int x, int y, uint32_t mbar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(tmap)), "r"(x), "r"(y), "r"(mbar)
      : "memory");
}

// TMA 3-D tile load: the box at (x, y, z) of `tmap` into shared memory at
// `dst`, completion counted in bytes on `mbar`.  No cluster multicast.
__device__ __forceinline__ void tma_load_3d(uint32_t dst, const void* tmap, int x, int y, int z, uint32_t mbar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(tmap)), "r"(x), "r"(y), "r"(z), "r"(mbar)
      : "memory");
}

// TMA row gather: rows r0..r3 of a 2-D tensor map (box: 64 elements x one
// row, 128-byte swizzle), columns c0 .. c0+63, into 4 consecutive 128-byte
// rows of shared memory at `dst` (128-byte aligned; the swizzle follows the
// address bits, so a 1024-byte aligned tile gets the SW128 K-major layout).
// Completion is counted in bytes on `mbar`.  No cluster multicast.
__device__ __forceinline__ void tma_gather4(uint32_t dst, const void* tmap, int c0, int r0, int r1, int r2, int r3,
                                            uint32_t mbar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile::gather4.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4, %5, %6}], [%7];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(tmap)), "r"(c0), "r"(r0), "r"(r1), "r"(r2), "r"(r3), "r"(mbar)
      : "memory");
}

}  // namespace tc
}  // namespace moba
