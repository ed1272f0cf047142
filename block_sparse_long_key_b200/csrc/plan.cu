// Sequence plan: sanitised cu_seqlens and per-sequence block / routing-tile
// offsets, computed on the device so that no call needs a host copy of the
// sequence lengths.
//
// Blocks partition every sequence into ceil(L/B) runs of B consecutive
// tokens ("Optimizing Mixture of Block Attention", §"Definizione del
// Compito": N keys in n = N/B blocks); block numbering restarts at each
// sequence, and global block gb = blk_off[s] + j names block j of sequence s.
#include "common.cuh"
#include "launch.h"

namespace moba {
namespace {

constexpr int kPlanThreads = 1024;

__global__ void __launch_bounds__(kPlanThreads)
plan_kernel(const int32_t* __restrict__ cu_in, int batch, int total, int block_size,
            int32_t* __restrict__ cu_out, int32_t* __restrict__ blk_off,
            int32_t* __restrict__ tile_off, int32_t* __restrict__ status) {
  __shared__ int32_t s_blk[kPlanThreads];
  __shared__ int32_t s_tile[kPlanThreads];
  __shared__ int32_t s_carry[3];  // blocks, tiles, last clamped boundary
  const int tid = threadIdx.x;
  if (tid == 0) {
    s_carry[0] = 0;
    s_carry[1] = 0;
    s_carry[2] = 0;
    if (__ldg(cu_in) != 0 || __ldg(cu_in + batch) != total) set_status(status, kStatusBadSeqlens);
    cu_out[0] = 0;
  }
  __syncthreads();
  for (int base = 0; base < batch; base += kPlanThreads) {
    const int s = base + tid;
    int nblk = 0, ntile = 0;
    int lo = 0, hi = 0;
    if (s < batch) {
      lo = __ldg(cu_in + s);
      hi = __ldg(cu_in + s + 1);
      // Clamp to [0, total] and to monotone order; anything clamped is reported.
      int clo = min(max(lo, 0), total);
      int chi = min(max(hi, 0), total);
      if (clo != lo || chi != hi || chi < clo) set_status(status, kStatusBadSeqlens);
      lo = clo;
      hi = max(chi, clo);
    }
    // The clamped end of sequence s must also be >= the clamped end of s-1;
    // a running max over the chunk restores monotone boundaries.
    s_blk[tid] = hi;
    __syncthreads();
    for (int off = 1; off < kPlanThreads; off <<= 1) {
      int v = tid >= off ? s_blk[tid - off] : 0;
      __syncthreads();
      s_blk[tid] = max(s_blk[tid], v);
      __syncthreads();
    }
    const int prev_end = tid == 0 ? s_carry[2] : max(s_carry[2], s_blk[tid - 1]);
    const int end = max(s_blk[tid], s_carry[2]);
    __syncthreads();
    if (s < batch) {
      const int L = end - prev_end;
      nblk = (L + block_size - 1) / block_size;
      ntile = (L + kRouteTile - 1) / kRouteTile;
      cu_out[s + 1] = end;
    }
    s_blk[tid] = nblk;
    s_tile[tid] = ntile;
    __syncthreads();
    for (int off = 1; off < kPlanThreads; off <<= 1) {
      int a = tid >= off ? s_blk[tid - off] : 0;
      int b = tid >= off ? s_tile[tid - off] : 0;
      __syncthreads();
      s_blk[tid] += a;
      s_tile[tid] += b;
      __syncthreads();
    }
    if (s < batch) {
      blk_off[s] = s_carry[0] + s_blk[tid] - nblk;
      tile_off[s] = s_carry[1] + s_tile[tid] - ntile;
    }
    __syncthreads();
    if (tid == kPlanThreads - 1) {
      s_carry[0] += s_blk[tid];
      s_carry[1] += s_tile[tid];
      s_carry[2] = max(s_carry[2], end);
    }
    __syncthreads();
  }
  if (tid == 0) {
    blk_off[batch] = s_carry[0];
    tile_off[batch] = s_carry[1];
  }
}

}  // namespace

cudaError_t launch_plan(const int32_t* cu_in, int batch, int total_tokens, int block_size,
                        int32_t* cu_out, int32_t* blk_off, int32_t* tile_off, int32_t* status,
                        cudaStream_t st) {
  plan_kernel<<<1, kPlanThreads, 0, st>>>(cu_in, batch, total_tokens, block_size, cu_out, blk_off,
                                          tile_off, status);
  return cudaGetLastError();
}

}  // namespace moba
