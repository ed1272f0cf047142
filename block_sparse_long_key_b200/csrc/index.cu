// Index builder: inverts the query -> block picks into per-KV-block query
// lists (CSR).
//
// "Optimizing Mixture of Block Attention", §"Progettazione del Kernel
// FlashMoBA", "Tre Kernel Fusi" 1 (Flash TopK stage 3: an epilogue that
// rewrites the query-major picks into a key-block-major varlen layout) and 2
// (the forward uses those varlen indices to find, for each key block, the
// queries that chose it).
//
// Bucket of (KV head kvh, global block gb) = kvh * nb_max + gb.  Each entry
// is a query row id r = token * H_q + q_head, so one entry addresses the
// query, its output and its statistics directly.  Own-block picks are
// included; the attention kernels apply the causal cut for them.
//
// Three passes: count (one atomic per pick), exclusive scan of the counts
// (one CTA), fill (one atomic per pick to claim a slot).  The order of rows
// inside a bucket is therefore not deterministic; no result depends on it
// beyond fp32 summation order.  Integer work, bound by the atomics.
#include <algorithm>

#include "common.cuh"
#include "launch.h"

namespace moba {
namespace {

constexpr int kThreads = 256;
constexpr int kScanThreads = 1024;

// Returns the bucket of pick `e` (row * topk + slot) or -1 if the slot is
// empty or invalid (invalid entries raise kStatusBadSelIdx).
__device__ __forceinline__ int pick_bucket(const int32_t* __restrict__ sel_idx, long long e, int topk,
                                           int h_q, int group, int block_size, const int32_t* cu,
                                           const int32_t* blk_off, int batch, int nb_max,
                                           int32_t* status) {
  const int j = __ldg(sel_idx + e);
  if (j < 0) {
    if (j != -1) set_status(status, kStatusBadSelIdx);
    return -1;
  }
  const long long row = e / topk;
  const int t = (int)(row / h_q);
  const int h = (int)(row % h_q);
  if (t >= __ldg(cu + batch)) return -1;  // token outside every sequence
  const int s = upper_seq(cu, batch, t);
  const int pos = t - __ldg(cu + s);
  if (j > pos / block_size) {
    set_status(status, kStatusBadSelIdx);
    return -1;
  }
  return (h / group) * nb_max + __ldg(blk_off + s) + j;
}

__global__ void __launch_bounds__(kThreads)
count_kernel(const int32_t* __restrict__ sel_idx, long long npicks, int topk, int h_q, int group,
             int block_size, const int32_t* __restrict__ cu, const int32_t* __restrict__ blk_off,
             int batch, int nb_max, int32_t* __restrict__ cnt, int32_t* __restrict__ status) {
  for (long long e = blockIdx.x * (long long)kThreads + threadIdx.x; e < npicks;
       e += (long long)gridDim.x * kThreads) {
    const int b = pick_bucket(sel_idx, e, topk, h_q, group, block_size, cu, blk_off, batch, nb_max, status);
    if (b >= 0) atomicAdd(cnt + b, 1);
  }
}

// Exclusive scan of cnt[0..n) into ptr[0..n]; cursor = ptr[0..n).
__global__ void __launch_bounds__(kScanThreads)
scan_kernel(const int32_t* __restrict__ cnt, int n, int32_t* __restrict__ ptr, int32_t* __restrict__ cursor) {
  __shared__ int32_t s_sum[kScanThreads];
  const int tid = threadIdx.x;
  const int per = (n + kScanThreads - 1) / kScanThreads;
  const int lo = min(tid * per, n), hi = min(lo + per, n);
  int local = 0;
  for (int i = lo; i < hi; ++i) local += cnt[i];
  s_sum[tid] = local;
  __syncthreads();
  for (int off = 1; off < kScanThreads; off <<= 1) {
    const int v = tid >= off ? s_sum[tid - off] : 0;
    __syncthreads();
    s_sum[tid] += v;
    __syncthreads();
  }
  int run = s_sum[tid] - local;
  for (int i = lo; i < hi; ++i) {
    ptr[i] = run;
    cursor[i] = run;
    run += cnt[i];
  }
  if (tid == kScanThreads - 1) ptr[n] = s_sum[tid];
}

__global__ void __launch_bounds__(kThreads)
fill_kernel(const int32_t* __restrict__ sel_idx, long long npicks, int topk, int h_q, int group,
            int block_size, const int32_t* __restrict__ cu, const int32_t* __restrict__ blk_off,
            int batch, int nb_max, const int32_t* __restrict__ ptr, int32_t* __restrict__ cursor,
            int32_t* __restrict__ rows, int32_t* __restrict__ status) {
  for (long long e = blockIdx.x * (long long)kThreads + threadIdx.x; e < npicks;
       e += (long long)gridDim.x * kThreads) {
    const int b = pick_bucket(sel_idx, e, topk, h_q, group, block_size, cu, blk_off, batch, nb_max, status);
    if (b < 0) continue;
    const int slot = atomicAdd(cursor + b, 1);
    if (slot < __ldg(ptr + b + 1)) rows[slot] = (int32_t)(e / topk);
    else set_status(status, kStatusIndexOverflow);
  }
}

}  // namespace

cudaError_t launch_build_index(const int32_t* sel_idx, const SeqPlan& p, int h_q, int h_kv, int block_size,
                               int topk, int32_t* cnt, int32_t* ptr, int32_t* cursor, int32_t* rows,
                               int32_t* status, cudaStream_t st) {
  const int nbk = h_kv * p.nb_max;
  const long long npicks = (long long)p.total_tokens * h_q * topk;
  cudaError_t e = cudaMemsetAsync(cnt, 0, sizeof(int32_t) * (size_t)nbk, st);
  if (e != cudaSuccess) return e;
  const int group = h_q / h_kv;
  const int grid = (int)std::min<long long>((npicks + kThreads - 1) / kThreads, 148LL * 16);
  if (npicks > 0) {
    count_kernel<<<grid, kThreads, 0, st>>>(sel_idx, npicks, topk, h_q, group, block_size, p.cu, p.blk_off,
                                            p.batch, p.nb_max, cnt, status);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  scan_kernel<<<1, kScanThreads, 0, st>>>(cnt, nbk, ptr, cursor);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  if (npicks > 0) {
    fill_kernel<<<grid, kThreads, 0, st>>>(sel_idx, npicks, topk, h_q, group, block_size, p.cu, p.blk_off,
                                           p.batch, p.nb_max, ptr, cursor, rows, status);
    e = cudaGetLastError();
  }
  return e;
}

}  // namespace moba
