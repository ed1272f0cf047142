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
// Main path (a KV head's blocks fit a shared-memory histogram): the picks of
// one KV head are cut into chunks of kChunkTokens tokens; one CTA per
// (chunk, KV head) counts its picks per block with shared-memory atomics and
// writes that histogram row; a per-bucket pass turns the rows into each
// chunk's starting offset inside the bucket; a one-CTA scan gives the bucket
// starts; the fill pass re-reads the picks and places them with
// shared-memory cursors.  Global traffic: the picks twice, the rows once, the
// histogram rows a few times.  Fallback (huge block counts, or no chunk
// buffer): one global atomic per pick to count and one to claim a slot.  The
// order of rows inside a bucket is not deterministic; no result depends on
// it beyond fp32 summation order.
#include <algorithm>

#include "common.cuh"
#include "launch.h"

namespace moba {
namespace {

constexpr int kThreads = 256;
constexpr int kScanThreads = 1024;
constexpr int kChunkTokens = 1024;
constexpr int kMaxSmemBuckets = 16384;  // 64 KB of shared-memory counters

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

// Exclusive scan of cnt[0..n) into ptr[0..n]; cursor = ptr[0..n).  One CTA:
// each warp owns a contiguous segment, read 32 entries at a time (coalesced);
// pass 1 sums the segments, a scan over the warp sums gives each segment's
// start, pass 2 re-reads the segment and writes the running prefix.
__global__ void __launch_bounds__(kScanThreads)
scan_kernel(const int32_t* __restrict__ cnt, int n, int32_t* __restrict__ ptr, int32_t* __restrict__ cursor) {
  constexpr int kWarps = kScanThreads / 32;
  __shared__ int32_t s_warp[kWarps];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int seg = (n + kWarps - 1) / kWarps;
  const int lo = min(warp * seg, n), hi = min(lo + seg, n);
  int sum = 0;
  for (int i = lo + lane; i < hi; i += 32) sum += __ldg(cnt + i);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
  if (lane == 0) s_warp[warp] = sum;
  __syncthreads();
  if (warp == 0) {
    const int v = s_warp[lane];  // kWarps == 32
    int incl = v;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int o = __shfl_up_sync(0xffffffffu, incl, off);
      if (lane >= off) incl += o;
    }
    s_warp[lane] = incl - v;
    if (lane == 31) ptr[n] = incl;
  }
  __syncthreads();
  int run = s_warp[warp];
  for (int i0 = lo; i0 < hi; i0 += 32) {
    const int i = i0 + lane;
    const int v = i < hi ? __ldg(cnt + i) : 0;
    int incl = v;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int o = __shfl_up_sync(0xffffffffu, incl, off);
      if (lane >= off) incl += o;
    }
    if (i < hi) {
      ptr[i] = run + incl - v;
      cursor[i] = run + incl - v;
    }
    run += __shfl_sync(0xffffffffu, incl, 31);
  }
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

// ---- shared-memory privatised path
//
// A CTA owns the picks of one (chunk of kChunkTokens tokens, KV head).  The
// count and the staged fill take a run of kRun consecutive slots of one
// query row per thread (coalesced loads, several picks in flight per
// thread); the unstaged fill takes one query row per thread and walks its
// topk picks.  The per-pick work is a load, a range check and one
// shared-memory atomic.

// For query row `r` of the chunk (ta: first token): its row id, its
// sequence's first global block and its own block; false past the chunk or
// outside every sequence.
__device__ __forceinline__ bool chunk_row(int r, int ntok, int ta, int kvh, int group, int h_q, int block_size,
                                          const int32_t* cu, const int32_t* blk_off, int batch, int seq_end,
                                          int& row, int& base, int& own) {
  if (r >= ntok * group) return false;
  const int t = ta + r / group;
  if (t >= seq_end) return false;
  row = t * h_q + kvh * group + r % group;
  const int s = upper_seq(cu, batch, t);
  base = __ldg(blk_off + s);
  own = (t - __ldg(cu + s)) / block_size;
  return true;
}

// Calls f(m, j) for the valid picks of a row (j in [0, own]); invalid
// entries are skipped (and raise kStatusBadSelIdx when `kReport`).
template <bool kReport, typename F>
__device__ __forceinline__ void for_row_picks(const int32_t* __restrict__ sel_idx, int row, int topk, int own,
                                              int32_t* status, F&& f) {
  const int32_t* p = sel_idx + (size_t)row * topk;
  auto one = [&](int m, int j) {
    if (j < 0) {
      if (kReport && j != -1) set_status(status, kStatusBadSelIdx);
    } else if (j > own) {
      if (kReport) set_status(status, kStatusBadSelIdx);
    } else {
      f(m, j);
    }
  };
  int m = 0;
  if ((topk & 3) == 0) {  // rows start 16-byte aligned
    for (; m < topk; m += 4) {
      const int4 v = __ldg(reinterpret_cast<const int4*>(p + m));
      one(m, v.x);
      one(m + 1, v.y);
      one(m + 2, v.z);
      one(m + 3, v.w);
    }
  }
  for (; m < topk; ++m) one(m, __ldg(p + m));
}

// Threads of the per-chunk count and staged fill.  A thread takes a run of
// kRun consecutive slots of one query row (two 16-byte loads when topk is a
// multiple of 4), so the row's sequence is located once per run and a warp's
// loads of sel_idx are contiguous; a CTA covers kPickThreads runs per step.
constexpr int kPickThreads = 1024;
constexpr int kRun = 8;

// Run q of a chunk (rpr = ceil(topk / kRun) runs per query row): slots
// [m0, m0 + kRun) of chunk row r = q / rpr.  Sets `row` and bk[i] to the
// block offset of slot m0 + i in the KV head's histogram (sequence base +
// block), or -1 for a slot past topk, an empty or invalid slot (invalid ones
// raise kStatusBadSelIdx when `kReport`) or a row outside every sequence.
template <bool kReport>
__device__ __forceinline__ void chunk_run(const int32_t* __restrict__ sel_idx, int q, int rpr, int topk, int ntok,
                                          int ta, int kvh, int group, int h_q, int block_size, const int32_t* cu,
                                          const int32_t* blk_off, int batch, int seq_end, int32_t* status, int& row,
                                          int (&bk)[kRun]) {
  const int r = q / rpr, m0 = (q - r * rpr) * kRun;
  int bb, own;
#pragma unroll
  for (int i = 0; i < kRun; ++i) bk[i] = -1;
  if (!chunk_row(r, ntok, ta, kvh, group, h_q, block_size, cu, blk_off, batch, seq_end, row, bb, own)) return;
  const int32_t* src = sel_idx + (size_t)row * topk + m0;
  int j[kRun];
  if ((topk & 3) == 0) {  // 16-byte aligned: m0 is a multiple of 8, row * topk of 4
#pragma unroll
    for (int i = 0; i < kRun; i += 4) {
      if (m0 + i < topk) {
        const int4 v = __ldg(reinterpret_cast<const int4*>(src + i));
        j[i] = v.x;
        j[i + 1] = v.y;
        j[i + 2] = v.z;
        j[i + 3] = v.w;
      } else {
        j[i] = j[i + 1] = j[i + 2] = j[i + 3] = -1;
      }
    }
  } else {
#pragma unroll
    for (int i = 0; i < kRun; ++i) j[i] = m0 + i < topk ? __ldg(src + i) : -1;
  }
#pragma unroll
  for (int i = 0; i < kRun; ++i) {
    if (j[i] < 0) {
      if (kReport && j[i] != -1) set_status(status, kStatusBadSelIdx);
    } else if (j[i] > own) {
      if (kReport) set_status(status, kStatusBadSelIdx);
    } else {
      bk[i] = bb + j[i];
    }
  }
}

__global__ void __launch_bounds__(kPickThreads)
chunk_count_kernel(const int32_t* __restrict__ sel_idx, int total_tokens, int topk, int h_q, int group,
                   int block_size, const int32_t* __restrict__ cu, const int32_t* __restrict__ blk_off, int batch,
                   int nb_max, int nchunks, int32_t* __restrict__ chunk_cnt, int32_t* __restrict__ status) {
  extern __shared__ int32_t hist[];
  const int c = blockIdx.x, kvh = blockIdx.y, tid = threadIdx.x;
  for (int b = tid; b < nb_max; b += kPickThreads) hist[b] = 0;
  __syncthreads();
  const int ta = c * kChunkTokens;
  const int ntok = max(0, min(kChunkTokens, total_tokens - ta));
  const int seq_end = __ldg(cu + batch);
  const int rpr = (topk + kRun - 1) / kRun;
  const int nruns = ntok * group * rpr;
  for (int q = tid; q < nruns; q += kPickThreads) {
    int row, bk[kRun];
    chunk_run<true>(sel_idx, q, rpr, topk, ntok, ta, kvh, group, h_q, block_size, cu, blk_off, batch, seq_end, status,
                    row, bk);
#pragma unroll
    for (int i = 0; i < kRun; ++i)
      if (bk[i] >= 0) atomicAdd(hist + bk[i], 1);
  }
  __syncthreads();
  int32_t* dst = chunk_cnt + ((size_t)kvh * nchunks + c) * nb_max;
  for (int b = tid; b < nb_max; b += kPickThreads) dst[b] = hist[b];
}

// Per bucket: chunk counts -> exclusive prefix over chunks (in place), total
// into cnt.  A thread reads eight chunks' counts before writing them back, so
// its loads overlap.
__global__ void __launch_bounds__(kThreads)
chunk_prefix_kernel(int32_t* __restrict__ chunk_cnt, int nb_max, int nchunks, int h_kv, int32_t* __restrict__ cnt) {
  constexpr int U = 8;
  const int b = blockIdx.x * kThreads + threadIdx.x;
  if (b >= h_kv * nb_max) return;
  const int kvh = b / nb_max, lb = b % nb_max;
  int32_t* col = chunk_cnt + (size_t)kvh * nchunks * nb_max + lb;
  int run = 0;
  for (int c0 = 0; c0 < nchunks; c0 += U) {
    int v[U];
#pragma unroll
    for (int u = 0; u < U; ++u) v[u] = c0 + u < nchunks ? col[(size_t)(c0 + u) * nb_max] : 0;
#pragma unroll
    for (int u = 0; u < U; ++u) {
      if (c0 + u < nchunks) col[(size_t)(c0 + u) * nb_max] = run;
      run += v[u];
    }
  }
  cnt[b] = run;
}

__global__ void __launch_bounds__(kThreads)
chunk_fill_kernel(const int32_t* __restrict__ sel_idx, int total_tokens, int topk, int h_q, int group,
                  int block_size, const int32_t* __restrict__ cu, const int32_t* __restrict__ blk_off, int batch,
                  int nb_max, int nchunks, const int32_t* __restrict__ chunk_cnt, const int32_t* __restrict__ ptr,
                  int32_t* __restrict__ rows, int32_t* __restrict__ status) {
  extern __shared__ int32_t cursor[];
  const int c = blockIdx.x, kvh = blockIdx.y;
  const int32_t* src = chunk_cnt + ((size_t)kvh * nchunks + c) * nb_max;
  const int32_t* bptr = ptr + (size_t)kvh * nb_max;
  for (int b = threadIdx.x; b < nb_max; b += kThreads) cursor[b] = __ldg(bptr + b) + __ldg(src + b);
  __syncthreads();
  const int ta = c * kChunkTokens;
  const int ntok = max(0, min(kChunkTokens, total_tokens - ta));
  const int seq_end = __ldg(cu + batch);
  // (invalid entries were reported by the count pass)
  for (int r = threadIdx.x; r < ntok * group; r += kThreads) {
    int row, base, own;
    if (!chunk_row(r, ntok, ta, kvh, group, h_q, block_size, cu, blk_off, batch, seq_end, row, base, own)) continue;
    for_row_picks<false>(sel_idx, row, topk, own, status,
                         [&](int, int j) { rows[atomicAdd(cursor + base + j, 1)] = row; });
  }
}

// Staged fill (blocks per KV head <= kMaxStagedBuckets): the chunk's runs
// are taken in passes of kPickThreads, one per thread (at most kStage
// picks).  A pass counts its picks per block in shared memory, scans the counts
// into local bucket starts, places each row id at its local slot (with its
// bucket as a tag; the picks' buckets stay in registers between the two
// steps) and then copies the staged entries out in order: consecutive
// entries of one bucket go to consecutive addresses, so the stores coalesce
// into runs instead of one scattered 4-byte store per pick.  `base[b]` is
// where the chunk's next entry for block b goes in rows[].
constexpr int kStage = kPickThreads * kRun;
constexpr int kMaxStagedBuckets = 8192;

__host__ __device__ constexpr size_t staged_fill_smem(int nb_max) {
  return sizeof(int32_t) * (2 * (size_t)nb_max + 1 + kStage) + sizeof(uint16_t) * kStage;
}

// In-place exclusive scan of a[0..n) by the whole CTA (NT threads, NT <=
// 1024); returns the total.  `part` holds NT / 32 + 1 ints of shared scratch.
template <int NT>
__device__ int block_exclusive_scan(int32_t* a, int n, int32_t* part) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int per = (n + NT - 1) / NT;
  const int lo = min(tid * per, n), hi = min(lo + per, n);
  int sum = 0;
  for (int i = lo; i < hi; ++i) sum += a[i];
  int incl = sum;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int o = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += o;
  }
  if (lane == 31) part[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const int v = lane < NT / 32 ? part[lane] : 0;
    int w = v;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int o = __shfl_up_sync(0xffffffffu, w, off);
      if (lane >= off) w += o;
    }
    if (lane < NT / 32) part[lane] = w - v;
    if (lane == 31) part[NT / 32] = w;  // total
  }
  __syncthreads();
  int run = part[warp] + incl - sum;
  for (int i = lo; i < hi; ++i) {
    const int v = a[i];
    a[i] = run;
    run += v;
  }
  const int total = part[NT / 32];
  __syncthreads();
  return total;
}

__global__ void __launch_bounds__(kPickThreads, 2)
chunk_fill_staged_kernel(const int32_t* __restrict__ sel_idx, int total_tokens, int topk, int h_q, int group,
                         int block_size, const int32_t* __restrict__ cu, const int32_t* __restrict__ blk_off,
                         int batch, int nb_max, int nchunks, const int32_t* __restrict__ chunk_cnt,
                         const int32_t* __restrict__ ptr, int32_t* __restrict__ rows) {
  extern __shared__ __align__(16) int32_t sm_fill[];
  int32_t* base = sm_fill;                  // [nb_max]
  int32_t* lc = base + nb_max;              // [nb_max + 1]: counts -> local starts -> cursors
  int32_t* stage = lc + nb_max + 1;         // [kStage]
  uint16_t* tag = reinterpret_cast<uint16_t*>(stage + kStage);  // [kStage]
  __shared__ int32_t part[kPickThreads / 32 + 1];
  const int c = blockIdx.x, kvh = blockIdx.y;
  const int tid = threadIdx.x;
  const int32_t* src = chunk_cnt + ((size_t)kvh * nchunks + c) * nb_max;
  const int32_t* bptr = ptr + (size_t)kvh * nb_max;
  for (int b = tid; b < nb_max; b += kPickThreads) base[b] = __ldg(bptr + b) + __ldg(src + b);
  const int ta = c * kChunkTokens;
  const int ntok = max(0, min(kChunkTokens, total_tokens - ta));
  const int seq_end = __ldg(cu + batch);
  const int rpr = (topk + kRun - 1) / kRun;
  const int nruns = ntok * group * rpr;
  for (int q0 = 0; q0 < nruns; q0 += kPickThreads) {
    for (int b = tid; b <= nb_max; b += kPickThreads) lc[b] = 0;
    __syncthreads();
    // 1. this pass's runs: bucket offsets (invalid entries were reported by
    //    the count pass and are skipped here), counted per block
    int row = 0, bk[kRun];
    if (q0 + tid < nruns) {
      chunk_run<false>(sel_idx, q0 + tid, rpr, topk, ntok, ta, kvh, group, h_q, block_size, cu, blk_off, batch,
                       seq_end, nullptr, row, bk);
    } else {
#pragma unroll
      for (int i = 0; i < kRun; ++i) bk[i] = -1;
    }
#pragma unroll
    for (int i = 0; i < kRun; ++i)
      if (bk[i] >= 0) atomicAdd(lc + bk[i], 1);
    __syncthreads();
    // 2. local bucket starts
    const int total = block_exclusive_scan<kPickThreads>(lc, nb_max, part);
    // 3. stage each row id at its local slot
#pragma unroll
    for (int i = 0; i < kRun; ++i) {
      if (bk[i] < 0) continue;
      const int slot = atomicAdd(lc + bk[i], 1);
      stage[slot] = row;
      tag[slot] = (uint16_t)bk[i];
    }
    __syncthreads();
    // 4. copy out in order; lc[b] is now the end of bucket b's local run, so
    //    the run starts at lc[b - 1]
    for (int i = tid; i < total; i += kPickThreads) {
      const int b = tag[i];
      const int start = b > 0 ? lc[b - 1] : 0;
      rows[base[b] + (i - start)] = stage[i];
    }
    __syncthreads();
    for (int b = tid; b < nb_max; b += kPickThreads) base[b] += lc[b] - (b > 0 ? lc[b - 1] : 0);
    __syncthreads();
  }
}

}  // namespace

size_t index_chunk_ints(int total_tokens, int h_kv, int nb_max) {
  if (nb_max > kMaxSmemBuckets) return 0;
  const size_t nchunks = ((size_t)total_tokens + kChunkTokens - 1) / kChunkTokens;
  return (size_t)h_kv * nchunks * nb_max;
}

cudaError_t launch_build_index(const int32_t* sel_idx, const SeqPlan& p, int h_q, int h_kv, int block_size,
                               int topk, int32_t* cnt, int32_t* ptr, int32_t* cursor, int32_t* rows,
                               int32_t* status, cudaStream_t st, int32_t* chunk_cnt) {
  const int nbk = h_kv * p.nb_max;
  const long long npicks = (long long)p.total_tokens * h_q * topk;
  const int group = h_q / h_kv;
  cudaError_t e;
  if (chunk_cnt != nullptr && p.nb_max <= kMaxSmemBuckets && p.total_tokens > 0) {
    const int nchunks = (p.total_tokens + kChunkTokens - 1) / kChunkTokens;
    const size_t smem = sizeof(int32_t) * (size_t)p.nb_max;
    if ((e = cudaFuncSetAttribute(chunk_count_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)) !=
        cudaSuccess)
      return e;
    if ((e = cudaFuncSetAttribute(chunk_fill_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)) !=
        cudaSuccess)
      return e;
    dim3 grid(nchunks, h_kv);
    chunk_count_kernel<<<grid, kPickThreads, smem, st>>>(sel_idx, p.total_tokens, topk, h_q, group, block_size, p.cu,
                                                     p.blk_off, p.batch, p.nb_max, nchunks, chunk_cnt, status);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    chunk_prefix_kernel<<<(nbk + kThreads - 1) / kThreads, kThreads, 0, st>>>(chunk_cnt, p.nb_max, nchunks, h_kv,
                                                                              cnt);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    scan_kernel<<<1, kScanThreads, 0, st>>>(cnt, nbk, ptr, cursor);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    if (p.nb_max <= kMaxStagedBuckets && topk <= kStage) {
      const size_t smem2 = staged_fill_smem(p.nb_max);
      if ((e = cudaFuncSetAttribute(chunk_fill_staged_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    (int)smem2)) != cudaSuccess)
        return e;
      chunk_fill_staged_kernel<<<grid, kPickThreads, smem2, st>>>(sel_idx, p.total_tokens, topk, h_q, group, block_size,
                                                              p.cu, p.blk_off, p.batch, p.nb_max, nchunks, chunk_cnt,
                                                              ptr, rows);
      return cudaGetLastError();
    }
    chunk_fill_kernel<<<grid, kThreads, smem, st>>>(sel_idx, p.total_tokens, topk, h_q, group, block_size, p.cu,
                                                    p.blk_off, p.batch, p.nb_max, nchunks, chunk_cnt, ptr, rows,
                                                    status);
    return cudaGetLastError();
  }
  e = cudaMemsetAsync(cnt, 0, sizeof(int32_t) * (size_t)nbk, st);
  if (e != cudaSuccess) return e;
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
