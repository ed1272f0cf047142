// Internal launchers of the MoBA kernels.  Every launcher enqueues work on
// `st` and returns the launch status; none of them allocates or
// synchronises.  Pointers are device pointers; layouts are documented in
// include/moba.h and at each kernel.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace moba {

typedef __nv_bfloat16 bf16;

// Query rows per routing tile.
constexpr int kRouteTile = 128;

struct SeqPlan {
  const int32_t* cu;        // sanitised cu_seqlens [batch + 1]
  const int32_t* blk_off;   // first global block of each sequence [batch + 1]
  const int32_t* tile_off;  // first routing tile of each sequence [batch + 1]
  int batch;
  int total_tokens;
  int nb_max;               // static bound on the number of blocks
};

cudaError_t launch_plan(const int32_t* cu_in, int batch, int total_tokens, int block_size,
                        int32_t* cu_out, int32_t* blk_off, int32_t* tile_off, int32_t* status,
                        cudaStream_t st);

// cent_norm_max (optional, h_kv floats, zeroed by the caller): receives each
// KV head's largest centroid 2-norm.
cudaError_t launch_conv_centroid(const bf16* k, const float* conv_w, int conv_width, const SeqPlan& p,
                                 int h_kv, int d, int block_size, bf16* k_out, float* cent,
                                 bf16* cent_hi, bf16* cent_lo, float* cent_norm_max, cudaStream_t st);

// Forward accumulator: rows of d floats (the unnormalised O, 256- or
// 512-byte rows, so each starts on an L2 line) and, separately, one float l
// per row.
__host__ __device__ constexpr int oacc_stride(int d) { return d; }

// How many head-windows early the attention kernels issue a head's longest
// CTAs (bucket_order): as many as let those heads' accumulator rows share
// half of L2 with the current head's, at most 2; 0 when one head's rows
// already fill that much.
inline int bucket_lead(long long rows_per_kv_head, int row_bytes) {
  const long long head = rows_per_kv_head * row_bytes;
  if (head <= 0) return 0;
  const long long n = (64ll << 20) / head - 1;
  return (int)(n < 0 ? 0 : (n > 2 ? 2 : n));
}

// cent_norm_max: each KV head's largest centroid 2-norm (launch_conv_centroid).
cudaError_t launch_route(const bf16* q, const bf16* k, const bf16* cent_hi, const bf16* cent_lo,
                         const float* cent_norm_max, const SeqPlan& p, int h_q, int h_kv, int d, int block_size,
                         int topk, int32_t* sel_idx, float* mref, int32_t* flag, float* oacc, float* lacc,
                         int32_t* status, cudaStream_t st);

// chunk_cnt (optional, index_chunk_ints() int32) selects the shared-memory
// privatised path; nullptr, or a zero size from index_chunk_ints(), uses one
// global atomic per pick.
size_t index_chunk_ints(int total_tokens, int h_kv, int nb_max);
cudaError_t launch_build_index(const int32_t* sel_idx, const SeqPlan& p, int h_q, int h_kv,
                               int block_size, int topk, int32_t* cnt, int32_t* ptr, int32_t* cursor,
                               int32_t* rows, int32_t* status, cudaStream_t st, int32_t* chunk_cnt = nullptr);

// Tensor map over a [nrows, d] bf16 row table (16-byte aligned base):
// 64-element boxes `box_rows` rows high, 128-byte swizzle (box_rows = 1 for
// the tile::gather4 row gathers).
cudaError_t make_row_map(CUtensorMap* map, const void* base, unsigned long long nrows, int d, int box_rows = 1);

// Tensor map over a [T, h_kv, d] bf16 key or value tensor: boxes of 64
// channels x one head x `box_tokens` tokens (a key block), 128-byte swizzle.
cudaError_t make_kv_map(CUtensorMap* map, const void* base, int total_tokens, int h_kv, int d, int box_tokens);

// tcgen05 forward attention (every supported d and B); `tm_q` is
// make_row_map over q as T*H_q rows, `tm_k` / `tm_v` make_kv_map over k and v
// with box_tokens = block_size.
cudaError_t launch_fwd_tc(const CUtensorMap& tm_q, const CUtensorMap& tm_k, const CUtensorMap& tm_v,
                          const SeqPlan& p, const int32_t* ptr, const int32_t* rows, const float* mref, int h_q,
                          int h_kv, int d, int block_size, float* oacc, float* lacc, int32_t* flag,
                          int32_t* status, cudaStream_t st);

cudaError_t launch_fwd_finalize(const float* oacc, const float* lacc, const float* mref, const int32_t* flag, int nrows,
                                int d, bf16* out, float* lse, int32_t* flag_list, cudaStream_t st);

cudaError_t launch_fwd_fallback(const bf16* q, const bf16* k, const bf16* v, const SeqPlan& p,
                                const int32_t* sel_idx, const int32_t* flag_list, int h_q, int h_kv,
                                int d, int block_size, int topk, bf16* out, float* lse, int32_t* status,
                                cudaStream_t st);

// stat[row] = (LSE_i, D_i = dO_i . O_i) for the tcgen05 backward (one 8-byte
// load per gathered row); zeroes the dQ accumulator.
cudaError_t launch_bwd_pre(const bf16* out, const bf16* dout, const float* lse, int nrows, int d, float2* stat,
                           float* dqacc, cudaStream_t st);

// tcgen05 backward attention (dK, dV written; dQ added into dqacc) for
// every supported d and B; tm_q / tm_do are make_row_map over q and dout as
// T*H_q rows, tm_k / tm_v make_kv_map over k and v.
cudaError_t launch_bwd_tc(const CUtensorMap& tm_q, const CUtensorMap& tm_k, const CUtensorMap& tm_v,
                          const CUtensorMap& tm_do, const float2* stat, const SeqPlan& p, const int32_t* ptr,
                          const int32_t* rows, int h_q, int h_kv, int d, int block_size, float* dqacc, bf16* dk,
                          bf16* dv, int32_t* status, cudaStream_t st);

cudaError_t launch_bwd_dq(const float* dqacc, int n, bf16* dq, cudaStream_t st);

// dw_part: h_kv * nb_max * d * conv_width floats of per-block partial sums.
cudaError_t launch_conv_bwd(const bf16* k, const float* conv_w, int conv_width, const bf16* dk_conv,
                            const SeqPlan& p, int h_kv, int d, int block_size, bf16* dk, float* dw,
                            float* dw_part, cudaStream_t st);

}  // namespace moba
