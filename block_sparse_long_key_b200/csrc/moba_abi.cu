// C ABI of the MoBA hot path: argument checks, workspace carving and the
// launch order on the caller's stream.  See include/moba.h for the contract.
#include <cuda_runtime.h>

#include <cstdint>
#include <cstring>

#include "moba.h"
#include "common.cuh"
#include "launch.h"

using moba::bf16;

namespace {

constexpr size_t kAlign = 256;

size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

bool shape_ok(const moba_shape* s) {
  if (!s) return false;
  if (s->batch < 1 || s->total_tokens < 0 || s->h_q < 1 || s->h_kv < 1) return false;
  if (s->h_q % s->h_kv != 0) return false;
  if (s->head_dim != 64 && s->head_dim != 128) return false;
  if (s->block_size != 16 && s->block_size != 32 && s->block_size != 64 && s->block_size != 128) return false;
  if (s->topk < 1 || s->topk > 64) return false;
  const long long rows = (long long)s->total_tokens * s->h_q;
  const long long widest = s->head_dim > s->topk ? s->head_dim : s->topk;
  if (rows * widest >= (1LL << 31)) return false;
  return true;
}

int nb_max_of(const moba_shape* s) { return s->total_tokens / s->block_size + s->batch; }

// Bump allocator over the caller's workspace (sizes in bytes).
struct Carve {
  size_t off = 0;
  char* base = nullptr;
  template <typename T>
  T* take(size_t count) {
    T* p = base ? reinterpret_cast<T*>(base + off) : nullptr;
    off = align_up(off + sizeof(T) * count);
    return p;
  }
};

struct PlanBufs {
  int32_t* status;
  int32_t* cu;
  int32_t* blk_off;
  int32_t* tile_off;
};

PlanBufs carve_plan(Carve& c, const moba_shape* s) {
  PlanBufs p;
  p.status = c.take<int32_t>(2);  // [0] status bits, [1] kernel-path bits
  p.cu = c.take<int32_t>(s->batch + 1);
  p.blk_off = c.take<int32_t>(s->batch + 1);
  p.tile_off = c.take<int32_t>(s->batch + 1);
  return p;
}

struct FwdBufs {
  PlanBufs plan;
  float* cent;
  bf16* hi;
  bf16* lo;
  float* cnorm;  // largest centroid norm per KV head (router screen margin)
  float* mref;
  int32_t* flag;
  float* oacc;  // rows of oacc_stride(d) floats: the unnormalised O
  float* lacc;  // one float per row: the softmax denominator l
  int32_t* cnt;
  int32_t* ptr;
  int32_t* cursor;
  int32_t* rows;
  int32_t* chunk_cnt;  // per-chunk bucket histograms of the index builder (may be null)
  int32_t* flag_list;
};

FwdBufs carve_fwd(Carve& c, const moba_shape* s) {
  const size_t nrow = (size_t)s->total_tokens * s->h_q;
  const size_t ncent = (size_t)s->h_kv * nb_max_of(s) * s->head_dim;
  const size_t nbk = (size_t)s->h_kv * nb_max_of(s);
  FwdBufs b;
  b.plan = carve_plan(c, s);
  b.cent = c.take<float>(ncent);
  b.hi = c.take<bf16>(ncent);
  b.lo = c.take<bf16>(ncent);
  b.cnorm = c.take<float>(s->h_kv);
  b.mref = c.take<float>(nrow);
  b.flag = c.take<int32_t>(nrow);
  b.oacc = c.take<float>(nrow * moba::oacc_stride(s->head_dim));
  b.lacc = c.take<float>(nrow);
  b.cnt = c.take<int32_t>(nbk);
  b.ptr = c.take<int32_t>(nbk + 1);
  b.cursor = c.take<int32_t>(nbk);
  b.rows = c.take<int32_t>(nrow * s->topk);
  const size_t nch = moba::index_chunk_ints(s->total_tokens, s->h_kv, nb_max_of(s));
  b.chunk_cnt = nch ? c.take<int32_t>(nch) : nullptr;
  b.flag_list = c.take<int32_t>(nrow + 1);
  return b;
}

struct BwdBufs {
  PlanBufs plan;
  int32_t* cnt;
  int32_t* ptr;
  int32_t* cursor;
  int32_t* rows;
  int32_t* chunk_cnt;
  float2* stat;  // (LSE, D) per row for the tcgen05 backward
  float* dqacc;
  float* dw_part;  // per-block key-conv dW partials (width <= 8)
};

BwdBufs carve_bwd(Carve& c, const moba_shape* s) {
  const size_t nrow = (size_t)s->total_tokens * s->h_q;
  const size_t nbk = (size_t)s->h_kv * nb_max_of(s);
  BwdBufs b;
  b.plan = carve_plan(c, s);
  b.cnt = c.take<int32_t>(nbk);
  b.ptr = c.take<int32_t>(nbk + 1);
  b.cursor = c.take<int32_t>(nbk);
  b.rows = c.take<int32_t>(nrow * s->topk);
  const size_t nch = moba::index_chunk_ints(s->total_tokens, s->h_kv, nb_max_of(s));
  b.chunk_cnt = nch ? c.take<int32_t>(nch) : nullptr;
  b.stat = c.take<float2>(nrow);
  b.dqacc = c.take<float>(nrow * s->head_dim);
  b.dw_part = c.take<float>((size_t)s->h_kv * nb_max_of(s) * s->head_dim * 8);
  return b;
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// Optional per-stage event table of the calling host thread (benchmarks).
thread_local cudaEvent_t const* g_stage_events = nullptr;
thread_local int g_stage_nevents = 0;

// idx < 0 (a plan run by a step entry point without a stage of its own) is not recorded.
void stage_mark(int idx, cudaStream_t st) {
  if (g_stage_events && idx >= 0 && idx < g_stage_nevents && g_stage_events[idx])
    cudaEventRecord(g_stage_events[idx], st);
}
#define STAGE_BEGIN(i) stage_mark(2 * (i), st)
#define STAGE_END(i) stage_mark(2 * (i) + 1, st)

#define MOBA_TRY(expr)                              \
  do {                                              \
    if ((expr) != cudaSuccess) return MOBA_ELAUNCH; \
  } while (0)

int begin_plan(const PlanBufs& pb, const int32_t* cu_seqlens, const moba_shape* s, cudaStream_t st,
               moba::SeqPlan* plan, int stage) {
  STAGE_BEGIN(stage);
  MOBA_TRY(cudaMemsetAsync(pb.status, 0, 2 * sizeof(int32_t), st));
  MOBA_TRY(moba::launch_plan(cu_seqlens, s->batch, s->total_tokens, s->block_size, pb.cu, pb.blk_off, pb.tile_off,
                             pb.status, st));
  STAGE_END(stage);
  plan->cu = pb.cu;
  plan->blk_off = pb.blk_off;
  plan->tile_off = pb.tile_off;
  plan->batch = s->batch;
  plan->total_tokens = s->total_tokens;
  plan->nb_max = nb_max_of(s);
  return MOBA_OK;
}

int check_ptrs(std::initializer_list<const void*> ps) {
  for (const void* p : ps) {
    if (!p) return MOBA_EINVAL;
    if (!aligned(p, 16)) return MOBA_EALIGN;
  }
  return MOBA_OK;
}

int check_ws(const void* ws, size_t have, size_t need) {
  if (!ws) return MOBA_EINVAL;
  if (!aligned(ws, kAlign)) return MOBA_EALIGN;
  if (have < need) return MOBA_EWORKSPACE;
  return MOBA_OK;
}

int check_conv(const float* conv_w, int conv_width, const void* k_out) {
  if (conv_width < 0 || conv_width > 8) return MOBA_EINVAL;
  if (conv_width == 0) return MOBA_OK;
  return check_ptrs({conv_w, k_out});
}

}  // namespace

extern "C" {

size_t moba_fwd_workspace_size(const moba_shape* shape) {
  if (!shape_ok(shape)) return 0;
  Carve c;
  carve_fwd(c, shape);
  return c.off;
}

size_t moba_bwd_workspace_size(const moba_shape* shape) {
  if (!shape_ok(shape)) return 0;
  Carve c;
  carve_bwd(c, shape);
  return c.off;
}

int moba_key_conv_centroid(const void* k, const float* conv_w, int conv_width, const int32_t* cu_seqlens,
                           const moba_shape* shape, void* k_out, float* centroid, void* workspace,
                           size_t workspace_bytes, void* stream) {
  if (!shape_ok(shape)) return MOBA_EINVAL;
  if (shape->total_tokens == 0) return MOBA_OK;
  int rc;
  if ((rc = check_ptrs({k, cu_seqlens, centroid})) != MOBA_OK) return rc;
  if ((rc = check_conv(conv_w, conv_width, k_out)) != MOBA_OK) return rc;
  if (conv_width > 0 && k_out == k) return MOBA_EINVAL;
  if ((rc = check_ws(workspace, workspace_bytes, moba_fwd_workspace_size(shape))) != MOBA_OK) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  Carve c;
  c.base = static_cast<char*>(workspace);
  FwdBufs b = carve_fwd(c, shape);
  moba::SeqPlan plan;
  if ((rc = begin_plan(b.plan, cu_seqlens, shape, st, &plan, -1)) != MOBA_OK) return rc;
  MOBA_TRY(moba::launch_conv_centroid(static_cast<const bf16*>(k), conv_w, conv_width, plan, shape->h_kv,
                                      shape->head_dim, shape->block_size, static_cast<bf16*>(k_out), centroid, b.hi,
                                      b.lo, nullptr, st));
  return MOBA_OK;
}

int moba_forward(const void* q, const void* k, const void* v, const int32_t* cu_seqlens, const moba_shape* shape,
                 const float* conv_w, int conv_width, void* k_conv_out, void* out, float* lse, int32_t* sel_idx,
                 void* workspace, size_t workspace_bytes, void* stream) {
  if (!shape_ok(shape)) return MOBA_EINVAL;
  if (shape->total_tokens == 0) return MOBA_OK;
  int rc;
  if ((rc = check_ptrs({q, k, v, cu_seqlens, out, lse, sel_idx})) != MOBA_OK) return rc;
  if ((rc = check_conv(conv_w, conv_width, k_conv_out)) != MOBA_OK) return rc;
  if (conv_width > 0 && k_conv_out == k) return MOBA_EINVAL;
  if ((rc = check_ws(workspace, workspace_bytes, moba_fwd_workspace_size(shape))) != MOBA_OK) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  Carve c;
  c.base = static_cast<char*>(workspace);
  FwdBufs b = carve_fwd(c, shape);
  moba::SeqPlan plan;
  if ((rc = begin_plan(b.plan, cu_seqlens, shape, st, &plan, MOBA_STAGE_FWD_PLAN)) != MOBA_OK) return rc;
  const int T = shape->total_tokens, hq = shape->h_q, hkv = shape->h_kv, d = shape->head_dim;
  const int B = shape->block_size, topk = shape->topk;
  const bf16* kq = static_cast<const bf16*>(q);
  const bf16* kk = conv_width > 0 ? static_cast<const bf16*>(k_conv_out) : static_cast<const bf16*>(k);
  const bf16* kv = static_cast<const bf16*>(v);
  STAGE_BEGIN(MOBA_STAGE_FWD_CENTROID);
  MOBA_TRY(cudaMemsetAsync(b.cnorm, 0, sizeof(float) * hkv, st));
  MOBA_TRY(moba::launch_conv_centroid(static_cast<const bf16*>(k), conv_w, conv_width, plan, hkv, d, B,
                                      static_cast<bf16*>(k_conv_out), b.cent, b.hi, b.lo, b.cnorm, st));
  STAGE_END(MOBA_STAGE_FWD_CENTROID);
  STAGE_BEGIN(MOBA_STAGE_FWD_ROUTE);
  MOBA_TRY(moba::launch_route(kq, kk, b.hi, b.lo, b.cnorm, plan, hq, hkv, d, B, topk, sel_idx, b.mref, b.flag, b.oacc,
                              b.lacc, b.plan.status, st));
  STAGE_END(MOBA_STAGE_FWD_ROUTE);
  STAGE_BEGIN(MOBA_STAGE_FWD_INDEX);
  MOBA_TRY(moba::launch_build_index(sel_idx, plan, hq, hkv, B, topk, b.cnt, b.ptr, b.cursor, b.rows,
                                    b.plan.status, st, b.chunk_cnt));
  STAGE_END(MOBA_STAGE_FWD_INDEX);
  STAGE_BEGIN(MOBA_STAGE_FWD_ATTN);
  CUtensorMap tm_q, tm_k, tm_v;
  MOBA_TRY(moba::make_row_map(&tm_q, kq, (unsigned long long)T * hq, d));
  MOBA_TRY(moba::make_kv_map(&tm_k, kk, T, hkv, d, B));
  MOBA_TRY(moba::make_kv_map(&tm_v, kv, T, hkv, d, B));
  MOBA_TRY(moba::launch_fwd_tc(tm_q, tm_k, tm_v, plan, b.ptr, b.rows, b.mref, hq, hkv, d, B, b.oacc, b.lacc, b.flag,
                               b.plan.status, st));
  STAGE_END(MOBA_STAGE_FWD_ATTN);
  STAGE_BEGIN(MOBA_STAGE_FWD_FINALIZE);
  MOBA_TRY(moba::launch_fwd_finalize(b.oacc, b.lacc, b.mref, b.flag, T * hq, d, static_cast<bf16*>(out), lse,
                                     b.flag_list, st));
  MOBA_TRY(moba::launch_fwd_fallback(kq, kk, kv, plan, sel_idx, b.flag_list, hq, hkv, d, B, topk,
                                     static_cast<bf16*>(out), lse, b.plan.status, st));
  STAGE_END(MOBA_STAGE_FWD_FINALIZE);
  return MOBA_OK;
}

int moba_build_index(const int32_t* sel_idx, const int32_t* cu_seqlens, const moba_shape* shape, int32_t* blk_ptr,
                     int32_t* blk_rows, void* workspace, size_t workspace_bytes, void* stream) {
  if (!shape_ok(shape)) return MOBA_EINVAL;
  if (shape->total_tokens == 0) return MOBA_OK;
  int rc;
  if ((rc = check_ptrs({sel_idx, cu_seqlens, blk_ptr, blk_rows})) != MOBA_OK) return rc;
  if ((rc = check_ws(workspace, workspace_bytes, moba_bwd_workspace_size(shape))) != MOBA_OK) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  Carve c;
  c.base = static_cast<char*>(workspace);
  BwdBufs b = carve_bwd(c, shape);
  moba::SeqPlan plan;
  if ((rc = begin_plan(b.plan, cu_seqlens, shape, st, &plan, -1)) != MOBA_OK) return rc;
  MOBA_TRY(moba::launch_build_index(sel_idx, plan, shape->h_q, shape->h_kv, shape->block_size, shape->topk, b.cnt,
                                    blk_ptr, b.cursor, blk_rows, b.plan.status, st, b.chunk_cnt));
  return MOBA_OK;
}

int moba_backward(const void* q, const void* k, const void* v, const void* out, const float* lse, const void* dout,
                  const int32_t* sel_idx, const int32_t* cu_seqlens, const moba_shape* shape, void* dq, void* dk,
                  void* dv, void* workspace, size_t workspace_bytes, const void* fwd_workspace, void* stream) {
  if (!shape_ok(shape)) return MOBA_EINVAL;
  if (shape->total_tokens == 0) return MOBA_OK;
  int rc;
  if ((rc = check_ptrs({q, k, v, out, lse, dout, sel_idx, cu_seqlens, dq, dk, dv})) != MOBA_OK) return rc;
  if ((rc = check_ws(workspace, workspace_bytes, moba_bwd_workspace_size(shape))) != MOBA_OK) return rc;
  if (fwd_workspace && !aligned(fwd_workspace, kAlign)) return MOBA_EALIGN;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  Carve c;
  c.base = static_cast<char*>(workspace);
  BwdBufs b = carve_bwd(c, shape);
  moba::SeqPlan plan;
  if ((rc = begin_plan(b.plan, cu_seqlens, shape, st, &plan, MOBA_STAGE_BWD_PLAN)) != MOBA_OK) return rc;
  const int T = shape->total_tokens, hq = shape->h_q, hkv = shape->h_kv, d = shape->head_dim;
  const int32_t* ptr = b.ptr;
  const int32_t* rows = b.rows;
  STAGE_BEGIN(MOBA_STAGE_BWD_INDEX);
  if (fwd_workspace) {
    // Reuse the block index the forward built in its workspace.
    Carve cf;
    cf.base = static_cast<char*>(const_cast<void*>(fwd_workspace));
    FwdBufs f = carve_fwd(cf, shape);
    ptr = f.ptr;
    rows = f.rows;
  } else {
    MOBA_TRY(moba::launch_build_index(sel_idx, plan, hq, hkv, shape->block_size, shape->topk, b.cnt, b.ptr, b.cursor,
                                      b.rows, b.plan.status, st, b.chunk_cnt));
  }
  STAGE_END(MOBA_STAGE_BWD_INDEX);
  STAGE_BEGIN(MOBA_STAGE_BWD_PRE);
  MOBA_TRY(moba::launch_bwd_pre(static_cast<const bf16*>(out), static_cast<const bf16*>(dout), lse, T * hq, d,
                                b.stat, b.dqacc, st));
  STAGE_END(MOBA_STAGE_BWD_PRE);
  STAGE_BEGIN(MOBA_STAGE_BWD_ATTN);
  CUtensorMap tm_q, tm_do, tm_k, tm_v;
  MOBA_TRY(moba::make_row_map(&tm_q, q, (unsigned long long)T * hq, d));
  MOBA_TRY(moba::make_row_map(&tm_do, dout, (unsigned long long)T * hq, d));
  MOBA_TRY(moba::make_kv_map(&tm_k, k, T, hkv, d, shape->block_size));
  MOBA_TRY(moba::make_kv_map(&tm_v, v, T, hkv, d, shape->block_size));
  MOBA_TRY(moba::launch_bwd_tc(tm_q, tm_k, tm_v, tm_do, b.stat, plan, ptr, rows, hq, hkv, d, shape->block_size,
                               b.dqacc, static_cast<bf16*>(dk), static_cast<bf16*>(dv), b.plan.status, st));
  STAGE_END(MOBA_STAGE_BWD_ATTN);
  STAGE_BEGIN(MOBA_STAGE_BWD_DQ);
  MOBA_TRY(moba::launch_bwd_dq(b.dqacc, T * hq * d, static_cast<bf16*>(dq), st));
  STAGE_END(MOBA_STAGE_BWD_DQ);
  return MOBA_OK;
}

int moba_key_conv_backward(const void* k, const float* conv_w, int conv_width, const int32_t* cu_seqlens,
                           const moba_shape* shape, const void* dk_conv, void* dk, float* dw, void* workspace,
                           size_t workspace_bytes, void* stream) {
  if (!shape_ok(shape)) return MOBA_EINVAL;
  if (conv_width < 1 || conv_width > 8) return MOBA_EINVAL;
  if (shape->total_tokens == 0) return MOBA_OK;
  int rc;
  if ((rc = check_ptrs({k, conv_w, cu_seqlens, dk_conv, dk, dw})) != MOBA_OK) return rc;
  if (dk == k || dk == dk_conv) return MOBA_EINVAL;
  if ((rc = check_ws(workspace, workspace_bytes, moba_bwd_workspace_size(shape))) != MOBA_OK) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  Carve c;
  c.base = static_cast<char*>(workspace);
  BwdBufs b = carve_bwd(c, shape);
  moba::SeqPlan plan;
  if ((rc = begin_plan(b.plan, cu_seqlens, shape, st, &plan, -1)) != MOBA_OK) return rc;
  STAGE_BEGIN(MOBA_STAGE_CONV_BWD);
  MOBA_TRY(moba::launch_conv_bwd(static_cast<const bf16*>(k), conv_w, conv_width, static_cast<const bf16*>(dk_conv),
                                 plan, shape->h_kv, shape->head_dim, shape->block_size, static_cast<bf16*>(dk), dw,
                                 b.dw_part, st));
  STAGE_END(MOBA_STAGE_CONV_BWD);
  return MOBA_OK;
}

int moba_set_stage_events(void* const* events, int n_events) {
  if (n_events < 0 || (n_events > 0 && !events)) return MOBA_EINVAL;
  g_stage_events = n_events ? reinterpret_cast<cudaEvent_t const*>(events) : nullptr;
  g_stage_nevents = n_events;
  return MOBA_OK;
}

int moba_check_status(const void* workspace, void* stream, int32_t* device_status) {
  if (!workspace || !device_status) return MOBA_EINVAL;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(st) != cudaSuccess) return MOBA_ELAUNCH;
  int32_t v = 0;
  if (cudaMemcpy(&v, workspace, sizeof(int32_t), cudaMemcpyDeviceToHost) != cudaSuccess) return MOBA_ELAUNCH;
  *device_status = v;
  return v ? MOBA_EDEVICE : MOBA_OK;
}

int moba_check_path(const void* workspace, void* stream, int32_t* path_bits) {
  if (!workspace || !path_bits) return MOBA_EINVAL;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(st) != cudaSuccess) return MOBA_ELAUNCH;
  int32_t v = 0;
  if (cudaMemcpy(&v, static_cast<const int32_t*>(workspace) + 1, sizeof(int32_t), cudaMemcpyDeviceToHost) !=
      cudaSuccess)
    return MOBA_ELAUNCH;
  *path_bits = v;
  return MOBA_OK;
}

const char* moba_status_string(int code) {
  switch (code) {
    case MOBA_OK: return "ok";
    case MOBA_EINVAL: return "invalid argument (null pointer, unsupported size or bad shape)";
    case MOBA_EALIGN: return "misaligned pointer (16 bytes; workspace 256 bytes)";
    case MOBA_EWORKSPACE: return "workspace too small";
    case MOBA_ELAUNCH: return "CUDA launch or stream error";
    case MOBA_EDEVICE: return "device flagged invalid input (see status bits)";
    default: return "unknown status";
  }
}

}  // extern "C"
