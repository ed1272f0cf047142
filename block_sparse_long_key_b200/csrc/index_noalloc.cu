// Allocation-free variant of moba_build_index.
//
// Some callers cannot hand this library a workspace: they run inside a host
// framework that owns every byte of device memory and forbids side
// allocations, or on a latency-critical path where cudaMalloc is off limits
// because it may synchronise the device.  For them this entry point keeps its
// scratch (sequence plan, per-bucket counters and fill cursors) in a
// fixed-size array compiled into the library, so a call needs nothing but
// its inputs and outputs.
//
// The array is a file-scope __device__ variable: every GPU that loads the
// library holds MOBA_NOALLOC_SCRATCH_BYTES of it until the process exits.
// In host code its name is only a host-side handle, not a device address, so
// every call looks the address up with cudaGetSymbolAddress on the current
// device.  The lookup is a host-side query (no device work, no allocation);
// re-doing it per call keeps the pointer valid for the context that is
// current now, also after a cudaDeviceReset re-created it.
#include <cuda_runtime.h>

#include <cstdint>

#include "moba.h"
#include "launch.h"

namespace {

static __device__ __align__(256) unsigned char g_index_scratch[MOBA_NOALLOC_SCRATCH_BYTES];

constexpr size_t kAlign = 256;

size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

// Device address of the scratch array in the current device's context.
int scratch_address(void** out) {
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_index_scratch) != cudaSuccess || !p) return MOBA_ELAUNCH;
  *out = p;
  return MOBA_OK;
}

bool shape_valid(const moba_shape* s) {
  if (!s) return false;
  if (s->batch < 1 || s->total_tokens < 0 || s->h_q < 1 || s->h_kv < 1) return false;
  if (s->h_q % s->h_kv != 0) return false;
  if (s->head_dim != 64 && s->head_dim != 128) return false;
  if (s->block_size != 16 && s->block_size != 32 && s->block_size != 64 && s->block_size != 128) return false;
  if (s->topk < 1 || s->topk > 64) return false;
  const long long rows = (long long)s->total_tokens * s->h_q;
  const long long widest = s->head_dim > s->topk ? s->head_dim : s->topk;
  return rows * widest < (1LL << 31);
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" int moba_build_index_noalloc(const int32_t* sel_idx, const int32_t* cu_seqlens, const moba_shape* shape,
                                        int32_t* blk_ptr, int32_t* blk_rows, void* stream) {
  if (!shape_valid(shape)) return MOBA_EINVAL;
  if (shape->total_tokens == 0) return MOBA_OK;
  for (const void* p : {static_cast<const void*>(sel_idx), static_cast<const void*>(cu_seqlens),
                        static_cast<const void*>(blk_ptr), static_cast<const void*>(blk_rows)}) {
    if (!p) return MOBA_EINVAL;
    if (!aligned16(p)) return MOBA_EALIGN;
  }
  // Scratch layout: status word | cu | blk_off | tile_off | counts | cursors.
  const size_t nb_max = (size_t)shape->total_tokens / shape->block_size + shape->batch;
  const size_t nbk = (size_t)shape->h_kv * nb_max;
  const size_t seq = sizeof(int32_t) * ((size_t)shape->batch + 1);
  const size_t off_cu = kAlign;
  const size_t off_blk = off_cu + align_up(seq);
  const size_t off_tile = off_blk + align_up(seq);
  const size_t off_cnt = off_tile + align_up(seq);
  const size_t off_cur = off_cnt + align_up(sizeof(int32_t) * nbk);
  const size_t need = off_cur + align_up(sizeof(int32_t) * nbk);
  if (need > MOBA_NOALLOC_SCRATCH_BYTES) return MOBA_EWORKSPACE;

  void* base = nullptr;
  int rc = scratch_address(&base);
  if (rc != MOBA_OK) return rc;
  char* b = static_cast<char*>(base);
  int32_t* status = reinterpret_cast<int32_t*>(b);
  int32_t* cu = reinterpret_cast<int32_t*>(b + off_cu);
  int32_t* blk_off = reinterpret_cast<int32_t*>(b + off_blk);
  int32_t* tile_off = reinterpret_cast<int32_t*>(b + off_tile);
  int32_t* cnt = reinterpret_cast<int32_t*>(b + off_cnt);
  int32_t* cursor = reinterpret_cast<int32_t*>(b + off_cur);

  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // The array keeps whatever the previous call left: clear what must start at
  // zero (the status word here; the counts inside launch_build_index).
  if (cudaMemsetAsync(status, 0, sizeof(int32_t), st) != cudaSuccess) return MOBA_ELAUNCH;
  if (moba::launch_plan(cu_seqlens, shape->batch, shape->total_tokens, shape->block_size, cu, blk_off, tile_off,
                        status, st) != cudaSuccess)
    return MOBA_ELAUNCH;
  moba::SeqPlan plan;
  plan.cu = cu;
  plan.blk_off = blk_off;
  plan.tile_off = tile_off;
  plan.batch = shape->batch;
  plan.total_tokens = shape->total_tokens;
  plan.nb_max = (int)nb_max;
  if (moba::launch_build_index(sel_idx, plan, shape->h_q, shape->h_kv, shape->block_size, shape->topk, cnt, blk_ptr,
                               cursor, blk_rows, status, st) != cudaSuccess)
    return MOBA_ELAUNCH;
  return MOBA_OK;
}
