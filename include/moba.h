/*
 * moba.h - C ABI of the B200 (sm_100a) MoBA hot path.
 *
 * MoBA (Mixture of Block Attention), as defined in "Optimizing Mixture of
 * Block Attention" (Xiao, Guo, Mazaheri, Han; summarised on the lowest.today
 * pages, Italian and German): keys are split into blocks of B tokens, each
 * block is represented by its mean key (centroid), every query scores the
 * causally visible centroids with q . k~_j, keeps its own block plus the
 * best-scoring earlier blocks (k blocks in all), and exact softmax attention
 * with scale 1/sqrt(d) runs over the selected tokens only.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  Tokens are packed ("varlen"): sequences s = 0..batch-1 occupy tokens
 *  [cu_seqlens[s], cu_seqlens[s+1]).  cu_seqlens is int32 [batch + 1] in
 *  DEVICE memory, non-decreasing, cu_seqlens[0] = 0, cu_seqlens[batch] = T.
 *  Blocks, causality and the key convolution restart at every sequence.
 *
 *  q, out, dout, dq:  bf16 [T, h_q,  d] row-major (d contiguous).
 *  k, v, dk, dv:      bf16 [T, h_kv, d] row-major.
 *  lse:               fp32 [T, h_q], natural log of sum exp(q.k/sqrt(d)).
 *  sel_idx:           int32 [T, h_q, topk]: the selected blocks of each
 *                     query, block numbers relative to the query's sequence,
 *                     sorted ascending, the query's own block last among the
 *                     valid entries, unused slots -1.
 *  Query head h reads KV head h / (h_q / h_kv) (grouped-query attention).
 *
 *  Every pointer is a device pointer owned by the caller, 16-byte aligned
 *  (the workspace: 256-byte aligned).  The library allocates no memory, keeps
 *  no state between calls (apart from the optional per-thread stage-timing
 *  table of moba_set_stage_events, a cached driver entry point used to build
 *  TMA tensor maps on the host, and the static device scratch of
 *  moba_build_index_noalloc) and never synchronises: each call only enqueues
 *  kernels on `stream` (a cudaStream_t; NULL = legacy default stream) and
 *  returns.  Argument errors are reported synchronously by the return code;
 *  data-dependent errors found on the device (bad cu_seqlens, out-of-range
 *  sel_idx entries) are recorded in the workspace's status word and read
 *  with moba_check_status().  No call ever traps the device.
 *
 *  Supported sizes: d in {64, 128}; B in {16, 32, 64, 128}; 1 <= topk <= 64;
 *  h_q a multiple of h_kv; T * h_q * max(d, topk) < 2^31.  T = 0 is valid:
 *  the call returns MOBA_OK after checking the shape, launches nothing and
 *  leaves the workspace (and its status word) untouched.
 */
#ifndef MOBA_H_
#define MOBA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Problem shape.  All fields are plain host values. */
typedef struct moba_shape {
  int32_t total_tokens; /* T = cu_seqlens[batch] */
  int32_t batch;        /* number of packed sequences, >= 1 */
  int32_t h_q;          /* query heads */
  int32_t h_kv;         /* key/value heads; divides h_q */
  int32_t head_dim;     /* d: 64 or 128 */
  int32_t block_size;   /* B: 16, 32, 64 or 128 */
  int32_t topk;         /* k: selected blocks per query, own block included */
} moba_shape;

/* Return codes. */
#define MOBA_OK 0
#define MOBA_EINVAL (-1)     /* null pointer, unsupported size, bad shape */
#define MOBA_EALIGN (-2)     /* pointer not 16-byte (workspace: 256-byte) aligned */
#define MOBA_EWORKSPACE (-3) /* workspace smaller than the *_workspace_size() */
#define MOBA_ELAUNCH (-4)    /* a kernel launch failed (CUDA error) */
#define MOBA_EDEVICE (-5)    /* moba_check_status(): the device flagged bad input */

/* Device status bits reported by moba_check_status(). */
#define MOBA_STATUS_BAD_SEQLENS 1 /* cu_seqlens not monotone or not ending at T */
#define MOBA_STATUS_BAD_SEL_IDX 2 /* a sel_idx entry outside [-1, own block]; skipped */
#define MOBA_STATUS_INDEX_OVERFLOW 4
#define MOBA_STATUS_TIMEOUT 8     /* a bounded device wait gave up; outputs of that call are invalid */

/* Kernel-path bits reported by moba_check_path(): which kernel families the
 * last call on a workspace ran (each kernel's first thread sets its bit). */
#define MOBA_PATH_ROUTE_TCGEN05 1 /* routing scores on the tcgen05 tensor cores */
#define MOBA_PATH_FWD_TCGEN05 2   /* forward attention on the tcgen05 tensor cores */
#define MOBA_PATH_BWD_TCGEN05 4   /* backward attention on the tcgen05 tensor cores */
#define MOBA_PATH_EXACT_ROWS 8    /* rows far above the softmax reference recomputed exactly */

/* Bytes of device workspace moba_forward / moba_key_conv_centroid need for
 * `shape` (0 for an invalid shape).  The caller allocates it; its contents
 * need no initialisation and are scratch after the call, except the status
 * word read by moba_check_status(). */
size_t moba_fwd_workspace_size(const moba_shape* shape);

/* Bytes of device workspace moba_backward / moba_build_index need. */
size_t moba_bwd_workspace_size(const moba_shape* shape);

/*
 * Key convolution (optional) and block centroids: the first two steps of
 * the forward, exposed on their own.
 *
 * Follows "Optimizing Mixture of Block Attention", section "Progettazione
 * della Convoluzione delle Chiavi (Appendice B)", "Forma Formale":
 *   k'_t = k_t + SiLU(sum_{l=0}^{W-1} w_l (.) k_{t-l})
 * depthwise (one filter per channel), causal with zero padding before the
 * sequence start, no bias; k' is rounded to bf16 (nearest even).  And section
 * "Architettura del Modello Statistico" 1: centroid of block j = mean of its
 * keys (k' when the conv is on; a partial last block averages its real
 * tokens).
 *
 *  k         bf16 [T, h_kv, d]   input keys
 *  conv_w    fp32 [h_kv, d, conv_width], tap l multiplies k_{t-l}; NULL and
 *            conv_width = 0 for no convolution; conv_width <= 8
 *  k_out     bf16 [T, h_kv, d]   k' (ignored when conv_width = 0); must not
 *            alias k
 *  centroid  fp32 [h_kv, nblk, d] where block j of sequence s is row
 *            blk_off[s] + j, blk_off[s] = sum_{s'<s} ceil(L_s'/B), and
 *            nblk = T / B + batch is the row capacity (unused rows untouched)
 */
int moba_key_conv_centroid(const void* k, const float* conv_w, int conv_width, const int32_t* cu_seqlens,
                           const moba_shape* shape, void* k_out, float* centroid, void* workspace,
                           size_t workspace_bytes, void* stream);

/*
 * MoBA forward: (key conv) -> centroids -> routing + top-k -> block index ->
 * gather-and-densify sparse attention -> normalisation.
 *
 * Routing: "Optimizing Mixture of Block Attention", section "Architettura del
 * Modello Statistico" 1 (s_j = q . k~_j) and "Definizione del Compito"
 * (top-k blocks); a query at local position p (block b = p / B) scores blocks
 * j < b, keeps the topk-1 best (exact ties: lower j) and always its own block.
 * Attention: "Definizione del Compito", O = softmax(Q K^T / sqrt(d)) V over
 * the selected tokens, causal inside the own block.
 *
 *  q, k, v           inputs (see conventions)
 *  conv_w, conv_width optional key convolution, as in moba_key_conv_centroid;
 *                    when on, k_conv_out (bf16 [T, h_kv, d]) receives k',
 *                    which routing and attention use and which the backward
 *                    must be given as its k
 *  out               bf16 [T, h_q, d]
 *  lse               fp32 [T, h_q]
 *  sel_idx           int32 [T, h_q, topk] (output)
 *  workspace         >= moba_fwd_workspace_size(shape) bytes
 */
int moba_forward(const void* q, const void* k, const void* v, const int32_t* cu_seqlens,
                 const moba_shape* shape, const float* conv_w, int conv_width, void* k_conv_out, void* out,
                 float* lse, int32_t* sel_idx, void* workspace, size_t workspace_bytes, void* stream);

/*
 * Block index: inverts sel_idx (query -> blocks) into per-(KV head, block)
 * query lists, the key-block-major varlen layout of "Optimizing Mixture of
 * Block Attention", section "Progettazione del Kernel FlashMoBA", "Tre Kernel
 * Fusi" 1 (stage 3) used by the forward and the backward.
 *
 *  blk_ptr   int32 [h_kv * nblk + 1]: bucket (kvh, gb) = kvh * nblk + gb
 *            holds entries blk_ptr[b] .. blk_ptr[b+1]-1; nblk = T / B + batch
 *  blk_rows  int32 [T * h_q * topk] capacity: query row ids t * h_q + h of
 *            every valid pick (own block included); order inside a bucket
 *            is unspecified
 */
int moba_build_index(const int32_t* sel_idx, const int32_t* cu_seqlens, const moba_shape* shape,
                     int32_t* blk_ptr, int32_t* blk_rows, void* workspace, size_t workspace_bytes,
                     void* stream);

/*
 * Allocation-free moba_build_index.  The paper has no counterpart: this entry
 * point exists for callers that cannot provide device scratch memory, such
 * as code running inside a host framework that owns all device memory and
 * forbids side allocations, or latency-critical paths that must not call
 * cudaMalloc because it can synchronise the device.
 *
 * Same inputs and outputs as moba_build_index, without the workspace: its
 * scratch lives in a static device array of MOBA_NOALLOC_SCRATCH_BYTES
 * compiled into the library, which every GPU that loads the library keeps
 * until the process exits.  The call allocates and frees nothing.  blk_ptr
 * is identical to moba_build_index's and every bucket holds the same row
 * ids, but the order of the ids inside a bucket may differ between the two
 * entry points and from call to call (consumers only sum over a bucket).
 *
 *  - Runs on the current device; `stream` must belong to it.  Every call
 *    looks up the array's device address on the current device
 *    (cudaGetSymbolAddress, a host-side query), so a device reset never
 *    leaves a stale address behind.  The first call on a device also makes
 *    the runtime set the array up in that device's context: make it before
 *    any stream capture.
 *  - Every call on a device shares the one array, and the array keeps what the
 *    last call left in it (this call clears what must start at zero).  Calls
 *    whose work overlaps on the GPU (other streams, other host threads) race
 *    on it and give wrong results: serialise them.
 *  - The scratch holds 4 * (h_kv * (T / B + batch)) * 2 bytes of counters and
 *    cursors plus 3 * 4 * (batch + 1) bytes of sequence plan (each part rounded
 *    up to 256 bytes, plus 256); a shape that needs more than
 *    MOBA_NOALLOC_SCRATCH_BYTES returns MOBA_EWORKSPACE and launches nothing.
 *  - Device-side input errors (bad cu_seqlens or sel_idx) are skipped, as in
 *    moba_build_index; the status word is not readable from outside here.
 */
#define MOBA_NOALLOC_SCRATCH_BYTES (8u << 20)
int moba_build_index_noalloc(const int32_t* sel_idx, const int32_t* cu_seqlens, const moba_shape* shape,
                             int32_t* blk_ptr, int32_t* blk_rows, void* stream);

/*
 * MoBA backward with the selection held fixed ("Optimizing Mixture of Block
 * Attention", section "Progettazione del Kernel FlashMoBA", "Tre Kernel
 * Fusi" 3: recompute per key block, dQ by atomic accumulation in fp32).
 *
 *  q, k, v, out, lse, sel_idx   as given to / returned by moba_forward (k is
 *                               k' when the forward used the key conv)
 *  dout              bf16 [T, h_q, d]
 *  dq                bf16 [T, h_q, d]  (output)
 *  dk, dv            bf16 [T, h_kv, d] (output; summed over the query heads
 *                    of each group).  The gradient stops at k': the key
 *                    convolution's own backward is not part of this call.
 *  workspace         >= moba_bwd_workspace_size(shape) bytes
 *  fwd_workspace     optional (NULL: rebuild the block index from sel_idx).
 *                    The workspace of the moba_forward call that produced
 *                    sel_idx, same shape, untouched since: its block index
 *                    is reused instead of being rebuilt.  Read only.
 */
int moba_backward(const void* q, const void* k, const void* v, const void* out, const float* lse,
                  const void* dout, const int32_t* sel_idx, const int32_t* cu_seqlens, const moba_shape* shape,
                  void* dq, void* dk, void* dv, void* workspace, size_t workspace_bytes,
                  const void* fwd_workspace, void* stream);

/*
 * Optional stage timing for benchmarks.  While a table is installed on the
 * calling host thread, moba_forward and moba_backward record events[2*i]
 * (a cudaEvent_t) on their stream before stage i and events[2*i+1] after it,
 * for every i with 2*i+1 < n_events; NULL entries are skipped.  The stages:
 * forward plan, key conv + centroids, routing, block index, attention,
 * normalisation (+ exact re-computation of flagged rows); backward plan,
 * block index, preprocessing, attention, dQ conversion; key-conv backward
 * (moba_key_conv_backward).  The table is read,
 * never written; the caller keeps it (and the events) alive while installed.
 * Pass (NULL, 0) to remove it.  Results are unaffected.
 */
#define MOBA_STAGE_FWD_PLAN 0
#define MOBA_STAGE_FWD_CENTROID 1
#define MOBA_STAGE_FWD_ROUTE 2
#define MOBA_STAGE_FWD_INDEX 3
#define MOBA_STAGE_FWD_ATTN 4
#define MOBA_STAGE_FWD_FINALIZE 5
#define MOBA_STAGE_BWD_PLAN 6
#define MOBA_STAGE_BWD_INDEX 7
#define MOBA_STAGE_BWD_PRE 8
#define MOBA_STAGE_BWD_ATTN 9
#define MOBA_STAGE_BWD_DQ 10
#define MOBA_STAGE_CONV_BWD 11
#define MOBA_NUM_STAGES 12
int moba_set_stage_events(void* const* events, int n_events);

/*
 * Backward of the key convolution, for training with it: from dK' (the
 * gradient moba_backward returns for k', which the attention used) to the
 * gradient of the original keys and of the conv weights.  Differentiates
 * "Optimizing Mixture of Block Attention", section "Progettazione della
 * Convoluzione delle Chiavi (Appendice B)", "Forma Formale", with
 * x_t = sum_l w_l (.) k_{t-l} and g_t = dK'_t (.) SiLU'(x_t):
 *   dK_t = dK'_t + sum_l w_l (.) g_{t+l}   (t + l inside the sequence)
 *   dW_l = sum_t g_t (.) k_{t-l}
 * The bf16 rounding of k' is treated as the identity.
 *
 *  k, conv_w, conv_width, cu_seqlens   as given to moba_forward (1 <= width <= 8)
 *  dk_conv   bf16 [T, h_kv, d]  dK' (e.g. moba_backward's dk)
 *  dk        bf16 [T, h_kv, d]  output; must alias neither k nor dk_conv
 *  dw        fp32 [h_kv, d, conv_width]  output (overwritten, not accumulated)
 *  workspace >= moba_bwd_workspace_size(shape) bytes
 */
int moba_key_conv_backward(const void* k, const float* conv_w, int conv_width, const int32_t* cu_seqlens,
                           const moba_shape* shape, const void* dk_conv, void* dk, float* dw, void* workspace,
                           size_t workspace_bytes, void* stream);

/* Synchronises `stream`, then reads the status word the last call on this
 * workspace left.  *device_status receives the MOBA_STATUS_* bits (0 = ok).
 * Returns MOBA_OK, MOBA_EDEVICE if any bit is set, or MOBA_ELAUNCH if the
 * stream reported a CUDA error. */
int moba_check_status(const void* workspace, void* stream, int32_t* device_status);

/* Synchronises `stream`, then reads which kernel families the last call on
 * this workspace ran (MOBA_PATH_* bits; forward workspace: routing, forward
 * attention, exact rows; backward workspace: backward attention).  Returns
 * MOBA_OK or MOBA_ELAUNCH if the stream reported a CUDA error.  Every shape
 * the library accepts runs the tcgen05 kernels: there is no other attention
 * or routing path. */
int moba_check_path(const void* workspace, void* stream, int32_t* path_bits);

/*
 * Self-test of the bounded device waits (the pages have no counterpart).
 * Every tensor-core kernel of this library waits on mbarriers for TMA copies,
 * MMA completions and hand-offs between warps; each such wait gives up after
 * a wall-clock limit, records MOBA_STATUS_TIMEOUT and lets the kernel return,
 * so a lost completion cannot hang the GPU.  This entry point runs that path
 * on purpose: one CTA waits, with limit `limit_ns` (1 ns .. 10 s), on an
 * mbarrier that is never completed (no copy or MMA is in flight), then sets
 * MOBA_STATUS_TIMEOUT in the status word of `workspace` (>= 256 bytes,
 * 256-byte aligned; only its first 8 bytes are written) and exits.  Read the
 * result with moba_check_status(); the device stays usable afterwards.
 */
int moba_selftest_bounded_wait(unsigned long long limit_ns, void* workspace, size_t workspace_bytes, void* stream);

/* Static description of a return code. */
const char* moba_status_string(int code);

#ifdef __cplusplus
}
#endif

#endif /* MOBA_H_ */
