/*
 * kascade.h -- C ABI of the Kascade head-aware, cross-layer-reused Top-k
 * sparse attention library for NVIDIA B200 (sm_100a).
 *
 * The method (page "A Practical Sparse Attention Method for Long-Context LLM
 * Inference", the Kascade README, Abstract): a few *anchor* layers compute
 * exact post-softmax attention, pool it per kv head and pick exact Top-k key
 * indices; the *reuse* layers in between attend only over the index set of an
 * anchor head chosen by a per-layer head map.  Selection is tile-level in
 * prefill (tile_size 32, README "Running Evaluations and Performance
 * Benchmarks") and the budget is a fraction of the context ("Top-k set to
 * 10%", Abstract figure caption).
 *
 * Conventions shared by every call
 * --------------------------------
 * Tensors are dense, row-major, bf16 unless stated:
 *   q   [B, Hq,  L, d]   L = q_len (1 in decode, N in prefill)
 *   k,v [B, Hkv, N, d]   one contiguous [N, d] slab per (batch, kv head)
 *   o   [B, Hq,  L, d]   bf16 output
 *   lse [B, Hq,  L]      fp32 natural-log softmax denominator of the scaled
 *                        scores (may be NULL); -inf for a row that sees no key
 * Query head qh belongs to kv head qh / G, G = Hq / Hkv.  Scores are
 * q.k / sqrt(d).
 *
 * Index sets (int32, ascending within each list):
 *   decode  idx [B, Hkv, K]          K = ceil(frac * N)
 *   prefill idx [B, Hkv, S]          S = sum_t k_t, k_t = ceil(frac * e_t),
 *                                    e_t = min(32 (t+1), N); the list of tile t
 *                                    starts at offsets[t] (kascade_index_offsets)
 *
 * Ownership: the caller owns every buffer (device memory for tensors, index
 * lists and the workspace; host memory for kascade_shape and offsets).  The
 * library never allocates or frees memory and keeps no state between calls.
 * All device work is enqueued on `stream` (a cudaStream_t; NULL = legacy
 * default stream) and is asynchronous: results are ready when the stream is.
 *
 * Workspace: every call takes `ws`/`ws_bytes` of device scratch of at
 * least kascade_workspace_bytes(shape, op) bytes, 256-byte aligned.  Its
 * first int is the device error word: kernels never trap or wait without
 * bound, and a bounded wait that gives up stores a non-zero code there
 * (read it with kascade_workspace_error).  Zero the workspace once before
 * first use (kascade_workspace_init); nothing else depends on its initial
 * contents.  The attention calls need only this 256-byte header (their
 * partial results stay on chip) and accept ws = NULL, in which case no error
 * word is kept.  One workspace sized for the largest op serves every call of
 * a shape; calls that may run concurrently must not share a workspace.
 *
 * Errors: every call returns KASCADE_OK (0) or a status below; argument
 * errors are detected on the host before anything is launched.  No kernel
 * traps or waits on another kernel; device-side failures go to the error
 * word described above.
 */
#ifndef KASCADE_H_
#define KASCADE_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define KASCADE_API __attribute__((visibility("default")))
#else
#define KASCADE_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

#define KASCADE_OK 0
#define KASCADE_ERR_INVALID_ARG 1  /* null pointer, bad dims, Hq % Hkv != 0, frac outside (0,1] */
#define KASCADE_ERR_UNSUPPORTED 2  /* d not 64/128, tile != 32, G > 8, q_len not 1 or N, misaligned pointer */
#define KASCADE_ERR_WORKSPACE 3    /* ws NULL, misaligned or smaller than kascade_workspace_bytes() */
#define KASCADE_ERR_CUDA 4         /* a CUDA launch or device query failed */
#define KASCADE_ERR_TOO_LARGE 5    /* the shape needs more scratch than a fixed library buffer holds */

/* Operations for kascade_workspace_bytes(). */
#define KASCADE_OP_SELECT 0
#define KASCADE_OP_SPARSE_DECODE 1
#define KASCADE_OP_SPARSE_PREFILL 2
#define KASCADE_OP_DENSE 3

typedef struct kascade_shape {
  int32_t batch;        /* B  >= 1 */
  int32_t num_q_heads;  /* Hq >= 1, multiple of Hkv */
  int32_t num_kv_heads; /* Hkv >= 1 */
  int32_t head_dim;     /* d: 64 or 128 */
  int32_t q_len;        /* 1 = decode; == kv_len = causal prefill */
  int32_t kv_len;       /* N >= 1 (N <= 2^20) */
  int32_t tile;         /* prefill query tile; must be 32 (ignored in decode) */
  int32_t topk_num;     /* frac = topk_num / topk_den, 0 < frac <= 1, */
  int32_t topk_den;     /*   e.g. 10/100 for the README's Top-k of 10 % */
  int32_t flags;        /* KASCADE_FLAG_* bits, 0 for plain stream ordering */
} kascade_shape;

/* Launch the call's kernels with programmatic dependent launch: a kernel may
 * begin (set-up only) while the previous kernel on the stream finishes; it
 * waits for that kernel's completion before reading any input, and lets the
 * next kernel start right after that wait.  Results are the same as without
 * the flag. */
#define KASCADE_FLAG_PDL 1
/* With KASCADE_FLAG_PDL, sparse decode: the caller guarantees that k, v, idx
 * and head_map were last written at least two kernel launches earlier on the
 * stream (or before it), so the gathers may start before the previous kernel
 * completes.  q and the outputs still wait.  Every kernel of this library
 * releases its successor only after its own wait, which is what makes the
 * two-launch rule sufficient.  Do not set it when the previous kernel on the
 * stream wrote any of those inputs (e.g. the anchor layer's own call right
 * after kascade_select). */
#define KASCADE_FLAG_INPUTS_STABLE 2

/* Bytes of workspace that `op` needs for `shape` (0 on an invalid shape). */
KASCADE_API size_t kascade_workspace_bytes(const kascade_shape* shape, int op);

/* Number of kernels that `op` launches for `shape` on the current device
 * (what a CUDA graph capturing the call will hold): KASCADE_OP_SELECT
 * launches 1 for decode shapes whose scores fit on chip (fused scoring and
 * selection in one cluster launch) and 2 otherwise (scoring, then
 * selection); the attention ops launch 1.  Host-only query (it reads the
 * device's cluster occupancy once).  Returns -1 on an invalid shape or op.
 * The pages describe no such call; it exists for callers that size graphs. */
KASCADE_API int kascade_launch_count(const kascade_shape* shape, int op);

/* Number of int32 entries of the index buffer: B * Hkv * K (decode) or
 * B * Hkv * sum_t k_t (prefill).  Returns -1 on an invalid shape. */
KASCADE_API int64_t kascade_index_count(const kascade_shape* shape);

/* Host-side: writes T+1 int64 tile offsets (T = ceil(N/32)) of one
 * (batch, kv head) index row to `offsets` (host memory, caller-owned);
 * offsets[T] is the row length.  Decode shapes write {0, K}. */
KASCADE_API int kascade_index_offsets(const kascade_shape* shape, int64_t* offsets);

/* Zero-fills `ws_bytes` bytes of device workspace on `stream` (optional:
 * no call depends on the workspace's initial contents). */
KASCADE_API int kascade_workspace_init(void* ws, size_t ws_bytes, void* stream);

/*
 * Anchor-layer selection (README Abstract: "exact Top-k indices ... in a
 * small set of anchor layers"; strategy post_softmax_pooled_prefill_topk).
 *
 * For every (b, kv head h) in decode, or (b, h, query tile t) in prefill:
 * softmax over the visible keys of every query row of h's G query heads,
 * mean of those probabilities over the rows (masked entries count as 0),
 * then the k (= ceil(frac * e)) keys with the largest pooled value among the
 * candidates [0, e), equal values going to the lower index, written in
 * ascending order to `idx` (layout above).  Selection is exact: near the
 * k-th value the pooled scores are recomputed in fp64.
 *   q, k  device, bf16, layouts above
 *   idx   device, int32, kascade_index_count(shape) entries, written
 */
KASCADE_API int kascade_select(const kascade_shape* shape, const void* q, const void* k,
                   int32_t* idx, void* ws, size_t ws_bytes, void* stream);

/*
 * Sparse decode attention of an anchor or reuse layer (README Abstract:
 * reuse layers attend over the anchor's indices; selection and reuse are
 * head-aware).  kv head h attends over the list idx[b, head_map[h]] (the
 * anchor layer's decode index buffer) and for each of its G query heads
 * writes o = softmax(q . k_S / sqrt(d)) v_S.
 *   head_map  device int32 [Hkv], entries in [0, Hkv); NULL = identity
 *             (an anchor layer attending over its own sets).  The host
 *             cannot read it, so the kernel guards it: a kv head whose entry
 *             is out of range attends over an empty list (o = 0, lse = -inf).
 *   idx       device int32 [B, Hkv, K] as written by kascade_select
 *   o, lse    device outputs (lse may be NULL)
 * Requires q_len == 1.  Index values must lie in [0, N) (not checked on the
 * device; kascade_select only writes such values).
 */
KASCADE_API int kascade_sparse_decode(const kascade_shape* shape, const void* q, const void* k,
                          const void* v, const int32_t* idx, const int32_t* head_map,
                          void* o, float* lse, void* ws, size_t ws_bytes, void* stream);

/*
 * Sparse causal prefill attention of an anchor or reuse layer (README
 * Abstract, tile-level operations in prefill).  For query tile t of kv head
 * h, the rows of h's G query heads attend over the keys j of list
 * (b, head_map[h], t) with j <= the row's position.  A row with no such key
 * writes o = 0 and lse = -inf.  Requires q_len == kv_len.
 */
KASCADE_API int kascade_sparse_prefill(const kascade_shape* shape, const void* q, const void* k,
                           const void* v, const int32_t* idx, const int32_t* head_map,
                           void* o, float* lse, void* ws, size_t ws_bytes, void* stream);

/*
 * Dense reference attention (the role FlashAttention-3 plays as the README's
 * speed-up baseline, Abstract): every query attends over all keys (decode,
 * q_len == 1) or causally over keys j <= i (prefill, q_len == N, causal != 0).
 */
KASCADE_API int kascade_dense_ref(const kascade_shape* shape, const void* q, const void* k,
                      const void* v, int causal, void* o, float* lse,
                      void* ws, size_t ws_bytes, void* stream);

/*
 * Decode anchor selection that allocates nothing and takes no workspace.
 * The paper has no counterpart: this serves callers that can neither pass
 * device scratch nor allocate (e.g. an operator inside a host runtime that
 * pre-plans all device memory).  Same inputs, outputs and results as
 * kascade_select for a decode shape (q_len == 1).  Its scratch is a fixed
 * array of kascade_select_decode_static_max_bytes() bytes (8 MiB) inside the
 * library, held by every GPU that loads the library until the process exits.
 * The first call on a device looks up the array's device address with that
 * device current; make that first call before any stream capture.  All calls
 * share the array: calls that may overlap on the GPU race and must be
 * serialised by the caller.  Returns KASCADE_ERR_TOO_LARGE, before launching
 * anything, when the shape needs more than the array holds, and
 * KASCADE_ERR_UNSUPPORTED for prefill shapes.
 */
KASCADE_API int kascade_select_decode_static(const kascade_shape* shape, const void* q, const void* k,
                                             int32_t* idx, void* stream);
/* Size in bytes of the fixed scratch array of kascade_select_decode_static. */
KASCADE_API size_t kascade_select_decode_static_max_bytes(void);

/* Synchronises `stream`, copies the device error word (the first int of
 * `ws`) to *error_out (0 = no failure; 1 = a bounded wait timed out) and, if
 * `clear` is non-zero, resets it. */
KASCADE_API int kascade_workspace_error(const void* ws, int* error_out, int clear, void* stream);

/* Static string for a status code. */
KASCADE_API const char* kascade_status_str(int status);

#ifdef __cplusplus
}
#endif

#endif /* KASCADE_H_ */
