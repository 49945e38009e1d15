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
 * Tensors are dense, row-major, bf16 (or the shape's KASCADE_DTYPE_*):
 *   q   [B, Hq,  L, d]   L = q_len (1 in decode; N, or a chunk's rows, in prefill)
 *   k,v [B, Hkv, N, d]   one contiguous [N, d] slab per (batch, kv head)
 *   o   [B, Hq,  L, d]   output, the input type
 *   lse [B, Hq,  L]      fp32 natural-log softmax denominator of the scaled
 *                        scores (may be NULL); -inf for a row that sees no key
 * Query head qh belongs to kv head qh / G, G = Hq / Hkv.  Scores are
 * q.k / sqrt(d).
 *
 * Index sets (int32, ascending within each list), L lists per batch row
 * (L = Hkv in the default GQA mode; see KASCADE_SELECT_*):
 *   decode  idx [B, L, K]            K = ceil(frac * N)
 *   prefill idx [B, L, S]            S = sum_t k_t over the call's query tiles,
 *                                    k_t = ceil(frac * e_t), e_t = min(32 (t+1), N);
 *                                    the list of the call's i-th tile starts at
 *                                    offsets[i] (kascade_index_offsets)
 *
 * Ownership: the caller owns every buffer (device memory for tensors, index
 * lists and the workspace; host memory for kascade_shape and offsets).  The
 * library never allocates or frees memory and keeps no state between calls,
 * with one exception: kascade_select_decode_static (below) runs on a fixed
 * __device__ array inside the library image, which every GPU that loads the
 * library holds and which keeps the last such call's contents.
 * All device work is enqueued on `stream` (a cudaStream_t; NULL = legacy
 * default stream) and is asynchronous: results are ready when the stream is.
 *
 * Workspace: every call takes `ws`/`ws_bytes` of device scratch of at
 * least kascade_workspace_bytes(shape, op) bytes, 256-byte aligned.  Its
 * first int is the device error word: kernels never trap or wait without
 * bound, and a bounded wait that gives up stores a non-zero code there
 * (read it with kascade_workspace_error; codes KASCADE_DEVERR_* below).
 * Zero the workspace once before first use (kascade_workspace_init);
 * nothing else depends on its initial contents.  The attention calls need
 * only this 256-byte header (their partial results stay on chip) and accept
 * ws = NULL, in which case no error word is kept (with
 * KASCADE_FLAG_CHECK_INDICES they need more, below).  One workspace sized for
 * the largest op serves every call of a shape; calls that may run
 * concurrently must not share a workspace.
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
#define KASCADE_ERR_UNSUPPORTED 2  /* d not 64/128, tile != 32, G > 8, q_len not 1 or N, misaligned pointer,
                                      dtype not built, all-heads mode with Hq > 64 */
#define KASCADE_ERR_WORKSPACE 3    /* ws NULL, misaligned or smaller than kascade_workspace_bytes() */
#define KASCADE_ERR_CUDA 4         /* a CUDA launch or device query failed */
#define KASCADE_ERR_TOO_LARGE 5    /* the shape needs more scratch than a fixed library buffer holds */

/* Codes a kernel stores in the device error word when one of its bounded
 * waits (about 2^32 SM clocks, a few seconds) gives up.  The kernel records
 * the code, carries on without the missing data and finishes; the call's
 * outputs are then not valid.  The word keeps the last code written until it
 * is cleared. */
#define KASCADE_DEVERR_NONE 0
#define KASCADE_DEVERR_SCORE_POOL 2      /* prefill scoring: a TMA or MMA stage never completed */
#define KASCADE_DEVERR_DECODE_MERGE 3    /* sparse decode: a peer CTA's partial never arrived */
#define KASCADE_DEVERR_PREFILL_ATTN 4    /* sparse prefill: a gather or MMA stage never completed */
#define KASCADE_DEVERR_DECODE_SELECT 5   /* decode selection: a cluster exchange never completed */
#define KASCADE_DEVERR_DECODE_GATHER 6   /* sparse decode: a bulk-copied K or V row never arrived */
#define KASCADE_DEVERR_INDEX_LIST 7      /* KASCADE_FLAG_CHECK_INDICES: an index input out of range or unsorted */

/* Operations for kascade_workspace_bytes(). */
#define KASCADE_OP_SELECT 0
#define KASCADE_OP_SPARSE_DECODE 1
#define KASCADE_OP_SPARSE_PREFILL 2
#define KASCADE_OP_DENSE 3
#define KASCADE_OP_REFINE 4   /* kascade_refine_select, any pool length up to N */
#define KASCADE_OP_SELECT_VARLEN 5   /* kascade_select_varlen */

typedef struct kascade_shape {
  int32_t batch;        /* B  >= 1 */
  int32_t num_q_heads;  /* Hq >= 1, multiple of Hkv */
  int32_t num_kv_heads; /* Hkv >= 1 */
  int32_t head_dim;     /* d: 64 or 128 */
  int32_t q_len;        /* 1 = decode; else causal prefill of the last q_len positions
                           of the context: q_len == kv_len is the whole prompt,
                           q_len < kv_len a rolling chunk (README, Python API,
                           rolling_prefill) whose first position kv_len - q_len is a
                           multiple of 32; the call then covers only the chunk's query
                           tiles, exactly as the whole prompt's call computes them */
  int32_t kv_len;       /* N >= 1 (N <= 2^20) */
  int32_t tile;         /* prefill query tile; must be 32 (ignored in decode) */
  int32_t topk_num;     /* frac = topk_num / topk_den, 0 < frac <= 1, */
  int32_t topk_den;     /*   e.g. 10/100 for the README's Top-k of 10 % */
  int32_t flags;        /* KASCADE_FLAG_* bits, 0 for plain stream ordering */
  int32_t select_mode;  /* KASCADE_SELECT_*: which query heads a selection pools */
  int32_t dtype;        /* KASCADE_DTYPE_*: element type of q, k, v and o */
} kascade_shape;

/* Head-selection modes (README, Reproducibility: the default strategy
 * post_softmax_pooled_prefill_topk beside oracle_topk, Figure 1, and
 * post_softmax_all_heads_pooled_oracle_topk, Figure 3; the Abstract calls
 * head-aware selection critical for accuracy).  The mode fixes the index
 * lists per batch row, L, and what head_map maps:
 *   GQA       L = Hkv: list h pools the G query heads of kv head h (default);
 *             head_map [Hkv] maps kv heads to anchor kv heads.
 *   PER_HEAD  L = Hq: list qh is query head qh's own selection (no pooling
 *             across heads; in prefill still pooled over the 32-row tile);
 *             head_map [Hq] maps query heads to anchor query heads.
 *   ALL_HEADS L = 1: one list per batch row pools every query head, each
 *             scored against its own kv head (head-unaware); every head of
 *             every layer reads it and head_map is ignored.  Hq <= 64.
 * Index buffers are [B, L, K] (decode) or [B, L, sum_t k_t] (prefill). */
#define KASCADE_SELECT_GQA 0
#define KASCADE_SELECT_PER_HEAD 1
#define KASCADE_SELECT_ALL_HEADS 2

/* Element types of q, k, v and o (lse is always fp32).  BF16 runs the
 * tensor-core kernels.  FP32 and FP16 run a CUDA-core path: selection scores
 * with fp64 products, attention in fp32, results rounded once to the output
 * type (fp32 outputs within 1e-4 of exact attention over the selected keys);
 * built for correctness, not for the bf16 path's speed.  (The README's own
 * kernels take fp16 only, Running Evaluations.) */
#define KASCADE_DTYPE_BF16 0
#define KASCADE_DTYPE_F32 1
#define KASCADE_DTYPE_F16 2

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
/* Test only, for checking failure reporting: the prefill scoring kernel of
 * kascade_select announces each CTA's first query-tile load but never issues
 * it.  The waits on that load give up after their bound (a few seconds),
 * the kernel finishes without further waiting, the workspace error word
 * reads KASCADE_DEVERR_SCORE_POOL and the call's outputs are not valid.  No
 * other call reads the flag. */
#define KASCADE_FLAG_TEST_DROP_LOAD (1 << 30)
/* Index validation, a debugging aid (the method has no counterpart): the
 * sparse decode calls (contiguous, paged, varlen), kascade_sparse_prefill and
 * kascade_refine_select first copy their index lists, head_map and kv_lens
 * into the workspace through a checking kernel, and the attention or refine
 * kernels read the copies.  Entries out of range (list entries outside the
 * keys their list may name: [0, ceil(frac n_b)) entries in [0, n_b) for a
 * decode row of n_b keys, tile t's entries in [0, min(32 (t + 1), N)), pool
 * entries in [0, N); head_map outside [0, lists per row); kv_lens outside
 * [1, N]) set the workspace error word to KASCADE_DEVERR_INDEX_LIST and are
 * clamped into range in the copy, so no load leaves the K and V buffers;
 * lists that are not strictly ascending set the word too.  The results of a
 * call that set the word are not valid.  Page-table entries are not checked
 * (the call carries no page count).  Requires a workspace of
 * kascade_workspace_bytes(shape, op) with the flag in shape->flags (the
 * copies live there); clears KASCADE_FLAG_INPUTS_STABLE for the call.  One
 * extra launch per call. */
#define KASCADE_FLAG_CHECK_INDICES 4

/* Bytes of workspace that `op` needs for `shape` (0 on an invalid shape). */
KASCADE_API size_t kascade_workspace_bytes(const kascade_shape* shape, int op);

/* Number of kernels that `op` launches for `shape` on the current device
 * (what a CUDA graph capturing the call will hold): KASCADE_OP_SELECT
 * launches 1 for decode shapes whose scores fit on chip (fused scoring and
 * selection in one cluster launch) and 2 otherwise (scoring, then
 * selection); the attention ops launch 1 (2 with KASCADE_FLAG_CHECK_INDICES,
 * except the dense form).  Host-only query (it reads the
 * device's cluster occupancy once).  Returns -1 on an invalid shape or op.
 * The pages describe no such call; it exists for callers that size graphs. */
KASCADE_API int kascade_launch_count(const kascade_shape* shape, int op);

/* Number of int32 entries of the index buffer: B * L * K (decode) or
 * B * L * sum_t k_t (prefill), L the lists per batch row of the shape's
 * select_mode.  Returns -1 on an invalid shape. */
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
 * For every (b, list l) in decode, or (b, l, query tile t) in prefill:
 * softmax over the visible keys of every query row of the list's query heads
 * (the G heads of kv head l by default; see KASCADE_SELECT_*), mean of those
 * probabilities over the rows (masked entries count as 0), then the
 * k (= ceil(frac * e)) keys with the largest pooled value among the
 * candidates [0, e), equal values going to the lower index, written in
 * ascending order to `idx` (layout above).  Selection is exact: near the
 * k-th value the pooled scores are recomputed in fp64.
 *   q, k  device, bf16, layouts above
 *   idx   device, int32, kascade_index_count(shape) entries, written
 */
KASCADE_API int kascade_select(const kascade_shape* shape, const void* q, const void* k,
                   int32_t* idx, void* ws, size_t ws_bytes, void* stream);

/*
 * Proposal-refine selection of a decode layer (Prism Attention page,
 * abstract and the caption of Table 9: a proposal layer builds a pool of
 * rho * kappa candidate indices and each refined layer picks its own top
 * kappa from the pool of its nearest preceding proposal layer; an
 * alternative to rigid reuse of one index set).
 *
 * kv head h scores only the keys of pool list head_map[h] (its own K rows
 * at those positions), takes the post-softmax probabilities of each of its
 * G query heads over the pool, pools them (mean over the G heads) and
 * writes the k = ceil(frac * N) keys with the largest pooled value, lower
 * index on ties, ascending, to idx [B, Hkv, k]; exact, with the same fp64
 * band as kascade_select.
 *   pool      device int32 [B, Hkv, pool_len], ascending key indices in
 *             [0, N), e.g. written by kascade_select for the proposal layer
 *             with a budget rho times this shape's (not checked on the
 *             device)
 *   pool_len  k <= pool_len <= N, else KASCADE_ERR_INVALID_ARG
 *   head_map  device int32 [Hkv], entries in [0, Hkv) (an out-of-range
 *             entry reads list 0); NULL = identity
 *   ws        kascade_workspace_bytes(shape, KASCADE_OP_REFINE) bytes
 * Requires q_len == 1 and the GQA selection mode (KASCADE_ERR_UNSUPPORTED
 * otherwise); bf16 or fp32 inputs.  The refined layer then attends with
 * kascade_sparse_decode over idx (head_map NULL).
 */
KASCADE_API int kascade_refine_select(const kascade_shape* shape, const void* q, const void* k,
                                      const int32_t* pool, int32_t pool_len, const int32_t* head_map,
                                      int32_t* idx, void* ws, size_t ws_bytes, void* stream);

/*
 * Sparse decode attention of an anchor or reuse layer (README Abstract:
 * reuse layers attend over the anchor's indices; selection and reuse are
 * head-aware).  kv head h attends over the list idx[b, head_map[h]] (the
 * anchor layer's decode index buffer) and for each of its G query heads
 * writes o = softmax(q . k_S / sqrt(d)) v_S.
 *   head_map  device int32 [Hkv] with entries in [0, Hkv) (GQA mode), or
 *             [Hq] with entries in [0, Hq) (per-head mode, query head qh
 *             reads list head_map[qh]); ignored in the all-heads mode; NULL =
 *             identity (an anchor layer attending over its own sets).  The
 *             host cannot read it, so the kernel guards it: a head whose
 *             entry is out of range attends over an empty list (o = 0,
 *             lse = -inf).
 *   idx       device int32 [B, L, K] as written by kascade_select
 *   o, lse    device outputs (lse may be NULL)
 * Requires q_len == 1.  Index values must lie in [0, N) (not checked on the
 * device; kascade_select only writes such values).
 */
KASCADE_API int kascade_sparse_decode(const kascade_shape* shape, const void* q, const void* k,
                          const void* v, const int32_t* idx, const int32_t* head_map,
                          void* o, float* lse, void* ws, size_t ws_bytes, void* stream);

/*
 * Variable-length decode batches (README, Kernel Benchmarks note: varlen
 * kernels are planned).  Batch row b holds kv_lens[b] keys, 1 <= kv_lens[b]
 * <= N = shape->kv_len (device int32 [B], not checked on the device), in
 * the first kv_lens[b] rows of its [N, d] slabs.  Row b's selection and
 * attention are those of a batch of one with context kv_lens[b].
 *
 * kascade_select_varlen: as kascade_select for a decode shape (any selection
 * mode), each row selecting ceil(frac kv_lens[b]) of its keys.  The index
 * buffer keeps the layout of kv_len = N, [B, L, ceil(frac N)]: row b's lists
 * hold their ceil(frac kv_lens[b]) keys ascending, then -1.  Workspace:
 * kascade_workspace_bytes(shape, KASCADE_OP_SELECT_VARLEN).  bf16.
 *
 * kascade_sparse_decode_varlen: as kascade_sparse_decode, row b attending
 * over the first ceil(frac kv_lens[b]) entries of its list (idx NULL: dense
 * over its kv_lens[b] keys).  With KASCADE_FLAG_INPUTS_STABLE, kv_lens counts
 * among the inputs that must be two launches old.  bf16.
 */
KASCADE_API int kascade_select_varlen(const kascade_shape* shape, const void* q, const void* k,
                                      const int32_t* kv_lens, int32_t* idx, void* ws, size_t ws_bytes,
                                      void* stream);
KASCADE_API int kascade_sparse_decode_varlen(const kascade_shape* shape, const void* q, const void* k,
                                             const void* v, const int32_t* kv_lens, const int32_t* idx,
                                             const int32_t* head_map, void* o, float* lse, void* ws,
                                             size_t ws_bytes, void* stream);

/*
 * kascade_sparse_decode over a paged KV cache (README, Kernel Benchmarks
 * note: paged kernels are planned; a paged cache stores the same keys in
 * fixed-size pages, so the results are those of kascade_sparse_decode on the
 * contiguous cache, bit for bit).
 *   k_pages, v_pages  device bf16 [num_pages, Hkv, page_size, d]: page p
 *             holds page_size consecutive positions of one sequence for
 *             every kv head
 *   page_table device int32 [B, max_pages]: key j of batch row b is row
 *             j % page_size of page page_table[b * max_pages + j / page_size]
 *             (entries must name allocated pages; not checked on the device)
 *   page_size a power of two in [16, 2^20]; max_pages >= ceil(N / page_size)
 *   idx       as for kascade_sparse_decode, or NULL for dense decode over
 *             the whole paged context
 * Other arguments as kascade_sparse_decode.  bf16 only.  Anchor selection
 * reads a contiguous K (kascade_select); this call serves the reuse layers.
 */
KASCADE_API int kascade_sparse_decode_paged(const kascade_shape* shape, const void* q, const void* k_pages,
                                            const void* v_pages, const int32_t* page_table, int32_t page_size,
                                            int32_t max_pages, const int32_t* idx, const int32_t* head_map,
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

/* The device error word of kascade_select_decode_static on the current
 * device: the first int of its fixed array, which plays the role the
 * workspace's first int plays for kascade_select.  Synchronises `stream`,
 * stores the word (KASCADE_DEVERR_*) in *error_out and, if `clear` is
 * non-zero, resets it.  Every static call on the device shares this word. */
KASCADE_API int kascade_select_decode_static_error(int* error_out, int clear, void* stream);

/* Synchronises `stream`, copies the device error word (the first int of
 * `ws`) to *error_out (KASCADE_DEVERR_NONE = no failure, else the code of
 * the kernel whose bounded wait gave up) and, if `clear` is non-zero,
 * resets it. */
KASCADE_API int kascade_workspace_error(const void* ws, int* error_out, int clear, void* stream);

/*
 * Anchor-layer selection (README, Abstract: the anchor layers are chosen by
 * a dynamic program that maximises cross-layer similarity over a
 * development set; Reproducibility, Figure 4, select_layers).
 *
 * kascade_index_overlap: for two index buffers a and b of one shape (layout
 * above, ascending lists, e.g. two layers' kascade_select outputs), writes
 * counts[p] = sum over the tiles of |a_t and b_t| for every (batch row,
 * list) p, B * L int64 values (device memory), on `stream`.  Divided by the
 * list length, this is the index-set overlap of the two layers.
 *
 * kascade_plan_anchors (host): sim is a row-major [n_layers][n_layers] host
 * array, sim[a][l] the similarity of layer l to an earlier layer a (only
 * a <= l is read; sim[l][l] is what an anchor scores for itself, e.g. 1).
 * Writes the n_anchors anchor layers, ascending and always starting at layer
 * 0, that maximise the sum over layers of sim[anchor(l)][l], anchor(l) the
 * nearest anchor at or before l (every other layer reuses it), and the
 * maximum to *objective (may be NULL).  Among equal sums the plan with the
 * smallest anchor list (lexicographically) wins.  O(n_anchors * n_layers^2).
 */
KASCADE_API int kascade_index_overlap(const kascade_shape* shape, const int32_t* a, const int32_t* b,
                                      int64_t* counts, void* stream);
KASCADE_API int kascade_plan_anchors(const double* sim, int32_t n_layers, int32_t n_anchors, int32_t* anchors,
                                     double* objective);

/* Static string for a status code. */
KASCADE_API const char* kascade_status_str(int status);

#ifdef __cplusplus
}
#endif

#endif /* KASCADE_H_ */
