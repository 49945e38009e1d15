// Internal launch interface between the C ABI layer (api.cu) and the kernels.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace kascade {

// Problems.  A selection or attention call is split into problems per batch
// row: problem p serves query heads [p G, p G + G) and reads the keys and
// values of kv head (p G) / Gkv (Gkv = Hq / Hkv).  GQA pooling (the default):
// Hp = Hkv problems of G = Gkv heads.  Per query head: Hp = Hq problems of
// G = 1 head.  All heads pooled (selection only): Hp = 1 problem of G = Hq
// heads, whose heads read different kv heads.
__host__ __device__ inline int kv_slab_of(int b, int qh, int Hkv, int Gkv) { return b * Hkv + qh / Gkv; }

struct DecodeScoreArgs {
  const __nv_bfloat16* q;  // [B, Hq, 1, D]
  const __nv_bfloat16* k;  // [B, Hkv, N, D]
  float* s2;               // [B, Hq, N]      scores * log2(e)/sqrt(D)
  float* m_part;           // [B, Hq, splits]
  double* l_part;          // [B, Hq, splits]
  int B, Hq, Hkv, G, D, N;
  int flags;
  // proposal-refine: score only the keys of a candidate list per (b, kv
  // head): list head_map[h] (NULL = h) of `cand` [B, cand_lists, N]; N is
  // then the list length and n_ctx the rows of each K slab
  const int32_t* cand;
  const int32_t* cand_map;
  int cand_lists;
  int n_ctx;
  const int32_t* kv_lens;  // varlen: batch row b scores keys [0, kv_lens[b]) (NULL: all N)
};
int decode_score_keys_per_split();
cudaError_t launch_decode_score(const DecodeScoreArgs& a, cudaStream_t stream);

// Top-k selection over pooled post-softmax scores (decode or prefill).
struct SelArgs {
  bool prefill;
  int B, Hq, Hkv, G, D, N, tile, num, den;
  int Hp;                  // problems per batch row (index lists per row)
  int Gkv;                 // query heads per kv head
  int q0, Lq;              // prefill: query rows are positions [q0, q0 + Lq = N) (rolling chunk)
  int in_type;             // element type of q and k: 0 bf16, 1 fp32, 2 fp16 (pointers reinterpreted)
  // decode proposal-refine: the N candidates of problem (b, h) are the keys
  // cand[(b * cand_lists + cand_map[h]) * N + j] (cand_map NULL = h); K slabs
  // hold n_ctx rows and the output keeps topk_count(n_ctx) keys
  const int32_t* cand;
  const int32_t* cand_map;
  int cand_lists;
  int n_ctx;
  const int32_t* kv_lens;  // decode varlen: batch row b selects among keys [0, kv_lens[b]) (NULL: N);
                           // lists keep the stride of N and end in -1 past ceil(frac kv_lens[b])
  const __nv_bfloat16* q;  // [B, Hq, Lq, D]
  const __nv_bfloat16* k;  // [B, Hkv, N, D]
  // decode inputs
  const float* s2;         // [B, Hq, N]
  const float* m_part;     // [B, Hq, splits]
  const double* l_part;    // [B, Hq, splits]
  int splits;
  // prefill inputs
  const float* pooled;     // [B, Hkv, sum_t e_t] fp32 pooled scores
  const float* row_m2;     // [B, Hq, N]  row max of s2
  const double* row_l;     // [B, Hq, N]  row sum of exp2(s2 - m2)
  // per-CTA scratch (grid CTAs, n_max entries each)
  float* v_scratch;        // decode only
  int32_t* band_idx;
  double* band_val;
  uint8_t* state;
  int n_max;
  int grid;
  int32_t* idx;            // output
  int flags;
  int* err;                // device error word (a bounded wait gave up), may be NULL
};
size_t select_scratch_bytes_per_cta(int n_max);
// decode: one 8-CTA cluster per (batch, kv head) when N / 8 <= 16384 (band
// scratch also sized for the fused kernel)
bool select_decode_cluster_ok(int N);
size_t select_decode_cluster_scratch(int B, int problems, int N);   // band entries (problems per batch row)
cudaError_t launch_select_decode_cluster(const SelArgs& a, cudaStream_t stream);
// decode: fused scoring + selection (one cluster per (batch, kv head), K
// streamed once, scores kept on chip) when the shape and device allow it
bool anchor_select_fused_ok(const SelArgs& a);
cudaError_t launch_anchor_select_fused(const SelArgs& a, cudaStream_t stream);
int select_grid(bool prefill, int problems, int num_sms);
cudaError_t launch_select(const SelArgs& a, cudaStream_t stream);

// Anchor prefill scoring and pooling (row statistics, then pooled scores).
struct ScorePoolArgs {
  const __nv_bfloat16* q;  // [B, Hq, N, D]
  const __nv_bfloat16* k;  // [B, Hkv, N, D]
  float* row_m2;           // [B, Hq, N]
  double* row_l;           // [B, Hq, N]
  float* pooled;           // [B, Hkv, sum_t e_t], or [B, Hq, sum_t e_t] with per_head (the chunk's tiles)
  int B, Hq, Hkv, G, D, N, tile;
  int q0, Lq;              // query rows: positions [q0, q0 + Lq = N); row stats are [B, Hq, Lq]
  int flags;
  bool per_head;           // pool each query head on its own (no GQA mean)
};
cudaError_t launch_score_pool(const ScorePoolArgs& a, cudaStream_t stream);
// tcgen05/TMEM + TMA version (G <= 4); err: device error word (may be NULL)
bool score_pool_tc_supported(const ScorePoolArgs& a);
cudaError_t launch_score_pool_tc(const ScorePoolArgs& a, int* err, int num_sms, cudaStream_t stream);

// Sparse / dense attention over an index list (decode: split-K + combine).
struct AttnArgs {
  const __nv_bfloat16* q;
  const __nv_bfloat16* k;
  const __nv_bfloat16* v;
  const int32_t* idx;        // NULL: dense
  const int32_t* head_map;   // NULL: identity
  __nv_bfloat16* o;
  float* lse;                // may be NULL
  int B, Hq, Hkv, G, D, N, tile, num, den;
  int Hp;                    // problems per batch row (G = query heads per problem)
  int Gkv;                   // query heads per kv head
  int q0, Lq;                // prefill: query (and o, lse) rows are positions [q0, q0 + Lq = N)
  // decode over a paged cache (NULL: contiguous slabs): k and v are pages
  // [num_pages, Hkv, page_size, D]; key j of batch row b is row j % page_size
  // of page page_table[b * max_pages + j / page_size]
  const int32_t* page_table;
  int page_size, page_shift, max_pages;
  const int32_t* kv_lens;    // decode varlen: batch row b attends over its first ceil(frac kv_lens[b])
                             // list entries (dense: keys [0, kv_lens[b])); NULL: all
  int n_lists;               // index lists per batch row
  bool one_list;             // every problem reads list 0 of its row (head_map unused)
  bool causal;               // prefill dense only
  int* err;                  // device error word (a bounded wait gave up), may be NULL
  int flags;                 // KASCADE_FLAG_* bits
};
// fp32- and fp16-input variants (q, k, v, o of that type behind the same
// pointers; half = fp16): scoring with fp64 products into the bf16 path's
// workspace layouts, then the shared Top-k; fp32 attention on CUDA cores
cudaError_t launch_decode_score_f32(const DecodeScoreArgs& a, bool half, cudaStream_t stream);
cudaError_t launch_score_pool_f32(const ScorePoolArgs& a, bool half, cudaStream_t stream);
cudaError_t launch_sparse_decode_f32(const AttnArgs& a, bool half, cudaStream_t stream);
cudaError_t launch_sparse_prefill_f32(const AttnArgs& a, bool half, cudaStream_t stream);

// mean over the Hkv rows of pooled scores: out[b, x] = (1/Hkv) sum_h in[b, h, x]
cudaError_t launch_pool_mean(const float* in, float* out, int B, int Hkv, int64_t row, int flags,
                             cudaStream_t stream);

// decode: one 16-CTA cluster per (batch, kv head), merge over DSMEM
// Checked copies of index inputs (KASCADE_FLAG_CHECK_INDICES): rows of
// `row_len` entries, B * L of them (L lists per batch row); decode lists,
// prefill tile lists (tiles t0 .. T - 1) or refine pools (`pool`: every
// entry in [0, N)); head_map (n_map entries, in [0, L)) and kv_lens (B
// entries, NULL = none) copied to hm_out / kv_out.
struct CheckArgs {
  const int32_t* idx;
  int32_t* idx_out;
  const int32_t* head_map;
  int32_t* hm_out;
  int n_map;
  const int32_t* kv_lens;
  int32_t* kv_out;
  int B, L, N, num, den, t0;
  int64_t row_len;
  bool prefill, pool, pdl;
  int* err;
};
cudaError_t launch_check_lists(const CheckArgs& c, cudaStream_t stream);

cudaError_t launch_decode_attn(const AttnArgs& a, cudaStream_t stream);
cudaError_t launch_prefill_attn(const AttnArgs& a, cudaStream_t stream);
// prefill on tcgen05 (G <= 4 or a multiple of 4, d in {64, 128}, tile 32)
bool prefill_attn_tc_supported(const AttnArgs& a);
cudaError_t launch_prefill_attn_tc(const AttnArgs& a, int num_sms, cudaStream_t stream);

}  // namespace kascade
