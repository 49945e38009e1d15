// Internal launch interface between the C ABI layer (api.cu) and the kernels.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace kascade {

struct DecodeScoreArgs {
  const __nv_bfloat16* q;  // [B, Hq, 1, D]
  const __nv_bfloat16* k;  // [B, Hkv, N, D]
  float* s2;               // [B, Hq, N]      scores * log2(e)/sqrt(D)
  float* m_part;           // [B, Hq, splits]
  double* l_part;          // [B, Hq, splits]
  int B, Hq, Hkv, G, D, N;
  int flags;
};
int decode_score_keys_per_split();
cudaError_t launch_decode_score(const DecodeScoreArgs& a, cudaStream_t stream);

// Top-k selection over pooled post-softmax scores (decode or prefill).
struct SelArgs {
  bool prefill;
  int B, Hq, Hkv, G, D, N, tile, num, den;
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
size_t select_decode_cluster_scratch(int B, int Hkv, int N);   // band entries
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
  float* pooled;           // [B, Hkv, sum_t e_t]
  int B, Hq, Hkv, G, D, N, tile;
  int flags;
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
  bool causal;               // prefill dense only
  int* err;                  // device error word (a bounded wait gave up), may be NULL
  int flags;                 // KASCADE_FLAG_* bits
};
// decode: one 16-CTA cluster per (batch, kv head), merge over DSMEM
cudaError_t launch_decode_attn(const AttnArgs& a, cudaStream_t stream);
cudaError_t launch_prefill_attn(const AttnArgs& a, cudaStream_t stream);
// prefill on tcgen05 (G <= 4 or a multiple of 4, d in {64, 128}, tile 32)
bool prefill_attn_tc_supported(const AttnArgs& a);
cudaError_t launch_prefill_attn_tc(const AttnArgs& a, int num_sms, cudaStream_t stream);

}  // namespace kascade
