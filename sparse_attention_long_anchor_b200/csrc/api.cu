// C ABI of the Kascade library: argument checks, workspace layout and kernel
// launches.  Declarations and the calling contract are in include/kascade.h.
#include <stdint.h>
#include <string.h>

#include "../../include/kascade.h"
#include "common.cuh"
#include "kernels.h"

namespace kascade {
namespace {

// Grids and workspace sizes are planned for the 148 SMs of a B200; other
// parts run the same grids in more or fewer waves.
constexpr int kPlanSMs = 148;
constexpr size_t kAlign = 256;

size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

bool aligned(const void* p, size_t a) { return ((uintptr_t)p % a) == 0; }

int check_shape(const kascade_shape* s) {
  if (!s) return KASCADE_ERR_INVALID_ARG;
  if (s->batch < 1 || s->num_q_heads < 1 || s->num_kv_heads < 1 || s->kv_len < 1 || s->q_len < 1)
    return KASCADE_ERR_INVALID_ARG;
  if (s->num_q_heads % s->num_kv_heads != 0) return KASCADE_ERR_INVALID_ARG;
  if (s->topk_num < 1 || s->topk_den < 1 || s->topk_num > s->topk_den) return KASCADE_ERR_INVALID_ARG;
  if (s->head_dim != 64 && s->head_dim != 128) return KASCADE_ERR_UNSUPPORTED;
  if (s->num_q_heads / s->num_kv_heads > 8) return KASCADE_ERR_UNSUPPORTED;
  if (s->kv_len > (1 << 20)) return KASCADE_ERR_UNSUPPORTED;
  if (s->topk_den > (1 << 20)) return KASCADE_ERR_UNSUPPORTED;
  // prefill: the query rows are the last q_len positions of the context (a
  // rolling chunk when q_len < kv_len), starting on a tile boundary
  if (s->q_len > s->kv_len || (s->q_len != 1 && (s->kv_len - s->q_len) % 32 != 0)) return KASCADE_ERR_UNSUPPORTED;
  if (s->q_len != 1 && s->tile != 32) return KASCADE_ERR_UNSUPPORTED;
  if (s->flags & ~(KASCADE_FLAG_PDL | KASCADE_FLAG_INPUTS_STABLE | KASCADE_FLAG_CHECK_INDICES |
                   KASCADE_FLAG_TEST_DROP_LOAD))
    return KASCADE_ERR_INVALID_ARG;
  if (s->select_mode < KASCADE_SELECT_GQA || s->select_mode > KASCADE_SELECT_ALL_HEADS) return KASCADE_ERR_INVALID_ARG;
  if (s->select_mode == KASCADE_SELECT_ALL_HEADS && s->num_q_heads > 64) return KASCADE_ERR_UNSUPPORTED;
  if (s->dtype != KASCADE_DTYPE_BF16 && s->dtype != KASCADE_DTYPE_F32 && s->dtype != KASCADE_DTYPE_F16)
    return KASCADE_ERR_UNSUPPORTED;
  return KASCADE_OK;
}

// Problems per batch row (= index lists per row) and query heads per
// problem of the selection (see kv_slab_of).
int n_lists(const kascade_shape* s) {
  switch (s->select_mode) {
    case KASCADE_SELECT_PER_HEAD: return s->num_q_heads;
    case KASCADE_SELECT_ALL_HEADS: return 1;
    default: return s->num_kv_heads;
  }
}
int sel_heads(const kascade_shape* s) { return s->num_q_heads / n_lists(s); }

bool is_decode(const kascade_shape* s) { return s->q_len == 1; }
// prefill: first query position and first query tile of the call
int q_first(const kascade_shape* s) { return is_decode(s) ? 0 : s->kv_len - s->q_len; }
int t_first(const kascade_shape* s) { return q_first(s) / 32; }
// fp32 and fp16 inputs run the CUDA-core path (is_f32: either of them)
bool is_f32(const kascade_shape* s) { return s->dtype == KASCADE_DTYPE_F32 || s->dtype == KASCADE_DTYPE_F16; }
bool is_f16(const kascade_shape* s) { return s->dtype == KASCADE_DTYPE_F16; }
int n_tiles(const kascade_shape* s) { return (s->kv_len + 31) / 32; }

int64_t prefill_row_len(const kascade_shape* s) {
  return chunk_row_len(s->kv_len, t_first(s), 32, s->topk_num, s->topk_den);
}

int64_t pooled_row_len(const kascade_shape* s) { return chunk_pooled_len(s->kv_len, t_first(s), 32); }

// ----------------------------------------------------------------- workspace plans

struct Carver {
  char* base;
  size_t off = 0;
  template <class T>
  T* take(size_t count) {
    T* p = base ? reinterpret_cast<T*>(base + off) : nullptr;
    off = align_up(off + count * sizeof(T));
    return p;
  }
};

struct SelectPlan {
  float* s2;
  float* m_part;
  double* l_part;
  int splits;
  float* row_m2;
  double* row_l;
  float* pooled;
  float* pooled_all;
  float* v_scratch;
  int32_t* band_idx;
  double* band_val;
  uint8_t* state;
  int grid;
  bool cluster;
  size_t bytes;
};

// Every workspace starts with a 256-byte header whose first int is the
// device error word (set when a bounded wait in a kernel gives up).
constexpr size_t kHeader = 256;

SelectPlan plan_select(const kascade_shape* s, void* ws, bool one_cta = false) {
  SelectPlan p{};
  Carver cv{static_cast<char*>(ws)};
  cv.take<char>(kHeader);
  const size_t B = s->batch, Hq = s->num_q_heads, Hkv = s->num_kv_heads, N = s->kv_len;
  const int n_max = s->kv_len;
  if (is_decode(s)) {
    p.splits = (s->kv_len + decode_score_keys_per_split() - 1) / decode_score_keys_per_split();
    p.s2 = cv.take<float>(B * Hq * N);
    p.m_part = cv.take<float>(B * Hq * p.splits);
    p.l_part = cv.take<double>(B * Hq * p.splits);
    if (!one_cta && s->select_mode != KASCADE_SELECT_ALL_HEADS && !is_f32(s) && select_decode_cluster_ok(s->kv_len)) {
      p.cluster = true;
      const size_t entries = select_decode_cluster_scratch(s->batch, n_lists(s), s->kv_len);
      p.band_idx = cv.take<int32_t>(entries);
      p.band_val = cv.take<double>(entries);
      p.bytes = cv.off;
      return p;
    }
    p.grid = select_grid(false, (int)(B * n_lists(s)), kPlanSMs);
    p.v_scratch = cv.take<float>((size_t)p.grid * n_max);
  } else {
    const size_t Lq = s->q_len;   // row statistics of the call's query rows
    p.row_m2 = cv.take<float>(B * Hq * Lq);
    p.row_l = cv.take<double>(B * Hq * Lq);
    // scoring writes one pooled row per kv head (per query head in the
    // per-head mode); the all-heads mode adds their mean per batch row
    const size_t score_rows = s->select_mode == KASCADE_SELECT_PER_HEAD ? Hq : Hkv;
    p.pooled = cv.take<float>(B * score_rows * (size_t)pooled_row_len(s));
    p.pooled_all = s->select_mode == KASCADE_SELECT_ALL_HEADS ? cv.take<float>(B * (size_t)pooled_row_len(s)) : nullptr;
    const int64_t problems = (int64_t)B * n_lists(s) * (n_tiles(s) - t_first(s));
    p.grid = select_grid(true, (int)(problems < (1 << 30) ? problems : (1 << 30)), kPlanSMs);
    p.v_scratch = nullptr;
  }
  p.band_idx = cv.take<int32_t>((size_t)p.grid * n_max);
  p.band_val = cv.take<double>((size_t)p.grid * n_max);
  p.state = cv.take<uint8_t>((size_t)p.grid * n_max);
  p.bytes = cv.off;
  return p;
}

// Proposal-refine selection (decode): scores of the pool's keys, split
// statistics, and the one-CTA-per-problem Top-k over the pool.
SelectPlan plan_refine(const kascade_shape* s, int pool_len, void* ws) {
  SelectPlan p{};
  Carver cv{static_cast<char*>(ws)};
  cv.take<char>(kHeader);
  const size_t B = s->batch, Hq = s->num_q_heads, Hkv = s->num_kv_heads, n = pool_len;
  p.splits = (pool_len + decode_score_keys_per_split() - 1) / decode_score_keys_per_split();
  p.s2 = cv.take<float>(B * Hq * n);
  p.m_part = cv.take<float>(B * Hq * p.splits);
  p.l_part = cv.take<double>(B * Hq * p.splits);
  p.grid = select_grid(false, (int)(B * Hkv), kPlanSMs);
  p.v_scratch = cv.take<float>((size_t)p.grid * n);
  p.band_idx = cv.take<int32_t>((size_t)p.grid * n);
  p.band_val = cv.take<double>((size_t)p.grid * n);
  p.state = cv.take<uint8_t>((size_t)p.grid * n);
  p.bytes = cv.off;
  return p;
}

int device_sms() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
      n <= 0)
    return kPlanSMs;
  return n;
}

// sparse / dense prefill: the tcgen05 kernel where it applies, else the
// warp-MMA kernel
cudaError_t launch_prefill(const AttnArgs& a, cudaStream_t st) {
  return prefill_attn_tc_supported(a) ? launch_prefill_attn_tc(a, device_sms(), st) : launch_prefill_attn(a, st);
}

int* err_word(void* ws, size_t ws_bytes) {
  return (ws && ws_bytes >= sizeof(int) && aligned(ws, 4)) ? static_cast<int*>(ws) : nullptr;
}

int cuda_status(cudaError_t e) { return e == cudaSuccess ? KASCADE_OK : KASCADE_ERR_CUDA; }

int check_ws(void* ws, size_t ws_bytes, size_t need) {
  if (need == 0) return KASCADE_OK;
  if (!ws || !aligned(ws, kAlign) || ws_bytes < need) return KASCADE_ERR_WORKSPACE;
  return KASCADE_OK;
}

int check_tensors(const void* q, const void* k, const void* v, const void* o) {
  if (!q || !k || !o) return KASCADE_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(o, 16) || (v && !aligned(v, 16)))
    return KASCADE_ERR_UNSUPPORTED;
  return KASCADE_OK;
}

// ----------------------------------------------------------------- index checks

bool checking(const kascade_shape* s) { return (s->flags & KASCADE_FLAG_CHECK_INDICES) != 0; }

int64_t index_entries(const kascade_shape* s) {
  const int64_t BH = (int64_t)s->batch * n_lists(s);
  return is_decode(s) ? BH * topk_count(s->kv_len, s->topk_num, s->topk_den) : BH * prefill_row_len(s);
}

// the checked copies (index rows, head_map, kv_lens) carved at `offset`
struct CheckPlan {
  int32_t* idx;
  int32_t* hm;
  int32_t* kv;
  size_t bytes;   // offset + the copies
};
CheckPlan plan_check(const kascade_shape* s, int64_t entries, size_t offset, void* ws) {
  CheckPlan p{};
  Carver cv{static_cast<char*>(ws), offset};
  p.idx = cv.take<int32_t>((size_t)entries);
  p.hm = cv.take<int32_t>((size_t)s->num_q_heads);
  p.kv = cv.take<int32_t>((size_t)s->batch);
  p.bytes = cv.off;
  return p;
}

// Runs the checking kernel and points idx / head_map / kv_lens at the
// copies.  rows: B * lists rows of row_len entries.
int run_check(const kascade_shape* s, int lists, int64_t row_len, bool pool, const int32_t*& idx,
              const int32_t*& head_map, const int32_t*& kv_lens, void* ws, size_t ws_bytes, size_t offset,
              cudaStream_t st) {
  const CheckPlan need = plan_check(s, (int64_t)s->batch * lists * row_len, offset, nullptr);
  if (!ws || !aligned(ws, kAlign) || ws_bytes < need.bytes) return KASCADE_ERR_WORKSPACE;
  const CheckPlan pl = plan_check(s, (int64_t)s->batch * lists * row_len, offset, ws);
  CheckArgs c{};
  c.idx = idx;
  c.idx_out = pl.idx;
  c.head_map = head_map;
  c.hm_out = pl.hm;
  c.n_map = head_map ? lists : 0;
  c.kv_lens = kv_lens;
  c.kv_out = pl.kv;
  c.B = s->batch;
  c.L = lists;
  c.N = s->kv_len;
  c.num = s->topk_num;
  c.den = s->topk_den;
  c.t0 = t_first(s);
  c.row_len = row_len;
  c.prefill = !is_decode(s);
  c.pool = pool;
  c.pdl = (s->flags & KASCADE_FLAG_PDL) != 0;
  c.err = static_cast<int*>(ws);
  const int rc = cuda_status(launch_check_lists(c, st));
  if (rc) return rc;
  idx = pl.idx;
  if (head_map) head_map = pl.hm;
  if (kv_lens) kv_lens = pl.kv;
  return KASCADE_OK;
}

// KASCADE_FLAG_CHECK_INDICES for an attention call: checked copies of the
// lists (none for the dense form), head_map and kv_lens
int check_attn_inputs(const kascade_shape* s, AttnArgs& a, void* ws, size_t ws_bytes, cudaStream_t st) {
  if (!checking(s)) return KASCADE_OK;
  const int64_t row_len =
      !a.idx ? 0 : is_decode(s) ? topk_count(s->kv_len, s->topk_num, s->topk_den) : prefill_row_len(s);
  const int32_t* hm = a.one_list ? nullptr : a.head_map;   // all heads pooled: one list, no map
  const int rc = run_check(s, n_lists(s), row_len, false, a.idx, hm, a.kv_lens, ws, ws_bytes, kHeader, st);
  if (rc) return rc;
  if (!a.one_list) a.head_map = hm;
  a.flags &= ~KASCADE_FLAG_INPUTS_STABLE;   // the copies are written just before
  return KASCADE_OK;
}

AttnArgs attn_args(const kascade_shape* s, const void* q, const void* k, const void* v,
                   const int32_t* idx, const int32_t* head_map, void* o, float* lse) {
  AttnArgs a{};
  a.q = static_cast<const __nv_bfloat16*>(q);
  a.k = static_cast<const __nv_bfloat16*>(k);
  a.v = static_cast<const __nv_bfloat16*>(v);
  a.idx = idx;
  a.head_map = head_map;
  a.o = static_cast<__nv_bfloat16*>(o);
  a.lse = lse;
  a.B = s->batch;
  a.Hq = s->num_q_heads;
  a.Hkv = s->num_kv_heads;
  a.G = a.Hq / a.Hkv;
  a.D = s->head_dim;
  a.N = s->kv_len;
  a.tile = 32;
  a.num = s->topk_num;
  a.den = s->topk_den;
  a.flags = s->flags;
  a.Gkv = a.G;
  a.Hp = a.Hkv;
  a.q0 = q_first(s);
  a.Lq = s->q_len;
  a.n_lists = n_lists(s);
  a.one_list = false;
  if (idx && s->select_mode == KASCADE_SELECT_PER_HEAD) {   // one problem per query head
    a.Hp = a.Hq;
    a.G = 1;
  } else if (idx && s->select_mode == KASCADE_SELECT_ALL_HEADS) {
    a.one_list = true;   // every kv head reads the row's single list
  }
  return a;
}

}  // namespace
}  // namespace kascade

using namespace kascade;

extern "C" {

size_t kascade_workspace_bytes(const kascade_shape* s, int op) {
  if (check_shape(s)) return 0;
  switch (op) {
    case KASCADE_OP_SELECT:
      return plan_select(s, nullptr).bytes;
    case KASCADE_OP_SPARSE_DECODE:
    case KASCADE_OP_SPARSE_PREFILL:
      // only the error word (partial results stay on chip), plus the checked
      // index copies with KASCADE_FLAG_CHECK_INDICES
      return checking(s) ? plan_check(s, index_entries(s), kHeader, nullptr).bytes : kHeader;
    case KASCADE_OP_DENSE:
      return kHeader;
    case KASCADE_OP_REFINE: {   // covers every pool length up to N
      if (!is_decode(s)) return 0;
      const size_t b = plan_refine(s, s->kv_len, nullptr).bytes;
      return checking(s) ? plan_check(s, (int64_t)s->batch * s->num_kv_heads * s->kv_len, b, nullptr).bytes : b;
    }
    case KASCADE_OP_SELECT_VARLEN:
      return is_decode(s) ? plan_select(s, nullptr, true).bytes : 0;
    default:
      return 0;
  }
}

int64_t kascade_index_count(const kascade_shape* s) {
  if (check_shape(s)) return -1;
  const int64_t BH = (int64_t)s->batch * n_lists(s);
  if (is_decode(s)) return BH * topk_count(s->kv_len, s->topk_num, s->topk_den);
  return BH * prefill_row_len(s);
}

int kascade_index_offsets(const kascade_shape* s, int64_t* offsets) {
  int rc = check_shape(s);
  if (rc) return rc;
  if (!offsets) return KASCADE_ERR_INVALID_ARG;
  if (is_decode(s)) {
    offsets[0] = 0;
    offsets[1] = topk_count(s->kv_len, s->topk_num, s->topk_den);
    return KASCADE_OK;
  }
  const int T = n_tiles(s), t0 = t_first(s);
  for (int t = t0; t < T; ++t) offsets[t - t0] = chunk_list_offset(t, t0, 32, s->topk_num, s->topk_den);
  offsets[T - t0] = prefill_row_len(s);
  return KASCADE_OK;
}

int kascade_launch_count(const kascade_shape* s, int op) {
  if (check_shape(s)) return -1;
  if (op == KASCADE_OP_DENSE) return 1;
  if (op == KASCADE_OP_SPARSE_DECODE || op == KASCADE_OP_SPARSE_PREFILL) return checking(s) ? 2 : 1;
  if (op != KASCADE_OP_SELECT) return -1;
  if (!is_decode(s)) return s->select_mode == KASCADE_SELECT_ALL_HEADS ? 3 : 2;
  if (s->select_mode == KASCADE_SELECT_ALL_HEADS || is_f32(s) || !select_decode_cluster_ok(s->kv_len)) return 2;
  SelArgs a{};
  a.B = s->batch;
  a.Hq = s->num_q_heads;
  a.Hkv = s->num_kv_heads;
  a.Hp = n_lists(s);
  a.G = sel_heads(s);
  a.Gkv = a.Hq / a.Hkv;
  a.D = s->head_dim;
  a.N = s->kv_len;
  return anchor_select_fused_ok(a) ? 1 : 2;
}

int kascade_workspace_init(void* ws, size_t ws_bytes, void* stream) {
  if (!ws && ws_bytes) return KASCADE_ERR_WORKSPACE;
  if (!ws_bytes) return KASCADE_OK;
  return cuda_status(cudaMemsetAsync(ws, 0, ws_bytes, static_cast<cudaStream_t>(stream)));
}

int kascade_select(const kascade_shape* s, const void* q, const void* k, int32_t* idx, void* ws,
                   size_t ws_bytes, void* stream) {
  int rc = check_shape(s);
  if (rc) return rc;
  if (!q || !k || !idx) return KASCADE_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(idx, 4)) return KASCADE_ERR_UNSUPPORTED;
  SelectPlan pl = plan_select(s, nullptr);
  rc = check_ws(ws, ws_bytes, pl.bytes);
  if (rc) return rc;
  pl = plan_select(s, ws);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  SelArgs a{};
  a.prefill = !is_decode(s);
  a.B = s->batch;
  a.Hq = s->num_q_heads;
  a.Hkv = s->num_kv_heads;
  a.Hp = n_lists(s);
  a.G = sel_heads(s);
  a.Gkv = a.Hq / a.Hkv;
  a.D = s->head_dim;
  a.N = s->kv_len;
  a.q0 = q_first(s);
  a.Lq = s->q_len;
  a.tile = 32;
  a.num = s->topk_num;
  a.den = s->topk_den;
  a.q = static_cast<const __nv_bfloat16*>(q);
  a.k = static_cast<const __nv_bfloat16*>(k);
  a.v_scratch = pl.v_scratch;
  a.band_idx = pl.band_idx;
  a.band_val = pl.band_val;
  a.state = pl.state;
  a.n_max = s->kv_len;
  a.grid = pl.grid;
  a.idx = idx;
  a.flags = s->flags & KASCADE_FLAG_PDL;
  a.err = err_word(ws, ws_bytes);
  a.in_type = s->dtype;
  const int test_flags = s->flags & KASCADE_FLAG_TEST_DROP_LOAD;
  if (is_decode(s)) {
    if (pl.cluster && anchor_select_fused_ok(a)) return cuda_status(launch_anchor_select_fused(a, st));
    DecodeScoreArgs d{};
    d.flags = a.flags;
    d.q = a.q;
    d.k = a.k;
    d.s2 = pl.s2;
    d.m_part = pl.m_part;
    d.l_part = pl.l_part;
    d.B = a.B;
    d.Hq = a.Hq;
    d.Hkv = a.Hkv;
    d.G = a.Gkv;   // scoring runs per kv head over its query heads
    d.D = a.D;
    d.N = a.N;
    rc = cuda_status(is_f32(s) ? launch_decode_score_f32(d, is_f16(s), st) : launch_decode_score(d, st));
    if (rc) return rc;
    a.s2 = pl.s2;
    a.m_part = pl.m_part;
    a.l_part = pl.l_part;
    a.splits = pl.splits;
    if (pl.cluster) return cuda_status(launch_select_decode_cluster(a, st));
  } else {
    ScorePoolArgs sp{};
    sp.flags = a.flags | test_flags;
    sp.q = a.q;
    sp.k = a.k;
    sp.row_m2 = pl.row_m2;
    sp.row_l = pl.row_l;
    sp.pooled = pl.pooled;
    sp.B = a.B;
    sp.Hq = a.Hq;
    sp.Hkv = a.Hkv;
    sp.G = a.Gkv;   // scoring runs per kv head over its query heads
    sp.D = a.D;
    sp.N = a.N;
    sp.q0 = a.q0;
    sp.Lq = a.Lq;
    sp.tile = 32;
    sp.per_head = s->select_mode == KASCADE_SELECT_PER_HEAD;
    rc = cuda_status(is_f32(s) ? launch_score_pool_f32(sp, is_f16(s), st)
                     : score_pool_tc_supported(sp) ? launch_score_pool_tc(sp, err_word(ws, ws_bytes), device_sms(), st)
                                                   : launch_score_pool(sp, st));
    if (rc) return rc;
    a.pooled = pl.pooled;
    if (s->select_mode == KASCADE_SELECT_ALL_HEADS) {
      rc = cuda_status(launch_pool_mean(pl.pooled, pl.pooled_all, a.B, a.Hkv, pooled_row_len(s), a.flags, st));
      if (rc) return rc;
      a.pooled = pl.pooled_all;
    }
    a.row_m2 = pl.row_m2;
    a.row_l = pl.row_l;
  }
  return cuda_status(launch_select(a, st));
}

int kascade_refine_select(const kascade_shape* s, const void* q, const void* k, const int32_t* pool,
                          int32_t pool_len, const int32_t* head_map, int32_t* idx, void* ws, size_t ws_bytes,
                          void* stream) {
  int rc = check_shape(s);
  if (rc) return rc;
  if (!is_decode(s) || s->select_mode != KASCADE_SELECT_GQA) return KASCADE_ERR_UNSUPPORTED;
  if (!q || !k || !pool || !idx) return KASCADE_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(idx, 4) || !aligned(pool, 4) ||
      (head_map && !aligned(head_map, 4)))
    return KASCADE_ERR_UNSUPPORTED;
  const int kk = topk_count(s->kv_len, s->topk_num, s->topk_den);
  if (pool_len < kk || pool_len > s->kv_len) return KASCADE_ERR_INVALID_ARG;
  SelectPlan pl = plan_refine(s, pool_len, nullptr);
  rc = check_ws(ws, ws_bytes, pl.bytes);
  if (rc) return rc;
  pl = plan_refine(s, pool_len, ws);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int flags = s->flags & KASCADE_FLAG_PDL;
  if (checking(s)) {
    const int32_t* no_lens = nullptr;
    rc = run_check(s, s->num_kv_heads, pool_len, true, pool, head_map, no_lens, ws, ws_bytes, pl.bytes, st);
    if (rc) return rc;
  }
  DecodeScoreArgs d{};
  d.flags = flags;
  d.q = static_cast<const __nv_bfloat16*>(q);
  d.k = static_cast<const __nv_bfloat16*>(k);
  d.s2 = pl.s2;
  d.m_part = pl.m_part;
  d.l_part = pl.l_part;
  d.B = s->batch;
  d.Hq = s->num_q_heads;
  d.Hkv = s->num_kv_heads;
  d.G = d.Hq / d.Hkv;
  d.D = s->head_dim;
  d.N = pool_len;
  d.cand = pool;
  d.cand_map = head_map;
  d.cand_lists = s->num_kv_heads;
  d.n_ctx = s->kv_len;
  rc = cuda_status(is_f32(s) ? launch_decode_score_f32(d, is_f16(s), st) : launch_decode_score(d, st));
  if (rc) return rc;
  SelArgs a{};
  a.prefill = false;
  a.B = d.B;
  a.Hq = d.Hq;
  a.Hkv = d.Hkv;
  a.Hp = d.Hkv;
  a.G = d.G;
  a.Gkv = d.G;
  a.D = d.D;
  a.N = pool_len;
  a.n_ctx = s->kv_len;
  a.cand = pool;
  a.cand_map = head_map;
  a.cand_lists = s->num_kv_heads;
  a.tile = 32;
  a.num = s->topk_num;
  a.den = s->topk_den;
  a.q = d.q;
  a.k = d.k;
  a.s2 = pl.s2;
  a.m_part = pl.m_part;
  a.l_part = pl.l_part;
  a.splits = pl.splits;
  a.v_scratch = pl.v_scratch;
  a.band_idx = pl.band_idx;
  a.band_val = pl.band_val;
  a.state = pl.state;
  a.n_max = pool_len;
  a.grid = pl.grid;
  a.idx = idx;
  a.flags = flags;
  a.err = err_word(ws, ws_bytes);
  a.in_type = s->dtype;
  return cuda_status(launch_select(a, st));
}

int kascade_sparse_decode(const kascade_shape* s, const void* q, const void* k, const void* v,
                          const int32_t* idx, const int32_t* head_map, void* o, float* lse, void* ws,
                          size_t ws_bytes, void* stream) {
  int rc = check_shape(s);
  if (rc) return rc;
  if (!is_decode(s)) return KASCADE_ERR_UNSUPPORTED;
  if (!v || !idx) return KASCADE_ERR_INVALID_ARG;
  rc = check_tensors(q, k, v, o);
  if (rc) return rc;
  if (!aligned(idx, 4) || (head_map && !aligned(head_map, 4)) || (lse && !aligned(lse, 4)))
    return KASCADE_ERR_UNSUPPORTED;
  AttnArgs a = attn_args(s, q, k, v, idx, head_map, o, lse);
  a.err = err_word(ws, ws_bytes);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  rc = check_attn_inputs(s, a, ws, ws_bytes, st);
  if (rc) return rc;
  if (is_f32(s)) return cuda_status(launch_sparse_decode_f32(a, is_f16(s), st));
  return cuda_status(launch_decode_attn(a, st));
}

int kascade_select_varlen(const kascade_shape* s, const void* q, const void* k, const int32_t* kv_lens,
                          int32_t* idx, void* ws, size_t ws_bytes, void* stream) {
  int rc = check_shape(s);
  if (rc) return rc;
  if (!is_decode(s) || s->dtype != KASCADE_DTYPE_BF16) return KASCADE_ERR_UNSUPPORTED;
  if (!q || !k || !kv_lens || !idx) return KASCADE_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(idx, 4) || !aligned(kv_lens, 4)) return KASCADE_ERR_UNSUPPORTED;
  SelectPlan pl = plan_select(s, nullptr, true);
  rc = check_ws(ws, ws_bytes, pl.bytes);
  if (rc) return rc;
  pl = plan_select(s, ws, true);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int flags = s->flags & KASCADE_FLAG_PDL;
  DecodeScoreArgs d{};
  d.flags = flags;
  d.q = static_cast<const __nv_bfloat16*>(q);
  d.k = static_cast<const __nv_bfloat16*>(k);
  d.s2 = pl.s2;
  d.m_part = pl.m_part;
  d.l_part = pl.l_part;
  d.B = s->batch;
  d.Hq = s->num_q_heads;
  d.Hkv = s->num_kv_heads;
  d.G = d.Hq / d.Hkv;
  d.D = s->head_dim;
  d.N = s->kv_len;
  d.kv_lens = kv_lens;
  rc = cuda_status(launch_decode_score(d, st));
  if (rc) return rc;
  SelArgs a{};
  a.prefill = false;
  a.B = d.B;
  a.Hq = d.Hq;
  a.Hkv = d.Hkv;
  a.Hp = n_lists(s);
  a.G = sel_heads(s);
  a.Gkv = d.G;
  a.D = d.D;
  a.N = d.N;
  a.kv_lens = kv_lens;
  a.tile = 32;
  a.num = s->topk_num;
  a.den = s->topk_den;
  a.q = d.q;
  a.k = d.k;
  a.s2 = pl.s2;
  a.m_part = pl.m_part;
  a.l_part = pl.l_part;
  a.splits = pl.splits;
  a.v_scratch = pl.v_scratch;
  a.band_idx = pl.band_idx;
  a.band_val = pl.band_val;
  a.state = pl.state;
  a.n_max = s->kv_len;
  a.grid = pl.grid;
  a.idx = idx;
  a.flags = flags;
  a.err = err_word(ws, ws_bytes);
  return cuda_status(launch_select(a, st));
}

int kascade_sparse_decode_varlen(const kascade_shape* s, const void* q, const void* k, const void* v,
                                 const int32_t* kv_lens, const int32_t* idx, const int32_t* head_map, void* o,
                                 float* lse, void* ws, size_t ws_bytes, void* stream) {
  int rc = check_shape(s);
  if (rc) return rc;
  if (!is_decode(s) || s->dtype != KASCADE_DTYPE_BF16) return KASCADE_ERR_UNSUPPORTED;
  if (!v || !kv_lens) return KASCADE_ERR_INVALID_ARG;
  rc = check_tensors(q, k, v, o);
  if (rc) return rc;
  if (!aligned(kv_lens, 4) || (idx && !aligned(idx, 4)) || (head_map && !aligned(head_map, 4)) ||
      (lse && !aligned(lse, 4)))
    return KASCADE_ERR_UNSUPPORTED;
  AttnArgs a = attn_args(s, q, k, v, idx, head_map, o, lse);
  a.err = err_word(ws, ws_bytes);
  a.kv_lens = kv_lens;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  rc = check_attn_inputs(s, a, ws, ws_bytes, st);
  if (rc) return rc;
  return cuda_status(launch_decode_attn(a, st));
}

int kascade_sparse_decode_paged(const kascade_shape* s, const void* q, const void* k_pages, const void* v_pages,
                                const int32_t* page_table, int32_t page_size, int32_t max_pages, const int32_t* idx,
                                const int32_t* head_map, void* o, float* lse, void* ws, size_t ws_bytes,
                                void* stream) {
  int rc = check_shape(s);
  if (rc) return rc;
  if (!is_decode(s) || s->dtype != KASCADE_DTYPE_BF16) return KASCADE_ERR_UNSUPPORTED;
  if (!v_pages || !page_table) return KASCADE_ERR_INVALID_ARG;
  rc = check_tensors(q, k_pages, v_pages, o);
  if (rc) return rc;
  if (page_size < 16 || page_size > (1 << 20) || (page_size & (page_size - 1)) != 0) return KASCADE_ERR_UNSUPPORTED;
  if (max_pages < (s->kv_len + page_size - 1) / page_size) return KASCADE_ERR_INVALID_ARG;
  if (!aligned(page_table, 4) || (idx && !aligned(idx, 4)) || (head_map && !aligned(head_map, 4)) ||
      (lse && !aligned(lse, 4)))
    return KASCADE_ERR_UNSUPPORTED;
  AttnArgs a = attn_args(s, q, k_pages, v_pages, idx, head_map, o, lse);
  a.err = err_word(ws, ws_bytes);
  a.page_table = page_table;
  a.page_size = page_size;
  a.max_pages = max_pages;
  int sh = 0;
  while ((1 << sh) < page_size) ++sh;
  a.page_shift = sh;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  rc = check_attn_inputs(s, a, ws, ws_bytes, st);
  if (rc) return rc;
  return cuda_status(launch_decode_attn(a, st));
}

int kascade_sparse_prefill(const kascade_shape* s, const void* q, const void* k, const void* v,
                           const int32_t* idx, const int32_t* head_map, void* o, float* lse, void* ws,
                           size_t ws_bytes, void* stream) {
  int rc = check_shape(s);
  if (rc) return rc;
  // N = 1 is both a decode and a prefill shape; both index layouts coincide there
  if (is_decode(s) && s->kv_len != 1) return KASCADE_ERR_UNSUPPORTED;
  if (!v || !idx) return KASCADE_ERR_INVALID_ARG;
  rc = check_tensors(q, k, v, o);
  if (rc) return rc;
  if (!aligned(idx, 4) || (head_map && !aligned(head_map, 4)) || (lse && !aligned(lse, 4)))
    return KASCADE_ERR_UNSUPPORTED;
  AttnArgs a = attn_args(s, q, k, v, idx, head_map, o, lse);
  a.err = err_word(ws, ws_bytes);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  rc = check_attn_inputs(s, a, ws, ws_bytes, st);
  if (rc) return rc;
  if (is_f32(s)) return cuda_status(launch_sparse_prefill_f32(a, is_f16(s), st));
  return cuda_status(launch_prefill(a, st));
}

int kascade_dense_ref(const kascade_shape* s, const void* q, const void* k, const void* v, int causal,
                      void* o, float* lse, void* ws, size_t ws_bytes, void* stream) {
  int rc = check_shape(s);
  if (rc) return rc;
  if (!v) return KASCADE_ERR_INVALID_ARG;
  rc = check_tensors(q, k, v, o);
  if (rc) return rc;
  if (lse && !aligned(lse, 4)) return KASCADE_ERR_UNSUPPORTED;
  AttnArgs a = attn_args(s, q, k, v, nullptr, nullptr, o, lse);
  a.err = err_word(ws, ws_bytes);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (is_decode(s)) {
    if (is_f32(s)) return cuda_status(launch_sparse_decode_f32(a, is_f16(s), st));
    return cuda_status(launch_decode_attn(a, st));
  }
  a.causal = causal != 0;
  if (is_f32(s)) return cuda_status(launch_sparse_prefill_f32(a, is_f16(s), st));
  return cuda_status(launch_prefill(a, st));
}

int kascade_workspace_error(const void* ws, int* error_out, int clear, void* stream) {
  if (!ws || !error_out) return KASCADE_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int host = 0;
  cudaError_t e = cudaMemcpyAsync(&host, ws, sizeof(int), cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e == cudaSuccess && clear && host) e = cudaMemsetAsync(const_cast<void*>(ws), 0, sizeof(int), st);
  if (e != cudaSuccess) return KASCADE_ERR_CUDA;
  *error_out = host;
  return KASCADE_OK;
}

const char* kascade_status_str(int status) {
  switch (status) {
    case KASCADE_OK:
      return "ok";
    case KASCADE_ERR_INVALID_ARG:
      return "invalid argument";
    case KASCADE_ERR_UNSUPPORTED:
      return "unsupported shape, alignment or option";
    case KASCADE_ERR_WORKSPACE:
      return "workspace missing, misaligned or too small";
    case KASCADE_ERR_CUDA:
      return "CUDA launch or device error";
    case KASCADE_ERR_TOO_LARGE:
      return "shape needs more scratch than the library's fixed buffer holds";
    default:
      return "unknown status";
  }
}

}  // extern "C"
