// Host side of the libqi21 C ABI (include/qi21.h): argument validation,
// workspace carving, and the kernel sequence of each entry point.
#include <stdarg.h>
#include <stdio.h>
#include <stdlib.h>
#include <stdint.h>
#include <string.h>

#include "../../include/qi21.h"
#include "qi21_internal.h"

namespace qi21 {

static thread_local char g_last_error[512] = "";
static thread_local uint64_t g_launches = 0;

void note_launch() { ++g_launches; }

static qi21_status fail(qi21_status s, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_last_error, sizeof(g_last_error), fmt, ap);
  va_end(ap);
  return s;
}

qi21_status report_error(qi21_status s, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_last_error, sizeof(g_last_error), fmt, ap);
  va_end(ap);
  return s;
}

static qi21_status cuda_fail(cudaError_t e, const char* what) {
  return fail(QI21_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

static bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

static size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

static size_t elem_bytes(qi21_dtype dt) { return dt == QI21_F32 ? 4 : 2; }

// Workspace: [header][cos/sin table: table_rows x 64 float2][rotated K: B x H x k_rows x 128]
// (the query rows need the table; the key rows not stored in a cache need the
// rotated-K room)
struct WsLayout {
  size_t table_off, k_off, total;
};
static WsLayout ws_layout(int64_t B, int64_t H, int64_t table_rows, int64_t k_rows, qi21_dtype dt) {
  WsLayout w;
  w.table_off = QI21_WORKSPACE_HEADER_BYTES;
  w.k_off = round_up(w.table_off + (size_t)table_rows * kPairs * sizeof(float2), 256);
  w.total = round_up(w.k_off + (size_t)B * H * k_rows * kHeadDim * elem_bytes(dt), 256);
  return w;
}

// Tail-split scratch of a cached step (the attention's last, partial wave of
// units split into key-range pieces): arrival counters for up to
// kSplitUnitsCap units, then per piece slot 64 KB of O / l (bf16) and 2 KB of
// (row max, row sum).  Slots: up to four per unit, at most kSplitSlotsCap.
constexpr int64_t kSplitUnitsCap = 512;
constexpr int64_t kSplitSlotsCap = 512;
constexpr size_t kSplitSlotPartBytes = (size_t)2 * 128 * kHeadDim * 2;
constexpr size_t kSplitSlotMlBytes = (size_t)2 * 128 * sizeof(float2);
struct SplitCaps {
  int64_t units, slots;
  size_t cnt_bytes;
};
static SplitCaps split_caps(int64_t B, int64_t H, int64_t T) {
  const int64_t units = B * H * ((T + 255) / 256);
  SplitCaps c;
  c.units = units < kSplitUnitsCap ? units : kSplitUnitsCap;
  c.slots = 4 * units < kSplitSlotsCap ? 4 * units : kSplitSlotsCap;
  c.cnt_bytes = round_up((size_t)c.units * 8 * sizeof(uint32_t), 256);
  return c;
}

// Bytes of the tail-split scratch for a call over `rows` query rows (bf16).
static size_t split_bytes(int64_t B, int64_t H, int64_t rows) {
  const SplitCaps c = split_caps(B, H, rows);
  return c.cnt_bytes + (size_t)c.slots * (kSplitSlotPartBytes + kSplitSlotMlBytes);
}

// Hands the attention the tail-split scratch that the workspace holds past
// its minimum layout (none: the call runs unsplit); the pre-pass zeroes the
// arrival counters.
static void carve_split(AttnArgs& a, RopePrepParams& rp, uint8_t* ws, size_t base, size_t workspace_bytes,
                        int64_t B, int64_t H, int64_t rows) {
  const SplitCaps c = split_caps(B, H, rows);
  const size_t avail = workspace_bytes - base;
  if (avail < c.cnt_bytes + kSplitSlotPartBytes + kSplitSlotMlBytes) return;
  int64_t slots = (int64_t)((avail - c.cnt_bytes) / (kSplitSlotPartBytes + kSplitSlotMlBytes));
  if (slots > c.slots) slots = c.slots;
  a.split_cnt = reinterpret_cast<uint32_t*>(ws + base);
  a.split_cnt_units = (int32_t)c.units;
  a.split_part = ws + base + c.cnt_bytes;
  a.split_ml = ws + base + c.cnt_bytes + (size_t)slots * kSplitSlotPartBytes;
  a.split_slots = (int32_t)slots;
  rp.zero_words = a.split_cnt;
  rp.n_zero_words = (int32_t)(c.units * 8);
}

static int sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 148;
  return n;
}

static qi21_status check_common(int32_t B, int32_t H, qi21_dtype dt) {
  if (B < 0 || H < 0) return fail(QI21_ERR_INVALID_ARG, "B and H must be >= 0 (got %d, %d)", B, H);
  if (dt != QI21_BF16 && dt != QI21_F32) return fail(QI21_ERR_UNSUPPORTED, "unknown dtype %d", (int)dt);
  return QI21_OK;
}

static qi21_status check_ptr(const void* p, const char* name) {
  if (p == nullptr) return fail(QI21_ERR_INVALID_ARG, "%s is NULL", name);
  if (!aligned16(p)) return fail(QI21_ERR_INVALID_ARG, "%s is not 16-byte aligned", name);
  return QI21_OK;
}

#define QI21_TRY(x)                        \
  do {                                     \
    qi21_status _s = (x);                  \
    if (_s != QI21_OK) return _s;          \
  } while (0)

// QK-RMSNorm arguments: both weight vectors or neither; eps finite, >= 0.
static qi21_status check_norm(const float* norm_q, const float* norm_k, float eps) {
  if (norm_q == nullptr && norm_k == nullptr) return QI21_OK;
  QI21_TRY(check_ptr(norm_q, "norm_q"));
  QI21_TRY(check_ptr(norm_k, "norm_k"));
  if (!(eps >= 0.f) || !(eps < 3.0e38f)) return fail(QI21_ERR_INVALID_ARG, "eps must be finite and >= 0");
  return QI21_OK;
}

// Runs the attention kernel that matches the dtype.
static qi21_status run_attention(const AttnArgs& a, qi21_dtype dt, cudaStream_t st) {
  const cudaError_t e =
      dt == QI21_F32 ? launch_attn_simt_f32(a, st) : launch_attn_tc_bf16(a, st, sm_count());
  if (e != cudaSuccess) return cuda_fail(e, "attention launch");
  return QI21_OK;
}

size_t attn_cached_workspace_min(int32_t B, int32_t H, int64_t T, qi21_dtype dt) {
  if (B < 0 || H < 0 || T < 0) return 0;
  return ws_layout(B, H, T, T, dt).total;
}

}  // namespace qi21

using namespace qi21;

extern "C" {

// Position table and visibility bound.  original = the earlier model: text
// positions start after the images (max over images of max(H//2, W//2)) and
// there is no mask.
static qi21_status rope_positions_impl(const qi21_segment* segs, int32_t n_segs, int64_t L, int32_t* pos,
                                       int32_t* kv_end, bool original, void* stream) {
  if (n_segs == 0 && L == 0) return QI21_OK;
  if (segs == nullptr) return fail(QI21_ERR_INVALID_ARG, "segs is NULL");
  if (n_segs < 1 || n_segs > QI21_MAX_SEGMENTS)
    return fail(QI21_ERR_INVALID_ARG, "n_segs must be in [1, %d] (got %d)", QI21_MAX_SEGMENTS, n_segs);
  if (pos == nullptr) return fail(QI21_ERR_INVALID_ARG, "pos is NULL");
  PositionsParams p;
  memset(&p, 0, sizeof(p));
  int64_t start = 0, text = 0;
  for (int i = 0; i < n_segs; ++i) {
    const qi21_segment& s = segs[i];
    int64_t n;
    if (s.kind == QI21_SEG_TEXT) {
      if (s.n < 1) return fail(QI21_ERR_INVALID_ARG, "segment %d: text needs n >= 1", i);
      n = s.n;
    } else if (s.kind == QI21_SEG_IMAGE) {
      if (s.H < 1 || s.W < 1) return fail(QI21_ERR_INVALID_ARG, "segment %d: image needs H, W >= 1", i);
      n = (int64_t)s.H * s.W;
    } else {
      return fail(QI21_ERR_INVALID_ARG, "segment %d: unknown kind %d", i, s.kind);
    }
    p.segs[i].kind = s.kind;
    p.segs[i].n = s.n;
    p.segs[i].H = s.H;
    p.segs[i].W = s.W;
    p.segs[i].frame = s.frame;
    p.segs[i].start = (int32_t)start;
    p.segs[i].text_base = (int32_t)text;
    if (s.kind == QI21_SEG_TEXT) text += n;
    start += n;
    if (start > INT32_MAX / 2) return fail(QI21_ERR_INVALID_ARG, "sequence too long");
  }
  if (start != L) return fail(QI21_ERR_INVALID_ARG, "segments hold %lld tokens, L = %lld", (long long)start, (long long)L);
  if (original) {
    int32_t max_vid_index = 0;
    for (int i = 0; i < n_segs; ++i)
      if (segs[i].kind == QI21_SEG_IMAGE) {
        max_vid_index = segs[i].H / 2 > max_vid_index ? segs[i].H / 2 : max_vid_index;
        max_vid_index = segs[i].W / 2 > max_vid_index ? segs[i].W / 2 : max_vid_index;
      }
    for (int i = 0; i < n_segs; ++i) p.segs[i].text_base += max_vid_index;
  }
  p.n_segs = n_segs;
  p.L = L;
  p.pos = pos;
  p.kv_end = kv_end;
  p.all_visible = original ? 1 : 0;
  cudaError_t e = launch_positions(p, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "positions launch");
  return QI21_OK;
}

qi21_status qi21_rope_positions(const qi21_segment* segs, int32_t n_segs, int64_t L, int32_t* pos,
                                int32_t* kv_end, void* stream) {
  return rope_positions_impl(segs, n_segs, L, pos, kv_end, false, stream);
}

qi21_status qi21_rope_positions_original(const qi21_segment* segs, int32_t n_segs, int64_t L, int32_t* pos,
                                         int32_t* kv_end, void* stream) {
  return rope_positions_impl(segs, n_segs, L, pos, kv_end, true, stream);
}

size_t qi21_attn_full_workspace_size(int32_t B, int32_t H, int64_t L, int64_t P, qi21_dtype dt) {
  if (B < 0 || H < 0 || L < 0 || P < 0 || P > L) return 0;
  const size_t base = ws_layout(B, H, L, L - P, dt).total;
  if (dt != QI21_BF16 || B == 0 || H == 0 || L == 0) return base;
  return base + split_bytes(B, H, L);
}

size_t qi21_attn_cached_workspace_size(int32_t B, int32_t H, int64_t P, int64_t T, qi21_dtype dt) {
  (void)P;
  if (B < 0 || H < 0 || T < 0) return 0;
  const size_t base = ws_layout(B, H, T, T, dt).total;
  if (dt != QI21_BF16 || B == 0 || H == 0 || T == 0) return base;
  return base + split_bytes(B, H, T);
}

// Ablation of where the keys are rotated: QI21_K_ROTATION=attention (read on
// every call) leaves the keys that do not go to the Prefix cache unrotated in
// the pre-pass and has the tensor-core kernel rotate each of their tiles in
// shared memory before its S MMAs.  bf16 calls without QK-RMSNorm only; such a
// call runs without tail split.  Default: every key is rotated once, in the
// pre-pass.
static bool k_rotation_in_attention(qi21_dtype dt, const float* norm_k) {
  if (dt != QI21_BF16 || norm_k != nullptr) return false;
  const char* s = getenv("QI21_K_ROTATION");
  return s != nullptr && strcmp(s, "attention") == 0;
}

static qi21_status attn_full_impl(int32_t B, int32_t H, int64_t L, int64_t P, qi21_dtype dt,
                                  const void* q, const void* k, const void* v, const int32_t* pos,
                                  const int32_t* kv_end, void* o, void* k_cache, void* v_cache,
                                  const float* norm_q, const float* norm_k, float eps,
                                  void* workspace, size_t workspace_bytes, void* stream) {
  QI21_TRY(check_common(B, H, dt));
  if (L < 0 || L > (int64_t)1 << 30) return fail(QI21_ERR_INVALID_ARG, "L out of range (%lld)", (long long)L);
  if (P < 0 || P > L) return fail(QI21_ERR_INVALID_ARG, "P must be in [0, L] (P=%lld, L=%lld)", (long long)P, (long long)L);
  if ((k_cache == nullptr) != (v_cache == nullptr))
    return fail(QI21_ERR_INVALID_ARG, "k_cache and v_cache must both be given or both be NULL");
  if (B == 0 || H == 0 || L == 0) return QI21_OK;
  QI21_TRY(check_ptr(q, "q"));
  QI21_TRY(check_ptr(k, "k"));
  QI21_TRY(check_ptr(v, "v"));
  QI21_TRY(check_ptr(o, "o"));
  QI21_TRY(check_ptr(pos, "pos"));
  if (kv_end != nullptr) QI21_TRY(check_ptr(kv_end, "kv_end"));
  if (k_cache != nullptr && P > 0) {
    QI21_TRY(check_ptr(k_cache, "k_cache"));
    QI21_TRY(check_ptr(v_cache, "v_cache"));
  }
  QI21_TRY(check_ptr(workspace, "workspace"));
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return fail(QI21_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
  QI21_TRY(check_norm(norm_q, norm_k, eps));
  const bool cache = k_cache != nullptr && P > 0;
  const int64_t split = cache ? P : L;
  const WsLayout w = ws_layout(B, H, L, L - (cache ? P : 0), dt);
  if (workspace_bytes < w.total)
    return fail(QI21_ERR_INVALID_ARG, "workspace too small: %zu < %zu bytes", workspace_bytes, w.total);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  uint32_t* status = reinterpret_cast<uint32_t*>(ws);
  float2* table = reinterpret_cast<float2*>(ws + w.table_off);
  void* ws_k = ws + w.k_off;

  RopePrepParams rp;
  memset(&rp, 0, sizeof(rp));
  rp.k = k;
  rp.v = v;
  rp.pos = pos;
  rp.B = B;
  rp.H = H;
  rp.Lk = L;
  rp.split = split;
  rp.k_dst0 = cache ? k_cache : ws_k;
  rp.k_dst1 = cache ? ws_k : nullptr;
  rp.v_dst0 = cache ? v_cache : nullptr;
  rp.table = table;
  rp.table_half = dt == QI21_BF16 ? 1 : 0;
  rp.unit_counter = &reinterpret_cast<WsHeader*>(ws)->unit_counter;
  rp.omega = make_omega();
  rp.k_norm_w = norm_k;
  rp.norm_eps = eps;
  // the target's keys (past the cached Prefix) may be left to the attention kernel
  const bool rot_k1 = cache && k_rotation_in_attention(dt, norm_k);
  rp.k_rot_end = rot_k1 ? split : L;
  AttnArgs a;
  memset(&a, 0, sizeof(a));
  // without a mask every unit costs the same, so the last wave may be split
  if (dt == QI21_BF16 && kv_end == nullptr && !rot_k1)
    carve_split(a, rp, ws, w.total, workspace_bytes, B, H, L);
  cudaError_t e = launch_rope_prep(rp, dt == QI21_F32, st);
  if (e != cudaSuccess) return cuda_fail(e, "rope pre-pass launch");

  const int64_t tokstride = (int64_t)H * kHeadDim;
  a.unit_counter = rp.unit_counter;
  a.B = B;
  a.H = H;
  a.Lq = L;
  a.q = q;
  a.table = table;
  a.kv_end = kv_end;
  // keys: rows [0, split) head-major in dst0, rows [split, L) head-major in ws_k
  a.k0 = KvSource{rp.k_dst0, split, kHeadDim, split * kHeadDim, (int64_t)H * split * kHeadDim};
  a.k1 = KvSource{cache ? ws_k : nullptr, L - split, kHeadDim, (L - split) * kHeadDim,
                  (int64_t)H * (L - split) * kHeadDim};
  const size_t eb = elem_bytes(dt);
  if (rot_k1) {
    // raw target keys straight from k (token-major)
    a.k1 = KvSource{static_cast<const uint8_t*>(k) + (size_t)split * tokstride * eb, L - split, tokstride,
                    kHeadDim, L * tokstride};
    a.rot_k1 = 1;
  }
  // values straight from v (token-major), split the same way
  a.v0 = KvSource{v, split, tokstride, kHeadDim, L * tokstride};
  a.v1 = KvSource{static_cast<const uint8_t*>(v) + (size_t)split * tokstride * eb, L - split, tokstride,
                  kHeadDim, L * tokstride};
  a.o = o;
  a.status = status;
  a.q_norm_w = norm_q;
  a.norm_eps = eps;
  return run_attention(a, dt, st);
}

// rope_table: the target's table from qi21_rope_table (its float32 pairs feed
// the pre-pass's key rotation, its float16 pairs the queries' rotation), or
// null: computed here from pos_tgt.
static qi21_status attn_cached_impl(int32_t B, int32_t H, int64_t P, int64_t T, qi21_dtype dt,
                                    const void* q, const void* k, const void* v,
                                    const int32_t* pos_tgt, const void* k_cache, const void* v_cache,
                                    void* o, const float* norm_q, const float* norm_k, float eps,
                                    void* workspace, size_t workspace_bytes, void* stream,
                                    const void* rope_table = nullptr) {
  QI21_TRY(check_common(B, H, dt));
  if (P < 0 || T < 0 || P > (int64_t)1 << 30 || T > (int64_t)1 << 30)
    return fail(QI21_ERR_INVALID_ARG, "P and T must be in [0, 2^30] (P=%lld, T=%lld)", (long long)P, (long long)T);
  if (B == 0 || H == 0 || T == 0) return QI21_OK;
  QI21_TRY(check_ptr(q, "q"));
  QI21_TRY(check_ptr(k, "k"));
  QI21_TRY(check_ptr(v, "v"));
  QI21_TRY(check_ptr(o, "o"));
  if (rope_table == nullptr)
    QI21_TRY(check_ptr(pos_tgt, "pos_tgt"));
  else
    QI21_TRY(check_ptr(rope_table, "rope_table"));
  if (P > 0) {
    QI21_TRY(check_ptr(k_cache, "k_cache"));
    QI21_TRY(check_ptr(v_cache, "v_cache"));
  }
  QI21_TRY(check_ptr(workspace, "workspace"));
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return fail(QI21_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
  QI21_TRY(check_norm(norm_q, norm_k, eps));
  const WsLayout w = ws_layout(B, H, T, T, dt);
  if (workspace_bytes < w.total)
    return fail(QI21_ERR_INVALID_ARG, "workspace too small: %zu < %zu bytes", workspace_bytes, w.total);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  uint32_t* status = reinterpret_cast<uint32_t*>(ws);
  float2* table = reinterpret_cast<float2*>(ws + w.table_off);
  void* ws_k = ws + w.k_off;

  RopePrepParams rp;
  memset(&rp, 0, sizeof(rp));
  rp.k = k;
  rp.v = v;
  rp.pos = pos_tgt;
  rp.B = B;
  rp.H = H;
  rp.Lk = T;
  rp.split = T;
  rp.k_dst0 = ws_k;
  rp.table = table;
  rp.table_half = dt == QI21_BF16 ? 1 : 0;
  rp.unit_counter = &reinterpret_cast<WsHeader*>(ws)->unit_counter;
  rp.omega = make_omega();
  rp.k_norm_w = norm_k;
  rp.norm_eps = eps;
  const bool rot_k1 = k_rotation_in_attention(dt, norm_k);
  rp.k_rot_end = rot_k1 ? 0 : T;
  // a given table: the pre-pass reads its float32 pairs, the attention its
  // float16 (bf16 path) or float32 pairs; the workspace's table is not written
  const void* table_t16 = nullptr;
  if (rope_table != nullptr) {
    rp.pos = nullptr;
    rp.table_in = rope_table;
    rp.table = nullptr;
    table_t16 = static_cast<const uint8_t*>(rope_table) + (size_t)T * kPairs * sizeof(float2);
  }

  // Tail-split scratch: whatever the workspace holds past the minimum layout
  // (none: the call runs unsplit).
  AttnArgs a;
  memset(&a, 0, sizeof(a));
  if (dt == QI21_BF16 && !rot_k1) carve_split(a, rp, ws, w.total, workspace_bytes, B, H, T);
  cudaError_t e = launch_rope_prep(rp, dt == QI21_F32, st);
  if (e != cudaSuccess) return cuda_fail(e, "rope pre-pass launch");

  const int64_t tokstride = (int64_t)H * kHeadDim;
  a.unit_counter = rp.unit_counter;
  a.B = B;
  a.H = H;
  a.Lq = T;
  a.q = q;
  a.table = rope_table == nullptr ? static_cast<const void*>(table)
                                  : (dt == QI21_BF16 ? table_t16 : rope_table);
  a.kv_end = nullptr;  // the target sees every key
  a.k0 = KvSource{k_cache, P, kHeadDim, P * kHeadDim, (int64_t)H * P * kHeadDim};
  a.k1 = KvSource{ws_k, T, kHeadDim, T * kHeadDim, (int64_t)H * T * kHeadDim};
  if (rot_k1) {
    a.k1 = KvSource{k, T, tokstride, kHeadDim, T * tokstride};  // raw target keys
    a.rot_k1 = 1;
  }
  a.v0 = KvSource{v_cache, P, kHeadDim, P * kHeadDim, (int64_t)H * P * kHeadDim};
  a.v1 = KvSource{v, T, tokstride, kHeadDim, T * tokstride};
  a.o = o;
  a.status = status;
  a.q_norm_w = norm_q;
  a.norm_eps = eps;
  return run_attention(a, dt, st);
}

qi21_status qi21_attn_full(int32_t B, int32_t H, int64_t L, int64_t P, qi21_dtype dt, const void* q,
                           const void* k, const void* v, const int32_t* pos, const int32_t* kv_end,
                           void* o, void* k_cache, void* v_cache, void* workspace,
                           size_t workspace_bytes, void* stream) {
  return attn_full_impl(B, H, L, P, dt, q, k, v, pos, kv_end, o, k_cache, v_cache, nullptr, nullptr,
                        0.f, workspace, workspace_bytes, stream);
}

qi21_status qi21_attn_full_qknorm(int32_t B, int32_t H, int64_t L, int64_t P, qi21_dtype dt,
                                  const void* q, const void* k, const void* v, const int32_t* pos,
                                  const int32_t* kv_end, void* o, void* k_cache, void* v_cache,
                                  const float* norm_q, const float* norm_k, float eps,
                                  void* workspace, size_t workspace_bytes, void* stream) {
  if (norm_q == nullptr || norm_k == nullptr)
    return fail(QI21_ERR_INVALID_ARG, "norm_q and norm_k must be given");
  return attn_full_impl(B, H, L, P, dt, q, k, v, pos, kv_end, o, k_cache, v_cache, norm_q, norm_k,
                        eps, workspace, workspace_bytes, stream);
}

qi21_status qi21_attn_cached(int32_t B, int32_t H, int64_t P, int64_t T, qi21_dtype dt, const void* q,
                             const void* k, const void* v, const int32_t* pos_tgt, const void* k_cache,
                             const void* v_cache, void* o, void* workspace, size_t workspace_bytes,
                             void* stream) {
  return attn_cached_impl(B, H, P, T, dt, q, k, v, pos_tgt, k_cache, v_cache, o, nullptr, nullptr,
                          0.f, workspace, workspace_bytes, stream);
}

size_t qi21_rope_table_size(int64_t n) {
  if (n < 0) return 0;
  return (size_t)n * kPairs * (sizeof(float2) + sizeof(uint32_t));
}

qi21_status qi21_rope_table(const int32_t* pos, int64_t n, void* table, size_t table_bytes, void* stream) {
  if (n < 0 || n > (int64_t)1 << 30) return fail(QI21_ERR_INVALID_ARG, "n out of range (%lld)", (long long)n);
  if (n == 0) return QI21_OK;
  QI21_TRY(check_ptr(pos, "pos"));
  QI21_TRY(check_ptr(table, "table"));
  if (table_bytes < qi21_rope_table_size(n))
    return fail(QI21_ERR_INVALID_ARG, "table too small: %zu < %zu bytes", table_bytes, qi21_rope_table_size(n));
  RopeTableParams p;
  p.pos = pos;
  p.n = n;
  p.t32 = table;
  p.t16 = static_cast<uint8_t*>(table) + (size_t)n * kPairs * sizeof(float2);
  p.omega = make_omega();
  const cudaError_t e = launch_rope_table(p, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "rotation table launch");
  return QI21_OK;
}

qi21_status qi21_attn_cached_tabled(int32_t B, int32_t H, int64_t P, int64_t T, qi21_dtype dt,
                                    const void* q, const void* k, const void* v, const void* rope_table,
                                    const void* k_cache, const void* v_cache, void* o, void* workspace,
                                    size_t workspace_bytes, void* stream) {
  return attn_cached_impl(B, H, P, T, dt, q, k, v, nullptr, k_cache, v_cache, o, nullptr, nullptr, 0.f,
                          workspace, workspace_bytes, stream, rope_table);
}

qi21_status qi21_attn_cached_qknorm(int32_t B, int32_t H, int64_t P, int64_t T, qi21_dtype dt,
                                    const void* q, const void* k, const void* v,
                                    const int32_t* pos_tgt, const void* k_cache, const void* v_cache,
                                    void* o, const float* norm_q, const float* norm_k, float eps,
                                    void* workspace, size_t workspace_bytes, void* stream) {
  if (norm_q == nullptr || norm_k == nullptr)
    return fail(QI21_ERR_INVALID_ARG, "norm_q and norm_k must be given");
  return attn_cached_impl(B, H, P, T, dt, q, k, v, pos_tgt, k_cache, v_cache, o, norm_q, norm_k, eps,
                          workspace, workspace_bytes, stream);
}

static qi21_status linear_impl(int64_t M, int64_t N, int64_t K, const void* x, const void* w, const void* bias,
                               void* const* out, int32_t n_out, const void* residual, float alpha,
                               bool swiglu, void* workspace, size_t workspace_bytes, void* stream) {
  if (M < 0 || N < 0 || K < 0 || M > INT32_MAX || N > INT32_MAX || K > INT32_MAX)
    return fail(QI21_ERR_INVALID_ARG, "M, N, K must be in [0, 2^31)");
  if (n_out < 1 || n_out > 4) return fail(QI21_ERR_INVALID_ARG, "n_out must be in [1, 4] (got %d)", n_out);
  if (N % n_out != 0 || (N / n_out) % 8 != 0)
    return fail(QI21_ERR_INVALID_ARG, "N / n_out must be a whole multiple of 8 (N=%lld, n_out=%d)",
                (long long)N, n_out);
  if (K % 8 != 0) return fail(QI21_ERR_INVALID_ARG, "K must be a multiple of 8 (got %lld)", (long long)K);
  if (M == 0 || N == 0) return QI21_OK;
  if (K == 0) return fail(QI21_ERR_INVALID_ARG, "K must be >= 8 when M and N are not 0");
  QI21_TRY(check_ptr(x, "x"));
  QI21_TRY(check_ptr(w, "w"));
  if (bias != nullptr) QI21_TRY(check_ptr(bias, "bias"));
  if (out == nullptr) return fail(QI21_ERR_INVALID_ARG, "out is NULL");
  for (int i = 0; i < n_out; ++i) QI21_TRY(check_ptr(out[i], "out[i]"));
  QI21_TRY(check_ptr(workspace, "workspace"));
  if (workspace_bytes < QI21_WORKSPACE_HEADER_BYTES)
    return fail(QI21_ERR_INVALID_ARG, "workspace too small: %zu < %d bytes", workspace_bytes,
                QI21_WORKSPACE_HEADER_BYTES);
  GemmArgs a;
  memset(&a, 0, sizeof(a));
  a.M = M;
  a.N = N;
  a.K = K;
  a.x = x;
  a.w = w;
  a.bias = bias;
  for (int i = 0; i < n_out; ++i) a.out[i] = out[i];
  a.n_out = n_out;
  a.residual = residual;
  a.alpha = alpha;
  a.swiglu = swiglu ? 1 : 0;
  a.status = static_cast<uint32_t*>(workspace);
  cudaError_t e = launch_gemm_tc(a, static_cast<cudaStream_t>(stream), sm_count());
  if (e != cudaSuccess) return cuda_fail(e, "linear launch");
  return QI21_OK;
}

qi21_status qi21_linear(int64_t M, int64_t N, int64_t K, const void* x, const void* w, const void* bias,
                        void* const* out, int32_t n_out, void* workspace, size_t workspace_bytes,
                        void* stream) {
  return linear_impl(M, N, K, x, w, bias, out, n_out, nullptr, 1.0f, false, workspace, workspace_bytes,
                     stream);
}

qi21_status qi21_linear_residual(int64_t M, int64_t N, int64_t K, const void* x, const void* w,
                                 const void* bias, const void* residual, float alpha, void* out,
                                 void* workspace, size_t workspace_bytes, void* stream) {
  if (M > 0 && N > 0) QI21_TRY(check_ptr(residual, "residual"));
  if (!(alpha == alpha) || alpha > 3.0e38f || alpha < -3.0e38f)
    return fail(QI21_ERR_INVALID_ARG, "alpha must be finite");
  void* outs[1] = {out};
  return linear_impl(M, N, K, x, w, bias, outs, 1, residual, alpha, false, workspace, workspace_bytes, stream);
}

qi21_status qi21_linear_swiglu(int64_t M, int64_t N, int64_t K, const void* x, const void* w,
                               const void* bias, void* out, void* workspace, size_t workspace_bytes,
                               void* stream) {
  if (N % 256 != 0)
    return fail(QI21_ERR_INVALID_ARG, "N must be a multiple of 256 (gate/up blocks of 128; got %lld)",
                (long long)N);
  void* outs[1] = {out};
  return linear_impl(M, N, K, x, w, bias, outs, 1, nullptr, 1.0f, true, workspace, workspace_bytes, stream);
}

qi21_status qi21_rmsnorm(int64_t M, int32_t D, const void* x, const void* w, float eps, void* y,
                         void* stream) {
  if (M < 0 || D < 8 || D % 8 != 0 || M > INT32_MAX)
    return fail(QI21_ERR_INVALID_ARG, "need M >= 0 and D a multiple of 8 (M=%lld, D=%d)", (long long)M, D);
  if (!(eps >= 0.f) || !(eps < 3.0e38f)) return fail(QI21_ERR_INVALID_ARG, "eps must be finite and >= 0");
  if (M == 0) return QI21_OK;
  QI21_TRY(check_ptr(x, "x"));
  QI21_TRY(check_ptr(w, "w"));
  QI21_TRY(check_ptr(y, "y"));
  cudaError_t e = launch_rmsnorm(M, D, x, w, eps, y, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "rmsnorm launch");
  return QI21_OK;
}

qi21_status qi21_swiglu(int64_t n, const void* g, const void* u, void* m, void* stream) {
  if (n < 0 || n % 8 != 0 || n / 8 > INT32_MAX)
    return fail(QI21_ERR_INVALID_ARG, "n must be a non-negative multiple of 8 (got %lld)", (long long)n);
  if (n == 0) return QI21_OK;
  QI21_TRY(check_ptr(g, "g"));
  QI21_TRY(check_ptr(u, "u"));
  QI21_TRY(check_ptr(m, "m"));
  cudaError_t e = launch_swiglu(n, g, u, m, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "swiglu launch");
  return QI21_OK;
}

// NULL names the built-in scratch of qi21_attn_cached_noalloc.
static qi21_status status_target(void** workspace) {
  if (*workspace != nullptr) return QI21_OK;
  const cudaError_t e = noalloc_scratch(workspace);
  if (e != cudaSuccess) return cuda_fail(e, "built-in scratch address");
  return QI21_OK;
}

qi21_status qi21_workspace_status(void* workspace, void* stream) {
  QI21_TRY(status_target(&workspace));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  WsHeader h;
  cudaError_t e = cudaMemcpyAsync(&h, workspace, sizeof(h), cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return cuda_fail(e, "status read");
  if (h.status == QI21_OK) return QI21_OK;
  const uint32_t zero[2] = {0, 0};  // status and site; the schedule counter is left alone
  e = cudaMemcpyAsync(workspace, zero, sizeof(zero), cudaMemcpyHostToDevice, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return cuda_fail(e, "status clear");
  return fail(static_cast<qi21_status>(h.status), "device wait ran out (site 0x%x)", h.where);
}

qi21_status qi21_selftest_wait_timeout(void* workspace, int64_t limit_ns, void* stream) {
  QI21_TRY(status_target(&workspace));
  if (limit_ns < 1 || limit_ns > 2000000000LL)
    return fail(QI21_ERR_INVALID_ARG, "limit_ns must be in [1, 2e9]");
  cudaError_t e = launch_wait_selftest(static_cast<uint32_t*>(workspace), (uint64_t)limit_ns,
                                       static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "self-test launch");
  return QI21_OK;
}

const char* qi21_status_string(qi21_status s) {
  switch (s) {
    case QI21_OK: return "QI21_OK";
    case QI21_ERR_INVALID_ARG: return "QI21_ERR_INVALID_ARG";
    case QI21_ERR_UNSUPPORTED: return "QI21_ERR_UNSUPPORTED";
    case QI21_ERR_CUDA: return "QI21_ERR_CUDA";
    case QI21_ERR_TIMEOUT: return "QI21_ERR_TIMEOUT";
  }
  return "QI21_ERR_UNKNOWN";
}

const char* qi21_last_error(void) { return g_last_error; }

uint64_t qi21_launch_count(void) { return g_launches; }

}  // extern "C"
