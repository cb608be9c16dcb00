// Internal declarations shared by the host entry points and the kernels of
// libqi21.  Not part of the public C ABI (include/qi21.h is).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/qi21.h"

namespace qi21 {

constexpr int kHeadDim = 128;
constexpr int kPairs = 64;           // complex pairs per head (8 + 28 + 28)
constexpr int kBandPairs0 = 8;       // frame band: dims [0, 16)
constexpr int kBandPairs01 = 36;     // frame + height bands: dims [0, 72)
constexpr uint32_t kStatusTimeout = 4;
constexpr uint64_t kWaitLimitNs = 1000000000ull;  // bounded device waits: 1 s

// Status words at the start of every workspace.
struct WsHeader {
  uint32_t status;        // 0 = OK, else a qi21_status
  uint32_t where;         // which wait ran out (role << 8 | barrier id)
  uint32_t unit_counter;  // next work unit of the attention kernel's dynamic schedule
};

// ---------------------------------------------------------------- positions
struct SegDev {
  int32_t kind, n, H, W, frame;
  int32_t start;      // first token of the segment
  int32_t text_base;  // position of the segment's first text token
};
constexpr int kMaxSegments = 128;
struct PositionsParams {
  SegDev segs[kMaxSegments];
  int32_t n_segs;
  int64_t L;
  int32_t* pos;
  int32_t* kv_end;
  int32_t all_visible;  // 1: no mask, every token sees all L keys
};
cudaError_t launch_positions(const PositionsParams& p, cudaStream_t stream);

// ------------------------------------------------- rotation / cache pre-pass
// Angular frequency of every pair: theta^(-2j/d_axis) for its band, float64.
struct Omega {
  double w[kPairs];
};
Omega make_omega();

struct RopePrepParams {
  const void* k;       // token-major [B, Lk, H, 128]
  const void* v;       // token-major [B, Lk, H, 128] (read only when v_dst0)
  const int32_t* pos;  // [Lk][3]
  int32_t B, H;
  int64_t Lk;
  int64_t split;   // tokens [0, split) -> dst0, [split, Lk) -> dst1
  void* k_dst0;    // head-major [B, H, split, 128]
  void* k_dst1;    // head-major [B, H, Lk - split, 128] (or null when split == Lk)
  void* v_dst0;    // head-major [B, H, split, 128] copy of V, or null
  void* table;     // [Lk][64] (cos, sin) of every token, or null: float2, or half2 when table_half
  int32_t table_half;
  uint32_t* unit_counter;  // zeroed here for the attention launch that follows, or null
  uint32_t* zero_words;    // also zeroed here (the attention's tail-split counters), or null
  int32_t n_zero_words;
  Omega omega;
  const float* k_norm_w;   // [128] QK-RMSNorm weight of K, or null (no norm)
  float norm_eps;
  // Keys of tokens [k_rot_end, Lk) are neither rotated nor written here (the
  // attention kernel rotates them itself); Lk: every token's key is rotated.
  int64_t k_rot_end;
  // [Lk][64] float2 (cos, sin) built earlier by the table kernel (pos is then
  // not read and no angle is computed), or null
  const void* table_in;
};
cudaError_t launch_rope_prep(const RopePrepParams& p, bool f32, cudaStream_t stream);

// A request's rotation table: per token its 64 (cos, sin) pairs, float2 in
// t32 [n][64] and rounded to half2 in t16 [n][64], the same values the
// pre-pass computes.
struct RopeTableParams {
  const int32_t* pos;  // [n][3]
  int64_t n;
  void* t32;
  void* t16;
  Omega omega;
};
cudaError_t launch_rope_table(const RopeTableParams& p, cudaStream_t stream);

// --------------------------------------------------------------- attention
// One key/value source: rows of one (batch, head) are `row` elements apart,
// heads `head` apart, batches `batch` apart (element strides).
struct KvSource {
  const void* ptr;
  int64_t n;  // rows in this source
  int64_t row, head, batch;
};

// Attention of Lq query rows over the keys [src0 rows || src1 rows]:
// O = softmax(rot(Q) K^T / sqrt(128) + M) V, M from kv_end (null = no mask).
struct AttnArgs {
  int32_t B, H;
  int64_t Lq;
  const void* q;          // token-major [B, Lq, H, 128] (not rotated)
  const void* table;      // [Lq][64] cos/sin of the query rows: half2 (bf16 path) or float2 (fp32)
  const int32_t* kv_end;  // [Lq] or null
  KvSource k0, k1;        // rotated keys
  KvSource v0, v1;        // values
  void* o;                // token-major [B, Lq, H, 128]
  uint32_t* status;       // workspace header status word
  uint32_t* unit_counter; // workspace header: dynamic-schedule counter (zeroed by the pre-pass)
  const float* q_norm_w;  // [128] QK-RMSNorm weight of Q, or null (no norm)
  float norm_eps;
  // Scratch for splitting the last, partial wave of units into key-range
  // pieces (unmasked calls only; null / 0: no split).  split_cnt holds
  // split_cnt_units x 8 arrival counters, zeroed by the pre-pass; split_part
  // and split_ml hold the O / l (bf16) and (row max, row sum) of up to
  // split_slots pieces.  The launcher decides how many pieces it uses.
  uint32_t* split_cnt;
  int32_t split_cnt_units;
  void* split_part;   // split_slots x 2 tiles x 128 rows x 128 bf16
  void* split_ml;     // split_slots x 2 tiles x 128 rows x float2
  int32_t split_slots;
  // 1: k1 holds the raw keys of the last k1.n query rows (token-major, not
  // rotated), and the tensor-core kernel rotates each of their tiles in shared
  // memory from the query table before its S MMAs (no tail split then).
  int32_t rot_k1;
};
cudaError_t launch_attn_simt_f32(const AttnArgs& a, cudaStream_t stream);
cudaError_t launch_attn_tc_bf16(const AttnArgs& a, cudaStream_t stream, int num_sms);

// ------------------------------------------------------------ linear layer
// Y = X W^T (+ b): X [M, K], W [N, K], b [N] or null, all bf16; the N output
// columns go to n_out equal segments out[i] = [M, N / n_out] (row-major).
struct GemmArgs {
  int64_t M, N, K;
  const void* x;
  const void* w;
  const void* bias;
  void* out[4];
  int32_t n_out;
  const void* residual;  // [M, N]: out = residual + alpha * (X W^T + b) (n_out = 1), or null
  float alpha;
  int32_t swiglu;        // 1: gate/up rows of W alternate in 128-row blocks; out[0] [M, N/2]
                         //    = silu(gate) * up (n_out = 1, N a multiple of 256)
  uint32_t* status;  // workspace header status word
};
cudaError_t launch_gemm_tc(const GemmArgs& a, cudaStream_t stream, int num_sms);

// ---------------------------------------------------------- row-wise ops
// y = x / sqrt(mean(x^2) + eps) * w over rows of D (bf16), one warp per row.
cudaError_t launch_rmsnorm(int64_t M, int32_t D, const void* x, const void* w, float eps, void* y,
                           cudaStream_t stream);
// m = silu(g) * u elementwise (bf16, n a multiple of 8).
cudaError_t launch_swiglu(int64_t n, const void* g, const void* u, void* m, cudaStream_t stream);

// --------------------------------------------------------------- self test
cudaError_t launch_wait_selftest(uint32_t* status, uint64_t limit_ns, cudaStream_t stream);

// Bytes a cached step needs at least (no tail-split scratch);
// qi21_attn_cached_workspace_size() adds the scratch that lets the last wave
// of units be split.
size_t attn_cached_workspace_min(int32_t B, int32_t H, int64_t T, qi21_dtype dt);

// Device address of qi21_attn_cached_noalloc's built-in scratch on the
// current device (noalloc.cu).
cudaError_t noalloc_scratch(void** ptr);

// Launch bookkeeping (thread-local counter of launches enqueued).
void note_launch();

// Records a message for qi21_last_error() and returns `s`.
qi21_status report_error(qi21_status s, const char* fmt, ...);

}  // namespace qi21
