/*
 * qi21.h -- C ABI of libqi21, the sm_100a (B200) hot path of the Qwen-Image-2.1
 * denoiser's joint attention: 3D axial RoPE, the Block-Causal mask and the
 * Prefix KV Cache.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * - Head dimension is fixed at 128, split into rotary bands (16, 56, 56) for
 *   the (frame, height, width) axes, theta = 10000, adjacent-pair rotation
 *   ("3A - 3D Axial RoPE (16, 56, 56)", section 1; "Qwen-Image-Edit close
 *   reading", section 7.1).  Softmax scale is 1/sqrt(128).
 * - Activations are contiguous [B, L, H, 128] (token-major), as the joint
 *   attention sees them after unflattening heads ("Qwen-Image-Edit close
 *   reading", section 6 and the shape table of section 8.2).  The KV cache is
 *   contiguous [B, H, P, 128] (head-major).
 * - Pointers named "device" must be device memory of the current CUDA device;
 *   every device buffer must be 16-byte aligned.  The caller owns every buffer;
 *   the library allocates nothing, and nothing one call leaves behind changes
 *   what a later call computes: the only state it keeps is, per calling
 *   thread, the last error message and a launch counter (the diagnostics at
 *   the end of this header), plus the built-in scratch of
 *   qi21_attn_cached_noalloc.
 * - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *   Calls validate their arguments on the host, enqueue kernels on `stream` and
 *   return without synchronising.  A failed launch returns QI21_ERR_CUDA.
 * - Errors: a non-OK status means nothing was enqueued (argument errors) or the
 *   launch failed; qi21_last_error() returns a message for the calling thread.
 * - Device-side waits are bounded (about one second); a wait that runs out
 *   sets a status word in the workspace header and the kernel returns early.
 *   qi21_workspace_status() reads and clears that word.
 * - Scratch: the attention calls take a caller-owned workspace (its header
 *   holds the status word and the kernel's work counter; the rest holds the
 *   per-token cos/sin table and the rotated keys of the call).  The paths
 *   that need no workspace are qi21_rope_positions and
 *   qi21_attn_cached_noalloc.
 * - Key rotation placement (an ablation; the result is the same up to
 *   rounding): by default every key is rotated once, by the call's pre-pass.
 *   With the environment variable QI21_K_ROTATION=attention (read on every
 *   call) a QI21_BF16 call without QK-RMSNorm leaves the keys that do not go
 *   to the Prefix cache unrotated, and the attention kernel rotates each of
 *   their tiles in shared memory (from the fp16 query table) before it reads
 *   them, once per query-tile pair that visits the tile; such a call does not
 *   split its last wave.  The Prefix keys stored in the cache are rotated by
 *   the pre-pass either way.
 */
#ifndef QI21_H
#define QI21_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  QI21_OK = 0,
  QI21_ERR_INVALID_ARG = 1, /* bad size, pointer, alignment or workspace */
  QI21_ERR_UNSUPPORTED = 2, /* valid request this build does not handle */
  QI21_ERR_CUDA = 3,        /* a CUDA runtime/driver call failed */
  QI21_ERR_TIMEOUT = 4      /* a device-side bounded wait ran out */
} qi21_status;

typedef enum {
  QI21_BF16 = 0, /* bf16 storage, fp32 accumulation (tcgen05 tensor cores) */
  QI21_F32 = 1   /* fp32 storage and arithmetic (CUDA cores) */
} qi21_dtype;

typedef enum { QI21_SEG_TEXT = 0, QI21_SEG_IMAGE = 1 } qi21_segment_kind;

/* One segment of the joint sequence, in sequence order.  Text: `n` tokens
 * (H, W, frame ignored).  Image: an H x W latent grid in row-major order
 * (width fastest), all tokens sharing frame index `frame` (n ignored). */
typedef struct {
  int32_t kind;  /* qi21_segment_kind */
  int32_t n;     /* text token count */
  int32_t H, W;  /* image grid */
  int32_t frame; /* image frame index */
} qi21_segment;

/* Bytes of the workspace header (status word); workspaces start with it. */
#define QI21_WORKSPACE_HEADER_BYTES 256
/* Most segments one qi21_rope_positions call accepts. */
#define QI21_MAX_SEGMENTS 128

/*
 * qi21_rope_positions -- position table and block-causal visibility bound.
 *
 * Follows "3A - 3D Axial RoPE (16, 56, 56) & Zero-Centered Grid", section 1
 * and its glossary: text tokens advance frame = height = width by +1 (the
 * counter starts at 0 and counts text tokens only); an image keeps its frame
 * index over the whole image and centres its grid, height running from
 * -(H - H//2) to H//2 - 1 and width likewise.  The visibility bound follows
 * the Block-Causal mask of the "Qwen-Image-2.1 architecture" overview (card
 * 3C): text token i sees keys [0, i]; an image token sees every key before its
 * image and its whole image.  Hence allowed(i, j) <=> j < kv_end[i].
 *
 *   segs    host array of n_segs segments (1 <= n_segs <= QI21_MAX_SEGMENTS);
 *           text n >= 1, image H, W >= 1.
 *   L       total tokens; must equal the sum over segments.
 *   pos     device int32 [L][3] (frame, height, width), written.
 *   kv_end  device int32 [L], written; may be NULL.
 * Returns QI21_ERR_INVALID_ARG when the segments are malformed or do not add
 * up to L.  L = 0 with n_segs = 0 is a no-op.
 */
qi21_status qi21_rope_positions(const qi21_segment* segs, int32_t n_segs, int64_t L,
                                int32_t* pos, int32_t* kv_end, void* stream);

/*
 * qi21_rope_positions_original -- the same table for the earlier Qwen-Image
 * model, a second workload for the attention with the mask off.  Images are
 * numbered exactly as above (close reading section 7.3); text tokens take
 * f = h = w = max_vid_index + (text tokens before them), where max_vid_index
 * is the largest max(H//2, W//2) over the image segments (section 7.2: the
 * text frequencies start at max_vid_index); kv_end[i] = L for every token (no
 * mask; section 6: is_causal=False).  That model orders its sequence
 * [text | target | references]; the segment order is the caller's.  Same
 * arguments, errors and layout as qi21_rope_positions.
 */
qi21_status qi21_rope_positions_original(const qi21_segment* segs, int32_t n_segs, int64_t L,
                                         int32_t* pos, int32_t* kv_end, void* stream);

/* Workspace bytes for qi21_attn_full with these sizes (header included).
 * P is the number of rows the call will store in a cache: pass the prefix
 * length when k_cache/v_cache are given and 0 when they are not (the call
 * checks workspace_bytes against the size for the rows it keeps).  For bf16
 * it includes the scratch for splitting the last wave of work units, used
 * only by calls without a mask (kv_end NULL); a workspace without it (the
 * table and the rotated keys) still works. */
size_t qi21_attn_full_workspace_size(int32_t B, int32_t H, int64_t L, int64_t P, qi21_dtype dt);

/*
 * qi21_attn_full -- the first denoising step: block-causal joint attention over
 * the whole sequence, optionally storing the Prefix KV Cache.
 *
 * O = softmax(rot(Q) rot(K)^T / sqrt(128) + M) V with M[i][j] = 0 if
 * j < kv_end[i] else -inf (overview cards 3C and 4A); key tiles that are fully
 * masked for a query tile are skipped.  The first P tokens form the Prefix
 * (text + reference images, before the target image); when k_cache/v_cache
 * are given, the rotated prefix K and the prefix V are stored there for the
 * later steps (overview card 6A: step 1 stores, steps 2..N load).
 *
 *   B, H, L     batch, heads, tokens (B, H >= 0; L >= 0).
 *   P           prefix length, 0 <= P <= L.
 *   dt          QI21_BF16 or QI21_F32; every tensor argument has this type.
 *   q, k, v     device [B, L, H, 128], read.
 *   pos         device int32 [L][3] from qi21_rope_positions.
 *   kv_end      device int32 [L] from qi21_rope_positions; must be
 *               non-decreasing with 1 <= kv_end[i] <= L (the builder's output
 *               always is).  NULL: no mask, every query sees all L keys (the
 *               earlier model's layout, where qi21_rope_positions_original
 *               writes kv_end = L); such a call may also split its last,
 *               partial wave of work units like qi21_attn_cached.
 *   o           device [B, L, H, 128], written.
 *   k_cache     device [B, H, P, 128] or NULL: rotated prefix K, written.
 *   v_cache     device [B, H, P, 128] or NULL: prefix V, written (both or
 *               neither must be given).
 *   workspace   device scratch of at least qi21_attn_full_workspace_size()
 *               bytes, 256-byte aligned; its header must be zero before the
 *               first use (a zeroed allocation) and is kept zero by the
 *               library unless a bounded wait runs out.
 * Calls on one workspace must be stream-ordered.
 */
qi21_status qi21_attn_full(int32_t B, int32_t H, int64_t L, int64_t P, qi21_dtype dt,
                           const void* q, const void* k, const void* v,
                           const int32_t* pos, const int32_t* kv_end, void* o,
                           void* k_cache, void* v_cache,
                           void* workspace, size_t workspace_bytes, void* stream);

/* Workspace bytes for qi21_attn_cached with these sizes (header included).
 * For bf16 this includes scratch for splitting the last, partial wave of
 * work units into key-range pieces (up to 512 pieces of 66 KB, and arrival
 * counters); a smaller workspace still works as long as it holds the table
 * and the rotated target keys -- the call then splits fewer units or none
 * (the no-allocation entry point below runs that way when its 32 MiB are
 * short). */
size_t qi21_attn_cached_workspace_size(int32_t B, int32_t H, int64_t P, int64_t T, qi21_dtype dt);

/*
 * qi21_attn_cached -- a later denoising step: only the T target tokens are
 * computed.  Their queries attend, with no mask (the target sees everything),
 * the cached prefix keys/values followed by their own fresh keys/values:
 * O_t = softmax(rot(Q_t) [Kc || rot(K_t)]^T / sqrt(128)) [Vc || V_t]
 * (overview card 6A and learning goals).
 *
 *   B, H, P, T  batch, heads, cached prefix length (>= 0), target tokens (>= 0).
 *   q, k, v     device [B, T, H, 128] target tensors, read.
 *   pos_tgt     device int32 [T][3]: the target rows of the position table.
 *   k_cache     device [B, H, P, 128] rotated prefix K from qi21_attn_full.
 *   v_cache     device [B, H, P, 128] prefix V from qi21_attn_full.
 *   o           device [B, T, H, 128], written.
 *   workspace   as for qi21_attn_full, sized by qi21_attn_cached_workspace_size().
 */
qi21_status qi21_attn_cached(int32_t B, int32_t H, int64_t P, int64_t T, qi21_dtype dt,
                             const void* q, const void* k, const void* v,
                             const int32_t* pos_tgt, const void* k_cache, const void* v_cache,
                             void* o, void* workspace, size_t workspace_bytes, void* stream);

/*
 * qi21_rope_table -- a request's rotation table: for each of n tokens the 64
 * (cos, sin) pairs of its axial angles pos * theta^(-2i/d_axis), computed in
 * float64 ("3A - 3D Axial RoPE (16, 56, 56)", section 1), stored rounded to
 * float32 ([n][64] float2, first) and to float16 ([n][64] half2, after it).
 * The target's positions do not change over the denoising steps, so the
 * table of its T tokens can be built once per request and handed to every
 * later step's qi21_attn_cached_tabled, whose pre-pass then computes no
 * angles; the result is bit-identical to qi21_attn_cached with the same
 * positions.
 *   pos     device [n][3] int32 (qi21_rope_positions' rows of those tokens).
 *   table   device, at least qi21_rope_table_size(n) bytes, 16-byte aligned;
 *           written (caller-owned; valid as long as the caller keeps it).
 * Returns QI21_ERR_INVALID_ARG for a bad size or pointer or a short buffer.
 */
size_t qi21_rope_table_size(int64_t n);
qi21_status qi21_rope_table(const int32_t* pos, int64_t n, void* table, size_t table_bytes, void* stream);

/*
 * qi21_attn_cached_tabled -- qi21_attn_cached with the target's rotation
 * table given (rope_table: device, qi21_rope_table of the T target tokens)
 * instead of its positions.  Every other argument, the workspace size and the
 * errors are those of qi21_attn_cached.
 */
qi21_status qi21_attn_cached_tabled(int32_t B, int32_t H, int64_t P, int64_t T, qi21_dtype dt,
                                    const void* q, const void* k, const void* v, const void* rope_table,
                                    const void* k_cache, const void* v_cache, void* o, void* workspace,
                                    size_t workspace_bytes, void* stream);

/*
 * qi21_attn_full_qknorm / qi21_attn_cached_qknorm -- the same two steps with
 * the QK-RMSNorm that precedes RoPE fused in (overview card 4A "Single-Stream
 * DiT Attention & QK-RMSNorm"; close reading section 6: norm_q and norm_k are
 * RMSNorm(head_dim = 128), applied to every head of every token before the
 * rotation).  Each Q and K head vector x becomes
 *     x / sqrt(mean(x^2) + eps) * w        (w = norm_q for Q, norm_k for K),
 * computed in fp32 from the stored values, then rotated and rounded once to
 * the storage type.  V is not normalised.
 *
 *   norm_q, norm_k  device float32 [128] each (16-byte aligned), read; both
 *                   must be given (QI21_ERR_INVALID_ARG otherwise).
 *   eps             finite, >= 0 (the pages print 1e-6 for the model's other
 *                   RMSNorms and none for these two).  An all-zero head row with
 *                   eps = 0 divides by zero, as the formula does.
 *   other arguments as for qi21_attn_full / qi21_attn_cached.
 * The cache written by qi21_attn_full_qknorm holds normalised, rotated prefix K;
 * use it with qi21_attn_cached_qknorm and the same norm_k.
 */
qi21_status qi21_attn_full_qknorm(int32_t B, int32_t H, int64_t L, int64_t P, qi21_dtype dt,
                                  const void* q, const void* k, const void* v,
                                  const int32_t* pos, const int32_t* kv_end, void* o,
                                  void* k_cache, void* v_cache,
                                  const float* norm_q, const float* norm_k, float eps,
                                  void* workspace, size_t workspace_bytes, void* stream);
qi21_status qi21_attn_cached_qknorm(int32_t B, int32_t H, int64_t P, int64_t T, qi21_dtype dt,
                                    const void* q, const void* k, const void* v,
                                    const int32_t* pos_tgt, const void* k_cache,
                                    const void* v_cache, void* o,
                                    const float* norm_q, const float* norm_k, float eps,
                                    void* workspace, size_t workspace_bytes, void* stream);

/*
 * qi21_linear -- the projections around the attention, on the tensor cores:
 *     Y = X W^T (+ b)
 * with X [M, K], W [N, K] (the nn.Linear weight layout: K contiguous) and b
 * [N], all bf16, accumulated in fp32 and rounded once to bf16.  The joint
 * attention's Q, K and V come from such projections of the hidden states and
 * its output goes through one (close reading section 6: to_q / to_k / to_v,
 * to_out); in steps 2..N only the target tokens' rows need projecting
 * (overview card 6A), which is M = B * T here.  The N output columns are cut
 * into n_out equal segments, segment i written to out[i] as a row-major
 * [M, N / n_out] tensor: with W = [W_q; W_k; W_v] and n_out = 3 one launch
 * leaves Q, K and V in the [B, T, H, 128] layout qi21_attn_* read.
 *
 *   M, N, K     sizes (>= 0; K a multiple of 8 and >= 8 unless M or N is 0).
 *   x, w        device bf16 [M, K], [N, K], 16-byte aligned, read.
 *   bias        device bf16 [N] (16-byte aligned) or NULL.
 *   out         HOST array of n_out (1..4) device pointers, each 16-byte
 *               aligned, [M, N / n_out] bf16 written; N / n_out must be a
 *               multiple of 8.
 *   workspace   device scratch of at least QI21_WORKSPACE_HEADER_BYTES (its
 *               status header, as for qi21_attn_full).
 * Returns QI21_ERR_INVALID_ARG for bad sizes, pointers or alignment before
 * enqueuing anything.
 */
qi21_status qi21_linear(int64_t M, int64_t N, int64_t K, const void* x, const void* w,
                        const void* bias, void* const* out, int32_t n_out,
                        void* workspace, size_t workspace_bytes, void* stream);

/*
 * The rest of a block of the denoising loop around the attention (overview
 * cards 4A and 5A: each of the stacked blocks runs attention, then a SwiGLU
 * feed-forward layer 3x wider than the model, each behind an RMSNorm and
 * added back to the residual stream; card 6B: the Euler step).
 *
 * qi21_linear_residual -- out = residual + alpha * (X W^T + b): qi21_linear
 *   with one output and a residual added in its epilogue (a residual
 *   connection with alpha = 1; the Euler step x + (sigma' - sigma) v with the
 *   velocity head as the projection).  residual: device bf16 [M, N], 16-byte
 *   aligned; it may be out itself (each element is read before it is
 *   written, by the same thread).  alpha finite.
 */
qi21_status qi21_linear_residual(int64_t M, int64_t N, int64_t K, const void* x, const void* w,
                                 const void* bias, const void* residual, float alpha, void* out,
                                 void* workspace, size_t workspace_bytes, void* stream);

/*
 * qi21_linear_swiglu -- out = silu(X W_gate^T + b_gate) * (X W_up^T + b_up)
 *   in one launch: the feed-forward layer's gated first half (card 5A) with
 *   the gate in the projection's epilogue.  W ([N, K]) and bias ([N]) hold
 *   the gate and up rows in alternating blocks of 128: rows 256j..256j+127 are
 *   the gates of output features 128j..128j+127, rows 256j+128..256j+255 their
 *   up projections.  N a multiple of 256; out: device bf16 [M, N / 2].  Other
 *   arguments and errors as for qi21_linear.
 */
qi21_status qi21_linear_swiglu(int64_t M, int64_t N, int64_t K, const void* x, const void* w,
                               const void* bias, void* out, void* workspace, size_t workspace_bytes,
                               void* stream);

/* qi21_rmsnorm -- y = x / sqrt(mean(x^2) + eps) * w over each of the M rows
 * of D values (bf16 x, w [D], y; D a multiple of 8; 16-byte aligned; eps
 * finite, >= 0).  y may not overlap x. */
qi21_status qi21_rmsnorm(int64_t M, int32_t D, const void* x, const void* w, float eps, void* y,
                         void* stream);

/* qi21_swiglu -- m = silu(g) * u elementwise, silu(g) = g / (1 + exp(-g)),
 * over n bf16 values (n a multiple of 8; 16-byte aligned; m may be g or u). */
qi21_status qi21_swiglu(int64_t n, const void* g, const void* u, void* m, void* stream);

/*
 * qi21_attn_cached_noalloc -- the cached step of qi21_attn_cached for callers
 * that may not allocate device memory (plugin hosts that only hand over a
 * stream and tensors, servers that reserve all memory at start-up, loops where
 * an allocation would synchronise the device).  The pages have no counterpart
 * of this entry point: it exists for such callers only.
 *
 * Same arguments and result as qi21_attn_cached minus the workspace: the
 * scratch is a 32 MiB array built into the library, held by every GPU that
 * loads the library until the process exits.  Calls needing more than that
 * (more than 32 MiB for the position table and the rotated target keys, about
 * B * H * T * 256 bytes + T * 512 bytes; the 2048^2 workload's cached step
 * needs ~200 MB) return QI21_ERR_INVALID_ARG
 * without enqueuing anything; so does every other argument error.  Each call
 * looks up the array's device address on the current device; the first call
 * on a device also loads the library's device code there, so make it before
 * any stream capture.  No call allocates (no cudaMalloc/cudaFree).  Every
 * call on a device shares the one array and the array keeps the last call's
 * contents (a call resets what must start at zero itself), so calls whose
 * kernels overlap on the GPU (other streams, other threads) race on the
 * scratch -- order them on one stream.  A device wait that runs out is
 * recorded in the array's status header and stays there until
 * qi21_workspace_status(NULL, stream) reads and clears it.
 */
qi21_status qi21_attn_cached_noalloc(int32_t B, int32_t H, int64_t P, int64_t T, qi21_dtype dt,
                                     const void* q, const void* k, const void* v,
                                     const int32_t* pos_tgt, const void* k_cache,
                                     const void* v_cache, void* o, void* stream);

/* Synchronises `stream`, then reads and clears the status word in the
 * workspace header: QI21_OK, or QI21_ERR_TIMEOUT if a device wait ran out.
 * workspace = NULL reads the built-in scratch of qi21_attn_cached_noalloc on
 * the current device. */
qi21_status qi21_workspace_status(void* workspace, void* stream);

/* ---------------------------------------------------------------------------
 * Diagnostics and test support.  Not part of the computation: a test hook for
 * the bounded waits, the message of the last error and a launch counter.
 * ------------------------------------------------------------------------- */

/* Test hook for the bounded-wait machinery: launches one CTA that waits on a
 * shared-memory barrier nobody arrives at, with a limit of `limit_ns`
 * nanoseconds (1..2e9).  The kernel records QI21_ERR_TIMEOUT in the workspace
 * header (workspace = NULL: the built-in scratch of qi21_attn_cached_noalloc)
 * and exits normally; read it with qi21_workspace_status(). */
qi21_status qi21_selftest_wait_timeout(void* workspace, int64_t limit_ns, void* stream);

const char* qi21_status_string(qi21_status s);

/* Message describing the last non-OK status returned to the calling thread. */
const char* qi21_last_error(void);

/* Number of kernel launches the calling thread has enqueued through this
 * library since it was loaded (every entry point counts its launches). */
uint64_t qi21_launch_count(void);

#ifdef __cplusplus
}
#endif

#endif /* QI21_H */
