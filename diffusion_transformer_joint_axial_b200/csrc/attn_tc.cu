// bf16 joint attention on the sm_100a tensor cores (tcgen05 + TMEM + TMA).
//
// Computes O = softmax(rot(Q) K^T / sqrt(128) + M) V for the Qwen-Image-2.1
// joint sequence ("Qwen-Image-2.1 architecture" overview, cards 3A/3C/4A/6A):
// the queries are rotated band-wise (16, 56, 56) inside the kernel right
// after their TMA load; the keys come already rotated (from the Prefix KV
// cache or the per-step pre-pass); M is the block-causal mask given by
// kv_end (allowed(i, j) <=> j < kv_end[i]) or no mask at all.
//
// Work unit: one (batch, head) and a pair of 128-row query tiles.  CTAs (one
// per SM, persistent) take units from a global counter in order of decreasing
// cost (longest-processing-time-first, decided at run time), heads grouped so
// that concurrent CTAs share K/V in L2.
// Without a mask (the cached step) every unit costs the same, and the units of
// the last, partial wave can leave most SMs idle (384 units on 148 SMs are 2.6
// waves); there the host may hand those units out as k key-range pieces each
// (chosen by a cost model): each piece writes its O / l (bf16) and its row
// max and row sum to the workspace, and the epilogue warp that finishes the
// last piece of a unit's rows (an arrival counter, no waiting) merges them.
// For each query tile only the key tiles that start below the tile's largest
// kv_end are visited: every visibility bound is a prefix of the keys, so
// fully masked tiles are skipped and never loaded; only tiles that straddle
// a row's bound (the diagonal of the text block, ragged ends) are masked
// element-wise.
//
// Warp roles (512 threads, registers rebalanced with setmaxnreg):
//   warps 0-3   query tile 0: rotates each item's query rows in shared memory
//               once the tile lands (one row per thread, its cos/sin chunks
//               requested before the wait), then the softmax (thread = row =
//               TMEM lane), 160 regs
//   warps 4-7   the same for query tile 1, 160 regs
//   warps 8-11  epilogue, 80 regs: drains each item's O (O / l -> bf16 ->
//               TMA store, or a piece's partial result and the merge) as soon
//               as its MMAs are done
//   warp  12    TMA producer of Q tiles and of the key tiles, 112 regs
//   warp  13    TMEM allocator and tcgen05.mma issuer, 112 regs
//   warp  14    TMA producer of the value tiles, 112 regs
//   warp  15    idle, 112 regs
// Key and value tiles share a two-slot ring: slot t holds key tile t and
// value tile t - 1 (numbered over the CTA's whole sequence of items), the two
// tiles one step of the MMA warp reads, so each step waits on one barrier
// and releases one (a unit's last slot, whose key tile is the next unit's
// first, is released after that unit's first S MMAs).
// TMEM (512 columns): S0 | S1 | O0 | O1, 128 fp32 columns each; P (bf16,
// packed in pairs) overwrites the upper 64 columns of its S and is the A
// operand of the P*V MMA, so P never touches shared memory.  P is released in
// two halves (keys 0-63, then 64-127) so the first half of P*V runs while the
// softmax finishes the second.
// Issue order per key tile n: PV0(n), S0(n+1), PV1(n), S1(n+1): while one
// softmax group works the tensor core runs the other tile's MMAs.
// The softmax keeps its dependency chains short (eight partial row sums, an
// eight-chain row max): on B200 a lone softmax warp per SMSP is bound by
// instruction latency more than by the MUFU exp2 rate.
// Online softmax uses a lazy rescale: O and l are rescaled only when a row
// maximum grows by more than 2^8, which keeps every P <= 256.  Each tile's
// row maximum is taken before its exponentials.
#include <cudaTypedefs.h>
#include <cuda_fp16.h>
#include <math.h>

#include "qi21_device.cuh"
#include "qi21_internal.h"

namespace qi21 {

namespace tc {

constexpr int BM = 128;  // query rows per tile
constexpr int BN = 128;  // keys per tile
constexpr int kStages = 2;
constexpr int kTileBytes = BM * kHeadDim * 2;  // 32 KB: two 64-column SW128 halves
constexpr int kHalfBytes = kTileBytes / 2;
constexpr int kThreads = 512;
constexpr int kWarpEpi = 8;  // first epilogue warp
constexpr int kWarpLoad = 12;   // Q and K tiles
constexpr int kWarpMma = 13;
constexpr int kWarpLoadV = 14;  // V tiles
constexpr uint32_t kTmemCols = 512;
// setmaxnreg budget: 128 x (160 + 160 + 80 + 112) = 65536 = 512 threads x 128.
constexpr int kRegsSoftmax = 160;
constexpr int kRegsEpilogue = 80;
constexpr int kRegsOther = 112;
static_assert(128 * (2 * kRegsSoftmax + kRegsEpilogue + kRegsOther) == 65536, "register split");

// Instruction descriptor of tcgen05.mma kind::f16: fp32 accumulate (bit 4),
// A and B bf16 (bits 7, 10), N >> 3 at bit 17, M >> 4 at bit 24; bit 16 marks
// B as MN-major (V: head dim contiguous).
constexpr uint32_t kIdescS = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) |
                             ((uint32_t)(BM >> 4) << 24);
constexpr uint32_t kIdescPV = (1u << 4) | (1u << 7) | (1u << 10) | (1u << 16) |
                              ((uint32_t)(kHeadDim >> 3) << 17) | ((uint32_t)(BM >> 4) << 24);

// P (bf16 pairs, 64 columns) lives in the upper half of its S region: the S
// values there (keys 64-127) are already in registers when P is written, and
// the lower half (keys 0-63) stays intact in TMEM until the next S MMA.
constexpr uint32_t kPCol = 64;

// log2(e) / sqrt(128) and the lazy-rescale threshold (8 in log2 units).
constexpr float kScaleLog2 = 0.12751743082459868f;
constexpr float kRescaleRaw = 8.0f / kScaleLog2;

struct Params {
  CUtensorMap tm_q;
  CUtensorMap tm_o;  // the output: 64 columns x 32 rows boxes (one epilogue warp's rows)
  CUtensorMap tm_k0, tm_k1, tm_v0, tm_v1;
  int32_t k0_tok, k1_tok, v0_tok, v1_tok;  // 1: token-major coords, 0: head-major
  int32_t B, H, Lq, n0, n1;
  int32_t nqp;        // query-tile pairs per (batch, head)
  int32_t num_units;  // B * H * nqp
  // Tail split: work items [0, head_units) are whole units; the remaining
  // num_units - head_units units (the last, partial wave) are handed out as
  // split_k key-range pieces each, so num_items = head_units + (num_units -
  // head_units) * split_k.  split_k == 1: every item is a whole unit.
  int32_t head_units, split_k, num_items;
  // 1: source-1 keys arrive unrotated and the epilogue warps rotate each of
  // their tiles (row r of source 1 uses table row ktab1 + r) before the MMA
  // warp may read it (k_rot); whole units only
  int32_t rot_k1, ktab1;
  uint4* part;         // [slot][tile][4 row quarters][16 chunks][32 rows]: a piece's O / l, 8 bf16 per chunk
  float2* part_ml;     // [slot][tile][128 rows]: the piece's (row max, row sum)
  uint32_t* part_cnt;  // [tail unit][tile][4 row quarters]: pieces finished (zeroed by the pre-pass)
  const uint4* table;  // per token 16 x (4 x half2 (cos, sin)): one 16-byte load per 8 dims
  const int32_t* kv_end;
  __nv_bfloat16* o;
  uint32_t* status;
  uint32_t* unit_counter;  // zeroed by the pre-pass kernel before this launch
  const float* q_norm_w;   // [128] QK-RMSNorm weight of Q, or null
  float norm_eps;
};

constexpr int kSchedSlots = 4;
// Threads that read every scheduled unit: warps 0-14 (warp 15 idles).
constexpr uint32_t kSchedReaders = 15 * 32;

struct __align__(1024) Smem {
  uint8_t q[2][kTileBytes];
  uint8_t k[kStages][kTileBytes];
  uint8_t v[kStages][kTileBytes];
  // 64 columns x 128 rows of O (bf16, 128B-swizzled): each epilogue warp
  // stages its 32 rows (4 KB) here for its own TMA store
  uint8_t ostage[kHalfBytes];
  float row_l[2][2][BM];  // [unit parity][tile][row]: softmax -> epilogue
  float row_m[2][2][BM];  // the rows' maxima (read for the pieces of a split unit)
  alignas(16) float qnw[kHeadDim];  // QK-RMSNorm weight of Q (when given)
  int32_t sched_unit[kSchedSlots];  // units handed out by the K producer (-1: none left)
  uint64_t q_full[2], q_rot[2], q_empty[2];
  // ring slot t holds key tile t and value tile t - 1 (global indices, in
  // stage t % kStages); full: both producers' loads landed, empty: the MMA
  // warp has read both tiles
  uint64_t slot_full[kStages], slot_empty[kStages];
  uint64_t k_rot[kStages];  // source-1 rotation done (rot_k1 only)
  uint64_t s_full[2], p_half[2], p_full[2], o_done[2], o_free[2];
  // [item parity][tile]: the epilogue can fall an item behind (while it
  // merges a split unit, say), and a tile with a single key tile can then
  // finish its softmax twice before the epilogue waits; one barrier per item
  // parity keeps the phases apart
  uint64_t l_ready[2][2];
  // [tile][epilogue warp]: bulk loads of the pieces to merge after a CTA's last item
  uint64_t mrg[2][4];
  uint64_t sched_full[kSchedSlots], sched_empty[kSchedSlots];
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
};

// Shared-memory descriptor of a 128B-swizzled operand (version 1, layout 2).
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr & 0x3FFFFu) >> 4);
  d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
  d |= (uint64_t)1 << 46;
  d |= (uint64_t)2 << 61;
  return d;
}
// K-major operands (Q, K tiles): the 16-element k-step kk lives in half kk/4 at
// byte offset 32*(kk%4) of each 128-byte row; 8-row groups are 1024 B apart
// (SBO), LBO unused.  MN-major operand (V tile, rows = keys): k-step kk is 16
// key rows = 2048 B further; the two 64-column halves are 16 KB apart (LBO).

__device__ __forceinline__ void setmaxnreg_inc_softmax() {
  asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegsSoftmax));
}
__device__ __forceinline__ void setmaxnreg_dec_epilogue() {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsEpilogue));
}
__device__ __forceinline__ void setmaxnreg_dec_other() {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsOther));
}

__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

struct Unit {
  int b, h, row0;
  int N[2];   // key tiles of each query tile in this item
  int kb;     // first key tile of the item (a piece of a split unit starts past 0)
  int slot;   // partial-result slot of a piece, -1 for a whole unit
  int grp;    // tail unit of a piece (its arrival counters)
};

__device__ __forceinline__ int ceil_div(int a, int b) { return (a + b - 1) / b; }

// Key tiles that start below kv_hi (keys are [source 0 rows || source 1 rows]).
__device__ __forceinline__ int tiles_below(const Params& p, int kv_hi) {
  const int nt0 = ceil_div(p.n0, BN);
  if (kv_hi <= p.n0) return ceil_div(kv_hi, BN);
  return nt0 + min(ceil_div(kv_hi - p.n0, BN), ceil_div(p.n1, BN));
}

// Units run in groups of kGroup query-tile pairs: group by group from the end
// of the sequence (kv_end is non-decreasing, so the most expensive pairs come
// first: longest-processing-time order), and inside a group head by head.  The
// CTAs running at the same time then share the K/V of a few heads instead of
// streaming every head's K/V through L2 at once (measured on the 2048^2
// workload: 14-15 % faster, the saved DRAM traffic letting the power-capped
// clock run higher).
constexpr int kGroup = 16;

// Most pieces a tail unit is split into.
constexpr int kMaxSplit = 4;

__device__ __forceinline__ Unit decode_unit(const Params& p, int u) {
  Unit U;
  const int bh_count = p.B * p.H;
  const int span = bh_count * kGroup;
  const int full = p.nqp / kGroup;
  int bh, qi;
  if (u < full * span) {
    const int r = u % span;
    bh = r / kGroup;
    qi = (u / span) * kGroup + r % kGroup;
  } else {
    const int rem = p.nqp - full * kGroup;
    const int r = u - full * span;
    bh = r / rem;
    qi = full * kGroup + r % rem;
  }
  const int qp = p.nqp - 1 - qi;
  U.b = bh / p.H;
  U.h = bh % p.H;
  U.row0 = qp * 2 * BM;
  for (int s = 0; s < 2; ++s) {
    const int first = U.row0 + s * BM;
    if (first >= p.Lq) {
      U.N[s] = 0;
      continue;
    }
    const int last = min(first + BM - 1, p.Lq - 1);
    const int kv_hi = p.kv_end ? min(p.kv_end[last], p.n0 + p.n1) : p.n0 + p.n1;
    U.N[s] = tiles_below(p, kv_hi);
  }
  U.kb = 0;
  U.slot = -1;
  U.grp = 0;
  return U;
}

// Work item w.  Piece i of a split tail unit covers key tiles
// [i N / k, (i+1) N / k) of both query tiles; a tail unit whose tiles differ in
// length or that has fewer than k key tiles goes whole as its piece 0, and its
// other pieces are empty items (N = 0 for both tiles: every role skips them).
__device__ __forceinline__ Unit decode_item(const Params& p, int w) {
  int u = w, g = 0, i = -1;
  if (w >= p.head_units) {
    const int j = w - p.head_units;
    g = j / p.split_k;
    i = j - g * p.split_k;
    u = p.head_units + g;
  }
  Unit U = decode_unit(p, u);
  if (i >= 0) {
    const int N = U.N[0];
    if (U.N[1] == N && N >= p.split_k) {
      const int kb = (int)((int64_t)i * N / p.split_k);
      const int ke = (int)((int64_t)(i + 1) * N / p.split_k);
      U.kb = kb;
      U.N[0] = U.N[1] = ke - kb;
      U.slot = w - p.head_units;
      U.grp = g;
    } else if (i > 0) {
      U.N[0] = U.N[1] = 0;
    }
  }
  return U;
}

// The token's sixteen 16-byte (cos, sin) chunks (fp16 pairs), all loads in
// flight at once: one round trip to L2, issued before the query tile lands.
__device__ __forceinline__ void load_table_row(const uint4* cs, uint4 (&tb)[16]) {
#pragma unroll
  for (int i = 0; i < 16; ++i) tb[i] = __ldg(cs + i);
}

// One 16-byte chunk (four adjacent pairs (2m, 2m+1)) turned by its four
// (cos, sin) fp16 pairs, rounded once to bf16.
__device__ __forceinline__ void turn_chunk(uint4& x, const uint4& tb) {
  const __half2* tc = reinterpret_cast<const __half2*>(&tb);
  uint32_t* w = reinterpret_cast<uint32_t*>(&x);
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const float2 xv = unpack_bf16x2(w[e]);
    const float2 r = __half22float2(tc[e]);  // (cos, sin) of pair e of the chunk
    w[e] = pack_bf16x2(fmaf(xv.x, r.x, -xv.y * r.y), fmaf(xv.x, r.y, xv.y * r.x));
  }
}
// Chunk c of row t of a 128B-swizzled 128 x 128 tile (two 64-column halves).
__device__ __forceinline__ uint4* tile_chunk(uint8_t* row, int c, int t) {
  return reinterpret_cast<uint4*>(row + (c >> 3) * kHalfBytes + (((c & 7) ^ (t & 7)) << 4));
}

// Rotation of one query row in its 128B-swizzled tile (row t): each adjacent
// pair (2m, 2m+1) turned by the token's (cos, sin), rounded once to bf16.
__device__ __forceinline__ void rotate_q_row(uint8_t* qrow, const uint4 (&tb)[16], int t) {
#pragma unroll
  for (int c = 0; c < 16; ++c) {
    uint4* ptr = tile_chunk(qrow, c, t);
    uint4 x = *ptr;
    turn_chunk(x, tb[c]);
    *ptr = x;
  }
}

// The same for one row of an unrotated key tile, with the table read two
// chunks at a time (the epilogue warps that do it run on 80 registers).
__device__ __forceinline__ void rotate_k_row(uint8_t* krow, const uint4* cs, int t) {
#pragma unroll
  for (int c0 = 0; c0 < 16; c0 += 2) {
    uint4 tb[2], x[2];
#pragma unroll
    for (int i = 0; i < 2; ++i) tb[i] = __ldg(cs + c0 + i);
#pragma unroll
    for (int i = 0; i < 2; ++i) x[i] = *tile_chunk(krow, c0 + i, t);
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      turn_chunk(x[i], tb[i]);
      *tile_chunk(krow, c0 + i, t) = x[i];
    }
  }
}

// QK-RMSNorm + rotation of one query row: the row's mean square (fp32, from
// the bf16 values), then each adjacent pair (2m, 2m+1) scaled by
// rsqrt(mean square + eps) and the weight and rotated by the token's
// (cos, sin), rounded once to bf16.
__device__ __forceinline__ void norm_rotate_q_row(uint8_t* qrow, const uint4 (&tb)[16], int t,
                                                  const float* wn, float eps) {
  float ss0 = 0.f, ss1 = 0.f;
#pragma unroll 4
  for (int c = 0; c < 16; ++c) {
    const uint4 x =
        *reinterpret_cast<const uint4*>(qrow + (c >> 3) * kHalfBytes + (((c & 7) ^ (t & 7)) << 4));
    const uint32_t* w = reinterpret_cast<const uint32_t*>(&x);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 v = unpack_bf16x2(w[e]);
      ss0 = fmaf(v.x, v.x, ss0);
      ss1 = fmaf(v.y, v.y, ss1);
    }
  }
  const float rs = rsqrtf((ss0 + ss1) * (1.f / kHeadDim) + eps);
#pragma unroll
  for (int c = 0; c < 16; ++c) {
    uint4* ptr = reinterpret_cast<uint4*>(qrow + (c >> 3) * kHalfBytes + (((c & 7) ^ (t & 7)) << 4));
    uint4 x = *ptr;
    const float4 w0 = *reinterpret_cast<const float4*>(wn + 8 * c);
    const float4 w1 = *reinterpret_cast<const float4*>(wn + 8 * c + 4);
    const float wv[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
    const __half2* tc = reinterpret_cast<const __half2*>(&tb[c]);
    uint32_t* w = reinterpret_cast<uint32_t*>(&x);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 v = unpack_bf16x2(w[e]);
      const float2 r = __half22float2(tc[e]);  // (cos, sin)
      const float x0 = v.x * rs * wv[2 * e], x1 = v.y * rs * wv[2 * e + 1];
      w[e] = pack_bf16x2(fmaf(x0, r.x, -x1 * r.y), fmaf(x0, r.y, x1 * r.x));
    }
    *ptr = x;
  }
}

// Key tile n: first key index j0 (in the joint key order), key count, source
// and first row inside the source.
struct KTile {
  int j0, cnt, src, row;
};
__device__ __forceinline__ KTile key_tile(const Params& p, int n) {
  KTile t;
  const int nt0 = ceil_div(p.n0, BN);
  if (n < nt0) {
    t.src = 0;
    t.row = n * BN;
    t.cnt = min(BN, p.n0 - t.row);
    t.j0 = t.row;
  } else {
    t.src = 1;
    t.row = (n - nt0) * BN;
    t.cnt = min(BN, p.n1 - t.row);
    t.j0 = p.n0 + t.row;
  }
  return t;
}

__device__ __forceinline__ void load_kv_tile(const CUtensorMap* map, int tok_major, uint32_t dst,
                                             uint32_t bar, int row, int h, int b) {
  for (int half = 0; half < 2; ++half) {
    if (tok_major)
      tma_load_4d(dst + half * kHalfBytes, map, bar, half * 64, h, row, b);
    else
      tma_load_4d(dst + half * kHalfBytes, map, bar, half * 64, row, h, b);
  }
}

// The start-address field of a descriptor is (address >> 4) in its low 14
// bits; shared-memory addresses stay below 256 KB, so moving a descriptor by a
// byte offset is a 32-bit add of offset >> 4 to its low word that never
// carries out of the field.  The MMA warp shares an SMSP with two softmax
// warps, which then reach their barriers last: every instruction it saves
// (this add, the per-stage descriptors built once) shortens the step
// (measured 1-2 % on every workload).
__device__ __forceinline__ uint64_t desc_lo_add(uint64_t d, uint32_t off) {
  const uint32_t lo = (uint32_t)d + off, hi = (uint32_t)(d >> 32);
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "r"(lo), "r"(hi));
  return r;
}
__device__ __forceinline__ void issue_s(uint32_t tmem_s, uint64_t qdesc, uint64_t kdesc) {
#pragma unroll
  for (int kk = 0; kk < kHeadDim / 16; ++kk) {
    const uint32_t off = (uint32_t)(((kk >> 2) * kHalfBytes + (kk & 3) * 32) >> 4);
    mma_ss(tmem_s, desc_lo_add(qdesc, off), desc_lo_add(kdesc, off), kIdescS, kk > 0);
  }
}
__device__ __forceinline__ void issue_pv(uint32_t tmem_o, uint32_t tmem_p, uint64_t vdesc, int kk0,
                                         bool first) {
#pragma unroll
  for (int kk = kk0; kk < kk0 + 4; ++kk)
    mma_ts(tmem_o, tmem_p + kk * 8, desc_lo_add(vdesc, (uint32_t)((kk * 2048) >> 4)), kIdescPV,
           (!first || kk > 0) ? 1u : 0u);
}

// Exponentials and bf16 packing of the 32 column pairs of one half of the
// row (pairs j0 .. j0+31), stored to TMEM in two 16-column pieces at P's
// columns (pair j -> column 64 + j of the S region): x = s * log2(e)/sqrt(128) -
// m * log2(e)/sqrt(128) (scalar FMAs: the packed fp32x2 forms have a ~26-cycle
// latency that lands in front of every exp2), exp2 on MUFU, the row sum in
// eight partial sums (the adds have a long latency: a single chain would
// serialise the loop).  The stores are not waited for here.
__device__ __forceinline__ void exp_pack_half(const float* sv, int j0, float mc, float (&acc)[8],
                                              uint32_t tS) {
#pragma unroll
  for (int q = 0; q < 2; ++q) {
    uint32_t pk[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      const int c = 2 * (j0 + 16 * q + j);
      const float e0 = ex2_approx(fmaf(sv[c], kScaleLog2, -mc));
      const float e1 = ex2_approx(fmaf(sv[c + 1], kScaleLog2, -mc));
      acc[(2 * j) & 7] += e0;
      acc[(2 * j + 1) & 7] += e1;
      pk[j] = pack_bf16x2(e0, e1);
    }
    tmem_st16(tS + kPCol + j0 + 16 * q, pk);
  }
}

// Folds the S values [c0, 128) into the eight maximum chains, then reduces them.
__device__ __forceinline__ float row_max_from(const float* sv, int c0, float (&mxc)[8]) {
#pragma unroll
  for (int c = c0; c < BN; c += 16) {
#pragma unroll
    for (int i = 0; i < 8; ++i) mxc[i] = fmax3(mxc[i], sv[c + i], sv[c + i + 8]);
  }
  return fmaxf(fmax3(mxc[0], mxc[1], mxc[2]), fmaxf(fmax3(mxc[3], mxc[4], mxc[5]), fmaxf(mxc[6], mxc[7])));
}

// O / l -> bf16 of one whole unit's tile, this warp's 32 rows, in two
// 64-column halves.  Each warp stages its own rows in shared memory (128B-
// swizzled, the TMA layout) and writes them with one TMA store (rows past Lq
// are clipped; a box wholly past Lq is not issued).  O's TMEM columns are
// released as soon as the second half has been read, long before the stores
// finish.  No barrier spans warps, so a warp that gives up on a timed-out
// wait cannot hold the others.
__device__ __forceinline__ void store_tile(Smem& S, const Params& p, uint32_t tO, float inv,
                                           uint8_t* stage, int lane, int s, int h, int b,
                                           int row_first) {
  for (int hh = 0; hh < 2; ++hh) {
    if (lane == 0) bulk_wait_read_all();  // this warp's slice of the stage is free
    __syncwarp();
#pragma unroll 1
    for (int c = 0; c < 2; ++c) {
      uint32_t orow[32];
      tmem_ld32(tO + 64 * hh + 32 * c, orow);
      tmem_wait_ld();
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        uint32_t w[4];
#pragma unroll
        for (int i = 0; i < 4; ++i)
          w[i] = pack_bf16x2(__uint_as_float(orow[8 * e + 2 * i]) * inv,
                             __uint_as_float(orow[8 * e + 2 * i + 1]) * inv);
        const int chunk = 4 * c + e;  // 16-byte chunk of the 128-byte row
        *reinterpret_cast<uint4*>(stage + lane * 128 + ((chunk ^ (lane & 7)) << 4)) =
            make_uint4(w[0], w[1], w[2], w[3]);
      }
    }
    if (hh == 1) {
      tc_fence_before();
      mbar_arrive(smem_u32(&S.o_free[s]));
    }
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0 && row_first < p.Lq) {
      tma_store_4d(&p.tm_o, smem_u32(stage), 64 * hh, h, row_first, b);
      bulk_commit_group();
    }
    __syncwarp();
  }
}

// Dynamic schedule: the K-producer warp takes the next unit from a global
// counter (units are numbered in decreasing-cost order) and publishes it in a
// shared-memory ring; every role reads the same sequence through next_unit().
__device__ __forceinline__ void publish_unit(Smem& S, const Params& p, uint32_t sc, bool leader,
                                             volatile int* abort, bool& ok) {
  const int slot = sc % kSchedSlots;
  ok = ok && __all_sync(0xffffffffu,
                        mbar_wait(smem_u32(&S.sched_empty[slot]), ((sc / kSchedSlots) & 1u) ^ 1u,
                                  abort, p.status, 0x500));
  if (ok && leader) {
    const uint32_t u = atomicAdd(p.unit_counter, 1u);
    S.sched_unit[slot] = u < (uint32_t)p.num_items ? (int32_t)u : -1;
    mbar_arrive(smem_u32(&S.sched_full[slot]));
  }
  __syncwarp();
}
__device__ __forceinline__ int next_unit(Smem& S, const Params& p, uint32_t& sc, volatile int* abort,
                                         bool& ok) {
  const int slot = sc % kSchedSlots;
  ok = ok && __all_sync(0xffffffffu,
                        mbar_wait(smem_u32(&S.sched_full[slot]), (sc / kSchedSlots) & 1u, abort,
                                  p.status, 0x510));
  int u = -1;
  if (ok) {
    u = *reinterpret_cast<volatile int32_t*>(&S.sched_unit[slot]);
    mbar_arrive(smem_u32(&S.sched_empty[slot]));
  }
  ++sc;
  return ok ? u : -1;
}

// Merge of the k pieces of one warp's 32 rows of a split unit's query tile:
// O = sum_i a_i (O_i / l_i) with a_i the piece's share of the row sum,
// a_i = 2^((m_i - M) c) l_i / sum_j 2^((m_j - M) c) l_j, written through the
// warp's slice of the output stage.  `src` holds the pieces' rows, 8 KB per
// piece ([16 chunks][32 rows] of 8 bf16) and piece_stride bytes apart, in
// global memory (read through L2) or, after the CTA's last item, copied into
// shared memory.
template <bool kShared>
__device__ __forceinline__ void merge_pieces(const Params& p, const uint8_t* src, size_t piece_stride,
                                             const float (&a)[kMaxSplit], uint8_t* stage, int lane, int h,
                                             int b, int row_first) {
  for (int hh = 0; hh < 2; ++hh) {
    if (lane == 0) bulk_wait_read_all();
    __syncwarp();
#pragma unroll 2
    for (int ch = 0; ch < 8; ++ch) {
      float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int i = 0; i < kMaxSplit; ++i) {
        if (i < p.split_k) {
          const uint4* ptr = reinterpret_cast<const uint4*>(src + i * piece_stride + (8 * hh + ch) * 512) + lane;
          const uint4 x = kShared ? *ptr : __ldcg(ptr);
          const uint32_t* xw = reinterpret_cast<const uint32_t*>(&x);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 v = unpack_bf16x2(xw[e]);
            acc[2 * e] = fmaf(a[i], v.x, acc[2 * e]);
            acc[2 * e + 1] = fmaf(a[i], v.y, acc[2 * e + 1]);
          }
        }
      }
      *reinterpret_cast<uint4*>(stage + lane * 128 + ((ch ^ (lane & 7)) << 4)) =
          make_uint4(pack_bf16x2(acc[0], acc[1]), pack_bf16x2(acc[2], acc[3]),
                     pack_bf16x2(acc[4], acc[5]), pack_bf16x2(acc[6], acc[7]));
    }
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0 && row_first < p.Lq) {
      tma_store_4d(&p.tm_o, smem_u32(stage), 64 * hh, h, row_first, b);
      bulk_commit_group();
    }
    __syncwarp();
  }
}

// Shares a_i of the k pieces of row t (see merge_pieces).
__device__ __forceinline__ void piece_weights(const Params& p, int slot0, int s, int t, float (&a)[kMaxSplit]) {
  float m[kMaxSplit], l[kMaxSplit];
  float mx = -INFINITY;
#pragma unroll
  for (int i = 0; i < kMaxSplit; ++i) {
    m[i] = -INFINITY;
    l[i] = 0.f;
    if (i < p.split_k) {
      const float2 ml = __ldcg(p.part_ml + ((size_t)(slot0 + i) * 2 + s) * BM + t);
      m[i] = ml.x;
      l[i] = ml.y;
      mx = fmaxf(mx, ml.x);
    }
  }
  float tot = 0.f;
#pragma unroll
  for (int i = 0; i < kMaxSplit; ++i) {
    a[i] = i < p.split_k ? ex2_approx((m[i] - mx) * kScaleLog2) * l[i] : 0.f;
    tot += a[i];
  }
  const float inv = 1.f / tot;
#pragma unroll
  for (int i = 0; i < kMaxSplit; ++i) a[i] *= inv;
}

// Epilogue warps of a call whose source-1 keys arrive unrotated (rot_k1):
// besides draining O they rotate every source-1 key tile in place, one row
// per thread from the query table, and arrive on k_rot for every key tile
// (source 0 is already rotated), which the MMA warp waits on as well as on
// the slot.  An item's O is drained once the next item's first two key tiles
// are done, so those are ready when the item's last P*V completes.  Whole
// units only (the launcher does not split such a call).
__device__ __forceinline__ void rotk1_epilogue(Smem& S, const Params& p, uint32_t tmem,
                                               volatile int* abort_flag, int warp, int lane) {
  const int t = threadIdx.x & 127;
  const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
  uint8_t* stage = S.ostage + (warp & 3) * 32 * 128;
  uint32_t kc = 0, cnt[2] = {0, 0}, sc = 0;
  bool ok = true, have_prev = false;
  Unit prev = {};
  auto drain = [&](const Unit& d) {
    for (int s = 0; s < 2 && ok; ++s) {
      if (d.N[s] == 0) continue;
      const uint32_t par = cnt[s] & 1u;
      const uint32_t lpar = (cnt[s] >> 1) & 1u;
      ++cnt[s];
      ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&S.l_ready[par][s]), lpar, abort_flag,
                                            p.status, 0x440 | s));
      if (!ok) break;
      ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&S.o_done[s]), par, abort_flag,
                                            p.status, 0x450 | s));
      if (!ok) break;
      tc_fence_after();
      store_tile(S, p, tmem + lane_base + 256 + s * kHeadDim, 1.f / S.row_l[par][s][t], stage, lane,
                 s, d.h, d.b, d.row0 + s * BM + (warp & 3) * 32);
    }
  };
  while (ok) {
    const int u = next_unit(S, p, sc, abort_flag, ok);
    if (u < 0) break;
    const Unit U = decode_item(p, u);
    const int N = max(U.N[0], U.N[1]);
    for (int n = 0; n < N && ok; ++n) {
      const KTile kt = key_tile(p, U.kb + n);
      const int st = kc % kStages;
      ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&S.slot_full[st]), (kc / kStages) & 1u, abort_flag,
                                            p.status, 0x430 | st));
      if (!ok) break;
      ++kc;
      // rows past the source's end were zero-filled by the load: left alone
      if (kt.src == 1 && kt.row + t < p.n1)
        rotate_k_row(S.k[st] + t * 128, p.table + (size_t)(p.ktab1 + kt.row + t) * 16, t);
      fence_proxy_async_smem();
      mbar_arrive(smem_u32(&S.k_rot[st]));
      if (have_prev && n == min(1, N - 1)) {
        drain(prev);
        have_prev = false;
      }
    }
    if (!ok) break;
    if (have_prev) drain(prev);  // an item without key tiles
    prev = U;
    have_prev = true;
  }
  if (ok && have_prev) drain(prev);
}

// kRotK1: source-1 keys arrive unrotated (Params::rot_k1); a separate
// instantiation, so the default kernel carries none of its checks.
template <bool kRotK1>
__global__ void __launch_bounds__(kThreads, 1) attn_tc_kernel(const __grid_constant__ Params p) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  Smem& S = *reinterpret_cast<Smem*>(smem_raw + (((raw + 1023u) & ~1023u) - raw));
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  volatile int* abort_flag = &S.abort_flag;

  if (threadIdx.x == 0) {
    for (int s = 0; s < 2; ++s) {
      mbar_init(smem_u32(&S.q_full[s]), 1);
      mbar_init(smem_u32(&S.q_rot[s]), BM);
      mbar_init(smem_u32(&S.q_empty[s]), 1);
      mbar_init(smem_u32(&S.s_full[s]), 1);
      mbar_init(smem_u32(&S.p_half[s]), BM);
      mbar_init(smem_u32(&S.p_full[s]), BM);
      mbar_init(smem_u32(&S.o_done[s]), 1);
      mbar_init(smem_u32(&S.o_free[s]), BM);
      mbar_init(smem_u32(&S.l_ready[0][s]), BM);
      mbar_init(smem_u32(&S.l_ready[1][s]), BM);
      for (int w = 0; w < 4; ++w) mbar_init(smem_u32(&S.mrg[s][w]), 1);
    }
    for (int s = 0; s < kStages; ++s) {
      mbar_init(smem_u32(&S.slot_full[s]), 2);  // the K and the V producer
      mbar_init(smem_u32(&S.slot_empty[s]), 1);
      mbar_init(smem_u32(&S.k_rot[s]), BM);
    }
    for (int s = 0; s < kSchedSlots; ++s) {
      mbar_init(smem_u32(&S.sched_full[s]), 1);
      mbar_init(smem_u32(&S.sched_empty[s]), kSchedReaders);
    }
    mbar_init(smem_u32(&S.drain), 1);
    S.abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kWarpMma) {
    tmem_alloc(smem_u32(&S.tmem_base), kTmemCols);
    tmem_relinquish();
  }
  if (p.q_norm_w != nullptr && threadIdx.x < kHeadDim) S.qnw[threadIdx.x] = p.q_norm_w[threadIdx.x];
  if (warp == kWarpLoad && lane == 0) {
    tma_prefetch_desc(&p.tm_q);
    tma_prefetch_desc(&p.tm_o);
    tma_prefetch_desc(&p.tm_k0);
    tma_prefetch_desc(&p.tm_v0);
    if (p.n1 > 0) {
      tma_prefetch_desc(&p.tm_k1);
      tma_prefetch_desc(&p.tm_v1);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = S.tmem_base;

  if (warp >= kWarpLoad) {
    setmaxnreg_dec_other();
    if (warp == kWarpLoad || warp == kWarpLoadV) {
      // --------------------------------------------------------- producers
      // Warp 12 loads Q and the key tiles, warp 14 the value tiles; both
      // count into the slot's barrier.
      const bool do_qk = warp == kWarpLoad;
      uint32_t sc = 0;
      // The whole warp runs the loop (every value is warp-uniform, so the
      // TMA operands stay in uniform registers); one elected lane issues.
      const bool leader = elect_one_sync();
      uint32_t kc = 0, vc = 0, ql[2] = {0, 0}, qi[2] = {0, 0};
      bool ok = true;
      // Ring slot t holds key tile t and value tile t - 1 (global indices):
      // the MMA warp uses both in the same step, and one barrier counts both
      // producers.  Slot 0 has no value tile: the V producer arrives alone.
      if (!do_qk && leader) mbar_arrive(smem_u32(&S.slot_full[0]));
      __syncwarp();
      while (ok) {
        if (do_qk) publish_unit(S, p, sc, leader, abort_flag, ok);
        const int u = next_unit(S, p, sc, abort_flag, ok);
        if (u < 0) break;
        const Unit U = decode_item(p, u);
        for (int s = 0; s < 2 && ok && do_qk; ++s) {
          if (U.N[s] == 0) continue;
          // the MMA warp releases Q_s once per unit that used it
          ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&S.q_empty[s]), (ql[s] & 1u) ^ 1u,
                                                abort_flag, p.status, 0x100 | s));
          ++ql[s];
          if (ok) ++qi[s];  // Q loads issued into buffer s
          if (ok && leader) {
            const uint32_t bar = smem_u32(&S.q_full[s]);
            mbar_arrive_expect_tx(bar, kTileBytes);
            const uint32_t dst = smem_u32(S.q[s]);
            tma_load_4d(dst, &p.tm_q, bar, 0, U.h, U.row0 + s * BM, U.b);
            tma_load_4d(dst + kHalfBytes, &p.tm_q, bar, 64, U.h, U.row0 + s * BM, U.b);
          }
        }
        const int N = max(U.N[0], U.N[1]);
        for (int n = 0; n < N && ok; ++n) {
          const KTile t = key_tile(p, U.kb + n);
          if (do_qk) {
            const int st = kc % kStages;
            ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&S.slot_empty[st]), ((kc / kStages) & 1u) ^ 1u,
                                                  abort_flag, p.status, 0x110 | st));
            if (!ok) break;
            if (leader) {
              const uint32_t bar = smem_u32(&S.slot_full[st]);
              mbar_arrive_expect_tx(bar, kTileBytes);
              load_kv_tile(t.src ? &p.tm_k1 : &p.tm_k0, t.src ? p.k1_tok : p.k0_tok,
                           smem_u32(S.k[st]), bar, t.row, U.h, U.b);
            }
            ++kc;
          } else {
            const uint32_t slot = vc + 1;
            const int st = slot % kStages;
            ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&S.slot_empty[st]), ((slot / kStages) & 1u) ^ 1u,
                                                  abort_flag, p.status, 0x120 | st));
            if (!ok) break;
            if (leader) {
              const uint32_t bar = smem_u32(&S.slot_full[st]);
              mbar_arrive_expect_tx(bar, kTileBytes);
              load_kv_tile(t.src ? &p.tm_v1 : &p.tm_v0, t.src ? p.v1_tok : p.v0_tok,
                           smem_u32(S.v[st]), bar, t.row, U.h, U.b);
            }
            ++vc;
          }
        }
      }
      // The last slot holds the last value tile and no key tile.
      if (ok && do_qk) {
        const int st = kc % kStages;
        ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&S.slot_empty[st]), ((kc / kStages) & 1u) ^ 1u,
                                              abort_flag, p.status, 0x130 | st));
        if (ok && leader) mbar_arrive(smem_u32(&S.slot_full[st]));
        __syncwarp();
      }
      // Every load this warp issued lands before the CTA may exit: wait
      // (bounded) for the last load issued into each stage.
      if (!ok) {
        for (int s = 0; s < 2 && do_qk; ++s)
          if (qi[s] > 0) mbar_wait(smem_u32(&S.q_full[s]), (qi[s] - 1) & 1u, nullptr, nullptr, 0);
        for (uint32_t st = 0; st < kStages; ++st) {
          if (kc > st && do_qk) {
            const uint32_t last = ((kc - 1 - st) / kStages) * kStages + st;
            mbar_wait(smem_u32(&S.slot_full[st]), (last / kStages) & 1u, nullptr, nullptr, 0);
          }
          if (!do_qk && vc >= 1) {  // value tiles sit in slots 1 .. vc
            const int last = (((int)vc - (int)st) / kStages) * kStages + (int)st;
            if (last >= 1 && last <= (int)vc)
              mbar_wait(smem_u32(&S.slot_full[st]), ((uint32_t)last / kStages) & 1u, nullptr, nullptr, 0);
          }
        }
      }
      __syncwarp();
    } else if (warp == kWarpMma) {
      // -------------------------------------------------------------- MMA
      // The whole warp runs the loop with warp-uniform values (MMA operands
      // stay in uniform registers); one fixed elected lane issues every
      // tcgen05.mma and tcgen05.commit, so each commit tracks all MMAs before it.
      const bool leader = elect_one_sync();
      const uint64_t qdesc[2] = {sw128_desc(smem_u32(S.q[0]), 16, 1024),
                                 sw128_desc(smem_u32(S.q[1]), 16, 1024)};
      const uint64_t kdesc0 = sw128_desc(smem_u32(S.k[0]), 16, 1024);
      const uint64_t kdesc1 = sw128_desc(smem_u32(S.k[1]), 16, 1024);
      const uint64_t vdesc0 = sw128_desc(smem_u32(S.v[0]), kHalfBytes, 1024);
      const uint64_t vdesc1 = sw128_desc(smem_u32(S.v[1]), kHalfBytes, 1024);
      uint32_t kc = 0, vc = 0, qv[2] = {0, 0}, ph[2] = {0, 0}, pf[2] = {0, 0}, of[2] = {0, 0};
      bool ok = true;
      auto wait = [&](uint64_t& bar, uint32_t parity, uint32_t where) -> bool {
        return __all_sync(0xffffffffu, mbar_wait(smem_u32(&bar), parity, abort_flag, p.status, where)) != 0;
      };
      // ring slot t (key tile t, value tile t - 1): slots below `waited` are full
      uint32_t waited = 0;
      auto need_slot = [&](uint32_t t, uint32_t where) -> bool {
        if (t < waited) return true;
        waited = t + 1;
        return wait(S.slot_full[t % kStages], (t / kStages) & 1u, where | (t % kStages));
      };
      uint32_t sc = 0;
      while (ok) {
        const int u = next_unit(S, p, sc, abort_flag, ok);
        if (u < 0) break;
        const Unit U = decode_item(p, u);
        const int N = max(U.N[0], U.N[1]);
        if (N == 0) continue;
        // prologue: S_s(0)
        {
          const int st = kc % kStages;
          ok = need_slot(kc, 0x210);
          if (ok && kRotK1) ok = wait(S.k_rot[st], (kc / kStages) & 1u, 0x214);
          if (!ok) break;
          tc_fence_after();
          const uint64_t kdesc = st ? kdesc1 : kdesc0;
          for (int s = 0; s < 2 && ok; ++s) {
            if (U.N[s] == 0) continue;
            ok = wait(S.q_rot[s], qv[s] & 1u, 0x220 | s);
            if (!ok) break;
            ++qv[s];
            tc_fence_after();
            if (leader) {
              issue_s(tmem + s * BN, qdesc[s], kdesc);
              mma_commit(smem_u32(&S.s_full[s]));
              if (U.N[s] == 1) mma_commit(smem_u32(&S.q_empty[s]));
            }
            __syncwarp();
          }
          if (!ok) break;
          if (leader) mma_commit(smem_u32(&S.slot_empty[st]));  // slot kc: both its tiles are read
          __syncwarp();
          ++kc;
        }
        for (int n = 0; n < N && ok; ++n) {
          const int vst = (vc + 1) % kStages;  // value tile vc sits in slot vc + 1
          ok = need_slot(vc + 1, 0x230);
          if (!ok) break;
          tc_fence_after();
          const uint64_t vdesc = vst ? vdesc1 : vdesc0;
          const int kst = kc % kStages;
          const uint64_t kdesc = kst ? kdesc1 : kdesc0;
          bool k_ready = false;
          for (int s = 0; s < 2 && ok; ++s) {
            const uint32_t tS = tmem + s * BN;
            const uint32_t tO = tmem + 256 + s * kHeadDim;
            if (n < U.N[s]) {
              ok = wait(S.p_half[s], ph[s] & 1u, 0x240 | s);
              if (!ok) break;
              ++ph[s];
              if (n == 0) {
                ok = wait(S.o_free[s], (of[s] & 1u) ^ 1u, 0x250 | s);
                if (!ok) break;
                ++of[s];
              }
              tc_fence_after();
              if (leader) issue_pv(tO, tS + kPCol, vdesc, 0, n == 0);
              __syncwarp();
              ok = wait(S.p_full[s], pf[s] & 1u, 0x270 | s);
              if (!ok) break;
              ++pf[s];
              tc_fence_after();
              if (leader) {
                issue_pv(tO, tS + kPCol, vdesc, 4, n == 0);
                if (n == U.N[s] - 1) mma_commit(smem_u32(&S.o_done[s]));
              }
              __syncwarp();
            }
            if (n + 1 < U.N[s]) {
              if (!k_ready) {
                // key tile kc is in the slot already waited for (kc == vc + 1)
                if (kRotK1) ok = wait(S.k_rot[kst], (kc / kStages) & 1u, 0x260 | kst);
                if (!ok) break;
                tc_fence_after();
                k_ready = true;
              }
              if (leader) {
                issue_s(tS, qdesc[s], kdesc);
                mma_commit(smem_u32(&S.s_full[s]));
                if (n + 2 == U.N[s]) mma_commit(smem_u32(&S.q_empty[s]));
              }
              __syncwarp();
            }
          }
          if (!ok) break;
          // slot vc + 1 is free once its key tile is read too: now, or (the
          // unit's last step) after the next unit's first S MMAs
          if (leader && k_ready) mma_commit(smem_u32(&S.slot_empty[vst]));
          __syncwarp();
          ++vc;
          if (k_ready) ++kc;
        }
      }
      // Drain: every MMA issued above completes before TMEM is released.
      if (leader) mma_commit(smem_u32(&S.drain));
      __syncwarp();
      mbar_wait(smem_u32(&S.drain), 0, nullptr, nullptr, 0);
      __syncwarp();
    }
  } else if (warp >= kWarpEpi) {
    // ------------------------------------------------------------ epilogue
    // Drains each item's O as soon as its MMAs are done (O / l -> bf16 ->
    // global, or a piece's partial result), releasing O's TMEM columns for the
    // next item's first P*V.  The next item is read from the schedule ring
    // before the drain: the K producer publishes it while this one's keys are
    // still being loaded, so the read does not delay the drain, and it tells
    // whether this is the CTA's last item.
    setmaxnreg_dec_epilogue();
    const int t = threadIdx.x & 127;  // row == TMEM lane (warp % 4 picks the lane quarter)
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    if constexpr (kRotK1) {
      rotk1_epilogue(S, p, tmem, abort_flag, warp, lane);
    } else {
    uint32_t cnt[2] = {0, 0}, sc = 0;
    bool ok = true;
    int u = next_unit(S, p, sc, abort_flag, ok);
    while (ok && u >= 0) {
      const Unit prev = decode_item(p, u);
      u = next_unit(S, p, sc, abort_flag, ok);  // -1: prev is the CTA's last item
      if (!ok) break;
      bool merge_pending[2] = {false, false};
      for (int s = 0; s < 2 && ok; ++s) {
        if (prev.N[s] == 0) continue;
        const uint32_t par = cnt[s] & 1u;
        const uint32_t lpar = (cnt[s] >> 1) & 1u;  // phase of l_ready[par][s]
        ++cnt[s];
        ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&S.l_ready[par][s]), lpar, abort_flag,
                                              p.status, 0x400 | s));
        if (!ok) break;
        ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&S.o_done[s]), par, abort_flag,
                                              p.status, 0x410 | s));
        if (!ok) break;
        tc_fence_after();
        const uint32_t tO = tmem + lane_base + 256 + s * kHeadDim;
        uint8_t* stage = S.ostage + (warp & 3) * 32 * 128;
        const int row_first = prev.row0 + s * BM + (warp & 3) * 32;
        if (prev.slot < 0) {
          store_tile(S, p, tO, 1.f / S.row_l[par][s][t], stage, lane, s, prev.h, prev.b, row_first);
          continue;
        }
        // A piece of a split unit: its O / l (bf16) and (row max, row sum)
        // go to the piece's slot; the warp that finishes the last piece of
        // these 32 rows merges all pieces.  Nothing waits for another CTA:
        // the arrival counter decides who merges.
        const size_t part_off = (((size_t)prev.slot * 2 + s) * 4 + (warp & 3)) * 8192;  // bytes
        {
          const float l = S.row_l[par][s][t];
          const float m = S.row_m[par][s][t];
          const float inv = 1.f / l;
          uint4* dst = reinterpret_cast<uint4*>(reinterpret_cast<uint8_t*>(p.part) + part_off) + lane;
#pragma unroll 1
          for (int c = 0; c < 4; ++c) {
            uint32_t orow[32];
            tmem_ld32(tO + 32 * c, orow);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              uint32_t w[4];
#pragma unroll
              for (int i = 0; i < 4; ++i)
                w[i] = pack_bf16x2(__uint_as_float(orow[8 * e + 2 * i]) * inv,
                                   __uint_as_float(orow[8 * e + 2 * i + 1]) * inv);
              dst[(4 * c + e) * 32] = make_uint4(w[0], w[1], w[2], w[3]);
            }
          }
          tc_fence_before();
          mbar_arrive(smem_u32(&S.o_free[s]));
          p.part_ml[(size_t)(prev.slot * 2 + s) * BM + t] = make_float2(m, l);
        }
        __threadfence();
        __syncwarp();
        uint32_t arrived = 0;
        if (lane == 0) arrived = atomicAdd(p.part_cnt + ((size_t)prev.grp * 2 + s) * 4 + (warp & 3), 1u);
        arrived = __shfl_sync(0xffffffffu, arrived, 0);
        if (arrived != (uint32_t)(p.split_k - 1)) continue;
        __syncwarp();
        __threadfence();
        if (u < 0) {
          // the CTA's last item: merged below, once both tiles' MMAs are done
          merge_pending[s] = true;
          continue;
        }
        {
          float a[kMaxSplit];
          const int slot0 = prev.grp * p.split_k;
          piece_weights(p, slot0, s, t, a);
          const uint8_t* src = reinterpret_cast<const uint8_t*>(p.part) +
                               (((size_t)slot0 * 2 + s) * 4 + (warp & 3)) * 8192;
          // consecutive slots are 2 tiles x 4 row quarters x 8 KB apart
          merge_pieces<false>(p, src, 65536, a, stage, lane, prev.h, prev.b, row_first);
        }
      }
      if (u < 0) {
        // Merges that fell to this warp on the CTA's last item.  Every MMA of
        // the CTA has completed (both tiles' o_done were waited above) and no
        // load is in flight, so the Q and K buffers are free: each warp bulk-
        // loads its rows of the k pieces (8 KB each) into its 32 KB of them,
        // one round trip instead of one per 16-byte chunk.
        for (int s = 0; s < 2 && ok; ++s) {
          if (!merge_pending[s]) continue;
          float a[kMaxSplit];
          const int slot0 = prev.grp * p.split_k;
          piece_weights(p, slot0, s, t, a);
          uint8_t* buf = S.q[0] + (warp & 3) * 32768;
          const uint32_t bar = smem_u32(&S.mrg[s][warp & 3]);
          fence_proxy_async_smem();  // earlier reads of buf come before the copies
          __syncwarp();
          if (lane == 0) {
            mbar_arrive_expect_tx(bar, (uint32_t)p.split_k * 8192u);
            for (int i = 0; i < p.split_k; ++i)
              bulk_load(smem_u32(buf) + i * 8192,
                        reinterpret_cast<const uint8_t*>(p.part) +
                            (((size_t)(slot0 + i) * 2 + s) * 4 + (warp & 3)) * 8192,
                        8192u, bar);
          }
          __syncwarp();
          ok = __all_sync(0xffffffffu, mbar_wait(bar, 0, abort_flag, p.status, 0x420 | s));
          if (!ok) break;
          merge_pieces<true>(p, buf, 8192, a, S.ostage + (warp & 3) * 32 * 128, lane, prev.h, prev.b,
                             prev.row0 + s * BM + (warp & 3) * 32);
        }
        break;
      }
    }
    }
    // the shared-memory stage must stay valid until the last stores read it
    if (lane == 0) bulk_wait_read_all();
    __syncwarp();
  } else {
    // ------------------------------------------------------------- softmax
    setmaxnreg_inc_softmax();
    const int s = warp >> 2;          // query tile of this group
    const int t = threadIdx.x & 127;  // row in the tile == TMEM lane
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + lane_base + s * BN;
    const uint32_t tO = tmem + lane_base + 256 + s * kHeadDim;
    uint32_t uc = 0, sf = 0, sc = 0, qv = 0;
    bool ok = true;
    while (ok) {
      const int u = next_unit(S, p, sc, abort_flag, ok);
      if (u < 0) break;
      const Unit U = decode_item(p, u);
      const int Ns = U.N[s];
      if (Ns == 0) continue;
      const int row = U.row0 + s * BM + t;
      const bool valid = row < p.Lq;
      const uint32_t par = uc & 1u;  // unit parity of this tile's l buffer
      ++uc;
      {
        // Rotate this thread's query row in place once the tile's TMA load
        // lands (the MMA warp waits for q_rot before the first S MMA).  The
        // group is idle here (its last tile of the previous item is done),
        // and the row's table chunks are requested before the wait (rows
        // past Lq read the last row's and leave their zero-filled Q alone).
        uint4 tb[16];
        load_table_row(p.table + (size_t)min(row, p.Lq - 1) * 16, tb);
        ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&S.q_full[s]), qv & 1u, abort_flag, p.status,
                                              0x300 | s));
        if (!ok) break;
        ++qv;
        if (valid) {
          uint8_t* qrow = S.q[s] + t * 128;
          if (p.q_norm_w == nullptr)
            rotate_q_row(qrow, tb, t);
          else
            norm_rotate_q_row(qrow, tb, t, S.qnw, p.norm_eps);
        }
        fence_proxy_async_smem();
        mbar_arrive(smem_u32(&S.q_rot[s]));
      }
      const int kv_i = valid ? (p.kv_end ? p.kv_end[row] : p.n0 + p.n1) : p.n0 + p.n1;
      float m = -INFINITY, l = 0.f;
      for (int n = 0; n < Ns; ++n) {
        ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&S.s_full[s]), sf & 1u, abort_flag,
                                              p.status, 0x310 | s));
        if (!ok) break;
        ++sf;
        tc_fence_after();
        uint32_t sr[128];
        tmem_ld32(tS + 0, *reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
        tmem_ld32(tS + 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
        tmem_ld32(tS + 64, *reinterpret_cast<uint32_t(*)[32]>(&sr[64]));
        tmem_ld32(tS + 96, *reinterpret_cast<uint32_t(*)[32]>(&sr[96]));
        tmem_wait_ld();
        float* sv = reinterpret_cast<float*>(sr);
        const KTile kt = key_tile(p, U.kb + n);
        const int lim = max(0, min(kt.cnt, kv_i - kt.j0));
        const bool masked = __any_sync(0xffffffffu, lim < BN);
        float alpha = 1.f, mc;
        bool rescale = false;
        float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        float mxc[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) mxc[i] = -INFINITY;
        // mask (only tiles that straddle a row's bound), row maximum, then
        // the exponentials (measured: starting the first half from the
        // running maximum with the tile maximum folded in was ~3 % slower)
        if (masked) {
#pragma unroll
          for (int c = 0; c < BN; ++c)
            if (c >= lim) sv[c] = -INFINITY;
        }
        const float mx = row_max_from(sv, 0, mxc);
        if (n == 0) {
          m = mx;
        } else if (mx > m + kRescaleRaw) {
          alpha = ex2_approx((m - mx) * kScaleLog2);
          m = mx;
          rescale = true;
        }
        mc = m * kScaleLog2;
        exp_pack_half(sv, 0, mc, acc, tS);
        if (__any_sync(0xffffffffu, rescale)) {
          // O holds PV(n-1): it is complete, since S(n) was committed after it.
#pragma unroll 1
          for (int c = 0; c < kHeadDim; c += 32) {
            uint32_t orow[32];
            tmem_ld32(tO + c, orow);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) orow[e] = __float_as_uint(__uint_as_float(orow[e]) * alpha);
            tmem_st32(tO + c, orow);
          }
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(smem_u32(&S.p_half[s]));
        // ---- second half of P (keys 64-127)
        exp_pack_half(sv, 32, mc, acc, tS);
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(smem_u32(&S.p_full[s]));
        l = l * alpha + (((acc[0] + acc[1]) + (acc[2] + acc[3])) + ((acc[4] + acc[5]) + (acc[6] + acc[7])));
      }
      if (!ok) break;
      S.row_l[par][s][t] = l;
      S.row_m[par][s][t] = m;
      mbar_arrive(smem_u32(&S.l_ready[par][s]));
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kWarpMma) tmem_dealloc(tmem, kTmemCols);
}

}  // namespace tc

// --------------------------------------------------------------- host side
static PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (fn == nullptr) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &ptr, 12000, cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  }
  return fn;
}

// 4-D bf16 map over (dim, a, b, c) with byte strides (sa, sb, sc); the box is
// 64 columns x (box_a, box_b) rows, 128-byte swizzle, zero fill out of range.
static bool encode_4d(CUtensorMap* m, const void* base, uint64_t da, uint64_t db, uint64_t dc,
                      uint64_t sa, uint64_t sb, uint64_t sc, uint32_t box_a, uint32_t box_b) {
  auto fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[4] = {(cuuint64_t)kHeadDim, da, db, dc};
  cuuint64_t strides[3] = {sa, sb, sc};
  cuuint32_t box[4] = {64, box_a, box_b, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Map of one key/value source; returns whether it is token-major.
static bool encode_source(CUtensorMap* m, const KvSource& s, int B, int H, int* tok_major) {
  if (s.n == 0) {
    *tok_major = 0;
    return true;
  }
  const uint64_t e = 2;  // bytes per bf16
  if (s.row > s.head) {  // token-major: (dim, head, row, batch)
    *tok_major = 1;
    return encode_4d(m, s.ptr, H, s.n, B, s.head * e, s.row * e, s.batch * e, 1, tc::BM);
  }
  *tok_major = 0;  // head-major: (dim, row, head, batch)
  return encode_4d(m, s.ptr, s.n, H, B, s.row * e, s.head * e, s.batch * e, tc::BM, 1);
}

// Tail-split cost model constants (key tiles), see launch_attn_tc_bf16.
constexpr float kSplitItemTiles = 3.5f;
constexpr float kSplitMergeTiles = 9.0f;

cudaError_t launch_attn_tc_bf16(const AttnArgs& a, cudaStream_t stream, int num_sms) {
  if (a.Lq == 0 || a.B == 0 || a.H == 0) return cudaSuccess;
  tc::Params p;
  memset(&p, 0, sizeof(p));
  const uint64_t tok = (uint64_t)a.H * kHeadDim * 2;
  if (!encode_4d(&p.tm_q, a.q, a.H, a.Lq, a.B, kHeadDim * 2, tok, tok * a.Lq, 1, tc::BM) ||
      !encode_4d(&p.tm_o, a.o, a.H, a.Lq, a.B, kHeadDim * 2, tok, tok * a.Lq, 1, 32))
    return cudaErrorInvalidValue;
  if (!encode_source(&p.tm_k0, a.k0, a.B, a.H, &p.k0_tok) ||
      !encode_source(&p.tm_k1, a.k1, a.B, a.H, &p.k1_tok) ||
      !encode_source(&p.tm_v0, a.v0, a.B, a.H, &p.v0_tok) ||
      !encode_source(&p.tm_v1, a.v1, a.B, a.H, &p.v1_tok))
    return cudaErrorInvalidValue;
  p.B = a.B;
  p.H = a.H;
  p.Lq = (int32_t)a.Lq;
  p.n0 = (int32_t)a.k0.n;
  p.n1 = (int32_t)a.k1.n;
  p.nqp = (int32_t)((a.Lq + 2 * tc::BM - 1) / (2 * tc::BM));
  p.num_units = a.B * a.H * p.nqp;
  p.table = static_cast<const uint4*>(a.table);
  p.kv_end = a.kv_end;
  p.o = static_cast<__nv_bfloat16*>(a.o);
  p.status = a.status;
  p.unit_counter = a.unit_counter;
  p.q_norm_w = a.q_norm_w;
  p.norm_eps = a.norm_eps;
  p.rot_k1 = a.rot_k1;
  p.ktab1 = (int32_t)(a.Lq - a.k1.n);
  // Tail split (unmasked calls, where every unit visits the same key tiles):
  // the r units of the last, partial wave go out as k pieces each when that
  // shortens the wave.  Costs in key tiles of one unit, from per-CTA
  // timelines: each item (the pipeline's fill and drain around its key tiles)
  // about 3.5; the merge the last CTA cannot overlap, plus the slowdown of
  // the whole units running beside the pieces, about 9 (with these the
  // 384-unit 1024^2 step, 34 key tiles per unit, stays unsplit: split into 3
  // it measured 3 % slower).
  p.head_units = p.num_units;
  p.split_k = 1;
  if (a.kv_end == nullptr && a.split_slots > 0 && num_sms > 0 && !a.rot_k1) {
    const int r = p.num_units % num_sms;
    const int N = (p.n0 + tc::BN - 1) / tc::BN + (p.n1 + tc::BN - 1) / tc::BN;
    if (r > 0 && r <= a.split_cnt_units) {
      float best = (float)N + kSplitItemTiles;
      for (int k = 2; k <= tc::kMaxSplit; ++k) {
        if (N < k || r * k > a.split_slots) break;
        const float cost = (float)((r * k + num_sms - 1) / num_sms) * ((float)N / k + kSplitItemTiles) +
                           kSplitMergeTiles;
        if (cost < best) {
          best = cost;
          p.split_k = k;
        }
      }
      if (p.split_k > 1) p.head_units = p.num_units - r;
    }
  }
  p.num_items = p.head_units + (p.num_units - p.head_units) * p.split_k;
  p.part = static_cast<uint4*>(a.split_part);
  p.part_ml = static_cast<float2*>(a.split_ml);
  p.part_cnt = a.split_cnt;
  const size_t smem = sizeof(tc::Smem) + 1024;
  cudaError_t err =
      cudaFuncSetAttribute(p.rot_k1 ? tc::attn_tc_kernel<true> : tc::attn_tc_kernel<false>,
                           cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (err != cudaSuccess) return err;
  const int grid = p.num_items < num_sms ? p.num_items : num_sms;
  if (p.rot_k1)
    tc::attn_tc_kernel<true><<<grid, tc::kThreads, smem, stream>>>(p);
  else
    tc::attn_tc_kernel<false><<<grid, tc::kThreads, smem, stream>>>(p);
  note_launch();
  return cudaGetLastError();
}

}  // namespace qi21
