// bf16 joint attention on the sm_100a tensor cores (tcgen05 + TMEM + TMA).
//
// Computes O = softmax(rot(Q) K^T / sqrt(128) + M) V for the Qwen-Image-2.1
// joint sequence ("Qwen-Image-2.1 architecture" overview, cards 3A/3C/4A/6A):
// the queries are rotated band-wise (16, 56, 56) inside the kernel right
// after their TMA load; the keys come already rotated (from the Prefix KV
// cache or the per-step pre-pass); M is the block-causal mask given by
// kv_end (allowed(i, j) <=> j < kv_end[i]) or no mask at all.
//
// Work unit: one (batch, head) and a pair of 128-row query tiles.  A CTA
// (one per SM, persistent) walks its units in order of decreasing cost.
// For each query tile only the key tiles that start below the tile's largest
// kv_end are visited: every visibility bound is a prefix of the keys, so
// fully masked tiles are skipped and never loaded; only tiles that straddle
// a row's bound (the diagonal of the text block, ragged ends) are masked
// element-wise.
//
// Warp roles (320 threads):
//   warps 0-3  softmax + epilogue for query tile 0 (thread = row = TMEM lane)
//   warps 4-7  softmax + epilogue for query tile 1
//   warp  8    TMA producer (Q tiles, K/V ring of 2 stages each)
//   warp  9    TMEM allocator and tcgen05.mma issuer
// TMEM (512 columns): S0 | S1 | O0 | O1, 128 fp32 columns each; P (bf16,
// packed in pairs) overwrites the first 64 columns of its S and is the A
// operand of the P*V MMA, so P never touches shared memory.
// Issue order per key tile n: PV0(n), S0(n+1), PV1(n), S1(n+1): while one
// softmax group works the tensor core runs the other tile's MMAs.
// Online softmax uses a lazy rescale: O and l are rescaled only when a row
// maximum grows by more than 2^8, which keeps every P <= 256.
#include <cudaTypedefs.h>
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
constexpr int kThreads = 320;
constexpr int kWarpLoad = 8;
constexpr int kWarpMma = 9;
constexpr uint32_t kTmemCols = 512;

// Instruction descriptor of tcgen05.mma kind::f16: fp32 accumulate (bit 4),
// A and B bf16 (bits 7, 10), N >> 3 at bit 17, M >> 4 at bit 24; bit 16 marks
// B as MN-major (V: head dim contiguous).
constexpr uint32_t kIdescS = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) |
                             ((uint32_t)(BM >> 4) << 24);
constexpr uint32_t kIdescPV = (1u << 4) | (1u << 7) | (1u << 10) | (1u << 16) |
                              ((uint32_t)(kHeadDim >> 3) << 17) | ((uint32_t)(BM >> 4) << 24);

// log2(e) / sqrt(128) and the lazy-rescale threshold (8 in log2 units).
constexpr float kScaleLog2 = 0.12751743082459868f;
constexpr float kRescaleRaw = 8.0f / kScaleLog2;

struct Params {
  CUtensorMap tm_q;
  CUtensorMap tm_k0, tm_k1, tm_v0, tm_v1;
  int32_t k0_tok, k1_tok, v0_tok, v1_tok;  // 1: token-major coords, 0: head-major
  int32_t B, H, Lq, n0, n1;
  int32_t nqp;        // query-tile pairs per (batch, head)
  int32_t num_units;  // B * H * nqp
  const float2* table;
  const int32_t* kv_end;
  __nv_bfloat16* o;
  uint32_t* status;
};

struct __align__(1024) Smem {
  uint8_t q[2][kTileBytes];
  uint8_t k[kStages][kTileBytes];
  uint8_t v[kStages][kTileBytes];
  uint64_t q_full[2], q_rot[2], q_empty[2];
  uint64_t k_full[kStages], k_empty[kStages], v_full[kStages], v_empty[kStages];
  uint64_t s_full[2], p_full[2], o_done[2], o_free[2];
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
// K-major operand (Q or K tile): 16-element k-step kk lives in half kk/4 at
// byte offset 32*(kk%4) of each 128-byte row; 8-row groups are 1024 B apart.
__device__ __forceinline__ uint64_t kmajor_desc(uint32_t tile, int kk) {
  return sw128_desc(tile + (kk >> 2) * kHalfBytes + (kk & 3) * 32, 16, 1024);
}
// MN-major operand (V tile, rows = keys): k-step kk = 16 key rows = 2048 B;
// the two 64-column halves are 16 KB apart.
__device__ __forceinline__ uint64_t mnmajor_desc(uint32_t tile, int kk) {
  return sw128_desc(tile + kk * 2048, kHalfBytes, 1024);
}

struct Unit {
  int b, h, row0;
  int N[2];
};

__device__ __forceinline__ int ceil_div(int a, int b) { return (a + b - 1) / b; }

// Key tiles that start below kv_hi (keys are [source 0 rows || source 1 rows]).
__device__ __forceinline__ int tiles_below(const Params& p, int kv_hi) {
  const int nt0 = ceil_div(p.n0, BN);
  if (kv_hi <= p.n0) return ceil_div(kv_hi, BN);
  return nt0 + min(ceil_div(kv_hi - p.n0, BN), ceil_div(p.n1, BN));
}

__device__ __forceinline__ Unit decode_unit(const Params& p, int u) {
  Unit U;
  const int bh_count = p.B * p.H;
  const int qp = p.nqp - 1 - u / bh_count;  // most expensive query tiles first
  const int bh = u % bh_count;
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
  return U;
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
      mbar_init(smem_u32(&S.p_full[s]), BM);
      mbar_init(smem_u32(&S.o_done[s]), 1);
      mbar_init(smem_u32(&S.o_free[s]), BM);
    }
    for (int s = 0; s < kStages; ++s) {
      mbar_init(smem_u32(&S.k_full[s]), 1);
      mbar_init(smem_u32(&S.k_empty[s]), 1);
      mbar_init(smem_u32(&S.v_full[s]), 1);
      mbar_init(smem_u32(&S.v_empty[s]), 1);
    }
    mbar_init(smem_u32(&S.drain), 1);
    S.abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kWarpMma) {
    tmem_alloc(smem_u32(&S.tmem_base), kTmemCols);
    tmem_relinquish();
  }
  if (warp == kWarpLoad && lane == 0) {
    tma_prefetch_desc(&p.tm_q);
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

  if (warp == kWarpLoad) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      uint32_t kc = 0, vc = 0, ql[2] = {0, 0};
      bool ok = true;
      for (int u = blockIdx.x; u < p.num_units && ok; u += gridDim.x) {
        const Unit U = decode_unit(p, u);
        for (int s = 0; s < 2 && ok; ++s) {
          if (U.N[s] == 0) continue;
          // the MMA thread releases Q_s once per unit that used it
          ok = mbar_wait(smem_u32(&S.q_empty[s]), (ql[s] & 1u) ^ 1u, abort_flag, p.status, 0x100 | s);
          ++ql[s];
          if (ok) {
            const uint32_t bar = smem_u32(&S.q_full[s]);
            mbar_arrive_expect_tx(bar, kTileBytes);
            const uint32_t dst = smem_u32(S.q[s]);
            tma_load_4d(dst, &p.tm_q, bar, 0, U.h, U.row0 + s * BM, U.b);
            tma_load_4d(dst + kHalfBytes, &p.tm_q, bar, 64, U.h, U.row0 + s * BM, U.b);
          }
        }
        const int N = max(U.N[0], U.N[1]);
        for (int n = 0; n < N && ok; ++n) {
          const KTile t = key_tile(p, n);
          {
            const int st = kc % kStages;
            ok = mbar_wait(smem_u32(&S.k_empty[st]), ((kc / kStages) & 1u) ^ 1u, abort_flag,
                           p.status, 0x110 | st);
            if (!ok) break;
            const uint32_t bar = smem_u32(&S.k_full[st]);
            mbar_arrive_expect_tx(bar, kTileBytes);
            load_kv_tile(t.src ? &p.tm_k1 : &p.tm_k0, t.src ? p.k1_tok : p.k0_tok, smem_u32(S.k[st]),
                         bar, t.row, U.h, U.b);
            ++kc;
          }
          {
            const int st = vc % kStages;
            ok = mbar_wait(smem_u32(&S.v_empty[st]), ((vc / kStages) & 1u) ^ 1u, abort_flag,
                           p.status, 0x120 | st);
            if (!ok) break;
            const uint32_t bar = smem_u32(&S.v_full[st]);
            mbar_arrive_expect_tx(bar, kTileBytes);
            load_kv_tile(t.src ? &p.tm_v1 : &p.tm_v0, t.src ? p.v1_tok : p.v0_tok, smem_u32(S.v[st]),
                         bar, t.row, U.h, U.b);
            ++vc;
          }
        }
      }
      // Every load this warp issued lands before the CTA may exit: wait
      // (bounded) for the last load issued into each stage.
      if (!ok) {
        for (uint32_t st = 0; st < kStages; ++st) {
          if (kc > st) {
            const uint32_t last = ((kc - 1 - st) / kStages) * kStages + st;
            mbar_wait(smem_u32(&S.k_full[st]), (last / kStages) & 1u, nullptr, nullptr, 0);
          }
          if (vc > st) {
            const uint32_t last = ((vc - 1 - st) / kStages) * kStages + st;
            mbar_wait(smem_u32(&S.v_full[st]), (last / kStages) & 1u, nullptr, nullptr, 0);
          }
        }
      }
    }
  } else if (warp == kWarpMma) {
    // -------------------------------------------------------------- MMA
    if (lane == 0) {
      uint32_t kc = 0, vc = 0, qv[2] = {0, 0}, pc[2] = {0, 0}, of[2] = {0, 0};
      bool ok = true;
      for (int u = blockIdx.x; u < p.num_units && ok; u += gridDim.x) {
        const Unit U = decode_unit(p, u);
        const int N = max(U.N[0], U.N[1]);
        if (N == 0) continue;
        // prologue: S_s(0)
        {
          const int st = kc % kStages;
          ok = mbar_wait(smem_u32(&S.k_full[st]), (kc / kStages) & 1u, abort_flag, p.status, 0x210);
          if (!ok) break;
          tc_fence_after();
          const uint32_t kt = smem_u32(S.k[st]);
          for (int s = 0; s < 2 && ok; ++s) {
            if (U.N[s] == 0) continue;
            ok = mbar_wait(smem_u32(&S.q_rot[s]), qv[s] & 1u, abort_flag, p.status, 0x220 | s);
            if (!ok) break;
            ++qv[s];
            tc_fence_after();
            const uint32_t qt = smem_u32(S.q[s]);
            for (int kk = 0; kk < kHeadDim / 16; ++kk)
              mma_ss(tmem + s * BN, kmajor_desc(qt, kk), kmajor_desc(kt, kk), kIdescS, kk > 0);
            mma_commit(smem_u32(&S.s_full[s]));
            if (U.N[s] == 1) mma_commit(smem_u32(&S.q_empty[s]));
          }
          if (!ok) break;
          mma_commit(smem_u32(&S.k_empty[st]));
          ++kc;
        }
        for (int n = 0; n < N && ok; ++n) {
          const int vst = vc % kStages;
          ok = mbar_wait(smem_u32(&S.v_full[vst]), (vc / kStages) & 1u, abort_flag, p.status,
                         0x230 | vst);
          if (!ok) break;
          tc_fence_after();
          const uint32_t vt = smem_u32(S.v[vst]);
          const int kst = kc % kStages;
          const uint32_t kt = smem_u32(S.k[kst]);
          bool k_ready = false;
          for (int s = 0; s < 2 && ok; ++s) {
            if (n < U.N[s]) {
              ok = mbar_wait(smem_u32(&S.p_full[s]), pc[s] & 1u, abort_flag, p.status, 0x240 | s);
              if (!ok) break;
              ++pc[s];
              if (n == 0) {
                ok = mbar_wait(smem_u32(&S.o_free[s]), (of[s] & 1u) ^ 1u, abort_flag, p.status,
                               0x250 | s);
                if (!ok) break;
                ++of[s];
              }
              tc_fence_after();
              for (int kk = 0; kk < BN / 16; ++kk)
                mma_ts(tmem + 256 + s * kHeadDim, tmem + s * BN + kk * 8, mnmajor_desc(vt, kk),
                       kIdescPV, (n > 0 || kk > 0) ? 1u : 0u);
              if (n == U.N[s] - 1) mma_commit(smem_u32(&S.o_done[s]));
            }
            if (n + 1 < U.N[s]) {
              if (!k_ready) {
                ok = mbar_wait(smem_u32(&S.k_full[kst]), (kc / kStages) & 1u, abort_flag, p.status,
                               0x260 | kst);
                if (!ok) break;
                tc_fence_after();
                k_ready = true;
              }
              const uint32_t qt = smem_u32(S.q[s]);
              for (int kk = 0; kk < kHeadDim / 16; ++kk)
                mma_ss(tmem + s * BN, kmajor_desc(qt, kk), kmajor_desc(kt, kk), kIdescS, kk > 0);
              mma_commit(smem_u32(&S.s_full[s]));
              if (n + 2 == U.N[s]) mma_commit(smem_u32(&S.q_empty[s]));
            }
          }
          if (!ok) break;
          mma_commit(smem_u32(&S.v_empty[vst]));
          ++vc;
          if (k_ready) {
            mma_commit(smem_u32(&S.k_empty[kst]));
            ++kc;
          }
        }
      }
      // Drain: every MMA issued above completes before TMEM is released.
      mma_commit(smem_u32(&S.drain));
      mbar_wait(smem_u32(&S.drain), 0, nullptr, nullptr, 0);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------- softmax / epilogue
    const int s = warp >> 2;             // query tile of this group
    const int t = threadIdx.x & 127;     // row in the tile == TMEM lane
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + lane_base + s * BN;
    const uint32_t tO = tmem + lane_base + 256 + s * kHeadDim;
    uint32_t qv = 0, sf = 0, od = 0;
    bool ok = true;
    for (int u = blockIdx.x; u < p.num_units && ok; u += gridDim.x) {
      const Unit U = decode_unit(p, u);
      const int Ns = U.N[s];
      if (Ns == 0) continue;
      const int row = U.row0 + s * BM + t;
      const bool valid = row < p.Lq;
      // ---- rotate this query row in place (bands 16/56/56, adjacent pairs)
      ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&S.q_full[s]), qv & 1u, abort_flag, p.status,
                                            0x300 | s));
      if (!ok) break;
      ++qv;
      if (valid) {
        const float4* cs = reinterpret_cast<const float4*>(p.table + (size_t)row * kPairs);
        uint8_t* qrow = S.q[s] + t * 128;
#pragma unroll 4
        for (int c = 0; c < 16; ++c) {
          const int half = c >> 3, cc = c & 7;
          uint4* ptr = reinterpret_cast<uint4*>(qrow + half * kHalfBytes + ((cc ^ (t & 7)) << 4));
          uint4 x = *ptr;
          const float4 r01 = __ldg(cs + 2 * c);
          const float4 r23 = __ldg(cs + 2 * c + 1);
          const float rc[4] = {r01.x, r01.z, r23.x, r23.z};
          const float rs[4] = {r01.y, r01.w, r23.y, r23.w};
          uint32_t* w = reinterpret_cast<uint32_t*>(&x);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 xv = unpack_bf16x2(w[e]);
            w[e] = pack_bf16x2(fmaf(xv.x, rc[e], -xv.y * rs[e]), fmaf(xv.x, rs[e], xv.y * rc[e]));
          }
          *ptr = x;
        }
      }
      fence_proxy_async_smem();
      mbar_arrive(smem_u32(&S.q_rot[s]));

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
        const KTile kt = key_tile(p, n);
        const int lim = max(0, min(kt.cnt, kv_i - kt.j0));
        if (__any_sync(0xffffffffu, lim < BN)) {
#pragma unroll
          for (int c = 0; c < BN; ++c)
            if (c >= lim) sv[c] = -INFINITY;
        }
        float mx0 = sv[0], mx1 = sv[1], mx2 = sv[2], mx3 = sv[3];
#pragma unroll
        for (int c = 4; c < BN; c += 4) {
          mx0 = fmaxf(mx0, sv[c]);
          mx1 = fmaxf(mx1, sv[c + 1]);
          mx2 = fmaxf(mx2, sv[c + 2]);
          mx3 = fmaxf(mx3, sv[c + 3]);
        }
        const float mx = fmaxf(fmaxf(mx0, mx1), fmaxf(mx2, mx3));
        float alpha = 1.f;
        bool rescale = false;
        if (n == 0) {
          m = mx;
        } else if (mx > m + kRescaleRaw) {
          alpha = ex2_approx((m - mx) * kScaleLog2);
          m = mx;
          rescale = true;
        }
        const float mc = m * kScaleLog2;
        float l0 = 0.f, l1 = 0.f;
        uint32_t pk[64];
#pragma unroll
        for (int c = 0; c < BN; c += 2) {
          const float p0 = ex2_approx(fmaf(sv[c], kScaleLog2, -mc));
          const float p1 = ex2_approx(fmaf(sv[c + 1], kScaleLog2, -mc));
          l0 += p0;
          l1 += p1;
          pk[c >> 1] = pack_bf16x2(p0, p1);
        }
        tmem_st32(tS + 0, *reinterpret_cast<uint32_t(*)[32]>(&pk[0]));
        tmem_st32(tS + 32, *reinterpret_cast<uint32_t(*)[32]>(&pk[32]));
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
        l = l * alpha + (l0 + l1);
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(smem_u32(&S.p_full[s]));
      }
      if (!ok) break;
      // ---- epilogue: O / l -> bf16 -> global
      ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&S.o_done[s]), od & 1u, abort_flag, p.status,
                                            0x320 | s));
      if (!ok) break;
      ++od;
      tc_fence_after();
      const float inv = 1.f / l;
      __nv_bfloat16* dst =
          p.o + (((size_t)U.b * p.Lq + (valid ? row : 0)) * p.H + U.h) * kHeadDim;
#pragma unroll 1
      for (int c = 0; c < kHeadDim; c += 32) {
        uint32_t orow[32];
        tmem_ld32(tO + c, orow);
        tmem_wait_ld();
        if (valid) {
          uint32_t pkd[16];
#pragma unroll
          for (int e = 0; e < 16; ++e)
            pkd[e] = pack_bf16x2(__uint_as_float(orow[2 * e]) * inv,
                                 __uint_as_float(orow[2 * e + 1]) * inv);
          uint4* d4 = reinterpret_cast<uint4*>(dst + c);
#pragma unroll
          for (int e = 0; e < 4; ++e)
            d4[e] = make_uint4(pkd[4 * e], pkd[4 * e + 1], pkd[4 * e + 2], pkd[4 * e + 3]);
        }
      }
      tc_fence_before();
      mbar_arrive(smem_u32(&S.o_free[s]));
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

cudaError_t launch_attn_tc_bf16(const AttnArgs& a, cudaStream_t stream, int num_sms) {
  if (a.Lq == 0 || a.B == 0 || a.H == 0) return cudaSuccess;
  tc::Params p;
  memset(&p, 0, sizeof(p));
  const uint64_t tok = (uint64_t)a.H * kHeadDim * 2;
  if (!encode_4d(&p.tm_q, a.q, a.H, a.Lq, a.B, kHeadDim * 2, tok, tok * a.Lq, 1, tc::BM))
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
  p.table = a.table;
  p.kv_end = a.kv_end;
  p.o = static_cast<__nv_bfloat16*>(a.o);
  p.status = a.status;
  const size_t smem = sizeof(tc::Smem) + 1024;
  cudaError_t err =
      cudaFuncSetAttribute(tc::attn_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (err != cudaSuccess) return err;
  const int grid = p.num_units < num_sms ? p.num_units : num_sms;
  tc::attn_tc_kernel<<<grid, tc::kThreads, smem, stream>>>(p);
  note_launch();
  return cudaGetLastError();
}

}  // namespace qi21
