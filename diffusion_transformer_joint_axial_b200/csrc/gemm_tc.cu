// bf16 linear layer on the sm_100a tensor cores: Y = X W^T (+ b).
//
// The projections around the attention of one Qwen-Image-2.1 DiT block
// (close reading section 6: to_q / to_k / to_v produce the joint Q, K, V and
// the output projection maps the attention output back; overview card 6A:
// steps 2..N compute only the target tokens, so only their rows are
// projected).  X is [M, K] row-major, W is [N, K] (the nn.Linear layout, K
// contiguous), b is [N] or absent; the N output columns are cut into n_out
// equal segments written to separate [M, N / n_out] row-major tensors, so one
// launch of the fused Q/K/V projection leaves Q, K and V exactly in the
// [B, T, H, 128] layout the attention kernels read.
//
// Tiles of 128 x 256 outputs; one persistent CTA per SM walks tiles
// t = blockIdx.x, blockIdx.x + gridDim.x, ... with the 128-row M blocks
// fastest, so CTAs working at the same time share one 256-row slice of W.
// Roles (256 threads):
//   warp 0     TMA producer: a 4-stage ring of (X 128x64, W 256x64) K-steps
//   warp 1     TMEM owner and tcgen05.mma issuer (M=128, N=256, K=16)
//   warps 4-7  epilogue: TMEM -> fp32 (+ bias, or residual + alpha * (. + bias),
//              or silu(gate) * up of a tile's two column halves) -> bf16 -> global,
//              row per thread
// TMEM holds two 256-column fp32 accumulators, so the epilogue of one tile
// overlaps the MMAs of the next.  Rows, columns and K past the end are
// zero-filled by TMA and never stored.  Every wait is bounded.
#include <cudaTypedefs.h>
#include <string.h>

#include "qi21_device.cuh"
#include "qi21_internal.h"

namespace qi21 {

namespace gemm {

constexpr int BM = 128;
constexpr int BN = 256;
constexpr int BK = 64;  // one 128-byte swizzle atom of bf16
constexpr int kStages = 4;
constexpr int kABytes = BM * BK * 2;  // 16 KB
constexpr int kBBytes = BN * BK * 2;  // 32 KB
constexpr int kThreads = 256;
constexpr int kWarpMma = 1;
constexpr int kWarpEpi = 4;
constexpr uint32_t kTmemCols = 2 * BN;
constexpr int kMaxOut = 4;

// tcgen05.mma kind::f16 instruction descriptor: fp32 accumulate (bit 4), A and
// B bf16 (bits 7, 10), both K-major, N >> 3 at bit 17, M >> 4 at bit 24.
constexpr uint32_t kIdesc = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) |
                            ((uint32_t)(BM >> 4) << 24);

struct Params {
  CUtensorMap tm_x, tm_w;
  int32_t M, N, K;
  int32_t n_seg;                // columns per output segment
  int32_t mt, nt, kt;           // tiles along M, N and K steps
  __nv_bfloat16* out[kMaxOut];  // [M, n_seg] each
  const __nv_bfloat16* bias;    // [N] or null
  const __nv_bfloat16* residual;  // [M, N] added to alpha * (X W^T + b), or null (may be out[0])
  float alpha;
  int32_t swiglu;  // 1: W holds gate/up rows in alternating 128-row blocks; out[0] = silu(gate) * up
  uint32_t* status;
};

struct __align__(1024) Smem {
  uint8_t a[kStages][kABytes];
  uint8_t b[kStages][kBBytes];
  uint64_t full[kStages], empty[kStages];
  uint64_t acc_full[2], acc_empty[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
};

// Shared-memory descriptor of a K-major operand in 128B-swizzled rows of
// 128 bytes: 8-row groups 1024 B apart (SBO), LBO unused, version 1, layout 2.
__device__ __forceinline__ uint64_t kmajor_sw128_desc(uint32_t saddr) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr & 0x3FFFFu) >> 4);
  d |= (uint64_t)(16u >> 4) << 16;
  d |= (uint64_t)(1024u >> 4) << 32;
  d |= (uint64_t)1 << 46;
  d |= (uint64_t)2 << 61;
  return d;
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const void* map, uint32_t bar, int c0, int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
      "l"(map), "r"(c0), "r"(c1), "r"(bar)
      : "memory");
}

__global__ void __launch_bounds__(kThreads, 1) gemm_tc_kernel(const __grid_constant__ Params p) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  Smem& S = *reinterpret_cast<Smem*>(smem_raw + (((raw + 1023u) & ~1023u) - raw));
  const int warp = threadIdx.x >> 5;
  volatile int* abort_flag = &S.abort_flag;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(smem_u32(&S.full[s]), 1);
      mbar_init(smem_u32(&S.empty[s]), 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(smem_u32(&S.acc_full[s]), 1);
      mbar_init(smem_u32(&S.acc_empty[s]), 128);
    }
    mbar_init(smem_u32(&S.drain), 1);
    S.abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kWarpMma) {
    tmem_alloc(smem_u32(&S.tmem_base), kTmemCols);
    tmem_relinquish();
  }
  if (warp == 0 && (threadIdx.x & 31) == 0) {
    tma_prefetch_desc(&p.tm_x);
    tma_prefetch_desc(&p.tm_w);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = S.tmem_base;
  const int tiles = p.mt * p.nt;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    const bool leader = elect_one_sync();
    uint32_t it = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < tiles && ok; t += gridDim.x) {
      const int m0 = (t % p.mt) * BM, n0 = (t / p.mt) * BN;
      for (int kb = 0; kb < p.kt; ++kb, ++it) {
        const int st = it % kStages;
        ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&S.empty[st]), ((it / kStages) & 1u) ^ 1u,
                                              abort_flag, p.status, 0x600 | st));
        if (!ok) break;
        if (leader) {
          const uint32_t bar = smem_u32(&S.full[st]);
          mbar_arrive_expect_tx(bar, kABytes + kBBytes);
          tma_load_2d(smem_u32(S.a[st]), &p.tm_x, bar, kb * BK, m0);
          tma_load_2d(smem_u32(S.b[st]), &p.tm_w, bar, kb * BK, n0);
        }
        __syncwarp();
      }
    }
    // every load issued lands before the CTA may exit
    if (!ok) {
      for (uint32_t st = 0; st < kStages; ++st)
        if (it > st) {
          const uint32_t last = ((it - 1 - st) / kStages) * kStages + st;
          mbar_wait(smem_u32(&S.full[st]), (last / kStages) & 1u, nullptr, nullptr, 0);
        }
    }
    __syncwarp();
  } else if (warp == kWarpMma) {
    // ---------------------------------------------------------------- MMA
    const bool leader = elect_one_sync();
    uint32_t it = 0, tc = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < tiles && ok; t += gridDim.x, ++tc) {
      const uint32_t buf = tc & 1u;
      ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&S.acc_empty[buf]), ((tc >> 1) & 1u) ^ 1u,
                                            abort_flag, p.status, 0x610 | buf));
      if (!ok) break;
      tc_fence_after();
      const uint32_t acc = tmem + buf * BN;
      for (int kb = 0; kb < p.kt; ++kb, ++it) {
        const int st = it % kStages;
        ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&S.full[st]), (it / kStages) & 1u, abort_flag,
                                              p.status, 0x620 | st));
        if (!ok) break;
        tc_fence_after();
        if (leader) {
          const uint64_t ad = kmajor_sw128_desc(smem_u32(S.a[st]));
          const uint64_t bd = kmajor_sw128_desc(smem_u32(S.b[st]));
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk)
            mma_ss(acc, ad + (uint64_t)(kk * 2), bd + (uint64_t)(kk * 2), kIdesc,
                   (kb > 0 || kk > 0) ? 1u : 0u);
          mma_commit(smem_u32(&S.empty[st]));
          if (kb == p.kt - 1) mma_commit(smem_u32(&S.acc_full[buf]));
        }
        __syncwarp();
      }
    }
    // every MMA issued completes before TMEM is released
    if (leader) mma_commit(smem_u32(&S.drain));
    __syncwarp();
    mbar_wait(smem_u32(&S.drain), 0, nullptr, nullptr, 0);
    __syncwarp();
  } else if (warp >= kWarpEpi) {
    // ----------------------------------------------------------- epilogue
    const int r = threadIdx.x - kWarpEpi * 32;  // row in the tile == TMEM lane
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    uint32_t tc = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < tiles && ok; t += gridDim.x, ++tc) {
      const uint32_t buf = tc & 1u;
      ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&S.acc_full[buf]), (tc >> 1) & 1u, abort_flag,
                                            p.status, 0x630 | buf));
      if (!ok) break;
      tc_fence_after();
      const int row = (t % p.mt) * BM + r;
      const int n0 = (t / p.mt) * BN;
      if (p.swiglu) {
        // columns [0, 128) of the tile are the gates of output features
        // n0/2 + [0, 128), columns [128, 256) their up projections
#pragma unroll 1
        for (int c = 0; c < BN / 2; c += 32) {
          uint32_t gv[32], uv[32];
          tmem_ld32(tmem + lane_base + buf * BN + c, gv);
          tmem_ld32(tmem + lane_base + buf * BN + BN / 2 + c, uv);
          tmem_wait_ld();
          if (row < p.M) {
#pragma unroll
            for (int g = 0; g < 4; ++g) {
              float gate[8], up[8];
#pragma unroll
              for (int e = 0; e < 8; ++e) {
                gate[e] = __uint_as_float(gv[8 * g + e]);
                up[e] = __uint_as_float(uv[8 * g + e]);
              }
              if (p.bias != nullptr) {
                const uint4 bg = __ldg(reinterpret_cast<const uint4*>(p.bias + n0 + c + 8 * g));
                const uint4 bu = __ldg(reinterpret_cast<const uint4*>(p.bias + n0 + BN / 2 + c + 8 * g));
                const uint32_t* bgw = reinterpret_cast<const uint32_t*>(&bg);
                const uint32_t* buw = reinterpret_cast<const uint32_t*>(&bu);
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                  const float2 a = unpack_bf16x2(bgw[e]), b = unpack_bf16x2(buw[e]);
                  gate[2 * e] += a.x;
                  gate[2 * e + 1] += a.y;
                  up[2 * e] += b.x;
                  up[2 * e + 1] += b.y;
                }
              }
              float f[8];
#pragma unroll
              for (int e = 0; e < 8; ++e) f[e] = gate[e] / (1.f + expf(-gate[e])) * up[e];
              __nv_bfloat16* dst = p.out[0] + (size_t)row * p.n_seg + n0 / 2 + c + 8 * g;
              *reinterpret_cast<uint4*>(dst) = make_uint4(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]),
                                                          pack_bf16x2(f[4], f[5]), pack_bf16x2(f[6], f[7]));
            }
          }
        }
        tc_fence_before();
        mbar_arrive(smem_u32(&S.acc_empty[buf]));
        continue;
      }
#pragma unroll 1
      for (int c = 0; c < BN; c += 32) {
        uint32_t v[32];
        tmem_ld32(tmem + lane_base + buf * BN + c, v);
        tmem_wait_ld();
        if (row < p.M) {
#pragma unroll
          for (int g = 0; g < 4; ++g) {  // 8 columns = 16 bytes
            const int col = n0 + c + 8 * g;
            if (col >= p.N) break;
            float f[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) f[e] = __uint_as_float(v[8 * g + e]);
            if (p.bias != nullptr) {
              const uint4 bb = __ldg(reinterpret_cast<const uint4*>(p.bias + col));
              const uint32_t* bw = reinterpret_cast<const uint32_t*>(&bb);
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const float2 bf = unpack_bf16x2(bw[e]);
                f[2 * e] += bf.x;
                f[2 * e + 1] += bf.y;
              }
            }
            const int seg = col / p.n_seg;
            __nv_bfloat16* dst = p.out[seg] + (size_t)row * p.n_seg + (col - seg * p.n_seg);
            if (p.residual != nullptr) {
              // the same thread reads this residual chunk and then writes the
              // output chunk, so the residual may be the output itself
              const uint4 rr = *reinterpret_cast<const uint4*>(p.residual + (size_t)row * p.N + col);
              const uint32_t* rw = reinterpret_cast<const uint32_t*>(&rr);
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const float2 rf = unpack_bf16x2(rw[e]);
                f[2 * e] = fmaf(p.alpha, f[2 * e], rf.x);
                f[2 * e + 1] = fmaf(p.alpha, f[2 * e + 1], rf.y);
              }
            }
            *reinterpret_cast<uint4*>(dst) = make_uint4(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]),
                                                        pack_bf16x2(f[4], f[5]), pack_bf16x2(f[6], f[7]));
          }
        }
      }
      tc_fence_before();
      mbar_arrive(smem_u32(&S.acc_empty[buf]));
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kWarpMma) tmem_dealloc(tmem, kTmemCols);
}

}  // namespace gemm

// --------------------------------------------------------------- host side
static PFN_cuTensorMapEncodeTiled_v12000 gemm_encode_fn() {
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

// 2-D bf16 map of a row-major [rows, K] matrix; box 64 (K) x box_rows, 128-byte
// swizzle, zero fill past the ends.
static bool encode_rows(CUtensorMap* m, const void* base, uint64_t rows, uint64_t K, uint32_t box_rows) {
  auto fn = gemm_encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[2] = {K, rows};
  cuuint64_t strides[1] = {K * 2};
  cuuint32_t box[2] = {(cuuint32_t)gemm::BK, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

cudaError_t launch_gemm_tc(const GemmArgs& a, cudaStream_t stream, int num_sms) {
  if (a.M == 0 || a.N == 0) return cudaSuccess;
  gemm::Params p;
  memset(&p, 0, sizeof(p));
  if (!encode_rows(&p.tm_x, a.x, a.M, a.K, gemm::BM) || !encode_rows(&p.tm_w, a.w, a.N, a.K, gemm::BN))
    return cudaErrorInvalidValue;
  p.M = (int32_t)a.M;
  p.N = (int32_t)a.N;
  p.K = (int32_t)a.K;
  p.n_seg = (int32_t)(a.swiglu ? a.N / 2 : a.N / a.n_out);
  p.swiglu = a.swiglu;
  p.mt = (int32_t)((a.M + gemm::BM - 1) / gemm::BM);
  p.nt = (int32_t)((a.N + gemm::BN - 1) / gemm::BN);
  p.kt = (int32_t)((a.K + gemm::BK - 1) / gemm::BK);
  for (int i = 0; i < a.n_out; ++i) p.out[i] = static_cast<__nv_bfloat16*>(a.out[i]);
  p.bias = static_cast<const __nv_bfloat16*>(a.bias);
  p.residual = static_cast<const __nv_bfloat16*>(a.residual);
  p.alpha = a.alpha;
  p.status = a.status;
  const size_t smem = sizeof(gemm::Smem) + 1024;
  cudaError_t err =
      cudaFuncSetAttribute(gemm::gemm_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (err != cudaSuccess) return err;
  const int64_t tiles = (int64_t)p.mt * p.nt;
  const int grid = tiles < num_sms ? (int)tiles : num_sms;
  gemm::gemm_tc_kernel<<<grid, gemm::kThreads, smem, stream>>>(p);
  note_launch();
  return cudaGetLastError();
}

}  // namespace qi21
