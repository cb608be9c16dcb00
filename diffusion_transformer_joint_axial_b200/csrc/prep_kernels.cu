// Position table builder, axial-rotation / cache pre-pass and the wait
// self-test kernel of libqi21.
#include <cuda_fp16.h>
#include <math.h>

#include "qi21_device.cuh"
#include "qi21_internal.h"

namespace qi21 {

// ============================================================== positions ==
// One thread per token.  "3A - 3D Axial RoPE (16, 56, 56) & Zero-Centered
// Grid", section 1: text advances (f, h, w) together by +1 (counting text
// tokens only, from the segment's text_base); an image freezes f and centres
// its row-major grid, h = r - (H - H//2), w = c - (W - W//2).  Visibility
// bound (overview card 3C): text token i sees [0, i]; an image token sees up
// to the end of its image; with all_visible (the earlier model, no mask)
// every token sees all L keys.
__global__ void positions_kernel(const __grid_constant__ PositionsParams p) {
  const int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  if (i >= p.L) return;
  // last segment whose start <= i
  int lo = 0, hi = p.n_segs - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (p.segs[mid].start <= i) lo = mid; else hi = mid - 1;
  }
  const SegDev s = p.segs[lo];
  const int32_t t = static_cast<int32_t>(i - s.start);
  int32_t f, h, w, end;
  if (s.kind == 0) {
    f = h = w = s.text_base + t;
    end = static_cast<int32_t>(i) + 1;
  } else {
    const int32_t r = t / s.W;
    const int32_t c = t - r * s.W;
    f = s.frame;
    h = r - (s.H - s.H / 2);
    w = c - (s.W - s.W / 2);
    end = s.start + s.H * s.W;
  }
  if (p.all_visible) end = static_cast<int32_t>(p.L);
  p.pos[3 * i + 0] = f;
  p.pos[3 * i + 1] = h;
  p.pos[3 * i + 2] = w;
  if (p.kv_end != nullptr) p.kv_end[i] = end;
}

cudaError_t launch_positions(const PositionsParams& p, cudaStream_t stream) {
  if (p.L == 0) return cudaSuccess;
  const int threads = 256;
  const int64_t blocks = (p.L + threads - 1) / threads;
  positions_kernel<<<static_cast<unsigned>(blocks), threads, 0, stream>>>(p);
  note_launch();
  return cudaGetLastError();
}

// ============================================== rotation / cache pre-pass ==
// Per token: the 64 (cos, sin) pairs of its axial angles, computed in float64
// and rounded once (to fp32 for the rotation here and the fp32 attention; to
// fp16 in the table the tensor-core attention reads for its queries: half the
// bytes and load instructions, within 2.4e-4 of the exact value).  Pair m < 8 uses the frame axis, m < 36 the
// height axis, the rest the width axis ("3A", section 1: bands 16/56/56).
// Every K row is rotated once here and stored head-major (the Prefix rows go
// straight into the KV cache); V's prefix rows are copied into the V cache.
// With a K norm weight, each head row is first divided by its root mean
// square (plus eps under the root) and multiplied by the weight: the
// QK-RMSNorm that precedes RoPE (overview card 4A; close reading section 6).

Omega make_omega() {
  Omega o;
  const int dims[3] = {16, 56, 56};
  int m = 0;
  for (int a = 0; a < 3; ++a)
    for (int j = 0; j < dims[a] / 2; ++j) o.w[m++] = pow(10000.0, -2.0 * j / dims[a]);
  return o;
}

// (cos, sin) of pair m of a token at (f, h, w) = pos[0..2], in float64.
__device__ __forceinline__ void pair_sincos(const int32_t* pos, int m, const Omega& om, double& c,
                                            double& s) {
  const int axis = m < kBandPairs0 ? 0 : (m < kBandPairs01 ? 1 : 2);
  sincos(static_cast<double>(pos[axis]) * om.w[m], &s, &c);
}

constexpr int kPrepTokens = 4;  // tokens per CTA
constexpr int kPrepThreads = 256;

template <typename T>
struct Vec16;  // 16-byte vector of T
template <>
struct Vec16<__nv_bfloat16> {
  static constexpr int N = 8;
};
template <>
struct Vec16<float> {
  static constexpr int N = 4;
};

// Sum of squares of a 16-byte chunk.
__device__ __forceinline__ float sumsq_chunk(const uint4& u, __nv_bfloat16*) {
  const uint32_t* w = reinterpret_cast<const uint32_t*>(&u);
  float s = 0.f;
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const float2 x = unpack_bf16x2(w[e]);
    s = fmaf(x.x, x.x, fmaf(x.y, x.y, s));
  }
  return s;
}
__device__ __forceinline__ float sumsq_chunk(const uint4& u, float*) {
  const float* x = reinterpret_cast<const float*>(&u);
  return fmaf(x[0], x[0], fmaf(x[1], x[1], fmaf(x[2], x[2], x[3] * x[3])));
}

// (x * scale * weight), then the rotation by the pairs' (cos, sin), on one
// chunk; wt is null when there is no norm (scale is then 1).
__device__ __forceinline__ void rotate_chunk(uint4& u, const float2* cs, float scale, const float* wt,
                                             __nv_bfloat16*) {
  uint32_t* w = reinterpret_cast<uint32_t*>(&u);
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const float2 xr = unpack_bf16x2(w[e]);
    float x0 = xr.x, x1 = xr.y;
    if (wt != nullptr) {
      x0 *= scale * wt[2 * e];
      x1 *= scale * wt[2 * e + 1];
    }
    const float2 r = cs[e];
    w[e] = pack_bf16x2(fmaf(x0, r.x, -x1 * r.y), fmaf(x0, r.y, x1 * r.x));
  }
}
__device__ __forceinline__ void rotate_chunk(uint4& u, const float2* cs, float scale, const float* wt,
                                             float*) {
  float* x = reinterpret_cast<float*>(&u);
#pragma unroll
  for (int e = 0; e < 2; ++e) {
    float x0 = x[2 * e], x1 = x[2 * e + 1];
    if (wt != nullptr) {
      x0 *= scale * wt[2 * e];
      x1 *= scale * wt[2 * e + 1];
    }
    const float2 r = cs[e];
    x[2 * e] = fmaf(x0, r.x, -x1 * r.y);
    x[2 * e + 1] = fmaf(x0, r.y, x1 * r.x);
  }
}

__device__ __forceinline__ uint4 ld_stream(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

// Thread layout: a CTA takes kPrepTokens tokens of one batch.  Thread i keeps
// one 16-byte chunk c = i % CPR of the head rows of one token and walks that
// token's heads h0, h0 + SPT, h0 + 2 SPT, ... (SPT head slots per token), so
// the chunk's (cos, sin) pairs are read once and reused for every head, and
// consecutive lanes cover consecutive bytes of a row (coalesced).
constexpr int kPrepHeadsInFlight = 8;  // head rows whose loads a thread keeps in flight

template <typename T>
__global__ void __launch_bounds__(kPrepThreads)
    rope_prep_kernel(const __grid_constant__ RopePrepParams p) {
  __shared__ __align__(16) float2 cs[kPrepTokens][kPairs];
  __shared__ __align__(16) float wn[kHeadDim];  // norm weight of K
  constexpr int EPC = Vec16<T>::N;       // elements per 16-byte chunk
  constexpr int CPR = kHeadDim / EPC;    // chunks per head row (a power of two)
  constexpr int SLOTS = kPrepThreads / CPR;
  constexpr int SPT = SLOTS / kPrepTokens;  // head slots per token
  static_assert(SPT >= 1 && SLOTS % kPrepTokens == 0, "thread layout");
  const int64_t tok0 = static_cast<int64_t>(blockIdx.x) * kPrepTokens;
  const int b = blockIdx.y;
  const int c = threadIdx.x % CPR;
  const int slot = threadIdx.x / CPR;
  const int t = slot / SPT;
  const int h0 = slot % SPT;
  const int64_t tok = tok0 + t;
  const int H = p.H;
  const bool has_tok = tok < p.Lk;
  const bool has_k = tok < p.k_rot_end && has_tok;  // this token's key is rotated here
  const int iters = (H + SPT - 1) / SPT;  // the same for every thread (shuffle reductions)
  if (blockIdx.x == 0 && blockIdx.y == 0) {
    if (p.unit_counter != nullptr && threadIdx.x == 0) *p.unit_counter = 0u;
    for (int i = threadIdx.x; i < p.n_zero_words; i += blockDim.x) p.zero_words[i] = 0u;
  }
  const bool norm = p.k_norm_w != nullptr;
  const T* __restrict__ kp = static_cast<const T*>(p.k) + ((static_cast<int64_t>(b) * p.Lk + tok) * H) *
                                                              kHeadDim + c * EPC;
  // destination of this token's rows: the cache for the first `split` tokens, the rest after
  const bool first = tok < p.split;
  T* const dst_base = static_cast<T*>(first ? p.k_dst0 : p.k_dst1);
  const int64_t rows = first ? p.split : p.Lk - p.split;
  const int64_t row = first ? tok : tok - p.split;

  // The first loads go out before the angles are computed: they do not need them.
  uint4 x[kPrepHeadsInFlight];
  auto load_batch = [&](int i0) {
#pragma unroll
    for (int j = 0; j < kPrepHeadsInFlight; ++j) {
      const int h = h0 + (i0 + j) * SPT;
      if (has_k && i0 + j < iters && h < H) x[j] = ld_stream(kp + static_cast<int64_t>(h) * kHeadDim);
    }
  };
  load_batch(0);

  if (norm && threadIdx.x < kHeadDim) wn[threadIdx.x] = p.k_norm_w[threadIdx.x];
  if (threadIdx.x < kPrepTokens * kPairs) {
    const int tt = threadIdx.x / kPairs, m = threadIdx.x % kPairs;
    if (tok0 + tt < p.Lk && p.table_in != nullptr) {
      cs[tt][m] = static_cast<const float2*>(p.table_in)[(tok0 + tt) * kPairs + m];
    } else if (tok0 + tt < p.Lk) {
      double sd, cd;
      pair_sincos(p.pos + 3 * (tok0 + tt), m, p.omega, cd, sd);
      const float2 v = make_float2(static_cast<float>(cd), static_cast<float>(sd));
      cs[tt][m] = v;
      if (p.table != nullptr && b == 0) {
        if (p.table_half)
          static_cast<__half2*>(p.table)[(tok0 + tt) * kPairs + m] = __halves2half2(__double2half(cd), __double2half(sd));
        else
          static_cast<float2*>(p.table)[(tok0 + tt) * kPairs + m] = v;
      }
    }
  }
  __syncthreads();
  // this chunk's (cos, sin) pairs, the same for every head of the token
  float2 r[EPC / 2];
#pragma unroll
  for (int e = 0; e < EPC / 2; ++e) r[e] = cs[t][c * (EPC / 2) + e];
  const float* wc = norm ? &wn[c * EPC] : nullptr;

  for (int i0 = 0; i0 < iters; i0 += kPrepHeadsInFlight) {
    if (i0 > 0) load_batch(i0);
#pragma unroll
    for (int j = 0; j < kPrepHeadsInFlight; ++j) {
      if (i0 + j >= iters) break;
      const int h = h0 + (i0 + j) * SPT;
      const bool live = has_k && h < H;
      float rs = 1.f;
      if (norm) {
        // the row's CPR chunks are CPR consecutive lanes
        float ss = live ? sumsq_chunk(x[j], static_cast<T*>(nullptr)) : 0.f;
#pragma unroll
        for (int o = CPR / 2; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
        rs = rsqrtf(ss * (1.f / kHeadDim) + p.norm_eps);
      }
      if (!live) continue;
      rotate_chunk(x[j], r, rs, wc, static_cast<T*>(nullptr));
      *reinterpret_cast<uint4*>(dst_base + ((static_cast<int64_t>(b) * H + h) * rows + row) * kHeadDim +
                                c * EPC) = x[j];
    }
  }

  // Prefix V rows: a plain copy into the V cache.
  if (p.v_dst0 != nullptr && has_tok && first) {
    const T* __restrict__ vp = static_cast<const T*>(p.v) + ((static_cast<int64_t>(b) * p.Lk + tok) * H) *
                                                                kHeadDim + c * EPC;
    T* const vd = static_cast<T*>(p.v_dst0);
    for (int i0 = 0; i0 < iters; i0 += kPrepHeadsInFlight) {
      uint4 y[kPrepHeadsInFlight];
#pragma unroll
      for (int j = 0; j < kPrepHeadsInFlight; ++j) {
        const int h = h0 + (i0 + j) * SPT;
        if (i0 + j < iters && h < H) y[j] = ld_stream(vp + static_cast<int64_t>(h) * kHeadDim);
      }
#pragma unroll
      for (int j = 0; j < kPrepHeadsInFlight; ++j) {
        const int h = h0 + (i0 + j) * SPT;
        if (i0 + j < iters && h < H)
          *reinterpret_cast<uint4*>(vd + ((static_cast<int64_t>(b) * H + h) * p.split + tok) * kHeadDim +
                                    c * EPC) = y[j];
      }
    }
  }
}

cudaError_t launch_rope_prep(const RopePrepParams& p, bool f32, cudaStream_t stream) {
  if (p.Lk == 0 || p.B == 0 || p.H == 0) {
    // the table still has to exist for zero heads/batches: nothing reads it then
    return cudaSuccess;
  }
  dim3 grid(static_cast<unsigned>((p.Lk + kPrepTokens - 1) / kPrepTokens),
            static_cast<unsigned>(p.B));
  if (f32)
    rope_prep_kernel<float><<<grid, kPrepThreads, 0, stream>>>(p);
  else
    rope_prep_kernel<__nv_bfloat16><<<grid, kPrepThreads, 0, stream>>>(p);
  note_launch();
  return cudaGetLastError();
}

// ======================================================= rotation table ==
// One thread per (token, pair): the pre-pass's float64 angle, rounded once to
// fp32 and once to fp16.
__global__ void rope_table_kernel(const __grid_constant__ RopeTableParams p) {
  const int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x;
  if (i >= p.n * kPairs) return;
  const int64_t tok = i / kPairs;
  const int m = static_cast<int>(i - tok * kPairs);
  double sd, cd;
  pair_sincos(p.pos + 3 * tok, m, p.omega, cd, sd);
  static_cast<float2*>(p.t32)[i] = make_float2(static_cast<float>(cd), static_cast<float>(sd));
  static_cast<__half2*>(p.t16)[i] = __halves2half2(__double2half(cd), __double2half(sd));
}

cudaError_t launch_rope_table(const RopeTableParams& p, cudaStream_t stream) {
  if (p.n == 0) return cudaSuccess;
  const int threads = 256;
  const int64_t blocks = (p.n * kPairs + threads - 1) / threads;
  rope_table_kernel<<<static_cast<unsigned>(blocks), threads, 0, stream>>>(p);
  note_launch();
  return cudaGetLastError();
}

// ============================================================ self test ==
// One CTA waits on a barrier that no one arrives at, with a short limit; the
// bounded wait must give up, record QI21_ERR_TIMEOUT and let the CTA exit.
__global__ void wait_selftest_kernel(uint32_t* status, uint64_t limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    mbar_wait(smem_u32(&bar), 0, &abort_flag, status, 0xFFu, limit_ns);
  }
  __syncthreads();
}

cudaError_t launch_wait_selftest(uint32_t* status, uint64_t limit_ns, cudaStream_t stream) {
  wait_selftest_kernel<<<1, 32, 0, stream>>>(status, limit_ns);
  note_launch();
  return cudaGetLastError();
}

}  // namespace qi21
