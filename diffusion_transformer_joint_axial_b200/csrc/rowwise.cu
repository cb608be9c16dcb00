// Row-wise and elementwise kernels of the denoising loop's blocks: the
// RMSNorm in front of the attention and of the feed-forward layer, and the
// SwiGLU gate between its two projections (overview cards 4A and 5A).  Both
// are memory-bound: 16-byte loads and stores, fp32 arithmetic, one rounding to
// bf16 per output.
#include "qi21_device.cuh"
#include "qi21_internal.h"

namespace qi21 {

// One warp per row of D bf16 values (D a multiple of 8): the first pass sums
// the squares, the second scales by rsqrt(mean + eps) and the weight.
__global__ void rmsnorm_kernel(int64_t M, int32_t D, const __nv_bfloat16* __restrict__ x,
                               const __nv_bfloat16* __restrict__ w, float eps, __nv_bfloat16* __restrict__ y) {
  const int64_t row = blockIdx.x * (int64_t)(blockDim.x / 32) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= M) return;  // whole warps leave together
  const uint4* xr = reinterpret_cast<const uint4*>(x + row * D);
  const int chunks = D / 8;
  float ss = 0.f;
  for (int c = lane; c < chunks; c += 32) {
    const uint4 u = xr[c];
    const uint32_t* p = reinterpret_cast<const uint32_t*>(&u);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 f = unpack_bf16x2(p[e]);
      ss = fmaf(f.x, f.x, fmaf(f.y, f.y, ss));
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  const float rs = rsqrtf(ss / static_cast<float>(D) + eps);
  uint4* yr = reinterpret_cast<uint4*>(y + row * D);
  const uint4* wr = reinterpret_cast<const uint4*>(w);
  for (int c = lane; c < chunks; c += 32) {
    const uint4 u = xr[c], wu = __ldg(wr + c);
    const uint32_t* p = reinterpret_cast<const uint32_t*>(&u);
    const uint32_t* q = reinterpret_cast<const uint32_t*>(&wu);
    uint4 out;
    uint32_t* o = reinterpret_cast<uint32_t*>(&out);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 f = unpack_bf16x2(p[e]), g = unpack_bf16x2(q[e]);
      o[e] = pack_bf16x2(f.x * rs * g.x, f.y * rs * g.y);
    }
    yr[c] = out;
  }
}

cudaError_t launch_rmsnorm(int64_t M, int32_t D, const void* x, const void* w, float eps, void* y,
                           cudaStream_t stream) {
  if (M == 0) return cudaSuccess;
  const int warps = 8;
  const int64_t blocks = (M + warps - 1) / warps;
  rmsnorm_kernel<<<static_cast<unsigned>(blocks), warps * 32, 0, stream>>>(
      M, D, static_cast<const __nv_bfloat16*>(x), static_cast<const __nv_bfloat16*>(w), eps,
      static_cast<__nv_bfloat16*>(y));
  note_launch();
  return cudaGetLastError();
}

// m = g * sigmoid(g) * u, eight elements (one 16-byte chunk of each) per thread.
__global__ void swiglu_kernel(int64_t chunks, const uint4* __restrict__ g, const uint4* __restrict__ u,
                              uint4* __restrict__ m) {
  const int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  if (i >= chunks) return;
  const uint4 gv = g[i], uv = u[i];
  const uint32_t* gp = reinterpret_cast<const uint32_t*>(&gv);
  const uint32_t* up = reinterpret_cast<const uint32_t*>(&uv);
  uint4 out;
  uint32_t* o = reinterpret_cast<uint32_t*>(&out);
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const float2 a = unpack_bf16x2(gp[e]), b = unpack_bf16x2(up[e]);
    o[e] = pack_bf16x2(a.x / (1.f + expf(-a.x)) * b.x, a.y / (1.f + expf(-a.y)) * b.y);
  }
  m[i] = out;
}

cudaError_t launch_swiglu(int64_t n, const void* g, const void* u, void* m, cudaStream_t stream) {
  if (n == 0) return cudaSuccess;
  const int64_t chunks = n / 8;
  const int threads = 256;
  swiglu_kernel<<<static_cast<unsigned>((chunks + threads - 1) / threads), threads, 0, stream>>>(
      chunks, static_cast<const uint4*>(g), static_cast<const uint4*>(u), static_cast<uint4*>(m));
  note_launch();
  return cudaGetLastError();
}

}  // namespace qi21
