// fp32 joint attention on the CUDA cores (the fp32 storage type has no
// dense tensor-core path that meets a 1e-4 bound in one pass).
//
// One CTA = 16 query rows of one (batch, head); 8 warps x 2 rows.  The query
// rows are rotated on load with the per-token (cos, sin) table (after the
// QK-RMSNorm, when its weight is given); keys arrive already rotated.  Key tiles of 32 that lie at or beyond the largest
// visibility bound of the CTA's rows are never loaded (block-causal skip);
// inside the loaded tiles each row masks keys j >= kv_end[i].  Online softmax
// in fp32 with expf.
#include <math.h>

#include "qi21_device.cuh"
#include "qi21_internal.h"

namespace qi21 {

constexpr int kSimtRows = 16;
constexpr int kRowsPerWarp = 2;
constexpr int kSimtKeys = 32;
constexpr int kSimtThreads = 256;

__device__ __forceinline__ const float* kv_row(const KvSource& s, int b, int h, int64_t r) {
  return static_cast<const float*>(s.ptr) + b * s.batch + h * s.head + r * s.row;
}

__global__ void __launch_bounds__(kSimtThreads)
    attn_simt_f32_kernel(const __grid_constant__ AttnArgs a) {
  __shared__ float sq[kSimtRows][kHeadDim];
  __shared__ float sk[kSimtKeys][kHeadDim + 1];
  __shared__ float sv[kSimtKeys][kHeadDim];
  __shared__ int s_kvhi;
  __shared__ float s_rs[kSimtRows];  // QK-RMSNorm: rsqrt(mean square + eps) of each query row

  const int b = blockIdx.z, h = blockIdx.y;
  const int64_t row0 = static_cast<int64_t>(blockIdx.x) * kSimtRows;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t n_keys = a.k0.n + a.k1.n;
  const int64_t tok_stride = static_cast<int64_t>(a.H) * kHeadDim;
  const float* q = static_cast<const float*>(a.q);

  // QK-RMSNorm of the query rows (when a weight is given): one warp per row,
  // four elements per lane, a shuffle sum
  const bool norm = a.q_norm_w != nullptr;
  if (norm) {
    for (int r = warp; r < kSimtRows; r += kSimtThreads / 32) {
      const int64_t row = row0 + r;
      float ss = 0.f;
      if (row < a.Lq) {
        const float4 x = *reinterpret_cast<const float4*>(q + (b * a.Lq + row) * tok_stride +
                                                          h * kHeadDim + 4 * lane);
        ss = x.x * x.x + x.y * x.y + x.z * x.z + x.w * x.w;
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
      if (lane == 0) s_rs[r] = rsqrtf(ss * (1.f / kHeadDim) + a.norm_eps);
    }
    __syncthreads();
  }
  // rotated query rows
  for (int e = threadIdx.x; e < kSimtRows * (kHeadDim / 2); e += blockDim.x) {
    const int r = e / (kHeadDim / 2), m = e % (kHeadDim / 2);
    const int64_t row = row0 + r;
    float y0 = 0.f, y1 = 0.f;
    if (row < a.Lq) {
      const float* src = q + (b * a.Lq + row) * tok_stride + h * kHeadDim + 2 * m;
      const float2 cs = static_cast<const float2*>(a.table)[row * kPairs + m];
      float x0 = src[0], x1 = src[1];
      if (norm) {
        x0 *= s_rs[r] * a.q_norm_w[2 * m];
        x1 *= s_rs[r] * a.q_norm_w[2 * m + 1];
      }
      y0 = fmaf(x0, cs.x, -x1 * cs.y);
      y1 = fmaf(x0, cs.y, x1 * cs.x);
    }
    sq[r][2 * m] = y0;
    sq[r][2 * m + 1] = y1;
  }
  if (warp == 0) {
    const int64_t row = row0 + lane;
    int64_t kv = 0;
    if (lane < kSimtRows && row < a.Lq) kv = a.kv_end ? a.kv_end[row] : n_keys;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) kv = max(kv, __shfl_xor_sync(0xffffffffu, kv, o));
    if (lane == 0) s_kvhi = static_cast<int>(min(kv, n_keys));
  }
  __syncthreads();
  const int64_t kv_hi = s_kvhi;

  int64_t kv_row_end[kRowsPerWarp];
#pragma unroll
  for (int r = 0; r < kRowsPerWarp; ++r) {
    const int64_t row = row0 + warp * kRowsPerWarp + r;
    kv_row_end[r] = row < a.Lq ? (a.kv_end ? a.kv_end[row] : n_keys) : n_keys;
  }
  float m_i[kRowsPerWarp], l_i[kRowsPerWarp], acc[kRowsPerWarp][4];
#pragma unroll
  for (int r = 0; r < kRowsPerWarp; ++r) {
    m_i[r] = -INFINITY;
    l_i[r] = 0.f;
#pragma unroll
    for (int t = 0; t < 4; ++t) acc[r][t] = 0.f;
  }
  const float scale = 0.08838834764831845f;  // 1/sqrt(128)

  for (int64_t j0 = 0; j0 < kv_hi; j0 += kSimtKeys) {
    __syncthreads();
    for (int e = threadIdx.x; e < kSimtKeys * kHeadDim; e += blockDim.x) {
      const int r = e / kHeadDim, d = e % kHeadDim;
      const int64_t j = j0 + r;
      float kk = 0.f, vv = 0.f;
      if (j < n_keys) {
        if (j < a.k0.n) {
          kk = kv_row(a.k0, b, h, j)[d];
          vv = kv_row(a.v0, b, h, j)[d];
        } else {
          kk = kv_row(a.k1, b, h, j - a.k0.n)[d];
          vv = kv_row(a.v1, b, h, j - a.k0.n)[d];
        }
      }
      sk[r][d] = kk;
      sv[r][d] = vv;
    }
    __syncthreads();

    const int64_t j = j0 + lane;
#pragma unroll
    for (int r = 0; r < kRowsPerWarp; ++r) {
      const float* qr = sq[warp * kRowsPerWarp + r];
      float s = 0.f;
#pragma unroll 16
      for (int d = 0; d < kHeadDim; ++d) s = fmaf(qr[d], sk[lane][d], s);
      const bool ok = j < n_keys && j < kv_row_end[r];
      s = ok ? s * scale : -INFINITY;
      float mx = s;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      const float m_new = fmaxf(m_i[r], mx);
      if (m_new == -INFINITY) continue;  // nothing visible yet for this row
      const float alpha = (m_i[r] == -INFINITY) ? 0.f : expf(m_i[r] - m_new);
      const float p = ok ? expf(s - m_new) : 0.f;
      float ps = p;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) ps += __shfl_xor_sync(0xffffffffu, ps, o);
      l_i[r] = l_i[r] * alpha + ps;
      m_i[r] = m_new;
#pragma unroll
      for (int t = 0; t < 4; ++t) acc[r][t] *= alpha;
#pragma unroll 8
      for (int jj = 0; jj < kSimtKeys; ++jj) {
        const float pj = __shfl_sync(0xffffffffu, p, jj);
#pragma unroll
        for (int t = 0; t < 4; ++t) acc[r][t] = fmaf(pj, sv[jj][lane + 32 * t], acc[r][t]);
      }
    }
  }

  float* o = static_cast<float*>(a.o);
#pragma unroll
  for (int r = 0; r < kRowsPerWarp; ++r) {
    const int64_t row = row0 + warp * kRowsPerWarp + r;
    if (row >= a.Lq) continue;
    const float inv = 1.f / l_i[r];
    float* dst = o + (b * a.Lq + row) * tok_stride + h * kHeadDim;
#pragma unroll
    for (int t = 0; t < 4; ++t) dst[lane + 32 * t] = acc[r][t] * inv;
  }
}

cudaError_t launch_attn_simt_f32(const AttnArgs& a, cudaStream_t stream) {
  if (a.Lq == 0 || a.B == 0 || a.H == 0) return cudaSuccess;
  dim3 grid(static_cast<unsigned>((a.Lq + kSimtRows - 1) / kSimtRows), a.H, a.B);
  attn_simt_f32_kernel<<<grid, kSimtThreads, 0, stream>>>(a);
  note_launch();
  return cudaGetLastError();
}

}  // namespace qi21
