// Step 3: the Estimator (inter-block importance).
//
// SPADE technical summary (gist.science/paper/2608.03335), Methodology 1,
// "Summarizer & Estimator Expressions": the Estimator scores query-block x
// key-block importance from the block summaries.  Concrete instance:
//   prob[h,i,:] = softmax_j( qmean[h,i,:] . kmean[h,j,:] / sqrt(d) ).
// One CTA per (head, 16 query rows); the 16 x nb score rows stay in shared
// memory so the softmax needs no second pass over global memory.
#include "spade_internal.cuh"

namespace spade {
namespace {

constexpr int kRows = 16;
constexpr int kCols = 64;
constexpr int kThreads = 256;

__global__ void __launch_bounds__(kThreads) estimate_kernel(const float* __restrict__ qm,
                                                            const float* __restrict__ km,
                                                            float* __restrict__ prob, int nb, int d,
                                                            float scale) {
  extern __shared__ __align__(16) float sm[];
  const int dp = d + 4;                       // padded row (keeps float4 alignment)
  float* qs = sm;                             // [kRows][d]
  float* ks = qs + kRows * d;                 // [kCols][dp]
  float* S = ks + kCols * dp;                 // [kRows][nb]
  const int h = blockIdx.y;
  const int r0 = blockIdx.x * kRows;
  const int tid = threadIdx.x;
  const float* qh = qm + (long long)h * nb * d;
  const float* kh = km + (long long)h * nb * d;

  for (int i = tid; i < kRows * d / 4; i += kThreads) {
    const int r = (i * 4) / d, c = (i * 4) % d;
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    if (r0 + r < nb) v = reinterpret_cast<const float4*>(qh + (long long)(r0 + r) * d)[c / 4];
    reinterpret_cast<float4*>(qs + r * d)[c / 4] = v;
  }
  const int r = tid / 16;
  const int cl = tid % 16;
  for (int j0 = 0; j0 < nb; j0 += kCols) {
    __syncthreads();
    for (int i = tid; i < kCols * d / 4; i += kThreads) {
      const int jr = (i * 4) / d, c = (i * 4) % d;
      float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
      if (j0 + jr < nb) v = reinterpret_cast<const float4*>(kh + (long long)(j0 + jr) * d)[c / 4];
      reinterpret_cast<float4*>(ks + jr * dp)[c / 4] = v;
    }
    __syncthreads();
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    for (int kk = 0; kk < d; kk += 4) {
      const float4 qv = reinterpret_cast<const float4*>(qs + r * d)[kk / 4];
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        const float4 kv = reinterpret_cast<const float4*>(ks + (cl + 16 * m) * dp)[kk / 4];
        acc[m] = fmaf(qv.x, kv.x, acc[m]);
        acc[m] = fmaf(qv.y, kv.y, acc[m]);
        acc[m] = fmaf(qv.z, kv.z, acc[m]);
        acc[m] = fmaf(qv.w, kv.w, acc[m]);
      }
    }
#pragma unroll
    for (int m = 0; m < 4; ++m) {
      const int j = j0 + cl + 16 * m;
      if (j < nb) S[r * nb + j] = acc[m] * scale;
    }
  }
  __syncthreads();
  // softmax: warp w handles rows 2w, 2w+1
  const int warp = tid >> 5, lane = tid & 31;
  for (int rr = warp * 2; rr < warp * 2 + 2; ++rr) {
    if (r0 + rr >= nb) break;
    const float* srow = S + rr * nb;
    float mx = -INFINITY;
    for (int j = lane; j < nb; j += 32) mx = fmaxf(mx, srow[j]);
#pragma unroll
    for (int o = 16; o; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    float sum = 0.f;
    for (int j = lane; j < nb; j += 32) sum += expf(srow[j] - mx);
#pragma unroll
    for (int o = 16; o; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
    const float inv = 1.0f / sum;
    float* prow = prob + ((long long)h * nb + r0 + rr) * nb;
    for (int j = lane; j < nb; j += 32) prow[j] = expf(srow[j] - mx) * inv;
  }
}

}  // namespace

cudaError_t launch_estimate(const float* qm, const float* km, float* prob, int heads, int nb, int d,
                            cudaStream_t s) {
  const size_t smem = sizeof(float) * ((size_t)kRows * d + (size_t)kCols * (d + 4) + (size_t)kRows * nb);
  cudaError_t e = cudaFuncSetAttribute(estimate_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid(cdiv(nb, kRows), heads);
  estimate_kernel<<<grid, kThreads, smem, s>>>(qm, km, prob, nb, d, 1.0f / sqrtf((float)d));
  return cudaGetLastError();
}

}  // namespace spade
