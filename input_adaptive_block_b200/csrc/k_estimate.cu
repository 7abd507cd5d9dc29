// Step 3: the Estimator (inter-block importance).
//
// SPADE technical summary (gist.science/paper/2608.03335), Methodology 1,
// "Summarizer & Estimator Expressions": the Estimator scores query-block x
// key-block importance from the block summaries.  Concrete instance:
//   prob[h,i,:] = softmax_j( qmean[h,i,:] . kmean[h,j,:] / sqrt(d) ).
//
// fp32 on the FMA pipe (the scores decide the kept sets, so they keep full
// single precision).  One CTA per (head, 32 query rows), eight warps; warp w
// owns rows 4w..4w+3 and lane l the key columns l, l+32, l+64, l+96 of each
// 128-column chunk: a 4 x 4 register tile, fed per four-element k step by
// four broadcast loads of Q (one row per load, same address in every lane)
// and four conflict-free loads of K (rows 528 B apart).  Each dot product is
// accumulated in ascending k with one FMA chain, as the plain definition
// reads.  Scores are staged in the output rows with a running row max and
// sum (online softmax over the chunks); a second pass over the warp's own
// rows turns them into probabilities.
#include "spade_internal.cuh"

namespace spade {
namespace {

constexpr int kRows = 32;       // query rows per CTA
constexpr int kCols = 128;      // key columns per chunk
constexpr int kThreads = 256;   // 8 warps x 4 rows

template <int D>
__global__ void __launch_bounds__(kThreads, 2) estimate_kernel(const float* __restrict__ qm,
                                                               const float* __restrict__ km,
                                                               float* __restrict__ prob, int nb, float scale) {
  constexpr int DP = D + 4;                   // padded row: 16-byte aligned, rows 4 banks apart
  extern __shared__ __align__(16) float sm[];
  float* qs = sm;                             // [kRows][DP]
  float* ks = qs + kRows * DP;                // [kCols][DP]
  const int h = blockIdx.y;
  const int r0 = blockIdx.x * kRows;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const float* qh = qm + (long long)h * nb * D;
  const float* kh = km + (long long)h * nb * D;
  float* ph = prob + (long long)h * nb * nb;

  for (int i = tid; i < kRows * D / 4; i += kThreads) {
    const int r = i / (D / 4), c4 = i % (D / 4);
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    if (r0 + r < nb) v = reinterpret_cast<const float4*>(qh + (long long)(r0 + r) * D)[c4];
    reinterpret_cast<float4*>(qs + r * DP)[c4] = v;
  }
  float m[4], l[4];
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    m[r] = -INFINITY;
    l[r] = 0.f;
  }
  const int row0 = warp * 4;
  for (int j0 = 0; j0 < nb; j0 += kCols) {
    __syncthreads();
    for (int i = tid; i < kCols * D / 4; i += kThreads) {
      const int jr = i / (D / 4), c4 = i % (D / 4);
      float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
      if (j0 + jr < nb) v = reinterpret_cast<const float4*>(kh + (long long)(j0 + jr) * D)[c4];
      reinterpret_cast<float4*>(ks + jr * DP)[c4] = v;
    }
    __syncthreads();
    float acc[4][4];
#pragma unroll
    for (int r = 0; r < 4; ++r)
#pragma unroll
      for (int c = 0; c < 4; ++c) acc[r][c] = 0.f;
#pragma unroll 4
    for (int k = 0; k < D; k += 4) {
      float4 qv[4], kv[4];
#pragma unroll
      for (int r = 0; r < 4; ++r) qv[r] = *reinterpret_cast<const float4*>(qs + (row0 + r) * DP + k);
#pragma unroll
      for (int c = 0; c < 4; ++c) kv[c] = *reinterpret_cast<const float4*>(ks + (lane + 32 * c) * DP + k);
#pragma unroll
      for (int r = 0; r < 4; ++r)
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          acc[r][c] = fmaf(qv[r].x, kv[c].x, acc[r][c]);
          acc[r][c] = fmaf(qv[r].y, kv[c].y, acc[r][c]);
          acc[r][c] = fmaf(qv[r].z, kv[c].z, acc[r][c]);
          acc[r][c] = fmaf(qv[r].w, kv[c].w, acc[r][c]);
        }
    }
    // stage the scaled scores; update the running row max and sum
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const int i = r0 + row0 + r;
      float cm = -INFINITY;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int j = j0 + lane + 32 * c;
        acc[r][c] = j < nb ? acc[r][c] * scale : -INFINITY;
        cm = fmaxf(cm, acc[r][c]);
        if (i < nb && j < nb) ph[(long long)i * nb + j] = acc[r][c];
      }
#pragma unroll
      for (int o = 16; o; o >>= 1) cm = fmaxf(cm, __shfl_xor_sync(0xffffffffu, cm, o));
      const float mn = fmaxf(m[r], cm);
      float cs = 0.f;
#pragma unroll
      for (int c = 0; c < 4; ++c) cs += expf(acc[r][c] - mn);
#pragma unroll
      for (int o = 16; o; o >>= 1) cs += __shfl_xor_sync(0xffffffffu, cs, o);
      l[r] = l[r] * expf(m[r] - mn) + cs;
      m[r] = mn;
    }
  }
  // probabilities: each warp rewrites its own staged rows (its own earlier
  // writes, so no cross-warp ordering is involved)
  __syncwarp();
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    const int i = r0 + row0 + r;
    if (i >= nb) break;
    const float inv = 1.0f / l[r];
    float* prow = ph + (long long)i * nb;
    for (int j0 = 0; j0 < nb; j0 += 32 * 8) {         // eight loads in flight per lane
      float v[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int j = j0 + 32 * u + lane;
        v[u] = j < nb ? prow[j] : 0.f;
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int j = j0 + 32 * u + lane;
        if (j < nb) prow[j] = expf(v[u] - m[r]) * inv;
      }
    }
  }
}

}  // namespace

cudaError_t launch_estimate(const float* qm, const float* km, float* prob, int heads, int nb, int d,
                            cudaStream_t s) {
  const dim3 grid(cdiv(nb, kRows), heads);
  const float scale = 1.0f / sqrtf((float)d);
  if (d == 128) {
    const size_t smem = sizeof(float) * (size_t)(kRows + kCols) * (128 + 4);
    cudaError_t e = cudaFuncSetAttribute(estimate_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    estimate_kernel<128><<<grid, kThreads, smem, s>>>(qm, km, prob, nb, scale);
  } else if (d == 64) {
    const size_t smem = sizeof(float) * (size_t)(kRows + kCols) * (64 + 4);
    cudaError_t e = cudaFuncSetAttribute(estimate_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    estimate_kernel<64><<<grid, kThreads, smem, s>>>(qm, km, prob, nb, scale);
  } else {
    return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace spade
