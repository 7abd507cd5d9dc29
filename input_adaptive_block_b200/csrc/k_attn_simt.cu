// Step 5 on CUDA cores: flash block-sparse attention for the shapes the
// tensor-core kernel does not take (fp32 data, blocks other than 128 slots).
//
// SPADE technical summary (gist.science/paper/2608.03335), Methodology 3,
// "Flash Block-Sparse Attention": each query block attends only to its kept
// key blocks; the softmax is evaluated online block by block, so no dense
// score matrix exists.  One CTA per work item (head, query block), one thread
// per query slot; each key block's K/V tile is gathered from token order into
// shared memory (padded slots flagged invalid and given no weight).
#include "spade_internal.cuh"

namespace spade {
namespace {

template <typename T>
__device__ __forceinline__ float to_f(T x);
template <>
__device__ __forceinline__ float to_f<float>(float x) { return x; }
template <>
__device__ __forceinline__ float to_f<__nv_bfloat16>(__nv_bfloat16 x) { return __bfloat162float(x); }
template <typename T>
__device__ __forceinline__ T from_f(float x);
template <>
__device__ __forceinline__ float from_f<float>(float x) { return x; }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float x) { return __float2bfloat16_rn(x); }

// Token id of slot s of block b (video, scheme g) or -1 for a padded slot.
__device__ __forceinline__ long long video_slot_token(const Geo& g, int b, int s) {
  int t0, y0, x0, et, eh, ew;
  block_box(g, b, t0, y0, x0, et, eh, ew);
  const int xl = s % g.bw, yl = (s / g.bw) % g.bh, tl = s / (g.bw * g.bh);
  if (tl >= et || yl >= eh || xl >= ew) return -1;
  return ((long long)(t0 + tl) * g.H + (y0 + yl)) * g.W + (x0 + xl);
}

// Key block #k of an item: kept video blocks (ascending), then text blocks.
__device__ __forceinline__ int item_key_block(const AttnArgs& a, const HeadInfo& hi, int qb, int ncnt, int k) {
  if (hi.dense || qb >= hi.nb) return k;
  if (k < ncnt) return a.idx[hi.idx_off + (long long)qb * hi.nb + k];
  return hi.nb + (k - ncnt);
}

template <typename T, int D>
__global__ void __launch_bounds__(128) attn_simt_kernel(const __grid_constant__ AttnArgs a, float scale) {
  extern __shared__ __align__(16) float smem[];
  float* Ks = smem;                 // [128][D]
  float* Vs = Ks + 128 * D;         // [128][D]
  long long* tok = reinterpret_cast<long long*>(Vs + 128 * D);   // [128]
  const int item = a.work[blockIdx.x];
  const int h = item >> 16, qb = item & 0xffff;
  const HeadInfo hi = a.head[h];
  const Geo g = a.geo[hi.scheme];
  const int ntb = text_blocks(a.text_tokens);
  const bool full_row = hi.dense || qb >= hi.nb;
  const int ncnt = full_row ? hi.nb : a.cnt[hi.cnt_off + qb];
  const int n = ncnt + ntb;
  const T* Q = static_cast<const T*>(a.q);
  const T* K = static_cast<const T*>(a.k);
  const T* V = static_cast<const T*>(a.v);
  T* O = static_cast<T*>(a.out);
  const long long rs = (long long)a.heads * D;   // token row stride (elements)
  const int r = threadIdx.x;

  long long qtok = -1;
  if (qb < hi.nb) {
    if (r < g.bs) qtok = video_slot_token(g, qb, r);
  } else {
    const int t = (qb - hi.nb) * 128 + r;
    if (t < a.text_tokens) qtok = a.N + t;
  }
  float q[D], o[D];
#pragma unroll
  for (int c = 0; c < D; ++c) {
    q[c] = qtok >= 0 ? to_f<T>(Q[qtok * rs + (long long)h * D + c]) * scale : 0.f;
    o[c] = 0.f;
  }
  float m = -INFINITY, l = 0.f;
  for (int kk = 0; kk < n; ++kk) {
    const int kb = item_key_block(a, hi, qb, ncnt, kk);
    const int slots = kb < hi.nb ? g.bs : 128;
    __syncthreads();
    for (int s = threadIdx.x; s < slots; s += blockDim.x) {
      long long t;
      if (kb < hi.nb) t = video_slot_token(g, kb, s);
      else {
        const int tt = (kb - hi.nb) * 128 + s;
        t = tt < a.text_tokens ? (long long)a.N + tt : -1;
      }
      tok[s] = t;
    }
    __syncthreads();
    for (int e = threadIdx.x; e < slots * D; e += blockDim.x) {
      const int s = e / D, c = e % D;
      const long long t = tok[s];
      Ks[e] = t >= 0 ? to_f<T>(K[t * rs + (long long)h * D + c]) : 0.f;
      Vs[e] = t >= 0 ? to_f<T>(V[t * rs + (long long)h * D + c]) : 0.f;
    }
    __syncthreads();
    // pass 1: block max; pass 2: weights and accumulation
    float bm = -INFINITY;
    for (int s = 0; s < slots; ++s) {
      if (tok[s] < 0) continue;
      float sc = 0.f;
#pragma unroll
      for (int c = 0; c < D; ++c) sc = fmaf(q[c], Ks[s * D + c], sc);
      bm = fmaxf(bm, sc);
    }
    const float mn = fmaxf(m, bm);
    const float alpha = expf(m - mn);
    l *= alpha;
#pragma unroll
    for (int c = 0; c < D; ++c) o[c] *= alpha;
    for (int s = 0; s < slots; ++s) {
      if (tok[s] < 0) continue;
      float sc = 0.f;
#pragma unroll
      for (int c = 0; c < D; ++c) sc = fmaf(q[c], Ks[s * D + c], sc);
      const float p = expf(sc - mn);
      l += p;
#pragma unroll
      for (int c = 0; c < D; ++c) o[c] = fmaf(p, Vs[s * D + c], o[c]);
    }
    m = mn;
  }
  if (qtok >= 0) {
    const float inv = 1.0f / l;
#pragma unroll
    for (int c = 0; c < D; ++c) O[qtok * rs + (long long)h * D + c] = from_f<T>(o[c] * inv);
  }
}

template <typename T, int D>
cudaError_t launch_t(const AttnArgs& a, cudaStream_t s) {
  const size_t smem = 2 * 128 * D * sizeof(float) + 128 * sizeof(long long);
  cudaError_t e =
      cudaFuncSetAttribute(attn_simt_kernel<T, D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  attn_simt_kernel<T, D><<<a.n_items, 128, smem, s>>>(a, 1.0f / sqrtf((float)D));
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attn_simt(const AttnArgs& a, cudaStream_t s) {
  if (a.dt == SPADE_F32) return a.d == 64 ? launch_t<float, 64>(a, s) : launch_t<float, 128>(a, s);
  return a.d == 64 ? launch_t<__nv_bfloat16, 64>(a, s) : launch_t<__nv_bfloat16, 128>(a, s);
}

}  // namespace spade
