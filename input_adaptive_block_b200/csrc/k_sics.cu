// Scheme generation: Sum of Intra-block Cosine Similarities (SICS).
//
// SPADE technical summary (gist.science/paper/2608.03335), Methodology 2,
// "Scheme Generation": every blocking candidate is scored by the sum of the
// cosine similarities between the embeddings inside each block, in an
// online form that costs O(BS * d_head) per block instead of O(BS^2); each
// head takes the candidate with the highest score.  The online form used
// here is the identity
//     sum_{i,j in b} cos(x_i, x_j) = || sum_{i in b} x_i / ||x_i|| ||^2 ,
// one pass over the block's tokens: each token's head vector is normalised
// (its norm reduced across the lanes that hold it) and accumulated; the
// block's score is the squared norm of the sum.  A head's score under a
// candidate is the sum over its blocks, for Q plus for K.
//
// Kernel 1 (one launch per candidate): work unit = (block, group of 32
// 16-byte chunks of the token row, i.e. 32 / lanes-per-head heads); one warp
// per unit, the block's tokens walked by pointer stepping with several loads
// in flight; writes one float per (head, block).  Kernel 2: per head, the
// blocks' values summed in a fixed order (deterministic) and the argmax over
// candidates (ties -> lower index).
#include <cuda_bf16.h>

#include "spade_internal.cuh"

namespace spade {
namespace {

template <bool BF16>
__device__ __forceinline__ void unpack(const uint4& v, float (&x)[BF16 ? 8 : 4]) {
  if (BF16) {
    const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 f = __bfloat1622float2(p[e]);
      x[2 * e] = f.x;
      x[2 * e + 1] = f.y;
    }
  } else {
    const float* f = reinterpret_cast<const float*>(&v);
#pragma unroll
    for (int e = 0; e < (BF16 ? 8 : 4); ++e) x[e] = f[e];
  }
}

// Adds x / ||x|| to u, where the head vector x is spread over LPH lanes.
template <bool BF16, int LPH>
__device__ __forceinline__ void add_unit(const uint4& raw, float (&u)[BF16 ? 8 : 4]) {
  constexpr int EPC = BF16 ? 8 : 4;
  float x[EPC];
  unpack<BF16>(raw, x);
  float ss = 0.f;
#pragma unroll
  for (int e = 0; e < EPC; ++e) ss = fmaf(x[e], x[e], ss);
#pragma unroll
  for (int o = LPH / 2; o; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  const float inv = ss > 0.f ? rsqrtf(ss) : 0.f;
#pragma unroll
  for (int e = 0; e < EPC; ++e) u[e] = fmaf(x[e], inv, u[e]);
}

template <bool BF16, int LPH>
__global__ void __launch_bounds__(256) sics_block_kernel(const uint8_t* __restrict__ q,
                                                          const uint8_t* __restrict__ k,
                                                          float* __restrict__ out,   // [heads][nb]
                                                          Geo g, long long row_bytes, int chunks) {
  constexpr int EPC = BF16 ? 8 : 4;
  constexpr int HPW = 32 / LPH;                     // heads per warp unit
  const int lane = threadIdx.x & 31;
  const int gwarp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int nwarps = (gridDim.x * blockDim.x) >> 5;
  const int groups = (chunks + 31) / 32;           // a partial last group holds whole heads
  const long long n_units = (long long)g.nb * groups;
  const long long sy = (long long)g.W * row_bytes;
  const long long st = (long long)g.H * sy;
  for (long long un = gwarp; un < n_units; un += nwarps) {
    const int b = (int)(un / groups);
    const int grp = (int)(un - (long long)b * groups);
    int t0, y0, x0, et, eh, ew;
    block_box(g, b, t0, y0, x0, et, eh, ew);
    const int nvalid = et * eh * ew;
    const bool act = grp * 32 + lane < chunks;
    const long long off = (long long)(act ? grp * 32 + lane : 0) * 16 +
                          (((long long)t0 * g.H + y0) * g.W + x0) * row_bytes;
    const uint8_t* pq = q + off;
    const uint8_t* pk = k + off;
    const long long wrap_y = sy - (long long)ew * row_bytes;
    const long long wrap_t = st - (long long)eh * sy;
    float uq[EPC], uk[EPC];
#pragma unroll
    for (int e = 0; e < EPC; ++e) uq[e] = uk[e] = 0.f;
    int xl = 0, yl = 0;
    long long pos = 0;                              // byte offset of the current token from the block origin
    auto step = [&]() {
      pos += row_bytes;
      if (++xl == ew) {
        xl = 0;
        pos += wrap_y;
        if (++yl == eh) {
          yl = 0;
          pos += wrap_t;
        }
      }
    };
    int i = 0;
    for (; i + 4 <= nvalid; i += 4) {
      uint4 vq[4], vk[4];
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        vq[r] = act ? __ldg(reinterpret_cast<const uint4*>(pq + pos)) : make_uint4(0u, 0u, 0u, 0u);
        vk[r] = act ? __ldg(reinterpret_cast<const uint4*>(pk + pos)) : make_uint4(0u, 0u, 0u, 0u);
        step();
      }
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        add_unit<BF16, LPH>(vq[r], uq);
        add_unit<BF16, LPH>(vk[r], uk);
      }
    }
    for (; i < nvalid; ++i) {
      add_unit<BF16, LPH>(act ? __ldg(reinterpret_cast<const uint4*>(pq + pos)) : make_uint4(0u, 0u, 0u, 0u), uq);
      add_unit<BF16, LPH>(act ? __ldg(reinterpret_cast<const uint4*>(pk + pos)) : make_uint4(0u, 0u, 0u, 0u), uk);
      step();
    }
    float s = 0.f;
#pragma unroll
    for (int e = 0; e < EPC; ++e) s = fmaf(uq[e], uq[e], fmaf(uk[e], uk[e], s));
#pragma unroll
    for (int o = LPH / 2; o; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if (act && lane % LPH == 0) {
      const int h = grp * HPW + lane / LPH;
      out[(long long)h * g.nb + b] = s;
    }
  }
}

struct SicsReduceArgs {
  int n_cand;
  int heads;
  long long off[SPADE_MAX_SCHEMES];   // float offset of candidate c's [heads][nb] values
  int nb[SPADE_MAX_SCHEMES];
};

// One CTA per head: fixed-order sum over blocks per candidate, then argmax.
__global__ void __launch_bounds__(256) sics_reduce_kernel(const float* __restrict__ ws,
                                                           const __grid_constant__ SicsReduceArgs a,
                                                           float* __restrict__ scores, int* __restrict__ choice) {
  __shared__ float part[256];
  __shared__ float tot[SPADE_MAX_SCHEMES];
  const int h = blockIdx.x, tid = threadIdx.x;
  for (int c = 0; c < a.n_cand; ++c) {
    const float* v = ws + a.off[c] + (long long)h * a.nb[c];
    float s = 0.f;
    for (int b = tid; b < a.nb[c]; b += 256) s += v[b];
    part[tid] = s;
    __syncthreads();
    for (int w = 128; w; w >>= 1) {
      if (tid < w) part[tid] += part[tid + w];
      __syncthreads();
    }
    if (tid == 0) tot[c] = part[0];
    __syncthreads();
  }
  if (tid == 0) {
    int best = 0;
    for (int c = 0; c < a.n_cand; ++c) {
      scores[h * a.n_cand + c] = tot[c];
      if (tot[c] > tot[best]) best = c;
    }
    choice[h] = best;
  }
}

template <bool BF16, int LPH>
cudaError_t launch_block(const void* q, const void* k, float* out, const Geo& g, long long row_bytes, int chunks,
                         cudaStream_t s) {
  const long long units = (long long)g.nb * ((chunks + 31) / 32);
  long long blocks = (units + 7) / 8;
  const long long cap = 4LL * num_sms();
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  sics_block_kernel<BF16, LPH><<<(int)blocks, 256, 0, s>>>(static_cast<const uint8_t*>(q),
                                                            static_cast<const uint8_t*>(k), out, g, row_bytes, chunks);
  return cudaGetLastError();
}

}  // namespace

size_t sics_workspace_floats(const Geo* cand, int n_cand, int heads) {
  size_t n = 0;
  for (int c = 0; c < n_cand; ++c) n += (size_t)heads * cand[c].nb;
  return n;
}

cudaError_t launch_sics(const void* q, const void* k, const Geo* cand, int n_cand, int heads, int d, spade_dtype dt,
                        float* ws, float* scores, int* choice, cudaStream_t s) {
  const int esz = dt == SPADE_BF16 ? 2 : 4;
  const int lph = d * esz / 16;                      // lanes per head vector
  const long long row_bytes = (long long)heads * d * esz;
  const int chunks = heads * lph;
  SicsReduceArgs ra;
  ra.n_cand = n_cand;
  ra.heads = heads;
  long long off = 0;
  for (int c = 0; c < n_cand; ++c) {
    ra.off[c] = off;
    ra.nb[c] = cand[c].nb;
    cudaError_t e;
    float* out = ws + off;
    if (dt == SPADE_BF16 && lph == 16) e = launch_block<true, 16>(q, k, out, cand[c], row_bytes, chunks, s);
    else if (dt == SPADE_BF16 && lph == 8) e = launch_block<true, 8>(q, k, out, cand[c], row_bytes, chunks, s);
    else if (dt == SPADE_F32 && lph == 32) e = launch_block<false, 32>(q, k, out, cand[c], row_bytes, chunks, s);
    else if (dt == SPADE_F32 && lph == 16) e = launch_block<false, 16>(q, k, out, cand[c], row_bytes, chunks, s);
    else return cudaErrorInvalidValue;
    if (e != cudaSuccess) return e;
    off += (long long)heads * cand[c].nb;
  }
  sics_reduce_kernel<<<heads, 256, 0, s>>>(ws, ra, scores, choice);
  return cudaGetLastError();
}

}  // namespace spade
