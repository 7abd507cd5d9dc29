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
// Block values, one float per (candidate, head, block), come from one of two
// kernels.  The one-pass kernel (below) reads Q and K once for all
// candidates through their common refinement; it serves every candidate set
// on one grid whose refinement region holds at most 64 cells.  Otherwise one
// launch per candidate: work unit = (block, group of 32 16-byte chunks of the
// token row, i.e. 32 / lanes-per-head heads); one warp per unit, the block's
// tokens walked by pointer stepping with several loads in flight.  Then per
// head the blocks' values are summed in a fixed order (deterministic) and the
// argmax taken over candidates (ties -> lower index).
#include <cuda_bf16.h>

#include <algorithm>

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

// Same as unpack, but opaque to the compiler, so that a second unpack of the
// same words is recomputed (two instructions per word) instead of keeping
// the first one's floats live across the norm reductions.
template <bool BF16>
__device__ __forceinline__ void unpack_again(const uint4& v, float (&x)[BF16 ? 8 : 4]) {
  if (BF16) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      uint32_t lo, hi;
      asm volatile("shl.b32 %0, %1, 16;" : "=r"(lo) : "r"(w[e]));
      asm volatile("and.b32 %0, %1, 0xffff0000;" : "=r"(hi) : "r"(w[e]));
      x[2 * e] = __uint_as_float(lo);
      x[2 * e + 1] = __uint_as_float(hi);
    }
  } else {
    unpack<BF16>(v, x);
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

// ---- all candidates in one pass ------------------------------------------
// The candidates' blockings have a common refinement: cells of
// (gcd bt, gcd bh, gcd bw) tokens, each inside exactly one block of every
// candidate, and regions of (lcm bt, lcm bh, lcm bw) tokens, each a union of
// whole blocks of every candidate.  A CTA takes one (region, head) unit.
// Its warps sum the normalised Q and K head vectors over each cell into
// shared memory: a warp load covers 32 / LPH tokens (one per group of LPH
// lanes, each group walking its own contiguous share of the cell's tokens in
// t, y, x order), the groups' partial sums are then added by a fixed
// butterfly.  Each candidate block of the region then sums its cells in
// (t, y, x) order and takes the squared norms, Q plus K.  Q and K are read
// once for every candidate instead of once per candidate, and every sum runs
// in a fixed order, so the result is deterministic.  Units are handed out by
// the block scheduler in order of decreasing region volume (full regions
// first, grid-edge regions last), which balances the last wave.
constexpr int kFusedMaxCells = 64;
constexpr int kFusedBatch = 4;        // tokens per lane group in flight (x2: Q and K)
constexpr int kFusedMinBlocks = 3;    // resident CTAs per SM the registers are sized for

// A box of region indices whose regions all have the same clipped volume.
struct RegionClass {
  int r0[3], nr[3];      // first region index and count along t, y, x
  int before;            // regions of the classes ahead of this one
};

struct SicsFusedArgs {
  int n_cand;
  Geo cand[SPADE_MAX_SCHEMES];
  long long out_off[SPADE_MAX_SCHEMES];   // float offset of candidate c's [heads][nb] values
  int T, H, W;
  int RT, RY, RX;        // region (lcm of the block extents)
  int CT, CY, CX;        // cell (gcd of the block extents)
  int NCT, NCY, NCX;     // cells per region axis
  int NRT, NRY, NRX;     // regions per grid axis
  int n_cls;             // region classes, by decreasing region volume
  RegionClass cls[8];
  int heads;
  long long row_bytes;
};

template <bool BF16, int LPH, int B>
__global__ void __launch_bounds__(256, kFusedMinBlocks) sics_fused_kernel(const uint8_t* __restrict__ q,
                                                             const uint8_t* __restrict__ k,
                                                             float* __restrict__ ws,
                                                             const __grid_constant__ SicsFusedArgs a) {
  constexpr int EPC = BF16 ? 8 : 4;
  constexpr int TPW = 32 / LPH;                       // tokens per warp load
  const int ncell = a.NCT * a.NCY * a.NCX;
  extern __shared__ float4 fused_smem[];
  float* cq = reinterpret_cast<float*>(fused_smem);   // [cell][EPC][LPH]: the cell's sum of Q / ||Q||
  float* ck = cq + ncell * EPC * LPH;                 // same for K
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int lg = lane / LPH, li = lane % LPH;         // lane group (token) and lane within the head
  const int nreg = a.NRT * a.NRY * a.NRX;
  const long long units = (long long)nreg * a.heads;
  const long long sy = (long long)a.W * a.row_bytes, st = (long long)a.H * sy;
  for (long long un = blockIdx.x; un < units; un += gridDim.x) {
    const int r = (int)(un / a.heads), h = (int)(un - (long long)r * a.heads);
    int kc = 0;
    while (kc + 1 < a.n_cls && a.cls[kc + 1].before <= r) ++kc;
    const RegionClass& rc = a.cls[kc];
    const int rl = r - rc.before;
    const int rk = rc.r0[2] + rl % rc.nr[2], rj = rc.r0[1] + (rl / rc.nr[2]) % rc.nr[1],
              ri = rc.r0[0] + rl / (rc.nr[2] * rc.nr[1]);
    const int t0r = ri * a.RT, y0r = rj * a.RY, x0r = rk * a.RX;
    const long long lane_off = (long long)(h * LPH + li) * 16;
    for (int c = warp; c < ncell; c += 8) {
      const int cx = c % a.NCX, cy = (c / a.NCX) % a.NCY, ct = c / (a.NCX * a.NCY);
      const int t0 = t0r + ct * a.CT, y0 = y0r + cy * a.CY, x0 = x0r + cx * a.CX;
      const int et = max(0, min(a.CT, a.T - t0)), eh = max(0, min(a.CY, a.H - y0)), ew = max(0, min(a.CX, a.W - x0));
      const int n = et * eh * ew;
      float uq[EPC], uk[EPC];
#pragma unroll
      for (int e = 0; e < EPC; ++e) uq[e] = uk[e] = 0.f;
      if (n > 0) {
        const int m = (n + TPW - 1) / TPW;                 // tokens per lane group (warp-uniform)
        const int s0 = lg * m;
        const int cnt = max(0, min(m, n - s0));           // this group's tokens: [s0, s0 + cnt)
        int tl = 0, yl = 0, xl = 0;
        if (cnt > 0) { tl = s0 / (eh * ew); yl = (s0 / ew) % eh; xl = s0 % ew; }
        long long pos = (((long long)(t0 + tl) * a.H + (y0 + yl)) * a.W + (x0 + xl)) * a.row_bytes + lane_off;
        const long long wrap_y = sy - (long long)ew * a.row_bytes;
        const long long wrap_t = st - (long long)eh * sy;
        for (int i0 = 0; i0 < m; i0 += B) {
          uint4 vq[B], vk[B];
#pragma unroll
          for (int rr = 0; rr < B; ++rr) {
            vq[rr] = vk[rr] = make_uint4(0u, 0u, 0u, 0u);
            if (i0 + rr < cnt) {
              vq[rr] = __ldg(reinterpret_cast<const uint4*>(q + pos));
              vk[rr] = __ldg(reinterpret_cast<const uint4*>(k + pos));
              pos += a.row_bytes;
              if (++xl == ew) {
                xl = 0;
                pos += wrap_y;
                if (++yl == eh) {
                  yl = 0;
                  pos += wrap_t;
                }
              }
            }
          }
          // squared norms with packed FMAs over element pairs (even and odd
          // elements summed apart, then added), reduced over the head's lanes;
          // the raw words stay live and are unpacked again for the sums
          // (cheaper than keeping the floats across the reductions)
          float nq[B], nk[B];
#pragma unroll
          for (int rr = 0; rr < B; ++rr) {
            float xq[EPC], xk[EPC];
            unpack<BF16>(vq[rr], xq);
            unpack<BF16>(vk[rr], xk);
            float2 aq = make_float2(0.f, 0.f), ak = make_float2(0.f, 0.f);
#pragma unroll
            for (int e = 0; e < EPC; e += 2) {
              const float2 pq = make_float2(xq[e], xq[e + 1]), pk = make_float2(xk[e], xk[e + 1]);
              aq = __ffma2_rn(pq, pq, aq);
              ak = __ffma2_rn(pk, pk, ak);
            }
            nq[rr] = aq.x + aq.y;
            nk[rr] = ak.x + ak.y;
          }
#pragma unroll
          for (int o = LPH / 2; o; o >>= 1)
#pragma unroll
            for (int rr = 0; rr < B; ++rr) {
              nq[rr] += __shfl_xor_sync(0xffffffffu, nq[rr], o);
              nk[rr] += __shfl_xor_sync(0xffffffffu, nk[rr], o);
            }
#pragma unroll
          for (int rr = 0; rr < B; ++rr) {
            const float iq = nq[rr] > 0.f ? rsqrtf(nq[rr]) : 0.f;    // zero rows (past the group's share) add nothing
            const float ik = nk[rr] > 0.f ? rsqrtf(nk[rr]) : 0.f;
            const float2 iq2 = make_float2(iq, iq), ik2 = make_float2(ik, ik);
            float xq[EPC], xk[EPC];
            unpack_again<BF16>(vq[rr], xq);
            unpack_again<BF16>(vk[rr], xk);
#pragma unroll
            for (int e = 0; e < EPC; e += 2) {
              float2 a = __ffma2_rn(make_float2(xq[e], xq[e + 1]), iq2, make_float2(uq[e], uq[e + 1]));
              uq[e] = a.x;
              uq[e + 1] = a.y;
              a = __ffma2_rn(make_float2(xk[e], xk[e + 1]), ik2, make_float2(uk[e], uk[e + 1]));
              uk[e] = a.x;
              uk[e + 1] = a.y;
            }
          }
        }
      }
      // the lane groups' partial sums, added by a fixed butterfly (every group ends with the same value)
#pragma unroll
      for (int o = 16; o >= LPH; o >>= 1)
#pragma unroll
        for (int e = 0; e < EPC; ++e) {
          uq[e] += __shfl_xor_sync(0xffffffffu, uq[e], o);
          uk[e] += __shfl_xor_sync(0xffffffffu, uk[e], o);
        }
      if (lg == 0) {
#pragma unroll
        for (int e = 0; e < EPC; ++e) {
          cq[(c * EPC + e) * LPH + li] = uq[e];
          ck[(c * EPC + e) * LPH + li] = uk[e];
        }
      }
    }
    __syncthreads();
    // every candidate block of the region (one per lane group): its cells summed in (t, y, x) order
    for (int cd = 0; cd < a.n_cand; ++cd) {
      const Geo& g = a.cand[cd];
      const int pbt = a.RT / g.bt, pbh = a.RY / g.bh, pbw = a.RX / g.bw;     // blocks per region axis
      const int ctb = g.bt / a.CT, cyb = g.bh / a.CY, cxb = g.bw / a.CX;      // cells per block axis
      const int nbr = pbt * pbh * pbw;
      for (int bl0 = warp * TPW; bl0 < nbr; bl0 += 8 * TPW) {
        const int bl = bl0 + lg;
        const int bk = bl % pbw, bj = (bl / pbw) % pbh, bi = bl / (pbw * pbh);
        const int gbi = ri * pbt + bi, gbj = rj * pbh + bj, gbk = rk * pbw + bk;
        const bool ok = bl < nbr && gbi < g.nbt && gbj < g.nbh && gbk < g.nbw;   // inside the region and the grid
        float sq[EPC], sk[EPC];
#pragma unroll
        for (int e = 0; e < EPC; ++e) sq[e] = sk[e] = 0.f;
        if (ok) {
          for (int ci = 0; ci < ctb; ++ci)
            for (int cj = 0; cj < cyb; ++cj)
              for (int cl = 0; cl < cxb; ++cl) {
                const int c = ((bi * ctb + ci) * a.NCY + (bj * cyb + cj)) * a.NCX + (bk * cxb + cl);
#pragma unroll
                for (int e = 0; e < EPC; ++e) {
                  sq[e] += cq[(c * EPC + e) * LPH + li];
                  sk[e] += ck[(c * EPC + e) * LPH + li];
                }
              }
        }
        float pq = 0.f, pk = 0.f;
#pragma unroll
        for (int e = 0; e < EPC; ++e) {
          pq = fmaf(sq[e], sq[e], pq);
          pk = fmaf(sk[e], sk[e], pk);
        }
#pragma unroll
        for (int o = LPH / 2; o; o >>= 1) {
          pq += __shfl_xor_sync(0xffffffffu, pq, o);
          pk += __shfl_xor_sync(0xffffffffu, pk, o);
        }
        if (ok && li == 0) ws[a.out_off[cd] + (long long)h * g.nb + (gbi * g.nbh + gbj) * g.nbw + gbk] = pq + pk;
      }
    }
    __syncthreads();
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

int gcd_i(int a, int b) { while (b) { const int t = a % b; a = b; b = t; } return a; }
long long lcm_ll(long long a, long long b) { return a / gcd_i((int)a, (int)b) * b; }

template <bool BF16, int LPH>
cudaError_t launch_fused(const void* q, const void* k, float* ws, const SicsFusedArgs& fa, cudaStream_t s) {
  constexpr int EPC = BF16 ? 8 : 4;
  constexpr int B = kFusedBatch;
  const size_t smem = 2ull * fa.NCT * fa.NCY * fa.NCX * EPC * LPH * sizeof(float);
  // the opt-in is per device, so it is set on every launch (it is cheap)
  const cudaError_t attr = cudaFuncSetAttribute(sics_fused_kernel<BF16, LPH, B>,
                                                cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                (int)(2 * kFusedMaxCells * EPC * LPH * sizeof(float)));
  if (attr != cudaSuccess) return attr;
  const long long units = (long long)fa.NRT * fa.NRY * fa.NRX * fa.heads;
  long long blocks = units;
  const long long cap = 1LL << 30;
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  sics_fused_kernel<BF16, LPH, B><<<(int)blocks, 256, smem, s>>>(static_cast<const uint8_t*>(q),
                                                                  static_cast<const uint8_t*>(k), ws, fa);
  return cudaGetLastError();
}

// Region and cell of the candidates' common refinement; false when a region
// holds more cells than the one-pass kernel keeps on chip.
bool sics_fused_plan(const Geo* cand, int n_cand, SicsFusedArgs& fa) {
  long long RT = 1, RY = 1, RX = 1;
  int CT = cand[0].bt, CY = cand[0].bh, CX = cand[0].bw;
  for (int c = 0; c < n_cand; ++c) {
    if (cand[c].T != cand[0].T || cand[c].H != cand[0].H || cand[c].W != cand[0].W) return false;
    RT = lcm_ll(RT, cand[c].bt); RY = lcm_ll(RY, cand[c].bh); RX = lcm_ll(RX, cand[c].bw);
    CT = gcd_i(CT, cand[c].bt); CY = gcd_i(CY, cand[c].bh); CX = gcd_i(CX, cand[c].bw);
    if (RT > 4096 || RY > 4096 || RX > 4096) return false;
  }
  const long long ncell = (RT / CT) * (RY / CY) * (RX / CX);
  long long nblk = 0;
  for (int c = 0; c < n_cand; ++c) nblk += (RT / cand[c].bt) * (RY / cand[c].bh) * (RX / cand[c].bw);
  if (ncell > kFusedMaxCells || nblk > (long long)SPADE_MAX_SCHEMES * kFusedMaxCells) return false;
  fa.n_cand = n_cand;
  for (int c = 0; c < n_cand; ++c) fa.cand[c] = cand[c];
  fa.T = cand[0].T; fa.H = cand[0].H; fa.W = cand[0].W;
  fa.RT = (int)RT; fa.RY = (int)RY; fa.RX = (int)RX;
  fa.CT = CT; fa.CY = CY; fa.CX = CX;
  fa.NCT = (int)(RT / CT); fa.NCY = (int)(RY / CY); fa.NCX = (int)(RX / CX);
  fa.NRT = cdiv(fa.T, fa.RT); fa.NRY = cdiv(fa.H, fa.RY); fa.NRX = cdiv(fa.W, fa.RX);
  // per axis: the full regions, then the clipped last one (if any)
  const int dim[3] = {fa.T, fa.H, fa.W}, ext[3] = {fa.RT, fa.RY, fa.RX};
  int ar0[3][2], anr[3][2], aext[3][2], na[3];
  for (int ax = 0; ax < 3; ++ax) {
    na[ax] = 0;
    const int full = dim[ax] / ext[ax], rem = dim[ax] % ext[ax];
    if (full > 0) { ar0[ax][na[ax]] = 0; anr[ax][na[ax]] = full; aext[ax][na[ax]] = ext[ax]; ++na[ax]; }
    if (rem > 0) { ar0[ax][na[ax]] = full; anr[ax][na[ax]] = 1; aext[ax][na[ax]] = rem; ++na[ax]; }
  }
  struct C { RegionClass rc; long long vol; };
  C cl[8];
  int n = 0;
  for (int a0 = 0; a0 < na[0]; ++a0)
    for (int a1 = 0; a1 < na[1]; ++a1)
      for (int a2 = 0; a2 < na[2]; ++a2) {
        C& c = cl[n++];
        c.rc.r0[0] = ar0[0][a0]; c.rc.nr[0] = anr[0][a0];
        c.rc.r0[1] = ar0[1][a1]; c.rc.nr[1] = anr[1][a1];
        c.rc.r0[2] = ar0[2][a2]; c.rc.nr[2] = anr[2][a2];
        c.vol = (long long)aext[0][a0] * aext[1][a1] * aext[2][a2];
      }
  std::stable_sort(cl, cl + n, [](const C& x, const C& y) { return x.vol > y.vol; });
  int before = 0;
  for (int i = 0; i < n; ++i) {
    fa.cls[i] = cl[i].rc;
    fa.cls[i].before = before;
    before += cl[i].rc.nr[0] * cl[i].rc.nr[1] * cl[i].rc.nr[2];
  }
  fa.n_cls = n;
  return true;
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
  SicsFusedArgs fa;
  if (sics_fused_plan(cand, n_cand, fa)) {
    long long off = 0;
    for (int c = 0; c < n_cand; ++c) {
      ra.off[c] = fa.out_off[c] = off;
      ra.nb[c] = cand[c].nb;
      off += (long long)heads * cand[c].nb;
    }
    fa.heads = heads;
    fa.row_bytes = row_bytes;
    cudaError_t e;
    if (dt == SPADE_BF16 && lph == 16) e = launch_fused<true, 16>(q, k, ws, fa, s);
    else if (dt == SPADE_BF16 && lph == 8) e = launch_fused<true, 8>(q, k, ws, fa, s);
    else if (dt == SPADE_F32 && lph == 32) e = launch_fused<false, 32>(q, k, ws, fa, s);
    else if (dt == SPADE_F32 && lph == 16) e = launch_fused<false, 16>(q, k, ws, fa, s);
    else return cudaErrorInvalidValue;
    if (e != cudaSuccess) return e;
    sics_reduce_kernel<<<heads, 256, 0, s>>>(ws, ra, scores, choice);
    return cudaGetLastError();
  }
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
