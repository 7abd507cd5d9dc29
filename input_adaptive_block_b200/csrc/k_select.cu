// Step 4: the executor's index search, and the cost-ranked work list.
//
// SPADE abstract (catalyzex.com): the executor performs a "low-overhead index
// search"; technical summary (gist.science/paper/2608.03335), Methodology 3,
// "Flash Block-Sparse Attention": masks are turned into a ranked block-sparse
// representation for sequential access.
//
// Per (head, query block i): keep i, then the other key blocks in descending
// probability (ties -> lower id) until the kept mass reaches tau.  One warp
// per row and no sort of the row:
//  * masses are fixed point, m_j = round(p_j * 2^30) (scaled down for a row
//    that sums to more than 1), so every sum is exact and the same in any
//    order; the keys are the IEEE-754 bit patterns of p_j, which order
//    non-negative floats like their values;
//  * a radix select finds the cut key theta.  Level 1 adds the masses into
//    1024 bins of 1/32 octave below 1.0 (shared-memory integer atomics, in
//    the same pass that forms the keys and masses); a prefix over the bins,
//    largest keys first, gives the bin holding the cut.  The keys inside that bin are compacted and then
//    sorted across the warp (up to 32 of them) or radix-selected on their
//    bits, 10 at a time.  Blocks above theta are kept, and of the blocks tied
//    at theta the lowest ids until the mass reaches tau;
//  * in score mode the row holds the scaled pooled scores
//    Qbar_i . Kbar_j / sqrt(d): the kernel forms the Estimator's softmax
//    itself, so the probabilities never travel through memory.
// Kept ids are written in ascending order (sequential K/V access) through a
// shared-memory stage, as whole 16-byte stores; a second kernel ranks the
// (head, query block) items by cost for the attention scheduler.
#include "spade_internal.cuh"

namespace spade {
namespace {

struct SelectTaus {
  float tau[SPADE_SELECT_MAX_HEADS];
  // static windows (WIN kernels only): block radii per head and the block grid
  unsigned char rad[SPADE_SELECT_MAX_HEADS][3];
  int nbh, nbw;
};

constexpr int kSelWarps = 4;
constexpr int kBins = 1024;
constexpr int kOctShift = 18;              // 1/32-octave bins: 5 mantissa bits above the low 18
constexpr uint32_t kOneKey = 0x3F800000u;  // bit pattern of 1.0f, the largest key
constexpr uint32_t kFull = 0xffffffffu;
constexpr float kMassOne = 1073741824.0f;  // 2^30: fixed-point mass of probability 1

__device__ __forceinline__ uint32_t warp_sum(uint32_t v) { return __reduce_add_sync(kFull, v); }
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(kFull, v, o);
  return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v = fmaxf(v, __shfl_xor_sync(kFull, v, o));
  return v;
}
// inclusive prefix over the lanes
__device__ __forceinline__ uint32_t warp_incl(uint32_t v, int lane) {
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t t = __shfl_up_sync(kFull, v, o);
    if (lane >= o) v += t;
  }
  return v;
}

__device__ __forceinline__ uint32_t fixed_mass(uint32_t key, float scale) {
  return __float2uint_rn(__uint_as_float(key) * scale);
}

__device__ __forceinline__ void zero_bins(uint32_t* bins, int lane) {
  for (int c = 4 * lane; c < kBins; c += 128) *reinterpret_cast<uint4*>(bins + c) = make_uint4(0u, 0u, 0u, 0u);
}

// bins[0..1024): masses by digit, digit 0 holding the largest keys.  Returns
// the smallest digit whose inclusive prefix reaches r (the whole array must
// reach it) and, in *before, the mass of the digits ahead of it.
__device__ __forceinline__ int find_bin(const uint32_t* bins, uint32_t r, int lane, uint32_t* before) {
  const uint4* b4 = reinterpret_cast<const uint4*>(bins + 32 * lane);
  uint32_t tot = 0;
#pragma unroll
  for (int q = 0; q < 8; ++q) {                 // rotated so the lanes of a phase hit different banks
    const uint4 v = b4[(q + lane) & 7];
    tot += (v.x + v.y) + (v.z + v.w);
  }
  const uint32_t pre = warp_incl(tot, lane);
  const int L = max(__ffs(__ballot_sync(kFull, pre >= r)) - 1, 0);
  const uint32_t base = __shfl_sync(kFull, pre - tot, L);
  const uint32_t w = bins[32 * L + lane];
  const uint32_t pre2 = warp_incl(w, lane);
  const int K = max(__ffs(__ballot_sync(kFull, base + pre2 >= r)) - 1, 0);
  *before = base + __shfl_sync(kFull, pre2 - w, K);
  return 32 * L + K;
}

// The index search of one row whose values (scores or probabilities) are in
// x[] -- lane owns blocks j = lane*NPL .. lane*NPL + NPL - 1, read as -inf
// (scores) or 0 (probabilities) past nb -- for row i of head h: writes the
// kept ids (ascending) to idx_row and their number to *cnt_out.  bins: the
// warp's 1024 shared-memory bins; cb: the warp's NPL * 32 words of
// shared-memory stage.  vec: idx_row is 16-byte aligned (nb % 4 == 0).
// WIN: the static window of block radii (rt, ry, rx) around i replaces the
// diagonal: its blocks are kept first and their mass counts toward tau.
// SCORES: x holds scores (softmax formed here) instead of probabilities.
template <int NPL, bool WIN, bool SCORES>
__device__ __forceinline__ void select_row(float (&x)[NPL], const SelectTaus& taus, int h, int i, int nb, int vec,
                                           uint32_t* bins, uint32_t* cb, int* cnt_out, int* idx_row, int lane) {
  const int j0 = lane * NPL;
  zero_bins(bins, lane);                           // while the row is in flight
  float scale = kMassOne, pmul = 1.0f;
  if (SCORES) {
    // the Estimator's softmax over the row's valid key blocks: p_j = x_j * pmul
    float mx = -INFINITY;
#pragma unroll
    for (int e = 0; e < NPL; ++e) mx = fmaxf(mx, x[e]);
    mx = warp_max(mx);
    float l = 0.f;
#pragma unroll
    for (int e = 0; e < NPL; ++e) {
      const float t = __expf(x[e] - mx);          // 0 past nb
      x[e] = t;
      l += t;
    }
    pmul = 1.0f / warp_sum(l);
  } else {
    float sum = 0.f;
#pragma unroll
    for (int e = 0; e < NPL; ++e) {
      x[e] = fminf(fmaxf(x[e], 0.f), 1.0f);      // NaN -> 0
      sum += x[e];
    }
    sum = warp_sum(sum);
    if (sum > 1.0f) scale = kMassOne / sum;      // masses of the whole row stay below 2^31
  }
  __syncwarp();                                    // bins zeroed by every lane
  // one pass: keys, fixed-point masses, the window (or the diagonal) set
  // aside, and level 1 of the radix select -- masses into bins of 1/32
  // octave below 1.0 (digit 0 = the largest keys; masses of keys below
  // 2^-31 round to zero, so every digit is < 1024)
  uint32_t key[NPL];
  uint32_t win = 0, dl = 0, ml = 0;
  int it = 0, iy = 0, ix = 0, jt = 0, jy = 0, jx = 0;
  if (WIN) {
    const int plane = taus.nbh * taus.nbw;
    it = i / plane; iy = (i / taus.nbw) % taus.nbh; ix = i % taus.nbw;
    jt = j0 / plane; jy = (j0 / taus.nbw) % taus.nbh; jx = j0 % taus.nbw;
  }
#pragma unroll
  for (int e = 0; e < NPL; ++e) {
    const int j = j0 + e;
    bool in_win = j == i;
    if (WIN) {
      in_win = abs(jt - it) <= taus.rad[h][0] && abs(jy - iy) <= taus.rad[h][1] && abs(jx - ix) <= taus.rad[h][2];
      if (++jx == taus.nbw) {
        jx = 0;
        if (++jy == taus.nbh) { jy = 0; ++jt; }
      }
    }
    const float p = SCORES ? x[e] * pmul : x[e];   // <= 1 (a product of two values <= 1); 0 past nb
    const uint32_t m = __float2uint_rn(p * scale);
    uint32_t k = 0u;
    if ((WIN ? j < nb : true) && in_win) {         // without a window, j == i < nb
      win |= 1u << e;
      dl += m;
    } else if (m > 0u) {                           // massless blocks are never needed
      k = __float_as_uint(p);
      ml += m;
      atomicAdd(&bins[(kOneKey - k) >> kOctShift], m);
    }
    key[e] = k;
  }
  const uint32_t D = warp_sum(dl), Mr = warp_sum(ml);
  const float tau = taus.tau[h];
  bool keep_all = !(tau < 1.0f);                   // tau >= 1 keeps every block
  uint32_t T = 0;
  if (!keep_all) {
    T = tau > 0.f ? (uint32_t)ceil((double)tau * (double)scale) : 0u;
    keep_all = (unsigned long long)D + Mr < (unsigned long long)T;   // the mass never reaches tau
  }
  uint32_t keep = 0;
  if (!keep_all && D < T) {
    __syncwarp();                                  // every lane's masses are in the bins
    uint32_t r = T - D;                            // mass still needed from the other blocks (<= Mr)
    uint32_t ahead;
    const int d1 = find_bin(bins, r, lane, &ahead);
    r -= ahead;
    // keys of bin d1: (hi - 2^kOctShift, hi]
    const uint32_t lo = kOneKey - ((uint32_t)(d1 + 1) << kOctShift);
    uint32_t mc = 0;
#pragma unroll
    for (int e = 0; e < NPL; ++e) mc += (key[e] - lo - 1u) < (1u << kOctShift);
    const uint32_t inc = warp_incl(mc, lane);
    const int n1 = (int)__shfl_sync(kFull, inc, 31);
    uint32_t at = inc - mc;
#pragma unroll
    for (int e = 0; e < NPL; ++e)
      if ((key[e] - lo - 1u) < (1u << kOctShift)) cb[at++] = key[e];
    __syncwarp();
    uint32_t theta = 0, ntie = 0;
    if (n1 <= 32) {
      // bitonic sort of the bin's keys across the warp, descending
      uint32_t k = lane < n1 ? cb[lane] : 0u;
#pragma unroll
      for (int kk = 2; kk <= 32; kk <<= 1)
#pragma unroll
        for (int jj = kk >> 1; jj > 0; jj >>= 1) {
          const uint32_t o = __shfl_xor_sync(kFull, k, jj);
          const bool take_max = ((lane & kk) == 0) == ((lane & jj) == 0);
          k = take_max ? max(k, o) : min(k, o);
        }
      const uint32_t m = k ? fixed_mass(k, scale) : 0u;
      const uint32_t pre = warp_incl(m, lane);
      const int L = max(__ffs(__ballot_sync(kFull, pre >= r)) - 1, 0);
      theta = __shfl_sync(kFull, k, L);
      const uint32_t tb = __ballot_sync(kFull, k == theta);
      ntie = __popc(tb);
      r -= __shfl_sync(kFull, pre - m, __ffs(tb) - 1);   // mass of the keys above theta
    } else {
      // many keys in one bin (flat rows): radix-select their bits, 10 at a time
      for (int sh = 20; sh >= 0; sh -= 10) {
        __syncwarp();                              // previous reads of the bins are done
        zero_bins(bins, lane);
        __syncwarp();
        for (int c = lane; c < n1; c += 32) {
          const uint32_t k = cb[c];
          if ((k >> (sh + 10)) == (theta >> (sh + 10)))
            atomicAdd(&bins[kBins - 1 - ((k >> sh) & (kBins - 1))], fixed_mass(k, scale));
        }
        __syncwarp();
        uint32_t a;
        const int dg = find_bin(bins, r, lane, &a);
        r -= a;
        theta |= (uint32_t)(kBins - 1 - dg) << sh;
      }
      uint32_t tl = 0;
      for (int c = lane; c < n1; c += 32) tl += cb[c] == theta;
      ntie = warp_sum(tl);
    }
    // keep the keys above theta, and of those equal to it the lowest ids
    // until the mass reaches tau
    const uint32_t mt = max(fixed_mass(theta, scale), 1u);
    const uint32_t need = (r + mt - 1) / mt;
    if (ntie <= need) {
#pragma unroll
      for (int e = 0; e < NPL; ++e) keep |= (uint32_t)(key[e] >= theta) << e;
    } else {
      uint32_t tl = 0;
#pragma unroll
      for (int e = 0; e < NPL; ++e) tl += key[e] == theta;
      uint32_t trank = warp_incl(tl, lane) - tl;
#pragma unroll
      for (int e = 0; e < NPL; ++e) {
        if (key[e] > theta) {
          keep |= 1u << e;
        } else if (key[e] == theta) {
          if (trank < need) keep |= 1u << e;
          ++trank;
        }
      }
    }
  }
  if (keep_all) {
    keep = 0;
#pragma unroll
    for (int e = 0; e < NPL; ++e)
      if (j0 + e < nb) keep |= 1u << e;
  } else {
    keep |= win;                                   // the diagonal (or the static window) is always kept
  }
  // ascending ids through the row's shared-memory stage
  const uint32_t mine = __popc(keep);
  const uint32_t oinc = warp_incl(mine, lane);
  const int total = (int)__shfl_sync(kFull, oinc, 31);
  uint32_t at = oinc - mine;
  uint32_t* ob = cb;
  __syncwarp();                                    // the compacted keys have been read
#pragma unroll
  for (int e = 0; e < NPL; ++e)
    if (keep & (1u << e)) ob[at++] = (uint32_t)(j0 + e);
  __syncwarp();
  int* out = idx_row;
  if (vec) {
    for (int c = 4 * lane; c < total; c += 128) {
      if (c + 4 <= total) {
        *reinterpret_cast<uint4*>(out + c) = *reinterpret_cast<const uint4*>(ob + c);
      } else {
        for (int t = c; t < total; ++t) out[t] = (int)ob[t];
      }
    }
  } else {
    for (int c = lane; c < total; c += 32) out[c] = (int)ob[c];
  }
  if (lane == 0) *cnt_out = total;
  __syncwarp();                                    // the stage and bins are free for the warp's next row
}

// NPL: blocks per lane (lane owns j = lane*NPL .. lane*NPL + NPL - 1).
// WIN, SCORES: as for select_row.  vec: rows of `in` and `idx` are 16-byte
// aligned (nb % 4 == 0).
template <int NPL, bool WIN, bool SCORES>
__global__ void __launch_bounds__(kSelWarps * 32, NPL > 24 ? 6 : 8) select_kernel(const float* __restrict__ in,
                                                                  const __grid_constant__ SelectTaus taus,
                                                                  int* __restrict__ cnt, int* __restrict__ idx,
                                                                  int heads, int nb, int vec) {
  __shared__ __align__(16) uint32_t sbuf[kSelWarps][NPL * 32];   // compacted keys, then the output stage
  __shared__ __align__(16) uint32_t sbin[kSelWarps][kBins];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long row = (long long)blockIdx.x * kSelWarps + warp;
  if (row >= (long long)heads * nb) return;
  const int h = (int)(row / nb);
  const int i = (int)(row - (long long)h * nb);
  const float* prow = in + row * nb;
  const int j0 = lane * NPL;
  // blocks past nb read as -inf (scores: exp gives 0) or 0 (probabilities),
  // so the passes of select_row need no per-block range test
  const float pad = SCORES ? -INFINITY : 0.f;
  float x[NPL];
  if (vec) {
#pragma unroll
    for (int q = 0; q < NPL / 4; ++q) {
      float4 v = make_float4(pad, pad, pad, pad);
      if (j0 + 4 * q < nb) v = __ldg(reinterpret_cast<const float4*>(prow + j0) + q);
      x[4 * q] = v.x; x[4 * q + 1] = v.y; x[4 * q + 2] = v.z; x[4 * q + 3] = v.w;
    }
  } else {
#pragma unroll
    for (int e = 0; e < NPL; ++e) x[e] = j0 + e < nb ? __ldg(prow + j0 + e) : pad;
  }
  select_row<NPL, WIN, SCORES>(x, taus, h, i, nb, vec, sbin[warp], sbuf[warp], cnt + row, idx + row * nb, lane);
}

// ------------------------------------------------------------ work list --
// Items (head, query block) in head-major order; inside a head, ranked by
// cost = number of key blocks walked, descending (longest first), by a
// counting sort -- one CTA per head.  Consecutive items then share a head, so
// the K/V blocks that persistent attention CTAs work on at any time stay
// L2-resident, and long lists start before short ones.  CTA 0 also resets the
// ticket the attention kernel hands the list out with.
struct WorklistArgs {
  int heads;
  int ntb;
  int n_items;
  int item_start[SPADE_MAX_HEADS + 1];   // prefix sum of items per head
  int nb[SPADE_MAX_HEADS];
  int dense[SPADE_MAX_HEADS];
  int cnt_off[SPADE_MAX_HEADS];
};

constexpr int kWlThreads = 512;

__device__ __forceinline__ int item_cost(const WorklistArgs& a, const int* cnt, int h, int qb) {
  const int nb = a.nb[h];
  if (a.dense[h] || qb >= nb) return nb + a.ntb;
  return cnt[a.cnt_off[h] + qb] + a.ntb;
}

__global__ void __launch_bounds__(kWlThreads) worklist_kernel(const __grid_constant__ WorklistArgs a,
                                                              const int* __restrict__ cnt,
                                                              int* __restrict__ work, int* __restrict__ ticket) {
  __shared__ int hist[SPADE_WORKLIST_MAX_COST];
  __shared__ int warp_tot[kWlThreads / 32];
  const int tid = threadIdx.x;
  const int h = blockIdx.x;
  if (h == 0 && tid == 0) *ticket = 0;
  const int base = a.item_start[h];
  const int n = a.item_start[h + 1] - base;
  for (int i = tid; i < SPADE_WORKLIST_MAX_COST; i += kWlThreads) hist[i] = 0;
  __syncthreads();
  for (int qb = tid; qb < n; qb += kWlThreads) {
    const int c = min(item_cost(a, cnt, h, qb), SPADE_WORKLIST_MAX_COST - 1);
    atomicAdd(&hist[SPADE_WORKLIST_MAX_COST - 1 - c], 1);
  }
  __syncthreads();
  // exclusive scan over bins: each thread owns PER consecutive bins
  constexpr int PER = SPADE_WORKLIST_MAX_COST / kWlThreads;
  int local[PER];
  int s = 0;
#pragma unroll
  for (int e = 0; e < PER; ++e) { local[e] = hist[tid * PER + e]; s += local[e]; }
  const int lane = tid & 31, warp = tid >> 5;
  int inc = s;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int t = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += t;
  }
  if (lane == 31) warp_tot[warp] = inc;
  __syncthreads();
  if (warp == 0) {
    int w = lane < kWlThreads / 32 ? warp_tot[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int t = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += t;
    }
    if (lane < kWlThreads / 32) warp_tot[lane] = w;
  }
  __syncthreads();
  int off = inc - s + (warp > 0 ? warp_tot[warp - 1] : 0);
#pragma unroll
  for (int e = 0; e < PER; ++e) { hist[tid * PER + e] = off; off += local[e]; }
  __syncthreads();
  for (int qb = tid; qb < n; qb += kWlThreads) {
    const int c = min(item_cost(a, cnt, h, qb), SPADE_WORKLIST_MAX_COST - 1);
    const int pos = atomicAdd(&hist[SPADE_WORKLIST_MAX_COST - 1 - c], 1);
    work[base + pos] = (h << 16) | qb;
  }
}

template <int NPL>
cudaError_t launch_select_t(const float* in, const SelectTaus& t, bool win, bool scores, int vec, int* cnt,
                            int* idx, int heads, int nb, cudaStream_t s) {
  const long long rows = (long long)heads * nb;
  const int blocks = (int)((rows + kSelWarps - 1) / kSelWarps);
  const dim3 grid(blocks), block(kSelWarps * 32);
  if (win) {
    if (scores) select_kernel<NPL, true, true><<<grid, block, 0, s>>>(in, t, cnt, idx, heads, nb, vec);
    else select_kernel<NPL, true, false><<<grid, block, 0, s>>>(in, t, cnt, idx, heads, nb, vec);
  } else {
    if (scores) select_kernel<NPL, false, true><<<grid, block, 0, s>>>(in, t, cnt, idx, heads, nb, vec);
    else select_kernel<NPL, false, false><<<grid, block, 0, s>>>(in, t, cnt, idx, heads, nb, vec);
  }
  return cudaGetLastError();
}


// Fills the per-thread staging of taus (and window radii); returns whether any window is set.
bool stage_taus(SelectTaus& t, const float* tau_host, int heads, const int* radius_host, const Geo* g) {
  for (int h = 0; h < heads; ++h) t.tau[h] = tau_host[h];
  bool win = false;
  if (radius_host && g) {
    for (int h = 0; h < heads; ++h)
      for (int a = 0; a < 3; ++a) {
        t.rad[h][a] = (unsigned char)(radius_host[3 * h + a] > 255 ? 255 : radius_host[3 * h + a]);
        win = win || radius_host[3 * h + a] > 0;
      }
    t.nbh = g->nbh;
    t.nbw = g->nbw;
  }
  return win;
}

}  // namespace

cudaError_t launch_select(const float* in, const float* tau_host, int* cnt, int* idx, int heads, int nb,
                          cudaStream_t s, const int* radius_host, const Geo* g, bool scores) {
  // host staging (large), one per calling thread: the launch copies it into
  // the kernel's parameter buffer, so concurrent callers never share it
  thread_local SelectTaus t;
  const bool win = stage_taus(t, tau_host, heads, radius_host, g);
  const int vec = (nb % 4 == 0) && (reinterpret_cast<uintptr_t>(in) % 16 == 0) &&
                  (reinterpret_cast<uintptr_t>(idx) % 16 == 0);
  const int npl = (nb + 31) / 32;
  if (npl <= 4) return launch_select_t<4>(in, t, win, scores, vec, cnt, idx, heads, nb, s);
  if (npl <= 8) return launch_select_t<8>(in, t, win, scores, vec, cnt, idx, heads, nb, s);
  if (npl <= 12) return launch_select_t<12>(in, t, win, scores, vec, cnt, idx, heads, nb, s);
  if (npl <= 16) return launch_select_t<16>(in, t, win, scores, vec, cnt, idx, heads, nb, s);
  if (npl <= 20) return launch_select_t<20>(in, t, win, scores, vec, cnt, idx, heads, nb, s);
  if (npl <= 24) return launch_select_t<24>(in, t, win, scores, vec, cnt, idx, heads, nb, s);
  return launch_select_t<32>(in, t, win, scores, vec, cnt, idx, heads, nb, s);
}

cudaError_t launch_worklist(const AttnArgs& a, cudaStream_t s) {
  WorklistArgs w;
  w.heads = a.heads;
  w.ntb = text_blocks(a.text_tokens);
  int acc = 0;
  for (int h = 0; h < a.heads; ++h) {
    w.item_start[h] = acc;
    w.nb[h] = a.head[h].nb;
    w.dense[h] = a.head[h].dense;
    w.cnt_off[h] = a.head[h].cnt_off;
    acc += a.head[h].nb + w.ntb;
  }
  w.item_start[a.heads] = acc;
  w.n_items = acc;
  worklist_kernel<<<a.heads, kWlThreads, 0, s>>>(w, a.cnt, a.work, a.ticket);
  return cudaGetLastError();
}

}  // namespace spade
