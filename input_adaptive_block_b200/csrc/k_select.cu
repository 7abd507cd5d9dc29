// Step 4: the executor's index search, and the cost-ranked work list.
//
// SPADE abstract (catalyzex.com): the executor performs a "low-overhead index
// search"; technical summary (gist.science/paper/2608.03335), Methodology 3,
// "Flash Block-Sparse Attention": masks are turned into a ranked block-sparse
// representation for sequential access.
//
// Per (head, query block i): keep i, then the other key blocks in descending
// probability (ties -> lower id) until the kept mass reaches tau.  Instead of
// sorting, one warp per row finds the cut value by a binary search over the
// IEEE-754 bit pattern (monotone for non-negative floats): the largest theta
// with  p_ii + sum_{j != i, p_j >= theta} p_j >= tau.  Blocks above theta are
// kept, ties at theta are taken lowest id first.  Kept ids are written in
// ascending order (sequential K/V access); a second kernel ranks the
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

constexpr int kSelWarps = 8;
constexpr int kFineBits = 18;   // low bits of theta bisected over the compacted candidates only

// WIN: the static window of block radii (rt, ry, rx) around i replaces the
// diagonal: its blocks are kept first and their mass counts toward tau.
template <int NPL, bool WIN>
__global__ void __launch_bounds__(kSelWarps * 32) select_kernel(const float* __restrict__ prob,
                                                               const __grid_constant__ SelectTaus taus,
                                                               int* __restrict__ cnt, int* __restrict__ idx,
                                                               int heads, int nb) {
  __shared__ float buf[kSelWarps][NPL * 32];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long row = (long long)blockIdx.x * kSelWarps + warp;
  if (row >= (long long)heads * nb) return;
  const int h = (int)(row / nb);
  const int i = (int)(row - (long long)h * nb);
  const float* prow = prob + row * nb;
  float* b = buf[warp];
  {
    // coalesced row load, every load in flight before the first store
    float t[NPL];
#pragma unroll
    for (int e = 0; e < NPL; ++e) {
      const int j = lane + 32 * e;
      t[e] = j < nb ? __ldg(prow + j) : 0.f;
    }
#pragma unroll
    for (int e = 0; e < NPL; ++e) b[lane + 32 * e] = t[e];
  }
  __syncwarp();
  const float tau = taus.tau[h];
  // lane owns j in [lane*NPL, lane*NPL + NPL): contiguous, so ascending output is a lane-order scan
  float v[NPL];
  uint32_t win = 0;   // bit e: element lane*NPL+e lies in the window (always kept)
#pragma unroll
  for (int e = 0; e < NPL; ++e) {
    const int j = lane * NPL + e;
    bool in = j == i;
    if (WIN && j < nb) {
      const int it = i / (taus.nbh * taus.nbw), iy = (i / taus.nbw) % taus.nbh, ix = i % taus.nbw;
      const int jt = j / (taus.nbh * taus.nbw), jy = (j / taus.nbw) % taus.nbh, jx = j % taus.nbw;
      in = abs(jt - it) <= taus.rad[h][0] && abs(jy - iy) <= taus.rad[h][1] && abs(jx - ix) <= taus.rad[h][2];
    }
    if (in && j < nb) win |= 1u << e;
    v[e] = (j < nb && !in) ? b[j] : -1.0f;   // -1: never reaches a non-negative threshold
  }
  // mass of the window (just p_ii without one: adding zeros is exact)
  float diag = 0.f;
#pragma unroll
  for (int e = 0; e < NPL; ++e)
    if (win & (1u << e)) diag += b[lane * NPL + e];
#pragma unroll
  for (int o = 16; o; o >>= 1) diag += __shfl_xor_sync(0xffffffffu, diag, o);
  uint32_t keep = 0;   // bit e: element lane*NPL+e kept
  bool keep_all = tau >= 1.0f;
  if (!keep_all && diag < tau) {
    uint32_t u = 0;
    // bits 29..18 over every element (p <= 1 < 2.0f = 0x40000000) ...
    for (int bit = 29; bit >= kFineBits; --bit) {
      const uint32_t cand = u | (1u << bit);
      const float thr = __uint_as_float(cand);
      float s4[4] = {0.f, 0.f, 0.f, 0.f};                // four short chains instead of one long one
#pragma unroll
      for (int e = 0; e < NPL; ++e) s4[e & 3] += (v[e] >= thr) ? v[e] : 0.f;
      float s = (s4[0] + s4[1]) + (s4[2] + s4[3]);
#pragma unroll
      for (int o = 16; o; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
      if (diag + s >= tau) u = cand;
    }
    // ... then theta lies in [u, u + 2^kFineBits): the mass above that bracket
    // counts as a constant and the remaining bits are bisected over the few
    // elements inside it, compacted into the row buffer
    {
      const uint32_t top = u + (1u << kFineBits);
      float s4[4] = {0.f, 0.f, 0.f, 0.f};
      int mc = 0;
#pragma unroll
      for (int e = 0; e < NPL; ++e) {
        const uint32_t bits = __float_as_uint(v[e]);
        const bool pos = v[e] >= 0.f;
        s4[e & 3] += (pos && bits >= top) ? v[e] : 0.f;
        mc += (pos && bits >= u && bits < top);
      }
      float above = (s4[0] + s4[1]) + (s4[2] + s4[3]);
#pragma unroll
      for (int o = 16; o; o >>= 1) above += __shfl_xor_sync(0xffffffffu, above, o);
      int at = mc;                                   // inclusive scan of the candidate counts
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int t = __shfl_up_sync(0xffffffffu, at, o);
        if (lane >= o) at += t;
      }
      const int ncand = __shfl_sync(0xffffffffu, at, 31);
      at -= mc;
      __syncwarp();                                  // every lane has read its row elements from b
#pragma unroll
      for (int e = 0; e < NPL; ++e) {
        const uint32_t bits = __float_as_uint(v[e]);
        if (v[e] >= 0.f && bits >= u && bits < top) b[at++] = v[e];
      }
      __syncwarp();
      const float base = diag + above;
      for (int bit = kFineBits - 1; bit >= 0; --bit) {
        const uint32_t cand = u | (1u << bit);
        const float thr = __uint_as_float(cand);
        float s2 = 0.f;
        for (int c = lane; c < ncand; c += 32) s2 += (b[c] >= thr) ? b[c] : 0.f;
#pragma unroll
        for (int o = 16; o; o >>= 1) s2 += __shfl_xor_sync(0xffffffffu, s2, o);
        if (base + s2 >= tau) u = cand;
      }
    }
    if (u == 0) {
      keep_all = true;                               // the mass never reaches tau
    } else {
      const float theta = __uint_as_float(u);
      float above = 0.f;
      int ties = 0;
#pragma unroll
      for (int e = 0; e < NPL; ++e) {
        if (v[e] > theta) { keep |= 1u << e; above += v[e]; }
        ties += (v[e] == theta);
      }
#pragma unroll
      for (int o = 16; o; o >>= 1) {
        above += __shfl_xor_sync(0xffffffffu, above, o);
        ties += __shfl_xor_sync(0xffffffffu, ties, o);
      }
      if (ties == 1) {
#pragma unroll
        for (int e = 0; e < NPL; ++e)
          if (v[e] == theta) keep |= 1u << e;
      } else {
        float mass = diag + above;                   // take tied blocks lowest id first
        for (int L = 0; L < 32; ++L) {
          for (int e = 0; e < NPL; ++e) {
            const bool tie = __shfl_sync(0xffffffffu, v[e] == theta ? 1 : 0, L) != 0;
            if (tie && mass < tau) {
              if (lane == L) keep |= 1u << e;
              mass += theta;
            }
          }
        }
      }
    }
  }
  if (keep_all) {
    keep = 0;
#pragma unroll
    for (int e = 0; e < NPL; ++e)
      if (lane * NPL + e < nb) keep |= 1u << e;
  } else {
    keep |= win;                                   // the diagonal (or the static window) is always kept
  }
  const int mine = __popc(keep);
  int pre = mine;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int t = __shfl_up_sync(0xffffffffu, pre, o);
    if (lane >= o) pre += t;
  }
  const int total = __shfl_sync(0xffffffffu, pre, 31);
  int* out = idx + row * nb + (pre - mine);
  int w = 0;
#pragma unroll
  for (int e = 0; e < NPL; ++e)
    if (keep & (1u << e)) out[w++] = lane * NPL + e;
  if (lane == 0) cnt[row] = total;
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
cudaError_t launch_select_t(const float* prob, const SelectTaus& t, bool win, int* cnt, int* idx, int heads, int nb,
                            cudaStream_t s) {
  const long long rows = (long long)heads * nb;
  const int blocks = (int)((rows + kSelWarps - 1) / kSelWarps);
  if (win) select_kernel<NPL, true><<<blocks, kSelWarps * 32, 0, s>>>(prob, t, cnt, idx, heads, nb);
  else select_kernel<NPL, false><<<blocks, kSelWarps * 32, 0, s>>>(prob, t, cnt, idx, heads, nb);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_select(const float* prob, const float* tau_host, int* cnt, int* idx, int heads, int nb,
                          cudaStream_t s, const int* radius_host, const Geo* g) {
  static SelectTaus t;   // host staging (large); launches copy it into the parameter buffer
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
  const int npl = (nb + 31) / 32;
  if (npl <= 4) return launch_select_t<4>(prob, t, win, cnt, idx, heads, nb, s);
  if (npl <= 8) return launch_select_t<8>(prob, t, win, cnt, idx, heads, nb, s);
  if (npl <= 16) return launch_select_t<16>(prob, t, win, cnt, idx, heads, nb, s);
  if (npl <= 24) return launch_select_t<24>(prob, t, win, cnt, idx, heads, nb, s);
  return launch_select_t<32>(prob, t, win, cnt, idx, heads, nb, s);
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
