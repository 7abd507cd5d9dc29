// Step 1 (3D tiling) and step 2 (block-mean Summarizer) of the SPADE executor.
//
// SPADE technical summary (gist.science/paper/2608.03335), Methodology 1,
// "Blocking Scheme Candidates" and "Summarizer & Estimator Expressions";
// Methodology 3, "Kernel Fusion" (layout transformation fused with
// summarization).  The summarizer below reads Q/K in token order and reduces
// each 3D block directly, so the tiled layout is never written on the hot
// path; the attention kernel gathers its tiles with TMA boxes instead.
#include "spade_internal.cuh"

namespace spade {
namespace {

// ---------------------------------------------------------------- tile3d --
// One CTA per block; each thread moves 16-byte chunks.  Source rows are whole
// token rows (all heads), so reads are fully coalesced; each (head, slot)
// destination segment is d*esz contiguous bytes.
__global__ void tile3d_kernel(const uint8_t* __restrict__ x, uint8_t* __restrict__ xt, Geo g, int heads,
                              int row_bytes_head) {
  const int b = blockIdx.x;
  int t0, y0, x0, et, eh, ew;
  block_box(g, b, t0, y0, x0, et, eh, ew);
  const int chunks_head = row_bytes_head / 16;
  const int chunks_tok = chunks_head * heads;
  const long long row_bytes = (long long)row_bytes_head * heads;
  const int total = g.bs * chunks_tok;
  for (int i = threadIdx.x; i < total; i += blockDim.x) {
    const int slot = i / chunks_tok;
    const int c = i - slot * chunks_tok;
    const int h = c / chunks_head;
    const int cc = c - h * chunks_head;
    const int xl = slot % g.bw;
    const int yl = (slot / g.bw) % g.bh;
    const int tl = slot / (g.bw * g.bh);
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (tl < et && yl < eh && xl < ew) {
      const long long tok = ((long long)(t0 + tl) * g.H + (y0 + yl)) * g.W + (x0 + xl);
      v = __ldg(reinterpret_cast<const uint4*>(x + tok * row_bytes) + c);
    }
    uint8_t* dst = xt + (((long long)h * g.nb + b) * g.bs + slot) * row_bytes_head;
    reinterpret_cast<uint4*>(dst)[cc] = v;
  }
}

// ------------------------------------------------------------- summarize --
// Work unit = (block b, group of 32 16-byte chunks of a token row restricted
// to heads [h0, h0+hc)).  One warp per unit; lane l owns chunk 32*group + l
// and sums it over the block's valid tokens in fp32.  The block's tokens are
// walked in (t, y, x) order by stepping a pointer (no integer division on
// the load path), eight loads in flight per lane.  Units are dealt
// round-robin to all warps.
// MODE: 0 mean (sum, divided at the end), 1 max, 2 min -- the Summarizer's
// reduces (Methodology 1 names max / min / mean).
template <int MODE>
__device__ __forceinline__ float combine(float a, float v) {
  return MODE == 0 ? a + v : (MODE == 1 ? fmaxf(a, v) : fminf(a, v));
}

template <bool BF16, int MODE>
__device__ __forceinline__ void accumulate(float (&acc)[BF16 ? 8 : 4], const uint4& v) {
  if (BF16) {
    const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 f = __bfloat1622float2(p[e]);
      acc[2 * e] = combine<MODE>(acc[2 * e], f.x);
      acc[2 * e + 1] = combine<MODE>(acc[2 * e + 1], f.y);
    }
  } else {
    const float* f = reinterpret_cast<const float*>(&v);
#pragma unroll
    for (int e = 0; e < (BF16 ? 8 : 4); ++e) acc[e] = combine<MODE>(acc[e], f[e]);
  }
}

// Two tensors (Q and K) can share one launch: units [0, n) read in0 into
// out0, units [n, 2n) read in1 into out1 (in1 == nullptr: one tensor).
template <bool BF16, int MODE>
__global__ void __launch_bounds__(256, 5) summarize_kernel(const uint8_t* __restrict__ in0,
                                                         const uint8_t* __restrict__ in1,
                                                         float* __restrict__ out0, float* __restrict__ out1,
                                                         Geo g, long long row_bytes, int head_off_bytes,
                                                         int chunks, int d) {
  constexpr int EPC = BF16 ? 8 : 4;  // elements per 16-byte chunk
  const int lane = threadIdx.x & 31;
  const int gwarp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int nwarps = (gridDim.x * blockDim.x) >> 5;
  const int groups = (chunks + 31) / 32;
  const long long n_units = (long long)g.nb * groups;
  const long long all_units = in1 ? 2 * n_units : n_units;
  const long long sy = (long long)g.W * row_bytes;     // next y row
  const long long st = (long long)g.H * sy;            // next frame
  for (long long uu = gwarp; uu < all_units; uu += nwarps) {
    const bool second = uu >= n_units;
    const long long u = second ? uu - n_units : uu;
    const uint8_t* x = second ? in1 : in0;
    float* out = second ? out1 : out0;
    const int b = (int)(u / groups);
    const int c = (int)(u - (long long)b * groups) * 32 + lane;
    int t0, y0, x0, et, eh, ew;
    block_box(g, b, t0, y0, x0, et, eh, ew);
    const int nvalid = et * eh * ew;
    float acc[EPC];
#pragma unroll
    for (int e = 0; e < EPC; ++e) acc[e] = MODE == 0 ? 0.f : (MODE == 1 ? -INFINITY : INFINITY);
    if (c < chunks) {
      // pointer to token (t0 + tl, y0 + yl, x0 + xl); stepping x, then y, then t
      const uint8_t* ptr = x + head_off_bytes + (long long)c * 16 +
                           (((long long)t0 * g.H + y0) * g.W + x0) * row_bytes;
      const long long wrap_y = sy - (long long)ew * row_bytes;
      const long long wrap_t = st - (long long)eh * sy;
      int xl = 0, yl = 0;
      auto step = [&]() {
        ptr += row_bytes;
        if (++xl == ew) {
          xl = 0;
          ptr += wrap_y;
          if (++yl == eh) {
            yl = 0;
            ptr += wrap_t;
          }
        }
      };
      int i = 0;
      for (; i + 8 <= nvalid; i += 8) {
        uint4 v[8];
#pragma unroll
        for (int r = 0; r < 8; ++r) {
          v[r] = __ldg(reinterpret_cast<const uint4*>(ptr));
          step();
        }
#pragma unroll
        for (int r = 0; r < 8; ++r) accumulate<BF16, MODE>(acc, v[r]);
      }
      for (; i < nvalid; ++i) {
        accumulate<BF16, MODE>(acc, __ldg(reinterpret_cast<const uint4*>(ptr)));
        step();
      }
      const float inv = MODE == 0 ? 1.0f / (float)nvalid : 1.0f;
      const int e0 = c * EPC;             // element index within the head-range row
      const int h = e0 / d, dd = e0 - h * d;
      float* o = out + ((long long)h * g.nb + b) * d + dd;
      reinterpret_cast<float4*>(o)[0] = make_float4(acc[0] * inv, acc[1] * inv, acc[2] * inv, acc[3] * inv);
      if (BF16)
        reinterpret_cast<float4*>(o)[1] = make_float4(acc[4] * inv, acc[5] * inv, acc[6] * inv, acc[7] * inv);
    }
  }
}

// Wide form (bf16): lane owns the two adjacent 16-byte chunks 2l, 2l+1 of a
// group of 64 (a warp covers 1 KB of the token row) and reads both with one
// 32-byte load per token: half the load instructions and pointer steps per
// byte.  Used when every row start is 32-byte aligned.
//
// Small layers have too few (block, chunk group) units to keep enough loads
// in flight with one warp per unit, so each unit's tokens can be split into
// S consecutive slices taken by S warps of one CTA (S = 1, 2, 4 or 8; the
// CTA's 8 warps hold 8 / S units per round).  The slices' partial results
// are combined through shared memory in slice order, so the result is
// deterministic and depends only on S, which the launcher derives from the
// geometry and the head range alone.
__device__ __forceinline__ void ld32(uint4& a, uint4& b, const uint8_t* p) {
  asm volatile("ld.global.nc.v8.u32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
               : "=r"(a.x), "=r"(a.y), "=r"(a.z), "=r"(a.w), "=r"(b.x), "=r"(b.y), "=r"(b.z), "=r"(b.w)
               : "l"(p));
}

template <bool BF16, int MODE>
__global__ void __launch_bounds__(256, 4) summarize_wide_kernel(const uint8_t* __restrict__ in0,
                                                              const uint8_t* __restrict__ in1,
                                                              float* __restrict__ out0, float* __restrict__ out1,
                                                              Geo g, long long row_bytes, int head_off_bytes,
                                                              int chunks, int d, int S) {
  constexpr int EPC = BF16 ? 8 : 4;  // elements per 16-byte chunk
  __shared__ float part[8][2 * EPC][32];   // per warp: its slice's partial result, element-major
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int per_cta = 8 / S;                 // units per CTA round
  const int slot = warp / S, sl = warp - slot * S;
  const int groups = (chunks + 63) / 64;
  const long long n_units = (long long)g.nb * groups;
  const long long all_units = in1 ? 2 * n_units : n_units;
  const long long sy = (long long)g.W * row_bytes;     // next y row
  const long long st = (long long)g.H * sy;            // next frame
  // the loop runs the same number of rounds on every warp of the CTA (S > 1 synchronises the CTA)
  for (long long ub = (long long)blockIdx.x * per_cta; ub < all_units; ub += (long long)gridDim.x * per_cta) {
    const long long uu = ub + slot;
    const bool active = uu < all_units;
    const bool second = active && uu >= n_units;
    const long long u = second ? uu - n_units : uu;
    const uint8_t* x = second ? in1 : in0;
    float* out = second ? out1 : out0;
    const int b = active ? (int)(u / groups) : 0;
    const int c = active ? (int)(u - (long long)b * groups) * 64 + 2 * lane : chunks;   // first of the lane's two
    int t0, y0, x0, et, eh, ew;
    block_box(g, b, t0, y0, x0, et, eh, ew);
    const int nvalid = et * eh * ew;
    float acc0[EPC], acc1[EPC];
#pragma unroll
    for (int e = 0; e < EPC; ++e) acc0[e] = acc1[e] = MODE == 0 ? 0.f : (MODE == 1 ? -INFINITY : INFINITY);
    // this warp's slice of the block's tokens, in (t, y, x) order
    const int per = (nvalid + S - 1) / S;
    const int i0 = min(nvalid, sl * per), i1 = min(nvalid, i0 + per);
    if (c < chunks && i0 < i1) {
      const int area = eh * ew;
      const int tl0 = i0 / area, r0 = i0 - tl0 * area;
      int yl = r0 / ew, xl = r0 - (r0 / ew) * ew;
      const uint8_t* ptr = x + head_off_bytes + (long long)c * 16 +
                           (((long long)(t0 + tl0) * g.H + (y0 + yl)) * g.W + (x0 + xl)) * row_bytes;
      const long long wrap_y = sy - (long long)ew * row_bytes;
      const long long wrap_t = st - (long long)eh * sy;
      auto step = [&]() {
        ptr += row_bytes;
        if (++xl == ew) {
          xl = 0;
          ptr += wrap_y;
          if (++yl == eh) {
            yl = 0;
            ptr += wrap_t;
          }
        }
      };
      const int n = i1 - i0;
      int i = 0;
      for (; i + 4 <= n; i += 4) {
        uint4 va[4], vb[4];
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          ld32(va[r], vb[r], ptr);
          step();
        }
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          accumulate<BF16, MODE>(acc0, va[r]);
          accumulate<BF16, MODE>(acc1, vb[r]);
        }
      }
      for (; i < n; ++i) {
        uint4 va, vb;
        ld32(va, vb, ptr);
        accumulate<BF16, MODE>(acc0, va);
        accumulate<BF16, MODE>(acc1, vb);
        step();
      }
    }
    if (S > 1) {
      // combine the S slices of each unit in slice order (the first warp of the unit writes)
#pragma unroll
      for (int e = 0; e < EPC; ++e) {
        part[warp][e][lane] = acc0[e];
        part[warp][EPC + e][lane] = acc1[e];
      }
      __syncthreads();
      if (sl == 0) {
        for (int o = 1; o < S; ++o) {
#pragma unroll
          for (int e = 0; e < EPC; ++e) {
            acc0[e] = combine<MODE>(acc0[e], part[warp + o][e][lane]);
            acc1[e] = combine<MODE>(acc1[e], part[warp + o][EPC + e][lane]);
          }
        }
      }
      __syncthreads();
    }
    if (sl == 0 && c < chunks) {
      const float inv = MODE == 0 ? 1.0f / (float)nvalid : 1.0f;
      const int e0 = c * EPC;             // element index within the head-range row (both chunks in one head)
      const int h = e0 / d, dd = e0 - h * d;
      float4* o = reinterpret_cast<float4*>(out + ((long long)h * g.nb + b) * d + dd);
      o[0] = make_float4(acc0[0] * inv, acc0[1] * inv, acc0[2] * inv, acc0[3] * inv);
      if (BF16) {
        o[1] = make_float4(acc0[4] * inv, acc0[5] * inv, acc0[6] * inv, acc0[7] * inv);
        o[2] = make_float4(acc1[0] * inv, acc1[1] * inv, acc1[2] * inv, acc1[3] * inv);
        o[3] = make_float4(acc1[4] * inv, acc1[5] * inv, acc1[6] * inv, acc1[7] * inv);
      } else {
        o[1] = make_float4(acc1[0] * inv, acc1[1] * inv, acc1[2] * inv, acc1[3] * inv);
      }
    }
  }
}

}  // namespace

cudaError_t launch_tile3d(const void* x, void* xt, const Geo& g, int heads, int d, spade_dtype dt,
                          cudaStream_t s) {
  const int esz = dt == SPADE_BF16 ? 2 : 4;
  tile3d_kernel<<<g.nb, 256, 0, s>>>(static_cast<const uint8_t*>(x), static_cast<uint8_t*>(xt), g, heads,
                                     d * esz);
  return cudaGetLastError();
}

// Grid: every warp takes the same number of (block, chunk group) units,
// dealt round-robin, with all warps resident at once (5 CTAs of 8 warps per
// SM): no partial last round of units while the rest of the GPU idles.
template <int MODE>
cudaError_t launch_summarize_m(const void* x0, const void* x1, float* out0, float* out1, const Geo& g,
                               int heads_total, int h0, int hc, int d, spade_dtype dt, cudaStream_t s) {
  const int esz = dt == SPADE_BF16 ? 2 : 4;
  const long long row_bytes = (long long)heads_total * d * esz;
  const int chunks = hc * d * esz / 16;
  const uint8_t* a = static_cast<const uint8_t*>(x0);
  const uint8_t* b = static_cast<const uint8_t*>(x1);
  const long long head_off = (long long)h0 * d * esz;
  const bool wide = dt == SPADE_BF16 && row_bytes % 32 == 0 && head_off % 32 == 0 &&
                    (reinterpret_cast<uintptr_t>(a) & 31) == 0 && (!b || (reinterpret_cast<uintptr_t>(b) & 31) == 0);
  const int groups = wide ? (chunks + 63) / 64 : (chunks + 31) / 32;
  const long long units = (long long)g.nb * groups * (x1 ? 2 : 1);
  const long long resident = (wide ? 4LL : 5LL) * num_sms() * 8;      // warps
  if (wide) {
    // slices per unit: the fewest (up to 8) with which the units of two
    // tensors fill the resident warps; a function of one tensor's units only,
    // so one- and two-tensor launches give identical results
    const long long one = (long long)g.nb * groups;
    int S = 1;
    while (S < 8 && one * S * 2 < resident) S *= 2;
    const long long per_cta = 8 / S;
    const long long ctas = (units + per_cta - 1) / per_cta;
    const long long rounds = (ctas + resident / 8 - 1) / (resident / 8);
    long long blocks = (ctas + rounds - 1) / rounds;
    if (blocks < 1) blocks = 1;
    summarize_wide_kernel<true, MODE><<<(int)blocks, 256, 0, s>>>(a, b, out0, out1, g, row_bytes, (int)head_off,
                                                                   chunks, d, S);
    return cudaGetLastError();
  }
  const long long per_warp = (units + resident - 1) / resident;
  const long long warps = (units + per_warp - 1) / per_warp;
  long long blocks = (warps + 7) / 8;
  if (blocks < 1) blocks = 1;
  if (dt == SPADE_BF16)
    summarize_kernel<true, MODE><<<(int)blocks, 256, 0, s>>>(a, b, out0, out1, g, row_bytes, h0 * d * esz, chunks, d);
  else
    summarize_kernel<false, MODE><<<(int)blocks, 256, 0, s>>>(a, b, out0, out1, g, row_bytes, h0 * d * esz, chunks, d);
  return cudaGetLastError();
}

cudaError_t launch_summarize(const void* x, float* out, const Geo& g, int heads_total, int h0, int hc, int d,
                             spade_dtype dt, int mode, cudaStream_t s) {
  if (mode == 1) return launch_summarize_m<1>(x, nullptr, out, nullptr, g, heads_total, h0, hc, d, dt, s);
  if (mode == 2) return launch_summarize_m<2>(x, nullptr, out, nullptr, g, heads_total, h0, hc, d, dt, s);
  return launch_summarize_m<0>(x, nullptr, out, nullptr, g, heads_total, h0, hc, d, dt, s);
}

cudaError_t launch_summarize_pair(const void* q, const void* k, float* qout, float* kout, const Geo& g,
                                  int heads_total, int h0, int hc, int d, spade_dtype dt, int mode, cudaStream_t s) {
  if (mode == 1) return launch_summarize_m<1>(q, k, qout, kout, g, heads_total, h0, hc, d, dt, s);
  if (mode == 2) return launch_summarize_m<2>(q, k, qout, kout, g, heads_total, h0, hc, d, dt, s);
  return launch_summarize_m<0>(q, k, qout, kout, g, heads_total, h0, hc, d, dt, s);
}

}  // namespace spade
