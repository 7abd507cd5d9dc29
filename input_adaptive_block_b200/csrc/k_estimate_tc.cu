// Step 3 on the tensor cores: the Estimator's pooled scores
//   score[h,i,j] = qmean[h,i,:] . kmean[h,j,:] / sqrt(d)
// and, for the standalone estimator, their softmax over j
// (SPADE technical summary (gist.science/paper/2608.03335), Methodology 1,
// "Summarizer & Estimator Expressions": inter-block importance from the
// block summaries).  On the grouped path the softmax is formed by the index
// search as it reads each row (k_select.cu), so only the scores are written.
//
// The block means are fp32 and the scores decide the kept sets, so the
// contraction keeps fp32-level accuracy with error-compensated split
// precision on the TF32 tensor cores: each operand x = hi + lo with
// hi = x truncated to TF32 (low 13 mantissa bits cleared) and lo = x - hi
// (exact in fp32), and S = Qhi Khi^T + Qhi Klo^T + Qlo Khi^T (the lo lo term
// and the TF32 rounding of lo are below 2^-20 relative).
//
//  * Persistent CTAs, each over a contiguous range of items (head, 128 query
//    rows, 128 key columns), so the query tile changes only a few times per
//    CTA.  The query tile lives in TMEM: its fp32 chunks come through the
//    stage ring ahead of time (TMA), and once the previous tile's MMAs are
//    done a converter warpgroup (thread = query row) splits them and writes
//    Qhi and Qlo with tcgen05.st; the MMAs read them as the A operand, so
//    only key chunks pass through shared memory as operands.  Per item and
//    32-element d chunk:
//    TMA loads the fp32 K chunk (128 rows x 128 B, 128-byte swizzled: the
//    K-major layout the MMA reads) into one of six stages; the converter
//    rewrites it as hi in place and lo beside it (elementwise, so the
//    swizzled layout carries over); one thread issues the 12 tcgen05.mma
//    (kind::tf32, M=128, K=8, N = the item's valid key columns rounded up to
//    16) into one of two S tiles in TMEM.
//  * Two epilogue warpgroups (64 columns each; thread = query row) read a
//    finished tile with tcgen05.ld, release it, scale it, transpose 8x8
//    blocks of 16-byte chunks across each 8-lane group with shuffles, and
//    store whole 128-byte row segments, four rows per store instruction
//    (a row per thread would touch 32 lines per instruction; a shared-memory
//    stage would compete with the MMA operands for shared-memory bandwidth).
//  * Every wait is bounded (globaltimer); a timeout latches SPADE_ERR_TIMEOUT
//    in the device status word and the CTA winds down.
#include <cudaTypedefs.h>

#include "ptx.cuh"
#include "spade_internal.cuh"

namespace spade {
namespace {

constexpr int kStages = 6;
constexpr int kChunk = 128 * 128;           // 128 rows x 128 B (32 fp32 of d)
constexpr int kStageBytes = 2 * kChunk;     // K hi (written over the landed chunk), K lo
constexpr int kThreads = 512;               // producer, MMA, 2 idle, converters (4 warps), 2 x epilogue (4 warps)
constexpr int kSmem = kStages * kStageBytes + 256 + 1024;
// TMEM columns: S tiles [0, 256), Qhi [256, 256 + d), Qlo [384, 384 + d)
constexpr uint32_t kColQhi = 256, kColQlo = 384;

struct __align__(64) EstTcParams {
  CUtensorMap tm_q;         // [heads][nb][d] fp32: dims {d, nb, heads}, box {32, 128, 1}
  CUtensorMap tm_k;         // same for the key means
  float* out;               // [heads][nb][nb] scores
  int nb, d, nt, n_items;
  float scale;
  int* status;
  long long timeout_ns;
};

struct EWaiter {
  volatile int* abort;
  int* status;
  long long timeout_ns;
};

__device__ __forceinline__ bool ewait(uint64_t* bar, uint32_t parity, const EWaiter& w) {
  if (ptx::mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = ptx::globaltimer();
  for (;;) {
    if (ptx::mbar_try_wait_sleep(bar, parity, 200000u)) return true;
    if (*w.abort) return false;
    if ((long long)(ptx::globaltimer() - t0) > w.timeout_ns) {
      *w.abort = 1;
      atomicExch(w.status, (int)SPADE_ERR_TIMEOUT);
      return false;
    }
  }
}
__device__ __forceinline__ void edrain(uint64_t* bar, uint32_t parity, long long limit_ns) {
  const uint64_t t0 = ptx::globaltimer();
  while (!ptx::mbar_try_wait(bar, parity)) {
    if ((long long)(ptx::globaltimer() - t0) > limit_ns) return;
  }
}

// K-major operand, 128-byte swizzle: rows of 128 B, 8-row groups 1024 B apart.
__device__ __forceinline__ uint64_t kdesc(uint32_t saddr) {
  return (uint64_t)((saddr & 0x3FFFFu) >> 4) | ((uint64_t)1 << 16) | ((uint64_t)(1024 >> 4) << 32) |
         ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}
// kind::tf32: D fp32 (bit 4), A and B TF32 (format 2 in bits 7 and 10), K-major, N >> 3, M >> 4.
__device__ __forceinline__ uint32_t idesc_tf32(uint32_t n) {
  return (1u << 4) | (2u << 7) | (2u << 10) | ((n >> 3) << 17) | ((128u >> 4) << 24);
}

__device__ __forceinline__ uint32_t tf32_hi(uint32_t x) { return x & 0xFFFFE000u; }
__device__ __forceinline__ uint32_t tf32_lo(uint32_t x) {
  return __float_as_uint(__uint_as_float(x) - __uint_as_float(tf32_hi(x)));
}

__device__ __forceinline__ float4 shfl_xor4(float4 v, int m) {
  return make_float4(__shfl_xor_sync(0xffffffffu, v.x, m), __shfl_xor_sync(0xffffffffu, v.y, m),
                     __shfl_xor_sync(0xffffffffu, v.z, m), __shfl_xor_sync(0xffffffffu, v.w, m));
}
// 8x8 transpose of 16-byte elements across each 8-lane group: on entry lane
// 8G + r holds e[k] = element (r, k); on exit lane 8G + k holds e[r] = (r, k).
__device__ __forceinline__ void transpose8(float4 (&e)[8], int lane) {
#pragma unroll
  for (int s = 4; s >= 1; s >>= 1) {
    const bool upper = (lane & s) != 0;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      if (j & s) continue;
      const float4 send = upper ? e[j] : e[j | s];
      const float4 recv = shfl_xor4(send, s);
      if (upper) e[j] = recv; else e[j | s] = recv;
    }
  }
}



// VEC: nb % 4 == 0 (16-byte aligned score rows): transposed whole-line
// stores; otherwise each thread stores its own row.
template <bool VEC>
__global__ void __launch_bounds__(kThreads, 1) estimate_tc_kernel(const __grid_constant__ EstTcParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kStages * kStageBytes);
  uint64_t* full = bars;                   // [kStages] TMA landed
  uint64_t* conv = bars + kStages;         // [kStages] split into hi / lo (128 threads)
  uint64_t* empty = bars + 2 * kStages;    // [kStages] MMAs done with the stage
  uint64_t* s_full = bars + 3 * kStages;   // [2] S tile complete
  uint64_t* s_free = s_full + 2;           // [2] S tile read (256 epilogue threads)
  uint64_t* q_full = s_full + 4;           // query tile in TMEM (128 threads)
  uint64_t* q_free = s_full + 5;           // MMAs of the previous query tile done
  uint64_t* fin = s_full + 6;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(fin + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      ptx::mbar_init(&full[s], 1);
      ptx::mbar_init(&conv[s], 128);
      ptx::mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      ptx::mbar_init(&s_full[b], 1);
      ptx::mbar_init(&s_free[b], 256);
    }
    ptx::mbar_init(q_full, 128);
    ptx::mbar_init(q_free, 1);
    ptx::mbar_init(fin, 1);
    *abort_flag = 0;
    ptx::fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    ptx::prefetch_tmap(&p.tm_q);
    ptx::prefetch_tmap(&p.tm_k);
  }
  if (warp == 1) {
    ptx::tmem_alloc(tmem_slot, 512);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const EWaiter W{abort_flag, p.status, p.timeout_ns};
  const int nt = p.nt;            // key tiles = query tiles (both cover nb in 128s)
  const int ndc = p.d / 32;
  // this CTA's items: a contiguous range of the (head, query tile, key tile) order
  const int it0 = (int)((long long)blockIdx.x * p.n_items / gridDim.x);
  const int it1 = (int)((long long)(blockIdx.x + 1) * p.n_items / gridDim.x);

  if (warp == 0) {
    // ------------------------------------------------------ TMA producer --
    uint32_t g = 0;
    bool ok = true;
    for (int it = it0; ok && it < it1; ++it) {
      const int h = it / (nt * nt), rt = (it / nt) % nt, ct = it % nt;
      // a new query tile: its d chunks go through the ring first (read into
      // TMEM by the converter), then the item's key chunks
      const bool qt = it == it0 || ct == 0;
      for (int k = qt ? 0 : ndc; ok && k < 2 * ndc; ++k, ++g) {
        const int s = (int)(g % kStages);
        ok = __all_sync(0xffffffffu, ewait(&empty[s], ((g / kStages) & 1) ^ 1, W));
        if (!ok) break;
        ptx::mbar_arrive_expect_tx_elect(&full[s], kChunk);
        if (k < ndc) ptx::tma_load_3d_elect(smem + s * kStageBytes, &p.tm_q, &full[s], 32 * k, 128 * rt, h);
        else ptx::tma_load_3d_elect(smem + s * kStageBytes, &p.tm_k, &full[s], 32 * (k - ndc), 128 * ct, h);
      }
    }
    if (lane == 0 && !ok && g > 0) {   // wind down: let the loads issued land
      for (uint32_t k = (g > (uint32_t)kStages ? g - kStages : 0); k < g; ++k)
        edrain(&full[k % kStages], (k / kStages) & 1, 100000000LL);
    }
  } else if (warp == 1) {
    // --------------------------------------------------------- MMA issuer --
    uint32_t g = 0, gi = 0, gq = 0;
    bool ok = true;
    for (int it = it0; ok && it < it1; ++it, ++gi) {
      if (it == it0 || it % nt == 0) {                 // a new query tile
        if (gq > 0) ptx::tc_commit_elect(q_free);      // fires once the previous tile's MMAs are done
        // its chunks' stages: read into TMEM by the converter, then released here
        for (int dc = 0; ok && dc < ndc; ++dc, ++g) {
          const int s = (int)(g % kStages);
          ok = __all_sync(0xffffffffu, ewait(&conv[s], (g / kStages) & 1, W));
          if (!ok) break;
          if (lane == 0) ptx::mbar_arrive(&empty[s]);
        }
        if (!ok) break;
        ok = __all_sync(0xffffffffu, ewait(q_full, gq & 1, W));
        if (!ok) break;
        ptx::tc_fence_after();
        ++gq;
      }
      const int ct = it % nt;
      const int nv = p.nb - 128 * ct < 128 ? p.nb - 128 * ct : 128;   // valid key columns
      const uint32_t idesc = idesc_tf32((uint32_t)((nv + 15) & ~15));
      const int b = (int)(gi & 1);
      ok = __all_sync(0xffffffffu, ewait(&s_free[b], ((gi >> 1) & 1) ^ 1, W));
      if (!ok) break;
      ptx::tc_fence_after();
      const uint32_t ts = tmem + 128 * b;
      for (int dc = 0; ok && dc < ndc; ++dc, ++g) {
        const int s = (int)(g % kStages);
        ok = __all_sync(0xffffffffu, ewait(&conv[s], (g / kStages) & 1, W));
        if (!ok) break;
        ptx::tc_fence_after();
        const uint32_t base = ptx::smem_u32(smem + s * kStageBytes);
        const uint64_t khi = kdesc(base), klo = kdesc(base + kChunk);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {           // 8 fp32 (32 B) of d per MMA
          const uint64_t off = (uint64_t)((kk * 32) >> 4);
          const uint32_t ac = (uint32_t)(32 * dc + 8 * kk);
          ptx::mma_ts_tf32_elect(ts, tmem + kColQhi + ac, khi + off, idesc, (dc > 0 || kk > 0) ? 1u : 0u);
          ptx::mma_ts_tf32_elect(ts, tmem + kColQhi + ac, klo + off, idesc, 1u);
          ptx::mma_ts_tf32_elect(ts, tmem + kColQlo + ac, khi + off, idesc, 1u);
        }
        ptx::tc_commit_elect(&empty[s]);
      }
      if (ok) ptx::tc_commit_elect(&s_full[b]);
    }
    ptx::tc_commit_elect(fin);
    edrain(fin, 0, 100000000LL);
  } else if (warp >= 4 && warp < 8) {
    // -------------------------- query tile into TMEM, K chunks into hi / lo --
    const int ctid = threadIdx.x - 128;
    const int quad = warp & 3;
    uint32_t g = 0, gq = 0;
    bool ok = true;
    for (int it = it0; ok && it < it1; ++it) {
      if (it == it0 || it % nt == 0) {
        // the new query tile's chunks have been loaded into the ring ahead of
        // time; once the previous tile's MMAs are done, thread = query row
        // reads its row of each chunk (128-byte swizzled: 16-byte chunk c at
        // position c ^ (row & 7)), splits it and writes Qhi / Qlo to TMEM
        if (gq > 0) {
          ok = ewait(q_free, (gq - 1) & 1, W);         // the previous tile's MMAs have read it
          if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
          ptx::tc_fence_after();
        }
        const uint32_t lane_base = (uint32_t)(quad * 32) << 16;
        for (int dc = 0; ok && dc < ndc; ++dc, ++g) {
          const int s = (int)(g % kStages);
          ok = ewait(&full[s], (g / kStages) & 1, W);
          if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
          const uint8_t* rowp = smem + s * kStageBytes + ctid * 128;
          uint4 v[8];
#pragma unroll
          for (int c = 0; c < 8; ++c) v[c] = *reinterpret_cast<const uint4*>(rowp + ((c ^ (ctid & 7)) << 4));
          uint32_t r[32];
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            r[4 * c] = tf32_hi(v[c].x); r[4 * c + 1] = tf32_hi(v[c].y);
            r[4 * c + 2] = tf32_hi(v[c].z); r[4 * c + 3] = tf32_hi(v[c].w);
          }
          ptx::tmem_st32(tmem + lane_base + kColQhi + 32 * dc, r);
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            r[4 * c] = tf32_lo(v[c].x); r[4 * c + 1] = tf32_lo(v[c].y);
            r[4 * c + 2] = tf32_lo(v[c].z); r[4 * c + 3] = tf32_lo(v[c].w);
          }
          ptx::tmem_st32(tmem + lane_base + kColQlo + 32 * dc, r);
          ptx::mbar_arrive(&conv[s]);                  // stage read: the MMA warp releases it
        }
        if (!ok) break;
        ptx::tc_fence_before();
        ptx::mbar_arrive(q_full);
        ++gq;
      }
      for (int dc = 0; ok && dc < ndc; ++dc, ++g) {
        const int s = (int)(g % kStages);
        ok = ewait(&full[s], (g / kStages) & 1, W);
        if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
        uint4* hi4 = reinterpret_cast<uint4*>(smem + s * kStageBytes);
        uint4* lo4 = reinterpret_cast<uint4*>(smem + s * kStageBytes + kChunk);
#pragma unroll 4
        for (int q = ctid; q < kChunk / 16; q += 128) {
          const uint4 v = hi4[q];
          hi4[q] = make_uint4(tf32_hi(v.x), tf32_hi(v.y), tf32_hi(v.z), tf32_hi(v.w));
          lo4[q] = make_uint4(tf32_lo(v.x), tf32_lo(v.y), tf32_lo(v.z), tf32_lo(v.w));
        }
        ptx::fence_proxy_async_smem();                 // generic writes -> tensor-core reads
        ptx::mbar_arrive(&conv[s]);
      }
    }
  } else if (warp >= 8) {
    // --------------------------------------------------------- epilogues --
    const int half = (warp - 8) >> 2;            // key columns 64*half .. 64*half + 63 of the tile
    const int quad = warp & 3;
    const uint32_t lane_base = (uint32_t)(quad * 32) << 16;
    uint32_t gi = 0;
    bool ok = true;
    for (int it = it0; ok && it < it1; ++it, ++gi) {
      const int h = it / (nt * nt), rt = (it / nt) % nt, ct = it % nt;
      const int b = (int)(gi & 1);
      ok = ewait(&s_full[b], (gi >> 1) & 1, W);
      if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
      ptx::tc_fence_after();
      const int j0 = 128 * ct + 64 * half;
      const int nv = p.nb - j0 < 64 ? p.nb - j0 : 64;   // valid columns of this half (warp-uniform)
      uint32_t sr[64];
      if (nv > 0) ptx::tmem_ld64(tmem + lane_base + 128 * b + 64 * half, sr);
      ptx::tc_fence_before();
      ptx::mbar_arrive(&s_free[b]);                // the tile may be overwritten now
      if (nv <= 0) continue;
      const int row0 = 128 * rt + 32 * quad;       // this warp's first query row
      float* base = p.out + (long long)h * p.nb * p.nb;
      if (VEC) {
        const int grp = lane >> 3, k = lane & 7;
#pragma unroll
        for (int blk = 0; blk < 2; ++blk) {
          float4 e[8];
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            const uint32_t* v = sr + 32 * blk + 4 * c;
            e[c] = make_float4(__uint_as_float(v[0]) * p.scale, __uint_as_float(v[1]) * p.scale,
                               __uint_as_float(v[2]) * p.scale, __uint_as_float(v[3]) * p.scale);
          }
          transpose8(e, lane);                     // lane 8G + k: chunk k of rows 8G .. 8G + 7
          const int col = j0 + 32 * blk + 4 * k;
          if (col < p.nb) {
#pragma unroll
            for (int r = 0; r < 8; ++r) {
              const int i = row0 + 8 * grp + r;
              if (i < p.nb) *reinterpret_cast<float4*>(base + (long long)i * p.nb + col) = e[r];
            }
          }
        }
      } else {
        const int i = row0 + lane;
        if (i < p.nb) {
          float* dst = base + (long long)i * p.nb + j0;
#pragma unroll
          for (int c = 0; c < 64; ++c)
            if (c < nv) dst[c] = __uint_as_float(sr[c]) * p.scale;
        }
      }
    }
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  if (warp == 1) ptx::tmem_dealloc(tmem, 512);
}

// The driver's tensor-map encoder, looked up once (initialisation of a
// function-local static is thread-safe); null without a driver.
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static const PFN_cuTensorMapEncodeTiled_v12000 fn = [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    return static_cast<PFN_cuTensorMapEncodeTiled_v12000>(nullptr);
  }();
  return fn;
}

bool map_means(CUtensorMap* m, const float* base, int heads, int nb, int d) {
  cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)nb, (cuuint64_t)heads};
  cuuint64_t strides[2] = {(cuuint64_t)d * 4, (cuuint64_t)nb * d * 4};
  cuuint32_t box[3] = {32, 128, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return encode_fn()(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<float*>(base), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Row softmax in place, one warp per row (the standalone estimator's
// probabilities from its scores): p_j = exp(s_j - max) / sum.
template <int NPL>
__global__ void __launch_bounds__(256) softmax_rows_kernel(float* __restrict__ s, long long rows, int nb) {
  const int lane = threadIdx.x & 31;
  const long long row = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
  if (row >= rows) return;
  float* r = s + row * nb;
  float v[NPL];
  float mx = -INFINITY;
#pragma unroll
  for (int e = 0; e < NPL; ++e) {
    const int j = lane + 32 * e;
    v[e] = j < nb ? r[j] : -INFINITY;
    mx = fmaxf(mx, v[e]);
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  float l = 0.f;
#pragma unroll
  for (int e = 0; e < NPL; ++e) {
    v[e] = lane + 32 * e < nb ? expf(v[e] - mx) : 0.f;
    l += v[e];
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) l += __shfl_xor_sync(0xffffffffu, l, o);
  const float inv = 1.0f / l;
#pragma unroll
  for (int e = 0; e < NPL; ++e)
    if (lane + 32 * e < nb) r[lane + 32 * e] = v[e] * inv;
}

template <int NPL>
cudaError_t launch_softmax_rows(float* s, long long rows, int nb, cudaStream_t st) {
  const long long blocks = (rows + 7) / 8;
  softmax_rows_kernel<NPL><<<(unsigned)blocks, 256, 0, st>>>(s, rows, nb);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_estimate_tc(const float* qm, const float* km, float* out, int heads, int nb, int d, int* status,
                               bool probs, cudaStream_t s) {
  if (!encode_fn()) return cudaErrorNotSupported;
  if (d % 32 != 0 || d > 128 || (reinterpret_cast<uintptr_t>(qm) & 15) || (reinterpret_cast<uintptr_t>(km) & 15))
    return cudaErrorInvalidValue;
  thread_local EstTcParams tp;   // per calling thread; the launch copies it
  memset(&tp, 0, sizeof(tp));
  if (!map_means(&tp.tm_q, qm, heads, nb, d) || !map_means(&tp.tm_k, km, heads, nb, d)) return cudaErrorInvalidValue;
  tp.out = out;
  tp.nb = nb;
  tp.d = d;
  tp.nt = (nb + 127) / 128;
  tp.n_items = heads * tp.nt * tp.nt;
  tp.scale = 1.0f / sqrtf((float)d);
  tp.status = status;
  tp.timeout_ns = device_wait_timeout_ns();
  static_assert(kSmem <= 232448, "shared memory budget");
  const bool vec = nb % 4 == 0 && (reinterpret_cast<uintptr_t>(out) & 15) == 0;
  cudaError_t e = cudaFuncSetAttribute(vec ? estimate_tc_kernel<true> : estimate_tc_kernel<false>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
  if (e != cudaSuccess) return e;
  const int grid = tp.n_items < num_sms() ? tp.n_items : num_sms();
  if (grid <= 0) return cudaSuccess;
  if (vec) estimate_tc_kernel<true><<<grid, kThreads, kSmem, s>>>(tp);
  else estimate_tc_kernel<false><<<grid, kThreads, kSmem, s>>>(tp);
  e = cudaGetLastError();
  if (e != cudaSuccess || !probs) return e;
  const long long rows = (long long)heads * nb;
  if (nb <= 256) return launch_softmax_rows<8>(out, rows, nb, s);
  if (nb <= 512) return launch_softmax_rows<16>(out, rows, nb, s);
  if (nb <= 1024) return launch_softmax_rows<32>(out, rows, nb, s);
  return launch_softmax_rows<64>(out, rows, nb, s);
}

}  // namespace spade
