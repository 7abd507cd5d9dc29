// Step 3 on the tensor cores: the Estimator
//   prob[h,i,:] = softmax_j( qmean[h,i,:] . kmean[h,j,:] / sqrt(d) )
// (SPADE technical summary (gist.science/paper/2608.03335), Methodology 1,
// "Summarizer & Estimator Expressions": inter-block importance from the
// block summaries).
//
// The block means are fp32 and the scores decide the kept sets, so the
// contraction keeps fp32-level accuracy with error-compensated split
// precision on the TF32 tensor cores: each operand x = hi + lo with
// hi = x truncated to TF32 (low 13 mantissa bits cleared) and lo = x - hi
// (exact in fp32), and S = Qhi Khi^T + Qhi Klo^T + Qlo Khi^T (the lo lo term
// and the TF32 rounding of lo are below 2^-20 relative).
//
//  * Persistent CTAs over items (head, 128 query rows).  Per item, per
//    128-column key tile, per 32-element d chunk: TMA loads the fp32 Q and K
//    chunks (128 rows x 128 B, 128-byte swizzled: the K-major layout the MMA
//    reads); a converter warpgroup rewrites each chunk as hi in place and lo
//    beside it (the split is elementwise, so the swizzled layout carries
//    over); one thread issues the 12 tcgen05.mma (kind::tf32, M=N=128, K=8)
//    of the chunk into one of two S tiles in TMEM.
//  * An epilogue warpgroup (thread = query row) reads each finished S tile
//    with tcgen05.ld, scales it, keeps a running row max and sum (online
//    softmax over the key tiles), stages the scores in the output row, and
//    after the last tile rewrites its row as probabilities.
//  * Every wait is bounded (globaltimer); a timeout latches SPADE_ERR_TIMEOUT
//    in the device status word and the CTA winds down.
#include <cudaTypedefs.h>

#include "ptx.cuh"
#include "spade_internal.cuh"

namespace spade {
namespace {

constexpr int kStages = 3;
constexpr int kChunk = 128 * 128;           // 128 rows x 128 B (32 fp32 of d)
constexpr int kStageBytes = 4 * kChunk;     // Q hi, Q lo, K hi, K lo
constexpr int kThreads = 384;               // producer, MMA, 2 idle, converters (4 warps), epilogue (4 warps)
constexpr int kSmem = kStages * kStageBytes + 256 + 1024;

struct __align__(64) EstTcParams {
  CUtensorMap tm_q, tm_k;   // [heads][nb][d] fp32: dims {d, nb, heads}, box {32, 128, 1}
  float* prob;              // [heads][nb][nb]
  int nb, d, nrt, n_items;
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
constexpr uint32_t kIdesc = (1u << 4) | (2u << 7) | (2u << 10) | ((128u >> 3) << 17) | ((128u >> 4) << 24);

__global__ void __launch_bounds__(kThreads, 1) estimate_tc_kernel(const __grid_constant__ EstTcParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kStages * kStageBytes);
  uint64_t* full = bars;                   // [kStages] TMA landed
  uint64_t* conv = bars + kStages;         // [kStages] split into hi / lo (128 threads)
  uint64_t* empty = bars + 2 * kStages;    // [kStages] MMAs done with the stage
  uint64_t* s_full = bars + 3 * kStages;   // [2] S tile complete
  uint64_t* s_free = s_full + 2;           // [2] S tile read (128 threads)
  uint64_t* fin = s_full + 4;
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
      ptx::mbar_init(&s_free[b], 128);
    }
    ptx::mbar_init(fin, 1);
    *abort_flag = 0;
    ptx::fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    ptx::prefetch_tmap(&p.tm_q);
    ptx::prefetch_tmap(&p.tm_k);
  }
  if (warp == 1) {
    ptx::tmem_alloc(tmem_slot, 256);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const EWaiter W{abort_flag, p.status, p.timeout_ns};
  const int nct = p.nrt;          // key tiles = query tiles (both cover nb in 128s)
  const int ndc = p.d / 32;

  if (warp == 0) {
    // ------------------------------------------------------ TMA producer --
    uint32_t g = 0;
    bool ok = true;
    for (int it = blockIdx.x; ok && it < p.n_items; it += gridDim.x) {
      const int h = it / p.nrt, rt = it - h * p.nrt;
      for (int ct = 0; ok && ct < nct; ++ct)
        for (int dc = 0; ok && dc < ndc; ++dc, ++g) {
          const int s = (int)(g % kStages);
          ok = __all_sync(0xffffffffu, ewait(&empty[s], ((g / kStages) & 1) ^ 1, W));
          if (!ok) break;
          uint8_t* st = smem + s * kStageBytes;
          ptx::mbar_arrive_expect_tx_elect(&full[s], 2 * kChunk);
          ptx::tma_load_3d_elect(st, &p.tm_q, &full[s], 32 * dc, 128 * rt, h);
          ptx::tma_load_3d_elect(st + 2 * kChunk, &p.tm_k, &full[s], 32 * dc, 128 * ct, h);
        }
    }
    if (lane == 0 && !ok && g > 0) {   // wind down: let the loads issued land
      for (uint32_t k = (g > (uint32_t)kStages ? g - kStages : 0); k < g; ++k)
        edrain(&full[k % kStages], (k / kStages) & 1, 100000000LL);
    }
  } else if (warp == 1) {
    // --------------------------------------------------------- MMA issuer --
    uint32_t g = 0, gct = 0;
    bool ok = true;
    for (int it = blockIdx.x; ok && it < p.n_items; it += gridDim.x) {
      for (int ct = 0; ok && ct < nct; ++ct, ++gct) {
        const int b = (int)(gct & 1);
        ok = __all_sync(0xffffffffu, ewait(&s_free[b], ((gct >> 1) & 1) ^ 1, W));
        if (!ok) break;
        const uint32_t ts = tmem + 128 * b;
        for (int dc = 0; ok && dc < ndc; ++dc, ++g) {
          const int s = (int)(g % kStages);
          ok = __all_sync(0xffffffffu, ewait(&conv[s], (g / kStages) & 1, W));
          if (!ok) break;
          ptx::tc_fence_after();
          const uint32_t base = ptx::smem_u32(smem + s * kStageBytes);
          const uint64_t qhi = kdesc(base), qlo = kdesc(base + kChunk);
          const uint64_t khi = kdesc(base + 2 * kChunk), klo = kdesc(base + 3 * kChunk);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {           // 8 fp32 (32 B) of d per MMA
            const uint64_t off = (uint64_t)((kk * 32) >> 4);
            ptx::mma_ss_tf32_elect(ts, qhi + off, khi + off, kIdesc, (dc > 0 || kk > 0) ? 1u : 0u);
            ptx::mma_ss_tf32_elect(ts, qhi + off, klo + off, kIdesc, 1u);
            ptx::mma_ss_tf32_elect(ts, qlo + off, khi + off, kIdesc, 1u);
          }
          ptx::tc_commit_elect(&empty[s]);
        }
        if (ok) ptx::tc_commit_elect(&s_full[b]);
      }
    }
    ptx::tc_commit_elect(fin);
    edrain(fin, 0, 100000000LL);
  } else if (warp >= 4 && warp < 8) {
    // ------------------------------------------------- hi / lo converters --
    const int ctid = threadIdx.x - 128;
    uint32_t g = 0;
    bool ok = true;
    for (int it = blockIdx.x; ok && it < p.n_items; it += gridDim.x)
      for (int ct = 0; ok && ct < nct; ++ct)
        for (int dc = 0; ok && dc < ndc; ++dc, ++g) {
          const int s = (int)(g % kStages);
          ok = ewait(&full[s], (g / kStages) & 1, W);
          if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
          uint8_t* st = smem + s * kStageBytes;
#pragma unroll 4
          for (int i = ctid; i < 2 * (kChunk / 16); i += 128) {
            const int region = i / (kChunk / 16);          // 0: Q, 1: K
            uint4* hi = reinterpret_cast<uint4*>(st + region * 2 * kChunk) + (i % (kChunk / 16));
            uint4* lo = reinterpret_cast<uint4*>(reinterpret_cast<uint8_t*>(hi) + kChunk);
            const uint4 v = *hi;
            const uint4 h4 = make_uint4(v.x & 0xFFFFE000u, v.y & 0xFFFFE000u, v.z & 0xFFFFE000u, v.w & 0xFFFFE000u);
            const uint4 l4 = make_uint4(__float_as_uint(__uint_as_float(v.x) - __uint_as_float(h4.x)),
                                        __float_as_uint(__uint_as_float(v.y) - __uint_as_float(h4.y)),
                                        __float_as_uint(__uint_as_float(v.z) - __uint_as_float(h4.z)),
                                        __float_as_uint(__uint_as_float(v.w) - __uint_as_float(h4.w)));
            *hi = h4;
            *lo = l4;
          }
          ptx::fence_proxy_async_smem();                   // generic writes -> tensor-core reads
          ptx::mbar_arrive(&conv[s]);
        }
  } else if (warp >= 8) {
    // ---------------------------------------------------------- epilogue --
    const int quad = warp & 3;
    const int row = quad * 32 + lane;
    const uint32_t lane_base = (uint32_t)(quad * 32) << 16;
    const bool vec = (p.nb & 3) == 0;
    uint32_t gct = 0;
    bool ok = true;
    for (int it = blockIdx.x; ok && it < p.n_items; it += gridDim.x) {
      const int h = it / p.nrt, rt = it - h * p.nrt;
      const int i = 128 * rt + row;
      float* prow = p.prob + ((long long)h * p.nb + (i < p.nb ? i : 0)) * p.nb;
      float m = -INFINITY, l = 0.f;
      for (int ct = 0; ct < nct; ++ct, ++gct) {
        const int b = (int)(gct & 1);
        ok = ewait(&s_full[b], (gct >> 1) & 1, W);
        if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
        ptx::tc_fence_after();
        const int j0 = 128 * ct;
        const int nv = p.nb - j0 < 128 ? p.nb - j0 : 128;   // valid key columns in this tile
        // four 32-column pieces: scale, mask, fold into the running max / sum
        // (online softmax), stage the scores in the output row
#pragma unroll 1
        for (int c0 = 0; c0 < 128; c0 += 32) {
          uint32_t sr[32];
          ptx::tmem_ld32(tmem + lane_base + 128 * b + c0, sr);
          float cm = -INFINITY;
#pragma unroll
          for (int c = 0; c < 32; ++c) {
            const float v = c0 + c < nv ? __uint_as_float(sr[c]) * p.scale : -INFINITY;
            sr[c] = __float_as_uint(v);
            cm = fmaxf(cm, v);
          }
          if (cm > -INFINITY) {
            const float mn = fmaxf(m, cm);
            float cs = 0.f;
#pragma unroll
            for (int c = 0; c < 32; ++c) cs += expf(__uint_as_float(sr[c]) - mn);
            l = l * expf(m - mn) + cs;
            m = mn;
          }
          if (i < p.nb) {
            if (vec) {
              float4* dst = reinterpret_cast<float4*>(prow + j0 + c0);
#pragma unroll
              for (int c4 = 0; c4 < 8; ++c4)
                if (c0 + 4 * c4 < nv)
                  dst[c4] = make_float4(__uint_as_float(sr[4 * c4]), __uint_as_float(sr[4 * c4 + 1]),
                                        __uint_as_float(sr[4 * c4 + 2]), __uint_as_float(sr[4 * c4 + 3]));
            } else {
#pragma unroll
              for (int c = 0; c < 32; ++c)
                if (c0 + c < nv) prow[j0 + c0 + c] = __uint_as_float(sr[c]);
            }
          }
        }
        ptx::tc_fence_before();
        ptx::mbar_arrive(&s_free[b]);
      }
      if (!ok) break;
      if (i < p.nb) {
        // probabilities: the thread rewrites its own staged row
        const float inv = 1.0f / l;
        if (vec) {
          float4* r4 = reinterpret_cast<float4*>(prow);
          for (int c0 = 0; c0 < p.nb / 4; c0 += 16) {     // sixteen 16-byte loads in flight
            float4 v[16];
#pragma unroll
            for (int u = 0; u < 16; ++u)
              if (c0 + u < p.nb / 4) v[u] = r4[c0 + u];
#pragma unroll
            for (int u = 0; u < 16; ++u)
              if (c0 + u < p.nb / 4)
                r4[c0 + u] = make_float4(expf(v[u].x - m) * inv, expf(v[u].y - m) * inv, expf(v[u].z - m) * inv,
                                         expf(v[u].w - m) * inv);
          }
        } else {
          for (int c = 0; c < p.nb; ++c) prow[c] = expf(prow[c] - m) * inv;
        }
      }
    }
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  if (warp == 1) ptx::tmem_dealloc(tmem, 256);
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  }
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

}  // namespace

cudaError_t launch_estimate_tc(const float* qm, const float* km, float* prob, int heads, int nb, int d, int* status,
                               cudaStream_t s) {
  if (!encode_fn()) return cudaErrorNotSupported;
  if (d % 32 != 0 || (reinterpret_cast<uintptr_t>(qm) & 15) || (reinterpret_cast<uintptr_t>(km) & 15))
    return cudaErrorInvalidValue;
  static EstTcParams tp;
  memset(&tp, 0, sizeof(tp));
  if (!map_means(&tp.tm_q, qm, heads, nb, d) || !map_means(&tp.tm_k, km, heads, nb, d)) return cudaErrorInvalidValue;
  tp.prob = prob;
  tp.nb = nb;
  tp.d = d;
  tp.nrt = (nb + 127) / 128;
  tp.n_items = heads * tp.nrt;
  tp.scale = 1.0f / sqrtf((float)d);
  tp.status = status;
  tp.timeout_ns = device_wait_timeout_ns();
  static_assert(kSmem <= 232448, "shared memory budget");
  cudaError_t e = cudaFuncSetAttribute(estimate_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
  if (e != cudaSuccess) return e;
  const int grid = tp.n_items < num_sms() ? tp.n_items : num_sms();
  if (grid <= 0) return cudaSuccess;
  estimate_tc_kernel<<<grid, kThreads, kSmem, s>>>(tp);
  return cudaGetLastError();
}

}  // namespace spade
