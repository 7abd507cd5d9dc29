// Step 5 on the 5th-generation tensor cores: flash block-sparse attention.
//
// SPADE technical summary (gist.science/paper/2608.03335), Methodology 3,
// "Flash Block-Sparse Attention": attention restricted to each query block's
// kept key blocks, walked in sequential (ascending) order, with an online
// softmax so that no dense score matrix exists; "Head Grouping": heads with
// different blocking schemes share one launch.  The pages' kernel targets
// Hopper (TMA + warp-group MMA); this one is written for sm_100a:
//
//  * 3D tiling by TMA: Q/K/V stay in token order [n, heads, d].  A 5-D tensor
//    map {d, head, x, y, t} with box {64, 1, bw, bh, bt} lands one block of one
//    head in shared memory as 128 rows x 128 B (slot order t, y, x), 128-byte
//    swizzled -- the layout the MMA reads.  Out-of-grid slots are zero-filled
//    by the TMA unit; the output goes back through the same map, and the TMA
//    store clips padded rows.  No tiled copy of Q/K/V is ever written.
//  * tcgen05.mma (kind::f16, bf16 in, fp32 accumulate), issued by one thread:
//    S = Q K^T (128x128, both operands in shared memory) into one of two TMEM
//    buffers; O += P V with P (bf16) read from TMEM and V from shared memory.
//  * Warp specialisation: warp 0 loads (TMA), warp 1 issues MMAs, warps 2-5
//    own one TMEM lane (query row) each: masked online softmax (exp2 domain,
//    lazy rescaling of O only when the running max grows by more than 2^8),
//    P back to TMEM, epilogue (O / l -> bf16 -> swizzled smem -> TMA store).
//  * Persistent CTAs walk a work list of (head, query block) items ranked by
//    cost, so long kept lists start first and short ones fill the tail.
//  * Every wait is bounded (globaltimer); a wait that runs out latches
//    SPADE_ERR_TIMEOUT in the device status word and the CTA winds down,
//    draining its own TMA loads and MMAs before freeing TMEM.
#include <cudaTypedefs.h>

#include "ptx.cuh"
#include "spade_internal.cuh"

namespace spade {
namespace {

constexpr int kAtomBytes = 128 * 128;   // 128 rows x 128 B: one 64-column swizzle atom of a tile

template <int D>
struct Cfg {
  static constexpr int ATOMS = D / 64;
  static constexpr int TILE = 128 * D * 2;
  // K/V ring stages; d=64 takes more so that shared memory keeps one CTA per SM
  // (each CTA allocates all 512 TMEM columns)
  static constexpr int NS = D == 128 ? 3 : 6;
  static constexpr int OFF_Q = 0;                    // 2 Q buffers
  static constexpr int OFF_KV = 2 * TILE;
  static constexpr int OFF_O = OFF_KV + NS * TILE;   // output staging
  static constexpr int OFF_BAR = OFF_O + TILE;
  static constexpr int SMEM = OFF_BAR + 256 + 1024;  // barriers + alignment slack
  static constexpr uint32_t COL_S0 = 0, COL_S1 = 128, COL_O = 256;
  static constexpr uint32_t COL_P0 = 256 + D, COL_P1 = 256 + D + 64;
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr int THREADS = 192;
};

struct __align__(64) TcParams {
  CUtensorMap tm_q[SPADE_MAX_SCHEMES];
  CUtensorMap tm_k[SPADE_MAX_SCHEMES];
  CUtensorMap tm_v[SPADE_MAX_SCHEMES];
  CUtensorMap tm_o[SPADE_MAX_SCHEMES];
  CUtensorMap tm_qt, tm_kt, tm_vt, tm_ot;   // text tokens (3-D maps), when present
  Geo geo[SPADE_MAX_SCHEMES];
  HeadInfo head[SPADE_MAX_HEADS];
  const int* cnt;
  const int* idx;
  const int* work;
  int n_items;
  int n_schemes;
  int ntb;
  int text_tokens;
  float scale_log2;
  int* status;
  long long timeout_ns;
};

// ----------------------------------------------------------- descriptors --
// Shared-memory matrix descriptor (sm_100 format): start address >> 4 in bits
// 0-13, leading byte offset >> 4 in 16-29, stride byte offset >> 4 in 32-45,
// version 1 in bits 46-47, swizzle mode in 61-63 (2 = 128-byte swizzle).
__device__ __forceinline__ uint64_t sdesc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  return (uint64_t)((saddr & 0x3FFFFu) >> 4) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
         ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}
// K-major operand (rows of 128 B, 8-row groups 1024 B apart).
__device__ __forceinline__ uint64_t kmajor_desc(uint32_t saddr) { return sdesc(saddr, 16, 1024); }
// MN-major operand (V: rows = keys (the K dim), 64-column atoms 16 KB apart).
__device__ __forceinline__ uint64_t mnmajor_desc(uint32_t saddr) { return sdesc(saddr, kAtomBytes, 1024); }

// Instruction descriptor, kind::f16: D fp32 (bit 4), A/B bf16 (bits 7, 10),
// B major-ness (bit 16), N >> 3 (bits 17-22), M >> 4 (bits 24-28).
__host__ __device__ constexpr uint32_t make_idesc(int M, int N, bool b_mn_major) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((b_mn_major ? 1u : 0u) << 16) | ((uint32_t)(N >> 3) << 17) |
         ((uint32_t)(M >> 4) << 24);
}

// ---------------------------------------------------------- bounded wait --
struct Waiter {
  volatile int* abort;
  int* status;
  long long timeout_ns;
};

__device__ __forceinline__ bool wait_bar(uint64_t* bar, uint32_t parity, const Waiter& w) {
  if (ptx::mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = ptx::globaltimer();
  for (uint32_t it = 1;; ++it) {
    if (ptx::mbar_try_wait(bar, parity)) return true;
    if ((it & 63u) == 0) {
      if (*w.abort) return false;
      if ((long long)(ptx::globaltimer() - t0) > w.timeout_ns) {
        *w.abort = 1;
        atomicExch(w.status, (int)SPADE_ERR_TIMEOUT);
        return false;
      }
    }
  }
}
// Used only while winding down: ignores the abort flag.
__device__ __forceinline__ void drain_bar(uint64_t* bar, uint32_t parity, long long limit_ns) {
  const uint64_t t0 = ptx::globaltimer();
  while (!ptx::mbar_try_wait(bar, parity)) {
    if ((long long)(ptx::globaltimer() - t0) > limit_ns) return;
  }
}

// ----------------------------------------------------------------- items --
struct Item {
  int h, qb, n, ncnt, scheme, nb;
  bool full_row;
};

__device__ __forceinline__ Item get_item(const TcParams& p, int it) {
  Item I;
  const int w = p.work[it];
  I.h = w >> 16;
  I.qb = w & 0xffff;
  const HeadInfo& hi = p.head[I.h];
  I.scheme = hi.scheme;
  I.nb = hi.nb;
  I.full_row = hi.dense || I.qb >= hi.nb;
  I.ncnt = I.full_row ? hi.nb : p.cnt[hi.cnt_off + I.qb];
  I.n = I.ncnt + p.ntb;
  return I;
}

// Key block #k of an item: its kept video blocks (ascending), then the text blocks.
__device__ __forceinline__ int key_block(const TcParams& p, const Item& I, int k) {
  if (I.full_row) return k;
  if (k < I.ncnt) return p.idx[p.head[I.h].idx_off + (long long)I.qb * I.nb + k];
  return I.nb + (k - I.ncnt);
}

template <int D>
__device__ __forceinline__ void load_tile(const TcParams& p, const CUtensorMap* vid, const CUtensorMap* txt,
                                          const Item& I, int blk, uint8_t* dst, uint64_t* bar) {
  if (blk < I.nb) {
    const Geo& g = p.geo[I.scheme];
    const int bk = blk % g.nbw, bj = (blk / g.nbw) % g.nbh, bi = blk / (g.nbw * g.nbh);
#pragma unroll
    for (int a = 0; a < Cfg<D>::ATOMS; ++a)
      ptx::tma_load_5d(dst + a * kAtomBytes, vid, bar, 64 * a, I.h, bk * g.bw, bj * g.bh, bi * g.bt);
  } else {
    const int tb = blk - I.nb;
#pragma unroll
    for (int a = 0; a < Cfg<D>::ATOMS; ++a) ptx::tma_load_3d(dst + a * kAtomBytes, txt, bar, 64 * a, I.h, tb * 128);
  }
}

// Validity of the 128 key columns of block `blk` as four 32-bit words
// (warp-cooperative: lane l decides columns l, l+32, l+64, l+96).
__device__ __forceinline__ bool key_mask(const TcParams& p, const Item& I, int blk, int lane, uint32_t (&m)[4]) {
  if (blk < I.nb) {
    const Geo& g = p.geo[I.scheme];
    int t0, y0, x0, et, eh, ew;
    block_box(g, blk, t0, y0, x0, et, eh, ew);
    if (et == g.bt && eh == g.bh && ew == g.bw) return true;
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      const int c = lane + 32 * w;
      const int xl = c % g.bw, yl = (c / g.bw) % g.bh, tl = c / (g.bw * g.bh);
      m[w] = __ballot_sync(0xffffffffu, tl < et && yl < eh && xl < ew);
    }
    return false;
  }
  const int valid = min(128, p.text_tokens - (blk - I.nb) * 128);
  if (valid >= 128) return true;
#pragma unroll
  for (int w = 0; w < 4; ++w) m[w] = __ballot_sync(0xffffffffu, lane + 32 * w < valid);
  return false;
}

template <int D>
__global__ void __launch_bounds__(Cfg<D>::THREADS, 1) attn_tc_kernel(const __grid_constant__ TcParams p) {
  using C = Cfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem + C::OFF_Q;
  uint8_t* sKV = smem + C::OFF_KV;
  uint8_t* sO = smem + C::OFF_O;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* kv_full = bars;
  uint64_t* kv_empty = bars + C::NS;
  uint64_t* q_full = bars + 2 * C::NS;
  uint64_t* q_empty = q_full + 2;
  uint64_t* s_full = q_full + 4;
  uint64_t* p_full = q_full + 6;
  uint64_t* pv_done = q_full + 8;
  uint64_t* o_free = q_full + 10;
  uint64_t* mma_fin = q_full + 11;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(q_full + 12);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < C::NS; ++s) {
      ptx::mbar_init(&kv_full[s], 1);
      ptx::mbar_init(&kv_empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      ptx::mbar_init(&q_full[b], 1);
      ptx::mbar_init(&q_empty[b], 1);
      ptx::mbar_init(&s_full[b], 1);
      ptx::mbar_init(&p_full[b], 128);
      ptx::mbar_init(&pv_done[b], 1);
    }
    ptx::mbar_init(o_free, 128);
    ptx::mbar_init(mma_fin, 1);
    *abort_flag = 0;
    ptx::fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    for (int s = 0; s < p.n_schemes; ++s) {
      ptx::prefetch_tmap(&p.tm_q[s]);
      ptx::prefetch_tmap(&p.tm_k[s]);
      ptx::prefetch_tmap(&p.tm_v[s]);
      ptx::prefetch_tmap(&p.tm_o[s]);
    }
  }
  if (warp == 1) {
    ptx::tmem_alloc(tmem_slot, C::TMEM_COLS);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const Waiter W{abort_flag, p.status, p.timeout_ns};

  if (warp == 0) {
    // ------------------------------------------------------ TMA producer --
    if (lane == 0) {
      uint32_t kvpos = 0;
      uint32_t last_par[C::NS];
      uint32_t used = 0;
      int qlast[2] = {-1, -1};
      int li = 0;
      bool ok = true;
      for (int it = blockIdx.x; ok && it < p.n_items; it += gridDim.x, ++li) {
        const Item I = get_item(p, it);
        const int qs = li & 1;
        if (!(ok = wait_bar(&q_empty[qs], ((li >> 1) & 1) ^ 1, W))) break;
        ptx::mbar_arrive_expect_tx(&q_full[qs], C::TILE);
        load_tile<D>(p, &p.tm_q[I.scheme], &p.tm_qt, I, I.qb, sQ + qs * C::TILE, &q_full[qs]);
        qlast[qs] = (li >> 1) & 1;
        auto push = [&](const CUtensorMap* vid, const CUtensorMap* txt, int blk) -> bool {
          const int st = kvpos % C::NS;
          const uint32_t par = (kvpos / C::NS) & 1;
          if (!wait_bar(&kv_empty[st], par ^ 1, W)) return false;
          ptx::mbar_arrive_expect_tx(&kv_full[st], C::TILE);
          load_tile<D>(p, vid, txt, I, blk, sKV + st * C::TILE, &kv_full[st]);
          last_par[st] = par;
          used |= 1u << st;
          ++kvpos;
          return true;
        };
        int prev = -1;
        for (int j = 0; ok && j < I.n; ++j) {
          const int kb = key_block(p, I, j);
          ok = push(&p.tm_k[I.scheme], &p.tm_kt, kb);
          if (ok && j >= 1) ok = push(&p.tm_v[I.scheme], &p.tm_vt, prev);
          prev = kb;
        }
        if (ok) ok = push(&p.tm_v[I.scheme], &p.tm_vt, prev);
      }
      if (!ok) {   // wind down: let every load this thread issued land before the CTA exits
        for (int st = 0; st < C::NS; ++st)
          if (used & (1u << st)) drain_bar(&kv_full[st], last_par[st], 100000000LL);
        for (int b = 0; b < 2; ++b)
          if (qlast[b] >= 0) drain_bar(&q_full[b], qlast[b], 100000000LL);
      }
    }
  } else if (warp == 1) {
    // -------------------------------------------------------- MMA issuer --
    if (lane == 0) {
      constexpr uint32_t idesc_qk = make_idesc(128, 128, false);
      constexpr uint32_t idesc_pv = make_idesc(128, D, true);
      uint32_t kvpos = 0, g = 0;
      int li = 0;
      bool ok = true;
      for (int it = blockIdx.x; ok && it < p.n_items; it += gridDim.x, ++li) {
        const Item I = get_item(p, it);
        const int qs = li & 1;
        if (!(ok = wait_bar(&q_full[qs], (li >> 1) & 1, W))) break;
        ptx::tc_fence_after();
        const uint32_t qaddr = ptx::smem_u32(sQ + qs * C::TILE);
        auto issue_pv = [&](int jj) -> bool {
          const uint32_t gj = g + jj, b = gj & 1;
          if (!wait_bar(&p_full[b], (gj >> 1) & 1, W)) return false;
          const int st = kvpos % C::NS;
          if (!wait_bar(&kv_full[st], (kvpos / C::NS) & 1, W)) return false;
          if (jj == 0 && !wait_bar(o_free, (li & 1) ^ 1, W)) return false;
          ptx::tc_fence_after();
          const uint32_t vaddr = ptx::smem_u32(sKV + st * C::TILE);
          const uint32_t pcol = b ? C::COL_P1 : C::COL_P0;
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            ptx::mma_ts(tmem + C::COL_O, tmem + pcol + kk * 8, mnmajor_desc(vaddr + kk * 2048), idesc_pv,
                        (jj > 0 || kk > 0) ? 1u : 0u);
          ptx::tc_commit(&pv_done[b]);
          ptx::tc_commit(&kv_empty[st]);
          ++kvpos;
          return true;
        };
        for (int j = 0; ok && j < I.n; ++j) {
          const int st = kvpos % C::NS;
          if (!(ok = wait_bar(&kv_full[st], (kvpos / C::NS) & 1, W))) break;
          ptx::tc_fence_after();
          const uint32_t b = (g + j) & 1;
          const uint32_t kaddr = ptx::smem_u32(sKV + st * C::TILE);
          const uint32_t scol = b ? C::COL_S1 : C::COL_S0;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (kk >> 2) * kAtomBytes + (kk & 3) * 32;
            ptx::mma_ss(tmem + scol, kmajor_desc(qaddr + off), kmajor_desc(kaddr + off), idesc_qk,
                        kk > 0 ? 1u : 0u);
          }
          ptx::tc_commit(&s_full[b]);
          ptx::tc_commit(&kv_empty[st]);
          ++kvpos;
          if (j == I.n - 1) ptx::tc_commit(&q_empty[qs]);
          if (j >= 1) ok = issue_pv(j - 1);
        }
        if (ok) ok = issue_pv(I.n - 1);
        g += I.n;
      }
      // every MMA this thread issued completes before TMEM is released
      ptx::tc_commit(mma_fin);
      drain_bar(mma_fin, 0, 100000000LL);
    }
  } else {
    // ---------------------------------------- softmax / correction / epilogue --
    const int quad = warp & 3;
    const int row = quad * 32 + lane;                  // TMEM lane = query slot
    const uint32_t lane_base = (uint32_t)(quad * 32) << 16;
    const bool store_thread = threadIdx.x == 64;
    const float sl2 = p.scale_log2;
    uint32_t g = 0;
    int li = 0;
    bool ok = true;
    for (int it = blockIdx.x; ok && it < p.n_items; it += gridDim.x, ++li) {
      const Item I = get_item(p, it);
      float m_use = 0.f, l = 0.f;
      for (int j = 0; j < I.n; ++j) {
        const uint32_t gj = g + j, b = gj & 1;
        ok = wait_bar(&s_full[b], (gj >> 1) & 1, W);
        if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
        ptx::tc_fence_after();
        uint32_t sr[128];
        const uint32_t tS = tmem + lane_base + (b ? C::COL_S1 : C::COL_S0);
        ptx::tmem_ld64(tS, sr);
        ptx::tmem_ld64(tS + 64, sr + 64);
        const int kb = key_block(p, I, j);
        uint32_t mw[4];
        const bool full = key_mask(p, I, kb, lane, mw);
        float mx = -INFINITY;
        if (full) {
#pragma unroll
          for (int c = 0; c < 128; ++c) mx = fmaxf(mx, __uint_as_float(sr[c]));
        } else {
#pragma unroll
          for (int c = 0; c < 128; ++c) {
            const bool v = (mw[c >> 5] >> (c & 31)) & 1u;
            const float s = v ? __uint_as_float(sr[c]) : -INFINITY;
            sr[c] = __float_as_uint(s);
            mx = fmaxf(mx, s);
          }
        }
        mx *= sl2;
        if (j == 0) {
          m_use = mx;
        } else {
          const bool need = mx > m_use + 8.0f;
          if (__any_sync(0xffffffffu, need)) {
            // rescale O by 2^(m_use - mx) once PV(j-1) has landed
            const uint32_t gp = gj - 1;
            ok = wait_bar(&pv_done[gp & 1], (gp >> 1) & 1, W);
            if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
            ptx::tc_fence_after();
            const float alpha = need ? ptx::ex2(m_use - mx) : 1.0f;
            if (need) { l *= alpha; m_use = mx; }
#pragma unroll 1
            for (int c0 = 0; c0 < D; c0 += 32) {
              uint32_t ob[32];
              ptx::tmem_ld32(tmem + lane_base + C::COL_O + c0, ob);
#pragma unroll
              for (int c = 0; c < 32; ++c) ob[c] = __float_as_uint(__uint_as_float(ob[c]) * alpha);
              ptx::tmem_st32(tmem + lane_base + C::COL_O + c0, ob);
            }
          }
        }
        const float nm = -m_use;
        float rs = 0.f;
        uint32_t pk[64];
#pragma unroll
        for (int c = 0; c < 64; ++c) {
          const float p0 = ptx::ex2(fmaf(__uint_as_float(sr[2 * c]), sl2, nm));
          const float p1 = ptx::ex2(fmaf(__uint_as_float(sr[2 * c + 1]), sl2, nm));
          rs += p0 + p1;
          pk[c] = ptx::pack_bf16x2(p0, p1);
        }
        l += rs;
        if (j >= 2) {                                  // P buffer b was read by PV(j-2)
          const uint32_t gp = gj - 2;
          ok = wait_bar(&pv_done[b], (gp >> 1) & 1, W);
          if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
        }
        const uint32_t tP = tmem + lane_base + (b ? C::COL_P1 : C::COL_P0);
        ptx::tmem_st32(tP, pk);
        ptx::tmem_st32(tP + 32, pk + 32);
        ptx::tc_fence_before();
        ptx::mbar_arrive(&p_full[b]);
      }
      if (!ok) break;
      // epilogue: O / l -> bf16 -> swizzled staging -> TMA store in token order
      const uint32_t gl = g + I.n - 1;
      ok = wait_bar(&pv_done[gl & 1], (gl >> 1) & 1, W);
      if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
      ptx::tc_fence_after();
      uint32_t ov[D];
#pragma unroll
      for (int c0 = 0; c0 < D; c0 += 64) ptx::tmem_ld64(tmem + lane_base + C::COL_O + c0, ov + c0);
      ptx::tc_fence_before();
      ptx::mbar_arrive(o_free);
      const float inv = 1.0f / l;
      if (store_thread) ptx::bulk_wait_read0();        // previous store has read the staging buffer
      ptx::named_bar_sync(1, 128);
#pragma unroll
      for (int a = 0; a < C::ATOMS; ++a) {
#pragma unroll
        for (int ch = 0; ch < 8; ++ch) {
          const int c = a * 64 + ch * 8;
          uint4 w;
          w.x = ptx::pack_bf16x2(__uint_as_float(ov[c + 0]) * inv, __uint_as_float(ov[c + 1]) * inv);
          w.y = ptx::pack_bf16x2(__uint_as_float(ov[c + 2]) * inv, __uint_as_float(ov[c + 3]) * inv);
          w.z = ptx::pack_bf16x2(__uint_as_float(ov[c + 4]) * inv, __uint_as_float(ov[c + 5]) * inv);
          w.w = ptx::pack_bf16x2(__uint_as_float(ov[c + 6]) * inv, __uint_as_float(ov[c + 7]) * inv);
          *reinterpret_cast<uint4*>(sO + a * kAtomBytes + row * 128 + ((ch ^ (row & 7)) << 4)) = w;
        }
      }
      ptx::fence_proxy_async_smem();
      ptx::named_bar_sync(1, 128);
      if (store_thread) {
        if (I.qb < I.nb) {
          const Geo& gg = p.geo[I.scheme];
          const int bk = I.qb % gg.nbw, bj = (I.qb / gg.nbw) % gg.nbh, bi = I.qb / (gg.nbw * gg.nbh);
#pragma unroll
          for (int a = 0; a < C::ATOMS; ++a)
            ptx::tma_store_5d(&p.tm_o[I.scheme], sO + a * kAtomBytes, 64 * a, I.h, bk * gg.bw, bj * gg.bh,
                              bi * gg.bt);
        } else {
#pragma unroll
          for (int a = 0; a < C::ATOMS; ++a)
            ptx::tma_store_3d(&p.tm_ot, sO + a * kAtomBytes, 64 * a, I.h, (I.qb - I.nb) * 128);
        }
        ptx::bulk_commit();
      }
      g += I.n;
    }
    if (store_thread) ptx::bulk_wait0();
  }

  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  if (warp == 1) ptx::tmem_dealloc(tmem, C::TMEM_COLS);
}

// ------------------------------------------------------------------ host --
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

bool map_video(CUtensorMap* m, const void* base, const Geo& g, int heads, int d) {
  const cuuint64_t es = 2;
  cuuint64_t dims[5] = {(cuuint64_t)d, (cuuint64_t)heads, (cuuint64_t)g.W, (cuuint64_t)g.H, (cuuint64_t)g.T};
  cuuint64_t strides[4] = {d * es, (cuuint64_t)heads * d * es, (cuuint64_t)g.W * heads * d * es,
                           (cuuint64_t)g.H * g.W * heads * d * es};
  cuuint32_t box[5] = {64, 1, (cuuint32_t)g.bw, (cuuint32_t)g.bh, (cuuint32_t)g.bt};
  cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  return encode_fn()(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void*>(base), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool map_text(CUtensorMap* m, const void* base, int text, int heads, int d) {
  const cuuint64_t es = 2;
  cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)heads, (cuuint64_t)text};
  cuuint64_t strides[2] = {d * es, (cuuint64_t)heads * d * es};
  cuuint32_t box[3] = {64, 1, 128};
  cuuint32_t estr[3] = {1, 1, 1};
  return encode_fn()(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int D>
cudaError_t launch_d(const TcParams& tp, int grid, cudaStream_t s) {
  const int smem = Cfg<D>::SMEM;
  cudaError_t e = cudaFuncSetAttribute(attn_tc_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  attn_tc_kernel<D><<<grid, Cfg<D>::THREADS, smem, s>>>(tp);
  return cudaGetLastError();
}

}  // namespace

bool attn_tc_supported(const AttnArgs& a) {
  if (a.dt != SPADE_BF16 || (a.d != 64 && a.d != 128)) return false;
  for (int s = 0; s < a.n_schemes; ++s)
    if (a.geo[s].bs != 128) return false;
  return true;
}

cudaError_t launch_attn_tc(const AttnArgs& a, cudaStream_t s, const char** why) {
  static TcParams tp;   // host staging (large); launches copy it into the parameter buffer
  if (!encode_fn()) { *why = "cuTensorMapEncodeTiled unavailable"; return cudaErrorNotSupported; }
  memset(&tp, 0, sizeof(tp));
  const int es = 2;
  for (int sc = 0; sc < a.n_schemes; ++sc) {
    const Geo& g = a.geo[sc];
    if (!map_video(&tp.tm_q[sc], a.q, g, a.heads, a.d) || !map_video(&tp.tm_k[sc], a.k, g, a.heads, a.d) ||
        !map_video(&tp.tm_v[sc], a.v, g, a.heads, a.d) || !map_video(&tp.tm_o[sc], a.out, g, a.heads, a.d)) {
      *why = "tensor map encoding failed (video)";
      return cudaErrorInvalidValue;
    }
    tp.geo[sc] = g;
  }
  if (a.text_tokens > 0) {
    const size_t off = (size_t)a.N * a.heads * a.d * es;
    const char* qb = static_cast<const char*>(a.q) + off;
    const char* kb = static_cast<const char*>(a.k) + off;
    const char* vb = static_cast<const char*>(a.v) + off;
    const char* ob = static_cast<const char*>(a.out) + off;
    if (!map_text(&tp.tm_qt, qb, a.text_tokens, a.heads, a.d) ||
        !map_text(&tp.tm_kt, kb, a.text_tokens, a.heads, a.d) ||
        !map_text(&tp.tm_vt, vb, a.text_tokens, a.heads, a.d) ||
        !map_text(&tp.tm_ot, ob, a.text_tokens, a.heads, a.d)) {
      *why = "tensor map encoding failed (text)";
      return cudaErrorInvalidValue;
    }
  }
  for (int h = 0; h < a.heads; ++h) tp.head[h] = a.head[h];
  tp.cnt = a.cnt;
  tp.idx = a.idx;
  tp.work = a.work;
  tp.n_items = a.n_items;
  tp.n_schemes = a.n_schemes;
  tp.ntb = text_blocks(a.text_tokens);
  tp.text_tokens = a.text_tokens;
  tp.scale_log2 = 1.4426950408889634f / sqrtf((float)a.d);
  tp.status = a.status;
  tp.timeout_ns = device_wait_timeout_ns();
  const int grid = a.n_items < num_sms() ? a.n_items : num_sms();
  if (grid <= 0) return cudaSuccess;
  return a.d == 128 ? launch_d<128>(tp, grid, s) : launch_d<64>(tp, grid, s);
}

// ------------------------------------------------- bounded-wait self test --
__global__ void bounded_wait_selftest_kernel(int* status, long long timeout_ns) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    ptx::mbar_init(&bar, 1);   // nothing ever arrives
    abort_flag = 0;
    ptx::fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const Waiter W{&abort_flag, status, timeout_ns};
    wait_bar(&bar, 0, W);
  }
}

cudaError_t launch_bounded_wait_selftest(int* status, long long timeout_ns, cudaStream_t s) {
  bounded_wait_selftest_kernel<<<1, 32, 0, s>>>(status, timeout_ns);
  return cudaGetLastError();
}

}  // namespace spade
