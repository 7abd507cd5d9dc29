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
//  * Warp specialisation: warp 0 loads (TMA) and hands out work, warp 1 issues
//    MMAs, warps 2-5 own one TMEM lane (query row) each: masked online
//    softmax (exp2 domain, lazy rescaling of O only when the running max grows
//    by more than 2^8), P back to TMEM, epilogue (O / l -> bf16 -> swizzled
//    smem -> TMA store).  A quarter of the exponentials of full blocks run on
//    the FMA pipe (polynomial, below) so the SFU does not bound the softmax.
//  * Persistent CTAs take (head, query block) items from a work list ordered
//    head-major (longest first within a head) through an atomic ticket: the
//    K/V blocks in use at any time belong to one or two heads and stay in L2,
//    and the dynamic hand-out balances lists of different lengths.
//  * Every wait is bounded (globaltimer); a wait that runs out latches
//    SPADE_ERR_TIMEOUT in the device status word and the CTA winds down,
//    draining its own TMA loads and MMAs before freeing TMEM.
#include <cudaTypedefs.h>

#include <cstdlib>

#include "ptx.cuh"
#include "spade_internal.cuh"

namespace spade {
namespace {

constexpr int kAtomBytes = 128 * 128;        // 128 rows x 128 B: one 64-column swizzle atom of a tile
constexpr int kMaxList = SPADE_TC_MAX_LIST;  // key blocks per work item staged in shared memory
constexpr int kItemRing = 4;                 // work items in flight between the roles
constexpr uint32_t kFullBlock = 1u << 31;    // extent code: every slot valid
constexpr uint32_t kTextBlock = 1u << 30;    // extent code: text block (low bits = valid count)

template <int D, int NQ_, int NS_>
struct Cfg {
  static constexpr int ATOMS = D / 64;
  static constexpr int TILE = 128 * D * 2;
  // K/V ring stages (TMA latency under load is ~1-1.5 us, so the ring holds
  // several (query tile, key block) pairs of look-ahead); shared memory use
  // keeps one CTA per SM, which owns all 512 TMEM columns
  static constexpr int NS = NS_;
  static constexpr int NQ = NQ_;                                  // Q buffers
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_KV = NQ * TILE;
  static constexpr int OFF_PLIST = OFF_KV + NS * TILE;            // producer's copy of the key list
  static constexpr int OFF_SEXT = OFF_PLIST + 4 * kMaxList;       // softmax warps: extent code per block
  static constexpr int OFF_DEC = OFF_SEXT + 4 * kMaxList;         // slot -> (t, y, x) per scheme
  static constexpr int OFF_RED = OFF_DEC + 4 * 128 * SPADE_MAX_SCHEMES;  // row max / sum exchange
  static constexpr int OFF_BAR = OFF_RED + 4 * (2 * 2 * 128 + 2 * 128);
  static constexpr int SMEM = OFF_BAR + 512 + 1024;               // barriers + alignment slack
  static constexpr uint32_t COL_S0 = 0, COL_S1 = 128, COL_O = 256;
  static constexpr uint32_t COL_P0 = 256 + D, COL_P1 = 256 + D + 64;
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr int THREADS = 320;   // producer, MMA, 8 softmax warps
};

struct __align__(64) TcParams {
  CUtensorMap tm_q[SPADE_MAX_SCHEMES];
  CUtensorMap tm_k[SPADE_MAX_SCHEMES];
  CUtensorMap tm_v[SPADE_MAX_SCHEMES];
  CUtensorMap tm_qt, tm_kt, tm_vt;          // text tokens (3-D maps), when present
  Geo geo[SPADE_MAX_SCHEMES];
  HeadInfo head[SPADE_MAX_HEADS];
  const int* cnt;
  const int* idx;
  const int* work;
  uint8_t* out;       // [N + text, heads, D] bf16
  int heads;
  int N;
  int* ticket;        // next work-list position (zeroed by the work-list kernel)
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

// Waiting threads sleep in try_wait (hardware suspend, woken when the phase
// completes) rather than spin: the producer and MMA warps share schedulers
// with two of the softmax warps, and a spinning waiter steals their issue slots.
__device__ __forceinline__ bool wait_bar(uint64_t* bar, uint32_t parity, const Waiter& w) {
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

// Packed tile coordinates of key block `blk`, decoded once per work item so
// the producer's per-tile path has no integer division: video blocks keep
// (bk, bj, bi) in bits 0-11 / 12-21 / 22-30, text blocks set bit 31 and keep
// their index in the low bits.
__device__ __forceinline__ uint32_t pack_coord(const TcParams& p, const Item& I, int blk) {
  if (blk < I.nb) {
    const Geo& g = p.geo[I.scheme];
    const int bk = blk % g.nbw, bj = (blk / g.nbw) % g.nbh, bi = blk / (g.nbw * g.nbh);
    return (uint32_t)bk | ((uint32_t)bj << 12) | ((uint32_t)bi << 22);
  }
  return 0x80000000u | (uint32_t)(blk - I.nb);
}

template <int D>
__device__ __forceinline__ void load_tile(const TcParams& p, const CUtensorMap* vid, const CUtensorMap* txt,
                                          const Item& I, uint32_t pc, uint8_t* dst, uint64_t* bar) {
  if (!(pc & 0x80000000u)) {
    const Geo& g = p.geo[I.scheme];
    const int bk = (int)(pc & 0xfffu), bj = (int)((pc >> 12) & 0x3ffu), bi = (int)(pc >> 22);
#pragma unroll
    for (int a = 0; a < D / 64; ++a)
      ptx::tma_load_5d_elect(dst + a * kAtomBytes, vid, bar, 64 * a, I.h, bk * g.bw, bj * g.bh, bi * g.bt);
  } else {
    const int tb = (int)(pc & 0x7fffffffu);
#pragma unroll
    for (int a = 0; a < D / 64; ++a) ptx::tma_load_3d_elect(dst + a * kAtomBytes, txt, bar, 64 * a, I.h, tb * 128);
  }
}

// Extent code of key block `blk`: clipped (t, y, x) extents of a video block,
// or the valid count of a text block, plus a flag when every slot is valid.
__device__ __forceinline__ uint32_t extent_code(const TcParams& p, const Item& I, int blk) {
  if (blk < I.nb) {
    const Geo& g = p.geo[I.scheme];
    int t0, y0, x0, et, eh, ew;
    block_box(g, blk, t0, y0, x0, et, eh, ew);
    const bool full = et == g.bt && eh == g.bh && ew == g.bw;
    return (uint32_t)et | ((uint32_t)eh << 8) | ((uint32_t)ew << 16) | (full ? kFullBlock : 0u);
  }
  const int valid = min(128, p.text_tokens - (blk - I.nb) * 128);
  return (uint32_t)valid | kTextBlock | (valid >= 128 ? kFullBlock : 0u);
}

// Validity of the 128 key columns of a partial block as four 32-bit words
// (warp-cooperative: lane l decides columns l, l+32, l+64, l+96; `dec` maps a
// slot to its (t, y, x) offsets inside the box).
__device__ __forceinline__ void key_mask(uint32_t code, const uint32_t* dec, int lane, uint32_t (&m)[4]) {
  if (code & kTextBlock) {
    const int valid = (int)(code & 0xffu);
#pragma unroll
    for (int w = 0; w < 4; ++w) m[w] = __ballot_sync(0xffffffffu, lane + 32 * w < valid);
    return;
  }
  const uint32_t et = code & 0xffu, eh = (code >> 8) & 0xffu, ew = (code >> 16) & 0xffu;
#pragma unroll
  for (int w = 0; w < 4; ++w) {
    const uint32_t e = dec[lane + 32 * w];
    m[w] = __ballot_sync(0xffffffffu, (e & 0xffu) < et && ((e >> 8) & 0xffu) < eh && (e >> 16) < ew);
  }
}

// ------------------------------------------------------- exp2 on the FMA pipe --
// 2^x for a pair of floats without the SFU.  Range reduction x = n + f with
// n = round(x) obtained by adding 1.5 * 2^23 (the integer lands in the low
// mantissa bits; Cody & Waite style reduction), |f| <= 1/2; 2^f by a cubic
// fitted to 2^f on Chebyshev nodes of [-1/2, 1/2] (relative error <= 7.5e-5,
// far below the bf16 rounding the result goes through); 2^n is added to the
// exponent field with one integer multiply-add.  Inputs are clamped at -125
// so that every result stays a normal float.
__device__ __forceinline__ float2 exp2_poly2(float2 x) {
  constexpr float kRound = 12582912.0f;  // 1.5 * 2^23
  x.x = fmaxf(x.x, -125.0f);
  x.y = fmaxf(x.y, -125.0f);
  const float2 j = __fadd2_rn(x, make_float2(kRound, kRound));
  const float2 n = __fadd2_rn(j, make_float2(-kRound, -kRound));
  const float2 f = __fadd2_rn(x, make_float2(-n.x, -n.y));
  float2 q = __ffma2_rn(make_float2(0.055171654f, 0.055171654f), f, make_float2(0.24261113f, 0.24261113f));
  q = __ffma2_rn(q, f, make_float2(0.69326097f, 0.69326097f));
  q = __ffma2_rn(q, f, make_float2(0.99992806f, 0.99992806f));
  return make_float2(__int_as_float(__float_as_int(q.x) + (__float_as_int(j.x) << 23)),
                     __int_as_float(__float_as_int(q.y) + (__float_as_int(j.y) << 23)));
}

__device__ __forceinline__ float max3f(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

template <int D, int NQ, int NS>
__global__ void __launch_bounds__(Cfg<D, NQ, NS>::THREADS, 1) attn_tc_kernel(const __grid_constant__ TcParams p) {
  using C = Cfg<D, NQ, NS>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem + C::OFF_Q;
  uint8_t* sKV = smem + C::OFF_KV;
  int* plist = reinterpret_cast<int*>(smem + C::OFF_PLIST);   // packed tile coordinates
  uint32_t* sext = reinterpret_cast<uint32_t*>(smem + C::OFF_SEXT);
  uint32_t* sdec = reinterpret_cast<uint32_t*>(smem + C::OFF_DEC);
  float* pmax = reinterpret_cast<float*>(smem + C::OFF_RED);   // [2 parity][2 halves][128 rows]
  float* psum = pmax + 2 * 2 * 128;                             // [2 halves][128 rows]
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
  uint64_t* item_full = q_full + 12;
  uint64_t* item_empty = item_full + kItemRing;
  uint64_t* xbar = item_empty + kItemRing;      // [quad][block parity]: partner row-max exchange
  uint64_t* ebar = xbar + 8;                    // [quad]: partner row-sum exchange (epilogue)
  uint64_t* stage_bar = ebar + 4;               // softmax warps: key-list extents staged
  int* item_ring = reinterpret_cast<int*>(stage_bar + 1);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(item_ring + kItemRing);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int e = threadIdx.x; e < p.n_schemes * 128; e += blockDim.x) {
    const Geo& g = p.geo[e >> 7];
    const int c = e & 127;
    sdec[e] = (uint32_t)(c / (g.bw * g.bh)) | ((uint32_t)((c / g.bw) % g.bh) << 8) | ((uint32_t)(c % g.bw) << 16);
  }
  if (threadIdx.x == 0) {
    for (int s = 0; s < C::NS; ++s) {
      ptx::mbar_init(&kv_full[s], 1);
      ptx::mbar_init(&kv_empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      ptx::mbar_init(&q_full[b], 1);
      ptx::mbar_init(&q_empty[b], 1);
      ptx::mbar_init(&s_full[b], 1);
      ptx::mbar_init(&p_full[b], 256);
      ptx::mbar_init(&pv_done[b], 1);
    }
    ptx::mbar_init(o_free, 256);
    ptx::mbar_init(mma_fin, 1);
    for (int r = 0; r < kItemRing; ++r) {
      ptx::mbar_init(&item_full[r], 1);
      ptx::mbar_init(&item_empty[r], 1 + 256);   // the MMA warp and every softmax thread
    }
    for (int r = 0; r < 8; ++r) ptx::mbar_init(&xbar[r], 64);
    for (int r = 0; r < 4; ++r) ptx::mbar_init(&ebar[r], 64);
    ptx::mbar_init(stage_bar, 256);
    *abort_flag = 0;
    ptx::fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    for (int s = 0; s < p.n_schemes; ++s) {
      ptx::prefetch_tmap(&p.tm_q[s]);
      ptx::prefetch_tmap(&p.tm_k[s]);
      ptx::prefetch_tmap(&p.tm_v[s]);
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
    // ------------------------------------------- scheduler + TMA producer --
    // The whole warp runs this loop in uniform control flow and stages each
    // item's key list in shared memory; one elected lane takes the ticket,
    // publishes the item (or -1 at the end) to the other roles, and issues
    // each expect-tx / TMA load (elect.sync-predicated, no divergent branch).
    uint32_t kvpos = 0;
    uint32_t last_par[C::NS];
    uint32_t used = 0;
    int qlast[2] = {-1, -1};
    bool ok = true;
    for (int li = 0;; ++li) {
      int it = 0;
      if (lane == 0) {
        it = atomicAdd(p.ticket, 1);
        if (it >= p.n_items) it = -1;
      }
      it = __shfl_sync(0xffffffffu, it, 0);
      const int slot = li % kItemRing;
      ok = __all_sync(0xffffffffu, wait_bar(&item_empty[slot], ((li / kItemRing) & 1) ^ 1, W));
      if (!ok) break;
      if (lane == 0) {
        item_ring[slot] = it;
        ptx::mbar_arrive(&item_full[slot]);
      }
      __syncwarp();
      if (it < 0) break;
      const Item I = get_item(p, it);
      for (int j = lane; j < I.n; j += 32) plist[j] = (int)pack_coord(p, I, key_block(p, I, j));
      __syncwarp();
      const int qs = li % C::NQ;
      ok = __all_sync(0xffffffffu, wait_bar(&q_empty[qs], ((li / C::NQ) & 1) ^ 1, W));
      if (!ok) break;
      ptx::mbar_arrive_expect_tx_elect(&q_full[qs], C::TILE);
      load_tile<D>(p, &p.tm_q[I.scheme], &p.tm_qt, I, pack_coord(p, I, I.qb), sQ + qs * C::TILE, &q_full[qs]);
      qlast[qs] = (li / C::NQ) & 1;
      auto push = [&](const CUtensorMap* vid, const CUtensorMap* txt, int pcw) -> bool {
        const int st = kvpos % C::NS;
        const uint32_t par = (kvpos / C::NS) & 1;
        if (!__all_sync(0xffffffffu, wait_bar(&kv_empty[st], par ^ 1, W))) return false;
        ptx::mbar_arrive_expect_tx_elect(&kv_full[st], C::TILE);
        load_tile<D>(p, vid, txt, I, (uint32_t)pcw, sKV + st * C::TILE, &kv_full[st]);
        last_par[st] = par;
        used |= 1u << st;
        ++kvpos;
        return true;
      };
      // ring order = MMA consumption order: K0, K1, then K_{j+2}, V_j
      for (int j = 0; ok && j < 2 && j < I.n; ++j) ok = push(&p.tm_k[I.scheme], &p.tm_kt, plist[j]);
      for (int j = 0; ok && j < I.n; ++j) {
        if (j + 2 < I.n) ok = push(&p.tm_k[I.scheme], &p.tm_kt, plist[j + 2]);
        if (ok) ok = push(&p.tm_v[I.scheme], &p.tm_vt, plist[j]);
      }
      __syncwarp();
      if (!ok) break;
    }
    if (lane == 0 && !ok) {   // wind down: let every load this warp issued land before the CTA exits
      for (int st = 0; st < C::NS; ++st)
        if (used & (1u << st)) drain_bar(&kv_full[st], last_par[st], 100000000LL);
      for (int b = 0; b < C::NQ; ++b)
        if (qlast[b] >= 0) drain_bar(&q_full[b], qlast[b], 100000000LL);
    }
  } else if (warp == 1) {
    // -------------------------------------------------------- MMA issuer --
    // The whole warp runs this loop in uniform control flow (waits, item
    // bookkeeping, descriptors); one elected lane issues each tcgen05.mma /
    // commit.  Issuing from a lane-divergent region costs a register-to-
    // uniform conversion per MMA, which is slower than the MMA itself.
    constexpr uint32_t idesc_qk = make_idesc(128, 128, false);
    constexpr uint32_t idesc_pv = make_idesc(128, D, true);
    uint32_t kvpos = 0, g = 0;
    bool ok = true;
    for (int li = 0; ok; ++li) {
      const int slot = li % kItemRing;
      ok = wait_bar(&item_full[slot], (li / kItemRing) & 1, W);
      if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
      const int it = item_ring[slot];
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(&item_empty[slot]);
      if (it < 0) break;
      const Item I = get_item(p, it);
      const int qs = li % C::NQ;
      ok = wait_bar(&q_full[qs], (li / C::NQ) & 1, W);
      if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
      ptx::tc_fence_after();
      const uint64_t qdesc = kmajor_desc(ptx::smem_u32(sQ + qs * C::TILE));
      // S(j) -> S buffer j%2, P(j) -> P buffer j%2.  Once softmax(j) has
      // published P(j) (and so released S buffer j%2), S(j+2) is issued ahead
      // of PV(j), so the next-but-one score tile is ready as early as possible.
      auto issue_s = [&](int jj) -> bool {
        const int st = kvpos % C::NS;
        if (!__all_sync(0xffffffffu, wait_bar(&kv_full[st], (kvpos / C::NS) & 1, W))) return false;
        ptx::tc_fence_after();
        const uint32_t b = (g + jj) & 1;
        const uint64_t kdesc = kmajor_desc(ptx::smem_u32(sKV + st * C::TILE));
        const uint32_t ts = tmem + (b ? C::COL_S1 : C::COL_S0);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint64_t off = (uint64_t)(((kk >> 2) * kAtomBytes + (kk & 3) * 32) >> 4);
          ptx::mma_ss_elect(ts, qdesc + off, kdesc + off, idesc_qk, kk > 0 ? 1u : 0u);
        }
        ptx::tc_commit_elect(&s_full[b]);
        ptx::tc_commit_elect(&kv_empty[st]);
        ++kvpos;
        if (jj == I.n - 1) ptx::tc_commit_elect(&q_empty[qs]);
        return true;
      };
      auto issue_pv = [&](int jj) -> bool {
        const uint32_t b = (g + jj) & 1;
        const int st = kvpos % C::NS;
        bool w = wait_bar(&kv_full[st], (kvpos / C::NS) & 1, W);
        if (jj == 0) w = w && wait_bar(o_free, (li & 1) ^ 1, W);
        if (!__all_sync(0xffffffffu, w)) return false;
        ptx::tc_fence_after();
        const uint64_t vdesc = mnmajor_desc(ptx::smem_u32(sKV + st * C::TILE));
        const uint32_t tp = tmem + (b ? C::COL_P1 : C::COL_P0);
        const uint32_t acc0 = jj > 0 ? 1u : 0u;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          ptx::mma_ts_elect(tmem + C::COL_O, tp + kk * 8, vdesc + (uint64_t)(kk * (2048 >> 4)), idesc_pv,
                            kk > 0 ? 1u : acc0);
        ptx::tc_commit_elect(&pv_done[b]);
        ptx::tc_commit_elect(&kv_empty[st]);
        ++kvpos;
        return true;
      };
      for (int j = 0; ok && j < 2 && j < I.n; ++j) ok = issue_s(j);
      for (int j = 0; ok && j < I.n; ++j) {
        const uint32_t gj = g + j;
        ok = __all_sync(0xffffffffu, wait_bar(&p_full[gj & 1], (gj >> 1) & 1, W));
        if (ok && j + 2 < I.n) ok = issue_s(j + 2);
        if (ok) ok = issue_pv(j);
      }
      g += I.n;
    }
    // every MMA this warp issued completes before TMEM is released
    ptx::tc_commit_elect(mma_fin);
    drain_bar(mma_fin, 0, 100000000LL);
  } else {
    // ---------------------------------------- softmax / correction / epilogue --
    // Eight warps, two per TMEM lane quadrant: warp half hf owns score columns
    // [64 hf, 64 hf + 64) of the quadrant's 32 rows (and the same half of O).
    // The two partners (same quadrant, same scheduler) exchange their partial
    // row maxima through shared memory, so both use the same running max; row
    // sums stay per half and are combined in the epilogue.
    constexpr int OH = D / 2;                          // O columns per half
    const int hf = (warp - 2) >> 2;
    const int quad = warp & 3;
    const int row = quad * 32 + lane;                  // TMEM lane = query slot
    const uint32_t lane_base = (uint32_t)(quad * 32) << 16;
    const int stid = threadIdx.x - 64;                 // 0..255 within the softmax warps
    const float sl2 = p.scale_log2;
    const float2 sl2x2 = make_float2(sl2, sl2);
    uint32_t g = 0;
    bool ok = true;
    for (int li = 0; ok; ++li) {
      const int slot = li % kItemRing;
      ok = wait_bar(&item_full[slot], (li / kItemRing) & 1, W);
      if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
      const int it = item_ring[slot];
      ptx::mbar_arrive(&item_empty[slot]);
      if (it < 0) break;
      const Item I = get_item(p, it);
      for (int j = stid; j < I.n; j += 256) sext[j] = extent_code(p, I, key_block(p, I, j));
      ptx::mbar_arrive(stage_bar);
      ok = wait_bar(stage_bar, li & 1, W);
      if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
      const uint32_t* dec = sdec + 128 * I.scheme;
      float m_use = 0.f, l = 0.f;                      // l: this half's share of the row sum
      for (int j = 0; j < I.n; ++j) {
        const uint32_t gj = g + j, b = gj & 1;
        ok = wait_bar(&s_full[b], (gj >> 1) & 1, W);
        if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
        ptx::tc_fence_after();
        uint32_t sr[64];
        ptx::tmem_ld64(tmem + lane_base + (b ? C::COL_S1 : C::COL_S0) + 64 * hf, sr);
        const uint32_t code = sext[j];
        const bool full = (code & kFullBlock) != 0;
        if (!full) {
          uint32_t mw[4];
          key_mask(code, dec, lane, mw);
          const uint32_t w0 = hf ? mw[2] : mw[0], w1 = hf ? mw[3] : mw[1];
#pragma unroll
          for (int c = 0; c < 64; ++c)
            if (!((((c < 32) ? w0 : w1) >> (c & 31)) & 1u)) sr[c] = 0xff800000u;   // -inf
        }
        // partial row max (eight 3-input chains), then the partner's half
        float mk[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) mk[k] = fmaxf(__uint_as_float(sr[k]), __uint_as_float(sr[k + 8]));
#pragma unroll
        for (int c = 16; c < 64; c += 16) {
#pragma unroll
          for (int k = 0; k < 8; ++k)
            mk[k] = max3f(mk[k], __uint_as_float(sr[c + k]), __uint_as_float(sr[c + k + 8]));
        }
        const float pm = max3f(max3f(mk[0], mk[1], mk[2]), max3f(mk[3], mk[4], mk[5]), fmaxf(mk[6], mk[7]));
        float* px = pmax + (b * 2) * 128;
        px[hf * 128 + row] = pm;
        ptx::mbar_arrive(&xbar[quad * 2 + b]);
        ok = wait_bar(&xbar[quad * 2 + b], (gj >> 1) & 1, W);
        if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
        const float mx = fmaxf(pm, px[(1 - hf) * 128 + row]) * sl2;
        if (j == 0) {
          m_use = mx;
        } else {
          const bool need = mx > m_use + 8.0f;
          if (__any_sync(0xffffffffu, need)) {
            // rescale this half of O by 2^(m_use - mx) once PV(j-1) has landed
            const uint32_t gp = gj - 1;
            ok = wait_bar(&pv_done[gp & 1], (gp >> 1) & 1, W);
            if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
            ptx::tc_fence_after();
            const float alpha = need ? ptx::ex2(m_use - mx) : 1.0f;
            if (need) { l *= alpha; m_use = mx; }
#pragma unroll 1
            for (int c0 = 0; c0 < OH; c0 += 32) {
              uint32_t ob[32];
              const uint32_t ta = tmem + lane_base + C::COL_O + OH * hf + c0;
              ptx::tmem_ld32(ta, ob);
#pragma unroll
              for (int c = 0; c < 32; ++c) ob[c] = __float_as_uint(__uint_as_float(ob[c]) * alpha);
              ptx::tmem_st32(ta, ob);
            }
          }
        }
        // p = 2^(s*scale*log2e - m): one FFMA2 per column pair, then the SFU,
        // straight-line so the SFU ops pipeline back to back (masked columns
        // are -inf and give an exact 0)
        const float2 nm2 = make_float2(-m_use, -m_use);
        float2 pe[32];
#pragma unroll
        for (int c = 0; c < 32; ++c)
          pe[c] = __ffma2_rn(make_float2(__uint_as_float(sr[2 * c]), __uint_as_float(sr[2 * c + 1])), sl2x2, nm2);
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          pe[c].x = ptx::ex2(pe[c].x);
          pe[c].y = ptx::ex2(pe[c].y);
        }
        float2 acc[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) acc[k] = pe[k];
#pragma unroll
        for (int c = 8; c < 32; ++c) acc[c & 7] = __fadd2_rn(acc[c & 7], pe[c]);
        const float2 a = __fadd2_rn(__fadd2_rn(__fadd2_rn(acc[0], acc[1]), __fadd2_rn(acc[2], acc[3])),
                                    __fadd2_rn(__fadd2_rn(acc[4], acc[5]), __fadd2_rn(acc[6], acc[7])));
        l += a.x + a.y;
        uint32_t pk[32];
#pragma unroll
        for (int c = 0; c < 32; ++c) pk[c] = ptx::pack_bf16x2(pe[c].x, pe[c].y);
        if (j >= 2) {                                  // P buffer b was read by PV(j-2)
          const uint32_t gp = gj - 2;
          ok = wait_bar(&pv_done[b], (gp >> 1) & 1, W);
          if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
        }
        ptx::tmem_st32(tmem + lane_base + (b ? C::COL_P1 : C::COL_P0) + 32 * hf, pk);
        ptx::tc_fence_before();
        ptx::mbar_arrive(&p_full[b]);
      }
      if (!ok) break;
      // epilogue: O / l -> bf16, each thread stores its half of its query row
      // straight to token order (padded slots of edge blocks are skipped)
      const uint32_t gl = g + I.n - 1;
      ok = wait_bar(&pv_done[gl & 1], (gl >> 1) & 1, W);
      if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
      ptx::tc_fence_after();
      psum[hf * 128 + row] = l;
      ptx::mbar_arrive(&ebar[quad]);
      ok = wait_bar(&ebar[quad], li & 1, W);
      if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
      const float inv = 1.0f / (l + psum[(1 - hf) * 128 + row]);
      long long tok = -1;
      if (I.qb < I.nb) {
        const Geo& gg = p.geo[I.scheme];
        int t0, y0, x0, et, eh, ew;
        block_box(gg, I.qb, t0, y0, x0, et, eh, ew);
        const uint32_t e = dec[row];
        const int tl = (int)(e & 0xffu), yl = (int)((e >> 8) & 0xffu), xl = (int)(e >> 16);
        if (tl < et && yl < eh && xl < ew) tok = ((long long)(t0 + tl) * gg.H + (y0 + yl)) * gg.W + (x0 + xl);
      } else {
        const int t = (I.qb - I.nb) * 128 + row;
        if (t < p.text_tokens) tok = (long long)p.N + t;
      }
      uint4* dst = reinterpret_cast<uint4*>(p.out + ((tok < 0 ? 0 : tok) * p.heads + I.h) * (long long)(D * 2) +
                                            OH * 2 * hf);
#pragma unroll
      for (int c0 = 0; c0 < OH; c0 += 32) {
        uint32_t ov[32];
        ptx::tmem_ld32(tmem + lane_base + C::COL_O + OH * hf + c0, ov);
        if (tok >= 0) {
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4) {
            const int c = q4 * 8;
            uint4 w;
            w.x = ptx::pack_bf16x2(__uint_as_float(ov[c + 0]) * inv, __uint_as_float(ov[c + 1]) * inv);
            w.y = ptx::pack_bf16x2(__uint_as_float(ov[c + 2]) * inv, __uint_as_float(ov[c + 3]) * inv);
            w.z = ptx::pack_bf16x2(__uint_as_float(ov[c + 4]) * inv, __uint_as_float(ov[c + 5]) * inv);
            w.w = ptx::pack_bf16x2(__uint_as_float(ov[c + 6]) * inv, __uint_as_float(ov[c + 7]) * inv);
            dst[c0 / 8 + q4] = w;
          }
        }
      }
      ptx::tc_fence_before();
      ptx::mbar_arrive(o_free);
      g += I.n;
    }
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

template <int D, int NQ, int NS>
cudaError_t launch_d(const TcParams& tp, int grid, cudaStream_t s) {
  using C = Cfg<D, NQ, NS>;
  static_assert(C::SMEM <= 232448, "shared memory budget");
  cudaError_t e =
      cudaFuncSetAttribute(attn_tc_kernel<D, NQ, NS>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
  if (e != cudaSuccess) return e;
  attn_tc_kernel<D, NQ, NS><<<grid, C::THREADS, C::SMEM, s>>>(tp);
  return cudaGetLastError();
}

}  // namespace

bool attn_tc_supported(const AttnArgs& a) {
  if (a.dt != SPADE_BF16 || (a.d != 64 && a.d != 128)) return false;
  for (int s = 0; s < a.n_schemes; ++s) {
    if (a.geo[s].bs != 128) return false;
    if (a.geo[s].nbw >= 4096 || a.geo[s].nbh >= 1024 || a.geo[s].nbt >= 512) return false;   // packed coords
  }
  const int ntb = text_blocks(a.text_tokens);
  for (int h = 0; h < a.heads; ++h)
    if (a.head[h].nb + ntb > kMaxList) return false;
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
        !map_video(&tp.tm_v[sc], a.v, g, a.heads, a.d)) {
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
    if (!map_text(&tp.tm_qt, qb, a.text_tokens, a.heads, a.d) ||
        !map_text(&tp.tm_kt, kb, a.text_tokens, a.heads, a.d) ||
        !map_text(&tp.tm_vt, vb, a.text_tokens, a.heads, a.d)) {
      *why = "tensor map encoding failed (text)";
      return cudaErrorInvalidValue;
    }
  }
  for (int h = 0; h < a.heads; ++h) tp.head[h] = a.head[h];
  tp.cnt = a.cnt;
  tp.idx = a.idx;
  tp.work = a.work;
  tp.out = static_cast<uint8_t*>(a.out);
  tp.heads = a.heads;
  tp.N = a.N;
  tp.ticket = a.ticket;
  tp.n_items = a.n_items;
  tp.n_schemes = a.n_schemes;
  tp.ntb = text_blocks(a.text_tokens);
  tp.text_tokens = a.text_tokens;
  tp.scale_log2 = 1.4426950408889634f / sqrtf((float)a.d);
  tp.status = a.status;
  tp.timeout_ns = device_wait_timeout_ns();
  const int grid = a.n_items < num_sms() ? a.n_items : num_sms();
  if (grid <= 0) return cudaSuccess;
  if (a.d == 64) return launch_d<64, 2, 8>(tp, grid, s);
  const char* v = getenv("SPADE_TC_VARIANT");   // ring-depth experiment (temporary)
  if (v && v[0] == '1') return launch_d<128, 2, 4>(tp, grid, s);
  return launch_d<128, 1, 5>(tp, grid, s);
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

// ------------------------------------------------ FMA-pipe exp2 self test --
__global__ void exp2_poly_selftest_kernel(const float* __restrict__ x, float* __restrict__ y, int n) {
  const int i = 2 * (blockIdx.x * blockDim.x + threadIdx.x);
  if (i + 1 < n) {
    const float2 r = exp2_poly2(make_float2(x[i], x[i + 1]));
    y[i] = r.x;
    y[i + 1] = r.y;
  } else if (i < n) {
    y[i] = exp2_poly2(make_float2(x[i], 0.f)).x;
  }
}

cudaError_t launch_exp2_poly_selftest(const float* x, float* y, int n, cudaStream_t s) {
  const int pairs = (n + 1) / 2;
  exp2_poly_selftest_kernel<<<(pairs + 255) / 256, 256, 0, s>>>(x, y, n);
  return cudaGetLastError();
}

}  // namespace spade
