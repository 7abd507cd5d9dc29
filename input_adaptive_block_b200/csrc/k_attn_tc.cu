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
//    swizzled -- the layout the MMA reads.  Out-of-grid query slots are
//    zero-filled by the TMA unit.  Key/value blocks clipped by the grid edge
//    are loaded with a box of their own clipped extents (one map per edge
//    case), so their valid tokens form a prefix of the tile: the score MMA's
//    N and the P V MMA's K stop at that prefix (rounded up to 16) instead of
//    computing padded columns, and the softmax masks the columns past it.  No
//    tiled copy of Q/K/V is ever written.
//  * tcgen05.mma (kind::f16, bf16 in, fp32 accumulate), issued by one thread.
//    TMEM (512 columns): five overlapping score slots of 128 fp32 columns,
//    64 columns apart (slot k = columns [64 k, 64 k + 128); key block g of the
//    CTA uses slot g % 5), then O (fp32, columns 384-511).  The softmax reads
//    S(g) into registers and writes P(g) (bf16) over the first half of its
//    slot, where P V(g) reads it.  A slot's upper half is the next slot's P
//    region, so S(g) is issued once S(g-1) is in registers and P V(g-4) has
//    completed: four blocks of P V -> S slack instead of the three that three
//    disjoint 128-column buffers would give, and a group never waits for its
//    previous P V before writing the next P.
//  * Warp specialisation: warp 0 hands out work and issues TMA loads (one K/V
//    ring), warp 1 issues the Q K^T MMAs and warp 2 the P V MMAs (so neither
//    stream's waits hold back the other's issue), warps 4-7 and 8-11 are two
//    softmax warpgroups (with most of the register file: setmaxnreg) taking the even and the odd kept blocks of
//    the query tile: each thread owns one query row (TMEM lane) with all 128
//    key columns.  The two groups accumulate into one O, so they share a
//    per-row reference maximum through shared memory: block j reads the
//    reference left by block j-1 (a short handshake), raises it only when its
//    own row maximum is more than 2^8 above (then rescales O once the P V
//    issued before it has landed), and every block's P is taken relative to
//    that reference.  Row sums stay per group and are combined in the epilogue
//    (O / l -> bf16 -> token order; each group writes half of the columns).
//  * Persistent CTAs take (head, query block) items from a work list ordered
//    head-major (longest first within a head) through an atomic ticket: the
//    K/V blocks in use at any time belong to one or two heads and stay in L2,
//    and the dynamic hand-out balances lists of different lengths.
//  * Every wait is bounded (globaltimer); a wait that runs out latches
//    SPADE_ERR_TIMEOUT in the device status word and the CTA winds down,
//    draining its own TMA loads and MMAs before freeing TMEM.
#include <cudaTypedefs.h>


#include "ptx.cuh"
#include "spade_internal.cuh"

namespace spade {
namespace {

constexpr int kAtomBytes = 128 * 128;        // 128 rows x 128 B: one 64-column swizzle atom of a tile
constexpr int kMaxList = SPADE_TC_MAX_LIST;  // key blocks per work item staged in shared memory
constexpr int kItemRing = 4;                 // work items in flight between the roles
constexpr uint32_t kFullBlock = 1u << 31;    // extent code: every slot valid (low bits = 128)
constexpr int kEdgeCases = 8;                // key/value maps per scheme: bit 0 t-, bit 1 y-, bit 2 x-edge

template <int D, int NS_>
struct Cfg {
  static constexpr int TILE = 128 * D * 2;
  // K/V ring stages (TMA latency under load is ~1-1.5 us, so the ring holds
  // several key blocks of look-ahead); shared memory use keeps one CTA per
  // SM, which owns all 512 TMEM columns
  static constexpr int NS = NS_;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_KV = TILE;
  static constexpr int OFF_PLIST = OFF_KV + NS * TILE;            // producer's copy of the key list
  static constexpr int OFF_SEXT = OFF_PLIST + 4 * kMaxList;       // softmax: extent code per block
  static constexpr int OFF_DEC = OFF_SEXT + 4 * kMaxList;         // slot -> (t, y, x) per scheme
  static constexpr int OFF_NV = OFF_DEC + 4 * 128 * SPADE_MAX_SCHEMES;     // valid rows per K/V ring stage
  static constexpr int OFF_MREF = OFF_NV + 4 * 16;                          // per-row reference max
  static constexpr int OFF_LX = OFF_MREF + 4 * 128;               // [2 groups][128 rows] row sums
  static constexpr int OFF_BAR = OFF_LX + 4 * 2 * 128;
  static constexpr int SMEM = OFF_BAR + 512 + 1024;               // barriers + alignment slack
  // five score slots 64 columns apart: S(g) at 64 (g % 5), g counting the
  // CTA's key blocks over all its items; P(g) (bf16 pairs) is written over
  // the first 64 columns of its slot, which the slot before it overlaps
  static constexpr uint32_t COL_S = 0;
  static constexpr int NSL = 5;                  // score slots, 64 columns apart
  static constexpr uint32_t COL_O = 384;
  static_assert(COL_S + 64 * (NSL - 1) + 128 <= COL_O && COL_O + D <= 512, "TMEM layout");
  static constexpr uint32_t TMEM_COLS = 512;
  // warpgroup 0: producer, two MMA issuers, one idle warp; warpgroups 1-2:
  // softmax.  Registers per thread after the split (setmaxnreg): the split
  // must fit in the launch-time pool of THREADS x (registers per thread).
  static constexpr int THREADS = 384;
  static constexpr int REG_CTRL = 64;            // the producer and MMA-issuer loops fit without spilling
  static constexpr int REG_SOFTMAX = 208;
  static constexpr int REG_POOL_NEEDED = 128 * REG_CTRL + 256 * REG_SOFTMAX;
};

struct __align__(64) TcParams {
  CUtensorMap tm_q[SPADE_MAX_SCHEMES];
  CUtensorMap tm_k[SPADE_MAX_SCHEMES][kEdgeCases];   // box = the clipped extents of each edge case
  CUtensorMap tm_v[SPADE_MAX_SCHEMES][kEdgeCases];
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

// Query tile: the full box (out-of-grid slots zero-filled, slot order t, y, x).
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

// Edge case of a video block (bit 0: clipped in t, 1: in y, 2: in x) and its
// number of valid tokens.
__device__ __forceinline__ int edge_case(const Geo& g, int bi, int bj, int bk, int& nv) {
  const int et = min(g.bt, g.T - bi * g.bt), eh = min(g.bh, g.H - bj * g.bh), ew = min(g.bw, g.W - bk * g.bw);
  nv = et * eh * ew;
  return (et < g.bt ? 1 : 0) | (eh < g.bh ? 2 : 0) | (ew < g.bw ? 4 : 0);
}

// Key or value tile into one ring stage: a video block through the map of its
// edge case (valid tokens = the first nv rows, in t, y, x order), a text
// block through the 3-D map (rows past the text end zero-filled).  The
// stage's valid row count goes to *nv_slot before the barrier is armed with
// the box's bytes (the arrival releases it to the MMA warps).  Whole warp,
// uniform control flow.
template <int D>
__device__ __forceinline__ void load_kv_tile(const TcParams& p, const CUtensorMap (&vid)[kEdgeCases],
                                             const CUtensorMap* txt, const Item& I, uint32_t pc, uint8_t* dst,
                                             uint64_t* bar, volatile int* nv_slot) {
  if (!(pc & 0x80000000u)) {
    const Geo& g = p.geo[I.scheme];
    const int bk = (int)(pc & 0xfffu), bj = (int)((pc >> 12) & 0x3ffu), bi = (int)(pc >> 22);
    int nv;
    const CUtensorMap* m = &vid[edge_case(g, bi, bj, bk, nv)];
    *nv_slot = nv;
    __syncwarp();
    ptx::mbar_arrive_expect_tx_elect(bar, (uint32_t)(nv * 2 * D));
#pragma unroll
    for (int a = 0; a < D / 64; ++a)
      ptx::tma_load_5d_elect(dst + a * kAtomBytes, m, bar, 64 * a, I.h, bk * g.bw, bj * g.bh, bi * g.bt);
    return;
  }
  const int tb = (int)(pc & 0x7fffffffu);
  *nv_slot = min(128, p.text_tokens - tb * 128);
  __syncwarp();
  ptx::mbar_arrive_expect_tx_elect(bar, (uint32_t)(128 * 2 * D));
#pragma unroll
  for (int a = 0; a < D / 64; ++a) ptx::tma_load_3d_elect(dst + a * kAtomBytes, txt, bar, 64 * a, I.h, tb * 128);
}

// Valid key columns of key block `blk` (a prefix of the tile: see
// load_kv_tile), with a flag when all 128 are valid.
__device__ __forceinline__ uint32_t extent_code(const TcParams& p, const Item& I, int blk) {
  int valid;
  if (blk < I.nb) {
    const Geo& g = p.geo[I.scheme];
    int t0, y0, x0, et, eh, ew;
    block_box(g, blk, t0, y0, x0, et, eh, ew);
    valid = et * eh * ew;
  } else {
    valid = min(128, p.text_tokens - (blk - I.nb) * 128);
  }
  return (uint32_t)valid | (valid >= 128 ? kFullBlock : 0u);
}

__device__ __forceinline__ float max3f(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

template <int D, int NS>
__global__ void __launch_bounds__(Cfg<D, NS>::THREADS, 1) attn_tc_kernel(const __grid_constant__ TcParams p) {
  using C = Cfg<D, NS>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem + C::OFF_Q;
  uint8_t* sKV = smem + C::OFF_KV;
  int* plist = reinterpret_cast<int*>(smem + C::OFF_PLIST);   // packed tile coordinates
  uint32_t* sext = reinterpret_cast<uint32_t*>(smem + C::OFF_SEXT);
  uint32_t* sdec = reinterpret_cast<uint32_t*>(smem + C::OFF_DEC);
  volatile int* stage_nv = reinterpret_cast<volatile int*>(smem + C::OFF_NV);   // valid rows of each ring stage
  float* mref = reinterpret_cast<float*>(smem + C::OFF_MREF);  // [128 rows] reference max (log2 domain)
  float* lx = reinterpret_cast<float*>(smem + C::OFF_LX);      // [2 groups][128 rows] final row sums
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* kv_full = bars;
  uint64_t* kv_empty = bars + NS;
  uint64_t* q_full = bars + 2 * NS;
  uint64_t* q_empty = q_full + 1;
  constexpr int NSL = C::NSL;
  uint64_t* s_full = q_full + 2;              // [NSL] S(g) in slot g % NSL (MMA commit)
  uint64_t* p_full = s_full + NSL;            // [NSL] P(g) written over the slot's first 64 columns (128 threads)
  uint64_t* buf_free = p_full + NSL;          // [NSL] P V(g) complete (MMA commit)
  uint64_t* s_read = buf_free + NSL;          // [NSL] S(g) loaded into registers by its softmax group (128 threads)
  uint64_t* md = s_read + NSL;                // [2] reference max of block j final (128 threads of its group)
  uint64_t* o_full = md + 2;                  // last P V of the item complete
  uint64_t* o_free = o_full + 1;              // epilogue has read O (256 threads)
  uint64_t* lx_bar = o_free + 1;              // both groups' final row sums published (256 threads)
  uint64_t* stage_bar = lx_bar + 1;           // extent codes of the item staged (256 threads)
  uint64_t* mma_fin = stage_bar + 1;          // [2] per MMA warp: all its MMAs complete
  uint64_t* item_full = mma_fin + 2;
  uint64_t* item_empty = item_full + kItemRing;
  int* item_ring = reinterpret_cast<int*>(item_empty + kItemRing);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(item_ring + kItemRing);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // A short key/value tile leaves the rows past its (16-rounded) prefix as
  // the ring stage last held them; zeroing the ring once keeps them finite
  // (0 * p = 0 in P V) before any tile has landed.
  for (int e = threadIdx.x; e < NS * C::TILE / 16; e += blockDim.x)
    reinterpret_cast<uint4*>(sKV)[e] = make_uint4(0u, 0u, 0u, 0u);
  ptx::fence_proxy_async_smem();
  for (int e = threadIdx.x; e < p.n_schemes * 128; e += blockDim.x) {
    const Geo& g = p.geo[e >> 7];
    const int c = e & 127;
    sdec[e] = (uint32_t)(c / (g.bw * g.bh)) | ((uint32_t)((c / g.bw) % g.bh) << 8) | ((uint32_t)(c % g.bw) << 16);
  }
  if (threadIdx.x == 0) {
    for (int s = 0; s < NS; ++s) {
      ptx::mbar_init(&kv_full[s], 1);
      ptx::mbar_init(&kv_empty[s], 1);
    }
    ptx::mbar_init(q_full, 1);
    ptx::mbar_init(q_empty, 1);
    for (int b = 0; b < NSL; ++b) {
      ptx::mbar_init(&s_full[b], 1);
      ptx::mbar_init(&p_full[b], 128);
      ptx::mbar_init(&buf_free[b], 1);
      ptx::mbar_init(&s_read[b], 128);
    }
    ptx::mbar_init(&md[0], 128);
    ptx::mbar_init(&md[1], 128);
    ptx::mbar_init(o_full, 1);
    ptx::mbar_init(o_free, 256);
    ptx::mbar_init(lx_bar, 256);
    ptx::mbar_init(stage_bar, 256);
    ptx::mbar_init(&mma_fin[0], 1);
    ptx::mbar_init(&mma_fin[1], 1);
    for (int r = 0; r < kItemRing; ++r) {
      ptx::mbar_init(&item_full[r], 1);
      ptx::mbar_init(&item_empty[r], 2 + 256);   // both MMA warps and every softmax thread
    }
    *abort_flag = 0;
    ptx::fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    for (int s = 0; s < p.n_schemes; ++s) {
      ptx::prefetch_tmap(&p.tm_q[s]);
      for (int c = 0; c < kEdgeCases; ++c) {
        ptx::prefetch_tmap(&p.tm_k[s][c]);
        ptx::prefetch_tmap(&p.tm_v[s][c]);
      }
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
  if (warp < 4) {
  // ------------------------------------------------ warpgroup 0: control --
  ptx::setmaxnreg_dec<C::REG_CTRL>();
  if (warp == 3) {
    // idle: its registers went to the softmax warpgroups
  } else if (warp == 0) {
    // ------------------------------------------- scheduler + TMA producer --
    // The whole warp runs this loop in uniform control flow and stages each
    // item's key list in shared memory; one elected lane takes the ticket,
    // publishes the item (or -1 at the end) to the other roles, and issues
    // each expect-tx / TMA load (elect.sync-predicated, no divergent branch).
    // Ring order = MMA consumption order: K0, K1, K2, then V_j, K_{j+3} (S(j+3) waits for P V(j) anyway).
    uint32_t kvpos = 0;
    uint32_t last_par[NS];
    uint32_t used = 0;
    int qlast = -1;
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
      ok = __all_sync(0xffffffffu, wait_bar(q_empty, (li & 1) ^ 1, W));
      if (!ok) break;
      ptx::mbar_arrive_expect_tx_elect(q_full, C::TILE);
      load_tile<D>(p, &p.tm_q[I.scheme], &p.tm_qt, I, pack_coord(p, I, I.qb), sQ, q_full);
      qlast = li & 1;
      auto push = [&](const CUtensorMap (&vid)[kEdgeCases], const CUtensorMap* txt, int pcw) -> bool {
        const int st = kvpos % NS;
        const uint32_t par = (kvpos / NS) & 1;
        if (!__all_sync(0xffffffffu, wait_bar(&kv_empty[st], par ^ 1, W))) return false;
        load_kv_tile<D>(p, vid, txt, I, (uint32_t)pcw, sKV + st * C::TILE, &kv_full[st], &stage_nv[st]);
        last_par[st] = par;
        used |= 1u << st;
        ++kvpos;
        return true;
      };
      for (int j = 0; ok && j < 3 && j < I.n; ++j) ok = push(p.tm_k[I.scheme], &p.tm_kt, plist[j]);
      for (int j = 0; ok && j < I.n; ++j) {
        ok = push(p.tm_v[I.scheme], &p.tm_vt, plist[j]);
        if (ok && j + 3 < I.n) ok = push(p.tm_k[I.scheme], &p.tm_kt, plist[j + 3]);
      }
      __syncwarp();
      if (!ok) break;
    }
    if (lane == 0 && !ok) {   // wind down: let every load this warp issued land before the CTA exits
      for (int st = 0; st < NS; ++st)
        if (used & (1u << st)) drain_bar(&kv_full[st], last_par[st], 100000000LL);
      if (qlast >= 0) drain_bar(q_full, qlast, 100000000LL);
    }
  } else if (warp == 1 || warp == 2) {
    // ------------------------------------------------------- MMA issuers --
    // Warp 1 issues the score MMAs S(g) = Q K_g^T, warp 2 the P V(g) MMAs.
    // Each commit tracks only its own warp's MMAs, so each warp blocks only on
    // its own events: S(g) waits for its K tile, for S(g-1) to be in the
    // softmax's registers (the lower half of slot g % 5 is the upper half of
    // the slot before) and for P V(g-4) to have completed (the upper half is
    // P(g-4)'s region); P V(g) waits for P(g) and V_g.  One warp waiting never holds back the other's issue,
    // which keeps the (shallow) tensor instruction queue fed; a single issuer
    // in a fixed order measured 23 % slower.  Each warp runs in uniform
    // control flow; one elected lane issues each tcgen05.mma / commit.
    //
    // Ring positions inside an item with n blocks (base B): K_k at B + k for
    // k < 3, at B + m + 2 (k - 3) + 1 otherwise; V_j at B + m + j + min(j, n - 3),
    // where m = min(n, 3) -- the producer's order K0, K1, K2, then V_j, K_{j+3}.
    const bool is_s = warp == 1;
    constexpr uint32_t idesc_pv = make_idesc(128, D, true);
    uint32_t base = 0;         // ring position of the item's first tile
    uint32_t g = 0;            // key blocks of this warp's stream so far (all items): slot g % 5
    bool ok = true;
    for (int li = 0; ok; ++li) {
      const int slot = li % kItemRing;
      ok = wait_bar(&item_full[slot], (li / kItemRing) & 1, W);
      if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
      const int it = item_ring[slot];
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(&item_empty[slot]);
      if (it < 0) break;
      const int n = get_item(p, it).n;
      const int m = n < 3 ? n : 3;
      const int nk3 = n > 3 ? n - 3 : 0;
      if (is_s) {
        ok = wait_bar(q_full, li & 1, W);
        if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
        ptx::tc_fence_after();
        const uint64_t qdesc = kmajor_desc(ptx::smem_u32(sQ));
        for (int k = 0; ok && k < n; ++k, ++g) {
          const uint32_t b = g % NSL;
          const uint32_t pos = base + (uint32_t)(k < 3 ? k : m + 2 * (k - 3) + 1);
          const int st = (int)(pos % NS);
          bool w = wait_bar(&kv_full[st], (pos / NS) & 1, W);
          // slot b = columns [64 b, 64 b + 128): its upper half is the P region of
          // slot b + 1, last used by block g - (NSL - 1) -- wait for that P V (which,
          // in order, also covers P(g - NSL) in the lower half); its lower half is
          // the upper half of slot b - 1 -- wait until S(g - 1) is in registers
          if (g >= NSL - 1) w = w && wait_bar(&buf_free[(g + 1) % NSL], ((g - (NSL - 1)) / NSL) & 1, W);
          if (b != 0) w = w && wait_bar(&s_read[b - 1], ((g - 1) / NSL) & 1, W);
          if (!__all_sync(0xffffffffu, w)) { ok = false; break; }
          ptx::tc_fence_after();
          const uint64_t kdesc = kmajor_desc(ptx::smem_u32(sKV + st * C::TILE));
          const uint32_t ts = tmem + C::COL_S + 64 * b;
          // N = valid key rows rounded up to 16 (the columns past it are masked by the softmax)
          const uint32_t idesc_qk = make_idesc(128, (stage_nv[st] + 15) & ~15, false);
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint64_t off = (uint64_t)(((kk >> 2) * kAtomBytes + (kk & 3) * 32) >> 4);
            ptx::mma_ss_elect(ts, qdesc + off, kdesc + off, idesc_qk, kk > 0 ? 1u : 0u);
          }
          ptx::tc_commit_elect(&s_full[b]);
          ptx::tc_commit_elect(&kv_empty[st]);
          if (k == n - 1) ptx::tc_commit_elect(q_empty);
        }
      } else {
        for (int j = 0; ok && j < n; ++j, ++g) {
          const uint32_t b = g % NSL;
          const uint32_t pos = base + (uint32_t)(m + j + (j < nk3 ? j : nk3));
          const int st = (int)(pos % NS);
          bool w = wait_bar(&p_full[b], (g / NSL) & 1, W);
          w = w && wait_bar(&kv_full[st], (pos / NS) & 1, W);
          if (j == 0) w = w && wait_bar(o_free, (li & 1) ^ 1, W);
          if (!__all_sync(0xffffffffu, w)) { ok = false; break; }
          ptx::tc_fence_after();
          const uint64_t vdesc = mnmajor_desc(ptx::smem_u32(sKV + st * C::TILE));
          const uint32_t tp = tmem + C::COL_S + 64 * b;    // P(g) over the first half of S(g)
          const uint32_t acc0 = j > 0 ? 1u : 0u;
          const int nk = (stage_nv[st] + 15) >> 4;       // K steps of 16 keys over the valid prefix
#pragma unroll 1
          for (int kk = 0; kk < nk; ++kk)
            ptx::mma_ts_elect(tmem + C::COL_O, tp + kk * 8, vdesc + (uint64_t)(kk * (2048 >> 4)), idesc_pv,
                              kk > 0 ? 1u : acc0);
          ptx::tc_commit_elect(&buf_free[b]);
          ptx::tc_commit_elect(&kv_empty[st]);
          if (j == n - 1) ptx::tc_commit_elect(o_full);
        }
      }
      base += 2u * (uint32_t)n;
    }
    // every MMA this warp issued completes before TMEM is released
    ptx::tc_commit_elect(&mma_fin[is_s ? 0 : 1]);
    drain_bar(&mma_fin[is_s ? 0 : 1], 0, 100000000LL);
  }
  } else {
    // ------------------------------------------------ softmax / epilogue --
    ptx::setmaxnreg_inc<C::REG_SOFTMAX>();
    // Group w (warps 4-7: w = 0, warps 8-11: w = 1) takes the item's blocks
    // j with j % 2 == w.  Thread = one query row (TMEM lane), all 128 columns.
    const int w = (warp - 4) >> 2;
    const int quad = warp & 3;
    const int row = quad * 32 + lane;
    const uint32_t lane_base = (uint32_t)(quad * 32) << 16;
    const int gtid = threadIdx.x - 128;                // 0..255 over both groups
    const uint32_t tO = tmem + lane_base + C::COL_O;
    const float sl2 = p.scale_log2;
    const float2 sl2x2 = make_float2(sl2, sl2);
    uint32_t nb_done[2] = {0, 0};                      // blocks of each group before this item
    uint32_t g0 = 0;                                   // key blocks of all previous items
    bool ok = true;
    for (int li = 0; ok; ++li) {
      const int slot = li % kItemRing;
      ok = wait_bar(&item_full[slot], (li / kItemRing) & 1, W);
      if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
      const int it = item_ring[slot];
      ptx::mbar_arrive(&item_empty[slot]);
      if (it < 0) break;
      const Item I = get_item(p, it);
      const int n = I.n;
      // both groups finished the previous item (its row sums were exchanged
      // after their last block), so the codes can be overwritten
      for (int j = gtid; j < n; j += 256) sext[j] = extent_code(p, I, key_block(p, I, j));
      ptx::mbar_arrive(stage_bar);
      ok = wait_bar(stage_bar, li & 1, W);
      if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
      float l = 0.f;          // this group's share of the row sum, relative to m_seen
      float m_seen = 0.f;     // reference max at this group's last block
      for (int j = w; j < n; j += 2) {
        const uint32_t g = g0 + (uint32_t)j;           // the CTA's key-block counter: slot g % NSL
        const uint32_t b = g % NSL;
        const uint32_t tS = tmem + lane_base + C::COL_S + 64 * b;
        ok = wait_bar(&s_full[b], (g / NSL) & 1, W);
        if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
        ptx::tc_fence_after();
        uint32_t sr[128];
        ptx::tmem_ld128(tS, sr);                       // waits for the loads: P may now overwrite S
        ptx::tc_fence_before();
        ptx::mbar_arrive(&s_read[b]);                  // S(g+1) may now overwrite the upper half
        const int nv = (int)(sext[j] & 0xffu);         // valid key columns: a prefix
        if (nv < 128) {
#pragma unroll
          for (int c = 0; c < 128; ++c)
            if (c >= nv) sr[c] = 0xff800000u;            // -inf
        }
        float mk[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) mk[k] = fmaxf(__uint_as_float(sr[k]), __uint_as_float(sr[k + 8]));
#pragma unroll
        for (int c = 16; c < 128; c += 16) {
#pragma unroll
          for (int k = 0; k < 8; ++k)
            mk[k] = max3f(mk[k], __uint_as_float(sr[c + k]), __uint_as_float(sr[c + k + 8]));
        }
        const float mx = max3f(max3f(mk[0], mk[1], mk[2]), max3f(mk[3], mk[4], mk[5]), fmaxf(mk[6], mk[7])) * sl2;
        // reference max: block 0 sets it; block j > 0 reads what block j-1
        // left and raises it only when its own max is more than 2^8 above
        float m_use = mx, alpha = 1.0f;
        bool raise = false;
        if (j > 0) {
          const uint32_t kother = nb_done[w ^ 1] + (uint32_t)((j - 1) >> 1);   // block j-1's index in its group
          ok = wait_bar(&md[w ^ 1], kother & 1, W);
          if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
          const float mprev = mref[row];
          if (mx > mprev + 8.0f) {
            raise = true;
            alpha = ptx::ex2(mprev - mx);
          } else {
            m_use = mprev;
          }
        }
        if (j == 0 || raise) mref[row] = m_use;
        ptx::mbar_arrive(&md[w]);
        if (l != 0.f && m_seen != m_use) l *= ptx::ex2(m_seen - m_use);
        m_seen = m_use;
        // p = 2^(s*scale*log2e - m): FFMA2 over the row, then exp2 (SFU),
        // row-sum FADD2, bf16 pack and TMEM store in four 32-column chunks;
        // masked columns are -inf and give 0 (chunks past a short block's
        // prefix are computed all the same: a branch between chunks costs
        // more than it saves)
        {
          // in place over the score row: x = s * scale * log2(e) - m for all
          // 128 columns (FFMA2), then 2^x chunk by chunk, each chunk's
          // exponentials issued before the previous chunk's sum, bf16 pack
          // and TMEM store, so the SFU always has queued work
          const float2 nm2 = make_float2(-m_use, -m_use);
          float2 acc4[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                            make_float2(0.f, 0.f)};
#pragma unroll
          for (int c = 0; c < 64; ++c) {
            const float2 x = __ffma2_rn(make_float2(__uint_as_float(sr[2 * c]), __uint_as_float(sr[2 * c + 1])),
                                        sl2x2, nm2);
            sr[2 * c] = __float_as_uint(x.x);
            sr[2 * c + 1] = __float_as_uint(x.y);
          }
          auto exp_chunk = [&](int q) {
#pragma unroll
            for (int c = 0; c < 32; ++c) sr[32 * q + c] = __float_as_uint(ptx::ex2(__uint_as_float(sr[32 * q + c])));
          };
          auto finish_chunk = [&](int q) {
            uint32_t pk[16];
#pragma unroll
            for (int c = 0; c < 16; ++c) {
              const float2 pv = make_float2(__uint_as_float(sr[32 * q + 2 * c]), __uint_as_float(sr[32 * q + 2 * c + 1]));
              acc4[c & 3] = __fadd2_rn(acc4[c & 3], pv);
              pk[c] = ptx::pack_bf16x2(pv.x, pv.y);
            }
            ptx::tmem_st16_nowait(tS + 16 * q, pk);
          };
          exp_chunk(0);
          exp_chunk(1);
          finish_chunk(0);
          exp_chunk(2);
          finish_chunk(1);
          exp_chunk(3);
          finish_chunk(2);
          finish_chunk(3);
          const float2 a = __fadd2_rn(__fadd2_rn(acc4[0], acc4[1]), __fadd2_rn(acc4[2], acc4[3]));
          l += a.x + a.y;
        }
        ptx::tmem_wait_st();
        if (__any_sync(0xffffffffu, raise)) {
          // O holds blocks < j relative to the old reference: rescale it once
          // P V(j-1) has landed (P V(j) waits for this group's P below)
          ok = wait_bar(&buf_free[(g - 1) % NSL], ((g - 1) / NSL) & 1, W);
          if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
          ptx::tc_fence_after();
#pragma unroll 1
          for (int c0 = 0; c0 < D; c0 += 32) {
            uint32_t ob[32];
            ptx::tmem_ld32(tO + c0, ob);
#pragma unroll
            for (int c = 0; c < 32; ++c) ob[c] = __float_as_uint(__uint_as_float(ob[c]) * alpha);
            ptx::tmem_st32(tO + c0, ob);
          }
        }
        ptx::tc_fence_before();
        ptx::mbar_arrive(&p_full[b]);
      }
      if (!ok) break;
      // ---- epilogue: combine the groups' row sums, O / l -> bf16 -> token order
      {
        const int jl = n - 1;                          // last block: its reference max is final
        if ((jl & 1) != w) {
          const uint32_t kl = nb_done[w ^ 1] + (uint32_t)(jl >> 1);
          ok = wait_bar(&md[w ^ 1], kl & 1, W);
          if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
        }
        const float mfin = mref[row];
        if (l != 0.f && m_seen != mfin) l *= ptx::ex2(m_seen - mfin);
        lx[w * 128 + row] = l;
        ptx::mbar_arrive(lx_bar);
        ok = wait_bar(lx_bar, li & 1, W);
        if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
        ok = wait_bar(o_full, li & 1, W);
        if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
        ptx::tc_fence_after();
      }
      nb_done[0] += (uint32_t)((n + 1) >> 1);
      nb_done[1] += (uint32_t)(n >> 1);
      g0 += (uint32_t)n;
      const float inv = 1.0f / (lx[row] + lx[128 + row]);
      const Item E = get_item(p, it);   // re-read: nothing of the item stays live across the block loop
      long long tok = -1;
      if (E.qb < E.nb) {
        const Geo& gg = p.geo[E.scheme];
        int t0, y0, x0, et, eh, ew;
        block_box(gg, E.qb, t0, y0, x0, et, eh, ew);
        const uint32_t e = sdec[128 * E.scheme + row];
        const int tl = (int)(e & 0xffu), yl = (int)((e >> 8) & 0xffu), xl = (int)(e >> 16);
        if (tl < et && yl < eh && xl < ew) tok = ((long long)(t0 + tl) * gg.H + (y0 + yl)) * gg.W + (x0 + xl);
      } else {
        const int t = (E.qb - E.nb) * 128 + row;
        if (t < p.text_tokens) tok = (long long)p.N + t;
      }
      constexpr int OH = D / 2;                        // this group's output columns
      uint4* dst = reinterpret_cast<uint4*>(p.out + ((tok < 0 ? 0 : tok) * p.heads + E.h) * (long long)(D * 2) +
                                            OH * 2 * w);
#pragma unroll 1
      for (int c0 = 0; c0 < OH; c0 += 32) {
        uint32_t ov[32];
        ptx::tmem_ld32(tO + OH * w + c0, ov);
        if (tok >= 0) {
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4) {
            const int c = q4 * 8;
            uint4 v4;
            v4.x = ptx::pack_bf16x2(__uint_as_float(ov[c + 0]) * inv, __uint_as_float(ov[c + 1]) * inv);
            v4.y = ptx::pack_bf16x2(__uint_as_float(ov[c + 2]) * inv, __uint_as_float(ov[c + 3]) * inv);
            v4.z = ptx::pack_bf16x2(__uint_as_float(ov[c + 4]) * inv, __uint_as_float(ov[c + 5]) * inv);
            v4.w = ptx::pack_bf16x2(__uint_as_float(ov[c + 6]) * inv, __uint_as_float(ov[c + 7]) * inv);
            dst[c0 / 8 + q4] = v4;
          }
        }
      }
      ptx::tc_fence_before();
      ptx::mbar_arrive(o_free);
    }
  }

  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  if (warp == 1) ptx::tmem_dealloc(tmem, C::TMEM_COLS);
}

// ------------------------------------------------------------------ host --
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

// box = (et, eh, ew) tokens of one head: the block shape, or the clipped
// extents of an edge block
bool map_video(CUtensorMap* m, const void* base, const Geo& g, int heads, int d, int et, int eh, int ew) {
  const cuuint64_t es = 2;
  cuuint64_t dims[5] = {(cuuint64_t)d, (cuuint64_t)heads, (cuuint64_t)g.W, (cuuint64_t)g.H, (cuuint64_t)g.T};
  cuuint64_t strides[4] = {d * es, (cuuint64_t)heads * d * es, (cuuint64_t)g.W * heads * d * es,
                           (cuuint64_t)g.H * g.W * heads * d * es};
  cuuint32_t box[5] = {64, 1, (cuuint32_t)ew, (cuuint32_t)eh, (cuuint32_t)et};
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

template <int D, int NS>
cudaError_t launch_d(const TcParams& tp, int grid, cudaStream_t s) {
  using C = Cfg<D, NS>;
  static_assert(C::SMEM <= 232448, "shared memory budget");
  static_assert(C::REG_POOL_NEEDED <= 65536, "register split");
  cudaError_t e =
      cudaFuncSetAttribute(attn_tc_kernel<D, NS>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
  if (e != cudaSuccess) return e;
  // The warpgroups' register increase waits for room in the block's
  // launch-time pool: never launch a build whose pool is smaller than the split.
  cudaFuncAttributes fa;
  e = cudaFuncGetAttributes(&fa, attn_tc_kernel<D, NS>);
  if (e != cudaSuccess) return e;
  if (fa.numRegs * C::THREADS < C::REG_POOL_NEEDED) return cudaErrorNotSupported;
  attn_tc_kernel<D, NS><<<grid, C::THREADS, C::SMEM, s>>>(tp);
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
  // host staging (large), one per calling thread: the launch copies it into
  // the kernel's parameter buffer, so concurrent callers never share it
  thread_local TcParams tp;
  if (!encode_fn()) { *why = "cuTensorMapEncodeTiled unavailable"; return cudaErrorNotSupported; }
  memset(&tp, 0, sizeof(tp));
  const int es = 2;
  for (int sc = 0; sc < a.n_schemes; ++sc) {
    const Geo& g = a.geo[sc];
    bool ok = map_video(&tp.tm_q[sc], a.q, g, a.heads, a.d, g.bt, g.bh, g.bw);
    // key/value maps per edge case (cases the grid does not have repeat the full box)
    const int lt = g.T - (g.nbt - 1) * g.bt, lh = g.H - (g.nbh - 1) * g.bh, lw = g.W - (g.nbw - 1) * g.bw;
    for (int c = 0; ok && c < kEdgeCases; ++c) {
      const int et = (c & 1) ? lt : g.bt, eh = (c & 2) ? lh : g.bh, ew = (c & 4) ? lw : g.bw;
      ok = map_video(&tp.tm_k[sc][c], a.k, g, a.heads, a.d, et, eh, ew) &&
           map_video(&tp.tm_v[sc][c], a.v, g, a.heads, a.d, et, eh, ew);
    }
    if (!ok) {
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
  if (a.d == 64) return launch_d<64, 8>(tp, grid, s);
  return launch_d<128, 5>(tp, grid, s);
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
