// C ABI of the SPADE executor hot path (declared in include/spade.h):
// argument validation, workspace layout, and the order of launches for the
// single steps and for the grouped (mixed-scheme) layer.
#include <algorithm>
#include <atomic>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <string>
#include <vector>

#include "spade_internal.cuh"
#include "spade_selftest.h"

// Latched device status (SPADE_OK / SPADE_ERR_TIMEOUT), one per device.
__device__ int g_spade_status;

// Fixed scratch for spade_block_sparse_attn_noalloc: the cost-ranked work list
// (up to SPADE_NOALLOC_MAX_ITEMS entries) followed by the work-hand-out ticket.
// Lives for as long as the library is loaded, on every device that uses it.
#define SPADE_NOALLOC_MAX_ITEMS 65536
static __device__ __align__(256) int g_noalloc_scratch[SPADE_NOALLOC_MAX_ITEMS + 64];

namespace spade {

namespace {

thread_local std::string g_err;

spade_status fail(spade_status s, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_err = buf;
  return s;
}

spade_status cuda_fail(cudaError_t e, const char* where) {
  return fail(SPADE_ERR_CUDA, "%s: %s", where, cudaGetErrorString(e));
}

constexpr int kMaxDevices = 64;

int current_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return -1;
  return dev;
}

// Per-device caches below are atomics: callers on several host threads may
// fill the same slot at once (with the same value).
int* status_ptr() {
  static std::atomic<int*> ptrs[kMaxDevices];
  const int dev = current_device();
  if (dev < 0 || dev >= kMaxDevices) return nullptr;
  int* p = ptrs[dev].load(std::memory_order_acquire);
  if (!p) {
    void* a = nullptr;
    if (cudaGetSymbolAddress(&a, g_spade_status) != cudaSuccess) return nullptr;
    p = static_cast<int*>(a);
    ptrs[dev].store(p, std::memory_order_release);
  }
  return p;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

spade_status check_geom(const spade_geom& g) {
  if (g.T <= 0 || g.H <= 0 || g.W <= 0 || g.bt <= 0 || g.bh <= 0 || g.bw <= 0)
    return fail(SPADE_ERR_INVALID, "geometry has a non-positive extent");
  if (g.bt > 256 || g.bh > 256 || g.bw > 256) return fail(SPADE_ERR_UNSUPPORTED, "block extent above 256");
  const long long bs = (long long)g.bt * g.bh * g.bw;
  if (bs > 1024) return fail(SPADE_ERR_UNSUPPORTED, "block size %lld above 1024", bs);
  const Geo gg = make_geo(g);
  if (gg.nb > 65535) return fail(SPADE_ERR_UNSUPPORTED, "more than 65535 blocks");
  return SPADE_OK;
}

spade_status check_d_dt(int d, spade_dtype dt) {
  if (d != 64 && d != 128) return fail(SPADE_ERR_UNSUPPORTED, "d=%d (supported: 64, 128)", d);
  if (dt != SPADE_F32 && dt != SPADE_BF16) return fail(SPADE_ERR_INVALID, "unknown dtype %d", (int)dt);
  return SPADE_OK;
}

cudaStream_t as_cuda(spade_stream_t s) { return reinterpret_cast<cudaStream_t>(s); }

// Layout of the grouped workspace (byte offsets).
struct GroupLayout {
  int n_sparse[SPADE_MAX_SCHEMES];
  std::vector<int> heads_of[SPADE_MAX_SCHEMES];   // sparse heads per scheme, ascending
  size_t qmean[SPADE_MAX_SCHEMES], kmean[SPADE_MAX_SCHEMES], prob[SPADE_MAX_SCHEMES];
  size_t cnt[SPADE_MAX_SCHEMES], idx[SPADE_MAX_SCHEMES];
  std::vector<int> pos;                             // position of head h in its scheme group
  size_t work;
  size_t ticket;
  int n_items;
  size_t total;
};

spade_status plan_group(const spade_geom* schemes, int n_schemes, const spade_head_scheme* table, int heads,
                        int d, int text_tokens, GroupLayout& L) {
  if (!schemes || !table) return fail(SPADE_ERR_INVALID, "null scheme table");
  if (n_schemes < 1 || n_schemes > SPADE_MAX_SCHEMES)
    return fail(SPADE_ERR_UNSUPPORTED, "n_schemes=%d (1..%d)", n_schemes, SPADE_MAX_SCHEMES);
  if (heads < 1 || heads > SPADE_MAX_HEADS) return fail(SPADE_ERR_UNSUPPORTED, "heads=%d (1..128)", heads);
  if (text_tokens < 0) return fail(SPADE_ERR_INVALID, "negative text_tokens");
  if (d != 64 && d != 128) return fail(SPADE_ERR_UNSUPPORTED, "d=%d (supported: 64, 128)", d);
  const long long N = (long long)schemes[0].T * schemes[0].H * schemes[0].W;
  for (int s = 0; s < n_schemes; ++s) {
    spade_status st = check_geom(schemes[s]);
    if (st != SPADE_OK) return st;
    if ((long long)schemes[s].T * schemes[s].H * schemes[s].W != N)
      return fail(SPADE_ERR_INVALID, "scheme %d covers a different number of tokens", s);
  }
  L.pos.assign(heads, -1);
  for (int s = 0; s < n_schemes; ++s) { L.n_sparse[s] = 0; L.heads_of[s].clear(); }
  for (int h = 0; h < heads; ++h) {
    const spade_head_scheme& r = table[h];
    if (r.scheme < 0 || r.scheme >= n_schemes) return fail(SPADE_ERR_INVALID, "head %d: scheme %d", h, r.scheme);
    if (r.dense != 0 && r.dense != 1) return fail(SPADE_ERR_INVALID, "head %d: dense flag %d", h, r.dense);
    if (!r.dense && !(r.tau > 0.f && r.tau <= 1e30f)) return fail(SPADE_ERR_INVALID, "head %d: tau", h);
    if (!r.dense) {
      L.pos[h] = L.n_sparse[r.scheme]++;
      L.heads_of[r.scheme].push_back(h);
    }
  }
  size_t off = 0;
  const int ntb = text_blocks(text_tokens);
  L.n_items = 0;
  for (int h = 0; h < heads; ++h) L.n_items += make_geo(schemes[table[h].scheme]).nb + ntb;
  for (int s = 0; s < n_schemes; ++s) {
    const Geo g = make_geo(schemes[s]);
    const size_t hs = L.n_sparse[s];
    if (hs > 0) {
      if (g.nb > SPADE_SELECT_MAX_NB) return fail(SPADE_ERR_UNSUPPORTED, "scheme %d: nb=%d above 1024", s, g.nb);
    }
    L.qmean[s] = off; off = align256(off + hs * g.nb * d * sizeof(float));
    L.kmean[s] = off; off = align256(off + hs * g.nb * d * sizeof(float));
    L.prob[s] = off;  off = align256(off + hs * g.nb * g.nb * sizeof(float));
    L.cnt[s] = off;   off = align256(off + hs * g.nb * sizeof(int));
    L.idx[s] = off;   off = align256(off + hs * g.nb * g.nb * sizeof(int));
  }
  L.work = off;
  off = align256(off + (size_t)L.n_items * sizeof(int));
  L.ticket = off;
  off = align256(off + sizeof(int));
  L.total = off;
  return SPADE_OK;
}

// Step 3: the tensor-core estimator (split-precision TF32); the FMA-pipe
// kernel only when the tensor-map encoder is unavailable.  want_probs = false
// asks for the scaled pooled scores (the index search then forms the
// softmax); *holds_scores says which of the two `out` received (the FMA-pipe
// kernel always writes probabilities).
cudaError_t run_estimate(const float* qm, const float* km, float* out, int heads, int nb, int d, int* status,
                         bool want_probs, bool* holds_scores, cudaStream_t s) {
  cudaError_t e = launch_estimate_tc(qm, km, out, heads, nb, d, status, want_probs, s);
  *holds_scores = !want_probs;
  if (e == cudaErrorNotSupported) {
    cudaGetLastError();
    e = launch_estimate(qm, km, out, heads, nb, d, s);
    *holds_scores = false;
  }
  return e;
}

// Host checks of an attention launch that do not depend on pointers; every
// entry point runs them before it enqueues anything.  A work item is packed
// as (head << 16) | query block, so a head's query blocks (video blocks plus
// text blocks) must number at most 65536; the CUDA-core kernel (taken when
// the tensor-core kernel does not support the shape) holds at most 128 slots
// per block.
spade_status check_attention(const AttnArgs& a) {
  const int ntb = text_blocks(a.text_tokens);
  for (int h = 0; h < a.heads; ++h)
    if ((long long)a.head[h].nb + ntb > 65536)
      return fail(SPADE_ERR_UNSUPPORTED, "head %d: %d blocks + %d text blocks exceed 65536 query blocks", h,
                  a.head[h].nb, ntb);
  if (!attn_tc_supported(a))
    for (int sc = 0; sc < a.n_schemes; ++sc)
      if (a.geo[sc].bs > 128) return fail(SPADE_ERR_UNSUPPORTED, "CUDA-core attention needs blocks <= 128 slots");
  return SPADE_OK;
}

// Enqueues the work list and the attention launch (check_attention has passed).
spade_status run_attention(AttnArgs& a, cudaStream_t s) {
  a.status = status_ptr();
  if (!a.status) return fail(SPADE_ERR_CUDA, "device status word unavailable");
  const bool tc = attn_tc_supported(a);
  cudaError_t e = launch_worklist(a, s);
  if (e != cudaSuccess) return cuda_fail(e, "work list");
  if (tc) {
    const char* why = "";
    e = launch_attn_tc(a, s, &why);
    if (e != cudaSuccess) return fail(SPADE_ERR_CUDA, "tensor-core attention: %s (%s)", cudaGetErrorString(e), why);
  } else {
    e = launch_attn_simt(a, s);
    if (e != cudaSuccess) return cuda_fail(e, "CUDA-core attention");
  }
  return SPADE_OK;
}

// The attention launch of a grouped layer: every head of the table, kept
// lists of the sparse heads read from their places in the grouped workspace.
void grouped_attn_args(const void* q, const void* k, const void* v, void* out, const spade_geom* schemes,
                       int n_schemes, const spade_head_scheme* table, int heads, int d, int text_tokens,
                       spade_dtype dt, const GroupLayout& L, uint8_t* ws, AttnArgs& a) {
  memset(&a, 0, sizeof(a));
  a.q = q; a.k = k; a.v = v; a.out = out;
  a.n_schemes = n_schemes;
  for (int sc = 0; sc < n_schemes; ++sc) a.geo[sc] = make_geo(schemes[sc]);
  a.heads = heads; a.d = d; a.text_tokens = text_tokens; a.N = schemes[0].T * schemes[0].H * schemes[0].W;
  a.dt = dt;
  for (int h = 0; h < heads; ++h) {
    const int sc = table[h].scheme;
    const Geo& g = a.geo[sc];
    a.head[h].scheme = sc;
    a.head[h].nb = g.nb;
    a.head[h].dense = table[h].dense;
    if (!table[h].dense) {
      a.head[h].cnt_off = (int)((L.cnt[sc] + (size_t)L.pos[h] * g.nb * sizeof(int)) / sizeof(int));
      a.head[h].idx_off = (long long)((L.idx[sc] + (size_t)L.pos[h] * g.nb * g.nb * sizeof(int)) / sizeof(int));
    }
  }
  a.cnt = reinterpret_cast<const int*>(ws);
  a.idx = reinterpret_cast<const int*>(ws);
  a.work = reinterpret_cast<int*>(ws + L.work);
  a.ticket = reinterpret_cast<int*>(ws + L.ticket);
  a.n_items = L.n_items;
}

// Device address of g_noalloc_scratch on the current device.  The name is only
// a host-side stand-in in host code, so the address is looked up once per
// device (with that device current) and cached.
int* noalloc_scratch(spade_status* st) {
  static std::atomic<int*> ptrs[kMaxDevices];
  const int dev = current_device();
  if (dev < 0 || dev >= kMaxDevices) {
    *st = fail(SPADE_ERR_CUDA, "no current CUDA device");
    return nullptr;
  }
  int* p = ptrs[dev].load(std::memory_order_acquire);
  if (!p) {
    void* a = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&a, g_noalloc_scratch);
    if (e != cudaSuccess) {
      *st = cuda_fail(e, "fixed scratch address");
      return nullptr;
    }
    p = static_cast<int*>(a);
    ptrs[dev].store(p, std::memory_order_release);
  }
  return p;
}

// ---- host-to-host pipelined layer (spade_grouped_attn_host) ----
constexpr int kHostSlots = 3;        // device group slots in flight
constexpr int kHostComputes = 2;     // compute streams the groups alternate over

// Layout of the caller's workspace for the host-to-host call.
struct HostLayout {
  int heads, head_chunk, n_groups, hc_max;
  size_t slot_bytes;       // one of Q, K, V, O for the largest group
  size_t ws_off;           // first grouped workspace
  size_t ws_bytes;         // each grouped workspace
  size_t total;
};

spade_status plan_host(const spade_geom* schemes, int n_schemes, const spade_head_scheme* table, int heads, int d,
                       int text_tokens, spade_dtype dt, int head_chunk, HostLayout& H) {
  GroupLayout L;
  spade_status st = plan_group(schemes, n_schemes, table, heads, d, text_tokens, L);   // the whole table
  if (st != SPADE_OK) return st;
  if ((st = check_d_dt(d, dt)) != SPADE_OK) return st;
  if (head_chunk < 1 || head_chunk > heads) return fail(SPADE_ERR_INVALID, "head_chunk=%d (1..%d)", head_chunk, heads);
  H.heads = heads;
  H.head_chunk = head_chunk;
  H.n_groups = (heads + head_chunk - 1) / head_chunk;
  H.hc_max = head_chunk;
  const size_t rows = (size_t)schemes[0].T * schemes[0].H * schemes[0].W + (size_t)text_tokens;
  const size_t esz = dt == SPADE_BF16 ? 2 : 4;
  H.slot_bytes = align256(rows * (size_t)H.hc_max * d * esz);
  H.ws_bytes = 0;
  for (int g = 0; g < H.n_groups; ++g) {
    const int h0 = g * head_chunk, hc = std::min(head_chunk, heads - h0);
    GroupLayout Lg;
    if ((st = plan_group(schemes, n_schemes, table + h0, hc, d, text_tokens, Lg)) != SPADE_OK) return st;
    H.ws_bytes = std::max(H.ws_bytes, Lg.total);
  }
  H.ws_bytes = align256(H.ws_bytes);
  const int ns = std::min(kHostSlots, H.n_groups);
  H.ws_off = (size_t)ns * 4 * H.slot_bytes;
  H.total = H.ws_off + (size_t)kHostComputes * H.ws_bytes;
  return SPADE_OK;
}

// Streams and events of the host-to-host call, created once per device.
struct HostPipe {
  std::mutex mu;                    // one call enqueues at a time
  bool ready = false;
  cudaStream_t up = nullptr, down = nullptr, comp[kHostComputes] = {nullptr, nullptr};
  std::vector<cudaEvent_t> ev;      // 3 per group (loaded, done, returned) + joins
};

HostPipe& host_pipe(int dev) {
  static HostPipe pipes[kMaxDevices];
  return pipes[dev];
}

// Creates the streams, and enough events for n_events (caller holds P.mu).
cudaError_t host_pipe_setup(HostPipe& P, size_t n_events) {
  cudaError_t e = cudaSuccess;
  if (!P.ready) {
    e = cudaStreamCreateWithFlags(&P.up, cudaStreamNonBlocking);
    if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&P.down, cudaStreamNonBlocking);
    for (int c = 0; e == cudaSuccess && c < kHostComputes; ++c)
      e = cudaStreamCreateWithFlags(&P.comp[c], cudaStreamNonBlocking);
    if (e != cudaSuccess) return e;
    P.ready = true;
  }
  while (P.ev.size() < n_events) {
    cudaEvent_t ev;
    if ((e = cudaEventCreateWithFlags(&ev, cudaEventDisableTiming)) != cudaSuccess) return e;
    P.ev.push_back(ev);
  }
  return cudaSuccess;
}

}  // namespace

int num_sms() {
  static std::atomic<int> sms[kMaxDevices];
  const int dev = current_device();
  if (dev < 0 || dev >= kMaxDevices) return 1;
  int v = sms[dev].load(std::memory_order_relaxed);
  if (!v) {
    cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev);
    if (v <= 0) v = 1;
    sms[dev].store(v, std::memory_order_relaxed);
  }
  return v;
}

long long device_wait_timeout_ns() {
  static const long long ns = [] {
    const char* e = getenv("SPADE_WAIT_TIMEOUT_MS");
    long long ms = e ? atoll(e) : 10000;
    if (ms <= 0) ms = 10000;
    return ms * 1000000LL;
  }();
  return ns;
}

}  // namespace spade

using namespace spade;

extern "C" {

int spade_version(void) { return 1; }

const char* spade_status_string(spade_status s) {
  switch (s) {
    case SPADE_OK: return "ok";
    case SPADE_ERR_INVALID: return "invalid argument";
    case SPADE_ERR_UNSUPPORTED: return "unsupported configuration";
    case SPADE_ERR_CUDA: return "CUDA error";
    case SPADE_ERR_TIMEOUT: return "device wait timed out";
    case SPADE_ERR_WORKSPACE: return "workspace missing or too small";
  }
  return "unknown status";
}

const char* spade_last_error_message(void) { return g_err.c_str(); }

spade_status spade_tile3d(const void* x, void* xt, spade_geom g, int heads, int d, spade_dtype dt,
                          spade_stream_t stream) {
  spade_status st = check_geom(g);
  if (st != SPADE_OK) return st;
  if ((st = check_d_dt(d, dt)) != SPADE_OK) return st;
  if (!x || !xt) return fail(SPADE_ERR_INVALID, "null pointer");
  if (!aligned16(x) || !aligned16(xt)) return fail(SPADE_ERR_INVALID, "pointers must be 16-byte aligned");
  if (heads < 1) return fail(SPADE_ERR_INVALID, "heads=%d", heads);
  cudaError_t e = launch_tile3d(x, xt, make_geo(g), heads, d, dt, as_cuda(stream));
  return e == cudaSuccess ? SPADE_OK : cuda_fail(e, "tile3d");
}

spade_status spade_summarize(const void* x, float* xmean, spade_geom g, int heads, int d, spade_dtype dt,
                             spade_stream_t stream) {
  spade_status st = check_geom(g);
  if (st != SPADE_OK) return st;
  if ((st = check_d_dt(d, dt)) != SPADE_OK) return st;
  if (!x || !xmean) return fail(SPADE_ERR_INVALID, "null pointer");
  if (!aligned16(x) || !aligned16(xmean)) return fail(SPADE_ERR_INVALID, "pointers must be 16-byte aligned");
  if (heads < 1) return fail(SPADE_ERR_INVALID, "heads=%d", heads);
  cudaError_t e = launch_summarize(x, xmean, make_geo(g), heads, 0, heads, d, dt, 0, as_cuda(stream));
  return e == cudaSuccess ? SPADE_OK : cuda_fail(e, "summarize");
}

spade_status spade_summarize_mode(const void* x, float* out, spade_geom g, int heads, int d, spade_dtype dt,
                                  spade_summary mode, spade_stream_t stream) {
  if (mode != SPADE_SUM_MEAN && mode != SPADE_SUM_MAX && mode != SPADE_SUM_MIN)
    return fail(SPADE_ERR_INVALID, "summary mode %d", (int)mode);
  if (mode == SPADE_SUM_MEAN) return spade_summarize(x, out, g, heads, d, dt, stream);
  spade_status st = check_geom(g);
  if (st != SPADE_OK) return st;
  if ((st = check_d_dt(d, dt)) != SPADE_OK) return st;
  if (!x || !out) return fail(SPADE_ERR_INVALID, "null pointer");
  if (!aligned16(x) || !aligned16(out)) return fail(SPADE_ERR_INVALID, "pointers must be 16-byte aligned");
  if (heads < 1) return fail(SPADE_ERR_INVALID, "heads=%d", heads);
  cudaError_t e = launch_summarize(x, out, make_geo(g), heads, 0, heads, d, dt, (int)mode, as_cuda(stream));
  return e == cudaSuccess ? SPADE_OK : cuda_fail(e, "summarize");
}

spade_status spade_summarize_qk(const void* q, const void* k, float* qmean, float* kmean, spade_geom g, int heads,
                                int d, spade_dtype dt, spade_stream_t stream) {
  spade_status st = check_geom(g);
  if (st != SPADE_OK) return st;
  if ((st = check_d_dt(d, dt)) != SPADE_OK) return st;
  if (!q || !k || !qmean || !kmean) return fail(SPADE_ERR_INVALID, "null pointer");
  if (!aligned16(q) || !aligned16(k) || !aligned16(qmean) || !aligned16(kmean))
    return fail(SPADE_ERR_INVALID, "pointers must be 16-byte aligned");
  if (heads < 1) return fail(SPADE_ERR_INVALID, "heads=%d", heads);
  cudaError_t e = launch_summarize_pair(q, k, qmean, kmean, make_geo(g), heads, 0, heads, d, dt, 0, as_cuda(stream));
  return e == cudaSuccess ? SPADE_OK : cuda_fail(e, "summarize");
}

static spade_status check_estimate_args(const float* qmean, const float* kmean, const float* out, int heads, int nb,
                                       int d) {
  if (!qmean || !kmean || !out) return fail(SPADE_ERR_INVALID, "null pointer");
  if (!aligned16(qmean) || !aligned16(kmean) || !aligned16(out))
    return fail(SPADE_ERR_INVALID, "pointers must be 16-byte aligned");
  if (heads < 1 || heads > 65535) return fail(SPADE_ERR_INVALID, "heads=%d", heads);
  if (nb < 1) return fail(SPADE_ERR_INVALID, "nb=%d", nb);
  if (nb > SPADE_ESTIMATE_MAX_NB) return fail(SPADE_ERR_UNSUPPORTED, "nb=%d above %d", nb, SPADE_ESTIMATE_MAX_NB);
  if (d != 64 && d != 128) return fail(SPADE_ERR_UNSUPPORTED, "d=%d (supported: 64, 128)", d);
  return SPADE_OK;
}

spade_status spade_estimate(const float* qmean, const float* kmean, float* prob, int heads, int nb, int d,
                            spade_stream_t stream) {
  spade_status st0 = check_estimate_args(qmean, kmean, prob, heads, nb, d);
  if (st0 != SPADE_OK) return st0;
  int* st = status_ptr();
  if (!st) return fail(SPADE_ERR_CUDA, "device status word unavailable");
  bool scores = false;
  cudaError_t e = run_estimate(qmean, kmean, prob, heads, nb, d, st, true, &scores, as_cuda(stream));
  return e == cudaSuccess ? SPADE_OK : cuda_fail(e, "estimate");
}

spade_status spade_estimate_scores(const float* qmean, const float* kmean, float* scores, int heads, int nb, int d,
                                   spade_stream_t stream) {
  spade_status st0 = check_estimate_args(qmean, kmean, scores, heads, nb, d);
  if (st0 != SPADE_OK) return st0;
  int* st = status_ptr();
  if (!st) return fail(SPADE_ERR_CUDA, "device status word unavailable");
  cudaError_t e = launch_estimate_tc(qmean, kmean, scores, heads, nb, d, st, false, as_cuda(stream));
  if (e == cudaErrorNotSupported) {
    cudaGetLastError();
    return fail(SPADE_ERR_UNSUPPORTED, "tensor-map encoder unavailable: no score-only estimator");
  }
  return e == cudaSuccess ? SPADE_OK : cuda_fail(e, "estimate scores");
}

static spade_status check_select_args(const float* in, const float* tau_host, const int* cnt, const int* idx,
                                     int heads, int nb) {
  if (!in || !tau_host || !cnt || !idx) return fail(SPADE_ERR_INVALID, "null pointer");
  if (heads < 1 || heads > SPADE_SELECT_MAX_HEADS) return fail(SPADE_ERR_UNSUPPORTED, "heads=%d (1..1024)", heads);
  if (nb < 1) return fail(SPADE_ERR_INVALID, "nb=%d", nb);
  if (nb > SPADE_SELECT_MAX_NB) return fail(SPADE_ERR_UNSUPPORTED, "nb=%d above %d", nb, SPADE_SELECT_MAX_NB);
  for (int h = 0; h < heads; ++h)
    if (!(tau_host[h] > 0.f && tau_host[h] <= 1e30f)) return fail(SPADE_ERR_INVALID, "tau[%d] must be > 0", h);
  return SPADE_OK;
}

spade_status spade_select(const float* prob, const float* tau_host, int* cnt, int* idx, int heads, int nb,
                          spade_stream_t stream) {
  spade_status st = check_select_args(prob, tau_host, cnt, idx, heads, nb);
  if (st != SPADE_OK) return st;
  cudaError_t e = launch_select(prob, tau_host, cnt, idx, heads, nb, as_cuda(stream));
  return e == cudaSuccess ? SPADE_OK : cuda_fail(e, "select");
}

spade_status spade_select_scores(const float* scores, const float* tau_host, int* cnt, int* idx, int heads, int nb,
                                 spade_stream_t stream) {
  spade_status st = check_select_args(scores, tau_host, cnt, idx, heads, nb);
  if (st != SPADE_OK) return st;
  cudaError_t e = launch_select(scores, tau_host, cnt, idx, heads, nb, as_cuda(stream), nullptr, nullptr, true);
  return e == cudaSuccess ? SPADE_OK : cuda_fail(e, "select scores");
}

spade_status spade_select_window(const float* prob, const float* tau_host, const int* radius_host, spade_geom g,
                                 int* cnt, int* idx, int heads, spade_stream_t stream) {
  spade_status st = check_geom(g);
  if (st != SPADE_OK) return st;
  if (!prob || !tau_host || !radius_host || !cnt || !idx) return fail(SPADE_ERR_INVALID, "null pointer");
  if (heads < 1 || heads > SPADE_SELECT_MAX_HEADS) return fail(SPADE_ERR_UNSUPPORTED, "heads=%d (1..1024)", heads);
  const Geo gg = make_geo(g);
  if (gg.nb > SPADE_SELECT_MAX_NB) return fail(SPADE_ERR_UNSUPPORTED, "nb=%d above %d", gg.nb, SPADE_SELECT_MAX_NB);
  for (int h = 0; h < heads; ++h) {
    if (!(tau_host[h] > 0.f && tau_host[h] <= 1e30f)) return fail(SPADE_ERR_INVALID, "tau[%d] must be > 0", h);
    for (int a = 0; a < 3; ++a)
      if (radius_host[3 * h + a] < 0) return fail(SPADE_ERR_INVALID, "window radius of head %d is negative", h);
  }
  cudaError_t e = launch_select(prob, tau_host, cnt, idx, heads, gg.nb, as_cuda(stream), radius_host, &gg);
  return e == cudaSuccess ? SPADE_OK : cuda_fail(e, "select");
}

size_t spade_attn_workspace_bytes(spade_geom g, int heads, int d, int text_tokens) {
  (void)d;
  if (heads < 1 || text_tokens < 0 || g.bt <= 0 || g.bh <= 0 || g.bw <= 0 || g.T <= 0 || g.H <= 0 || g.W <= 0)
    return 0;
  const Geo gg = make_geo(g);
  return align256((size_t)heads * (gg.nb + text_blocks(text_tokens)) * sizeof(int)) + 256;   // + ticket
}

spade_status spade_block_sparse_attn(const void* q, const void* k, const void* v, void* out, const int* cnt,
                                     const int* idx, spade_geom g, int heads, int d, int text_tokens,
                                     spade_dtype dt, void* workspace, size_t ws_bytes, spade_stream_t stream) {
  spade_status st = check_geom(g);
  if (st != SPADE_OK) return st;
  if ((st = check_d_dt(d, dt)) != SPADE_OK) return st;
  if (!q || !k || !v || !out) return fail(SPADE_ERR_INVALID, "null tensor pointer");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out))
    return fail(SPADE_ERR_INVALID, "pointers must be 16-byte aligned");
  if ((cnt == nullptr) != (idx == nullptr)) return fail(SPADE_ERR_INVALID, "cnt and idx must both be set or both NULL");
  if (heads < 1 || heads > SPADE_MAX_HEADS) return fail(SPADE_ERR_UNSUPPORTED, "heads=%d (1..128)", heads);
  if (text_tokens < 0) return fail(SPADE_ERR_INVALID, "negative text_tokens");
  const size_t need = spade_attn_workspace_bytes(g, heads, d, text_tokens);
  if (!workspace || ws_bytes < need) return fail(SPADE_ERR_WORKSPACE, "workspace needs %zu bytes", need);
  AttnArgs a;
  memset(&a, 0, sizeof(a));
  a.q = q; a.k = k; a.v = v; a.out = out;
  a.n_schemes = 1;
  a.geo[0] = make_geo(g);
  a.heads = heads; a.d = d; a.text_tokens = text_tokens; a.N = g.T * g.H * g.W; a.dt = dt;
  const int nb = a.geo[0].nb;
  for (int h = 0; h < heads; ++h) {
    a.head[h].scheme = 0;
    a.head[h].nb = nb;
    a.head[h].dense = cnt == nullptr;
    a.head[h].cnt_off = h * nb;
    a.head[h].idx_off = (long long)h * nb * nb;
  }
  a.cnt = cnt; a.idx = idx;
  a.work = static_cast<int*>(workspace);
  a.n_items = heads * (nb + text_blocks(text_tokens));
  a.ticket = reinterpret_cast<int*>(static_cast<uint8_t*>(workspace) + need - 256);
  if ((st = check_attention(a)) != SPADE_OK) return st;
  return run_attention(a, as_cuda(stream));
}

spade_status spade_block_sparse_attn_noalloc(const void* q, const void* k, const void* v, void* out,
                                             const int* cnt, const int* idx, spade_geom g, int heads, int d,
                                             int text_tokens, spade_dtype dt, spade_stream_t stream) {
  spade_status st = check_geom(g);
  if (st != SPADE_OK) return st;
  if ((st = check_d_dt(d, dt)) != SPADE_OK) return st;
  if (!q || !k || !v || !out) return fail(SPADE_ERR_INVALID, "null tensor pointer");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out))
    return fail(SPADE_ERR_INVALID, "pointers must be 16-byte aligned");
  if ((cnt == nullptr) != (idx == nullptr)) return fail(SPADE_ERR_INVALID, "cnt and idx must both be set or both NULL");
  if (heads < 1 || heads > SPADE_MAX_HEADS) return fail(SPADE_ERR_UNSUPPORTED, "heads=%d (1..128)", heads);
  if (text_tokens < 0) return fail(SPADE_ERR_INVALID, "negative text_tokens");
  const int nb = make_geo(g).nb;
  const long long n_items = (long long)heads * (nb + text_blocks(text_tokens));
  if (n_items > SPADE_NOALLOC_MAX_ITEMS)
    return fail(SPADE_ERR_UNSUPPORTED, "heads * (blocks + text blocks) = %lld exceeds the fixed scratch of %d work items",
                n_items, SPADE_NOALLOC_MAX_ITEMS);
  AttnArgs a;
  memset(&a, 0, sizeof(a));
  a.q = q; a.k = k; a.v = v; a.out = out;
  a.n_schemes = 1;
  a.geo[0] = make_geo(g);
  a.heads = heads; a.d = d; a.text_tokens = text_tokens; a.N = g.T * g.H * g.W; a.dt = dt;
  for (int h = 0; h < heads; ++h) {
    a.head[h].scheme = 0;
    a.head[h].nb = nb;
    a.head[h].dense = cnt == nullptr;
    a.head[h].cnt_off = h * nb;
    a.head[h].idx_off = (long long)h * nb * nb;
  }
  a.cnt = cnt; a.idx = idx;
  a.n_items = (int)n_items;
  if ((st = check_attention(a)) != SPADE_OK) return st;
  int* scratch = noalloc_scratch(&st);
  if (!scratch) return st;
  a.work = scratch;                                   // written in full by the work-list kernel
  a.ticket = scratch + SPADE_NOALLOC_MAX_ITEMS;       // reset to 0 by the work-list kernel
  return run_attention(a, as_cuda(stream));
}

size_t spade_grouped_workspace_bytes(const spade_geom* schemes, int n_schemes, const spade_head_scheme* table,
                                     int heads, int d, int text_tokens) {
  GroupLayout L;
  if (plan_group(schemes, n_schemes, table, heads, d, text_tokens, L) != SPADE_OK) return 0;
  return L.total;
}

spade_status spade_copy_head_slice(void* device, void* host, int64_t rows, int heads_total, int h0, int hc, int d,
                                   spade_dtype dt, int to_device, spade_stream_t stream) {
  if (!device || !host) return fail(SPADE_ERR_INVALID, "null pointer");
  if (rows < 1 || heads_total < 1 || d < 1 || h0 < 0 || hc < 1 || h0 + hc > heads_total)
    return fail(SPADE_ERR_INVALID, "slice [%d, %d) of %d heads, %lld rows", h0, h0 + hc, heads_total, (long long)rows);
  if (dt != SPADE_F32 && dt != SPADE_BF16) return fail(SPADE_ERR_INVALID, "unknown dtype %d", (int)dt);
  const size_t esz = dt == SPADE_BF16 ? 2 : 4;
  const size_t hpitch = (size_t)heads_total * d * esz, dpitch = (size_t)hc * d * esz;
  char* hp = static_cast<char*>(host) + (size_t)h0 * d * esz;
  cudaError_t e = to_device
                      ? cudaMemcpy2DAsync(device, dpitch, hp, hpitch, dpitch, (size_t)rows, cudaMemcpyHostToDevice,
                                          as_cuda(stream))
                      : cudaMemcpy2DAsync(hp, hpitch, device, dpitch, dpitch, (size_t)rows, cudaMemcpyDeviceToHost,
                                          as_cuda(stream));
  return e == cudaSuccess ? SPADE_OK : cuda_fail(e, "copy_head_slice");
}

size_t spade_sics_workspace_bytes(const spade_geom* candidates, int n_candidates, int heads) {
  if (!candidates || n_candidates < 1 || n_candidates > SPADE_MAX_SCHEMES || heads < 1) return 0;
  Geo g[SPADE_MAX_SCHEMES];
  for (int c = 0; c < n_candidates; ++c) g[c] = make_geo(candidates[c]);
  return sics_workspace_floats(g, n_candidates, heads) * sizeof(float);
}

spade_status spade_sics(const void* q, const void* k, const spade_geom* candidates, int n_candidates, int heads,
                        int d, spade_dtype dt, float* scores, int* choice, void* workspace, size_t ws_bytes,
                        spade_stream_t stream) {
  if (!q || !k || !candidates || !scores || !choice || !workspace) return fail(SPADE_ERR_INVALID, "null pointer");
  if (!aligned16(q) || !aligned16(k) || !aligned16(workspace))
    return fail(SPADE_ERR_INVALID, "pointers must be 16-byte aligned");
  if (n_candidates < 1 || n_candidates > SPADE_MAX_SCHEMES)
    return fail(SPADE_ERR_INVALID, "n_candidates=%d (1..%d)", n_candidates, SPADE_MAX_SCHEMES);
  if (heads < 1 || heads > 1024) return fail(SPADE_ERR_INVALID, "heads=%d", heads);
  spade_status st = check_d_dt(d, dt);
  if (st != SPADE_OK) return st;
  Geo g[SPADE_MAX_SCHEMES];
  for (int c = 0; c < n_candidates; ++c) {
    if ((st = check_geom(candidates[c])) != SPADE_OK) return st;
    if ((long long)candidates[c].T * candidates[c].H * candidates[c].W !=
        (long long)candidates[0].T * candidates[0].H * candidates[0].W)
      return fail(SPADE_ERR_INVALID, "candidate %d covers a different number of tokens", c);
    g[c] = make_geo(candidates[c]);
  }
  const size_t need = sics_workspace_floats(g, n_candidates, heads) * sizeof(float);
  if (ws_bytes < need) return fail(SPADE_ERR_WORKSPACE, "workspace needs %zu bytes", need);
  cudaError_t e = launch_sics(q, k, g, n_candidates, heads, d, dt, static_cast<float*>(workspace), scores, choice,
                              as_cuda(stream));
  return e == cudaSuccess ? SPADE_OK : cuda_fail(e, "sics");
}

spade_status spade_grouped_head_lists(const spade_geom* schemes, int n_schemes, const spade_head_scheme* table,
                                      int heads, int d, int text_tokens, int head, int64_t* cnt_offset,
                                      int64_t* idx_offset) {
  GroupLayout L;
  spade_status st = plan_group(schemes, n_schemes, table, heads, d, text_tokens, L);
  if (st != SPADE_OK) return st;
  if (head < 0 || head >= heads || !cnt_offset || !idx_offset) return fail(SPADE_ERR_INVALID, "head/outputs");
  if (table[head].dense) { *cnt_offset = -1; *idx_offset = -1; return SPADE_OK; }
  const int s = table[head].scheme;
  const Geo g = make_geo(schemes[s]);
  *cnt_offset = (int64_t)(L.cnt[s] + (size_t)L.pos[head] * g.nb * sizeof(int));
  *idx_offset = (int64_t)(L.idx[s] + (size_t)L.pos[head] * g.nb * g.nb * sizeof(int));
  return SPADE_OK;
}

spade_status spade_grouped_attn(const void* q, const void* k, const void* v, void* out, const spade_geom* schemes,
                                int n_schemes, const spade_head_scheme* table, int heads, int d, int text_tokens,
                                spade_dtype dt, void* workspace, size_t ws_bytes, spade_stream_t stream) {
  return spade_grouped_attn_ex(q, k, v, out, schemes, n_schemes, table, heads, d, text_tokens, dt, SPADE_SUM_MEAN,
                               SPADE_SUM_MEAN, nullptr, workspace, ws_bytes, stream);
}

spade_status spade_grouped_attn_ex(const void* q, const void* k, const void* v, void* out, const spade_geom* schemes,
                                   int n_schemes, const spade_head_scheme* table, int heads, int d, int text_tokens,
                                   spade_dtype dt, spade_summary q_summary, spade_summary k_summary,
                                   const int* window_radius, void* workspace, size_t ws_bytes,
                                   spade_stream_t stream) {
  if (window_radius)
    for (int h = 0; h < heads; ++h)
      for (int a = 0; a < 3; ++a)
        if (window_radius[3 * h + a] < 0) return fail(SPADE_ERR_INVALID, "window radius of head %d is negative", h);
  if ((q_summary != SPADE_SUM_MEAN && q_summary != SPADE_SUM_MAX && q_summary != SPADE_SUM_MIN) ||
      (k_summary != SPADE_SUM_MEAN && k_summary != SPADE_SUM_MAX && k_summary != SPADE_SUM_MIN))
    return fail(SPADE_ERR_INVALID, "summary modes %d/%d", (int)q_summary, (int)k_summary);
  GroupLayout L;
  spade_status st = plan_group(schemes, n_schemes, table, heads, d, text_tokens, L);
  if (st != SPADE_OK) return st;
  if ((st = check_d_dt(d, dt)) != SPADE_OK) return st;
  if (!q || !k || !v || !out) return fail(SPADE_ERR_INVALID, "null tensor pointer");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(workspace))
    return fail(SPADE_ERR_INVALID, "pointers must be 16-byte aligned");
  if (!workspace || ws_bytes < L.total) return fail(SPADE_ERR_WORKSPACE, "workspace needs %zu bytes", L.total);
  cudaStream_t s = as_cuda(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  // the attention launch of step 5, set up (and checked) before anything is enqueued
  AttnArgs a;
  grouped_attn_args(q, k, v, out, schemes, n_schemes, table, heads, d, text_tokens, dt, L, ws, a);
  if ((st = check_attention(a)) != SPADE_OK) return st;
  // steps 1-4 per scheme, for its non-dense heads
  for (int sc = 0; sc < n_schemes; ++sc) {
    const int hs = L.n_sparse[sc];
    if (hs == 0) continue;
    const Geo g = make_geo(schemes[sc]);
    float* qm = reinterpret_cast<float*>(ws + L.qmean[sc]);
    float* km = reinterpret_cast<float*>(ws + L.kmean[sc]);
    const std::vector<int>& hl = L.heads_of[sc];
    for (int i = 0; i < hs;) {                        // contiguous runs of heads
      int j = i + 1;
      while (j < hs && hl[j] == hl[j - 1] + 1) ++j;
      const size_t o = (size_t)i * g.nb * d;
      cudaError_t e;
      if (q_summary == k_summary) {               // Q and K in one launch
        e = launch_summarize_pair(q, k, qm + o, km + o, g, heads, hl[i], j - i, d, dt, (int)q_summary, s);
      } else {
        e = launch_summarize(q, qm + o, g, heads, hl[i], j - i, d, dt, (int)q_summary, s);
        if (e == cudaSuccess) e = launch_summarize(k, km + o, g, heads, hl[i], j - i, d, dt, (int)k_summary, s);
      }
      if (e != cudaSuccess) return cuda_fail(e, "summarize");
      i = j;
    }
    std::vector<float> taus(hs);
    std::vector<int> rad(3 * hs, 0);
    for (int i = 0; i < hs; ++i) {
      taus[i] = table[hl[i]].tau;
      if (window_radius)
        for (int a = 0; a < 3; ++a) rad[3 * i + a] = window_radius[3 * hl[i] + a];
    }
    int* cnt_s = reinterpret_cast<int*>(ws + L.cnt[sc]);
    int* idx_s = reinterpret_cast<int*>(ws + L.idx[sc]);
    float* prob = reinterpret_cast<float*>(ws + L.prob[sc]);
    int* st = status_ptr();
    if (!st) return fail(SPADE_ERR_CUDA, "device status word unavailable");
    bool scores = false;
    cudaError_t e = run_estimate(qm, km, prob, hs, g.nb, d, st, false, &scores, s);
    if (e != cudaSuccess) return cuda_fail(e, "estimate");
    e = launch_select(prob, taus.data(), cnt_s, idx_s, hs, g.nb, s, window_radius ? rad.data() : nullptr, &g, scores);
    if (e != cudaSuccess) return cuda_fail(e, "select");
  }
  // step 5: one grouped launch over every head
  return run_attention(a, s);
}

spade_status spade_grouped_attn_lists(const void* q, const void* k, const void* v, void* out,
                                      const spade_geom* schemes, int n_schemes, const spade_head_scheme* table,
                                      int heads, int d, int text_tokens, spade_dtype dt, void* workspace,
                                      size_t ws_bytes, spade_stream_t stream) {
  GroupLayout L;
  spade_status st = plan_group(schemes, n_schemes, table, heads, d, text_tokens, L);
  if (st != SPADE_OK) return st;
  if ((st = check_d_dt(d, dt)) != SPADE_OK) return st;
  if (!q || !k || !v || !out) return fail(SPADE_ERR_INVALID, "null tensor pointer");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(workspace))
    return fail(SPADE_ERR_INVALID, "pointers must be 16-byte aligned");
  if (!workspace || ws_bytes < L.total) return fail(SPADE_ERR_WORKSPACE, "workspace needs %zu bytes", L.total);
  AttnArgs a;
  grouped_attn_args(q, k, v, out, schemes, n_schemes, table, heads, d, text_tokens, dt, L,
                    static_cast<uint8_t*>(workspace), a);
  if ((st = check_attention(a)) != SPADE_OK) return st;
  return run_attention(a, as_cuda(stream));
}

size_t spade_grouped_host_workspace_bytes(const spade_geom* schemes, int n_schemes, const spade_head_scheme* table,
                                          int heads, int d, int text_tokens, spade_dtype dt, int head_chunk) {
  HostLayout H;
  if (plan_host(schemes, n_schemes, table, heads, d, text_tokens, dt, head_chunk, H) != SPADE_OK) return 0;
  return H.total;
}

spade_status spade_grouped_attn_host(const void* q_host, const void* k_host, const void* v_host, void* out_host,
                                     const spade_geom* schemes, int n_schemes, const spade_head_scheme* table,
                                     int heads, int d, int text_tokens, spade_dtype dt, int head_chunk,
                                     void* workspace, size_t ws_bytes, spade_stream_t stream) {
  HostLayout H;
  spade_status st = plan_host(schemes, n_schemes, table, heads, d, text_tokens, dt, head_chunk, H);
  if (st != SPADE_OK) return st;
  if (!q_host || !k_host || !v_host || !out_host) return fail(SPADE_ERR_INVALID, "null host pointer");
  if (!workspace || ws_bytes < H.total) return fail(SPADE_ERR_WORKSPACE, "workspace needs %zu bytes", H.total);
  if (!aligned16(workspace)) return fail(SPADE_ERR_INVALID, "pointers must be 16-byte aligned");
  // every group's grouped call is checked before anything is enqueued
  const int N = schemes[0].T * schemes[0].H * schemes[0].W;
  for (int g = 0; g < H.n_groups; ++g) {
    const int h0 = g * head_chunk, hc = std::min(head_chunk, heads - h0);
    AttnArgs a;
    memset(&a, 0, sizeof(a));
    a.n_schemes = n_schemes;
    for (int sc = 0; sc < n_schemes; ++sc) a.geo[sc] = make_geo(schemes[sc]);
    a.heads = hc; a.d = d; a.text_tokens = text_tokens; a.N = N; a.dt = dt;
    for (int h = 0; h < hc; ++h) {
      a.head[h].scheme = table[h0 + h].scheme;
      a.head[h].nb = a.geo[table[h0 + h].scheme].nb;
      a.head[h].dense = table[h0 + h].dense;
    }
    if ((st = check_attention(a)) != SPADE_OK) return st;
  }
  const int dev = current_device();
  if (dev < 0 || dev >= kMaxDevices) return fail(SPADE_ERR_CUDA, "no current CUDA device");
  HostPipe& P = host_pipe(dev);
  std::lock_guard<std::mutex> lock(P.mu);
  const int G = H.n_groups, ns = std::min(kHostSlots, G);
  cudaError_t e = host_pipe_setup(P, (size_t)3 * G + 1 + 2 + kHostComputes);
  if (e != cudaSuccess) return cuda_fail(e, "stream/event set-up");
  cudaEvent_t* loaded = P.ev.data();
  cudaEvent_t* done = loaded + G;
  cudaEvent_t* returned = done + G;
  cudaEvent_t* joins = returned + G;            // [0] entry, [1] up, [2] down, [3..] computes
  const cudaStream_t caller = as_cuda(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const int64_t rows = (int64_t)N + text_tokens;
  const void* src[3] = {q_host, k_host, v_host};
  // everything below is ordered after the caller's stream at this point
  if ((e = cudaEventRecord(joins[0], caller)) != cudaSuccess) return cuda_fail(e, "event record");
  cudaStreamWaitEvent(P.up, joins[0], 0);
  cudaStreamWaitEvent(P.down, joins[0], 0);
  for (int c = 0; c < kHostComputes; ++c) cudaStreamWaitEvent(P.comp[c], joins[0], 0);
  auto slot_buf = [&](int g, int which) { return ws + ((size_t)(g % ns) * 4 + which) * H.slot_bytes; };
  auto load = [&](int g) -> spade_status {
    const int h0 = g * head_chunk, hc = std::min(head_chunk, heads - h0);
    if (g >= ns) cudaStreamWaitEvent(P.up, returned[g - ns], 0);   // the slot's previous group is back
    for (int t = 0; t < 3; ++t) {
      spade_status s2 = spade_copy_head_slice(slot_buf(g, t), const_cast<void*>(src[t]), rows, heads, h0, hc, d, dt,
                                              1, reinterpret_cast<spade_stream_t>(P.up));
      if (s2 != SPADE_OK) return s2;
    }
    const cudaError_t e2 = cudaEventRecord(loaded[g], P.up);
    return e2 == cudaSuccess ? SPADE_OK : cuda_fail(e2, "event record");
  };
  for (int g = 0; g < ns - 1; ++g)
    if ((st = load(g)) != SPADE_OK) return st;
  for (int g = 0; g < G; ++g) {
    if (g + ns - 1 < G && (st = load(g + ns - 1)) != SPADE_OK) return st;
    const int h0 = g * head_chunk, hc = std::min(head_chunk, heads - h0);
    const cudaStream_t comp = P.comp[g % kHostComputes];
    cudaStreamWaitEvent(comp, loaded[g], 0);
    st = spade_grouped_attn(slot_buf(g, 0), slot_buf(g, 1), slot_buf(g, 2), slot_buf(g, 3), schemes, n_schemes,
                            table + h0, hc, d, text_tokens, dt, ws + H.ws_off + (size_t)(g % kHostComputes) * H.ws_bytes,
                            H.ws_bytes, reinterpret_cast<spade_stream_t>(comp));
    if (st != SPADE_OK) return st;
    if ((e = cudaEventRecord(done[g], comp)) != cudaSuccess) return cuda_fail(e, "event record");
    cudaStreamWaitEvent(P.down, done[g], 0);
    st = spade_copy_head_slice(slot_buf(g, 3), out_host, rows, heads, h0, hc, d, dt, 0,
                               reinterpret_cast<spade_stream_t>(P.down));
    if (st != SPADE_OK) return st;
    if ((e = cudaEventRecord(returned[g], P.down)) != cudaSuccess) return cuda_fail(e, "event record");
  }
  // the caller's stream waits for every stream of the call
  cudaEventRecord(joins[1], P.up);
  cudaEventRecord(joins[2], P.down);
  cudaStreamWaitEvent(caller, joins[1], 0);
  cudaStreamWaitEvent(caller, joins[2], 0);
  for (int c = 0; c < kHostComputes; ++c) {
    cudaEventRecord(joins[3 + c], P.comp[c]);
    cudaStreamWaitEvent(caller, joins[3 + c], 0);
  }
  e = cudaGetLastError();
  return e == cudaSuccess ? SPADE_OK : cuda_fail(e, "host-to-host layer");
}

spade_status spade_last_device_status(spade_stream_t stream) {
  cudaError_t e = cudaStreamSynchronize(as_cuda(stream));
  if (e != cudaSuccess) return cuda_fail(e, "stream synchronize");
  int v = 0;
  e = cudaMemcpyFromSymbol(&v, g_spade_status, sizeof(int));
  if (e != cudaSuccess) return cuda_fail(e, "read status");
  const int zero = 0;
  e = cudaMemcpyToSymbol(g_spade_status, &zero, sizeof(int));
  if (e != cudaSuccess) return cuda_fail(e, "clear status");
  return static_cast<spade_status>(v);
}

spade_status spade_selftest_bounded_wait(int64_t timeout_ns, spade_stream_t stream) {
  if (timeout_ns <= 0 || timeout_ns > 10000000000LL) return fail(SPADE_ERR_INVALID, "timeout_ns out of range");
  int* sp = status_ptr();
  if (!sp) return fail(SPADE_ERR_CUDA, "device status word unavailable");
  cudaError_t e = launch_bounded_wait_selftest(sp, timeout_ns, as_cuda(stream));
  return e == cudaSuccess ? SPADE_OK : cuda_fail(e, "bounded-wait self test");
}

}  // extern "C"
