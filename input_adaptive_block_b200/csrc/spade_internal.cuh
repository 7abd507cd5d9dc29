// Internal interface between the C-ABI layer (spade_api.cu) and the kernels.
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "spade.h"

#define SPADE_MAX_SCHEMES 4
#define SPADE_MAX_HEADS 128
#define SPADE_SELECT_MAX_NB 1024
#define SPADE_SELECT_MAX_HEADS 1024
#define SPADE_ESTIMATE_MAX_NB 2048
#define SPADE_WORKLIST_MAX_COST 4096
#define SPADE_TC_MAX_LIST 1280   // tensor-core path: key blocks per item (nb + text blocks)

namespace spade {

// Geometry of one blocking scheme, with derived block counts.
struct Geo {
  int T, H, W, bt, bh, bw;
  int nbt, nbh, nbw, nb, bs;
};

__host__ __device__ inline int cdiv(int a, int b) { return (a + b - 1) / b; }

__host__ __device__ inline Geo make_geo(const spade_geom& g) {
  Geo r;
  r.T = g.T; r.H = g.H; r.W = g.W; r.bt = g.bt; r.bh = g.bh; r.bw = g.bw;
  r.nbt = cdiv(g.T, g.bt); r.nbh = cdiv(g.H, g.bh); r.nbw = cdiv(g.W, g.bw);
  r.nb = r.nbt * r.nbh * r.nbw;
  r.bs = g.bt * g.bh * g.bw;
  return r;
}

// Origin (t0, y0, x0) and clipped extents (et, eh, ew) of block b.
__host__ __device__ inline void block_box(const Geo& g, int b, int& t0, int& y0, int& x0, int& et, int& eh,
                                          int& ew) {
  const int bk = b % g.nbw;
  const int bj = (b / g.nbw) % g.nbh;
  const int bi = b / (g.nbw * g.nbh);
  t0 = bi * g.bt; y0 = bj * g.bh; x0 = bk * g.bw;
  et = min(g.bt, g.T - t0); eh = min(g.bh, g.H - y0); ew = min(g.bw, g.W - x0);
}

// Per-head row of the attention launch.
struct HeadInfo {
  int scheme;      // index into the launch's scheme table
  int nb;          // blocks of that scheme
  int dense;       // attends every key block
  int cnt_off;     // element offset of this head's cnt[nb] from AttnArgs::cnt
  long long idx_off;  // element offset of this head's idx[nb][nb] from AttnArgs::idx
};

// Everything an attention launch needs (both kernel paths).
struct AttnArgs {
  const void* q; const void* k; const void* v; void* out;
  int n_schemes;
  Geo geo[SPADE_MAX_SCHEMES];
  int heads;           // total heads in the Q/K/V layout
  int d;
  int text_tokens;
  int N;               // video tokens = T*H*W (same for every scheme)
  HeadInfo head[SPADE_MAX_HEADS];
  const int* cnt;      // base of the kept counts
  const int* idx;      // base of the kept ids
  int* work;           // [n_items] work list (built on device)
  int* ticket;         // one int next to the work list: dynamic work hand-out
  int n_items;
  spade_dtype dt;
  int* status;         // device status word
};

// Items per head: one per query block of the head's scheme, plus the text
// query blocks (128 text tokens each).
__host__ __device__ inline int text_blocks(int text_tokens) { return (text_tokens + 127) / 128; }

// ---- launchers (return the CUDA error of the launch) ----
cudaError_t launch_tile3d(const void* x, void* xt, const Geo& g, int heads, int d, spade_dtype dt,
                          cudaStream_t s);
cudaError_t launch_summarize(const void* x, float* out, const Geo& g, int heads_total, int h0, int hc, int d,
                             spade_dtype dt, int mode, cudaStream_t s);
// Q and K with the same reduce, in one launch.
cudaError_t launch_summarize_pair(const void* q, const void* k, float* qout, float* kout, const Geo& g,
                                  int heads_total, int h0, int hc, int d, spade_dtype dt, int mode, cudaStream_t s);
// probs = false: out = the scaled pooled scores; true: their row softmax.
cudaError_t launch_estimate_tc(const float* qm, const float* km, float* out, int heads, int nb, int d, int* status,
                               bool probs, cudaStream_t s);
cudaError_t launch_estimate(const float* qm, const float* km, float* prob, int heads, int nb, int d,
                            cudaStream_t s);
// scores = true: `in` holds scaled pooled scores and the kernel forms the
// softmax itself; false: `in` holds probabilities.
cudaError_t launch_select(const float* in, const float* tau_host, int* cnt, int* idx, int heads, int nb,
                          cudaStream_t s, const int* radius_host = nullptr, const Geo* g = nullptr,
                          bool scores = false);
cudaError_t launch_worklist(const AttnArgs& a, cudaStream_t s);
cudaError_t launch_attn_simt(const AttnArgs& a, cudaStream_t s);
// Returns cudaErrorNotSupported if the shape is not for the tensor-core path.
bool attn_tc_supported(const AttnArgs& a);
cudaError_t launch_attn_tc(const AttnArgs& a, cudaStream_t s, const char** why);
cudaError_t launch_bounded_wait_selftest(int* status, long long timeout_ns, cudaStream_t s);
size_t sics_workspace_floats(const Geo* cand, int n_cand, int heads);
cudaError_t launch_sics(const void* q, const void* k, const Geo* cand, int n_cand, int heads, int d, spade_dtype dt,
                        float* ws, float* scores, int* choice, cudaStream_t s);

int num_sms();                               // SM count of the current device
long long device_wait_timeout_ns();          // limit for every bounded device wait

}  // namespace spade
