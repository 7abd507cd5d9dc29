/*
 * spade.h -- C ABI of the SPADE executor hot path on NVIDIA B200 (sm_100a).
 *
 * What it computes (SPADE: "An Input-Adaptive Sparse Attention Engine for Fast
 * Video Diffusion Models Inference"; authors' abstract on catalyzex.com, and
 * the technical summary on gist.science/paper/2608.03335):
 * the input-adaptive block-sparse self-attention of one video-DiT layer.  Per
 * attention head:
 *   1. 3D tiling of the latent token grid (T,H,W) into (bt,bh,bw) blocks
 *      (technical summary, Methodology 1 "Blocking Scheme Candidates");
 *   2. a Summarizer reducing each Q/K block to one vector -- block mean
 *      (Methodology 1, "Summarizer & Estimator Expressions");
 *   3. an Estimator of block-to-block importance -- softmax over key blocks of
 *      the pooled scores Qbar_i . Kbar_j / sqrt(d) (same passage);
 *   4. the "low-overhead index search" of the executor (abstract): per query
 *      block, the smallest set of key blocks whose probability mass reaches
 *      tau, diagonal block always kept;
 *   5. flash block-sparse attention over only the kept blocks, online softmax,
 *      no dense score matrix (Methodology 3, "Flash Block-Sparse Attention");
 * with heads of different blocking schemes run in one grouped launch
 * (Methodology 3, "Head Grouping"; abstract, "kernel grouping").
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - All tensor pointers are DEVICE pointers owned by the caller; the library
 *    never allocates, frees or synchronises (except spade_last_device_status).
 *    Work is enqueued on `stream` (a cudaStream_t; NULL = legacy default) and
 *    returns before it runs.
 *  - Token order: n = (t*H + y)*W + x.  Q/K/V/O are contiguous
 *    [n_tokens, heads, d] (batch 1).  When text_tokens > 0 the text tokens
 *    follow the N = T*H*W video tokens: n_tokens = N + text_tokens.
 *  - Blocks of a scheme are numbered raster-order over (block-t, block-y,
 *    block-x); the slots of a block raster-order over (t, y, x) inside the box.
 *    nb = ceil(T/bt)*ceil(H/bh)*ceil(W/bw); BS = bt*bh*bw.  Edge blocks are
 *    padded: padded slots hold zeros, padded keys get no weight, padded query
 *    slots produce no output, and block means divide by the VALID count.
 *  - Host-side argument errors are returned synchronously and nothing is
 *    enqueued.  Errors detected on the device (a bounded wait that ran out)
 *    are latched in a device status word, readable with
 *    spade_last_device_status().
 *  - Pointers must be 16-byte aligned.  bf16 = IEEE bfloat16 bit pattern.
 *  - Several host threads may call the library at once: each call stages its
 *    launch parameters in storage of its own thread, and the launch copies
 *    them.  The GPU-side rules are the caller's: calls whose buffers (or,
 *    for spade_block_sparse_attn_noalloc, the library's fixed scratch)
 *    overlap must be ordered on the GPU (one stream, or events).
 */
#ifndef SPADE_H_
#define SPADE_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* spade_stream_t;   /* same handle as cudaStream_t */

typedef enum {
  SPADE_OK = 0,
  SPADE_ERR_INVALID = 1,       /* bad pointer, size or shape                    */
  SPADE_ERR_UNSUPPORTED = 2,   /* valid but not implemented (e.g. d not 64/128)  */
  SPADE_ERR_CUDA = 3,          /* a CUDA runtime/driver call failed             */
  SPADE_ERR_TIMEOUT = 4,       /* a bounded device-side wait ran out            */
  SPADE_ERR_WORKSPACE = 5      /* workspace missing or smaller than required    */
} spade_status;

typedef enum { SPADE_F32 = 0, SPADE_BF16 = 1 } spade_dtype;

/* Summarizer reduce of a Q/K block (Methodology 1, "Summarizer & Estimator
 * Expressions": max / min / mean), over the block's valid tokens. */
typedef enum { SPADE_SUM_MEAN = 0, SPADE_SUM_MAX = 1, SPADE_SUM_MIN = 2 } spade_summary;

/* One blocking scheme: the (T,H,W) latent grid cut into (bt,bh,bw) boxes.
 * A dense head may use the flat scheme {1,1,N, 1,1,128}. */
typedef struct { int32_t T, H, W, bt, bh, bw; } spade_geom;

/* Row of the per-head scheme table: which scheme the head uses, its
 * cumulative-mass threshold tau (tau >= 1 keeps every block) and whether the
 * head is dense (attends every key; no estimation or selection). */
typedef struct { int32_t scheme; float tau; int32_t dense; } spade_head_scheme;

/* ---- step 1: 3D tiling --------------------------------------------------
 * Methodology 1, "Blocking Scheme Candidates" (contiguous 3D blocks of the
 * latent grid) and Methodology 3, "Kernel Fusion" (layout transformation).
 * x  : [>= N, heads, d] token order, dtype `dt` (rows past N are ignored).
 * xt : [heads, nb, BS, d] same dtype; padded slots written as zero.
 * Pure data movement: bit-exact. */
spade_status spade_tile3d(const void* x, void* xt, spade_geom g, int heads, int d,
                          spade_dtype dt, spade_stream_t stream);

/* ---- step 2: Summarizer (block mean) -------------------------------------
 * Methodology 1, "Summarizer & Estimator Expressions" (mean reduce of a Q/K
 * block), fused with the tiling as in Methodology 3 "Kernel Fusion": reads x
 * in token order and never materialises tiles.
 * x     : [>= N, heads, d] token order, dtype `dt`.
 * xmean : [heads, nb, d] float32, mean over each block's valid tokens
 *         (accumulated in float32). */
spade_status spade_summarize(const void* x, float* xmean, spade_geom g, int heads, int d,
                             spade_dtype dt, spade_stream_t stream);

/* spade_summarize of Q and of K in one launch (the form spade_grouped_attn
 * runs): qmean from q and kmean from k, each exactly as spade_summarize
 * computes it.  q, k: [>= N, heads, d] token order, dtype `dt`; qmean,
 * kmean: [heads, nb, d] float32. */
spade_status spade_summarize_qk(const void* q, const void* k, float* qmean, float* kmean, spade_geom g,
                                int heads, int d, spade_dtype dt, spade_stream_t stream);

/* The same pass with another of the Summarizer's reduces: mode
 * SPADE_SUM_MAX / SPADE_SUM_MIN give the elementwise max / min over each
 * block's valid tokens (exact: no rounding), SPADE_SUM_MEAN is
 * spade_summarize. */
spade_status spade_summarize_mode(const void* x, float* out, spade_geom g, int heads, int d,
                                  spade_dtype dt, spade_summary mode, spade_stream_t stream);

/* ---- step 3: Estimator ---------------------------------------------------
 * Methodology 1, "Summarizer & Estimator Expressions" (inter-block importance).
 * prob[h,i,j] = softmax_j( qmean[h,i,:] . kmean[h,j,:] / sqrt(d) ), float32.
 * qmean, kmean : [heads, nb, d] float32;  prob : [heads, nb, nb] float32.
 * Limits: 1 <= nb <= 2048, d in {64, 128}. */
spade_status spade_estimate(const float* qmean, const float* kmean, float* prob,
                            int heads, int nb, int d, spade_stream_t stream);

/* Step 3 without its softmax: scores[h,i,j] = qmean[h,i,:] . kmean[h,j,:] /
 * sqrt(d), float32, computed exactly as spade_estimate computes them before
 * its softmax (split-precision TF32 on the tensor cores, fp32-level
 * accuracy).  This is the form spade_grouped_attn runs: the softmax is then
 * formed by spade_select_scores as it reads each row, so the probabilities
 * never pass through memory.  Same arguments and limits as spade_estimate;
 * returns SPADE_ERR_UNSUPPORTED where the driver's tensor-map encoder is
 * unavailable (spade_estimate then falls back to a CUDA-core kernel). */
spade_status spade_estimate_scores(const float* qmean, const float* kmean, float* scores,
                                   int heads, int nb, int d, spade_stream_t stream);

/* ---- step 4: index search -----------------------------------------------
 * Abstract, executor "low-overhead index search"; Methodology 3, ranked
 * block-sparse representation.  Per (head h, query block i): kept set = {i},
 * then other blocks in descending prob (ties -> lower id) until the mass
 * (prob[h,i,i] + sum of added) >= tau[h]; tau >= 1 or a mass that never
 * reaches tau keeps every block.  Probabilities are compared as float32;
 * masses are summed in fixed point (units of 2^-30, or of 2^-30 times the
 * row sum when a row sums to more than 1), so every sum is exact and the
 * result does not depend on summation order.  Entries are clamped to [0, 1]
 * (NaN counts as 0).
 * prob    : [heads, nb, nb] float32 (device).
 * tau_host: [heads] float32 HOST array, read during the call.
 * cnt     : [heads, nb] int32 out, number of kept blocks (>= 1).
 * idx     : [heads, nb, nb] int32 out; row (h,i) holds its cnt[h,i] kept ids in
 *           ascending order; entries past cnt[h,i] are left untouched.
 * Limits: nb <= 1024, heads <= 1024. */
spade_status spade_select(const float* prob, const float* tau_host, int* cnt, int* idx,
                          int heads, int nb, spade_stream_t stream);

/* Steps 3 and 4 fused: the Estimator's softmax over each row of `scores`
 * (from spade_estimate_scores: prob = exp(s - max) / sum, float32) followed
 * by the same index search as spade_select, in one pass over the row.
 * scores: [heads, nb, nb] float32 (device); other arguments, outputs and
 * limits as spade_select. */
spade_status spade_select_scores(const float* scores, const float* tau_host, int* cnt, int* idx,
                                 int heads, int nb, spade_stream_t stream);

/* Static windows merged with dynamic selection (Methodology 2, Policy
 * Application: "balancing static windows and dynamic selection").  The
 * window of query block i -- the blocks whose (block-t, block-y, block-x)
 * coordinates in geometry g lie within radius_per_head[h] = (rt, ry, rx) of
 * block i's -- takes the place of the diagonal: it is always kept and its
 * mass counts first; the other blocks follow by descending probability
 * until the mass reaches tau.  Radius (0, 0, 0) is exactly spade_select.
 * prob: [heads, nb, nb] with nb = the block count of g; radius_per_head:
 * host int32 [heads][3], non-negative.  Same outputs and limits as
 * spade_select. */
spade_status spade_select_window(const float* prob, const float* tau_per_head, const int* radius_per_head,
                                 spade_geom g, int* cnt, int* idx, int heads, spade_stream_t stream);

/* ---- step 5: flash block-sparse attention (one scheme) -------------------
 * Methodology 3, "Flash Block-Sparse Attention": exact softmax attention of
 * every valid query token of block i over the valid tokens of its kept key
 * blocks (plus every text token), scale 1/sqrt(d), online softmax.  Text
 * query rows attend every key.  Output written in token order.
 * q,k,v   : [N + text_tokens, heads, d], dtype `dt`.
 * out     : [N + text_tokens, heads, d], dtype `dt`; every row written.
 * cnt,idx : from spade_select for this scheme ([heads, nb], [heads, nb, nb]);
 *           cnt == NULL means every head is dense.
 * workspace: device scratch of spade_attn_workspace_bytes() bytes (work list).
 * Paths: bf16 with BS == 128, d in {64,128} and nb + ceil(text_tokens/128)
 * <= 1280 runs the tcgen05/TMEM/TMA kernel; everything else (fp32, other
 * block sizes, longer lists) the CUDA-core kernel (blocks of <= 128 slots). */
size_t spade_attn_workspace_bytes(spade_geom g, int heads, int d, int text_tokens);
spade_status spade_block_sparse_attn(const void* q, const void* k, const void* v, void* out,
                                     const int* cnt, const int* idx, spade_geom g,
                                     int heads, int d, int text_tokens, spade_dtype dt,
                                     void* workspace, size_t ws_bytes, spade_stream_t stream);

/* ---- step 5 without a caller workspace ------------------------------------
 * Not from the SPADE pages (they have no counterpart): the same computation
 * and arguments as spade_block_sparse_attn, minus the workspace, for callers
 * that cannot allocate device memory themselves -- for example code running
 * where another component owns every allocation, or a runtime that forbids
 * allocation on the call path.  The per-call scratch (the work list and its
 * hand-out counter) lives instead in one fixed device array inside the
 * library: 65536 work items (256 KiB), held on every device that uses it
 * until the library is unloaded.
 *  - heads * (nb + ceil(text_tokens/128)) must be <= 65536; larger calls
 *    return SPADE_ERR_UNSUPPORTED and enqueue nothing.
 *  - The library allocates nothing here (no cudaMalloc/cudaFree).  The first
 *    call on each device looks up the array's device address (with that
 *    device current) and caches it; make that first call before any stream
 *    capture.
 *  - Every call shares the one array, and each call rewrites it in full
 *    (the counter is reset on the device at the start of each call).  Calls
 *    from any host threads may be made, but calls whose work overlaps on the
 *    GPU (on different streams) race on the array; order them (one stream,
 *    or events). */
spade_status spade_block_sparse_attn_noalloc(const void* q, const void* k, const void* v, void* out,
                                             const int* cnt, const int* idx, spade_geom g,
                                             int heads, int d, int text_tokens, spade_dtype dt,
                                             spade_stream_t stream);

/* ---- steps 1-5 for heads of mixed schemes, one grouped attention launch ---
 * Methodology 3, "Head Grouping"; abstract, "kernel grouping".  Runs the
 * summarizer, estimator and index search per scheme for the non-dense heads,
 * builds one cost-ranked work list over all heads, and runs ONE attention
 * launch over every head.
 * schemes : n_schemes (1..4) geometries, all with the same T*H*W = N.
 * table   : [heads] per-head rows (host array, read during the call).
 * workspace: device scratch of spade_grouped_workspace_bytes() bytes.
 * Limits: heads <= 128, as for the single steps. */
size_t spade_grouped_workspace_bytes(const spade_geom* schemes, int n_schemes,
                                     const spade_head_scheme* table, int heads, int d,
                                     int text_tokens);
spade_status spade_grouped_attn(const void* q, const void* k, const void* v, void* out,
                                const spade_geom* schemes, int n_schemes,
                                const spade_head_scheme* table, int heads, int d,
                                int text_tokens, spade_dtype dt,
                                void* workspace, size_t ws_bytes, spade_stream_t stream);

/* spade_grouped_attn with the Summarizer reduce chosen for Q and for K
 * (the estimator then scores the pooled Q and K summaries as usual) and an
 * optional static window per head (window_radius: host int32 [heads][3]
 * block radii (rt, ry, rx), see spade_select_window; NULL keeps the
 * diagonal rule).  spade_grouped_attn is this call with SPADE_SUM_MEAN for
 * both and no window. */
spade_status spade_grouped_attn_ex(const void* q, const void* k, const void* v, void* out,
                                   const spade_geom* schemes, int n_schemes,
                                   const spade_head_scheme* table, int heads, int d,
                                   int text_tokens, spade_dtype dt,
                                   spade_summary q_summary, spade_summary k_summary,
                                   const int* window_radius,
                                   void* workspace, size_t ws_bytes, spade_stream_t stream);

/* Step 5 alone for a grouped layer: the one attention launch over every
 * head, under the kept lists that an earlier spade_grouped_attn /
 * spade_grouped_attn_ex call with the same schemes, table, d and text_tokens
 * left in `workspace` (for instance to reuse a layer's mask on new Q/K/V, or
 * to time the attention apart from the selection).  Same arguments as
 * spade_grouped_attn; the workspace's kept lists are read, not written. */
spade_status spade_grouped_attn_lists(const void* q, const void* k, const void* v, void* out,
                                      const spade_geom* schemes, int n_schemes,
                                      const spade_head_scheme* table, int heads, int d,
                                      int text_tokens, spade_dtype dt,
                                      void* workspace, size_t ws_bytes, spade_stream_t stream);

/* Where, inside a grouped workspace, head `head`'s kept lists live (byte
 * offsets of its int32 cnt [nb] and idx [nb, nb] arrays); -1 for dense heads.
 * Lets a caller read back the mask the grouped call used. */
spade_status spade_grouped_head_lists(const spade_geom* schemes, int n_schemes,
                                      const spade_head_scheme* table, int heads, int d,
                                      int text_tokens, int head,
                                      int64_t* cnt_offset, int64_t* idx_offset);

/* ---- scheme generation: Sum of Intra-block Cosine Similarities -----------
 * Technical summary, Methodology 2 "Scheme Generation": every blocking
 * candidate is scored by the sum of the cosine similarities between the
 * embeddings inside each of its blocks (Aggregation Evaluation, in the
 * O(BS * d) online form), and each head takes the candidate with the
 * highest score (Policy Application); the result fills the per-head scheme
 * table of spade_grouped_attn.  Score of head h under candidate c:
 *   sum over blocks b of sum_{i,j valid in b} cos(q_i, q_j) + cos(k_i, k_j)
 * (ordered pairs, i = j included; a zero vector counts 0), evaluated as
 * || sum_i q_i/||q_i|| ||^2 + || sum_i k_i/||k_i|| ||^2 per block.
 * q, k      : device [N, heads, d] in dt, token order (text tokens, if any,
 *             follow the video tokens and are not scored).
 * candidates: n_candidates (1..4) geometries over the same T*H*W = N.
 * scores    : device float [heads, n_candidates] (written).
 * choice    : device int32 [heads]: index of the best candidate, ties to the
 *             lower index (written).
 * workspace : device scratch of spade_sics_workspace_bytes() bytes (one
 *             float per head, block and candidate); sums run in a fixed
 *             order, so results are deterministic.
 * Cost: when the candidates share one T x H x W grid and their common
 * refinement (cells of the gcd block extents inside regions of the lcm
 * extents) has at most 64 cells per region, Q and K are read once for all
 * candidates; otherwise once per candidate.
 * Supported: d in {64, 128}, dt bf16 or f32, heads <= 1024. */
size_t spade_sics_workspace_bytes(const spade_geom* candidates, int n_candidates, int heads);
spade_status spade_sics(const void* q, const void* k, const spade_geom* candidates, int n_candidates,
                        int heads, int d, spade_dtype dt, float* scores, int* choice,
                        void* workspace, size_t ws_bytes, spade_stream_t stream);

/* ---- host <-> device head slices (pipelined execution from host memory) ----
 * Copies the head slice [rows, h0 .. h0+hc, d] of a token-order array
 * [rows, heads_total, d] between host memory (ideally pinned) and a
 * contiguous device array [rows, hc, d]: to_device = 1 copies host -> device,
 * 0 copies device -> host.  One strided 2-D copy on `stream`
 * (asynchronous for pinned host memory); no kernels.  Lets a caller stream
 * a layer through the GPU head group by head group -- heads are independent
 * in every step -- overlapping the transfers of one group with the compute
 * of another. */
spade_status spade_copy_head_slice(void* device, void* host, int64_t rows, int heads_total, int h0, int hc,
                                   int d, spade_dtype dt, int to_device, spade_stream_t stream);

/* ---- steps 1-5 from host memory to host memory ------------------------------
 * One layer whose Q/K/V live in host memory and whose output goes back to
 * host memory.  Every step is per head (Methodology 3, "Head Grouping"), so
 * the layer is streamed through the GPU in groups of head_chunk heads: group
 * g is copied in (strided 2-D copies of its head slice) while an earlier
 * group runs spade_grouped_attn and a finished group is copied out, on
 * streams of the library's own.  Three device slots hold the groups in
 * flight and two compute streams alternate, so a group's kernels start on
 * the SMs the previous group's attention releases.
 * q_host, k_host, v_host : [N + text_tokens, heads, d] host arrays, dtype dt;
 *                          page-locked (cudaHostAlloc / cudaHostRegister)
 *                          for the copies to overlap the compute (pageable
 *                          memory works, with synchronous copies).
 * out_host               : [N + text_tokens, heads, d] host array, written.
 * schemes, table         : as for spade_grouped_attn (table: all heads).
 * head_chunk             : heads per group, 1 .. heads.
 * workspace              : device scratch of
 *                          spade_grouped_host_workspace_bytes() bytes (the
 *                          slots and one grouped workspace per compute
 *                          stream); the call allocates nothing.
 * The work is ordered after what `stream` holds at the call, and `stream`
 * waits for all of it: out_host is complete once `stream` is.  The library
 * creates its streams and events once per device and reuses them; calls on
 * one device from several host threads are enqueued one at a time. */
size_t spade_grouped_host_workspace_bytes(const spade_geom* schemes, int n_schemes,
                                          const spade_head_scheme* table, int heads, int d,
                                          int text_tokens, spade_dtype dt, int head_chunk);
spade_status spade_grouped_attn_host(const void* q_host, const void* k_host, const void* v_host, void* out_host,
                                     const spade_geom* schemes, int n_schemes,
                                     const spade_head_scheme* table, int heads, int d,
                                     int text_tokens, spade_dtype dt, int head_chunk,
                                     void* workspace, size_t ws_bytes, spade_stream_t stream);

/* ---- status ---------------------------------------------------------------
 * spade_last_device_status synchronises `stream`, returns the latched device
 * status (SPADE_OK or SPADE_ERR_TIMEOUT) and clears it. */
spade_status spade_last_device_status(spade_stream_t stream);
const char* spade_status_string(spade_status s);
const char* spade_last_error_message(void);   /* detail of the last host error */
int spade_version(void);

#ifdef __cplusplus
}
#endif
#endif /* SPADE_H_ */
