"""Plain, slow, fp64 CPU oracle of SPADE's input-adaptive block-sparse attention.

TEST INFRASTRUCTURE ONLY.  This module is what the CUDA library is checked
against; the library itself never imports, links or calls it.  It shares no
code with the CUDA path: the only thing both sides take from a common place is
the seeded input generator (package spade_workloads), which holds none of the
method's arithmetic.

Source: "SPADE: An Input-Adaptive Sparse Attention Engine for Fast Video
Diffusion Models Inference" (authors' abstract on catalyzex.com; technical
summary on gist.science/paper/2608.03335).  The pipeline per attention head:

  1. 3D tiling ("Blocking Scheme Candidates", vDiT-SSR): the latent token grid
     (T, H, W) is cut into contiguous (bt, bh, bw) boxes.
  2. Summarizer ("Summarizer & Estimator Expressions"): each Q/K block is
     reduced to one d-vector; the concrete instance here is the block mean.
  3. Estimator (same section): block-to-block importance, here the softmax
     over key blocks of the pooled scores  Qbar_i . Kbar_j / sqrt(d).
  4. Index search (abstract: "low-overhead index search"): per query block,
     the smallest set of key blocks whose probability mass reaches tau, with
     the diagonal block always kept.
  5. Flash block-sparse attention ("Head-wise Sparse Attention Execution"):
     exact softmax attention restricted to the kept blocks.  (Online softmax is
     how a kernel evaluates it; the oracle evaluates the definition directly.)

Readings taken where the pages are silent (each function below restates the
one it relies on):
  - token n = (t*H + y)*W + x; tensors [N (+text), heads, d]; batch 1;
  - edge blocks are padded; padded keys never receive weight; padded query
    slots produce no output; block means divide by the number of VALID tokens;
  - the softmax over key blocks is unweighted (no block-size correction);
  - selection: diagonal first, then the other blocks by descending probability
    (ties -> lower block id), stopping at the first prefix whose mass >= tau;
    tau >= 1, or a mass that never reaches tau, keeps every block;
  - text tokens are excluded from estimation/selection; every video query also
    attends every text key, and text queries attend every key;
  - dense heads attend every key;
  - softmax scale 1/sqrt(d) in both the estimator and the attention.

Every function works in float64 on numpy arrays; bf16/fp32 inputs convert to
float64 exactly.
"""
from __future__ import annotations

import math
from functools import lru_cache
from typing import Dict, List, Optional, Sequence, Tuple

import numpy as np

__all__ = [
    "block_tokens", "valid_counts", "tile3d", "untile3d", "summarize", "pooled_scores", "estimate", "softmax_rows",
    "select_row", "select", "selection_margin", "window_blocks", "attention_rows", "block_sparse_attention",
    "dense_attention", "pipeline", "kept_token_pairs",
    "block_sics", "sics", "choose_schemes",
]


# ---------------------------------------------------------------------------
# 1. 3D tiling
# ---------------------------------------------------------------------------

@lru_cache(maxsize=32)
def block_tokens(T: int, H: int, W: int, bt: int, bh: int, bw: int
                 ) -> Tuple[Tuple[np.ndarray, np.ndarray], ...]:
    """Per block (raster order over block-t, block-y, block-x): the token ids
    of its valid slots and the slot numbers they occupy, both in slot order.

    Slots inside a block are raster order over (t, y, x) within the box; a slot
    whose (t, y, x) falls outside the grid is padding (vDiT-SSR, "Blocking
    Scheme Candidates": contiguous 3D blocks of the latent grid)."""
    nbt, nbh, nbw = -(-T // bt), -(-H // bh), -(-W // bw)
    out = []
    for bi in range(nbt):
        for bj in range(nbh):
            for bk in range(nbw):
                toks, slots = [], []
                for tl in range(bt):
                    t = bi * bt + tl
                    for yl in range(bh):
                        y = bj * bh + yl
                        for xl in range(bw):
                            x = bk * bw + xl
                            if t < T and y < H and x < W:
                                toks.append((t * H + y) * W + x)
                                slots.append((tl * bh + yl) * bw + xl)
                out.append((np.asarray(toks, dtype=np.int64), np.asarray(slots, dtype=np.int64)))
    return tuple(out)


def valid_counts(geom: Sequence[int]) -> np.ndarray:
    return np.asarray([len(t) for t, _ in block_tokens(*geom)], dtype=np.int64)


def tile3d(x: np.ndarray, geom: Sequence[int]) -> np.ndarray:
    """x [N(+text), heads, d] -> tiles [heads, nb, bt*bh*bw, d] (float64),
    padded slots zero."""
    T, H, W, bt, bh, bw = geom
    blocks = block_tokens(*geom)
    heads, d = x.shape[1], x.shape[2]
    out = np.zeros((heads, len(blocks), bt * bh * bw, d), dtype=np.float64)
    for b, (toks, slots) in enumerate(blocks):
        out[:, b, slots, :] = np.transpose(x[toks].astype(np.float64), (1, 0, 2))
    return out


def untile3d(xt: np.ndarray, geom: Sequence[int]) -> np.ndarray:
    """Inverse of tile3d on the valid slots: tiles -> [N, heads, d]."""
    T, H, W = geom[:3]
    blocks = block_tokens(*geom)
    heads, d = xt.shape[0], xt.shape[3]
    out = np.zeros((T * H * W, heads, d), dtype=np.float64)
    for b, (toks, slots) in enumerate(blocks):
        out[toks] = np.transpose(xt[:, b, slots, :], (1, 0, 2))
    return out


# ---------------------------------------------------------------------------
# 2. Summarizer: block mean over valid tokens
# ---------------------------------------------------------------------------

def summarize(x: np.ndarray, geom: Sequence[int], mode: str = "mean") -> np.ndarray:
    """Reduce each block's valid tokens: [N, heads, d] -> [heads, nb, d].
    mode "mean" (the instance the estimator is specified with), or the other
    reduces the Summarizer names, "max" / "min" (elementwise over the block's
    valid tokens; padding never takes part)."""
    blocks = block_tokens(*geom)
    heads, d = x.shape[1], x.shape[2]
    out = np.zeros((heads, len(blocks), d), dtype=np.float64)
    for b, (toks, _) in enumerate(blocks):
        xb = x[toks].astype(np.float64)
        if mode == "mean":
            out[:, b, :] = xb.sum(axis=0) / len(toks)
        elif mode == "max":
            out[:, b, :] = xb.max(axis=0)
        elif mode == "min":
            out[:, b, :] = xb.min(axis=0)
        else:
            raise ValueError(mode)
    return out


# ---------------------------------------------------------------------------
# 3. Estimator: softmax over key blocks of pooled scores
# ---------------------------------------------------------------------------

def pooled_scores(qmean: np.ndarray, kmean: np.ndarray) -> np.ndarray:
    """S[h, i, j] = Qbar[h,i] . Kbar[h,j] / sqrt(d): the Estimator's
    inter-block score before its softmax."""
    d = qmean.shape[-1]
    return np.einsum("hid,hjd->hij", qmean.astype(np.float64), kmean.astype(np.float64)) / math.sqrt(d)


def estimate(qmean: np.ndarray, kmean: np.ndarray) -> np.ndarray:
    """P[h, i, j] = softmax_j(Qbar[h,i] . Kbar[h,j] / sqrt(d))."""
    return softmax_rows(pooled_scores(qmean, kmean))


def softmax_rows(s: np.ndarray) -> np.ndarray:
    """softmax over the last axis, float64."""
    s = np.asarray(s, dtype=np.float64)
    s = s - s.max(axis=-1, keepdims=True)
    e = np.exp(s)
    return e / e.sum(axis=-1, keepdims=True)


# ---------------------------------------------------------------------------
# 4. Index search: smallest diagonal-containing set reaching mass tau
# ---------------------------------------------------------------------------

def window_blocks(geom: Sequence[int], i: int, radius: Sequence[int]) -> List[int]:
    """Static window of query block i: the blocks whose (block-t, block-y,
    block-x) coordinates lie within radius = (rt, ry, rx) of block i's
    (technical summary, Methodology 2, Policy Application: "balancing static
    windows and dynamic selection").  Radius (0, 0, 0) is block i alone."""
    T, H, W, bt, bh, bw = (int(g) for g in geom)
    nbt, nbh, nbw = -(-T // bt), -(-H // bh), -(-W // bw)
    it, iy, ix = i // (nbh * nbw), (i // nbw) % nbh, i % nbw
    out = []
    for j in range(nbt * nbh * nbw):
        jt, jy, jx = j // (nbh * nbw), (j // nbw) % nbh, j % nbw
        if abs(jt - it) <= radius[0] and abs(jy - iy) <= radius[1] and abs(jx - ix) <= radius[2]:
            out.append(j)
    return out


def select_row(p: np.ndarray, i: int, tau: float, window: Optional[Sequence[int]] = None) -> List[int]:
    """Kept key blocks (ascending) for query block i of one head.  The
    static window (default: block i alone -- the diagonal) is kept first and
    its mass counts; the other blocks follow in descending probability."""
    nb = len(p)
    if tau >= 1.0:
        return list(range(nb))
    win = sorted(set(window)) if window is not None else [i]
    kept = list(win)
    mass = float(sum(float(p[j]) for j in win))
    inwin = set(win)
    others = sorted((j for j in range(nb) if j not in inwin), key=lambda j: (-p[j], j))
    for j in others:
        if mass >= tau:
            break
        kept.append(j)
        mass += float(p[j])
    return sorted(kept)


def select(P: np.ndarray, taus: Sequence[float]) -> Tuple[np.ndarray, np.ndarray]:
    """P [heads, nb, nb] -> (cnt [heads, nb] int32, idx [heads, nb, nb] int32,
    row-wise ascending kept ids, unused entries -1)."""
    heads, nb, _ = P.shape
    cnt = np.zeros((heads, nb), dtype=np.int32)
    idx = np.full((heads, nb, nb), -1, dtype=np.int32)
    for h in range(heads):
        for i in range(nb):
            kept = select_row(P[h, i], i, float(taus[h]))
            cnt[h, i] = len(kept)
            idx[h, i, : len(kept)] = kept
    return cnt, idx


def selection_margin(p: np.ndarray, i: int, tau: float, window: Optional[Sequence[int]] = None) -> float:
    """How far row i is from changing its kept set, in the estimator's score
    units (pooled logits; a probability ratio p_a/p_b is a score difference
    ln(p_a/p_b)).  It is the smallest of
      * ln(p_last_kept / p_first_dropped): the score gap at the cut;
      * (tau - C_before_last) / (C (1 - C)) and (C_after_last - tau) / (C (1 - C)):
        the mass slack on either side of tau divided by its first-order
        sensitivity to a shift of the kept blocks' scores against the rest
        (d C / d shift = C (1 - C) for a softmax).
    Rows whose margin is small may legitimately differ between a float32 and
    a float64 evaluation; rows above the threshold may not."""
    nb = len(p)
    if tau >= 1.0:
        return math.inf
    win = sorted(set(window)) if window is not None else [i]
    inwin = set(win)
    others = sorted((j for j in range(nb) if j not in inwin), key=lambda j: (-p[j], j))

    def sens(c):
        return max(c * (1.0 - c), 1e-300)

    mass = float(sum(float(p[j]) for j in win))
    k = 0
    prev = None
    while mass < tau and k < len(others):
        prev = mass
        mass += float(p[others[k]])
        k += 1
    if mass < tau:            # every block kept because the mass never reached tau
        return 0.0
    if k == 0:                # the diagonal (or the static window) alone reached tau
        return (mass - tau) / sens(mass)
    m = min((tau - prev) / sens(prev), (mass - tau) / sens(mass))
    if k < len(others):
        a, b = float(p[others[k - 1]]), float(p[others[k]])
        m = min(m, math.log(a / b) if b > 0.0 else math.inf)
    return m


# ---------------------------------------------------------------------------
# 5. Block-sparse attention: exact softmax attention over kept blocks
# ---------------------------------------------------------------------------

def attention_rows(q: np.ndarray, k: np.ndarray, v: np.ndarray, head: int,
                   rows: np.ndarray, keys: np.ndarray) -> np.ndarray:
    """softmax(q[rows] k[keys]^T / sqrt(d)) v[keys] for one head, float64."""
    d = q.shape[-1]
    qq = q[rows, head, :].astype(np.float64)
    kk = k[keys, head, :].astype(np.float64)
    vv = v[keys, head, :].astype(np.float64)
    s = (qq @ kk.T) / math.sqrt(d)
    s = s - s.max(axis=1, keepdims=True)
    e = np.exp(s)
    return (e / e.sum(axis=1, keepdims=True)) @ vv


def block_sparse_attention(q: np.ndarray, k: np.ndarray, v: np.ndarray,
                           head_geom: Sequence[Sequence[int]],
                           head_kept: Sequence[Optional[Sequence[Sequence[int]]]],
                           text_tokens: int = 0,
                           q_blocks: Optional[Dict[int, Sequence[int]]] = None) -> np.ndarray:
    """O [N + text, heads, d] float64.

    head_kept[h] is the kept-block list per query block of head h, or None for
    a dense head.  q_blocks optionally restricts which query blocks (per head)
    are evaluated; rows not evaluated are NaN.  Query blocks are numbered in
    the head's scheme; for text rows use block id nb (all text rows at once)."""
    n_tot, heads, d = q.shape
    N = n_tot - text_tokens
    out = np.full((n_tot, heads, d), np.nan, dtype=np.float64)
    text = np.arange(N, n_tot, dtype=np.int64)
    all_keys = np.arange(n_tot, dtype=np.int64)
    for h in range(heads):
        blocks = block_tokens(*head_geom[h])
        nb = len(blocks)
        want = range(nb + (1 if text_tokens else 0)) if q_blocks is None else q_blocks.get(h, [])
        for i in want:
            if i == nb:                                   # text query rows: dense
                out[text, h] = attention_rows(q, k, v, h, text, all_keys)
                continue
            rows = blocks[i][0]
            if head_kept[h] is None:
                keys = all_keys
            else:
                parts = [blocks[j][0] for j in head_kept[h][i]]
                if text_tokens:
                    parts.append(text)
                keys = np.concatenate(parts)
            out[rows, h] = attention_rows(q, k, v, h, rows, keys)
    return out


def dense_attention(q: np.ndarray, k: np.ndarray, v: np.ndarray) -> np.ndarray:
    """Plain full softmax attention over every token, per head (float64)."""
    n, heads, d = q.shape
    out = np.empty((n, heads, d), dtype=np.float64)
    rows = np.arange(n)
    for h in range(heads):
        out[:, h] = attention_rows(q, k, v, h, rows, rows)
    return out


def kept_token_pairs(head_geom, head_kept, text_tokens: int = 0,
                     q_blocks: Optional[Dict[int, Sequence[int]]] = None) -> int:
    """Number of (valid query, valid key) pairs the attention evaluates."""
    total = 0
    for h, geom in enumerate(head_geom):
        vc = valid_counts(geom)
        N = int(vc.sum())
        nb = len(vc)
        want = range(nb + (1 if text_tokens else 0)) if q_blocks is None else q_blocks.get(h, [])
        for i in want:
            if i == nb:
                total += text_tokens * (N + text_tokens)
            elif head_kept[h] is None:
                total += int(vc[i]) * (N + text_tokens)
            else:
                total += int(vc[i]) * (int(vc[list(head_kept[h][i])].sum()) + text_tokens)
    return total


# ---------------------------------------------------------------------------
# Scheme generation: Sum of Intra-block Cosine Similarities (SICS)
# ---------------------------------------------------------------------------
# Technical summary, Methodology 2 "Scheme Generation", Aggregation
# Evaluation: every blocking candidate is scored by the sum of the cosine
# similarities between the embeddings inside each block (tightly clustered
# blocks score high); Policy Application: each head takes the candidate with
# the highest score.  Readings (the pages give no formula): the embeddings
# are the head's Q and K tokens, scored separately and added; the sum runs
# over ordered pairs (i, j) of valid tokens of a block, i = j included (that
# adds N to every candidate alike, so the choice is unaffected); a zero
# vector has cosine 0 with everything; ties go to the lower candidate index.

def block_sics(xb: np.ndarray) -> float:
    """sum_{i, j} cos(x_i, x_j) over the rows of xb, by the plain pairwise
    definition: O(n^2 d)."""
    x = np.asarray(xb, dtype=np.float64)
    nrm = np.sqrt(np.sum(x * x, axis=1))
    total = 0.0
    for i in range(x.shape[0]):
        for j in range(x.shape[0]):
            if nrm[i] > 0.0 and nrm[j] > 0.0:
                total += float(np.dot(x[i], x[j]) / (nrm[i] * nrm[j]))
    return total


def sics(x: np.ndarray, geom: Sequence[int]) -> np.ndarray:
    """[heads] SICS of one tensor x [N, heads, d] under one blocking scheme:
    the sum over its blocks of block_sics of the block's valid tokens."""
    T, H, W, bt, bh, bw = (int(g) for g in geom)
    heads = x.shape[1]
    out = np.zeros(heads, dtype=np.float64)
    for ids, _slots in block_tokens(T, H, W, bt, bh, bw):
        for h in range(heads):
            out[h] += block_sics(x[ids, h, :])
    return out


def choose_schemes(q: np.ndarray, k: np.ndarray, candidates: Sequence[Sequence[int]]):
    """Per head: the SICS of every candidate (Q plus K) and the index of the
    best one.  Returns (scores [heads, n_candidates], choice [heads])."""
    heads = q.shape[1]
    scores = np.zeros((heads, len(candidates)), dtype=np.float64)
    for c, geom in enumerate(candidates):
        scores[:, c] = sics(q, geom) + sics(k, geom)
    choice = np.zeros(heads, dtype=np.int64)
    for h in range(heads):
        best = 0
        for c in range(1, len(candidates)):
            if scores[h, c] > scores[h, best]:
                best = c
        choice[h] = best
    return scores, choice


# ---------------------------------------------------------------------------
# The whole path for one layer
# ---------------------------------------------------------------------------

def pipeline(q: np.ndarray, k: np.ndarray, v: np.ndarray,
             schemes: Sequence[Sequence[int]], head_scheme: Sequence[int],
             head_tau: Sequence[float], head_dense: Sequence[bool],
             text_tokens: int = 0,
             q_blocks: Optional[Dict[int, Sequence[int]]] = None,
             kept_override: Optional[Dict[int, Sequence[Sequence[int]]]] = None,
             summary: Tuple[str, str] = ("mean", "mean")) -> dict:
    """Steps 1-5 for every head.  Returns the per-scheme summaries and
    probabilities, the kept lists and the output.  kept_override replaces the
    oracle's own selection for the given heads (used to evaluate attention
    under another implementation's mask); summary picks the Q and K reduces."""
    heads = q.shape[1]
    N = q.shape[0] - text_tokens
    head_geom = [tuple(schemes[head_scheme[h]]) for h in range(heads)]
    res = {"qmean": {}, "kmean": {}, "prob": {}, "kept": [None] * heads}
    for s_id, geom in enumerate(schemes):
        hs = [h for h in range(heads) if head_scheme[h] == s_id and not head_dense[h]]
        if not hs:
            continue
        qm = summarize(q[:N, hs], geom, summary[0])
        km = summarize(k[:N, hs], geom, summary[1])
        P = estimate(qm, km)
        res["qmean"][s_id], res["kmean"][s_id], res["prob"][s_id] = qm, km, P
        for n, h in enumerate(hs):
            res["kept"][h] = [select_row(P[n, i], i, float(head_tau[h])) for i in range(P.shape[1])]
    if kept_override:
        for h, kl in kept_override.items():
            res["kept"][h] = [list(x) for x in kl]
    kept = [None if head_dense[h] else res["kept"][h] for h in range(heads)]
    res["out"] = block_sparse_attention(q, k, v, head_geom, kept, text_tokens, q_blocks)
    return res
