"""Workload shapes.

The five layer shapes follow the models the SPADE pages evaluate on
(Hunyuan-Video and Wan 2.1/2.2, 720p; gist.science technical summary,
"Experimental Results"); the grid sizes are the latent grids of those models'
VAEs at 720p/480p.  Blocking schemes are 3D boxes over the (T, H, W) latent
grid ("Blocking Scheme Candidates", vDiT-SSR section of the same summary).

Token order inside a tensor is row-major over (t, y, x):
    n = (t * H + y) * W + x
and Q/K/V are laid out [N (+ text), heads, d].  Text tokens, when present, are
appended after the N video tokens.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import Tuple


def _cdiv(a: int, b: int) -> int:
    return -(-a // b)


@dataclass(frozen=True)
class Scheme:
    """One blocking scheme: a (T, H, W) grid cut into (bt, bh, bw) boxes.

    Blocks are numbered raster-order over (block-t, block-y, block-x) and the
    slots inside a block raster-order over (t, y, x).  Edge blocks are padded
    to the full box size.
    """
    T: int
    H: int
    W: int
    bt: int
    bh: int
    bw: int

    @property
    def nbt(self) -> int:
        return _cdiv(self.T, self.bt)

    @property
    def nbh(self) -> int:
        return _cdiv(self.H, self.bh)

    @property
    def nbw(self) -> int:
        return _cdiv(self.W, self.bw)

    @property
    def nb(self) -> int:
        return self.nbt * self.nbh * self.nbw

    @property
    def bs(self) -> int:
        return self.bt * self.bh * self.bw

    @property
    def n_tokens(self) -> int:
        return self.T * self.H * self.W

    def as_tuple(self) -> Tuple[int, int, int, int, int, int]:
        return (self.T, self.H, self.W, self.bt, self.bh, self.bw)


def flat_scheme(n_tokens: int, bs: int = 128) -> Scheme:
    """A 1D scheme over the flattened token sequence (used for dense heads,
    where the blocking does not change the result)."""
    return Scheme(1, 1, n_tokens, 1, 1, bs)


@dataclass(frozen=True)
class Workload:
    name: str
    config_id: int
    T: int
    H: int
    W: int
    heads: int
    d: int
    dtype: str                      # "f32" or "bf16"
    text_tokens: int
    schemes: Tuple[Scheme, ...]
    head_scheme: Tuple[int, ...]    # scheme index per head
    head_tau: Tuple[float, ...]     # cumulative-mass threshold per head
    head_dense: Tuple[bool, ...]    # dense heads attend to every key
    description: str = ""
    tau_sweep: Tuple[float, ...] = field(default=())

    @property
    def N(self) -> int:
        return self.T * self.H * self.W

    @property
    def n_total(self) -> int:
        return self.N + self.text_tokens

    def with_tau(self, tau: float) -> "Workload":
        taus = tuple(tau if not dn else t for t, dn in zip(self.head_tau, self.head_dense))
        return Workload(self.name + f"@tau={tau}", self.config_id, self.T, self.H, self.W,
                        self.heads, self.d, self.dtype, self.text_tokens, self.schemes,
                        self.head_scheme, taus, self.head_dense, self.description, ())

    def with_heads(self, heads: int) -> "Workload":
        """Same shape with only the first `heads` heads (for CPU-sized tests)."""
        return Workload(self.name + f"[h<{heads}]", self.config_id, self.T, self.H, self.W,
                        heads, self.d, self.dtype, self.text_tokens, self.schemes,
                        self.head_scheme[:heads], self.head_tau[:heads],
                        self.head_dense[:heads], self.description, self.tau_sweep)


def _uniform(name, cid, T, H, W, heads, d, dtype, text, block, tau, desc, sweep=()):
    sc = Scheme(T, H, W, *block)
    return Workload(name, cid, T, H, W, heads, d, dtype, text, (sc,),
                    (0,) * heads, (tau,) * heads, (False,) * heads, desc, tuple(sweep))


def _mixed() -> Workload:
    T, H, W, heads = 21, 45, 80, 40
    N = T * H * W
    schemes = (flat_scheme(N, 128), Scheme(T, H, W, 1, 8, 16), Scheme(T, H, W, 8, 4, 4))
    hs, taus, dense = [], [], []
    for h in range(heads):
        if h <= 12:
            hs.append(0); dense.append(True); taus.append(1.0)
        elif h <= 26:
            hs.append(1); dense.append(False); taus.append((0.85, 0.90, 0.95)[h % 3])
        else:
            hs.append(2); dense.append(False); taus.append((0.85, 0.90, 0.95)[h % 3])
    return Workload("mixed", 4, T, H, W, heads, 128, "bf16", 0, schemes, tuple(hs),
                    tuple(taus), tuple(dense),
                    "Wan-14B shape, heads 0-12 dense, 13-26 spatial 1x8x16, "
                    "27-39 temporal 8x4x4, per-head tau 0.85/0.90/0.95 by head mod 3")


CONFIGS = {
    "tiny": _uniform("tiny", 0, 4, 8, 8, 2, 64, "f32", 0, (2, 4, 4), 0.8,
                     "latent grid 4x8x8, blocks 2x4x4, 2 heads, d=64, fp32"),
    "wan1.3b": _uniform("wan1.3b", 1, 21, 30, 52, 12, 128, "bf16", 0, (2, 8, 8), 0.9,
                        "Wan-1.3B shape: grid 21x30x52, 12 heads, d=128, blocks 2x8x8"),
    "wan14b": _uniform("wan14b", 2, 21, 45, 80, 40, 128, "bf16", 0, (2, 8, 8), 0.9,
                       "Wan-14B 720p shape: grid 21x45x80, 40 heads, d=128, blocks 2x8x8",
                       sweep=(0.8, 0.9, 0.95)),
    "hunyuan": _uniform("hunyuan", 3, 33, 45, 80, 24, 128, "bf16", 256, (2, 8, 8), 0.9,
                        "Hunyuan-Video shape: grid 33x45x80 + 256 dense text tokens, "
                        "24 heads, d=128, blocks 2x8x8"),
    "mixed": _mixed(),
}


def config_names():
    return list(CONFIGS.keys())


def get_config(name: str) -> Workload:
    return CONFIGS[name]
