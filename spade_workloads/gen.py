"""Seeded input generation (counter-based, device independent bits).

Every random draw is SplitMix64 (Steele, Lea & Flood, "Fast splittable
pseudorandom number generators", OOPSLA 2014) applied to a counter, so element
i of a stream is a pure function of (stream key, i) and the same on CPU and
GPU.  Uniforms take the top 53 bits; normals use the Box-Muller transform.

Workload recipe (the pages give no activations; this stands in for the
Hunyuan-Video / Wan layer inputs they measure on):
  Q, K [t, y, x, head, c] = sum_{m<4} sin(2 pi (f_t t/T + f_y y/H + f_x x/W) + phi) + N(0, 0.5^2)
      f_* ~ U[0, 2) cycles per grid extent, phi ~ U[0, 2 pi), independent per
      (tensor, head, channel, m): a smooth 3D field plus noise.
  V ~ N(0, 1);  text tokens (if any): Q, K, V ~ N(0, 1).
Values are computed in float64 and rounded once to the workload dtype.
"""
from __future__ import annotations

import math
from typing import Optional, Tuple

import torch

from .configs import Workload

SEED_BASE = 20260805
_GOLDEN = 0x9E3779B97F4A7C15
_C1 = 0xBF58476D1CE4E5B9
_C2 = 0x94D049BB133111EB
_M64 = (1 << 64) - 1

TENSOR_Q, TENSOR_K, TENSOR_V = 0, 1, 2
_TEXT_OFFSET = 8
_PARAM_OFFSET = 16


def _as_i64(u: int) -> int:
    u &= _M64
    return u - (1 << 64) if u >= (1 << 63) else u


def _srl(z: torch.Tensor, s: int) -> torch.Tensor:
    """Logical right shift of int64 tensors holding uint64 bit patterns."""
    return (z >> s) & ((1 << (64 - s)) - 1)


def splitmix64(x: torch.Tensor) -> torch.Tensor:
    """SplitMix64 output of state x (int64 tensor, uint64 bits, wraps mod 2^64)."""
    z = x + _as_i64(_GOLDEN)
    z = (z ^ _srl(z, 30)) * _as_i64(_C1)
    z = (z ^ _srl(z, 27)) * _as_i64(_C2)
    return z ^ _srl(z, 31)


def _splitmix64_int(x: int) -> int:
    z = (x + _GOLDEN) & _M64
    z = ((z ^ (z >> 30)) * _C1) & _M64
    z = ((z ^ (z >> 27)) * _C2) & _M64
    return z ^ (z >> 31)


def stream_key(config_id: int, tensor: int, head: int, seed: int = SEED_BASE) -> int:
    k = _splitmix64_int(seed)
    k = _splitmix64_int(k ^ (config_id << 40) ^ (tensor << 32) ^ head)
    return k


def counter_uniform(key: int, n: int, device="cpu", start: int = 0) -> torch.Tensor:
    """n uniforms in (0, 1] (float64): ((bits >> 11) + 1) * 2^-53."""
    ctr = torch.arange(start, start + n, dtype=torch.int64, device=device) + _as_i64(key)
    z = splitmix64(ctr)
    return (_srl(z, 11) + 1).to(torch.float64) * (2.0 ** -53)


def counter_normal(key: int, n: int, device="cpu") -> torch.Tensor:
    """n standard normals (float64) by Box-Muller on counters 2i, 2i+1."""
    u1 = counter_uniform(key, n, device, start=0)
    u2 = counter_uniform(_splitmix64_int(key ^ 0x5DEECE66D), n, device, start=0)
    return torch.sqrt(-2.0 * torch.log(u1)) * torch.cos((2.0 * math.pi) * u2)


def _field_params(wl: Workload, tensor: int, head: int) -> torch.Tensor:
    """[4 (f_t, f_y, f_x, phi), d, 4 sinusoids] float64 on CPU."""
    key = stream_key(wl.config_id, tensor + _PARAM_OFFSET, head)
    u = counter_uniform(key, 4 * wl.d * 4).reshape(4, wl.d, 4)
    out = u.clone()
    out[:3] = 2.0 * u[:3]            # cycles per grid extent in [0, 2)
    out[3] = 2.0 * math.pi * u[3]    # phase in [0, 2 pi)
    return out


def smooth_field(wl: Workload, tensor: int, head: int, device="cpu") -> torch.Tensor:
    """[N, d] float64 field (no noise) for tensor Q or K of one head."""
    p = _field_params(wl, tensor, head).to(device)
    t = torch.arange(wl.T, dtype=torch.float64, device=device).view(-1, 1, 1, 1) / wl.T
    y = torch.arange(wl.H, dtype=torch.float64, device=device).view(1, -1, 1, 1) / wl.H
    x = torch.arange(wl.W, dtype=torch.float64, device=device).view(1, 1, -1, 1) / wl.W
    acc = torch.zeros(wl.T, wl.H, wl.W, wl.d, dtype=torch.float64, device=device)
    for m in range(4):
        arg = (t * p[0, :, m] + y * p[1, :, m] + x * p[2, :, m]) * (2.0 * math.pi) + p[3, :, m]
        acc += torch.sin(arg)
    return acc.reshape(wl.N, wl.d)


def torch_dtype(wl: Workload) -> torch.dtype:
    return torch.float32 if wl.dtype == "f32" else torch.bfloat16


def make_qkv(wl: Workload, device="cpu", heads: Optional[int] = None,
             out_dtype: Optional[torch.dtype] = None,
             head_list: Optional[list] = None) -> Tuple[torch.Tensor, torch.Tensor, torch.Tensor]:
    """Q, K, V as [N + text, heads, d] tensors in the workload dtype.  With
    head_list, only those heads are generated (slot i holds head head_list[i]);
    each head's values do not depend on which other heads are generated."""
    hl = list(head_list) if head_list is not None else list(range(wl.heads if heads is None else heads))
    dt = torch_dtype(wl) if out_dtype is None else out_dtype
    n_tot = wl.n_total
    outs = []
    for tensor in (TENSOR_Q, TENSOR_K, TENSOR_V):
        out = torch.empty(n_tot, len(hl), wl.d, dtype=dt, device=device)
        for slot, h in enumerate(hl):
            noise = counter_normal(stream_key(wl.config_id, tensor, h), wl.N * wl.d, device)
            noise = noise.view(wl.N, wl.d)
            if tensor == TENSOR_V:
                vals = noise
            else:
                vals = smooth_field(wl, tensor, h, device) + 0.5 * noise
            out[: wl.N, slot, :] = vals.to(dt)
            if wl.text_tokens:
                tk = stream_key(wl.config_id, tensor + _TEXT_OFFSET, h)
                txt = counter_normal(tk, wl.text_tokens * wl.d, device).view(wl.text_tokens, wl.d)
                out[wl.N:, slot, :] = txt.to(dt)
            del noise, vals
        outs.append(out)
    return outs[0], outs[1], outs[2]
