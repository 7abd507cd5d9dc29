"""The seeded input generator: SplitMix64 against its published reference
outputs, determinism, and the value recipe (smooth field + noise, V ~ N(0,1))."""
import math

import numpy as np
import torch

from spade_workloads import CONFIGS, get_config, make_qkv, splitmix64
from spade_workloads.gen import _GOLDEN, _as_i64, counter_normal, counter_uniform


def test_splitmix64_reference_vector():
    # reference outputs of Vigna's splitmix64.c seeded with 1234567
    expect = [6457827717110365317, 3203168211198807973, 9817491932198370423,
              4593380528125082431, 16408922859458223821]
    states = torch.tensor([_as_i64(1234567 + k * _GOLDEN) for k in range(5)])
    got = [int(v) & ((1 << 64) - 1) for v in splitmix64(states)]
    assert got == expect


def test_uniform_and_normal_moments():
    u = counter_uniform(12345, 200000)
    assert 0.0 < float(u.min()) and float(u.max()) <= 1.0
    assert abs(float(u.mean()) - 0.5) < 5e-3
    n = counter_normal(999, 200000)
    assert abs(float(n.mean())) < 1e-2 and abs(float(n.std()) - 1.0) < 1e-2


def test_generation_deterministic_and_shaped():
    wl = get_config("tiny")
    a = make_qkv(wl)
    b = make_qkv(wl)
    for x, y in zip(a, b):
        assert x.shape == (256, 2, 64) and x.dtype == torch.float32
        assert torch.equal(x, y)
    q, k, v = a
    assert not torch.equal(q, k)
    assert abs(float(v.mean())) < 0.05 and abs(float(v.std()) - 1.0) < 0.05
    # Q = smooth field (4 unit sinusoids: variance 2) + N(0, 0.25)
    assert abs(float(q.var()) - 2.25) < 0.5


def test_configs_geometry():
    assert CONFIGS["wan14b"].N == 75600 and CONFIGS["wan14b"].schemes[0].nb == 660
    assert CONFIGS["wan1.3b"].schemes[0].nb == 308
    assert CONFIGS["hunyuan"].schemes[0].nb == 1020 and CONFIGS["hunyuan"].n_total == 119056
    m = CONFIGS["mixed"]
    assert [s.nb for s in m.schemes] == [591, 630, 720]
    assert sum(m.head_dense) == 13 and m.head_scheme[13] == 1 and m.head_scheme[39] == 2
    assert m.head_tau[13] == 0.9 and m.head_tau[14] == 0.95 and m.head_tau[15] == 0.85
