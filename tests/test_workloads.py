"""Workload tables and seeded generators (CPU)."""

import numpy as np
import pytest

import workloads as W


@pytest.mark.parametrize("name,n,C,largest", [
    ("tiny", 1_048_576, 1, 1_048_576),
    ("bert-base", 109_482_240, 199, 23_440_896),
    ("gpt2xl-flat", 1_500_000_000, 23, 1 << 26),
    ("bert-large", 335_141_888, 391, 31_254_528),
    ("lamb-1.3b", 1_315_723_264, 292, 102_926_336),
])
def test_tables(name, n, C, largest):
    wl = W.get_workload(name)
    assert wl.n == n and wl.C == C and max(wl.sizes) == largest
    assert wl.offsets[0] == 0 and wl.offsets[-1] == n
    assert all(s % 32 == 0 for s in wl.sizes)


def test_gpt2xl_tail():
    wl = W.get_workload("gpt2xl-flat")
    assert wl.sizes[:22] == (1 << 26,) * 22 and wl.sizes[22] == 23_604_992


def test_generators_are_deterministic_and_blockwise():
    wl = W.get_workload("tiny").with_(sizes=(W.BLOCK + 1000, 64))
    a = W.chunk_grads(wl, 3, 1, 0)
    b = W.chunk_grads(wl, 3, 1, 0)
    assert np.array_equal(a, b)
    tail = W.chunk_grads(wl, 3, 1, 0, lo=W.BLOCK)
    assert np.array_equal(a[W.BLOCK:], tail)
    assert not np.array_equal(W.chunk_grads(wl, 4, 1, 0)[:100], a[:100])
    out = np.zeros((wl.W, wl.n), np.float32)
    W.fill_grads(wl, 3, out)
    assert np.array_equal(out[1, : wl.sizes[0]], a)
    p, v = W.chunk_state(wl, 1)
    pf, vf = np.zeros(wl.n, np.float32), np.zeros(wl.n, np.float32)
    W.fill_state(wl, pf, vf)
    assert np.array_equal(pf[wl.offsets[1]:], p) and np.array_equal(vf[wl.offsets[1]:], v)


def test_distributions():
    wl = W.get_workload("tiny")
    g = W.chunk_grads(wl, 0, 0, 0)
    assert abs(float(g.std()) - 1e-3) < 2e-5
    p, v = W.chunk_state(wl, 0)
    assert abs(float(p.std()) - 0.02) < 5e-4
    assert v.min() >= 1e-8 and v.max() <= 1e-6
    bl = W.get_workload("bert-large")
    t = W.chunk_grads(bl, 0, 0, 3)  # a 2048-element LayerNorm tensor
    assert 0.02 < np.mean(t == 0) < 0.09
    gx = W.get_workload("gpt2xl-flat")
    b = W.chunk_grads(gx, 0, 0, 22, lo=0, hi=1000)
    assert b.dtype == np.uint16
    f = W.bf16_bits_to_f32(b)
    assert np.all(W.f32_to_bf16_bits(f) == b)
    bb = W.get_workload("bert-base")
    assert bb.freeze_step == 5
    _, v0 = W.chunk_state(bb, 0)
    assert np.all(v0 == 0)


def test_bf16_rounding_ties_to_even():
    x = np.array([1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -(1.0 + 2 ** -8), 1.0 + 2 ** -8 + 2 ** -20],
                 np.float32)
    got = W.f32_to_bf16_bits(x)
    # ties go to the even mantissa; above the tie rounds up
    assert list(got) == [0x3F80, 0x3F82, 0xBF80, 0x3F81]
