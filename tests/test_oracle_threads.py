"""The multi-threaded oracle step equals the single-thread oracle bit for bit.

``oracle/onebit_oracle_mt.c`` runs the oracle's per-element statements over
element ranges on several host threads and keeps every reduction (a chunk's
sum of squares, a layer's trust-ratio sums) as one ascending loop, so its
results must be identical to ``orc_step`` for any thread count.  That is what
lets the all-cores CPU baseline and the long full-size chained parity runs use
it.  Cases: ragged multi-chunk layouts with chunks longer than one range task
(2^16 elements), tails, one-element and empty chunks; W = 1..5; float32 and
bfloat16 gradients; float32 and bfloat16 error buffers; clipping; Adam and
LAMB; several chained steps; a NaN gradient.  CPU only.
"""

import numpy as np
import pytest

import oracle
from workloads import aux_normal, aux_uniform

SEED = 0x7A11
B1, LR, EPS = np.float32(0.9), np.float32(1e-4), np.float32(1e-8)


def offsets_of(sizes):
    off = np.zeros(len(sizes) + 1, np.int64)
    np.cumsum(np.asarray(sizes, np.int64), out=off[1:])
    return off


def bf16_bits(x):
    u = np.ascontiguousarray(x, np.float32).view(np.uint32)
    return ((u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)).astype(np.uint16)


CASES = [
    # (sizes, W, grad bf16, err bf16, clip, optimizer, steps)
    ((200_003, 33, 0, 1, 131_072, 4_104), 1, False, False, 0.0, oracle.ADAM, 3),
    ((70_000, 65_536, 17), 3, True, False, 0.0, oracle.ADAM, 2),
    ((150_000, 0, 96), 4, False, True, 0.0, oracle.LAMB, 2),
    ((66_000, 1_000, 65_537), 5, True, True, 2.5e-4, oracle.LAMB, 2),
    ((300_000,), 2, False, False, 1e-4, oracle.ADAM, 3),
]


def _state(sizes, W, err_bf16, key):
    off = offsets_of(sizes)
    n = int(off[-1])
    p = aux_normal(SEED, (key, 1), n, 0.02)
    v = aux_uniform(SEED, (key, 2), n, 1e-8, 1e-6)
    m = aux_normal(SEED, (key, 3), n, 1e-4)
    err = aux_normal(SEED, (key, 4), W * n, 1e-4).reshape(W, n)
    srv = aux_normal(SEED, (key, 5), n, 1e-4)
    if err_bf16:
        err, srv = bf16_bits(err), bf16_bits(srv)
    return off, n, {"p": p, "m": m, "v": v, "err": err, "srv_err": srv}


def _grads(n, W, bf16, key, step):
    g = aux_normal(SEED, (key, 10, step), W * n, 1e-3).reshape(W, n)
    return bf16_bits(g) if bf16 else g


@pytest.mark.parametrize("case", range(len(CASES)))
@pytest.mark.parametrize("threads", [2, 5, 16])
def test_threaded_step_equals_single_thread(case, threads):
    sizes, W, gbf, ebf, clip, opt, steps = CASES[case]
    off, n, ref = _state(sizes, W, ebf, case)
    got = {k: v.copy() for k, v in ref.items()}
    o1, omt = oracle.get(), oracle.get_mt()
    for t in range(steps):
        g = _grads(n, W, gbf, case, t)
        f1 = o1.step(off, g, ref, B1, LR, EPS, clip=clip, optimizer=opt)
        f2 = omt.step(off, g, got, B1, LR, EPS, clip=clip, optimizer=opt, threads=threads)
        assert f1 == f2
        for k in ("p", "m", "v", "err", "srv_err", "bits_w", "s_w", "bits_srv", "s_srv"):
            a, b = np.ascontiguousarray(ref[k]), np.ascontiguousarray(got[k])
            assert a.shape == b.shape, k
            assert np.array_equal(a.view(np.uint8), b.view(np.uint8)), f"step {t}: {k} differs"


def test_threaded_step_flags_nan():
    sizes = (100_000, 40)
    off, n, ref = _state(sizes, 2, False, 99)
    got = {k: v.copy() for k, v in ref.items()}
    g = _grads(n, 2, False, 99, 0)
    g[1, 77_777] = np.nan
    f1 = oracle.get().step(off, g, ref, B1, LR, EPS)
    f2 = oracle.get_mt().step(off, g, got, B1, LR, EPS, threads=8)
    assert f1 == f2 == oracle.STATUS_NONFINITE
    for k in ("p", "m", "err", "srv_err", "bits_w", "bits_srv"):
        assert np.array_equal(np.ascontiguousarray(ref[k]).view(np.uint8),
                              np.ascontiguousarray(got[k]).view(np.uint8)), k
    assert np.array_equal(np.isnan(ref["s_w"]), np.isnan(got["s_w"]))


def test_plain_build_refuses_threads():
    off, n, st = _state((64,), 1, False, 7)
    with pytest.raises(RuntimeError):
        oracle.get().step(off, _grads(n, 1, False, 7, 0), st, B1, LR, EPS, threads=4)
