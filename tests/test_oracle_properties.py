"""The oracle's invariants over many seeded random shapes (CPU).

The pins in oracle_pins.py check each invariant on fixed inputs; here the
strongest ones run over 40 random chunk tables, worker counts and
hyper-parameters each, so a mistake that only shows on some shape (an empty
chunk, a tail word, W = 1, a chunk of one element) still fails:

  * scaled signs: the two-level error feedback telescopes,
    sum_t g_hat_t = mean_w(sum_t g_w,t - err_w,T) - srv_err_T;
  * momentum-error rule: eps_T - eps_0 = (1 - beta1) sum_t (g_t - q_t);
  * 2-bit Adam: the worker stage is the 1-bit stage applied twice, bit for bit,
    and the two-level error feedback telescopes as well.
"""

import numpy as np
import pytest

from oracle_pins import EPS, LR, _codes_of, _ghat, _ghat2, offsets_of, ulp32
from workloads import aux_normal, aux_uniform

CASES = 40


def draw(case, salt):
    rng = np.random.default_rng([0x0B17, salt, case])
    C = int(rng.integers(1, 6))
    sizes = [int(rng.choice([0, 1, 2, 7, 31, 32, 33, 64, 100, 257])) for _ in range(C)]
    W = int(rng.integers(1, 6))
    T = int(rng.integers(2, 6))
    beta1 = np.float32(rng.choice([0.5, 0.8, 0.9, 0.95]))
    return sizes, W, T, beta1


def state(n, W, key):
    return {"p": aux_normal(0x0B17, (*key, 1), n, 0.02), "m": np.zeros(n, np.float32),
            "v": aux_uniform(0x0B17, (*key, 2), n, 1e-8, 1e-6),
            "err": np.zeros((W, n), np.float32), "srv_err": np.zeros(n, np.float32)}


@pytest.mark.parametrize("case", range(CASES))
def test_scaled_error_feedback_telescopes(orc, case):
    sizes, W, T, beta1 = draw(case, 1)
    off = offsets_of(sizes)
    n = int(off[-1])
    st = state(n, W, (1, case))
    gsum, ghat = np.zeros((W, n)), np.zeros(n)
    for t in range(T):
        g = aux_normal(0x0B17, (3, case, t), W * n, 1e-3).reshape(W, n)
        gsum += g
        orc.step(off, g, st, beta1, LR, EPS)
        ghat += _ghat(st["bits_srv"], st["s_srv"], sizes) if n else 0.0
    want = (gsum - st["err"]).mean(0) - st["srv_err"]
    assert np.max(np.abs(ghat - want), initial=0.0) <= 1e-8


@pytest.mark.parametrize("case", range(CASES))
def test_momentum_error_telescopes(orc, case):
    sizes, W, T, beta1 = draw(case, 2)
    off = offsets_of(sizes)
    n = int(off[-1])
    omb1 = float(np.float32(1) - beta1)
    err = aux_normal(0x0B17, (4, case), W * n, 0.1).reshape(W, n)
    err0 = err.astype(np.float64)
    acc, tol = np.zeros((W, n)), np.zeros((W, n))
    for t in range(T):
        g = aux_normal(0x0B17, (5, case, t), W * n, 0.3).reshape(W, n)
        before = err.astype(np.float64)
        codes, _ = orc.ternary_compress(off, g, err, beta1)
        q = np.stack([_codes_of(codes[w], sizes) for w in range(W)]).astype(np.float64) if n else \
            np.zeros((W, 0))
        acc += g - q
        tol += 4 * ulp32(np.abs(g) + np.abs(before) + np.abs(q) + np.abs(err))
    assert np.all(np.abs((err - err0) - omb1 * acc) <= tol)


@pytest.mark.parametrize("case", range(CASES))
def test_two_bit_is_one_bit_twice_and_telescopes(orc, case):
    sizes, W, T, beta1 = draw(case, 3)
    off = offsets_of(sizes)
    n = int(off[-1])
    wb = [0]
    for s in sizes:
        wb.append(wb[-1] + (s + 31) // 32)
    g = aux_normal(0x0B17, (6, case), W * n, 1e-3).reshape(W, n)
    err = aux_normal(0x0B17, (7, case), W * n, 1e-3).reshape(W, n)
    e2 = err.copy()
    bits2, s2, _ = orc.twobit_compress(off, g, e2)
    e1 = err.copy()
    b1, s1, _ = orc.compress(off, g, e1)
    zero = np.zeros_like(e1)
    b1b, s1b, _ = orc.compress(off, e1.copy(), zero)
    for w in range(W):
        for k in range(len(sizes)):
            nw = wb[k + 1] - wb[k]
            assert np.array_equal(bits2[w, 2 * wb[k]: 2 * wb[k] + nw], b1[w, wb[k]: wb[k + 1]])
            assert np.array_equal(bits2[w, 2 * wb[k] + nw: 2 * wb[k + 1]], b1b[w, wb[k]: wb[k + 1]])
    assert np.array_equal(s2[..., 0], s1) and np.array_equal(s2[..., 1], s1b) and np.array_equal(e2, zero)

    st = state(n, W, (8, case))
    gsum, ghat = np.zeros((W, n)), np.zeros(n)
    for t in range(T):
        gt = aux_normal(0x0B17, (9, case, t), W * n, 1e-3).reshape(W, n)
        gsum += gt
        orc.twobit_step(off, gt, st, beta1, LR, EPS)
        ghat += _ghat2(st["bits_srv"], st["s_srv"], sizes) if n else 0.0
    want = (gsum - st["err"]).mean(0) - st["srv_err"]
    assert np.max(np.abs(ghat - want), initial=0.0) <= 1e-8
