"""Pins of the CPU oracle against things other than itself.

Each ``pin_*`` function takes an ``oracle.Oracle`` and raises AssertionError
when the oracle disagrees with a hand-worked case, a closed form, an
invariant of the method, an exact (rational) brute-force computation, or an
independent library routine (numpy's bit packing, norms, means).  They are
run against the real oracle (tests/test_oracle_pins.py) and against oracle
builds with planted mistakes, each of which must fail at least one pin
(tests/test_oracle_mutants.py).

Passages the checks rest on ('DeepSpeed Communication Compression and
Hiding', section '1-bit Adam' 机制; same page '基线' for the Adam moments and
'1-bit LAMB' for the trust ratio; the CANN article section 3.2 for clipping and
the NaN check), with the scale s = ||c||_2/sqrt(n), sign(0) = +1, LSB-first
uint32 packing, per-worker error c - s*sign(c), and the server stage that
averages scaled signs and re-compresses with its own error buffer.
"""

from __future__ import annotations

import json
import math
import os
from fractions import Fraction

import numpy as np

from workloads import aux_bits, aux_normal, aux_uniform

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")
SEED = 0x0B17
B1, B2, LR, EPS = np.float32(0.9), np.float32(0.999), np.float32(1e-4), np.float32(1e-8)


# -- independent helpers (numpy library routines, no oracle code) ---------------

def offsets_of(sizes):
    off = np.zeros(len(sizes) + 1, np.int64)
    np.cumsum(np.asarray(sizes, np.int64), out=off[1:])
    return off


def word_base(sizes):
    wb = [0]
    for s in sizes:
        wb.append(wb[-1] + (s + 31) // 32)
    return wb


def pack_ref(mask: np.ndarray) -> np.ndarray:
    """Pack booleans LSB-first into uint32 words with numpy (independent packer)."""
    nw = (len(mask) + 31) // 32
    padded = np.zeros(nw * 32, np.uint8)
    padded[: len(mask)] = mask
    return np.packbits(padded, bitorder="little").view("<u4").astype(np.uint32)


def unpack_ref(words: np.ndarray, nk: int) -> np.ndarray:
    bits = np.unpackbits(np.ascontiguousarray(words, dtype="<u4").view(np.uint8), bitorder="little")
    return bits[:nk].astype(bool)


def ulp32(x) -> np.ndarray:
    return np.spacing(np.abs(np.asarray(x, np.float32))).astype(np.float64)


# -- hand-worked cases ----------------------------------------------------------

def _case_c(case) -> np.ndarray:
    if "c" in case:
        return np.array([float(v) for v in case["c"]], np.float32)
    name = case["name"]
    if name.startswith("n33"):
        return np.array([(-1) ** i * (i + 1) for i in range(33)], np.float32)
    if name.startswith("n64"):
        return np.array([i - 31.5 for i in range(64)], np.float32)
    raise KeyError(name)


def pin_hand_cases(o):
    cases = json.load(open(os.path.join(GOLDEN, "pack_hand_cases.json")))["cases"]
    for case in cases:
        c = _case_c(case)
        n = len(c)
        g = c[None, :].copy()
        err = np.zeros_like(g)
        bits, s, flags = o.compress([0, n], g, err)
        want_words = [int(w, 16) for w in case["words"]]
        assert [int(x) for x in bits[0]] == want_words, (case["name"], [hex(x) for x in bits[0]])
        assert sum(bin(int(x)).count("1") for x in bits[0]) == case["popcount"], case["name"]
        assert flags == 0
        s_exact = math.sqrt(float(Fraction(case["s_squared"])))
        assert abs(float(s[0, 0]) - s_exact) <= ulp32(s_exact), (case["name"], s[0, 0], s_exact)
        assert Fraction(case["sum_sq"]) == sum(Fraction(float(x)) ** 2 for x in c)
        sign = np.where(unpack_ref(bits[0], n), 1.0, -1.0)
        want_err = c.astype(np.float64) - float(s[0, 0]) * sign
        assert np.all(np.abs(err[0] - want_err) <= 0.5 * ulp32(err[0])), case["name"]


# -- worker stage invariants ----------------------------------------------------

RAGGED = [33, 64, 1, 100, 0, 257, 31, 32]


def _worker_inputs(W, sizes, key, gscale=1e-3, escale=1e-3):
    n = int(sum(sizes))
    g = aux_normal(SEED, (1, *key), W * n, gscale).reshape(W, n)
    err = aux_normal(SEED, (2, *key), W * n, escale).reshape(W, n)
    return g, err


def pin_worker_invariants(o):
    W, sizes = 3, RAGGED
    off, wb = offsets_of(sizes), word_base(sizes)
    g, err0 = _worker_inputs(W, sizes, (10,))
    err = err0.copy()
    bits, s, flags = o.compress(off, g, err)
    assert flags == 0
    assert bits.shape == (W, wb[-1]) and s.shape == (W, len(sizes))
    c = g + err0  # float32 addition: the compensated gradient
    for w in range(W):
        for k, nk in enumerate(sizes):
            lo, hi = off[k], off[k + 1]
            q = bits[w, wb[k]: wb[k + 1]]
            ck = c[w, lo:hi]
            # packing: LSB-first, bit = (c >= 0), fresh word per chunk, zero padding
            assert np.array_equal(q, pack_ref(ck >= 0)), (w, k)
            assert sum(bin(int(x)).count("1") for x in q) == int(np.count_nonzero(ck >= 0))
            if nk == 0:
                assert s[w, k] == 0.0
                continue
            # scale: ||s * sign(c)||_2 = s sqrt(n) = ||c||_2
            norm = np.linalg.norm(ck.astype(np.float64))
            assert abs(float(s[w, k]) * math.sqrt(nk) - norm) <= 2e-7 * norm, (w, k)
            # error: c = s*sign(c) + err, exact up to one rounding of err
            sign = np.where(unpack_ref(q, nk), 1.0, -1.0)
            exact = ck.astype(np.float64) - float(s[w, k]) * sign
            assert np.all(np.abs(err[w, lo:hi] - exact) <= 0.5 * ulp32(err[w, lo:hi])), (w, k)


def pin_chunk_independence(o):
    """A multi-chunk call equals the chunks compressed one at a time."""
    W, sizes = 2, RAGGED
    off, wb = offsets_of(sizes), word_base(sizes)
    g, err0 = _worker_inputs(W, sizes, (11,))
    err = err0.copy()
    bits, s, _ = o.compress(off, g, err)
    for k, nk in enumerate(sizes):
        lo, hi = off[k], off[k + 1]
        ek = np.ascontiguousarray(err0[:, lo:hi])
        bk, sk, _ = o.compress([0, nk], np.ascontiguousarray(g[:, lo:hi]), ek)
        assert np.array_equal(bk, bits[:, wb[k]: wb[k + 1]]), k
        assert np.array_equal(sk[:, 0], s[:, k]), k
        assert np.array_equal(ek, err[:, lo:hi]), k


def pin_clip(o):
    g = np.array([[10.0, -10.0, 3.0, -7.0]], np.float32)
    e = np.zeros_like(g)
    _, s, _ = o.compress([0, 4], g, e, clip=5.0)
    assert abs(float(s[0, 0]) - math.sqrt(21.0)) <= ulp32(math.sqrt(21.0))  # c = [5,-5,3,-5]
    want = np.array([5 - math.sqrt(21), -5 + math.sqrt(21), 3 - math.sqrt(21), -5 + math.sqrt(21)])
    assert np.all(np.abs(e[0] - want) <= ulp32(math.sqrt(21.0)) + ulp32(want))
    e = np.zeros_like(g)
    _, s, _ = o.compress([0, 4], g, e, clip=0.0)
    assert abs(float(s[0, 0]) - math.sqrt(64.5)) <= ulp32(math.sqrt(64.5))  # no clip


def pin_nonfinite(o):
    g = np.array([[1.0, float("nan"), -2.0, 0.5]], np.float32)
    e = np.zeros_like(g)
    bits, s, flags = o.compress([0, 4], g, e)
    assert flags & 1
    assert int(bits[0, 0]) == 0b1001  # NaN quantises to -1 (bit 0)
    g = np.array([[1.0, 2.0, -2.0, 0.5]], np.float32)
    e = np.zeros_like(g)
    _, _, flags = o.compress([0, 4], g, e)
    assert flags == 0


# bfloat16 bit patterns with their exact values, decoded by hand:
# 0x3C23 = +2^(120-127) * (1 + 35/128);  0xBA83 = -2^(117-127) * (1 + 3/128)
BF16_TABLE = [(0x3F80, 1.0), (0xBF80, -1.0), (0x4040, 3.0), (0x3F00, 0.5), (0xC0A0, -5.0),
              (0x0000, 0.0), (0x8000, -0.0), (0x3C23, 0.00994873046875),
              (0xBA83, -0.00099945068359375)]


def pin_bf16(o):
    bits16 = np.array([[b for b, _ in BF16_TABLE]], np.uint16)
    vals = np.array([[v for _, v in BF16_TABLE]], np.float32)
    n = bits16.shape[1]
    e1, e2 = np.zeros((1, n), np.float32), np.zeros((1, n), np.float32)
    b1, s1, _ = o.compress([0, n], bits16, e1)
    b2, s2, _ = o.compress([0, n], vals, e2)
    assert np.array_equal(b1, b2) and np.array_equal(s1, s2) and np.array_equal(e1, e2)


def pin_empty_chunk(o):
    sizes = [0, 8, 0]
    g = np.array([[0.5, -1, 0, 2, -0.0, -3, 1, -2]], np.float32)
    e = np.zeros_like(g)
    bits, s, _ = o.compress(offsets_of(sizes), g, e)
    assert bits.shape == (1, 1) and int(bits[0, 0]) == 0x5D
    assert s[0, 0] == 0.0 and s[0, 2] == 0.0 and s[0, 1] > 0


def _bf16_of(a: np.ndarray) -> np.ndarray:
    """float32 -> bfloat16 patterns with torch's conversion (round to nearest even)."""
    import torch
    return torch.from_numpy(np.ascontiguousarray(a, np.float32)).to(torch.bfloat16) \
        .view(torch.int16).numpy().view(np.uint16)


def _widen(b: np.ndarray) -> np.ndarray:
    return (b.astype(np.uint32) << np.uint32(16)).view(np.float32)


def pin_bf16_error_storage(o):
    """Error buffers stored as bfloat16 hold the float32 results rounded to
    nearest-even (checked against torch's conversion, on data with exact ties),
    and the next step reads them back widened exactly."""
    W, sizes = 2, [1 << 18, 1000, 33]
    off = offsets_of(sizes)
    n = int(off[-1])
    g = aux_normal(SEED, (90,), W * n, 1e-3).reshape(W, n)
    e32 = np.zeros((W, n), np.float32)
    e16 = np.zeros((W, n), np.uint16)
    b32, s32, _ = o.compress(off, g, e32)
    b16, s16, _ = o.compress(off, g, e16)
    assert np.array_equal(b32, b16) and np.array_equal(s32, s16)
    ties = (e32.view(np.uint32) & np.uint32(0xFFFF)) == np.uint32(0x8000)
    assert ties.sum() >= 1, "no exact bfloat16 ties in the data"
    assert np.array_equal(e16, _bf16_of(e32))
    # step 2 from the stored bfloat16 errors == float32 mode fed their widened values
    g2 = aux_normal(SEED, (91,), W * n, 1e-3).reshape(W, n)
    e32b = _widen(e16)
    o.compress(off, g2, e32b)
    o.compress(off, g2, e16)
    assert np.array_equal(e16, _bf16_of(e32b))
    # server error buffer, from a state both modes can hold
    srv16 = _bf16_of(aux_normal(SEED, (92,), n, 1e-3))
    srv32 = _widen(srv16)
    bs32, ss32, _ = o.server_reduce(off, b32, s32, srv32)
    bs16, ss16, _ = o.server_reduce(off, b32, s32, srv16)
    assert np.array_equal(bs32, bs16) and np.array_equal(ss32, ss16)
    assert np.array_equal(srv16, _bf16_of(srv32))


# -- server stage ----------------------------------------------------------------

def pin_server_single_worker(o):
    """W = 1 and a zero server error: the server re-quantisation is the identity."""
    sizes = [40, 64, 1, 77]
    off = offsets_of(sizes)
    g, err = _worker_inputs(1, sizes, (20,))
    bits_w, s_w, _ = o.compress(off, g, err)
    srv_err = np.zeros(off[-1], np.float32)
    bits_srv, s_srv, _ = o.server_reduce(off, bits_w, s_w, srv_err)
    assert np.array_equal(bits_srv, bits_w[0])
    assert np.array_equal(s_srv, s_w[0])
    assert np.all(srv_err == 0.0)


def pin_server_identical_workers(o):
    sizes = [40, 64, 1, 77]
    off = offsets_of(sizes)
    for W in (2, 4):
        g1, e1 = _worker_inputs(1, sizes, (21,))
        g, err = np.repeat(g1, W, 0), np.repeat(e1, W, 0)
        bits_w, s_w, _ = o.compress(off, g, err)
        srv_err = np.zeros(off[-1], np.float32)
        bits_srv, s_srv, _ = o.server_reduce(off, bits_w, s_w, srv_err)
        assert np.array_equal(bits_srv, bits_w[0]) and np.array_equal(s_srv, s_w[0]), W
        assert np.all(srv_err == 0.0), W


def pin_server_opposite_workers(o):
    """Two workers with opposite gradients: the scaled signs cancel exactly."""
    sizes = [40, 64, 33]
    off, wb = offsets_of(sizes), word_base(sizes)
    g1, _ = _worker_inputs(1, sizes, (22,))
    g = np.concatenate([g1, -g1])
    err = np.zeros_like(g)
    bits_w, s_w, _ = o.compress(off, g, err)
    srv_err = np.zeros(off[-1], np.float32)
    bits_srv, s_srv, _ = o.server_reduce(off, bits_w, s_w, srv_err)
    assert np.all(s_srv == 0.0)
    assert np.all(srv_err == 0.0)
    for k, nk in enumerate(sizes):
        assert np.array_equal(bits_srv[wb[k]: wb[k + 1]], pack_ref(np.ones(nk, bool)))


def pin_server_bruteforce(o):
    """Exact rational reconstruction of the server stage on tiny random inputs."""
    sizes = [5, 32, 33, 64, 17]
    off, wb = offsets_of(sizes), word_base(sizes)
    n = int(off[-1])
    for W in (1, 2, 3, 4):
        bits_w = np.stack([aux_bits(SEED, (30, W, w), wb[-1]) for w in range(W)])
        for w in range(W):  # padding bits must be zero on input as well
            for k, nk in enumerate(sizes):
                bits_w[w, wb[k]: wb[k + 1]] &= pack_ref(np.ones(nk, bool))
        s_w = aux_uniform(SEED, (31, W), W * len(sizes), 0.1, 2.0).reshape(W, len(sizes))
        srv0 = aux_normal(SEED, (32, W), n, 0.5)
        srv_err = srv0.copy()
        bits_srv, s_srv, _ = o.server_reduce(off, bits_w, s_w, srv_err)
        for k, nk in enumerate(sizes):
            lo = int(off[k])
            exact = []
            for i in range(nk):
                acc = Fraction(0)
                for w in range(W):
                    bit = unpack_ref(bits_w[w, wb[k]: wb[k + 1]], nk)[i]
                    acc += Fraction(float(s_w[w, k])) * (1 if bit else -1)
                exact.append(acc / W + Fraction(float(srv0[lo + i])))
            ex = np.array([float(x) for x in exact])
            mag = np.max(np.abs(s_w[:, k])) + np.max(np.abs(srv0[lo: lo + nk]))
            tol = (W + 3) * float(np.spacing(np.float32(mag)))
            s_exact = math.sqrt(float(sum(x * x for x in exact)) / nk)
            assert abs(float(s_srv[k]) - s_exact) <= 4 * tol, (W, k)
            sgn = unpack_ref(bits_srv[wb[k]: wb[k + 1]], nk)
            clear = np.abs(ex) > tol
            assert np.array_equal(sgn[clear], ex[clear] >= 0), (W, k)
            rec = srv_err[lo: lo + nk].astype(np.float64) + float(s_srv[k]) * np.where(sgn, 1.0, -1.0)
            assert np.all(np.abs(rec - ex) <= 2 * tol), (W, k)
            assert np.array_equal(bits_srv[wb[k]: wb[k + 1]], pack_ref(sgn))


def pin_error_feedback_telescopes(o):
    """Over T steps the transmitted directions add up to the gradients minus the
    final residuals:  sum_t g_hat_t = mean_w(sum_t g_w,t - err_w,T) - srv_err_T."""
    W, T, sizes = 3, 6, [50, 64, 33]
    off, wb = offsets_of(sizes), word_base(sizes)
    n = int(off[-1])
    st = {"p": aux_normal(SEED, (40,), n, 0.02), "m": np.zeros(n, np.float32),
          "v": aux_uniform(SEED, (41,), n, 1e-8, 1e-6),
          "err": np.zeros((W, n), np.float32), "srv_err": np.zeros(n, np.float32)}
    gsum = np.zeros((W, n))
    ghat_sum = np.zeros(n)
    for t in range(T):
        g = aux_normal(SEED, (42, t), W * n, 1e-3).reshape(W, n)
        gsum += g
        o.step(off, g, st, B1, LR, EPS)
        for k, nk in enumerate(sizes):
            sg = np.where(unpack_ref(st["bits_srv"][wb[k]: wb[k + 1]], nk), 1.0, -1.0)
            ghat_sum[off[k]: off[k + 1]] += float(st["s_srv"][k]) * sg
    want = (gsum - st["err"]).mean(0) - st["srv_err"]
    assert np.max(np.abs(ghat_sum - want)) <= 1e-8, np.max(np.abs(ghat_sum - want))


# -- updates ---------------------------------------------------------------------

def _fixed_direction(sizes, key):
    wb = word_base(sizes)
    bits = aux_bits(SEED, key, wb[-1])
    for k, nk in enumerate(sizes):
        bits[wb[k]: wb[k + 1]] &= pack_ref(np.ones(nk, bool))
    return bits


def _ghat(bits, s, sizes):
    wb = word_base(sizes)
    out = []
    for k, nk in enumerate(sizes):
        out.append(float(s[k]) * np.where(unpack_ref(bits[wb[k]: wb[k + 1]], nk), 1.0, -1.0))
    return np.concatenate(out)


def pin_adam_closed_form(o):
    """Constant g_hat from m = 0: m_t = (1 - b1^t) g_hat and
    p_t = p_0 - lr g_hat/(sqrt(v)+eps) * (t - b1 (1 - b1^t)/(1 - b1)); v untouched."""
    sizes, T = [40, 24], 20
    off = offsets_of(sizes)
    n = int(off[-1])
    bits = _fixed_direction(sizes, (50,))
    s = np.array([0.3, 0.7], np.float32)
    m = np.zeros(n, np.float32)
    v = aux_uniform(SEED, (51,), n, 1e-4, 1e-2)
    v0 = v.copy()
    p0 = aux_normal(SEED, (52,), n, 0.02)
    p = p0.copy()
    for _ in range(T):
        o.adam_apply(off, bits, s, m, v, p, B1, LR, EPS)
    gh = _ghat(bits, s, sizes)
    b1 = float(B1)
    assert np.allclose(m, (1 - b1 ** T) * gh, rtol=2e-6, atol=0)
    sum_m = T - b1 * (1 - b1 ** T) / (1 - b1)
    want_p = p0 - float(LR) * gh * sum_m / (np.sqrt(v0.astype(np.float64)) + float(EPS))
    assert np.max(np.abs(p - want_p)) <= 2e-7, np.max(np.abs(p - want_p))
    assert np.array_equal(v, v0)


def pin_lamb_proportional(o):
    """With u proportional to p inside a layer the trust ratio cancels the scale:
    p_new = (1 - lr) p; a zero layer takes r = 1."""
    sizes = [48, 40, 16]
    off, wb = offsets_of(sizes), word_base(sizes)
    n = int(off[-1])
    bits = _fixed_direction(sizes, (60,))
    s = np.array([0.25, 0.5, 0.125], np.float32)
    sgn = _ghat(bits, np.ones(3, np.float32), sizes)
    a = np.repeat(np.array([0.05, 2.0, 0.0]), sizes)
    p0 = (a * sgn).astype(np.float32)
    p = p0.copy()
    m = np.zeros(n, np.float32)
    v = np.full(n, 0.04, np.float32)
    r, _ = o.lamb_apply(off, bits, s, m, v, p, B1, LR, EPS)
    lr = float(LR)
    l0 = slice(0, sizes[0] + sizes[1])
    assert np.allclose(p[l0], (1 - lr) * p0[l0].astype(np.float64), rtol=1e-6, atol=0)
    beta = (1 - float(B1)) * s.astype(np.float64) / (math.sqrt(0.04) + float(EPS))
    assert abs(float(r[0]) - 0.05 / beta[0]) <= 1e-6 * 0.05 / beta[0]
    assert abs(float(r[1]) - 2.0 / beta[1]) <= 1e-6 * 2.0 / beta[1]
    assert float(r[2]) == 1.0
    u2 = (1 - float(B1)) * 0.125 * sgn[off[2]:] / (0.2 + float(EPS))
    assert np.allclose(p[off[2]:], -lr * u2, rtol=1e-6, atol=0)


def pin_lamb_step_norm(o):
    """Every LAMB update moves a layer by exactly lr * ||p_l|| (r ||u|| = ||p||)."""
    sizes = [64, 33, 100]
    off = offsets_of(sizes)
    n = int(off[-1])
    bits = _fixed_direction(sizes, (61,))
    s = np.array([1e-3, 2e-3, 5e-4], np.float32)
    p0 = aux_normal(SEED, (62,), n, 0.02)
    p = p0.copy()
    m = aux_normal(SEED, (63,), n, 1e-3)
    v = aux_uniform(SEED, (64,), n, 1e-8, 1e-6)
    o.lamb_apply(off, bits, s, m, v, p, B1, LR, EPS)
    for k in range(len(sizes)):
        sl = slice(off[k], off[k + 1])
        step = np.linalg.norm((p[sl] - p0[sl]).astype(np.float64))
        want = float(LR) * np.linalg.norm(p0[sl].astype(np.float64))
        assert abs(step - want) <= 1e-3 * want, (k, step, want)


def pin_warmup_closed_form(o):
    """From m = v = 0 with a constant gradient g (mean over workers):
    m_t = (1 - b1^t) g, v_t = (1 - b2^t) g^2, and the first Adam move is
    lr (1 - b1) g / (sqrt(1 - b2)|g| + eps)."""
    W, sizes = 4, [60, 40]
    off = offsets_of(sizes)
    n = int(off[-1])
    grads = aux_normal(SEED, (70,), W * n, 1e-3).reshape(W, n)
    gbar = grads.astype(np.float64).mean(0)
    m, v = np.zeros(n, np.float32), np.zeros(n, np.float32)
    p0 = aux_normal(SEED, (71,), n, 0.02)
    p = p0.copy()
    o.warmup(off, grads, m, v, p, B1, B2, LR, EPS)
    b1, b2, lr, eps = float(B1), float(B2), float(LR), float(EPS)
    assert np.allclose(m, (1 - b1) * gbar, rtol=1e-5, atol=0)
    assert np.allclose(v, (1 - b2) * gbar ** 2, rtol=1e-4, atol=0)
    move = lr * (1 - b1) * gbar / (math.sqrt(1 - b2) * np.abs(gbar) + eps)
    assert np.all(np.abs((p0.astype(np.float64) - p) - move) <= 2 * ulp32(p) + 1e-5 * np.abs(move))
    o.warmup(off, grads, m, v, p, B1, B2, LR, EPS)
    assert np.allclose(m, (1 - b1 ** 2) * gbar, rtol=1e-5, atol=0)
    assert np.allclose(v, (1 - b2 ** 2) * gbar ** 2, rtol=1e-4, atol=0)


def pin_warmup_lamb(o):
    """Warmup with the LAMB update: each layer moves by lr ||p_l|| along -m."""
    W, sizes = 2, [60, 40]
    off = offsets_of(sizes)
    n = int(off[-1])
    grads = aux_normal(SEED, (72,), W * n, 1e-3).reshape(W, n)
    m, v = np.zeros(n, np.float32), np.zeros(n, np.float32)
    p0 = aux_normal(SEED, (73,), n, 0.02)
    p = p0.copy()
    o.warmup(off, grads, m, v, p, B1, B2, LR, EPS, optimizer=1)
    for k in range(len(sizes)):
        sl = slice(off[k], off[k + 1])
        d = (p[sl] - p0[sl]).astype(np.float64)
        want = float(LR) * np.linalg.norm(p0[sl].astype(np.float64))
        assert abs(np.linalg.norm(d) - want) <= 1e-3 * want
        assert np.all(np.sign(d) == -np.sign(m[sl]))


def pin_step_composition(o):
    """The whole-step entry equals its three stages called in order."""
    W, sizes = 3, [50, 64, 33]
    off = offsets_of(sizes)
    n = int(off[-1])
    g = aux_normal(SEED, (80,), W * n, 1e-3).reshape(W, n)
    base = {"p": aux_normal(SEED, (81,), n, 0.02), "m": aux_normal(SEED, (82,), n, 1e-4),
            "v": aux_uniform(SEED, (83,), n, 1e-8, 1e-6),
            "err": aux_normal(SEED, (84,), W * n, 1e-4).reshape(W, n),
            "srv_err": aux_normal(SEED, (85,), n, 1e-4)}
    for opt in (0, 1):
        a = {k: v.copy() for k, v in base.items()}
        o.step(off, g, a, B1, LR, EPS, optimizer=opt)
        b = {k: v.copy() for k, v in base.items()}
        bw, sw, _ = o.compress(off, g, b["err"])
        bs, ss, _ = o.server_reduce(off, bw, sw, b["srv_err"])
        if opt == 0:
            o.adam_apply(off, bs, ss, b["m"], b["v"], b["p"], B1, LR, EPS)
        else:
            o.lamb_apply(off, bs, ss, b["m"], b["v"], b["p"], B1, LR, EPS)
        for key in ("p", "m", "err", "srv_err"):
            assert np.array_equal(a[key], b[key]), (opt, key)
        assert np.array_equal(a["bits_w"], bw) and np.array_equal(a["bits_srv"], bs)




# -- the momentum-error rule (int8 ternary codes) ---------------------------------------

def _f32(x) -> np.float32:
    return np.float32(float(x))


def code_base(sizes):
    """First 4-byte word of every chunk's codes (ceil(n_k / 4) words per chunk)."""
    cb = [0]
    for s in sizes:
        cb.append(cb[-1] + (s + 3) // 4)
    return cb


def pin_ternary_hand_cases(o):
    doc = json.load(open(os.path.join(GOLDEN, "ternary_hand_cases.json")))
    for case in doc["cases"]:
        sizes = case["sizes"]
        g = np.array([[_f32(x) for x in case["g"]]], np.float32)
        err = np.array([[_f32(x) for x in case["err0"]]], np.float32)
        codes, flags = o.ternary_compress(offsets_of(sizes), g, err, _f32(case["beta1"]))
        want = np.array([int(b, 16) for b in case["codes_bytes"]], np.uint8).view(np.int8)
        assert np.array_equal(codes[0], want), (case["name"], codes[0])
        want_err = [float(Fraction(str(x))) for x in case["err1"]]
        assert [float(x) for x in err[0]] == want_err, (case["name"], err[0])
        assert flags == 0
    srv = doc["server"]
    cw = np.array(srv["codes"], np.int8)
    out = o.ternary_server([0, cw.shape[1]], cw)
    assert [int(x) for x in out] == srv["sum"], out


def _ternary_inputs(W, sizes, key, gscale=0.3, escale=0.1):
    n = int(sum(sizes))
    g = aux_normal(SEED, (70, *key), W * n, gscale).reshape(W, n)
    err = aux_normal(SEED, (71, *key), W * n, escale).reshape(W, n)
    return g, err


def _codes_of(codes_row, sizes):
    """Unpack one row of chunk-laid codes to one value per element."""
    cb = code_base(sizes)
    return np.concatenate([codes_row[4 * cb[k]: 4 * cb[k] + nk] for k, nk in enumerate(sizes)]) \
        if sizes else np.zeros(0, np.int8)


def pin_ternary_codes_are_signs(o):
    """Every code is numpy's sign of the compensated value g + eps (float32 sum),
    and every padding byte is 0."""
    sizes = RAGGED
    off, cb = offsets_of(sizes), code_base(sizes)
    for W in (1, 3):
        g, err = _ternary_inputs(W, sizes, (W,))
        c = g + err
        codes, flags = o.ternary_compress(off, g, err, B1)
        assert flags == 0
        for w in range(W):
            assert np.array_equal(_codes_of(codes[w], sizes), np.sign(c[w]).astype(np.int8)), W
            pad = np.ones(codes.shape[1], bool)
            for k, nk in enumerate(sizes):
                pad[4 * cb[k]: 4 * cb[k] + nk] = False
            assert not codes[w][pad].any()


def pin_ternary_error_telescopes(o):
    """eps <- beta1 eps + (1 - beta1)(c - q) with c = g + eps is
    eps <- eps + (1 - beta1)(g - q), since beta1 + (1 - beta1) = 1 exactly for the
    float32 constants; so over T steps eps_T - eps_0 = (1 - beta1) sum_t (g_t - q_t),
    up to the roundings of each step."""
    sizes, T, W = [40, 33, 64], 40, 2
    off = offsets_of(sizes)
    n = int(off[-1])
    omb1 = float(np.float32(1) - B1)
    _, err = _ternary_inputs(W, sizes, (80,))
    err0 = err.astype(np.float64)
    acc = np.zeros((W, n))
    tol = np.zeros((W, n))
    for t in range(T):
        g = aux_normal(SEED, (81, t), W * n, 0.3).reshape(W, n)
        before = err.astype(np.float64)
        codes, _ = o.ternary_compress(off, g, err, B1)
        q = np.stack([_codes_of(codes[w], sizes) for w in range(W)]).astype(np.float64)
        acc += g.astype(np.float64) - q
        mag = np.abs(g) + np.abs(before) + np.abs(q) + np.abs(err)
        tol += 4 * ulp32(mag)
    diff = np.abs((err.astype(np.float64) - err0) - omb1 * acc)
    assert np.all(diff <= tol), float(np.max(diff - tol))


def pin_ternary_beta1_limits(o):
    """beta1 = 1 keeps the error buffer bit for bit; beta1 = 0 leaves the plain
    quantisation residual c - q."""
    sizes = [40, 33]
    off = offsets_of(sizes)
    g, err = _ternary_inputs(2, sizes, (90,))
    keep = err.copy()
    o.ternary_compress(off, g, err, np.float32(1.0))
    assert np.array_equal(err.view(np.uint32), keep.view(np.uint32))
    c = g + keep
    o.ternary_compress(off, g, err, np.float32(0.0))
    assert np.array_equal(err, c - np.sign(c))


def pin_ternary_server_bruteforce(o):
    """The server sum equals an integer brute-force sum of the unpacked codes, for
    W up to 127 (all +1 and all -1 reach the int8 limits); padding stays 0."""
    sizes = RAGGED
    off, cb = offsets_of(sizes), code_base(sizes)
    nb = 4 * cb[-1]
    for W in (1, 2, 5, 127):
        u = aux_uniform(SEED, (100, W), W * int(off[-1]), 0.0, 3.0).reshape(W, -1)
        vals = np.floor(u).astype(np.int64) - 1
        vals = np.clip(vals, -1, 1)
        if W == 127:
            vals[:, :5] = 1
            vals[:, 5:10] = -1
        codes = np.zeros((W, nb), np.int8)
        for w in range(W):
            for k, nk in enumerate(sizes):
                codes[w, 4 * cb[k]: 4 * cb[k] + nk] = vals[w, off[k]: off[k + 1]]
        out = o.ternary_server(off, codes)
        want = [sum(int(vals[w, i]) for w in range(W)) for i in range(int(off[-1]))]
        assert [int(x) for x in _codes_of(out, sizes)] == want, W
        pad = np.ones(nb, bool)
        for k, nk in enumerate(sizes):
            pad[4 * cb[k]: 4 * cb[k] + nk] = False
        assert not out[pad].any()
    try:
        o.ternary_server(off, np.zeros((128, nb), np.int8))
    except ValueError:
        pass
    else:
        raise AssertionError("W = 128 accepted: the int8 code sum could overflow")


def pin_ternary_adam_closed_form(o):
    """Constant code sums per chunk with W = 4 give g_hat in {1, -1/2, 0, 3/4}
    exactly; then m_t = (1 - b1^t) g_hat and p follows the closed form of
    pin_adam_closed_form; v untouched."""
    sizes, T, W = [8, 12, 5, 9], 20, 4
    off, cb = offsets_of(sizes), code_base(sizes)
    n = int(off[-1])
    sums = [4, -2, 0, 3]
    codes = np.zeros(4 * cb[-1], np.int8)
    gh = np.zeros(n)
    for k, nk in enumerate(sizes):
        codes[4 * cb[k]: 4 * cb[k] + nk] = sums[k]
        gh[off[k]: off[k + 1]] = sums[k] / W
    m = np.zeros(n, np.float32)
    v = aux_uniform(SEED, (110,), n, 1e-4, 1e-2)
    v0 = v.copy()
    p0 = aux_normal(SEED, (111,), n, 0.02)
    p = p0.copy()
    for _ in range(T):
        _, flags = o.ternary_apply(off, W, codes, m, v, p, B1, LR, EPS)
        assert flags == 0
    b1 = float(B1)
    assert np.allclose(m, (1 - b1 ** T) * gh, rtol=2e-6, atol=0)
    sum_m = T - b1 * (1 - b1 ** T) / (1 - b1)
    want_p = p0 - float(LR) * gh * sum_m / (np.sqrt(v0.astype(np.float64)) + float(EPS))
    assert np.max(np.abs(p - want_p)) <= 2e-7, np.max(np.abs(p - want_p))
    assert np.array_equal(v, v0)


def pin_ternary_lamb_proportional(o):
    """LAMB with the momentum-error rule: a layer whose u = m/(sqrt v + eps) is
    proportional to p (constant g_hat, v and p of one sign) moves to (1 - lr) p;
    a layer with all codes 0 has u = 0, r = 1 and keeps p."""
    sizes, W = [16, 12], 2
    off, cb = offsets_of(sizes), code_base(sizes)
    n = int(off[-1])
    codes = np.zeros(4 * cb[-1], np.int8)
    codes[: sizes[0]] = 2                   # g_hat = 1 on layer 0, 0 on layer 1
    m = np.zeros(n, np.float32)
    v = np.full(n, 0.25, np.float32)
    p = np.concatenate([np.full(sizes[0], 0.3), aux_normal(SEED, (120,), sizes[1], 0.02)]).astype(np.float32)
    p0 = p.copy()
    lr = np.float32(0.01)
    r, flags = o.ternary_apply(off, W, codes, m, v, p, B1, lr, EPS, optimizer=1)
    assert flags == 0
    assert np.allclose(p[: sizes[0]], (1 - float(lr)) * 0.3, rtol=1e-6)
    assert np.array_equal(p[sizes[0]:], p0[sizes[0]:]) and float(r[1]) == 1.0
    u0 = float(np.float32(1) - B1) / (0.5 + float(EPS))
    assert abs(float(r[0]) - 0.3 / u0) <= 1e-6 * 0.3 / u0


def pin_ternary_step_composition(o):
    """The whole step equals worker stage -> server sum -> update, Adam and LAMB."""
    sizes, W = [40, 33, 64, 0, 7], 3
    off = offsets_of(sizes)
    n = int(off[-1])
    for opt in (0, 1):
        g, err = _ternary_inputs(W, sizes, (130, opt))
        st = {"p": aux_normal(SEED, (131,), n, 0.02), "m": aux_normal(SEED, (132,), n, 1e-3),
              "v": aux_uniform(SEED, (133,), n, 1e-8, 1e-6), "err": err.copy()}
        ref = {k: v.copy() for k, v in st.items()}
        flags = o.ternary_step(off, g, st, B1, LR, EPS, optimizer=opt)
        codes, f1 = o.ternary_compress(off, g, ref["err"], B1)
        srv = o.ternary_server(off, codes)
        _, f2 = o.ternary_apply(off, W, srv, ref["m"], ref["v"], ref["p"], B1, LR, EPS, optimizer=opt)
        assert flags == f1 | f2
        for k in ("p", "m", "v", "err"):
            assert np.array_equal(st[k], ref[k]), (opt, k)
        assert np.array_equal(st["codes_w"], codes) and np.array_equal(st["codes_srv"], srv)


def pin_ternary_nonfinite(o):
    """A NaN gradient gives code 0 and a NaN error; +inf gives code +1 and an
    infinite error; both raise the flag (the check after the error update).
    Large finite values do not."""
    off = [0, 4]
    g = np.array([[np.nan, np.inf, -3e38, 1.0]], np.float32)
    err = np.zeros_like(g)
    codes, flags = o.ternary_compress(off, g, err, B1)
    assert flags == 1
    assert [int(x) for x in codes[0][:4]] == [0, 1, -1, 1]
    assert np.isnan(err[0, 0]) and np.isposinf(err[0, 1]) and np.isfinite(err[0, 2:]).all()
    g2 = np.array([[-3e38, 3e38, 0.0, 1.0]], np.float32)
    _, flags = o.ternary_compress(off, g2, np.zeros_like(g2), B1)
    assert flags == 0


def pin_ternary_clip(o):
    """clip > 0 clamps the raw gradient before eps is added: a clipped run equals
    the run on numpy's clamped gradient, bit for bit; NaN passes through."""
    sizes = [40, 33]
    off = offsets_of(sizes)
    g, err = _ternary_inputs(2, sizes, (140,), gscale=8.0)
    e1, e2 = err.copy(), err.copy()
    c1, _ = o.ternary_compress(off, g, e1, B1, clip=5.0)
    c2, _ = o.ternary_compress(off, np.clip(g, -5, 5).astype(np.float32), e2, B1)
    assert np.array_equal(c1, c2) and np.array_equal(e1, e2)
    assert np.abs(g).max() > 5


def pin_ternary_bf16(o):
    """bf16 gradients widen exactly (same result as their float32 values); bf16
    error storage keeps torch's round-to-nearest-even bfloat16 of the float32
    result."""
    sizes = RAGGED
    off = offsets_of(sizes)
    g, err = _ternary_inputs(2, sizes, (150,))
    gb = _bf16_of(g)
    eb = _bf16_of(err)
    e32 = _widen(eb)
    c_b, _ = o.ternary_compress(off, gb, eb, B1)
    c_f, _ = o.ternary_compress(off, _widen(gb), e32, B1)
    assert np.array_equal(c_b, c_f)
    assert np.array_equal(eb, _bf16_of(e32))




# -- 2-bit Adam (two residual sign planes) ----------------------------------------------

def _twobit_case_c(case):
    if "c" in case:
        return np.array(case["c"], np.float32)
    return np.array([(-1) ** i * 3.0 for i in range(33)] + [2, -2, 2, -2], np.float32)


def pin_twobit_hand_cases(o):
    doc = json.load(open(os.path.join(GOLDEN, "twobit_hand_cases.json")))
    for case in doc["cases"]:
        c = _twobit_case_c(case)
        sizes = case["sizes"]
        g = c[None, :].copy()
        err = np.zeros_like(g)
        bits, s, flags = o.twobit_compress(offsets_of(sizes), g, err)
        assert [int(x) for x in bits[0]] == [int(w, 16) for w in case["words"]], (case["name"], bits)
        s1sq = case["s1_squared"] if isinstance(case["s1_squared"], list) else [case["s1_squared"]]
        s2sq = case["s2_squared"] if isinstance(case["s2_squared"], list) else [case["s2_squared"]]
        for k in range(len(sizes)):
            for plane, sq in ((0, s1sq[k]), (1, s2sq[k])):
                want = math.sqrt(float(Fraction(sq)))
                assert abs(float(s[0, k, plane]) - want) <= ulp32(want), (case["name"], k, plane)
        if "r" in case:
            r = np.array(case["r"], np.float64)
            sign2 = np.where(r >= 0, 1.0, -1.0)
            want_err = r - float(s[0, 0, 1]) * sign2
            assert np.all(np.abs(err[0] - want_err) <= 0.5 * ulp32(err[0])), case["name"]
        assert flags == 0


def pin_twobit_is_one_bit_twice(o):
    """Plane 1 and s1 are the 1-bit stage of c; plane 2, s2 and the error are the
    1-bit stage of the 1-bit residual (with a zero error buffer) -- bit for bit."""
    sizes = RAGGED
    off, wb = offsets_of(sizes), word_base(sizes)
    for W, clip in ((1, 0.0), (3, 0.0), (2, 2e-3)):
        g, err = _worker_inputs(W, sizes, (160, W))
        e2 = err.copy()
        bits2, s2, f2 = o.twobit_compress(off, g, e2, clip=clip)
        e1 = err.copy()
        b1, s1, _ = o.compress(off, g, e1, clip=clip)
        zero = np.zeros_like(e1)
        b1b, s1b, _ = o.compress(off, e1.copy(), zero)
        for w in range(W):
            for k, nk in enumerate(sizes):
                nw = wb[k + 1] - wb[k]
                base = 2 * wb[k]
                assert np.array_equal(bits2[w, base: base + nw], b1[w, wb[k]: wb[k + 1]]), (W, k, 1)
                assert np.array_equal(bits2[w, base + nw: base + 2 * nw], b1b[w, wb[k]: wb[k + 1]]), (W, k, 2)
        assert np.array_equal(s2[:, :, 0], s1) and np.array_equal(s2[:, :, 1], s1b)
        assert np.array_equal(e2, zero), W
        assert f2 == 0


def pin_twobit_residual_norm_identity(o):
    """sum r^2 = sum c^2 - 2 s1 sum |c| + n s1^2 for r = c - s1 sign(c): the second
    scale agrees with the closed form of the first plane's residual norm."""
    sizes = [40, 64, 257, 1000]
    off = offsets_of(sizes)
    g, err = _worker_inputs(2, sizes, (170,))
    c = (g + err).astype(np.float64)
    _, s, _ = o.twobit_compress(off, g, err.copy())
    for w in range(2):
        for k, nk in enumerate(sizes):
            ck = c[w, off[k]: off[k + 1]]
            s1 = float(s[w, k, 0])
            r2 = (ck ** 2).sum() - 2 * s1 * np.abs(ck).sum() + nk * s1 * s1
            assert abs(float(s[w, k, 1]) - math.sqrt(r2 / nk)) <= 1e-5 * math.sqrt(r2 / nk), (w, k)


def _ghat2(bits, s, sizes):
    wb = word_base(sizes)
    out = []
    for k, nk in enumerate(sizes):
        nw = wb[k + 1] - wb[k]
        base = 2 * wb[k]
        p1 = np.where(unpack_ref(bits[base: base + nw], nk), 1.0, -1.0)
        p2 = np.where(unpack_ref(bits[base + nw: base + 2 * nw], nk), 1.0, -1.0)
        out.append(float(s[k, 0]) * p1 + float(s[k, 1]) * p2)
    return np.concatenate(out)


def pin_twobit_error_feedback_telescopes(o):
    """With two planes the two-level error feedback still telescopes:
    sum_t g_hat_t = mean_w(sum_t g_w,t - err_w,T) - srv_err_T."""
    W, T, sizes = 3, 6, [50, 64, 33]
    off = offsets_of(sizes)
    n = int(off[-1])
    st = {"p": aux_normal(SEED, (180,), n, 0.02), "m": np.zeros(n, np.float32),
          "v": aux_uniform(SEED, (181,), n, 1e-8, 1e-6),
          "err": np.zeros((W, n), np.float32), "srv_err": np.zeros(n, np.float32)}
    gsum = np.zeros((W, n))
    ghat_sum = np.zeros(n)
    for t in range(T):
        g = aux_normal(SEED, (182, t), W * n, 1e-3).reshape(W, n)
        gsum += g
        o.twobit_step(off, g, st, B1, LR, EPS)
        ghat_sum += _ghat2(st["bits_srv"], st["s_srv"], sizes)
    want = (gsum - st["err"]).mean(0) - st["srv_err"]
    assert np.max(np.abs(ghat_sum - want)) <= 1e-8, np.max(np.abs(ghat_sum - want))


def pin_twobit_server_special_cases(o):
    """Opposite workers cancel exactly, so the server quantises its own error
    (= the worker stage applied to srv_err); two identical workers equal one."""
    sizes = [40, 33, 64]
    off = offsets_of(sizes)
    n = int(off[-1])
    g, err = _worker_inputs(1, sizes, (190,))
    bits, s, _ = o.twobit_compress(off, g, err)
    bits_neg = ~bits
    srv0 = aux_normal(SEED, (191,), n, 1e-3)
    wb = word_base(sizes)
    for k, nk in enumerate(sizes):            # padding bits stay 0 in the negated message
        for base in (2 * wb[k], 2 * wb[k] + (wb[k + 1] - wb[k])):
            nw = wb[k + 1] - wb[k]
            bits_neg[0, base: base + nw] &= pack_ref(np.ones(nk, bool))
    srv = srv0.copy()
    b_s, s_s, _ = o.twobit_server(off, np.concatenate([bits, bits_neg]), np.concatenate([s, s]), srv)
    e = np.zeros((1, n), np.float32)
    b_ref, s_ref, _ = o.twobit_compress(off, srv0[None, :].copy(), e)
    assert np.array_equal(b_s, b_ref[0]) and np.array_equal(s_s, s_ref[0]) and np.array_equal(srv, e[0])
    one = srv0.copy()
    two = srv0.copy()
    b1, s1, _ = o.twobit_server(off, bits, s, one)
    b2, s2, _ = o.twobit_server(off, np.concatenate([bits, bits]), np.concatenate([s, s]), two)
    assert np.array_equal(b1, b2) and np.array_equal(s1, s2) and np.array_equal(one, two)


def pin_twobit_adam_closed_form(o):
    """Constant server planes: m_t = (1 - b1^t) g_hat with g_hat = +-s1 +-s2 per
    element, and p follows the closed form of pin_adam_closed_form."""
    sizes, T = [40, 24], 20
    off, wb = offsets_of(sizes), word_base(sizes)
    n = int(off[-1])
    bits = np.zeros(2 * wb[-1], np.uint32)
    for k, nk in enumerate(sizes):
        nw = wb[k + 1] - wb[k]
        bits[2 * wb[k]: 2 * wb[k] + nw] = _fixed_direction([nk], (200, k, 1))
        bits[2 * wb[k] + nw: 2 * wb[k + 1]] = _fixed_direction([nk], (200, k, 2))
    s = np.array([[0.3, 0.125], [0.7, 0.25]], np.float32)
    m = np.zeros(n, np.float32)
    v = aux_uniform(SEED, (201,), n, 1e-4, 1e-2)
    v0 = v.copy()
    p0 = aux_normal(SEED, (202,), n, 0.02)
    p = p0.copy()
    for _ in range(T):
        _, flags = o.twobit_apply(off, bits, s, m, v, p, B1, LR, EPS)
        assert flags == 0
    gh = _ghat2(bits, s, sizes)
    b1 = float(B1)
    assert np.allclose(m, (1 - b1 ** T) * gh, rtol=2e-6, atol=0)
    sum_m = T - b1 * (1 - b1 ** T) / (1 - b1)
    want_p = p0 - float(LR) * gh * sum_m / (np.sqrt(v0.astype(np.float64)) + float(EPS))
    assert np.max(np.abs(p - want_p)) <= 2e-7, np.max(np.abs(p - want_p))
    assert np.array_equal(v, v0)


def pin_twobit_step_composition(o):
    sizes, W = [40, 33, 64, 0, 7], 3
    off = offsets_of(sizes)
    n = int(off[-1])
    for opt in (0, 1):
        g, err = _worker_inputs(W, sizes, (210, opt))
        st = {"p": aux_normal(SEED, (211,), n, 0.02), "m": aux_normal(SEED, (212,), n, 1e-3),
              "v": aux_uniform(SEED, (213,), n, 1e-8, 1e-6), "err": err.copy(),
              "srv_err": aux_normal(SEED, (214,), n, 1e-4)}
        ref = {k: v.copy() for k, v in st.items()}
        flags = o.twobit_step(off, g, st, B1, LR, EPS, optimizer=opt)
        b, s, f1 = o.twobit_compress(off, g, ref["err"])
        bs, ss, f2 = o.twobit_server(off, b, s, ref["srv_err"])
        _, f3 = o.twobit_apply(off, bs, ss, ref["m"], ref["v"], ref["p"], B1, LR, EPS, optimizer=opt)
        assert flags == f1 | f2 | f3
        for k in ("p", "m", "v", "err", "srv_err"):
            assert np.array_equal(st[k], ref[k]), (opt, k)
        assert np.array_equal(st["bits_srv"], bs) and np.array_equal(st["s_srv"], ss)




# -- monitoring: the quantisation rate ---------------------------------------------------

def pin_sign_rates_hand_cases(o):
    """The hand-worked packing cases: rate = popcount / n (5/8, 17/33, 32/64)."""
    cases = json.load(open(os.path.join(GOLDEN, "pack_hand_cases.json")))["cases"]
    for case in cases:
        c = _case_c(case)
        n = len(c)
        words = np.array([int(w, 16) for w in case["words"]], np.uint32)
        rate = o.sign_rates([0, n], words)
        assert rate.shape == (1, 1, 1)
        assert float(rate[0, 0, 0]) == float(np.float32(Fraction(case["popcount"], n))), case["name"]


def pin_sign_rates_count_real_bits_only(o):
    """Rates count the n_k real bits of each chunk: set padding bits change
    nothing; an empty chunk has rate 0; rows are independent."""
    sizes = [33, 0, 64, 5, 100]
    off, wb = offsets_of(sizes), word_base(sizes)
    c = aux_normal(SEED, (300,), 2 * int(off[-1]), 1.0).reshape(2, -1)
    rows = np.stack([np.concatenate([pack_ref(c[r, off[k]:off[k + 1]] >= 0) for k in range(len(sizes))])
                     for r in range(2)])
    want = np.zeros((2, len(sizes), 1), np.float32)
    for r in range(2):
        for k, nk in enumerate(sizes):
            if nk:
                want[r, k, 0] = np.float32(Fraction(int(np.count_nonzero(c[r, off[k]:off[k + 1]] >= 0)), nk))
    assert np.array_equal(o.sign_rates(off, rows), want)
    dirty = rows.copy()
    for k, nk in enumerate(sizes):
        if nk % 32:
            dirty[:, wb[k + 1] - 1] |= np.uint32((0xFFFFFFFF << (nk % 32)) & 0xFFFFFFFF)
    assert np.array_equal(o.sign_rates(off, dirty), want)
    assert np.array_equal(o.sign_rates(off, rows[1]), want[1:2])


def pin_sign_rates_of_the_stages(o):
    """Worker rates equal the fraction of compensated values c >= 0 (numpy, from c
    itself); the 2-bit layout has two planes per chunk, plane 1 the signs of c,
    plane 2 the bits numpy unpacks from the second plane's words."""
    W, sizes = 2, [70, 33, 0, 128]
    off = offsets_of(sizes)
    g, err0 = _worker_inputs(W, sizes, (301,))
    err = err0.copy()
    bits, _, _ = o.compress(off, g, err)
    c = g + err0
    rates = o.sign_rates(off, bits)
    err2 = err0.copy()
    bits2, _, _ = o.twobit_compress(off, g, err2)
    rates2 = o.sign_rates(off, bits2, planes=2)
    assert rates2.shape == (W, len(sizes), 2)
    base = 0
    for k, nk in enumerate(sizes):
        nw = (nk + 31) // 32
        for w in range(W):
            want = np.float32(Fraction(int(np.count_nonzero(c[w, off[k]:off[k + 1]] >= 0)), nk)) if nk else 0.0
            assert rates[w, k, 0] == want and rates2[w, k, 0] == want, (w, k)
            plane2 = unpack_ref(bits2[w, base + nw: base + 2 * nw], nk)
            want2 = np.float32(Fraction(int(plane2.sum()), nk)) if nk else 0.0
            assert rates2[w, k, 1] == want2, (w, k)
        base += 2 * nw


# -- 0/1 Adam: the local step ------------------------------------------------------------

def _local_state(sizes, W, key):
    off = offsets_of(sizes)
    n = int(off[-1])
    return off, n, {"p": aux_normal(SEED, (key, 1), n, 0.02), "m": aux_normal(SEED, (key, 2), n, 1e-3),
                    "v": aux_uniform(SEED, (key, 3), n, 1e-8, 1e-6),
                    "err": aux_normal(SEED, (key, 4), W * n, 1e-3).reshape(W, n),
                    "srv_err": aux_normal(SEED, (key, 5), n, 1e-4)}


def pin_local_step_moves_p_with_the_current_momentum(o):
    """A local step's parameter move is the compressed-phase update with beta1 = 1
    (m kept, whatever g_hat): equal p bit for bit, Adam and LAMB; m and v are
    untouched."""
    sizes = [48, 33, 0, 64]
    for opt in (0, 1):
        off, n, st = _local_state(sizes, 2, 310 + opt)
        m0, v0 = st["m"].copy(), st["v"].copy()
        p_ref = st["p"].copy()
        bits = _fixed_direction(sizes, (312,))
        s = np.array([0.5, 0.25, 0.0, 0.125], np.float32)
        if opt == 0:
            o.adam_apply(off, bits, s, st["m"].copy(), st["v"], p_ref, np.float32(1.0), LR, EPS)
        else:
            o.lamb_apply(off, bits, s, st["m"].copy(), st["v"], p_ref, np.float32(1.0), LR, EPS)
        g = aux_normal(SEED, (313,), 2 * n, 1e-3).reshape(2, n)
        flags = o.local_step(off, g, st, LR, EPS, optimizer=opt)
        assert flags == 0
        assert np.array_equal(st["p"], p_ref), opt
        assert np.array_equal(st["m"], m0) and np.array_equal(st["v"], v0)


def pin_local_steps_telescope_with_error_feedback(o):
    """Over a schedule mixing synchronised and local steps, the transmitted
    directions still add up to all the gradients minus the final residuals:
    sum over synchronised t of g_hat_t = mean_w(sum over all t of g_w,t - err_w,T)
    - srv_err_T.  The local steps' gradients are not lost."""
    W, sizes = 3, [50, 64, 33]
    off, wb = offsets_of(sizes), word_base(sizes)
    n = int(off[-1])
    st = {"p": aux_normal(SEED, (320,), n, 0.02), "m": np.zeros(n, np.float32),
          "v": aux_uniform(SEED, (321,), n, 1e-8, 1e-6),
          "err": np.zeros((W, n), np.float32), "srv_err": np.zeros(n, np.float32)}
    gsum = np.zeros((W, n))
    ghat_sum = np.zeros(n)
    for t, kind in enumerate("SLLSLSLLLS"):
        g = aux_normal(SEED, (322, t), W * n, 1e-3).reshape(W, n)
        gsum += g
        if kind == "L":
            assert o.local_step(off, g, st, LR, EPS) == 0
            continue
        o.step(off, g, st, B1, LR, EPS)
        for k, nk in enumerate(sizes):
            sg = np.where(unpack_ref(st["bits_srv"][wb[k]: wb[k + 1]], nk), 1.0, -1.0)
            ghat_sum[off[k]: off[k + 1]] += float(st["s_srv"][k]) * sg
    want = (gsum - st["err"]).mean(0) - st["srv_err"]
    assert np.max(np.abs(ghat_sum - want)) <= 2e-8, np.max(np.abs(ghat_sum - want))


def pin_local_step_clip_and_nonfinite(o):
    """The kept gradient is clipped like the worker stage's (numpy's clamp), and
    a NaN gradient raises the flag."""
    sizes = [40]
    off, n, st = _local_state(sizes, 1, 330)
    g = aux_normal(SEED, (331,), n, 3.0).reshape(1, n)
    e0 = st["err"].copy()
    assert o.local_step(off, g, st, LR, EPS, clip=2.5) == 0
    want = (np.clip(g, np.float32(-2.5), np.float32(2.5)).astype(np.float32) + e0).astype(np.float32)
    assert np.array_equal(st["err"], want)
    g[0, 7] = np.nan
    assert o.local_step(off, g, st, LR, EPS) == 1


ALL_PINS = [v for k, v in sorted(globals().items()) if k.startswith("pin_") and callable(v)]
