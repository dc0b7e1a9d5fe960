"""Quantisation-rate monitoring and the 0/1 Adam local step: CUDA path
(through the C ABI, via OneBitAdam) against the CPU oracle.

* ``ob_quant_rates`` (the CANN article's section 8 quantisation-rate check):
  per-chunk fractions of elements sent as +1, for every worker and for the
  server, one plane (scaled-sign rule) or two (2-bit Adam).  Rates come from
  integer counts and one double division, so they must equal the oracle's
  bit for bit, from the GPU's own sign words and from the oracle's.
* ``ob_local_step`` ("DeepSpeed Communication Compression and Hiding",
  section "0/1 Adam"): schedules that mix synchronised compressed steps, local
  steps and variance refreshes, Adam and LAMB, float32 and bfloat16 gradients
  and error buffers, clipping, one and several workers, compared with the
  oracle after every step at the parity bar (sign words bit-exact).
"""

import numpy as np
import pytest
import torch

import oracle
import workloads as WL
from bit_adam_error_b200 import OneBitAdam, _lib as L
from gpu_harness import (F, HP, Pair, assert_bits, assert_scales, assert_state, dev, grads_for,
                         np_of, state_for, to_dev)

pytestmark = pytest.mark.gpu

RAGGED = [1, 7, 8, 9, 31, 32, 33, 511, 512, 513, 1024, 1031, 4104, 1792, 0, 2, 5, 3000, 0, 6]
ALIGNED = [512, 8, 1536, 4352, 24, 2048, 40, 6216, 0, 65536 + 2056]
LAYOUTS = {"ragged": RAGGED, "aligned": ALIGNED}


def small(sizes, W, **kw):
    return WL.get_workload("tiny").with_(sizes=tuple(sizes), W=W, **kw)


# -- quantisation rate -------------------------------------------------------------------

@pytest.mark.parametrize("layout", sorted(LAYOUTS))
@pytest.mark.parametrize("W", [1, 3, 4])
def test_quant_rates_scaled_rule(layout, W):
    wl = small(LAYOUTS[layout], W, grad_dist="student_t_zeros", zero_frac=0.05)
    p, v = state_for(wl)
    pr = Pair(wl.offsets, W, p0=p, v0=v)
    for t in range(2):
        pr.step(grads_for(wl, t), warm=False)
    wr, sr = pr.gpu.quant_rates()
    torch.cuda.synchronize()
    o = oracle.get()
    # from the GPU's own sign words, and from the oracle's (equal words)
    want_w = o.sign_rates(wl.offsets, np_of(pr.gpu.bits_w))[:, :, 0]
    want_s = o.sign_rates(wl.offsets, np_of(pr.gpu.bits_srv))[0, :, 0]
    assert np.array_equal(np_of(wr), want_w)
    assert np.array_equal(np_of(sr), want_s)
    assert np.array_equal(np_of(wr), o.sign_rates(wl.offsets, pr.ref["bits_w"])[:, :, 0])
    assert np.array_equal(np_of(sr), o.sign_rates(wl.offsets, pr.ref["bits_srv"])[0, :, 0])
    sizes = np.diff(wl.offsets)
    assert np.all(np_of(wr)[:, sizes == 0] == 0)
    big = sizes >= 4096                   # symmetric gradients: near the theoretical 1/2
    assert np.all(np.abs(np_of(wr)[:, big] - 0.5) < 0.1)
    pr.gpu.close()


def test_quant_rates_two_bit_rule():
    W = 3
    wl = small(ALIGNED, W)
    p, v = state_for(wl)
    gpu = OneBitAdam(wl.offsets, W, rule="twobit", device=dev(), p=to_dev(p), v=to_dev(v), **HP)
    gpu.step(to_dev(grads_for(wl, 0)))
    wr, sr = gpu.quant_rates()
    torch.cuda.synchronize()
    assert tuple(wr.shape) == (W, wl.C, 2) and tuple(sr.shape) == (wl.C, 2)
    o = oracle.get()
    assert np.array_equal(np_of(wr), o.sign_rates(wl.offsets, np_of(gpu.bits_w), planes=2))
    assert np.array_equal(np_of(sr), o.sign_rates(wl.offsets, np_of(gpu.bits_srv), planes=2)[0])
    gpu.close()


def test_quant_rates_refusals():
    wl = small([64, 32], 2)
    gpu = OneBitAdam(wl.offsets, 2, rule="momentum", device=dev(), **HP)
    with pytest.raises(L.OneBitError) as ei:
        gpu.quant_rates()
    assert ei.value.code == L.OB_EINVAL
    gpu.close()
    gpu = OneBitAdam(wl.offsets, 2, device=dev(), **HP)
    with pytest.raises(L.OneBitError) as ei:
        L.ob_quant_rates(gpu.ctx, 0, 0, 0)
    assert ei.value.code == L.OB_EINVAL
    gpu.close()


# -- 0/1 Adam local steps ----------------------------------------------------------------

def run_schedule(wl, schedule, *, optimizer="adam", clip=0.0, err_dtype="f32"):
    """S = synchronised compressed step, L = local step, R = variance refresh."""
    p, v = state_for(wl)
    pr = Pair(wl.offsets, wl.W, grad_dtype=wl.grad_dtype, optimizer=optimizer, clip=clip,
              err_dtype=err_dtype, p0=p, v0=v)
    o = oracle.get()
    for t, kind in enumerate(schedule):
        g = grads_for(wl, t)
        r = pr.ref
        if kind == "L":
            pr.gpu.local_step(to_dev(g))
            pr.ref_flags |= o.local_step(wl.offsets, g, r, F["lr"], F["eps"], clip=clip, optimizer=pr.opt_code)
        elif kind == "R":
            pr.gpu.refresh_step(to_dev(g))
            o.warmup(wl.offsets, g, r["m"], r["v"], r["p"], F["beta1"], F["beta2"], F["lr"], F["eps"],
                     optimizer=pr.opt_code)
        else:
            pr.step(g, warm=False)
        pr.compare(tag=f"step {t} ({kind}) ", bits=kind == "S")
    assert pr.gpu.step_count == len(schedule)
    assert pr.gpu.status() == 0 and pr.ref_flags == 0
    return pr


@pytest.mark.parametrize("layout", sorted(LAYOUTS))
@pytest.mark.parametrize("W,gdt,opt,clip", [(1, "bf16", "adam", 0.0), (3, "f32", "adam", 0.0),
                                            (2, "f32", "lamb", 0.0), (4, "bf16", "adam", 2e-3)])
def test_local_steps_between_synchronisations(layout, W, gdt, opt, clip):
    wl = small(LAYOUTS[layout], W, grad_dtype=gdt)
    run_schedule(wl, "SLLSLRSLLLS", optimizer=opt, clip=clip)


def test_local_steps_bf16_error_buffers():
    run_schedule(small(ALIGNED, 2), "SLSLLS", err_dtype="bf16")


def test_zero_length_local_phase_is_the_plain_path():
    """A schedule without local steps equals today's chained compressed steps,
    and a local phase changes p and err but not m, v or the words."""
    wl = small(ALIGNED, 2)
    a = run_schedule(wl, "SSS")
    b = run_schedule(wl, "SLS")
    torch.cuda.synchronize()
    assert not np.array_equal(np_of(a.gpu.p), np_of(b.gpu.p))
    c = run_schedule(wl, "S")
    m0, v0, bits0 = np_of(c.gpu.m).copy(), np_of(c.gpu.v).copy(), np_of(c.gpu.bits_srv).copy()
    c.gpu.local_step(to_dev(grads_for(wl, 5)))
    torch.cuda.synchronize()
    assert np.array_equal(np_of(c.gpu.m), m0) and np.array_equal(np_of(c.gpu.v), v0)
    assert np.array_equal(np_of(c.gpu.bits_srv), bits0)


def test_local_steps_two_bit_rule():
    W = 2
    wl = small(ALIGNED, W)
    p, v = state_for(wl)
    gpu = OneBitAdam(wl.offsets, W, rule="twobit", device=dev(), p=to_dev(p), v=to_dev(v), **HP)
    o = oracle.get()
    ref = {"p": p.copy(), "m": np.zeros_like(p), "v": v.copy(), "err": np.zeros((W, wl.n), np.float32),
           "srv_err": np.zeros_like(p)}
    for t, kind in enumerate("SLLS"):
        g = grads_for(wl, t)
        if kind == "L":
            gpu.local_step(to_dev(g))
            o.local_step(wl.offsets, g, ref, F["lr"], F["eps"])
        else:
            gpu.step(to_dev(g))
            o.twobit_step(wl.offsets, g, ref, F["beta1"], F["lr"], F["eps"])
        torch.cuda.synchronize()
        for key in ("p", "m", "v", "srv_err"):
            assert_state(f"step {t} {key}", np_of(getattr(gpu, key)), ref[key], wl.offsets)
        assert_state(f"step {t} err", np_of(gpu.err), ref["err"], wl.offsets)
    assert_bits("bits_srv", np_of(gpu.bits_srv), ref["bits_srv"])
    gpu.close()


def test_local_step_refusals_and_nonfinite():
    wl = small([512, 40], 2)
    warm = OneBitAdam(wl.offsets, 2, freeze_step=2, device=dev(), **HP)
    with pytest.raises(L.OneBitError) as ei:
        warm.local_step(to_dev(grads_for(wl, 0)))
    assert ei.value.code == L.OB_EPHASE and warm.step_count == 0
    warm.close()
    mom = OneBitAdam(wl.offsets, 2, rule="momentum", device=dev(), **HP)
    with pytest.raises(L.OneBitError) as ei:
        mom.local_step(to_dev(grads_for(wl, 0)))
    assert ei.value.code == L.OB_EINVAL
    mom.close()
    gpu = OneBitAdam(wl.offsets, 2, device=dev(), **HP)
    g = grads_for(wl, 0)
    g[1, 300] = np.float32("nan")
    gpu.local_step(to_dev(g))
    assert gpu.status(clear=True) & L.OB_STATUS_NONFINITE
    assert gpu.step_count == 1
    assert torch.ones(4, device=dev()).sum().item() == 4     # the context is still usable
    gpu.close()


# -- the warmup's full-precision average -------------------------------------------------

@pytest.mark.parametrize("layout", sorted(LAYOUTS))
@pytest.mark.parametrize("W,gdt", [(1, "f32"), (3, "bf16"), (4, "f32"), (5, "f32")])
def test_mean_grads_then_one_worker_warmup_equals_the_w_worker_warmup(layout, W, gdt):
    """ob_mean_grads on W gradients, then ob_warmup_step on a one-worker float32
    ctx over the average, leaves p, m, v where the oracle's W-worker warmup
    leaves them (two steps, Adam)."""
    wl = small(LAYOUTS[layout], W, grad_dtype=gdt, freeze_step=2)
    p, v = state_for(wl)
    v[:] = 0
    one = OneBitAdam(wl.offsets, 1, freeze_step=2, device=dev(), p=to_dev(p), v=to_dev(v), **HP)
    many = OneBitAdam(wl.offsets, W, grad_dtype=gdt, freeze_step=2, device=dev(), **HP)
    mean = torch.zeros(wl.n, dtype=torch.float32, device=dev())
    ref = {"p": p.copy(), "m": np.zeros_like(p), "v": v.copy()}
    o = oracle.get()
    for t in range(2):
        g = grads_for(wl, t)
        G = to_dev(g)
        L.ob_mean_grads(many.ctx, int(G.data_ptr()), int(mean.data_ptr()),
                        int(torch.cuda.current_stream().cuda_stream))
        one.step(mean.reshape(1, -1))
        o.warmup(wl.offsets, g, ref["m"], ref["v"], ref["p"], F["beta1"], F["beta2"], F["lr"], F["eps"])
    torch.cuda.synchronize()
    for key in ("p", "m", "v"):
        assert_state(key, np_of(getattr(one, key)), ref[key], wl.offsets)
    assert many.step_count == 0 and one.step_count == 2
    one.close()
    many.close()
