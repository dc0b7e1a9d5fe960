"""2-bit Adam (two residual sign planes) on the GPU against the oracle, through
the C ABI.

Stage by stage with identical input state (worker planes, scales and errors;
the server stage from seeded planes and scales; the update), then runs of fused
steps on ragged and aligned layouts (Adam, LAMB, bf16 gradients and error
buffers, clip, many workers), each step from the oracle's state, fused =
stages, and the non-finite flag.  Planes compare bit for bit, scales within
1e-5, state at the parity bar (bf16 error buffers: plus one bf16 step, see
gpu_harness).
"""

import numpy as np
import pytest
import torch

import oracle
import workloads as WL
from bit_adam_error_b200 import OneBitAdam, _lib as L
from gpu_harness import (F, HP, as_f32, assert_bits, assert_scales, assert_state, dev, grads_for, np_of,
                         state_for, sync_state, to_dev)

pytestmark = pytest.mark.gpu

RAGGED = [1, 7, 8, 9, 31, 32, 33, 511, 512, 513, 1024, 1031, 4104, 1792, 0, 2, 5, 3000, 0, 6]
ALIGNED = [512, 8, 1536, 4352, 24, 2048, 40, 6216, 0, 65536 + 2056]
LAYOUTS = {"ragged": RAGGED, "aligned": ALIGNED}


def small(sizes, W, **kw):
    return WL.get_workload("tiny").with_(sizes=tuple(sizes), W=W, **kw)


def make_gpu(off, W, **kw):
    return OneBitAdam(off, W, rule="twobit", device=dev(), **{**HP, **kw})


def word_base2(sizes):
    wb = np.zeros(len(sizes) + 1, np.int64)
    np.cumsum([2 * ((s + 31) // 32) for s in sizes], out=wb[1:])
    return wb


def seeded_planes(sizes, W, key):
    """Random sign planes with zero padding bits, [W, words2]."""
    wb = word_base2(sizes)
    out = np.zeros((W, wb[-1]), np.uint32)
    for w in range(W):
        raw = WL.aux_bits(21, (key, w), int(wb[-1]))
        for k, nk in enumerate(sizes):
            nw = (nk + 31) // 32
            mask = np.zeros(nw * 32, np.uint8)
            mask[:nk] = 1
            m = np.packbits(mask, bitorder="little").view("<u4").astype(np.uint32)
            out[w, wb[k]: wb[k] + nw] = raw[wb[k]: wb[k] + nw] & m
            out[w, wb[k] + nw: wb[k + 1]] = raw[wb[k] + nw: wb[k + 1]] & m
    return out


@pytest.mark.parametrize("layout", sorted(LAYOUTS))
@pytest.mark.parametrize("W,gdt,edt,clip", [(1, "f32", "f32", 0.0), (3, "f32", "f32", 0.0),
                                            (4, "bf16", "f32", 0.0), (2, "f32", "bf16", 2e-3),
                                            (16, "f32", "f32", 0.0)])
def test_worker_stage(layout, W, gdt, edt, clip):
    wl = small(LAYOUTS[layout], W, grad_dtype=gdt, clip=clip)
    off = wl.offsets
    g = grads_for(wl, 0)
    e32 = WL.aux_normal(22, (W,), W * wl.n, 1e-3).reshape(W, wl.n)
    err0 = (e32.view(np.uint32) >> np.uint32(16)).astype(np.uint16) if edt == "bf16" else e32
    gpu = make_gpu(off, W, grad_dtype=gdt, clip=clip, err_dtype=edt)
    gpu.err.copy_(to_dev(err0))
    gpu.bits_w.fill_(-1)
    gpu.compress(to_dev(g))
    ref_err = err0.copy()
    bits, s_w, flags = oracle.get().twobit_compress(off, g, ref_err, clip=clip)
    torch.cuda.synchronize()
    assert_bits("bits_w", np_of(gpu.bits_w), bits)
    assert_scales("s_w", np_of(gpu.s_w), s_w)
    assert_state("err", as_f32(np_of(gpu.err)), as_f32(ref_err), off)
    assert gpu.status() == flags == 0


@pytest.mark.parametrize("layout", sorted(LAYOUTS))
@pytest.mark.parametrize("W,edt", [(1, "f32"), (2, "f32"), (5, "bf16"), (16, "f32")])
def test_server_stage(layout, W, edt):
    sizes = LAYOUTS[layout]
    off = small(sizes, 1).offsets
    n = int(off[-1])
    bits_w = seeded_planes(sizes, W, 23)
    s_w = WL.aux_uniform(24, (W,), W * len(sizes) * 2, 1e-4, 1e-2).reshape(W, len(sizes), 2)
    s32 = WL.aux_normal(25, (1,), n, 1e-3)
    srv0 = (s32.view(np.uint32) >> np.uint32(16)).astype(np.uint16) if edt == "bf16" else s32
    gpu = make_gpu(off, W, err_dtype=edt)
    gpu.bits_w.copy_(to_dev(bits_w))
    gpu.s_w.copy_(to_dev(s_w))
    gpu.srv_err.copy_(to_dev(srv0))
    gpu.server_reduce()
    srv = srv0.copy()
    bits_srv, s_srv, flags = oracle.get().twobit_server(off, bits_w, s_w, srv)
    torch.cuda.synchronize()
    assert_bits("bits_srv", np_of(gpu.bits_srv), bits_srv)
    assert_scales("s_srv", np_of(gpu.s_srv), s_srv)
    assert_state("srv_err", as_f32(np_of(gpu.srv_err)), as_f32(srv), off)
    assert gpu.status() == flags == 0


@pytest.mark.parametrize("layout", sorted(LAYOUTS))
@pytest.mark.parametrize("opt", ["adam", "lamb"])
def test_update_stage(layout, opt):
    sizes = LAYOUTS[layout]
    off = small(sizes, 1).offsets
    n = int(off[-1])
    bits_srv = seeded_planes(sizes, 1, 26)[0]
    s_srv = WL.aux_uniform(27, (1,), len(sizes) * 2, 1e-4, 1e-2).reshape(len(sizes), 2)
    p = WL.aux_normal(28, (1,), n, 0.02)
    v = WL.aux_uniform(28, (2,), n, 1e-8, 1e-6)
    m = WL.aux_normal(28, (3,), n, 1e-4)
    gpu = make_gpu(off, 2, optimizer=opt, p=to_dev(p), m=to_dev(m), v=to_dev(v))
    gpu.bits_srv.copy_(to_dev(bits_srv))
    gpu.s_srv.copy_(to_dev(s_srv))
    gpu.apply()
    mr, pr = m.copy(), p.copy()
    oracle.get().twobit_apply(off, bits_srv, s_srv, mr, v, pr, F["beta1"], F["lr"], F["eps"],
                              optimizer=oracle.LAMB if opt == "lamb" else oracle.ADAM)
    torch.cuda.synchronize()
    assert_state("m", np_of(gpu.m), mr, off)
    assert_state("p", np_of(gpu.p), pr, off)
    assert np.array_equal(np_of(gpu.v), v)


def run_chain(wl, steps, err_dtype="f32", sync=True):
    p, v = state_for(wl)
    gpu = make_gpu(wl.offsets, wl.W, grad_dtype=wl.grad_dtype, optimizer=wl.optimizer, clip=wl.clip,
                   freeze_step=wl.freeze_step, err_dtype=err_dtype, p=to_dev(p), v=to_dev(v))
    edt = np.uint16 if err_dtype == "bf16" else np.float32
    ref = {"p": p.copy(), "m": np.zeros(wl.n, np.float32), "v": v.copy(),
           "err": np.zeros((wl.W, wl.n), edt), "srv_err": np.zeros(wl.n, edt)}
    o = oracle.get()
    opt = oracle.LAMB if wl.optimizer == "lamb" else oracle.ADAM
    flags = 0
    exact = True
    for t in range(steps):
        g = grads_for(wl, t)
        gpu.step(to_dev(g))
        if t < wl.freeze_step:
            flags |= o.warmup(wl.offsets, g, ref["m"], ref["v"], ref["p"], F["beta1"], F["beta2"],
                              F["lr"], F["eps"], optimizer=opt)
        else:
            flags |= o.twobit_step(wl.offsets, g, ref, F["beta1"], F["lr"], F["eps"], clip=wl.clip,
                                   optimizer=opt)
        torch.cuda.synchronize()
        for k in ("p", "m", "v", "err", "srv_err"):
            got = np_of(getattr(gpu, k))
            want = ref[k].reshape(got.shape)
            assert_state(f"step {t} {k}", as_f32(got), as_f32(want), wl.offsets,
                         bf16_step=got.dtype == np.uint16)
            exact &= np.array_equal(got, want)
        if t >= wl.freeze_step:
            assert_bits(f"step {t} bits_w", np_of(gpu.bits_w), ref["bits_w"])
            assert_bits(f"step {t} bits_srv", np_of(gpu.bits_srv), ref["bits_srv"])
            assert_scales(f"step {t} s_w", np_of(gpu.s_w), ref["s_w"])
            assert_scales(f"step {t} s_srv", np_of(gpu.s_srv), ref["s_srv"])
        if sync:
            sync_state(gpu, ref)
    assert gpu.status() == flags == 0
    return gpu, exact


@pytest.mark.parametrize("layout", sorted(LAYOUTS))
@pytest.mark.parametrize("W,gdt,opt,clip,edt", [(1, "bf16", "adam", 0.0, "f32"), (4, "f32", "adam", 0.0, "f32"),
                                                (3, "f32", "lamb", 0.0, "f32"), (16, "f32", "adam", 5.0, "f32"),
                                                (2, "bf16", "lamb", 0.0, "bf16"), (5, "f32", "adam", 0.0, "bf16")])
def test_fused_steps(layout, W, gdt, opt, clip, edt):
    wl = small(LAYOUTS[layout], W, grad_dtype=gdt, optimizer=opt, clip=clip,
               grad_dist="student_t_zeros" if clip else "normal", zero_frac=0.05 if clip else 0.0)
    _, exact = run_chain(wl, 4, err_dtype=edt)
    print(f"2-bit {layout} W={W} {gdt} {opt}: bit-identical to the oracle: {exact}")


@pytest.mark.parametrize("layout", sorted(LAYOUTS))
@pytest.mark.parametrize("W,gdt,opt,clip", [(1, "bf16", "adam", 0.0), (4, "f32", "lamb", 0.0),
                                            (16, "f32", "adam", 5.0)])
def test_fused_steps_free_running(layout, W, gdt, opt, clip):
    """Six steps with no state sync between them (f32 error buffers): the
    second scale's possible one-ulp difference does not compound into
    different planes or state beyond the bar."""
    wl = small(LAYOUTS[layout], W, grad_dtype=gdt, optimizer=opt, clip=clip,
               grad_dist="student_t_zeros" if clip else "normal", zero_frac=0.05 if clip else 0.0)
    _, exact = run_chain(wl, 6, sync=False)
    print(f"2-bit free-running {layout} W={W} {gdt} {opt}: bit-identical to the oracle: {exact}")


@pytest.mark.parametrize("W", [1, 2])
def test_equal_magnitudes_give_an_exact_zero_second_scale(W):
    """Gradients of one magnitude per chunk (random signs, the same for every
    worker): |c| equals s1 everywhere, so the residual is exactly 0 and both
    second scales are exactly 0 -- on the GPU, whose second scale comes from
    shifted tile sums of |c|, as in the oracle.  Chunks of 1, 33, 512, 1000 and
    4104 elements (ragged tiles, the scalar and 8-wide paths) and an empty one."""
    sizes = [1, 33, 512, 0, 1000, 4104]
    wl = small(sizes, W)
    p, v = state_for(wl)
    rng = np.random.default_rng(17)
    mags = np.float32([3.0517578e-05, 1e-3, 0.25, 1.0, 7.5e-4, 2.0 ** -20])
    row = np.concatenate([np.where(rng.random(n) < 0.5, -1.0, 1.0).astype(np.float32) * mags[k]
                          for k, n in enumerate(sizes)]).astype(np.float32)
    g = np.stack([row] * W)
    gpu = make_gpu(wl.offsets, W, p=to_dev(p), v=to_dev(v))
    gpu.step(to_dev(g))
    torch.cuda.synchronize()
    ref = {"p": p.copy(), "m": np.zeros(wl.n, np.float32), "v": v.copy(),
           "err": np.zeros((W, wl.n), np.float32), "srv_err": np.zeros(wl.n, np.float32)}
    o = oracle.get()
    assert o.twobit_step(wl.offsets, g, ref, F["beta1"], F["lr"], F["eps"]) == 0
    s_w, s_srv = np_of(gpu.s_w).reshape(W, len(sizes), 2), np_of(gpu.s_srv).reshape(len(sizes), 2)
    assert np.array_equal(s_w, ref["s_w"]) and np.array_equal(s_srv, ref["s_srv"])
    assert np.all(s_w[:, :, 1] == 0) and np.all(s_srv[:, 1] == 0)
    assert np.array_equal(s_w[0, :, 0], np.where(np.array(sizes) > 0, mags, 0))
    assert_bits("bits_w", np_of(gpu.bits_w), ref["bits_w"])
    assert_bits("bits_srv", np_of(gpu.bits_srv), ref["bits_srv"])
    for k in ("p", "m", "err", "srv_err"):
        assert np.array_equal(np_of(getattr(gpu, k)), ref[k].reshape(np_of(getattr(gpu, k)).shape)), k
    assert gpu.status() == 0


def test_warmup_then_compressed():
    run_chain(small(ALIGNED, 4, freeze_step=2), 5)


@pytest.mark.parametrize("W", [3, 8])
def test_fused_equals_stages(W):
    """Bit for bit; from W = 4 on the fused step's server passes read the server
    value pass 2 kept, the stage calls rebuild it."""
    wl = small(RAGGED, W)
    p, v = state_for(wl)
    a = make_gpu(wl.offsets, W, p=to_dev(p), v=to_dev(v))
    b = make_gpu(wl.offsets, W, p=to_dev(p), v=to_dev(v))
    for t in range(3):
        g = to_dev(grads_for(wl, t))
        a.step(g)
        b.compress(g)
        b.server_reduce()
        b.apply()
    torch.cuda.synchronize()
    for k in ("p", "m", "err", "srv_err", "bits_w", "s_w", "bits_srv", "s_srv"):
        assert torch.equal(getattr(a, k), getattr(b, k)), k


def test_many_tiles_per_cta():
    run_chain(small([(1 << 22) + 8, 3 * (1 << 20)], 2, grad_dtype="bf16"), 2)


def test_nonfinite_sets_status_without_trapping():
    wl = small([512, 1000, 33], 2)
    p, v = state_for(wl)
    gpu = make_gpu(wl.offsets, 2, p=to_dev(p), v=to_dev(v))
    g = grads_for(wl, 0)
    g[1, 700] = np.float32("nan")
    gpu.step(to_dev(g))
    assert gpu.status() & L.OB_STATUS_NONFINITE
    assert gpu.status(clear=True) & L.OB_STATUS_NONFINITE
    assert torch.ones(4, device=dev()).sum().item() == 4
