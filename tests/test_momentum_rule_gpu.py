"""The momentum-error rule (CANN 1-bit Adam article, sections 2.1-3.2) on the GPU
against the oracle, through the C ABI.

Stage by stage with identical input state (worker codes and errors, the code
sum, the update), then chained fused one-pass steps on ragged and aligned
layouts, warmup -> compressed, bfloat16 gradients and error buffers, clip,
LAMB, non-finite values, and the calls this rule refuses.  Codes are int8
bytes and compare bit for bit; the per-element arithmetic has no reduction, so
errors, m and p of Adam are expected to be bit-identical as well (checked at
the parity bar, with exactness reported); LAMB's trust ratio sums in a
different order and is held to the bar.
"""

import numpy as np
import pytest
import torch

import oracle
import workloads as WL
from bit_adam_error_b200 import OneBitAdam, _lib as L
from gpu_harness import F, HP, as_f32, assert_state, dev, grads_for, np_of, state_for, to_dev

pytestmark = pytest.mark.gpu

RAGGED = [1, 7, 8, 9, 31, 32, 33, 511, 512, 513, 1024, 1031, 4104, 1792, 0, 2, 5, 3000, 0, 6]
ALIGNED = [512, 8, 1536, 4352, 24, 2048, 40, 6216, 0, 65536 + 2056]
LAYOUTS = {"ragged": RAGGED, "aligned": ALIGNED}


def small(sizes, W, **kw):
    return WL.get_workload("tiny").with_(sizes=tuple(sizes), W=W, **kw)


def make_gpu(off, W, **kw):
    return OneBitAdam(off, W, rule="momentum", device=dev(), **{**HP, **kw})


def codes_np(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().view(torch.int8).numpy()


# -- stage by stage ----------------------------------------------------------------------

@pytest.mark.parametrize("layout", sorted(LAYOUTS))
@pytest.mark.parametrize("W,gdt,edt,clip", [(1, "f32", "f32", 0.0), (3, "f32", "f32", 0.0),
                                            (4, "bf16", "f32", 0.0), (2, "f32", "bf16", 5.0),
                                            (5, "bf16", "bf16", 0.0)])
def test_worker_stage(layout, W, gdt, edt, clip):
    wl = small(LAYOUTS[layout], W, grad_dtype=gdt, clip=clip, grad_scale=0.3 if not clip else 3.0)
    off = wl.offsets
    g = grads_for(wl, 0)
    e32 = WL.aux_normal(11, (W, 1), W * wl.n, 0.2).reshape(W, wl.n)
    if edt == "bf16":
        err0 = (e32.view(np.uint32) >> np.uint32(16)).astype(np.uint16)   # any bf16 patterns will do
    else:
        err0 = e32
    gpu = make_gpu(off, W, grad_dtype=gdt, clip=clip, err_dtype=edt)
    gpu.err.copy_(to_dev(err0))
    gpu.bits_w.fill_(-1)                       # padding must be written as 0
    gpu.compress(to_dev(g))
    ref_err = err0.copy()
    codes, flags = oracle.get().ternary_compress(off, g, ref_err, F["beta1"], clip=clip)
    torch.cuda.synchronize()
    assert np.array_equal(codes_np(gpu.bits_w), codes), "codes differ"
    got = np_of(gpu.err)
    assert_state("err", as_f32(got), as_f32(ref_err), off)
    assert np.array_equal(got, ref_err), "worker errors not bit-identical"
    assert gpu.status() == flags == 0


@pytest.mark.parametrize("layout", sorted(LAYOUTS))
@pytest.mark.parametrize("W", [1, 2, 5, 127])
def test_server_stage(layout, W):
    sizes = LAYOUTS[layout]
    off = small(sizes, 1).offsets
    o = oracle.get()
    nb = 4 * o.code_words_total(off)
    u = WL.aux_uniform(12, (W,), W * nb, 0.0, 3.0).reshape(W, nb)
    vals = (np.floor(u).astype(np.int64) - 1).clip(-1, 1).astype(np.int8)
    if W == 127:
        vals[:, :64] = 1
        vals[:, 64:128] = -1
    codes = np.zeros((W, nb), np.int8)        # codes only where elements are; padding 0
    cb = np.zeros(len(sizes) + 1, np.int64)
    np.cumsum([(s + 3) // 4 for s in sizes], out=cb[1:])
    for k, nk in enumerate(sizes):
        codes[:, 4 * cb[k]: 4 * cb[k] + nk] = vals[:, 4 * cb[k]: 4 * cb[k] + nk]
    gpu = make_gpu(off, W)
    gpu.bits_w.copy_(torch.from_numpy(codes.view(np.int32).copy()).to(dev()))
    gpu.server_reduce()
    want = o.ternary_server(off, codes)
    torch.cuda.synchronize()
    assert np.array_equal(codes_np(gpu.bits_srv), want)


@pytest.mark.parametrize("layout", sorted(LAYOUTS))
@pytest.mark.parametrize("W,opt", [(4, "adam"), (3, "adam"), (5, "lamb"), (2, "lamb")])
def test_update_stage(layout, W, opt):
    sizes = LAYOUTS[layout]
    off = small(sizes, 1).offsets
    n = int(off[-1])
    o = oracle.get()
    nb = 4 * o.code_words_total(off)
    sums = (np.floor(WL.aux_uniform(13, (W,), nb, 0.0, 2 * W + 1)).astype(np.int64) - W).astype(np.int8)
    p = WL.aux_normal(14, (1,), n, 0.02)
    v = WL.aux_uniform(14, (2,), n, 1e-8, 1e-6)
    m = WL.aux_normal(14, (3,), n, 1e-4)
    gpu = make_gpu(off, W, optimizer=opt, p=to_dev(p), m=to_dev(m), v=to_dev(v))
    gpu.bits_srv.copy_(torch.from_numpy(sums.view(np.int32).copy()).to(dev()))
    gpu.apply()
    mr, pr = m.copy(), p.copy()
    o.ternary_apply(off, W, sums, mr, v, pr, F["beta1"], F["lr"], F["eps"],
                    optimizer=oracle.LAMB if opt == "lamb" else oracle.ADAM)
    torch.cuda.synchronize()
    assert_state("m", np_of(gpu.m), mr, off)
    assert_state("p", np_of(gpu.p), pr, off)
    assert np.array_equal(np_of(gpu.m), mr)
    if opt == "adam":
        assert np.array_equal(np_of(gpu.p), pr), "Adam parameters not bit-identical"
    assert np.array_equal(np_of(gpu.v), v)
    assert gpu.step_count == 1


# -- whole steps --------------------------------------------------------------------------

def run_chain(wl, steps, err_dtype="f32"):
    p, v = state_for(wl)
    gpu = make_gpu(wl.offsets, wl.W, grad_dtype=wl.grad_dtype, optimizer=wl.optimizer, clip=wl.clip,
                   freeze_step=wl.freeze_step, err_dtype=err_dtype, p=to_dev(p), v=to_dev(v))
    edt = np.uint16 if err_dtype == "bf16" else np.float32
    ref = {"p": p.copy(), "m": np.zeros(wl.n, np.float32), "v": v.copy(),
           "err": np.zeros((wl.W, wl.n), edt)}
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
            flags |= o.ternary_step(wl.offsets, g, ref, F["beta1"], F["lr"], F["eps"], clip=wl.clip,
                                    optimizer=opt)
        torch.cuda.synchronize()
        for k in ("p", "m", "v", "err"):
            got = np_of(getattr(gpu, k))
            want = ref[k].reshape(got.shape)
            assert_state(f"step {t} {k}", as_f32(got), as_f32(want), wl.offsets)
            exact &= np.array_equal(got, want)
    assert gpu.status() == flags == 0
    return gpu, exact


@pytest.mark.parametrize("layout", sorted(LAYOUTS))
@pytest.mark.parametrize("W,gdt,opt,clip,edt", [(1, "bf16", "adam", 0.0, "f32"), (4, "f32", "adam", 0.0, "f32"),
                                                (3, "f32", "lamb", 0.0, "f32"), (16, "f32", "adam", 5.0, "f32"),
                                                (2, "bf16", "lamb", 0.0, "bf16"), (5, "f32", "adam", 0.0, "bf16")])
def test_fused_steps(layout, W, gdt, opt, clip, edt):
    wl = small(LAYOUTS[layout], W, grad_dtype=gdt, optimizer=opt, clip=clip,
               grad_dist="student_t_zeros" if clip else "normal", zero_frac=0.05 if clip else 0.0)
    _, exact = run_chain(wl, 5, err_dtype=edt)
    if opt == "adam":
        assert exact, "Adam steps of the momentum-error rule are not bit-identical to the oracle"


def test_warmup_then_compressed():
    wl = small(ALIGNED, 4, freeze_step=2)
    run_chain(wl, 5)


def test_fused_equals_stages():
    """One fused pass gives the state of compress -> server sum -> update."""
    wl = small(RAGGED, 3)
    p, v = state_for(wl)
    a = make_gpu(wl.offsets, 3, p=to_dev(p), v=to_dev(v))
    b = make_gpu(wl.offsets, 3, p=to_dev(p), v=to_dev(v))
    for t in range(3):
        g = to_dev(grads_for(wl, t))
        a.step(g)
        b.compress(g)
        b.server_reduce()
        b.apply()
    torch.cuda.synchronize()
    for k in ("p", "m", "err"):
        assert torch.equal(getattr(a, k), getattr(b, k)), k


def test_many_tiles_per_cta():
    wl = small([(1 << 22) + 8, 3 * (1 << 20)], 2, grad_dtype="bf16")
    run_chain(wl, 2)


def test_nonfinite_sets_status_without_trapping():
    wl = small([512, 1000, 33], 2)
    p, v = state_for(wl)
    gpu = make_gpu(wl.offsets, 2, p=to_dev(p), v=to_dev(v))
    g = grads_for(wl, 0)
    g[1, 700] = np.float32("nan")
    g[0, 1530] = np.float32("inf")
    gpu.step(to_dev(g))
    assert gpu.status() & L.OB_STATUS_NONFINITE
    assert gpu.status(clear=True) & L.OB_STATUS_NONFINITE
    assert gpu.status() == 0
    assert torch.ones(4, device=dev()).sum().item() == 4


def test_host_entry_matches_device_path():
    wl = small(ALIGNED, 2, grad_dtype="bf16")
    p, v = state_for(wl)
    a = make_gpu(wl.offsets, 2, grad_dtype="bf16", p=to_dev(p), v=to_dev(v))
    b = make_gpu(wl.offsets, 2, grad_dtype="bf16", p=to_dev(p), v=to_dev(v))
    for t in range(3):
        g = to_dev(grads_for(wl, t))
        a.step(g)
        b.step(g.cpu().pin_memory())
    torch.cuda.synchronize()
    for k in ("p", "m", "err"):
        assert torch.equal(getattr(a, k), getattr(b, k)), k


def test_refused_calls():
    off = small([1024, 40], 1).offsets
    gpu = make_gpu(off, 2)
    assert gpu.srv_err is None and gpu.s_w is None and gpu.s_srv is None
    wn, sn = gpu.error_norms()                  # worker norms only
    assert sn is None and wn.shape == (2, 2)
    stream = int(torch.cuda.current_stream().cuda_stream)
    out = torch.zeros(4, device=dev())
    with pytest.raises(L.OneBitError) as ei:    # no server error under this rule
        L.ob_error_norms(gpu.ctx, wn.data_ptr(), out.data_ptr(), stream)
    assert ei.value.code == L.OB_EINVAL
    with pytest.raises(L.OneBitError) as ei:    # int8 sums: at most 127 workers
        make_gpu(off, 128)
    assert ei.value.code == L.OB_EINVAL
    cfg, _keep = L.make_config(int(off[-1]), off, 1, rule=L.OB_RULE_MOMENTUM_ERROR)
    g = torch.zeros(int(off[-1]), device=dev())
    with pytest.raises(L.OneBitError) as ei:    # the no-alloc worker stage is the scaled rule's
        L.ob_compress_noalloc(cfg, g.data_ptr(), gpu.err.data_ptr(), gpu.bits_w.data_ptr(), 0, stream)
    assert ei.value.code == L.OB_EINVAL


def test_error_norms_of_worker_buffers():
    wl = small(RAGGED, 3)
    p, v = state_for(wl)
    gpu = make_gpu(wl.offsets, 3, p=to_dev(p), v=to_dev(v))
    for t in range(2):
        gpu.step(to_dev(grads_for(wl, t)))
    wn, _ = gpu.error_norms()
    e = np_of(gpu.err).astype(np.float64)
    off = wl.offsets
    want = np.array([[np.sqrt((e[w, off[k]:off[k + 1]] ** 2).sum()) for k in range(wl.C)] for w in range(3)])
    assert np.allclose(np_of(wn), want, rtol=1e-6, atol=0)


@pytest.mark.parametrize("rule", ["momentum", "twobit"])
def test_step_replays_from_a_cuda_graph(rule):
    """The fused step of the other rules captures into a CUDA graph too; replays
    equal eager steps bit for bit."""
    wl = WL.get_workload("tiny")
    p, v = state_for(wl)
    kw = dict(rule=rule, device=dev(), p=to_dev(p), v=to_dev(v), **HP)
    eager = OneBitAdam(wl.offsets, wl.W, **kw)
    graphed = OneBitAdam(wl.offsets, wl.W, **kw)
    G = torch.empty((wl.W, wl.n), dtype=torch.float32, device=dev())
    s = torch.cuda.Stream(device=dev())
    s.wait_stream(torch.cuda.current_stream())
    graph = torch.cuda.CUDAGraph()
    G.copy_(to_dev(grads_for(wl, 0)))
    with torch.cuda.stream(s):
        graphed.step(G)
    torch.cuda.current_stream().wait_stream(s)
    with torch.cuda.graph(graph, stream=s):
        graphed.step(G)
    graphed.set_step(1)
    eager.step(to_dev(grads_for(wl, 0)))
    for t in range(1, 4):
        gt = to_dev(grads_for(wl, t))
        eager.step(gt)
        G.copy_(gt)
        graph.replay()
    torch.cuda.synchronize()
    for k in ("p", "m", "err"):
        assert np.array_equal(np_of(getattr(eager, k)), np_of(getattr(graphed, k))), k


@pytest.mark.parametrize("rule", ["momentum", "twobit"])
def test_checkpoint_resume_bitwise(rule):
    """10 steps equal 5 steps, state_dict, a fresh optimizer, load, 5 more steps."""
    wl = small(ALIGNED, 2, freeze_step=2)
    p, v = state_for(wl)
    kw = dict(rule=rule, device=dev(), freeze_step=2, **HP)
    a = OneBitAdam(wl.offsets, 2, p=to_dev(p), v=to_dev(v), **kw)
    for t in range(10):
        a.step(to_dev(grads_for(wl, t)))
    b = OneBitAdam(wl.offsets, 2, p=to_dev(p), v=to_dev(v), **kw)
    for t in range(5):
        b.step(to_dev(grads_for(wl, t)))
    sd = b.state_dict()
    b.close()
    assert ("srv_err" in sd) == (rule == "twobit")
    c = OneBitAdam(wl.offsets, 2, **kw)
    c.load_state_dict(sd)
    assert c.step_count == 5
    for t in range(5, 10):
        c.step(to_dev(grads_for(wl, t)))
    torch.cuda.synchronize()
    for k in ("p", "m", "v", "err") + (("srv_err",) if rule == "twobit" else ()):
        assert np.array_equal(np_of(getattr(a, k)), np_of(getattr(c, k))), k
