"""CUDA path (through the C ABI) vs the CPU oracle on identical seeded inputs.

Stage by stage (worker stage, server stage, update) with identical input state,
then whole fused steps chained, warmup -> compressed transitions, ragged layouts
(vector and scalar paths, empty chunks, tails), edge cases, error paths that
must return a status instead of faulting, determinism, checkpoint/resume and
the host-buffer entry point.  Full-size workloads are compared on sampled
chunks in test_full_size_gpu.py.
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

# Chunk layouts.  RAGGED mixes chunk starts that are / are not multiples of 8
# (vector vs scalar path), lengths around the 32-element word and the
# 512-element warp tile, empty chunks and a multi-tile tail.
RAGGED = [1, 7, 8, 9, 31, 32, 33, 511, 512, 513, 1024, 1031, 4104, 1792, 0, 2, 5, 3000, 0, 6]
ALIGNED = [512, 8, 1536, 4352, 24, 2048, 40, 6216, 0, 65536 + 2056]
LAYOUTS = {"ragged": RAGGED, "aligned": ALIGNED}


def small(sizes, W, **kw):
    return WL.get_workload("tiny").with_(sizes=tuple(sizes), W=W, **kw)


def aux_state(n, key, W=1):
    p = WL.aux_normal(7, (key, 1), n, 0.02)
    v = WL.aux_uniform(7, (key, 2), n, 1e-8, 1e-6)
    m = WL.aux_normal(7, (key, 3), n, 1e-4)
    err = WL.aux_normal(7, (key, 4), W * n, 1e-4).reshape(W, n)
    srv = WL.aux_normal(7, (key, 5), n, 1e-4)
    return p, v, m, err, srv


# -- stage by stage -------------------------------------------------------------------

@pytest.mark.parametrize("layout", sorted(LAYOUTS))
@pytest.mark.parametrize("W,gdt,clip", [(1, "f32", 0.0), (3, "f32", 0.0), (4, "bf16", 0.0),
                                        (16, "f32", 5.0), (1, "bf16", 0.0)])
def test_worker_stage(layout, W, gdt, clip):
    wl = small(LAYOUTS[layout], W, grad_dtype=gdt, grad_dist="student_t_zeros", zero_frac=0.05)
    p, v, m, err0, srv = aux_state(wl.n, 11, W)
    pr = Pair(wl.offsets, W, grad_dtype=gdt, clip=clip, p0=p, v0=v, m0=m, err0=err0, srv0=srv)
    g = grads_for(wl, 0)
    if clip:
        g[:, ::97] = np.float32(9.0)   # values the clip must cut
    pr.gpu.compress(to_dev(g))
    err = err0.copy()
    bits_w, s_w, _ = oracle.get().compress(wl.offsets, g, err, clip=clip)
    torch.cuda.synchronize()
    assert_bits("bits_w", np_of(pr.gpu.bits_w), bits_w)
    assert_scales("s_w", np_of(pr.gpu.s_w), s_w)
    assert_state("err", np_of(pr.gpu.err), err, wl.offsets)
    # the stage call leaves the rest of the state alone and does not count a step
    assert np.array_equal(np_of(pr.gpu.p), p) and np.array_equal(np_of(pr.gpu.srv_err), srv)
    assert pr.gpu.step_count == 0


def _aux_bits(sizes, W, key):
    wb = [0]
    for s in sizes:
        wb.append(wb[-1] + (s + 31) // 32)
    bits = np.stack([WL.aux_bits(9, (key, w), wb[-1]) for w in range(W)])
    return bits


@pytest.mark.parametrize("layout", sorted(LAYOUTS))
@pytest.mark.parametrize("W", [1, 2, 5, 16])
def test_server_stage(layout, W):
    sizes = LAYOUTS[layout]
    off = WL.get_workload("tiny").with_(sizes=tuple(sizes)).offsets
    n = int(off[-1])
    bits_w = _aux_bits(sizes, W, 21)
    s_w = WL.aux_uniform(9, (22,), W * len(sizes), 1e-4, 1e-2).reshape(W, len(sizes))
    srv0 = WL.aux_normal(9, (23,), n, 1e-3)
    pr = Pair(off, W, srv0=srv0)
    pr.gpu.bits_w.copy_(to_dev(bits_w))
    pr.gpu.s_w.copy_(to_dev(s_w))
    pr.gpu.server_reduce()
    srv = srv0.copy()
    bits_srv, s_srv, _ = oracle.get().server_reduce(off, bits_w, s_w, srv)
    torch.cuda.synchronize()
    assert_bits("bits_srv", np_of(pr.gpu.bits_srv), bits_srv)
    assert_scales("s_srv", np_of(pr.gpu.s_srv), s_srv)
    assert_state("srv_err", np_of(pr.gpu.srv_err), srv, off)


@pytest.mark.parametrize("layout", sorted(LAYOUTS))
@pytest.mark.parametrize("opt", ["adam", "lamb"])
def test_update_stage(layout, opt):
    sizes = LAYOUTS[layout]
    off = WL.get_workload("tiny").with_(sizes=tuple(sizes)).offsets
    n = int(off[-1])
    p, v, m, _, _ = aux_state(n, 31)
    bits_srv = _aux_bits(sizes, 1, 32)[0]
    s_srv = WL.aux_uniform(9, (33,), len(sizes), 1e-4, 1e-2)
    pr = Pair(off, 2, optimizer=opt, p0=p, v0=v, m0=m)
    pr.gpu.bits_srv.copy_(to_dev(bits_srv))
    pr.gpu.s_srv.copy_(to_dev(s_srv))
    pr.gpu.apply()
    mr, pr_ = m.copy(), p.copy()
    o = oracle.get()
    if opt == "adam":
        o.adam_apply(off, bits_srv, s_srv, mr, v, pr_, F["beta1"], F["lr"], F["eps"])
    else:
        o.lamb_apply(off, bits_srv, s_srv, mr, v, pr_, F["beta1"], F["lr"], F["eps"])
    torch.cuda.synchronize()
    assert_state("m", np_of(pr.gpu.m), mr, off)
    assert_state("p", np_of(pr.gpu.p), pr_, off)
    assert np.array_equal(np_of(pr.gpu.v), v)
    assert pr.gpu.step_count == 1


# -- whole steps -------------------------------------------------------------------------

def run_chain(wl, steps, compare_every=True, err_dtype="f32", **pair_kw):
    p, v = state_for(wl)
    pair_kw["err_dtype"] = err_dtype
    pr = Pair(wl.offsets, wl.W, grad_dtype=wl.grad_dtype, optimizer=wl.optimizer, clip=wl.clip,
              freeze_step=wl.freeze_step, p0=p, v0=v, **pair_kw)
    for t in range(steps):
        pr.step(grads_for(wl, t), warm=t < wl.freeze_step)
        if compare_every or t == steps - 1:
            pr.compare(tag=f"step {t} ", bits=t >= wl.freeze_step)
    assert pr.gpu.status() == 0      # no non-finite value, no pipeline timeout
    return pr


def test_tiny_config_ten_steps():
    wl = WL.get_workload("tiny")
    pr = run_chain(wl, wl.steps)
    print("tiny: bit-identical to the oracle:", pr.exact())


@pytest.mark.parametrize("layout", sorted(LAYOUTS))
@pytest.mark.parametrize("W,gdt,opt,clip", [(1, "bf16", "adam", 0.0), (4, "f32", "adam", 0.0),
                                            (3, "f32", "lamb", 0.0), (16, "f32", "adam", 5.0),
                                            (2, "bf16", "lamb", 0.0)])
def test_fused_steps_ragged(layout, W, gdt, opt, clip):
    wl = small(LAYOUTS[layout], W, grad_dtype=gdt, optimizer=opt, clip=clip,
               grad_dist="student_t_zeros" if clip else "normal", zero_frac=0.05 if clip else 0.0)
    run_chain(wl, 4)


@pytest.mark.parametrize("layout", sorted(LAYOUTS))
@pytest.mark.parametrize("W,gdt,opt,clip", [(1, "bf16", "adam", 0.0), (4, "f32", "lamb", 0.0),
                                            (16, "f32", "adam", 5.0), (3, "f32", "adam", 0.0)])
def test_fused_steps_bf16_error_buffers(layout, W, gdt, opt, clip):
    """Error buffers stored as bfloat16 (rounded to nearest even): every step
    equals the oracle run with the same storage."""
    wl = small(LAYOUTS[layout], W, grad_dtype=gdt, optimizer=opt, clip=clip,
               grad_dist="student_t_zeros" if clip else "normal", zero_frac=0.05 if clip else 0.0)
    pr = run_chain(wl, 4, err_dtype="bf16")
    assert pr.gpu.err.dtype == torch.bfloat16


def test_stages_bf16_error_buffers():
    """Worker and server stages alone with bfloat16 error buffers."""
    wl = small(RAGGED, 3)
    p, v, m, err0, srv = aux_state(wl.n, 41, 3)
    from oracle_pins import _bf16_of
    err0, srv = _bf16_of(err0).reshape(3, -1), _bf16_of(srv)
    pr = Pair(wl.offsets, 3, err_dtype="bf16", p0=p, v0=v, m0=m, err0=err0, srv0=srv)
    g = grads_for(wl, 0)
    pr.gpu.compress(to_dev(g))
    pr.gpu.server_reduce()
    e, sv = err0.copy(), srv.copy()
    o = oracle.get()
    bits_w, s_w, _ = o.compress(wl.offsets, g, e)
    bits_srv, s_srv, _ = o.server_reduce(wl.offsets, bits_w, s_w, sv)
    torch.cuda.synchronize()
    assert_bits("bits_w", np_of(pr.gpu.bits_w), bits_w)
    assert_bits("bits_srv", np_of(pr.gpu.bits_srv), bits_srv)
    assert np.array_equal(np_of(pr.gpu.err), e) and np.array_equal(np_of(pr.gpu.srv_err), sv)
    wn, sn = pr.gpu.error_norms()
    torch.cuda.synchronize()
    widen = lambda a: (a.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)  # noqa: E731
    off = wl.offsets
    want = np.array([np.linalg.norm(widen(sv[off[k]:off[k + 1]])) for k in range(wl.C)])
    assert_scales("server error norms", np_of(sn), want)


@pytest.mark.parametrize("opt", ["adam", "lamb"])
def test_warmup_then_compressed(opt):
    sizes = WL.configs.bert_tensor_sizes(64, 2, 256, 1000)
    wl = small(sizes, 8, optimizer=opt, grad_dist="normal_layer", freeze_step=3)
    run_chain(wl, 6)


@pytest.mark.parametrize("W,gdt,opt", [(1, "bf16", "adam"), (3, "f32", "adam"), (2, "f32", "lamb")])
def test_fused_steps_many_tiles_per_warp(W, gdt, opt):
    # ~12M elements: every warp of the persistent grid strides over many
    # 512-element warp tiles, across chunk boundaries; chunks of uneven size,
    # one of 40 elements and ones that end part-way through a tile.
    wl = small([1 << 23, 3 * (1 << 20) + 2048 * 7 + 8, 40, 2048 * 300 - 8 * 3], W, grad_dtype=gdt,
               optimizer=opt)
    run_chain(wl, 3)


def test_fused_steps_1024_workers():
    # W = 1024, the largest worker count the library accepts: passes 1-2 loop
    # over 1024 workers per tile, and pass 3 reads the cached server value.
    run_chain(small([2048, 1000, 24], 1024), 2)


def test_hundred_chained_steps_parameter_norm():
    wl = small([40000, 24576, 1000], 2)
    pr = run_chain(wl, 100, compare_every=False)
    torch.cuda.synchronize()
    pg = np_of(pr.gpu.p).astype(np.float64)
    pref = pr.ref["p"].astype(np.float64)
    rel = abs(np.linalg.norm(pg) - np.linalg.norm(pref)) / np.linalg.norm(pref)
    assert rel <= 1e-3, rel
    print("100 steps: relative parameter-norm difference", rel, "exact:", pr.exact())


# -- edge cases ------------------------------------------------------------------------------

def test_empty_problem():
    pr = Pair([0, 0, 0], 3)
    g = np.zeros((3, 0), np.float32)
    pr.gpu.step(torch.zeros((3, 0), dtype=torch.float32, device=dev()))
    torch.cuda.synchronize()
    assert pr.gpu.step_count == 1
    assert np.all(np_of(pr.gpu.s_srv) == 0) and np.all(np_of(pr.gpu.s_w) == 0)
    assert g.size == 0


def test_zero_gradient_chunk():
    """An all-zero chunk: scale 0, every sign +1, error unchanged (stays 0)."""
    wl = small([64, 100, 1024], 2)
    p, v = state_for(wl)
    pr = Pair(wl.offsets, 2, p0=p, v0=v)
    g = grads_for(wl, 0)
    g[:, 64:164] = 0.0
    pr.step(g, warm=False)
    pr.compare()
    sw = np_of(pr.gpu.s_w)
    assert np.all(sw[:, 1] == 0)


def test_nonfinite_sets_status_without_trapping():
    wl = small([512, 1000, 33], 2)
    p, v = state_for(wl)
    pr = Pair(wl.offsets, 2, p0=p, v0=v)
    g = grads_for(wl, 0)
    g[1, 700] = np.float32("nan")
    g[0, 1530] = np.float32("inf")
    pr.step(g, warm=False)
    assert pr.gpu.status() & L.OB_STATUS_NONFINITE
    assert pr.ref_flags & oracle.STATUS_NONFINITE
    pr.compare()   # NaN patterns and every finite value still match
    assert pr.gpu.status(clear=True) & L.OB_STATUS_NONFINITE
    assert pr.gpu.status() == 0
    torch.cuda.synchronize()  # the context is still usable
    assert torch.ones(4, device=dev()).sum().item() == 4


def test_phase_errors():
    wl = small([1024], 2, freeze_step=1)
    pr = Pair(wl.offsets, 2, freeze_step=1)
    g = to_dev(grads_for(wl, 0))
    with pytest.raises(L.OneBitError) as ei:
        pr.gpu.compress(g)
    assert ei.value.code == L.OB_EPHASE
    with pytest.raises(L.OneBitError):
        pr.gpu.server_reduce()
    pr.gpu.step(g)                     # warmup step
    with pytest.raises(L.OneBitError) as ei:
        pr.gpu.warmup_step(g)
    assert ei.value.code == L.OB_EPHASE
    pr.gpu.step(g)                     # compressed step
    assert pr.gpu.step_count == 2


def test_bad_pointers_are_rejected():
    wl = small([1024], 1)
    pr = Pair(wl.offsets, 1)
    stream = int(torch.cuda.current_stream().cuda_stream)
    big = torch.zeros(1025, dtype=torch.float32, device=dev())
    with pytest.raises(L.OneBitError) as ei:          # 4-byte offset: misaligned
        L.ob_step(pr.gpu.ctx, big.data_ptr() + 4, stream)
    assert ei.value.code == L.OB_EINVAL
    host = torch.zeros(1024, dtype=torch.float32)    # pageable host memory
    with pytest.raises(L.OneBitError) as ei:
        L.ob_step(pr.gpu.ctx, host.data_ptr(), stream)
    assert ei.value.code == L.OB_EINVAL
    assert pr.gpu.step_count == 0


def test_determinism_bitwise():
    wl = small(ALIGNED, 4)
    outs = []
    for _ in range(2):
        p, v = state_for(wl)
        opt = OneBitAdam(wl.offsets, 4, device=dev(), p=to_dev(p), v=to_dev(v), **HP)
        for t in range(3):
            opt.step(to_dev(grads_for(wl, t)))
        torch.cuda.synchronize()
        outs.append({k: np_of(getattr(opt, k)).copy() for k in
                     ("p", "m", "err", "srv_err", "bits_w", "bits_srv", "s_w", "s_srv")})
        opt.close()
    for k in outs[0]:
        assert np.array_equal(outs[0][k], outs[1][k]), k


def test_checkpoint_resume_bitwise():
    wl = small(ALIGNED, 2, freeze_step=2)
    p, v = state_for(wl)
    kw = dict(device=dev(), freeze_step=2, **HP)
    a = OneBitAdam(wl.offsets, 2, p=to_dev(p), v=to_dev(v), **kw)
    for t in range(10):
        a.step(to_dev(grads_for(wl, t)))
    b = OneBitAdam(wl.offsets, 2, p=to_dev(p), v=to_dev(v), **kw)
    for t in range(5):
        b.step(to_dev(grads_for(wl, t)))
    sd = b.state_dict()
    b.close()
    c = OneBitAdam(wl.offsets, 2, **kw)
    c.load_state_dict(sd)
    assert c.step_count == 5
    for t in range(5, 10):
        c.step(to_dev(grads_for(wl, t)))
    torch.cuda.synchronize()
    for k in ("p", "m", "v", "err", "srv_err"):
        assert np.array_equal(np_of(getattr(a, k)), np_of(getattr(c, k))), k


def test_host_buffer_entry_point_matches_device_path():
    wl = small(ALIGNED, 2, grad_dtype="bf16")
    p, v = state_for(wl)
    a = OneBitAdam(wl.offsets, 2, grad_dtype="bf16", device=dev(), p=to_dev(p), v=to_dev(v), **HP)
    b = OneBitAdam(wl.offsets, 2, grad_dtype="bf16", device=dev(), p=to_dev(p), v=to_dev(v), **HP)
    for t in range(3):
        g = grads_for(wl, t)
        a.step(to_dev(g))
        host = torch.from_numpy(g.view(np.int16)).view(torch.bfloat16).pin_memory()
        b.step(host)
        torch.cuda.synchronize()   # the pinned buffer must outlive its asynchronous copy
    torch.cuda.synchronize()
    for k in ("p", "m", "err", "srv_err", "bits_srv"):
        assert np.array_equal(np_of(getattr(a, k)), np_of(getattr(b, k))), k
    assert b.step_count == 3


def test_host_entry_overlapped_steps_match_device_path():
    """Back-to-back host-gradient steps (no synchronisation between them): the
    upload of step t+1 overlaps step t's compute through the internal copy
    stream and the alternating staging buffers; results equal the device path."""
    wl = small([1 << 20, 4096, 40], 2)
    p, v = state_for(wl)
    a = OneBitAdam(wl.offsets, 2, device=dev(), p=to_dev(p), v=to_dev(v), **HP)
    b = OneBitAdam(wl.offsets, 2, device=dev(), p=to_dev(p), v=to_dev(v), **HP)
    hosts = [torch.from_numpy(grads_for(wl, t)).pin_memory() for t in range(4)]
    for t in range(4):
        a.step(hosts[t].to(dev()))
    for t in range(4):
        b.step(hosts[t])                 # no synchronisation in between
    torch.cuda.synchronize()
    for k in ("p", "m", "err", "srv_err", "bits_srv", "s_srv"):
        assert np.array_equal(np_of(getattr(a, k)), np_of(getattr(b, k))), k
    assert b.step_count == 4


def test_step_replays_from_a_cuda_graph():
    """The fused step's launches capture into a CUDA graph; replaying it equals
    eager execution bit for bit (small workloads are launch-bound)."""
    wl = WL.get_workload("tiny")
    p, v = state_for(wl)
    eager = OneBitAdam(wl.offsets, wl.W, device=dev(), p=to_dev(p), v=to_dev(v), **HP)
    graphed = OneBitAdam(wl.offsets, wl.W, device=dev(), p=to_dev(p), v=to_dev(v), **HP)
    G = torch.empty((wl.W, wl.n), dtype=torch.float32, device=dev())
    s = torch.cuda.Stream(device=dev())
    s.wait_stream(torch.cuda.current_stream())
    graph = torch.cuda.CUDAGraph()
    G.copy_(to_dev(grads_for(wl, 0)))
    with torch.cuda.stream(s):
        graphed.step(G)                   # first call outside capture (occupancy queries)
    torch.cuda.current_stream().wait_stream(s)
    with torch.cuda.graph(graph, stream=s):
        graphed.step(G)
    graphed.set_step(1)                   # the capture call counted a step without running it
    eager.step(to_dev(grads_for(wl, 0)))
    for t in range(1, 4):
        gt = to_dev(grads_for(wl, t))
        eager.step(gt)
        G.copy_(gt)
        graph.replay()
    torch.cuda.synchronize()
    for k in ("p", "m", "err", "srv_err", "bits_srv", "s_srv"):
        assert np.array_equal(np_of(getattr(eager, k)), np_of(getattr(graphed, k))), k


@pytest.mark.parametrize("opt", ["adam", "lamb"])
def test_zero_one_adam_variance_refresh(opt):
    """0/1 Adam: full-precision refresh steps (m and v) interleaved with
    compressed steps; error buffers carry through the refreshes untouched."""
    wl = small(ALIGNED, 3, optimizer=opt)
    p, v = state_for(wl)
    pr = Pair(wl.offsets, 3, optimizer=opt, p0=p, v0=v)
    o = oracle.get()
    for t, refresh in enumerate([False, False, True, False, True, True, False]):
        g = grads_for(wl, t)
        if refresh:
            pr.gpu.refresh_step(to_dev(g))
            r = pr.ref
            o.warmup(wl.offsets, g, r["m"], r["v"], r["p"], F["beta1"], F["beta2"], F["lr"], F["eps"],
                     optimizer=pr.opt_code)
        else:
            pr.step(g, warm=False)
        pr.compare(tag=f"step {t} ", bits=not refresh)
    assert pr.gpu.step_count == 7 and pr.gpu.status() == 0


@pytest.mark.parametrize("layout", sorted(LAYOUTS))
def test_error_norms_monitoring(layout):
    """Per-chunk L2 norms of the worker and server error buffers after a few
    steps equal numpy's norms of the oracle's buffers (same state)."""
    wl = small(LAYOUTS[layout], 3)
    pr = run_chain(wl, 3, compare_every=False)
    wn, sn = pr.gpu.error_norms()
    torch.cuda.synchronize()
    off = wl.offsets
    want_w = np.array([[np.linalg.norm(pr.ref["err"][w, off[k]:off[k + 1]].astype(np.float64))
                        for k in range(wl.C)] for w in range(3)])
    want_s = np.array([np.linalg.norm(pr.ref["srv_err"][off[k]:off[k + 1]].astype(np.float64))
                       for k in range(wl.C)])
    assert_scales("worker error norms", np_of(wn), want_w)
    assert_scales("server error norms", np_of(sn), want_s)
    assert np.all(np_of(wn)[:, np.diff(off) == 0] == 0)


@pytest.mark.parametrize("W", [2, 4, 16])
def test_fused_equals_stages_bitwise(W):
    """From W = 4 on the fused step keeps the server value of pass 2 for pass 3
    instead of rebuilding it from the workers' words; it must equal the stage
    calls (which rebuild it) bit for bit, as it does below that."""
    wl = small(RAGGED, W)
    p, v = state_for(wl)
    a = OneBitAdam(wl.offsets, W, device=dev(), p=to_dev(p), v=to_dev(v), **HP)
    b = OneBitAdam(wl.offsets, W, device=dev(), p=to_dev(p), v=to_dev(v), **HP)
    for t in range(3):
        g = to_dev(grads_for(wl, t))
        a.step(g)
        b.compress(g)
        b.server_reduce()
        b.apply()
    torch.cuda.synchronize()
    for k in ("p", "m", "err", "srv_err", "bits_w", "s_w", "bits_srv", "s_srv"):
        assert torch.equal(getattr(a, k), getattr(b, k)), k
