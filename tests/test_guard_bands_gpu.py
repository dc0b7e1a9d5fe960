"""Out-of-bounds writes, caught without a sanitizer: guard bands.

Every device buffer a ctx is given is carved out of a larger allocation whose
margins (4 KiB before and after) hold a sentinel byte pattern.  All calls of
every rule then run through the C ABI on layouts with ragged chunks, tails
and empty chunks: warmup, fused steps, the three stage calls, the variance
refresh, the error norms, the host entry, and the no-alloc worker stage.
Afterwards every margin must still hold the sentinel, byte for byte.  Writes
inside a buffer (padding words included) are legitimate; a single byte written
outside one fails the test and names the buffer and side.
"""

import numpy as np
import pytest
import torch

import workloads as WL
from bit_adam_error_b200 import _lib as L
from gpu_harness import dev, grads_for, state_for

pytestmark = pytest.mark.gpu

GUARD = 4096
SENTINEL = 0xA5
RAGGED = [1, 7, 8, 9, 31, 32, 33, 511, 512, 513, 1031, 0, 2, 5, 3000, 0, 6]
ALIGNED = [512, 8, 1536, 24, 2048, 40, 0, 4104]


class Guarded:
    """Device buffers with sentinel margins."""

    def __init__(self):
        self.bufs = {}

    def alloc(self, name, count, dtype):
        itemsize = torch.tensor([], dtype=dtype).element_size()
        nbytes = count * itemsize
        raw = torch.full((GUARD + nbytes + GUARD,), SENTINEL, dtype=torch.uint8, device=dev())
        view = raw[GUARD: GUARD + nbytes].view(dtype)
        view.zero_()
        self.bufs[name] = (raw, nbytes)
        return view

    def ptr(self, name):
        raw, nbytes = self.bufs[name]
        return int(raw.data_ptr()) + GUARD if nbytes else 0

    def check(self):
        torch.cuda.synchronize()
        for name, (raw, nbytes) in self.bufs.items():
            before = raw[:GUARD].cpu().numpy()
            after = raw[GUARD + nbytes:].cpu().numpy()
            assert (before == SENTINEL).all(), f"{name}: write before the buffer"
            assert (after == SENTINEL).all(), f"{name}: write after the buffer (first at +{int(np.argmax(after != SENTINEL))})"


def run_all_calls(sizes, W, rule, gdt, edt, opt):
    wl = WL.get_workload("tiny").with_(sizes=tuple(sizes), W=W, grad_dtype=gdt, optimizer=opt)
    n, C = wl.n, wl.C
    rcode = {"scaled": L.OB_RULE_SCALED_SIGN, "momentum": L.OB_RULE_MOMENTUM_ERROR,
             "twobit": L.OB_RULE_TWO_BIT}[rule]
    cfg, _keep = L.make_config(n, wl.offsets, W, L.OB_BF16 if gdt == "bf16" else L.OB_F32,
                               L.OB_LAMB if opt == "lamb" else L.OB_ADAM, freeze_step=1,
                               err_dtype=L.OB_BF16 if edt == "bf16" else L.OB_F32, rule=rcode)
    words = L.ob_layout(cfg)
    planes = 2 if rule == "twobit" else 1
    scales = 0 if rule == "momentum" else planes
    g = Guarded()
    f32, et = torch.float32, (torch.bfloat16 if edt == "bf16" else torch.float32)
    gt = torch.bfloat16 if gdt == "bf16" else torch.float32
    p = g.alloc("p", n, f32)
    g.alloc("m", n, f32)
    v = g.alloc("v", n, f32)
    g.alloc("err", W * n, et)
    g.alloc("srv_err", n if scales else 0, et)
    g.alloc("bits_w", W * words, torch.int32)
    g.alloc("s_w", W * C * scales, f32)
    g.alloc("bits_srv", words, torch.int32)
    g.alloc("s_srv", C * scales, f32)
    grads = g.alloc("grads", W * n, gt)
    g.alloc("wnorm", W * C, f32)
    g.alloc("snorm", C if scales else 0, f32)
    p0, v0 = state_for(wl)
    p.copy_(torch.from_numpy(p0))
    v.copy_(torch.from_numpy(v0))
    ctx = L.ob_create(cfg, g.ptr("p"), g.ptr("m"), g.ptr("v"), g.ptr("err"), g.ptr("srv_err"),
                      g.ptr("bits_w"), g.ptr("s_w"), g.ptr("bits_srv"), g.ptr("s_srv"))
    st = int(torch.cuda.current_stream().cuda_stream)
    try:
        def load(t):
            a = grads_for(wl, t)
            src = torch.from_numpy(a.view(np.int16)).view(torch.bfloat16) if a.dtype == np.uint16 \
                else torch.from_numpy(a)
            grads.copy_(src.reshape(-1).to(dev()))
        load(0)
        L.ob_warmup_step(ctx, g.ptr("grads"), st)
        for t in (1, 2):
            load(t)
            L.ob_step(ctx, g.ptr("grads"), st)
        load(3)
        L.ob_compress(ctx, g.ptr("grads"), st)
        L.ob_server_reduce(ctx, st)
        L.ob_step(ctx, 0, st)
        L.ob_refresh_step(ctx, g.ptr("grads"), st)
        L.ob_error_norms(ctx, g.ptr("wnorm"), g.ptr("snorm") if scales else 0, st)
        host = grads.cpu().pin_memory()
        L.ob_step_host(ctx, int(host.data_ptr()), g.ptr("grads"), st)
        if rule == "scaled" and edt == "f32":
            L.ob_compress_noalloc(cfg, g.ptr("grads"), g.ptr("err"), g.ptr("bits_w"), g.ptr("s_w"), st)
        assert L.ob_get_status(ctx, False, st) == 0
    finally:
        L.ob_destroy(ctx)
    g.check()


@pytest.mark.parametrize("layout", ["ragged", "aligned"])
@pytest.mark.parametrize("rule", ["scaled", "momentum", "twobit"])
@pytest.mark.parametrize("W,gdt,edt,opt", [(1, "bf16", "f32", "adam"), (3, "f32", "bf16", "lamb"),
                                           (4, "f32", "f32", "adam")])
def test_no_write_outside_any_buffer(layout, rule, W, gdt, edt, opt):
    run_all_calls(RAGGED if layout == "ragged" else ALIGNED, W, rule, gdt, edt, opt)


def test_empty_problem_writes_nothing():
    for rule in ("scaled", "momentum", "twobit"):
        run_all_calls([0, 0], 2, rule, "f32", "f32", "adam")
