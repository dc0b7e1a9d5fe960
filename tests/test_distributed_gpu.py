"""Data-parallel driver with the CUDA stages (one GPU here).

world 1 over NCCL (the exchanges reduce to local copies) and worlds 2 and 3
over gloo with all ranks on the same GPU (packed words staged through host
memory; no kernel waits on another process), in the grouped and the pipelined
schedule, for all three rules.  Every rank's state is compared with the
single-process W-worker oracle at the GPU parity bar: sign words bit-exact,
scales and state within 1e-5.
"""

import pytest

from bit_adam_error_b200.distributed import plan
from dist_harness import compare, reference, run_ranks

pytestmark = pytest.mark.gpu

SIZES = [4096, 1000, 640, 33, 20480, 7, 512, 96, 0, 3000]


@pytest.mark.parametrize("world,backend,wl_kw,steps,pipelined", [
    (1, "nccl", dict(freeze_step=1), 3, True),
    (2, "gloo", dict(), 4, False),
    (2, "gloo", dict(), 4, True),
    (2, "gloo", dict(freeze_step=2, optimizer="lamb"), 4, True),
    (2, "gloo", dict(grad_dtype="bf16", clip=5.0, grad_dist="student_t_zeros", zero_frac=0.05), 3, False),
    (3, "gloo", dict(grad_dtype="bf16", clip=5.0, grad_dist="student_t_zeros", zero_frac=0.05), 3, True),
])
def test_gpu_ranks_match_oracle(world, backend, wl_kw, steps, pipelined):
    """Owner slices of SIZES start on 16-element boundaries for 2 and 3 ranks, so
    the per-slice ctxs (pipelined schedule) are taken there."""
    outs = run_ranks(SIZES, world, wl_kw, steps, backend=backend, device="cuda:0", pipelined=pipelined)
    wl, ref = reference(SIZES, world, wl_kw, steps)
    compare(plan(SIZES, world), wl, ref, outs, exact=False)
    assert all(o["flags"] == 0 for o in outs)
    want = "pipelined" if pipelined and world > 1 else "grouped"
    assert all(o["schedule"] == want for o in outs)


@pytest.mark.parametrize("world,pipelined", [(1, True), (2, True), (3, False)])
def test_gpu_ranks_momentum_rule(world, pipelined):
    backend = "nccl" if world == 1 else "gloo"
    wl_kw = dict(grad_dtype="bf16", freeze_step=1)
    outs = run_ranks(SIZES, world, wl_kw, 3, backend=backend, device="cuda:0", pipelined=pipelined,
                     rule="momentum")
    wl, ref = reference(SIZES, world, wl_kw, 3, rule="momentum")
    compare(plan(SIZES, world, 4), wl, ref, outs, exact=False)
    assert all(o["flags"] == 0 for o in outs)
    want = "pipelined" if pipelined and world > 1 else "grouped"
    assert all(o["schedule"] == want for o in outs)


@pytest.mark.parametrize("world,pipelined", [(1, True), (2, True), (3, False)])
def test_gpu_ranks_two_bit_rule(world, pipelined):
    backend = "nccl" if world == 1 else "gloo"
    wl_kw = dict(grad_dtype="bf16", freeze_step=1)
    outs = run_ranks(SIZES, world, wl_kw, 3, backend=backend, device="cuda:0", pipelined=pipelined,
                     rule="twobit")
    wl, ref = reference(SIZES, world, wl_kw, 3, rule="twobit")
    compare(plan(SIZES, world, 32, 2), wl, ref, outs, exact=False)
    assert all(o["flags"] == 0 for o in outs)
    want = "pipelined" if pipelined and world > 1 else "grouped"
    assert all(o["schedule"] == want for o in outs)


@pytest.mark.parametrize("world,backend,wl_kw,schedule,pipelined", [
    (1, "nccl", dict(freeze_step=2, grad_dtype="bf16"), "WWSLLS", True),
    (2, "gloo", dict(freeze_step=1), "WSLSLL", True),
    (3, "gloo", dict(freeze_step=2, optimizer="lamb", grad_dtype="bf16"), "WWSLS", False),
])
def test_gpu_ranks_warmup_exchange_and_local_steps(world, backend, wl_kw, schedule, pipelined):
    """The owner-averaged warmup (each owner averages the ranks' slices of its
    chunks with ob_mean_grads, then every rank runs a one-worker warmup on the
    average) and 0/1 Adam local steps (ob_local_step, no exchange), against the
    W-worker oracle with the same schedule."""
    outs = run_ranks(SIZES, world, wl_kw, len(schedule), backend=backend, device="cuda:0",
                     pipelined=pipelined, schedule=schedule)
    wl, ref = reference(SIZES, world, wl_kw, len(schedule), schedule=schedule)
    compare(plan(SIZES, world), wl, ref, outs, exact=False)
    assert all(o["flags"] == 0 for o in outs)
