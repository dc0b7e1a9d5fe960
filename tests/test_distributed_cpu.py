"""Data-parallel driver on CPU ranks (gloo, world size 2 and 3).

The ranks exchange packed words with the driver's real exchange code; the
per-rank arithmetic is the oracle (OracleStages).  Every rank's final state
must equal the single-process W-worker oracle, bit for bit: chunk ownership
and the two exchanges must not change a single operation.
"""

import time

import pytest

from bit_adam_error_b200.distributed import plan
from dist_harness import compare, reference, run_ranks, run_with_dead_rank

SIZES = [40, 1000, 64, 33, 2048, 7, 512, 96, 0, 300]


def test_plan_balances_and_groups_by_owner():
    lay = plan(SIZES, 3)
    loads = [sum(SIZES[k] for k in range(len(SIZES)) if lay.owner[k] == r) for r in range(3)]
    assert max(loads) - min(loads) <= max(SIZES)
    assert [lay.owner[k] for k in lay.order] == sorted(lay.owner)
    assert lay.offsets[-1] == sum(SIZES)
    for r in range(3):
        ks = lay.kslice(r)
        assert all(lay.owner[lay.order[i]] == r for i in range(ks.start, ks.stop))
    one = plan(SIZES, 1)
    assert one.order == tuple(range(len(SIZES)))
    many = plan([10, 20], 4)            # more ranks than chunks: some own nothing
    assert sum(many.kslice(r).stop - many.kslice(r).start for r in range(4)) == 2


@pytest.mark.parametrize("pipelined", [False, True], ids=["grouped", "pipelined"])
@pytest.mark.parametrize("world,wl_kw,steps", [
    (2, dict(), 4),
    (3, dict(freeze_step=2), 4),
    (2, dict(optimizer="lamb", freeze_step=1), 3),
    (3, dict(grad_dtype="bf16", clip=5.0, grad_dist="student_t_zeros", zero_frac=0.05), 3),
])
def test_ranks_match_single_process_oracle(world, wl_kw, steps, pipelined):
    outs = run_ranks(SIZES, world, wl_kw, steps, pipelined=pipelined)
    wl, ref = reference(SIZES, world, wl_kw, steps)
    compare(plan(SIZES, world), wl, ref, outs)
    assert all(o["flags"] == 0 for o in outs)
    assert all(o["schedule"] == ("pipelined" if pipelined else "grouped") for o in outs)


@pytest.mark.parametrize("world", [4, 5])
def test_pipelined_rounds_pair_every_rank(world):
    """Shifted rounds with 4 and 5 ranks (the pairing differs from world 2/3;
    with 5 ranks over 10 chunks some ranks own one chunk, one owns the empty one)."""
    outs = run_ranks(SIZES, world, dict(freeze_step=1), 3, pipelined=True)
    wl, ref = reference(SIZES, world, dict(freeze_step=1), 3)
    compare(plan(SIZES, world), wl, ref, outs)
    assert all(o["schedule"] == "pipelined" for o in outs)


def test_a_dead_rank_ends_the_others_step_with_an_error():
    """Failure detection on the host: rank 1 exits between steps; rank 0's next
    exchange must fail (peer gone or process-group timeout), not hang."""
    t0 = time.monotonic()
    results, codes = run_with_dead_rank(SIZES, 2, dict(), steps=3, die=(1, 1), timeout_s=10)
    assert codes[1] == 17
    assert "error" in results[0], "the surviving rank finished instead of reporting the lost peer"
    assert time.monotonic() - t0 < 120


@pytest.mark.parametrize("pipelined", [False, True], ids=["grouped", "pipelined"])
@pytest.mark.parametrize("world,wl_kw,steps", [
    (2, dict(freeze_step=1), 3),
    (3, dict(grad_dtype="bf16", clip=5.0, grad_dist="student_t_zeros", zero_frac=0.05), 3),
    (3, dict(optimizer="lamb"), 2),
])
def test_momentum_rule_ranks_match_single_process_oracle(world, wl_kw, steps, pipelined):
    """The momentum-error rule across ranks: int8 codes to the owners, code sums
    back; every rank equals the W-worker oracle bit for bit."""
    outs = run_ranks(SIZES, world, wl_kw, steps, pipelined=pipelined, rule="momentum")
    wl, ref = reference(SIZES, world, wl_kw, steps, rule="momentum")
    compare(plan(SIZES, world, 4), wl, ref, outs)
    assert all(o["flags"] == 0 for o in outs)


def test_plan_code_words():
    lay = plan(SIZES, 3, 4)
    assert int(lay.words[-1]) == sum((s + 3) // 4 for s in SIZES)
    with pytest.raises(ValueError):
        plan(SIZES, 2, 8)
    two = plan(SIZES, 3, 32, 2)
    assert int(two.words[-1]) == sum(2 * ((s + 31) // 32) for s in SIZES)
    with pytest.raises(ValueError):
        plan(SIZES, 2, 4, 2)


@pytest.mark.parametrize("pipelined", [False, True], ids=["grouped", "pipelined"])
@pytest.mark.parametrize("world,wl_kw,steps", [
    (2, dict(freeze_step=1), 3),
    (3, dict(grad_dtype="bf16", clip=5.0, grad_dist="student_t_zeros", zero_frac=0.05), 3),
    (3, dict(optimizer="lamb"), 2),
])
def test_two_bit_ranks_match_single_process_oracle(world, wl_kw, steps, pipelined):
    """2-bit Adam across ranks: both planes and both scales of owned chunks to
    the owners, the server planes back; bit for bit with the W-worker oracle."""
    outs = run_ranks(SIZES, world, wl_kw, steps, pipelined=pipelined, rule="twobit")
    wl, ref = reference(SIZES, world, wl_kw, steps, rule="twobit")
    compare(plan(SIZES, world, 32, 2), wl, ref, outs)
    assert all(o["flags"] == 0 for o in outs)


@pytest.mark.parametrize("world,wl_kw", [
    (2, dict(freeze_step=3)),
    (3, dict(freeze_step=3, grad_dtype="bf16")),
    (4, dict(freeze_step=2, optimizer="lamb")),
    (5, dict(freeze_step=3, grad_dtype="bf16", optimizer="lamb")),
])
def test_warmup_exchange_owner_average(world, wl_kw):
    """Warmup steps: every rank sends each owner its slice of the owner's
    chunks, the owner averages the W slices in rank order, the averaged slices
    return to every rank, and a one-worker warmup runs on the average.  The
    result equals the W-worker oracle warmup bit for bit (all-warmup runs)."""
    steps = wl_kw["freeze_step"]
    outs = run_ranks(SIZES, world, wl_kw, steps)
    wl, ref = reference(SIZES, world, wl_kw, steps)
    lay = plan(SIZES, world)
    import numpy as np
    off = wl.offsets
    for r, out in enumerate(outs):
        for key in ("p", "m", "v"):
            want = lay.to_layout([ref[key][off[k]:off[k + 1]] for k in range(wl.C)])
            np.testing.assert_array_equal(out[key], want, err_msg=f"rank {r} {key}")
        assert out["flags"] == 0


@pytest.mark.parametrize("pipelined", [False, True], ids=["grouped", "pipelined"])
@pytest.mark.parametrize("world,wl_kw,schedule", [
    (2, dict(), "SLLSLS"),
    (3, dict(freeze_step=1, grad_dtype="bf16"), "WSLSLL"),
    (2, dict(optimizer="lamb", clip=2e-3), "SLSL"),
])
def test_local_steps_across_ranks(world, wl_kw, schedule, pipelined):
    """0/1 Adam local steps in the data-parallel driver: no exchange, each rank
    keeps its gradient in its error buffer and moves its replica; every rank
    equals the W-worker oracle with the same schedule, bit for bit."""
    outs = run_ranks(SIZES, world, wl_kw, len(schedule), pipelined=pipelined, schedule=schedule)
    wl, ref = reference(SIZES, world, wl_kw, len(schedule), schedule=schedule)
    compare(plan(SIZES, world), wl, ref, outs)
    assert all(o["flags"] == 0 for o in outs)
