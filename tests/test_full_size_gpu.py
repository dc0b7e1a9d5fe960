"""Full-size workloads on the GPU, compared with the oracle on sampled chunks.

Each workload runs at its full size through the same call the benchmark times
(``OneBitAdam.step`` -> ``ob_step`` / ``ob_warmup_step``), from the seeded
initial state.  Chunks are independent in the method (each has its own scales,
and LAMB layers are chunks), so the oracle recomputes a few sampled chunks on
their own -- regenerating their inputs from the same per-chunk seeded streams
-- and every output of those chunks is compared: packed words bit-exact,
scales and state within the parity bar.
"""

import numpy as np
import pytest
import torch

import oracle
import workloads as WL
from bit_adam_error_b200 import OneBitAdam
from gpu_harness import (F, HP, assert_bits, assert_scales, assert_state, dev, np_of,
                         upload_grads, upload_state)

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

# The scaled-sign rule's oracle step runs on every host core (bit-identical to
# the single-thread oracle; tests/test_oracle_threads.py), which keeps the
# full-size comparisons short.
THREADS = oracle.host_threads()


def sampled_chunks(wl):
    C = wl.C
    return sorted({0, C // 2, C - 1, int(np.argmax(wl.sizes))})


@pytest.mark.parametrize("name", ["tiny", "bert-base", "gpt2xl-flat", "bert-large", "lamb-1.3b"])
def test_full_size_sampled_chunks(name):
    wl = WL.get_workload(name)
    steps = wl.freeze_step + 1
    torch.cuda.empty_cache()
    opt = OneBitAdam(wl.offsets, wl.W, grad_dtype=wl.grad_dtype, optimizer=wl.optimizer,
                     clip=wl.clip, freeze_step=wl.freeze_step, device=dev(), **HP)
    upload_state(wl, opt.p, opt.v)
    gdt = torch.bfloat16 if wl.grad_dtype == "bf16" else torch.float32
    G = torch.empty((wl.W, wl.n), dtype=gdt, device=dev())
    for t in range(steps):
        upload_grads(wl, t, G)
        opt.step(G)
    torch.cuda.synchronize()
    assert opt.status() == 0
    del G

    o = oracle.get_mt()
    wb = np.zeros(wl.C + 1, np.int64)
    np.cumsum([(s + 31) // 32 for s in wl.sizes], out=wb[1:])
    for k in sampled_chunks(wl):
        nk = wl.sizes[k]
        lo, hi = int(wl.offsets[k]), int(wl.offsets[k + 1])
        off = np.array([0, nk], np.int64)
        pk, vk = WL.chunk_state(wl, k)
        ref = {"p": pk, "m": np.zeros(nk, np.float32), "v": vk,
               "err": np.zeros((wl.W, nk), np.float32), "srv_err": np.zeros(nk, np.float32)}
        opt_code = oracle.LAMB if wl.optimizer == "lamb" else oracle.ADAM
        for t in range(steps):
            g = np.stack([WL.chunk_grads(wl, t, w, k) for w in range(wl.W)])
            if t < wl.freeze_step:
                o.warmup(off, g, ref["m"], ref["v"], ref["p"], F["beta1"], F["beta2"], F["lr"],
                         F["eps"], optimizer=opt_code)
            else:
                o.step(off, g, ref, F["beta1"], F["lr"], F["eps"], clip=wl.clip, optimizer=opt_code,
                       threads=THREADS)
        tag = f"{name} chunk {k}: "
        for key in ("p", "m", "v", "srv_err"):
            assert_state(tag + key, np_of(getattr(opt, key)[lo:hi]), ref[key], off)
        assert_state(tag + "err", np_of(opt.err[:, lo:hi]), ref["err"], off)
        assert_bits(tag + "bits_w", np_of(opt.bits_w[:, wb[k]:wb[k + 1]]), ref["bits_w"])
        assert_bits(tag + "bits_srv", np_of(opt.bits_srv[wb[k]:wb[k + 1]]), ref["bits_srv"])
        assert_scales(tag + "s_w", np_of(opt.s_w[:, k]), ref["s_w"][:, 0])
        assert_scales(tag + "s_srv", np_of(opt.s_srv[k:k + 1]), ref["s_srv"])
    opt.close()


def test_gpt2xl_flat_hundred_chained_steps():
    """The headline workload chained at full size: 100 compressed steps of the
    1.5e9-element gpt2xl-flat buffer (W = 1, bf16 gradients) through
    OneBitAdam.step, the call the benchmark times.  The gradient of step t is
    pre-generated batch t mod 4 (four 3 GB batches stay on the device).

    The oracle runs the same 100 steps on the first chunk (2^26 elements) and
    the 23,604,992-element tail chunk, on their own (chunks are independent).
    Checked:
      * after 100 steps, each sampled chunk's p, m, err and srv_err within the
        per-step parity bar of the oracle's, scales within 1e-5, and the
        chunk's parameter norm within 1e-3 of the oracle's;
      * the last step from identical input state: the oracle's step 100 run on
        the GPU's own state after step 99 gives bit-exact sign words and the
        same state (within the parity bar) as the GPU's step 100.
    """
    wl = WL.get_workload("gpt2xl-flat")
    steps, batches = 100, 4
    ks = (0, wl.C - 1)
    torch.cuda.empty_cache()
    opt = OneBitAdam(wl.offsets, wl.W, grad_dtype=wl.grad_dtype, optimizer=wl.optimizer,
                     clip=wl.clip, freeze_step=wl.freeze_step, device=dev(), **HP)
    upload_state(wl, opt.p, opt.v)
    Gs = []
    for j in range(batches):
        G = torch.empty((wl.W, wl.n), dtype=torch.bfloat16, device=dev())
        upload_grads(wl, j, G)
        Gs.append(G)
    spans = [(int(wl.offsets[k]), int(wl.offsets[k + 1])) for k in ks]
    before_last = None
    for t in range(steps):
        if t == steps - 1:
            torch.cuda.synchronize()
            before_last = {key: np.concatenate([np_of(getattr(opt, key)[..., lo:hi]) for lo, hi in spans], axis=-1)
                           for key in ("p", "m", "v", "err", "srv_err")}
        opt.step(Gs[t % batches])
    torch.cuda.synchronize()
    assert opt.status() == 0
    del Gs
    torch.cuda.empty_cache()

    wb = np.zeros(wl.C + 1, np.int64)
    np.cumsum([(s + 31) // 32 for s in wl.sizes], out=wb[1:])
    gpu = {key: np.concatenate([np_of(getattr(opt, key)[..., lo:hi]) for lo, hi in spans], axis=-1)
           for key in ("p", "m", "v", "err", "srv_err")}
    gpu["bits_w"] = np.concatenate([np_of(opt.bits_w[:, wb[k]:wb[k + 1]]) for k in ks], axis=-1)
    gpu["bits_srv"] = np.concatenate([np_of(opt.bits_srv[wb[k]:wb[k + 1]]) for k in ks])
    gpu["s_w"] = np.stack([np_of(opt.s_w[:, k]) for k in ks], axis=-1)
    gpu["s_srv"] = np.array([np_of(opt.s_srv[k:k + 1])[0] for k in ks], np.float32)
    opt.close()

    # The two sampled chunks as one two-chunk problem, from the seeded state.
    sizes = [wl.sizes[k] for k in ks]
    off = np.array([0, sizes[0], sizes[0] + sizes[1]], np.int64)
    n2 = int(off[-1])
    grads = []
    for j in range(batches):
        g = np.empty((1, n2), np.uint16)
        for i, k in enumerate(ks):
            g[0, off[i]:off[i + 1]] = WL.chunk_grads(wl, j, 0, k)
        grads.append(g)
    p0, v0 = zip(*(WL.chunk_state(wl, k) for k in ks))
    ref = {"p": np.concatenate(p0), "m": np.zeros(n2, np.float32), "v": np.concatenate(v0),
           "err": np.zeros((1, n2), np.float32), "srv_err": np.zeros(n2, np.float32)}
    o = oracle.get_mt()
    for t in range(steps):
        assert o.step(off, grads[t % batches], ref, F["beta1"], F["lr"], F["eps"], threads=THREADS) == 0

    for key in ("p", "m", "v", "srv_err"):
        assert_state("100 steps: " + key, gpu[key], ref[key], off)
    assert_state("100 steps: err", gpu["err"], ref["err"], off)
    assert_scales("100 steps: s_w", gpu["s_w"], ref["s_w"])
    assert_scales("100 steps: s_srv", gpu["s_srv"], ref["s_srv"])
    for i, k in enumerate(ks):
        pg = gpu["p"][off[i]:off[i + 1]].astype(np.float64)
        pr = ref["p"][off[i]:off[i + 1]].astype(np.float64)
        rel = abs(np.linalg.norm(pg) - np.linalg.norm(pr)) / np.linalg.norm(pr)
        assert rel <= 1e-3, (k, rel)

    # Step 100 again, on the oracle, from the GPU's state after step 99.
    last = {key: np.ascontiguousarray(val) for key, val in before_last.items()}
    assert o.step(off, grads[(steps - 1) % batches], last, F["beta1"], F["lr"], F["eps"], threads=THREADS) == 0
    assert_bits("step 100: bits_w", gpu["bits_w"], last["bits_w"])
    assert_bits("step 100: bits_srv", gpu["bits_srv"], last["bits_srv"])
    assert_scales("step 100: s_w", gpu["s_w"], last["s_w"])
    assert_scales("step 100: s_srv", gpu["s_srv"], last["s_srv"])
    for key in ("p", "m", "srv_err"):
        assert_state("step 100: " + key, gpu[key], last[key], off)
    assert_state("step 100: err", gpu["err"], last["err"], off)


def test_gpt2xl_flat_local_step_and_quant_rates():
    """0/1 Adam's local step and the quantisation rates at full size: on the
    1.5e9-element workload, a synchronised step, a local step and another
    synchronised step; chunk 0 and the tail chunk are compared with the oracle
    (state within the parity bar, sign words bit-exact), and the per-chunk
    quantisation rates of every chunk equal the oracle's count of the GPU's
    own sign words (and, on the sampled chunks, of the oracle's)."""
    wl = WL.get_workload("gpt2xl-flat")
    ks = (0, wl.C - 1)
    torch.cuda.empty_cache()
    opt = OneBitAdam(wl.offsets, 1, grad_dtype="bf16", device=dev(), **HP)
    upload_state(wl, opt.p, opt.v)
    G = torch.empty((1, wl.n), dtype=torch.bfloat16, device=dev())
    for t, kind in enumerate("SLS"):
        upload_grads(wl, t, G)
        (opt.local_step if kind == "L" else opt.step)(G)
    wr, sr = opt.quant_rates()
    torch.cuda.synchronize()
    assert opt.status() == 0
    del G
    o = oracle.get_mt()
    bits_w, bits_srv = np_of(opt.bits_w), np_of(opt.bits_srv)
    assert np.array_equal(np_of(wr), o.sign_rates(wl.offsets, bits_w)[:, :, 0])
    assert np.array_equal(np_of(sr), o.sign_rates(wl.offsets, bits_srv)[0, :, 0])
    wb = np.zeros(wl.C + 1, np.int64)
    np.cumsum([(s + 31) // 32 for s in wl.sizes], out=wb[1:])
    for k in ks:
        nk = wl.sizes[k]
        lo, hi = int(wl.offsets[k]), int(wl.offsets[k + 1])
        off = np.array([0, nk], np.int64)
        pk, vk = WL.chunk_state(wl, k)
        ref = {"p": pk, "m": np.zeros(nk, np.float32), "v": vk,
               "err": np.zeros((1, nk), np.float32), "srv_err": np.zeros(nk, np.float32)}
        for t, kind in enumerate("SLS"):
            g = WL.chunk_grads(wl, t, 0, k)[None, :]
            if kind == "L":
                assert o.local_step(off, g, ref, F["lr"], F["eps"]) == 0
            else:
                assert o.step(off, g, ref, F["beta1"], F["lr"], F["eps"], threads=THREADS) == 0
        tag = f"chunk {k}: "
        for key in ("p", "m", "v", "srv_err"):
            assert_state(tag + key, np_of(getattr(opt, key)[lo:hi]), ref[key], off)
        assert_state(tag + "err", np_of(opt.err[:, lo:hi]), ref["err"], off)
        assert_bits(tag + "bits_w", bits_w[:, wb[k]:wb[k + 1]], ref["bits_w"])
        assert_bits(tag + "bits_srv", bits_srv[wb[k]:wb[k + 1]], ref["bits_srv"])
        assert np_of(wr)[0, k] == o.sign_rates(off, ref["bits_w"])[0, 0, 0]
        assert np_of(sr)[k] == o.sign_rates(off, ref["bits_srv"])[0, 0, 0]
    opt.close()


def test_row_longer_than_two_to_the_31():
    """Maximum-size indexing: one worker row of 2^31 + 2^20 elements (bf16
    gradients; about 48 GB resident), so element, word and tile indices pass
    2^31.  The first chunk and the chunks past 2^31 are compared with the oracle."""
    n = (1 << 31) + (1 << 20)
    wl = WL.get_workload("gpt2xl-flat").with_(name="row-2^31", sizes=tuple(WL.configs.flat_slices(n, 1 << 26)))
    torch.cuda.empty_cache()
    opt = OneBitAdam(wl.offsets, 1, grad_dtype="bf16", device=dev(), **HP)
    upload_state(wl, opt.p, opt.v)
    G = torch.empty((1, n), dtype=torch.bfloat16, device=dev())
    upload_grads(wl, 0, G)
    opt.step(G)
    torch.cuda.synchronize()
    assert opt.status() == 0
    del G
    o = oracle.get_mt()
    wb = np.zeros(wl.C + 1, np.int64)
    np.cumsum([(s + 31) // 32 for s in wl.sizes], out=wb[1:])
    for k in (0, wl.C - 2, wl.C - 1):
        nk = wl.sizes[k]
        lo, hi = int(wl.offsets[k]), int(wl.offsets[k + 1])
        off = np.array([0, nk], np.int64)
        pk, vk = WL.chunk_state(wl, k)
        ref = {"p": pk, "m": np.zeros(nk, np.float32), "v": vk, "err": np.zeros((1, nk), np.float32),
               "srv_err": np.zeros(nk, np.float32)}
        o.step(off, WL.chunk_grads(wl, 0, 0, k)[None, :], ref, F["beta1"], F["lr"], F["eps"], threads=THREADS)
        tag = f"chunk {k} [{lo}, {hi}): "
        for key in ("p", "m", "srv_err"):
            assert_state(tag + key, np_of(getattr(opt, key)[lo:hi]), ref[key], off)
        assert_state(tag + "err", np_of(opt.err[:, lo:hi]), ref["err"], off)
        assert_bits(tag + "bits_srv", np_of(opt.bits_srv[wb[k]:wb[k + 1]]), ref["bits_srv"])
        assert_scales(tag + "s_srv", np_of(opt.s_srv[k:k + 1]), ref["s_srv"])
    assert wl.offsets[wl.C - 1] >= (1 << 31)
    opt.close()


@pytest.mark.parametrize("name", ["gpt2xl-flat", "bert-large", "lamb-1.3b"])
def test_full_size_momentum_rule(name):
    """The momentum-error rule's one-pass step at full size (two compressed
    steps from the seeded state), compared with the oracle on sampled chunks."""
    wl = WL.get_workload(name)
    steps = 2
    torch.cuda.empty_cache()
    opt = OneBitAdam(wl.offsets, wl.W, grad_dtype=wl.grad_dtype, optimizer=wl.optimizer,
                     clip=wl.clip, rule="momentum", device=dev(), **HP)
    upload_state(wl, opt.p, opt.v)
    gdt = torch.bfloat16 if wl.grad_dtype == "bf16" else torch.float32
    G = torch.empty((wl.W, wl.n), dtype=gdt, device=dev())
    for t in range(steps):
        upload_grads(wl, t, G)
        opt.step(G)
    torch.cuda.synchronize()
    assert opt.status() == 0
    del G
    o = oracle.get()
    opt_code = oracle.LAMB if wl.optimizer == "lamb" else oracle.ADAM
    for k in sampled_chunks(wl):
        nk = wl.sizes[k]
        lo, hi = int(wl.offsets[k]), int(wl.offsets[k + 1])
        off = np.array([0, nk], np.int64)
        pk, vk = WL.chunk_state(wl, k)
        ref = {"p": pk, "m": np.zeros(nk, np.float32), "v": vk, "err": np.zeros((wl.W, nk), np.float32)}
        for t in range(steps):
            g = np.stack([WL.chunk_grads(wl, t, w, k) for w in range(wl.W)])
            o.ternary_step(off, g, ref, F["beta1"], F["lr"], F["eps"], clip=wl.clip, optimizer=opt_code)
        tag = f"{name} chunk {k}: "
        for key in ("p", "m", "v"):
            assert_state(tag + key, np_of(getattr(opt, key)[lo:hi]), ref[key], off)
        assert_state(tag + "err", np_of(opt.err[:, lo:hi]), ref["err"], off)
    opt.close()


@pytest.mark.parametrize("name", ["gpt2xl-flat", "bert-large"])
def test_full_size_two_bit_rule(name):
    """2-bit Adam at full size (one compressed step from the seeded state),
    compared with the oracle on sampled chunks."""
    wl = WL.get_workload(name)
    torch.cuda.empty_cache()
    opt = OneBitAdam(wl.offsets, wl.W, grad_dtype=wl.grad_dtype, optimizer=wl.optimizer,
                     clip=wl.clip, rule="twobit", device=dev(), **HP)
    upload_state(wl, opt.p, opt.v)
    gdt = torch.bfloat16 if wl.grad_dtype == "bf16" else torch.float32
    G = torch.empty((wl.W, wl.n), dtype=gdt, device=dev())
    upload_grads(wl, 0, G)
    opt.step(G)
    torch.cuda.synchronize()
    assert opt.status() == 0
    del G
    o = oracle.get()
    wb = np.zeros(wl.C + 1, np.int64)
    np.cumsum([2 * ((s + 31) // 32) for s in wl.sizes], out=wb[1:])
    opt_code = oracle.LAMB if wl.optimizer == "lamb" else oracle.ADAM
    for k in sampled_chunks(wl):
        nk = wl.sizes[k]
        lo, hi = int(wl.offsets[k]), int(wl.offsets[k + 1])
        off = np.array([0, nk], np.int64)
        pk, vk = WL.chunk_state(wl, k)
        ref = {"p": pk, "m": np.zeros(nk, np.float32), "v": vk,
               "err": np.zeros((wl.W, nk), np.float32), "srv_err": np.zeros(nk, np.float32)}
        g = np.stack([WL.chunk_grads(wl, 0, w, k) for w in range(wl.W)])
        o.twobit_step(off, g, ref, F["beta1"], F["lr"], F["eps"], clip=wl.clip, optimizer=opt_code)
        tag = f"{name} chunk {k}: "
        for key in ("p", "m", "v", "srv_err"):
            assert_state(tag + key, np_of(getattr(opt, key)[lo:hi]), ref[key], off)
        assert_state(tag + "err", np_of(opt.err[:, lo:hi]), ref["err"], off)
        assert_bits(tag + "bits_w", np_of(opt.bits_w[:, wb[k]:wb[k + 1]]), ref["bits_w"])
        assert_bits(tag + "bits_srv", np_of(opt.bits_srv[wb[k]:wb[k + 1]]), ref["bits_srv"])
        assert_scales(tag + "s_w", np_of(opt.s_w[:, k]), ref["s_w"][:, 0])
        assert_scales(tag + "s_srv", np_of(opt.s_srv[k]), ref["s_srv"][0])
    opt.close()
