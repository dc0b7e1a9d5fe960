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

    o = oracle.get()
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
                o.step(off, g, ref, F["beta1"], F["lr"], F["eps"], clip=wl.clip, optimizer=opt_code)
        tag = f"{name} chunk {k}: "
        for key in ("p", "m", "v", "srv_err"):
            assert_state(tag + key, np_of(getattr(opt, key)[lo:hi]), ref[key], off)
        assert_state(tag + "err", np_of(opt.err[:, lo:hi]), ref["err"], off)
        assert_bits(tag + "bits_w", np_of(opt.bits_w[:, wb[k]:wb[k + 1]]), ref["bits_w"])
        assert_bits(tag + "bits_srv", np_of(opt.bits_srv[wb[k]:wb[k + 1]]), ref["bits_srv"])
        assert_scales(tag + "s_w", np_of(opt.s_w[:, k]), ref["s_w"][:, 0])
        assert_scales(tag + "s_srv", np_of(opt.s_srv[k:k + 1]), ref["s_srv"])
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
    o = oracle.get()
    wb = np.zeros(wl.C + 1, np.int64)
    np.cumsum([(s + 31) // 32 for s in wl.sizes], out=wb[1:])
    for k in (0, wl.C - 2, wl.C - 1):
        nk = wl.sizes[k]
        lo, hi = int(wl.offsets[k]), int(wl.offsets[k + 1])
        off = np.array([0, nk], np.int64)
        pk, vk = WL.chunk_state(wl, k)
        ref = {"p": pk, "m": np.zeros(nk, np.float32), "v": vk, "err": np.zeros((1, nk), np.float32),
               "srv_err": np.zeros(nk, np.float32)}
        o.step(off, WL.chunk_grads(wl, 0, 0, k)[None, :], ref, F["beta1"], F["lr"], F["eps"])
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
