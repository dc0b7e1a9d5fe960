"""Seeded random configurations, every rule, against the oracle.

Each case draws a chunk table (empty chunks, lengths around the 8-element
vector grid, the 32-element word and the 512-element tile, a few multi-tile
chunks), a worker count, gradient and error-buffer types, clip, optimizer and
a warmup length, then runs a short chain of fused steps on the GPU through the
C ABI and the same chain in the oracle, comparing every state tensor at the
parity bar (and the sign planes bit for bit where the rule has them).  The
draws are fixed by the case index, so a failure names a reproducible case.
"""

import numpy as np
import pytest
import torch

import oracle
import workloads as WL
from bit_adam_error_b200 import OneBitAdam
from gpu_harness import F, HP, as_f32, assert_bits, assert_scales, assert_state, dev, grads_for, np_of, \
    state_for, sync_state, to_dev

pytestmark = pytest.mark.gpu

CASES = 24


def draw(case: int, rule: str):
    rng = np.random.default_rng([0x5EED, case, ("scaled", "momentum", "twobit").index(rule)])
    C = int(rng.integers(1, 12))
    pool = [0, 1, 2, 7, 8, 9, 31, 32, 33, 63, 64, 65, 255, 256, 511, 512, 513, 1000, 1024, 1031, 4104]
    sizes = [int(rng.choice(pool)) for _ in range(C)]
    if rng.random() < 0.3:
        sizes.append(int(rng.integers(5000, 70000)))
    W = int(rng.choice([1, 2, 3, 4, 5, 8, 16]))
    gdt = str(rng.choice(["f32", "bf16"]))
    edt = str(rng.choice(["f32", "bf16"]))
    opt = str(rng.choice(["adam", "lamb"]))
    clip = float(rng.choice([0.0, 0.0, 2e-3]))
    freeze = int(rng.integers(0, 2))
    wl = WL.get_workload("tiny").with_(sizes=tuple(sizes), W=W, grad_dtype=gdt, optimizer=opt, clip=clip,
                                       freeze_step=freeze, seed=WL.configs.SEED_BASE + 100 + case)
    return wl, edt


@pytest.mark.parametrize("rule", ["scaled", "momentum", "twobit"])
@pytest.mark.parametrize("case", range(CASES))
def test_random_config(rule, case):
    wl, edt = draw(case, rule)
    p, v = state_for(wl)
    gpu = OneBitAdam(wl.offsets, wl.W, grad_dtype=wl.grad_dtype, optimizer=wl.optimizer, clip=wl.clip,
                     freeze_step=wl.freeze_step, err_dtype=edt, rule=rule, device=dev(),
                     p=to_dev(p), v=to_dev(v), **HP)
    e = np.uint16 if edt == "bf16" else np.float32
    ref = {"p": p.copy(), "m": np.zeros(wl.n, np.float32), "v": v.copy(),
           "err": np.zeros((wl.W, wl.n), e), "srv_err": np.zeros(wl.n, e)}
    o = oracle.get()
    opt = oracle.LAMB if wl.optimizer == "lamb" else oracle.ADAM
    step = {"scaled": o.step, "momentum": o.ternary_step, "twobit": o.twobit_step}[rule]
    flags = 0
    keys = ("p", "m", "v", "err") if rule == "momentum" else ("p", "m", "v", "err", "srv_err")
    tag = f"case {case} {rule} sizes={list(wl.sizes)} W={wl.W} {wl.grad_dtype}/{edt} {wl.optimizer} clip={wl.clip}"
    for t in range(wl.freeze_step + 2):
        g = grads_for(wl, t)
        gpu.step(to_dev(g))
        if t < wl.freeze_step:
            flags |= o.warmup(wl.offsets, g, ref["m"], ref["v"], ref["p"], F["beta1"], F["beta2"], F["lr"],
                              F["eps"], optimizer=opt)
            continue
        flags |= step(wl.offsets, g, ref, F["beta1"], F["lr"], F["eps"], clip=wl.clip, optimizer=opt)
        torch.cuda.synchronize()
        for k in keys:
            got = np_of(getattr(gpu, k))
            assert_state(f"{tag} step {t} {k}", as_f32(got), as_f32(ref[k].reshape(got.shape)), wl.offsets,
                         bf16_step=rule == "twobit" and got.dtype == np.uint16)
        if rule != "momentum":          # (the momentum rule's fused step keeps its codes in registers)
            assert_bits(f"{tag} bits_w", np_of(gpu.bits_w), ref["bits_w"])
            assert_bits(f"{tag} bits_srv", np_of(gpu.bits_srv), ref["bits_srv"])
            assert_scales(f"{tag} s_w", np_of(gpu.s_w), ref["s_w"])
            assert_scales(f"{tag} s_srv", np_of(gpu.s_srv), ref["s_srv"])
        if rule == "twobit":            # the next step from the oracle's state (second scale to an ulp)
            sync_state(gpu, ref)
    assert gpu.status() == flags == 0, tag
    gpu.close()
