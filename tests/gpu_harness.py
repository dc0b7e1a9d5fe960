"""Shared helpers of the GPU parity tests: run the CUDA path (through the C ABI,
via the OneBitAdam binding) and the CPU oracle on the same seeded inputs, and
compare them.

Comparison bar (per step, identical input state):
  * packed sign words: bit-exact;
  * scales: relative error <= 1e-5;
  * state tensors X (err, srv_err, m, v, p), per row and per chunk:
      max_i |X_gpu - X_ref| <= 1e-5 * max(|X_ref,i|, RMS_chunk(X_ref)),
    plus, for error buffers stored as bf16 under 2-bit Adam, one bf16 step
    (bf16_step=True): the CUDA path's second scale may differ from the
    oracle's by one float ulp (it is formed from moments of |c|, the oracle
    sums the float residuals), and a float value within the bar can round to
    the neighbouring bf16 value.
"""

from __future__ import annotations

from typing import Dict, Optional, Sequence

import numpy as np
import torch

import oracle
import workloads as WL
from bit_adam_error_b200 import OneBitAdam

RTOL = 1e-5
HP = dict(lr=1e-4, beta1=0.9, beta2=0.999, eps=1e-8)
F = {k: np.float32(v) for k, v in HP.items()}


def dev():
    return torch.device("cuda", 0)


def to_dev(a: np.ndarray) -> torch.Tensor:
    if a.dtype == np.uint16:
        return torch.from_numpy(a.view(np.int16).copy()).to(dev()).view(torch.bfloat16)
    if a.dtype == np.uint32:
        return torch.from_numpy(a.view(np.int32).copy()).to(dev())
    return torch.from_numpy(np.ascontiguousarray(a)).to(dev())


def np_of(t: torch.Tensor) -> np.ndarray:
    """Host copy; int32 words as uint32, bfloat16 as uint16 bit patterns."""
    t = t.detach().cpu().contiguous()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    a = t.numpy()
    return a.view(np.uint32) if a.dtype == np.int32 else a


def as_f32(a: np.ndarray) -> np.ndarray:
    """bfloat16 patterns widened to float32 (other arrays unchanged)."""
    if a.dtype == np.uint16:
        return (a.astype(np.uint32) << np.uint32(16)).view(np.float32)
    return a


def assert_bits(name, got: np.ndarray, ref: np.ndarray):
    got, ref = np.asarray(got, np.uint32), np.asarray(ref, np.uint32)
    assert got.shape == ref.shape, (name, got.shape, ref.shape)
    bad = np.nonzero(got != ref)
    assert bad[0].size == 0, f"{name}: {bad[0].size} words differ, first at {tuple(b[0] for b in bad)}"


def assert_scales(name, got, ref, rtol=RTOL):
    got, ref = np.asarray(got, np.float64), np.asarray(ref, np.float64)
    same_nan = np.isnan(got) & np.isnan(ref)
    with np.errstate(invalid="ignore"):
        ok = same_nan | (got == ref) | (np.abs(got - ref) <= rtol * np.abs(ref))
    assert ok.all(), f"{name}: max rel err {np.nanmax(np.abs(got - ref) / np.maximum(np.abs(ref), 1e-300))}"


def bf16_ulp(x: np.ndarray) -> np.ndarray:
    """Spacing of bfloat16 values (8 significant bits) at |x| (normal range)."""
    _, e = np.frexp(np.abs(x))
    return np.ldexp(1.0, e - 8)


def assert_state(name, got, ref, offsets, rtol=RTOL, bf16_step=False):
    got = np.atleast_2d(np.asarray(got, np.float64))
    ref = np.atleast_2d(np.asarray(ref, np.float64))
    assert got.shape == ref.shape, (name, got.shape, ref.shape)
    for r in range(ref.shape[0]):
        for k in range(len(offsets) - 1):
            lo, hi = int(offsets[k]), int(offsets[k + 1])
            if hi == lo:
                continue
            g, x = got[r, lo:hi], ref[r, lo:hi]
            fin = np.isfinite(x)
            assert np.array_equal(np.isnan(g), np.isnan(x)), f"{name}[{r}] chunk {k}: NaN pattern"
            inf = np.isinf(x)
            assert np.array_equal(g[inf], x[inf]), f"{name}[{r}] chunk {k}: infinities differ"
            if not fin.any():
                continue
            rms = np.sqrt(np.mean(x[fin] ** 2))
            bound = rtol * np.maximum(np.abs(x[fin]), rms)
            if bf16_step:
                bound = bound + bf16_ulp(np.maximum(np.abs(g[fin]), np.abs(x[fin])))
            err = np.abs(g[fin] - x[fin])
            assert (err <= bound).all(), (
                f"{name}[{r}] chunk {k}: max |diff| {err.max():.3e} vs bound {bound[np.argmax(err - bound)]:.3e}")


def sync_state(gpu, ref, keys=("p", "m", "err", "srv_err")):
    """Copy the oracle's state into the GPU optimizer's buffers, so that the
    next step starts from identical input state."""
    for k in keys:
        t = getattr(gpu, k)
        t.copy_(to_dev(np.ascontiguousarray(ref[k])).reshape(t.shape))


class Pair:
    """A GPU optimizer and the oracle state it is compared with."""

    def __init__(self, offsets: Sequence[int], W: int, *, grad_dtype="f32", optimizer="adam",
                 clip=0.0, freeze_step=0, err_dtype="f32", p0: Optional[np.ndarray] = None,
                 v0: Optional[np.ndarray] = None, m0: Optional[np.ndarray] = None,
                 err0: Optional[np.ndarray] = None, srv0: Optional[np.ndarray] = None):
        self.off = np.asarray(offsets, np.int64)
        self.n = int(self.off[-1])
        self.W = W
        self.clip = clip
        self.optimizer = optimizer
        self.orc = oracle.get()
        n = self.n
        p0 = np.zeros(n, np.float32) if p0 is None else p0
        v0 = np.zeros(n, np.float32) if v0 is None else v0
        m0 = np.zeros(n, np.float32) if m0 is None else m0
        edt = np.uint16 if err_dtype == "bf16" else np.float32
        err0 = np.zeros((W, n), edt) if err0 is None else err0
        srv0 = np.zeros(n, edt) if srv0 is None else srv0
        self.gpu = OneBitAdam(self.off, W, grad_dtype=grad_dtype, optimizer=optimizer, clip=clip,
                              freeze_step=freeze_step, err_dtype=err_dtype, device=dev(),
                              p=to_dev(p0), m=to_dev(m0), v=to_dev(v0), **HP)
        if err0.any():
            self.gpu.err.copy_(to_dev(err0))
        if srv0.any():
            self.gpu.srv_err.copy_(to_dev(srv0))
        self.ref: Dict[str, np.ndarray] = {"p": p0.copy(), "m": m0.copy(), "v": v0.copy(),
                                           "err": err0.copy(), "srv_err": srv0.copy()}
        self.ref_flags = 0

    @property
    def opt_code(self):
        return oracle.LAMB if self.optimizer == "lamb" else oracle.ADAM

    def step(self, g: np.ndarray, warm: bool) -> None:
        self.gpu.step(to_dev(g))
        r = self.ref
        if warm:
            self.ref_flags |= self.orc.warmup(self.off, g, r["m"], r["v"], r["p"], F["beta1"],
                                              F["beta2"], F["lr"], F["eps"], optimizer=self.opt_code)
        else:
            self.ref_flags |= self.orc.step(self.off, g, r, F["beta1"], F["lr"], F["eps"],
                                            clip=self.clip, optimizer=self.opt_code)

    def compare(self, what=("p", "m", "v", "err", "srv_err"), bits=True, tag=""):
        torch.cuda.synchronize()
        for k in what:
            got = np_of(getattr(self.gpu, k))
            want = self.ref[k].reshape(got.shape)       # bfloat16 buffers compare widened
            assert_state(f"{tag}{k}", as_f32(got), as_f32(want), self.off)
        if bits and "bits_w" in self.ref:
            assert_bits(f"{tag}bits_w", np_of(self.gpu.bits_w), self.ref["bits_w"])
            assert_bits(f"{tag}bits_srv", np_of(self.gpu.bits_srv), self.ref["bits_srv"])
            assert_scales(f"{tag}s_w", np_of(self.gpu.s_w), self.ref["s_w"])
            assert_scales(f"{tag}s_srv", np_of(self.gpu.s_srv), self.ref["s_srv"])

    def exact(self) -> bool:
        """True when every state tensor equals the oracle's bit for bit."""
        torch.cuda.synchronize()
        return all(np.array_equal(np_of(getattr(self.gpu, k)).reshape(-1), self.ref[k].reshape(-1))
                   for k in ("p", "m", "v", "err", "srv_err"))


def grads_for(wl: WL.Workload, step: int) -> np.ndarray:
    dt = np.uint16 if wl.grad_dtype == "bf16" else np.float32
    g = np.zeros((wl.W, wl.n), dt)
    WL.fill_grads(wl, step, g)
    return g


def state_for(wl: WL.Workload):
    p = np.zeros(wl.n, np.float32)
    v = np.zeros(wl.n, np.float32)
    WL.fill_state(wl, p, v)
    return p, v


def upload_state(wl: WL.Workload, p_dev: torch.Tensor, v_dev: torch.Tensor) -> None:
    """Seeded initial p, v of the workload into device tensors, a chunk group at a
    time (bounded host memory)."""
    for k0, k1 in WL.chunk_groups(wl):
        lo, hi = int(wl.offsets[k0]), int(wl.offsets[k1])
        p = np.empty(hi - lo, np.float32)
        v = np.empty(hi - lo, np.float32)
        WL.fill_state(wl, p, v, chunks=(k0, k1))
        p_dev[lo:hi].copy_(torch.from_numpy(p))
        v_dev[lo:hi].copy_(torch.from_numpy(v))


def upload_grads(wl: WL.Workload, step: int, G: torch.Tensor) -> None:
    """The step's gradients into the device tensor G [W, n], a worker row and a
    chunk group at a time."""
    bf = wl.grad_dtype == "bf16"
    for w in range(wl.W):
        for k0, k1 in WL.chunk_groups(wl):
            lo, hi = int(wl.offsets[k0]), int(wl.offsets[k1])
            row = np.empty(hi - lo, np.uint16 if bf else np.float32)
            WL.fill_grads_row(wl, step, w, row, chunks=(k0, k1))
            src = torch.from_numpy(row.view(np.int16)).view(torch.bfloat16) if bf else torch.from_numpy(row)
            G[w, lo:hi].copy_(src)
