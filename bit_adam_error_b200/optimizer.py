"""User-facing 1-bit Adam / 1-bit LAMB optimizer over the C ABI.

PyTorch supplies device memory and the current CUDA stream; every step of the
method runs in ``libonebit.so``.  The optimizer keeps the whole state resident
in HBM as flat buffers:

  p, m, v          : float32 [n]
  err              : [W, n]  (one error buffer per virtual worker; float32 or bfloat16)
  srv_err          : [n]     (server error buffer; same type as err)
  bits_w           : uint32  [W, words]   (packed worker signs; stored as int32)
  s_w              : float32 [W, C]
  bits_srv         : uint32  [words]
  s_srv            : float32 [C]

With ``rule="momentum"`` (the momentum-error rule of the CANN 1-bit Adam
article, sections 2.1-3.2) bits_w / bits_srv hold int8 codes and their sums
(``codes_w`` / ``codes_srv`` give int8 views), and srv_err, s_w, s_srv are
absent (None): that rule has no scale and no server error.  With
``rule="twobit"`` (2-bit Adam: two residual sign planes) bits_w / bits_srv
hold both planes of every chunk and s_w / s_srv are [W, C, 2] / [C, 2].

Phases follow "DeepSpeed Communication Compression and Hiding" (section
"1-bit Adam", 机制): ``step()`` runs the full-precision warmup while
``step_count < freeze_step`` and the fused compressed step afterwards (the
CANN 1-bit Adam article's use_full_precision / use_1bit_compression switch,
section 6.1, is the same switch driven by the step counter).
"""

from __future__ import annotations

from typing import Dict, Optional, Sequence

import numpy as np
import torch

from . import _lib as L


def _ptr(t: Optional[torch.Tensor]) -> int:
    return 0 if t is None else int(t.data_ptr())


class OneBitAdam:
    def __init__(self, offsets: Sequence[int], W: int, *, grad_dtype: str = "f32",
                 optimizer: str = "adam", lr: float = 1e-4, beta1: float = 0.9,
                 beta2: float = 0.999, eps: float = 1e-8, clip: float = 0.0,
                 freeze_step: int = 0, err_dtype: str = "f32", rule: str = "scaled", device=None,
                 p: Optional[torch.Tensor] = None, m: Optional[torch.Tensor] = None,
                 v: Optional[torch.Tensor] = None):
        self.device = torch.device(device) if device is not None else torch.device("cuda", torch.cuda.current_device())
        self.offsets = np.asarray(offsets, dtype=np.int64)
        self.C = len(self.offsets) - 1
        self.n = int(self.offsets[-1])
        self.W = int(W)
        self.grad_dtype = {"f32": L.OB_F32, "bf16": L.OB_BF16}[grad_dtype]
        self.grad_torch_dtype = torch.float32 if self.grad_dtype == L.OB_F32 else torch.bfloat16
        self.optimizer = {"adam": L.OB_ADAM, "lamb": L.OB_LAMB}[optimizer]
        self.err_dtype = {"f32": L.OB_F32, "bf16": L.OB_BF16}[err_dtype]
        edt = torch.float32 if self.err_dtype == L.OB_F32 else torch.bfloat16
        self.rule = {"scaled": L.OB_RULE_SCALED_SIGN, "momentum": L.OB_RULE_MOMENTUM_ERROR,
                     "twobit": L.OB_RULE_TWO_BIT}[rule]
        scaled = self.rule != L.OB_RULE_MOMENTUM_ERROR        # has scales and a server error
        planes = (2,) if self.rule == L.OB_RULE_TWO_BIT else ()
        self.cfg, self._off_keep = L.make_config(self.n, self.offsets, self.W, self.grad_dtype,
                                                 self.optimizer, lr, beta1, beta2, eps, clip,
                                                 freeze_step, self.err_dtype, self.rule)
        self.words = L.ob_layout(self.cfg)
        dev, f32 = self.device, torch.float32

        def state(src, shape):
            t = torch.zeros(shape, dtype=f32, device=dev)
            if src is not None:
                t.copy_(src.reshape(shape))
            return t

        self.p = state(p, (self.n,))
        self.m = state(m, (self.n,))
        self.v = state(v, (self.n,))
        self.err = torch.zeros((self.W, self.n), dtype=edt, device=dev)
        self.srv_err = torch.zeros(self.n, dtype=edt, device=dev) if scaled else None
        self.bits_w = torch.zeros((self.W, self.words), dtype=torch.int32, device=dev)
        self.s_w = torch.zeros((self.W, self.C, *planes), dtype=f32, device=dev) if scaled else None
        self.bits_srv = torch.zeros(self.words, dtype=torch.int32, device=dev)
        self.s_srv = torch.zeros((self.C, *planes), dtype=f32, device=dev) if scaled else None
        with torch.cuda.device(dev):
            self.ctx = L.ob_create(self.cfg, _ptr(self.p), _ptr(self.m), _ptr(self.v),
                                   _ptr(self.err), _ptr(self.srv_err), _ptr(self.bits_w),
                                   _ptr(self.s_w), _ptr(self.bits_srv), _ptr(self.s_srv))
        self._staging: list = []       # two device buffers for host gradients, used alternately
        self._staging_turn = 0

    @property
    def codes_w(self) -> torch.Tensor:
        """Momentum-error rule: the workers' int8 codes [W, 4 * words] (a view)."""
        return self.bits_w.view(torch.int8)

    @property
    def codes_srv(self) -> torch.Tensor:
        """Momentum-error rule: the per-element code sums, int8 [4 * words] (a view)."""
        return self.bits_srv.view(torch.int8)

    # -- plumbing -----------------------------------------------------------------
    def _stream(self) -> int:
        return int(torch.cuda.current_stream(self.device).cuda_stream)

    def _grads_ptr(self, grads: torch.Tensor) -> int:
        if grads.device != self.device:
            raise ValueError(f"grads must live on {self.device} (got {grads.device})")
        if grads.dtype != self.grad_torch_dtype or not grads.is_contiguous() \
                or grads.numel() != self.W * self.n:
            raise ValueError(f"grads must be a contiguous {self.grad_torch_dtype} tensor of "
                             f"{self.W} x {self.n} elements")
        return _ptr(grads)

    # -- phases -------------------------------------------------------------------
    @property
    def step_count(self) -> int:
        return L.ob_get_step(self.ctx)

    def set_step(self, step: int) -> None:
        L.ob_set_step(self.ctx, step)

    @property
    def in_warmup(self) -> bool:
        return self.step_count < self.cfg.freeze_step

    def step(self, grads: torch.Tensor) -> None:
        """One optimizer step on the [W, n] gradients of the W virtual workers.

        Device gradients run the warmup or the fused compressed step in place;
        CPU gradients (pinned for an asynchronous copy) go through
        ``ob_step_host`` with two device staging buffers used alternately, so
        the upload of a step's gradients overlaps the previous step's compute
        (compressed phase only; keep the host tensor unchanged until the
        current stream has passed the step).
        """
        if grads.device.type == "cpu":
            if self.in_warmup:
                raise L.OneBitError(L.OB_EPHASE, "step", "host gradients are taken in the compressed phase only")
            if grads.dtype != self.grad_torch_dtype or not grads.is_contiguous() \
                    or grads.numel() != self.W * self.n:
                raise ValueError("host grads must be contiguous, of the configured dtype and size")
            if not self._staging:
                self._staging = [torch.empty((self.W, self.n), dtype=self.grad_torch_dtype, device=self.device)
                                 for _ in range(2)]
            staging = self._staging[self._staging_turn]
            self._staging_turn ^= 1
            L.ob_step_host(self.ctx, _ptr(grads), _ptr(staging), self._stream())
            return
        g = self._grads_ptr(grads)
        if self.in_warmup:
            L.ob_warmup_step(self.ctx, g, self._stream())
        else:
            L.ob_step(self.ctx, g, self._stream())

    def warmup_step(self, grads: torch.Tensor) -> None:
        L.ob_warmup_step(self.ctx, self._grads_ptr(grads), self._stream())

    def refresh_step(self, grads: torch.Tensor) -> None:
        """0/1 Adam variance refresh: a full-precision step (m and v) in any phase;
        error buffers untouched.  Which steps refresh is the caller's schedule."""
        L.ob_refresh_step(self.ctx, self._grads_ptr(grads), self._stream())

    def local_step(self, grads: torch.Tensor) -> None:
        """0/1 Adam local step (compressed phase): nothing is sent; each worker's
        gradient is kept in its error buffer for the next synchronised step, and
        p moves with the current m and v.  Which steps are local is the caller's
        schedule."""
        L.ob_local_step(self.ctx, self._grads_ptr(grads), self._stream())

    def compress(self, grads: torch.Tensor) -> None:
        """Worker stage: err, bits_w, s_w."""
        L.ob_compress(self.ctx, self._grads_ptr(grads), self._stream())

    def server_reduce(self) -> None:
        """Server stage (compressed allreduce): srv_err, bits_srv, s_srv."""
        L.ob_server_reduce(self.ctx, self._stream())

    def apply(self) -> None:
        """Update from bits_srv / s_srv (after compress + server_reduce)."""
        L.ob_step(self.ctx, None, self._stream())

    def error_norms(self):
        """(worker norms [W, C], server norms [C]) of the error buffers, per chunk,
        as device tensors (monitoring; the CANN article's error-norm check)."""
        wn = torch.empty((self.W, self.C), dtype=torch.float32, device=self.device)
        sn = torch.empty(self.C, dtype=torch.float32, device=self.device) \
            if self.srv_err is not None else None
        L.ob_error_norms(self.ctx, _ptr(wn) if wn.numel() else 0,
                         _ptr(sn) if sn is not None and sn.numel() else 0, self._stream())
        return wn, sn

    def quant_rates(self):
        """(worker rates [W, C(, 2)], server rates [C(, 2)]): per chunk the fraction
        of elements the last step sent as +1 (theoretical value 1/2), as device
        tensors (monitoring; the CANN article's quantisation-rate check).  Not
        available under the momentum-error rule."""
        planes = (2,) if self.rule == L.OB_RULE_TWO_BIT else ()
        wr = torch.empty((self.W, self.C, *planes), dtype=torch.float32, device=self.device)
        sr = torch.empty((self.C, *planes), dtype=torch.float32, device=self.device)
        L.ob_quant_rates(self.ctx, _ptr(wr) if wr.numel() else 0, _ptr(sr) if sr.numel() else 0,
                         self._stream())
        return wr, sr

    def status(self, clear: bool = False) -> int:
        return L.ob_get_status(self.ctx, clear, self._stream())

    # -- checkpoint ----------------------------------------------------------------
    def state_dict(self) -> Dict[str, object]:
        keys = [k for k in ("p", "m", "v", "err", "srv_err") if getattr(self, k) is not None]
        sd: Dict[str, object] = {k: getattr(self, k).detach().cpu().clone() for k in keys}
        sd["step"] = self.step_count
        return sd

    def load_state_dict(self, sd: Dict[str, object]) -> None:
        for k in ("p", "m", "v", "err", "srv_err"):
            if getattr(self, k) is not None:
                getattr(self, k).copy_(sd[k])  # type: ignore[arg-type]
        self.set_step(int(sd["step"]))  # type: ignore[arg-type]

    def close(self) -> None:
        if getattr(self, "ctx", 0):
            L.ob_destroy(self.ctx)
            self.ctx = 0

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
