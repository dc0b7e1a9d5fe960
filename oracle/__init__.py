"""CPU oracle of the 1-bit Adam compressed-phase step -- TEST INFRASTRUCTURE.

Thin numpy/ctypes wrapper around ``onebit_oracle.c`` (plain single-threaded C).
Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product library
(``bit_adam_error_b200``) never imports it and shares no code with it.

Every function mirrors one step of the method as the pages state it; see the
header of ``onebit_oracle.c`` for the passages followed and the readings taken
where the pages are silent.
"""

from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional, Tuple

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "onebit_oracle.c")
_LIB = os.path.join(_HERE, "libonebit_oracle.so")
# The multi-threaded step (onebit_oracle_mt.c compiles onebit_oracle.c into the
# same unit, so this library also exports every single-thread function).
_SRC_MT = os.path.join(_HERE, "onebit_oracle_mt.c")
_LIB_MT = os.path.join(_HERE, "libonebit_oracle_mt.so")

F32, BF16 = 0, 1
ADAM, LAMB = 0, 1
STATUS_NONFINITE = 1

CFLAGS = ["-O2", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared", "-std=c11"]


def build(force: bool = False, src: str = _SRC, out: str = _LIB, defines=(), threads: bool = False) -> str:
    """Compile the oracle with gcc (no FMA contraction).  Returns the .so path.

    ``threads``: the multi-threaded step (``onebit_oracle_mt.c``, linked with
    ``-pthread``) when ``src``/``out`` are left at their defaults.
    """
    if threads and src == _SRC and out == _LIB:
        src, out = _SRC_MT, _LIB_MT
    deps = [src] + ([_SRC] if src == _SRC_MT else [])
    if not force and os.path.exists(out) and all(os.path.getmtime(out) >= os.path.getmtime(d) for d in deps):
        return out
    extra = ["-pthread"] if src == _SRC_MT else []
    cmd = ["gcc", *CFLAGS, *extra, *[f"-D{d}" for d in defines], "-o", out, src, "-lm"]
    subprocess.run(cmd, check=True)
    return out


def build_all(force: bool = False) -> None:
    """Both oracle libraries: the plain one and the multi-threaded step."""
    build(force=force)
    build(force=force, threads=True)


_P = ctypes.c_void_p
_I32 = ctypes.c_int32
_I64 = ctypes.c_int64
_F = ctypes.c_float
_U32 = ctypes.c_uint32

_SIGS = {
    "orc_words_total": (_I64, [_I32, _P]),
    "orc_compress": (_U32, [_I32, _I64, _I32, _P, _P, _I32, _F, _P, _I32, _P, _P]),
    "orc_server_reduce": (_U32, [_I32, _I64, _I32, _P, _P, _P, _P, _I32, _P, _P]),
    "orc_adam_apply": (_U32, [_I64, _I32, _P, _P, _P, _F, _F, _F, _P, _P, _P]),
    "orc_lamb_apply": (_U32, [_I64, _I32, _P, _P, _P, _F, _F, _F, _P, _P, _P, _P]),
    "orc_warmup": (_U32, [_I32, _I64, _I32, _P, _P, _I32, _I32, _F, _F, _F, _F, _P, _P, _P]),
    "orc_step": (_U32, [_I32, _I64, _I32, _P, _P, _I32, _I32, _F, _F, _F, _F,
                        _P, _P, _P, _P, _P, _I32, _P, _P, _P, _P]),
    "orc_code_words_total": (_I64, [_I32, _P]),
    "orc_ternary_compress": (_U32, [_I32, _I64, _I32, _P, _P, _I32, _F, _F, _P, _I32, _P]),
    "orc_ternary_server": (_U32, [_I32, _I32, _P, _P, _P]),
    "orc_ternary_apply": (_U32, [_I64, _I32, _P, _I32, _P, _I32, _F, _F, _F, _P, _P, _P, _P]),
    "orc_ternary_step": (_U32, [_I32, _I64, _I32, _P, _P, _I32, _I32, _F, _F, _F, _F,
                                _P, _P, _P, _P, _I32, _P, _P]),
    "orc_words2_total": (_I64, [_I32, _P]),
    "orc_twobit_compress": (_U32, [_I32, _I64, _I32, _P, _P, _I32, _F, _P, _I32, _P, _P]),
    "orc_twobit_server": (_U32, [_I32, _I64, _I32, _P, _P, _P, _P, _I32, _P, _P]),
    "orc_twobit_apply": (_U32, [_I64, _I32, _P, _P, _P, _I32, _F, _F, _F, _P, _P, _P, _P]),
    "orc_twobit_step": (_U32, [_I32, _I64, _I32, _P, _P, _I32, _I32, _F, _F, _F, _F,
                               _P, _P, _P, _P, _P, _I32, _P, _P, _P, _P]),
}
_SIGS.update({
    "orc_sign_rates": (None, [_I32, _I32, _P, _I32, _P, _P]),
    "orc_local_step": (_U32, [_I32, _I64, _I32, _P, _P, _I32, _I32, _F, _F, _F, _P, _P, _P, _P, _I32]),
})
_SIGS_MT = {
    "orc_step_mt": (_U32, [_I32, _I32, _I64, _I32, _P, _P, _I32, _I32, _F, _F, _F, _F,
                           _P, _P, _P, _P, _P, _I32, _P, _P, _P, _P]),
}

MAX_TERNARY_WORKERS = 127   # the int8 sum of W codes in {-1, 0, 1} is exact up to here


class Oracle:
    """ctypes handle on one build of the oracle library."""

    def __init__(self, path: Optional[str] = None):
        self.path = path or build()
        self.lib = ctypes.CDLL(self.path)
        sigs = dict(_SIGS)
        if hasattr(self.lib, "orc_step_mt"):
            sigs.update(_SIGS_MT)
        for name, (res, args) in sigs.items():
            fn = getattr(self.lib, name)
            fn.restype = res
            fn.argtypes = args

    # -- helpers -----------------------------------------------------------------
    @staticmethod
    def _ptr(a: Optional[np.ndarray]):
        if a is None:
            return None
        assert a.flags["C_CONTIGUOUS"], "oracle arrays must be contiguous"
        return a.ctypes.data

    @staticmethod
    def _off(offsets) -> np.ndarray:
        return np.ascontiguousarray(offsets, dtype=np.int64)

    def words_total(self, offsets) -> int:
        off = self._off(offsets)
        return int(self.lib.orc_words_total(len(off) - 1, self._ptr(off)))

    @staticmethod
    def _err_dtype(err: np.ndarray) -> int:
        if err.dtype == np.float32:
            return F32
        if err.dtype == np.uint16:
            return BF16
        raise TypeError("error buffers must be float32 or uint16 bfloat16 bit patterns")

    @staticmethod
    def _dtype_of(grads: np.ndarray) -> int:
        if grads.dtype == np.float32:
            return F32
        if grads.dtype == np.uint16:
            return BF16
        raise TypeError("grads must be float32 values or uint16 bfloat16 bit patterns")

    # -- stages ------------------------------------------------------------------
    def compress(self, offsets, grads: np.ndarray, err: np.ndarray, clip: float = 0.0
                 ) -> Tuple[np.ndarray, np.ndarray, int]:
        """Worker stage.  ``grads``/``err``: [W, n]; ``err`` updated in place.

        Returns (bits_w [W, words], s_w [W, C], flags).
        """
        off = self._off(offsets)
        W, n = grads.shape
        C = len(off) - 1
        words = self.words_total(off)
        bits_w = np.zeros((W, words), np.uint32)
        s_w = np.zeros((W, C), np.float32)
        flags = self.lib.orc_compress(W, n, C, self._ptr(off), self._ptr(grads),
                                      self._dtype_of(grads), float(clip), self._ptr(err),
                                      self._err_dtype(err), self._ptr(bits_w), self._ptr(s_w))
        return bits_w, s_w, int(flags)

    def server_reduce(self, offsets, bits_w: np.ndarray, s_w: np.ndarray, srv_err: np.ndarray
                      ) -> Tuple[np.ndarray, np.ndarray, int]:
        """Server stage.  ``srv_err`` [n] updated in place.  Returns (bits_srv, s_srv, flags)."""
        off = self._off(offsets)
        W = bits_w.shape[0]
        C = len(off) - 1
        n = int(off[-1])
        words = self.words_total(off)
        bits_srv = np.zeros(words, np.uint32)
        s_srv = np.zeros(C, np.float32)
        flags = self.lib.orc_server_reduce(W, n, C, self._ptr(off), self._ptr(bits_w),
                                           self._ptr(s_w), self._ptr(srv_err),
                                           self._err_dtype(srv_err), self._ptr(bits_srv),
                                           self._ptr(s_srv))
        return bits_srv, s_srv, int(flags)

    def adam_apply(self, offsets, bits_srv, s_srv, m, v, p, beta1, lr, eps) -> int:
        off = self._off(offsets)
        return int(self.lib.orc_adam_apply(int(off[-1]), len(off) - 1, self._ptr(off),
                                           self._ptr(bits_srv), self._ptr(s_srv), beta1, lr,
                                           eps, self._ptr(m), self._ptr(v), self._ptr(p)))

    def lamb_apply(self, offsets, bits_srv, s_srv, m, v, p, beta1, lr, eps
                   ) -> Tuple[np.ndarray, int]:
        off = self._off(offsets)
        r = np.zeros(len(off) - 1, np.float32)
        flags = self.lib.orc_lamb_apply(int(off[-1]), len(off) - 1, self._ptr(off),
                                        self._ptr(bits_srv), self._ptr(s_srv), beta1, lr, eps,
                                        self._ptr(m), self._ptr(v), self._ptr(p), self._ptr(r))
        return r, int(flags)

    def warmup(self, offsets, grads, m, v, p, beta1, beta2, lr, eps, optimizer=ADAM) -> int:
        off = self._off(offsets)
        W, n = grads.shape
        return int(self.lib.orc_warmup(W, n, len(off) - 1, self._ptr(off), self._ptr(grads),
                                       self._dtype_of(grads), optimizer, beta1, beta2, lr, eps,
                                       self._ptr(m), self._ptr(v), self._ptr(p)))

    def step(self, offsets, grads, state: dict, beta1, lr, eps, clip=0.0, optimizer=ADAM,
             threads: int = 1) -> int:
        """One compressed step.  ``state`` holds p, m, v, err, srv_err (updated in place;
        err and srv_err float32, or both uint16 bfloat16 patterns) and receives
        bits_w, s_w, bits_srv, s_srv.

        ``threads`` > 1 runs the multi-threaded step (bit-identical results); it
        needs an ``Oracle`` loaded from the multi-threaded library (``get_mt()``).
        """
        off = self._off(offsets)
        W, n = grads.shape
        C = len(off) - 1
        words = self.words_total(off)
        for key, shape, dt in (("bits_w", (W, words), np.uint32), ("s_w", (W, C), np.float32),
                               ("bits_srv", (words,), np.uint32), ("s_srv", (C,), np.float32)):
            if key not in state or state[key].shape != shape:
                state[key] = np.zeros(shape, dt)
        args = (W, n, C, self._ptr(off), self._ptr(grads), self._dtype_of(grads), optimizer,
                float(clip), beta1, lr, eps, self._ptr(state["p"]), self._ptr(state["m"]),
                self._ptr(state["v"]), self._ptr(state["err"]), self._ptr(state["srv_err"]),
                self._err_dtype(state["err"]),
                self._ptr(state["bits_w"]), self._ptr(state["s_w"]), self._ptr(state["bits_srv"]),
                self._ptr(state["s_srv"]))
        if threads > 1:
            if not hasattr(self.lib, "orc_step_mt"):
                raise RuntimeError("this oracle build has no multi-threaded step; use oracle.get_mt()")
            flags = int(self.lib.orc_step_mt(int(threads), *args))
            if flags & 0x80000000:
                raise MemoryError("orc_step_mt: scratch allocation failed")
            return flags
        return int(self.lib.orc_step(*args))

    # -- the momentum-error rule (int8 ternary codes) --------------------------------
    def code_words_total(self, offsets) -> int:
        off = self._off(offsets)
        return int(self.lib.orc_code_words_total(len(off) - 1, self._ptr(off)))

    def ternary_compress(self, offsets, grads: np.ndarray, err: np.ndarray, beta1, clip: float = 0.0
                         ) -> Tuple[np.ndarray, int]:
        """Worker stage.  ``grads``/``err``: [W, n]; ``err`` updated in place.

        Returns (codes_w int8 [W, 4 * code_words], flags).
        """
        off = self._off(offsets)
        W, n = grads.shape
        codes = np.zeros((W, 4 * self.code_words_total(off)), np.int8)
        flags = self.lib.orc_ternary_compress(W, n, len(off) - 1, self._ptr(off), self._ptr(grads),
                                              self._dtype_of(grads), float(clip), beta1,
                                              self._ptr(err), self._err_dtype(err), self._ptr(codes))
        return codes, int(flags)

    def ternary_server(self, offsets, codes_w: np.ndarray) -> np.ndarray:
        """Per-element sum of the W workers' codes (int8, W <= 127)."""
        off = self._off(offsets)
        W = codes_w.shape[0]
        if W > MAX_TERNARY_WORKERS:
            raise ValueError(f"W = {W} > {MAX_TERNARY_WORKERS}: the int8 code sum could overflow")
        out = np.zeros(4 * self.code_words_total(off), np.int8)
        self.lib.orc_ternary_server(W, len(off) - 1, self._ptr(off),
                                    self._ptr(np.ascontiguousarray(codes_w, np.int8)), self._ptr(out))
        return out

    def ternary_apply(self, offsets, W, codes_srv, m, v, p, beta1, lr, eps, optimizer=ADAM
                      ) -> Tuple[np.ndarray, int]:
        off = self._off(offsets)
        r = np.zeros(len(off) - 1, np.float32)
        flags = self.lib.orc_ternary_apply(int(off[-1]), len(off) - 1, self._ptr(off), int(W),
                                           self._ptr(np.ascontiguousarray(codes_srv, np.int8)),
                                           optimizer, beta1, lr, eps, self._ptr(m), self._ptr(v),
                                           self._ptr(p), self._ptr(r))
        return r, int(flags)

    def ternary_step(self, offsets, grads, state: dict, beta1, lr, eps, clip=0.0, optimizer=ADAM) -> int:
        """One compressed step of the momentum-error rule.  ``state`` holds p, m, v,
        err (updated in place) and receives codes_w and codes_srv."""
        off = self._off(offsets)
        W, n = grads.shape
        if W > MAX_TERNARY_WORKERS:
            raise ValueError(f"W = {W} > {MAX_TERNARY_WORKERS}: the int8 code sum could overflow")
        nb = 4 * self.code_words_total(off)
        for key, shape in (("codes_w", (W, nb)), ("codes_srv", (nb,))):
            if key not in state or state[key].shape != shape:
                state[key] = np.zeros(shape, np.int8)
        return int(self.lib.orc_ternary_step(
            W, n, len(off) - 1, self._ptr(off), self._ptr(grads), self._dtype_of(grads), optimizer,
            float(clip), beta1, lr, eps, self._ptr(state["p"]), self._ptr(state["m"]),
            self._ptr(state["v"]), self._ptr(state["err"]), self._err_dtype(state["err"]),
            self._ptr(state["codes_w"]), self._ptr(state["codes_srv"])))

    # -- 2-bit Adam (two residual sign planes) ---------------------------------------
    def words2_total(self, offsets) -> int:
        off = self._off(offsets)
        return int(self.lib.orc_words2_total(len(off) - 1, self._ptr(off)))

    def twobit_compress(self, offsets, grads: np.ndarray, err: np.ndarray, clip: float = 0.0
                        ) -> Tuple[np.ndarray, np.ndarray, int]:
        """Worker stage.  Returns (bits_w [W, words2], s_w [W, C, 2], flags); err in place."""
        off = self._off(offsets)
        W, n = grads.shape
        C = len(off) - 1
        bits_w = np.zeros((W, self.words2_total(off)), np.uint32)
        s_w = np.zeros((W, C, 2), np.float32)
        flags = self.lib.orc_twobit_compress(W, n, C, self._ptr(off), self._ptr(grads),
                                             self._dtype_of(grads), float(clip), self._ptr(err),
                                             self._err_dtype(err), self._ptr(bits_w), self._ptr(s_w))
        return bits_w, s_w, int(flags)

    def twobit_server(self, offsets, bits_w: np.ndarray, s_w: np.ndarray, srv_err: np.ndarray
                      ) -> Tuple[np.ndarray, np.ndarray, int]:
        """Server stage.  Returns (bits_srv [words2], s_srv [C, 2], flags); srv_err in place."""
        off = self._off(offsets)
        W = bits_w.shape[0]
        C = len(off) - 1
        bits_srv = np.zeros(self.words2_total(off), np.uint32)
        s_srv = np.zeros((C, 2), np.float32)
        flags = self.lib.orc_twobit_server(W, int(off[-1]), C, self._ptr(off),
                                           self._ptr(np.ascontiguousarray(bits_w, np.uint32)),
                                           self._ptr(np.ascontiguousarray(s_w, np.float32)),
                                           self._ptr(srv_err), self._err_dtype(srv_err),
                                           self._ptr(bits_srv), self._ptr(s_srv))
        return bits_srv, s_srv, int(flags)

    def twobit_apply(self, offsets, bits_srv, s_srv, m, v, p, beta1, lr, eps, optimizer=ADAM
                     ) -> Tuple[np.ndarray, int]:
        off = self._off(offsets)
        r = np.zeros(len(off) - 1, np.float32)
        flags = self.lib.orc_twobit_apply(int(off[-1]), len(off) - 1, self._ptr(off),
                                          self._ptr(np.ascontiguousarray(bits_srv, np.uint32)),
                                          self._ptr(np.ascontiguousarray(s_srv, np.float32)), optimizer,
                                          beta1, lr, eps, self._ptr(m), self._ptr(v), self._ptr(p),
                                          self._ptr(r))
        return r, int(flags)

    def twobit_step(self, offsets, grads, state: dict, beta1, lr, eps, clip=0.0, optimizer=ADAM) -> int:
        """One compressed step of 2-bit Adam; ``state`` as for ``step`` (bits_w,
        s_w [W, C, 2], bits_srv, s_srv [C, 2] are (re)allocated when missing)."""
        off = self._off(offsets)
        W, n = grads.shape
        C = len(off) - 1
        words = self.words2_total(off)
        for key, shape, dt in (("bits_w", (W, words), np.uint32), ("s_w", (W, C, 2), np.float32),
                               ("bits_srv", (words,), np.uint32), ("s_srv", (C, 2), np.float32)):
            if key not in state or state[key].shape != shape:
                state[key] = np.zeros(shape, dt)
        return int(self.lib.orc_twobit_step(
            W, n, C, self._ptr(off), self._ptr(grads), self._dtype_of(grads), optimizer,
            float(clip), beta1, lr, eps, self._ptr(state["p"]), self._ptr(state["m"]),
            self._ptr(state["v"]), self._ptr(state["err"]), self._ptr(state["srv_err"]),
            self._err_dtype(state["err"]),
            self._ptr(state["bits_w"]), self._ptr(state["s_w"]), self._ptr(state["bits_srv"]),
            self._ptr(state["s_srv"])))


    # -- monitoring and 0/1 Adam's local step ----------------------------------------
    def sign_rates(self, offsets, bits: np.ndarray, planes: int = 1) -> np.ndarray:
        """Quantisation rate: per row, chunk and plane the fraction of the chunk's
        elements whose sign bit is set.  ``bits`` [rows, words] (or one row).
        Returns float32 [rows, C, planes]."""
        off = self._off(offsets)
        C = len(off) - 1
        b = np.ascontiguousarray(np.atleast_2d(bits), dtype=np.uint32)
        rows = b.shape[0]
        out = np.zeros((rows, C, planes), np.float32)
        self.lib.orc_sign_rates(rows, C, self._ptr(off), int(planes), self._ptr(b), self._ptr(out))
        return out

    def local_step(self, offsets, grads, state: dict, lr, eps, clip=0.0, optimizer=ADAM) -> int:
        """0/1 Adam local step: err += clip(g) per worker; p moves with the current
        m and v (both unchanged).  ``state`` holds p, m, v, err (in place)."""
        off = self._off(offsets)
        W, n = grads.shape
        return int(self.lib.orc_local_step(
            W, n, len(off) - 1, self._ptr(off), self._ptr(grads), self._dtype_of(grads), optimizer,
            float(clip), lr, eps, self._ptr(state["p"]), self._ptr(state["m"]), self._ptr(state["v"]),
            self._ptr(state["err"]), self._err_dtype(state["err"])))


_default: Optional[Oracle] = None
_default_mt: Optional[Oracle] = None


def get() -> Oracle:
    """The default (unmodified) oracle build."""
    global _default
    if _default is None:
        _default = Oracle()
    return _default


def get_mt() -> Oracle:
    """The multi-threaded build: every function of ``get()``, plus ``step(...,
    threads=N)`` on N host threads."""
    global _default_mt
    if _default_mt is None:
        _default_mt = Oracle(build(threads=True))
    return _default_mt


def host_threads() -> int:
    """Threads this process may run on (its CPU affinity), at least 1."""
    try:
        return max(1, len(os.sched_getaffinity(0)))
    except (AttributeError, OSError):
        return max(1, os.cpu_count() or 1)
