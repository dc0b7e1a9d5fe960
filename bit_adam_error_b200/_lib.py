"""ctypes binding of the C ABI in include/onebit.h (argument marshalling only).

Every function here has the C name and forwards plain integers/pointers to
``libonebit.so``; all arithmetic runs in the library's CUDA kernels.  Loading
fails loudly when the library is missing: there is no fallback path.
"""

from __future__ import annotations

import ctypes
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libonebit.so")

OB_OK, OB_EINVAL, OB_ECUDA, OB_EPHASE, OB_ENOMEM = 0, -1, -2, -3, -4
OB_F32, OB_BF16 = 0, 1
OB_ADAM, OB_LAMB = 0, 1
OB_RULE_SCALED_SIGN, OB_RULE_MOMENTUM_ERROR, OB_RULE_TWO_BIT = 0, 1, 2
OB_STATUS_NONFINITE = 1

ERR_NAMES = {OB_OK: "OB_OK", OB_EINVAL: "OB_EINVAL", OB_ECUDA: "OB_ECUDA",
             OB_EPHASE: "OB_EPHASE", OB_ENOMEM: "OB_ENOMEM"}


class ob_config(ctypes.Structure):
    _fields_ = [
        ("n", ctypes.c_int64),
        ("num_chunks", ctypes.c_int32),
        ("chunk_offsets", ctypes.POINTER(ctypes.c_int64)),
        ("W", ctypes.c_int32),
        ("grad_dtype", ctypes.c_int32),
        ("optimizer", ctypes.c_int32),
        ("lr", ctypes.c_float),
        ("beta1", ctypes.c_float),
        ("beta2", ctypes.c_float),
        ("eps", ctypes.c_float),
        ("clip", ctypes.c_float),
        ("freeze_step", ctypes.c_int32),
        ("err_dtype", ctypes.c_int32),
        ("rule", ctypes.c_int32),
    ]


class OneBitError(RuntimeError):
    def __init__(self, code: int, call: str, msg: str):
        super().__init__(f"{call} -> {ERR_NAMES.get(code, code)}: {msg}")
        self.code = code


_P = ctypes.c_void_p
_SIGS = {
    "ob_layout": (ctypes.c_int, [ctypes.POINTER(ob_config), ctypes.POINTER(ctypes.c_int64)]),
    "ob_create": (ctypes.c_int, [ctypes.POINTER(ob_config), _P, _P, _P, _P, _P, _P, _P, _P, _P,
                                 ctypes.POINTER(_P)]),
    "ob_warmup_step": (ctypes.c_int, [_P, _P, _P]),
    "ob_refresh_step": (ctypes.c_int, [_P, _P, _P]),
    "ob_compress": (ctypes.c_int, [_P, _P, _P]),
    "ob_server_reduce": (ctypes.c_int, [_P, _P]),
    "ob_step": (ctypes.c_int, [_P, _P, _P]),
    "ob_step_host": (ctypes.c_int, [_P, _P, _P, _P]),
    "ob_destroy": (ctypes.c_int, [_P]),
    "ob_get_status": (ctypes.c_int, [_P, ctypes.POINTER(ctypes.c_uint32), ctypes.c_int32, _P]),
    "ob_get_step": (ctypes.c_int64, [_P]),
    "ob_set_step": (ctypes.c_int, [_P, ctypes.c_int64]),
    "ob_profile_start": (ctypes.c_int, [_P, ctypes.c_int32]),
    "ob_profile_stop": (ctypes.c_int, [_P, ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_int64)]),
    "ob_kernel_name": (ctypes.c_char_p, [ctypes.c_int32]),
    "ob_launch_count": (ctypes.c_int64, [_P]),
    "ob_compress_noalloc": (ctypes.c_int, [ctypes.POINTER(ob_config), _P, _P, _P, _P, _P]),
    "ob_error_norms": (ctypes.c_int, [_P, _P, _P, _P]),
    "ob_quant_rates": (ctypes.c_int, [_P, _P, _P, _P]),
    "ob_local_step": (ctypes.c_int, [_P, _P, _P]),
    "ob_mean_grads": (ctypes.c_int, [_P, _P, _P, _P]),
    "ob_last_error": (ctypes.c_char_p, []),
}

OB_K_KINDS = 24

_lib = None


def load() -> ctypes.CDLL:
    """Load libonebit.so (built in-tree by bit_adam_error_b200.build)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with `python bit_adam_error_b200/build.py` "
            "(the 1-bit Adam step has no non-CUDA implementation)")
    lib = ctypes.CDLL(LIB_PATH)
    for name, (res, args) in _SIGS.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


def declared_symbols():
    return sorted(_SIGS)


def last_error() -> str:
    return (load().ob_last_error() or b"").decode(errors="replace")


def check(code: int, call: str) -> None:
    if code != OB_OK:
        raise OneBitError(code, call, last_error())


def make_config(n, offsets, W, grad_dtype=OB_F32, optimizer=OB_ADAM, lr=1e-4, beta1=0.9,
                beta2=0.999, eps=1e-8, clip=0.0, freeze_step=0, err_dtype=OB_F32,
                rule=OB_RULE_SCALED_SIGN):
    """Build an ob_config; returns (config, offsets_array) -- keep both alive."""
    arr = (ctypes.c_int64 * len(offsets))(*[int(x) for x in offsets])
    cfg = ob_config(int(n), len(offsets) - 1, arr, int(W), int(grad_dtype), int(optimizer),
                    float(lr), float(beta1), float(beta2), float(eps), float(clip), int(freeze_step),
                    int(err_dtype), int(rule))
    return cfg, arr


# -- C-named wrappers: integers in, integers out ------------------------------------

def ob_layout(cfg: ob_config) -> int:
    out = ctypes.c_int64(0)
    check(load().ob_layout(ctypes.byref(cfg), ctypes.byref(out)), "ob_layout")
    return out.value


def ob_create(cfg: ob_config, p, m, v, err, srv_err, bits_w, s_w, bits_srv, s_srv) -> int:
    out = _P(0)
    check(load().ob_create(ctypes.byref(cfg), p, m, v, err, srv_err, bits_w, s_w, bits_srv,
                           s_srv, ctypes.byref(out)), "ob_create")
    return out.value


def ob_warmup_step(ctx: int, grads: int, stream: int) -> None:
    check(load().ob_warmup_step(ctx, grads, stream), "ob_warmup_step")


def ob_refresh_step(ctx: int, grads: int, stream: int) -> None:
    check(load().ob_refresh_step(ctx, grads, stream), "ob_refresh_step")


def ob_compress(ctx: int, grads: int, stream: int) -> None:
    check(load().ob_compress(ctx, grads, stream), "ob_compress")


def ob_server_reduce(ctx: int, stream: int) -> None:
    check(load().ob_server_reduce(ctx, stream), "ob_server_reduce")


def ob_step(ctx: int, grads, stream: int) -> None:
    check(load().ob_step(ctx, grads, stream), "ob_step")


def ob_step_host(ctx: int, host_grads: int, dev_staging: int, stream: int) -> None:
    check(load().ob_step_host(ctx, host_grads, dev_staging, stream), "ob_step_host")


def ob_destroy(ctx) -> None:
    check(load().ob_destroy(ctx), "ob_destroy")


def ob_get_status(ctx: int, clear: bool, stream: int) -> int:
    out = ctypes.c_uint32(0)
    check(load().ob_get_status(ctx, ctypes.byref(out), int(bool(clear)), stream), "ob_get_status")
    return out.value


def ob_get_step(ctx) -> int:
    return int(load().ob_get_step(ctx))


def ob_set_step(ctx: int, step: int) -> None:
    check(load().ob_set_step(ctx, step), "ob_set_step")


def ob_error_norms(ctx: int, worker_norms: int, server_norms: int, stream: int) -> None:
    check(load().ob_error_norms(ctx, worker_norms, server_norms, stream), "ob_error_norms")


def ob_quant_rates(ctx: int, worker_rates: int, server_rates: int, stream: int) -> None:
    check(load().ob_quant_rates(ctx, worker_rates, server_rates, stream), "ob_quant_rates")


def ob_local_step(ctx: int, grads: int, stream: int) -> None:
    check(load().ob_local_step(ctx, grads, stream), "ob_local_step")


def ob_mean_grads(ctx: int, grads: int, mean: int, stream: int) -> None:
    check(load().ob_mean_grads(ctx, grads, mean, stream), "ob_mean_grads")


def ob_profile_start(ctx: int, capacity: int) -> None:
    check(load().ob_profile_start(ctx, capacity), "ob_profile_start")


def ob_profile_stop(ctx: int):
    """Returns {kernel name: (total ms, timed launches)} for the kinds that ran."""
    ms = (ctypes.c_double * OB_K_KINDS)()
    n = (ctypes.c_int64 * OB_K_KINDS)()
    check(load().ob_profile_stop(ctx, ms, n), "ob_profile_stop")
    return {ob_kernel_name(k): (ms[k], n[k]) for k in range(OB_K_KINDS) if n[k]}


def ob_kernel_name(kind: int) -> str:
    return (load().ob_kernel_name(kind) or b"").decode()


def ob_launch_count(ctx) -> int:
    return int(load().ob_launch_count(ctx))


def ob_compress_noalloc(cfg: ob_config, grads: int, err: int, bits_w: int, s_w: int, stream: int) -> None:
    """Worker stage without a ctx and without device allocation (fixed scratch)."""
    check(load().ob_compress_noalloc(ctypes.byref(cfg), grads, err, bits_w, s_w, stream),
          "ob_compress_noalloc")
