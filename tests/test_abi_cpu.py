"""The C-ABI library loads, exports what include/onebit.h declares, and rejects
bad arguments on the host (no GPU needed; no kernel is launched)."""

import ctypes
import os
import re

import pytest

from bit_adam_error_b200 import _lib as L

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def header_symbols():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            text = open(os.path.join(ROOT, "include", fn)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names |= set(re.findall(r"\b(ob_[a-z_]+)\s*\(", text))
    return sorted(names)


def test_library_exports_every_declared_symbol():
    lib = L.load()
    syms = header_symbols()
    assert len(syms) >= 12
    for s in syms:
        assert hasattr(lib, s), s
    assert set(syms) <= set(L.declared_symbols())


def test_layout_counts_words_per_chunk():
    cfg, _k = L.make_config(100, [0, 33, 33, 97, 100], 3)
    assert L.ob_layout(cfg) == 2 + 0 + 2 + 1
    cfg, _k = L.make_config(0, [0, 0], 1)
    assert L.ob_layout(cfg) == 0


def test_layout_counts_code_words_under_the_momentum_rule():
    """int8 codes, four to a word, every chunk on a fresh word."""
    cfg, _k = L.make_config(100, [0, 33, 33, 97, 100], 3, rule=L.OB_RULE_MOMENTUM_ERROR)
    assert L.ob_layout(cfg) == 9 + 0 + 16 + 1
    cfg, _k = L.make_config(8, [0, 8], 127, rule=L.OB_RULE_MOMENTUM_ERROR)
    assert L.ob_layout(cfg) == 2


def test_layout_counts_two_planes_under_the_two_bit_rule():
    cfg, _k = L.make_config(100, [0, 33, 33, 97, 100], 3, rule=L.OB_RULE_TWO_BIT)
    assert L.ob_layout(cfg) == 2 * (2 + 0 + 2 + 1)


@pytest.mark.parametrize("kw,frag", [
    (dict(n=10, offsets=[0, 5, 9], W=1), "!= n"),
    (dict(n=10, offsets=[1, 10], W=1), "[0] must be 0"),
    (dict(n=10, offsets=[0, 6, 4, 10], W=1), "decrease"),
    (dict(n=10, offsets=[0, 10], W=0), "W = 0"),
    (dict(n=10, offsets=[0, 10], W=1025), "W = 1025"),
    (dict(n=10, offsets=[0, 10], W=1, grad_dtype=7), "grad_dtype"),
    (dict(n=10, offsets=[0, 10], W=1, optimizer=5), "optimizer"),
    (dict(n=10, offsets=[0, 10], W=1, lr=float("nan")), "finite"),
    (dict(n=10, offsets=[0, 10], W=1, freeze_step=-1), "freeze_step"),
    (dict(n=-1, offsets=[0, -1], W=1), "n = -1"),
    (dict(n=10, offsets=[0, 10], W=1, rule=3), "rule = 3"),
    (dict(n=10, offsets=[0, 10], W=128, rule=1), "W = 128 > 127"),
])
def test_layout_rejects_bad_configs(kw, frag):
    n, off, W = kw.pop("n"), kw.pop("offsets"), kw.pop("W")
    cfg, _k = L.make_config(n, off, W, **kw)
    with pytest.raises(L.OneBitError) as ei:
        L.ob_layout(cfg)
    assert ei.value.code == L.OB_EINVAL and frag in str(ei.value)


def test_null_arguments_are_errors_not_crashes():
    lib = L.load()
    assert lib.ob_layout(None, None) == L.OB_EINVAL
    cfg, _k = L.make_config(8, [0, 8], 1)
    assert lib.ob_layout(ctypes.byref(cfg), None) == L.OB_EINVAL
    assert lib.ob_create(ctypes.byref(cfg), *([None] * 9), None) == L.OB_EINVAL
    assert lib.ob_destroy(None) == L.OB_OK
    assert lib.ob_get_step(None) == -1
    assert lib.ob_set_step(None, 3) == L.OB_EINVAL
    for fn in ("ob_warmup_step", "ob_compress", "ob_step"):
        assert getattr(lib, fn)(None, None, None) == L.OB_EINVAL, fn
    assert lib.ob_server_reduce(None, None) == L.OB_EINVAL
    assert lib.ob_step_host(None, None, None, None) == L.OB_EINVAL
    flags = ctypes.c_uint32(0)
    assert lib.ob_get_status(None, ctypes.byref(flags), 0, None) == L.OB_EINVAL
    assert "ctx is NULL" in L.last_error()


def test_create_with_bad_config_fails_before_touching_cuda():
    cfg, _k = L.make_config(10, [0, 5, 9], 1)
    with pytest.raises(L.OneBitError) as ei:
        L.ob_create(cfg, *([0] * 9))
    assert ei.value.code == L.OB_EINVAL
