"""ob_compress_noalloc, the worker stage for callers that cannot allocate.

Some users of this library may not allocate device memory: their GPU memory is
owned by another allocator (a framework pool that reserved the device up front)
or they run on a latency-critical path where cudaMalloc/cudaFree could stall
the device.  They cannot call ob_create, so ob_compress_noalloc runs the worker
stage with a fixed scratch array inside the library instead.  These tests
check, through the C ABI, that two calls in a row give what the ctx path
(ob_compress) gives on the same inputs and what the CPU oracle's worker stage
gives, within the tolerance of the other parity tests (sign words bit-exact),
on layouts that take the 8-wide vector path and the scalar path, for one, two
and three workers; that a non-finite gradient shows in the chunk's scale; that
the call refuses a stream under graph capture; and that sizes beyond the fixed
scratch are refused up front.  This file is collected last on purpose; it
needs no state from other tests.
"""

import numpy as np
import pytest
import torch

import oracle
import workloads as WL
from bit_adam_error_b200 import OneBitAdam, _lib as L
from gpu_harness import HP, assert_bits, assert_scales, assert_state, dev, grads_for, np_of, to_dev

pytestmark = pytest.mark.gpu

# Ragged: chunks off the 8-element grid, odd n -- every chunk on the scalar path.
SIZES = [512, 8, 1536, 33, 4352, 1, 2048, 40, 6216, 0, 65536 + 2056, 7]
# Aligned: the first four chunks start and end on the 8-element grid and n is a
# multiple of 8 (the vector path with 256-bit loads and shuffle-packed words);
# the last two are ragged (scalar path).
SIZES_VEC = [512, 1536, 4352, 65536 + 2056, 33, 7]


def _run_two_calls(sizes, W, gdt, clip):
    wl = WL.get_workload("tiny").with_(sizes=tuple(sizes), W=W, grad_dtype=gdt)
    err0 = WL.aux_normal(5, (1, W), W * wl.n, 1e-3).reshape(W, wl.n)
    ref = OneBitAdam(wl.offsets, W, grad_dtype=gdt, clip=clip, device=dev(), **HP)
    ref.err.copy_(to_dev(err0))
    orc_err = err0.copy()
    # The caller's own buffers for the allocation-free call.
    err = to_dev(err0)
    bits = torch.zeros((W, ref.words), dtype=torch.int32, device=dev())
    s = torch.zeros((W, wl.C), dtype=torch.float32, device=dev())
    cfg, _keep = L.make_config(wl.n, wl.offsets, W, grad_dtype=L.OB_BF16 if gdt == "bf16" else L.OB_F32,
                               clip=clip)
    stream = int(torch.cuda.current_stream().cuda_stream)
    for t in range(2):
        g = grads_for(wl, t)
        if clip:                        # values the clip must cut (-8.0; 0xC100 as bfloat16 bits)
            g[:, ::53] = np.float32(-8.0) if g.dtype == np.float32 else np.uint16(0xC100)
        G = to_dev(g)
        ref.compress(G)
        L.ob_compress_noalloc(cfg, G.data_ptr(), err.data_ptr(), bits.data_ptr(), s.data_ptr(), stream)
        orc_bits, orc_s, flags = oracle.get().compress(wl.offsets, g, orc_err, clip=clip)
        assert flags == 0
        torch.cuda.synchronize()
        # against the ctx path
        assert_bits(f"call {t} bits_w vs ctx", np_of(bits), np_of(ref.bits_w))
        assert_scales(f"call {t} s_w vs ctx", np_of(s), np_of(ref.s_w))
        assert_state(f"call {t} err vs ctx", np_of(err), np_of(ref.err), wl.offsets)
        # against the oracle
        assert_bits(f"call {t} bits_w vs oracle", np_of(bits), orc_bits)
        assert_scales(f"call {t} s_w vs oracle", np_of(s), orc_s)
        assert_state(f"call {t} err vs oracle", np_of(err), orc_err, wl.offsets)
    ref.close()


@pytest.mark.parametrize("gdt,clip", [("f32", 0.0), ("bf16", 0.0), ("f32", 5.0)])
def test_noalloc_matches_ctx_path_on_two_calls(gdt, clip):
    _run_two_calls(SIZES, 3, gdt, clip)


@pytest.mark.parametrize("W", [1, 2, 3])
@pytest.mark.parametrize("gdt,clip", [("f32", 0.0), ("bf16", 0.0), ("bf16", 5.0)])
def test_noalloc_vector_path_matches_ctx_path_and_oracle(W, gdt, clip):
    _run_two_calls(SIZES_VEC, W, gdt, clip)


def test_noalloc_nonfinite_gradient_shows_in_the_scale():
    W = 2
    wl = WL.get_workload("tiny").with_(sizes=tuple(SIZES_VEC), W=W)
    g = grads_for(wl, 0)
    g[1, int(wl.offsets[2]) + 100] = np.float32("nan")
    g[0, int(wl.offsets[3]) + 5] = np.float32("inf")
    err = torch.zeros((W, wl.n), dtype=torch.float32, device=dev())
    words = sum((n + 31) // 32 for n in SIZES_VEC)
    bits = torch.zeros((W, words), dtype=torch.int32, device=dev())
    s = torch.zeros((W, wl.C), dtype=torch.float32, device=dev())
    cfg, _keep = L.make_config(wl.n, wl.offsets, W)
    G = to_dev(g)
    L.ob_compress_noalloc(cfg, G.data_ptr(), err.data_ptr(), bits.data_ptr(), s.data_ptr(),
                          int(torch.cuda.current_stream().cuda_stream))
    torch.cuda.synchronize()
    sc = np_of(s)
    assert np.isnan(sc[1, 2]) and np.isposinf(sc[0, 3])
    bad = np.zeros_like(sc, bool)
    bad[1, 2] = bad[0, 3] = True
    assert np.isfinite(sc[~bad]).all()


def test_noalloc_refuses_a_capturing_stream():
    W = 1
    wl = WL.get_workload("tiny").with_(sizes=(512, 40), W=W)
    G = to_dev(grads_for(wl, 0))
    err = torch.zeros((W, wl.n), dtype=torch.float32, device=dev())
    bits = torch.zeros((W, 16 + 2), dtype=torch.int32, device=dev())
    s = torch.zeros((W, wl.C), dtype=torch.float32, device=dev())
    cfg, _keep = L.make_config(wl.n, wl.offsets, W)
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    graph = torch.cuda.CUDAGraph()
    x = torch.zeros(4, device=dev())
    with torch.cuda.stream(side):
        graph.capture_begin()
        try:
            with pytest.raises(L.OneBitError) as ei:
                L.ob_compress_noalloc(cfg, G.data_ptr(), err.data_ptr(), bits.data_ptr(), s.data_ptr(),
                                      int(side.cuda_stream))
            x.add_(1.0)
        finally:
            graph.capture_end()
    assert ei.value.code == L.OB_EINVAL and "captured" in str(ei.value)
    torch.cuda.synchronize()
    del graph


def test_noalloc_refuses_sizes_beyond_its_scratch():
    cfg, _k = L.make_config(40_000_000, [0, 40_000_000], 16)     # W*n = 6.4e8 elements
    with pytest.raises(L.OneBitError) as ei:
        L.ob_compress_noalloc(cfg, 0, 0, 0, 0, 0)
    assert ei.value.code == L.OB_EINVAL and "scratch" in str(ei.value)
    off = list(range(0, 4098 * 8, 8))                            # 4097 chunks
    cfg, _k = L.make_config(off[-1], off, 1)
    with pytest.raises(L.OneBitError) as ei:
        L.ob_compress_noalloc(cfg, 0, 0, 0, 0, 0)
    assert ei.value.code == L.OB_EINVAL and "chunks" in str(ei.value)
