"""ob_compress_noalloc, the worker stage for callers that cannot allocate.

Some users of this library may not allocate device memory: their GPU memory is
owned by another allocator (a framework pool that reserved the device up front)
or they run on a latency-critical path where cudaMalloc/cudaFree could stall
the device.  They cannot call ob_create, so ob_compress_noalloc runs the worker
stage with a fixed scratch array inside the library instead.  These tests
check, through the C ABI, that two calls in a row give what the ctx path
(ob_compress) gives on the same inputs, within the tolerance of the other
parity tests, and that sizes beyond the fixed scratch are refused up front.
This file is collected last on purpose; it needs no state from other tests.
"""

import numpy as np
import pytest
import torch

import workloads as WL
from bit_adam_error_b200 import OneBitAdam, _lib as L
from gpu_harness import HP, assert_bits, assert_scales, assert_state, dev, grads_for, np_of, to_dev

pytestmark = pytest.mark.gpu

SIZES = [512, 8, 1536, 33, 4352, 1, 2048, 40, 6216, 0, 65536 + 2056, 7]


@pytest.mark.parametrize("gdt,clip", [("f32", 0.0), ("bf16", 0.0), ("f32", 5.0)])
def test_noalloc_matches_ctx_path_on_two_calls(gdt, clip):
    W = 3
    wl = WL.get_workload("tiny").with_(sizes=tuple(SIZES), W=W, grad_dtype=gdt)
    err0 = WL.aux_normal(5, (1,), W * wl.n, 1e-3).reshape(W, wl.n)
    ref = OneBitAdam(wl.offsets, W, grad_dtype=gdt, clip=clip, device=dev(), **HP)
    ref.err.copy_(to_dev(err0))
    # The caller's own buffers for the allocation-free call.
    err = to_dev(err0)
    bits = torch.zeros((W, ref.words), dtype=torch.int32, device=dev())
    s = torch.zeros((W, wl.C), dtype=torch.float32, device=dev())
    cfg, _keep = L.make_config(wl.n, wl.offsets, W, grad_dtype=L.OB_BF16 if gdt == "bf16" else L.OB_F32,
                               clip=clip)
    stream = int(torch.cuda.current_stream().cuda_stream)
    for t in range(2):
        g = grads_for(wl, t)
        if clip:
            g[:, ::53] = np.float32(-8.0)
        G = to_dev(g)
        ref.compress(G)
        L.ob_compress_noalloc(cfg, G.data_ptr(), err.data_ptr(), bits.data_ptr(), s.data_ptr(), stream)
        torch.cuda.synchronize()
        assert_bits(f"call {t} bits_w", np_of(bits), np_of(ref.bits_w))
        assert_scales(f"call {t} s_w", np_of(s), np_of(ref.s_w))
        assert_state(f"call {t} err", np_of(err), np_of(ref.err), wl.offsets)
    ref.close()


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
