"""Seeded input generators (no method arithmetic here).

Every value is drawn from its own counter-based stream: numpy's Philox-4x32
bit generator keyed through a ``SeedSequence`` of
``(seed, kind, step, worker, chunk, block)``.  A block is a fixed
``BLOCK``-element slice of a chunk, so any chunk (or any block of it) can be
regenerated on its own, in any order, by any number of threads, with the same
bits.  That is what lets a test regenerate one sampled chunk of a 1.5e9-element
workload for the oracle without touching the rest.
"""

from __future__ import annotations

import os
from concurrent.futures import ThreadPoolExecutor
from typing import Optional, Tuple

import numpy as np

from .configs import Workload

BLOCK = 1 << 22

KIND_GRAD = 1
KIND_P = 2
KIND_V = 3
KIND_LAYER_MULT = 4
KIND_AUX = 5          # free-form streams for tests (e.g. synthetic server-stage state)


def _rng(seed: int, *key: int) -> np.random.Generator:
    ss = np.random.SeedSequence([int(seed) & 0xFFFFFFFF, *[int(k) for k in key]])
    return np.random.Generator(np.random.Philox(ss))


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bfloat16 (round to nearest, ties to even).

    Returns the raw 16-bit patterns as uint16.  Finite inputs only.
    """
    # For every finite float32 pattern u, u + 0x8000 stays below 2^32.
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    r = ((u >> np.uint32(16)) & np.uint32(1)) + np.uint32(0x7FFF)
    return ((u + r) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Exact widening of bfloat16 bit patterns to float32."""
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def layer_multiplier(wl: Workload, k: int) -> float:
    """Per-chunk gradient std multiplier u_k ~ U(0.5, 2) ('normal_layer' workloads)."""
    return float(_rng(wl.seed, KIND_LAYER_MULT, k).uniform(0.5, 2.0))


def _grad_block(wl: Workload, step: int, worker: int, k: int, b: int, size: int) -> np.ndarray:
    rng = _rng(wl.seed, KIND_GRAD, step, worker, k, b)
    if wl.grad_dist == "normal":
        g = rng.standard_normal(size, dtype=np.float32) * np.float32(wl.grad_scale)
    elif wl.grad_dist == "normal_layer":
        std = np.float32(wl.grad_scale * layer_multiplier(wl, k))
        g = rng.standard_normal(size, dtype=np.float32) * std
    elif wl.grad_dist == "student_t_zeros":
        g = (rng.standard_t(3.0, size) * wl.grad_scale).astype(np.float32)
        if wl.zero_frac > 0:
            g[rng.random(size) < wl.zero_frac] = np.float32(0.0)
    else:
        raise ValueError(f"unknown grad_dist {wl.grad_dist!r}")
    return g.astype(np.float32, copy=False)


def _blocks(nk: int):
    for b, lo in enumerate(range(0, nk, BLOCK)):
        yield b, lo, min(nk, lo + BLOCK)


def chunk_grads(wl: Workload, step: int, worker: int, k: int,
                lo: int = 0, hi: Optional[int] = None) -> np.ndarray:
    """Gradient of ``worker`` at ``step`` for chunk ``k`` (elements [lo, hi) of it).

    float32 values for f32 workloads, uint16 bfloat16 bit patterns for bf16 ones.
    ``lo`` must be a multiple of ``BLOCK``.
    """
    nk = wl.sizes[k]
    hi = nk if hi is None else hi
    assert lo % BLOCK == 0 and 0 <= lo <= hi <= nk
    parts = [_grad_block(wl, step, worker, k, b, b_hi - b_lo)
             for b, b_lo, b_hi in _blocks(nk) if b_lo < hi and b_lo >= lo]
    g = np.concatenate(parts) if parts else np.zeros(0, np.float32)
    g = g[: hi - lo]
    return f32_to_bf16_bits(g) if wl.grad_dtype == "bf16" else g


def _state_block(wl: Workload, k: int, b: int, size: int) -> Tuple[np.ndarray, np.ndarray]:
    p = _rng(wl.seed, KIND_P, k, b).standard_normal(size, dtype=np.float32) * np.float32(0.02)
    if wl.freeze_step > 0:
        v = np.zeros(size, np.float32)
    else:
        u = _rng(wl.seed, KIND_V, k, b).random(size, dtype=np.float32)
        v = (u * np.float32(1e-6 - 1e-8) + np.float32(1e-8)).astype(np.float32)
    return p.astype(np.float32, copy=False), v


def chunk_state(wl: Workload, k: int) -> Tuple[np.ndarray, np.ndarray]:
    """Initial (p, v) of chunk ``k``; m, err and srv_err start at zero."""
    nk = wl.sizes[k]
    ps, vs = [], []
    for b, lo, hi in _blocks(nk):
        p, v = _state_block(wl, k, b, hi - lo)
        ps.append(p)
        vs.append(v)
    if not ps:
        return np.zeros(0, np.float32), np.zeros(0, np.float32)
    return np.concatenate(ps), np.concatenate(vs)


def _threads() -> int:
    return max(1, min(32, os.cpu_count() or 1))


def chunk_groups(wl: Workload, max_elems: int = 1 << 28):
    """Consecutive chunk ranges [k0, k1) holding at most max_elems elements each
    (a single larger chunk forms a group of its own)."""
    k0, tot = 0, 0
    for k, s in enumerate(wl.sizes):
        if k > k0 and tot + s > max_elems:
            yield k0, k
            k0, tot = k, 0
        tot += s
    if k0 < wl.C:
        yield k0, wl.C


def fill_grads(wl: Workload, step: int, out: np.ndarray, workers=None, rows=None,
               chunks=None) -> None:
    """Fill ``out`` (shape [W, n]; float32 or uint16) with the step's gradients.

    ``workers`` selects which workers to generate; ``rows`` (same length) the
    rows of ``out`` they go to (default: row = worker).  ``chunks = (k0, k1)``
    restricts it to those chunks; ``out`` then holds only their elements.
    """
    workers = list(range(wl.W)) if workers is None else list(workers)
    rows = workers if rows is None else list(rows)
    k0, k1 = (0, wl.C) if chunks is None else chunks
    off = wl.offsets - wl.offsets[k0]
    jobs = [(w, r, k, b, lo, hi) for w, r in zip(workers, rows) for k in range(k0, k1)
            for b, lo, hi in _blocks(wl.sizes[k])]

    def run(job):
        w, r, k, b, lo, hi = job
        g = _grad_block(wl, step, w, k, b, hi - lo)
        if wl.grad_dtype == "bf16":
            g = f32_to_bf16_bits(g)
        out[r, off[k] + lo: off[k] + hi] = g

    with ThreadPoolExecutor(_threads()) as ex:
        list(ex.map(run, jobs))


def fill_grads_row(wl: Workload, step: int, worker: int, out: np.ndarray, chunks=None) -> None:
    """Fill the flat row ``out`` with one worker's gradients at ``step`` (all
    chunks, or chunks = (k0, k1) only)."""
    fill_grads(wl, step, out.reshape(1, -1), workers=[worker], rows=[0], chunks=chunks)


def fill_state(wl: Workload, p_out: np.ndarray, v_out: Optional[np.ndarray], chunks=None) -> None:
    """Fill flat ``p_out`` / ``v_out`` (float32) with the initial state of all
    chunks (length n) or of chunks = (k0, k1) only."""
    k0, k1 = (0, wl.C) if chunks is None else chunks
    off = wl.offsets - wl.offsets[k0]
    jobs = [(k, b, lo, hi) for k in range(k0, k1) for b, lo, hi in _blocks(wl.sizes[k])]

    def run(job):
        k, b, lo, hi = job
        p, v = _state_block(wl, k, b, hi - lo)
        p_out[off[k] + lo: off[k] + hi] = p
        if v_out is not None:
            v_out[off[k] + lo: off[k] + hi] = v

    with ThreadPoolExecutor(_threads()) as ex:
        list(ex.map(run, jobs))


def aux_normal(seed: int, key: Tuple[int, ...], size: int, scale: float = 1.0) -> np.ndarray:
    """Free-form seeded N(0, scale^2) float32 draws (test fixtures)."""
    return _rng(seed, KIND_AUX, *key).standard_normal(size, dtype=np.float32) * np.float32(scale)


def aux_bits(seed: int, key: Tuple[int, ...], words: int) -> np.ndarray:
    """Free-form seeded uint32 words (test fixtures)."""
    return _rng(seed, KIND_AUX, *key).integers(0, 1 << 32, size=words, dtype=np.uint64).astype(np.uint32)


def aux_uniform(seed: int, key: Tuple[int, ...], size: int, lo: float, hi: float) -> np.ndarray:
    """Free-form seeded U(lo, hi) float32 draws (test fixtures)."""
    return _rng(seed, KIND_AUX, *key).uniform(lo, hi, size).astype(np.float32)
