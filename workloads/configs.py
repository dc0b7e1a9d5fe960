"""Workload definitions: chunk tables and input distributions.

A *chunk* is the unit that owns one scale (one parameter tensor, or one fixed
slice of a flat buffer).  Chunks are laid out back to back in one flattened
buffer of ``n`` elements; ``offsets`` has ``C + 1`` entries with
``offsets[0] == 0`` and ``offsets[C] == n``.

The five parameter sets are the workloads the 1-bit Adam pages talk about
(BERT-base / BERT-large pre-training, GPT-sized models, a 1-bit LAMB run on a
large transformer), written out as the standard tensor lists of those
architectures.  Only sizes are needed; no weights are involved.
"""

from __future__ import annotations

from dataclasses import dataclass, field
from typing import Dict, List, Tuple

import numpy as np

SEED_BASE = 0x1B17ADA0


def bert_tensor_sizes(hidden: int, layers: int, ffn: int, vocab: int,
                      positions: int = 512, token_types: int = 2) -> List[int]:
    """Tensor sizes of a BERT encoder with pooler, in parameter order.

    5 embedding tensors (word, position, token type, LayerNorm gamma/beta),
    16 per encoder layer (Q/K/V/attention-output weight+bias, attention
    LayerNorm, FFN in/out weight+bias, output LayerNorm), 2 pooler tensors.
    """
    h = hidden
    sizes = [vocab * h, positions * h, token_types * h, h, h]
    for _ in range(layers):
        for _qkvo in range(4):
            sizes += [h * h, h]
        sizes += [h, h]              # attention-output LayerNorm
        sizes += [h * ffn, ffn]      # intermediate dense
        sizes += [ffn * h, h]        # output dense
        sizes += [h, h]              # output LayerNorm
    sizes += [h * h, h]              # pooler
    return sizes


def gpt_tensor_sizes(hidden: int, layers: int, ffn: int, vocab: int,
                     positions: int) -> List[int]:
    """Tensor sizes of a GPT-2-style decoder with fused QKV, in parameter order.

    token + position tables, 12 per block (ln_1, fused qkv weight+bias,
    attention projection weight+bias, ln_2, MLP in/out weight+bias), ln_f.
    """
    h = hidden
    sizes = [vocab * h, positions * h]
    for _ in range(layers):
        sizes += [h, h]                  # ln_1
        sizes += [h * 3 * h, 3 * h]      # fused qkv
        sizes += [h * h, h]              # attention projection
        sizes += [h, h]                  # ln_2
        sizes += [h * ffn, ffn]          # mlp in
        sizes += [ffn * h, h]            # mlp out
    sizes += [h, h]                      # ln_f
    return sizes


def flat_slices(n: int, slice_elems: int) -> List[int]:
    """A flat buffer of ``n`` elements cut into fixed slices (last one shorter)."""
    full, tail = divmod(n, slice_elems)
    return [slice_elems] * full + ([tail] if tail else [])


@dataclass(frozen=True)
class Workload:
    """One synthetic workload of the compressed-phase step.

    ``grad_dist``:
      * ``"normal"``          g ~ N(0, grad_scale^2)
      * ``"normal_layer"``    g ~ N(0, (grad_scale * u_k)^2), one u_k ~ U(0.5, 2)
                              per chunk (per tensor)
      * ``"student_t_zeros"`` g = grad_scale * t_3, then each element set to +0.0
                              with probability ``zero_frac``
    State init: p ~ N(0, 0.02^2); v ~ U(1e-8, 1e-6) (or 0 when the workload
    starts with full-precision warmup steps); m = err = srv_err = 0.
    """

    name: str
    sizes: Tuple[int, ...]
    W: int
    grad_dtype: str = "f32"          # "f32" | "bf16"
    err_dtype: str = "f32"           # storage of the error buffers: "f32" | "bf16"
    optimizer: str = "adam"          # "adam" | "lamb"
    grad_dist: str = "normal"
    grad_scale: float = 1e-3
    zero_frac: float = 0.0
    clip: float = 0.0                # <= 0: off
    freeze_step: int = 0             # number of full-precision warmup steps
    steps: int = 10                  # steps the workload is quoted on
    lr: float = 1e-4
    beta1: float = 0.9
    beta2: float = 0.999
    eps: float = 1e-8
    seed: int = SEED_BASE
    description: str = ""
    _cache: Dict[str, object] = field(default_factory=dict, compare=False,
                                      repr=False, hash=False)

    @property
    def C(self) -> int:
        return len(self.sizes)

    @property
    def n(self) -> int:
        return int(sum(self.sizes))

    @property
    def offsets(self) -> np.ndarray:
        if "offsets" not in self._cache:
            off = np.zeros(self.C + 1, dtype=np.int64)
            np.cumsum(np.asarray(self.sizes, dtype=np.int64), out=off[1:])
            self._cache["offsets"] = off
        return self._cache["offsets"]  # type: ignore[return-value]

    @property
    def grad_bytes(self) -> int:
        return 2 if self.grad_dtype == "bf16" else 4

    @property
    def err_bytes(self) -> int:
        return 2 if self.err_dtype == "bf16" else 4

    def with_(self, **kw) -> "Workload":
        d = {k: getattr(self, k) for k in self.__dataclass_fields__ if k != "_cache"}
        d.update(kw)
        if "sizes" in kw:
            d["sizes"] = tuple(int(s) for s in kw["sizes"])
        return Workload(**d)


def _mk() -> Dict[str, Workload]:
    w: Dict[str, Workload] = {}
    w["tiny"] = Workload(
        name="tiny", sizes=(1 << 20,), W=4, grad_dist="normal", grad_scale=1e-3,
        steps=10, seed=SEED_BASE + 0,
        description="n=1,048,576, one chunk, W=4 fp32 workers, 10 compressed steps")
    w["bert-base"] = Workload(
        name="bert-base",
        sizes=tuple(bert_tensor_sizes(768, 12, 3072, 30522)), W=8,
        grad_dist="normal_layer", grad_scale=1e-3, freeze_step=5, steps=10,
        seed=SEED_BASE + 1,
        description="BERT-base tensor set, 109,482,240 params in 199 chunks, W=8, "
                    "5 fp32 warmup steps then compressed steps")
    w["gpt2xl-flat"] = Workload(
        name="gpt2xl-flat", sizes=tuple(flat_slices(1_500_000_000, 1 << 26)), W=1,
        grad_dtype="bf16", grad_dist="normal", grad_scale=1e-4, steps=100,
        seed=SEED_BASE + 2,
        description="flat 1.5e9-element buffer in 2^26-element chunks (23 chunks), "
                    "W=1, bf16 gradients upcast in-kernel, fp32 state")
    w["bert-large"] = Workload(
        name="bert-large",
        sizes=tuple(bert_tensor_sizes(1024, 24, 4096, 30522)), W=16,
        grad_dist="student_t_zeros", grad_scale=1e-3, zero_frac=0.05, clip=5.0,
        steps=10, seed=SEED_BASE + 3,
        description="BERT-large tensor set, 335,141,888 params in 391 chunks, W=16, "
                    "Student-t(3) gradients with 5% exact zeros, clip +/-5")
    w["lamb-1.3b"] = Workload(
        name="lamb-1.3b",
        sizes=tuple(gpt_tensor_sizes(2048, 24, 8192, 50257, 2048)), W=4,
        optimizer="lamb", grad_dist="normal", grad_scale=1e-4, steps=10,
        seed=SEED_BASE + 4,
        description="1.3B-param 24-layer GPT-style transformer, 292 tensors = LAMB "
                    "layers, W=4, 1-bit LAMB trust ratio per layer")
    return w


WORKLOADS: Dict[str, Workload] = _mk()


def get_workload(name: str) -> Workload:
    try:
        return WORKLOADS[name]
    except KeyError:
        raise KeyError(f"unknown workload {name!r}; known: {sorted(WORKLOADS)}")
