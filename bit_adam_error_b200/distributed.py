"""1-bit Adam across real GPUs: worker w = rank w, one process per GPU.

The single-GPU library keeps W virtual workers in one GPU's memory.  Here the
W workers are the ranks of a torch.distributed group and the compressed
allreduce ("DeepSpeed Communication Compression and Hiding", section "1-bit
Adam", 机制) becomes two exchanges of packed words:

  1. every rank runs the worker stage on its own gradient (one worker):
     signs + per-chunk scales + its worker error;
  2. exchange 1: the words and scales of chunk k go to the rank that owns k;
  3. every owner runs the server stage over the W workers of its chunks
     (server error kept only by the owner);
  4. exchange 2: the owners' server words and scales go to every rank;
  5. every rank applies the update to its replica of p, m (v frozen).

Chunks are owned whole (greedy balance by size), so each chunk's server scale
and every float operation are the ones the single-GPU path (and the oracle)
computes with W workers: the result is the same, bit for bit.  The flat
buffer groups chunks by owner, so each exchange moves one contiguous slice
per peer: about n/32 words plus C scales in each direction per step, 1/32 of an
fp32 allreduce.  A warmup step averages the full-precision gradients owner by
owner: every rank sends owner o its gradient slice of o's chunks (n / W
elements to each peer), the owner averages the W slices in rank order (the
oracle's float sum, then / W), and the owners send the averaged slices to
every rank (float32), which runs a one-worker warmup on the average.  Per rank
that moves about n gradient elements plus n floats, instead of the W whole
gradients an all-gather of gradients would.  The averaging and the one-worker
warmup round exactly as the W-worker warmup does.

0/1 Adam's local steps (``local_step``) exchange nothing: every rank keeps its
gradient in its error buffer and moves its replica with the current m and v.

The arithmetic runs in the CUDA library (``CudaStages``); this module only
plans the layout and moves packed words between ranks (NCCL on GPUs; gloo
stages CUDA tensors through host memory).  The stage backend is an object with
a fixed interface, so the exchange logic can also be exercised on CPU ranks.

Compression overlapped with transfer (the CANN 1-bit Adam article, section
4.2): with one worker ctx per owner slice, each slice is compressed just
before its exchange round is posted, and updated as soon as its owner's server
words arrive.  On NCCL the transfers run on the communicator's own stream, so
they overlap the kernels of the next slice.
"""

from __future__ import annotations

from dataclasses import dataclass
from typing import List, Optional, Sequence, Tuple

import numpy as np
import torch
import torch.distributed as dist


# ---- layout ------------------------------------------------------------------------

@dataclass(frozen=True)
class DPLayout:
    """Chunk ownership and the owner-grouped flat layout.

    ``sizes`` are the chunks in the caller's order; ``order`` lists them in
    layout order (grouped by owner rank, ascending chunk index inside a group).
    Offsets and word offsets are in layout order.
    """

    sizes: Tuple[int, ...]
    world: int
    owner: Tuple[int, ...]           # owner rank of each chunk (caller's order)
    order: Tuple[int, ...]           # caller's chunk index at each layout position
    offsets: np.ndarray              # [C+1] element offsets, layout order
    words: np.ndarray                # [C+1] packed-word offsets, layout order
    kbounds: Tuple[int, ...]         # [world+1] layout positions: rank r owns [kbounds[r], kbounds[r+1])
    codes_per_word: int = 32         # 32 sign bits, or 4 int8 codes (momentum-error rule)
    planes: int = 1                  # sign planes per chunk (2: 2-bit Adam)

    @property
    def n(self) -> int:
        return int(self.offsets[-1])

    @property
    def C(self) -> int:
        return len(self.sizes)

    def kslice(self, r: int) -> slice:
        return slice(self.kbounds[r], self.kbounds[r + 1])

    def eslice(self, r: int) -> slice:
        return slice(int(self.offsets[self.kbounds[r]]), int(self.offsets[self.kbounds[r + 1]]))

    def wslice(self, r: int) -> slice:
        return slice(int(self.words[self.kbounds[r]]), int(self.words[self.kbounds[r + 1]]))

    def to_layout(self, per_chunk: Sequence[np.ndarray]) -> np.ndarray:
        """Concatenate per-chunk arrays (caller's order) in layout order."""
        return np.concatenate([per_chunk[k] for k in self.order]) if self.C else np.zeros(0)

    def chunk_position(self, k: int) -> int:
        return self.order.index(k)


def plan(sizes: Sequence[int], world: int, codes_per_word: int = 32, planes: int = 1) -> DPLayout:
    """Assign chunks to ranks (largest first to the least-loaded rank, ties to the
    lower rank) and lay the buffer out grouped by owner.  ``codes_per_word``: 32
    for the sign bits of the scaled-sign rule, 4 for the int8 codes of the
    momentum-error rule; ``planes``: 2 for the two sign planes of 2-bit Adam.
    Every chunk starts on a fresh word."""
    if codes_per_word not in (4, 32):
        raise ValueError("codes_per_word must be 32 (sign bits) or 4 (int8 codes)")
    if planes not in (1, 2) or (planes == 2 and codes_per_word != 32):
        raise ValueError("planes must be 1, or 2 with sign bits")
    sizes = tuple(int(s) for s in sizes)
    if world < 1:
        raise ValueError("world must be >= 1")
    load = [0] * world
    owner = [0] * len(sizes)
    for k in sorted(range(len(sizes)), key=lambda k: (-sizes[k], k)):
        r = min(range(world), key=lambda r: (load[r], r))
        owner[k] = r
        load[r] += sizes[k]
    order = tuple(sorted(range(len(sizes)), key=lambda k: (owner[k], k)))
    lay_sizes = [sizes[k] for k in order]
    offsets = np.zeros(len(sizes) + 1, np.int64)
    np.cumsum(np.asarray(lay_sizes, np.int64), out=offsets[1:])
    words = np.zeros(len(sizes) + 1, np.int64)
    cpw = codes_per_word
    np.cumsum(np.asarray([planes * ((s + cpw - 1) // cpw) for s in lay_sizes], np.int64), out=words[1:])
    kb = [0] * (world + 1)
    for r in range(world):
        kb[r + 1] = kb[r] + sum(1 for k in order if owner[k] == r)
    return DPLayout(sizes, world, tuple(owner), order, offsets, words, tuple(kb), cpw, planes)


# ---- CUDA stage backend ------------------------------------------------------------------

class CudaStages:
    """Per-rank state and the C-ABI ctxs that compute on it.

    local  (W = 1): p, m, v, this rank's err, its words/scales, the full server
                    words/scales (filled by exchange 2) -> worker stage, update.
    server (W = world, owned chunks only): srv_err, the W workers' words/scales
                    of the owned chunks (filled by exchange 1) -> server stage.
    warm   (W = 1, float32 gradients, shares p, m, v): the full-precision warmup
                    step on the averaged gradient (the server ctx averages the
                    owned slices of the W ranks' gradients).
    update (momentum-error rule only; W = world, shares p, m, v, bits_srv): the
                    update divides the code sums by W, which the local ctx's W = 1
                    would get wrong.
    slice_ctx / slice_upd (pipelined schedule): the local (and update) ctxs again,
                    one per owner slice, as views into the same buffers.
    ``rule``: "scaled" (default), "momentum" or "twobit"; the layout must be
    planned for it (codes per word, planes).
    Phases are the driver's: every ctx is created with freeze_step 0 (local,
    server, update) or never leaving warmup (warm).
    """

    def __init__(self, layout: DPLayout, rank: int, *, grad_dtype: str = "f32",
                 optimizer: str = "adam", lr: float = 1e-4, beta1: float = 0.9,
                 beta2: float = 0.999, eps: float = 1e-8, clip: float = 0.0,
                 warmup: bool = True, pipelined: bool = True, rule: str = "scaled", device=None):
        from . import _lib as L
        self.L = L
        self.device = torch.device(device) if device is not None else torch.device("cuda", torch.cuda.current_device())
        self.layout, self.rank = layout, rank
        W, n = layout.world, layout.n
        momentum, twobit = rule == "momentum", rule == "twobit"
        if (layout.codes_per_word, layout.planes) != ((4, 1) if momentum else (32, 2) if twobit else (32, 1)):
            raise ValueError(f"layout planned with {layout.codes_per_word} codes per word and "
                             f"{layout.planes} plane(s), not for rule {rule!r}")
        # The momentum-error rule has no scales and no server error: those are
        # empty.  2-bit Adam has two scales per chunk: [.., C, 2].
        C = 0 if momentum else layout.C
        sp = (2,) if twobit else ()
        code_rule = (L.OB_RULE_MOMENTUM_ERROR if momentum else L.OB_RULE_TWO_BIT if twobit
                     else L.OB_RULE_SCALED_SIGN)
        gd = L.OB_BF16 if grad_dtype == "bf16" else L.OB_F32
        opt = L.OB_LAMB if optimizer == "lamb" else L.OB_ADAM
        hp = dict(lr=lr, beta1=beta1, beta2=beta2, eps=eps, clip=clip)
        dev, f32, i32 = self.device, torch.float32, torch.int32
        words = int(layout.words[-1])
        z = lambda shape, dt=f32: torch.zeros(shape, dtype=dt, device=dev)  # noqa: E731
        self.p, self.m, self.v = z(n), z(n), z(n)
        self.err = z((1, n))
        self.bits_w, self.s_w = z((1, words), i32), z((1, C, *sp))
        self.bits_srv, self.s_srv = z(words, i32), z((C, *sp))
        ptr = lambda t: 0 if t is None or t.numel() == 0 else int(t.data_ptr())  # noqa: E731
        self._keep = []

        def cfg(offsets, workers, freeze):
            c, arr = L.make_config(int(offsets[-1]), offsets, workers, gd, opt, freeze_step=freeze,
                                   rule=code_rule, **hp)
            self._keep.append(arr)
            return c

        with torch.cuda.device(dev):
            self.local = L.ob_create(cfg(layout.offsets, 1, 0), ptr(self.p), ptr(self.m), ptr(self.v),
                                     ptr(self.err), 0, ptr(self.bits_w), ptr(self.s_w),
                                     ptr(self.bits_srv), ptr(self.s_srv))
            ks = layout.kslice(rank)
            off_own = layout.offsets[ks.start: ks.stop + 1] - layout.offsets[ks.start]
            self.n_own, self.C_own = int(off_own[-1]), ks.stop - ks.start
            w_own = layout.wslice(rank).stop - layout.wslice(rank).start
            self.srv_err = z(0 if momentum else self.n_own)
            C_own_scales = 0 if momentum else self.C_own
            self.bits_w_srv, self.s_w_srv = z((W, w_own), i32), z((W, C_own_scales, *sp))
            self.bits_srv_own, self.s_srv_own = z(w_own, i32), z((C_own_scales, *sp))
            self.server = 0
            if self.C_own > 0:
                self.server = L.ob_create(cfg(off_own, W, 0), 0, 0, 0, 0, ptr(self.srv_err),
                                          ptr(self.bits_w_srv), ptr(self.s_w_srv),
                                          ptr(self.bits_srv_own), ptr(self.s_srv_own))
            self.warm = 0
            if warmup:
                c_warm, arr = L.make_config(n, layout.offsets, 1, L.OB_F32, opt, freeze_step=1 << 30,
                                            rule=code_rule, **hp)
                self._keep.append(arr)
                self.warm = L.ob_create(c_warm, ptr(self.p), ptr(self.m), ptr(self.v), 0, 0, 0, 0, 0, 0)
            self.grad_dtype = torch.bfloat16 if gd == L.OB_BF16 else f32
            self._warm_grads: Optional[torch.Tensor] = None   # [W, n_own]: the owned slices of every rank
            self._warm_own: Optional[torch.Tensor] = None     # [n_own]: their average (aligned for the kernel)
            self._warm_mean: Optional[torch.Tensor] = None    # [n]: the averaged gradient
            # The momentum-error rule's update divides the code sums by W, so it runs
            # on a ctx of W = world workers (the worker stage's ctx has one).  The
            # scaled rules' update reads averaged scales: the local ctx serves.
            self.update = 0
            if momentum:
                self.update = L.ob_create(cfg(layout.offsets, W, 0), ptr(self.p), ptr(self.m), ptr(self.v),
                                          0, 0, 0, 0, ptr(self.bits_srv), 0)
            # One worker+update ctx per owner slice (views into the same buffers), so a
            # slice can be compressed and sent while the next one is compressed.  Element
            # arrays of a slice must start 32-byte aligned (16 bf16 elements).
            self.slice_ctx: Optional[List[int]] = None
            self.slice_upd: Optional[List[int]] = None
            if pipelined and W > 1 and all(layout.eslice(o).start % 16 == 0 for o in range(W)):
                self.slice_ctx, self.slice_upd = [], []
                for o in range(W):
                    ks, es, ws = layout.kslice(o), layout.eslice(o), layout.wslice(o)
                    if ks.stop == ks.start:
                        self.slice_ctx.append(0)
                        self.slice_upd.append(0)
                        continue
                    so = layout.offsets[ks.start: ks.stop + 1] - es.start
                    e4, w4, k4 = 4 * es.start, 4 * ws.start, 4 * (2 if twobit else 1) * ks.start
                    at = lambda t, b: ptr(t) + b if t.numel() else 0  # noqa: E731
                    h = L.ob_create(cfg(so, 1, 0), at(self.p, e4), at(self.m, e4), at(self.v, e4),
                                    at(self.err, e4), 0, at(self.bits_w, w4), at(self.s_w, k4),
                                    at(self.bits_srv, w4), at(self.s_srv, k4))
                    self.slice_ctx.append(h)
                    self.slice_upd.append(L.ob_create(cfg(so, W, 0), at(self.p, e4), at(self.m, e4),
                                                      at(self.v, e4), 0, 0, 0, 0, at(self.bits_srv, w4), 0)
                                          if momentum else h)

    def _stream(self) -> int:
        return int(torch.cuda.current_stream(self.device).cuda_stream)

    # -- warmup: average owner by owner, then a one-worker step on the average --
    def warm_buffers(self) -> Tuple[torch.Tensor, torch.Tensor, torch.Tensor]:
        """([W, n_own] owned gradient slices of every rank, [n_own] their float32
        average, [n] float32 averaged gradient), allocated on the first warmup step."""
        if self._warm_grads is None:
            dev = self.device
            self._warm_grads = torch.zeros((self.layout.world, self.n_own), dtype=self.grad_dtype, device=dev)
            self._warm_own = torch.zeros(self.n_own, dtype=torch.float32, device=dev)
            self._warm_mean = torch.zeros(self.layout.n, dtype=torch.float32, device=dev)
        return self._warm_grads, self._warm_own, self._warm_mean

    def warm_mean_own(self) -> None:
        """Average the W ranks' slices of the owned chunks (into the [n_own] buffer)."""
        if self.server:
            self.L.ob_mean_grads(self.server, int(self._warm_grads.data_ptr()), int(self._warm_own.data_ptr()),
                                 self._stream())

    def warmup(self) -> None:
        """The full-precision step on the averaged gradient."""
        self.L.ob_warmup_step(self.warm, int(self._warm_mean.data_ptr()), self._stream())

    def local_step(self, grad: torch.Tensor) -> None:
        self.L.ob_local_step(self.local, int(grad.data_ptr()), self._stream())

    def compress(self, grad: torch.Tensor) -> None:
        self.L.ob_compress(self.local, int(grad.data_ptr()), self._stream())

    @property
    def pipelined(self) -> bool:
        return self.slice_ctx is not None

    def compress_slice(self, o: int, grad_slice: torch.Tensor) -> None:
        if self.slice_ctx[o]:
            self.L.ob_compress(self.slice_ctx[o], int(grad_slice.data_ptr()), self._stream())

    def apply_slice(self, o: int) -> None:
        if self.slice_upd[o]:
            self.L.ob_step(self.slice_upd[o], None, self._stream())

    def server_reduce(self) -> None:
        if self.server:
            self.L.ob_server_reduce(self.server, self._stream())

    def apply(self) -> None:
        self.L.ob_step(self.update or self.local, None, self._stream())

    def status(self) -> int:
        st = self._stream()
        f = self.L.ob_get_status(self.local, False, st)
        if self.server:
            f |= self.L.ob_get_status(self.server, False, st)
        if self.warm:
            f |= self.L.ob_get_status(self.warm, False, st)
        if self.update:
            f |= self.L.ob_get_status(self.update, False, st)
        for h in set(self.slice_ctx or []) | set(self.slice_upd or []):
            if h:
                f |= self.L.ob_get_status(h, False, st)
        return f

    def close(self) -> None:
        for name in ("local", "server", "warm", "update"):
            h = getattr(self, name, 0)
            if h:
                self.L.ob_destroy(h)
                setattr(self, name, 0)
        for h in set(self.slice_ctx or []) | set(self.slice_upd or []):
            if h:
                self.L.ob_destroy(h)
        self.slice_ctx = self.slice_upd = None


# ---- the data-parallel optimizer -------------------------------------------------------

class _Pending:
    """Posted point-to-point works plus the host-staged receives to copy back."""

    def __init__(self, works, copy_back):
        self.works, self.copy_back = works, copy_back

    def wait(self) -> None:
        for w in self.works:
            w.wait()
        for t, dst in self.copy_back:
            t.copy_(dst)
        self.works, self.copy_back = [], []


class DistributedOneBitAdam:
    """One rank of data-parallel 1-bit Adam (worker w = rank w).

    ``step(grad)`` takes this rank's gradient as a flat tensor in layout order
    (``layout.to_layout`` / ``layout.eslice``) and runs a warmup step while
    ``step_count < freeze_step``, the compressed step afterwards.
    """

    def __init__(self, layout: DPLayout, stages, *, freeze_step: int = 0, group=None):
        self.layout, self.stages = layout, stages
        self.group = group
        self.rank = dist.get_rank(group)
        self.world = dist.get_world_size(group)
        if self.world != layout.world:
            raise ValueError(f"layout planned for {layout.world} ranks, group has {self.world}")
        self.freeze_step = int(freeze_step)
        self.step_count = 0
        self._stage_on_host = dist.get_backend(group) == "gloo"

    # -- point-to-point with optional host staging (gloo has no CUDA transport) --
    def _p2p(self, sends: List[Tuple[torch.Tensor, int]], recvs: List[Tuple[torch.Tensor, int]],
             wait: bool = True) -> "_Pending":
        """Post one grouped batch of sends and receives.  With ``wait=False`` the
        caller waits on the returned handle later (on NCCL that makes the current
        stream wait for the transfer, so kernels enqueued meanwhile overlap it)."""
        host = self._stage_on_host
        ops, copy_back = [], []
        as_bits = lambda t: t.view(torch.int16) if t.dtype == torch.bfloat16 else t  # noqa: E731
        sends = [(as_bits(t), peer) for t, peer in sends]
        recvs = [(as_bits(t), peer) for t, peer in recvs]
        for t, peer in sends:
            if t.numel():
                src = t.detach().to("cpu") if host and t.is_cuda else t.contiguous()
                ops.append(dist.P2POp(dist.isend, src, peer, self.group))
        for t, peer in recvs:
            if t.numel():
                dst = torch.empty(t.shape, dtype=t.dtype) if host and t.is_cuda else t
                ops.append(dist.P2POp(dist.irecv, dst, peer, self.group))
                if dst is not t:
                    copy_back.append((t, dst))
        pending = _Pending(dist.batch_isend_irecv(ops) if ops else [], copy_back)
        if wait:
            pending.wait()
        return pending

    def _to_owners(self) -> None:
        """Exchange 1: this rank's words/scales of owner o's chunks -> rank o."""
        L, s, r = self.layout, self.stages, self.rank
        sends, recvs = [], []
        for o in range(self.world):
            wsl, ksl = L.wslice(o), L.kslice(o)
            if o == r:
                s.bits_w_srv[r].copy_(s.bits_w[0, wsl])
                s.s_w_srv[r].copy_(s.s_w[0, ksl])
            else:
                sends += [(s.bits_w[0, wsl], o), (s.s_w[0, ksl], o)]
                recvs += [(s.bits_w_srv[o], o), (s.s_w_srv[o], o)]
        self._p2p(sends, recvs)

    def _from_owners(self) -> None:
        """Exchange 2: owner o's server words/scales -> every rank."""
        L, s, r = self.layout, self.stages, self.rank
        sends, recvs = [], []
        for o in range(self.world):
            wsl, ksl = L.wslice(o), L.kslice(o)
            if o == r:
                s.bits_srv[wsl].copy_(s.bits_srv_own)
                s.s_srv[ksl].copy_(s.s_srv_own)
            else:
                sends += [(s.bits_srv_own, o), (s.s_srv_own, o)]
                recvs += [(s.bits_srv[wsl], o), (s.s_srv[ksl], o)]
        self._p2p(sends, recvs)

    def _compressed_step_pipelined(self, grad: torch.Tensor) -> None:
        """Exchange 1 and 2 as W-1 shifted rounds.  In round i this rank sends to
        rank r+i and receives from rank r-i, so every round pairs the ranks
        consistently whatever their number.  Exchange 1: slice r+i is compressed
        just before its round is posted, so its transfer overlaps the
        compression of the next slice; the server stage waits for all rounds.
        Exchange 2: all rounds are posted at once, then slice r-i is updated as
        soon as round i has arrived."""
        L, s, r, W = self.layout, self.stages, self.rank, self.world
        pending = []
        for i in range(1, W):
            to, frm = (r + i) % W, (r - i) % W
            s.compress_slice(to, grad[L.eslice(to)])
            pending.append(self._p2p(
                [(s.bits_w[0, L.wslice(to)], to), (s.s_w[0, L.kslice(to)], to)],
                [(s.bits_w_srv[frm], frm), (s.s_w_srv[frm], frm)], wait=False))
        s.compress_slice(r, grad[L.eslice(r)])
        s.bits_w_srv[r].copy_(s.bits_w[0, L.wslice(r)])
        s.s_w_srv[r].copy_(s.s_w[0, L.kslice(r)])
        for pend in pending:
            pend.wait()
        s.server_reduce()
        pending = []
        for i in range(1, W):
            to, frm = (r + i) % W, (r - i) % W
            pending.append(self._p2p(
                [(s.bits_srv_own, to), (s.s_srv_own, to)],
                [(s.bits_srv[L.wslice(frm)], frm), (s.s_srv[L.kslice(frm)], frm)], wait=False))
        s.bits_srv[L.wslice(r)].copy_(s.bits_srv_own)
        s.s_srv[L.kslice(r)].copy_(s.s_srv_own)
        s.apply_slice(r)
        for i, pend in enumerate(pending, 1):
            pend.wait()
            s.apply_slice((r - i) % W)

    def _warmup_step(self, grad: torch.Tensor) -> None:
        """Full-precision step: (1) every rank sends owner o its gradient slice of
        o's chunks; (2) each owner averages the W slices in rank order; (3) the
        owners send their averaged slices to every rank; (4) every rank runs the
        one-worker warmup on the averaged gradient."""
        L, s, r = self.layout, self.stages, self.rank
        G, own, gbar = s.warm_buffers()
        sends, recvs = [], []
        for o in range(self.world):
            es = L.eslice(o)
            if o == r:
                G[r].copy_(grad[es])
            else:
                sends.append((grad[es], o))
                recvs.append((G[o], o))
        self._p2p(sends, recvs)
        s.warm_mean_own()
        gbar[L.eslice(r)].copy_(own)
        sends = [(own, o) for o in range(self.world) if o != r]
        recvs = [(gbar[L.eslice(o)], o) for o in range(self.world) if o != r]
        self._p2p(sends, recvs)
        s.warmup()

    @property
    def in_warmup(self) -> bool:
        return self.step_count < self.freeze_step

    def step(self, grad: torch.Tensor) -> None:
        if grad.numel() != self.layout.n:
            raise ValueError(f"gradient must hold {self.layout.n} elements (layout order)")
        if self.in_warmup:
            self._warmup_step(grad.reshape(-1))
        elif getattr(self.stages, "pipelined", False):
            self._compressed_step_pipelined(grad.reshape(-1))
        else:
            self.stages.compress(grad)
            self._to_owners()
            self.stages.server_reduce()
            self._from_owners()
            self.stages.apply()
        self.step_count += 1

    def local_step(self, grad: torch.Tensor) -> None:
        """0/1 Adam local step (compressed phase): no exchange; this rank keeps its
        gradient in its error buffer for the next synchronised step and moves its
        replica with the current m and v.  Every rank must take the same
        schedule of local and synchronised steps."""
        if grad.numel() != self.layout.n:
            raise ValueError(f"gradient must hold {self.layout.n} elements (layout order)")
        if self.in_warmup:
            raise ValueError("local steps belong to the compressed phase")
        self.stages.local_step(grad.reshape(-1))
        self.step_count += 1

    def status(self) -> int:
        """Status flags OR-ed over all ranks."""
        f = torch.tensor([self.stages.status()], dtype=torch.int64)
        if not self._stage_on_host and torch.cuda.is_available():
            f = f.to(self.stages.device)
        dist.all_reduce(f, op=dist.ReduceOp.MAX, group=self.group)  # one flag bit in use
        return int(f.item())
