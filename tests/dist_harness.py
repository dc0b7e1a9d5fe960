"""Multi-rank harness for the data-parallel driver (bit_adam_error_b200.distributed).

``OracleStages`` is a CPU stage backend with the interface of ``CudaStages``,
computing with the oracle, so the driver's ownership plan and both exchanges
run under gloo on CPU ranks; ``run_ranks`` spawns the ranks and collects each
rank's final state; ``reference`` runs the same workload as one W-worker
oracle problem in the caller's chunk order.  Test infrastructure only.
"""

from __future__ import annotations

import datetime
import os
import socket
import traceback

import numpy as np
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

HP = dict(lr=1e-4, beta1=0.9, beta2=0.999, eps=1e-8)


class OracleStages:
    """``pipelined``: also offer the per-owner-slice stages (compress_slice,
    apply_slice), so the driver takes its overlapped schedule."""

    def __init__(self, layout, rank, optimizer="adam", clip=0.0, pipelined=False, rule="scaled",
                 grad_dtype="f32"):
        import oracle
        self.o = oracle.get()
        self.grad_dtype = grad_dtype
        self.layout, self.rank = layout, rank
        self.opt = oracle.LAMB if optimizer == "lamb" else oracle.ADAM
        self.clip = clip
        self.device = torch.device("cpu")
        self.momentum, self.twobit = rule == "momentum", rule == "twobit"
        W, n = layout.world, layout.n
        C = 0 if self.momentum else layout.C
        sp = (2,) if self.twobit else ()
        words = int(layout.words[-1])
        f32, i32 = torch.float32, torch.int32
        self.p, self.m, self.v = torch.zeros(n), torch.zeros(n), torch.zeros(n)
        self.err = torch.zeros((1, n))
        self.bits_w, self.s_w = torch.zeros((1, words), dtype=i32), torch.zeros((1, C, *sp))
        self.bits_srv, self.s_srv = torch.zeros(words, dtype=i32), torch.zeros((C, *sp))
        ks, wsl = layout.kslice(rank), layout.wslice(rank)
        self.off_own = layout.offsets[ks.start: ks.stop + 1] - layout.offsets[ks.start]
        c_own = 0 if self.momentum else ks.stop - ks.start
        self.srv_err = torch.zeros(0 if self.momentum else int(self.off_own[-1]))
        self.bits_w_srv = torch.zeros((W, wsl.stop - wsl.start), dtype=i32)
        self.s_w_srv = torch.zeros((W, c_own, *sp), dtype=f32)
        self.bits_srv_own = torch.zeros(wsl.stop - wsl.start, dtype=i32)
        self.s_srv_own = torch.zeros((c_own, *sp), dtype=f32)
        self.flags = 0
        self.pipelined = bool(pipelined) and layout.world > 1

    @staticmethod
    def _u32(t):
        return t.numpy().view(np.uint32)

    # -- warmup: the owned slices of every rank are averaged by the owner ------------
    def warm_buffers(self):
        if not hasattr(self, "_warm"):
            n_own = int(self.off_own[-1])
            gdt = torch.bfloat16 if self.grad_dtype == "bf16" else torch.float32
            self._warm = (torch.zeros((self.layout.world, n_own), dtype=gdt), torch.zeros(n_own),
                          torch.zeros(self.layout.n))
        return self._warm

    def warm_mean_own(self):
        """The owner's average of the W slices: float32 additions in rank order,
        then one division by W (numpy's IEEE float32 arithmetic, the statement
        the oracle's warmup makes before its moments)."""
        G, own, _ = self._warm
        rows = self._grad_rows(G) if G.dtype == torch.bfloat16 else G.numpy()
        if rows.dtype == np.uint16:
            rows = (rows.astype(np.uint32) << np.uint32(16)).view(np.float32).reshape(G.shape)
        acc = np.zeros(rows.shape[1], np.float32)
        for w in range(rows.shape[0]):
            acc = (acc + rows[w]).astype(np.float32)
        own.numpy()[:] = (acc / np.float32(rows.shape[0])).astype(np.float32)

    def warmup(self):
        """The oracle's warmup with one worker on the averaged gradient."""
        f = {k: np.float32(v) for k, v in HP.items()}
        gbar = np.ascontiguousarray(self._warm[2].numpy().reshape(1, -1))
        self.flags |= self.o.warmup(self.layout.offsets, gbar, self.m.numpy(), self.v.numpy(), self.p.numpy(),
                                    f["beta1"], f["beta2"], f["lr"], f["eps"], optimizer=self.opt)

    def local_step(self, grad):
        f = {k: np.float32(v) for k, v in HP.items()}
        st = {"p": self.p.numpy(), "m": self.m.numpy(), "v": self.v.numpy(), "err": self.err.numpy()}
        self.flags |= self.o.local_step(self.layout.offsets, self._grad_rows(grad), st, f["lr"], f["eps"],
                                        clip=self.clip, optimizer=self.opt)

    @staticmethod
    def _grad_rows(grad):
        if grad.dtype == torch.bfloat16:
            return np.ascontiguousarray(grad.view(torch.int16).numpy().view(np.uint16).reshape(1, -1))
        return np.ascontiguousarray(grad.numpy().reshape(1, -1))

    def compress(self, grad):
        if self.momentum:
            codes, fl = self.o.ternary_compress(self.layout.offsets, self._grad_rows(grad), self.err.numpy(),
                                                np.float32(HP["beta1"]), clip=self.clip)
            self.bits_w.numpy().view(np.int8)[:] = codes
            self.flags |= fl
            return
        fn = self.o.twobit_compress if self.twobit else self.o.compress
        bits, s, fl = fn(self.layout.offsets, self._grad_rows(grad), self.err.numpy(), clip=self.clip)
        self._u32(self.bits_w)[:] = bits
        self.s_w.numpy()[:] = s
        self.flags |= fl

    def _slice_offsets(self, o):
        ks, es = self.layout.kslice(o), self.layout.eslice(o)
        return self.layout.offsets[ks.start: ks.stop + 1] - es.start

    def compress_slice(self, o, grad_slice):
        L = self.layout
        ks, es, wsl = L.kslice(o), L.eslice(o), L.wslice(o)
        if ks.stop == ks.start:
            return
        err = self.err.numpy()[0, es].reshape(1, -1)
        if self.momentum:
            codes, fl = self.o.ternary_compress(self._slice_offsets(o), self._grad_rows(grad_slice), err,
                                                np.float32(HP["beta1"]), clip=self.clip)
            self.bits_w.numpy().view(np.int8)[0, 4 * wsl.start: 4 * wsl.stop] = codes[0]
            self.flags |= fl
            return
        fn = self.o.twobit_compress if self.twobit else self.o.compress
        bits, s, fl = fn(self._slice_offsets(o), self._grad_rows(grad_slice), err, clip=self.clip)
        self._u32(self.bits_w)[0, wsl] = bits[0]
        self.s_w.numpy()[0, ks] = s[0]
        self.flags |= fl

    def server_reduce(self):
        if self.momentum:
            if self.bits_w_srv.shape[1]:
                sums = self.o.ternary_server(self.off_own, np.ascontiguousarray(self.bits_w_srv.numpy().view(np.int8)))
                self.bits_srv_own.numpy().view(np.int8)[:] = sums
            return
        if self.s_w_srv.shape[1] == 0:
            return
        fn = self.o.twobit_server if self.twobit else self.o.server_reduce
        bits, s, fl = fn(self.off_own, np.ascontiguousarray(self._u32(self.bits_w_srv)),
                         np.ascontiguousarray(self.s_w_srv.numpy()), self.srv_err.numpy())
        self._u32(self.bits_srv_own)[:] = bits
        self.s_srv_own.numpy()[:] = s
        self.flags |= fl

    def apply(self):
        f = {k: np.float32(v) for k, v in HP.items()}
        if self.momentum:
            self.flags |= self.o.ternary_apply(self.layout.offsets, self.layout.world,
                                               self.bits_srv.numpy().view(np.int8), self.m.numpy(),
                                               self.v.numpy(), self.p.numpy(), f["beta1"], f["lr"], f["eps"],
                                               optimizer=self.opt)[1]
            return
        args = (self.layout.offsets, self._u32(self.bits_srv), self.s_srv.numpy(), self.m.numpy(),
                self.v.numpy(), self.p.numpy(), f["beta1"], f["lr"], f["eps"])
        if self.twobit:
            self.flags |= self.o.twobit_apply(*args, optimizer=self.opt)[1]
        elif self.opt:
            self.flags |= self.o.lamb_apply(*args)[1]
        else:
            self.flags |= self.o.adam_apply(*args)

    def apply_slice(self, o):
        L = self.layout
        ks, es, wsl = L.kslice(o), L.eslice(o), L.wslice(o)
        if ks.stop == ks.start:
            return
        f = {k: np.float32(v) for k, v in HP.items()}
        if self.momentum:
            sums = np.ascontiguousarray(self.bits_srv.numpy().view(np.int8)[4 * wsl.start: 4 * wsl.stop])
            self.flags |= self.o.ternary_apply(self._slice_offsets(o), L.world, sums, self.m.numpy()[es],
                                               self.v.numpy()[es], self.p.numpy()[es], f["beta1"], f["lr"],
                                               f["eps"], optimizer=self.opt)[1]
            return
        args = (self._slice_offsets(o), self._u32(self.bits_srv)[wsl], self.s_srv.numpy()[ks],
                self.m.numpy()[es], self.v.numpy()[es], self.p.numpy()[es], f["beta1"], f["lr"], f["eps"])
        if self.twobit:
            self.flags |= self.o.twobit_apply(*args, optimizer=self.opt)[1]
        elif self.opt:
            self.flags |= self.o.lamb_apply(*args)[1]
        else:
            self.flags |= self.o.adam_apply(*args)

    def status(self):
        return self.flags


def free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def workload(sizes, world, **kw):
    import workloads as WL
    return WL.get_workload("tiny").with_(sizes=tuple(sizes), W=world, **kw)


def rank_inputs(wl, layout, rank, step):
    """This rank's gradient at `step` in layout order (worker = rank)."""
    import workloads as WL
    return layout.to_layout([WL.chunk_grads(wl, step, rank, k) for k in range(wl.C)])


def initial_state(wl, layout):
    import workloads as WL
    ps, vs = zip(*[WL.chunk_state(wl, k) for k in range(wl.C)])
    return layout.to_layout(ps).astype(np.float32), layout.to_layout(vs).astype(np.float32)


def _rank_main(rank, world, port, sizes, wl_kw, steps, backend, device, q, die=None, timeout_s=120,
               pipelined=False, rule="scaled", schedule=None):
    try:
        import sys
        sys.path.insert(0, ROOT)
        sys.path.insert(0, os.path.join(ROOT, "tests"))
        import torch.distributed as dist
        from bit_adam_error_b200.distributed import DistributedOneBitAdam, plan
        os.environ["MASTER_ADDR"] = "127.0.0.1"
        os.environ["MASTER_PORT"] = str(port)
        if device != "cpu":
            torch.cuda.set_device(torch.device(device))
        dist.init_process_group(backend, rank=rank, world_size=world,
                                timeout=datetime.timedelta(seconds=timeout_s))
        wl = workload(sizes, world, **wl_kw)
        layout = plan(sizes, world, 4 if rule == "momentum" else 32, 2 if rule == "twobit" else 1)
        if device == "cpu":
            stages = OracleStages(layout, rank, optimizer=wl.optimizer, clip=wl.clip, pipelined=pipelined,
                                  rule=rule, grad_dtype=wl.grad_dtype)
        else:
            from bit_adam_error_b200.distributed import CudaStages
            stages = CudaStages(layout, rank, grad_dtype=wl.grad_dtype, optimizer=wl.optimizer,
                                clip=wl.clip, warmup=wl.freeze_step > 0, pipelined=pipelined,
                                rule=rule, device=device, **HP)
        p0, v0 = initial_state(wl, layout)
        stages.p.copy_(torch.from_numpy(p0))
        stages.v.copy_(torch.from_numpy(v0))
        drv = DistributedOneBitAdam(layout, stages, freeze_step=wl.freeze_step)
        for t in range(steps):
            if die is not None and die == (rank, t):
                os._exit(17)             # an injected rank failure between steps
            g = rank_inputs(wl, layout, rank, t)
            gt = torch.from_numpy(g.view(np.int16)).view(torch.bfloat16) if g.dtype == np.uint16 \
                else torch.from_numpy(g)
            if schedule is not None and schedule[t] == "L":
                drv.local_step(gt.to(stages.device))
            else:
                drv.step(gt.to(stages.device))
        flags = drv.status()
        schedule = "pipelined" if getattr(stages, "pipelined", False) else "grouped"
        if device != "cpu":
            torch.cuda.synchronize()

        def host(t):
            a = t.detach().cpu().numpy()
            return a.view(np.uint32) if a.dtype == np.int32 else a.copy()

        out = {k: host(getattr(stages, k)) for k in ("p", "m", "v", "err", "srv_err", "bits_srv", "s_srv")}
        out["flags"] = flags
        out["schedule"] = schedule
        if hasattr(stages, "close"):
            stages.close()
        dist.destroy_process_group()
        q.put((rank, out))
    except Exception:
        q.put((rank, {"error": traceback.format_exc()}))


def run_ranks(sizes, world, wl_kw, steps, backend="gloo", device="cpu", timeout=600, pipelined=False,
              rule="scaled", schedule=None):
    """Spawn `world` ranks; returns the list of per-rank final states.  ``schedule``:
    one letter per step, "L" for a 0/1 Adam local step (else a regular step)."""
    import multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, sizes, wl_kw, steps, backend, device, q),
                         kwargs=dict(pipelined=pipelined, rule=rule, schedule=schedule)) for r in range(world)]
    for pr in procs:
        pr.start()
    results = {}
    try:
        for _ in range(world):
            r, out = q.get(timeout=timeout)
            results[r] = out
    finally:
        for pr in procs:
            pr.join(timeout=30)
            if pr.is_alive():
                pr.kill()
    for r, out in results.items():
        assert "error" not in out, f"rank {r} failed:\n{out['error']}"
    return [results[r] for r in range(world)]


def reference(sizes, world, wl_kw, steps, rule="scaled", schedule=None):
    """The same workload as one W-worker oracle problem (caller's chunk order);
    ``schedule`` as for run_ranks."""
    import oracle
    import workloads as WL
    wl = workload(sizes, world, **wl_kw)
    o = oracle.get()
    n = wl.n
    p = np.zeros(n, np.float32)
    v = np.zeros(n, np.float32)
    WL.fill_state(wl, p, v)
    st = {"p": p, "m": np.zeros(n, np.float32), "v": v, "err": np.zeros((world, n), np.float32),
          "srv_err": np.zeros(n, np.float32)}
    f = {k: np.float32(x) for k, x in HP.items()}
    opt = oracle.LAMB if wl.optimizer == "lamb" else oracle.ADAM
    for t in range(steps):
        dt = np.uint16 if wl.grad_dtype == "bf16" else np.float32
        g = np.zeros((world, n), dt)
        WL.fill_grads(wl, t, g)
        if t < wl.freeze_step:
            o.warmup(wl.offsets, g, st["m"], st["v"], st["p"], f["beta1"], f["beta2"], f["lr"], f["eps"],
                     optimizer=opt)
        elif schedule is not None and schedule[t] == "L":
            o.local_step(wl.offsets, g, st, f["lr"], f["eps"], clip=wl.clip, optimizer=opt)
        elif rule == "momentum":
            o.ternary_step(wl.offsets, g, st, f["beta1"], f["lr"], f["eps"], clip=wl.clip, optimizer=opt)
        elif rule == "twobit":
            o.twobit_step(wl.offsets, g, st, f["beta1"], f["lr"], f["eps"], clip=wl.clip, optimizer=opt)
        else:
            o.step(wl.offsets, g, st, f["beta1"], f["lr"], f["eps"], clip=wl.clip, optimizer=opt)
    return wl, st


def compare(layout, wl, ref, outs, exact=True):
    planes = layout.planes
    """Every rank's state against the W-worker oracle, mapped to layout order:
    bit for bit (exact) or to the parity bar of the GPU tests."""
    off = wl.offsets

    def lay(a):  # caller-order flat array -> layout order
        return layout.to_layout([a[..., off[k]:off[k + 1]] for k in range(wl.C)]) if a.ndim == 1 else \
            np.stack([lay(r) for r in a])

    if "bits_srv" in ref:          # the scaled-sign rule: server words, scales, server error
        wb = np.zeros(wl.C + 1, np.int64)
        np.cumsum([planes * ((s + 31) // 32) for s in wl.sizes], out=wb[1:])
        bits_ref = layout.to_layout([ref["bits_srv"][wb[k]:wb[k + 1]] for k in range(wl.C)]).astype(np.uint32)
        s_ref = np.array([ref["s_srv"][k] for k in layout.order], np.float32)
        srv_ref = lay(ref["srv_err"])
    if exact:
        same = lambda name, got, want: np.testing.assert_array_equal(got, want, err_msg=name)  # noqa: E731
        scales = same
    else:
        from gpu_harness import assert_scales, assert_state
        same = lambda name, got, want: assert_state(name, got, want, layout.offsets)  # noqa: E731
        scales = assert_scales
    for r, out in enumerate(outs):
        for key in ("p", "m", "v"):
            same(f"rank {r} {key}", out[key], lay(ref[key]))
        same(f"rank {r} err", out["err"][0], lay(ref["err"][r]))
        if "codes_srv" in ref:        # momentum-error rule: the code sums, byte for byte
            cb = np.zeros(wl.C + 1, np.int64)
            np.cumsum([(s + 3) // 4 for s in wl.sizes], out=cb[1:])
            want = layout.to_layout([ref["codes_srv"][4 * cb[k]: 4 * cb[k + 1]] for k in range(wl.C)])
            assert np.array_equal(out["bits_srv"].view(np.int8), want.astype(np.int8)), (r, "code sums")
        if "bits_w" in ref:
            assert np.array_equal(out["bits_srv"], bits_ref), (r, "bits_srv")
            scales(f"rank {r} s_srv", out["s_srv"], s_ref)
            es = layout.eslice(r)
            own_off = layout.offsets[layout.kslice(r).start: layout.kslice(r).stop + 1] - es.start
            got, want = out["srv_err"], srv_ref[es]
            if exact:
                np.testing.assert_array_equal(got, want, err_msg=f"rank {r} srv_err")
            else:
                from gpu_harness import assert_state
                assert_state(f"rank {r} srv_err", got, want, own_off)


def run_with_dead_rank(sizes, world, wl_kw, steps, die, timeout_s=15):
    """Spawn the ranks with rank die[0] exiting before its step die[1]; returns
    ({rank: result or error}, {rank: exit code})."""
    import multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, sizes, wl_kw, steps, "gloo", "cpu", q,
                                                  die, timeout_s)) for r in range(world)]
    for pr in procs:
        pr.start()
    results = {}
    try:
        for _ in range(world - 1):
            r, out = q.get(timeout=timeout_s * 6)
            results[r] = out
    finally:
        for pr in procs:
            pr.join(timeout=30)
            if pr.is_alive():
                pr.kill()
    return results, {r: pr.exitcode for r, pr in enumerate(procs)}
