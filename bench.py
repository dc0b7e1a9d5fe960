#!/usr/bin/env python
"""Benchmark of the 1-bit Adam compressed-phase step on B200.

One step = one pass of the whole fused compressed step (worker stage with
per-chunk scales, server stage, frozen-v Adam update) over one batch of
synthetic gradients of the workload, through ``OneBitAdam.step`` ->
``ob_step``.  Default workload: the flat 1.5e9-element GPT-2-XL-sized buffer
(23 chunks of 2^26 elements, W = 1 worker, bf16 gradients, fp32 state).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Prints one JSON line (rank 0).  ``value`` is whole-job Gelem/s (elements of
all replicas / max-over-ranks device time per step), measured with CUDA
events with all inputs resident in HBM; ``e2e`` is the same metric through
the public call with host (pinned) gradients, so the host-to-device copy of
every step's gradients and a device-to-host read of its scales are inside
the timed region.  ``roofline`` reports the dominant kernel's algorithmic
bytes per launch over its CUDA-event time on its launch stream against the
measured HBM copy bandwidth.  ``cpu_baseline`` times the CPU oracle (the
plain C statement of the method) on one host thread and on all host cores, on
the same sample of whole chunks.  ``--impl reference`` times the oracle on all
host cores, one bounded sample (chunk 0) per bench step.

Multi-GPU (N > 1 under torchrun): real data parallelism -- rank w is worker
w, holding the whole model and its own gradient of the workload; the
compressed allreduce runs as two NCCL point-to-point exchanges of packed words
around a chunk-owner server stage.  Per-rank work is fixed, so scaling is weak
and ``value`` counts the gradient elements of all ranks.  ``--replicas`` times
independent single-GPU replicas instead (no collective).
"""

from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

METRIC = "compressed-phase 1-bit Adam step: Gelem/s and HBM GB/s as % of B200 peak"
UNIT = "Gelem/s"
FALLBACK_HBM_GBS = 6650.0
E2E_MAX_HOST_BYTES = 16e9        # pinned host gradients per step the e2e leg may hold
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "ncu_traffic.txt")
KERNEL_SOURCES = [os.path.join(ROOT, "bit_adam_error_b200", "csrc", f)
                  for f in ("kernels.cuh", "ternary.cuh", "twobit.cuh", "onebit.cu")]


def parse_args():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="gpt2xl-flat")
    ap.add_argument("--chunks", type=int, default=0,
                    help="use only the first K chunks of the workload (a smaller case, e.g. for ncu)")
    ap.add_argument("--grad-buffers", type=int, default=2,
                    help="distinct gradient batches cycled through the timed steps")
    ap.add_argument("--phase", choices=["compressed", "refresh", "local"], default="compressed",
                    help="time the compressed step (default), the full-precision variance-refresh "
                         "step of 0/1 Adam, or its local step")
    ap.add_argument("--rule", choices=["scaled", "momentum", "twobit"], default="scaled",
                    help="compression rule: scaled sign bits with worker and server error "
                         "(default), the momentum-error rule with int8 ternary codes, or "
                         "2-bit Adam (two residual sign planes)")
    ap.add_argument("--err-dtype", choices=["f32", "bf16"], default=None,
                    help="storage of the error buffers (default: the workload's, f32)")
    ap.add_argument("--dp", action="store_true",
                    help="time the real data-parallel path (worker w = rank w, NCCL exchanges) even "
                         "at one GPU (with more than one GPU it is the default)")
    ap.add_argument("--replicas", action="store_true",
                    help="with more than one GPU, time independent replicas of the single-GPU step "
                         "(no collective) instead of the data-parallel step")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    a = ap.parse_args()
    if a.warmup < 3:
        ap.error("--warmup must be >= 3")
    if a.steps < 1:
        ap.error("--steps must be >= 1")
    return a


# -- algorithmic traffic per element (three-pass schedule) ---------------------------

def algo_bytes_per_elem(kind: str, wl) -> float:
    """HBM bytes per element that kernel kind must move in the fused step
    (gb = gradient bytes, eb = error-buffer bytes: 4, or 2 when stored as bf16)."""
    W, gb, eb = wl.W, wl.grad_bytes, wl.err_bytes
    if kind == "k_worker_norm":          # read g, err for every worker
        return (gb + eb) * W
    if kind == "k_worker_pack":          # read g, err, write err, signs; read srv_err
        return (gb + 2 * eb) * W + W / 8 + eb
    if kind == "k_server_update":
        if wl.optimizer == "lamb":       # signs, srv_err r/w, server signs, m r/w, v, p reads
            return W / 8 + 2 * eb + 1 / 8 + 16
        return W / 8 + 2 * eb + 1 / 8 + 20  # + m, v, p reads and m, p writes
    if kind == "k_lamb_param":           # m, v, p reads, p write
        return 16.0
    if kind == "k_warmup":               # g (xW), m, v, p reads; m, v (+ p for Adam) writes
        return gb * W + (20 if wl.optimizer == "lamb" else 24)
    # the momentum-error rule
    if kind == "k_ternary_step":         # g, err r/w per worker; m r/w, v, p r (+ p w for Adam)
        return (gb + 2 * eb) * W + (16 if wl.optimizer == "lamb" else 20)
    if kind == "k_ternary_compress":     # g, err r/w, one code byte per worker
        return (gb + 2 * eb + 1) * W
    if kind == "k_ternary_server":       # W code bytes in, one sum byte out
        return W + 1.0
    if kind == "k_ternary_update":       # one sum byte, m r/w, v, p r (+ p w for Adam)
        return 1 + (16 if wl.optimizer == "lamb" else 20)
    # 2-bit Adam: two sign planes per message
    if kind == "k_tb_worker_norm":       # g, err of every worker (both scales' sums)
        return (gb + eb) * W
    if kind == "k_tb_pack":              # g, err r/w, both planes; srv_err read
        return (gb + 2 * eb) * W + W / 4 + eb
    if kind == "k_tb_server_norm":       # both planes of every worker, srv_err (stage call)
        return W / 4 + eb
    if kind == "k_tb_server_update":     # planes, srv_err r/w, server planes (+ m, v, p as Adam/LAMB)
        return W / 4 + 2 * eb + 1 / 4 + (16 if wl.optimizer == "lamb" else 20)
    # W >= 4: pass 2 also stores c_srv (4 B); pass 3 reads it instead of the W
    # workers' words and the server error
    upd = 16 if wl.optimizer == "lamb" else 20
    if kind == "k_worker_pack_cached":
        return algo_bytes_per_elem("k_worker_pack", wl) + 4
    if kind == "k_server_update_cached":  # c_srv, srv_err written, server signs, m, v, p
        return 4 + eb + 1 / 8 + upd
    if kind == "k_tb_pack_cached":
        return algo_bytes_per_elem("k_tb_pack", wl) + 4
    if kind == "k_tb_server_update_cached":
        return 4 + eb + 1 / 4 + upd
    # 0/1 Adam's local step: g, err r/w per worker; m, v, p reads (+ p write for Adam)
    if kind == "k_local_step":
        return (gb + 2 * eb) * W + (12 if wl.optimizer == "lamb" else 16)
    if kind == "k_sign_count":           # the packed signs of every worker (monitoring)
        return W / 8
    if kind == "k_grad_mean":            # g of every worker in, one float out
        return gb * W + 4.0
    return 0.0                           # finalisers: a few bytes per chunk


CACHE_MIN_W = 4     # the library's fused step stores c_srv from this many workers on


def step_bytes_per_elem(wl, phase: str = "compressed", rule: str = "scaled") -> float:
    """The step's algorithmic bytes per element, from the kernels it launches
    (bench.py also sums them from the kernels the timed steps actually ran)."""
    if phase == "refresh":
        return algo_bytes_per_elem("k_warmup", wl) + (16.0 if wl.optimizer == "lamb" else 0.0)
    if phase == "local":
        return algo_bytes_per_elem("k_local_step", wl) + (16.0 if wl.optimizer == "lamb" else 0.0)
    if rule == "momentum":
        return algo_bytes_per_elem("k_ternary_step", wl) + (16.0 if wl.optimizer == "lamb" else 0.0)
    cached = "_cached" if wl.W >= CACHE_MIN_W else ""
    if rule == "twobit":
        kinds = ["k_tb_worker_norm", "k_tb_pack" + cached, "k_tb_server_update" + cached]
        return sum(algo_bytes_per_elem(k, wl) for k in kinds) + (16.0 if wl.optimizer == "lamb" else 0.0)
    kinds = ["k_worker_norm", "k_worker_pack" + cached, "k_server_update" + cached]
    if wl.optimizer == "lamb":
        kinds.append("k_lamb_param")
    return sum(algo_bytes_per_elem(k, wl) for k in kinds)


def measured_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def kernel_source_sha() -> str:
    h = hashlib.sha256()
    for p in KERNEL_SOURCES:
        with open(p, "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def ncu_traffic(kernel: str, workload: str):
    """DRAM bytes per launch of `kernel` from the committed ncu summary, or None
    when there is none for this kernel/workload or the kernel source changed."""
    if not os.path.exists(TRAFFIC_FILE):
        return None
    sha = kernel_source_sha()
    with open(TRAFFIC_FILE) as f:
        for line in f:
            parts = line.split()
            if len(parts) < 3 or line.startswith("#"):
                continue
            kv = dict(p.split("=", 1) for p in parts[2:] if "=" in p)
            if parts[0] == kernel and parts[1] == workload and kv.get("source_sha") == sha:
                return float(kv["dram_bytes_per_launch"])
    return None


# -- clocks during the timed region ------------------------------------------------------

class ClockSampler:
    FIELDS = ("timestamp,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")
    REASONS = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")

    def __init__(self, gpu_id: str):
        self.gpu_id = gpu_id
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(prefix="clocks_", suffix=".csv")
            self.fh = os.fdopen(fd, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "50", "-i", self.gpu_id], stdout=self.fh, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self, t0: float, t1: float):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "note": "nvidia-smi unavailable"}
        time.sleep(0.1)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.fh.close()
        rows = []
        with open(self.path) as f:
            for line in f:
                p = [x.strip() for x in line.split(",")]
                if len(p) < 8:
                    continue
                try:
                    ts = datetime.datetime.strptime(p[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
                    rows.append((ts, float(p[1]), float(p[2]), float(p[3]) if p[3] not in ("[N/A]", "") else 0.0,
                                 p[4:8]))
                except ValueError:
                    continue
        os.unlink(self.path)
        inside = [r for r in rows if t0 - 0.05 <= r[0] <= t1 + 0.05] or rows
        if not inside:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "note": "no samples"}
        reasons = sorted({name for r in inside for name, val in zip(self.REASONS, r[4])
                          if val.lower() == "active"})
        return {"sm_mhz": statistics.median(r[1] for r in inside),
                "sm_max_mhz": max(r[2] for r in inside),
                "reasons": reasons, "samples": len(inside),
                "power_w_max": max(r[3] for r in inside)}


# -- distributed plumbing ------------------------------------------------------------------

def dp_bytes_per_elem(kind: str, role: str, wl, world: int, rule: str) -> float:
    """HBM bytes per element of a data-parallel stage kernel: role "worker" (a
    ctx over the rank's gradient or a slice of it: the worker stage, or the
    update alone), "server" (the owner's W-worker server stage).  0 for the
    finalisers and the monitoring kernels."""
    gb, eb = wl.grad_bytes, wl.err_bytes
    upd = 16.0 if wl.optimizer == "lamb" else 20.0
    if rule == "scaled" and role == "worker":
        return {"k_worker_norm": gb + eb,                      # g, err
                "k_worker_pack": gb + 2 * eb + 1 / 8,          # g, err r/w, signs
                "k_server_update": 1 / 8 + upd,                # server signs, m r/w, v, p (+ p w)
                "k_lamb_param": 16.0}.get(kind, 0.0)
    if rule == "scaled" and role == "server":
        return {"k_server_norm": world / 8 + eb,               # W workers' signs, srv_err
                "k_server_update": world / 8 + 2 * eb + 1 / 8}.get(kind, 0.0)  # signs, srv_err r/w, server signs
    if rule == "twobit" and role == "worker":
        return {"k_tb_worker_norm": gb + eb,                   # g, err
                "k_tb_pack": gb + 2 * eb + 1 / 4,              # g, err r/w, both planes
                "k_tb_server_update": 1 / 4 + upd,             # server planes, m r/w, v, p (+ p w)
                "k_lamb_param": 16.0}.get(kind, 0.0)
    if rule == "twobit" and role == "server":
        return {"k_tb_server_norm": world / 4 + eb,            # W workers' planes, srv_err
                "k_tb_server_update": world / 4 + 2 * eb + 1 / 4}.get(kind, 0.0)
    if rule == "momentum" and role == "worker":
        return {"k_ternary_compress": gb + 2 * eb + 1,         # g, err r/w, one code byte
                "k_ternary_update": 1 + upd,                   # one sum byte, m r/w, v, p (+ p w)
                "k_lamb_param": 16.0}.get(kind, 0.0)
    if rule == "momentum" and role == "server":
        return {"k_ternary_server": world + 1.0}.get(kind, 0.0)  # W code bytes in, one sum byte out
    return 0.0
    gb, eb = wl.grad_bytes, wl.err_bytes
    upd = 16.0 if wl.optimizer == "lamb" else 20.0
    if role == "worker":
        return {"k_worker_norm": gb + eb,                      # g, err
                "k_worker_pack": gb + 2 * eb + 1 / 8,          # g, err r/w, signs
                "k_server_update": 1 / 8 + upd,                # server signs, m r/w, v, p (+ p w)
                "k_lamb_param": 16.0}.get(kind, 0.0)
    if role == "server":
        return {"k_server_norm": world / 8 + eb,               # W workers' signs, srv_err
                "k_server_update": world / 8 + 2 * eb + 1 / 8}.get(kind, 0.0)  # signs, srv_err r/w, server signs
    return 0.0


def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def init_dist(world, local):
    import torch
    import torch.distributed as dist
    if world > 1 and not dist.is_initialized():
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    return dist if world > 1 else None


def barrier(dist):
    if dist is not None:
        dist.barrier()


def max_over_ranks(dist, x: float, device) -> float:
    if dist is None:
        return x
    import torch
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# -- CPU oracle timing ----------------------------------------------------------------------

def _chunk_inputs(wl, k, nk):
    """Seeded gradients and initial state of chunk k (its first nk elements)."""
    import workloads as WL
    g = np.stack([WL.chunk_grads(wl, 0, w, k, 0, nk) for w in range(wl.W)])
    p, v = WL.chunk_state(wl, k)
    edt = np.uint16 if wl.err_dtype == "bf16" else np.float32
    st = {"p": p[:nk].copy(), "m": np.zeros(nk, np.float32), "v": v[:nk].copy(),
          "err": np.zeros((wl.W, nk), edt), "srv_err": np.zeros(nk, edt)}
    return g, st


def _oracle_step(o, wl, off, g, st, phase, rule, threads=1):
    import oracle
    f = np.float32
    opt = oracle.LAMB if wl.optimizer == "lamb" else oracle.ADAM
    if phase == "refresh":
        o.warmup(off, g, st["m"], st["v"], st["p"], f(wl.beta1), f(wl.beta2), f(wl.lr), f(wl.eps),
                 optimizer=opt)
    elif phase == "local":
        o.local_step(off, g, st, f(wl.lr), f(wl.eps), clip=wl.clip, optimizer=opt)
    elif rule == "momentum":
        o.ternary_step(off, g, st, f(wl.beta1), f(wl.lr), f(wl.eps), clip=wl.clip, optimizer=opt)
    elif rule == "twobit":
        o.twobit_step(off, g, st, f(wl.beta1), f(wl.lr), f(wl.eps), clip=wl.clip, optimizer=opt)
    else:
        o.step(off, g, st, f(wl.beta1), f(wl.lr), f(wl.eps), clip=wl.clip, optimizer=opt, threads=threads)


def oracle_rate(wl, chunks, max_elems=None, min_seconds=0.0, steps=1, phase="compressed", rule="scaled"):
    """Time the single-threaded oracle's compressed step (or full-precision
    refresh step) on whole chunks (or on the first max_elems elements of a
    chunk, taken as one chunk), until min_seconds have passed."""
    import oracle
    o = oracle.get()
    elems = 0
    secs = 0.0
    per_step = []
    used = []
    for k in chunks:
        nk = wl.sizes[k] if max_elems is None else min(max_elems, wl.sizes[k])
        g, st = _chunk_inputs(wl, k, nk)
        for _ in range(steps):
            t = time.perf_counter()
            _oracle_step(o, wl, [0, nk], g, st, phase, rule)
            dt = time.perf_counter() - t
            per_step.append(dt)
            secs += dt
            elems += nk
        used.append((k, nk))
        if secs >= min_seconds:
            break
    return elems, secs, per_step, used


def oracle_rate_all_cores(wl, used, threads, steps=1, phase="compressed", rule="scaled"):
    """Time the oracle on `threads` host threads over the same chunk sample.

    The scaled rule's compressed step runs the multi-threaded oracle step
    (element ranges of every chunk on all threads, each reduction one ascending
    loop: bit-identical to the single-thread oracle) on the sampled chunks as
    one problem.  Other rules and the refresh step run the single-thread oracle
    on the chunks concurrently, one chunk per thread (the oracle releases the
    interpreter lock inside its C calls).  Returns (elements, seconds per step
    list, how)."""
    import oracle
    from concurrent.futures import ThreadPoolExecutor
    inputs = [_chunk_inputs(wl, k, nk) for k, nk in used]
    elems = sum(nk for _, nk in used)
    per_step = []
    if phase == "compressed" and rule == "scaled":
        o = oracle.get_mt()
        off = np.zeros(len(used) + 1, np.int64)
        np.cumsum([nk for _, nk in used], out=off[1:])
        g = np.concatenate([gi for gi, _ in inputs], axis=1)
        st = {key: np.concatenate([si[key] for _, si in inputs], axis=-1) for key in inputs[0][1]}
        del inputs
        for _ in range(steps):
            t = time.perf_counter()
            _oracle_step(o, wl, off, g, st, phase, rule, threads=threads)
            per_step.append(time.perf_counter() - t)
        return elems, per_step, f"multi-threaded oracle step, {threads} threads over element ranges"
    o = oracle.get()
    workers = max(1, min(threads, len(used)))
    with ThreadPoolExecutor(workers) as ex:
        for _ in range(steps):
            t = time.perf_counter()
            list(ex.map(lambda gs: _oracle_step(o, wl, [0, gs[0].shape[1]], gs[0], gs[1], phase, rule),
                        inputs))
            per_step.append(time.perf_counter() - t)
    return elems, per_step, f"single-thread oracle on {workers} chunk(s) at once, one thread each"


def run_reference(args):
    """The reference arm: the CPU oracle on all host cores, one step per bench
    step on a bounded sample of the workload (chunk 0, whole, taken as one
    chunk), rank 0 only."""
    world, rank, local = dist_env()
    if rank != 0:
        return 0
    import oracle
    wl = select_workload(args)
    cores = oracle.host_threads()
    nk = wl.sizes[0]
    elems, per_step, how = oracle_rate_all_cores(wl, [(0, nk)], cores, steps=args.warmup + args.steps,
                                                 rule=args.rule)
    timed = per_step[args.warmup:]
    ms = 1e3 * sum(timed) / len(timed)
    value = elems / (ms / 1e3) / 1e9
    sample_txt = (f"chunk 0 of {wl.name} ({nk} elements, whole), W={wl.W}, one compressed step per bench "
                  f"step ({args.rule} rule); {how}")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": workload_config(wl, args.gpus, args.rule),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                             "sample": sample_txt, "nproc": os.cpu_count()},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def select_workload(args):
    import workloads as WL
    wl = WL.get_workload(args.workload)
    if getattr(args, "err_dtype", None):
        wl = wl.with_(err_dtype=args.err_dtype)
    if args.chunks:
        k = min(args.chunks, wl.C)
        wl = wl.with_(sizes=wl.sizes[:k], name=f"{wl.name}-first{k}",
                      description=f"first {k} chunk(s) of {wl.name} ({wl.description})")
    return wl


L2_BYTES = 126 * 1000 * 1000           # B200 L2 cache


def flushes_l2(wl, rule="scaled") -> bool:
    """Steps whose traffic is not well above L2 are timed one at a time with an
    L2 flush (an untimed 2 x L2 write) between them."""
    return step_bytes_per_elem(wl, "compressed", rule) * wl.n < 4 * L2_BYTES


def workload_config(wl, n_gpus, rule="scaled"):
    return {"workload": f"{wl.name}: {wl.description}", "n": wl.n, "chunks": wl.C, "W": wl.W,
            "grad_dtype": wl.grad_dtype, "state_dtype": "f32", "err_dtype": wl.err_dtype,
            "optimizer": wl.optimizer, "rule": rule,
            "global_batch": wl.W * n_gpus, "parallelism": f"{n_gpus} replica(s) x {wl.W} virtual workers",
            "l2": (f"L2 flushed between timed steps ({2 * L2_BYTES // 1000000} MB write, untimed; "
                   f"{step_bytes_per_elem(wl, 'compressed', rule) * wl.n / 1e9:.2f} GB of traffic per step)")
                  if flushes_l2(wl, rule) else
                  f"inputs larger than L2: {step_bytes_per_elem(wl, 'compressed', rule) * wl.n / 1e9:.1f} "
                  "GB of traffic per step"}


# -- our arm -------------------------------------------------------------------------------

def run_ours(args):
    import torch
    world, rank, local = dist_env()
    if world != args.gpus:
        print(f"warning: --gpus {args.gpus} but WORLD_SIZE={world}", file=sys.stderr)
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    dist = init_dist(world, local)

    import workloads as WL
    from bit_adam_error_b200 import OneBitAdam, _lib as L

    wl = select_workload(args)
    n, W = wl.n, wl.W
    gdt = torch.bfloat16 if wl.grad_dtype == "bf16" else torch.float32

    # State: seeded p, v generated a chunk group at a time and uploaded once.
    opt = OneBitAdam(wl.offsets, W, grad_dtype=wl.grad_dtype, optimizer=wl.optimizer, clip=wl.clip,
                     freeze_step=0, lr=wl.lr, beta1=wl.beta1, beta2=wl.beta2, eps=wl.eps,
                     err_dtype=wl.err_dtype, rule=args.rule, device=device)
    swl = wl.with_(freeze_step=0)
    for k0, k1 in WL.chunk_groups(wl):
        lo, hi = int(wl.offsets[k0]), int(wl.offsets[k1])
        p_h = np.empty(hi - lo, np.float32)
        v_h = np.empty(hi - lo, np.float32)
        WL.fill_state(swl, p_h, v_h, chunks=(k0, k1))
        opt.p[lo:hi].copy_(torch.from_numpy(p_h))
        opt.v[lo:hi].copy_(torch.from_numpy(v_h))
    del p_h, v_h

    # Gradient batches in HBM (distinct seeded steps), generated a chunk group at a time.
    nbuf = max(1, args.grad_buffers)
    dev_g = []
    for b in range(nbuf):
        G = torch.empty((W, n), dtype=gdt, device=device)
        fill_device_grads(wl, b + 1000 * rank, G)
        dev_g.append(G)
    stream = torch.cuda.current_stream(device)

    step_fn = {"refresh": opt.refresh_step, "local": opt.local_step}.get(args.phase, opt.step)
    for i in range(args.warmup):
        step_fn(dev_g[i % nbuf])
    torch.cuda.synchronize()

    # -- timed region: inputs resident in HBM ------------------------------------
    # Large workloads: per-kernel CUDA events ride along in the timed steps (a few
    # microseconds against milliseconds).  Small workloads (L2 flushed between
    # steps): events between the launches would stop each kernel's launch from
    # overlapping the previous kernel's tail, so the steps are timed without them
    # and a second pass of the same steps, with the per-kernel events, gives the
    # kernel breakdown.
    per_step_launches = 16
    flush = flushes_l2(wl, args.rule)
    if not flush:
        L.ob_profile_start(opt.ctx, args.steps * per_step_launches)
    launches0 = L.ob_launch_count(opt.ctx)
    sampler = ClockSampler(gpu_id(device))
    sampler.start()
    time.sleep(0.3)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    flush_buf = torch.empty(2 * L2_BYTES, dtype=torch.uint8, device=device) if flush else None
    step_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(args.steps)] if flush else []
    barrier(dist)
    torch.cuda.synchronize()
    w0 = time.time()
    e0.record(stream)
    for i in range(args.steps):
        if flush:                          # small workload: evict it from L2, outside the step's events
            flush_buf.zero_()
            step_ev[i][0].record(stream)
        step_fn(dev_g[i % nbuf])
        if flush:
            step_ev[i][1].record(stream)
    e1.record(stream)
    torch.cuda.synchronize()
    w1 = time.time()
    barrier(dist)
    clocks = sampler.stop(w0, w1)
    launches = L.ob_launch_count(opt.ctx) - launches0
    ms = (sum(a.elapsed_time(b) for a, b in step_ev) if flush else e0.elapsed_time(e1)) / args.steps
    ms_max = max_over_ranks(dist, ms, device)
    if flush:                              # the kernel breakdown: the same steps, with per-kernel events
        L.ob_profile_start(opt.ctx, args.steps * per_step_launches)
        for i in range(args.steps):
            flush_buf.zero_()
            step_fn(dev_g[i % nbuf])
        torch.cuda.synchronize()
    prof = L.ob_profile_stop(opt.ctx)
    status = opt.status()

    # Dominant kernel roofline (this rank's CUDA events on the launch stream).
    peak, peak_src = measured_peak()
    # Dominant kernel: the one with the most time among those that stream the
    # step's bytes (on a launch-bound workload a finaliser can take longer).
    dom = max((k for k in prof if algo_bytes_per_elem(k, wl) > 0), key=lambda k: prof[k][0])
    dom_ms = prof[dom][0] / prof[dom][1]
    dom_bytes = algo_bytes_per_elem(dom, wl) * n
    achieved = dom_bytes / (dom_ms / 1e3) / 1e9
    traffic = ncu_traffic(dom, wl.name)
    total_ms = sum(v[0] for v in prof.values())
    roofline = {"bound": "hbm", "kernel": dom, "achieved": achieved, "peak": peak,
                "peak_source": f"{peak_src} (copy bandwidth)", "unit": "GB/s",
                "frac": achieved / peak, "traffic": traffic,
                "algorithmic_bytes_per_launch": dom_bytes, "launch_ms": dom_ms,
                "share_of_kernel_time": prof[dom][0] / total_ms}
    kernels = {k: {"ms_per_launch": v[0] / v[1], "launches": v[1], "share": v[0] / total_ms,
                   "algorithmic_GBps": (algo_bytes_per_elem(k, wl) * n / (v[0] / v[1] / 1e3) / 1e9)
                   if algo_bytes_per_elem(k, wl) else None}
               for k, v in prof.items()}
    # Step bytes from the kernels the timed steps ran (the library picks the schedule).
    step_bpe = sum(algo_bytes_per_elem(k, wl) * v[1] for k, v in prof.items()) / args.steps
    step_gbs = step_bpe * n / (ms_max / 1e3) / 1e9

    # -- small workloads: the same steps back to back, inputs left in L2 -------------
    l2_resident = None
    if flush:
        for i in range(3):
            step_fn(dev_g[i % nbuf])
        torch.cuda.synchronize()
        e0.record(stream)
        for i in range(args.steps):
            step_fn(dev_g[i % nbuf])
        e1.record(stream)
        torch.cuda.synchronize()
        ms_res = max_over_ranks(dist, e0.elapsed_time(e1) / args.steps, device)
        l2_resident = {"ms_per_step": ms_res, "value": world * n / (ms_res / 1e3) / 1e9, "unit": UNIT,
                       "note": "no L2 flush between steps: the step's inputs stay in the 126 MB L2"}

    # -- error-buffer monitoring (one call, timed alone) -----------------------------
    monitor = None
    if args.phase == "compressed":
        opt.error_norms()                  # first call: host-side set-up outside the timing
        torch.cuda.synchronize()
        e0.record(stream)
        opt.error_norms()
        e1.record(stream)
        torch.cuda.synchronize()
        mon_ms = e0.elapsed_time(e1)
        mon_bytes = wl.err_bytes * n * (W + (1 if opt.srv_err is not None else 0))
        monitor = {"ms": mon_ms, "GBps": mon_bytes / (mon_ms / 1e3) / 1e9,
                   "frac": mon_bytes / (mon_ms / 1e3) / 1e9 / peak, "bytes": mon_bytes}

    # -- quantisation-rate monitoring (one call, timed alone; sign-bit rules) ----------
    rates = None
    if args.phase == "compressed" and args.rule != "momentum":
        opt.quant_rates()
        torch.cuda.synchronize()
        e0.record(stream)
        opt.quant_rates()
        e1.record(stream)
        torch.cuda.synchronize()
        r_ms = e0.elapsed_time(e1)
        r_bytes = 4 * opt.words * (W + 1)          # every worker's packed words and the server's
        rates = {"ms": r_ms, "GBps": r_bytes / (r_ms / 1e3) / 1e9, "bytes": r_bytes}

    # -- end to end: host gradients through the public call ---------------------------
    e2e = None
    host_bytes = W * n * wl.grad_bytes
    if not args.no_e2e and args.phase != "compressed":
        e2e = {"value": None, "unit": UNIT, "note": "host gradients are taken by the compressed step only"}
    elif not args.no_e2e and host_bytes > E2E_MAX_HOST_BYTES:
        e2e = {"value": None, "unit": UNIT, "note": f"skipped: {host_bytes / 1e9:.1f} GB of pinned host "
               f"gradients per step exceeds the {E2E_MAX_HOST_BYTES / 1e9:.0f} GB cap"}
    elif not args.no_e2e:
        # Pinned host copies of the gradient batches, filled from the same seeded streams.
        host_g = []
        for b in range(min(nbuf, 2)):
            h = torch.empty((W, n), dtype=gdt, pin_memory=True)
            arr = h.view(torch.int16).numpy().view(np.uint16) if wl.grad_dtype == "bf16" else h.numpy()
            WL.fill_grads(wl, b + 1000 * rank, arr)
            host_g.append(h)
        nh = len(host_g)
        # The step's result read back each step: the server scales, or (the
        # momentum-error rule has none) the first C parameters.
        result = opt.s_srv if opt.s_srv is not None else opt.p[: wl.C]
        s_host = torch.empty(result.shape, dtype=torch.float32, pin_memory=True)
        for i in range(2):
            opt.step(host_g[i % nh])
        torch.cuda.synchronize()
        barrier(dist)
        torch.cuda.synchronize()
        e0.record(stream)
        for i in range(args.steps):
            opt.step(host_g[i % nh])
            s_host.copy_(result, non_blocking=True)
        e1.record(stream)
        torch.cuda.synchronize()
        barrier(dist)
        ms_e2e = max_over_ranks(dist, e0.elapsed_time(e1) / args.steps, device)
        e2e = {"value": world * n / (ms_e2e / 1e3) / 1e9, "unit": UNIT, "ms_per_step": ms_e2e,
               "h2d_bytes_per_step": host_bytes, "d2h_bytes_per_step": 4 * s_host.numel()}
        del host_g

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(wl, args)

    if rank == 0:
        line = {"metric": METRIC, "value": world * n / (ms_max / 1e3) / 1e9, "unit": UNIT,
                "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_max,
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
                "data": "synthetic (seeded Philox streams; shapes and distributions of the workload)",
                "config": workload_config(wl, world, args.rule),
                "phase": args.phase,
                "hbm": {"step_achieved_GBps": step_gbs, "step_frac": step_gbs / peak,
                        "algorithmic_bytes_per_elem": step_bpe, "peak": peak,
                        "peak_source": peak_src},
                "roofline": roofline, "kernels": kernels,
                "kernel_timing": ("a second pass of the same steps with per-kernel CUDA events"
                                  if flush else "per-kernel CUDA events in the timed steps"),
                "error_norms_call": monitor, "quant_rates_call": rates,
                "l2_resident": l2_resident,
                "cpu_baseline": cpu, "e2e": e2e,
                "gpu_launches": launches, "status_flags": status, "clocks": clocks}
        print(json.dumps(line), flush=True)
    opt.close()
    if dist is not None:
        dist.destroy_process_group()
    return 0


def cpu_baseline(wl, args):
    """The CPU oracle on the machine's host: one thread, then all host cores, on the
    same sample of whole chunks (as many as about 10 s of single-thread work
    takes).  The record's value is the all-cores figure; both legs are listed."""
    import oracle
    elems, secs, _, used = oracle_rate(wl, list(range(wl.C)), min_seconds=10.0, phase=args.phase,
                                       rule=args.rule)
    one = elems / secs / 1e9
    cores = oracle.host_threads()
    e_all, per_step, how = oracle_rate_all_cores(wl, used, cores, phase=args.phase, rule=args.rule)
    t_all = sum(per_step)
    allv = e_all / t_all / 1e9
    sample = (f"{len(used)} whole chunk(s) {[k for k, _ in used]} of {wl.name} ({elems} elements), "
              f"one {args.phase} step ({args.rule} rule)")
    return {"value": allv, "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": f"{sample}; {how}, {t_all:.2f} s",
            "nproc": os.cpu_count(),
            "legs": [{"cores": 1, "value": one, "seconds": secs, "how": "single-thread oracle, chunk by chunk"},
                     {"cores": cores, "value": allv, "seconds": t_all, "how": how}]}


def fill_device_grads(wl, step, G) -> None:
    """Seeded gradients of one step into the device tensor G [W, n], a worker row
    and a chunk group at a time."""
    import torch
    import workloads as WL
    bf = wl.grad_dtype == "bf16"
    for w in range(wl.W):
        for k0, k1 in WL.chunk_groups(wl):
            lo, hi = int(wl.offsets[k0]), int(wl.offsets[k1])
            row = np.empty(hi - lo, np.uint16 if bf else np.float32)
            WL.fill_grads_row(wl, step, w, row, chunks=(k0, k1))
            src = torch.from_numpy(row.view(np.int16)).view(torch.bfloat16) if bf else torch.from_numpy(row)
            G[w, lo:hi].copy_(src)


def run_dp(args):
    """Data-parallel 1-bit Adam over the ranks: each rank is one worker (W = N)
    holding the whole model and its own gradient; it compresses its gradient,
    serves the chunks it owns (server stage between the two point-to-point
    exchanges) and applies the update to its replica.  Per-rank work is one
    gradient of n elements whatever N is, so scaling is weak and ``value`` is
    the gradient elements of all ranks per second (N n / max-over-ranks step
    time); ``model_value`` is n / step time."""
    import torch
    world, rank, local = dist_env()
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    import torch.distributed as tdist
    if not tdist.is_initialized():
        os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
        os.environ.setdefault("MASTER_PORT", "29517")
        os.environ.setdefault("RANK", str(rank))
        os.environ.setdefault("WORLD_SIZE", str(world))
        tdist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=device)
    import workloads as WL
    from bit_adam_error_b200 import _lib as L
    from bit_adam_error_b200.distributed import CudaStages, DistributedOneBitAdam, plan
    wl = select_workload(args).with_(W=world, freeze_step=0)
    layout = plan(wl.sizes, world, 4 if args.rule == "momentum" else 32, 2 if args.rule == "twobit" else 1)
    stages = CudaStages(layout, rank, grad_dtype=wl.grad_dtype, optimizer=wl.optimizer, clip=wl.clip,
                        lr=wl.lr, beta1=wl.beta1, beta2=wl.beta2, eps=wl.eps, warmup=False,
                        rule=args.rule, device=device)
    bf = wl.grad_dtype == "bf16"
    gdt = torch.bfloat16 if bf else torch.float32
    nbuf = max(1, args.grad_buffers)
    G = [torch.empty(layout.n, dtype=gdt, device=device) for _ in range(nbuf)]
    for pos, k in enumerate(layout.order):            # layout order: chunks grouped by owner
        lo, hi = int(layout.offsets[pos]), int(layout.offsets[pos + 1])
        p_h = np.empty(hi - lo, np.float32)
        v_h = np.empty(hi - lo, np.float32)
        WL.fill_state(wl, p_h, v_h, chunks=(k, k + 1))
        stages.p[lo:hi].copy_(torch.from_numpy(p_h))
        stages.v[lo:hi].copy_(torch.from_numpy(v_h))
        for b in range(nbuf):
            row = np.empty(hi - lo, np.uint16 if bf else np.float32)
            WL.fill_grads_row(wl, b, rank, row, chunks=(k, k + 1))
            src = torch.from_numpy(row.view(np.int16)).view(torch.bfloat16) if bf else torch.from_numpy(row)
            G[b][lo:hi].copy_(src)
    drv = DistributedOneBitAdam(layout, stages, freeze_step=0)
    ctxs = [h for h in {stages.local, stages.server, stages.update, *(stages.slice_ctx or []),
                        *(stages.slice_upd or [])} if h]
    # Elements and role of every ctx, for the byte model of its kernels.
    ctx_info = {stages.local: (layout.n, "worker")}
    if stages.server:
        ctx_info[stages.server] = (stages.n_own, "server")
    if stages.update:
        ctx_info[stages.update] = (layout.n, "worker")
    for o, h in enumerate(stages.slice_ctx or []):
        if h:
            es = layout.eslice(o)
            ctx_info[h] = (es.stop - es.start, "worker")
    for o, h in enumerate(stages.slice_upd or []):
        if h and h not in ctx_info:
            es = layout.eslice(o)
            ctx_info[h] = (es.stop - es.start, "worker")
    stream = torch.cuda.current_stream(device)
    for i in range(args.warmup):
        drv.step(G[i % nbuf])
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    launches0 = sum(L.ob_launch_count(h) for h in ctxs)
    for h in ctxs:
        L.ob_profile_start(h, args.steps * 16)
    sampler = ClockSampler(gpu_id(device))
    sampler.start()
    time.sleep(0.3)
    barrier(tdist)
    torch.cuda.synchronize()
    w0 = time.time()
    e0.record(stream)
    for i in range(args.steps):
        drv.step(G[i % nbuf])
    e1.record(stream)
    torch.cuda.synchronize()
    w1 = time.time()
    barrier(tdist)
    clocks = sampler.stop(w0, w1)
    launches = sum(L.ob_launch_count(h) for h in ctxs) - launches0
    ms = max_over_ranks(tdist, e0.elapsed_time(e1) / args.steps, device)
    # Per kernel and ctx role: time (CUDA events on the launch stream) and bytes.
    agg = {}
    for h in ctxs:
        n_ctx, role = ctx_info.get(h, (0, "worker"))
        for kname, (kms, kl) in L.ob_profile_stop(h).items():
            key = f"{kname} ({role})"
            t, c, b = agg.get(key, (0.0, 0, 0.0))
            agg[key] = (t + kms, c + kl, b + kl * n_ctx * dp_bytes_per_elem(kname, role, wl, world, args.rule))
    peak, peak_src = measured_peak()
    streamed = {k: v for k, v in agg.items() if v[2] > 0}
    roofline, dp_kernels = None, None
    if streamed:
        total_ms = sum(v[0] for v in agg.values())
        dom = max(streamed, key=lambda k: streamed[k][0])
        t, c, b = streamed[dom]
        achieved = b / (t / 1e3) / 1e9
        roofline = {"bound": "hbm", "kernel": dom, "achieved": achieved, "peak": peak,
                    "peak_source": f"{peak_src} (copy bandwidth)", "unit": "GB/s", "frac": achieved / peak,
                    "traffic": None, "algorithmic_bytes_per_launch": b / c, "launch_ms": t / c,
                    "share_of_kernel_time": t / total_ms, "rank": rank}
        dp_kernels = {k: {"ms_per_launch": v[0] / v[1], "launches": v[1], "share": v[0] / total_ms,
                          "algorithmic_GBps": (v[2] / (v[0] / 1e3) / 1e9) if v[2] else None}
                      for k, v in agg.items()}

    # End to end: this rank's gradient from pinned host memory every step (one
    # host-to-device copy), the step, and a device-to-host read of the scales.
    e2e = None
    if not args.no_e2e:
        host = [torch.empty(layout.n, dtype=gdt, pin_memory=True) for _ in range(min(2, nbuf))]
        for b, hb in enumerate(host):
            hb.copy_(G[b])
        dev_in = torch.empty(layout.n, dtype=gdt, device=device)
        result = stages.s_srv if stages.s_srv.numel() else stages.p[: max(1, layout.C)]
        out_h = torch.empty(result.shape, dtype=torch.float32, pin_memory=True)
        for i in range(2):
            dev_in.copy_(host[i % len(host)], non_blocking=True)
            drv.step(dev_in)
        torch.cuda.synchronize()
        barrier(tdist)
        torch.cuda.synchronize()
        e0.record(stream)
        for i in range(args.steps):
            dev_in.copy_(host[i % len(host)], non_blocking=True)
            drv.step(dev_in)
            out_h.copy_(result, non_blocking=True)
        e1.record(stream)
        torch.cuda.synchronize()
        barrier(tdist)
        ms_e2e = max_over_ranks(tdist, e0.elapsed_time(e1) / args.steps, device)
        e2e = {"value": world * layout.n / (ms_e2e / 1e3) / 1e9, "unit": UNIT, "ms_per_step": ms_e2e,
               "h2d_bytes_per_step": layout.n * wl.grad_bytes, "d2h_bytes_per_step": 4 * out_h.numel()}
    flags = drv.status()
    if rank == 0:
        own = [layout.eslice(r).stop - layout.eslice(r).start for r in range(world)]
        scales_per_chunk = {"scaled": 1, "momentum": 0, "twobit": 2}[args.rule]
        line = {"metric": METRIC, "value": world * layout.n / (ms / 1e3) / 1e9, "unit": UNIT,
                "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
                "data": "synthetic (seeded Philox streams; shapes and distributions of the workload)",
                "config": dict(workload_config(wl, world, args.rule),
                               parallelism=f"dp{world}: worker w = rank w (whole model and one gradient per "
                                           f"rank), chunk-owner server stage, NCCL point-to-point exchanges "
                                           f"({'pipelined' if stages.pipelined else 'grouped'})",
                               owned_elements=own, units="gradient elements of all ranks per second"),
                "model_value": layout.n / (ms / 1e3) / 1e9,
                "exchange_bytes_per_step_per_rank": 2 * 4 * (int(layout.words[-1]) + scales_per_chunk * layout.C),
                "roofline": roofline, "kernels": dp_kernels,
                "kernel_timing": "per-kernel CUDA events of every ctx in the timed steps",
                "gpu_launches": launches, "status_flags": flags, "e2e": e2e, "clocks": clocks}
        print(json.dumps(line), flush=True)
    stages.close()
    tdist.destroy_process_group()
    return 0


def gpu_id(device) -> str:
    import torch
    try:
        return "GPU-" + str(torch.cuda.get_device_properties(device).uuid)
    except Exception:
        return str(device.index)


def main():
    args = parse_args()
    if args.impl == "reference":
        return run_reference(args)
    world = dist_env()[0]
    if args.dp or (world > 1 and not args.replicas):
        return run_dp(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
