"""Benchmark of one token-sparse decode step (and the dense reference path).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                    [--impl ours|reference] [--no-sweep] [--cpu-seconds S]

A step is the whole hot path for one decode token of every sequence in the
batch: append the new token's label row, score every cached token on the
label channels and keep the top k, then exact attention over the kept rows --
one ds_decode_step call (one launch where the sizes allow; the same step as
separate calls is timed beside it for per-kernel stage times).  Inputs are seeded and synthetic (``dsgen``) and resident
in HBM; the step is one CUDA graph; L2 is flushed (256 MiB written, then read) between
steps and each step is timed with CUDA events, so every step reads its bytes
from HBM.

Printed value: achieved algorithmic HBM bandwidth of the step, GB/s, summed
over ranks (label bytes + k*2*d*2 bytes of selected K/V + Q and O per query
head, divided by the device time of a step).  ``us_per_step`` and
``tokens_heads_per_s`` are reported beside it, with the dense path and the
CPU oracle.  Multi-GPU runs are independent replicas (one process per GPU,
each with its own seeded batch): the decode step has no cross-GPU exchange.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import dsgen  # noqa: E402

HEADLINE = "llama2-7b-B8-H32-T4K"
METRIC = "sparse decode µs/step & HBM GB/s (% of 8 TB/s) vs dense, T=1K–256K"
FLUSH_BYTES = 256 << 20
# the B200's nominal HBM3e bandwidth (DGX figure), beside the measured copy peak
NOMINAL_HBM_GBS = 8000.0
PROFILE_TRAFFIC = os.path.join(ROOT, "profiles", "traffic_llama2-7b-B8-H32-T4K.txt")
CSRC = os.path.join(ROOT, "post_token_sparse_b200", "csrc")


def flush_l2(buf):
    """Evict L2 between timed steps: write a buffer larger than L2, then read it
    back, so that L2 holds clean lines (a write alone leaves about 126 MB of dirty
    lines whose write-back would be charged to the next timed kernel)."""
    import torch

    buf.zero_()
    torch.sum(buf.view(torch.int64), dtype=torch.int64)


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=1000)
    p.add_argument("--warmup", type=int, default=20)
    p.add_argument("--workload", default=HEADLINE, choices=list(dsgen.CONFIGS))
    p.add_argument("--impl", default="ours", choices=["ours", "reference"])
    p.add_argument("--no-sweep", action="store_true")
    p.add_argument("--unfused", action="store_true",
                   help="separate score and top-k launches instead of the fused one")
    p.add_argument("--mode", default="step", choices=["step", "calls"],
                   help="step: ds_decode_step; calls: label append, score+top-k and "
                        "sparse attention as separate calls")
    p.add_argument("--cpu-seconds", type=float, default=10.0)
    p.add_argument("--batch", type=int, default=None,
                   help="override the workload's batch size (smaller captures for ncu)")
    p.add_argument("--summarize-ncu", metavar="DIR", default=None,
                   help="no GPU: write the profiles/ summaries from DIR/launches.csv and "
                        "DIR/k_step_headline.ncu-rep (the ncu runs of the small command)")
    return p.parse_args()


def rank_env():
    return (int(os.environ.get("RANK", 0)), int(os.environ.get("LOCAL_RANK", 0)),
            int(os.environ.get("WORLD_SIZE", 1)))


# ---------------------------------------------------------------------------
# replicas: one process per GPU, each with its own seeded batch, no exchange

def replica_workload(base: dsgen.Workload, rank: int) -> dsgen.Workload:
    """The workload of one rank: the same shapes, its own seed."""
    return base.with_(seed=base.seed + rank)


def max_over_ranks(x: float, world: int, device) -> float:
    """The largest of every rank's x (a device time): the job ends with its slowest rank."""
    import torch

    t = torch.tensor([x], dtype=torch.float64, device=device)
    if world > 1:
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return t.item()


def job_gbs(bytes_per_rank_step: int, world: int, ms_per_step: float) -> float:
    """Whole-job algorithmic bandwidth: every rank's bytes over the slowest rank's time."""
    return world * bytes_per_rank_step / (ms_per_step * 1e-3) / 1e9


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as fh:
            j = json.load(fh)
        return float(j["hbm_gbs"]), "measured"
    except Exception:  # noqa: BLE001
        return 6650.0, "fallback"


def kernel_source_hash() -> str:
    h = hashlib.sha256()
    for n in sorted(os.listdir(CSRC)):
        if n.endswith((".cu", ".cuh")):
            h.update(open(os.path.join(CSRC, n), "rb").read())
    return h.hexdigest()[:16]


def profiled_traffic(kernel: str):
    """DRAM bytes per launch from the committed ncu summary, if it is current."""
    try:
        lines = open(PROFILE_TRAFFIC).read().splitlines()
    except OSError:
        return None
    kv = dict(line.split(":", 1) for line in lines if ":" in line and not line.startswith("#"))
    kv = {k.strip(): v.strip() for k, v in kv.items()}
    if kv.get("kernel_source_hash") != kernel_source_hash():
        return None
    v = kv.get(f"dram_bytes_per_launch[{kernel}]")
    return float(v) if v else None


# ---------------------------------------------------------------------------
# clocks during the timed region (NVML, read only)

class ClockSampler:
    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x100: "display_clock_setting"}

    def __init__(self, cuda_index: int, period_s: float = 0.01):
        self.samples, self.reasons = [], 0
        self.max_mhz = None
        self._stop = threading.Event()
        self._period = period_s
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            self._nv = pynvml
            # NVML numbers every GPU of the machine; match the CUDA device by UUID
            try:
                uuid = "GPU-" + str(torch.cuda.get_device_properties(cuda_index).uuid)
                self._h = pynvml.nvmlDeviceGetHandleByUUID(uuid.encode())
            except Exception:  # noqa: BLE001
                self._h = pynvml.nvmlDeviceGetHandleByIndex(cuda_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception:  # noqa: BLE001
            self._nv = None

    def _run(self):
        nv = self._nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
                self.reasons |= nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
            except Exception:  # noqa: BLE001
                pass
            time.sleep(self._period)

    def __enter__(self):
        if self._nv:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self._nv:
            self._t.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unavailable"]}
        names = [n for b, n in self.REASONS.items() if self.reasons & b and b != 0x1]
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": names, "samples": len(self.samples)}


# ---------------------------------------------------------------------------
# the device side

class Step:
    """One decode step of workload ``w`` on the current GPU, captured as a CUDA graph.

    mode "step": ds_decode_step (label row of the new token, selection and
    attention; one launch when the sizes allow).  mode "calls": the same step as
    separate calls, one stage each: [0] label row of the new token, [1] score +
    top-k (fused, or score then top-k with fused=False), [2] sparse attention.
    dense=True: ds_decode over every token.
    """

    STAGES = ("label_append", "score_topk", "sparse_decode")

    def __init__(self, w: dsgen.Workload, fused: bool = True, dense: bool = False,
                 inputs=None, mode: str = "calls"):
        import torch

        import post_token_sparse_b200 as ds

        self.ds, self.torch, self.w, self.fused, self.dense = ds, torch, w, fused, dense
        self.mode = "dense" if dense else mode
        self.Q, self.K, self.V = inputs if inputs is not None else device_inputs(w)
        self.C = torch.from_numpy(dsgen.channels(w)).cuda()
        BH = w.B * w.Hq
        self.O = torch.empty((w.B, w.Hq, w.d), dtype=torch.float32, device="cuda")
        self.lse = torch.empty((w.B, w.Hq), dtype=torch.float32, device="cuda")
        if not dense:
            self.label = torch.empty((w.B, w.Hq, w.T, w.r), dtype=torch.bfloat16, device="cuda")
            ds.label_append(self.K, self.C, self.label, 0, w.T)  # prompt (setup)
            self.idx = torch.empty((BH, w.k), dtype=torch.int32, device="cuda")
            self.scores = None if fused else torch.empty((BH, w.T), dtype=torch.float32,
                                                         device="cuda")
            dims = ds.dims_of(self.Q, self.K, w.r)
            op = ds.OP_DECODE_STEP if self.mode == "step" else ds.OP_SPARSE_DECODE
            self.ws = ds.workspace(op, dims, w.T, w.k, "cuda")
        else:
            dims = ds.dims_of(self.Q, self.K, w.r)
            self.ws = ds.workspace(ds.OP_DECODE, dims, w.T, w.T, "cuda")
        self.flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device="cuda")
        torch.cuda.synchronize()
        self._capture()

    # the calls of one step, stage by stage
    def stages(self):
        ds, w = self.ds, self.w
        if self.dense:
            return [lambda: ds.decode(self.Q, self.K, self.V, self.O, w.T, w.scale, lse=self.lse,
                                      ws=self.ws)]
        if self.mode == "step":
            return [lambda: ds.decode_step(self.Q, self.K, self.V, self.C, self.label, self.idx,
                                           self.O, w.T, w.scale, append=True, lse=self.lse,
                                           ws=self.ws)]
        s0 = lambda: ds.label_append(self.K, self.C, self.label, w.T - 1, 1)  # noqa: E731
        if self.fused:
            s1 = lambda: ds.score_topk(self.Q, self.C, self.label, self.idx, w.T)  # noqa: E731
        else:
            def s1():
                ds.score(self.Q, self.C, self.label, self.scores, w.T)
                ds.topk(self.scores, self.idx)
        s2 = lambda: ds.sparse_decode(self.Q, self.K, self.V, self.idx, self.O, w.T,  # noqa
                                      w.scale, lse=self.lse, ws=self.ws)
        return [s0, s1, s2]

    def _capture(self):
        torch, ds = self.torch, self.ds
        st = self.stages()
        for s in st:  # eager once: one-time attribute setup happens outside capture
            s()
        torch.cuda.synchronize()
        self.events = [torch.cuda.Event(enable_timing=True, external=True)
                       for _ in range(len(st) + 1)]
        self.graph = torch.cuda.CUDAGraph()
        n0 = ds.kernel_launches()
        with torch.cuda.graph(self.graph):
            self.events[0].record()
            for i, s in enumerate(st):
                s()
                self.events[i + 1].record()
        self.launches_per_step = ds.kernel_launches() - n0
        torch.cuda.synchronize()

    def replay(self):
        self.graph.replay()

    def timed(self, flush: bool = True):
        """One step after an L2 flush (or without one): (step ms, [stage ms])."""
        if flush:
            flush_l2(self.flush)
        self.graph.replay()
        self.torch.cuda.synchronize()
        ev = self.events
        stage = [ev[i].elapsed_time(ev[i + 1]) for i in range(len(ev) - 1)]
        return ev[0].elapsed_time(ev[-1]), stage

    def release(self):
        self.graph = None
        for n in ("Q", "K", "V", "C", "label", "idx", "scores", "O", "lse", "ws", "flush"):
            if hasattr(self, n):
                setattr(self, n, None)
        self.torch.cuda.empty_cache()


def device_inputs(w: dsgen.Workload):
    """Q, K, V of workload ``w`` on the current GPU (bf16)."""
    import numpy as np
    import torch

    out = []
    for bits in dsgen.qkv(w):
        out.append(torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).cuda())
        del bits
    return tuple(out)


def step_bytes(w: dsgen.Workload) -> int:
    return w.sparse_step_bytes()


def stage_bytes(w: dsgen.Workload):
    """Algorithmic bytes per launch of each stage."""
    BH = w.B * w.Hq
    st = {
        "label_append": w.B * w.Hkv * w.d * 2 + BH * w.r * 2,
        "score_topk": w.label_bytes() + BH * (w.r * 2 + w.k * 4),
        "sparse_decode": w.sparse_decode_bytes(),
    }
    st["decode_step"] = sum(st.values())
    return st


def time_device(step: Step, steps: int, warmup: int):
    for _ in range(warmup):
        step.timed()
    total, per_stage = 0.0, [0.0] * len(step.events[:-1])
    for _ in range(steps):
        ms, st = step.timed()
        total += ms
        per_stage = [a + b for a, b in zip(per_stage, st)]
    return total, per_stage


def time_e2e(step: Step, steps: int, warmup: int):
    """Same step end to end through the public API with host buffers: each step
    is one call of the Python binding's decode_step_kv (which marshals the
    arguments and calls ds_decode_step_kv of the C ABI, whose host-side checks
    then launch the kernels) with the query, the new token's K/V rows and O in
    pinned host memory, followed by a host synchronisation, timed on the host
    clock.  The new rows are stored into the caches at T-1 and O written into
    host memory over the host link inside the step.  L2 is flushed before each
    step, outside the timed region.

    Beside it (``graph``): the same call captured once in a CUDA graph and
    replayed, timed by device events (what a decode loop replaying a graph per
    token sees on the GPU, without host launch and synchronisation costs).
    Returns (host ms total, graph ms total, h2d bytes, d2h bytes)."""
    import torch

    w = step.w
    ds = step.ds
    # the step's own query and newest K/V rows, staged in pinned host memory
    q_h = step.Q.cpu().pin_memory()
    kv_h = [c[:, :, w.T - 1, :].contiguous().cpu().pin_memory() for c in (step.K, step.V)]
    o_h = torch.empty((w.B, w.Hq, w.d), dtype=torch.float32).pin_memory()
    stream = torch.cuda.current_stream()

    def call():
        if step.mode == "step":
            ds.decode_step_kv(q_h, kv_h[0], kv_h[1], step.K, step.V, step.C, step.label,
                              step.idx, o_h, w.T, w.scale, ws=step.ws)
        else:  # the separate calls take device buffers: copy the query in, O out
            ds.kv_append(kv_h[0], kv_h[1], step.K, step.V, w.T - 1)
            step.Q.copy_(q_h, non_blocking=True)
            for s in step.stages():
                s()
            o_h.copy_(step.O, non_blocking=True)

    def host_step():
        flush_l2(step.flush)
        torch.cuda.synchronize()
        t0 = time.perf_counter()
        call()
        stream.synchronize()
        return (time.perf_counter() - t0) * 1e3

    for _ in range(warmup):
        host_step()
    host_ms = sum(host_step() for _ in range(steps))

    e0 = torch.cuda.Event(enable_timing=True, external=True)
    e1 = torch.cuda.Event(enable_timing=True, external=True)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        e0.record()
        call()
        e1.record()

    def graph_step():
        flush_l2(step.flush)
        g.replay()
        torch.cuda.synchronize()
        return e0.elapsed_time(e1)

    for _ in range(warmup):
        graph_step()
    graph_ms = sum(graph_step() for _ in range(steps))
    del g
    h2d = q_h.numel() * 2 + 2 * kv_h[0].numel() * 2
    return host_ms, graph_ms, h2d, o_h.numel() * 4


# ---------------------------------------------------------------------------
# the CPU oracle, timed on a bounded sample of heads

def _oracle_slabs(w: dsgen.Workload, max_bytes: int = 2 << 30):
    """Per-head inputs of the CPU oracle: the query, channels, label rows and the
    KV head's rows of every head when they fit in max_bytes, else of a seeded
    sample of heads (the first and last included)."""
    import numpy as np

    import oracle as orc_np

    per_head = w.T * w.d * 2 * 2 + w.T * w.r * 2
    n = w.B * w.Hq if per_head * w.B * w.Hq <= max_bytes else max(1, max_bytes // per_head)
    rng = np.random.default_rng(1)
    heads = (np.arange(w.B * w.Hq) if n == w.B * w.Hq
             else np.sort(rng.permutation(w.B * w.Hq)[:n]))
    C = dsgen.channels(w)
    Qs = np.empty((n, w.d), np.uint16)
    Ks = np.empty((n, w.T, w.d), np.uint16)
    Vs = np.empty((n, w.T, w.d), np.uint16)
    Ls = np.empty((n, w.T, w.r), np.uint16)
    Cs = np.empty((n, w.r), np.int32)
    full = None
    if n == w.B * w.Hq:
        full = dsgen.qkv(w)
    for i, p in enumerate(heads):
        b, h = divmod(int(p), w.Hq)
        g = h // w.G
        if full is not None:
            Qs[i], Ks[i], Vs[i] = full[0][b, h], full[1][b, g], full[2][b, g]
        else:
            Qs[i] = dsgen.q_slab(w, b, h)
            Ks[i] = dsgen.kv_slab(w, "K", b, g)
            Vs[i] = dsgen.kv_slab(w, "V", b, g)
        Cs[i] = C[h]
        Ls[i] = orc_np.label_head(Ks[i], C[h])  # label cache: setup, not timed
    return heads, Qs, Cs, Ls, Ks, Vs


def time_oracle(w: dsgen.Workload, budget_s: float, with_dense: bool = False,
                max_bytes: int = 2 << 30, slabs=None):
    """The C++ oracle (float64, std::sort, std::exp) on the host cores: score,
    top-k and attention per head, the heads spread over every core by
    std::thread (cores = the threads it used), repeated over the heads until the
    time budget is spent; dense attention the same way when with_dense.  The
    numpy oracle on one head, one thread, is reported beside it.  Without a C++
    compiler the numpy oracle alone is timed, one thread, and `sample` says so."""
    import numpy as np

    import oracle as orc_np

    heads, Qs, Cs, Ls, Ks, Vs = slabs if slabs is not None else _oracle_slabs(w, max_bytes)
    n = len(heads)
    per_head = w.T * w.r * 2 + w.k * 4 * w.d + w.d * 6
    try:
        import oracle.cxx as orc_cxx
        orc_cxx.build()
    except Exception:  # noqa: BLE001  (no C++ compiler: numpy alone, said so)
        orc_cxx = None

    def numpy_head(i, dense=False):
        t0 = time.perf_counter()
        if dense:
            orc_np.attend_head(Qs[i], Ks[i], Vs[i], np.arange(w.T), w.scale)
        else:
            s = orc_np.to_f32(orc_np.score_head(Qs[i], Cs[i], Ls[i]))
            orc_np.attend_head(Qs[i], Ks[i], Vs[i], orc_np.topk_head(s, w.k), w.scale)
        return time.perf_counter() - t0

    t_np = numpy_head(0)
    np_rate = per_head / t_np / 1e9
    if orc_cxx is None:
        done, el = 1, t_np
        while el < budget_s and done < 100000:
            el += numpy_head(done % n)
            done += 1
        return {"value": per_head * done / el / 1e9, "unit": "GB/s", "cores": 1,
                "kind": "oracle", "us_per_step": el / done * w.B * w.Hq * 1e6,
                "sample": f"{done} head-steps of {w.name} in the float64 numpy oracle, one "
                          f"thread (no C++ compiler)", "by_oracle": {"float64 numpy": np_rate}}

    def cxx_pass(sparse, dense):
        t0 = time.perf_counter()
        res = orc_cxx.step_heads_mt(Qs, Cs, Ls, Ks, Vs, w.k, w.scale, sparse=sparse,
                                    dense=dense)
        return time.perf_counter() - t0, res[-1]

    el, passes, threads = 0.0, 0, 1
    while passes == 0 or el < budget_s:
        dt, threads = cxx_pass(True, False)
        el += dt
        passes += 1
    done = passes * n
    out = {"value": per_head * done / el / 1e9, "unit": "GB/s", "cores": threads,
           "kind": "oracle", "us_per_step": el / done * w.B * w.Hq * 1e6,
           "sample": f"{done} head-steps ({passes} pass(es) over {n} of the {w.B * w.Hq} heads) "
                     f"of {w.name}: score + top-k + attention per head in the float64 C++ "
                     f"oracle (std::sort, std::exp), heads spread over {threads} host threads "
                     f"(std::thread, {el:.1f} s); the float64 numpy oracle, one thread, one "
                     f"head: {np_rate:.3f} GB/s",
           "by_oracle": {"float64 C++ (std::sort, std::exp), all cores":
                         per_head * done / el / 1e9, "float64 numpy, one thread": np_rate}}
    if with_dense:
        eld, pd = 0.0, 0
        while pd == 0 or eld < budget_s / 2:
            dt, _ = cxx_pass(False, True)
            eld += dt
            pd += 1
        dense_bytes = w.T * w.d * 2 * 2 + w.d * 6
        out["dense_us_per_step"] = eld / (pd * n) * w.B * w.Hq * 1e6
        out["dense_gbs"] = dense_bytes * pd * n / eld / 1e9
    return out


# ---------------------------------------------------------------------------

def config_of(w: dsgen.Workload, args, world: int) -> dict:
    """The benchmark configuration both arms report: the workload and how it is run."""
    return {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "d": w.d,
            "T": w.T, "r": w.r, "k": w.k, "path": args.mode,
            "fused_score_topk": not args.unfused,
            "l2": "flushed between steps (256 MiB written, then read back)",
            "cuda_graph": True, "parallelism": f"replicas x{world}"}


def run_reference(args, rank, world):
    if rank != 0:
        return 0
    w = dsgen.workload(args.workload)
    slabs = _oracle_slabs(w)  # inputs drawn once (setup, not timed)
    per_step, n = [], 0
    budget = max(0.25, args.cpu_seconds / max(1, args.steps))
    for _ in range(args.warmup):
        time_oracle(w, budget / 4, slabs=slabs)
    for _ in range(args.steps):
        r = time_oracle(w, budget, slabs=slabs)
        per_step.append(r)
        n += 1
    us = statistics.mean(r["us_per_step"] for r in per_step)
    val = step_bytes(w) / (us * 1e-6) / 1e9
    line = {"impl": "reference", "metric": METRIC, "value": val, "unit": "GB/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": us / 1e3, "us_per_step": us, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": config_of(w, args, world),
            "cpu_baseline": {"value": val, "unit": "GB/s", "cores": per_step[-1]["cores"],
                             "kind": "oracle", "sample": per_step[-1]["sample"] + " per step"},
            "e2e": {"value": val, "unit": "GB/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def sweep_entry(w, steps, warmup, hbm_peak, fused=True, inputs=None):
    """The decode step (ds_decode_step) and, beside it, the separate calls' stages."""
    st = Step(w, fused=fused, inputs=inputs, mode="step")
    tot, _ = time_device(st, steps, warmup)
    st.release()
    ms = tot / steps
    sc = Step(w, fused=fused, inputs=inputs, mode="calls")
    _, stg = time_device(sc, steps, warmup)
    sc.release()
    su = Step(w, fused=False, inputs=inputs, mode="calls")  # score, then top-k over the scores
    _, stu = time_device(su, steps, warmup)
    su.release()
    sb = stage_bytes(w)
    att_ms = stg[2] / steps
    step_gbs = step_bytes(w) / (ms * 1e-3) / 1e9
    att_gbs = sb["sparse_decode"] / (att_ms * 1e-3) / 1e9
    sel_gbs = sb["score_topk"] / (stg[1] / steps * 1e-3) / 1e9
    return {"us_per_step": ms * 1e3, "gbs": step_gbs,
            "frac_of_measured_hbm": step_gbs / hbm_peak,
            "frac_of_8TBs": step_gbs / NOMINAL_HBM_GBS,
            "calls_us_per_step": sum(stg) / steps * 1e3,
            "sparse_decode_us": att_ms * 1e3,
            "sparse_decode_frac": att_gbs / hbm_peak,
            "sparse_decode_frac_of_8TBs": att_gbs / NOMINAL_HBM_GBS,
            "score_topk_us": stg[1] / steps * 1e3,
            "score_topk_frac": sel_gbs / hbm_peak,
            "score_topk_frac_of_8TBs": sel_gbs / NOMINAL_HBM_GBS,
            "score_then_topk_us": stu[1] / steps * 1e3,
            "tokens_heads_per_s": w.B * w.Hq * w.T / (ms * 1e-3)}


def dense_entry(w, steps, warmup, hbm_peak, inputs=None):
    st = Step(w, dense=True, inputs=inputs)
    tot, _ = time_device(st, steps, warmup)
    st.release()
    ms = tot / steps
    gbs = w.dense_bytes() / (ms * 1e-3) / 1e9
    return {"us_per_step": ms * 1e3, "gbs": gbs, "frac_of_measured_hbm": gbs / hbm_peak,
            "frac_of_8TBs": gbs / NOMINAL_HBM_GBS}


def time_graph(fn, steps: int, warmup: int) -> float:
    """Mean device ms of fn() (a few launches) replayed as a CUDA graph, with the
    L2 flushed (256 MiB written, then read back) before each replay."""
    import torch

    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device="cuda")
    fn()  # eager once: one-time setup outside the capture
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True, external=True)
    e1 = torch.cuda.Event(enable_timing=True, external=True)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        e0.record()
        fn()
        e1.record()
    for _ in range(warmup):
        flush_l2(flush)
        g.replay()
    tot = 0.0
    for _ in range(steps):
        flush_l2(flush)
        g.replay()
        torch.cuda.synchronize()
        tot += e0.elapsed_time(e1)
    del g
    return tot / steps


def calib_entry(w, K, hbm_peak, nq: int = 16, steps: int = 50):
    """Offline channel calibration (ds_calibrate) over the workload's keys and nq
    calibration queries per head: reads K once and the queries once."""
    import numpy as np
    import torch

    import post_token_sparse_b200 as ds

    qc = dsgen.q_calib(w, nq)
    Qc = torch.from_numpy(qc.view(np.int16)).view(torch.bfloat16).cuda()
    C = torch.empty((w.Hq, w.r), dtype=torch.int32, device="cuda")
    imp = torch.empty((w.Hq, w.d), dtype=torch.float32, device="cuda")
    dims = ds.Dims(w.B, w.Hq, w.Hkv, w.d, K.shape[2], w.r)
    ws = ds.workspace(ds.OP_CALIBRATE, dims, w.T, nq, "cuda")
    n0 = ds.kernel_launches()
    ds.calibrate(Qc, K, C, w.T, importance=imp, ws=ws)
    launches = ds.kernel_launches() - n0
    ms = time_graph(lambda: ds.calibrate(Qc, K, C, w.T, importance=imp, ws=ws), steps, 5)
    nbytes = w.B * w.Hkv * w.T * w.d * 2 + w.B * w.Hq * nq * w.d * 2
    return {"us": ms * 1e3, "gbs": nbytes / (ms * 1e-3) / 1e9,
            "frac_of_measured_hbm": nbytes / (ms * 1e-3) / 1e9 / hbm_peak,
            "bytes": nbytes, "calibration_queries_per_head": nq, "launches": launches}


def group_entry(w, inputs, hbm_peak, steps: int = 50):
    """Group-shared selection on grouped KV heads: ds_group_decode_step (the step's
    label append, group scores, one selection per KV group, attention with each kept
    row read once for the group's query heads; three launches)."""
    import torch

    import post_token_sparse_b200 as ds

    Q, K, V = inputs
    C = torch.from_numpy(dsgen.channels(w)).cuda()
    label = torch.empty((w.B, w.Hq, w.T, w.r), dtype=torch.bfloat16, device="cuda")
    ds.label_append(K, C, label, 0, w.T)
    sg = torch.empty((w.B * w.Hkv, w.T), dtype=torch.float32, device="cuda")
    idx = torch.empty((w.B * w.Hkv, w.k), dtype=torch.int32, device="cuda")
    O = torch.empty((w.B, w.Hq, w.d), dtype=torch.float32, device="cuda")
    ws = ds.workspace(ds.OP_GROUP_DECODE_STEP, ds.dims_of(Q, K, w.r), w.T, w.k, "cuda")

    def step():
        ds.group_decode_step(Q, K, V, C, label, sg, idx, O, w.T, w.scale, ws=ws)

    ms = time_graph(step, steps, 3)
    nb = w.group_step_bytes()
    return {"us_per_step": ms * 1e3, "bytes": nb, "gbs": nb / (ms * 1e-3) / 1e9,
            "frac_of_measured_hbm": nb / (ms * 1e-3) / 1e9 / hbm_peak,
            "tokens_heads_per_s": w.B * w.Hq * w.T / (ms * 1e-3)}


def block_entry(w, inputs, hbm_peak, bs: int = 64, steps: int = 50):
    """Block-granular selection with blocks of bs tokens and the same token budget
    as the workload's k (kb = k / bs blocks): the step's label append,
    ds_block_score_topk and ds_block_sparse_decode."""
    import torch

    import post_token_sparse_b200 as ds

    Q, K, V = inputs
    kb = max(1, w.k // bs)
    C = torch.from_numpy(dsgen.channels(w)).cuda()
    label = torch.empty((w.B, w.Hq, w.T, w.r), dtype=torch.bfloat16, device="cuda")
    ds.label_append(K, C, label, 0, w.T)
    BH = w.B * w.Hq
    sb = torch.empty((BH, -(-w.T // bs)), dtype=torch.float32, device="cuda")
    bidx = torch.empty((BH, kb), dtype=torch.int32, device="cuda")
    O = torch.empty((w.B, w.Hq, w.d), dtype=torch.float32, device="cuda")
    ws = ds.workspace(ds.OP_BLOCK_SPARSE_DECODE, ds.dims_of(Q, K, w.r), w.T, kb * bs, "cuda")

    def step():
        ds.label_append(K, C, label, w.T - 1, 1)
        ds.block_score_topk(Q, C, label, sb, bidx, w.T, bs)
        ds.block_sparse_decode(Q, K, V, bidx, O, w.T, bs, w.scale, ws=ws)

    ms = time_graph(step, steps, 3)
    nb = w.block_step_bytes(bs, kb)
    return {"us_per_step": ms * 1e3, "block": bs, "blocks_kept": kb, "bytes": nb,
            "gbs": nb / (ms * 1e-3) / 1e9, "frac_of_measured_hbm": nb / (ms * 1e-3) / 1e9 / hbm_peak,
            "tokens_heads_per_s": w.B * w.Hq * w.T / (ms * 1e-3)}


def offload_entry(w, hbm_peak):
    """KV offload: K and V of the workload in page-locked host memory, the label
    cache on the GPU.  A step (new label row, score + top-k, sparse attention)
    reads over the host link only the kept K/V rows; dense decode reads all."""
    import numpy as np
    import torch

    import post_token_sparse_b200 as ds

    Qb, Kb, Vb = dsgen.qkv(w)
    Q = torch.from_numpy(Qb.view(np.int16)).view(torch.bfloat16).cuda()
    K = torch.from_numpy(Kb.view(np.int16)).view(torch.bfloat16).pin_memory()
    del Kb
    V = torch.from_numpy(Vb.view(np.int16)).view(torch.bfloat16).pin_memory()
    del Vb
    C = torch.from_numpy(dsgen.channels(w)).cuda()
    label = torch.empty((w.B, w.Hq, w.T, w.r), dtype=torch.bfloat16, device="cuda")
    ds.label_append(K, C, label, 0, w.T)  # the prompt (setup)
    BH = w.B * w.Hq
    idx = torch.empty((BH, w.k), dtype=torch.int32, device="cuda")
    O = torch.empty((w.B, w.Hq, w.d), dtype=torch.float32, device="cuda")
    dims = ds.dims_of(Q, K, w.r)
    ws = ds.workspace(ds.OP_SPARSE_DECODE, dims, w.T, w.k, "cuda")
    wsd = ds.workspace(ds.OP_DECODE, dims, w.T, w.T, "cuda")

    def step():
        ds.label_append(K, C, label, w.T - 1, 1)
        ds.score_topk(Q, C, label, idx, w.T)
        ds.sparse_decode(Q, K, V, idx, O, w.T, w.scale, ws=ws)

    ms = time_graph(step, 5, 2)
    msd = time_graph(lambda: ds.decode(Q, K, V, O, w.T, w.scale, ws=wsd), 2, 1)
    link = w.B * w.Hq * w.k * 2 * w.d * 2 + w.B * w.Hkv * w.d * 2
    del K, V
    return {"us_per_step": ms * 1e3, "host_link_bytes_per_step": link,
            "host_link_gbs": link / (ms * 1e-3) / 1e9, "dense_us_per_step": msd * 1e3,
            "dense_host_link_bytes": w.dense_bytes(), "speedup_vs_dense": msd / ms}


def hier_entry(w, inputs, hbm_peak, steps: int = 50):
    """Hierarchical (top-down) selection in place of the exact top-k: the step's
    label append, ds_hier_score_topk and ds_sparse_decode over its k tokens."""
    import math

    import torch

    import post_token_sparse_b200 as ds

    Q, K, V = inputs
    C = torch.from_numpy(dsgen.channels(w)).cuda()
    label = torch.empty((w.B, w.Hq, w.T, w.r), dtype=torch.bfloat16, device="cuda")
    ds.label_append(K, C, label, 0, w.T)
    BH = w.B * w.Hq
    idx = torch.empty((BH, w.k), dtype=torch.int32, device="cuda")
    O = torch.empty((w.B, w.Hq, w.d), dtype=torch.float32, device="cuda")
    ws = ds.workspace(ds.OP_SPARSE_DECODE, ds.dims_of(Q, K, w.r), w.T, w.k, "cuda")

    def step():
        ds.label_append(K, C, label, w.T - 1, 1)
        ds.hier_score_topk(Q, C, label, idx, w.T)
        ds.sparse_decode(Q, K, V, idx, O, w.T, w.scale, ws=ws)

    ms = time_graph(step, steps, 3)
    levels = max(0, math.ceil(math.log2(-(-w.T // w.k)))) if w.T > w.k else 0
    rows = 2 * w.k * levels
    nb = BH * (rows * w.r * 2 + w.k * (2 * w.d * 2 + 4) + w.d * 6)
    return {"us_per_step": ms * 1e3, "levels": levels, "label_rows_read_per_head": rows,
            "bytes": nb, "gbs": nb / (ms * 1e-3) / 1e9,
            "frac_of_measured_hbm": nb / (ms * 1e-3) / 1e9 / hbm_peak,
            "tokens_heads_per_s": BH * w.T / (ms * 1e-3)}


def _rounded(e):
    return {k: (_rounded(v) if isinstance(v, dict) else round(v, 4) if isinstance(v, float)
                else v) for k, v in e.items()}


def run_sweep(skip: str, hbm_peak: float):
    """Every other named workload: sparse step and stage times, dense path beside it.

    The T=32K sweep cells share one input set (one seed); the r = d, k = T cell
    runs the whole sparse pipeline with every channel and every token.
    """
    import torch

    out, shared = {}, {}
    for name in dsgen.ORDER:
        if name == skip:
            continue
        ww = dsgen.workload(name)
        key = (ww.seed, ww.B, ww.Hq, ww.Hkv, ww.T)
        if key not in shared:
            shared.clear()
            torch.cuda.empty_cache()
            shared[key] = device_inputs(ww)
        inp = shared[key]
        n = 30 if ww.T >= 16384 else 200
        e = sweep_entry(ww, n, 3, hbm_peak, inputs=inp)
        first_of_set = not name.startswith("sweep") or name.endswith("r8-k512")
        if first_of_set:
            e["dense"] = dense_entry(ww, max(10, n // 3), 2, hbm_peak, inputs=inp)
        if ww.Hq > ww.Hkv:
            e["group_shared"] = group_entry(ww, inp, hbm_peak)
        if first_of_set and ww.T >= 16384:
            e["block_select"] = block_entry(ww, inp, hbm_peak, steps=20)
        if ww.T >= 262144:
            e["kv_offload"] = offload_entry(ww, hbm_peak)
        if ww.k <= 2048 and (first_of_set or ww.Hq > ww.Hkv) and ww.T > 4096:
            e["hier_select"] = hier_entry(ww, inp, hbm_peak, steps=20)
        try:  # the oracle on the host cores beside each workload: a few heads
            e["cpu_baseline"] = time_oracle(ww, 1.0, max_bytes=512 << 20)
        except Exception as ex:  # noqa: BLE001  (the GPU figures stand without it)
            e["cpu_baseline"] = {"kind": "oracle", "error": repr(ex)[:200]}
        out[name] = _rounded(e)
        if name == dsgen.ORDER[-1] and name.startswith("sweep"):
            full = ww.with_(name="sweep-B32-H32-T32K-r128-kT", r=ww.d, k=ww.T)
            out[full.name] = _rounded(sweep_entry(full, 10, 2, hbm_peak, inputs=inp))
    shared.clear()
    torch.cuda.empty_cache()
    return out


# ---------------------------------------------------------------------------
# profiles/: text summaries of the ncu runs of the small bench command

SMALL_CMD = "python bench.py --steps 20 --warmup 5 --no-sweep --cpu-seconds 1"


def summarize_ncu(src: str) -> None:
    """Write profiles/ from an ncu launch list (src/launches.csv, made by
    ``ncu --metrics gpu__time_duration.sum --clock-control none --csv --log-file
    launches.csv <SMALL_CMD>``) and a full capture of the step kernel
    (src/k_step_headline.ncu-rep, ``ncu --set full --clock-control none -k
    regex:k_step -s 5 -c 1 -o k_step_headline <SMALL_CMD>``), read with ``ncu -i``."""
    import collections
    import csv
    import io
    import re
    import subprocess

    w = dsgen.workload(HEADLINE)
    shape = f"B={w.B} Hq={w.Hq} Hkv={w.Hkv} T={w.T} r={w.r} k={w.k}"
    prof = os.path.join(ROOT, "profiles")
    made = "# command (one B200; the same command exited 0 without ncu first, in the same call):"
    # launch list: launches, total time and share per kernel
    rows = [r for r in csv.reader(open(os.path.join(src, "launches.csv"))) if len(r) > 10]
    ki, vi = rows[0].index("Kernel Name"), rows[0].index("Metric Value")
    agg = collections.OrderedDict()
    for r in rows[1:]:
        a = agg.setdefault(re.sub(r"\(.*", "", r[ki]).replace("void ", ""), [0, 0.0])
        a[0] += 1
        a[1] += float(r[vi]) / 1e3
    tot = sum(v[1] for v in agg.values())
    ours = sum(v[1] for k, v in agg.items() if k.startswith("ds::"))
    lines = [f"# Launch list of the small bench run, workload {w.name} ({shape})", made,
             "#   ncu --metrics gpu__time_duration.sum --clock-control none --csv --log-file "
             "launches.csv \\", f"#       {SMALL_CMD}",
             f"# summarised by: python bench.py --summarize-ncu <dir of the ncu outputs>",
             "# Under ncu every launch runs serialised with cold caches: compare shares, not "
             "absolute times.",
             "# at::...FillFunctor<unsigned char> is the bench's 256 MiB L2 flush between timed "
             "steps (outside",
             "# the timed region); the other at:: kernels are setup.  Shares of the library's own "
             "kernels are",
             "# also given relative to their sum.", "",
             f"{'kernel':58s} {'launches':>8s} {'total us':>11s} {'share':>7s} {'share(ds)':>9s} "
             f"{'avg us':>8s}"]
    for k, (n, t) in sorted(agg.items(), key=lambda x: -x[1][1]):
        sd = f"{100 * t / ours:8.1f}%" if k.startswith("ds::") else " " * 9
        lines.append(f"{k[:58]:58s} {n:8d} {t:11.1f} {100 * t / tot:6.1f}% {sd} {t / n:8.2f}")
    lines.append(f"{'total':58s} {len(rows) - 1:8d} {tot:11.1f}")
    open(os.path.join(prof, f"launches_{w.name}.txt"), "w").write("\n".join(lines) + "\n")

    # the step kernel's full capture
    raw = subprocess.run(["ncu", "-i", os.path.join(src, "k_step_headline.ncu-rep"), "--page",
                          "raw", "--csv"], capture_output=True, text=True, check=True).stdout
    rr = list(csv.reader(io.StringIO(raw)))
    h, units, vals = rr[0], rr[1], rr[2]

    def get(m):
        return (vals[h.index(m)], units[h.index(m)]) if m in h else ("n/a", "")

    def num(m):
        v, u = get(m)
        return float(v.replace(",", "")) * {"Kbyte": 1e3, "Mbyte": 1e6, "Gbyte": 1e9}.get(u, 1)

    rd, wr = num("dram__bytes_read.sum"), num("dram__bytes_write.sum")
    dur = num("gpu__time_duration.sum") / (1e3 if get("gpu__time_duration.sum")[1] == "ns"
                                           else 1)
    alg = stage_bytes(w)["decode_step"]
    pre, post = "smsp__average_warps_issue_stalled_", "_per_issue_active.ratio"
    stalls = sorted(((float(vals[i] or 0), m[len(pre):-len(post)]) for i, m in enumerate(h)
                     if m.startswith(pre) and m.endswith(post) and float(vals[i] or 0) >= 0.05),
                    reverse=True)
    cmd = f"ncu --set full --clock-control none -k regex:k_step -s 5 -c 1 -o k_step_headline " \
          f"{SMALL_CMD}"
    L = [f"# k_step<{w.r}> (ds_decode_step, one launch per decode step), workload {w.name}", made,
         f"#   {cmd}", "# summarised by: python bench.py --summarize-ncu <dir of the ncu outputs>",
         "# the 6th k_step launch (a graph-replayed timed step); ncu flushes caches before it "
         "(cold).",
         f"duration_us (under ncu, cold): {dur:.2f}",
         f"dram_bytes_read: {rd:.0f}", f"dram_bytes_write: {wr:.0f}",
         f"dram_bytes_total: {rd + wr:.0f}",
         f"algorithmic_bytes_per_launch: {alg}  (labels + selected K/V rows + idx + Q/O + new "
         "label rows)",
         f"traffic / algorithmic: {(rd + wr) / alg:.3f}",
         "dram throughput (% of peak, elapsed): "
         f"{get('gpu__dram_throughput.avg.pct_of_peak_sustained_elapsed')[0]}",
         "sm throughput (% of peak, elapsed): "
         f"{get('sm__throughput.avg.pct_of_peak_sustained_elapsed')[0]}",
         "issue active (% of active cycles): "
         f"{get('smsp__issue_active.avg.pct_of_peak_sustained_active')[0]}",
         f"registers/thread: {get('launch__registers_per_thread')[0]}  grid: "
         f"{get('launch__grid_size')[0]}  block: {get('launch__block_size')[0]}",
         f"dynamic smem/block: {get('launch__shared_mem_per_block_dynamic')[0]} "
         f"{get('launch__shared_mem_per_block_dynamic')[1]}",
         f"occupancy limit (registers): {get('launch__occupancy_limit_registers')[0]} blocks/SM",
         "warps active (% of peak, active cycles): "
         f"{get('sm__warps_active.avg.pct_of_peak_sustained_active')[0]}",
         f"L2 hit rate (%): {get('lts__t_sector_hit_rate.pct')[0]}",
         "shared-memory bank conflicts (sum): "
         f"{get('l1tex__data_bank_conflicts_pipe_lsu_mem_shared.sum')[0]}",
         "warp stall reasons (cycles per issued instruction, >= 0.05):"]
    L += [f"  {n:24s} {v:.2f}" for v, n in stalls]
    open(os.path.join(prof, f"k_step_{w.name}.txt"), "w").write("\n".join(L) + "\n")

    T = [f"# DRAM traffic per launch of the dominant kernel, workload {w.name} ({shape})",
         f"# from the full capture summarised in profiles/k_step_{w.name}.txt:", f"#   {cmd}",
         "# read by bench.py for roofline.traffic while kernel_source_hash matches the sources.",
         f"kernel_source_hash: {kernel_source_hash()}",
         f"dram_bytes_per_launch[k_step]: {rd + wr:.0f}",
         f"gpu_time_ns[k_step]: {dur * 1e3:.0f}"]
    open(os.path.join(prof, f"traffic_{w.name}.txt"), "w").write("\n".join(T) + "\n")

    # the group-by-group attention kernel, when its capture is present
    grep = os.path.join(src, "k_attend_group_gqa.ncu-rep")
    if os.path.exists(grep):
        g = dsgen.workload("gqa-B16-Hq64-Hkv8-T16K")
        raw = subprocess.run(["ncu", "-i", grep, "--page", "raw", "--csv"], capture_output=True,
                             text=True, check=True).stdout
        rr = list(csv.reader(io.StringIO(raw)))
        h, units, vals = rr[0], rr[1], rr[2]
        rd, wr = num("dram__bytes_read.sum"), num("dram__bytes_write.sum")
        dur = num("gpu__time_duration.sum") / (1e3 if get("gpu__time_duration.sum")[1] == "ns"
                                               else 1)
        alg = g.dense_bytes()
        stalls = sorted(((float(vals[i] or 0), m[len(pre):-len(post)]) for i, m in enumerate(h)
                         if m.startswith(pre) and m.endswith(post) and float(vals[i] or 0) >= 0.05),
                        reverse=True)
        gcmd = ("ncu --set full --clock-control none -k regex:k_attend_group -c 1 -o "
                "k_attend_group_gqa python -m pytest tests/test_gpu_attend_group.py -q -k "
                "full_gqa_workload_dense")
        G = [f"# k_attend_group<false> (ds_decode, dense, 8 query heads per KV head), workload "
             f"{g.name} (B={g.B} Hq={g.Hq} Hkv={g.Hkv} T={g.T})", made, f"#   {gcmd}",
             "# summarised by: python bench.py --summarize-ncu <dir of the ncu outputs>",
             "# ncu flushes caches before the captured launch (cold).",
             f"duration_us (under ncu, cold): {dur:.2f}",
             f"dram_bytes_read: {rd:.0f}", f"dram_bytes_write: {wr:.0f}",
             f"algorithmic_bytes_per_launch: {alg}  (K and V once per KV head + Q/O)",
             f"traffic / algorithmic: {(rd + wr) / alg:.3f}",
             f"achieved (algorithmic / duration): {alg / dur / 1e3:.0f} GB/s",
             "dram throughput (% of peak, elapsed): "
             f"{get('gpu__dram_throughput.avg.pct_of_peak_sustained_elapsed')[0]}",
             *[f"{m}: {vals[i]}" for i, m in enumerate(h)
               if "pipe_tensor" in m and "pct_of_peak_sustained" in m][:6],
             f"registers/thread: {get('launch__registers_per_thread')[0]}  grid: "
             f"{get('launch__grid_size')[0]}  block: {get('launch__block_size')[0]}",
             "warps active (% of peak, active cycles): "
             f"{get('sm__warps_active.avg.pct_of_peak_sustained_active')[0]}",
             "warp stall reasons (cycles per issued instruction, >= 0.05):"]
        G += [f"  {n:24s} {v:.2f}" for v, n in stalls]
        open(os.path.join(prof, f"k_attend_group_{g.name}.txt"), "w").write("\n".join(G) + "\n")


def main():
    args = parse()
    if args.summarize_ncu:
        summarize_ncu(args.summarize_ncu)
        return 0
    rank, local_rank, world = rank_env()
    if args.impl == "reference":
        return run_reference(args, rank, world)

    import torch

    torch.cuda.set_device(local_rank)
    if world > 1:
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    hbm_peak, peak_kind = peaks()

    base = dsgen.workload(args.workload)
    if args.batch:
        base = base.with_(B=args.batch)
    w = replica_workload(base, rank)
    inputs = device_inputs(w)
    step = Step(w, fused=not args.unfused, inputs=inputs, mode=args.mode)

    def barrier():
        if world > 1:
            torch.distributed.barrier()
        torch.cuda.synchronize()

    barrier()
    with ClockSampler(local_rank) as clocks:
        total_ms, stage_ms = time_device(step, args.steps, args.warmup)
    barrier()
    ms_step = max_over_ranks(total_ms, world, "cuda") / args.steps
    value = job_gbs(step_bytes(w), world, ms_step)

    e2e_steps = max(10, min(args.steps, 200))
    e2e_ms, e2e_graph_ms, h2d, d2h = time_e2e(step, e2e_steps, 5)
    e2e_step_ms = max_over_ranks(e2e_ms, world, "cuda") / e2e_steps
    e2e_val = job_gbs(step_bytes(w), world, e2e_step_ms)
    e2e_graph_step_ms = max_over_ranks(e2e_graph_ms, world, "cuda") / e2e_steps

    # dominant stage of the step and its roofline
    sb = stage_bytes(w)
    names = ("decode_step",) if args.mode == "step" else Step.STAGES
    dom = max(range(len(stage_ms)), key=lambda i: stage_ms[i])
    dom_ms = stage_ms[dom] / args.steps
    kern = {"label_append": "k_label_append", "score_topk": "k_topk",
            "sparse_decode": "k_attend", "decode_step": "k_step"}[names[dom]]
    achieved = sb[names[dom]] / (dom_ms * 1e-3) / 1e9
    traffic = profiled_traffic(kern)
    roofline = {"bound": "hbm", "achieved": achieved, "peak": hbm_peak, "unit": "GB/s",
                "frac": achieved / hbm_peak, "traffic": traffic,
                "kernel": names[dom], "peak_kind": f"{peak_kind} hbm_gbs (copy)",
                "algorithmic_bytes_per_launch": sb[names[dom]],
                "avg_launch_us": dom_ms * 1e3}
    stages = {n: {"us": stage_ms[i] / args.steps * 1e3,
                  "gbs": sb[n] / (stage_ms[i] / args.steps * 1e-3) / 1e9}
              for i, n in enumerate(names)}

    line = {"metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
            "us_per_step": ms_step * 1e3,
            "tokens_heads_per_s": world * w.B * w.Hq * w.T / (ms_step * 1e-3),
            "frac_of_8TBs": value / world / NOMINAL_HBM_GBS,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f32", "storage": "bf16", "data": "synthetic",
            "config": config_of(w, args, world),
            "stages": stages, "roofline": roofline,
            "gpu_launches": step.launches_per_step * args.steps,
            "clocks": clocks.summary(),
            "e2e": {"value": e2e_val, "unit": "GB/s", "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h, "steps": e2e_steps,
                    "us_per_step": e2e_step_ms * 1e3,
                    "timing": "host clock around each public-API call (Python binding "
                              "decode_step_kv -> C ABI ds_decode_step_kv, pinned host Q, new "
                              "K/V rows and O) and the host synchronisation after it; L2 "
                              "flushed before each call, outside the timed region",
                    "graph": {"us_per_step": e2e_graph_step_ms * 1e3,
                              "gbs": job_gbs(step_bytes(w), world, e2e_graph_step_ms),
                              "timing": "the same call captured in a CUDA graph, replayed, "
                                        "device events"}}}
    if rank == 0 and world == 1:
        try:  # the same step without the flush: L2 as the previous step left it
            wn = min(args.steps, 200)
            for _ in range(3):
                step.timed(flush=False)
            warm_ms = sum(step.timed(flush=False)[0] for _ in range(wn)) / wn
            line["warm"] = {"us_per_step": warm_ms * 1e3, "steps": wn,
                            "gbs": step_bytes(w) / (warm_ms * 1e-3) / 1e9,
                            "l2": f"not flushed between steps (the step reads "
                                  f"{step_bytes(w) / 1e6:.0f} MB; L2 holds 126 MB)"}
        except Exception as e:  # noqa: BLE001  (the flushed figures stand without it)
            line["warm"] = {"error": repr(e)[:200]}
    step.release()
    if args.mode == "step":
        # the same step as separate calls: per-kernel stage times
        calls = Step(w, fused=not args.unfused, inputs=inputs, mode="calls")
        ctot, cst = time_device(calls, max(20, args.steps // 5), 3)
        cn = max(20, args.steps // 5)
        calls.release()
        line["calls"] = {"us_per_step": ctot / cn * 1e3,
                         "stages": {n: {"us": cst[i] / cn * 1e3,
                                        "gbs": sb[n] / (cst[i] / cn * 1e-3) / 1e9,
                                        "frac_of_measured_hbm":
                                            sb[n] / (cst[i] / cn * 1e-3) / 1e9 / hbm_peak}
                                    for i, n in enumerate(Step.STAGES)}}
    if rank == 0 and world == 1:
        dn = dense_entry(w, max(20, args.steps // 10), 3, hbm_peak, inputs=inputs)
        line["dense"] = dn
        line["speedup_vs_dense"] = dn["us_per_step"] / line["us_per_step"]
        try:
            line["cpu_baseline"] = time_oracle(base, args.cpu_seconds, with_dense=True)
        except Exception as e:  # noqa: BLE001  (the GPU figures stand without it)
            line["cpu_baseline"] = {"kind": "oracle", "error": repr(e)[:200]}
        line["calibrate"] = _rounded(calib_entry(w, inputs[1], hbm_peak))
        line["block_select"] = _rounded(block_entry(w, inputs, hbm_peak))
        line["hier_select"] = _rounded(hier_entry(w, inputs, hbm_peak))
    del inputs
    torch.cuda.empty_cache()
    if rank == 0 and world == 1:
        if not args.no_sweep:
            line["sweep"] = run_sweep(w.name, hbm_peak)
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
