#!/usr/bin/env python
"""Benchmarks of the compressed-KV hot path (one JSON line on rank 0).

  python bench.py [--config 1..5] [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Workloads (--config; 3 is the default and the headline line):

  1  Tiny single RoPE head: d=64, 256 keys/values, 4 queries, fp32 N(0,1) with
     channels 3, 17, 40 scaled x20, RoPE base 10000. Step = quantise keys
     (RoPE + QJL) and values, then decode the 4 queries (RoPE at position 256).
     value = tokens/s; the figure that matters is the latency of one step,
     eager and replayed from a CUDA graph.
  2  ESM-2-650M-shaped cache: 33 layers x 20 heads x d=64, 1024 tokens, bf16,
     per-head SVD rotations and dual (K/V) empirical codebooks. Step = quantise
     the whole cache (one call for keys, one for values), then one
     bidirectional 1024-query attention pass per layer. value = tokens/s.
  3  Llama-3.1-8B-shaped decode: 32 layers, batch 8, 32 q / 8 kv heads,
     head_dim 128, context 32768, bf16 N(0,1) with 2% of channels x10.
     Step = quantise every layer's keys (3-bit + QJL) and values (3-bit), then
     one decode query per (batch, query head) per layer. value = context
     tokens/s.
  4  Long context: 1 layer, batch 1, 8 kv / 32 q heads, d=128, context 131072,
     bf16 with heavy-tailed outlier channels. Key bits 2, 3 and 4 (each with
     QJL), 3-bit values. Step = one decode call per key bit width, L2 flushed
     before each call. value = keys scored/s; per bit width: keys/s, HBM
     fraction, key-quantise time and the score error against exact
     q.k/sqrt(d).
  5  Vector search: 1,000,000 unit vectors d=200 from a 100-component Gaussian
     mixture, 10,000 queries, 3-bit + QJL codes. Step = top-10 of every query
     by estimated inner product over the whole corpus. value = estimated
     scores/s; recall@10 of all 10,000 queries against exact fp32 search.

Timing: W untimed warm-up steps, then K timed steps between CUDA events on the
launching stream, bracketed by barrier + synchronize; max over ranks. Where a
workload's bytes fit in L2 (configs 4, 5) the L2 is flushed before every timed
call and only the calls are timed. "gpu_launches" is the library's own count
of kernels it launched inside the timed region (tq_kernel_launches).

Multi-GPU: every rank runs an independent replica with its own seeded data (no
data-path collective); value sums the ranks' work over the slowest rank's time.
`--gpus N` without a launcher re-executes this script under
torch.distributed.run with N processes; under a launcher WORLD_SIZE must
equal N.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import platform
import socket
import statistics
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "decode-attn keys scored/s & HBM GB/s on 3+1-bit KV; quantize tokens/s"

WORKLOADS = {
    1: ("Tiny single head: d=64, N=256 keys/values, 4 queries, fp32 N(0,1) with channels 3,17,40 x20; "
        "RoPE base 10000 on q,k; 3-bit keys+values, 1-bit QJL; seed 0"),
    2: ("ESM-2-650M-shaped KV: 33 layers x 20 heads x head_dim 64, seq 1024, batch 1, bf16 K/V after RoPE, "
        "4 of 64 channels per head lognormal(2,1) x random sign; per-head SVD basis from 256 calibration tokens, "
        "dual K/V codebooks; quantise the whole cache, then one full-sequence attention pass per layer"),
    3: ("Llama-3.1-8B-shaped decode: 32 layers, batch 8, 32 q / 8 kv heads, head_dim 128, context 32768, "
        "bf16 N(0,1) K/V with 2% channels x10; 3-bit+QJL keys, 3-bit values; one decode step per layer"),
    4: ("Long-context sweep: 1 layer, 8 kv / 32 q heads, head_dim 128, context 131072, batch 1, bf16 K/V with "
        "8 of 128 channels lognormal(2,1) x random sign; key bits 2/3/4 each with QJL, 3-bit values"),
    5: ("Vector search: 1,000,000 database vectors d=200 from a 100-component Gaussian mixture, L2-normalised, "
        "fp32; 10,000 queries from the same mixture; 3-bit+QJL codes; top-10 by estimated inner product"),
}

# DRAM traffic of a kernel per unit of work: dram__bytes_read.sum +
# dram__bytes_write.sum of one launch on a smaller case of the same shape
# (one kernel, one launch, ncu), divided by the units that launch processed.
# An entry counts only while the listed sources still hash to `sha`; after any
# change to them the traffic is reported as null until it is captured again.
# Captured on the Llama-shaped cache at context 8192 (1 layer, 524,288 vectors
# per call); at that size part of a call's output is still in L2 when the
# kernel ends, so the write bytes are a lower bound. The quantise entries sum
# the main kernel and its fixup (the call the roofline times). The quantise
# entries' sha covers a later change of the fixup's grid size only (host code;
# the kernels' device code is the captured one, and the fixup reads the flag
# words and the flagged rows once whatever its grid).
TRAFFIC = {
    "decode_fused3_d128": {"bytes_per_unit": (65_936_640 + 58_624) / 524_288, "sha": "d958b2d61582ac83",
                           "sources": ["tq_decode_tc.cu", "tq_decode_tc.h", "tq_sm100.cuh"]},
    "quantize_tc_key3_d128": {"bytes_per_unit": (134_523_136 + 17_896_448 + 2_691_072) / 524_288,
                              "sha": "6813150f16aa91eb", "sources": ["tq_quantize_tc.cu", "tq_tc.h", "tq_sm100.cuh"]},
    "quantize_tc_value3_d128": {"bytes_per_unit": (134_339_072 + 9_486_336 + 2_416_640) / 524_288,
                                "sha": "6813150f16aa91eb",
                                "sources": ["tq_quantize_tc.cu", "tq_tc.h", "tq_sm100.cuh"]},
}

CSRC = os.path.join(ROOT, "kv_cache_vector_rope_b200", "csrc")


def parse(argv=None):
    p = argparse.ArgumentParser()
    p.add_argument("--config", type=int, choices=[1, 2, 3, 4, 5], default=3)
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=None, help="timed steps (default per config)")
    p.add_argument("--warmup", type=int, default=3)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--layers", type=int, default=32, help="config 3: layers of the cache (32 = the full workload)")
    p.add_argument("--context", type=int, default=32768,
                   help="config 3: context length (32768 = the full workload; smaller only for profiling)")
    p.add_argument("--e2e-steps", type=int, default=2)
    p.add_argument("--incremental-steps", type=int, default=8,
                   help="config 3: generated tokens timed for the append-then-decode line (0: skip)")
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--no-cpu", action="store_true")
    p.add_argument("--cpu-budget", type=float, default=12.0,
                   help="seconds of oracle work for each of the two cpu_baseline timings")
    a = p.parse_args(argv)
    if a.steps is None:
        a.steps = {1: 5000, 2: 20, 3: 20, 4: 300, 5: 5}[a.config]
    return a


# ---------------------------------------------------------------------------
# Clock sampling during the timed region.
# ---------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device: int):
        self.proc = None
        self.lines = []
        try:
            uuid = str(torch.cuda.get_device_properties(device).uuid)
            ident = uuid if uuid.startswith("GPU-") else f"GPU-{uuid}"
            self.proc = subprocess.Popen(["nvidia-smi", "-i", ident, f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "50"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
            t0 = time.time()                      # the first sample precedes the timed region
            while not self.lines and time.time() - t0 < 5.0:
                time.sleep(0.01)
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [x.strip() for x in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx.append(float(parts[2]))
            except ValueError:
                continue
            for nm, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------------------
# Process launch and distributed plumbing (one process per GPU; no data-path
# collective).
# ---------------------------------------------------------------------------
def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def launch_or_check(args, argv=None) -> None:
    """--gpus N: re-execute under torch.distributed.run when no launcher set
    WORLD_SIZE; under a launcher, WORLD_SIZE must be N."""
    world_env = os.environ.get("WORLD_SIZE")
    if world_env is None:
        if args.gpus > 1:
            argv = sys.argv[1:] if argv is None else argv
            cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={args.gpus}",
                   "--master-addr", "127.0.0.1", f"--master-port={_free_port()}", os.path.abspath(__file__)] + argv
            sys.exit(subprocess.call(cmd))
        return
    if int(world_env) != args.gpus:
        sys.exit(f"bench.py: --gpus {args.gpus} but WORLD_SIZE={world_env}; run one process per GPU "
                 f"(e.g. torch.distributed.run --nproc-per-node {args.gpus})")
    if torch.cuda.is_available() and torch.cuda.device_count() < int(world_env):
        sys.exit(f"bench.py: WORLD_SIZE={world_env} but only {torch.cuda.device_count()} GPU(s) visible")


def dist_setup(args=None, timeout_s: float = 600.0):
    """One process per GPU (NCCL); without a GPU the same plumbing runs on gloo."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
            torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=timeout_s),
                                                 device_id=torch.device("cuda", local))
        else:
            torch.distributed.init_process_group("gloo", timeout=datetime.timedelta(seconds=timeout_s))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    if world > 1:
        torch.distributed.barrier()


def max_over_ranks(world, x: float) -> float:
    """The slowest rank's time (every rank takes part)."""
    if world == 1:
        return x
    nccl = torch.distributed.get_backend() == "nccl"
    t = torch.tensor([x], dtype=torch.float64, device="cuda" if nccl else "cpu")
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def replica_seed(rank: int) -> int:
    """Each rank quantises and attends over its own data (independent units)."""
    return rank


# ---------------------------------------------------------------------------
# Peaks, rooflines and traffic.
# ---------------------------------------------------------------------------
def load_peaks() -> dict:
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            pk = json.load(f)
    except Exception:
        pk = {}
    out = {"hbm_gbs": float(pk.get("hbm_gbs", 6650.0)), "hbm_src": "measured" if "hbm_gbs" in pk else "fallback"}
    return out


def alu_peak_tops(clk: dict) -> tuple[float, str]:
    """FP32 lane operations per second: SMs x 128 FP32 lanes x max SM clock."""
    sms = torch.cuda.get_device_properties(torch.cuda.current_device()).multi_processor_count
    mhz = clk.get("sm_max_mhz") or 1965.0
    return sms * 128 * mhz * 1e6 / 1e12, f"{sms} SMs x 128 FP32 lanes x {mhz:.0f} MHz (one op per lane per clock)"


def _sources_sha(files) -> str:
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(CSRC, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def traffic_for(key: str, units: float):
    e = TRAFFIC.get(key)
    if e is None or _sources_sha(e["sources"]) != e["sha"]:
        return None
    return e["bytes_per_unit"] * units


def hbm_roofline(kernel, alg_bytes, seconds, peaks, per_unit, traffic_key=None, units=None):
    achieved = alg_bytes / seconds / 1e9
    return {"kernel": kernel, "bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
            "frac": achieved / peaks["hbm_gbs"], "peak_source": peaks["hbm_src"],
            "traffic": traffic_for(traffic_key, units) if traffic_key else None, "per_unit": per_unit}


def alu_roofline(kernel, ops, seconds, clk, per_unit):
    peak, how = alu_peak_tops(clk)
    achieved = ops / seconds / 1e12
    return {"kernel": kernel, "bound": "alu", "achieved": achieved, "peak": peak, "unit": "Top/s",
            "frac": achieved / peak, "peak_source": f"derived: {how}", "traffic": None, "per_unit": per_unit}


class L2Flush:
    """Writes a buffer larger than the 126 MB L2 (outside the timed calls)."""

    def __init__(self, dev, mib: int = 384):
        self.buf = torch.empty(mib << 20, dtype=torch.uint8, device=dev)
        self.v = 0

    def __call__(self):
        self.v = (self.v + 1) & 255
        self.buf.fill_(self.v)


def packed_bytes(d: int, bits: int, key: bool) -> int:
    """Bytes of one packed vector: codes, (signs, residual norm) and the norm."""
    return d * bits // 8 + 4 + ((d + 31) // 32 * 4 + 4 if key else 0)


def dev_tensor(x, dev, dtype=torch.float32):
    return torch.as_tensor(np.ascontiguousarray(x), device=dev).to(dtype)


def ev():
    return torch.cuda.Event(enable_timing=True)


# ---------------------------------------------------------------------------
# Oracle baselines on the host cores (bounded samples of each workload).
# ---------------------------------------------------------------------------
def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for ln in f:
                if ln.startswith("model name"):
                    return ln.split(":", 1)[1].strip()
    except Exception:
        pass
    return platform.processor() or "unknown"


def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        return max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    except Exception:
        return os.cpu_count() or 1


def _tiny_oracle_inputs(seed=0):
    th = synth.tiny_head(seed)
    return th


def cpu_sample(cfg: int, budget_s: float) -> dict:
    """The oracle on a bounded sample of config `cfg`; returns value/unit/sample."""
    from oracle import attention as oa
    from oracle import codebook as ocb
    from oracle import quantize as oq
    rg = np.random.default_rng(12345)
    f32 = lambda a: np.asarray(a, dtype=np.float32).astype(np.float64)

    def book(d, bits):
        b = ocb.lloyd_max_beta(d, bits)
        return f32(b.centroids), f32(0.5 * (b.centroids[1:] + b.centroids[:-1]))

    if cfg == 1:
        th = synth.tiny_head(0)
        c, t = book(th.d, 3)
        reps, t0 = 0, time.perf_counter()
        while True:
            kq = oq.quantize(th.K, th.Pi, c, t, 3, S=th.S, positions=th.k_pos, rope_base=th.rope_base)
            vq = oq.quantize(th.V, th.Pi, c, t, 3)
            oa.attention(th.Q, oa.KeyPlanes(kq.idx_plane, kq.sign_plane, kq.norm, kq.rnorm, 3),
                         oa.ValuePlanes(vq.idx_plane, vq.norm, 3), th.Pi, th.Pi, th.S, c, c,
                         q_positions=th.q_pos, rope_base=th.rope_base)
            reps += 1
            if time.perf_counter() - t0 > budget_s:
                break
        per = (time.perf_counter() - t0) / reps
        return {"value": th.K.shape[0] / per, "unit": "tokens/s", "seconds_per_step": per,
                "sample": f"the whole workload ({reps} repetitions); no extrapolation"}
    if cfg == 2:
        d, n = 64, 1024
        c, t = book(d, 3)
        Pi = synth.random_rotation(d, 0)
        S = synth.gaussian_projection(d, 0)
        chans = rg.choice(d, 4, replace=False)

        def draw():
            x = rg.standard_normal((n, d))
            x[:, chans] = rg.lognormal(2.0, 1.0, (n, 4)) * np.where(rg.random((n, 4)) < 0.5, -1.0, 1.0)
            return synth.to_bf16(x.astype(np.float32)).float().numpy().astype(np.float64)

        K, V, Q = draw(), draw(), rg.standard_normal((n, d))
        heads, t0 = 0, time.perf_counter()
        while True:
            kq = oq.quantize(K, Pi, c, t, 3, S=S)
            vq = oq.quantize(V, Pi, c, t, 3)
            oa.attention(Q, oa.KeyPlanes(kq.idx_plane, kq.sign_plane, kq.norm, kq.rnorm, 3),
                         oa.ValuePlanes(vq.idx_plane, vq.norm, 3), Pi, Pi, S, c, c)
            heads += 1
            if time.perf_counter() - t0 > budget_s:
                break
        per_head = (time.perf_counter() - t0) / heads
        return {"value": n / (33 * 20 * per_head), "unit": "tokens/s", "seconds_per_head": per_head,
                "sample": (f"{heads} (layer, head) unit(s): quantise 1024 keys + 1024 values (d=64, 3-bit, QJL), "
                           f"1024-query attention over them; extrapolated x660 heads (33 layers x 20)")}
    if cfg in (3, 4):
        d = 128
        c, t = book(d, 3)
        Pi = synth.random_rotation(d, 0)
        S = synth.gaussian_projection(d, 0)
        shape = synth.LlamaDecodeShape()

        def draw(m):
            x = rg.standard_normal((m, d))
            x[:, rg.choice(d, shape.n_outlier, replace=False)] *= shape.outlier_scale
            return synth.to_bf16(x.astype(np.float32)).float().numpy().astype(np.float64)

        probe = draw(256)
        t0 = time.perf_counter()
        oq.quantize(probe, Pi, c, t, 3, S=S)
        oq.quantize(probe, Pi, c, t, 3)
        per_q = (time.perf_counter() - t0) / 256
        m = int(max(256, min(1 << 16, 0.5 * budget_s / max(per_q, 1e-9))))
        Kx, Vx = draw(m), draw(m)
        t0 = time.perf_counter()
        kq = oq.quantize(Kx, Pi, c, t, 3, S=S)
        t_k = time.perf_counter() - t0
        t0 = time.perf_counter()
        vq = oq.quantize(Vx, Pi, c, t, 3)
        t_v = time.perf_counter() - t0
        kp = oa.KeyPlanes(kq.idx_plane, kq.sign_plane, kq.norm, kq.rnorm, 3)
        vp = oa.ValuePlanes(vq.idx_plane, vq.norm, 3)
        q = rg.standard_normal((4, d))
        reps, t0 = 0, time.perf_counter()
        while True:
            oa.attention(q, kp, vp, Pi, Pi, S, c, c)
            reps += 1
            if time.perf_counter() - t0 > 0.4 * budget_s:
                break
        t_att = (time.perf_counter() - t0) / reps
        if cfg == 3:
            per_token_head = (t_k + t_v + t_att) / m
            units = shape.layers * shape.hkv
            return {"value": 1.0 / (units * per_token_head), "unit": "tokens/s",
                    "seconds": {"quantize_k": t_k, "quantize_v": t_v, "attention": t_att},
                    "sample": (f"quantise {m} key + {m} value vectors (d=128, 3-bit, QJL), decode attention of 4 "
                               f"query heads over those {m} packed tokens; extrapolated to {units} (layer, kv-head) "
                               f"units per context token")}
        return {"value": 4 * m / t_att, "unit": "keys scored/s", "seconds": {"attention": t_att},
                "sample": (f"decode attention of 4 query heads (one GQA group) over {m} packed 3-bit+QJL tokens; "
                           f"keys scored/s (per-key cost is independent of the context length)")}
    # cfg 5
    from oracle import search as osr
    d = 200
    c, t = book(d, 3)
    Pi = synth.random_rotation(d, 0)
    S = synth.gaussian_projection(d, 0)
    m = 20000
    X = rg.standard_normal((m, d))
    X /= np.linalg.norm(X, axis=1, keepdims=True)
    kq = oq.quantize(X, Pi, c, t, 3, S=S)
    kp = oa.KeyPlanes(kq.idx_plane, kq.sign_plane, kq.norm, kq.rnorm, 3)
    Q = rg.standard_normal((8, d))
    reps, t0 = 0, time.perf_counter()
    while True:
        sc = osr.estimated_scores(Q, kp, Pi, S, c)
        osr.top_k(sc, 10)
        reps += 1
        if time.perf_counter() - t0 > budget_s:
            break
    per = (time.perf_counter() - t0) / reps
    return {"value": 8 * m / per, "unit": "scores/s", "seconds_per_block": per,
            "sample": (f"estimated scores + top-10 of 8 queries over {m} packed vectors (d=200, 3-bit, QJL); "
                       f"scores/s (per-score cost is independent of the corpus size)")}


def cpu_baseline(cfg: int, budget_s: float) -> dict:
    """The oracle timed on all host cores and on one core, same sample."""
    from threadpoolctl import threadpool_limits
    full = cpu_sample(cfg, budget_s)
    cores = blas_threads()
    with threadpool_limits(limits=1):
        one = cpu_sample(cfg, budget_s)
    out = {"value": full["value"], "unit": full["unit"], "cores": cores, "kind": "oracle",
           "sample": full["sample"], "value_1core": one["value"], "nproc": os.cpu_count(),
           "cpu_model": cpu_model(),
           "note": "fp64 NumPy oracle as it stands (not tuned); cores = BLAS threads; the rest of NumPy is one thread"}
    for k in ("seconds", "seconds_per_step", "seconds_per_head", "seconds_per_block"):
        if k in full:
            out[k] = full[k]
    return out


# ---------------------------------------------------------------------------
# Shared result skeleton.
# ---------------------------------------------------------------------------
def base_result(args, world, cfg, value, unit, ms_step, dtype, config, clk, launches):
    return {"metric": METRIC, "value": value, "unit": unit, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": dtype,
            "data": "synthetic (seeded; shapes and value laws of the workload; random orthogonal Pi, Gaussian S)",
            "config": dict({"workload": WORKLOADS[cfg], "config_id": cfg,
                            "parallelism": f"replicas x{world} (independent data per rank, no collective)"},
                           **config),
            "clocks": clk, "gpu_launches": launches}


class Timed:
    """Barrier + synchronize, clocks, launch count and CUDA events around a region."""

    def __init__(self, tq, world, dev):
        self.tq, self.world, self.dev = tq, world, dev

    def __enter__(self):
        self.clocks = ClockSampler(self.dev.index)
        barrier(self.world)
        torch.cuda.synchronize()
        self.n0 = self.tq.tq_kernel_launches()
        self.s, self.e = ev(), ev()
        self.s.record()
        return self

    def __exit__(self, *exc):
        self.e.record()
        torch.cuda.synchronize()
        self.launches = self.tq.tq_kernel_launches() - self.n0
        barrier(self.world)
        self.clk = self.clocks.stop()
        self.ms = self.s.elapsed_time(self.e)
        return False


# ---------------------------------------------------------------------------
# Config 1: tiny RoPE head (launch latency).
# ---------------------------------------------------------------------------
def run_c1(args, world, rank, tq):
    dev = torch.device("cuda", torch.cuda.current_device())
    th = synth.tiny_head(replica_seed(rank))
    d, n, nq = th.d, th.K.shape[0], th.Q.shape[0]
    lay = tq.layout(d, 3, 3)
    c, t, _ = tq.tq_make_codebook(d, 3, 0)
    cd, td = dev_tensor(c, dev), dev_tensor(t, dev)
    K, V, Q = dev_tensor(th.K, dev), dev_tensor(th.V, dev), dev_tensor(th.Q, dev).reshape(1, 1, nq, d)
    Pi, S = dev_tensor(th.Pi, dev), dev_tensor(th.S, dev)
    kpos = torch.as_tensor(th.k_pos, device=dev)
    qpos = torch.as_tensor(th.q_pos, device=dev)
    kp, vp = tq.alloc_planes(n, d, 3, True, dev), tq.alloc_planes(n, d, 3, False, dev)
    out = torch.empty((1, 1, nq, d), device=dev)
    ws = tq.decode_workspace(lay, 1, 1, 1, nq, n, dev)
    st = torch.zeros(1, dtype=torch.int32, device=dev)

    def step():
        tq.tq_quantize_kv(lay, True, K, kp, Pi, cd, td, S=S, positions=kpos, rope_base=th.rope_base, d_status=st)
        tq.tq_quantize_kv(lay, False, V, vp, Pi, cd, td, d_status=st)
        tq.tq_decode_attention(lay, Q, kp, vp, 1, n, Pi, Pi, S, cd, cd, out, ws, q_positions=qpos,
                               rope_base=th.rope_base, d_status=st)

    for _ in range(max(args.warmup, 3)):
        step()
    torch.cuda.synchronize()
    with Timed(tq, world, dev) as T:
        for _ in range(args.steps):
            step()
    assert int(st.item()) == 0, f"device status {int(st.item())}"
    ms = max_over_ranks(world, T.ms) / args.steps
    # The same three calls captured once into a CUDA graph and replayed.
    graph = {}
    try:
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            step()
        torch.cuda.current_stream().wait_stream(side)
        g = torch.cuda.CUDAGraph()
        n0 = tq.tq_kernel_launches()
        with torch.cuda.graph(g):
            step()
        captured = tq.tq_kernel_launches() - n0
        for _ in range(3):
            g.replay()
        torch.cuda.synchronize()
        s, e = ev(), ev()
        s.record()
        for _ in range(args.steps):
            g.replay()
        e.record()
        torch.cuda.synchronize()
        assert int(st.item()) == 0, f"device status {int(st.item())}"
        graph = {"us_per_step": 1e3 * s.elapsed_time(e) / args.steps, "kernels_per_step": captured}
    except Exception as exc:  # capture is reported, not required
        graph = {"error": str(exc).splitlines()[0][:200]}
    alg = n * (packed_bytes(d, 3, True) + packed_bytes(d, 3, False) + 2 * 4 * d)
    peaks = load_peaks()
    res = base_result(args, world, 1, world * n / (ms * 1e-3), "tokens/s", ms, "fp32 in, fp32 math, 3+1-bit cache",
                      {"head_dim": d, "tokens": n, "queries": nq, "rope_base": th.rope_base, "key_bits": 3,
                       "value_bits": 3, "qjl": True,
                       "l2": "the whole workload (≈0.2 MB) stays in L2: a latency measurement, not bandwidth"},
                      T.clk, T.launches)
    res["latency"] = {"eager_us_per_step": 1e3 * ms, "graph": graph,
                      "note": "one step = 3 library calls (RoPE+quantise keys, quantise values, RoPE+decode)"}
    res["roofline"] = hbm_roofline("whole step (quantize_kernel x2 + decode kernels)", alg, ms * 1e-3, peaks,
                                   "fp32 K and V in (256 B each) + packed out (36 B key, 28 B value) per token")
    res["roofline"]["note"] = "latency-bound: the step moves ~0.2 MB; the fraction is not a target here"
    e2e = None
    if not args.no_e2e:
        hK, hV, hQ = (t.cpu().pin_memory() for t in (K, V, Q))
        hout = torch.empty_like(out, device="cpu").pin_memory()

        def e2e_step():
            K.copy_(hK, non_blocking=True)
            V.copy_(hV, non_blocking=True)
            Q.copy_(hQ, non_blocking=True)
            step()
            hout.copy_(out, non_blocking=True)

        saved = args.e2e_steps
        args.e2e_steps = max(saved, 200)
        e2e = run_e2e_loop(args, world, e2e_step, n, "tokens/s", h2d=4 * (K.numel() + V.numel() + Q.numel()),
                           d2h=4 * out.numel())
        args.e2e_steps = saved
        e2e["note"] = "per step: fp32 K, V and queries copied in, attention outputs read back"
    return res, e2e


# ---------------------------------------------------------------------------
# Config 2: ESM-2-shaped cache, per-head rotations, full-sequence attention.
# ---------------------------------------------------------------------------
def esm_setup(tq, seed, dev):
    data = synth.esm_cache(seed)
    L, H, N, d = data.K.shape
    cK = data.calib_K.float().numpy()
    cV = data.calib_V.float().numpy()
    PiK = np.stack([tq.tq_fit_rotation(cK[l, h], data.Pi) for l in range(L) for h in range(H)])
    PiV = np.stack([tq.tq_fit_rotation(cV[l, h], data.Pi) for l in range(L) for h in range(H)])
    uk = np.concatenate([tq.tq_rotate_normalize(cK[l, h], PiK[l * H + h]).ravel() for l in range(L) for h in range(H)])
    uv = np.concatenate([tq.tq_rotate_normalize(cV[l, h], PiV[l * H + h]).ravel() for l in range(L) for h in range(H)])
    ck, tk, _ = tq.tq_make_codebook(d, 3, 1, uk)
    cv, tv, _ = tq.tq_make_codebook(d, 3, 1, uv)
    return data, PiK, PiV, (ck, tk), (cv, tv), (uk, uv)


def variants_c2(tq, data, PiK_h, PiV_h, books, samples, dev, layer=7):
    """Layout and correction variants on one layer of the ESM-shaped cache (untimed, evaluation only).

    Reconstructions (library kernels) against the bf16 inputs, scores q.k/sqrt(d) and softmax outputs of all
    1024 queries per head against fp32 attention on the inputs (torch, as the measuring stick):
      qjl        3-bit codes + QJL signs of S r + ||r|| (the configs' keys; tq_dequantize)
      sign_mean  3-bit codes + signs of r itself + ||x||, corrected by e_bar (TurboESM; S = I)
      plain      3-bit codes + ||x|| (the configs' values)
      b-1+1      TurboQuant's budget at b = 3: 2-bit codes + QJL (keys)
      shared     one table fitted on K and V samples pooled, instead of one each (dual)"""
    (ck, tk), (cv, tv) = books
    uk, uv = samples
    L, H, N, d = data.K.shape
    rows = slice(layer * H * N, (layer + 1) * H * N)
    n = H * N
    K = data.K.reshape(-1, d)[rows].to(dev)
    V = data.V.reshape(-1, d)[rows].to(dev)
    Q = data.Q[layer].to(dev).float()                                   # [H, N, d]
    PiK = torch.as_tensor(PiK_h[layer * H:(layer + 1) * H], device=dev).reshape(H * d, d).contiguous()
    PiV = torch.as_tensor(PiV_h[layer * H:(layer + 1) * H], device=dev).reshape(H * d, d).contiguous()
    S = torch.as_tensor(data.S, device=dev)
    eye = torch.eye(d, device=dev)
    lay3 = tq.layout(d, 3, 3)
    cs, ts, _ = tq.tq_make_codebook(d, 3, 1, np.concatenate([uk, uv]))
    ck2, tk2, _ = tq.tq_make_codebook(d, 2, 1, uk)
    e_k = tq.tq_residual_mean(uk, ck, tk, 3)
    e_v = tq.tq_residual_mean(uv, cv, tv, 3)
    T = lambda a: torch.as_tensor(np.ascontiguousarray(a), device=dev, dtype=torch.float32)

    def quant(x, Pi, c, t, bits, Sm):
        lay = tq.layout(d, bits, bits)
        p = tq.alloc_planes(n, d, bits, Sm is not None, dev)
        tq.tq_quantize_kv(lay, Sm is not None, x, p, Pi, T(c), T(t), S=Sm, vectors_per_pi=N, pi_stride=d * d)
        return lay, p

    def deq(lay, p, Pi, c, mode, e=0.0):
        o = torch.empty((n, d), device=dev)
        if mode == "qjl":
            tq.tq_dequantize(lay, True, p, n, Pi, T(c), o, S=S, vectors_per_pi=N, pi_stride=d * d)
        elif mode == "sign_mean":
            tq.tq_dequantize_sign_mean(lay, True, p, n, Pi, T(c), e, o, vectors_per_pi=N, pi_stride=d * d)
        else:
            tq.tq_dequantize(lay, False, p, n, Pi, T(c), o, vectors_per_pi=N, pi_stride=d * d)
        return o

    lk, pk = quant(K, PiK, ck, tk, 3, S)
    lki, pki = quant(K, PiK, ck, tk, 3, eye)
    lvi, pvi = quant(V, PiV, cv, tv, 3, eye)
    lk2, pk2 = quant(K, PiK, ck2, tk2, 2, S)
    lks, pks = quant(K, PiK, cs, ts, 3, None)
    lvs, pvs = quant(V, PiV, cs, ts, 3, None)
    rec = {
        "K": {"plain": deq(lk, pk, PiK, ck, "plain"), "qjl": deq(lk, pk, PiK, ck, "qjl"),
              "sign_mean": deq(lki, pki, PiK, ck, "sign_mean", e_k), "b-1+1": deq(lk2, pk2, PiK, ck2, "qjl"),
              "plain_shared": deq(lks, pks, PiK, cs, "plain")},
        "V": {"plain": deq(lvi, pvi, PiV, cv, "plain"), "sign_mean": deq(lvi, pvi, PiV, cv, "sign_mean", e_v),
              "plain_shared": deq(lvs, pvs, PiV, cs, "plain")},
    }
    torch.cuda.synchronize()
    Kf, Vf = K.float(), V.float()

    def snr(x, y):
        return float(10 * torch.log10((x * x).sum() / ((x - y) ** 2).sum()))

    out = {"e_bar": {"K": e_k, "V": e_v}, "snr_db": {t_: {m: snr(Kf if t_ == "K" else Vf, r) for m, r in rec[t_].items()}
                                                   for t_ in rec}}
    out["dual_vs_shared_db"] = {"K": out["snr_db"]["K"]["plain"] - out["snr_db"]["K"]["plain_shared"],
                                "V": out["snr_db"]["V"]["plain"] - out["snr_db"]["V"]["plain_shared"]}
    Kh, Vh = Kf.reshape(H, N, d), Vf.reshape(H, N, d)
    s_exact = torch.einsum("hqd,hkd->hqk", Q, Kh) / np.sqrt(d)
    o_exact = torch.softmax(s_exact, -1) @ Vh
    errs = {}
    for kname, vname in (("qjl", "plain"), ("sign_mean", "sign_mean"), ("b-1+1", "plain"), ("plain", "plain")):
        s_a = torch.einsum("hqd,hkd->hqk", Q, rec["K"][kname].reshape(H, N, d)) / np.sqrt(d)
        ds = s_a - s_exact
        o_a = torch.softmax(s_a, -1) @ rec["V"][vname].reshape(H, N, d)
        cos = torch.nn.functional.cosine_similarity(o_a, o_exact, dim=-1)
        errs[f"K {kname} / V {vname}"] = {"score_err_rel_rms": float(ds.pow(2).mean().sqrt() / s_exact.pow(2).mean().sqrt()),
                                          "score_err_mean": float(ds.mean()), "out_cos_mean": float(cos.mean()),
                                          "out_cos_min": float(cos.min())}
        del s_a, ds, o_a
    out["attention_vs_fp32"] = errs
    from_bytes = lambda kb, vb: L * H * N * (kb + vb)
    fp32 = L * H * N * 2 * d * 4
    kq = d * 3 // 8 + (d + 31) // 32 * 4 + 8
    layouts = {"configs (K codes+QJL signs+2 norms, V codes+norm)": (kq, d * 3 // 8 + 4),
               "TurboESM sign+e_bar (K and V codes+signs+norm)": (d * 3 // 8 + d // 8 + 4, d * 3 // 8 + d // 8 + 4),
               "TurboQuant (b-1)+1 at b=3 (K 2-bit+QJL, V 3-bit)": (d * 2 // 8 + (d + 31) // 32 * 4 + 8, d * 3 // 8 + 4)}
    out["layouts"] = {k: {"bytes_per_token_head": kb + vb, "MiB": from_bytes(kb, vb) / 2 ** 20,
                          "ratio_vs_fp32": fp32 / from_bytes(kb, vb)} for k, (kb, vb) in layouts.items()}
    out["fp32_MiB"] = fp32 / 2 ** 20
    out["layer"] = layer
    return out


def run_c2(args, world, rank, tq):
    dev = torch.device("cuda", torch.cuda.current_device())
    data, PiK_h, PiV_h, (ck, tk), (cv, tv), calib_u = esm_setup(tq, replica_seed(rank), dev)
    L, H, N, d = data.K.shape
    n = L * H * N
    lay = tq.layout(d, 3, 3)
    K = data.K.reshape(n, d).to(dev)
    V = data.V.reshape(n, d).to(dev)
    Q = data.Q.reshape(L, 1, H, N, d).to(dev)
    PiK, PiV = dev_tensor(PiK_h, dev), dev_tensor(PiV_h, dev)
    S = dev_tensor(data.S, dev)
    cKd, tKd, cVd, tVd = (dev_tensor(x, dev) for x in (ck, tk, cv, tv))
    kp, vp = tq.alloc_planes(n, d, 3, True, dev), tq.alloc_planes(n, d, 3, False, dev)
    out = torch.empty((L, 1, H, N, d), dtype=torch.bfloat16, device=dev)
    ws = tq.decode_workspace(lay, 1, H, H, N, N, dev)
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    kps = [kp.rows(l * H * N, (l + 1) * H * N) for l in range(L)]
    vps = [vp.rows(l * H * N, (l + 1) * H * N) for l in range(L)]

    def step(evs=None):
        if evs:
            evs[0].record()
        tq.tq_quantize_kv(lay, True, K, kp, PiK, cKd, tKd, S=S, vectors_per_pi=N, pi_stride=d * d, d_status=st)
        if evs:
            evs[1].record()
        tq.tq_quantize_kv(lay, False, V, vp, PiV, cVd, tVd, vectors_per_pi=N, pi_stride=d * d, d_status=st)
        if evs:
            evs[2].record()
        for l in range(L):
            tq.tq_decode_attention(lay, Q[l], kps[l], vps[l], H, N, PiK[l * H:(l + 1) * H], PiV[l * H:(l + 1) * H],
                                   S, cKd, cVd, out[l], ws, pi_stride=d * d, d_status=st)
        if evs:
            evs[3].record()

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    marks = [[ev() for _ in range(4)] for _ in range(args.steps)]
    with Timed(tq, world, dev) as T:
        for s in range(args.steps):
            step(marks[s])
    assert int(st.item()) == 0, f"device status {int(st.item())}"
    ms = max_over_ranks(world, T.ms) / args.steps
    kq_ms = statistics.mean(m[0].elapsed_time(m[1]) for m in marks)
    vq_ms = statistics.mean(m[1].elapsed_time(m[2]) for m in marks)
    at_ms = statistics.mean(m[2].elapsed_time(m[3]) for m in marks)
    pairs = L * H * N * N
    # Attention work per (query, key) pair at head_dim d, in FP32 lane ops:
    # d adds of the per-coordinate code table, d/4 adds of the sign-nibble
    # table, d FMAs of the value accumulation, 4 for scale/max/exp/sum.
    ops_pair = d + d // 4 + d + 4
    peaks = load_peaks()
    kb, vb = 2 * d + packed_bytes(d, 3, True), 2 * d + packed_bytes(d, 3, False)
    res = base_result(args, world, 2, world * N / (ms * 1e-3), "tokens/s", ms, "bf16 in, fp32 math, 3+1-bit cache",
                      {"layers": L, "heads": H, "head_dim": d, "seq": N, "batch": 1, "key_bits": 3, "value_bits": 3,
                       "qjl": True, "rotation": "per-head Pi_rand V_h^T (SVD of 256 calibration tokens)",
                       "codebooks": "dual empirical Lloyd (keys, values)",
                       "l2": "bf16 K/V (173 MB) read per step exceed the 126 MB L2; no flush"},
                      T.clk, T.launches)
    res["phases"] = {
        "quantize": {"key_call_us": 1e3 * kq_ms, "value_call_us": 1e3 * vq_ms,
                     "tokens_per_s": N / ((kq_ms + vq_ms) * 1e-3),
                     "vectors_per_s": 2 * n / ((kq_ms + vq_ms) * 1e-3),
                     "algorithmic_gbs": n * (kb + vb) / ((kq_ms + vq_ms) * 1e-3) / 1e9},
        "attention": {"ms": at_ms, "pairs_per_s": pairs / (at_ms * 1e-3), "calls": L,
                      "pairs": pairs},
    }
    att = alu_roofline("tq_decode_attention (1024 queries per head): decode_prologue + decode_main_v2<64> + "
                       "decode_combine, per layer", pairs * ops_pair, at_ms * 1e-3, T.clk,
                       f"{ops_pair} FP32 lane ops per (query, key) pair at d={d}; {pairs:,} pairs per step")
    quant = hbm_roofline("tq_quantize_kv(keys, per-head Pi): quantize_tc_kernel<64,key,3,per-head> + quantize_fixup",
                         n * kb, kq_ms * 1e-3, peaks,
                         f"bf16 in {2 * d} B + packed out {packed_bytes(d, 3, True)} B per key vector; {n:,} per call")
    quant_v = hbm_roofline("tq_quantize_kv(values, per-head Pi): quantize_tc_kernel<64,value,3,per-head> + "
                           "quantize_fixup", n * vb, vq_ms * 1e-3, peaks,
                           f"bf16 in {2 * d} B + packed out {packed_bytes(d, 3, False)} B per value vector")
    if at_ms >= kq_ms + vq_ms:
        res["roofline"], res["roofline_quantize"], res["roofline_quantize_value"] = att, quant, quant_v
    else:
        res["roofline"], res["roofline_attention"], res["roofline_quantize_value"] = quant, att, quant_v
    res["variants"] = variants_c2(tq, data, PiK_h, PiV_h, ((ck, tk), (cv, tv)), calib_u, dev)
    e2e = None
    if not args.no_e2e:
        hK = K.cpu().pin_memory()
        hV = V.cpu().pin_memory()
        hQ = Q.cpu().pin_memory()
        hout = torch.empty_like(out, device="cpu").pin_memory()

        def e2e_step():
            K.copy_(hK, non_blocking=True)
            V.copy_(hV, non_blocking=True)
            Q.copy_(hQ, non_blocking=True)
            step()
            hout.copy_(out, non_blocking=True)

        e2e = run_e2e_loop(args, world, e2e_step, N, "tokens/s",
                           h2d=hK.numel() * 2 + hV.numel() * 2 + hQ.numel() * 2, d2h=hout.numel() * 2)
    return res, e2e


# ---------------------------------------------------------------------------
# Config 3: Llama-3.1-8B-shaped decode (the headline line).
# ---------------------------------------------------------------------------
def run_c3(args, world, rank, tq):
    dev = torch.device("cuda", torch.cuda.current_device())
    shape = synth.LlamaDecodeShape(n_ctx=args.context)
    L = args.layers
    B, HQ, HKV, D, N = shape.batch, shape.hq, shape.hkv, shape.d, shape.n_ctx
    n_vec = B * HKV * N
    lay = tq.layout(D, 3, 3)
    c, t, _ = tq.tq_make_codebook(D, 3, 0)
    cd = torch.as_tensor(c, device=dev)
    td = torch.as_tensor(t, device=dev)
    Pi = torch.as_tensor(synth.random_rotation(D, 0), device=dev)
    S = torch.as_tensor(synth.gaussian_projection(D, 0), device=dev)
    seed = replica_seed(rank)
    K = [synth.llama_layer_kv(shape, seed, l, dev, "K").reshape(n_vec, D) for l in range(L)]
    V = [synth.llama_layer_kv(shape, seed, l, dev, "V").reshape(n_vec, D) for l in range(L)]
    Q = synth.llama_queries(shape, seed, dev)[:L].reshape(L, B, HQ, 1, D).contiguous()
    kp = [tq.alloc_planes(n_vec, D, 3, True, dev) for _ in range(L)]
    vp = [tq.alloc_planes(n_vec, D, 3, False, dev) for _ in range(L)]
    out = torch.empty((L, B, HQ, 1, D), dtype=torch.bfloat16, device=dev)
    ws = tq.decode_workspace(lay, B, HQ, HKV, 1, N, dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)

    def step(e=None):
        # e: events [K start, K end = V start, V end] per layer, then decode
        # boundaries (L + 1), all on the launching stream.
        for l in range(L):
            if e is not None:
                e[3 * l].record()
            tq.tq_quantize_kv(lay, True, K[l], kp[l], Pi, cd, td, S=S, d_status=status)
            if e is not None:
                e[3 * l + 1].record()
            tq.tq_quantize_kv(lay, False, V[l], vp[l], Pi, cd, td, d_status=status)
            if e is not None:
                e[3 * l + 2].record()
        for l in range(L):
            if e is not None:
                e[3 * L + l].record()
            tq.tq_decode_attention(lay, Q[l], kp[l], vp[l], HKV, N, Pi, Pi, S, cd, cd, out[l], ws, d_status=status)
        if e is not None:
            e[4 * L].record()

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    assert int(status.item()) == 0, f"device status {int(status.item())}"
    marks = [[ev() for _ in range(4 * L + 1)] for _ in range(args.steps)]
    with Timed(tq, world, dev) as T:
        for s in range(args.steps):
            step(marks[s])
    assert int(status.item()) == 0, f"device status {int(status.item())}"
    n_calls = args.steps * L
    k_ms = sum(e[3 * l].elapsed_time(e[3 * l + 1]) for e in marks for l in range(L)) / n_calls
    v_ms = sum(e[3 * l + 1].elapsed_time(e[3 * l + 2]) for e in marks for l in range(L)) / n_calls
    dl_ms = sum(e[3 * L + l].elapsed_time(e[3 * L + l + 1]) for e in marks for l in range(L)) / n_calls
    q_ms = sum(e[0].elapsed_time(e[3 * L - 1]) for e in marks) / args.steps
    d_ms = sum(e[3 * L].elapsed_time(e[4 * L]) for e in marks) / args.steps
    ms_step = max_over_ranks(world, T.ms) / args.steps

    tokens_step = B * N * L / shape.layers
    keys_scored_step = L * B * HQ * N
    k_bytes = 2 * D + packed_bytes(D, 3, True)
    v_bytes = 2 * D + packed_bytes(D, 3, False)
    dec_unit = packed_bytes(D, 3, True) + packed_bytes(D, 3, False)
    peaks = load_peaks()
    res = base_result(args, world, 3, world * tokens_step / (ms_step * 1e-3), "tokens/s", ms_step,
                      "bf16 in, fp32 math, 3+1-bit cache",
                      {"layers": L, "batch": B, "hq": HQ, "hkv": HKV, "head_dim": D, "context": N, "key_bits": 3,
                       "value_bits": 3, "qjl": True,
                       "l2": "inputs (34 GB) and packed cache (8.3 GB) per step exceed the 126 MB L2; no flush"},
                      T.clk, T.launches)
    res["phases"] = {
        "quantize": {"ms": q_ms, "tokens_per_s": tokens_step / (q_ms * 1e-3),
                     "token_heads_per_s": 2 * L * n_vec / (q_ms * 1e-3),
                     "algorithmic_gbs": L * n_vec * (k_bytes + v_bytes) / (q_ms * 1e-3) / 1e9,
                     "key_call_us": 1e3 * k_ms, "value_call_us": 1e3 * v_ms},
        "decode": {"ms": d_ms, "keys_scored_per_s": keys_scored_step / (d_ms * 1e-3),
                   "algorithmic_gbs": L * n_vec * dec_unit / (d_ms * 1e-3) / 1e9, "call_us": 1e3 * dl_ms},
    }
    # The dominant call of the step: tq_quantize_kv of one layer's keys.
    res["roofline"] = hbm_roofline("tq_quantize_kv(keys): quantize_tc_kernel<128,key,3> + quantize_fixup",
                                   n_vec * k_bytes, k_ms * 1e-3, peaks,
                                   f"bf16 in 256 B + packed out {packed_bytes(D, 3, True)} B per key vector; "
                                   f"{n_vec:,} vectors per call", "quantize_tc_key3_d128", n_vec)
    res["roofline_value"] = hbm_roofline("tq_quantize_kv(values): quantize_tc_kernel<128,value,3> + quantize_fixup",
                                         n_vec * v_bytes, v_ms * 1e-3, peaks,
                                         f"bf16 in 256 B + packed out {packed_bytes(D, 3, False)} B per value "
                                         f"vector; {n_vec:,} per call", "quantize_tc_value3_d128", n_vec)
    res["roofline_decode"] = hbm_roofline("tq_decode_attention: decode_qprep_kernel + decode_fused_kernel<3>",
                                          n_vec * dec_unit, dl_ms * 1e-3, peaks,
                                          f"{dec_unit} B per (token, kv head); {n_vec:,} per call",
                                          "decode_fused3_d128", n_vec)
    if args.incremental_steps > 0:
        res["incremental"] = run_incremental_c3(args, tq, lay, Q, kp, vp, out, ws, Pi, S, cd, td, status, shape,
                                                world, L, dev)
    e2e = None
    if not args.no_e2e:
        e2e = run_e2e_c3(args, tq, lay, K, V, Q, kp, vp, out, ws, Pi, S, cd, td, status, shape, world)
    return res, e2e


def run_incremental_c3(args, tq, lay, Q, kp, vp, out, ws, Pi, S, cd, td, status, shape, world, L, dev):
    """One generated token per step: every layer appends one key (RoPE at its position) and one value per
    (batch, kv head) stream with tq_append_kv, then decodes over the grown cache. The cache holds N - T tokens
    before the first of T steps (its capacity, ctx_stride, stays N)."""
    B, HKV, D, N = shape.batch, shape.hkv, shape.d, shape.n_ctx
    T = args.incremental_steps
    streams = B * HKV
    base = 500000.0                                # Llama-3.1 RoPE base
    g = torch.Generator(device=dev)
    g.manual_seed(1234)
    kn = torch.randn((T, L, streams, D), generator=g, device=dev).to(torch.bfloat16)
    vn = torch.randn((T, L, streams, D), generator=g, device=dev).to(torch.bfloat16)
    slots = [N - T + i for i in range(T)]
    kpos = [torch.full((streams,), sl, dtype=torch.int32, device=dev) for sl in slots]
    qpos = [torch.full((B, 1), sl, dtype=torch.int32, device=dev) for sl in slots]
    marks = [(ev(), ev(), ev()) for _ in range(T)]
    barrier(world)
    torch.cuda.synchronize()
    n0 = tq.tq_kernel_launches()
    for i, sl in enumerate(slots):
        marks[i][0].record()
        for l in range(L):
            tq.tq_append_kv(lay, True, kn[i, l], kp[l], N, sl, Pi, cd, td, S=S, positions=kpos[i], rope_base=base,
                            d_status=status)
            tq.tq_append_kv(lay, False, vn[i, l], vp[l], N, sl, Pi, cd, td, d_status=status)
            if l == 0:
                marks[i][1].record()
            tq.tq_decode_attention(lay, Q[l], kp[l], vp[l], HKV, sl + 1, Pi, Pi, S, cd, cd, out[l], ws,
                                   q_positions=qpos[i], rope_base=base, ctx_stride=N, d_status=status)
        marks[i][2].record()
    torch.cuda.synchronize()
    launches = tq.tq_kernel_launches() - n0
    assert int(status.item()) == 0, f"device status {int(status.item())}"
    per_token = max_over_ranks(world, statistics.mean(m[0].elapsed_time(m[2]) for m in marks))
    append_l0 = statistics.mean(m[0].elapsed_time(m[1]) for m in marks)

    # The same steps, each captured once as a CUDA graph (the host's launch
    # cost leaves the timed region), replayed in order.
    def one_step(i, sl):
        for l in range(L):
            tq.tq_append_kv(lay, True, kn[i, l], kp[l], N, sl, Pi, cd, td, S=S, positions=kpos[i], rope_base=base,
                            d_status=status)
            tq.tq_append_kv(lay, False, vn[i, l], vp[l], N, sl, Pi, cd, td, d_status=status)
            tq.tq_decode_attention(lay, Q[l], kp[l], vp[l], HKV, sl + 1, Pi, Pi, S, cd, cd, out[l], ws,
                                   q_positions=qpos[i], rope_base=base, ctx_stride=N, d_status=status)

    graph = {}
    try:
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        graphs = []
        with torch.cuda.stream(side):
            for i, sl in enumerate(slots):
                g = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g, stream=side):
                    one_step(i, sl)
                graphs.append(g)
            ga = torch.cuda.CUDAGraph()                # 100 appends of one layer's 64 keys
            with torch.cuda.graph(ga, stream=side):
                for _ in range(100):
                    tq.tq_append_kv(lay, True, kn[0, 0], kp[0], N, slots[0], Pi, cd, td, S=S, positions=kpos[0],
                                    rope_base=base, d_status=status)
        torch.cuda.current_stream().wait_stream(side)
        torch.cuda.synchronize()
        barrier(world)
        s0, s1 = ev(), ev()
        s0.record()
        for g in graphs:
            g.replay()
        s1.record()
        torch.cuda.synchronize()
        a0, a1 = ev(), ev()
        a0.record()
        ga.replay()
        a1.record()
        torch.cuda.synchronize()
        assert int(status.item()) == 0, f"device status {int(status.item())}"
        g_tok = max_over_ranks(world, s0.elapsed_time(s1) / T)
        graph = {"us_per_generated_token": 1e3 * g_tok, "tokens_per_s": world * B / (g_tok * 1e-3),
                 "append_call_us": 1e3 * a0.elapsed_time(a1) / 100}
        del graphs, ga
    except Exception as exc:  # capture is reported, not required
        graph = {"error": str(exc).splitlines()[0][:200]}
    barrier(world)
    return {"us_per_generated_token": 1e3 * per_token, "tokens_per_s": world * B / (per_token * 1e-3),
            "layers": L, "steps": T, "append_us_layer0": 1e3 * append_l0, "gpu_launches": launches,
            "graph": graph,
            "note": (f"per step and layer: tq_append_kv of {streams} keys (RoPE) and {streams} values at slot "
                     f"N-{T}+i, then tq_decode_attention over slot+1 tokens (ctx_stride {N}); eager launches from "
                     f"Python, and each step replayed from a CUDA graph; tokens_per_s counts the batch's {B} "
                     f"sequences")}


def run_e2e_c3(args, tq, lay, K, V, Q, kp, vp, out, ws, Pi, S, cd, td, status, shape, world):
    """The same step through the public API with host inputs: per step the pinned host K/V of every layer are
    copied to the device (copy stream, overlapped with the previous layer's quantisation), and the
    attention outputs are read back."""
    import psutil
    L = len(K)
    per_layer = 2 * K[0].numel() * K[0].element_size()
    avail = psutil.virtual_memory().available
    # Pinned host copies of up to 30% of the free host memory, shared by the
    # ranks of this node (each takes its 1/world part).
    pool = max(1, min(L, int(0.3 / world * avail // per_layer)))
    hostK = [torch.empty_like(K[i], device="cpu").pin_memory() for i in range(pool)]
    hostV = [torch.empty_like(V[i], device="cpu").pin_memory() for i in range(pool)]
    for i in range(pool):
        hostK[i].copy_(K[i])
        hostV[i].copy_(V[i])
    host_out = torch.empty_like(out, device="cpu").pin_memory()
    comp = torch.cuda.current_stream()
    copy = torch.cuda.Stream()
    done = [torch.cuda.Event() for _ in range(L)]
    ready = [torch.cuda.Event() for _ in range(L)]
    HKV, N = shape.hkv, shape.n_ctx

    def step():
        for l in range(L):
            copy.wait_event(done[l])
            with torch.cuda.stream(copy):
                K[l].copy_(hostK[l % pool], non_blocking=True)
                V[l].copy_(hostV[l % pool], non_blocking=True)
            ready[l].record(copy)
        for l in range(L):
            comp.wait_event(ready[l])
            tq.tq_quantize_kv(lay, True, K[l], kp[l], Pi, cd, td, S=S, d_status=status)
            tq.tq_quantize_kv(lay, False, V[l], vp[l], Pi, cd, td, d_status=status)
            done[l].record(comp)
        for l in range(L):
            tq.tq_decode_attention(lay, Q[l], kp[l], vp[l], HKV, N, Pi, Pi, S, cd, cd, out[l], ws, d_status=status)
        host_out.copy_(out, non_blocking=True)

    for l in range(L):
        done[l].record(comp)
    tokens = shape.batch * N * L / shape.layers
    res = run_e2e_loop(args, world, step, tokens, "tokens/s", h2d=int(L * per_layer),
                       d2h=int(out.numel() * out.element_size()))
    res["host_pool_layers"] = pool
    return res


def run_e2e_loop(args, world, step, units, unit, h2d, d2h):
    step()
    torch.cuda.synchronize()
    steps = max(1, args.e2e_steps)
    barrier(world)
    torch.cuda.synchronize()
    s0, s1 = ev(), ev()
    s0.record()
    for _ in range(steps):
        step()
    s1.record()
    torch.cuda.synchronize()
    barrier(world)
    ms = max_over_ranks(world, s0.elapsed_time(s1)) / steps
    return {"value": world * units / (ms * 1e-3), "unit": unit, "ms_per_step": ms, "steps": steps,
            "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h)}


# ---------------------------------------------------------------------------
# Config 4: long context, key bits 2/3/4.
# ---------------------------------------------------------------------------
def run_c4(args, world, rank, tq):
    dev = torch.device("cuda", torch.cuda.current_device())
    lc = synth.long_context(replica_seed(rank), device=dev)
    _, hkv, n, d = lc.K.shape
    hq = lc.Q.shape[1]
    G = hq // hkv
    bits_list = (2, 3, 4)
    K = lc.K.reshape(-1, d)
    V = lc.V.reshape(-1, d)
    nv = K.shape[0]
    Pi, S = dev_tensor(lc.Pi, dev), dev_tensor(lc.S, dev)
    cv, tv, _ = tq.tq_make_codebook(d, 3, 0)
    cVd, tVd = dev_tensor(cv, dev), dev_tensor(tv, dev)
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    books, kps, lays = {}, {}, {}
    vp = tq.alloc_planes(nv, d, 3, False, dev)
    tq.tq_quantize_kv(tq.layout(d, 3, 3), False, V, vp, Pi, cVd, tVd, d_status=st)
    for b in bits_list:
        c, t, _ = tq.tq_make_codebook(d, b, 0)
        books[b] = (dev_tensor(c, dev), dev_tensor(t, dev))
        lays[b] = tq.layout(d, b, 3)
        kps[b] = tq.alloc_planes(nv, d, b, True, dev)
    q = lc.Q.reshape(1, hq, 1, d).contiguous()
    out = torch.empty((1, hq, 1, d), dtype=torch.bfloat16, device=dev)
    ws = tq.decode_workspace(lays[4], 1, hq, hkv, 1, n, dev)
    flush = L2Flush(dev)

    def quantize_keys(b):
        tq.tq_quantize_kv(lays[b], True, K, kps[b], Pi, books[b][0], books[b][1], S=S, d_status=st)

    def decode(b, scores=None):
        tq.tq_decode_attention(lays[b], q, kps[b], vp, hkv, n, Pi, Pi, S, books[b][0], cVd, out, ws,
                               scores_out=scores, d_status=st)

    # Key quantisation per bit width (timed once each, cold L2; not part of the step).
    qt = {}
    for b in bits_list:
        quantize_keys(b)
        flush()
        s, e = ev(), ev()
        s.record()
        quantize_keys(b)
        e.record()
        torch.cuda.synchronize()
        qt[b] = s.elapsed_time(e)
    for _ in range(args.warmup):
        for b in bits_list:
            decode(b)
    torch.cuda.synchronize()
    marks = [[(ev(), ev()) for _ in bits_list] for _ in range(args.steps)]
    with Timed(tq, world, dev) as T:
        for s in range(args.steps):
            for j, b in enumerate(bits_list):
                flush()
                marks[s][j][0].record()
                decode(b)
                marks[s][j][1].record()
    assert int(st.item()) == 0, f"device status {int(st.item())}"
    launches = T.launches
    call_ms = {b: statistics.mean(m[j][0].elapsed_time(m[j][1]) for m in marks) for j, b in enumerate(bits_list)}
    ms_step = max_over_ranks(world, sum(call_ms.values()))
    keys_call = hq * n
    # Score error of each bit width against exact q.k/sqrt(d) (fp32 from the bf16 inputs).
    Kf = lc.K[0].float()                                              # [hkv, n, d]
    qf = lc.Q[0].float()                                              # [hq, d]
    exact = torch.einsum("hgd,hnd->hgn", qf.reshape(hkv, G, d), Kf).reshape(hq, n) / math.sqrt(d)
    sc = torch.empty((1, hq, 1, n), device=dev)
    peaks = load_peaks()
    per_bits = {}
    for b in bits_list:
        decode(b, sc)
        torch.cuda.synchronize()
        err = sc[0, :, 0] - exact
        unit = packed_bytes(d, b, True) + packed_bytes(d, 3, False)
        ms = call_ms[b]
        per_bits[str(b)] = {
            "decode_call_us": 1e3 * ms, "keys_scored_per_s": keys_call / (ms * 1e-3),
            "algorithmic_gbs": nv * unit / (ms * 1e-3) / 1e9,
            "hbm_frac": nv * unit / (ms * 1e-3) / 1e9 / peaks["hbm_gbs"], "bytes_per_token_head": unit,
            "key_quantize_us": 1e3 * qt[b],
            "key_quantize_gbs": nv * (2 * d + packed_bytes(d, b, True)) / (qt[b] * 1e-3) / 1e9,
            "score_err_rms": float(err.pow(2).mean().sqrt()), "score_err_max": float(err.abs().max()),
            "score_rms": float(exact.pow(2).mean().sqrt()),
            "score_err_rel_rms": float(err.pow(2).mean().sqrt() / exact.pow(2).mean().sqrt()),
        }
    unit3 = packed_bytes(d, 3, True) + packed_bytes(d, 3, False)
    res = base_result(args, world, 4, world * len(bits_list) * keys_call / (ms_step * 1e-3), "keys scored/s",
                      ms_step, "bf16 in, fp32 math, {2,3,4}+1-bit keys, 3-bit values",
                      {"layers": 1, "batch": 1, "hq": hq, "hkv": hkv, "head_dim": d, "context": n,
                       "key_bits": list(bits_list), "value_bits": 3, "qjl": True,
                       "step": "one decode call per key bit width (3 calls)",
                       "l2": "L2 flushed (384 MiB write) before every timed call; only the calls are timed"},
                      T.clk, launches)
    res["per_key_bits"] = per_bits
    res["score_error_reference"] = "exact q.k/sqrt(d) in fp32 from the same bf16 inputs (torch matmul)"
    res["roofline"] = hbm_roofline("tq_decode_attention (key bits 3): decode_qprep_kernel + decode_fused_kernel<3>",
                                   nv * unit3, call_ms[3] * 1e-3, peaks,
                                   f"{unit3} B per (token, kv head); {nv:,} per call", "decode_fused3_d128", nv)
    e2e = None
    if not args.no_e2e:
        hK, hV = K.cpu().pin_memory(), V.cpu().pin_memory()
        hq_ = q.cpu().pin_memory()
        hout = torch.empty((len(bits_list),) + tuple(out.shape), dtype=out.dtype).pin_memory()

        def e2e_step():
            K.copy_(hK, non_blocking=True)
            V.copy_(hV, non_blocking=True)
            q.copy_(hq_, non_blocking=True)
            tq.tq_quantize_kv(tq.layout(d, 3, 3), False, V, vp, Pi, cVd, tVd, d_status=st)
            for j, b in enumerate(bits_list):
                quantize_keys(b)
                decode(b)
                hout[j].copy_(out, non_blocking=True)

        e2e = run_e2e_loop(args, world, e2e_step, len(bits_list) * keys_call, "keys scored/s",
                           h2d=2 * K.numel() * 2 + q.numel() * 2, d2h=hout.numel() * 2)
        e2e["note"] = "per step: K/V bf16 copied in, values + keys at 3 bit widths quantised, 3 decode calls"
    return res, e2e


# ---------------------------------------------------------------------------
# Config 5: vector search over compressed codes.
# ---------------------------------------------------------------------------
def exact_top10(Xd, Qd, k=10, block=65536):
    best_s = best_i = None
    for s0 in range(0, Xd.shape[0], block):
        sc = Qd @ Xd[s0:s0 + block].T
        ts, ti = torch.topk(sc, k, dim=1)
        ti = ti + s0
        if best_s is None:
            best_s, best_i = ts, ti
        else:
            cs, ci = torch.cat([best_s, ts], 1), torch.cat([best_i, ti], 1)
            best_s, o = torch.topk(cs, k, dim=1)
            best_i = torch.gather(ci, 1, o)
    return best_i


def run_c5(args, world, rank, tq):
    dev = torch.device("cuda", torch.cuda.current_device())
    corpus = synth.search_corpus(replica_seed(rank))
    X, Qh, d = corpus.X, corpus.Q, corpus.d
    n_db, nq, k = X.shape[0], Qh.shape[0], 10
    lay = tq.layout(d, 3, 3)
    c, t, _ = tq.tq_make_codebook(d, 3, 0)
    cd, td = dev_tensor(c, dev), dev_tensor(t, dev)
    Pi, S = dev_tensor(corpus.Pi, dev), dev_tensor(corpus.S, dev)
    Xd, Qd = dev_tensor(X, dev), dev_tensor(Qh, dev)
    planes = tq.alloc_planes(n_db, d, 3, True, dev)
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    flush = L2Flush(dev)
    # Index build (quantise the corpus), timed once with a cold L2.
    tq.tq_quantize_kv(lay, True, Xd, planes, Pi, cd, td, S=S, d_status=st)
    flush()
    s, e = ev(), ev()
    s.record()
    tq.tq_quantize_kv(lay, True, Xd, planes, Pi, cd, td, S=S, d_status=st)
    e.record()
    torch.cuda.synchronize()
    build_ms = s.elapsed_time(e)
    top_i = torch.empty((nq, k), dtype=torch.int64, device=dev)
    top_s = torch.empty((nq, k), dtype=torch.float32, device=dev)
    ws = torch.empty(tq.tq_search_workspace_bytes(lay, nq, n_db, k) + 256, dtype=torch.uint8, device=dev)

    def search():
        tq.tq_search_topk(lay, Qd, planes, n_db, Pi, S, cd, k, top_i, top_s, ws)

    for _ in range(args.warmup):
        search()
    torch.cuda.synchronize()
    marks = [(ev(), ev()) for _ in range(args.steps)]
    with Timed(tq, world, dev) as T:
        for m in marks:
            flush()
            m[0].record()
            search()
            m[1].record()
    assert int(st.item()) == 0, f"device status {int(st.item())}"
    ms_step = max_over_ranks(world, statistics.mean(m[0].elapsed_time(m[1]) for m in marks))
    scores = nq * n_db
    prev = torch.backends.cuda.matmul.allow_tf32
    torch.backends.cuda.matmul.allow_tf32 = False
    exact = exact_top10(Xd, Qd, k).cpu().numpy()
    torch.backends.cuda.matmul.allow_tf32 = prev
    got = top_i.cpu().numpy()
    recall = float(np.mean([len(set(a.tolist()) & set(b.tolist())) for a, b in zip(got, exact)]) / k)
    # The pages' measure, recall 1@k: how often the true best inner product
    # is among the first k estimated results (one untimed call with k = 32).
    k32 = 32
    ti32 = torch.empty((nq, k32), dtype=torch.int64, device=dev)
    ts32 = torch.empty((nq, k32), dtype=torch.float32, device=dev)
    ws32 = torch.empty(tq.tq_search_workspace_bytes(lay, nq, n_db, k32) + 256, dtype=torch.uint8, device=dev)
    tq.tq_search_topk(lay, Qd, planes, n_db, Pi, S, cd, k32, ti32, ts32, ws32)
    g32 = ti32.cpu().numpy()
    assert np.array_equal(g32[:, :k], got), "top-10 is the head of top-32"
    one_at = {str(kk): float(np.mean([exact[r, 0] in g32[r, :kk] for r in range(nq)])) for kk in (1, 2, 4, 8, 16, 32)}
    # Work per estimated score at head_dim d, in FP32 lane ops: d adds of the
    # per-coordinate code table, d/4 adds of the sign-nibble table, 2 for the
    # norm-weighted combination.
    ops_score = d + d // 4 + 2
    peaks = load_peaks()
    res = base_result(args, world, 5, world * scores / (ms_step * 1e-3), "scores/s", ms_step,
                      "fp32 in, fp32 math, 3+1-bit codes",
                      {"n_db": n_db, "n_queries": nq, "d": d, "k": k, "bits": 3, "qjl": True,
                       "step": "top-10 of all 10,000 queries over the whole corpus (one tq_search_topk call)",
                       "l2": "L2 flushed (384 MiB write) before every timed call; only the calls are timed"},
                      T.clk, T.launches)
    res["recall_at_10"] = recall
    res["recall_1_at_k"] = one_at
    res["recall_reference"] = "exact fp32 inner-product top-10 of all 10,000 queries (torch matmul, TF32 off)"
    res["index_build"] = {"quantize_us": 1e3 * build_ms, "vectors_per_s": n_db / (build_ms * 1e-3),
                          "roofline": hbm_roofline("tq_quantize_kv(d=200 fp32 keys): quantize_kernel<200>",
                                                   n_db * (4 * d + packed_bytes(d, 3, True)), build_ms * 1e-3,
                                                   peaks, f"fp32 in {4 * d} B + packed out "
                                                          f"{packed_bytes(d, 3, True)} B per vector")}
    res["roofline"] = alu_roofline("tq_search_topk: search_prologue + search_main<200> + search_merge",
                                   scores * ops_score, ms_step * 1e-3, T.clk,
                                   f"{ops_score} FP32 lane ops per estimated score at d={d}; {scores:,} per call")
    e2e = None
    if not args.no_e2e:
        hQ = Qd.cpu().pin_memory()
        hi = torch.empty_like(top_i, device="cpu").pin_memory()
        hs = torch.empty_like(top_s, device="cpu").pin_memory()

        def e2e_step():
            Qd.copy_(hQ, non_blocking=True)
            search()
            hi.copy_(top_i, non_blocking=True)
            hs.copy_(top_s, non_blocking=True)

        e2e = run_e2e_loop(args, world, e2e_step, scores, "scores/s", h2d=hQ.numel() * 4,
                           d2h=hi.numel() * 8 + hs.numel() * 4)
        e2e["note"] = "queries copied in and top-10 ids/scores read back per step; the packed index stays resident"
    return res, e2e


RUNNERS = {1: run_c1, 2: run_c2, 3: run_c3, 4: run_c4, 5: run_c5}


# ---------------------------------------------------------------------------
# Reference arm: the oracle on the host cores.
# ---------------------------------------------------------------------------
def run_reference(args, world):
    cfg = args.config
    per = min(args.cpu_budget, max(1.0, min(20.0, 60.0 / max(1, args.steps + args.warmup))))
    for _ in range(args.warmup):
        cpu_sample(cfg, per)
    vals, last = [], None
    t0 = time.perf_counter()
    for _ in range(args.steps):
        last = cpu_sample(cfg, per)
        vals.append(last["value"])
    wall = time.perf_counter() - t0
    v = statistics.median(vals)
    cb = {"value": v, "unit": last["unit"], "cores": blas_threads(), "kind": "oracle", "sample": last["sample"],
          "cpu_model": cpu_model(), "nproc": os.cpu_count()}
    return {"impl": "reference", "metric": METRIC, "value": v, "unit": last["unit"], "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * wall / max(1, args.steps),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded)",
            "config": {"workload": WORKLOADS[cfg], "config_id": cfg, "sample": "bounded per step"},
            "cpu_baseline": cb, "e2e": {"value": v, "unit": last["unit"], "h2d_bytes_per_step": 0,
                                        "d2h_bytes_per_step": 0}}


def main(argv=None):
    args = parse(argv)
    launch_or_check(args, argv)
    if args.impl == "reference":
        # Every rank joins the group once (the launch check); rank 0 alone
        # then runs the oracle and prints, the others exit without work.
        world, rank, _ = dist_setup(args, timeout_s=120.0)
        barrier(world)
        if world > 1:
            world = torch.distributed.get_world_size()
            torch.distributed.destroy_process_group()
        if rank == 0:
            print(json.dumps(run_reference(args, world)), flush=True)
        return
    import kv_cache_vector_rope_b200 as tq
    if not torch.cuda.is_available():
        sys.exit("bench.py: the CUDA path needs a GPU (use --impl reference for the oracle on the host)")
    world, rank, _ = dist_setup(args)
    res, e2e = RUNNERS[args.config](args, world, rank, tq)
    if e2e is not None:
        res["e2e"] = e2e
    if rank == 0 and not args.no_cpu:
        res["cpu_baseline"] = cpu_baseline(args.config, args.cpu_budget)
    if rank == 0:
        print(json.dumps(res), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
