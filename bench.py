"""Benchmark of one decode step: paged KV-cache write + paged GQA decode attention.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

A step is the whole hot path over one batch: the cache write of this step's
new K/V (one token per sequence, at position L_b - 1) followed by decode
attention over every sequence's paged context, split-KV partitions and their
log-sum-exp merge included. Inputs are seeded synthetic tensors shaped like
the Qwen2.5 serving workloads ("rvLLM 소개" (discuss.pytorch.kr),
§PagedAttention과 FlashAttention-3 and §H100 SXM 80GB 직접 엔진 벤치마크),
resident in HBM before timing. The K timed steps are replayed from CUDA
graphs, as the serving engine replays its decode step (same page, §CUDA
그래프 리플레이); consecutive steps read different replicas of the KV pool, and
the replicas together are larger than the L2 cache, so no step finds its KV
in L2.

The headline workload is the largest single-GPU one at the pages' f16
precision: Qwen2.5-7B-shaped, B=128, 28/4 heads, contexts U[512, 4096], with
the 128-token cache write fused into the step. The same line carries the
other decode workloads (FP8 E4M3 cache, Qwen2.5-1.5B-shaped, and the skewed
long-context batch at 512-token partitions and under the balanced plan), each
with its own roofline, and the standalone cache write.

Metric: algorithmic HBM bytes of the step (KV + Q + O + block tables +
lengths for attention, plus the cache write's reads and writes) per second of
step time, GB/s; `seq_steps_per_s` is batch * steps / time. One JSON line on
rank 0. Under torchrun every rank runs its own batch (weak scaling, no
collective on the data path); time is the max over ranks.

--impl reference times the float64 CPU oracle on the host cores on a bounded
sample of the same workload (there is no other implementation of this path to
compare with).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads as W  # noqa: E402

METRIC = "paged GQA decode attn: KV-read GB/s (% of B200 HBM peak), seq-steps/s"
FALLBACK_HBM_GBS = 6650.0
L2_BYTES = 126 * 2 ** 20
PROFILE_SUMMARY = os.path.join(ROOT, "profiles", "decode_attention_traffic.json")
# the largest single-GPU decode workload at f16, and the others reported beside it (partition -1 is
# the balanced plan, P > 0 fixed partitions of P tokens)
HEADLINE = "qwen2.5-7b"
SUBLINES = (("fp8-e4m3", -1), ("qwen2.5-1.5b", -1), ("skewed-split", 512), ("skewed-split", -1))


# ------------------------------------------------------------------ byte model
def kv_bytes(lens, kv_heads, head_dim, elem_bytes) -> int:
    """K and V bytes one decode step must read: each cached token once per KV head."""
    return int(sum(2 * int(L) * kv_heads * head_dim * elem_bytes for L in lens))


def attention_bytes(lens, Hq, Hkv, D, elem_bytes, block_size) -> int:
    """KV + Q (f16 read) + out (f16 write) + block-table entries + context lengths."""
    lens = [int(L) for L in lens]
    tables = sum(4 * (-(-L // block_size)) for L in lens)
    return kv_bytes(lens, Hkv, D, elem_bytes) + 2 * len(lens) * Hq * D * 2 + tables + 4 * len(lens)


def cache_write_bytes(T, Hkv, D, elem_bytes) -> int:
    """New K/V read (f16) + cache rows written + slots read."""
    return T * Hkv * D * 2 * 2 + T * Hkv * D * elem_bytes * 2 + 8 * T


def step_bytes(w, lens, n_new):
    e = 1 if w.kv_dtype == "fp8" else 2
    a = attention_bytes(lens, w.Hq, w.Hkv, w.head_dim, e, w.block_size)
    return a, cache_write_bytes(n_new, w.Hkv, w.head_dim, e)


DECODE_SOURCES = ("cache_write.cuh", "decode_attention.cuh", "decode_balanced.cuh", "decode_page.cuh",
                  "pkv_device.cuh")


def kernel_source_digest() -> str:
    """Hash of what the decode kernels are built from: their device headers and the launch-shape
    constants in pagedkv.cu (worker warps, ring slots). Other kernels of the library do not enter."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "paged_kv_decode_gqa_b200", "csrc")
    for name in DECODE_SOURCES:
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(name.encode() + f.read())
    with open(os.path.join(csrc, "pagedkv.cu"), "rb") as f:
        for line in f:
            if b"PKV_BAL_" in line or b"constexpr int kStages" in line or b"constexpr int kConsumers" in line:
                h.update(line)
    return h.hexdigest()[:16]


def measured_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return json.load(f), "measured"
    except (OSError, ValueError):
        return {"hbm_gbs": FALLBACK_HBM_GBS}, "fallback"


def recorded_traffic(workload: str, partition: int):
    """ncu DRAM bytes per attention launch recorded for this kernel source, else None."""
    try:
        with open(PROFILE_SUMMARY) as f:
            rec = json.load(f)
    except (OSError, ValueError):
        return None
    for r in rec.get("captures", []):
        if (r.get("workload") == workload and r.get("partition_tokens") == partition
                and r.get("source_digest") == kernel_source_digest()):
            return r.get("dram_bytes_per_launch")
    return None


# -------------------------------------------------------------------- clocks
class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML in a thread."""

    REASONS = {
        "gpu_idle": 0x1, "applications_clocks_setting": 0x2, "sw_power_cap": 0x4,
        "hw_slowdown": 0x8, "sync_boost": 0x10, "sw_thermal_slowdown": 0x20,
        "hw_thermal_slowdown": 0x40, "hw_power_brake_slowdown": 0x80,
    }

    def __init__(self, device_index: int, period_s: float = 0.005):
        self.samples, self.period, self._stop = [], period_s, threading.Event()
        self.ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # pragma: no cover - no NVML
            self.err = str(e)

    def _run(self):
        while not self._stop.is_set():
            try:
                mhz = self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM)
                rs = self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                self.samples.append((time.perf_counter(), mhz, rs))
            except Exception:
                pass
            time.sleep(self.period)

    def start(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def stop(self):
        if self.ok:
            self._stop.set()
            self.t.join()

    def summary(self, t0: float, t1: float):
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "note": "NVML unavailable"}
        inside = [s for s in self.samples if t0 <= s[0] <= t1]
        note = "sampled during the timed region"
        if not inside:                          # timed region shorter than a sample period
            inside = sorted(self.samples, key=lambda s: min(abs(s[0] - t0), abs(s[0] - t1)))[:3]
            note = "nearest samples to a timed region shorter than the sampling period"
        reasons = set()
        for _, _, rs in inside:
            for name, bit in self.REASONS.items():
                if rs & bit and name != "gpu_idle":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(s[1] for s in inside) if inside else None,
                "sm_max_mhz": self.max_mhz, "reasons": sorted(reasons), "samples": len(inside),
                "note": note}


# ---------------------------------------------------------------- distributed
def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def reduce_max(value: float, world: int, device=None) -> float:
    if world == 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_gbs(world: int, bytes_per_rank_step: int, steps: int, elapsed_max_ms: float) -> float:
    """Throughput of all ranks (weak scaling: every rank does the same work) over the slowest rank."""
    return world * bytes_per_rank_step * steps / (elapsed_max_ms * 1e-3) / 1e9


def barrier(world: int, device=None):
    if world > 1:
        import torch.distributed as dist
        if device is not None:
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


# -------------------------------------------------------------- CPU baseline
def time_oracle(w, x, budget_s: float, max_reps: int = 10_000):
    """Whole steps of the oracle (cache write + attention) on the host cores."""
    import oracle
    fp8 = w.kv_dtype == "fp8"
    if fp8:
        kc = oracle.quantize_e4m3(x["k_pool"], float(x["k_scale"]))
        vc = oracle.quantize_e4m3(x["v_pool"], float(x["v_scale"]))
    else:
        kc, vc = x["k_pool"].copy(), x["v_pool"].copy()
    reps, t0 = 0, time.perf_counter()
    while reps < max_reps:
        oracle.paged_kv_cache_write(x["k_new"], x["v_new"], kc, vc, x["slot_mapping"],
                                    kv_dtype=w.kv_dtype, k_scale=float(x["k_scale"]),
                                    v_scale=float(x["v_scale"]))
        oracle.paged_gqa_decode(x["q"], kc, vc, x["block_tables"], x["context_lens"],
                                float(x["softmax_scale"]), kv_dtype=w.kv_dtype,
                                k_scale=float(x["k_scale"]), v_scale=float(x["v_scale"]),
                                partition_tokens=w.partition_tokens)
        reps += 1
        if time.perf_counter() - t0 >= budget_s:
            break
    return reps, time.perf_counter() - t0, oracle.num_threads()


def oracle_sample(w, x, max_seqs: int):
    """The first `max_seqs` sequences of the workload (same pool and lengths)."""
    n = min(w.B, max_seqs)
    xs = dict(x)
    for k in ("q", "block_tables", "context_lens", "k_new", "v_new", "slot_mapping"):
        xs[k] = x[k][:n]
    return xs, n


# ---------------------------------------------------------------------- main
def qkv_bytes(T: int, H: int, N: int, bias: bool) -> int:
    """Algorithmic bytes of one fused add + RMSNorm + QKV launch: W once, x and residual in,
    residual_out and q|k|v out, gamma and bias."""
    return 2 * (N * H + 3 * T * H + T * N + H + (N if bias else 0))


def time_qkv_projection(w, device, stream, peak, seed=0):
    """fused_add_rmsnorm_qkv at the workload's model shape (H = Hq * D) for its batch, from a CUDA
    graph that rotates over enough weight replicas that W is read from HBM every launch."""
    import torch

    import paged_kv_decode_gqa_b200 as pkv
    Hq, Hkv, D, T = w.Hq, w.Hkv, w.head_dim, w.B
    H, N = Hq * D, (Hq + 2 * Hkv) * D
    d = W.make_qkv_inputs(T, H, Hq, Hkv, D, seed)
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(device)
    x, r, g, b = t(d["x"]), t(d["residual"]), t(d["gamma"]), t(d["bias"])
    w0 = t(d["w_qkv"])
    R = max(2, min(64, -(-2 * L2_BYTES // (N * H * 2))))
    ws = [w0] + [w0.clone() for _ in range(R - 1)]
    res = torch.empty((T, H), dtype=torch.float16, device=device)
    q = torch.empty((T, Hq, D), dtype=torch.float16, device=device)
    kn = torch.empty((T, Hkv, D), dtype=torch.float16, device=device)
    vn = torch.empty((T, Hkv, D), dtype=torch.float16, device=device)
    call = lambda wi: pkv.fused_add_rmsnorm_qkv(x, r, g, wi, b, res, q, kn, vn, eps=W.RMS_EPS,
                                                flags=pkv.PKV_STEP_OVERLAP_PREVIOUS, stream=stream)
    with torch.cuda.stream(stream):
        for wi in ws[:3]:
            call(wi)
        stream.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=stream):
            for wi in ws:
                call(wi)
        for _ in range(3):
            graph.replay()
        reps = max(1, 2000 // R)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(reps):
            graph.replay()
        e1.record(stream)
    torch.cuda.synchronize()
    us = e0.elapsed_time(e1) * 1000 / (reps * R)
    nbytes = qkv_bytes(T, H, N, True)
    del graph
    return {"what": "fused_add_rmsnorm_qkv (residual add + RMSNorm + QKV projection, q/k/v out)",
            "T": T, "H": H, "N": N, "bias": True, "algorithmic_bytes": nbytes, "us": us,
            "achieved": nbytes / us / 1e3, "peak": peak, "unit": "GB/s", "frac": nbytes / us / 1e3 / peak,
            "bound": "hbm", "launches": reps * R, "plan": pkv.fused_add_rmsnorm_qkv_plan(T, H, Hq, Hkv, D),
            "l2": f"{R} weight replicas rotated ({R * N * H * 2 / 2**20:.0f} MiB), graph of {R} launches, "
                  "PKV_STEP_OVERLAP_PREVIOUS"}


def prefill_flops(lens, n_new, Hq, D) -> int:
    """Attention FLOPs of a chunked prefill: per query at position p, 2 D (p + 1) for the logits
    and as many for the weighted values, per query head."""
    total = 0
    for L, n in zip(lens, n_new):
        pos = np.arange(int(L) - int(n), int(L), dtype=np.int64)
        total += int(4 * D * Hq * (pos + 1).sum())
    return total


def time_prefill(w, device, stream, peak_tflops, seed=0):
    """paged_gqa_prefill_attention at the workload's head shape: 8 sequences append 512 tokens each
    to contexts of 2048 (f16 cache), timed over back-to-back launches."""
    import torch

    import paged_kv_decode_gqa_b200 as pkv
    B, n_new, L = 8, 512, 2048
    pw = W.with_sizes(w, B=B, num_blocks=B * L // w.block_size + 64, ctx=("fixed", (L,) * B), kv_dtype="f16")
    x = W.make_inputs(pw, seed, poison=False)
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(device)
    qs = np.arange(0, (B + 1) * n_new, n_new, dtype=np.int32)
    q = (np.random.default_rng(seed).standard_normal((B * n_new, w.Hq, w.head_dim), dtype=np.float32)
         .astype(np.float16))
    qd, kc, vc, bt, cl, qsd = t(q), t(x["k_pool"]), t(x["v_pool"]), t(x["block_tables"]), t(x["context_lens"]), t(qs)
    out = torch.empty_like(qd)
    ws = torch.zeros(pkv.paged_gqa_prefill_workspace_size(w.Hq, w.Hkv, w.head_dim), dtype=torch.uint8,
                     device=device)
    reps = 20

    def timed(workspace):
        call = lambda: pkv.paged_gqa_prefill_attention(out, qd, kc, vc, bt, cl, qsd, max_query_len=n_new,
                                                       max_context_len=L, softmax_scale=float(x["softmax_scale"]),
                                                       workspace=workspace, stream=stream)
        with torch.cuda.stream(stream):
            for _ in range(3):
                call()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            for _ in range(reps):
                call()
            e1.record(stream)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) * 1000 / reps

    us_items = timed(None)                 # whole items, no workspace
    us = timed(ws)                         # the load-balanced schedule (items cut at CTA boundaries)
    flops = prefill_flops([L] * B, [n_new] * B, w.Hq, w.head_dim)
    tflops = flops / us / 1e6
    return {"what": "paged_gqa_prefill_attention (chunked prefill, f16 cache, load-balanced schedule)", "B": B,
            "new_tokens": n_new, "context": L, "Hq": w.Hq, "Hkv": w.Hkv, "flops": flops, "us": us,
            "achieved": tflops, "peak": peak_tflops, "unit": "TFLOP/s", "frac": tflops / peak_tflops,
            "bound": "tensor", "us_whole_items": us_items, "frac_whole_items": flops / us_items / 1e6 / peak_tflops,
            "launches": reps, "l2": "cache of 8 x 2048 tokens re-read by every chunk; L2-resident after the first"}


def parse_args(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--workload", default=HEADLINE, choices=sorted(W.WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--partition", type=int, default=-1,
                    help="split-KV plan: -1 the library's balanced plan (default), 0 single pass, "
                         "P > 0 fixed partitions of P tokens")
    ap.add_argument("--graph-steps", type=int, default=500, help="steps per captured CUDA graph")
    ap.add_argument("--no-overlap", action="store_true",
                    help="fused step without PKV_STEP_OVERLAP_PREVIOUS")
    ap.add_argument("--unfused", action="store_true",
                    help="two launches per step (cache write, then attention) instead of the fused step")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-prefill", action="store_true",
                    help="skip timing the chunked prefill attention at the workload's head shape")
    ap.add_argument("--no-qkv", action="store_true",
                    help="skip timing the fused add + RMSNorm + QKV projection at the workload's shape")
    ap.add_argument("--no-sublines", action="store_true",
                    help="skip the other decode workloads (FP8, 1.5B, skewed at 512-token partitions and "
                         "under the balanced plan) and the standalone cache write")
    ap.add_argument("--sub-steps", type=int, default=200, help="timed steps of each other workload")
    ap.add_argument("--fp8-scales", default="tensor", choices=["tensor", "per-head"],
                    help="FP8 workloads: per-tensor host scales, or per-KV-head scales computed on the "
                         "device and passed to the device-scale entry points")
    ap.add_argument("--kv-read-ratio", action="store_true",
                    help="only compare the grouped decode kernel with per-query-head launches on the "
                         "workload (one launch of each, then timed repeats): the KV bytes the grouping "
                         "saves, for an ncu capture of dram__bytes_read")
    ap.add_argument("--cpu-baseline-s", type=float, default=10.0)
    ap.add_argument("--seed", type=int, default=0)
    return ap.parse_args(argv)


def run_reference(args):
    world, rank, _ = dist_setup()
    if rank != 0:
        return 0
    w = W.WORKLOADS[args.workload]
    x = W.make_inputs(w, args.seed)
    # bounded sample: enough sequences for about a second of oracle work per step
    xs, n = oracle_sample(w, x, max_seqs={"qwen2.5-1.5b": 64, "qwen2.5-7b": 16, "fp8-e4m3": 8,
                                           "skewed-split": 8, "tiny": 2}.get(w.name, 8))
    # keep the whole K-step run within about two minutes: shrink the sample if needed
    _, t1, _ = time_oracle(w, xs, budget_s=0.0, max_reps=1)
    if t1 * (args.steps + args.warmup) > 120.0 and n > 1:
        n = max(1, int(n * 120.0 / (t1 * (args.steps + args.warmup))))
        xs, n = oracle_sample(w, x, max_seqs=n)
    wa, wc = step_bytes(w, xs["context_lens"], n)
    time_oracle(w, xs, budget_s=0.0, max_reps=max(args.warmup, 1))
    reps, secs, cores = time_oracle(w, xs, budget_s=1e9, max_reps=args.steps)
    value = (wa + wc) * reps / secs / 1e9
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world,
        "steps": reps, "warmup": args.warmup, "ms_per_step": secs / reps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "seq_steps_per_s": n * reps / secs,
        "config": {"workload": w.name, "sample": f"first {n} of {w.B} sequences, whole steps",
                   "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "head_dim": w.head_dim,
                   "block_size": w.block_size, "kv_dtype": w.kv_dtype},
        "cpu_baseline": {"value": value, "unit": "GB/s", "cores": cores, "kind": "oracle",
                         "sample": f"first {n} of {w.B} sequences of {w.name}, {reps} whole steps"},
        "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line))
    return 0


# A spin of about 0.5 ms queued in front of every timed region: the GPU is busy
# while the host enqueues the timed graph replays, so the region measures the
# steps on the device and not the host's submission latency.
LEAD_IN_CYCLES = 1_000_000


def lead_in(stream):
    import torch
    with torch.cuda.stream(stream):
        torch.cuda._sleep(LEAD_IN_CYCLES)


class StepBench:
    """One decode workload resident on the device, and the library calls of its step.

    The step is the whole hot path over the batch: this step's new K/V written at
    position L_b - 1 of every sequence, then decode attention over the paged
    contexts. With the balanced plan (partition -1) it is one fused launch
    (paged_gqa_decode_step); with fixed partitions, or `unfused`, it is
    paged_kv_cache_write followed by paged_gqa_decode_attention.

    The KV pool is replicated R times and step i uses replica i % R, so that the
    KV touched between two reads of one replica is at least 4x the L2 size; with
    the overlap flag R >= 2, so that the launch before a step never writes the
    pages that step reads before its grid-dependency wait (the flag's promise).
    """

    def __init__(self, w, device, stream, seed, partition, *, unfused=False, overlap=True,
                 fp8_scales="tensor"):
        import torch

        import paged_kv_decode_gqa_b200 as pkv
        self.torch, self.pkv = torch, pkv
        self.w, self.device, self.stream, self.P = w, device, stream, partition
        x = W.make_inputs(w, seed)
        self.x = x
        lens = x["context_lens"]
        B, Hq, Hkv, D, bs = w.B, w.Hq, w.Hkv, w.head_dim, w.block_size
        self.B = B
        self.max_len = int(lens.max())
        self.fp8 = fp8 = w.kv_dtype == "fp8"
        self.attn_b, self.cw_b = step_bytes(w, lens, B)
        self.step_b = self.attn_b + self.cw_b
        self.fused = not unfused and partition == pkv.PKV_PARTITION_AUTO
        self.flags = pkv.PKV_STEP_OVERLAP_PREVIOUS if (overlap and self.fused) else 0
        t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(device)
        self.t = t
        self.q, self.bt, self.cl = t(x["q"]), t(x["block_tables"]), t(x["context_lens"])
        self.k_new, self.v_new, self.slots = t(x["k_new"]), t(x["v_new"]), t(x["slot_mapping"])
        self.ks, self.vs, self.scale = float(x["k_scale"]), float(x["v_scale"]), float(x["softmax_scale"])

        self.touched = kv_bytes(lens, Hkv, D, 1 if fp8 else 2)
        R = max(1, min(16, -(-4 * L2_BYTES // max(self.touched, 1))))
        if self.flags:
            R = max(R, 2)
        self.R = R
        k16, v16 = t(x["k_pool"]), t(x["v_pool"])
        self.per_head = fp8 and fp8_scales == "per-head"
        self.scales_kernel = None
        if fp8:                                    # quantise the pool with the library's cache write
            kq = torch.empty(k16.shape, dtype=torch.uint8, device=device)
            vq = torch.empty_like(kq)
            n_rows = w.num_blocks * bs
            rows_k, rows_v = k16.view(n_rows, Hkv, D), v16.view(n_rows, Hkv, D)
            all_slots = torch.arange(n_rows, dtype=torch.int64, device=device)
            if self.per_head:
                # per-KV-head scales computed on the device from the pool (its free rows are NaN
                # and do not count); the scales kernel is timed over the K pool
                self.ks_t = torch.empty(Hkv, dtype=torch.float32, device=device)
                self.vs_t = torch.empty(Hkv, dtype=torch.float32, device=device)
                for _ in range(3):
                    pkv.paged_kv_fp8_scales(rows_k, self.ks_t, per_head=True, stream=stream)
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                reps = 10
                e0.record(stream)
                for _ in range(reps):
                    pkv.paged_kv_fp8_scales(rows_k, self.ks_t, per_head=True, stream=stream)
                e1.record(stream)
                pkv.paged_kv_fp8_scales(rows_v, self.vs_t, per_head=True, stream=stream)
                torch.cuda.synchronize()
                us = e0.elapsed_time(e1) * 1000 / reps
                nbytes = rows_k.numel() * 2
                self.scales_kernel = {
                    "input_bytes": nbytes, "us": us, "gbs": nbytes / us / 1e3,
                    "what": "paged_kv_fp8_scales, per KV head, over the f16 K pool (memset + 2 launches)"}
                pkv.paged_kv_cache_write_fp8_scaled(rows_k, rows_v, kq, vq, all_slots, self.ks_t, self.vs_t,
                                                    stream=stream)
            else:
                pkv.paged_kv_cache_write(rows_k, rows_v, kq, vq, all_slots, kv_dtype="fp8", k_scale=self.ks,
                                         v_scale=self.vs, stream=stream)
            base_k, base_v = kq, vq
            del k16, v16, rows_k, rows_v
        else:
            base_k, base_v = k16, v16
        self.pools = [(base_k, base_v)] + [(base_k.clone(), base_v.clone()) for _ in range(R - 1)]
        ws_n = pkv.paged_gqa_decode_workspace_size(B, Hq, Hkv, D, self.max_len, partition)
        self.ws = torch.zeros(max(ws_n, 256), dtype=torch.uint8, device=device)
        self.out = torch.empty((B, Hq, D), dtype=torch.float16, device=device)
        torch.cuda.synchronize()

    # ---- the library calls of one step: per-tensor scales or per-KV-head device scales ----
    def write_call(self, kn, vn, kc, vc, sl):
        if self.per_head:
            self.pkv.paged_kv_cache_write_fp8_scaled(kn, vn, kc, vc, sl, self.ks_t, self.vs_t, stream=self.stream)
        else:
            self.pkv.paged_kv_cache_write(kn, vn, kc, vc, sl, kv_dtype=self.w.kv_dtype, k_scale=self.ks,
                                          v_scale=self.vs, stream=self.stream)

    def step_call(self, qq, kn, vn, kc, vc, bb, cc, flags):
        if self.per_head:
            self.pkv.paged_gqa_decode_step_fp8_scaled(self.out, qq, kn, vn, kc, vc, bb, cc, self.ks_t, self.vs_t,
                                                      max_context_len=self.max_len, softmax_scale=self.scale,
                                                      workspace=self.ws, flags=flags, stream=self.stream)
        else:
            self.pkv.paged_gqa_decode_step(self.out, qq, kn, vn, kc, vc, bb, cc, max_context_len=self.max_len,
                                           softmax_scale=self.scale, kv_dtype=self.w.kv_dtype, k_scale=self.ks,
                                           v_scale=self.vs, workspace=self.ws, flags=flags, stream=self.stream)

    def attention_call(self, qq, kc, vc, bb, cc):
        if self.per_head:
            self.pkv.paged_gqa_decode_attention_fp8_scaled(self.out, qq, kc, vc, bb, cc, self.ks_t, self.vs_t,
                                                           max_context_len=self.max_len, softmax_scale=self.scale,
                                                           partition_tokens=self.P, workspace=self.ws,
                                                           stream=self.stream)
        else:
            self.pkv.paged_gqa_decode_attention(self.out, qq, kc, vc, bb, cc, max_context_len=self.max_len,
                                                softmax_scale=self.scale, kv_dtype=self.w.kv_dtype,
                                                k_scale=self.ks, v_scale=self.vs, partition_tokens=self.P,
                                                workspace=self.ws, stream=self.stream)

    def step(self, i, events=None):
        """Step i on pool replica i % R; `events` = (before, after) the attention launch."""
        kc, vc = self.pools[i % self.R]
        if self.fused:
            self.step_call(self.q, self.k_new, self.v_new, kc, vc, self.bt, self.cl, self.flags)
            return
        self.write_call(self.k_new, self.v_new, kc, vc, self.slots)
        if events:
            events[0].record(self.stream)
        self.attention_call(self.q, kc, vc, self.bt, self.cl)
        if events:
            events[1].record(self.stream)

    @property
    def launches_per_step(self):
        return 1 if self.fused else 2

    def warmup(self, n):
        for i in range(n):
            self.step(i)
        self.torch.cuda.synchronize()

    def time(self, K, graph_steps, world=1, sampler=None):
        """Times exactly K steps replayed from CUDA graphs. Returns the device time of the region
        (max over ranks), the attention kernel's mean launch duration and the host wall clock.

        Graphs hold a multiple of R steps, so consecutive steps always use different replicas.
        Fused: one launch per step and nothing between launches, so each launch overlaps the
        previous one's tail (programmatic dependent launch); the kernel's average duration is the
        region over K. Unfused: events around every attention launch give its own duration."""
        torch = self.torch
        S = max(1, min(graph_steps, K))
        S = max(self.R, S - S % self.R)
        chunks = [S] * (K // S) + ([K % S] if K % S else [])
        graphs = {}
        for n in sorted(set(chunks)):
            evs = [] if self.fused else [(torch.cuda.Event(enable_timing=True, external=True),
                                          torch.cuda.Event(enable_timing=True, external=True)) for _ in range(n)]
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=self.stream):
                for i in range(n):
                    self.step(i, evs[i] if evs else None)
            graphs[n] = (g, evs)
        torch.cuda.synchronize()
        start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier(world, self.device)
        torch.cuda.synchronize()
        if sampler:
            sampler.start()
        lead_in(self.stream)
        wall0 = time.perf_counter()
        start.record(self.stream)
        for n in chunks:
            graphs[n][0].replay()
        end.record(self.stream)
        torch.cuda.synchronize()
        wall1 = time.perf_counter()
        if sampler:
            sampler.stop()
        barrier(world, self.device)
        elapsed_ms = start.elapsed_time(end)
        if self.fused:
            attn_ms = elapsed_ms / K
        else:        # per-launch durations of the attention kernel in the last replay of each graph
            d = [a.elapsed_time(b) for n in set(chunks) for a, b in graphs[n][1]]
            attn_ms = sum(d) / len(d)
        del graphs
        return {"elapsed_ms": reduce_max(elapsed_ms, world, self.device), "attn_ms": attn_ms,
                "wall": (wall0, wall1), "graph_steps": S, "replays": len(chunks)}

    def e2e(self, n_steps, world=1):
        """The same step through the public API on pinned host buffers: every step copies its
        inputs host to device, runs, copies the output back and waits for it."""
        torch = self.torch
        x = self.x
        h = {k: torch.from_numpy(np.ascontiguousarray(x[k])).pin_memory()
             for k in ("q", "k_new", "v_new", "slot_mapping", "block_tables", "context_lens")}
        d = {k: torch.empty(v.shape, dtype=v.dtype, device=self.device) for k, v in h.items()}
        out_h = torch.empty(tuple(self.out.shape), dtype=torch.float16).pin_memory()
        h2d = sum(v.numel() * v.element_size() for v in h.values())
        d2h = out_h.numel() * out_h.element_size()

        def one(i):
            for k in h:
                d[k].copy_(h[k], non_blocking=True)
            kc, vc = self.pools[i % self.R]
            if self.fused:
                self.step_call(d["q"], d["k_new"], d["v_new"], kc, vc, d["block_tables"], d["context_lens"], 0)
            else:
                self.write_call(d["k_new"], d["v_new"], kc, vc, d["slot_mapping"])
                self.attention_call(d["q"], kc, vc, d["block_tables"], d["context_lens"])
            out_h.copy_(self.out, non_blocking=True)
            self.stream.synchronize()

        with torch.cuda.stream(self.stream):
            for i in range(3):
                one(i)
            barrier(world, self.device)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(self.stream)
            for i in range(n_steps):
                one(i)
            e1.record(self.stream)
        torch.cuda.synchronize()
        ms = reduce_max(e0.elapsed_time(e1), world, self.device)
        return {"value": world * self.step_b * n_steps / (ms * 1e-3) / 1e9, "unit": "GB/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": n_steps,
                "ms_per_step": ms / n_steps, "note": "eager calls, one host sync per step"}

    def describe(self):
        s = ("one fused launch (cache write + attention)" +
             (", PKV_STEP_OVERLAP_PREVIOUS" if self.flags else "")) if self.fused \
            else "cache write + attention launches"
        return {"step": s,
                "l2": f"inputs larger than L2: {self.R} KV pool replicas rotated, "
                      f"{self.R * self.touched / 2**20:.0f} MiB touched per cycle"}


def kernel_line(sb, timing, peak, peak_src):
    """Roofline of the step's dominant kernel: algorithmic bytes per launch over its mean duration."""
    kern_b = sb.step_b if sb.fused else sb.attn_b      # the fused launch also does the cache write
    achieved = kern_b / (timing["attn_ms"] * 1e-3) / 1e9
    return {"bound": "hbm",
            "kernel": "decode_balanced_kernel (fused step)" if sb.fused else "decode attention",
            "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
            "peak_source": f"{peak_src} hbm_gbs", "traffic": recorded_traffic(sb.w.name, sb.P),
            "algorithmic_bytes_per_launch": kern_b, "mean_launch_us": timing["attn_ms"] * 1e3}


def time_subline(name, partition, device, stream, peak, peak_src, steps, seed, fp8_scales):
    """One other decode workload: its own step, timed like the headline's, as a sub-object."""
    import torch
    w = W.WORKLOADS[name]
    sb = StepBench(w, device, stream, seed, partition, fp8_scales=fp8_scales)
    sb.warmup(5)
    tm = sb.time(steps, 500)
    roof = kernel_line(sb, tm, peak, peak_src)
    res = {"workload": name, "partition_tokens": partition, **sb.describe(),
           "steps": steps, "us_per_step": tm["elapsed_ms"] * 1e3 / steps,
           "value": sb.step_b * steps / (tm["elapsed_ms"] * 1e-3) / 1e9, "unit": "GB/s",
           "seq_steps_per_s": w.B * steps / (tm["elapsed_ms"] * 1e-3),
           "us": roof["mean_launch_us"], "achieved": roof["achieved"], "frac": roof["frac"],
           "algorithmic_bytes_per_launch": roof["algorithmic_bytes_per_launch"], "traffic": roof["traffic"],
           "kernel": roof["kernel"], "gpu_launches": sb.launches_per_step * steps}
    del sb
    torch.cuda.empty_cache()
    return res


def time_cache_write(w, device, stream, peak, seed=0, reps=200):
    """paged_kv_cache_write alone at the workload's shape (one new token per sequence), from a
    CUDA graph of `reps` launches that rotates over cache replicas larger than L2 in total."""
    import torch

    import paged_kv_decode_gqa_b200 as pkv
    x = W.make_inputs(w, seed, poison=False)
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(device)
    fp8 = w.kv_dtype == "fp8"
    k_new, v_new, slots = t(x["k_new"]), t(x["v_new"]), t(x["slot_mapping"])
    shape = x["k_pool"].shape
    dt = torch.uint8 if fp8 else torch.float16
    pool_bytes = 2 * int(np.prod(shape)) * (1 if fp8 else 2)
    R = max(2, min(16, -(-2 * L2_BYTES // pool_bytes)))
    pools = [(torch.zeros(shape, dtype=dt, device=device), torch.zeros(shape, dtype=dt, device=device))
             for _ in range(R)]
    call = lambda i: pkv.paged_kv_cache_write(k_new, v_new, pools[i % R][0], pools[i % R][1], slots,
                                              kv_dtype=w.kv_dtype, k_scale=float(x["k_scale"]),
                                              v_scale=float(x["v_scale"]), stream=stream)
    with torch.cuda.stream(stream):
        for i in range(3):
            call(i)
        torch.cuda.synchronize()
        n = max(R, reps - reps % R)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for i in range(n):
                call(i)
        g.replay()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        lead_in(stream)
        e0.record(stream)
        g.replay()
        e1.record(stream)
    torch.cuda.synchronize()
    us = e0.elapsed_time(e1) * 1000 / n
    T = int((x["slot_mapping"] >= 0).sum())
    nbytes = cache_write_bytes(T, w.Hkv, w.head_dim, 1 if fp8 else 2)
    del g
    return {"what": "paged_kv_cache_write (reshape_and_cache) alone", "workload": w.name, "T": T,
            "Hkv": w.Hkv, "head_dim": w.head_dim, "kv_dtype": w.kv_dtype, "algorithmic_bytes": nbytes,
            "us": us, "achieved": nbytes / us / 1e3, "peak": peak, "unit": "GB/s",
            "frac": nbytes / us / 1e3 / peak, "bound": "hbm (launch-bound at this size)", "launches": n,
            "l2": f"{R} cache replicas rotated; graph of {n} launches"}


def run_kv_read_ratio(args):
    """The grouped kernel against per-query-head launches on one workload: one launch of the
    grouped attention (all G query heads of a KV head from one read of its K/V), then G launches
    with Hq = Hkv, launch m serving query head m of every group, so every query head reads the
    KV on its own. The first 1 + G decode launches of this process are exactly these, in this
    order, for an ncu capture of dram__bytes_read.sum; timed repeats with L2 flushed follow."""
    import torch

    import paged_kv_decode_gqa_b200 as pkv
    device = torch.device("cuda", 0)
    torch.cuda.set_device(device)
    stream = torch.cuda.Stream(device)
    w = W.WORKLOADS[args.workload]
    x = W.make_inputs(w, args.seed)
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(device)
    B, Hq, Hkv, D, G = w.B, w.Hq, w.Hkv, w.head_dim, w.group
    if w.kv_dtype != "f16":
        raise SystemExit("--kv-read-ratio takes an f16 workload")
    k, v, bt, cl, q = t(x["k_pool"]), t(x["v_pool"]), t(x["block_tables"]), t(x["context_lens"]), t(x["q"])
    max_len, scale = int(x["context_lens"].max()), float(x["softmax_scale"])
    q_m = [q.view(B, Hkv, G, D)[:, :, m, :].contiguous() for m in range(G)]
    out = torch.empty_like(q)
    out_m = [torch.empty_like(qm) for qm in q_m]
    P = pkv.PKV_PARTITION_AUTO
    ws = torch.zeros(max(pkv.paged_gqa_decode_workspace_size(B, Hq, Hkv, D, max_len, P), 256),
                     dtype=torch.uint8, device=device)
    flush = torch.empty(2 * L2_BYTES, dtype=torch.uint8, device=device)

    def grouped():
        pkv.paged_gqa_decode_attention(out, q, k, v, bt, cl, max_context_len=max_len, softmax_scale=scale,
                                       partition_tokens=P, workspace=ws, stream=stream)

    def per_head(m):
        pkv.paged_gqa_decode_attention(out_m[m], q_m[m], k, v, bt, cl, max_context_len=max_len,
                                       softmax_scale=scale, partition_tokens=P, workspace=ws, stream=stream)

    with torch.cuda.stream(stream):
        grouped()
        for m in range(G):
            per_head(m)
        torch.cuda.synchronize()
        ref = out.view(B, Hkv, G, D)
        same = all(torch.equal(out_m[m], ref[:, :, m, :]) for m in range(G))
        max_diff = max(float((out_m[m].float() - ref[:, :, m, :].float()).abs().max()) for m in range(G))

        def timed(fn, reps=20):
            ms = []
            for _ in range(reps):
                flush.fill_(1)
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record(stream)
                fn()
                e1.record(stream)
                torch.cuda.synchronize()
                ms.append(e0.elapsed_time(e1))
            return statistics.median(ms) * 1e3

        us_grouped = timed(grouped)
        us_per_head = timed(lambda: [per_head(m) for m in range(G)])
    kv = kv_bytes(x["context_lens"], Hkv, D, 2)
    print(json.dumps({
        "what": "grouped decode attention vs per-query-head launches (Hq = Hkv, one launch per group member)",
        "workload": w.name, "B": B, "Hq": Hq, "Hkv": Hkv, "G": G,
        "kv_bytes_grouped": kv, "kv_bytes_per_query_head": G * kv,
        "outputs_bitwise_equal": same, "max_abs_diff": max_diff,
        "us_grouped": us_grouped, "us_per_query_head_total": us_per_head,
        "time_ratio": us_per_head / us_grouped,
        "timing": "median of 20, L2 flushed (256 MiB write) before each"}), flush=True)
    return 0


def run_ours(args):
    import torch
    world, rank, local = dist_setup()
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)

    w = W.WORKLOADS[args.workload]
    stream = torch.cuda.Stream(device)
    torch.cuda.set_stream(stream)
    sb = StepBench(w, device, stream, W.shard_seed(args.seed, rank), args.partition, unfused=args.unfused,
                   overlap=not args.no_overlap, fp8_scales=args.fp8_scales)
    B = w.B
    K = args.steps

    # ---- warm-up: W eager steps (also sets kernel attributes and TMA maps), then K timed steps ----
    sb.warmup(args.warmup)
    sampler = ClockSampler(torch.cuda.current_device())
    tm = sb.time(K, args.graph_steps, world, sampler)
    elapsed_max = tm["elapsed_ms"]
    e2e = None if args.no_e2e else sb.e2e(max(3, min(K, 200)), world)

    if rank == 0:
        peaks, peak_src = measured_peaks()
        peak = float(peaks.get("hbm_gbs", FALLBACK_HBM_GBS))
        value = whole_job_gbs(world, sb.step_b, K, elapsed_max)
        line = {
            "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": K,
            "warmup": args.warmup, "ms_per_step": elapsed_max / K, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f16" if not sb.fp8 else "fp8-e4m3 KV, f16 q/out",
            "data": "synthetic",
            "seq_steps_per_s": world * B * K / (elapsed_max * 1e-3),
            "pct_of_hbm_peak": 100.0 * value / peak,
            "config": {"workload": w.name, "B": B, "Hq": w.Hq, "Hkv": w.Hkv, "head_dim": w.head_dim,
                       "block_size": w.block_size, "kv_dtype": w.kv_dtype, "context_lens": list(w.ctx),
                       **({"fp8_scales": "per KV head, computed on the device"} if sb.per_head else {}),
                       "partition_tokens": args.partition, "parallelism": f"dp{world} (independent batches)",
                       **sb.describe(),
                       "timing": f"{tm['replays']} CUDA graph replays of <= {tm['graph_steps']} steps after a "
                                 "0.5 ms lead-in spin, CUDA events on the launching stream"},
            "roofline": kernel_line(sb, tm, peak, peak_src),
            "gpu_launches": sb.launches_per_step * K,
            "clocks": sampler.summary(*tm["wall"]),
        }
        if sb.scales_kernel:
            line["fp8_scales_kernel"] = sb.scales_kernel
        if e2e:
            line["e2e"] = e2e
        del sb
        torch.cuda.empty_cache()
        # side measurements: a failure is reported in its key, and the step's line is still printed
        side = []
        if not args.no_sublines and world == 1:
            subs = {}
            for name, P in SUBLINES:
                if name == w.name and P == args.partition:
                    continue
                key = f"{name}/{'auto' if P == -1 else f'P{P}'}"
                try:
                    subs[key] = time_subline(name, P, device, stream, peak, peak_src, args.sub_steps, args.seed,
                                             args.fp8_scales)
                except Exception as exc:  # noqa: BLE001 -- reported, never silent
                    subs[key] = {"error": f"{type(exc).__name__}: {exc}"}
            line["workloads"] = subs
            side.append(("cache_write_kernel", lambda: time_cache_write(W.WORKLOADS[HEADLINE], device, stream,
                                                                        peak, args.seed)))
        if not args.no_qkv:
            side.append(("qkv_kernel", lambda: time_qkv_projection(w, device, stream, peak, args.seed)))
        if not args.no_prefill:
            side.append(("prefill_kernel", lambda: time_prefill(
                w, device, stream, float(peaks.get("bf16_tflops", 1590.0)), args.seed)))
        for key, measure in side:
            try:
                line[key] = measure()
            except Exception as exc:  # noqa: BLE001 -- reported, never silent
                line[key] = {"error": f"{type(exc).__name__}: {exc}"}
        if world == 1 and args.cpu_baseline_s > 0:
            x = W.make_inputs(w, W.shard_seed(args.seed, rank))
            reps, secs, cores = time_oracle(w, x, args.cpu_baseline_s)
            attn_b, cw_b = step_bytes(w, x["context_lens"], B)
            line["cpu_baseline"] = {
                "value": (attn_b + cw_b) * reps / secs / 1e9, "unit": "GB/s", "cores": cores, "kind": "oracle",
                "sample": f"{reps} whole steps of {w.name} (all {B} sequences), {secs:.1f} s"}
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.barrier(device_ids=[local])
        dist.destroy_process_group()
    return 0


def main(argv=None):
    args = parse_args(argv)
    if args.impl == "reference":
        return run_reference(args)
    if args.kv_read_ratio:
        return run_kv_read_ratio(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
