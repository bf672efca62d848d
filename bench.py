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
그래프 리플레이); consecutive steps read different replicas of the KV pool so
that the L2 cache never holds a step's KV.

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
    call = lambda: pkv.paged_gqa_prefill_attention(out, qd, kc, vc, bt, cl, qsd, max_query_len=n_new,
                                                   max_context_len=L, softmax_scale=float(x["softmax_scale"]),
                                                   stream=stream)
    with torch.cuda.stream(stream):
        for _ in range(3):
            call()
        reps = 20
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(reps):
            call()
        e1.record(stream)
    torch.cuda.synchronize()
    us = e0.elapsed_time(e1) * 1000 / reps
    flops = prefill_flops([L] * B, [n_new] * B, w.Hq, w.head_dim)
    tflops = flops / us / 1e6
    return {"what": "paged_gqa_prefill_attention (chunked prefill, f16 cache)", "B": B, "new_tokens": n_new,
            "context": L, "Hq": w.Hq, "Hkv": w.Hkv, "flops": flops, "us": us, "achieved": tflops,
            "peak": peak_tflops, "unit": "TFLOP/s", "frac": tflops / peak_tflops, "bound": "tensor",
            "launches": reps, "l2": "cache of 8 x 2048 tokens re-read by every chunk; L2-resident after the first"}


def parse_args(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--workload", default="qwen2.5-1.5b", choices=sorted(W.WORKLOADS))
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
    ap.add_argument("--fp8-scales", default="tensor", choices=["tensor", "per-head"],
                    help="FP8 workloads: per-tensor host scales, or per-KV-head scales computed on the "
                         "device and passed to the device-scale entry points")
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
    import paged_kv_decode_gqa_b200 as pkv

    w = W.WORKLOADS[args.workload]
    x = W.make_inputs(w, W.shard_seed(args.seed, rank))
    lens = x["context_lens"]
    B, Hq, Hkv, D, bs = w.B, w.Hq, w.Hkv, w.head_dim, w.block_size
    max_len = int(lens.max())
    fp8 = w.kv_dtype == "fp8"
    P = args.partition
    attn_b, cw_b = step_bytes(w, lens, B)
    step_b = attn_b + cw_b

    stream = torch.cuda.Stream(device)
    torch.cuda.set_stream(stream)
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(device)
    q, bt, cl = t(x["q"]), t(x["block_tables"]), t(x["context_lens"])
    k_new, v_new, slots = t(x["k_new"]), t(x["v_new"]), t(x["slot_mapping"])
    ks, vs, scale = float(x["k_scale"]), float(x["v_scale"]), float(x["softmax_scale"])

    # KV pool replicas: enough that the KV touched between two reads of a replica exceeds 4x L2.
    touched = kv_bytes(lens, Hkv, D, 1 if fp8 else 2)
    R = max(1, min(16, -(-4 * L2_BYTES // max(touched, 1))))
    k16, v16 = t(x["k_pool"]), t(x["v_pool"])
    per_head = fp8 and args.fp8_scales == "per-head"
    scales_kernel = None
    if fp8:                                        # quantise the pool with the library's cache write
        kq = torch.empty(k16.shape, dtype=torch.uint8, device=device)
        vq = torch.empty_like(kq)
        n_rows = w.num_blocks * bs
        rows_k, rows_v = k16.view(n_rows, Hkv, D), v16.view(n_rows, Hkv, D)
        all_slots = torch.arange(n_rows, dtype=torch.int64, device=device)
        if per_head:
            # per-KV-head scales computed on the device from the pool (its free rows are NaN and
            # do not count); the scales kernel is timed over the K pool
            ks_t = torch.empty(Hkv, dtype=torch.float32, device=device)
            vs_t = torch.empty(Hkv, dtype=torch.float32, device=device)
            for _ in range(3):
                pkv.paged_kv_fp8_scales(rows_k, ks_t, per_head=True, stream=stream)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            reps = 10
            e0.record(stream)
            for _ in range(reps):
                pkv.paged_kv_fp8_scales(rows_k, ks_t, per_head=True, stream=stream)
            e1.record(stream)
            pkv.paged_kv_fp8_scales(rows_v, vs_t, per_head=True, stream=stream)
            torch.cuda.synchronize()
            us = e0.elapsed_time(e1) * 1000 / reps
            nbytes = rows_k.numel() * 2
            scales_kernel = {"input_bytes": nbytes, "us": us, "gbs": nbytes / us / 1e3,
                             "what": "paged_kv_fp8_scales, per KV head, over the f16 K pool (memset + 2 launches)"}
            pkv.paged_kv_cache_write_fp8_scaled(rows_k, rows_v, kq, vq, all_slots, ks_t, vs_t, stream=stream)
        else:
            pkv.paged_kv_cache_write(rows_k, rows_v, kq, vq, all_slots, kv_dtype="fp8", k_scale=ks, v_scale=vs)
        base_k, base_v = kq, vq
        del k16, v16, rows_k, rows_v
    else:
        base_k, base_v = k16, v16
    pools = [(base_k, base_v)] + [(base_k.clone(), base_v.clone()) for _ in range(R - 1)]
    ws_n = pkv.paged_gqa_decode_workspace_size(B, Hq, Hkv, D, max_len, P)
    ws = torch.zeros(max(ws_n, 256), dtype=torch.uint8, device=device)
    out = torch.empty((B, Hq, D), dtype=torch.float16, device=device)

    fused = not args.unfused and P == pkv.PKV_PARTITION_AUTO
    step_flags = 0 if args.no_overlap else pkv.PKV_STEP_OVERLAP_PREVIOUS

    # the library calls of one step, per-tensor scales or per-KV-head device scales
    def write_call(kn, vn, kc, vc, sl):
        if per_head:
            pkv.paged_kv_cache_write_fp8_scaled(kn, vn, kc, vc, sl, ks_t, vs_t, stream=stream)
        else:
            pkv.paged_kv_cache_write(kn, vn, kc, vc, sl, kv_dtype=w.kv_dtype, k_scale=ks, v_scale=vs,
                                     stream=stream)

    def step_call(qq, kn, vn, kc, vc, bb, cc, flags):
        if per_head:
            pkv.paged_gqa_decode_step_fp8_scaled(out, qq, kn, vn, kc, vc, bb, cc, ks_t, vs_t,
                                                 max_context_len=max_len, softmax_scale=scale,
                                                 workspace=ws, flags=flags, stream=stream)
        else:
            pkv.paged_gqa_decode_step(out, qq, kn, vn, kc, vc, bb, cc, max_context_len=max_len,
                                      softmax_scale=scale, kv_dtype=w.kv_dtype, k_scale=ks, v_scale=vs,
                                      workspace=ws, flags=flags, stream=stream)

    def attention_call(qq, kc, vc, bb, cc):
        if per_head:
            pkv.paged_gqa_decode_attention_fp8_scaled(out, qq, kc, vc, bb, cc, ks_t, vs_t,
                                                      max_context_len=max_len, softmax_scale=scale,
                                                      partition_tokens=P, workspace=ws, stream=stream)
        else:
            pkv.paged_gqa_decode_attention(out, qq, kc, vc, bb, cc, max_context_len=max_len,
                                           softmax_scale=scale, kv_dtype=w.kv_dtype, k_scale=ks,
                                           v_scale=vs, partition_tokens=P, workspace=ws, stream=stream)

    def cache_write(i):
        if fused:                                  # the step kernel writes the new tokens itself
            return
        kc, vc = pools[i % R]
        write_call(k_new, v_new, kc, vc, slots)

    def attention(i):
        kc, vc = pools[i % R]
        if fused:
            # consecutive steps read different pool replicas, so no launch writes
            # the pages the next one reads: the overlap promise holds
            step_call(q, k_new, v_new, kc, vc, bt, cl, step_flags)
        else:
            attention_call(q, kc, vc, bt, cl)

    # ---- warm-up: W eager steps (also sets kernel attributes and TMA maps) ----
    for i in range(args.warmup):
        cache_write(i)
        attention(i)
    torch.cuda.synchronize()

    # ---- capture the timed steps as CUDA graphs with events around each attention launch ----
    K = args.steps
    S = max(1, min(args.graph_steps, K))
    chunks = [S] * (K // S) + ([K % S] if K % S else [])
    graphs, ev_pairs = {}, []
    # Fused: one launch per step and nothing between launches, so that each
    # launch overlaps the previous one's tail (programmatic dependent launch);
    # its average duration is the timed region over K. Unfused: events around
    # every attention launch give that kernel's own duration.
    for n in sorted(set(chunks)):
        evs = [] if fused else [(torch.cuda.Event(enable_timing=True, external=True),
                                 torch.cuda.Event(enable_timing=True, external=True)) for _ in range(n)]
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for i in range(n):
                cache_write(i)
                if evs:
                    evs[i][0].record(stream)
                attention(i)
                if evs:
                    evs[i][1].record(stream)
        graphs[n] = (g, evs)
    torch.cuda.synchronize()

    sampler = ClockSampler(torch.cuda.current_device()).start()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    attn_ms = []
    barrier(world, device)
    torch.cuda.synchronize()
    wall0 = time.perf_counter()
    start.record(stream)
    for n in chunks:
        graphs[n][0].replay()
    end.record(stream)
    torch.cuda.synchronize()
    wall1 = time.perf_counter()
    barrier(world, device)
    sampler.stop()
    elapsed_ms = start.elapsed_time(end)
    if fused:
        attn_ms = [elapsed_ms / K]
    else:        # per-launch durations of the attention kernel in the last replay of each graph
        for n in set(chunks):
            attn_ms += [a.elapsed_time(b) for a, b in graphs[n][1]]
    elapsed_max = reduce_max(elapsed_ms, world, device)
    launches = (1 if fused else 2) * K

    # ---- e2e: the public API on host buffers, copies in the timed region ----
    e2e = None
    if not args.no_e2e:
        h = {k: torch.from_numpy(np.ascontiguousarray(x[k])).pin_memory()
             for k in ("q", "k_new", "v_new", "slot_mapping", "block_tables", "context_lens")}
        d = {k: torch.empty(v.shape, dtype=v.dtype, device=device) for k, v in h.items()}
        out_h = torch.empty((B, Hq, D), dtype=torch.float16).pin_memory()
        h2d = sum(v.numel() * v.element_size() for v in h.values())
        d2h = out_h.numel() * out_h.element_size()
        n_e2e = max(3, min(K, 200))

        def e2e_step(i):
            for k in h:
                d[k].copy_(h[k], non_blocking=True)
            kc, vc = pools[i % R]
            if fused:
                step_call(d["q"], d["k_new"], d["v_new"], kc, vc, d["block_tables"], d["context_lens"], 0)
            else:
                write_call(d["k_new"], d["v_new"], kc, vc, d["slot_mapping"])
                attention_call(d["q"], kc, vc, d["block_tables"], d["context_lens"])
            out_h.copy_(out, non_blocking=True)
            stream.synchronize()

        for i in range(3):
            e2e_step(i)
        barrier(world, device)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for i in range(n_e2e):
            e2e_step(i)
        e1.record(stream)
        torch.cuda.synchronize()
        e2e_ms = reduce_max(e0.elapsed_time(e1), world, device)
        e2e = {"value": world * step_b * n_e2e / (e2e_ms * 1e-3) / 1e9, "unit": "GB/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": n_e2e,
               "ms_per_step": e2e_ms / n_e2e, "note": "eager calls, one host sync per step"}

    if rank == 0:
        peaks, peak_src = measured_peaks()
        peak = float(peaks.get("hbm_gbs", FALLBACK_HBM_GBS))
        mean_attn_ms = sum(attn_ms) / len(attn_ms)
        kern_b = step_b if fused else attn_b          # the fused launch also does the cache write
        achieved = kern_b / (mean_attn_ms * 1e-3) / 1e9
        traffic = recorded_traffic(w.name, P)
        value = whole_job_gbs(world, step_b, K, elapsed_max)
        line = {
            "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": K,
            "warmup": args.warmup, "ms_per_step": elapsed_max / K, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f16" if not fp8 else "fp8-e4m3 KV, f16 q/out",
            "data": "synthetic",
            "seq_steps_per_s": world * B * K / (elapsed_max * 1e-3),
            "pct_of_hbm_peak": 100.0 * value / peak,
            "config": {"workload": w.name, "B": B, "Hq": Hq, "Hkv": Hkv, "head_dim": D,
                       "block_size": bs, "kv_dtype": w.kv_dtype, "context_lens": list(w.ctx),
                       **({"fp8_scales": "per KV head, computed on the device"} if per_head else {}),
                       "partition_tokens": P, "parallelism": f"dp{world} (independent batches)",
                       "l2": f"inputs larger than L2: {R} KV pool replicas rotated, "
                             f"{R * touched / 2**20:.0f} MiB touched per cycle",
                       "timing": f"{len(chunks)} CUDA graph replays of <= {S} steps",
                       "step": ("one fused launch (cache write + attention)" +
                                ("" if args.no_overlap else ", PKV_STEP_OVERLAP_PREVIOUS"))
                               if fused else "cache write + attention launches"},
            "roofline": {"bound": "hbm",
                         "kernel": "decode_balanced_kernel (fused step)" if fused else "decode attention",
                         "achieved": achieved, "peak": peak, "unit": "GB/s",
                         "frac": achieved / peak, "peak_source": f"{peak_src} hbm_gbs",
                         "traffic": traffic, "algorithmic_bytes_per_launch": kern_b,
                         "mean_launch_us": mean_attn_ms * 1e3},
            "gpu_launches": launches,
            "clocks": sampler.summary(wall0, wall1),
        }
        if scales_kernel:
            line["fp8_scales_kernel"] = scales_kernel
        # side measurements of the other kernels: a failure is reported in its key, and the
        # step's line is still printed
        side = []
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
        if e2e:
            line["e2e"] = e2e
        if world == 1 and args.cpu_baseline_s > 0:
            reps, secs, cores = time_oracle(w, x, args.cpu_baseline_s)
            line["cpu_baseline"] = {
                "value": step_b * reps / secs / 1e9, "unit": "GB/s", "cores": cores, "kind": "oracle",
                "sample": f"{reps} whole steps of {w.name} (all {B} sequences), {secs:.1f} s"}
        print(json.dumps(line), flush=True)
    del graphs
    if world > 1:
        import torch.distributed as dist
        dist.barrier(device_ids=[local])
        dist.destroy_process_group()
    return 0


def main(argv=None):
    args = parse_args(argv)
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
