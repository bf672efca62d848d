"""The entry point that allocates nothing: paged_gqa_decode_attention_static_workspace.

Some callers cannot allocate device memory for per-call scratch -- a serving
engine that handed all free GPU memory to its KV-cache pool at start-up, a
decode step being recorded into a CUDA graph (no cudaMalloc allowed there), or
a foreign-language caller without the process's allocator. This entry point
takes its split-KV scratch from a fixed array inside the library instead of a
caller workspace, for every plan: the balanced default (PKV_PARTITION_AUTO),
fixed partitions and the single pass. Its results must match the float64
oracle within the attention tolerance, and the regular entry point (same
kernel, same plan) bit for bit, on two calls in a row that share the array.

This file is named to be collected last, so that a run that stops at the first
failure has run every other test first; it also passes alone.
"""
import numpy as np
import pytest
import torch

import paged_kv_decode_gqa_b200 as pkv
import workloads as W
from _gpu_helpers import DecodeRun, assert_attention_close, fp8_caches, host

pytestmark = pytest.mark.gpu

AUTO = pkv.PKV_PARTITION_AUTO

CASES = [
    ("qwen2.5-1.5b", dict(B=16), "f16", 128),                   # fixed partitions: scratch from the array
    ("qwen2.5-1.5b", dict(B=16), "f16", AUTO),                  # balanced plan: piece slots and tickets
    ("skewed-split", {}, "f16", 512),                           # the full skewed workload, 7.1 MiB
    ("skewed-split", {}, "f16", AUTO),                          # one 32k sequence over hundreds of workers
    ("fp8-e4m3", dict(B=12, num_blocks=6144), "fp8", AUTO),    # FP8 balanced plan (the largest slots)
    ("fp8-e4m3", dict(B=12, num_blocks=6144), "fp8", 1024),
    ("qwen2.5-7b", dict(B=4, num_blocks=2048), "f16", 0),       # single pass: no scratch
]


def _case_id(c):
    return f"{c[0]}-{c[2]}-{'auto' if c[3] == AUTO else c[3]}"


@pytest.mark.parametrize("name,sizes,kv,P", CASES, ids=[_case_id(c) for c in CASES])
def test_static_workspace_matches_oracle_and_regular_entry_point_twice(name, sizes, kv, P):
    w = W.with_sizes(W.WORKLOADS[name], **sizes)
    x = W.make_inputs(w, seed=21)
    if kv == "fp8":
        kq, vq = fp8_caches(x)
        r = DecodeRun(w, x, kv_dtype="fp8", k_cache=kq, v_cache=vq)
    else:
        r = DecodeRun(w, x)
    B, Hq, D = r.q.shape
    ref = r.oracle(partition_tokens=max(P, 0))
    regular = host(r.attention(P))                          # caller workspace, same plan
    for call in range(2):                                   # two calls in a row share the array
        out = torch.full((B, Hq, D), float("nan"), dtype=torch.float16, device="cuda")
        pkv.paged_gqa_decode_attention_static_workspace(
            out, r.q, r.k, r.v, r.bt, r.cl, max_context_len=r.max_len,
            softmax_scale=float(x["softmax_scale"]), kv_dtype=kv, k_scale=float(x["k_scale"]),
            v_scale=float(x["v_scale"]), partition_tokens=P)
        torch.cuda.synchronize()
        got = host(out)
        assert_attention_close(got, ref, f"{_case_id((name, sizes, kv, P))} call {call}")
        assert np.array_equal(got.view(np.uint16), regular.view(np.uint16)), f"call {call} differs from the regular entry point"
    assert pkv.pkv_device_error() == 0


def test_static_workspace_rejects_sizes_beyond_its_limit():
    w = W.WORKLOADS["qwen2.5-7b"]
    B, Hq, D, max_len, P = w.B, w.Hq, w.head_dim, 4096, 256
    assert pkv.paged_gqa_decode_workspace_size(B, Hq, w.Hkv, D, max_len, P) > pkv.STATIC_WORKSPACE_BYTES
    t = lambda *s, dt=torch.float16: torch.zeros(s, dtype=dt, device="cuda")
    with pytest.raises(pkv.PagedKVError) as e:
        pkv.paged_gqa_decode_attention_static_workspace(
            t(B, Hq, D), t(B, Hq, D), t(64, 16, w.Hkv, D), t(64, 16, w.Hkv, D),
            t(B, 256, dt=torch.int32), t(B, dt=torch.int32), max_context_len=max_len,
            softmax_scale=0.088, partition_tokens=P)
    assert e.value.status == pkv.PKV_ERR_WORKSPACE
