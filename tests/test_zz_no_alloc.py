"""The entry point that allocates nothing: paged_gqa_decode_attention_static_workspace.

Some callers cannot allocate device memory for per-call scratch -- a serving
engine that handed all free GPU memory to its KV-cache pool at start-up, a
decode step being recorded into a CUDA graph (no cudaMalloc allowed there), or
a foreign-language caller without the process's allocator. This entry point
takes its split-KV scratch from a fixed array inside the library instead of a
caller workspace. Its results must match the regular entry point's, within the
tolerance the parity tests use, on two calls in a row that share the array.

This file is named to be collected last, so that a run that stops at the first
failure has run every other test first; it also passes alone.
"""
import numpy as np
import pytest
import torch

import paged_kv_decode_gqa_b200 as pkv
import workloads as W
from _gpu_helpers import ATOL, RTOL_OF_MAX, DecodeRun, host

pytestmark = pytest.mark.gpu


def _close(a, b, what):
    a = a.astype(np.float64)
    b = b.astype(np.float64)
    err = np.abs(a - b).max()
    assert np.isfinite(a).all(), what
    assert err <= ATOL and err <= RTOL_OF_MAX * np.abs(b).max(), f"{what}: {err:.3e}"


CASES = [
    ("qwen2.5-1.5b", dict(B=16), 128),                   # split-KV: uses the static scratch
    ("skewed-split", {}, 512),                           # full skewed workload, 7.1 MiB of scratch
    ("qwen2.5-7b", dict(B=4, num_blocks=2048), 0),       # single pass: no scratch
]


@pytest.mark.parametrize("name,sizes,P", CASES)
def test_static_workspace_matches_regular_entry_point_twice(name, sizes, P):
    w = W.with_sizes(W.WORKLOADS[name], **sizes)
    x = W.make_inputs(w, seed=21)
    r = DecodeRun(w, x)
    B, Hq, D = r.q.shape
    assert pkv.paged_gqa_decode_workspace_size(B, Hq, w.Hkv, D, r.max_len, P) <= pkv.STATIC_WORKSPACE_BYTES
    ref = host(r.attention(P))                           # regular entry point, caller workspace
    for call in range(2):                                # two calls in a row share the array
        out = torch.full((B, Hq, D), float("nan"), dtype=torch.float16, device="cuda")
        pkv.paged_gqa_decode_attention_static_workspace(
            out, r.q, r.k, r.v, r.bt, r.cl, max_context_len=r.max_len,
            softmax_scale=float(x["softmax_scale"]), partition_tokens=P)
        torch.cuda.synchronize()
        _close(host(out), ref, f"{name} call {call}")


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
