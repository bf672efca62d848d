"""Failure detection on the GPU: a barrier wait that runs out ends the kernel
with an error status instead of a hang, and the context stays usable.

Every wait of the decode kernels on a page's transaction barrier has a time
limit; when it runs out, the kernel flags PKV_DEVERR_WAIT_TIMEOUT in the
device error word, waits (again with the limit) for the copies it still has
in flight, and returns. The self-test flag PKV_STEP_SELFTEST_WAIT_TIMEOUT of
paged_gqa_decode_step makes one worker warp issue none of its page loads, so
its first wait can never complete, with no copy in flight, and shortens the
limit to 2 ms. Nothing here faults, traps or hangs the GPU.
"""
import numpy as np
import pytest
import torch

import oracle
import paged_kv_decode_gqa_b200 as pkv
import workloads as W
from _gpu_helpers import assert_attention_close, dev, host

pytestmark = pytest.mark.gpu


def _step_inputs(name, sizes, seed):
    w = W.with_sizes(W.WORKLOADS[name], **sizes)
    x = W.make_inputs(w, seed=seed)
    return w, x


@pytest.mark.parametrize("name,sizes", [("qwen2.5-1.5b", dict(B=16)), ("skewed-split", {})])
def test_wait_timeout_is_flagged_and_the_next_call_is_correct(name, sizes):
    w, x = _step_inputs(name, sizes, seed=5)
    B, Hq, D = x["q"].shape
    kc, vc = dev(x["k_pool"]), dev(x["v_pool"])
    q, kn, vn = dev(x["q"]), dev(x["k_new"]), dev(x["v_new"])
    bt, cl = dev(x["block_tables"]), dev(x["context_lens"])
    max_len = int(x["context_lens"].max())
    n = pkv.paged_gqa_decode_workspace_size(B, Hq, w.Hkv, D, max_len, pkv.PKV_PARTITION_AUTO)
    ws = torch.zeros(n, dtype=torch.uint8, device="cuda")
    out = torch.full((B, Hq, D), float("nan"), dtype=torch.float16, device="cuda")
    assert pkv.pkv_device_error() == 0

    call = lambda flags: pkv.paged_gqa_decode_step(
        out, q, kn, vn, kc, vc, bt, cl, max_context_len=max_len, softmax_scale=float(x["softmax_scale"]),
        workspace=ws, flags=flags)
    call(pkv.PKV_STEP_SELFTEST_WAIT_TIMEOUT)
    torch.cuda.synchronize()                      # the launch ends: no hang, no CUDA error
    assert pkv.pkv_device_error() & pkv.DEVERR_WAIT_TIMEOUT
    assert not torch.isfinite(out).all()          # the stalled worker's rows were never written

    # the context is usable: zero the workspace again (its tickets may be set) and step normally
    ws.zero_()
    out.fill_(float("nan"))
    call(0)
    torch.cuda.synchronize()
    assert pkv.pkv_device_error() == 0
    kr, vr = x["k_pool"].copy(), x["v_pool"].copy()
    oracle.paged_kv_cache_write(x["k_new"], x["v_new"], kr, vr, x["slot_mapping"])
    ref = oracle.paged_gqa_decode(x["q"], kr, vr, x["block_tables"], x["context_lens"], float(x["softmax_scale"]))
    assert_attention_close(host(out), ref, f"{name} after a wait timeout")
    assert np.array_equal(host(kc).view(np.uint16), kr.view(np.uint16))
    assert np.array_equal(host(vc).view(np.uint16), vr.view(np.uint16))

