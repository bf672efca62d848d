"""Parity of the FP8 entry points with device-side scales (per tensor or per KV head) and of the
scales computed from data, against the float64 oracle.

Scales and cache bytes: bit-exact. Attention: the tolerance of tests/test_gpu_parity.py, with the
oracle run on the same E4M3 bytes and the same scales.
"""
import numpy as np
import pytest
import torch

import oracle
import paged_kv_decode_gqa_b200 as pkv
import workloads as W
from _gpu_helpers import assert_attention_close, dev, host

pytestmark = pytest.mark.gpu
AUTO = pkv.PKV_PARTITION_AUTO


@pytest.fixture(autouse=True)
def _clear_device_error():
    pkv.pkv_device_error()
    yield
    torch.cuda.synchronize()


def _device_scales(x, per_head):
    s = torch.full((x.shape[1] if per_head else 1,), -7.0, dtype=torch.float32, device="cuda")
    pkv.paged_kv_fp8_scales(dev(x), s, per_head=per_head)
    return host(s)


# ------------------------------------------------------------------ scales from data
@pytest.mark.parametrize("Hkv", [1, 2, 4, 7, 8])
@pytest.mark.parametrize("per_head", [False, True])
def test_scales_from_data_bit_exact(Hkv, per_head):
    rng = np.random.default_rng(Hkv)
    x = (rng.standard_normal((333, Hkv, 128)) * rng.uniform(0.01, 50.0, size=(1, Hkv, 1))).astype(np.float16)
    x[5, 0, 3] = np.nan                                 # NaN never counts
    x[7, Hkv - 1, 100] = np.float16(-300.0)             # a negative maximum
    got = _device_scales(x, per_head)
    assert np.array_equal(got.view(np.uint32), oracle.fp8_scales(x, per_head).view(np.uint32))
    assert pkv.pkv_device_error() == 0


def test_scales_of_zero_and_empty_data_are_one():
    z = np.zeros((16, 2, 128), np.float16)
    z[:, 1] = np.nan
    assert _device_scales(z, True).tolist() == [1.0, 1.0]
    e = torch.empty((0, 4, 128), dtype=torch.float16, device="cuda")
    s = torch.zeros(4, dtype=torch.float32, device="cuda")
    pkv.paged_kv_fp8_scales(e, s, per_head=True)
    assert host(s).tolist() == [1.0] * 4


def test_scales_of_the_7b_pool_bit_exact():
    """The full 32k-block Qwen2.5-7B-shaped pool (268M f16 values, NaN-poisoned free rows)."""
    w = W.WORKLOADS["qwen2.5-7b"]
    x = W.make_inputs(w, 3)
    pool = x["k_pool"].reshape(-1, w.Hkv, w.head_dim)
    for per_head in (False, True):
        got = _device_scales(pool, per_head)
        assert np.array_equal(got.view(np.uint32), oracle.fp8_scales(pool, per_head).view(np.uint32))


# ------------------------------------------------------------------ per-head cache write
@pytest.mark.parametrize("per_head", [False, True])
def test_cache_write_with_device_scales_bit_exact(per_head):
    w = W.with_sizes(W.WORKLOADS["qwen2.5-7b"], kv_dtype="fp8")
    x = W.make_inputs(w, 4)
    T = w.B
    ks = oracle.fp8_scales(x["k_new"], per_head) * np.float32(3.0)     # any positive scales
    vs = oracle.fp8_scales(x["v_new"], per_head)
    kc = np.zeros((w.num_blocks, w.block_size, w.Hkv, w.head_dim), np.uint8)
    vc = np.zeros_like(kc)
    slots = x["slot_mapping"].copy()
    slots[1] = -1
    k_dev, v_dev = dev(kc), dev(vc)
    pkv.paged_kv_cache_write_fp8_scaled(dev(x["k_new"]), dev(x["v_new"]), k_dev, v_dev, dev(slots),
                                        dev(ks), dev(vs))
    kr, vr = kc.copy(), vc.copy()
    oracle.paged_kv_cache_write(x["k_new"], x["v_new"], kr, vr, slots, kv_dtype="fp8",
                                k_scale=ks if per_head else float(ks[0]),
                                v_scale=vs if per_head else float(vs[0]))
    assert np.array_equal(host(k_dev), kr) and np.array_equal(host(v_dev), vr)
    assert T > 0 and pkv.pkv_device_error() == 0


# ------------------------------------------------------------------ attention and step
class _Case:
    """An FP8 decode case quantised per KV head with scales computed on the device."""

    def __init__(self, w, seed):
        self.w, x = w, W.make_inputs(w, seed)
        self.x = x
        live = np.concatenate([x["k_pool"].reshape(-1, w.Hkv, w.head_dim)])
        self.ks = _device_scales(live, True) * np.array([1, 2, 0.5, 1.5, 1, 3, 0.25, 1][:w.Hkv], np.float32)
        self.vs = _device_scales(x["v_pool"].reshape(-1, w.Hkv, w.head_dim), True)
        self.kq = np.ascontiguousarray(np.stack(
            [oracle.quantize_e4m3(x["k_pool"][:, :, h], float(self.ks[h])) for h in range(w.Hkv)], axis=2))
        self.vq = np.ascontiguousarray(np.stack(
            [oracle.quantize_e4m3(x["v_pool"][:, :, h], float(self.vs[h])) for h in range(w.Hkv)], axis=2))
        self.max_len = max(int(x["context_lens"].max()), 1)

    def oracle(self, k=None, v=None, seqs=None):
        sel = slice(None) if seqs is None else np.asarray(seqs)
        x = self.x
        return oracle.paged_gqa_decode(x["q"][sel], self.kq if k is None else k, self.vq if v is None else v,
                                       x["block_tables"][sel], x["context_lens"][sel], float(x["softmax_scale"]),
                                       kv_dtype="fp8", k_scale=self.ks, v_scale=self.vs)


@pytest.mark.parametrize("P", [0, 64, AUTO])
@pytest.mark.parametrize("name,sizes", [
    ("fp8-e4m3", dict(B=4, num_blocks=4096, ctx=("uniform", 17, 2600))),
    ("qwen2.5-7b", dict(B=5, num_blocks=2048, kv_dtype="fp8")),
])
def test_attention_with_per_head_device_scales(name, sizes, P):
    c = _Case(W.with_sizes(W.WORKLOADS[name], **sizes), 9)
    x = c.x
    B, Hq, D = x["q"].shape
    out = torch.full((B, Hq, D), float("nan"), dtype=torch.float16, device="cuda")
    ws = None
    if P:
        ws = torch.zeros(pkv.paged_gqa_decode_workspace_size(B, Hq, c.w.Hkv, D, c.max_len, P),
                         dtype=torch.uint8, device="cuda")
    pkv.paged_gqa_decode_attention_fp8_scaled(out, dev(x["q"]), dev(c.kq), dev(c.vq), dev(x["block_tables"]),
                                              dev(x["context_lens"]), dev(c.ks), dev(c.vs),
                                              max_context_len=c.max_len, softmax_scale=float(x["softmax_scale"]),
                                              partition_tokens=P, workspace=ws)
    assert_attention_close(host(out), c.oracle(), f"{name} per-head P={P}")
    assert pkv.pkv_device_error() == 0


def test_attention_with_one_device_scale_is_the_per_tensor_entry_point():
    w = W.with_sizes(W.WORKLOADS["fp8-e4m3"], B=4, num_blocks=4096, ctx=("uniform", 17, 2600))
    x = W.make_inputs(w, 10)
    kq = oracle.quantize_e4m3(x["k_pool"], float(x["k_scale"]))
    vq = oracle.quantize_e4m3(x["v_pool"], float(x["v_scale"]))
    B, Hq, D = x["q"].shape
    ml = int(x["context_lens"].max())
    outs = []
    for scaled in (False, True):
        out = torch.empty((B, Hq, D), dtype=torch.float16, device="cuda")
        args = (out, dev(x["q"]), dev(kq), dev(vq), dev(x["block_tables"]), dev(x["context_lens"]))
        if scaled:
            pkv.paged_gqa_decode_attention_fp8_scaled(
                *args, dev(np.array([x["k_scale"]], np.float32)), dev(np.array([x["v_scale"]], np.float32)),
                max_context_len=ml, softmax_scale=float(x["softmax_scale"]))
        else:
            pkv.paged_gqa_decode_attention(*args, max_context_len=ml, softmax_scale=float(x["softmax_scale"]),
                                           kv_dtype="fp8", k_scale=float(x["k_scale"]),
                                           v_scale=float(x["v_scale"]))
        outs.append(host(out))
    ref = oracle.paged_gqa_decode(x["q"], kq, vq, x["block_tables"], x["context_lens"],
                                  float(x["softmax_scale"]), kv_dtype="fp8", k_scale=float(x["k_scale"]),
                                  v_scale=float(x["v_scale"]))
    for o in outs:
        assert_attention_close(o, ref, "one device scale")


@pytest.mark.parametrize("flags", [0, pkv.PKV_STEP_OVERLAP_PREVIOUS])
def test_fused_step_with_per_head_device_scales(flags):
    c = _Case(W.with_sizes(W.WORKLOADS["qwen2.5-7b"], B=6, num_blocks=2048, kv_dtype="fp8"), 11)
    x = c.x
    B, Hq, D = x["q"].shape
    k_dev, v_dev = dev(c.kq), dev(c.vq)
    out = torch.full((B, Hq, D), float("nan"), dtype=torch.float16, device="cuda")
    ws = torch.zeros(pkv.paged_gqa_decode_workspace_size(B, Hq, c.w.Hkv, D, c.max_len, AUTO),
                     dtype=torch.uint8, device="cuda")
    pkv.paged_gqa_decode_step_fp8_scaled(out, dev(x["q"]), dev(x["k_new"]), dev(x["v_new"]), k_dev, v_dev,
                                         dev(x["block_tables"]), dev(x["context_lens"]), dev(c.ks), dev(c.vs),
                                         max_context_len=c.max_len, softmax_scale=float(x["softmax_scale"]),
                                         workspace=ws, flags=flags)
    kr, vr = c.kq.copy(), c.vq.copy()
    oracle.paged_kv_cache_write(x["k_new"], x["v_new"], kr, vr, x["slot_mapping"], kv_dtype="fp8",
                                k_scale=c.ks, v_scale=c.vs)
    assert np.array_equal(host(k_dev), kr) and np.array_equal(host(v_dev), vr)
    assert_attention_close(host(out), c.oracle(k=kr, v=vr), f"fused per-head flags={flags}")
    assert pkv.pkv_device_error() == 0


def test_a_non_positive_device_scale_is_flagged_not_faulted():
    c = _Case(W.with_sizes(W.WORKLOADS["qwen2.5-7b"], B=2, num_blocks=512, kv_dtype="fp8"), 12)
    x = c.x
    B, Hq, D = x["q"].shape
    ks = c.ks.copy()
    ks[1] = 0.0
    out = torch.empty((B, Hq, D), dtype=torch.float16, device="cuda")
    pkv.paged_gqa_decode_attention_fp8_scaled(out, dev(x["q"]), dev(c.kq), dev(c.vq), dev(x["block_tables"]),
                                              dev(x["context_lens"]), dev(ks), dev(c.vs),
                                              max_context_len=c.max_len, softmax_scale=float(x["softmax_scale"]))
    assert pkv.pkv_device_error() & pkv.DEVERR_SCALE
    kc = torch.zeros((16, 16, 4, 128), dtype=torch.uint8, device="cuda")
    kn = torch.ones((1, 4, 128), dtype=torch.float16, device="cuda")
    pkv.paged_kv_cache_write_fp8_scaled(kn, kn, kc, kc.clone(), torch.zeros(1, dtype=torch.int64, device="cuda"),
                                        dev(np.array([1, 1, float("inf"), 1], np.float32)),
                                        dev(np.ones(4, np.float32)))
    assert pkv.pkv_device_error() & pkv.DEVERR_SCALE
