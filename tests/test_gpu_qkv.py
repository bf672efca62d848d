"""Parity of fused_add_rmsnorm_qkv (residual add + RMSNorm + QKV projection) with the float64 oracle.

residual_out: bit-exact. q, k_new, v_new: |gpu - oracle| <= ulp16(oracle) + 2^-10 * C[t, n], with
C[t, n] = sum_k |W[n, k] * y[t, k]| (y the oracle's normalised activations). The bound follows
from the kernel's arithmetic: the weight operand W * gamma is rounded once to f16 (relative 2^-11
per term) while the activation operand s is exact, the dot product is accumulated in fp32 (at
most H * 2^-24 relative to C: 2.2e-4 at the models' H <= 3584; the H = 8192 case relies on the
usual square-root growth of rounding errors), the sum of squares in fp32 moves 1/RMS by about
1e-4 relative, and the result is rounded once to f16 (half an ulp; a full ulp covers a rounding
that crosses a binade). The first three add up to under 2^-10 * C.
"""
import numpy as np
import pytest
import torch

import oracle
import paged_kv_decode_gqa_b200 as pkv
import workloads as W
from _gpu_helpers import dev, host

pytestmark = pytest.mark.gpu
F16 = np.float16


@pytest.fixture(autouse=True)
def _clear_device_error():
    pkv.pkv_device_error()
    yield
    torch.cuda.synchronize()


def _ulp16(v):
    a = np.abs(v.astype(np.float64))
    e = np.floor(np.log2(np.maximum(a, 2.0 ** -14)))
    return np.exp2(e - 10)


def qkv_bound(d, res_out, eps, rows=None):
    """ulp16 + 2^-10 * sum_k |W y| per (token, feature) for the tokens `rows`."""
    s = res_out.astype(np.float64)
    if rows is not None:
        s = s[rows]
    y = s / np.sqrt((s * s).mean(axis=1, keepdims=True) + eps) * d["gamma"].astype(np.float64)
    return np.abs(y) @ np.abs(d["w_qkv"].astype(np.float64)).T * 2.0 ** -10


def run_gpu(d, Hq, Hkv, D, eps, flags=0):
    T, H = d["x"].shape
    res = torch.full((T, H), float("nan"), dtype=torch.float16, device="cuda")
    q = torch.full((T, Hq, D), float("nan"), dtype=torch.float16, device="cuda")
    k = torch.full((T, Hkv, D), float("nan"), dtype=torch.float16, device="cuda")
    v = torch.full((T, Hkv, D), float("nan"), dtype=torch.float16, device="cuda")
    pkv.fused_add_rmsnorm_qkv(dev(d["x"]), dev(d["residual"]), dev(d["gamma"]), dev(d["w_qkv"]),
                              None if d["bias"] is None else dev(d["bias"]), res, q, k, v, eps=eps, flags=flags)
    return host(res), host(q), host(k), host(v)


def check(d, Hq, Hkv, D, eps=W.RMS_EPS, rows=None, flags=0, what=""):
    T = d["x"].shape[0]
    res, q, k, v = run_gpu(d, Hq, Hkv, D, eps, flags)
    sel = np.arange(T) if rows is None else np.asarray(rows)
    sub = {key: (val[sel] if key in ("x", "residual") else val) for key, val in d.items()}
    ref_res, rq, rk, rv = oracle.add_rmsnorm_qkv(sub["x"], sub["residual"], d["gamma"], d["w_qkv"], d["bias"],
                                                 eps, Hq, Hkv, D)
    assert np.array_equal(res[sel].view(np.uint16), ref_res.view(np.uint16)), f"{what}: residual_out"
    got = np.concatenate([q[sel].reshape(len(sel), -1), k[sel].reshape(len(sel), -1),
                          v[sel].reshape(len(sel), -1)], axis=1).astype(np.float64)
    ref = np.concatenate([rq.reshape(len(sel), -1), rk.reshape(len(sel), -1), rv.reshape(len(sel), -1)], axis=1)
    tol = _ulp16(ref) + qkv_bound(d, ref_res, eps)
    err = np.abs(got - ref)
    assert np.isfinite(got).all(), f"{what}: non-finite output"
    worst = np.unravel_index(np.argmax(err - tol), err.shape)
    assert (err <= tol).all(), f"{what}: err {err[worst]:.3g} > tol {tol[worst]:.3g} at {worst}"
    assert pkv.pkv_device_error() == 0
    return float(err.max())


# ------------------------------------------------------------------ small cases: tiles, slices, tails
@pytest.mark.parametrize("T,H,Hq,Hkv,D", [
    (1, 64, 2, 1, 64),          # one k block: no split
    (5, 192, 4, 2, 32),         # 3 k blocks, N = 256
    (64, 1536, 12, 2, 128),     # Qwen2.5-1.5B shape, one token tile
    (70, 1536, 12, 2, 128),     # a ragged second token tile
    (130, 512, 6, 1, 64),       # one partial token tile of 256, N = 512
    (300, 512, 6, 1, 64),       # two token tiles of 256, the second ragged
    (33, 3584, 28, 4, 128),     # Qwen2.5-7B shape: 256-row weight tiles
    (3, 8192, 2, 1, 128),       # the largest H
    (9, 640, 1, 1, 8),          # N = 24: one partial weight tile
])
@pytest.mark.parametrize("bias", [True, False])
def test_parity_small(T, H, Hq, Hkv, D, bias):
    d = W.make_qkv_inputs(T, H, Hq, Hkv, D, seed=T + H, bias=bias)
    check(d, Hq, Hkv, D, what=f"T={T} H={H}")


@pytest.mark.parametrize("name", sorted(W.QKV_SHAPES))
def test_parity_outlier_channels(name):
    """Residual channels near 3e4 with gamma 8: s * gamma would pass the f16 range before the RMS division
    (the kernel scales W by gamma and keeps s exact)."""
    sh = W.QKV_SHAPES[name]
    d = W.make_qkv_inputs(16, sh["H"], sh["Hq"], sh["Hkv"], sh["D"], seed=7, outliers=True)
    check(d, sh["Hq"], sh["Hkv"], sh["D"], what=f"{name} outliers")


def test_tiny_and_huge_rows():
    """Rows scaled by 2^-20 and 2^10: the activation operand is s itself, exact at any scale."""
    d = W.make_qkv_inputs(8, 1536, 12, 2, 128, seed=3)
    for t, sc in [(0, 2.0 ** -20), (1, 2.0 ** -20), (5, 2.0 ** 10)]:
        d["x"][t] = (d["x"][t].astype(np.float32) * sc).astype(F16)
        d["residual"][t] = (d["residual"][t].astype(np.float32) * sc).astype(F16)
    d["x"][2] = 0
    d["residual"][2] = 0                    # an all-zero row gives the bias
    check(d, 12, 2, 128, what="tiny/huge rows")


def test_empty_batch_is_a_no_op():
    d = W.make_qkv_inputs(0, 1536, 12, 2, 128, seed=0)
    e = torch.empty((0, 1536), dtype=torch.float16, device="cuda")
    q = torch.empty((0, 12, 128), dtype=torch.float16, device="cuda")
    kv = [torch.empty((0, 2, 128), dtype=torch.float16, device="cuda") for _ in range(2)]
    pkv.fused_add_rmsnorm_qkv(e, e.clone(), dev(d["gamma"]), dev(d["w_qkv"]), dev(d["bias"]), e.clone(), q, *kv)
    assert pkv.pkv_device_error() == 0


def test_overlap_flag_gives_the_same_bytes():
    sh = W.QKV_SHAPES["qwen2.5-1.5b"]
    d = W.make_qkv_inputs(40, sh["H"], sh["Hq"], sh["Hkv"], sh["D"], seed=11)
    a = run_gpu(d, sh["Hq"], sh["Hkv"], sh["D"], W.RMS_EPS, 0)
    b = run_gpu(d, sh["Hq"], sh["Hkv"], sh["D"], W.RMS_EPS, pkv.PKV_STEP_OVERLAP_PREVIOUS)
    for x, y in zip(a, b):
        assert np.array_equal(x.view(np.uint16), y.view(np.uint16))


# ------------------------------------------------------------------ full sizes
@pytest.mark.parametrize("name", sorted(W.QKV_SHAPES))
def test_parity_full_size(name):
    """Batch and hidden size of the benchmark's model shapes; the 7B case is checked on sampled tokens."""
    sh = W.QKV_SHAPES[name]
    d = W.make_qkv_inputs(sh["T"], sh["H"], sh["Hq"], sh["Hkv"], sh["D"], seed=1)
    rows = None if sh["T"] <= 64 else np.random.default_rng(0).choice(sh["T"], 24, replace=False)
    check(d, sh["Hq"], sh["Hkv"], sh["D"], rows=rows, what=name)
    # the same call twice gives the same bytes (fixed summation order)
    a = run_gpu(d, sh["Hq"], sh["Hkv"], sh["D"], W.RMS_EPS)
    b = run_gpu(d, sh["Hq"], sh["Hkv"], sh["D"], W.RMS_EPS)
    for x, y in zip(a, b):
        assert np.array_equal(x.view(np.uint16), y.view(np.uint16))


def test_batch_256_of_the_small_model():
    d = W.make_qkv_inputs(256, 1536, 12, 2, 128, seed=5)
    check(d, 12, 2, 128, rows=np.arange(0, 256, 9), what="T=256")


# ------------------------------------------------------------------ feeding the decode step
def test_projection_feeds_the_fused_step():
    """q, k_new, v_new go straight into paged_gqa_decode_step: the cache rows it writes are the
    projection's k/v bytes and its attention matches the oracle on the projection's q."""
    w = W.with_sizes(W.WORKLOADS["qwen2.5-1.5b"], B=12, num_blocks=1024)
    x = W.make_inputs(w, 21)
    B, Hq, Hkv, D = w.B, w.Hq, w.Hkv, w.head_dim
    d = W.make_qkv_inputs(B, Hq * D, Hq, Hkv, D, seed=22)
    res = torch.empty((B, Hq * D), dtype=torch.float16, device="cuda")
    q = torch.empty((B, Hq, D), dtype=torch.float16, device="cuda")
    kn = torch.empty((B, Hkv, D), dtype=torch.float16, device="cuda")
    vn = torch.empty((B, Hkv, D), dtype=torch.float16, device="cuda")
    kc, vc = dev(x["k_pool"]), dev(x["v_pool"])
    ml = int(x["context_lens"].max())
    ws = torch.zeros(pkv.paged_gqa_decode_workspace_size(B, Hq, Hkv, D, ml, pkv.PKV_PARTITION_AUTO),
                     dtype=torch.uint8, device="cuda")
    out = torch.empty((B, Hq, D), dtype=torch.float16, device="cuda")
    pkv.fused_add_rmsnorm_qkv(dev(d["x"]), dev(d["residual"]), dev(d["gamma"]), dev(d["w_qkv"]), dev(d["bias"]),
                              res, q, kn, vn)
    pkv.paged_gqa_decode_step(out, q, kn, vn, kc, vc, dev(x["block_tables"]), dev(x["context_lens"]),
                              max_context_len=ml, softmax_scale=float(x["softmax_scale"]),
                              workspace=ws, flags=pkv.PKV_STEP_OVERLAP_PREVIOUS)
    kr, vr = x["k_pool"].copy(), x["v_pool"].copy()
    oracle.paged_kv_cache_write(host(kn), host(vn), kr, vr, x["slot_mapping"])
    got_k, got_v = host(kc), host(vc)
    assert np.array_equal(got_k.view(np.uint16), kr.view(np.uint16))
    assert np.array_equal(got_v.view(np.uint16), vr.view(np.uint16))
    ref = oracle.paged_gqa_decode(host(q), kr, vr, x["block_tables"], x["context_lens"], float(x["softmax_scale"]))
    from _gpu_helpers import assert_attention_close
    assert_attention_close(host(out), ref, "projection -> step")
    assert pkv.pkv_device_error() == 0
