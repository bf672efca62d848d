"""Shared helpers of the GPU parity tests: upload seeded inputs, run the CUDA
path through the C-ABI binding, run the oracle on the same host arrays, and
compare with the stated tolerance."""
import numpy as np
import torch

import oracle
import paged_kv_decode_gqa_b200 as pkv

# Attention tolerance: max |gpu - oracle| <= 2e-3 and that maximum <= 1e-2 of
# max |oracle| over the output tensor.
ATOL = 2e-3
RTOL_OF_MAX = 1e-2


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def host(t):
    return t.cpu().numpy()


def assert_attention_close(gpu_f16, ref_f64, what=""):
    g = np.asarray(gpu_f16, dtype=np.float64)
    assert g.shape == ref_f64.shape
    assert np.isfinite(g).all(), f"{what}: non-finite output"
    err = np.abs(g - ref_f64).max() if g.size else 0.0
    scale = np.abs(ref_f64).max() if g.size else 1.0
    assert err <= ATOL, f"{what}: max abs error {err:.3e} > {ATOL}"
    assert scale == 0 or err / scale <= RTOL_OF_MAX, f"{what}: max rel error {err / scale:.3e}"
    return err


def fp8_caches(x):
    """E4M3 codes of the workload's f16 pools, quantised by the oracle (tests only)."""
    kq = oracle.quantize_e4m3(x["k_pool"], float(x["k_scale"]))
    vq = oracle.quantize_e4m3(x["v_pool"], float(x["v_scale"]))
    return kq, vq


class DecodeRun:
    """The inputs of one workload on the device plus a call of the CUDA path."""

    def __init__(self, w, x, kv_dtype="f16", k_cache=None, v_cache=None):
        self.w, self.x, self.kv_dtype = w, x, kv_dtype
        if k_cache is None:
            k_cache, v_cache = x["k_pool"], x["v_pool"]
        self.k_host, self.v_host = k_cache, v_cache
        self.k = dev(k_cache)
        self.v = dev(v_cache)
        self.q = dev(x["q"])
        self.bt = dev(x["block_tables"])
        self.cl = dev(x["context_lens"])
        self.max_len = max(int(x["context_lens"].max()), 0) if x["context_lens"].size else 0
        self.max_len = max(self.max_len, 1)

    def attention(self, partition_tokens=0, q=None, bt=None, cl=None, k=None, v=None, max_len=None):
        q = self.q if q is None else q
        B, Hq, D = q.shape
        out = torch.full((B, Hq, D), float("nan"), dtype=torch.float16, device="cuda")
        max_len = self.max_len if max_len is None else max_len
        ws = None
        if partition_tokens:
            n = pkv.paged_gqa_decode_workspace_size(B, Hq, self.w.Hkv, D, max_len, partition_tokens)
            ws = torch.zeros(n, dtype=torch.uint8, device="cuda")
        pkv.paged_gqa_decode_attention(
            out, q, self.k if k is None else k, self.v if v is None else v,
            self.bt if bt is None else bt, self.cl if cl is None else cl,
            max_context_len=max_len, softmax_scale=float(self.x["softmax_scale"]),
            kv_dtype=self.kv_dtype, k_scale=float(self.x["k_scale"]), v_scale=float(self.x["v_scale"]),
            partition_tokens=partition_tokens, workspace=ws)
        torch.cuda.synchronize()
        return out

    def oracle(self, partition_tokens=0, seqs=None):
        x = self.x
        sel = slice(None) if seqs is None else np.asarray(seqs)
        return oracle.paged_gqa_decode(
            x["q"][sel], self.k_host, self.v_host, x["block_tables"][sel], x["context_lens"][sel],
            float(x["softmax_scale"]), kv_dtype=self.kv_dtype, k_scale=float(x["k_scale"]),
            v_scale=float(x["v_scale"]), partition_tokens=partition_tokens)
