"""The C-ABI library loads, exports every entry point include/pagedkv.h declares,
and rejects bad arguments on the host before any launch (no GPU needed)."""
import ctypes
import os
import re

import pytest

import paged_kv_decode_gqa_b200 as pkv

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "pagedkv.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?[\w]+\s*\*?\s*(\w+)\s*\(", text, flags=re.M)))


def test_header_declares_the_binding_entry_points():
    assert declared_functions() == sorted(pkv.EXPORTED)


def test_library_exports_every_declared_symbol():
    lib = pkv.load_library()
    for name in declared_functions():
        assert hasattr(lib, name), name


def test_status_strings():
    lib = pkv.load_library()
    for code in range(5):
        assert lib.pkv_status_string(code)
    assert lib.pkv_status_string(99) == b"unknown status"


def test_workspace_size():
    assert pkv.paged_gqa_decode_workspace_size(8, 28, 4, 128, 32768, 0) == 0
    n = pkv.paged_gqa_decode_workspace_size(8, 28, 4, 128, 32768, 512)
    rows = 8 * 28 * 64
    assert n >= rows * 128 * 4 + 2 * rows * 4 + 2 * 8 * 4 * 64 * 4   # two tree levels of tickets for 64 partitions
    assert n % 256 == 0
    assert pkv.paged_gqa_decode_workspace_size(8, 28, 4, 64, 32768, 512) == 0   # D != 128


def test_suggest_partition_is_a_multiple_of_the_page():
    for B, Hkv, L in [(64, 2, 2048), (128, 4, 4096), (256, 2, 8192), (8, 4, 32768), (1, 1, 64)]:
        P = pkv.paged_gqa_decode_suggest_partition(B, Hkv, L, 16, 148)
        assert P == 0 or (P % 16 == 0 and 16 <= P < L)
    assert pkv.paged_gqa_decode_suggest_partition(2, 2, 40, 16, 148) == 0


# Fake but aligned device pointers: every call below must be rejected by the
# host-side checks, before the library touches CUDA.
A = 1 << 20


def _attn(**kw):
    args = dict(out=A, q=A, k=A, v=A, bt=A, cl=A, B=2, Hq=12, Hkv=2, D=128, bs=16, mb=4, NB=64,
                maxlen=40, scale=0.088, dt=0, ks=1.0, vs=1.0, P=0, ws=0, wsb=0)
    args.update(kw)
    a = args
    return pkv.load_library().paged_gqa_decode_attention(
        a["out"], a["q"], a["k"], a["v"], a["bt"], a["cl"], a["B"], a["Hq"], a["Hkv"], a["D"], a["bs"],
        a["mb"], a["NB"], a["maxlen"], a["scale"], a["dt"], a["ks"], a["vs"], a["P"], a["ws"], a["wsb"],
        None)


@pytest.mark.parametrize("kw,status", [
    (dict(q=0), pkv.PKV_ERR_INVALID_ARG),
    (dict(out=A + 8), pkv.PKV_ERR_INVALID_ARG),            # misaligned
    (dict(Hq=13), pkv.PKV_ERR_INVALID_ARG),                # Hq % Hkv != 0
    (dict(Hq=20), pkv.PKV_ERR_UNSUPPORTED),                # group of 10 > 8
    (dict(D=64), pkv.PKV_ERR_UNSUPPORTED),
    (dict(bs=32, mb=2), pkv.PKV_ERR_UNSUPPORTED),
    (dict(maxlen=65), pkv.PKV_ERR_INVALID_ARG),            # > max_blocks * bs
    (dict(P=20), pkv.PKV_ERR_INVALID_ARG),                 # not a multiple of bs
    (dict(P=-2), pkv.PKV_ERR_INVALID_ARG),                 # below PKV_PARTITION_AUTO
    (dict(P=16), pkv.PKV_ERR_WORKSPACE),                   # split without workspace
    (dict(P=16, ws=A, wsb=64), pkv.PKV_ERR_WORKSPACE),     # too small
    (dict(dt=1, ks=0.0), pkv.PKV_ERR_INVALID_ARG),         # FP8 needs positive scales
    (dict(dt=7), pkv.PKV_ERR_INVALID_ARG),
    (dict(B=-1), pkv.PKV_ERR_INVALID_ARG),
    (dict(scale=float("nan")), pkv.PKV_ERR_INVALID_ARG),
    (dict(B=0), pkv.PKV_OK),                                # empty batch: nothing to do
])
def test_attention_rejects_bad_arguments_on_host(kw, status):
    assert _attn(**kw) == status


@pytest.mark.parametrize("kw,status", [
    (dict(k_new=0), pkv.PKV_ERR_INVALID_ARG),
    (dict(D=12), pkv.PKV_ERR_UNSUPPORTED),
    (dict(dt=1, ks=-1.0), pkv.PKV_ERR_INVALID_ARG),
    (dict(slots=A + 4), pkv.PKV_ERR_INVALID_ARG),
    (dict(T=0), pkv.PKV_OK),
])
def test_cache_write_rejects_bad_arguments_on_host(kw, status):
    a = dict(k_new=A, v_new=A, kc=A, vc=A, slots=A, T=4, Hkv=2, D=128, NB=64, bs=16, dt=0,
             ks=1.0, vs=1.0)
    a.update(kw)
    rc = pkv.load_library().paged_kv_cache_write(a["k_new"], a["v_new"], a["kc"], a["vc"], a["slots"],
                                                 a["T"], a["Hkv"], a["D"], a["NB"], a["bs"], a["dt"],
                                                 a["ks"], a["vs"], None)
    assert rc == status


@pytest.mark.parametrize("kw,status", [
    (dict(ks=0), pkv.PKV_ERR_INVALID_ARG),                 # device scales missing
    (dict(ks=A + 2), pkv.PKV_ERR_INVALID_ARG),             # misaligned float array
    (dict(per_head=2), pkv.PKV_ERR_INVALID_ARG),
    (dict(q=0), pkv.PKV_ERR_INVALID_ARG),                  # the attention checks still apply
    (dict(Hq=20), pkv.PKV_ERR_UNSUPPORTED),
    (dict(B=0), pkv.PKV_OK),
])
def test_fp8_scaled_attention_rejects_bad_arguments_on_host(kw, status):
    a = dict(out=A, q=A, k=A, v=A, bt=A, cl=A, B=2, Hq=12, Hkv=2, D=128, bs=16, mb=4, NB=64,
             maxlen=40, scale=0.088, ks=A, vs=A, per_head=1, P=0, ws=0, wsb=0)
    a.update(kw)
    rc = pkv.load_library().paged_gqa_decode_attention_fp8_scaled(
        a["out"], a["q"], a["k"], a["v"], a["bt"], a["cl"], a["B"], a["Hq"], a["Hkv"], a["D"], a["bs"],
        a["mb"], a["NB"], a["maxlen"], a["scale"], a["ks"], a["vs"], a["per_head"], a["P"], a["ws"],
        a["wsb"], None)
    assert rc == status


@pytest.mark.parametrize("kw,status", [
    (dict(vs=0), pkv.PKV_ERR_INVALID_ARG),
    (dict(per_head=-1), pkv.PKV_ERR_INVALID_ARG),
    (dict(D=12), pkv.PKV_ERR_UNSUPPORTED),
    (dict(T=0), pkv.PKV_OK),
])
def test_fp8_scaled_cache_write_rejects_bad_arguments_on_host(kw, status):
    a = dict(k_new=A, v_new=A, kc=A, vc=A, slots=A, T=4, Hkv=2, D=128, NB=64, bs=16, ks=A, vs=A, per_head=0)
    a.update(kw)
    rc = pkv.load_library().paged_kv_cache_write_fp8_scaled(
        a["k_new"], a["v_new"], a["kc"], a["vc"], a["slots"], a["T"], a["Hkv"], a["D"], a["NB"], a["bs"],
        a["ks"], a["vs"], a["per_head"], None)
    assert rc == status


@pytest.mark.parametrize("kw,status", [
    (dict(scales=0), pkv.PKV_ERR_INVALID_ARG),
    (dict(x=0), pkv.PKV_ERR_INVALID_ARG),
    (dict(x=A + 8), pkv.PKV_ERR_INVALID_ARG),              # chunks are 16-byte loads
    (dict(D=12), pkv.PKV_ERR_UNSUPPORTED),
    (dict(Hkv=2000), pkv.PKV_ERR_UNSUPPORTED),             # per-head maxima live in shared memory
    (dict(rows=-1), pkv.PKV_ERR_INVALID_ARG),
    (dict(per_head=3), pkv.PKV_ERR_INVALID_ARG),
])
def test_fp8_scales_rejects_bad_arguments_on_host(kw, status):
    a = dict(x=A, rows=64, Hkv=2, D=128, per_head=1, scales=A)
    a.update(kw)
    rc = pkv.load_library().paged_kv_fp8_scales(a["x"], a["rows"], a["Hkv"], a["D"], a["per_head"],
                                                a["scales"], None)
    assert rc == status


_QKV_BASE = 1 << 40                         # fake, 16-byte aligned, far apart
_QKV_PTRS = {n: _QKV_BASE + (i << 32) for i, n in enumerate(
    ("x", "residual", "gamma", "w", "bias", "res", "q", "k", "v"))}


@pytest.mark.parametrize("kw,status", [
    (dict(x=0), pkv.PKV_ERR_INVALID_ARG),
    (dict(w=0), pkv.PKV_ERR_INVALID_ARG),
    (dict(v=0), pkv.PKV_ERR_INVALID_ARG),
    (dict(q=_QKV_PTRS["q"] + 8), pkv.PKV_ERR_INVALID_ARG),        # 16-byte loads and stores
    (dict(bias=_QKV_PTRS["bias"] + 4), pkv.PKV_ERR_INVALID_ARG),
    (dict(res=_QKV_PTRS["residual"]), pkv.PKV_ERR_INVALID_ARG),   # in place: other CTAs still read it
    (dict(q=_QKV_PTRS["x"] + 1024), pkv.PKV_ERR_INVALID_ARG),     # an output inside an input
    (dict(k=_QKV_PTRS["q"] + 4096), pkv.PKV_ERR_INVALID_ARG),     # two outputs overlap
    (dict(T=-1), pkv.PKV_ERR_INVALID_ARG),
    (dict(Hkv=0), pkv.PKV_ERR_INVALID_ARG),
    (dict(eps=-1e-6), pkv.PKV_ERR_INVALID_ARG),
    (dict(eps=float("nan")), pkv.PKV_ERR_INVALID_ARG),
    (dict(flags=2), pkv.PKV_ERR_INVALID_ARG),
    (dict(H=1000), pkv.PKV_ERR_UNSUPPORTED),                     # H a multiple of 64
    (dict(H=8256), pkv.PKV_ERR_UNSUPPORTED),                     # above 8 slices of 16 blocks
    (dict(D=12), pkv.PKV_ERR_UNSUPPORTED),
    (dict(T=65535 * 64 + 1), pkv.PKV_ERR_UNSUPPORTED),
])
def test_qkv_rejects_bad_arguments_on_host(kw, status):
    a = dict(_QKV_PTRS, T=64, H=1536, Hq=12, Hkv=2, D=128, eps=1e-6, flags=0)
    a.update(kw)
    rc = pkv.load_library().fused_add_rmsnorm_qkv(
        a["x"], a["residual"], a["gamma"], a["w"], a["bias"], a["res"], a["q"], a["k"], a["v"],
        a["T"], a["H"], a["Hq"], a["Hkv"], a["D"], a["eps"], a["flags"], None)
    assert rc == status


def test_qkv_empty_batch_returns_before_any_cuda_call():
    a = _QKV_PTRS
    lib = pkv.load_library()
    rc = lib.fused_add_rmsnorm_qkv(a["x"], a["residual"], a["gamma"], a["w"], None, a["res"],
                                   a["q"], a["k"], a["v"], 0, 1536, 12, 2, 128, 1e-6, 0, None)
    assert rc == pkv.PKV_OK
    # empty per-token tensors may have null data pointers
    rc = lib.fused_add_rmsnorm_qkv(0, 0, a["gamma"], a["w"], None, 0, 0, 0, 0, 0, 1536, 12, 2, 128, 1e-6, 0, None)
    assert rc == pkv.PKV_OK
    rc = lib.fused_add_rmsnorm_qkv(a["x"], a["residual"], 0, a["w"], None, a["res"],
                                   a["q"], a["k"], a["v"], 0, 1536, 12, 2, 128, 1e-6, 0, None)
    assert rc == pkv.PKV_ERR_INVALID_ARG


@pytest.mark.parametrize("args,status", [
    ((64, 1536, 12, 2, 128, None), pkv.PKV_ERR_INVALID_ARG),
    ((0, 1536, 12, 2, 128, "buf"), pkv.PKV_ERR_INVALID_ARG),
    ((64, 1000, 12, 2, 128, "buf"), pkv.PKV_ERR_UNSUPPORTED),
    ((64, 1536, 12, 2, 12, "buf"), pkv.PKV_ERR_UNSUPPORTED),
])
def test_qkv_plan_rejects_bad_arguments_on_host(args, status):
    buf = (ctypes.c_int32 * 5)()
    a = list(args)
    a[5] = buf if a[5] == "buf" else None
    assert pkv.load_library().fused_add_rmsnorm_qkv_plan(*a) == status


@pytest.mark.parametrize("kw,status", [
    (dict(qs=0), pkv.PKV_ERR_INVALID_ARG),
    (dict(qs=A + 2), pkv.PKV_ERR_INVALID_ARG),
    (dict(out=0), pkv.PKV_ERR_INVALID_ARG),
    (dict(total=-1), pkv.PKV_ERR_INVALID_ARG),
    (dict(maxq=5000), pkv.PKV_ERR_INVALID_ARG),           # above max_context_len
    (dict(dtype=7), pkv.PKV_ERR_INVALID_ARG),
    (dict(D=64), pkv.PKV_ERR_UNSUPPORTED),
    (dict(Hq=36, Hkv=4), pkv.PKV_ERR_UNSUPPORTED),        # groups above 8
    (dict(total=0), pkv.PKV_OK),                          # nothing to do
])
def test_prefill_rejects_bad_arguments_on_host(kw, status):
    a = dict(out=A, q=A, k=A, v=A, bt=A, cl=A, qs=A, B=4, total=64, maxq=16, Hq=12, Hkv=2, D=128, bs=16,
             mb=256, nb=1024, maxc=4096, scale=0.088, dtype=0)
    a.update(kw)
    rc = pkv.load_library().paged_gqa_prefill_attention(
        a["out"], a["q"], a["k"], a["v"], a["bt"], a["cl"], a["qs"], a["B"], a["total"], a["maxq"], a["Hq"],
        a["Hkv"], a["D"], a["bs"], a["mb"], a["nb"], a["maxc"], a["scale"], a["dtype"], 1.0, 1.0, None, 0, None)
    assert rc == status


@pytest.mark.parametrize("args", [(0, 2, 128, 0), (12, 0, 128, 0), (12, 5, 128, 0), (12, 2, 64, 0),
                                  (36, 4, 128, 0), (12, 2, 128, 7), (12, 2, 128, 1)])
def test_prefill_workspace_size_zero_without_a_schedule_to_serve(args):
    """Invalid sizes and an FP8 cache (whose kernel takes no workspace) need none; the size of a valid
    f16 call needs the device's SM count, so it is checked on the GPU."""
    assert pkv.load_library().paged_gqa_prefill_workspace_size(*args) == 0


def test_prefill_flops_closed_form():
    """One sequence prefilled from an empty cache: sum over positions of 4 D Hq (p + 1)."""
    import bench
    L, Hq, D = 100, 12, 128
    assert bench.prefill_flops([L], [L], Hq, D) == 4 * D * Hq * L * (L + 1) // 2
    assert bench.prefill_flops([L], [1], Hq, D) == 4 * D * Hq * L            # decode


def test_measured_kv_read_cut_matches_the_pages_6x():
    """The page's 6x KV-bandwidth cut for Qwen2.5's 12 query / 2 KV heads, against DRAM bytes
    measured by ncu: the per-query-head launches together read 6x what the grouped kernel reads,
    within 5%, and the grouped kernel reads the KV about once."""
    import json
    g = json.load(open(os.path.join(ROOT, "tests", "golden", "qwen25_gqa_heads.json")))
    m = json.load(open(os.path.join(ROOT, "profiles", "gqa_kv_read_ratio.json")))
    per_head = m["per_query_head_dram_bytes_read"]
    assert len(per_head) == g["Hq"] // g["Hkv"]
    ratio = sum(per_head) / m["grouped_dram_bytes_read"]
    assert abs(ratio / g["kv_bandwidth_reduction"] - 1) <= 0.05, ratio
    assert 1.0 <= m["grouped_dram_bytes_read"] / m["algorithmic_kv_bytes_grouped"] <= 1.02


def test_header_macros_match_the_binding():
    text = open(HEADER).read()
    macros = {m: int(v, 0) for m, v in re.findall(r"#define\s+(PKV_\w+)\s+\(?([0-9x]+)u?\)?", text)}
    m = re.search(r"#define\s+PKV_STATIC_WORKSPACE_BYTES\s+\((\d+)u\s*<<\s*(\d+)\)", text)
    assert pkv.STATIC_WORKSPACE_BYTES == int(m.group(1)) << int(m.group(2))
    assert macros["PKV_STEP_OVERLAP_PREVIOUS"] == pkv.PKV_STEP_OVERLAP_PREVIOUS
    assert macros["PKV_STEP_SELFTEST_WAIT_TIMEOUT"] == pkv.PKV_STEP_SELFTEST_WAIT_TIMEOUT
    assert macros["PKV_DEVERR_WAIT_TIMEOUT"] == pkv.DEVERR_WAIT_TIMEOUT


def _step(flags, **kw):
    a = dict(out=A, q=A, kn=A, vn=A, k=A, v=A, bt=A, cl=A, B=2, Hq=12, Hkv=2, D=128, bs=16, mb=4, NB=64,
             maxlen=40, scale=0.088, dt=0, ks=1.0, vs=1.0, ws=0, wsb=0)
    a.update(kw)
    return pkv.load_library().paged_gqa_decode_step(
        a["out"], a["q"], a["kn"], a["vn"], a["k"], a["v"], a["bt"], a["cl"], a["B"], a["Hq"], a["Hkv"],
        a["D"], a["bs"], a["mb"], a["NB"], a["maxlen"], a["scale"], a["dt"], a["ks"], a["vs"], a["ws"],
        a["wsb"], flags, None)


@pytest.mark.parametrize("flags", [0x2, 0x200, 0x80000000])
def test_step_rejects_unknown_flags_on_host(flags):
    assert _step(flags) == pkv.PKV_ERR_INVALID_ARG


def test_static_workspace_entry_rejects_bad_arguments_on_host():
    lib = pkv.load_library()
    call = lambda **kw: lib.paged_gqa_decode_attention_static_workspace(
        *[kw.get(k, A) for k in ("out", "q", "k", "v", "bt", "cl")], kw.get("B", 2), 12, 2, kw.get("D", 128), 16,
        4, 64, 40, 0.088, 0, 1.0, 1.0, kw.get("P", 0), None)
    assert call(q=0) == pkv.PKV_ERR_INVALID_ARG
    assert call(D=64) == pkv.PKV_ERR_UNSUPPORTED
    assert call(P=20) == pkv.PKV_ERR_INVALID_ARG
    assert call(B=0) == pkv.PKV_OK
