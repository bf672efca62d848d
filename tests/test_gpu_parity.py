"""Parity of the CUDA path (through the C-ABI binding) with the float64 oracle.

Cache write: bit-exact. Attention: max |gpu - oracle| <= 2e-3 and <= 1e-2 of
max |oracle| (FP8: the oracle runs on the same E4M3 bytes). Sizes span several
stages of the shared-memory ring and ragged last blocks; the full workload
sizes run in the launch configuration the benchmark times, checked on sampled
sequences.
"""
import numpy as np
import pytest
import torch

import oracle
import paged_kv_decode_gqa_b200 as pkv
import workloads as W
from _gpu_helpers import DecodeRun, assert_attention_close, dev, fp8_caches, host

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _clear_device_error():
    pkv.pkv_device_error()
    yield
    torch.cuda.synchronize()


def _run(w, seed, kv_dtype=None):
    x = W.make_inputs(w, seed)
    kv_dtype = kv_dtype or w.kv_dtype
    if kv_dtype == "fp8":
        kq, vq = fp8_caches(x)
        return DecodeRun(w, x, "fp8", kq, vq)
    return DecodeRun(w, x)


# ------------------------------------------------------------------ cache write
def _cache_write_case(w, seed, kv_dtype):
    x = W.make_inputs(w, seed)
    if kv_dtype == "fp8":
        kc, vc = fp8_caches(x)
    else:
        kc, vc = x["k_pool"], x["v_pool"]
    slots = x["slot_mapping"].copy()
    if slots.size > 2:
        slots[1] = -1                                       # padding token: skipped
    k_dev, v_dev = dev(kc), dev(vc)
    pkv.paged_kv_cache_write(dev(x["k_new"]), dev(x["v_new"]), k_dev, v_dev, dev(slots),
                             kv_dtype=kv_dtype, k_scale=float(x["k_scale"]), v_scale=float(x["v_scale"]))
    kr, vr = kc.copy(), vc.copy()
    oracle.paged_kv_cache_write(x["k_new"], x["v_new"], kr, vr, slots, kv_dtype=kv_dtype,
                                k_scale=float(x["k_scale"]), v_scale=float(x["v_scale"]))
    view = (lambda a: a.view(np.uint16)) if kv_dtype == "f16" else (lambda a: a)
    assert np.array_equal(view(host(k_dev)), view(kr))
    assert np.array_equal(view(host(v_dev)), view(vr))
    assert pkv.pkv_device_error() == 0


@pytest.mark.parametrize("kv_dtype", ["f16", "fp8"])
def test_cache_write_tiny_bit_exact(kv_dtype):
    _cache_write_case(W.WORKLOADS["tiny"], 0, kv_dtype)


@pytest.mark.parametrize("kv_dtype", ["f16", "fp8"])
def test_cache_write_7b_step_bit_exact(kv_dtype):
    """128 new tokens into the full 32k-block pool (Qwen2.5-7B shape), whole caches compared."""
    w = W.WORKLOADS["qwen2.5-7b"]
    if kv_dtype == "fp8":
        w = W.with_sizes(w, kv_dtype="fp8")
    _cache_write_case(w, 1, kv_dtype)


@pytest.mark.parametrize("scale", [1.0, 0.0078125, 0.0133, 3.7])
def test_cache_write_fp8_every_f16_value(scale):
    """Every finite f16 value (and +-inf, NaN) through the device quantiser, compared bytewise."""
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    vals = bits.view(np.float16)
    n = -(-vals.size // 128) * 128
    flat = np.zeros(n, dtype=np.float16)
    flat[:vals.size] = vals
    T = n // 128
    k_new = flat.reshape(T, 1, 128)
    v_new = k_new[::-1].copy()
    NB = -(-T // 16)
    kc = np.zeros((NB, 16, 1, 128), np.uint8)
    vc = np.zeros_like(kc)
    slots = np.arange(T, dtype=np.int64)
    k_dev, v_dev = dev(kc), dev(vc)
    pkv.paged_kv_cache_write(dev(k_new), dev(v_new), k_dev, v_dev, dev(slots), kv_dtype="fp8",
                             k_scale=scale, v_scale=scale)
    kr, vr = kc.copy(), vc.copy()
    oracle.paged_kv_cache_write(k_new, v_new, kr, vr, slots, kv_dtype="fp8", k_scale=scale,
                                v_scale=scale)
    assert np.array_equal(host(k_dev), kr)
    assert np.array_equal(host(v_dev), vr)


def test_cache_write_flags_slot_outside_pool():
    kc = torch.zeros((4, 16, 1, 128), dtype=torch.float16, device="cuda")
    vc = torch.zeros_like(kc)
    kn = torch.ones((2, 1, 128), dtype=torch.float16, device="cuda")
    slots = torch.tensor([3, 64], dtype=torch.int64, device="cuda")
    pkv.paged_kv_cache_write(kn, kn, kc, vc, slots)
    assert pkv.pkv_device_error() == pkv.DEVERR_SLOT
    assert kc[0, 3].eq(1).all() and kc.sum().item() == 128


# ------------------------------------------------------------- attention parity
AUTO = pkv.PKV_PARTITION_AUTO


@pytest.mark.parametrize("P", [0, 16, 32, AUTO])
@pytest.mark.parametrize("seed", [0, 1, 2])
def test_tiny_config_f16(P, seed):
    r = _run(W.WORKLOADS["tiny"], seed)
    assert_attention_close(host(r.attention(P)), r.oracle(), f"tiny P={P}")
    assert pkv.pkv_device_error() == 0


REDUCED = {
    "qwen2.5-1.5b": dict(B=8),
    "qwen2.5-7b": dict(B=6, num_blocks=2048),
    "fp8-e4m3": dict(B=4, num_blocks=4096, ctx=("uniform", 17, 2600)),
    "skewed-split": dict(B=4, num_blocks=1024, ctx=("skewed", 4100, 3, 1, 700)),
}


@pytest.mark.parametrize("name", sorted(REDUCED))
@pytest.mark.parametrize("P", [0, 64, 512, AUTO])
def test_reduced_configs(name, P):
    w = W.with_sizes(W.WORKLOADS[name], **REDUCED[name])
    for seed in (0, 3):
        r = _run(w, seed)
        assert_attention_close(host(r.attention(P)), r.oracle(), f"{name} P={P} seed={seed}")
    assert pkv.pkv_device_error() == 0


@pytest.mark.parametrize("name", ["qwen2.5-1.5b", "qwen2.5-7b", "fp8-e4m3", "skewed-split"])
def test_full_size_configs_sampled(name):
    """Full workload on the device in the benchmark's plan; oracle on sampled sequences."""
    w = W.WORKLOADS[name]
    r = _run(w, 0)
    lens = r.x["context_lens"]
    rng = np.random.default_rng(5)
    seqs = sorted(set([int(np.argmax(lens)), int(np.argmin(lens))]
                      + list(rng.choice(w.B, size=min(w.B, 6), replace=False))))
    ref = r.oracle(seqs=seqs)
    P_bench = w.partition_tokens or pkv.paged_gqa_decode_suggest_partition(w.B, w.Hkv, r.max_len)
    for P in sorted({0, P_bench, AUTO}):
        out = host(r.attention(P))
        assert_attention_close(out[seqs], ref, f"{name} P={P}")
    assert pkv.pkv_device_error() == 0


# ------------------------------------------------------- invariants and edges
def test_context_one_is_exactly_v0():
    w = W.with_sizes(W.WORKLOADS["qwen2.5-7b"], B=5, num_blocks=64, ctx=("fixed", (1, 1, 1, 1, 1)))
    r = _run(w, 2)
    out = host(r.attention())
    for b in range(w.B):
        blk = r.x["block_tables"][b, 0]
        v0 = r.x["v_pool"][blk, 0]                          # [Hkv, D]
        assert np.array_equal(out[b].view(np.uint16), np.repeat(v0, w.group, axis=0).view(np.uint16))


def test_block_permutation_invariance_bitwise():
    w = W.with_sizes(W.WORKLOADS["qwen2.5-1.5b"], B=6, num_blocks=1024)
    r = _run(w, 4)
    out1 = host(r.attention(128))
    auto1 = host(r.attention(AUTO))
    perm = np.random.default_rng(9).permutation(w.num_blocks)
    k2 = np.empty_like(r.k_host); v2 = np.empty_like(r.v_host)
    k2[perm] = r.k_host; v2[perm] = r.v_host
    bt = r.x["block_tables"]
    bt2 = np.where(bt >= 0, perm[np.maximum(bt, 0)], -1).astype(np.int32)
    out2 = host(r.attention(128, bt=dev(bt2), k=dev(k2), v=dev(v2)))
    assert np.array_equal(out1.view(np.uint16), out2.view(np.uint16))
    auto2 = host(r.attention(AUTO, bt=dev(bt2), k=dev(k2), v=dev(v2)))
    assert np.array_equal(auto1.view(np.uint16), auto2.view(np.uint16))


def test_split_with_partition_covering_context_is_bitwise_single_pass():
    w = W.with_sizes(W.WORKLOADS["qwen2.5-7b"], B=4, num_blocks=2048)
    r = _run(w, 6)
    single = host(r.attention(0))
    P = -(-r.max_len // 16) * 16
    assert np.array_equal(single.view(np.uint16), host(r.attention(P)).view(np.uint16))


def test_split_equals_single_within_tolerance_and_workspace_reuse():
    w = W.with_sizes(W.WORKLOADS["skewed-split"], B=4, num_blocks=1024, ctx=("skewed", 5000, 3, 16, 900))
    r = _run(w, 7)
    ref = r.oracle()
    B, Hq, D = r.q.shape
    for P in (256, AUTO):
        n = pkv.paged_gqa_decode_workspace_size(B, Hq, w.Hkv, D, r.max_len, P)
        ws = torch.zeros(n, dtype=torch.uint8, device="cuda")
        outs = []
        for _ in range(3):                                  # the same workspace, reused
            out = torch.empty((B, Hq, D), dtype=torch.float16, device="cuda")
            pkv.paged_gqa_decode_attention(out, r.q, r.k, r.v, r.bt, r.cl, max_context_len=r.max_len,
                                           softmax_scale=float(r.x["softmax_scale"]),
                                           partition_tokens=P, workspace=ws)
            outs.append(host(out))
        for o in outs:
            assert_attention_close(o, ref, f"split {P}")
            assert np.array_equal(o.view(np.uint16), outs[0].view(np.uint16))
    assert_attention_close(host(r.attention(0)), ref, "single")


def test_poison_never_read_bitwise():
    w = W.with_sizes(W.WORKLOADS["qwen2.5-7b"], B=6, num_blocks=2048, ctx=("uniform", 1, 300))
    xa = W.make_inputs(w, 8, poison=True)
    xb = W.make_inputs(w, 8, poison=False)
    ra, rb = DecodeRun(w, xa), DecodeRun(w, xb)
    for P in (0, 64, AUTO):
        a, b = host(ra.attention(P)), host(rb.attention(P))
        assert np.isfinite(a.astype(np.float32)).all()
        assert np.array_equal(a.view(np.uint16), b.view(np.uint16))


def test_fp8_poison_code_never_read():
    w = W.with_sizes(W.WORKLOADS["fp8-e4m3"], B=5, num_blocks=1024, ctx=("uniform", 1, 200))
    x = W.make_inputs(w, 9)
    kq, vq = fp8_caches(x)                                  # NaN rows quantise to 0x7F
    assert (kq == 0x7F).any()
    r = DecodeRun(w, x, "fp8", kq, vq)
    for P in (0, 32, AUTO):
        assert_attention_close(host(r.attention(P)), r.oracle(), f"fp8 poison P={P}")


def test_head_map_contiguous_groups():
    w = W.with_sizes(W.WORKLOADS["qwen2.5-7b"], B=3, num_blocks=1024)
    x = W.make_inputs(w, 10, poison=False)
    x["v_pool"][:] = np.arange(w.Hkv, dtype=np.float16)[None, None, :, None]
    r = DecodeRun(w, x)
    expect = np.repeat(np.arange(w.Hkv, dtype=np.float64), w.group)[None, :, None]
    for P in (64, AUTO):
        out = host(r.attention(P)).astype(np.float64)
        assert np.array_equal(out, np.broadcast_to(expect, out.shape))


@pytest.mark.parametrize("Hq,Hkv", [(4, 4), (8, 4), (16, 4), (14, 2), (8, 1), (32, 4)])
def test_group_sizes(Hq, Hkv):
    w = W.with_sizes(W.WORKLOADS["qwen2.5-7b"], B=3, Hq=Hq, Hkv=Hkv, num_blocks=1024,
                     ctx=("uniform", 1, 1000))
    r = _run(w, 11)
    for P in (0, 128, AUTO):
        assert_attention_close(host(r.attention(P)), r.oracle(), f"Hq={Hq} Hkv={Hkv} P={P}")


def test_empty_contexts_give_zero_rows():
    w = W.with_sizes(W.WORKLOADS["qwen2.5-1.5b"], B=4, num_blocks=512, ctx=("fixed", (0, 33, 0, 700)))
    r = _run(w, 12)
    for P in (0, 64, AUTO):
        out = host(r.attention(P))
        assert not out[0].any() and not out[2].any()
        assert_attention_close(out, r.oracle(), f"empty P={P}")


def test_all_contexts_empty_and_zero_max_len():
    w = W.with_sizes(W.WORKLOADS["tiny"], ctx=("fixed", (0, 0)))
    r = _run(w, 0)
    for P in (0, AUTO):
        out = host(r.attention(P, max_len=0))
        assert not out.any()


def test_bad_block_id_and_length_are_flagged_not_faulted():
    w = W.with_sizes(W.WORKLOADS["tiny"])
    r = _run(w, 1)
    bt = r.x["block_tables"].copy()
    bt[1, 0] = w.num_blocks + 5                              # outside the pool: reads zeros
    r.attention(0, bt=dev(bt))
    assert pkv.pkv_device_error() == pkv.DEVERR_BLOCK_ID
    cl = r.x["context_lens"].copy()
    cl[0] = 10_000                                           # beyond max_context_len: clamped
    r.attention(0, cl=dev(cl))
    # clamped to 40 tokens, sequence 0 (17 live tokens) also reaches its unused
    # third table entry (-1), which is flagged as well
    assert pkv.pkv_device_error() == pkv.DEVERR_CONTEXT_LEN | pkv.DEVERR_BLOCK_ID


def test_step_captured_in_cuda_graph():
    """Cache write + attention captured once and replayed on the caller's stream."""
    w = W.with_sizes(W.WORKLOADS["qwen2.5-1.5b"], B=8, num_blocks=2048)
    x = W.make_inputs(w, 13)
    r = DecodeRun(w, x)
    P = AUTO
    B, Hq, D = r.q.shape
    ws = torch.zeros(pkv.paged_gqa_decode_workspace_size(B, Hq, w.Hkv, D, r.max_len, P),
                     dtype=torch.uint8, device="cuda")
    out = torch.empty((B, Hq, D), dtype=torch.float16, device="cuda")
    kn, vn, sl = dev(x["k_new"]), dev(x["v_new"]), dev(x["slot_mapping"])

    def step():
        pkv.paged_kv_cache_write(kn, vn, r.k, r.v, sl)
        pkv.paged_gqa_decode_attention(out, r.q, r.k, r.v, r.bt, r.cl, max_context_len=r.max_len,
                                       softmax_scale=float(x["softmax_scale"]), partition_tokens=P,
                                       workspace=ws)

    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        step()                                               # warm-up (attribute set-up, maps)
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        step()
    out.fill_(float("nan"))
    g.replay()
    torch.cuda.synchronize()
    kr, vr = x["k_pool"].copy(), x["v_pool"].copy()
    oracle.paged_kv_cache_write(x["k_new"], x["v_new"], kr, vr, x["slot_mapping"])
    ref = oracle.paged_gqa_decode(x["q"], kr, vr, x["block_tables"], x["context_lens"],
                                  float(x["softmax_scale"]))
    assert_attention_close(host(out), ref, "graph replay")
    del g


# ------------------------------------------------------- the balanced plan
def test_auto_many_short_sequences():
    """Thousands of 1..40-token sequences: many whole segments per worker."""
    w = W.with_sizes(W.WORKLOADS["qwen2.5-1.5b"], B=3000, num_blocks=9000, ctx=("uniform", 1, 40))
    r = _run(w, 14)
    seqs = np.random.default_rng(1).choice(w.B, 200, replace=False)
    out = host(r.attention(AUTO))
    assert_attention_close(out[np.sort(seqs)], r.oracle(seqs=np.sort(seqs)), "auto short")
    assert pkv.pkv_device_error() == 0


@pytest.mark.parametrize("kv_dtype", ["f16", "fp8"])
def test_auto_many_segments_per_cta(kv_dtype):
    """1500 sequences of 1..100 tokens: a few dozen segments per SM's range, most of them
    split over several consumer warps, so the per-CTA accumulators are reused many times."""
    base = W.WORKLOADS["fp8-e4m3" if kv_dtype == "fp8" else "qwen2.5-1.5b"]
    w = W.with_sizes(base, B=1500, num_blocks=12000, ctx=("uniform", 1, 100))
    r = _run(w, 17)
    seqs = np.sort(np.random.default_rng(2).choice(w.B, 150, replace=False))
    out = host(r.attention(AUTO))
    assert_attention_close(out[seqs], r.oracle(seqs=seqs), f"auto many segments {kv_dtype}")
    assert pkv.pkv_device_error() == 0


def test_auto_one_sequence_split_over_many_workers():
    """One 32k-token sequence among short ones: its segments span hundreds of workers."""
    w = W.with_sizes(W.WORKLOADS["skewed-split"], B=3, num_blocks=4096, ctx=("skewed", 32768, 2, 1, 50))
    r = _run(w, 15)
    assert_attention_close(host(r.attention(AUTO)), r.oracle(), "auto long")


@pytest.mark.parametrize("kv_dtype", ["f16", "fp8"])
@pytest.mark.parametrize("P", [16, 64, 512])
def test_fixed_partitions_merge_tree(P, kv_dtype):
    """One 32k-token sequence in 2048, 512 or 64 partitions: a merge tree of fan-in 8 with 4, 3 or
    2 levels and ragged groups, beside short one-partition sequences. The same workspace serves a
    second call (every ticket back at zero) with the same bytes."""
    base = "skewed-split" if kv_dtype == "f16" else "fp8-e4m3"
    w = W.with_sizes(W.WORKLOADS[base], B=3, num_blocks=4096, ctx=("skewed", 32768, 2, 1, 50))
    r = _run(w, 16)
    B, Hq, D = r.q.shape
    n = pkv.paged_gqa_decode_workspace_size(B, Hq, w.Hkv, D, r.max_len, P)
    ws = torch.zeros(n, dtype=torch.uint8, device="cuda")
    outs = []
    for _ in range(2):
        out = torch.full((B, Hq, D), float("nan"), dtype=torch.float16, device="cuda")
        pkv.paged_gqa_decode_attention(out, r.q, r.k, r.v, r.bt, r.cl, max_context_len=r.max_len,
                                       softmax_scale=float(r.x["softmax_scale"]), kv_dtype=r.kv_dtype,
                                       k_scale=float(r.x["k_scale"]), v_scale=float(r.x["v_scale"]),
                                       partition_tokens=P, workspace=ws)
        outs.append(host(out))
    assert_attention_close(outs[0], r.oracle(), f"tree P={P} {kv_dtype}")
    assert np.array_equal(outs[0].view(np.uint16), outs[1].view(np.uint16))
    assert pkv.pkv_device_error() == 0


def test_auto_fp8_batch_beyond_its_tables_falls_back():
    """4000 sequences: the FP8 balanced tables no longer fit in shared memory while the f16
    ones do, so FP8 runs fixed partitions inside the workspace sized for the automatic plan."""
    w = W.with_sizes(W.WORKLOADS["fp8-e4m3"], B=4000, num_blocks=12000, ctx=("uniform", 1, 40))
    r = _run(w, 18)
    seqs = np.arange(0, w.B, 20)
    out = host(r.attention(AUTO))
    assert_attention_close(out[seqs], r.oracle(seqs=seqs), "auto fp8 fallback")
    assert pkv.pkv_device_error() == 0


def test_auto_batch_beyond_balanced_tables_falls_back():
    w = W.with_sizes(W.WORKLOADS["qwen2.5-1.5b"], B=9000, num_blocks=20000, ctx=("uniform", 1, 40))
    r = _run(w, 16)
    seqs = np.arange(0, w.B, 45)
    out = host(r.attention(AUTO))
    assert_attention_close(out[seqs], r.oracle(seqs=seqs), "auto fallback")


# ------------------------------------------------------- fused decode step
def _step(r, kn, vn, ws=None, flags=0):
    B, Hq, D = r.q.shape
    out = torch.full((B, Hq, D), float("nan"), dtype=torch.float16, device="cuda")
    if ws is None:
        ws = torch.zeros(pkv.paged_gqa_decode_workspace_size(B, Hq, r.w.Hkv, D, r.max_len, AUTO),
                         dtype=torch.uint8, device="cuda")
    pkv.paged_gqa_decode_step(out, r.q, kn, vn, r.k, r.v, r.bt, r.cl, max_context_len=r.max_len,
                              softmax_scale=float(r.x["softmax_scale"]), kv_dtype=r.kv_dtype,
                              k_scale=float(r.x["k_scale"]), v_scale=float(r.x["v_scale"]), workspace=ws,
                              flags=flags)
    torch.cuda.synchronize()
    return out


STEP_CASES = {
    "tiny": {},
    "qwen2.5-1.5b": dict(B=8),
    "qwen2.5-7b": dict(B=6, num_blocks=2048),
    "fp8-e4m3": dict(B=4, num_blocks=4096, ctx=("uniform", 1, 2600)),
    "skewed-split": dict(B=4, num_blocks=1024, ctx=("skewed", 4100, 3, 1, 700)),
}


@pytest.mark.parametrize("flags", [0, pkv.PKV_STEP_OVERLAP_PREVIOUS])
@pytest.mark.parametrize("name", sorted(STEP_CASES))
def test_fused_step_writes_cache_and_matches_oracle(name, flags):
    w = W.with_sizes(W.WORKLOADS[name], **STEP_CASES[name])
    r = _run(w, 17)
    x = r.x
    out = host(_step(r, dev(x["k_new"]), dev(x["v_new"]), flags=flags))
    kr, vr = r.k_host.copy(), r.v_host.copy()
    oracle.paged_kv_cache_write(x["k_new"], x["v_new"], kr, vr, x["slot_mapping"], kv_dtype=r.kv_dtype,
                                k_scale=float(x["k_scale"]), v_scale=float(x["v_scale"]))
    view = (lambda a: a.view(np.uint16)) if r.kv_dtype == "f16" else (lambda a: a)
    assert np.array_equal(view(host(r.k)), view(kr))
    assert np.array_equal(view(host(r.v)), view(vr))
    ref = oracle.paged_gqa_decode(x["q"], kr, vr, x["block_tables"], x["context_lens"],
                                  float(x["softmax_scale"]), kv_dtype=r.kv_dtype,
                                  k_scale=float(x["k_scale"]), v_scale=float(x["v_scale"]))
    assert_attention_close(out, ref, f"step {name}")
    assert pkv.pkv_device_error() == 0


@pytest.mark.parametrize("name", ["qwen2.5-1.5b", "fp8-e4m3"])
def test_fused_step_equals_write_then_attention_bitwise(name):
    w = W.with_sizes(W.WORKLOADS[name], **STEP_CASES[name])
    x = W.make_inputs(w, 18)
    if w.kv_dtype == "fp8":
        kq, vq = fp8_caches(x)
        r1, r2 = DecodeRun(w, x, "fp8", kq, vq), DecodeRun(w, x, "fp8", kq, vq)
    else:
        r1, r2 = DecodeRun(w, x), DecodeRun(w, x)
    fused = host(_step(r1, dev(x["k_new"]), dev(x["v_new"])))
    pkv.paged_kv_cache_write(dev(x["k_new"]), dev(x["v_new"]), r2.k, r2.v, dev(x["slot_mapping"]),
                             kv_dtype=w.kv_dtype, k_scale=float(x["k_scale"]), v_scale=float(x["v_scale"]))
    two = host(r2.attention(AUTO))
    assert np.array_equal(fused.view(np.uint16), two.view(np.uint16))
    bits = (lambda t: t.view(torch.int16)) if w.kv_dtype == "f16" else (lambda t: t)
    assert torch.equal(bits(r1.k), bits(r2.k)) and torch.equal(bits(r1.v), bits(r2.v))


@pytest.mark.parametrize("name", ["qwen2.5-1.5b", "qwen2.5-7b", "fp8-e4m3", "skewed-split"])
def test_fused_step_full_size_sampled(name):
    w = W.WORKLOADS[name]
    r = _run(w, 19)
    x = r.x
    out = host(_step(r, dev(x["k_new"]), dev(x["v_new"])))
    lens = x["context_lens"]
    seqs = np.array(sorted(set([int(np.argmax(lens)), int(np.argmin(lens))]
                               + list(np.random.default_rng(6).choice(w.B, min(w.B, 6), replace=False)))))
    kr, vr = r.k_host, r.v_host                          # updated in place: only the new rows change
    oracle.paged_kv_cache_write(x["k_new"], x["v_new"], kr, vr, x["slot_mapping"], kv_dtype=r.kv_dtype,
                                k_scale=float(x["k_scale"]), v_scale=float(x["v_scale"]))
    ref = oracle.paged_gqa_decode(x["q"][seqs], kr, vr, x["block_tables"][seqs], lens[seqs],
                                  float(x["softmax_scale"]), kv_dtype=r.kv_dtype,
                                  k_scale=float(x["k_scale"]), v_scale=float(x["v_scale"]))
    assert_attention_close(out[seqs], ref, f"step full {name}")
    assert pkv.pkv_device_error() == 0


def test_fused_step_empty_contexts_and_graph_replay():
    w = W.with_sizes(W.WORKLOADS["qwen2.5-7b"], B=5, num_blocks=1024, ctx=("fixed", (0, 33, 0, 700, 16)))
    x = W.make_inputs(w, 20)
    r = DecodeRun(w, x)
    B, Hq, D = r.q.shape
    ws = torch.zeros(pkv.paged_gqa_decode_workspace_size(B, Hq, w.Hkv, D, r.max_len, AUTO),
                     dtype=torch.uint8, device="cuda")
    kn, vn = dev(x["k_new"]), dev(x["v_new"])
    _step(r, kn, vn, ws)                                   # warm-up outside the capture
    g = torch.cuda.CUDAGraph()
    out = torch.empty((B, Hq, D), dtype=torch.float16, device="cuda")
    with torch.cuda.graph(g):
        pkv.paged_gqa_decode_step(out, r.q, kn, vn, r.k, r.v, r.bt, r.cl, max_context_len=r.max_len,
                                  softmax_scale=float(x["softmax_scale"]), workspace=ws)
    out.fill_(float("nan"))
    g.replay()
    torch.cuda.synchronize()
    kr, vr = x["k_pool"].copy(), x["v_pool"].copy()
    oracle.paged_kv_cache_write(x["k_new"], x["v_new"], kr, vr, x["slot_mapping"])
    ref = oracle.paged_gqa_decode(x["q"], kr, vr, x["block_tables"], x["context_lens"],
                                  float(x["softmax_scale"]))
    o = host(out)
    assert not o[0].any() and not o[2].any()
    assert_attention_close(o, ref, "step graph")
    del g


def test_fused_steps_back_to_back_with_overlap_flag():
    """Steps on alternating pools with PKV_STEP_OVERLAP_PREVIOUS, in a graph: each
    step's output matches the oracle (the promise holds: consecutive steps use
    different pools and tables)."""
    w = W.with_sizes(W.WORKLOADS["qwen2.5-1.5b"], B=16, num_blocks=2048)
    xs = [W.make_inputs(w, 30 + i) for i in range(2)]
    rs = [DecodeRun(w, x) for x in xs]
    B, Hq, D = rs[0].q.shape
    ws = torch.zeros(pkv.paged_gqa_decode_workspace_size(B, Hq, w.Hkv, D, 2048, AUTO),
                     dtype=torch.uint8, device="cuda")
    outs = [torch.empty((B, Hq, D), dtype=torch.float16, device="cuda") for _ in range(2)]
    kns = [(dev(x["k_new"]), dev(x["v_new"])) for x in xs]

    def steps():
        for i in range(6):
            r, (kn, vn) = rs[i % 2], kns[i % 2]
            pkv.paged_gqa_decode_step(outs[i % 2], r.q, kn, vn, r.k, r.v, r.bt, r.cl, max_context_len=2048,
                                      softmax_scale=float(r.x["softmax_scale"]), workspace=ws,
                                      flags=pkv.PKV_STEP_OVERLAP_PREVIOUS)

    steps()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        steps()
    for o in outs:
        o.fill_(float("nan"))
    g.replay()
    torch.cuda.synchronize()
    for i, (x, o) in enumerate(zip(xs, outs)):
        kr, vr = x["k_pool"].copy(), x["v_pool"].copy()
        oracle.paged_kv_cache_write(x["k_new"], x["v_new"], kr, vr, x["slot_mapping"])
        ref = oracle.paged_gqa_decode(x["q"], kr, vr, x["block_tables"], x["context_lens"],
                                      float(x["softmax_scale"]))
        assert_attention_close(host(o), ref, f"overlapped steps, pool {i}")
    del g
