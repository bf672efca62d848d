"""Pins of the float64 oracle to things other than itself.

Every check here compares the oracle with an independent statement of the
result: a library routine (NumPy's binary16, torch's float8_e4m3fn), a dense
NumPy brute force over contiguous (unpaged) K/V, a closed form, or an
invariant of the definition (paged decode attention as the pages describe it:
"rvLLM 소개" (discuss.pytorch.kr), §PagedAttention과 FlashAttention-3, and the
vLLM talk summary (aitrends.kr), §용어 해설). Mistakes a plausible bug would
make -- a dropped term, a transposed operand, a wrong head or block index, a
sign error in the merge -- each fail at least one test below.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import workloads as W

RTOL_DENSE = 1e-12


# ----------------------------------------------------------------- helpers
def dense_attention(q, K, V, scale):
    """Contiguous GQA attention by dense NumPy ops: q [Hq,D], K/V [L,Hkv,D] (f64)."""
    Hq, Hkv = q.shape[0], K.shape[1]
    G = Hq // Hkv
    Kr = np.repeat(K, G, axis=1)          # [L, Hq, D]  (query head h -> KV head h // G)
    Vr = np.repeat(V, G, axis=1)
    s = scale * np.einsum("hd,lhd->hl", q, Kr)
    s = s - s.max(axis=1, keepdims=True)
    p = np.exp(s)
    p /= p.sum(axis=1, keepdims=True)
    return np.einsum("hl,lhd->hd", p, Vr)


def paged_from_contiguous(Ks, Vs, bs, NB, rng, fill=np.nan):
    """Scatter per-sequence contiguous K/V ([L,Hkv,D] each) into a shuffled pool."""
    Hkv, D = Ks[0].shape[1], Ks[0].shape[2]
    dtype = Ks[0].dtype
    kp = np.full((NB, bs, Hkv, D), fill, dtype=dtype)
    vp = np.full((NB, bs, Hkv, D), fill, dtype=dtype)
    nbs = [-(-k.shape[0] // bs) for k in Ks]
    mb = max(max(nbs), 1)
    bt = np.full((len(Ks), mb), -1, dtype=np.int32)
    perm = rng.permutation(NB)
    pos = 0
    for b, (k, v) in enumerate(zip(Ks, Vs)):
        for j in range(nbs[b]):
            phys = int(perm[pos]); pos += 1
            bt[b, j] = phys
            rows = slice(j * bs, min((j + 1) * bs, k.shape[0]))
            n = rows.stop - rows.start
            kp[phys, :n] = k[rows]
            vp[phys, :n] = v[rows]
    return kp, vp, bt


def random_case(rng, lens, Hq, Hkv, D=16, bs=4, extra_blocks=5):
    Ks = [rng.standard_normal((L, Hkv, D)).astype(np.float16) for L in lens]
    Vs = [rng.standard_normal((L, Hkv, D)).astype(np.float16) for L in lens]
    q = rng.standard_normal((len(lens), Hq, D)).astype(np.float16)
    NB = sum(-(-L // bs) for L in lens) + extra_blocks
    kp, vp, bt = paged_from_contiguous(Ks, Vs, bs, NB, rng)
    return q, Ks, Vs, kp, vp, bt, np.array(lens, dtype=np.int32)


def e4m3_table_torch():
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    return codes.view(torch.float8_e4m3fn).to(torch.float32).double().numpy()


def e4m3_round_bruteforce(x):
    """Nearest finite E4M3 value to fp32 x, ties to the even code, clamp at 448."""
    tab = e4m3_table_torch()
    finite = [c for c in range(0x7F) if np.isfinite(tab[c])]      # 0x00..0x7E
    a = abs(float(x))
    best = min(finite, key=lambda c: (abs(tab[c] - a), c & 1))
    sign = 0x80 if math.copysign(1.0, float(x)) < 0 else 0
    return sign | best


# ------------------------------------------------------------- number formats
def test_f16_decode_all_codes_matches_numpy():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ours = oracle.f16_to_f64(bits)
    ref = bits.view(np.float16).astype(np.float64)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(ours), nan)
    assert np.array_equal(ours[~nan], ref[~nan])
    assert np.array_equal(np.signbit(ours[~nan]), np.signbit(ref[~nan]))


def test_e4m3_decode_all_codes_matches_torch():
    ours = oracle.e4m3_to_f64(np.arange(256, dtype=np.uint8))
    ref = e4m3_table_torch()
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(ours), nan)
    assert nan.sum() == 2                                   # 0x7F and 0xFF only
    assert np.array_equal(ours[~nan], ref[~nan])


def test_e4m3_decode_closed_forms():
    d = lambda c: float(oracle.e4m3_to_f64(np.array([c], dtype=np.uint8))[0])
    assert d(0x7E) == 448.0                                 # 1.75 * 2^8, largest finite
    assert d(0xFE) == -448.0
    assert d(0x38) == 1.0                                   # e = 7 (bias), m = 0
    assert d(0x08) == 2.0 ** -6                             # smallest normal
    assert d(0x01) == 2.0 ** -9                             # smallest subnormal
    assert d(0x07) == 7 * 2.0 ** -9                         # largest subnormal
    assert d(0x00) == 0.0 and math.copysign(1, d(0x80)) < 0
    assert math.isnan(d(0x7F))


def test_e4m3_round_matches_bruteforce_and_torch():
    rng = np.random.default_rng(1)
    tab = e4m3_table_torch()
    finite = np.array(sorted(set(abs(v) for v in tab[:0x7F])))
    mids = (finite[1:] + finite[:-1]) / 2                    # exact ties (fp32-representable)
    xs = np.concatenate([
        finite, -finite, mids, -mids,
        np.nextafter(mids.astype(np.float32), np.float32(np.inf)),
        np.nextafter(mids.astype(np.float32), np.float32(-np.inf)),
        rng.standard_normal(3000) * 40, rng.uniform(-2 ** -6, 2 ** -6, 500),
    ]).astype(np.float32)
    ours = oracle.e4m3_from_f32(xs)
    brute = np.array([e4m3_round_bruteforce(x) for x in xs], dtype=np.uint8)
    assert np.array_equal(ours, brute)
    inrange = np.abs(xs) < 464                               # torch's cast is RNE but not satfinite
    t = torch.from_numpy(xs[inrange]).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(ours[inrange], t)


def test_e4m3_round_saturation_and_ties():
    r = lambda x: int(oracle.e4m3_from_f32(np.array([x], dtype=np.float32))[0])
    assert r(448.0) == 0x7E and r(449.0) == 0x7E
    assert r(464.0) == 0x7E                                  # tie between 448 (m=6) and 480: even
    assert r(470.0) == 0x7E and r(1e9) == 0x7E and r(np.inf) == 0x7E
    assert r(-1e9) == 0xFE and r(-np.inf) == 0xFE
    assert r(np.nan) == 0x7F
    assert r(2.0 ** -10) == 0x00                             # tie between 0 and 2^-9: even (0)
    assert r(-(2.0 ** -10)) == 0x80
    assert r(3 * 2.0 ** -10) == 0x02                         # tie between 1 and 2 (x 2^-9): even
    assert r(1.0625) == 0x38                                 # tie between 1.0 and 1.125: even
    assert r(1.1875) == 0x3A                                 # tie between 1.125 and 1.25: even


def test_quantize_divides_in_fp32():
    rng = np.random.default_rng(2)
    x = rng.standard_normal(4096).astype(np.float16)
    scale = np.float32(0.0137)
    ours = oracle.quantize_e4m3(x, float(scale))
    quot = (x.astype(np.float32) / scale).astype(np.float32)
    assert np.array_equal(ours, oracle.e4m3_from_f32(quot))


# -------------------------------------------------------------- cache write
@pytest.mark.parametrize("kv_dtype", ["f16", "fp8"])
def test_cache_write_touches_only_target_slots(kv_dtype):
    rng = np.random.default_rng(3)
    NB, bs, Hkv, D, T = 10, 4, 2, 8, 5
    cdt = np.uint8 if kv_dtype == "fp8" else np.float16
    if kv_dtype == "fp8":
        kc = rng.integers(0, 256, (NB, bs, Hkv, D)).astype(np.uint8)
        vc = rng.integers(0, 256, (NB, bs, Hkv, D)).astype(np.uint8)
    else:
        kc = rng.standard_normal((NB, bs, Hkv, D)).astype(np.float16)
        vc = rng.standard_normal((NB, bs, Hkv, D)).astype(np.float16)
    k0, v0 = kc.copy(), vc.copy()
    kn = rng.standard_normal((T, Hkv, D)).astype(np.float16)
    vn = rng.standard_normal((T, Hkv, D)).astype(np.float16)
    slots = np.array([7, 39, -1, 0, 22], dtype=np.int64)
    ks, vs = 0.01, 0.02
    oracle.paged_kv_cache_write(kn, vn, kc, vc, slots, kv_dtype=kv_dtype, k_scale=ks, v_scale=vs)
    changed = np.zeros((NB, bs), dtype=bool)
    for i, s in enumerate(slots):
        if s < 0:
            continue
        blk, row = divmod(int(s), bs)
        changed[blk, row] = True
        if kv_dtype == "fp8":
            exp_k = oracle.e4m3_from_f32((kn[i].astype(np.float32) / np.float32(ks)).ravel())
            exp_v = oracle.e4m3_from_f32((vn[i].astype(np.float32) / np.float32(vs)).ravel())
            assert np.array_equal(kc[blk, row].ravel(), exp_k)
            assert np.array_equal(vc[blk, row].ravel(), exp_v)
        else:
            assert np.array_equal(kc[blk, row].view(np.uint16), kn[i].view(np.uint16))
            assert np.array_equal(vc[blk, row].view(np.uint16), vn[i].view(np.uint16))
    view = (lambda a: a.view(np.uint16)) if cdt == np.float16 else (lambda a: a)
    assert np.array_equal(view(kc)[~changed], view(k0)[~changed])
    assert np.array_equal(view(vc)[~changed], view(v0)[~changed])


def test_cache_write_rejects_slot_outside_pool():
    kc = np.zeros((2, 4, 1, 8), np.float16)
    with pytest.raises(ValueError):
        oracle.paged_kv_cache_write(np.zeros((1, 1, 8), np.float16), np.zeros((1, 1, 8), np.float16),
                                    kc, kc.copy(), np.array([8], np.int64))


# ------------------------------------------------------- attention: brute force
@pytest.mark.parametrize("Hq,Hkv", [(4, 4), (12, 2), (7, 1), (28, 4)])
@pytest.mark.parametrize("seed", [0, 1])
def test_decode_matches_dense_bruteforce(Hq, Hkv, seed):
    rng = np.random.default_rng(10 + seed)
    lens = [1, 5, 4, 13, 30]
    q, Ks, Vs, kp, vp, bt, cl = random_case(rng, lens, Hq, Hkv)
    scale = np.float32(1 / math.sqrt(16))
    out, lse = oracle.paged_gqa_decode(q, kp, vp, bt, cl, float(scale), return_lse=True)
    for b, L in enumerate(lens):
        ref = dense_attention(q[b].astype(np.float64), Ks[b].astype(np.float64),
                              Vs[b].astype(np.float64), float(scale))
        np.testing.assert_allclose(out[b], ref, rtol=RTOL_DENSE, atol=1e-14)
        G = Hq // Hkv
        s = float(scale) * np.einsum("hd,lhd->hl", q[b].astype(np.float64),
                                     np.repeat(Ks[b].astype(np.float64), G, axis=1))
        from scipy.special import logsumexp
        np.testing.assert_allclose(lse[b], logsumexp(s, axis=1), rtol=1e-13)


def test_tiny_workload_matches_dense_bruteforce():
    w = W.WORKLOADS["tiny"]
    x = W.make_inputs(w, seed=0)
    out = oracle.paged_gqa_decode(x["q"], x["k_pool"], x["v_pool"], x["block_tables"],
                                  x["context_lens"], float(x["softmax_scale"]))
    for b in range(w.B):
        L = int(x["context_lens"][b])
        rows = [(int(x["block_tables"][b, t // 16]), t % 16) for t in range(L)]
        K = np.stack([x["k_pool"][p, r] for p, r in rows]).astype(np.float64)
        V = np.stack([x["v_pool"][p, r] for p, r in rows]).astype(np.float64)
        ref = dense_attention(x["q"][b].astype(np.float64), K, V, float(x["softmax_scale"]))
        np.testing.assert_allclose(out[b], ref, rtol=RTOL_DENSE, atol=1e-14)
    assert np.isfinite(out).all()                             # NaN poison never read


def test_fp8_decode_matches_dense_on_dequantised_values():
    rng = np.random.default_rng(20)
    lens = [3, 16, 21]
    Hq, Hkv, D, bs = 6, 2, 16, 4
    q, Ks, Vs, kp, vp, bt, cl = random_case(rng, lens, Hq, Hkv, D=D, bs=bs)
    ks, vs = 0.0091, 0.0123
    kq = oracle.quantize_e4m3(np.nan_to_num(kp), ks)
    vq = oracle.quantize_e4m3(np.nan_to_num(vp), vs)
    out = oracle.paged_gqa_decode(q, kq, vq, bt, cl, 0.25, kv_dtype="fp8", k_scale=ks, v_scale=vs)
    tab = e4m3_table_torch()
    for b, L in enumerate(lens):
        rows = [(int(bt[b, t // bs]), t % bs) for t in range(L)]
        K = np.stack([tab[kq[p, r]] for p, r in rows]) * float(np.float32(ks))
        V = np.stack([tab[vq[p, r]] for p, r in rows]) * float(np.float32(vs))
        ref = dense_attention(q[b].astype(np.float64), K, V, 0.25)
        np.testing.assert_allclose(out[b], ref, rtol=RTOL_DENSE, atol=1e-14)


# --------------------------------------------------- closed forms and invariants
def test_worked_example_closed_form():
    """s = (0, 1, 2) by construction, so p = (1, e, e^2) / (1 + e + e^2)."""
    q = np.array([[[2.0, 0.0]]], dtype=np.float16)            # B=1, Hq=1, D=2
    K = np.array([[[0, 0]], [[1, 0]], [[2, 0]]], dtype=np.float16)
    V = np.array([[[1, 0]], [[0, 1]], [[1, 1]]], dtype=np.float16)
    kp, vp, bt = paged_from_contiguous([K], [V], 2, 4, np.random.default_rng(0))
    out = oracle.paged_gqa_decode(q, kp, vp, bt, np.array([3], np.int32), 0.5)
    e = math.e
    z = 1 + e + e * e
    np.testing.assert_allclose(out[0, 0], [(1 + e * e) / z, (e + e * e) / z], rtol=1e-15)


def test_context_one_returns_v0_exactly():
    rng = np.random.default_rng(4)
    q, Ks, Vs, kp, vp, bt, cl = random_case(rng, [1, 1], 6, 2)
    out = oracle.paged_gqa_decode(q, kp, vp, bt, cl, 0.3)
    for b in range(2):
        assert np.array_equal(out[b], np.repeat(Vs[b][0].astype(np.float64), 3, axis=0))


def test_identical_keys_and_zero_scale_give_mean_of_v():
    rng = np.random.default_rng(5)
    L, Hq, Hkv, D = 23, 6, 2, 16
    k1 = rng.standard_normal((1, Hkv, D)).astype(np.float16)
    K = np.repeat(k1, L, axis=0)
    V = rng.standard_normal((L, Hkv, D)).astype(np.float16)
    q = rng.standard_normal((1, Hq, D)).astype(np.float16)
    kp, vp, bt = paged_from_contiguous([K], [V], 4, 9, rng)
    mean = np.repeat(V.astype(np.float64).mean(axis=0), Hq // Hkv, axis=0)
    out = oracle.paged_gqa_decode(q, kp, vp, bt, np.array([L], np.int32), 0.7)
    np.testing.assert_allclose(out[0], mean, rtol=1e-13, atol=1e-15)
    Kr = rng.standard_normal((L, Hkv, D)).astype(np.float16)
    kp2, vp2, bt2 = paged_from_contiguous([Kr], [V], 4, 9, rng)
    out0 = oracle.paged_gqa_decode(q, kp2, vp2, bt2, np.array([L], np.int32), 0.0)
    np.testing.assert_allclose(out0[0], mean, rtol=1e-13, atol=1e-15)


def test_block_permutation_invariance_is_bitwise():
    rng = np.random.default_rng(6)
    q, Ks, Vs, kp, vp, bt, cl = random_case(rng, [9, 17, 30], 12, 2, extra_blocks=7)
    out = oracle.paged_gqa_decode(q, kp, vp, bt, cl, 0.25)
    NB = kp.shape[0]
    perm = rng.permutation(NB)                                 # new position of block i
    kp2 = np.empty_like(kp); vp2 = np.empty_like(vp)
    kp2[perm] = kp; vp2[perm] = vp
    bt2 = np.where(bt >= 0, perm[np.maximum(bt, 0)], -1).astype(np.int32)
    out2 = oracle.paged_gqa_decode(q, kp2, vp2, bt2, cl, 0.25)
    assert np.array_equal(out, out2)


@pytest.mark.parametrize("P", [4, 8, 12, 64])
def test_split_merge_equals_single_pass(P):
    rng = np.random.default_rng(7)
    q, Ks, Vs, kp, vp, bt, cl = random_case(rng, [1, 4, 5, 31, 40], 12, 2)
    single, lse1 = oracle.paged_gqa_decode(q, kp, vp, bt, cl, 0.25, return_lse=True)
    split, lse2 = oracle.paged_gqa_decode(q, kp, vp, bt, cl, 0.25, partition_tokens=P,
                                          return_lse=True)
    np.testing.assert_allclose(split, single, rtol=1e-12, atol=1e-15)
    np.testing.assert_allclose(lse2, lse1, rtol=1e-13)
    if P >= 40:
        assert np.array_equal(split, single)


def test_head_map_contiguous_groups():
    rng = np.random.default_rng(8)
    L, Hq, Hkv, D = 11, 28, 4, 8
    K = rng.standard_normal((L, Hkv, D)).astype(np.float16)
    V = np.broadcast_to(np.arange(Hkv, dtype=np.float16)[None, :, None], (L, Hkv, D)).copy()
    q = rng.standard_normal((1, Hq, D)).astype(np.float16)
    kp, vp, bt = paged_from_contiguous([K], [V], 4, 6, rng)
    out = oracle.paged_gqa_decode(q, kp, vp, bt, np.array([L], np.int32), 0.5)
    G = Hq // Hkv
    expect = np.repeat(np.arange(Hkv, dtype=np.float64), G)[:, None] * np.ones(D)
    np.testing.assert_allclose(out[0], expect, rtol=1e-14, atol=1e-14)


def test_poison_in_unused_rows_and_entries_is_never_read():
    w = W.with_sizes(W.WORKLOADS["tiny"], ctx=("fixed", (17, 40)))
    a = W.make_inputs(w, seed=3, poison=True)
    b = W.make_inputs(w, seed=3, poison=False)
    assert np.isnan(a["k_pool"]).any()
    oa = oracle.paged_gqa_decode(a["q"], a["k_pool"], a["v_pool"], a["block_tables"],
                                 a["context_lens"], 0.088)
    ob = oracle.paged_gqa_decode(b["q"], b["k_pool"], b["v_pool"], b["block_tables"],
                                 b["context_lens"], 0.088)
    assert np.array_equal(oa, ob)


def test_one_hot_logit_returns_that_value():
    """One logit exceeds the others by Delta: |out - V_j| <= (L-1) e^-Delta max|V_t - V_j|."""
    rng = np.random.default_rng(9)
    L, D = 20, 16
    K = (rng.standard_normal((L, 1, D)) * 0.1).astype(np.float16)
    j = 13
    K[j, 0] = np.float16(4.0)
    q = np.full((1, 1, D), 4.0, dtype=np.float16)
    V = rng.standard_normal((L, 1, D)).astype(np.float16)
    kp, vp, bt = paged_from_contiguous([K], [V], 4, 7, rng)
    out = oracle.paged_gqa_decode(q, kp, vp, bt, np.array([L], np.int32), 1.0)
    s = (q[0, 0].astype(np.float64) * K[:, 0].astype(np.float64)).sum(axis=1)
    delta = s[j] - np.delete(s, j).max()
    assert delta > 200
    bound = (L - 1) * math.exp(-delta) * np.abs(V[:, 0].astype(np.float64) - V[j, 0]).max()
    assert np.abs(out[0, 0] - V[j, 0].astype(np.float64)).max() <= bound + 1e-300


def test_empty_context_gives_zero_row_and_minus_inf_lse():
    rng = np.random.default_rng(11)
    q, Ks, Vs, kp, vp, bt, cl = random_case(rng, [5, 7], 4, 2)
    cl = np.array([0, 7], np.int32)
    for P in (0, 4):
        out, lse = oracle.paged_gqa_decode(q, kp, vp, bt, cl, 0.25, partition_tokens=P,
                                           return_lse=True)
        assert np.array_equal(out[0], np.zeros_like(out[0]))
        assert np.all(np.isneginf(lse[0]))
        assert np.isfinite(lse[1]).all()


def test_rejects_bad_lengths_and_tables():
    rng = np.random.default_rng(12)
    q, Ks, Vs, kp, vp, bt, cl = random_case(rng, [5, 7], 4, 2)
    with pytest.raises(ValueError):
        oracle.paged_gqa_decode(q, kp, vp, bt, np.array([5, 7 + 4 * bt.shape[1]], np.int32), 0.25)
    bad = bt.copy(); bad[0, 0] = kp.shape[0]
    with pytest.raises(ValueError):
        oracle.paged_gqa_decode(q, kp, vp, bad, cl, 0.25)
