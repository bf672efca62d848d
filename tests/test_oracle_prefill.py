"""Pins of the oracle's chunked prefill attention (reading R12).

The pages name prefill only as engine work besides decode ("rvLLM 소개" (discuss.pytorch.kr),
§H100 SXM 80GB 직접 엔진 벤치마크). The reading: sequence b brings n_b query tokens, the last n_b of
its context_lens[b] tokens (their K/V already cached); query i sits at position L_b - n_b + i and
attends causally to positions [0, p] through the block table. The pins: one query per sequence
is decode; a dense causal brute force on the gathered K/V (the textbook masked softmax); the
last query of a sequence is that sequence's decode; the first position returns V_0; changing
later positions leaves a query unchanged; physical block order does not matter.
"""
import numpy as np
import pytest

import oracle
import workloads as W

F16 = np.float16


def _case(seed, n_new, ctx=("uniform", 1, 70), B=5, Hq=6, Hkv=2, kv_dtype="f16"):
    """Pool, tables and lengths from the decode generator (no poison), plus the queries."""
    w = W.with_sizes(W.WORKLOADS["tiny"], B=B, Hq=Hq, Hkv=Hkv, num_blocks=64, ctx=ctx, kv_dtype=kv_dtype)
    x = W.make_inputs(w, seed, poison=False)
    lens = x["context_lens"]
    n = np.array([min(int(L), k) for L, k in zip(lens, n_new)], np.int32)
    qs = np.concatenate([[0], np.cumsum(n)]).astype(np.int32)
    rng = np.random.default_rng(seed + 100)
    q = rng.standard_normal((int(qs[-1]), Hq, w.head_dim)).astype(F16)
    return w, x, q, qs


def _dense(w, x, q, qs, k_scale=1.0, v_scale=1.0, kq=None, vq=None):
    """Causal softmax attention on the gathered, contiguous K/V of each sequence (float64)."""
    out = np.zeros(q.shape, np.float64)
    G = w.Hq // w.Hkv
    scale = float(x["softmax_scale"])
    for b in range(w.B):
        L = int(x["context_lens"][b])
        n = int(qs[b + 1] - qs[b])
        if n == 0:
            continue
        t = np.arange(L)
        phys = x["block_tables"][b, t // w.block_size]
        if kq is None:
            K = x["k_pool"][phys, t % w.block_size].astype(np.float64)            # [L, Hkv, D]
            V = x["v_pool"][phys, t % w.block_size].astype(np.float64)
        else:
            K = oracle.e4m3_to_f64(kq[phys, t % w.block_size]).reshape(L, w.Hkv, -1) * k_scale
            V = oracle.e4m3_to_f64(vq[phys, t % w.block_size]).reshape(L, w.Hkv, -1) * v_scale
        pos = L - n + np.arange(n)                                                  # [n]
        mask = t[None, :] <= pos[:, None]                                           # [n, L]
        for h in range(w.Hq):
            g = h // G
            qq = q[qs[b]:qs[b + 1], h].astype(np.float64)                           # [n, D]
            logits = scale * (qq @ K[:, g].T)
            logits = np.where(mask, logits, -np.inf)
            p = np.exp(logits - logits.max(axis=1, keepdims=True))
            out[qs[b]:qs[b + 1], h] = (p / p.sum(axis=1, keepdims=True)) @ V[:, g]
    return out


def _prefill(w, x, q, qs, **kw):
    return oracle.paged_prefill(q, x["k_pool"], x["v_pool"], x["block_tables"], x["context_lens"], qs,
                                float(x["softmax_scale"]), **kw)


def test_one_query_per_sequence_is_decode():
    w, x, q, qs = _case(1, [1] * 5)
    out, lse = _prefill(w, x, q, qs, return_lse=True)
    ref, rlse = oracle.paged_gqa_decode(q, x["k_pool"], x["v_pool"], x["block_tables"], x["context_lens"],
                                        float(x["softmax_scale"]), return_lse=True)
    assert np.array_equal(out, ref) and np.array_equal(lse, rlse)


@pytest.mark.parametrize("n_new", [[3, 1, 7, 40, 2], [70, 70, 70, 70, 70], [0, 5, 0, 1, 16]])
def test_matches_dense_causal_bruteforce(n_new):
    w, x, q, qs = _case(2, n_new)
    out = _prefill(w, x, q, qs)
    assert np.allclose(out, _dense(w, x, q, qs), rtol=1e-12, atol=1e-13)


def test_gqa_group_of_seven():
    w, x, q, qs = _case(3, [4, 9, 1, 30, 6], Hq=28, Hkv=4)
    assert np.allclose(_prefill(w, x, q, qs), _dense(w, x, q, qs), rtol=1e-12, atol=1e-13)


def test_last_query_of_a_sequence_is_its_decode():
    w, x, q, qs = _case(4, [6, 2, 11, 3, 8])
    out = _prefill(w, x, q, qs)
    last = qs[1:] - 1
    ref = oracle.paged_gqa_decode(np.ascontiguousarray(q[last]), x["k_pool"], x["v_pool"], x["block_tables"],
                                  x["context_lens"], float(x["softmax_scale"]))
    assert np.array_equal(out[last], ref)


def test_first_position_returns_v0():
    """A prefill from an empty cache: query 0 sees only token 0, so its output is V_0 exactly."""
    w, x, q, qs = _case(5, [100] * 5)
    out = _prefill(w, x, q, qs)
    G = w.Hq // w.Hkv
    for b in range(w.B):
        v0 = x["v_pool"][x["block_tables"][b, 0], 0].astype(np.float64)          # [Hkv, D]
        for h in range(w.Hq):
            assert np.array_equal(out[qs[b], h], v0[h // G])


def test_later_positions_do_not_reach_earlier_queries():
    w, x, q, qs = _case(6, [12, 12, 12, 12, 12], ctx=("fixed", (40, 33, 17, 60, 12)))
    base = _prefill(w, x, q, qs)
    b, i = 3, 4                                    # a middle query of sequence 3
    L, n = int(x["context_lens"][b]), int(qs[b + 1] - qs[b])
    pos = L - n + i
    row = qs[b] + i
    for t, changes in [(pos + 1, False), (L - 1, False), (pos, True), (0, True)]:
        y = {k: v.copy() if isinstance(v, np.ndarray) else v for k, v in x.items()}
        phys = y["block_tables"][b, t // w.block_size]
        y["k_pool"][phys, t % w.block_size] = F16(3.0)
        y["v_pool"][phys, t % w.block_size] = F16(-2.0)
        out = _prefill(w, y, q, qs)
        assert np.array_equal(out[row], base[row]) != changes, (t, changes)
        assert np.array_equal(out[:qs[b]], base[:qs[b]])         # other sequences never change


def test_block_permutation_is_invisible():
    w, x, q, qs = _case(7, [9, 4, 17, 2, 30])
    base = _prefill(w, x, q, qs)
    perm = np.random.default_rng(0).permutation(w.num_blocks)
    y = dict(x)
    y["k_pool"], y["v_pool"] = np.empty_like(x["k_pool"]), np.empty_like(x["v_pool"])
    y["k_pool"][perm], y["v_pool"][perm] = x["k_pool"], x["v_pool"]
    bt = x["block_tables"].copy()
    bt[bt >= 0] = perm[bt[bt >= 0]]
    y["block_tables"] = bt
    assert np.array_equal(_prefill(w, y, q, qs), base)


def test_fp8_matches_dense_on_dequantised_values():
    w, x, q, qs = _case(8, [5, 3, 20, 1, 9], kv_dtype="fp8")
    ks, vs = float(x["k_scale"]), float(x["v_scale"])
    kq, vq = oracle.quantize_e4m3(x["k_pool"], ks), oracle.quantize_e4m3(x["v_pool"], vs)
    out = oracle.paged_prefill(q, kq, vq, x["block_tables"], x["context_lens"], qs, float(x["softmax_scale"]),
                               kv_dtype="fp8", k_scale=ks, v_scale=vs)
    ref = _dense(w, x, q, qs, np.float32(ks), np.float32(vs), kq, vq)
    assert np.allclose(out, ref, rtol=1e-12, atol=1e-13)


def test_bad_lengths_are_rejected():
    w, x, q, qs = _case(9, [2, 2, 2, 2, 2], ctx=("fixed", (5, 5, 5, 5, 5)))
    bad = qs.copy()
    bad[1:] = [6, 8, 10, 12, 14]                   # sequence 0 asks for 6 queries of a 5-token context
    q6 = np.zeros((14, w.Hq, w.head_dim), F16)
    with pytest.raises(ValueError):
        oracle.paged_prefill(q6, x["k_pool"], x["v_pool"], x["block_tables"], x["context_lens"], bad,
                             float(x["softmax_scale"]))


def test_lse_matches_dense_logsumexp():
    """The returned log-sum-exp is that of the masked logits (natural log, scaled logits)."""
    w, x, q, qs = _case(10, [4, 9, 1, 30, 6])
    _, lse = _prefill(w, x, q, qs, return_lse=True)
    G = w.Hq // w.Hkv
    for b in range(w.B):
        L, n = int(x["context_lens"][b]), int(qs[b + 1] - qs[b])
        t = np.arange(L)
        K = x["k_pool"][x["block_tables"][b, t // w.block_size], t % w.block_size].astype(np.float64)
        for i in range(n):
            pos = L - n + i
            for h in range(w.Hq):
                s = float(x["softmax_scale"]) * (K[:pos + 1, h // G] @ q[qs[b] + i, h].astype(np.float64))
                want = s.max() + np.log(np.exp(s - s.max()).sum())
                assert abs(lse[qs[b] + i, h] - want) <= 1e-12 * max(1.0, abs(want))
