"""Pins of the oracle's FP8 scale paths: scales computed from data, and one scale per KV head.

"rvLLM 소개" (discuss.pytorch.kr), §PagedAttention과 FlashAttention-3 names an FP8 E4M3 KV
cache and nothing more. The readings (oracle header, R8): a scale may be given per KV head,
replacing the per-tensor scale for that head; a scale computed from data is fp32(amax) / 448,
amax being the largest |x| over the non-NaN elements, and 1 when that is 0. Each pin below
holds by construction or reduces the new path to an already pinned one.
"""
import numpy as np
import pytest

import oracle
import workloads as W

E4M3_MAX_CODE = 0x7E          # +448, the largest finite E4M3 (FN) code


def _normal(shape, seed, scale=1.0):
    return (np.random.default_rng(seed).standard_normal(shape) * scale).astype(np.float16)


# ------------------------------------------------------------------ amax and scales
def test_absmax_planted_values():
    x = np.zeros((4, 3, 8), dtype=np.float16)
    x[1, 0, 5] = 2.25
    x[3, 1, 0] = -3.5                       # a negative value counts by magnitude
    x[0, 2, 7] = 0.75
    x[2, 2, 1] = np.nan                     # NaN never counts
    x[0, 0, 0] = -1.0
    assert oracle.absmax_f16(x, True).tolist() == [2.25, 3.5, 0.75]
    assert oracle.absmax_f16(x, False).tolist() == [3.5]


def test_absmax_of_nothing_gives_scale_one():
    x = np.full((2, 2, 4), np.nan, dtype=np.float16)
    x[:, 1] = 0
    assert oracle.absmax_f16(x, True).tolist() == [0.0, 0.0]
    assert oracle.fp8_scales(x, True).tolist() == [1.0, 1.0]


def test_absmax_invariants():
    a, b = _normal((6, 2, 16), 1, 3.0), _normal((5, 2, 16), 2, 0.5)
    both = np.concatenate([a, b])
    for per_head in (True, False):
        assert np.array_equal(oracle.absmax_f16(both, per_head),
                              np.maximum(oracle.absmax_f16(a, per_head), oracle.absmax_f16(b, per_head)))
        assert np.array_equal(oracle.absmax_f16(-a, per_head), oracle.absmax_f16(a, per_head))
        assert np.array_equal(oracle.absmax_f16(a * np.float16(2), per_head), 2 * oracle.absmax_f16(a, per_head))


def test_scale_from_amax_values():
    assert oracle.fp8_scale_from_amax([448.0, 224.0, 0.0, 896.0]).tolist() == [1.0, 0.5, 1.0, 2.0]
    a = np.float32(3.1416015625)            # a binary16 value; the quotient is not exact
    assert oracle.fp8_scale_from_amax(a)[0] == a / np.float32(448)      # IEEE fp32 division


@pytest.mark.parametrize("seed", range(4))
def test_amax_element_maps_onto_the_largest_code(seed):
    """With scale = fp32(amax) / 448 the largest magnitude quantises to +-448 exactly."""
    x = _normal((32, 2, 128), 10 + seed, [0.01, 1.0, 37.0, 300.0][seed])
    s = oracle.fp8_scales(x, False)[0]
    codes = oracle.quantize_e4m3(x, float(s))
    amax_pos = np.unravel_index(np.nanargmax(np.abs(x.astype(np.float32))), x.shape)
    assert codes[amax_pos] & 0x7F == E4M3_MAX_CODE
    assert ((codes & 0x7F) <= E4M3_MAX_CODE).all()      # nothing else saturates past it or is NaN


# ------------------------------------------------------------------ per-head cache write
def test_per_head_write_is_the_pinned_quantiser_head_by_head():
    T, Hkv, D, NB, bs = 5, 4, 128, 8, 16
    k_new, v_new = _normal((T, Hkv, D), 3, 4.0), _normal((T, Hkv, D), 4, 0.2)
    ks = np.array([0.01, 0.02, 0.005, 0.04], np.float32)
    vs = np.array([0.001, 0.003, 0.0005, 0.0007], np.float32)
    slots = np.array([3, 17, -1, 40, 127], np.int64)
    kc = np.zeros((NB, bs, Hkv, D), np.uint8)
    vc = np.zeros_like(kc)
    oracle.paged_kv_cache_write(k_new, v_new, kc, vc, slots, kv_dtype="fp8", k_scale=ks, v_scale=vs)
    for i, s in enumerate(slots):
        if s < 0:
            continue
        for h in range(Hkv):
            assert np.array_equal(kc[s // bs, s % bs, h], oracle.quantize_e4m3(k_new[i, h], float(ks[h])))
            assert np.array_equal(vc[s // bs, s % bs, h], oracle.quantize_e4m3(v_new[i, h], float(vs[h])))
    untouched = np.ones(NB * bs, bool)
    untouched[slots[slots >= 0]] = False
    assert not kc.reshape(NB * bs, -1)[untouched].any() and not vc.reshape(NB * bs, -1)[untouched].any()


def test_per_head_write_with_equal_scales_is_the_per_tensor_write():
    w = W.WORKLOADS["tiny"]
    x = W.make_inputs(w, 5, poison=False)
    a = np.zeros((w.num_blocks, w.block_size, w.Hkv, w.head_dim), np.uint8)
    b, c, d = a.copy(), a.copy(), a.copy()
    oracle.paged_kv_cache_write(x["k_new"], x["v_new"], a, b, x["slot_mapping"], kv_dtype="fp8",
                                k_scale=0.01, v_scale=0.02)
    oracle.paged_kv_cache_write(x["k_new"], x["v_new"], c, d, x["slot_mapping"], kv_dtype="fp8",
                                k_scale=np.full(w.Hkv, 0.01), v_scale=np.full(w.Hkv, 0.02))
    assert np.array_equal(a, c) and np.array_equal(b, d)


# ------------------------------------------------------------------ per-head attention
def _fp8_case(seed, Hkv=4, G=3, B=3, NB=64):
    w = W.with_sizes(W.WORKLOADS["qwen2.5-7b"], B=B, Hq=G * Hkv, Hkv=Hkv, num_blocks=NB,
                     ctx=("uniform", 1, 120), kv_dtype="fp8")
    x = W.make_inputs(w, seed, poison=False)
    ks = np.float32(x["k_scale"]) * np.array([1.0, 0.5, 2.0, 0.25][:Hkv], np.float32)
    vs = np.float32(x["v_scale"]) * np.array([0.25, 1.0, 0.5, 2.0][:Hkv], np.float32)
    kq = np.stack([oracle.quantize_e4m3(x["k_pool"][:, :, h], float(ks[h])) for h in range(Hkv)], axis=2)
    vq = np.stack([oracle.quantize_e4m3(x["v_pool"][:, :, h], float(vs[h])) for h in range(Hkv)], axis=2)
    return w, x, ks, vs, np.ascontiguousarray(kq), np.ascontiguousarray(vq)


@pytest.mark.parametrize("P", [0, 32])
def test_per_head_attention_is_per_tensor_attention_per_kv_head(P):
    w, x, ks, vs, kq, vq = _fp8_case(6)
    G = w.group
    out = oracle.paged_gqa_decode(x["q"], kq, vq, x["block_tables"], x["context_lens"],
                                  float(x["softmax_scale"]), kv_dtype="fp8", k_scale=ks, v_scale=vs,
                                  partition_tokens=P)
    for g in range(w.Hkv):
        ref = oracle.paged_gqa_decode(np.ascontiguousarray(x["q"][:, g * G:(g + 1) * G]),
                                      np.ascontiguousarray(kq[:, :, g:g + 1]),
                                      np.ascontiguousarray(vq[:, :, g:g + 1]),
                                      x["block_tables"], x["context_lens"], float(x["softmax_scale"]),
                                      kv_dtype="fp8", k_scale=float(ks[g]), v_scale=float(vs[g]),
                                      partition_tokens=P)
        assert np.array_equal(out[:, g * G:(g + 1) * G], ref)


def test_per_head_attention_with_equal_scales_is_per_tensor_attention():
    w, x, ks, vs, kq, vq = _fp8_case(7)
    args = (x["q"], kq, vq, x["block_tables"], x["context_lens"], float(x["softmax_scale"]))
    a = oracle.paged_gqa_decode(*args, kv_dtype="fp8", k_scale=0.01, v_scale=0.02)
    b = oracle.paged_gqa_decode(*args, kv_dtype="fp8", k_scale=np.full(w.Hkv, 0.01, np.float32),
                                v_scale=np.full(w.Hkv, 0.02, np.float32))
    assert np.array_equal(a, b)


def test_doubling_one_heads_v_scale_doubles_exactly_its_group():
    w, x, ks, vs, kq, vq = _fp8_case(8)
    G = w.group
    args = (x["q"], kq, vq, x["block_tables"], x["context_lens"], float(x["softmax_scale"]))
    base = oracle.paged_gqa_decode(*args, kv_dtype="fp8", k_scale=ks, v_scale=vs)
    vs2 = vs.copy()
    vs2[2] *= 2
    twice = oracle.paged_gqa_decode(*args, kv_dtype="fp8", k_scale=ks, v_scale=vs2)
    assert np.array_equal(twice[:, 2 * G:3 * G], 2 * base[:, 2 * G:3 * G])
    keep = np.ones(w.Hq, bool)
    keep[2 * G:3 * G] = False
    assert np.array_equal(twice[:, keep], base[:, keep])
