"""Parity of paged_gqa_prefill_attention (chunked prefill through the block tables) with the float64
oracle, at the attention tolerance (2e-3 max-abs, 1e-2 of max |oracle|); FP8 on the same E4M3 bytes."""
import numpy as np
import pytest
import torch

import oracle
import paged_kv_decode_gqa_b200 as pkv
import workloads as W
from _gpu_helpers import assert_attention_close, dev, fp8_caches, host

pytestmark = pytest.mark.gpu
F16 = np.float16


@pytest.fixture(autouse=True)
def _clear_device_error():
    pkv.pkv_device_error()
    yield
    torch.cuda.synchronize()


def _case(name, seed, n_new, **sizes):
    w = W.with_sizes(W.WORKLOADS[name], **sizes)
    x = W.make_inputs(w, seed)                     # unused pool rows are NaN: never read
    lens = x["context_lens"]
    n = np.array([min(int(L), k) for L, k in zip(lens, n_new)], np.int32)
    qs = np.concatenate([[0], np.cumsum(n)]).astype(np.int32)
    q = np.random.default_rng(seed + 7).standard_normal((int(qs[-1]), w.Hq, w.head_dim)).astype(F16)
    return w, x, q, qs


# The two schedules of the f16 kernel: whole items (no workspace) and the load-balanced one that
# cuts items at CTA boundaries and merges their pieces (a zero-filled workspace).
SCHEDULES = ["items", "balanced"]
PART_BYTES = 128 * 128 * 4 + 128 * 8           # one piece's partial rows of one query tile


def _workspace(w):
    n = pkv.paged_gqa_prefill_workspace_size(w.Hq, w.Hkv, w.head_dim)
    assert n > 0
    return torch.zeros(n, dtype=torch.uint8, device="cuda")


def _run(w, x, q, qs, kv_dtype="f16", kc=None, vc=None, schedule="items", ws=None):
    out = torch.full(q.shape, float("nan"), dtype=torch.float16, device="cuda")
    kc = x["k_pool"] if kc is None else kc
    vc = x["v_pool"] if vc is None else vc
    n = qs[1:] - qs[:-1]
    if schedule == "balanced" and ws is None:
        ws = _workspace(w)
    pkv.paged_gqa_prefill_attention(out, dev(q), dev(kc), dev(vc), dev(x["block_tables"]), dev(x["context_lens"]),
                                    dev(qs), max_query_len=max(int(n.max()), 1),
                                    max_context_len=max(int(x["context_lens"].max()), 1),
                                    softmax_scale=float(x["softmax_scale"]), kv_dtype=kv_dtype,
                                    k_scale=float(x["k_scale"]), v_scale=float(x["v_scale"]),
                                    workspace=ws if schedule == "balanced" else None)
    return host(out)


def _check_sampled_rows(x, q, qs, got, what, seed, first=()):
    """Sampled query rows (40 at random, the first and the last, and `first`) against the float64
    oracle: query i of sequence b is decode attention at context length L_b - n_b + i + 1 over the
    same block table. Every row must be finite."""
    rng = np.random.default_rng(seed)
    total = int(qs[-1])
    rows = np.unique(np.concatenate([rng.choice(total, min(40, total), replace=False), [0, total - 1],
                                     np.asarray(first, np.int64)])).astype(np.int64)
    b_of = np.searchsorted(qs, rows, side="right") - 1
    ctx = (x["context_lens"][b_of] - (qs[b_of + 1] - qs[b_of]) + (rows - qs[b_of]) + 1).astype(np.int32)
    ref = oracle.paged_gqa_decode(q[rows], x["k_pool"], x["v_pool"], x["block_tables"][b_of], ctx,
                                  float(x["softmax_scale"]))
    assert_attention_close(got[rows], ref, f"{what}: sampled rows of {total}")
    assert np.isfinite(got).all()


def _tickets_clear(ws):
    """The merge tickets (after the partial results of two slots x two tiles per SM) are back at 0."""
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    return bool((ws[4 * sms * PART_BYTES:] == 0).all())


def _oracle(w, x, q, qs, kv_dtype="f16", kc=None, vc=None):
    return oracle.paged_prefill(q, x["k_pool"] if kc is None else kc, x["v_pool"] if vc is None else vc,
                                x["block_tables"], x["context_lens"], qs, float(x["softmax_scale"]),
                                kv_dtype=kv_dtype, k_scale=float(x["k_scale"]), v_scale=float(x["v_scale"]))


@pytest.mark.parametrize("name,n_new,sizes", [
    ("qwen2.5-1.5b", [1] * 6, dict(B=6, num_blocks=1024)),                          # decode as prefill
    ("qwen2.5-1.5b", [3, 1, 7, 40, 2, 17], dict(B=6, num_blocks=1024)),             # chunked, ragged chunks
    ("qwen2.5-1.5b", [300] * 4, dict(B=4, num_blocks=1024, ctx=("uniform", 1, 300))),  # from an empty cache
    ("qwen2.5-7b", [9, 0, 64, 33], dict(B=4, num_blocks=2048)),                      # G = 7, a sequence without queries
    ("tiny", [17, 40], {}),
])
@pytest.mark.parametrize("schedule", SCHEDULES)
def test_prefill_parity_f16(name, n_new, sizes, schedule):
    w, x, q, qs = _case(name, 3, n_new, **sizes)
    assert_attention_close(_run(w, x, q, qs, schedule=schedule), _oracle(w, x, q, qs), f"{name} {n_new[:3]}")
    assert pkv.pkv_device_error() == 0


@pytest.mark.parametrize("n_new", [[1] * 5, [5, 30, 2, 64, 11]])
def test_prefill_parity_fp8(n_new):
    w, x, q, qs = _case("fp8-e4m3", 4, n_new, B=5, num_blocks=4096, ctx=("uniform", 70, 1500))
    kq, vq = fp8_caches(x)
    got = _run(w, x, q, qs, "fp8", kq, vq)
    assert_attention_close(got, _oracle(w, x, q, qs, "fp8", kq, vq), f"fp8 {n_new}")
    assert pkv.pkv_device_error() == 0


def test_one_query_per_sequence_matches_decode():
    w, x, q, qs = _case("qwen2.5-7b", 5, [1] * 6, B=6, num_blocks=2048)
    got = _run(w, x, q, qs)
    out = torch.empty(q.shape, dtype=torch.float16, device="cuda")
    pkv.paged_gqa_decode_attention(out, dev(q), dev(x["k_pool"]), dev(x["v_pool"]), dev(x["block_tables"]),
                                   dev(x["context_lens"]), max_context_len=int(x["context_lens"].max()),
                                   softmax_scale=float(x["softmax_scale"]))
    ref = _oracle(w, x, q, qs)
    assert_attention_close(got, ref, "prefill n=1")
    assert_attention_close(host(out), ref, "decode")


@pytest.mark.parametrize("schedule", SCHEDULES)
def test_long_chunked_prefill(schedule):
    """Two sequences append 256 tokens to contexts of up to 2048 (Qwen2.5-7B heads)."""
    w, x, q, qs = _case("qwen2.5-7b", 6, [256, 256], B=2, num_blocks=1024, ctx=("uniform", 1024, 2048))
    assert_attention_close(_run(w, x, q, qs, schedule=schedule), _oracle(w, x, q, qs), "long chunked prefill")


@pytest.mark.parametrize("schedule", SCHEDULES)
def test_inconsistent_lengths_are_flagged_not_faulted(schedule):
    w, x, q, qs = _case("qwen2.5-1.5b", 8, [4, 4, 4], B=3, num_blocks=256, ctx=("fixed", (20, 3, 30)))
    # sequence 1 has a 3-token context; ask for 4 queries by moving the boundaries
    qs_bad = np.array([0, 4, 8, 12], np.int32)
    q_bad = np.zeros((12, w.Hq, w.head_dim), F16)
    out = torch.full(q_bad.shape, 7.0, dtype=torch.float16, device="cuda")
    pkv.paged_gqa_prefill_attention(out, dev(q_bad), dev(x["k_pool"]), dev(x["v_pool"]), dev(x["block_tables"]),
                                    dev(x["context_lens"]), dev(qs_bad), max_query_len=4, max_context_len=30,
                                    softmax_scale=float(x["softmax_scale"]),
                                    workspace=_workspace(w) if schedule == "balanced" else None)
    got = host(out)
    assert pkv.pkv_device_error() & pkv.DEVERR_CONTEXT_LEN
    assert (got[4:8] == 7.0).all()                  # the flagged sequence's rows are left alone
    assert np.isfinite(got[:4]).all() and np.isfinite(got[8:]).all()


@pytest.mark.parametrize("Hq,Hkv", [(8, 8), (8, 4), (12, 4), (16, 4), (10, 2), (16, 2)])
@pytest.mark.parametrize("schedule", SCHEDULES)
def test_prefill_group_sizes(Hq, Hkv, schedule):
    """Every group size packs floor(128 / G) query tokens x G heads into the tile's rows
    (128, 64, 42, 32, 25 and 16 tokens); several tiles per sequence, a one-query sequence."""
    w, x, q, qs = _case("qwen2.5-1.5b", 9, [150, 1, 77], B=3, num_blocks=512, Hq=Hq, Hkv=Hkv,
                        ctx=("uniform", 150, 600))
    assert_attention_close(_run(w, x, q, qs, schedule=schedule), _oracle(w, x, q, qs), f"Hq {Hq} / Hkv {Hkv}")
    assert pkv.pkv_device_error() == 0


@pytest.mark.parametrize("schedule", SCHEDULES)
def test_prefill_large_logits(schedule):
    """Logits that grow along the sequence: q scaled by 3 and each key by 1 + position / 256, so
    the running maximum of a row rises by more than the rescale threshold (8 in the exp2 domain)
    several times over its KV tiles and the output accumulated so far is rescaled each time."""
    w, x, q, qs = _case("qwen2.5-7b", 10, [64, 200], B=2, num_blocks=1024, ctx=("uniform", 1500, 2000))
    q = (q.astype(np.float32) * 3).astype(F16)
    k = x["k_pool"].astype(np.float32)
    for b, L in enumerate(x["context_lens"]):
        for j in range(-(-int(L) // 16)):
            pos = 16 * j + np.arange(16, dtype=np.float32)
            k[x["block_tables"][b, j]] *= (1 + pos / 256)[:, None, None]
    x["k_pool"] = k.astype(F16)                     # NaN rows stay NaN
    assert_attention_close(_run(w, x, q, qs, schedule=schedule), _oracle(w, x, q, qs), "large logits")
    assert pkv.pkv_device_error() == 0


@pytest.mark.parametrize("schedule", SCHEDULES)
def test_prefill_zero_scale_is_the_causal_mean(schedule):
    """softmax_scale = 0: every query averages V over its causal window (masked entries stay out
    of the average even though 0 times their logit is 0)."""
    w, x, q, qs = _case("qwen2.5-7b", 11, [40, 150], B=2, num_blocks=512, ctx=("uniform", 200, 400))
    x["softmax_scale"] = np.float32(0.0)
    assert_attention_close(_run(w, x, q, qs, schedule=schedule), _oracle(w, x, q, qs), "zero scale")
    assert pkv.pkv_device_error() == 0


@pytest.mark.parametrize("name", ["qwen2.5-7b", "qwen2.5-1.5b"])
@pytest.mark.parametrize("schedule", SCHEDULES)
def test_prefill_more_items_than_ctas_sampled(name, schedule):
    """The bench's case at full size: 8 sequences append 512 tokens each to 2048-token contexts.
    At 7B heads that is 480 work items (two 18-token query tiles, KV head, sequence), at 1.5B heads
    208, more than the 148 CTAs of the persistent grid, so CTAs run several items each and carry
    their barrier phases, Q reloads and accumulators from one item to the next. Sampled query rows
    are checked against the float64 oracle: query i of sequence b is decode attention at context
    length L_b - n_b + i + 1 over the same block table."""
    B, n_new, L = 8, 512, 2048
    w, x, q, qs = _case(name, 12, [n_new] * B, B=B, num_blocks=B * L // 16 + 64, ctx=("fixed", (L,) * B))
    got = _run(w, x, q, qs, schedule=schedule)
    _check_sampled_rows(x, q, qs, got, name, 13)
    assert pkv.pkv_device_error() == 0


def test_balanced_items_cut_into_many_pieces():
    """300 queries at the end of a 6000-token context and three one-query sequences, at 7B heads:
    the grid has one CTA per (query group, KV head, sequence) the longest sequence allows (144),
    but only 48 items, so the 1800 KV tiles give each CTA 12 or 13 and the 36 long items of about
    47 tiles are each cut into 4 or 5 pieces: a head piece, middle pieces spanning a whole CTA and
    a tail piece. A tail piece can start past the first queries' positions, whose rows then see
    nothing there (maximum -inf, sum 0) and must get weight 0: the first 60 query rows, at
    positions 5700-5759, are all checked."""
    w, x, q, qs = _case("qwen2.5-7b", 14, [300, 1, 1, 1], B=4, num_blocks=1024,
                        ctx=("fixed", (6000, 900, 50, 3000)))
    ws = _workspace(w)
    got = _run(w, x, q, qs, schedule="balanced", ws=ws)
    _check_sampled_rows(x, q, qs, got, "many pieces", 19, first=np.arange(60))
    assert pkv.pkv_device_error() == 0
    assert _tickets_clear(ws)


def test_balanced_workspace_is_reusable():
    """Calls that complete leave the tickets at zero: the same workspace serves the next call, with
    the same result bit for bit, and a different batch after it."""
    w, x, q, qs = _case("qwen2.5-7b", 15, [100, 7, 260, 33], B=4, num_blocks=2048, ctx=("uniform", 300, 3000))
    ws = _workspace(w)
    first = _run(w, x, q, qs, schedule="balanced", ws=ws)
    assert _tickets_clear(ws)
    second = _run(w, x, q, qs, schedule="balanced", ws=ws)
    assert np.array_equal(first.view(np.uint16), second.view(np.uint16))
    _check_sampled_rows(x, q, qs, second, "reused workspace", 20)
    w2, x2, q2, qs2 = _case("qwen2.5-7b", 16, [1, 64], B=2, num_blocks=512, ctx=("uniform", 64, 900))
    assert_attention_close(_run(w2, x2, q2, qs2, schedule="balanced", ws=ws), _oracle(w2, x2, q2, qs2),
                           "another batch on the same workspace")
    assert pkv.pkv_device_error() == 0 and _tickets_clear(ws)


def test_balanced_small_work_uses_fewer_ctas():
    """Fewer KV tiles than 4 per SM: the schedule gives every CTA at least 4 and leaves the rest idle."""
    w, x, q, qs = _case("qwen2.5-1.5b", 17, [5, 130, 1], B=3, num_blocks=256, ctx=("uniform", 130, 700))
    assert_attention_close(_run(w, x, q, qs, schedule="balanced"), _oracle(w, x, q, qs), "few tiles")
    assert pkv.pkv_device_error() == 0


def test_balanced_workspace_too_small_is_rejected():
    w, x, q, qs = _case("tiny", 18, [17, 40])
    small = torch.zeros(pkv.paged_gqa_prefill_workspace_size(w.Hq, w.Hkv, w.head_dim) - 256, dtype=torch.uint8,
                        device="cuda")
    with pytest.raises(pkv.PagedKVError):
        _run(w, x, q, qs, schedule="balanced", ws=small)
