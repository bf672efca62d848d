"""Seeded synthetic inputs for paged GQA decode attention and the KV-cache write.

Shared by the tests, the benchmark and the smoke check. This module only
draws random numbers and lays them out (pools, block tables, lengths, slots);
it holds none of the attention, softmax or FP8 quantisation arithmetic, and it
imports neither the CUDA library nor the oracle.

Shapes follow the serving workloads the pages describe for Qwen2.5: 12 query
heads sharing 2 KV heads for the 1.5B model ("rvLLM 소개" (discuss.pytorch.kr),
§PagedAttention과 FlashAttention-3) at batch sizes 64-256 (same page, §H100 SXM
80GB 직접 엔진 벤치마크), and 28/4 heads for the 7B model; the pages name no
dataset, so everything here is synthetic:
  * q, K, V, new K/V: float32 N(0, 1) draws rounded to float16;
  * physical blocks: a seeded permutation of the whole pool; sequence b takes
    its ceil(L_b / block_size) blocks consecutively from that permutation;
  * unused block-table entries are -1; unused pool rows (free blocks and the
    rows past L_b in a sequence's last block) hold NaN, so any read of them
    would show in the output;
  * this step's token of sequence b sits at position L_b - 1 (the context
    length counts it) and is written there by the cache write;
  * FP8 workloads carry per-tensor scales fp32(max|x| / 448) over the pool's
    live values and the new tokens.
"""
from __future__ import annotations

from dataclasses import dataclass, field, replace

import numpy as np

E4M3_MAX = 448.0


@dataclass(frozen=True)
class Workload:
    """One decode-step workload. Context lengths are drawn by ``ctx``:
    ("fixed", (L0, L1, ...)), ("uniform", lo, hi) inclusive, or
    ("skewed", long_len, n_short, lo, hi): sequence 0 is long, the rest uniform."""
    name: str
    B: int
    Hq: int
    Hkv: int
    head_dim: int
    block_size: int
    num_blocks: int
    ctx: tuple
    kv_dtype: str = "f16"
    partition_tokens: int = 0
    description: str = ""
    extra: dict = field(default_factory=dict)

    @property
    def group(self) -> int:
        return self.Hq // self.Hkv

    @property
    def max_context_len(self) -> int:
        kind = self.ctx[0]
        if kind == "fixed":
            return max(self.ctx[1])
        if kind == "uniform":
            return self.ctx[2]
        if kind == "skewed":
            return max(self.ctx[1], self.ctx[4])
        raise ValueError(kind)

    @property
    def max_blocks_per_seq(self) -> int:
        return -(-self.max_context_len // self.block_size)


WORKLOADS = {
    "tiny": Workload(
        "tiny", B=2, Hq=12, Hkv=2, head_dim=128, block_size=16, num_blocks=64,
        ctx=("fixed", (17, 40)),
        description="tiny paged decode: B=2, context_lens {17,40}, Hq=12/Hkv=2, D=128, "
                    "bs=16, 64-block shuffled pool, cache write of 1 new token per seq"),
    "qwen2.5-1.5b": Workload(
        "qwen2.5-1.5b", B=64, Hq=12, Hkv=2, head_dim=128, block_size=16, num_blocks=16384,
        ctx=("uniform", 32, 2048),
        description="Qwen2.5-1.5B-shaped decode: B=64, Hq=12/Hkv=2, D=128, bs=16, "
                    "context_lens U[32,2048], f16 KV, 16k-block shuffled pool"),
    "qwen2.5-7b": Workload(
        "qwen2.5-7b", B=128, Hq=28, Hkv=4, head_dim=128, block_size=16, num_blocks=32768,
        ctx=("uniform", 512, 4096),
        description="Qwen2.5-7B-shaped decode: B=128, Hq=28/Hkv=4, D=128, bs=16, "
                    "context_lens U[512,4096], f16 KV, 32k-block shuffled pool, "
                    "cache write of 128 new tokens"),
    "fp8-e4m3": Workload(
        "fp8-e4m3", B=256, Hq=12, Hkv=2, head_dim=128, block_size=16, num_blocks=98304,
        ctx=("uniform", 1024, 8192), kv_dtype="fp8",
        description="FP8 E4M3 KV cache: B=256, Hq=12/Hkv=2, D=128, bs=16, context_lens "
                    "U[1024,8192], per-tensor fp32 scales, f16 q/out, 96k-block pool"),
    "skewed-split": Workload(
        "skewed-split", B=8, Hq=28, Hkv=4, head_dim=128, block_size=16, num_blocks=4096,
        ctx=("skewed", 32768, 7, 128, 1024), partition_tokens=512,
        description="skewed long-context split-KV: B=8, Hq=28/Hkv=4, D=128, bs=16, one "
                    "seq at 32768 tokens and seven U[128,1024], 512-token partitions"),
}


def with_sizes(w: Workload, **kw) -> Workload:
    """A copy of ``w`` with some fields replaced (for reduced test cases)."""
    return replace(w, **kw)


def draw_context_lens(w: Workload, rng: np.random.Generator) -> np.ndarray:
    kind = w.ctx[0]
    if kind == "fixed":
        lens = np.array(w.ctx[1], dtype=np.int32)
        if lens.size != w.B:
            raise ValueError("fixed lengths must list B values")
    elif kind == "uniform":
        lens = rng.integers(w.ctx[1], w.ctx[2] + 1, size=w.B).astype(np.int32)
    elif kind == "skewed":
        long_len, n_short, lo, hi = w.ctx[1:]
        if n_short + 1 != w.B:
            raise ValueError("skewed workload: B must be 1 + n_short")
        lens = np.concatenate([[long_len], rng.integers(lo, hi + 1, size=n_short)]).astype(np.int32)
    else:
        raise ValueError(kind)
    return lens


def draw_block_tables(w: Workload, lens: np.ndarray, rng: np.random.Generator) -> np.ndarray:
    """[B, max_blocks] int32: consecutive runs of a seeded pool permutation; -1 unused."""
    nb = -(-lens.astype(np.int64) // w.block_size)
    if nb.sum() > w.num_blocks:
        raise ValueError(f"{w.name}: pool of {w.num_blocks} blocks < {nb.sum()} needed")
    perm = rng.permutation(w.num_blocks).astype(np.int32)
    mb = max(w.max_blocks_per_seq, 1)
    bt = np.full((w.B, mb), -1, dtype=np.int32)
    pos = 0
    for b in range(w.B):
        bt[b, :nb[b]] = perm[pos:pos + nb[b]]
        pos += nb[b]
    return bt


def _normal_f16(rng: np.random.Generator, shape) -> np.ndarray:
    return rng.standard_normal(size=shape, dtype=np.float32).astype(np.float16)


def make_inputs(w: Workload, seed: int = 0, *, poison: bool = True) -> dict:
    """All inputs of one decode step of ``w``, as NumPy arrays.

    Keys: q [B,Hq,D] f16; k_pool, v_pool [NB,bs,Hkv,D] f16 (live rows N(0,1),
    other rows NaN when ``poison``, else 0); block_tables [B,max_blocks] i32;
    context_lens [B] i32; k_new, v_new [B,Hkv,D] f16; slot_mapping [B] i64
    (slot of position L_b - 1, -1 for an empty sequence); softmax_scale
    (fp32 1/sqrt(D)); k_scale, v_scale (fp32, FP8 workloads; 1.0 otherwise).
    For FP8 workloads the pools are the f16 values the cache is quantised from.
    """
    rng = np.random.default_rng(seed)
    B, Hq, Hkv, D, bs, NB = w.B, w.Hq, w.Hkv, w.head_dim, w.block_size, w.num_blocks
    lens = draw_context_lens(w, rng)
    bt = draw_block_tables(w, lens, rng)
    q = _normal_f16(rng, (B, Hq, D))
    fill = np.float16(np.nan) if poison else np.float16(0)
    k_pool = np.full((NB, bs, Hkv, D), fill, dtype=np.float16)
    v_pool = np.full((NB, bs, Hkv, D), fill, dtype=np.float16)
    amax_k = amax_v = 0.0
    for b in range(B):
        L = int(lens[b])
        nb = -(-L // bs)
        if nb == 0:
            continue
        blocks = bt[b, :nb]
        kv = _normal_f16(rng, (2, nb * bs, Hkv, D))
        kv[:, L:] = fill                     # tail rows of the last block stay unused
        k_pool[blocks] = kv[0].reshape(nb, bs, Hkv, D)
        v_pool[blocks] = kv[1].reshape(nb, bs, Hkv, D)
        if w.kv_dtype == "fp8":
            amax_k = max(amax_k, _amax(kv[0, :L]))
            amax_v = max(amax_v, _amax(kv[1, :L]))
    k_new = _normal_f16(rng, (B, Hkv, D))
    v_new = _normal_f16(rng, (B, Hkv, D))
    slot = np.full(B, -1, dtype=np.int64)
    for b in range(B):
        L = int(lens[b])
        if L > 0:
            slot[b] = int(bt[b, (L - 1) // bs]) * bs + (L - 1) % bs
    k_scale = v_scale = np.float32(1.0)
    if w.kv_dtype == "fp8":
        k_scale = np.float32(max(amax_k, _amax(k_new)) / E4M3_MAX)
        v_scale = np.float32(max(amax_v, _amax(v_new)) / E4M3_MAX)
    return dict(q=q, k_pool=k_pool, v_pool=v_pool, block_tables=bt, context_lens=lens,
                k_new=k_new, v_new=v_new, slot_mapping=slot,
                softmax_scale=np.float32(1.0 / np.sqrt(D)),
                k_scale=k_scale, v_scale=v_scale)


def _amax(x: np.ndarray) -> float:
    return float(np.abs(x.astype(np.float32)).max()) if x.size else 0.0


# Hidden sizes of the two Qwen2.5 shapes: H = Hq * D (12 * 128 and 28 * 128).
QKV_SHAPES = {
    "qwen2.5-1.5b": dict(T=64, H=1536, Hq=12, Hkv=2, D=128),
    "qwen2.5-7b": dict(T=128, H=3584, Hq=28, Hkv=4, D=128),
}
RMS_EPS = 1e-6


def make_qkv_inputs(T: int, H: int, Hq: int, Hkv: int, D: int, seed: int = 0, *,
                    bias: bool = True, outliers: bool = False) -> dict:
    """Inputs of the fused residual add + RMSNorm + QKV projection, as NumPy arrays.

    Keys: x [T,H] f16 ~ N(0,1) (the sublayer output); residual [T,H] f16 ~ N(0, 4^2)
    (the residual stream); gamma [H] f16 ~ N(1, 0.25^2); w_qkv [(Hq+2Hkv)D, H] f16
    ~ N(0, 1/H) (random-init weights, rows q heads | k heads | v heads); bias [N]
    f16 ~ N(0, 0.5^2) or None. ``outliers`` plants a few large residual channels
    (|value| up to 3e4, gamma up to 8 there), as real residual streams carry.
    """
    rng = np.random.default_rng(seed)
    N = (Hq + 2 * Hkv) * D
    x = _normal_f16(rng, (T, H))
    residual = (rng.standard_normal((T, H), dtype=np.float32) * 4.0).astype(np.float16)
    gamma = (1.0 + 0.25 * rng.standard_normal(H, dtype=np.float32)).astype(np.float16)
    w = (rng.standard_normal((N, H), dtype=np.float32) / np.float32(np.sqrt(H))).astype(np.float16)
    b = (0.5 * rng.standard_normal(N, dtype=np.float32)).astype(np.float16) if bias else None
    if outliers and T > 0:
        ch = rng.choice(H, size=min(4, H), replace=False)
        residual[:, ch] = (rng.choice([-1.0, 1.0], size=(T, ch.size)) *
                           rng.uniform(1e4, 3e4, size=(T, ch.size))).astype(np.float16)
        gamma[ch] = np.float16(8.0)
    return dict(x=x, residual=residual, gamma=gamma, w_qkv=w, bias=b)


def shard_seed(seed: int, rank: int) -> int:
    """Seed of rank ``rank`` when every rank runs its own batch (weak scaling)."""
    return seed * 1000003 + rank
