"""Paged GQA decode attention and paged KV-cache write for B200 (sm_100a).

A thin ctypes binding over the C ABI declared in ``include/pagedkv.h`` and
implemented by the in-tree CUDA library ``libpagedkv_b200.so``. The functions
here only marshal arguments (shapes, device pointers, the current CUDA stream)
and raise on a non-OK status: every step of the computation runs in the
library's kernels. There is no CPU fallback; importing this package fails if
the library has not been built (``python -m paged_kv_decode_gqa_b200.build``).

Tensors are torch CUDA tensors used as plain device memory:
  q, out            [B, Hq, D]              float16 (prefill: [total queries, Hq, D])
  k_cache, v_cache  [NB, block_size, Hkv, D] float16, or uint8 (FP8 E4M3 codes)
  k_new, v_new      [T, Hkv, D]             float16
  block_tables      [B, max_blocks]         int32
  context_lens      [B]                     int32
  slot_mapping      [T]                     int64
  query_start       [B + 1]                 int32 (prefill)
  x, residual       [T, H]                  float16 (QKV projection; w_qkv [N, H], gamma [H])
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
# PKV_LIBRARY may name another build of the same library (e.g. a tuning build).
LIBRARY_PATH = os.environ.get("PKV_LIBRARY") or os.path.join(_HERE, "libpagedkv_b200.so")

_P, _i32, _f32, _sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_float, ctypes.c_size_t
_SIGNATURES = {
    "paged_kv_cache_write": ([_P, _P, _P, _P, _P, _i32, _i32, _i32, _i32, _i32, _i32, _f32, _f32, _P],
                             ctypes.c_int),
    "paged_gqa_decode_workspace_size": ([_i32, _i32, _i32, _i32, _i32, _i32], _sz),
    "paged_gqa_decode_suggest_partition": ([_i32, _i32, _i32, _i32, _i32], _i32),
    "paged_gqa_decode_attention": ([_P, _P, _P, _P, _P, _P, _i32, _i32, _i32, _i32, _i32, _i32, _i32,
                                    _i32, _f32, _i32, _f32, _f32, _i32, _P, _sz, _P], ctypes.c_int),
    "paged_gqa_decode_step": ([_P, _P, _P, _P, _P, _P, _P, _P, _i32, _i32, _i32, _i32, _i32, _i32, _i32,
                               _i32, _f32, _i32, _f32, _f32, _P, _sz, ctypes.c_uint32, _P], ctypes.c_int),
    "pkv_status_string": ([ctypes.c_int], ctypes.c_char_p),
    "pkv_device_error": ([ctypes.POINTER(ctypes.c_uint32)], ctypes.c_int),
    "paged_gqa_decode_attention_static_workspace": (
        [_P, _P, _P, _P, _P, _P, _i32, _i32, _i32, _i32, _i32, _i32, _i32, _i32, _f32, _i32, _f32,
         _f32, _i32, _P], ctypes.c_int),
    "paged_kv_fp8_scales": ([_P, ctypes.c_int64, _i32, _i32, _i32, _P, _P], ctypes.c_int),
    "paged_kv_cache_write_fp8_scaled": ([_P, _P, _P, _P, _P, _i32, _i32, _i32, _i32, _i32, _P, _P, _i32, _P],
                                        ctypes.c_int),
    "paged_gqa_decode_attention_fp8_scaled": (
        [_P, _P, _P, _P, _P, _P, _i32, _i32, _i32, _i32, _i32, _i32, _i32, _i32, _f32, _P, _P, _i32, _i32,
         _P, _sz, _P], ctypes.c_int),
    "paged_gqa_decode_step_fp8_scaled": (
        [_P, _P, _P, _P, _P, _P, _P, _P, _i32, _i32, _i32, _i32, _i32, _i32, _i32, _i32, _f32, _P, _P, _i32,
         _P, _sz, ctypes.c_uint32, _P], ctypes.c_int),
    "fused_add_rmsnorm_qkv": ([_P, _P, _P, _P, _P, _P, _P, _P, _P, _i32, _i32, _i32, _i32, _i32, _f32,
                               ctypes.c_uint32, _P], ctypes.c_int),
    "fused_add_rmsnorm_qkv_plan": ([_i32, _i32, _i32, _i32, _i32, _P], ctypes.c_int),
    "paged_gqa_prefill_workspace_size": ([_i32, _i32, _i32, _i32], _sz),
    "paged_gqa_prefill_attention": ([_P, _P, _P, _P, _P, _P, _P, _i32, _i32, _i32, _i32, _i32, _i32, _i32,
                                     _i32, _i32, _i32, _f32, _i32, _f32, _f32, _P, _sz, _P], ctypes.c_int),
}
# The symbols include/pagedkv.h declares (checked by the CPU tests).
EXPORTED = tuple(_SIGNATURES)

_lib = None


def load_library() -> ctypes.CDLL:
    """The CUDA library, loaded on first use. Raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIBRARY_PATH):
            raise ImportError(
                f"CUDA library not built: {LIBRARY_PATH} is missing "
                "(run `python -m paged_kv_decode_gqa_b200.build`)")
        lib = ctypes.CDLL(LIBRARY_PATH)
        for name, (args, res) in _SIGNATURES.items():
            fn = getattr(lib, name)
            fn.argtypes = args
            fn.restype = res
        _lib = lib
    return _lib


def __getattr__(name):
    if name == "lib":
        return load_library()
    raise AttributeError(name)


PKV_OK, PKV_ERR_INVALID_ARG, PKV_ERR_UNSUPPORTED, PKV_ERR_WORKSPACE, PKV_ERR_CUDA = range(5)
PKV_KV_F16, PKV_KV_FP8_E4M3 = 0, 1
PKV_PARTITION_AUTO = -1         # partition_tokens: the library's load-balanced plan
PKV_STEP_OVERLAP_PREVIOUS = 0x1  # paged_gqa_decode_step flag (see include/pagedkv.h)
PKV_STEP_SELFTEST_WAIT_TIMEOUT = 0x100  # self-test: one worker loads nothing, its wait runs out
DEVERR_CONTEXT_LEN, DEVERR_BLOCK_ID, DEVERR_SLOT, DEVERR_WAIT_TIMEOUT, DEVERR_SCALE = 0x1, 0x2, 0x4, 0x8, 0x10
_KV_DTYPES = {"f16": PKV_KV_F16, "fp8": PKV_KV_FP8_E4M3}


class PagedKVError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        text = load_library().pkv_status_string(status).decode()
        super().__init__(f"{where}: {text} (status {status})")


def _check(status: int, where: str) -> None:
    if status != PKV_OK:
        raise PagedKVError(status, where)


def _stream(stream):
    if stream is None:
        import torch
        return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, int):
        return ctypes.c_void_p(stream)
    return ctypes.c_void_p(stream.cuda_stream)


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else ctypes.c_void_p(0)


def _dense(name, t, *dtypes):
    """Checks that `t` is a dense CUDA tensor of one of `dtypes` (names)."""
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if str(t.dtype).replace("torch.", "") not in dtypes:
        raise TypeError(f"{name} must be {' or '.join(dtypes)}, got {t.dtype}")


def kv_dtype_code(kv_dtype: str) -> int:
    try:
        return _KV_DTYPES[kv_dtype]
    except KeyError:
        raise ValueError(f"kv_dtype must be one of {sorted(_KV_DTYPES)}") from None


def paged_kv_cache_write(k_new, v_new, k_cache, v_cache, slot_mapping, *, kv_dtype="f16",
                         k_scale=1.0, v_scale=1.0, stream=None) -> None:
    """reshape_and_cache: k_cache[slot // bs, slot % bs] = k_new[i] (and V)."""
    cdt = "uint8" if kv_dtype == "fp8" else "float16"
    for n, t in (("k_new", k_new), ("v_new", v_new)):
        _dense(n, t, "float16")
    for n, t in (("k_cache", k_cache), ("v_cache", v_cache)):
        _dense(n, t, cdt)
    _dense("slot_mapping", slot_mapping, "int64")
    T, Hkv, D = k_new.shape
    NB, bs = k_cache.shape[0], k_cache.shape[1]
    _check(load_library().paged_kv_cache_write(
        _ptr(k_new), _ptr(v_new), _ptr(k_cache), _ptr(v_cache), _ptr(slot_mapping), T, Hkv, D, NB,
        bs, kv_dtype_code(kv_dtype), float(k_scale), float(v_scale), _stream(stream)),
        "paged_kv_cache_write")


def paged_gqa_decode_workspace_size(batch, num_q_heads, num_kv_heads, head_dim, max_context_len,
                                    partition_tokens) -> int:
    return int(load_library().paged_gqa_decode_workspace_size(
        batch, num_q_heads, num_kv_heads, head_dim, max_context_len, partition_tokens))


def paged_gqa_decode_suggest_partition(batch, num_kv_heads, max_context_len, block_size=16,
                                       sm_count=0) -> int:
    return int(load_library().paged_gqa_decode_suggest_partition(
        batch, num_kv_heads, max_context_len, block_size, sm_count))


def paged_gqa_decode_attention(out, q, k_cache, v_cache, block_tables, context_lens, *,
                               max_context_len, softmax_scale, kv_dtype="f16", k_scale=1.0,
                               v_scale=1.0, partition_tokens=0, workspace=None, stream=None) -> None:
    """out[b, h] = softmax(scale * q[b, h] . K^T) V over the paged context of b."""
    cdt = "uint8" if kv_dtype == "fp8" else "float16"
    _dense("out", out, "float16")
    _dense("q", q, "float16")
    _dense("k_cache", k_cache, cdt)
    _dense("v_cache", v_cache, cdt)
    _dense("block_tables", block_tables, "int32")
    _dense("context_lens", context_lens, "int32")
    if workspace is not None:
        _dense("workspace", workspace, "uint8", "float32", "int32")
    B, Hq, D = q.shape
    NB, bs, Hkv, _ = k_cache.shape
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check(load_library().paged_gqa_decode_attention(
        _ptr(out), _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_tables), _ptr(context_lens),
        B, Hq, Hkv, D, bs, block_tables.shape[1], NB, int(max_context_len), float(softmax_scale),
        kv_dtype_code(kv_dtype), float(k_scale), float(v_scale), int(partition_tokens),
        _ptr(workspace), ws_bytes, _stream(stream)), "paged_gqa_decode_attention")


def paged_gqa_decode_step(out, q, k_new, v_new, k_cache, v_cache, block_tables, context_lens, *,
                          max_context_len, softmax_scale, kv_dtype="f16", k_scale=1.0, v_scale=1.0,
                          workspace=None, flags=0, stream=None) -> None:
    """One decode step in one launch: k_new/v_new [B, Hkv, D] go to position
    context_lens[b] - 1 of each sequence's pages, then out = attention over the
    updated cache (the load-balanced plan; workspace sized for PKV_PARTITION_AUTO)."""
    cdt = "uint8" if kv_dtype == "fp8" else "float16"
    _dense("out", out, "float16")
    _dense("q", q, "float16")
    _dense("k_new", k_new, "float16")
    _dense("v_new", v_new, "float16")
    _dense("k_cache", k_cache, cdt)
    _dense("v_cache", v_cache, cdt)
    _dense("block_tables", block_tables, "int32")
    _dense("context_lens", context_lens, "int32")
    if workspace is not None:
        _dense("workspace", workspace, "uint8", "float32", "int32")
    B, Hq, D = q.shape
    NB, bs, Hkv, _ = k_cache.shape
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check(load_library().paged_gqa_decode_step(
        _ptr(out), _ptr(q), _ptr(k_new), _ptr(v_new), _ptr(k_cache), _ptr(v_cache), _ptr(block_tables),
        _ptr(context_lens), B, Hq, Hkv, D, bs, block_tables.shape[1], NB, int(max_context_len),
        float(softmax_scale), kv_dtype_code(kv_dtype), float(k_scale), float(v_scale), _ptr(workspace),
        ws_bytes, int(flags), _stream(stream)), "paged_gqa_decode_step")


def pkv_device_error() -> int:
    """Reads and clears the device error word (DEVERR_* bits). Synchronises the device."""
    flags = ctypes.c_uint32(0)
    _check(load_library().pkv_device_error(ctypes.byref(flags)), "pkv_device_error")
    return int(flags.value)


# Size of the library's own split-KV scratch (PKV_STATIC_WORKSPACE_BYTES).
STATIC_WORKSPACE_BYTES = 16 << 20


def paged_gqa_decode_attention_static_workspace(out, q, k_cache, v_cache, block_tables,
                                                context_lens, *, max_context_len, softmax_scale,
                                                kv_dtype="f16", k_scale=1.0, v_scale=1.0,
                                                partition_tokens=0, stream=None) -> None:
    """paged_gqa_decode_attention without a caller workspace, for callers that
    cannot allocate device memory (an engine that gave all free HBM to its KV
    pool, a step being captured into a CUDA graph, a foreign-language caller
    without the process's allocator). Split-KV scratch comes from a fixed
    STATIC_WORKSPACE_BYTES array inside the library, shared by every call on a
    device: calls must not overlap on the GPU. Sizes needing more scratch raise
    PagedKVError (workspace). The first call on a device looks up the array's
    address and should come before any stream capture."""
    cdt = "uint8" if kv_dtype == "fp8" else "float16"
    _dense("out", out, "float16")
    _dense("q", q, "float16")
    _dense("k_cache", k_cache, cdt)
    _dense("v_cache", v_cache, cdt)
    _dense("block_tables", block_tables, "int32")
    _dense("context_lens", context_lens, "int32")
    B, Hq, D = q.shape
    NB, bs, Hkv, _ = k_cache.shape
    _check(load_library().paged_gqa_decode_attention_static_workspace(
        _ptr(out), _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_tables), _ptr(context_lens),
        B, Hq, Hkv, D, bs, block_tables.shape[1], NB, int(max_context_len), float(softmax_scale),
        kv_dtype_code(kv_dtype), float(k_scale), float(v_scale), int(partition_tokens),
        _stream(stream)), "paged_gqa_decode_attention_static_workspace")


# ----------------------------------------------------------------------------
# FP8 E4M3 caches with device-side scales: one float per tensor, or one per KV
# head (float32 CUDA tensors of 1 or Hkv elements).

def _scales(k_scales, v_scales, Hkv):
    _dense("k_scales", k_scales, "float32")
    _dense("v_scales", v_scales, "float32")
    n = k_scales.numel()
    if v_scales.numel() != n or n not in (1, Hkv):
        raise ValueError("k_scales and v_scales need 1 (per tensor) or num_kv_heads (per head) elements")
    return int(n == Hkv and Hkv > 1)


def paged_kv_fp8_scales(x, scales, *, per_head, stream=None) -> None:
    """scales[h] = max|x[:, h, :]| / 448 over the non-NaN elements of x [rows, Hkv, D]
    float16 (per KV head), or of all of x (per_head=False, one scale); 1 for a maximum of 0."""
    _dense("x", x, "float16")
    _dense("scales", scales, "float32")
    rows, Hkv, D = x.shape
    if scales.numel() != (Hkv if per_head else 1):
        raise ValueError("scales needs num_kv_heads elements per head, else 1")
    _check(load_library().paged_kv_fp8_scales(_ptr(x), rows, Hkv, D, int(bool(per_head)), _ptr(scales),
                                              _stream(stream)), "paged_kv_fp8_scales")


def paged_kv_cache_write_fp8_scaled(k_new, v_new, k_cache, v_cache, slot_mapping, k_scales, v_scales, *,
                                    stream=None) -> None:
    """paged_kv_cache_write into an FP8 cache, quantising head h with k_scales[h] / v_scales[h]
    (or the single scale)."""
    for n, t in (("k_new", k_new), ("v_new", v_new)):
        _dense(n, t, "float16")
    for n, t in (("k_cache", k_cache), ("v_cache", v_cache)):
        _dense(n, t, "uint8")
    _dense("slot_mapping", slot_mapping, "int64")
    T, Hkv, D = k_new.shape
    NB, bs = k_cache.shape[0], k_cache.shape[1]
    per_head = _scales(k_scales, v_scales, Hkv)
    _check(load_library().paged_kv_cache_write_fp8_scaled(
        _ptr(k_new), _ptr(v_new), _ptr(k_cache), _ptr(v_cache), _ptr(slot_mapping), T, Hkv, D, NB, bs,
        _ptr(k_scales), _ptr(v_scales), per_head, _stream(stream)), "paged_kv_cache_write_fp8_scaled")


def paged_gqa_decode_attention_fp8_scaled(out, q, k_cache, v_cache, block_tables, context_lens, k_scales,
                                          v_scales, *, max_context_len, softmax_scale, partition_tokens=0,
                                          workspace=None, stream=None) -> None:
    """paged_gqa_decode_attention on an FP8 cache whose KV head g dequantises with
    k_scales[g] / v_scales[g] (or the single scale)."""
    _dense("out", out, "float16")
    _dense("q", q, "float16")
    _dense("k_cache", k_cache, "uint8")
    _dense("v_cache", v_cache, "uint8")
    _dense("block_tables", block_tables, "int32")
    _dense("context_lens", context_lens, "int32")
    if workspace is not None:
        _dense("workspace", workspace, "uint8", "float32", "int32")
    B, Hq, D = q.shape
    NB, bs, Hkv, _ = k_cache.shape
    per_head = _scales(k_scales, v_scales, Hkv)
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check(load_library().paged_gqa_decode_attention_fp8_scaled(
        _ptr(out), _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_tables), _ptr(context_lens),
        B, Hq, Hkv, D, bs, block_tables.shape[1], NB, int(max_context_len), float(softmax_scale),
        _ptr(k_scales), _ptr(v_scales), per_head, int(partition_tokens), _ptr(workspace), ws_bytes,
        _stream(stream)), "paged_gqa_decode_attention_fp8_scaled")


def paged_gqa_decode_step_fp8_scaled(out, q, k_new, v_new, k_cache, v_cache, block_tables, context_lens,
                                     k_scales, v_scales, *, max_context_len, softmax_scale, workspace=None,
                                     flags=0, stream=None) -> None:
    """paged_gqa_decode_step on an FP8 cache with device-side scales (per tensor or per KV head)."""
    _dense("out", out, "float16")
    _dense("q", q, "float16")
    _dense("k_new", k_new, "float16")
    _dense("v_new", v_new, "float16")
    _dense("k_cache", k_cache, "uint8")
    _dense("v_cache", v_cache, "uint8")
    _dense("block_tables", block_tables, "int32")
    _dense("context_lens", context_lens, "int32")
    if workspace is not None:
        _dense("workspace", workspace, "uint8", "float32", "int32")
    B, Hq, D = q.shape
    NB, bs, Hkv, _ = k_cache.shape
    per_head = _scales(k_scales, v_scales, Hkv)
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check(load_library().paged_gqa_decode_step_fp8_scaled(
        _ptr(out), _ptr(q), _ptr(k_new), _ptr(v_new), _ptr(k_cache), _ptr(v_cache), _ptr(block_tables),
        _ptr(context_lens), B, Hq, Hkv, D, bs, block_tables.shape[1], NB, int(max_context_len),
        float(softmax_scale), _ptr(k_scales), _ptr(v_scales), per_head, _ptr(workspace), ws_bytes,
        int(flags), _stream(stream)), "paged_gqa_decode_step_fp8_scaled")


def fused_add_rmsnorm_qkv(x, residual, gamma, w_qkv, bias, residual_out, q, k_new, v_new, *, eps=1e-6,
                          flags=0, stream=None) -> None:
    """residual_out = x + residual (f16); q, k_new, v_new = the QKV projection of its RMSNorm.

    x, residual, residual_out [T, H]; gamma [H]; w_qkv [(Hq + 2 Hkv) D, H] (rows q heads | k | v);
    bias [N] or None; q [T, Hq, D]; k_new, v_new [T, Hkv, D]; all float16.
    """
    for n, t in (("x", x), ("residual", residual), ("gamma", gamma), ("w_qkv", w_qkv),
                 ("residual_out", residual_out), ("q", q), ("k_new", k_new), ("v_new", v_new)):
        _dense(n, t, "float16")
    if bias is not None:
        _dense("bias", bias, "float16")
    T, H = x.shape
    _, Hq, D = q.shape
    Hkv = k_new.shape[1]
    if (residual.shape != (T, H) or residual_out.shape != (T, H) or gamma.shape != (H,)
            or q.shape != (T, Hq, D) or k_new.shape != (T, Hkv, D) or v_new.shape != (T, Hkv, D)
            or w_qkv.shape != ((Hq + 2 * Hkv) * D, H)
            or (bias is not None and bias.shape != ((Hq + 2 * Hkv) * D,))):
        raise ValueError("shape mismatch")
    _check(load_library().fused_add_rmsnorm_qkv(
        _ptr(x), _ptr(residual), _ptr(gamma), _ptr(w_qkv), _ptr(bias), _ptr(residual_out), _ptr(q),
        _ptr(k_new), _ptr(v_new), T, H, Hq, Hkv, D, float(eps), int(flags), _stream(stream)),
        "fused_add_rmsnorm_qkv")


def fused_add_rmsnorm_qkv_plan(T, H, Hq, Hkv, D) -> dict:
    """The launch plan of fused_add_rmsnorm_qkv for these sizes on the current device."""
    plan = (ctypes.c_int32 * 5)()
    _check(load_library().fused_add_rmsnorm_qkv_plan(T, H, Hq, Hkv, D, plan), "fused_add_rmsnorm_qkv_plan")
    return dict(zip(("tile_rows", "slices", "token_tile", "ctas", "token_tiles"), list(plan)))


def paged_gqa_prefill_workspace_size(num_q_heads, num_kv_heads, head_dim, kv_dtype="f16") -> int:
    """Bytes of workspace for the load-balanced prefill schedule on the current device (0: none)."""
    return int(load_library().paged_gqa_prefill_workspace_size(num_q_heads, num_kv_heads, head_dim,
                                                                kv_dtype_code(kv_dtype)))


def paged_gqa_prefill_attention(out, q, k_cache, v_cache, block_tables, context_lens, query_start, *,
                                max_query_len, max_context_len, softmax_scale, kv_dtype="f16",
                                k_scale=1.0, v_scale=1.0, workspace=None, stream=None) -> None:
    """Chunked prefill: query rows q [total, Hq, D] of each sequence (query_start [B+1] int32), the
    last n_b tokens of its context, attending causally through the block tables; out [total, Hq, D].
    With a zero-filled workspace of paged_gqa_prefill_workspace_size bytes the f16 kernel balances
    its work over the SMs (items cut at CTA boundaries and merged); without one, whole items."""
    _dense("out", out, "float16")
    _dense("q", q, "float16")
    for n, t in (("k_cache", k_cache), ("v_cache", v_cache)):
        _dense(n, t, "float16", "uint8")
    _dense("block_tables", block_tables, "int32")
    _dense("context_lens", context_lens, "int32")
    _dense("query_start", query_start, "int32")
    total, Hq, D = q.shape
    NB, bs, Hkv, _ = k_cache.shape
    B = context_lens.shape[0]
    if out.shape != q.shape or query_start.shape[0] != B + 1:
        raise ValueError("shape mismatch")
    if workspace is not None:
        _dense("workspace", workspace, "uint8", "float32", "int32")
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check(load_library().paged_gqa_prefill_attention(
        _ptr(out), _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_tables), _ptr(context_lens), _ptr(query_start),
        B, total, int(max_query_len), Hq, Hkv, D, bs, block_tables.shape[1], NB, int(max_context_len),
        float(softmax_scale), kv_dtype_code(kv_dtype), float(k_scale), float(v_scale), _ptr(workspace), ws_bytes,
        _stream(stream)), "paged_gqa_prefill_attention")
