"""Float64 CPU oracle for paged GQA decode attention and the paged KV-cache write.

TEST INFRASTRUCTURE ONLY. Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package. The CUDA library
under ``paged_kv_decode_gqa_b200`` never imports, links or calls it, and the
two share no code: this package wraps ``pkv_oracle.c`` (plain C, float64),
compiled here with gcc into ``oracle/_build/liboracle.so``.

What each function computes, and the readings it takes where the pages are
silent, is stated in ``pkv_oracle.c``. Sources: "rvLLM 소개"
(discuss.pytorch.kr), §PagedAttention과 FlashAttention-3 (paged KV cache,
grouped-query heads, f16 and FP8 E4M3 caches), §퓨즈드 CUDA 커널 (the fused
Add+RMSNorm+QKV step before attention) and the vLLM talk summary (aitrends.kr),
§용어 해설 (KV cache, PagedAttention).

Arrays are NumPy. binary16 data is passed as ``np.float16`` (its bits are
read, never converted by NumPy); FP8 caches are ``np.uint8`` codes.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "pkv_oracle.c")
_BUILD_DIR = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_BUILD_DIR, "liboracle.so")
_CFLAGS = ["-O2", "-fopenmp", "-fPIC", "-shared", "-ffp-contract=off", "-fno-fast-math", "-std=c11"]

_lib = None


def build(force: bool = False) -> str:
    """Compile ``pkv_oracle.c`` with gcc (no-op when the library is current)."""
    os.makedirs(_BUILD_DIR, exist_ok=True)
    stale = (not os.path.exists(_LIB_PATH)
             or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC))
    if force or stale:
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.run(["gcc", *_CFLAGS, "-o", tmp, _SRC, "-lm"], check=True)
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        P = ctypes.c_void_p
        i32, i64, f32 = ctypes.c_int, ctypes.c_int64, ctypes.c_float
        lib.oracle_f16_to_f64.argtypes = [ctypes.c_uint16]
        lib.oracle_f16_to_f64.restype = ctypes.c_double
        lib.oracle_e4m3_to_f64.argtypes = [ctypes.c_uint8]
        lib.oracle_e4m3_to_f64.restype = ctypes.c_double
        lib.oracle_e4m3_from_f32.argtypes = [ctypes.c_float]
        lib.oracle_e4m3_from_f32.restype = ctypes.c_uint8
        lib.oracle_quantize_e4m3.argtypes = [P, i64, f32, P]
        lib.oracle_quantize_e4m3.restype = None
        lib.oracle_paged_kv_cache_write.argtypes = [P, P, P, P, P, i32, i32, i32, i32, i32, i32, f32, f32]
        lib.oracle_paged_kv_cache_write.restype = i32
        lib.oracle_paged_gqa_decode.argtypes = [P, P, P, P, P, P, P, i32, i32, i32, i32, i32,
                                                i32, i32, f32, i32, f32, f32, i32]
        lib.oracle_paged_gqa_decode.restype = i32
        lib.oracle_paged_kv_cache_write_scaled.argtypes = [P, P, P, P, P, i32, i32, i32, i32, i32, i32, P, P]
        lib.oracle_paged_kv_cache_write_scaled.restype = i32
        lib.oracle_paged_gqa_decode_scaled.argtypes = [P, P, P, P, P, P, P, i32, i32, i32, i32, i32,
                                                       i32, i32, f32, i32, P, P, i32]
        lib.oracle_paged_gqa_decode_scaled.restype = i32
        lib.oracle_absmax_f16.argtypes = [P, i64, i32, i32, i32, P]
        lib.oracle_absmax_f16.restype = None
        lib.oracle_fp8_scale_from_amax.argtypes = [f32]
        lib.oracle_fp8_scale_from_amax.restype = f32
        lib.oracle_f16_from_f64.argtypes = [ctypes.c_double]
        lib.oracle_f16_from_f64.restype = ctypes.c_uint16
        lib.oracle_add_rmsnorm_qkv.argtypes = [P, P, P, P, P, i32, i32, i32, ctypes.c_double, P, P]
        lib.oracle_add_rmsnorm_qkv.restype = i32
        lib.oracle_paged_prefill.argtypes = [P, P, P, P, P, P, P, P, i32, i32, i32, i32, i32, i32, i32,
                                             f32, i32, f32, f32]
        lib.oracle_paged_prefill.restype = i32
        lib.oracle_num_threads.argtypes = []
        lib.oracle_num_threads.restype = i32
        _lib = lib
    return _lib


def _ptr(a: np.ndarray):
    return ctypes.c_void_p(a.ctypes.data) if a is not None else None


def _c(a: np.ndarray, dtype) -> np.ndarray:
    a = np.asarray(a)
    if a.dtype != dtype:
        raise TypeError(f"expected {np.dtype(dtype)}, got {a.dtype}")
    return np.ascontiguousarray(a)


def num_threads() -> int:
    """Threads the oracle's OpenMP loops use (OMP_NUM_THREADS, else all cores)."""
    return int(_load().oracle_num_threads())


def f16_to_f64(bits: np.ndarray) -> np.ndarray:
    """Decode binary16 codes (uint16) to float64 from the IEEE definition."""
    lib = _load()
    bits = np.asarray(bits, dtype=np.uint16).ravel()
    return np.array([lib.oracle_f16_to_f64(int(b)) for b in bits], dtype=np.float64)


def e4m3_to_f64(codes: np.ndarray) -> np.ndarray:
    """Decode E4M3 codes (uint8) to float64 from the OCP E4M3 definition."""
    lib = _load()
    codes = np.asarray(codes, dtype=np.uint8).ravel()
    return np.array([lib.oracle_e4m3_to_f64(int(c)) for c in codes], dtype=np.float64)


def e4m3_from_f32(x: np.ndarray) -> np.ndarray:
    """Round fp32 values to E4M3 codes: nearest, ties to even, saturate at 448."""
    lib = _load()
    x = np.asarray(x, dtype=np.float32).ravel()
    return np.array([lib.oracle_e4m3_from_f32(float(v)) for v in x], dtype=np.uint8)


def quantize_e4m3(x_f16: np.ndarray, scale: float) -> np.ndarray:
    """E4M3 codes of ``fp32(x) / scale`` (division in fp32); same shape as x."""
    x = _c(x_f16, np.float16)
    out = np.empty(x.shape, dtype=np.uint8)
    _load().oracle_quantize_e4m3(_ptr(x), x.size, ctypes.c_float(scale), _ptr(out))
    return out


def _head_scales(scale, Hkv):
    """A scale argument as float32[Hkv]: per KV head if it has Hkv entries, else one per-tensor value."""
    a = np.asarray(scale, dtype=np.float32).ravel()
    if a.size == 1:
        return np.full(Hkv, a[0], dtype=np.float32), False
    if a.size != Hkv:
        raise ValueError("a per-head scale needs one value per KV head")
    return np.ascontiguousarray(a), True


def paged_kv_cache_write(k_new, v_new, k_cache, v_cache, slot_mapping, *,
                         kv_dtype: str = "f16", k_scale=1.0, v_scale=1.0):
    """In-place cache write on NumPy copies of the caches (reshape_and_cache).

    k_new, v_new: [T, Hkv, D] float16. k_cache, v_cache: [NB, bs, Hkv, D],
    float16 or uint8 (FP8 codes). slot_mapping: [T] int64, negative = skip.
    k_scale / v_scale: one per-tensor value, or one value per KV head.
    """
    k_new = _c(k_new, np.float16)
    v_new = _c(v_new, np.float16)
    fp8 = kv_dtype == "fp8"
    cdt = np.uint8 if fp8 else np.float16
    if k_cache.dtype != cdt or v_cache.dtype != cdt:
        raise TypeError("cache dtype does not match kv_dtype")
    if not (k_cache.flags.c_contiguous and v_cache.flags.c_contiguous):
        raise ValueError("caches must be C-contiguous")
    slots = _c(slot_mapping, np.int64)
    T, Hkv, D = k_new.shape
    NB, bs = k_cache.shape[0], k_cache.shape[1]
    ks, k_ph = _head_scales(k_scale, Hkv)
    vs, v_ph = _head_scales(v_scale, Hkv)
    if k_ph or v_ph:
        rc = _load().oracle_paged_kv_cache_write_scaled(_ptr(k_new), _ptr(v_new), _ptr(k_cache),
                                                        _ptr(v_cache), _ptr(slots), T, Hkv, D, NB, bs,
                                                        int(fp8), _ptr(ks), _ptr(vs))
    else:
        rc = _load().oracle_paged_kv_cache_write(_ptr(k_new), _ptr(v_new), _ptr(k_cache), _ptr(v_cache),
                                                 _ptr(slots), T, Hkv, D, NB, bs, int(fp8),
                                                 ctypes.c_float(ks[0]), ctypes.c_float(vs[0]))
    if rc != 0:
        raise ValueError("slot outside the pool")


def paged_gqa_decode(q, k_cache, v_cache, block_tables, context_lens, softmax_scale, *,
                     kv_dtype: str = "f16", k_scale=1.0, v_scale=1.0,
                     partition_tokens: int = 0, return_lse: bool = False):
    """Decode attention in float64 through the block tables.

    q: [B, Hq, D] float16. k_cache, v_cache: [NB, bs, Hkv, D] float16 or
    uint8 (FP8). block_tables: [B, max_blocks] int32. context_lens: [B] int32.
    k_scale / v_scale (FP8): one per-tensor value, or one value per KV head.
    Returns out [B, Hq, D] float64 (and lse [B, Hq] float64 if asked).
    """
    q = _c(q, np.float16)
    fp8 = kv_dtype == "fp8"
    cdt = np.uint8 if fp8 else np.float16
    k_cache = _c(k_cache, cdt)
    v_cache = _c(v_cache, cdt)
    bt = _c(block_tables, np.int32)
    cl = _c(context_lens, np.int32)
    B, Hq, D = q.shape
    NB, bs, Hkv, D2 = k_cache.shape
    if D2 != D or v_cache.shape != k_cache.shape:
        raise ValueError("shape mismatch")
    out = np.zeros((B, Hq, D), dtype=np.float64)
    lse = np.zeros((B, Hq), dtype=np.float64)
    ks, k_ph = _head_scales(k_scale, Hkv)
    vs, v_ph = _head_scales(v_scale, Hkv)
    if k_ph or v_ph:
        rc = _load().oracle_paged_gqa_decode_scaled(_ptr(out), _ptr(lse), _ptr(q), _ptr(k_cache),
                                                    _ptr(v_cache), _ptr(bt), _ptr(cl), B, Hq, Hkv, D, bs,
                                                    bt.shape[1], NB, ctypes.c_float(softmax_scale),
                                                    int(fp8), _ptr(ks), _ptr(vs), int(partition_tokens))
    else:
        rc = _load().oracle_paged_gqa_decode(_ptr(out), _ptr(lse), _ptr(q), _ptr(k_cache), _ptr(v_cache),
                                             _ptr(bt), _ptr(cl), B, Hq, Hkv, D, bs, bt.shape[1], NB,
                                             ctypes.c_float(softmax_scale), int(fp8),
                                             ctypes.c_float(ks[0]), ctypes.c_float(vs[0]),
                                             int(partition_tokens))
    if rc == -1:
        raise ValueError("block table entry outside the pool")
    if rc != 0:
        raise ValueError("bad head counts or context length")
    return (out, lse) if return_lse else out


def absmax_f16(x, per_head: bool):
    """Largest |x| over the non-NaN elements of x [rows, Hkv, D] float16: float32[Hkv]
    per KV head, or float32[1] over the tensor; 0 where nothing counts."""
    x = _c(x, np.float16)
    if x.ndim != 3:
        raise ValueError("x must be [rows, Hkv, D]")
    rows, Hkv, D = x.shape
    out = np.zeros(Hkv if per_head else 1, dtype=np.float32)
    _load().oracle_absmax_f16(_ptr(x), rows, Hkv, D, int(bool(per_head)), _ptr(out))
    return out


def fp8_scale_from_amax(amax):
    """E4M3 cache scale(s) fp32(amax) / 448 (fp32 division); 1 where amax is 0."""
    a = np.asarray(amax, dtype=np.float32).ravel()
    lib = _load()
    return np.array([lib.oracle_fp8_scale_from_amax(float(v)) for v in a], dtype=np.float32)


def fp8_scales(x, per_head: bool):
    """Scales an E4M3 cache would use for the data x [rows, Hkv, D] float16."""
    return fp8_scale_from_amax(absmax_f16(x, per_head))


def f16_from_f64(x) -> np.ndarray:
    """Round float64 values to binary16 codes (uint16): nearest, ties to even, overflow to inf."""
    lib = _load()
    x = np.asarray(x, dtype=np.float64).ravel()
    return np.array([lib.oracle_f16_from_f64(float(v)) for v in x], dtype=np.uint16)


def add_rmsnorm_qkv(x, residual, gamma, w_qkv, bias, eps, Hq, Hkv, D):
    """Residual add, RMSNorm and QKV projection of one decode step, in float64.

    x, residual: [T, H] float16. gamma: [H] float16. w_qkv: [(Hq + 2 Hkv) D, H]
    float16, rows ordered query heads, key heads, value heads. bias: [N]
    float16 or None. Returns (residual_out [T, H] float16, q [T, Hq, D],
    k [T, Hkv, D], v [T, Hkv, D] float64).
    """
    x = _c(x, np.float16)
    residual = _c(residual, np.float16)
    gamma = _c(gamma, np.float16)
    w_qkv = _c(w_qkv, np.float16)
    T, H = x.shape
    N = (Hq + 2 * Hkv) * D
    if residual.shape != (T, H) or gamma.shape != (H,) or w_qkv.shape != (N, H):
        raise ValueError("shape mismatch")
    if bias is not None:
        bias = _c(bias, np.float16)
        if bias.shape != (N,):
            raise ValueError("bias must be [N]")
    res_out = np.empty((T, H), dtype=np.float16)
    qkv = np.empty((T, N), dtype=np.float64)
    rc = _load().oracle_add_rmsnorm_qkv(_ptr(x), _ptr(residual), _ptr(gamma), _ptr(w_qkv), _ptr(bias),
                                        T, H, N, float(eps), _ptr(res_out), _ptr(qkv))
    if rc != 0:
        raise ValueError("bad sizes or eps")
    q = qkv[:, :Hq * D].reshape(T, Hq, D)
    k = qkv[:, Hq * D:(Hq + Hkv) * D].reshape(T, Hkv, D)
    v = qkv[:, (Hq + Hkv) * D:].reshape(T, Hkv, D)
    return res_out, q, k, v


def paged_prefill(q, k_cache, v_cache, block_tables, context_lens, query_start, softmax_scale, *,
                  kv_dtype: str = "f16", k_scale: float = 1.0, v_scale: float = 1.0, return_lse: bool = False):
    """Chunked prefill attention in float64 through the block tables (reading R12).

    q: [total, Hq, D] float16, the n_b = query_start[b+1] - query_start[b] new tokens of each
    sequence b, which are the last n_b of its context_lens[b] tokens (already in the cache).
    k_cache, v_cache: [NB, bs, Hkv, D] float16 or uint8 (FP8). block_tables: [B, max_blocks]
    int32. context_lens: [B] int32. query_start: [B + 1] int32. Returns out [total, Hq, D]
    float64 (and lse [total, Hq]).
    """
    q = _c(q, np.float16)
    fp8 = kv_dtype == "fp8"
    cdt = np.uint8 if fp8 else np.float16
    k_cache = _c(k_cache, cdt)
    v_cache = _c(v_cache, cdt)
    bt = _c(block_tables, np.int32)
    cl = _c(context_lens, np.int32)
    qs = _c(query_start, np.int32)
    total, Hq, D = q.shape
    NB, bs, Hkv, D2 = k_cache.shape
    B = cl.shape[0]
    if D2 != D or v_cache.shape != k_cache.shape or qs.shape != (B + 1,) or qs[-1] != total:
        raise ValueError("shape mismatch")
    out = np.zeros((total, Hq, D), dtype=np.float64)
    lse = np.zeros((total, Hq), dtype=np.float64)
    rc = _load().oracle_paged_prefill(_ptr(out), _ptr(lse), _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(bt),
                                      _ptr(cl), _ptr(qs), B, Hq, Hkv, D, bs, bt.shape[1], NB,
                                      ctypes.c_float(softmax_scale), int(fp8), ctypes.c_float(k_scale),
                                      ctypes.c_float(v_scale))
    if rc == -1:
        raise ValueError("block table entry outside the pool")
    if rc != 0:
        raise ValueError("bad lengths or head counts")
    return (out, lse) if return_lse else out
