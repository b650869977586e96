"""fp64 CPU oracle for paged decode attention, reshape_and_cache and copy_blocks.

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, by ``__graft_entry__.smoke()``
and by the CPU-baseline / reference arm of ``bench.py``; never by the product
package.  It shares no code with the CUDA path.  All arithmetic lives in
``pa_oracle.c`` (plain C, fp64, libm ``exp``); this module only marshals numpy
arrays into it.

What each function follows (web pages on vLLM / PagedAttention):
  * ``decode`` -- "vLLM 深度解读", section 3 (PagedAttention CUDA kernel): the
    block-table gather of K/V rows, score = scale * q.k, softmax, weighted sum
    of V; GQA reading: query head hq uses KV head hq // (Hq/Hkv).
  * ``reshape_and_cache`` -- "vLLM 深度解读", section 7 (the attention layer
    stores each new token's K/V into its slot before attention runs).
  * ``copy_blocks`` -- "详解vLLM推理引擎架构", section "Copy-on-Write 与内存共享"
    (copy_block(old, new) before writing a shared block).
  * ``swap_blocks`` -- "详解vLLM推理引擎架构", scheduler section (preempted requests' KV
    cache swapped out to CPU memory and back).
  * ``reshape_and_cache_e4m3`` / ``decode(..., kv_dtype="e4m3")`` -- the FP8 KV cache of
    "详解vLLM推理引擎架构", section "量化集成与部署" (--kv-cache-dtype fp8), read as OCP E4M3
    codes with one fp32 scale for K and one for V.

Every function is pinned in ``tests/test_oracle_pins.py`` against things other
than itself: the pages' block-table example, closed forms, torch's
scaled_dot_product_attention (fp64) on contiguous K/V, numpy fancy indexing for
the cache operations, and invariants (placement permutation, shared prefixes,
copy-on-write, GQA == MHA with repeated KV).
"""
import ctypes
import os

import numpy as np

from . import build as _build

DTYPES = {"f32": 0, "f16": 1, "bf16": 2, "e4m3": 3}
ELEM_BYTES = {"f32": 4, "f16": 2, "bf16": 2, "e4m3": 1}

_lib = None


def _load(path=None):
    global _lib
    if path is not None:
        lib = ctypes.CDLL(path)
    else:
        if _lib is not None:
            return _lib
        lib = ctypes.CDLL(_build.build())
    P = ctypes.c_void_p
    i32, i64 = ctypes.c_int, ctypes.c_int64
    lib.oracle_decode.argtypes = [P, P, i32, P, P, i32, P, P, i32, i32, i32, i32, i32, i32, i64,
                                  ctypes.c_float, i32]
    lib.oracle_decode.restype = i32
    lib.oracle_reshape_and_cache.argtypes = [P, P, P, P, P, i64, i32, i32, i32, i64, i32, i64, i64]
    lib.oracle_reshape_and_cache.restype = i32
    lib.oracle_copy_blocks.argtypes = [P, P, P, i64, i64, i64]
    lib.oracle_copy_blocks.restype = i32
    lib.oracle_decode_scaled.argtypes = [P, P, i32, P, P, i32, P, P, i32, i32, i32, i32, i32, i32, i64,
                                         ctypes.c_float, ctypes.c_float, ctypes.c_float, i32]
    lib.oracle_decode_scaled.restype = i32
    lib.oracle_decode_multi.argtypes = [P, P, i32, P, P, i32, P, P, i32, i32, i32, i32, i32, i32, i32, i64,
                                        ctypes.c_float, i32]
    lib.oracle_decode_multi.restype = i32
    lib.oracle_reshape_and_cache_e4m3.argtypes = [P, P, P, P, P, i64, i32, i32, i32, i64, i32,
                                                  ctypes.c_float, ctypes.c_float, i64, i64]
    lib.oracle_reshape_and_cache_e4m3.restype = i32
    lib.oracle_e4m3_to_f64.argtypes = [ctypes.c_uint8]
    lib.oracle_e4m3_to_f64.restype = ctypes.c_double
    lib.oracle_f32_to_e4m3.argtypes = [ctypes.c_float]
    lib.oracle_f32_to_e4m3.restype = ctypes.c_uint8
    lib.oracle_swap_blocks.argtypes = [P, P, P, P, P, i64, i64, i64, i64]
    lib.oracle_swap_blocks.restype = i32
    lib.oracle_f16_to_f64.argtypes = [ctypes.c_uint16]
    lib.oracle_f16_to_f64.restype = ctypes.c_double
    lib.oracle_bf16_to_f64.argtypes = [ctypes.c_uint16]
    lib.oracle_bf16_to_f64.restype = ctypes.c_double
    if path is None:
        _lib = lib
    return lib


class OracleError(RuntimeError):
    pass


def _ptr(a: np.ndarray):
    return ctypes.c_void_p(a.ctypes.data)


def _check_storage(a: np.ndarray, dtype: str, name: str):
    want = {"f32": np.float32, "e4m3": np.uint8}.get(dtype, np.uint16)
    if a.dtype != want:
        raise TypeError(f"{name}: {dtype} data must be stored as {np.dtype(want)}, got {a.dtype}")
    if not a.flags.c_contiguous:
        raise ValueError(f"{name} must be C-contiguous")


def default_threads() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1


def decode(q, q_dtype, k_cache, v_cache, kv_dtype, block_tables, seq_lens, scale,
           num_threads=None, lib=None, k_scale=1.0, v_scale=1.0):
    """fp64 paged decode attention.

    q: [N, Hq, D] (float32 for "f32", uint16 bit patterns for "f16"/"bf16");
    k_cache, v_cache: [NB, bs, Hkv, D] in kv_dtype storage (uint8 codes for "e4m3", whose
    values are code * k_scale and code * v_scale); block_tables int32 [N, MB]; seq_lens
    int32 [N].  Returns float64 [N, Hq, D].
    """
    lib = lib or _load()
    _check_storage(q, q_dtype, "q")
    _check_storage(k_cache, kv_dtype, "k_cache")
    _check_storage(v_cache, kv_dtype, "v_cache")
    block_tables = np.ascontiguousarray(block_tables, dtype=np.int32)
    seq_lens = np.ascontiguousarray(seq_lens, dtype=np.int32)
    N, Hq, D = q.shape
    NB, bs, Hkv, D2 = k_cache.shape
    if D2 != D or v_cache.shape != k_cache.shape:
        raise ValueError("shape mismatch between q and the caches")
    if block_tables.ndim != 2 or block_tables.shape[0] != N or seq_lens.shape != (N,):
        raise ValueError("block_tables must be [N, MB] and seq_lens [N]")
    MB = block_tables.shape[1]
    out = np.zeros((N, Hq, D), dtype=np.float64)
    threads = num_threads if num_threads else default_threads()
    if kv_dtype == "e4m3":
        rc = lib.oracle_decode_scaled(_ptr(out), _ptr(q), DTYPES[q_dtype], _ptr(k_cache), _ptr(v_cache),
                                      DTYPES[kv_dtype], _ptr(block_tables), _ptr(seq_lens), N, Hq, Hkv, D, bs,
                                      MB, NB, ctypes.c_float(scale), ctypes.c_float(k_scale),
                                      ctypes.c_float(v_scale), threads)
    else:
        rc = lib.oracle_decode(_ptr(out), _ptr(q), DTYPES[q_dtype], _ptr(k_cache), _ptr(v_cache),
                               DTYPES[kv_dtype], _ptr(block_tables), _ptr(seq_lens), N, Hq, Hkv, D, bs,
                               MB, NB, ctypes.c_float(scale), threads)
    if rc != 0:
        raise OracleError(f"oracle_decode failed with status {rc}")
    return out


def decode_multi(q, q_dtype, k_cache, v_cache, kv_dtype, block_tables, seq_lens, scale, num_threads=None,
                 lib=None):
    """fp64 causal multi-token attention over the paged cache.

    q: [N, T, Hq, D] in q_dtype storage; query token t of sequence i is the token at position
    seq_lens[i] - T + t and attends to tokens 0 .. seq_lens[i] - T + t (a sequence holds 0
    or at least T tokens).  Caches, block_tables and seq_lens as in decode (16-bit or f32
    caches).  Returns float64 [N, T, Hq, D].
    """
    lib = lib or _load()
    _check_storage(q, q_dtype, "q")
    _check_storage(k_cache, kv_dtype, "k_cache")
    _check_storage(v_cache, kv_dtype, "v_cache")
    if kv_dtype == "e4m3":
        raise ValueError("decode_multi takes a 16-bit or f32 cache")
    block_tables = np.ascontiguousarray(block_tables, dtype=np.int32)
    seq_lens = np.ascontiguousarray(seq_lens, dtype=np.int32)
    N, T, Hq, D = q.shape
    NB, bs, Hkv, D2 = k_cache.shape
    if D2 != D or v_cache.shape != k_cache.shape:
        raise ValueError("shape mismatch between q and the caches")
    if block_tables.ndim != 2 or block_tables.shape[0] != N or seq_lens.shape != (N,):
        raise ValueError("block_tables must be [N, MB] and seq_lens [N]")
    MB = block_tables.shape[1]
    out = np.zeros((N, T, Hq, D), dtype=np.float64)
    threads = num_threads if num_threads else default_threads()
    rc = lib.oracle_decode_multi(_ptr(out), _ptr(q), DTYPES[q_dtype], _ptr(k_cache), _ptr(v_cache),
                                 DTYPES[kv_dtype], _ptr(block_tables), _ptr(seq_lens), N, T, Hq, Hkv, D, bs, MB,
                                 NB, ctypes.c_float(scale), threads)
    if rc != 0:
        raise OracleError(f"oracle_decode_multi failed with status {rc}")
    return out


def reshape_and_cache(k, v, k_cache, v_cache, slot_mapping, kv_dtype, lib=None):
    """In place: write token t's K/V rows ([T, Hkv, D]) to slot slot_mapping[t] (skip if < 0)."""
    lib = lib or _load()
    for a, n in ((k, "k"), (v, "v"), (k_cache, "k_cache"), (v_cache, "v_cache")):
        _check_storage(a, kv_dtype, n)
    slot_mapping = np.ascontiguousarray(slot_mapping, dtype=np.int64)
    T, Hkv, D = k.shape
    NB, bs, Hkv2, D2 = k_cache.shape
    if (Hkv2, D2) != (Hkv, D) or v.shape != k.shape or slot_mapping.shape != (T,):
        raise ValueError("shape mismatch")
    rc = lib.oracle_reshape_and_cache(_ptr(k), _ptr(v), _ptr(k_cache), _ptr(v_cache),
                                      _ptr(slot_mapping), T, Hkv, D, bs, NB, ELEM_BYTES[kv_dtype],
                                      Hkv * D, Hkv * D)
    if rc != 0:
        raise OracleError(f"oracle_reshape_and_cache failed with status {rc}")


def reshape_and_cache_e4m3(k, v, k_cache, v_cache, slot_mapping, in_dtype, k_scale, v_scale, lib=None):
    """In place: quantise token t's K/V rows ([T, Hkv, D], in_dtype) to E4M3 codes
    e4m3(x / scale) at slot slot_mapping[t] of the uint8 caches (skip if < 0)."""
    lib = lib or _load()
    _check_storage(k, in_dtype, "k")
    _check_storage(v, in_dtype, "v")
    _check_storage(k_cache, "e4m3", "k_cache")
    _check_storage(v_cache, "e4m3", "v_cache")
    slot_mapping = np.ascontiguousarray(slot_mapping, dtype=np.int64)
    T, Hkv, D = k.shape
    NB, bs, Hkv2, D2 = k_cache.shape
    if (Hkv2, D2) != (Hkv, D) or v.shape != k.shape or slot_mapping.shape != (T,):
        raise ValueError("shape mismatch")
    rc = lib.oracle_reshape_and_cache_e4m3(_ptr(k), _ptr(v), _ptr(k_cache), _ptr(v_cache), _ptr(slot_mapping),
                                           T, Hkv, D, bs, NB, DTYPES[in_dtype], ctypes.c_float(k_scale),
                                           ctypes.c_float(v_scale), Hkv * D, Hkv * D)
    if rc != 0:
        raise OracleError(f"oracle_reshape_and_cache_e4m3 failed with status {rc}")


def copy_blocks(k_cache, v_cache, pairs, lib=None):
    """In place: for each (src, dst) row of pairs, in order, copy physical block src to dst."""
    lib = lib or _load()
    if not (k_cache.flags.c_contiguous and v_cache.flags.c_contiguous):
        raise ValueError("caches must be C-contiguous")
    pairs = np.ascontiguousarray(pairs, dtype=np.int32).reshape(-1, 2)
    NB = k_cache.shape[0]
    block_bytes = k_cache.nbytes // NB
    rc = lib.oracle_copy_blocks(_ptr(k_cache), _ptr(v_cache), _ptr(pairs), pairs.shape[0], NB,
                                block_bytes)
    if rc != 0:
        raise OracleError(f"oracle_copy_blocks failed with status {rc}")


def swap_blocks(dst_k, dst_v, src_k, src_v, pairs, lib=None):
    """In place: for each (src, dst) row of pairs, in order, copy block src of the source pool
    (src_k, src_v) to block dst of the destination pool (dst_k, dst_v)."""
    lib = lib or _load()
    for a in (dst_k, dst_v, src_k, src_v):
        if not a.flags.c_contiguous:
            raise ValueError("pools must be C-contiguous")
    pairs = np.ascontiguousarray(pairs, dtype=np.int32).reshape(-1, 2)
    block_bytes = src_k.nbytes // src_k.shape[0]
    if dst_k.nbytes // dst_k.shape[0] != block_bytes:
        raise ValueError("the pools' blocks differ in size")
    rc = lib.oracle_swap_blocks(_ptr(dst_k), _ptr(dst_v), _ptr(src_k), _ptr(src_v), _ptr(pairs), pairs.shape[0],
                                src_k.shape[0], dst_k.shape[0], block_bytes)
    if rc != 0:
        raise OracleError(f"oracle_swap_blocks failed with status {rc}")


def f16_to_f64(bits: int) -> float:
    return _load().oracle_f16_to_f64(bits)


def bf16_to_f64(bits: int) -> float:
    return _load().oracle_bf16_to_f64(bits)


def e4m3_to_f64(code: int) -> float:
    return _load().oracle_e4m3_to_f64(code)


def f32_to_e4m3(x: float) -> int:
    return int(_load().oracle_f32_to_e4m3(x))
