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

DTYPES = {"f32": 0, "f16": 1, "bf16": 2}
ELEM_BYTES = {"f32": 4, "f16": 2, "bf16": 2}

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
    want = np.float32 if dtype == "f32" else np.uint16
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
           num_threads=None, lib=None):
    """fp64 paged decode attention.

    q: [N, Hq, D] (float32 for "f32", uint16 bit patterns for "f16"/"bf16");
    k_cache, v_cache: [NB, bs, Hkv, D] in kv_dtype storage; block_tables int32
    [N, MB]; seq_lens int32 [N].  Returns float64 [N, Hq, D].
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
    rc = lib.oracle_decode(_ptr(out), _ptr(q), DTYPES[q_dtype], _ptr(k_cache), _ptr(v_cache),
                           DTYPES[kv_dtype], _ptr(block_tables), _ptr(seq_lens), N, Hq, Hkv, D, bs,
                           MB, NB, ctypes.c_float(scale),
                           num_threads if num_threads else default_threads())
    if rc != 0:
        raise OracleError(f"oracle_decode failed with status {rc}")
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


def f16_to_f64(bits: int) -> float:
    return _load().oracle_f16_to_f64(bits)


def bf16_to_f64(bits: int) -> float:
    return _load().oracle_bf16_to_f64(bits)
