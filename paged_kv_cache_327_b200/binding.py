"""ctypes binding of libpa.so (include/pa.h), with the ABI's own names.

Argument marshalling only: torch tensors are turned into device pointers, sizes and
pa_dtype codes, and every computation happens in the library's CUDA kernels.  Loading
fails loudly (ImportError) when libpa.so has not been built; there is no fallback.
"""
from __future__ import annotations

import ctypes
import dataclasses
import os
from typing import Optional

import numpy as np
import torch

from . import workload as W

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libpa.so")

PA_F32, PA_F16, PA_BF16, PA_FP8_E4M3 = 0, 1, 2, 3
PA_OK, PA_ERR_INVALID, PA_ERR_UNSUPPORTED, PA_ERR_WORKSPACE, PA_ERR_CUDA = 0, -1, -2, -3, -4
(PA_DEV_OK, PA_DEV_BAD_BLOCK_ID, PA_DEV_BAD_SEQ_LEN, PA_DEV_BAD_SLOT, PA_DEV_BAD_PAIR, PA_DEV_TIMEOUT,
 PA_DEV_BAD_PREFIX) = range(7)

EXPORTED = ("pa_decode_workspace_size", "pa_decode", "pa_reshape_and_cache", "pa_copy_blocks",
            "pa_strerror", "pa_get_device_error", "pa_version", "pa_decode_static_workspace",
            "pa_decode_fp8", "pa_reshape_and_cache_fp8", "pa_swap_blocks", "pa_decode_multi", "pa_decode_prefix",
            "pa_selftest_wait_timeout", "pa_set_option")
PA_ERR_TOO_LARGE = -5
PA_DECODE_STATIC_WORKSPACE_BYTES = 64 << 20

_TORCH_CODE = {torch.float32: PA_F32, torch.float16: PA_F16, torch.bfloat16: PA_BF16}
_NAME_CODE = {"f32": PA_F32, "f16": PA_F16, "bf16": PA_BF16}
_NAME_TORCH = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}

_lib = None


def load_library(path: str = _LIB_PATH):
    """Load libpa.so once and declare the ABI's signatures."""
    global _lib
    if _lib is not None and path == _LIB_PATH:
        return _lib
    if not os.path.exists(path):
        raise ImportError(f"{path} is missing: build it with `python paged_kv_cache_327_b200/build.py` "
                          "(the CUDA path has no fallback)")
    lib = ctypes.CDLL(path)
    P, I, I64, SZ = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_size_t
    lib.pa_decode_workspace_size.argtypes = [I, I, I, I, I]
    lib.pa_decode_workspace_size.restype = SZ
    lib.pa_decode.argtypes = [P, P, P, P, P, P, I, I, I, I, I, ctypes.c_float, I, I64, I, I, I, I, P, SZ, P]
    lib.pa_decode.restype = I
    lib.pa_reshape_and_cache.argtypes = [P, P, P, P, P, I, I, I, I, I64, I, I64, I64, P]
    lib.pa_reshape_and_cache.restype = I
    lib.pa_copy_blocks.argtypes = [P, P, P, I, I64, SZ, P, P]
    lib.pa_copy_blocks.restype = I
    lib.pa_strerror.argtypes = [I]
    lib.pa_strerror.restype = ctypes.c_char_p
    lib.pa_get_device_error.argtypes = [P]
    lib.pa_get_device_error.restype = I
    lib.pa_version.argtypes = []
    lib.pa_version.restype = I
    lib.pa_decode_static_workspace.argtypes = [P, P, P, P, P, P, I, I, I, I, I, ctypes.c_float, I, I64, I, I, I, I, P]
    lib.pa_decode_static_workspace.restype = I
    F = ctypes.c_float
    lib.pa_decode_fp8.argtypes = [P, P, P, P, P, P, I, I, I, I, I, F, F, F, I, I64, I, I, I, P, SZ, P]
    lib.pa_decode_fp8.restype = I
    lib.pa_reshape_and_cache_fp8.argtypes = [P, P, P, P, P, I, I, I, I, I64, I, F, F, I64, I64, P]
    lib.pa_reshape_and_cache_fp8.restype = I
    lib.pa_swap_blocks.argtypes = [P, P, P, P, P, I, I64, I64, SZ, P]
    lib.pa_swap_blocks.restype = I
    lib.pa_decode_multi.argtypes = [P, P, P, P, P, P, I, I, I, I, I, I, F, I, I64, I, I, I, I, P, SZ, P]
    lib.pa_decode_multi.restype = I
    lib.pa_decode_prefix.argtypes = [P, P, P, P, P, P, I, I, I, I, I, F, I, I64, I, I, I, I, P, I, I, P, SZ, P]
    lib.pa_decode_prefix.restype = I
    lib.pa_selftest_wait_timeout.argtypes = [I, P]
    lib.pa_selftest_wait_timeout.restype = I
    lib.pa_set_option.argtypes = [I, I]
    lib.pa_set_option.restype = I
    if path == _LIB_PATH:
        _lib = lib
    return lib


class PAError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {pa_strerror(status)} (status {status})")


def pa_strerror(status: int) -> str:
    return load_library().pa_strerror(int(status)).decode()


def _ptr(t: Optional[torch.Tensor]):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else ctypes.c_void_p(0)


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _check(rc: int, what: str) -> None:
    if rc != PA_OK:
        raise PAError(rc, what)


def pa_decode_workspace_size(num_seqs: int, num_q_heads: int, head_dim: int, max_seq_len: int,
                             partition_size: int = 0) -> int:
    return int(load_library().pa_decode_workspace_size(num_seqs, num_q_heads, head_dim, max_seq_len,
                                                       partition_size))


def pa_decode(out: torch.Tensor, q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
              block_tables: torch.Tensor, seq_lens: torch.Tensor, scale: float, workspace: torch.Tensor,
              partition_size: int = 0, stream=None) -> None:
    """out[N,Hq,D] <- paged decode attention (see include/pa.h); shapes give the sizes."""
    N, Hq, D = q.shape
    NB, bs, Hkv, D2 = k_cache.shape
    if D2 != D or tuple(out.shape) != (N, Hq, D) or v_cache.shape != k_cache.shape:
        raise ValueError("shape mismatch between q, out and the caches")
    for t in (out, q, k_cache, v_cache, block_tables, seq_lens, workspace):
        if not t.is_contiguous():
            raise ValueError("tensors must be contiguous")
    if block_tables.dtype != torch.int32 or seq_lens.dtype != torch.int32:
        raise TypeError("block_tables and seq_lens must be int32")
    rc = load_library().pa_decode(
        _ptr(out), _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_tables), _ptr(seq_lens), N, Hq, Hkv, D, bs,
        ctypes.c_float(scale), block_tables.shape[1], NB, _TORCH_CODE[q.dtype], _TORCH_CODE[k_cache.dtype],
        _TORCH_CODE[out.dtype], partition_size, _ptr(workspace), workspace.numel() * workspace.element_size(),
        _stream(stream))
    _check(rc, "pa_decode")


def pa_decode_multi(out: torch.Tensor, q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
                    block_tables: torch.Tensor, seq_lens: torch.Tensor, scale: float, workspace: torch.Tensor,
                    partition_size: int = 0, stream=None) -> None:
    """out[N,T,Hq,D] <- causal attention of each sequence's last T tokens over the paged cache.

    Query token t of sequence i sits at position seq_lens[i] - T + t and attends to positions
    0 .. seq_lens[i] - T + t (see include/pa.h).  The workspace is that of pa_decode for
    T * Hq query heads (DecodeWorkspace.for_multi).
    """
    N, T, Hq, D = q.shape
    NB, bs, Hkv, D2 = k_cache.shape
    if D2 != D or tuple(out.shape) != (N, T, Hq, D) or v_cache.shape != k_cache.shape:
        raise ValueError("shape mismatch between q, out and the caches")
    for t in (out, q, k_cache, v_cache, block_tables, seq_lens, workspace):
        if not t.is_contiguous():
            raise ValueError("tensors must be contiguous")
    if block_tables.dtype != torch.int32 or seq_lens.dtype != torch.int32:
        raise TypeError("block_tables and seq_lens must be int32")
    rc = load_library().pa_decode_multi(
        _ptr(out), _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_tables), _ptr(seq_lens), N, T, Hq, Hkv, D, bs,
        ctypes.c_float(scale), block_tables.shape[1], NB, _TORCH_CODE[q.dtype], _TORCH_CODE[k_cache.dtype],
        _TORCH_CODE[out.dtype], partition_size, _ptr(workspace), workspace.numel() * workspace.element_size(),
        _stream(stream))
    _check(rc, "pa_decode_multi")


def pa_decode_prefix(out: torch.Tensor, q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
                     block_tables: torch.Tensor, seq_lens: torch.Tensor, scale: float, workspace: torch.Tensor,
                     prefix_groups: torch.Tensor, max_members: int, partition_size: int = 0, stream=None) -> None:
    """pa_decode where each prefix group's shared blocks are read once for all its members.

    prefix_groups: device int32 [num_groups, 3] rows (first, members, shared tokens), e.g. from
    block_manager.find_prefix_groups; max_members * (Hq / Hkv) <= 32 (see include/pa.h).
    """
    N, Hq, D = q.shape
    NB, bs, Hkv, D2 = k_cache.shape
    if D2 != D or tuple(out.shape) != (N, Hq, D) or v_cache.shape != k_cache.shape:
        raise ValueError("shape mismatch between q, out and the caches")
    for t in (out, q, k_cache, v_cache, block_tables, seq_lens, workspace, prefix_groups):
        if not t.is_contiguous():
            raise ValueError("tensors must be contiguous")
    if block_tables.dtype != torch.int32 or seq_lens.dtype != torch.int32 or prefix_groups.dtype != torch.int32:
        raise TypeError("block_tables, seq_lens and prefix_groups must be int32")
    if prefix_groups.numel() and (prefix_groups.dim() != 2 or prefix_groups.shape[1] != 3):
        raise ValueError("prefix_groups must be [num_groups, 3]")
    rc = load_library().pa_decode_prefix(
        _ptr(out), _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_tables), _ptr(seq_lens), N, Hq, Hkv, D, bs,
        ctypes.c_float(scale), block_tables.shape[1], NB, _TORCH_CODE[q.dtype], _TORCH_CODE[k_cache.dtype],
        _TORCH_CODE[out.dtype], partition_size, _ptr(prefix_groups), prefix_groups.shape[0] if prefix_groups.numel()
        else 0, max_members, _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream))
    _check(rc, "pa_decode_prefix")


def max_prefix_members(num_q_heads: int, num_kv_heads: int) -> int:
    """Largest max_members pa_decode_prefix takes: 32 query rows per KV head in one shared pass."""
    return max(1, 32 // (num_q_heads // num_kv_heads))


def pa_decode_static_workspace(out: torch.Tensor, q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
                               block_tables: torch.Tensor, seq_lens: torch.Tensor, scale: float,
                               partition_size: int = 0, stream=None) -> None:
    """pa_decode with the library's built-in scratch buffer instead of a caller workspace.

    For callers that cannot allocate device memory when they decode (for example when the
    KV-cache pool already holds nearly all free HBM).  Raises PAError (PA_ERR_TOO_LARGE) when
    the call needs more than PA_DECODE_STATIC_WORKSPACE_BYTES of scratch.  Calls that could
    run concurrently on the GPU share that buffer and must be serialised (one stream).
    """
    N, Hq, D = q.shape
    NB, bs, Hkv, D2 = k_cache.shape
    if D2 != D or tuple(out.shape) != (N, Hq, D) or v_cache.shape != k_cache.shape:
        raise ValueError("shape mismatch between q, out and the caches")
    for t in (out, q, k_cache, v_cache, block_tables, seq_lens):
        if not t.is_contiguous():
            raise ValueError("tensors must be contiguous")
    if block_tables.dtype != torch.int32 or seq_lens.dtype != torch.int32:
        raise TypeError("block_tables and seq_lens must be int32")
    rc = load_library().pa_decode_static_workspace(
        _ptr(out), _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_tables), _ptr(seq_lens), N, Hq, Hkv, D, bs,
        ctypes.c_float(scale), block_tables.shape[1], NB, _TORCH_CODE[q.dtype], _TORCH_CODE[k_cache.dtype],
        _TORCH_CODE[out.dtype], partition_size, _stream(stream))
    _check(rc, "pa_decode_static_workspace")


def pa_decode_fp8(out: torch.Tensor, q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
                  block_tables: torch.Tensor, seq_lens: torch.Tensor, scale: float, k_scale: float, v_scale: float,
                  workspace: torch.Tensor, partition_size: int = 0, stream=None) -> None:
    """pa_decode over an FP8 E4M3 cache (uint8 tensors of codes; value = code * scale)."""
    N, Hq, D = q.shape
    NB, bs, Hkv, D2 = k_cache.shape
    if D2 != D or tuple(out.shape) != (N, Hq, D) or v_cache.shape != k_cache.shape:
        raise ValueError("shape mismatch between q, out and the caches")
    if k_cache.dtype != torch.uint8 or v_cache.dtype != torch.uint8:
        raise TypeError("FP8 caches are uint8 tensors of E4M3 codes")
    rc = load_library().pa_decode_fp8(
        _ptr(out), _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_tables), _ptr(seq_lens), N, Hq, Hkv, D, bs,
        ctypes.c_float(scale), ctypes.c_float(k_scale), ctypes.c_float(v_scale), block_tables.shape[1], NB,
        _TORCH_CODE[q.dtype], _TORCH_CODE[out.dtype], partition_size, _ptr(workspace),
        workspace.numel() * workspace.element_size(), _stream(stream))
    _check(rc, "pa_decode_fp8")


def pa_reshape_and_cache_fp8(k: torch.Tensor, v: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
                             slot_mapping: torch.Tensor, k_scale: float, v_scale: float, stream=None) -> None:
    """Quantise token rows k/v[t] to E4M3 codes e4m3(x / scale) at their slots (skip if < 0)."""
    T, Hkv, D = k.shape
    NB, bs = k_cache.shape[:2]
    if slot_mapping.dtype != torch.int64:
        raise TypeError("slot_mapping must be int64")
    rc = load_library().pa_reshape_and_cache_fp8(
        _ptr(k), _ptr(v), _ptr(k_cache), _ptr(v_cache), _ptr(slot_mapping), T, Hkv, D, bs, NB,
        _TORCH_CODE[k.dtype], ctypes.c_float(k_scale), ctypes.c_float(v_scale), k.stride(0), v.stride(0),
        _stream(stream))
    _check(rc, "pa_reshape_and_cache_fp8")


def pa_reshape_and_cache(k: torch.Tensor, v: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
                         slot_mapping: torch.Tensor, stream=None) -> None:
    """k_cache/v_cache[slot // bs, slot % bs] <- k/v[t] for each token t with slot >= 0."""
    T, Hkv, D = k.shape
    NB, bs = k_cache.shape[:2]
    if slot_mapping.dtype != torch.int64:
        raise TypeError("slot_mapping must be int64")
    rc = load_library().pa_reshape_and_cache(
        _ptr(k), _ptr(v), _ptr(k_cache), _ptr(v_cache), _ptr(slot_mapping), T, Hkv, D, bs, NB,
        _TORCH_CODE[k_cache.dtype], k.stride(0), v.stride(0), _stream(stream))
    _check(rc, "pa_reshape_and_cache")


def pa_copy_blocks(k_cache: torch.Tensor, v_cache: torch.Tensor, src_dst_pairs: torch.Tensor,
                   host_pairs: Optional[np.ndarray] = None, stream=None) -> None:
    """Copy physical block pairs[p,0] over pairs[p,1] in both caches (copy-on-write)."""
    P = src_dst_pairs.shape[0]
    NB = k_cache.shape[0]
    block_bytes = k_cache[0].numel() * k_cache.element_size()
    hp = None
    if host_pairs is not None:
        hp = np.ascontiguousarray(host_pairs, dtype=np.int32)
    rc = load_library().pa_copy_blocks(
        _ptr(k_cache), _ptr(v_cache), _ptr(src_dst_pairs), P, NB, block_bytes,
        ctypes.c_void_p(hp.ctypes.data) if hp is not None else ctypes.c_void_p(0), _stream(stream))
    _check(rc, "pa_copy_blocks")


def pa_swap_blocks(dst_k: torch.Tensor, dst_v: torch.Tensor, src_k: torch.Tensor, src_v: torch.Tensor,
                   src_dst_pairs: torch.Tensor, stream=None) -> None:
    """Copy block pairs[p,0] of the source pool to block pairs[p,1] of the destination pool.

    Either pool may be a pinned host tensor (``pin_memory()``), which the device addresses
    directly; ``src_dst_pairs`` (int32 [P, 2]) must be on the device or in pinned memory.
    """
    block_bytes = src_k[0].numel() * src_k.element_size()
    if dst_k[0].numel() * dst_k.element_size() != block_bytes:
        raise ValueError("the pools' blocks differ in size")
    rc = load_library().pa_swap_blocks(_ptr(dst_k), _ptr(dst_v), _ptr(src_k), _ptr(src_v), _ptr(src_dst_pairs),
                                       src_dst_pairs.shape[0], src_k.shape[0], dst_k.shape[0], block_bytes,
                                       _stream(stream))
    _check(rc, "pa_swap_blocks")


def pa_selftest_wait_timeout(polls: int, stream=None) -> None:
    """Run the library's bounded wait on a barrier nothing completes (see include/pa.h)."""
    _check(load_library().pa_selftest_wait_timeout(int(polls), _stream(stream)), "pa_selftest_wait_timeout")


PA_OPT_WIDE_KERNEL = 1
WIDE_KERNELS = {"mma": 0, "tcgen05": 1, "auto": 2}
PA_OPT_ITEM_SPLIT = 2
ITEM_SPLITS = {"adaptive": 0, "fixed": 1}


def pa_set_option(option: int, value: int) -> None:
    """Process-wide library option (see include/pa.h)."""
    _check(load_library().pa_set_option(int(option), int(value)), "pa_set_option")


def set_wide_kernel(name: str) -> None:
    """Kernel for items of more than 8 query rows per KV head: "auto" (default: tcgen05 for items of
    more than 32 rows, the warp-MMA kernel below that), "mma" or "tcgen05"."""
    if name not in WIDE_KERNELS:
        raise ValueError(f"wide kernel must be one of {sorted(WIDE_KERNELS)}, not {name!r}")
    pa_set_option(PA_OPT_WIDE_KERNEL, WIDE_KERNELS[name])


def set_item_split(name: str) -> None:
    """How decode calls cut sequences into work items: "adaptive" (default: pieces of one to four
    partitions, sized to the batch) or "fixed" (one partition each: batch-invariant bits)."""
    if name not in ITEM_SPLITS:
        raise ValueError(f"item split must be one of {sorted(ITEM_SPLITS)}, not {name!r}")
    pa_set_option(PA_OPT_ITEM_SPLIT, ITEM_SPLITS[name])


def pa_get_device_error(stream=None) -> int:
    return int(load_library().pa_get_device_error(_stream(stream)))


# ---------------------------------------------------------------------------------------
# convenience: a workload on the device and one decode step through the ABI
# ---------------------------------------------------------------------------------------
def to_torch(a: np.ndarray, dtype: str, device) -> torch.Tensor:
    """Storage array (float32, uint16 bit patterns, or uint8 E4M3 codes) -> torch tensor."""
    if dtype == "f32":
        t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32))
    elif dtype == "e4m3":
        t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.uint8))
    else:
        t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.uint16).view(np.int16)).view(_NAME_TORCH[dtype])
    return t.to(device)


def from_torch(t: torch.Tensor) -> np.ndarray:
    """torch tensor -> storage array (float32, or uint16 bit patterns for 16-bit types)."""
    t = t.detach().cpu().contiguous()
    if t.dtype in (torch.float32, torch.uint8):
        return t.numpy()
    return t.view(torch.int16).numpy().view(np.uint16)


@dataclasses.dataclass
class DeviceWorkload:
    w: W.Workload
    q: torch.Tensor
    k_cache: torch.Tensor
    v_cache: torch.Tensor
    block_tables: torch.Tensor
    seq_lens: torch.Tensor
    new_k: torch.Tensor
    new_v: torch.Tensor
    slot_mapping: torch.Tensor
    copy_pairs: torch.Tensor


def device_workload(w: W.Workload, device="cuda") -> DeviceWorkload:
    return DeviceWorkload(
        w=w, q=to_torch(w.q, w.q_dtype, device), k_cache=to_torch(w.k_cache, w.kv_dtype, device),
        v_cache=to_torch(w.v_cache, w.kv_dtype, device),
        block_tables=torch.from_numpy(w.block_tables).to(device),
        seq_lens=torch.from_numpy(w.seq_lens).to(device), new_k=to_torch(w.new_k, w.new_kv_dtype, device),
        new_v=to_torch(w.new_v, w.new_kv_dtype, device), slot_mapping=torch.from_numpy(w.slot_mapping).to(device),
        copy_pairs=torch.from_numpy(np.ascontiguousarray(w.copy_pairs, dtype=np.int32).reshape(-1, 2)).to(device))


class DecodeWorkspace:
    """Caller-owned decode workspace sized by pa_decode_workspace_size()."""

    def __init__(self, num_seqs, num_q_heads, head_dim, max_seq_len, partition_size=0, device="cuda"):
        n = pa_decode_workspace_size(num_seqs, num_q_heads, head_dim, max_seq_len, partition_size)
        if n == 0:
            raise ValueError("invalid workspace request")
        self.tensor = torch.empty(n, dtype=torch.uint8, device=device)

    @classmethod
    def for_workload(cls, dw: DeviceWorkload, partition_size=0):
        w = dw.w
        return cls(w.num_seqs, w.num_q_tokens * w.num_q_heads, w.head_dim, w.max_blocks_per_seq * w.block_size,
                   partition_size, device=dw.q.device)

    @classmethod
    def for_multi(cls, num_seqs, num_q_tokens, num_q_heads, head_dim, max_seq_len, partition_size=0,
                  device="cuda"):
        """Workspace of pa_decode_multi: pa_decode's for num_q_tokens * num_q_heads heads."""
        return cls(num_seqs, num_q_tokens * num_q_heads, head_dim, max_seq_len, partition_size, device=device)


def run_step(dw: DeviceWorkload, out: torch.Tensor, ws: DecodeWorkspace, partition_size=0, stream=None) -> None:
    """One decode step: copy_blocks -> reshape_and_cache -> decode (all through the C ABI).

    A workload with several query tokens per sequence runs pa_decode_multi as its decode."""
    w = dw.w
    if dw.copy_pairs.shape[0]:
        pa_copy_blocks(dw.k_cache, dw.v_cache, dw.copy_pairs, stream=stream)
    if w.kv_dtype == "e4m3":
        if dw.slot_mapping.shape[0]:
            pa_reshape_and_cache_fp8(dw.new_k, dw.new_v, dw.k_cache, dw.v_cache, dw.slot_mapping, w.k_scale,
                                     w.v_scale, stream=stream)
        pa_decode_fp8(out, dw.q, dw.k_cache, dw.v_cache, dw.block_tables, dw.seq_lens, w.scale, w.k_scale,
                      w.v_scale, ws.tensor, partition_size=partition_size, stream=stream)
        return
    if dw.slot_mapping.shape[0]:
        pa_reshape_and_cache(dw.new_k, dw.new_v, dw.k_cache, dw.v_cache, dw.slot_mapping, stream=stream)
    if w.num_q_tokens > 1:
        pa_decode_multi(out, dw.q, dw.k_cache, dw.v_cache, dw.block_tables, dw.seq_lens, w.scale, ws.tensor,
                        partition_size=partition_size, stream=stream)
        return
    pa_decode(out, dw.q, dw.k_cache, dw.v_cache, dw.block_tables, dw.seq_lens, dw.w.scale, ws.tensor,
              partition_size=partition_size, stream=stream)
