"""pa_decode_static_workspace: decode without a caller-provided workspace (needs a B200).

Some callers cannot allocate device memory when they decode -- a serving engine that has
already given nearly all free HBM to its KV-cache pool, or a plugin with no allocator of its
own.  This entry point takes its scratch from a buffer built into the library.  Its results
must match pa_decode (which takes a caller workspace) within the parity tolerance, call
after call, since every call reuses the same buffer and finds the previous call's contents
in it.  Both entry points run the same kernels on the same inputs, and their arithmetic does
not depend on where the scratch lives, so the outputs must be bit-identical.  This file is
collected last so that a stop at its first failure leaves every other test already run; it
also passes on its own in a fresh process.
"""
import ctypes

import numpy as np
import pytest
import torch

from paged_kv_cache_327_b200 import binding as B
from paged_kv_cache_327_b200 import workload as W

pytestmark = pytest.mark.gpu

TOL = {"f16": 2e-3, "bf16": 1e-2}


@pytest.fixture(scope="module", autouse=True)
def _require_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    B.load_library()


def _with_caller_workspace(w, dw):
    out = torch.empty((w.num_seqs, w.num_q_heads, w.head_dim), dtype=torch.float32, device="cuda")
    ws = B.DecodeWorkspace.for_workload(dw)
    B.pa_decode(out, dw.q, dw.k_cache, dw.v_cache, dw.block_tables, dw.seq_lens, w.scale, ws.tensor)
    torch.cuda.synchronize()
    return out


@pytest.mark.parametrize("name,kw", [("8b", {"num_seqs": 96}), ("tiny", {})])
def test_static_workspace_matches_caller_workspace_twice(name, kw):
    w = W.make_config(name, **kw)
    need = B.pa_decode_workspace_size(w.num_seqs, w.num_q_heads, w.head_dim,
                                      w.max_blocks_per_seq * w.block_size)
    assert need <= B.PA_DECODE_STATIC_WORKSPACE_BYTES, "the test workload must fit the built-in buffer"
    dw = B.device_workload(w)
    if len(w.copy_pairs):
        B.pa_copy_blocks(dw.k_cache, dw.v_cache, dw.copy_pairs)
    B.pa_reshape_and_cache(dw.new_k, dw.new_v, dw.k_cache, dw.v_cache, dw.slot_mapping)
    ref = _with_caller_workspace(w, dw)
    assert torch.isfinite(ref).all()
    for call in range(2):  # the second call finds the first call's data in the shared buffer
        out = torch.full_like(ref, float("nan"))
        B.pa_decode_static_workspace(out, dw.q, dw.k_cache, dw.v_cache, dw.block_tables, dw.seq_lens, w.scale)
        torch.cuda.synchronize()
        assert B.pa_get_device_error() == B.PA_DEV_OK
        err = float((out - ref).abs().max())
        assert err <= TOL[w.kv_dtype], f"call {call}: max|err| vs pa_decode = {err}"
        assert torch.equal(out, ref), f"call {call}: not bit-identical to pa_decode (max|err| {err})"


def test_static_workspace_rejects_oversized_calls():
    lib = B.load_library()
    V = ctypes.c_void_p
    fake = 0x10000  # never dereferenced: the size check comes first
    # 4096 sequences of up to 32768 tokens with 64 query heads need far more than 64 MiB
    rc = lib.pa_decode_static_workspace(V(fake), V(fake), V(fake), V(fake), V(fake), V(fake), 4096, 64, 8, 128,
                                        16, ctypes.c_float(0.088), 2048, 100000, 2, 2, 2, 0, V(0))
    assert rc == B.PA_ERR_TOO_LARGE
    assert "64 MiB" in B.pa_strerror(rc)
