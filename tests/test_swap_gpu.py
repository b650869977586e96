"""swap_blocks on the GPU: preemption to pinned host memory and back (needs a B200).

Bit-exact against the oracle in both directions; a swapped-out and swapped-back sequence
group, placed in different GPU blocks, decodes to the same bits as before.
"""
import numpy as np
import pytest
import torch

import oracle
from paged_kv_cache_327_b200 import binding as B
from paged_kv_cache_327_b200 import workload as W

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _require_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    B.load_library()


@pytest.mark.parametrize("kv_dtype", ["bf16", "e4m3"])
def test_swap_round_trip(kv_dtype):
    w = W.make_config("8b", num_seqs=24, kv_dtype=None if kv_dtype == "bf16" else "e4m3")
    dw = B.device_workload(w)
    out = torch.empty((w.num_seqs, w.num_q_heads, w.head_dim), dtype=torch.float32, device="cuda")
    ws = B.DecodeWorkspace.for_workload(dw)
    B.run_step(dw, out, ws)
    torch.cuda.synchronize()
    ref = out.clone()
    # preempt sequences 0..5: their blocks go to a pinned host pool
    bs = w.block_size
    seqs = range(6)
    gpu_blocks = [int(b) for i in seqs for b in w.block_tables[i, :-(-int(w.seq_lens[i]) // bs)]]
    host_shape = (len(gpu_blocks) + 3,) + tuple(dw.k_cache.shape[1:])
    hk = torch.zeros(host_shape, dtype=dw.k_cache.dtype).pin_memory()
    hv = torch.zeros(host_shape, dtype=dw.k_cache.dtype).pin_memory()
    cpu_ids = np.random.default_rng(1).permutation(host_shape[0])[:len(gpu_blocks)]
    out_pairs = np.stack([gpu_blocks, cpu_ids], 1).astype(np.int32)
    B.pa_swap_blocks(hk, hv, dw.k_cache, dw.v_cache, torch.from_numpy(out_pairs).cuda())
    torch.cuda.synchronize()
    assert B.pa_get_device_error() == B.PA_DEV_OK
    ek, ev = np.zeros_like(B.from_torch(hk)), np.zeros_like(B.from_torch(hv))
    oracle.swap_blocks(ek, ev, B.from_torch(dw.k_cache), B.from_torch(dw.v_cache), out_pairs)
    assert np.array_equal(B.from_torch(hk), ek) and np.array_equal(B.from_torch(hv), ev)
    # the GPU blocks are reused by someone else meanwhile
    dw.k_cache[torch.as_tensor(gpu_blocks, device="cuda")] = 0x7F if kv_dtype == "e4m3" else 0
    # resume into GPU blocks in a different placement: the group's own (clobbered) blocks,
    # shuffled so that no block returns to its old place (pairs from pinned host memory)
    new_ids = np.roll(np.asarray(gpu_blocks, np.int32), 1)
    assert not np.any(new_ids == np.asarray(gpu_blocks))
    in_pairs = torch.from_numpy(np.stack([cpu_ids, new_ids], 1).astype(np.int32)).pin_memory()
    B.pa_swap_blocks(dw.k_cache, dw.v_cache, hk, hv, in_pairs)
    torch.cuda.synchronize()
    assert B.pa_get_device_error() == B.PA_DEV_OK
    remap = dict(zip(gpu_blocks, new_ids.tolist()))
    bt = w.block_tables.copy()
    for i in seqs:
        n = -(-int(w.seq_lens[i]) // bs)
        bt[i, :n] = [remap[int(b)] for b in bt[i, :n]]
    dw.block_tables.copy_(torch.from_numpy(bt))
    out2 = torch.empty_like(ref)
    if kv_dtype == "e4m3":
        B.pa_decode_fp8(out2, dw.q, dw.k_cache, dw.v_cache, dw.block_tables, dw.seq_lens, w.scale, w.k_scale,
                        w.v_scale, ws.tensor)
    else:
        B.pa_decode(out2, dw.q, dw.k_cache, dw.v_cache, dw.block_tables, dw.seq_lens, w.scale, ws.tensor)
    torch.cuda.synchronize()
    assert torch.equal(out2, ref), "a swapped-out and swapped-back group must decode to the same bits"


def test_swap_rejects_bad_pairs_without_touching_memory():
    w = W.make_config("tiny")
    dw = B.device_workload(w)
    before = B.from_torch(dw.k_cache)
    hk = torch.zeros_like(dw.k_cache, device="cpu").pin_memory()
    hv = torch.zeros_like(hk).pin_memory()
    pairs = torch.tensor([[w.num_blocks, 0]], dtype=torch.int32, device="cuda")   # source id out of range
    B.pa_swap_blocks(hk, hv, dw.k_cache, dw.v_cache, pairs)
    assert B.pa_get_device_error() == B.PA_DEV_BAD_PAIR
    assert not hk.any() and np.array_equal(B.from_torch(dw.k_cache), before)
