"""CUDA path vs the fp64 oracle, element by element, through the C ABI (needs a B200).

Tolerances (compared in fp32): attention max|err| <= 2e-3 with fp16 KV and <= 1e-2 with
bf16 KV; when the output itself is stored in 16 bits, half an ulp of that format at the
oracle's value is added.  reshape_and_cache and copy_blocks must be bit-exact.
"""
import numpy as np
import pytest
import torch

import oracle
from paged_kv_cache_327_b200 import binding as B
from paged_kv_cache_327_b200 import workload as W

pytestmark = pytest.mark.gpu

TOL = {"f16": 2e-3, "bf16": 1e-2}


@pytest.fixture(scope="module", autouse=True)
def _require_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    B.load_library()


def half_ulp(x: np.ndarray, dtype: str) -> np.ndarray:
    if dtype == "f32":
        return np.zeros_like(x)
    mant = {"f16": 10, "bf16": 7}[dtype]
    e = np.floor(np.log2(np.maximum(np.abs(x), 2.0 ** -14)))
    return 2.0 ** (e - mant - 1)


def oracle_post_step(w: W.Workload):
    kc, vc = w.k_cache.copy(), w.v_cache.copy()
    oracle.copy_blocks(kc, vc, w.copy_pairs)
    oracle.reshape_and_cache(w.new_k, w.new_v, kc, vc, w.slot_mapping, w.kv_dtype)
    return kc, vc


def oracle_decode(w: W.Workload, kc, vc, seqs=None):
    idx = np.arange(w.num_seqs) if seqs is None else np.asarray(seqs)
    return idx, oracle.decode(np.ascontiguousarray(w.q[idx]), w.q_dtype, kc, vc, w.kv_dtype,
                              np.ascontiguousarray(w.block_tables[idx]), np.ascontiguousarray(w.seq_lens[idx]),
                              w.scale)


def gpu_step(w: W.Workload, out_dtype="f32", partition_size=0, dw=None):
    dw = dw or B.device_workload(w)
    out = torch.full((w.num_seqs, w.num_q_heads, w.head_dim), float("nan"), dtype=B._NAME_TORCH[out_dtype],
                     device="cuda")
    ws = B.DecodeWorkspace.for_workload(dw, partition_size)
    B.run_step(dw, out, ws, partition_size=partition_size)
    torch.cuda.synchronize()
    assert B.pa_get_device_error() == B.PA_DEV_OK
    return dw, out


def out_f32(out: torch.Tensor) -> np.ndarray:
    return out.float().cpu().numpy()


def assert_close(got32: np.ndarray, ref64: np.ndarray, kv_dtype: str, out_dtype: str, what=""):
    ref32 = ref64.astype(np.float32).astype(np.float64)
    err = np.abs(got32.astype(np.float64) - ref32)
    bound = TOL[kv_dtype] + half_ulp(ref64, out_dtype)
    bad = ~(err <= bound)
    assert not bad.any(), (f"{what}: {bad.sum()} elements out of tolerance, max|err| = {np.nanmax(err):.3e} "
                           f"at {np.unravel_index(np.nanargmax(err), err.shape)}")
    return float(np.max(err))


def test_tiny_config_step():
    w = W.make_config("tiny")
    dw, out = gpu_step(w)
    kc, vc = oracle_post_step(w)
    assert np.array_equal(B.from_torch(dw.k_cache), kc), "K cache differs after copy_blocks + reshape_and_cache"
    assert np.array_equal(B.from_torch(dw.v_cache), vc), "V cache differs after copy_blocks + reshape_and_cache"
    _, ref = oracle_decode(w, kc, vc)
    assert_close(out_f32(out), ref, w.kv_dtype, "f32", "tiny")


CASES = [
    # Hq, Hkv, D, bs, q_dtype, kv_dtype, out_dtype, partition_size
    (2, 2, 64, 16, "f32", "f16", "f32", 0),
    (8, 2, 128, 16, "bf16", "bf16", "f32", 0),
    (8, 1, 128, 16, "bf16", "bf16", "bf16", 0),
    (32, 8, 128, 16, "bf16", "bf16", "f32", 0),
    (64, 8, 128, 16, "bf16", "bf16", "bf16", 0),
    (6, 2, 128, 32, "f16", "f16", "f32", 0),
    (4, 4, 64, 32, "f16", "f16", "f16", 0),
    (4, 2, 64, 16, "f32", "bf16", "f32", 256),
    (16, 2, 128, 32, "f32", "f16", "f32", 1024),
    (5, 5, 128, 16, "f16", "f16", "f32", 16),
    (14, 2, 64, 32, "bf16", "bf16", "f32", 64),
]
LENS = [1, 15, 16, 17, 100, 511, 512, 513, 1025, 2000, 0, 3]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "-".join(map(str, c)))
def test_decode_matches_oracle(case):
    Hq, Hkv, D, bs, qd, kd, od, P = case
    w = W.independent("case", LENS, num_q_heads=Hq, num_kv_heads=Hkv, head_dim=D, block_size=bs, q_dtype=qd,
                      kv_dtype=kd, seed=1000 + CASES.index(case))
    dw, out = gpu_step(w, od, P)
    kc, vc = oracle_post_step(w)
    assert np.array_equal(B.from_torch(dw.k_cache), kc)
    assert np.array_equal(B.from_torch(dw.v_cache), vc)
    _, ref = oracle_decode(w, kc, vc)
    assert_close(out_f32(out), ref, kd, od, str(case))
    assert np.all(out_f32(out)[LENS.index(0)] == 0.0), "a zero-length sequence gives zeros"


@pytest.mark.parametrize("name,bs,step", [("tiny", 16, None), ("7b", 16, None), ("13b", 16, None), ("13b", 32, None),
                                          ("8b", 16, None), ("70b", 16, "decode"), ("70b", 16, "fork")])
def test_named_config_full_size(name, bs, step):
    """Full-size step as the bench runs it (copy_blocks -> reshape_and_cache -> decode, the
    output in the query dtype): the caches compared in full, bit for bit, and every output row
    of every sequence against the oracle, element by element.  The 70B batch runs both as one
    decode step (one new token per sequence) and as the fork step (every sample's suffix and
    all 192 copy-on-write pairs in the step)."""
    w = W.make_config(name, block_size=bs, **({"step": step} if step else {}))
    out_dtype = w.q_dtype
    dw, out = gpu_step(w, out_dtype)
    kc, vc = oracle_post_step(w)
    assert np.array_equal(B.from_torch(dw.k_cache), kc)
    assert np.array_equal(B.from_torch(dw.v_cache), vc)
    _, ref = oracle_decode(w, kc, vc)
    assert ref.shape == tuple(out.shape)
    assert_close(out_f32(out), ref, w.kv_dtype, out_dtype, name)
    # every output finite (no stray read of a poisoned slot)
    assert torch.isfinite(out.float()).all()


def test_bf16_output_is_rounding_of_f32_output():
    w = W.make_config("8b", num_seqs=24)
    dw = B.device_workload(w)
    _, o32 = gpu_step(w, "f32", dw=dw)
    dw2 = B.device_workload(w)
    _, o16 = gpu_step(w, "bf16", dw=dw2)
    assert torch.equal(o32.to(torch.bfloat16), o16)


def test_deterministic_and_placement_invariant():
    w = W.independent("inv", [700, 1, 1500, 33, 512, 2049], num_q_heads=32, num_kv_heads=8, head_dim=128,
                      block_size=16, q_dtype="bf16", kv_dtype="bf16", seed=77)
    _, a = gpu_step(w)
    _, b = gpu_step(w)
    assert torch.equal(a, b), "two runs differ"
    # move every physical block elsewhere in a bigger pool
    kc, vc = oracle_post_step(w)
    perm = np.random.default_rng(3).permutation(w.num_blocks + 50)[:w.num_blocks]
    NB2 = w.num_blocks + 50
    kc2 = np.full((NB2,) + kc.shape[1:], W.NAN_BITS["bf16"], np.uint16)
    vc2 = kc2.copy()
    kc2[perm], vc2[perm] = kc, vc
    bt2 = np.where(w.block_tables >= 0, perm[np.maximum(w.block_tables, 0)], -1).astype(np.int32)
    out2 = torch.empty_like(a)
    ws = B.DecodeWorkspace(w.num_seqs, w.num_q_heads, w.head_dim, bt2.shape[1] * 16)
    B.pa_decode(out2, B.to_torch(w.q, "bf16", "cuda"), B.to_torch(kc2, "bf16", "cuda"),
                B.to_torch(vc2, "bf16", "cuda"), torch.from_numpy(bt2).cuda(),
                torch.from_numpy(w.seq_lens).cuda(), w.scale, ws.tensor)
    torch.cuda.synchronize()
    assert torch.equal(a, out2), "physical placement changed the result"


def test_batch_invariance():
    """A sequence gives the same bits alone and inside a batch."""
    w = W.make_config("8b", num_seqs=40)
    dw, full = gpu_step(w)
    kc = dw.k_cache
    vc = dw.v_cache
    for i in (0, 7, int(np.argmax(w.seq_lens))):
        out = torch.empty((1, w.num_q_heads, w.head_dim), dtype=torch.float32, device="cuda")
        ws = B.DecodeWorkspace(1, w.num_q_heads, w.head_dim, w.max_blocks_per_seq * w.block_size)
        B.pa_decode(out, dw.q[i:i + 1].contiguous(), kc, vc, dw.block_tables[i:i + 1].contiguous(),
                    dw.seq_lens[i:i + 1].contiguous(), w.scale, ws.tensor)
        torch.cuda.synchronize()
        assert torch.equal(out[0], full[i]), f"sequence {i} differs alone vs in the batch"


def test_block_size_16_and_32_agree():
    a = W.independent("a", [300, 1000, 45], num_q_heads=8, num_kv_heads=2, head_dim=128, block_size=16,
                      q_dtype="f16", kv_dtype="f16", seed=8)
    b = W.independent("b", [300, 1000, 45], num_q_heads=8, num_kv_heads=2, head_dim=128, block_size=32,
                      q_dtype="f16", kv_dtype="f16", seed=8)
    _, oa = gpu_step(a)
    _, ob = gpu_step(b)
    assert float((oa - ob).abs().max()) <= 2 * TOL["f16"]


def test_bad_block_id_poisons_only_its_sequence():
    w = W.independent("bad", [40, 700, 20], num_q_heads=4, num_kv_heads=2, head_dim=64, block_size=16,
                      q_dtype="bf16", kv_dtype="bf16", seed=4)
    dw = B.device_workload(w)
    dw.block_tables[1, 3] = w.num_blocks + 5
    out = torch.zeros((3, 4, 64), dtype=torch.float32, device="cuda")
    ws = B.DecodeWorkspace.for_workload(dw)
    B.run_step(dw, out, ws)
    assert B.pa_get_device_error() == B.PA_DEV_BAD_BLOCK_ID
    assert torch.isnan(out[1]).all()
    assert torch.isfinite(out[0]).all() and torch.isfinite(out[2]).all()
    assert B.pa_get_device_error() == B.PA_DEV_OK, "reading the error word clears it"


def test_bad_seq_len_and_slot_and_pair_are_reported():
    w = W.independent("bad", [40, 20], num_q_heads=2, num_kv_heads=2, head_dim=64, block_size=16,
                      q_dtype="f16", kv_dtype="f16", seed=6)
    dw = B.device_workload(w)
    B.pa_reshape_and_cache(dw.new_k, dw.new_v, dw.k_cache, dw.v_cache, dw.slot_mapping)
    dw.seq_lens[0] = w.max_blocks_per_seq * 16 + 1
    out = torch.zeros((2, 2, 64), dtype=torch.float32, device="cuda")
    ws = B.DecodeWorkspace.for_workload(dw)
    B.pa_decode(out, dw.q, dw.k_cache, dw.v_cache, dw.block_tables, dw.seq_lens, w.scale, ws.tensor)
    assert B.pa_get_device_error() == B.PA_DEV_BAD_SEQ_LEN
    assert torch.isnan(out[0]).all() and torch.isfinite(out[1]).all()
    before = B.from_torch(dw.k_cache)
    slots = torch.tensor([w.num_blocks * 16], dtype=torch.int64, device="cuda")
    B.pa_reshape_and_cache(dw.new_k[:1], dw.new_v[:1], dw.k_cache, dw.v_cache, slots)
    assert B.pa_get_device_error() == B.PA_DEV_BAD_SLOT
    pairs = torch.tensor([[0, w.num_blocks]], dtype=torch.int32, device="cuda")
    B.pa_copy_blocks(dw.k_cache, dw.v_cache, pairs)
    assert B.pa_get_device_error() == B.PA_DEV_BAD_PAIR
    assert np.array_equal(B.from_torch(dw.k_cache), before), "an out-of-range write touched the cache"


def test_negative_slots_are_skipped_and_strided_input_works():
    w = W.independent("s", [30, 50], num_q_heads=4, num_kv_heads=2, head_dim=128, block_size=16,
                      q_dtype="bf16", kv_dtype="bf16", seed=12)
    dw = B.device_workload(w)
    # a fused [T, 3 * Hkv * D] buffer: k and v are strided views into it
    T = w.new_k.shape[0]
    fused = torch.zeros((T, 3, 2, 128), dtype=torch.bfloat16, device="cuda")
    fused[:, 1] = dw.new_k
    fused[:, 2] = dw.new_v
    slots = dw.slot_mapping.clone()
    slots[0] = -1
    B.pa_reshape_and_cache(fused[:, 1], fused[:, 2], dw.k_cache, dw.v_cache, slots)
    torch.cuda.synchronize()
    kc, vc = w.k_cache.copy(), w.v_cache.copy()
    sm = w.slot_mapping.copy()
    sm[0] = -1
    oracle.reshape_and_cache(w.new_k, w.new_v, kc, vc, sm, "bf16")
    assert np.array_equal(B.from_torch(dw.k_cache), kc) and np.array_equal(B.from_torch(dw.v_cache), vc)


def test_copy_blocks_host_validation():
    w = W.make_config("tiny")
    dw = B.device_workload(w)
    with pytest.raises(B.PAError):
        bad = np.asarray([[1, 2], [3, 2]], np.int32)          # repeated destination
        B.pa_copy_blocks(dw.k_cache, dw.v_cache, torch.from_numpy(bad).cuda(), host_pairs=bad)
    with pytest.raises(B.PAError):
        bad = np.asarray([[1, 2], [2, 3]], np.int32)          # a destination that is also a source
        B.pa_copy_blocks(dw.k_cache, dw.v_cache, torch.from_numpy(bad).cuda(), host_pairs=bad)


def test_thousands_of_short_and_empty_sequences():
    """4096 sequences of 0 to 40 tokens (8B shapes): the plan spreads its work over the whole
    CTA, the merge kernel writes the rows of empty sequences, and every row matches the oracle."""
    rng = np.random.default_rng(4096)
    lens = [int(x) for x in rng.integers(0, 41, size=4096)]
    w = W.independent("short", lens, num_q_heads=32, num_kv_heads=8, head_dim=128, block_size=16, q_dtype="bf16",
                      kv_dtype="bf16", seed=4096)
    dw, out = gpu_step(w, "f32")
    kc, vc = oracle_post_step(w)
    _, ref = oracle_decode(w, kc, vc)
    assert_close(out_f32(out), ref, "bf16", "f32", "4096 short sequences")
    empty = np.asarray(lens) == 0
    assert empty.sum() > 50 and np.all(out_f32(out)[empty] == 0.0)


def test_invalid_lengths_in_a_large_batch_give_nan_rows():
    """Invalid lengths scattered over 3000 sequences: exactly those rows are NaN (written by the
    merge kernel), the error is reported, and every other row matches the oracle."""
    rng = np.random.default_rng(3000)
    lens = [int(x) for x in rng.integers(0, 70, size=3000)]
    w = W.independent("inv", lens, num_q_heads=8, num_kv_heads=2, head_dim=64, block_size=16, q_dtype="f16",
                      kv_dtype="f16", seed=3000)
    dw = B.device_workload(w)
    B.pa_reshape_and_cache(dw.new_k, dw.new_v, dw.k_cache, dw.v_cache, dw.slot_mapping)
    bad = rng.choice(3000, 40, replace=False)
    sl = dw.seq_lens.clone()
    sl[torch.from_numpy(bad).cuda()] = -1 - torch.arange(40, dtype=torch.int32, device="cuda")
    out = torch.zeros((3000, 8, 64), device="cuda")
    ws = B.DecodeWorkspace.for_workload(dw)
    B.pa_decode(out, dw.q, dw.k_cache, dw.v_cache, dw.block_tables, sl, w.scale, ws.tensor)
    assert B.pa_get_device_error() == B.PA_DEV_BAD_SEQ_LEN
    got = out_f32(out)
    mask = np.zeros(3000, bool)
    mask[bad] = True
    assert np.isnan(got[mask]).all() and not np.isnan(got[~mask]).any()
    kc, vc = oracle_post_step(w)
    good = np.flatnonzero(~mask)
    _, ref = oracle_decode(w, kc, vc, good)
    assert_close(got[good], ref, "f16", "f32", "valid rows beside invalid ones")
