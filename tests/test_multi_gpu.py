"""Multi-token causal paged attention on the GPU vs the fp64 oracle, through the C ABI.

Each sequence's step stores its last T tokens (reshape_and_cache); its T query tokens then
attend causally: query token t of a sequence of L tokens sees positions 0 .. L - T + t.
Tolerances are those of single-token decode (2e-3 with fp16 KV, 1e-2 with bf16 KV, plus
half an ulp of a 16-bit output): the kernel's arithmetic per (query row, key) is the same.
Cases cover items of 1 to 4 eight-row query tiles (T x G = 2 .. 32 query rows per KV head),
sequences with more query rows than an item holds (split into column groups of tokens),
both block sizes, partition tails that lie wholly after some query tokens' positions (those
rows see none of the tail partition's keys), empty sequences, sequences of exactly T tokens,
and an invalid length 0 < L < T.
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


def half_ulp(x, dtype):
    if dtype == "f32":
        return np.zeros_like(x)
    mant = {"f16": 10, "bf16": 7}[dtype]
    e = np.floor(np.log2(np.maximum(np.abs(x), 2.0 ** -14)))
    return 2.0 ** (e - mant - 1)


def gpu_multi(w, out_dtype="f32", P=0, dw=None):
    dw = dw or B.device_workload(w)
    out = torch.full((w.num_seqs, w.num_q_tokens, w.num_q_heads, w.head_dim), float("nan"),
                     dtype=B._NAME_TORCH[out_dtype], device="cuda")
    ws = B.DecodeWorkspace.for_workload(dw, P)
    B.run_step(dw, out, ws, partition_size=P)
    torch.cuda.synchronize()
    return dw, out


def oracle_multi(w, seqs=None):
    kc, vc = w.k_cache.copy(), w.v_cache.copy()
    oracle.copy_blocks(kc, vc, w.copy_pairs)
    oracle.reshape_and_cache(w.new_k, w.new_v, kc, vc, w.slot_mapping, w.kv_dtype)
    idx = np.arange(w.num_seqs) if seqs is None else np.asarray(seqs)
    ref = oracle.decode_multi(np.ascontiguousarray(w.q[idx]), w.q_dtype, kc, vc, w.kv_dtype,
                              np.ascontiguousarray(w.block_tables[idx]), np.ascontiguousarray(w.seq_lens[idx]),
                              w.scale)
    return idx, ref, kc, vc


def assert_close(got, ref, kv_dtype, out_dtype, what=""):
    err = np.abs(got.astype(np.float64) - ref.astype(np.float32).astype(np.float64))
    bad = ~(err <= TOL[kv_dtype] + half_ulp(ref, out_dtype))
    assert not bad.any(), (f"{what}: {bad.sum()} elements out of tolerance, max|err| = {np.nanmax(err):.3e} "
                           f"at {np.unravel_index(np.nanargmax(err), err.shape)}")


CASES = [
    # Hq, Hkv, T, D, bs, q_dtype, out_dtype, partition   (query rows per item = T * Hq / Hkv)
    (8, 4, 2, 128, 16, "bf16", "f32", 0),      # 4 rows: one tile
    (8, 8, 5, 128, 16, "f16", "f32", 0),       # MHA, 5 rows
    (4, 4, 8, 64, 32, "f16", "f16", 0),        # head_dim 64, 8 rows
    (32, 8, 3, 128, 16, "bf16", "bf16", 0),    # 12 rows: two tiles
    (32, 8, 5, 128, 16, "bf16", "f32", 0),     # 20 rows: three tiles
    (16, 2, 4, 128, 32, "f16", "f32", 256),    # 32 rows: four tiles, block size 32
    (64, 8, 4, 128, 16, "bf16", "bf16", 0),    # 32 rows (G = 8)
    (32, 8, 8, 128, 32, "bf16", "f32", 128),   # 32 rows, short partitions
    # more query rows than one item holds: the query tokens are split into column groups
    (32, 8, 16, 128, 16, "bf16", "f32", 0),    # 64 rows: 2 groups of 8 tokens
    (64, 8, 9, 128, 16, "bf16", "bf16", 0),    # G = 8: groups of 4, 4 and 1 tokens
    (8, 8, 40, 128, 32, "f16", "f32", 256),    # MHA: groups of 32 and 8 tokens
    (8, 2, 11, 64, 16, "bf16", "f32", 0),      # head_dim 64: groups of 2 tokens (8 rows)
]


def lens_for(T):
    # exactly T, ragged, one page, a partition tail of one token (512 + 1), a tail shorter
    # than T, long, empty
    return [T, T + 1, 15 + T, 100, 511, 512, 513, 512 + T - 1, 1030, 2047, 0, 3 * T]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "-".join(map(str, c)))
def test_multi_matches_oracle(case):
    Hq, Hkv, T, D, bs, qd, od, P = case
    kvd = qd
    lens = lens_for(T)
    w = W.independent("multi", lens, num_q_tokens=T, num_q_heads=Hq, num_kv_heads=Hkv, head_dim=D, block_size=bs,
                      q_dtype=qd, kv_dtype=kvd, seed=4100 + CASES.index(case))
    dw, out = gpu_multi(w, od, P)
    assert B.pa_get_device_error() == B.PA_DEV_OK
    _, ref, kc, vc = oracle_multi(w)
    assert np.array_equal(B.from_torch(dw.k_cache), kc), "the step's T tokens were not stored as the oracle's"
    got = out.float().cpu().numpy()
    assert_close(got, ref, kvd, od, f"case {case}")
    assert np.all(got[lens.index(0)] == 0.0), "an empty sequence gives zero rows"


def test_one_query_token_is_decode():
    """num_q_tokens = 1 through pa_decode_multi is pa_decode, bit for bit."""
    w = W.make_config("8b", num_seqs=32)
    dw = B.device_workload(w)
    B.pa_reshape_and_cache(dw.new_k, dw.new_v, dw.k_cache, dw.v_cache, dw.slot_mapping)
    ws = B.DecodeWorkspace.for_workload(dw)
    a = torch.empty((w.num_seqs, w.num_q_heads, w.head_dim), device="cuda")
    b = torch.empty((w.num_seqs, 1, w.num_q_heads, w.head_dim), device="cuda")
    B.pa_decode(a, dw.q, dw.k_cache, dw.v_cache, dw.block_tables, dw.seq_lens, w.scale, ws.tensor)
    B.pa_decode_multi(b, dw.q[:, None].contiguous(), dw.k_cache, dw.v_cache, dw.block_tables, dw.seq_lens, w.scale,
                      ws.tensor)
    torch.cuda.synchronize()
    assert torch.equal(a, b[:, 0])


@pytest.mark.parametrize("T", [5, 8, 16])
def test_multi_8b_full_size(T):
    """The 8B-shaped batch (256 sequences, lognormal lengths) with T query tokens, as the bench
    runs it (T = 16 takes two column groups per partition): the step's stored tokens bit-exact
    and every output row of every sequence against the oracle."""
    w = W.make_config("8b", num_q_tokens=T)
    dw, out = gpu_multi(w, "bf16")
    assert B.pa_get_device_error() == B.PA_DEV_OK
    _, ref, kc, vc = oracle_multi(w)
    assert np.array_equal(B.from_torch(dw.k_cache), kc) and np.array_equal(B.from_torch(dw.v_cache), vc)
    assert_close(out.float().cpu().numpy(), ref, w.kv_dtype, "bf16", f"8b T={T}")
    assert torch.isfinite(out.float()).all()


def test_multi_is_deterministic_and_batch_invariant():
    """Same bits on a second call, and (PA_SPLIT_FIXED) for a sequence decoded on its own."""
    B.set_item_split("fixed")
    try:
        check_deterministic_and_batch_invariant()
    finally:
        B.set_item_split("adaptive")


def check_deterministic_and_batch_invariant():
    w = W.make_config("8b", num_seqs=24, num_q_tokens=4)
    dw, a = gpu_multi(w)
    ws = B.DecodeWorkspace.for_workload(dw)
    b = torch.empty_like(a)
    B.pa_decode_multi(b, dw.q, dw.k_cache, dw.v_cache, dw.block_tables, dw.seq_lens, w.scale, ws.tensor)
    torch.cuda.synchronize()
    assert torch.equal(a, b)
    i = int(np.argmax(w.seq_lens))
    one = torch.empty((1,) + tuple(a.shape[1:]), device="cuda")
    ws1 = B.DecodeWorkspace.for_multi(1, 4, w.num_q_heads, w.head_dim, w.max_blocks_per_seq * w.block_size)
    B.pa_decode_multi(one, dw.q[i:i + 1].contiguous(), dw.k_cache, dw.v_cache, dw.block_tables[i:i + 1].contiguous(),
                      dw.seq_lens[i:i + 1].contiguous(), w.scale, ws1.tensor)
    torch.cuda.synchronize()
    assert torch.equal(one[0], a[i])


def test_sequence_shorter_than_its_queries_is_flagged():
    """0 < seq_lens[i] < T is invalid: its rows are NaN, the device error is set, and the
    other sequences are unaffected."""
    T = 4
    w = W.independent("short", [40, 600, 9], num_q_tokens=T, num_q_heads=8, num_kv_heads=2, head_dim=128,
                      block_size=16, q_dtype="bf16", kv_dtype="bf16", seed=4200)
    dw = B.device_workload(w)
    B.pa_reshape_and_cache(dw.new_k, dw.new_v, dw.k_cache, dw.v_cache, dw.slot_mapping)
    sl = dw.seq_lens.clone()
    sl[2] = T - 1
    out = torch.zeros((3, T, 8, 128), device="cuda")
    ws = B.DecodeWorkspace.for_workload(dw)
    B.pa_decode_multi(out, dw.q, dw.k_cache, dw.v_cache, dw.block_tables, sl, w.scale, ws.tensor)
    torch.cuda.synchronize()
    assert B.pa_get_device_error() == B.PA_DEV_BAD_SEQ_LEN
    assert torch.isnan(out[2]).all()
    _, ref, _, _ = oracle_multi(w, [0, 1])
    assert_close(out[:2].cpu().numpy(), ref, "bf16", "f32", "valid sequences beside an invalid one")


@pytest.mark.parametrize("case", [(2, 1, 16, "f16"), (6, 2, 9, "bf16"), (5, 1, 7, "f16")],
                         ids=lambda c: "-".join(map(str, c)))
def test_multi_head_dim_64_many_column_groups(case):
    """head_dim 64 with few KV heads: items of 5 to 8 query rows, so a sequence's T query tokens
    make several column groups per partition.  64 sequences of up to 2048 tokens give a work
    list far larger than the workspace's alignment padding: every group must have its own
    reserved work item (none may spill into the partial results)."""
    Hq, Hkv, T, dt = case
    rng = np.random.default_rng(4300 + Hq)
    lens = [int(x) for x in rng.integers(T, 2049, size=64)]
    lens[:3] = [0, T, 2048]
    w = W.independent("d64", lens, num_q_tokens=T, num_q_heads=Hq, num_kv_heads=Hkv, head_dim=64, block_size=16,
                      q_dtype=dt, kv_dtype=dt, seed=4300 + Hq)
    dw, out = gpu_multi(w, "f32")
    assert B.pa_get_device_error() == B.PA_DEV_OK
    _, ref, _, _ = oracle_multi(w)
    assert_close(out.float().cpu().numpy(), ref, dt, "f32", f"head_dim 64 case {case}")
