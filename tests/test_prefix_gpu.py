"""Prefix-aware decode (pa_decode_prefix) on the GPU vs the fp64 oracle, through the C ABI.

Prefix-aware decode computes plain decode attention: each group's shared blocks are only read
once for all its members.  So the expectation is the oracle's decode, and the tolerances are
those of pa_decode (2e-3 with fp16 KV, 1e-2 with bf16 KV, plus half an ulp of a 16-bit
output).  Cases: groups of 2 to 9 members (split into shared passes of max_members), shared
lengths that end inside a partition, a member with no tokens of its own, items of 8 to 32
query rows, both block sizes, the 70B-shaped batch of the benchmark (64 groups x 4 samples plus
long standalone sequences), a malformed group (ignored, reported) and members whose tables
disagree (NaN, reported).
"""
import numpy as np
import pytest
import torch

import oracle
from paged_kv_cache_327_b200 import binding as B
from paged_kv_cache_327_b200 import block_manager as BM
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


def assert_close(got, ref, kv_dtype, out_dtype, what=""):
    err = np.abs(got.astype(np.float64) - ref.astype(np.float32).astype(np.float64))
    bad = ~(err <= TOL[kv_dtype] + half_ulp(ref, out_dtype))
    assert not bad.any(), (f"{what}: {bad.sum()} elements out of tolerance, max|err| = {np.nanmax(err):.3e} "
                           f"at {np.unravel_index(np.nanargmax(err), err.shape)}")


def stepped(w):
    """Device workload after the step (copy_blocks + reshape_and_cache) and the oracle's caches."""
    dw = B.device_workload(w)
    if len(w.copy_pairs):
        B.pa_copy_blocks(dw.k_cache, dw.v_cache, dw.copy_pairs)
    B.pa_reshape_and_cache(dw.new_k, dw.new_v, dw.k_cache, dw.v_cache, dw.slot_mapping)
    kc, vc = w.k_cache.copy(), w.v_cache.copy()
    oracle.copy_blocks(kc, vc, w.copy_pairs)
    oracle.reshape_and_cache(w.new_k, w.new_v, kc, vc, w.slot_mapping, w.kv_dtype)
    return dw, kc, vc


def prefix_decode(w, dw, groups, max_members, out_dtype="f32", P=0):
    out = torch.full((w.num_seqs, w.num_q_heads, w.head_dim), float("nan"), dtype=B._NAME_TORCH[out_dtype],
                     device="cuda")
    ws = B.DecodeWorkspace.for_workload(dw, P)
    g = torch.from_numpy(np.ascontiguousarray(groups, dtype=np.int32).reshape(-1, 3)).cuda()
    B.pa_decode_prefix(out, dw.q, dw.k_cache, dw.v_cache, dw.block_tables, dw.seq_lens, w.scale, ws.tensor, g,
                       max_members, partition_size=P)
    torch.cuda.synchronize()
    return out


def oracle_decode(w, kc, vc, seqs=None):
    idx = np.arange(w.num_seqs) if seqs is None else np.asarray(seqs)
    return idx, oracle.decode(np.ascontiguousarray(w.q[idx]), w.q_dtype, kc, vc, w.kv_dtype,
                              np.ascontiguousarray(w.block_tables[idx]), np.ascontiguousarray(w.seq_lens[idx]),
                              w.scale)


CASES = [
    # Hq, Hkv, bs, q_dtype, out_dtype, partition, max_members, groups as (prefix, [step tokens per member])
    (32, 8, 16, "bf16", "f32", 0, 8, [(700, [1, 5, 30]), (40, [3]), (1030, [1, 1, 1, 1, 1, 1, 1, 1, 1]),
                                      (64, [0, 2])]),
    (64, 8, 16, "bf16", "bf16", 0, 4, [(4100, [1, 200, 17, 512]), (513, [2, 2]), (9, [1, 1])]),
    (16, 8, 32, "f16", "f32", 256, 16, [(300, [1, 64, 5]), (2000, [7, 1]), (31, [1, 1, 1])]),
    (8, 8, 16, "f32", "f32", 0, 8, [(520, [1, 1, 1, 1, 1]), (100, [1]), (33, [1, 1])]),  # MHA, f32 query
    (24, 8, 32, "bf16", "f16", 128, 2, [(1500, [1, 9]), (77, [1, 1, 40])]),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "-".join(map(str, c[:7])))
def test_prefix_decode_matches_oracle(case):
    Hq, Hkv, bs, qd, od, P, mm, spec = case
    kvd = "f16" if qd == "f16" else ("bf16" if qd == "bf16" else "f16")
    groups = [W.Group(p, st) for p, st in spec]
    w = W.build_groups("prefix", groups, num_q_heads=Hq, num_kv_heads=Hkv, head_dim=128, block_size=bs, q_dtype=qd,
                       kv_dtype=kvd, seed=5100 + CASES.index(case))
    pg = BM.find_prefix_groups(w.block_tables, w.seq_lens, bs)
    assert len(pg) >= 2, "the case must exercise shared prefixes"
    dw, kc, vc = stepped(w)
    out = prefix_decode(w, dw, pg, mm, od, P)
    assert B.pa_get_device_error() == B.PA_DEV_OK
    _, ref = oracle_decode(w, kc, vc)
    assert_close(out.float().cpu().numpy(), ref, kvd, od, f"case {case[:7]}")


def test_prefix_70b_batch_matches_decode_and_oracle():
    """The 70B-shaped batch as the bench runs it: every row agrees with pa_decode and, element by
    element, with the oracle."""
    w = W.make_config("70b")
    pg = BM.find_prefix_groups(w.block_tables, w.seq_lens, w.block_size)
    dw, kc, vc = stepped(w)
    out = prefix_decode(w, dw, pg, B.max_prefix_members(w.num_q_heads, w.num_kv_heads))
    assert B.pa_get_device_error() == B.PA_DEV_OK
    plain = torch.empty_like(out)
    ws = B.DecodeWorkspace.for_workload(dw)
    B.pa_decode(plain, dw.q, dw.k_cache, dw.v_cache, dw.block_tables, dw.seq_lens, w.scale, ws.tensor)
    torch.cuda.synchronize()
    assert float((out - plain).abs().max()) <= TOL[w.kv_dtype]
    _, ref = oracle_decode(w, kc, vc)
    assert_close(out.float().cpu().numpy(), ref, w.kv_dtype, "f32", "70b")


def test_prefix_decode_is_deterministic():
    w = W.build_groups("det", [W.Group(1500, [1, 3, 9, 27]), W.Group(900, [2, 2])], num_q_heads=32, num_kv_heads=8,
                       head_dim=128, block_size=16, q_dtype="bf16", kv_dtype="bf16", seed=5200)
    pg = BM.find_prefix_groups(w.block_tables, w.seq_lens, 16)
    dw, _, _ = stepped(w)
    a = prefix_decode(w, dw, pg, 8)
    b = prefix_decode(w, dw, pg, 8)
    assert torch.equal(a, b)


def test_malformed_group_is_ignored_and_reported():
    w = W.build_groups("bad", [W.Group(600, [1, 4]), W.Group(300, [2, 2, 2])], num_q_heads=32, num_kv_heads=8,
                       head_dim=128, block_size=16, q_dtype="bf16", kv_dtype="bf16", seed=5300)
    pg = BM.find_prefix_groups(w.block_tables, w.seq_lens, 16)
    dw, kc, vc = stepped(w)
    _, ref = oracle_decode(w, kc, vc)
    for bad in ([[0, 2, 600]],                          # shared tokens not a multiple of the block size
                [[0, 2, 592], [1, 3, 288]],             # overlapping groups: both are ignored
                [[0, 5, 16], [1, 1, 16], [3, 2, 16]],   # one group overlapping two others
                [[0, 9, 16]]):                          # past the last sequence
        out = prefix_decode(w, dw, np.asarray(bad), 8)
        assert B.pa_get_device_error() == B.PA_DEV_BAD_PREFIX, bad
        assert_close(out.float().cpu().numpy(), ref, "bf16", "f32", f"groups {bad}")
    assert pg.tolist() == [[0, 2, 592], [2, 3, 288]]
    out = prefix_decode(w, dw, pg[::-1].copy(), 8)              # order does not matter
    assert B.pa_get_device_error() == B.PA_DEV_OK
    assert_close(out.float().cpu().numpy(), ref, "bf16", "f32", "groups in reverse order")


def test_members_with_different_tables_get_nan():
    """A group claiming shared blocks its members do not share: those members are NaN and the
    error is reported; sequences outside the group are unaffected."""
    w = W.build_groups("lie", [W.Group(200, [1]), W.Group(200, [1]), W.Group(300, [1, 1])], num_q_heads=32,
                       num_kv_heads=8, head_dim=128, block_size=16, q_dtype="bf16", kv_dtype="bf16", seed=5400)
    dw, kc, vc = stepped(w)
    out = prefix_decode(w, dw, np.asarray([[0, 2, 192]]), 8)    # sequences 0 and 1 are independent
    assert B.pa_get_device_error() == B.PA_DEV_BAD_PREFIX
    got = out.float().cpu().numpy()
    assert np.isnan(got[0]).all() and np.isnan(got[1]).all()
    _, ref = oracle_decode(w, kc, vc, [2, 3])
    assert_close(got[2:], ref, "bf16", "f32", "sequences outside the bad group")


def test_large_group_beside_many_small_groups():
    """One system prompt shared by 600 requests, beside 150 forks of 2 to 4 samples: the plan
    validates every group in parallel over its members; all groups are valid, so none may be
    dropped (no PA_DEV_BAD_PREFIX), and every row matches the oracle."""
    rng = np.random.default_rng(5500)
    groups = [W.Group(1500, [1] * 600)]
    groups += [W.Group(int(rng.integers(16, 600)), [int(x) for x in rng.integers(1, 30, size=int(rng.integers(2, 5)))])
               for _ in range(150)]
    w = W.build_groups("big", groups, num_q_heads=32, num_kv_heads=8, head_dim=128, block_size=16, q_dtype="bf16",
                       kv_dtype="bf16", seed=5500)
    pg = BM.find_prefix_groups(w.block_tables, w.seq_lens, 16)
    assert pg[0].tolist() == [0, 600, 1488] and len(pg) > 100
    dw, kc, vc = stepped(w)
    out = prefix_decode(w, dw, pg, 8)
    assert B.pa_get_device_error() == B.PA_DEV_OK
    _, ref = oracle_decode(w, kc, vc)
    assert_close(out.float().cpu().numpy(), ref, "bf16", "f32", "large group")


def test_long_shared_items_check_every_page():
    """Many groups (160 pairs sharing 1040 tokens, 8 KV heads) make the plan take shared items of
    several partitions: here the whole 1040-token prefix, 65 pages, whose block-table entries the
    producer reads in windows of 32.  A member whose table differs from its leader's only in the
    second window (page 40) poisons its group's item (NaN rows, PA_DEV_BAD_PREFIX); every other
    row matches the oracle."""
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    groups = [W.Group(1040, [1, 1]) for _ in range(160)]
    w = W.build_groups("long", groups, num_q_heads=32, num_kv_heads=8, head_dim=128, block_size=16, q_dtype="bf16",
                       kv_dtype="bf16", seed=5600)
    pg = BM.find_prefix_groups(w.block_tables, w.seq_lens, 16)
    assert len(pg) == 160 and (pg[:, 2] == 1040).all()
    # at 512 tokens the shared items would outnumber the partition kernel's page pipelines four to one
    assert 160 * 3 * 8 >= 4 * 4 * sms
    # member 1 of group 0 reads a different (valid) block at page 40 of the shared tokens
    s0, s1 = int(pg[0, 0]), int(pg[0, 0]) + 1
    other = int(w.block_tables[int(pg[1, 0]), 3])
    w.block_tables[s1, 40] = other
    dw, kc, vc = stepped(w)
    out = prefix_decode(w, dw, pg, 8)
    assert B.pa_get_device_error() == B.PA_DEV_BAD_PREFIX
    got = out.float().cpu().numpy()
    assert np.isnan(got[s0]).all() and np.isnan(got[s1]).all()
    rest = [i for i in range(w.num_seqs) if i not in (s0, s1)]
    _, ref = oracle_decode(w, kc, vc, rest)
    assert_close(got[rest], ref, "bf16", "f32", "groups with consistent tables")
    # the same batch without the inconsistency: every row matches
    w.block_tables[s1, 40] = w.block_tables[s0, 40]
    dw, kc, vc = stepped(w)
    out = prefix_decode(w, dw, pg, 8)
    assert B.pa_get_device_error() == B.PA_DEV_OK
    _, ref = oracle_decode(w, kc, vc)
    assert_close(out.float().cpu().numpy(), ref, "bf16", "f32", "long shared items")
