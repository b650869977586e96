"""The 5th-generation tensor-core kernel for wide work items (PA_WIDE_TCGEN05) vs the fp64 oracle.

Items of more than 8 query rows per KV head (several query tokens, or the members of a shared
prefix) on a 16-bit cache with head_dim 128 and block size 16 run on this kernel once
pa_set_option(PA_OPT_WIDE_KERNEL, PA_WIDE_TCGEN05) is called, and by default (PA_WIDE_AUTO) when a
call's rows per KV head exceed the warp-MMA kernel's 32.  An item holds up to 64 query rows
(the M of its products); wider sequences are split into column groups.  The cases mirror the
warp-MMA kernel's: 12..64 query rows, column groups, short partitions (two chunks of 4 pages) and
long ones (several chunks, a ragged last chunk and page), empty sequences, causal tails, shared
prefixes of up to 64 rows, a bad block id and members whose tables differ.
Tolerances are the attention ones (2e-3 with fp16 KV, 1e-2 with bf16 KV, plus half an ulp of a
16-bit output).
"""
import numpy as np
import pytest
import torch

from paged_kv_cache_327_b200 import binding as B
from paged_kv_cache_327_b200 import block_manager as BM
from paged_kv_cache_327_b200 import workload as W
from tests import test_multi_gpu as TM
from tests import test_prefix_gpu as TP

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _tcgen05_kernel():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    B.load_library()
    B.set_wide_kernel("tcgen05")
    yield
    B.set_wide_kernel("auto")


MULTI = [
    # Hq, Hkv, T, D, bs, q_dtype, out_dtype, partition   (query rows per item = T * Hq / Hkv)
    (32, 8, 3, 128, 16, "bf16", "bf16", 0),    # 12 rows
    (16, 4, 4, 128, 16, "f16", "f16", 0),      # 16 rows, fp16
    (32, 8, 5, 128, 16, "bf16", "f32", 0),     # 20 rows
    (64, 8, 4, 128, 16, "bf16", "bf16", 0),    # 32 rows (G = 8)
    (32, 8, 8, 128, 16, "bf16", "f32", 128),   # 32 rows, two chunks per partition
    (32, 8, 16, 128, 16, "bf16", "f32", 0),    # 64 rows: one item per partition
    (64, 8, 9, 128, 16, "bf16", "bf16", 0),    # G = 8, 72 rows: column groups of 8 and 1 tokens
    (8, 8, 40, 128, 16, "f16", "f32", 256),    # MHA, 40 rows, four chunks per partition
    (8, 8, 100, 128, 16, "bf16", "f32", 0),    # MHA, 100 rows: column groups of 64 and 36 tokens
    (32, 8, 20, 128, 16, "f16", "bf16", 64),   # 80 rows: groups of 16 and 4 tokens, one-chunk partitions
]


@pytest.mark.parametrize("case", MULTI, ids=lambda c: "-".join(map(str, c)))
def test_multi_matches_oracle(case):
    Hq, Hkv, T, D, bs, qd, od, P = case
    lens = TM.lens_for(T)
    w = W.independent("multi", lens, num_q_tokens=T, num_q_heads=Hq, num_kv_heads=Hkv, head_dim=D, block_size=bs,
                      q_dtype=qd, kv_dtype=qd, seed=4700 + MULTI.index(case))
    dw, out = TM.gpu_multi(w, od, P)
    assert B.pa_get_device_error() == B.PA_DEV_OK
    _, ref, _, _ = TM.oracle_multi(w)
    got = out.float().cpu().numpy()
    TM.assert_close(got, ref, qd, od, f"case {case}")
    assert np.all(got[lens.index(0)] == 0.0), "an empty sequence gives zero rows"


@pytest.mark.parametrize("T", [5, 16])
def test_multi_8b_full_size(T):
    """The 8B-shaped batch (256 sequences, lognormal lengths) with T query tokens: every row of
    every sequence against the oracle, every row finite, and every row within tolerance of the
    warp-MMA kernel."""
    w = W.make_config("8b", num_q_tokens=T)
    dw, out = TM.gpu_multi(w, "bf16")
    assert B.pa_get_device_error() == B.PA_DEV_OK
    _, ref, _, _ = TM.oracle_multi(w)
    TM.assert_close(out.float().cpu().numpy(), ref, w.kv_dtype, "bf16", f"8b T={T}")
    assert torch.isfinite(out.float()).all()
    # the same decode (the cache already holds the step's tokens) on both kernels
    ws = B.DecodeWorkspace.for_workload(dw)
    a = torch.empty_like(out, dtype=torch.float32)
    b = torch.empty_like(a)
    B.pa_decode_multi(a, dw.q, dw.k_cache, dw.v_cache, dw.block_tables, dw.seq_lens, w.scale, ws.tensor)
    B.set_wide_kernel("mma")
    try:
        B.pa_decode_multi(b, dw.q, dw.k_cache, dw.v_cache, dw.block_tables, dw.seq_lens, w.scale, ws.tensor)
    finally:
        B.set_wide_kernel("tcgen05")
    torch.cuda.synchronize()
    assert float((a - b).abs().max()) <= 2 * TM.TOL[w.kv_dtype]


def test_multi_is_deterministic():
    w = W.make_config("8b", num_seqs=24, num_q_tokens=4)
    dw, a = TM.gpu_multi(w)
    ws = B.DecodeWorkspace.for_workload(dw)
    b = torch.empty_like(a)
    B.pa_decode_multi(b, dw.q, dw.k_cache, dw.v_cache, dw.block_tables, dw.seq_lens, w.scale, ws.tensor)
    torch.cuda.synchronize()
    assert torch.equal(a, b)


def test_bad_block_id_poisons_only_its_sequence():
    T = 4
    w = W.independent("bad", [40, 700, 1300, 20], num_q_tokens=T, num_q_heads=32, num_kv_heads=8, head_dim=128,
                      block_size=16, q_dtype="bf16", kv_dtype="bf16", seed=4790)
    dw = B.device_workload(w)
    dw.block_tables[2, 40] = w.num_blocks + 5   # in the sequence's second partition
    out = torch.zeros((4, T, 32, 128), dtype=torch.float32, device="cuda")
    ws = B.DecodeWorkspace.for_workload(dw)
    B.run_step(dw, out, ws)
    assert B.pa_get_device_error() == B.PA_DEV_BAD_BLOCK_ID
    assert torch.isnan(out[2]).all()
    assert torch.isfinite(out[[0, 1, 3]]).all()


@pytest.mark.parametrize("case", [c for c in TP.CASES if c[2] == 16 and c[3] != "f32"],
                         ids=lambda c: "-".join(map(str, c[:7])))
def test_prefix_decode_matches_oracle(case):
    Hq, Hkv, bs, qd, od, P, mm, spec = case
    kvd = qd
    groups = [W.Group(p, st) for p, st in spec]
    w = W.build_groups("prefix", groups, num_q_heads=Hq, num_kv_heads=Hkv, head_dim=128, block_size=bs, q_dtype=qd,
                       kv_dtype=kvd, seed=5100 + TP.CASES.index(case))
    pg = BM.find_prefix_groups(w.block_tables, w.seq_lens, bs)
    dw, kc, vc = TP.stepped(w)
    out = TP.prefix_decode(w, dw, pg, mm, od, P)
    assert B.pa_get_device_error() == B.PA_DEV_OK
    _, ref = TP.oracle_decode(w, kc, vc)
    TP.assert_close(out.float().cpu().numpy(), ref, kvd, od, f"case {case[:7]}")


def test_prefix_70b_batch():
    TP.test_prefix_70b_batch_matches_decode_and_oracle()


def test_prefix_members_with_different_tables_get_nan():
    TP.test_members_with_different_tables_get_nan()


def test_prefix_64_rows():
    """A shared pass of 8 members x G = 8 = 64 query rows (the tensor-core kernel's widest item)."""
    groups = [W.Group(1100, [1, 3, 9, 27, 2, 5, 40, 1]), W.Group(600, [1] * 11), W.Group(70, [4])]
    w = W.build_groups("p64", groups, num_q_heads=64, num_kv_heads=8, head_dim=128, block_size=16, q_dtype="bf16",
                       kv_dtype="bf16", seed=5600)
    pg = BM.find_prefix_groups(w.block_tables, w.seq_lens, 16)
    dw, kc, vc = TP.stepped(w)
    out = TP.prefix_decode(w, dw, pg, 8)
    assert B.pa_get_device_error() == B.PA_DEV_OK
    _, ref = TP.oracle_decode(w, kc, vc)
    TP.assert_close(out.float().cpu().numpy(), ref, "bf16", "f32", "64-row shared passes")


@pytest.mark.parametrize("T,kernel", [(16, "tcgen05"), (8, "mma")])
def test_default_option_picks_by_rows(T, kernel):
    """PA_WIDE_AUTO (the default) runs items of more than 32 query rows per KV head (8B shapes:
    4 grouped heads, so T = 16 gives 64 rows) on the tensor-core kernel and narrower ones on the
    warp-MMA kernel: its result is bit-identical to the kernel it picks (both are deterministic)."""
    w = W.make_config("8b", num_seqs=48, num_q_tokens=T)
    dw, _ = TM.gpu_multi(w)  # the step's tokens are stored
    ws = B.DecodeWorkspace.for_workload(dw)
    outs = {}
    try:
        for mode in ("auto", kernel):
            B.set_wide_kernel(mode)
            o = torch.empty(tuple(dw.q.shape), dtype=torch.float32, device="cuda")
            B.pa_decode_multi(o, dw.q, dw.k_cache, dw.v_cache, dw.block_tables, dw.seq_lens, w.scale, ws.tensor)
            outs[mode] = o
    finally:
        B.set_wide_kernel("tcgen05")
    torch.cuda.synchronize()
    assert B.pa_get_device_error() == B.PA_DEV_OK
    assert torch.equal(outs["auto"], outs[kernel])
