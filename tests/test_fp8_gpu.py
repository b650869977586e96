"""FP8 (E4M3) KV cache on the GPU vs the fp64 oracle, through the C ABI (needs a B200).

The quantising store must be bit-exact.  Decode is compared in fp32 with the fp16-KV
tolerance, 2e-3 (plus half an ulp of a 16-bit output): every E4M3 code is exact in f16, so
the kernel's only roundings are the f16 softmax weights of the PV product and fp32
accumulation -- the same as on an fp16 cache.
"""
import numpy as np
import pytest
import torch

import oracle
from paged_kv_cache_327_b200 import binding as B
from paged_kv_cache_327_b200 import workload as W

pytestmark = pytest.mark.gpu

TOL = 2e-3


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


def oracle_post_step(w):
    kc, vc = w.k_cache.copy(), w.v_cache.copy()
    oracle.copy_blocks(kc, vc, w.copy_pairs)
    oracle.reshape_and_cache_e4m3(w.new_k, w.new_v, kc, vc, w.slot_mapping, w.new_kv_dtype, w.k_scale, w.v_scale)
    return kc, vc


def run(w, out_dtype="f32", P=0):
    dw = B.device_workload(w)
    out = torch.full((w.num_seqs, w.num_q_heads, w.head_dim), float("nan"), dtype=B._NAME_TORCH[out_dtype],
                     device="cuda")
    ws = B.DecodeWorkspace.for_workload(dw, P)
    B.run_step(dw, out, ws, partition_size=P)
    torch.cuda.synchronize()
    assert B.pa_get_device_error() == B.PA_DEV_OK
    return dw, out


def check(w, dw, out, out_dtype, seqs=None):
    kc, vc = oracle_post_step(w)
    assert np.array_equal(B.from_torch(dw.k_cache), kc), "FP8 K cache differs from the oracle's store"
    assert np.array_equal(B.from_torch(dw.v_cache), vc), "FP8 V cache differs from the oracle's store"
    idx = np.arange(w.num_seqs) if seqs is None else np.asarray(seqs)
    ref = oracle.decode(np.ascontiguousarray(w.q[idx]), w.q_dtype, kc, vc, "e4m3",
                        np.ascontiguousarray(w.block_tables[idx]), np.ascontiguousarray(w.seq_lens[idx]), w.scale,
                        k_scale=w.k_scale, v_scale=w.v_scale)
    got = out.float().cpu().numpy()[idx].astype(np.float64)
    err = np.abs(got - ref.astype(np.float32))
    bad = ~(err <= TOL + half_ulp(ref, out_dtype))
    assert not bad.any(), f"{bad.sum()} elements off, max|err| {np.nanmax(err):.3e}"


@pytest.mark.parametrize("in_dt", ["bf16", "f16", "f32"])
def test_fp8_store_is_bit_exact(in_dt):
    w = W.independent("s", [5, 40, 17, 1, 64], num_q_heads=8, num_kv_heads=4, head_dim=128, block_size=16,
                      q_dtype="bf16", kv_dtype="e4m3", new_dtype=in_dt, seed=31)
    dw = B.device_workload(w)
    # large rows exercise saturation at +-448, a skipped token the negative-slot rule
    dw.new_k[1] *= 40.0
    slots = dw.slot_mapping.clone()
    slots[2] = -1
    B.pa_reshape_and_cache_fp8(dw.new_k, dw.new_v, dw.k_cache, dw.v_cache, slots, w.k_scale, w.v_scale)
    torch.cuda.synchronize()
    kc, vc = w.k_cache.copy(), w.v_cache.copy()
    nk = B.from_torch(dw.new_k)
    sm = w.slot_mapping.copy()
    sm[2] = -1
    oracle.reshape_and_cache_e4m3(nk, w.new_v, kc, vc, sm, in_dt, w.k_scale, w.v_scale)
    assert np.array_equal(B.from_torch(dw.k_cache), kc)
    assert np.array_equal(B.from_torch(dw.v_cache), vc)
    assert ((B.from_torch(dw.k_cache) & 0x7f) == 0x7e).any(), "saturated codes expected"


CASES = [
    # Hq, Hkv, bs, q_dtype, out_dtype, partition
    (32, 8, 16, "bf16", "f32", 0),
    (64, 8, 16, "bf16", "bf16", 0),
    (8, 8, 16, "f16", "f32", 0),
    (8, 2, 32, "f32", "f32", 0),
    (12, 4, 32, "bf16", "f16", 256),
    (6, 6, 16, "f32", "bf16", 128),
]
LENS = [1, 15, 16, 17, 100, 511, 512, 513, 1025, 2000, 0, 3]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "-".join(map(str, c)))
def test_fp8_decode_matches_oracle(case):
    Hq, Hkv, bs, qd, od, P = case
    new_dt = "bf16" if qd == "f32" else qd
    w = W.independent("fp8", LENS, num_q_heads=Hq, num_kv_heads=Hkv, head_dim=128, block_size=bs, q_dtype=qd,
                      kv_dtype="e4m3", new_dtype=new_dt, seed=2000 + CASES.index(case))
    dw, out = run(w, od, P)
    check(w, dw, out, od)
    assert np.all(out.float().cpu().numpy()[LENS.index(0)] == 0.0)


@pytest.mark.parametrize("name,bs", [("8b", 16), ("7b", 16), ("13b", 32)])
def test_fp8_full_size(name, bs):
    """A named config over an FP8 cache, as the bench runs it: the quantising store bit-exact over
    the whole cache and every output row of every sequence against the oracle."""
    w = W.make_config(name, block_size=bs, kv_dtype="e4m3")
    dw, out = run(w, "bf16")
    check(w, dw, out, "bf16")
    assert torch.isfinite(out.float()).all()


def test_fp8_is_deterministic_and_batch_invariant():
    """Same bits on a second call, and (PA_SPLIT_FIXED) for a sequence decoded on its own."""
    B.set_item_split("fixed")
    try:
        check_deterministic_and_batch_invariant()
    finally:
        B.set_item_split("adaptive")


def check_deterministic_and_batch_invariant():
    w = W.make_config("8b", kv_dtype="e4m3", num_seqs=24)
    dw, a = run(w)
    ws = B.DecodeWorkspace.for_workload(dw)
    b = torch.empty_like(a)
    B.pa_decode_fp8(b, dw.q, dw.k_cache, dw.v_cache, dw.block_tables, dw.seq_lens, w.scale, w.k_scale, w.v_scale,
                    ws.tensor)
    torch.cuda.synchronize()
    assert torch.equal(a, b)
    i = int(np.argmax(w.seq_lens))
    one = torch.empty((1, w.num_q_heads, w.head_dim), dtype=torch.float32, device="cuda")
    ws1 = B.DecodeWorkspace(1, w.num_q_heads, w.head_dim, w.max_blocks_per_seq * w.block_size)
    B.pa_decode_fp8(one, dw.q[i:i + 1].contiguous(), dw.k_cache, dw.v_cache, dw.block_tables[i:i + 1].contiguous(),
                    dw.seq_lens[i:i + 1].contiguous(), w.scale, w.k_scale, w.v_scale, ws1.tensor)
    torch.cuda.synchronize()
    assert torch.equal(one[0], a[i])


def test_fp8_argument_checks():
    w = W.independent("a", [20], num_q_heads=2, num_kv_heads=2, head_dim=128, block_size=16, q_dtype="bf16",
                      kv_dtype="e4m3", seed=3)
    dw = B.device_workload(w)
    out = torch.empty((1, 2, 128), device="cuda")
    ws = B.DecodeWorkspace.for_workload(dw)
    with pytest.raises(B.PAError):  # scales must be positive
        B.pa_decode_fp8(out, dw.q, dw.k_cache, dw.v_cache, dw.block_tables, dw.seq_lens, w.scale, 0.0, 1.0, ws.tensor)
    lib = B.load_library()
    import ctypes
    V = ctypes.c_void_p
    # pa_decode refuses an FP8 cache (it has no scales)
    rc = lib.pa_decode(V(out.data_ptr()), V(dw.q.data_ptr()), V(dw.k_cache.data_ptr()), V(dw.v_cache.data_ptr()),
                       V(dw.block_tables.data_ptr()), V(dw.seq_lens.data_ptr()), 1, 2, 2, 128, 16,
                       ctypes.c_float(0.1), w.max_blocks_per_seq, w.num_blocks, B.PA_BF16, B.PA_FP8_E4M3, 0, 0,
                       V(ws.tensor.data_ptr()), ws.tensor.numel(), V(0))
    assert rc == B.PA_ERR_UNSUPPORTED
