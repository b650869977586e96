"""Pins of the fp64 oracle to things other than itself (CPU only).

Each ``check_*`` function takes an oracle library handle so that
``test_oracle_mutants.py`` can run the same checks against deliberately broken
copies of the oracle and show that every planted mistake is caught.

What pins what:
  * fp16 / bf16 element decoding -- every one of the 65536 bit patterns against
    numpy's float16 and torch's bfloat16 conversions;
  * decode -- torch's scaled_dot_product_attention in fp64 on contiguous K/V that
    the test itself scatters into the paged pool (so the oracle's gather is checked
    against the inverse mapping), for MHA and GQA, head_dim 64/128, block size 16/32,
    ragged lengths; closed forms (one token, zero query, equal keys, a dominant key,
    three keys with weights 1 : e : e^2); the pages' block-table example (logical
    blocks 0, 1, 2 -> physical 5, 12, 3); invariants (placement permutation, shared
    prefix == private copy, copy-on-write leaves the parent unchanged, GQA == MHA
    with repeated KV, block size 16 == 32);
  * reshape_and_cache / copy_blocks -- numpy fancy-index assignment;
  * multi-token causal attention -- torch SDPA in fp64 with an explicit causal mask
    (query token t of a sequence of L tokens sees positions 0 .. L - T + t) on contiguous
    K/V scattered into the pool; a closed form (zero keys: each query token averages V
    over exactly the positions it sees); and the reduction of every query token to a
    single-token decode of the sequence cut after the token's own position.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from paged_kv_cache_327_b200 import workload as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# --------------------------------------------------------------------------------------
# helpers that build inputs without the oracle
# --------------------------------------------------------------------------------------
def _rng(*key):
    return np.random.default_rng(list(key))


def paged_from_logical(Ks, Vs, block_size, num_blocks, rng, kv_dtype):
    """Scatter per-sequence logical K/V ([L, Hkv, D] float32) into a shuffled paged pool.

    Returns (k_cache, v_cache, block_tables, seq_lens) in storage form; unused pool
    positions hold NaN.
    """
    Hkv, D = Ks[0].shape[1], Ks[0].shape[2]
    nan = W.NAN_BITS[kv_dtype]
    kc = np.full((num_blocks, block_size, Hkv, D), nan, np.uint16)
    vc = np.full_like(kc, nan)
    free = list(rng.permutation(num_blocks))
    MB = max(1, max(-(-len(K) // block_size) for K in Ks))
    bt = np.full((len(Ks), MB), -1, np.int32)
    for i, (K, V) in enumerate(zip(Ks, Vs)):
        L = len(K)
        for b in range(-(-L // block_size)):
            phys = free.pop(0)
            bt[i, b] = phys
            n = min(block_size, L - b * block_size)
            kc[phys, :n] = W.to_storage(K[b * block_size:b * block_size + n], kv_dtype)
            vc[phys, :n] = W.to_storage(V[b * block_size:b * block_size + n], kv_dtype)
    lens = np.asarray([len(K) for K in Ks], np.int32)
    return kc, vc, bt, lens


def sdpa_reference(q32, Ks, Vs, scale, G):
    """torch SDPA in fp64 on contiguous per-sequence K/V (values already rounded)."""
    outs = []
    for i, (K, V) in enumerate(zip(Ks, Vs)):
        qi = torch.from_numpy(q32[i].astype(np.float64))[None, :, None, :]       # [1,Hq,1,D]
        if len(K) == 0:
            outs.append(np.zeros(q32.shape[1:], np.float64))
            continue
        k = torch.from_numpy(K.astype(np.float64)).permute(1, 0, 2)[None]        # [1,Hkv,L,D]
        v = torch.from_numpy(V.astype(np.float64)).permute(1, 0, 2)[None]
        o = torch.nn.functional.scaled_dot_product_attention(qi, k, v, scale=scale, enable_gqa=G > 1)
        outs.append(o[0, :, 0, :].numpy())
    return np.stack(outs)


def random_case(seed, lens, Hq, Hkv, D, bs, q_dtype, kv_dtype, pool_slack=3):
    rng = _rng(seed)
    q32 = W.storage_to_f32(W.to_storage(rng.standard_normal((len(lens), Hq, D), dtype=np.float32), q_dtype), q_dtype)
    Ks, Vs = [], []
    for L in lens:
        Ks.append(W.storage_to_f32(W.to_storage(rng.standard_normal((L, Hkv, D), dtype=np.float32), kv_dtype), kv_dtype))
        Vs.append(W.storage_to_f32(W.to_storage(rng.standard_normal((L, Hkv, D), dtype=np.float32), kv_dtype), kv_dtype))
    nb = sum(-(-L // bs) for L in lens) + pool_slack
    kc, vc, bt, sl = paged_from_logical(Ks, Vs, bs, nb, rng, kv_dtype)
    q = W.to_storage(q32, q_dtype)
    return q, q32, Ks, Vs, kc, vc, bt, sl


# --------------------------------------------------------------------------------------
# checks (shared with the mutation tests)
# --------------------------------------------------------------------------------------
def check_f16_decode(lib):
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ref = bits.view(np.float16).astype(np.float64)
    got = np.array([lib.oracle_f16_to_f64(int(b)) for b in bits])
    both_nan = np.isnan(ref) & np.isnan(got)
    assert np.array_equal(got[~both_nan], ref[~both_nan]), "fp16 decoding differs from numpy"
    assert np.array_equal(np.isnan(got), np.isnan(ref))


def check_bf16_decode(lib):
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ref = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).double().numpy()
    got = np.array([lib.oracle_bf16_to_f64(int(b)) for b in bits])
    both_nan = np.isnan(ref) & np.isnan(got)
    assert np.array_equal(got[~both_nan], ref[~both_nan]), "bf16 decoding differs from torch"


SDPA_CASES = [
    # lens, Hq, Hkv, D, bs, q_dtype, kv_dtype
    ([1, 17, 40, 5], 2, 2, 64, 16, "f32", "f16"),
    ([33, 64, 7], 4, 1, 64, 16, "bf16", "bf16"),
    ([50, 3, 96], 8, 2, 128, 16, "bf16", "bf16"),
    ([31, 70], 6, 3, 128, 32, "f16", "f16"),
    ([129, 2], 8, 8, 128, 32, "f32", "bf16"),
]


def check_decode_vs_sdpa(lib, cases=SDPA_CASES):
    for n, (lens, Hq, Hkv, D, bs, qd, kd) in enumerate(cases):
        q, q32, Ks, Vs, kc, vc, bt, sl = random_case(100 + n, lens, Hq, Hkv, D, bs, qd, kd)
        scale = float(np.float32(1 / math.sqrt(D)))
        got = oracle.decode(q, qd, kc, vc, kd, bt, sl, scale, num_threads=2, lib=lib)
        ref = sdpa_reference(q32, Ks, Vs, scale, Hq // Hkv)
        err = np.max(np.abs(got - ref))
        assert err < 1e-12, f"case {n}: oracle vs SDPA max|err| = {err}"


def _single(lib, K, V, qvec, scale, kv_dtype="f16", q_dtype="f32", bs=16):
    """One sequence, one head: K, V float32 [L, D] (representable), qvec float32 [D]."""
    L, D = K.shape
    kc, vc, bt, sl = paged_from_logical([K[:, None, :]], [V[:, None, :]], bs, -(-L // bs) + 2,
                                        _rng(7), kv_dtype)
    q = W.to_storage(qvec[None, None, :], q_dtype)
    return oracle.decode(q, q_dtype, kc, vc, kv_dtype, bt, sl, scale, num_threads=1, lib=lib)[0, 0]


def check_closed_forms(lib):
    rng = _rng(11)
    D = 64
    rep = lambda x: W.storage_to_f32(W.to_storage(x, "f16"), "f16")
    # one token: the output is that token's V row, exactly
    K = rep(rng.standard_normal((1, D), dtype=np.float32))
    V = rep(rng.standard_normal((1, D), dtype=np.float32))
    out = _single(lib, K, V, rng.standard_normal(D, dtype=np.float32), 0.125)
    assert np.array_equal(out, V[0].astype(np.float64)), "L=1 must return V_0"
    # zero query: uniform weights -> mean of V
    K = rep(rng.standard_normal((37, D), dtype=np.float32))
    V = rep(rng.standard_normal((37, D), dtype=np.float32))
    out = _single(lib, K, V, np.zeros(D, np.float32), 0.125)
    assert np.max(np.abs(out - V.astype(np.float64).mean(0))) < 1e-14, "q=0 must give mean(V)"
    # identical keys: uniform weights again
    K = np.repeat(rep(rng.standard_normal((1, D), dtype=np.float32)), 29, axis=0)
    out = _single(lib, K, V[:29], rng.standard_normal(D, dtype=np.float32), 0.125)
    assert np.max(np.abs(out - V[:29].astype(np.float64).mean(0))) < 1e-14, "equal keys must give mean(V)"
    # a dominant key: weights concentrate on it
    K = rep(rng.standard_normal((20, D), dtype=np.float32))
    kk = K[13].astype(np.float64)
    qv = (200.0 * kk / np.linalg.norm(kk)).astype(np.float32)
    out = _single(lib, K, V[:20], qv, 1.0)
    assert np.max(np.abs(out - V[13])) < 1e-6, "a dominant key must select its V row"
    # three keys with scores 0, 1, 2 (scale 1/8, q = 8 e_0, K_j[0] = j): weights 1 : e : e^2
    K = np.zeros((3, D), np.float32)
    K[:, 0] = [0.0, 1.0, 2.0]
    V = np.zeros((3, D), np.float32)
    V[0, :], V[1, :], V[2, :] = 1.0, 2.0, -1.0
    V[:, 5] = [3.0, -4.0, 0.5]
    qv = np.zeros(D, np.float32)
    qv[0] = 8.0
    out = _single(lib, K, V, qv, 0.125)
    e = math.e
    z = 1 + e + e * e
    assert abs(out[0] - (1 + 2 * e - e * e) / z) < 1e-14
    assert abs(out[5] - (3 - 4 * e + 0.5 * e * e) / z) < 1e-14


def check_page_block_table_example(lib):
    with open(os.path.join(GOLDEN, "page1_block_table.json"), encoding="utf-8") as f:
        g = json.load(f)
    bs, phys = g["block_size"], g["logical_to_physical"]
    L = sum(g["tokens_per_logical_block"]) - 7          # ragged last block too
    D, H = 64, 2
    rng = _rng(12)
    rep = lambda x: W.storage_to_f32(W.to_storage(x, "f16"), "f16")
    K = rep(rng.standard_normal((L, H, D), dtype=np.float32))
    V = rep(rng.standard_normal((L, H, D), dtype=np.float32))
    q32 = rng.standard_normal((1, H, D), dtype=np.float32)
    NB = max(phys) + 2
    nan = W.NAN_BITS["f16"]
    kc = np.full((NB, bs, H, D), nan, np.uint16)
    vc = np.full_like(kc, nan)
    for b, p in enumerate(phys):
        n = min(bs, L - b * bs)
        kc[p, :n] = W.to_storage(K[b * bs:b * bs + n], "f16")
        vc[p, :n] = W.to_storage(V[b * bs:b * bs + n], "f16")
    bt = np.asarray([phys], np.int32)
    sl = np.asarray([L], np.int32)
    got = oracle.decode(q32, "f32", kc, vc, "f16", bt, sl, 0.125, lib=lib)
    ref = sdpa_reference(q32, [K], [V], 0.125, 1)
    assert np.max(np.abs(got - ref)) < 1e-12
    # the same sequence stored in physical blocks 0, 1, 2 gives the same bits
    kc2 = np.full_like(kc, nan)
    vc2 = np.full_like(kc, nan)
    for b, p in enumerate(phys):
        kc2[b], vc2[b] = kc[p], vc[p]
    got2 = oracle.decode(q32, "f32", kc2, vc2, "f16", np.asarray([[0, 1, 2]], np.int32), sl, 0.125, lib=lib)
    assert np.array_equal(got, got2)


def check_invariants(lib):
    lens = [40, 77, 16, 1]
    Hq, Hkv, D, bs = 8, 2, 64, 16
    q, q32, Ks, Vs, kc, vc, bt, sl = random_case(21, lens, Hq, Hkv, D, bs, "bf16", "bf16", pool_slack=9)
    base = oracle.decode(q, "bf16", kc, vc, "bf16", bt, sl, 0.125, lib=lib)
    # 1. any permutation of physical placement gives identical bits
    perm = _rng(22).permutation(kc.shape[0])
    kc_p = np.empty_like(kc)
    vc_p = np.empty_like(vc)
    kc_p[perm], vc_p[perm] = kc, vc
    bt_p = np.where(bt >= 0, perm[np.maximum(bt, 0)], -1).astype(np.int32)
    assert np.array_equal(base, oracle.decode(q, "bf16", kc_p, vc_p, "bf16", bt_p, sl, 0.125, lib=lib))
    # 2. GQA equals MHA with each KV head repeated G times (contiguous groups)
    G = Hq // Hkv
    kc_r = np.repeat(kc, G, axis=2)
    vc_r = np.repeat(vc, G, axis=2)
    assert np.array_equal(base, oracle.decode(q, "bf16", kc_r, vc_r, "bf16", bt, sl, 0.125, lib=lib))
    # 3. block size 16 vs 32 on the same logical data
    kc32, vc32, bt32, sl32 = paged_from_logical(Ks, Vs, 32, 12, _rng(23), "bf16")
    assert np.array_equal(base, oracle.decode(q, "bf16", kc32, vc32, "bf16", bt32, sl32, 0.125, lib=lib))
    # 4. a sequence whose table shares another's prefix blocks equals its private copy
    #    (sequence 1 reuses sequence 0's first two blocks, i.e. tokens 0..31)
    bt_s = bt.copy()
    kc_s, vc_s = kc.copy(), vc.copy()
    for b in range(2):
        kc_s[bt[1, b]], vc_s[bt[1, b]] = kc[bt[0, b]], vc[bt[0, b]]
    private = oracle.decode(q, "bf16", kc_s, vc_s, "bf16", bt_s, sl, 0.125, lib=lib)
    bt_s[1, :2] = bt[0, :2]
    shared = oracle.decode(q, "bf16", kc_s, vc_s, "bf16", bt_s, sl, 0.125, lib=lib)
    assert np.array_equal(private, shared)


def check_cow_leaves_parent(lib):
    # parent of 21 tokens, child forks it and writes token 21 through copy-on-write
    from paged_kv_cache_327_b200.block_manager import BlockAllocator, BlockTable
    bs, H, D = 16, 1, 64
    alloc = BlockAllocator(8, bs, seed=5)
    parent = BlockTable(bs)
    slots = parent.append_tokens(21, alloc)
    child = BlockTable(bs)
    child.fork_from(parent, alloc)
    rng = _rng(31)
    kc = np.full((8, bs, H, D), W.NAN_BITS["f16"], np.uint16)
    vc = kc.copy()
    kc.reshape(-1, H, D)[slots] = W.to_storage(rng.standard_normal((21, H, D), dtype=np.float32), "f16")
    vc.reshape(-1, H, D)[slots] = W.to_storage(rng.standard_normal((21, H, D), dtype=np.float32), "f16")
    q = rng.standard_normal((1, H, D), dtype=np.float32)
    bt_p = np.asarray([parent.get_physical_blocks()], np.int32)
    before = oracle.decode(q, "f32", kc, vc, "f16", bt_p, np.asarray([21], np.int32), 0.125, lib=lib)
    slot = child.append_token(alloc)
    pairs = alloc.take_pending_copies()
    assert len(pairs) == 1
    oracle.copy_blocks(kc, vc, pairs, lib=lib)
    newk = W.to_storage(rng.standard_normal((1, H, D), dtype=np.float32), "f16")
    oracle.reshape_and_cache(newk, newk.copy(), kc, vc, np.asarray([slot], np.int64), "f16", lib=lib)
    after = oracle.decode(q, "f32", kc, vc, "f16", bt_p, np.asarray([21], np.int32), 0.125, lib=lib)
    assert np.array_equal(before, after), "copy-on-write changed the parent's output"
    # and the child sees the parent's 21 tokens plus its own
    bt_c = np.asarray([child.get_physical_blocks()], np.int32)
    kc_ref = kc.copy()
    child_out = oracle.decode(q, "f32", kc, vc, "f16", bt_c, np.asarray([22], np.int32), 0.125, lib=lib)
    Kl = np.concatenate([W.storage_to_f32(kc.reshape(-1, H, D)[slots], "f16"), W.storage_to_f32(newk, "f16")])
    Vl = np.concatenate([W.storage_to_f32(vc.reshape(-1, H, D)[slots], "f16"), W.storage_to_f32(newk, "f16")])
    ref = sdpa_reference(q, [Kl], [Vl], 0.125, 1)
    assert np.max(np.abs(child_out - ref)) < 1e-12
    assert np.array_equal(kc, kc_ref)


def check_reshape_and_cache(lib):
    rng = _rng(41)
    NB, bs, H, D, T = 6, 16, 3, 64, 20
    for dt in ("f16", "bf16"):
        kc = W.to_storage(rng.standard_normal((NB, bs, H, D), dtype=np.float32), dt)
        vc = W.to_storage(rng.standard_normal((NB, bs, H, D), dtype=np.float32), dt)
        k = W.to_storage(rng.standard_normal((T, H, D), dtype=np.float32), dt)
        v = W.to_storage(rng.standard_normal((T, H, D), dtype=np.float32), dt)
        slots = rng.choice(NB * bs, size=T, replace=False).astype(np.int64)
        slots[[3, 11]] = -1                                    # skipped tokens
        ek, ev = kc.copy(), vc.copy()
        keep = slots >= 0
        ek.reshape(NB * bs, H, D)[slots[keep]] = k[keep]
        ev.reshape(NB * bs, H, D)[slots[keep]] = v[keep]
        oracle.reshape_and_cache(k, v, kc, vc, slots, dt, lib=lib)
        assert np.array_equal(kc, ek) and np.array_equal(vc, ev)


def check_copy_blocks(lib):
    rng = _rng(51)
    NB, bs, H, D = 9, 16, 2, 64
    kc = W.to_storage(rng.standard_normal((NB, bs, H, D), dtype=np.float32), "bf16")
    vc = W.to_storage(rng.standard_normal((NB, bs, H, D), dtype=np.float32), "bf16")
    pairs = np.asarray([[2, 7], [0, 5], [2, 8]], np.int32)
    ek, ev = kc.copy(), vc.copy()
    for s, d in pairs:
        ek[d], ev[d] = ek[s], ev[s]
    oracle.copy_blocks(kc, vc, pairs, lib=lib)
    assert np.array_equal(kc, ek) and np.array_equal(vc, ev)


# ------------------------------------------------------------------ FP8 (E4M3) KV cache
E4M3_FINITE = [c for c in range(256) if (c & 0x7f) != 0x7f]


def _e4m3_values():
    return torch.arange(256, dtype=torch.int32).to(torch.uint8).view(torch.float8_e4m3fn).double().numpy()


def brute_force_e4m3(x: float) -> int:
    """Nearest finite E4M3 code by exhaustive search; ties to the even code; |x| > 448 saturates."""
    vals = _e4m3_values()
    if abs(x) > 448.0:
        return 0xFE if x < 0 else 0x7E
    best, bd = None, None
    for c in E4M3_FINITE:
        if (c >> 7) != (1 if math.copysign(1.0, x) < 0 else 0):
            continue
        d = abs(float(vals[c]) - x)
        if bd is None or d < bd or (d == bd and (c & 1) == 0 and (best & 1) == 1):
            best, bd = c, d
    return best


def check_e4m3_decode(lib):
    ref = _e4m3_values()
    got = np.array([lib.oracle_e4m3_to_f64(c) for c in range(256)])
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan) and np.array_equal(got[~nan], ref[~nan])
    assert lib.oracle_e4m3_to_f64(0x7E) == 448.0 and lib.oracle_e4m3_to_f64(0x01) == 2.0 ** -9


def check_e4m3_encode(lib):
    rng = _rng(71)
    vals = _e4m3_values()
    pos = np.sort(np.unique(vals[[c for c in E4M3_FINITE if c < 0x80]]))
    mids = ((pos[1:] + pos[:-1]) / 2).astype(np.float32)      # exact ties between neighbours
    xs = np.concatenate([rng.standard_normal(300).astype(np.float32) * 10 ** rng.uniform(-3, 2.5, 300).astype(np.float32),
                         mids, -mids, pos.astype(np.float32), np.float32([0.0, -0.0, 447.9, 448.0, 449.0, 460.0,
                                                                          465.0, 1e6, -1e6, 2.0 ** -10, 2.0 ** -11])])
    for x in xs:
        got = lib.oracle_f32_to_e4m3(ctypes_float(x))
        want = brute_force_e4m3(float(x))
        assert got == want, (float(x), got, want)
    # in range, torch's round-to-nearest-even cast agrees
    inr = xs[np.abs(xs) <= 448]
    t = torch.from_numpy(inr).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = np.array([lib.oracle_f32_to_e4m3(ctypes_float(x)) for x in inr], dtype=np.uint8)
    assert np.array_equal(got, t)


def ctypes_float(x):
    import ctypes
    return ctypes.c_float(float(x))


def check_reshape_and_cache_e4m3(lib):
    rng = _rng(72)
    NB, bs, H, D, T = 5, 16, 2, 64, 12
    for in_dt in ("bf16", "f16", "f32"):
        kc = rng.integers(0, 256, size=(NB, bs, H, D), dtype=np.uint8)
        vc = rng.integers(0, 256, size=(NB, bs, H, D), dtype=np.uint8)
        k = W.to_storage(rng.standard_normal((T, H, D), dtype=np.float32) * 3, in_dt)
        v = W.to_storage(rng.standard_normal((T, H, D), dtype=np.float32) * 3, in_dt)
        ks, vs = np.float32(0.0371), np.float32(0.0459)   # |x / scale| stays below 448
        slots = rng.choice(NB * bs, size=T, replace=False).astype(np.int64)
        slots[4] = -1
        ek, ev = kc.copy(), vc.copy()
        keep = slots >= 0
        qk = (torch.from_numpy(W.storage_to_f32(k, in_dt)) / torch.tensor(ks)).to(torch.float8_e4m3fn)
        qv = (torch.from_numpy(W.storage_to_f32(v, in_dt)) / torch.tensor(vs)).to(torch.float8_e4m3fn)
        ek.reshape(NB * bs, H, D)[slots[keep]] = qk.view(torch.uint8).numpy()[keep]
        ev.reshape(NB * bs, H, D)[slots[keep]] = qv.view(torch.uint8).numpy()[keep]
        oracle.reshape_and_cache_e4m3(k, v, kc, vc, slots, in_dt, float(ks), float(vs), lib=lib)
        assert np.array_equal(kc, ek) and np.array_equal(vc, ev), in_dt


def check_decode_e4m3_vs_sdpa(lib):
    rng = _rng(73)
    for n, (lens, Hq, Hkv, D, bs, qd) in enumerate([([40, 1, 77], 8, 2, 128, 16, "bf16"),
                                                     ([33, 130], 4, 4, 64, 32, "f32")]):
        ks, vs = 0.0123, 0.0211
        codes_k = [rng.choice(E4M3_FINITE, size=(L, Hkv, D)).astype(np.uint8) for L in lens]
        codes_v = [rng.choice(E4M3_FINITE, size=(L, Hkv, D)).astype(np.uint8) for L in lens]
        vals = _e4m3_values()
        Ks = [vals[c] * np.float64(np.float32(ks)) for c in codes_k]
        Vs = [vals[c] * np.float64(np.float32(vs)) for c in codes_v]
        NB = sum(-(-L // bs) for L in lens) + 2
        kc = np.zeros((NB, bs, Hkv, D), np.uint8)
        vc = np.zeros_like(kc)
        perm = list(_rng(74 + n).permutation(NB))
        bt = np.full((len(lens), max(-(-L // bs) for L in lens)), -1, np.int32)
        for i, L in enumerate(lens):
            for b in range(-(-L // bs)):
                phys = perm.pop(0)
                bt[i, b] = phys
                m = min(bs, L - b * bs)
                kc[phys, :m] = codes_k[i][b * bs:b * bs + m]
                vc[phys, :m] = codes_v[i][b * bs:b * bs + m]
        q32 = W.storage_to_f32(W.to_storage(rng.standard_normal((len(lens), Hq, D), dtype=np.float32), qd), qd)
        scale = float(np.float32(1 / math.sqrt(D)))
        got = oracle.decode(W.to_storage(q32, qd), qd, kc, vc, "e4m3", bt, np.asarray(lens, np.int32), scale,
                            lib=lib, k_scale=ks, v_scale=vs)
        ref = sdpa_reference(q32, Ks, Vs, scale, Hq // Hkv)
        assert np.max(np.abs(got - ref)) < 1e-12, n


def check_swap_blocks(lib):
    rng = _rng(81)
    src_k = rng.integers(0, 256, size=(7, 16, 2, 64, 2), dtype=np.uint8)
    src_v = rng.integers(0, 256, size=src_k.shape, dtype=np.uint8)
    dst_k = rng.integers(0, 256, size=(5, 16, 2, 64, 2), dtype=np.uint8)
    dst_v = rng.integers(0, 256, size=dst_k.shape, dtype=np.uint8)
    pairs = np.asarray([[6, 0], [2, 4], [0, 1]], np.int32)
    ek, ev = dst_k.copy(), dst_v.copy()
    for s_, d_ in pairs:
        ek[d_], ev[d_] = src_k[s_], src_v[s_]
    sk, sv = src_k.copy(), src_v.copy()
    oracle.swap_blocks(dst_k, dst_v, src_k, src_v, pairs, lib=lib)
    assert np.array_equal(dst_k, ek) and np.array_equal(dst_v, ev)
    assert np.array_equal(src_k, sk) and np.array_equal(src_v, sv), "the source pool is left as it was"


MULTI_CASES = [
    # lens, T, Hq, Hkv, D, bs, q_dtype, kv_dtype
    ([5, 17, 40, 0], 5, 4, 2, 64, 16, "f32", "f16"),
    ([33, 64, 4], 4, 8, 2, 128, 16, "bf16", "bf16"),
    ([70, 3], 3, 6, 3, 128, 32, "f16", "f16"),
    ([20, 48], 8, 4, 1, 64, 32, "bf16", "bf16"),
]


def random_multi_case(seed, lens, T, Hq, Hkv, D, bs, q_dtype, kv_dtype):
    rng = _rng(seed)
    q32 = W.storage_to_f32(W.to_storage(rng.standard_normal((len(lens), T, Hq, D), dtype=np.float32), q_dtype),
                           q_dtype)
    Ks, Vs = [], []
    for L in lens:
        Ks.append(W.storage_to_f32(W.to_storage(rng.standard_normal((L, Hkv, D), dtype=np.float32), kv_dtype), kv_dtype))
        Vs.append(W.storage_to_f32(W.to_storage(rng.standard_normal((L, Hkv, D), dtype=np.float32), kv_dtype), kv_dtype))
    kc, vc, bt, sl = paged_from_logical(Ks, Vs, bs, sum(-(-L // bs) for L in lens) + 2, rng, kv_dtype)
    return W.to_storage(q32, q_dtype), q32, Ks, Vs, kc, vc, bt, sl


def causal_sdpa_reference(q32, Ks, Vs, scale, G):
    """torch SDPA in fp64 with a boolean mask: query token t sees key positions <= L - T + t."""
    N, T = q32.shape[:2]
    outs = []
    for i, (K, V) in enumerate(zip(Ks, Vs)):
        L = len(K)
        if L == 0:
            outs.append(np.zeros(q32.shape[1:], np.float64))
            continue
        qi = torch.from_numpy(q32[i].astype(np.float64)).permute(1, 0, 2)[None]   # [1,Hq,T,D]
        k = torch.from_numpy(K.astype(np.float64)).permute(1, 0, 2)[None]        # [1,Hkv,L,D]
        v = torch.from_numpy(V.astype(np.float64)).permute(1, 0, 2)[None]
        mask = torch.arange(L)[None, :] <= (L - T + torch.arange(T))[:, None]    # [T, L]
        o = torch.nn.functional.scaled_dot_product_attention(qi, k, v, attn_mask=mask, scale=scale,
                                                             enable_gqa=G > 1)
        outs.append(o[0].permute(1, 0, 2).numpy())                               # [T,Hq,D]
    return np.stack(outs)


def check_multi_vs_sdpa(lib, cases=MULTI_CASES):
    for n, (lens, T, Hq, Hkv, D, bs, qd, kd) in enumerate(cases):
        q, q32, Ks, Vs, kc, vc, bt, sl = random_multi_case(300 + n, lens, T, Hq, Hkv, D, bs, qd, kd)
        scale = float(np.float32(1 / math.sqrt(D)))
        got = oracle.decode_multi(q, qd, kc, vc, kd, bt, sl, scale, num_threads=2, lib=lib)
        ref = causal_sdpa_reference(q32, Ks, Vs, scale, Hq // Hkv)
        err = np.max(np.abs(got - ref))
        assert err < 1e-12, f"case {n}: multi-token oracle vs causal SDPA max|err| = {err}"


def check_multi_causal_closed_form(lib):
    """Zero keys make every visible score equal: query token t of a sequence of L tokens
    returns the mean of V over positions 0 .. L - T + t, exactly the positions it sees."""
    rng = _rng(17)
    T, L, D, bs = 6, 37, 64, 16
    K = np.zeros((L, 1, D), np.float32)
    V = rng.integers(-8, 9, size=(L, 1, D)).astype(np.float32)
    kc, vc, bt, sl = paged_from_logical([K], [V], bs, 6, rng, "f16")
    q = W.to_storage(rng.standard_normal((1, T, 1, D), dtype=np.float32), "f32")
    got = oracle.decode_multi(q, "f32", kc, vc, "f16", bt, sl, 0.3, num_threads=1, lib=lib)[0, :, 0]
    for t in range(T):
        want = V[:L - T + t + 1, 0].astype(np.float64).mean(axis=0)
        assert np.max(np.abs(got[t] - want)) < 1e-12, f"query token {t}"


def check_multi_reduces_to_decode(lib):
    """Query token t equals a one-token decode of the sequence cut after position L - T + t."""
    lens, T = [9, 40, 0, 4], 4
    q, q32, Ks, Vs, kc, vc, bt, sl = random_multi_case(77, lens, T, 4, 2, 64, 16, "bf16", "bf16")
    got = oracle.decode_multi(q, "bf16", kc, vc, "bf16", bt, sl, 0.125, num_threads=1, lib=lib)
    for t in range(T):
        cut = np.where(sl > 0, sl - T + t + 1, 0).astype(np.int32)
        one = oracle.decode(np.ascontiguousarray(q[:, t]), "bf16", kc, vc, "bf16", bt, cut, 0.125, num_threads=1,
                            lib=lib)
        assert np.array_equal(got[:, t], one), f"query token {t}"


ALL_CHECKS = [check_swap_blocks, check_f16_decode, check_bf16_decode, check_decode_vs_sdpa, check_closed_forms,
              check_page_block_table_example, check_invariants, check_cow_leaves_parent,
              check_reshape_and_cache, check_copy_blocks, check_e4m3_decode, check_e4m3_encode,
              check_reshape_and_cache_e4m3, check_decode_e4m3_vs_sdpa, check_multi_vs_sdpa,
              check_multi_causal_closed_form, check_multi_reduces_to_decode]


@pytest.fixture(scope="module")
def lib():
    return oracle._load()


@pytest.mark.parametrize("check", ALL_CHECKS, ids=lambda c: c.__name__)
def test_oracle_pin(lib, check):
    check(lib)


def test_oracle_thread_count_does_not_change_bits(lib):
    q, q32, Ks, Vs, kc, vc, bt, sl = random_case(61, [100, 5, 64, 33, 1, 0], 4, 2, 64, 16, "bf16", "bf16")
    a = oracle.decode(q, "bf16", kc, vc, "bf16", bt, sl, 0.125, num_threads=1, lib=lib)
    b = oracle.decode(q, "bf16", kc, vc, "bf16", bt, sl, 0.125, num_threads=5, lib=lib)
    assert np.array_equal(a, b)
    assert np.all(a[5] == 0.0), "a zero-length sequence gives a zero row"


def test_oracle_rejects_bad_indices(lib):
    q, q32, Ks, Vs, kc, vc, bt, sl = random_case(62, [20, 5], 2, 2, 64, 16, "f16", "f16")
    bad = bt.copy()
    bad[0, 1] = kc.shape[0]
    with pytest.raises(oracle.OracleError):
        oracle.decode(q, "f16", kc, vc, "f16", bad, sl, 0.125, lib=lib)
    with pytest.raises(oracle.OracleError):
        oracle.copy_blocks(kc, vc, np.asarray([[0, kc.shape[0]]], np.int32), lib=lib)
    with pytest.raises(oracle.OracleError):
        oracle.reshape_and_cache(kc[0], vc[0], kc, vc, np.full(16, kc.shape[0] * 16, np.int64), "f16", lib=lib)
    # a sequence must hold at least its query tokens
    qm = np.zeros((2, 6, 2, 64), np.uint16)
    with pytest.raises(oracle.OracleError):
        oracle.decode_multi(qm, "f16", kc, vc, "f16", bt, sl, 0.125, lib=lib)
