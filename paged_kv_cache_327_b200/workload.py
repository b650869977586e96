"""Seeded synthetic decode-step workloads shaped like the models on the vLLM pages.

This module only builds inputs: sequence lengths, block tables (through the
refcounted allocator in ``block_manager``), the pre-step paged K/V pool, the step's
new K/V tokens with their slots, the copy-on-write pairs and the queries.  It holds
none of the attention arithmetic and is shared, as the single input source, by the
tests, the bench and the oracle-side checks.

A decode step, as the Llama attention layer on "vLLM 深度解读" (section 7) orders it:
  1. copy_blocks    -- duplicate every shared block that a sequence is about to
                       write into (copy-on-write, "详解vLLM推理引擎架构", "Copy-on-Write");
  2. reshape_and_cache -- store the step's new K/V tokens into their slots;
  3. decode         -- attend with one query per sequence over seq_lens[i] tokens,
                       the new ones included.

Value recipe: every K, V and q element is drawn from N(0, 1) in float32 and rounded
to nearest-even into the stored dtype (fp16 / bf16; fp32 q stays as drawn).  Pool
positions that no sequence has written hold a NaN pattern, so any stray read of them
poisons the output.  Each config draws from ``numpy.random.default_rng([seed, stream])``
with seed = 3270 + config index and separate streams for lengths, placement, q,
history K/V and new K/V, so logical values do not depend on the block size or the pool.
"""
from __future__ import annotations

import concurrent.futures
import dataclasses
import math
import os
from typing import Dict, List, Optional, Sequence, Tuple

import numpy as np

from .block_manager import BlockAllocator, BlockTable, tables_to_array

ELEM_BYTES = {"f32": 4, "f16": 2, "bf16": 2, "e4m3": 1}
NAN_BITS = {"f16": 0x7E00, "bf16": 0x7FC0, "e4m3": 0x7F}

# Default per-tensor scales of an FP8 (E4M3) cache for N(0,1) data: |x| / scale stays well
# inside the format's +-448 for every draw (|x| < 7).
FP8_K_SCALE, FP8_V_SCALE = 0.0171, 0.0193

# random streams
_S_LENS, _S_PLACE, _S_Q, _S_HIST, _S_NEW, _S_EXTRA = range(6)


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 to bfloat16 (nearest, ties to even); returns the uint16 bit patterns."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    bias = ((u >> np.uint32(16)) & np.uint32(1)) + np.uint32(0x7FFF)
    return ((u + bias) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def to_storage(x: np.ndarray, dtype: str) -> np.ndarray:
    """float32 values -> storage array (float32, or uint16 bit patterns for f16 / bf16)."""
    if dtype == "f32":
        return np.ascontiguousarray(x, dtype=np.float32)
    if dtype == "f16":
        return np.ascontiguousarray(x, dtype=np.float32).astype(np.float16).view(np.uint16)
    if dtype == "bf16":
        return f32_to_bf16_bits(x)
    raise ValueError(f"unknown dtype {dtype!r}")


def storage_to_f32(a: np.ndarray, dtype: str) -> np.ndarray:
    if dtype == "f32":
        return np.asarray(a, dtype=np.float32)
    if dtype == "f16":
        return np.asarray(a, dtype=np.uint16).view(np.float16).astype(np.float32)
    if dtype == "bf16":
        return bf16_bits_to_f32(a)
    raise ValueError(f"unknown dtype {dtype!r}")


_CHUNK = 1 << 22


def to_e4m3_codes(x: np.ndarray, scale: float) -> np.ndarray:
    """float32 values -> FP8 E4M3 codes of x / scale (torch's round-to-nearest-even cast),
    clamped to the format's +-448 first."""
    import torch
    y = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)) / torch.tensor(np.float32(scale))
    y = torch.clamp(y, -448.0, 448.0)
    return y.to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def _draw(key: Tuple[int, ...], shape, dtype: str) -> np.ndarray:
    """N(0,1) values rounded into ``dtype`` storage, generated in fixed 4 Mi-element chunks.

    Chunk c is drawn from default_rng(key + (c,)), so the values depend only on ``key``
    and the element count, never on the thread count.
    """
    n = int(np.prod(shape, dtype=np.int64))
    fp8_scale = None
    if isinstance(dtype, tuple):  # ("e4m3", scale): codes of N(0,1) / scale
        dtype, fp8_scale = dtype
    out = np.empty(n, dtype={"f32": np.float32, "e4m3": np.uint8}.get(dtype, np.uint16))

    def fill(c: int) -> None:
        lo, hi = c * _CHUNK, min(n, (c + 1) * _CHUNK)
        x = np.random.default_rng(list(key) + [c]).standard_normal(hi - lo, dtype=np.float32)
        out[lo:hi] = to_e4m3_codes(x, fp8_scale) if dtype == "e4m3" else to_storage(x, dtype)

    chunks = range(-(-n // _CHUNK))
    if n > _CHUNK:
        with concurrent.futures.ThreadPoolExecutor(max_workers=min(16, os.cpu_count() or 1)) as ex:
            list(ex.map(fill, chunks))
    else:
        for c in chunks:
            fill(c)
    return out.reshape(shape)


@dataclasses.dataclass
class Group:
    """Sequences that share a prefix: member 0 owns the prefix, members 1.. fork from it.

    prefix: tokens cached before the step (shared by every member).
    step_tokens: tokens each member appends in this step (through reshape_and_cache).
    own_history: tokens each member appended after the fork and before the step (None: none).
        Their first write into a shared partial block went through copy-on-write then, so
        those copies are part of the cache state before the step, not of the step.
    """
    prefix: int
    step_tokens: List[int]
    own_history: Optional[List[int]] = None


@dataclasses.dataclass
class Workload:
    name: str
    num_seqs: int
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    block_size: int
    num_blocks: int
    q_dtype: str
    kv_dtype: str
    scale: float                  # float32 value of 1/sqrt(head_dim)
    q: np.ndarray                 # [N, Hq, D]; [N, T, Hq, D] with T = num_q_tokens > 1
    k_cache: np.ndarray           # [NB, bs, Hkv, D], state before the step
    v_cache: np.ndarray
    block_tables: np.ndarray      # int32 [N, MB], padded with -1
    seq_lens: np.ndarray          # int32 [N], after the step
    new_k: np.ndarray             # [T, Hkv, D]
    new_v: np.ndarray
    slot_mapping: np.ndarray      # int64 [T]
    copy_pairs: np.ndarray        # int32 [P, 2]
    notes: Dict[str, object] = dataclasses.field(default_factory=dict)
    new_dtype: str = ""           # dtype of new_k / new_v ("" = kv_dtype)
    k_scale: float = 1.0          # FP8 cache: value = code * scale
    v_scale: float = 1.0
    num_q_tokens: int = 1         # query tokens per sequence: the last T tokens, stored in the step

    @property
    def new_kv_dtype(self) -> str:
        return self.new_dtype or self.kv_dtype

    @property
    def max_blocks_per_seq(self) -> int:
        return int(self.block_tables.shape[1])

    @property
    def group_size(self) -> int:
        return self.num_q_heads // self.num_kv_heads

    @property
    def kv_row_bytes(self) -> int:
        """Bytes of one token's K (or V) row over all KV heads."""
        return self.num_kv_heads * self.head_dim * ELEM_BYTES[self.kv_dtype]

    @property
    def block_bytes(self) -> int:
        return self.block_size * self.kv_row_bytes

    def total_tokens(self) -> int:
        return int(self.seq_lens.astype(np.int64).sum())

    def kv_bytes_logical(self) -> int:
        """K+V bytes decode reads: each (token, KV head) of each sequence counted once."""
        return 2 * self.total_tokens() * self.kv_row_bytes

    def kv_bytes_unique(self) -> int:
        """K+V bytes of distinct physical token slots reached by any sequence (shared blocks once)."""
        used: Dict[int, int] = {}
        bs = self.block_size
        for i in range(self.num_seqs):
            L = int(self.seq_lens[i])
            nb = -(-L // bs)
            for b in range(nb):
                phys = int(self.block_tables[i, b])
                n = min(bs, L - b * bs)
                if used.get(phys, 0) < n:
                    used[phys] = n
        return 2 * sum(used.values()) * self.kv_row_bytes

    def num_partitions(self, partition_size: int = 512) -> int:
        L = self.seq_lens.astype(np.int64)
        return int(((L + partition_size - 1) // partition_size).sum())

    def io_bytes(self) -> Dict[str, int]:
        """Algorithmic bytes of one decode call other than K/V."""
        q_bytes = self.q.nbytes
        return {"q": q_bytes, "block_tables": int(sum(-(-int(L) // self.block_size) for L in self.seq_lens)) * 4,
                "seq_lens": self.num_seqs * 4}


def build_groups(name: str, groups: Sequence[Group], *, num_q_heads: int, num_kv_heads: int,
                 head_dim: int, block_size: int, q_dtype: str, kv_dtype: str, seed: int,
                 pool_factor: float = 1.25, num_blocks: Optional[int] = None,
                 notes: Optional[dict] = None, new_dtype: str = "bf16",
                 k_scale: float = FP8_K_SCALE, v_scale: float = FP8_V_SCALE, num_q_tokens: int = 1) -> Workload:
    """Materialise a decode step from groups of prefix-sharing sequences.

    Sequence order is group by group, member by member.  The pool holds
    ``num_blocks`` blocks, or ceil(pool_factor * blocks the step needs).  With kv_dtype
    "e4m3" the pool holds FP8 codes of N(0,1) / scale, and the step's new tokens are
    ``new_dtype`` values that the step itself quantises.  With num_q_tokens T > 1 the
    queries are [N, T, Hq, D]: each sequence's step appends T tokens (or none, for an empty
    sequence), which its T query tokens then attend to causally.
    """
    if num_q_heads % num_kv_heads:
        raise ValueError("num_q_heads must be a multiple of num_kv_heads")
    for g in groups:
        if g.prefix < 0 or not g.step_tokens or min(g.step_tokens) < 0:
            raise ValueError("bad group")
        if g.own_history is not None and (len(g.own_history) != len(g.step_tokens) or min(g.own_history) < 0):
            raise ValueError("own_history needs one non-negative count per member")
    bs = block_size

    def run(allocator: BlockAllocator):
        tables: List[BlockTable] = []
        prefix_slots: List[np.ndarray] = []
        own_slots: List[np.ndarray] = []
        step_slots: List[List[np.ndarray]] = []
        hist_pairs: List[np.ndarray] = []
        step_pairs: List[np.ndarray] = []
        for g in groups:
            parent = BlockTable(bs)
            prefix_slots.append(parent.append_tokens(g.prefix, allocator))
            members = [parent]
            for _ in g.step_tokens[1:]:
                child = BlockTable(bs)
                child.fork_from(parent, allocator)
                members.append(child)
            if g.own_history is not None:
                own_slots.extend(m.append_tokens(n, allocator) for m, n in zip(members, g.own_history))
            hist_pairs.append(allocator.take_pending_copies())
            step_slots.append([m.append_tokens(n, allocator) for m, n in zip(members, g.step_tokens)])
            step_pairs.append(allocator.take_pending_copies())
            tables.extend(members)
        return (tables, prefix_slots, own_slots, step_slots, np.concatenate(hist_pairs + [np.zeros((0, 2), np.int32)]),
                np.concatenate(step_pairs + [np.zeros((0, 2), np.int32)]))

    # dry run on an identity-ordered pool large enough for anything: counts the blocks needed
    upper = sum(-(-g.prefix // bs) + sum(-(-n // bs) + 1 for n in g.step_tokens) +
                sum(-(-n // bs) + 1 for n in (g.own_history or [])) for g in groups) + 1
    probe = BlockAllocator(upper, bs)
    run(probe)
    need = upper - probe.get_num_free_blocks()
    if num_blocks is None:
        num_blocks = max(1, int(math.ceil(pool_factor * need)))
    if num_blocks < need:
        raise ValueError(f"pool of {num_blocks} blocks is smaller than the {need} the step needs")

    place_rng = np.random.default_rng([seed, _S_PLACE])
    allocator = BlockAllocator(num_blocks, bs, rng=place_rng)
    tables, prefix_slots, own_slots, step_slots, hist_pairs, pairs = run(allocator)

    N = len(tables)
    Hkv, D = num_kv_heads, head_dim
    if num_q_tokens > 1 and any(n not in (0, num_q_tokens) for g in groups for n in g.step_tokens):
        raise ValueError("with several query tokens every sequence appends exactly that many tokens (or none)")
    # the [N, Hq, D] draw of one query token is the [N, 1, Hq, D] draw
    q = _draw((seed, _S_Q), (N, num_q_tokens, num_q_heads, head_dim), q_dtype)
    if num_q_tokens == 1:
        q = q.reshape(N, num_q_heads, head_dim)

    # history: every group's prefix tokens, in group order, K then V
    nan = NAN_BITS[kv_dtype]
    fp8 = kv_dtype == "e4m3"
    pool_t = np.uint8 if fp8 else np.uint16
    k_cache = np.full((num_blocks, bs, Hkv, D), nan, dtype=pool_t)
    v_cache = np.full((num_blocks, bs, Hkv, D), nan, dtype=pool_t)
    hist_slots = np.concatenate([np.zeros(0, np.int64)] + prefix_slots)
    H = len(hist_slots)
    kdt = ("e4m3", k_scale) if fp8 else kv_dtype
    vdt = ("e4m3", v_scale) if fp8 else kv_dtype
    if H:
        k_cache.reshape(num_blocks * bs, Hkv, D)[hist_slots] = _draw((seed, _S_HIST, 0), (H, Hkv, D), kdt)
        v_cache.reshape(num_blocks * bs, Hkv, D)[hist_slots] = _draw((seed, _S_HIST, 1), (H, Hkv, D), vdt)
    # members' own history: the copy-on-write copies of their first writes, then the tokens
    for src, dst in hist_pairs:
        k_cache[dst] = k_cache[src]
        v_cache[dst] = v_cache[src]
    own = np.concatenate([np.zeros(0, np.int64)] + own_slots)
    if len(own):
        k_cache.reshape(num_blocks * bs, Hkv, D)[own] = _draw((seed, _S_HIST, 2), (len(own), Hkv, D), kdt)
        v_cache.reshape(num_blocks * bs, Hkv, D)[own] = _draw((seed, _S_HIST, 3), (len(own), Hkv, D), vdt)

    all_slots = np.concatenate([np.zeros(0, np.int64)] +
                               [s for per_group in step_slots for s in per_group]).astype(np.int64)
    T = len(all_slots)
    ndt = new_dtype if fp8 else kv_dtype
    new_k = _draw((seed, _S_NEW, 0), (T, Hkv, D), ndt)
    new_v = _draw((seed, _S_NEW, 1), (T, Hkv, D), ndt)

    seq_lens = np.asarray([t.num_tokens for t in tables], dtype=np.int32)
    block_tables = tables_to_array(tables)
    info = {"groups": len(groups), "blocks_needed": int(need), "cow_pairs": int(len(pairs)),
            "cow_pairs_before_step": int(len(hist_pairs)), "new_tokens": int(T), "pool_factor": pool_factor}
    if notes:
        info.update(notes)
    return Workload(name=name, num_seqs=N, num_q_heads=num_q_heads, num_kv_heads=num_kv_heads,
                    head_dim=head_dim, block_size=bs, num_blocks=num_blocks, q_dtype=q_dtype,
                    kv_dtype=kv_dtype, scale=float(np.float32(1.0 / math.sqrt(head_dim))), q=q,
                    k_cache=k_cache, v_cache=v_cache, block_tables=block_tables, seq_lens=seq_lens,
                    new_k=new_k, new_v=new_v, slot_mapping=all_slots, copy_pairs=pairs, notes=info,
                    new_dtype=ndt, k_scale=float(np.float32(k_scale)) if fp8 else 1.0,
                    v_scale=float(np.float32(v_scale)) if fp8 else 1.0, num_q_tokens=num_q_tokens)


def independent(name: str, seq_lens: Sequence[int], num_q_tokens: int = 1, **kw) -> Workload:
    """Each sequence on its own; seq_lens are post-step lengths, the last num_q_tokens tokens
    stored in the step (a sequence holds 0 or at least num_q_tokens tokens)."""
    T = num_q_tokens
    if any(0 < int(L) < T for L in seq_lens):
        raise ValueError("a sequence must hold 0 or at least num_q_tokens tokens")
    groups = [Group(prefix=max(int(L) - T, 0), step_tokens=[T if L > 0 else 0]) for L in seq_lens]
    return build_groups(name, groups, num_q_tokens=T, **kw)


def _fp8_kw(kw: dict, fp8: bool) -> dict:
    """A config over an FP8 cache: the config's own dtype becomes the new tokens' dtype."""
    if fp8:
        kw = dict(kw, new_dtype=kw["kv_dtype"], kv_dtype="e4m3")
    return kw


# ---------------------------------------------------------------------------------------
# The five named decode configurations.
# ---------------------------------------------------------------------------------------
CONFIG_NAMES = ("tiny", "7b", "13b", "8b", "70b")
CONFIG_INDEX = {n: i + 1 for i, n in enumerate(CONFIG_NAMES)}


def config_seed(name: str) -> int:
    return 3270 + CONFIG_INDEX[name]


def _tiny(seed: int, block_size: int, fp8: bool = False) -> Workload:
    # 4 sequences, post-step lengths uniform in [1, 64]; sequence 3 is a fork of sequence 2
    # (parallel sampling), so the step's first write into their shared partial block is the
    # one copy-on-write pair.  Fixed pool of 64 blocks.
    rng = np.random.default_rng([seed, _S_LENS])
    L = [int(x) for x in rng.integers(1, 65, size=2)]
    while True:
        L2 = int(rng.integers(1, 65))
        if (L2 - 1) % block_size != 0:
            break
    groups = [Group(L[0] - 1, [1]), Group(L[1] - 1, [1]), Group(L2 - 1, [1, 1])]
    if fp8:
        raise ValueError("the tiny config (head_dim 64) has no FP8 variant")
    return build_groups("tiny", groups, num_q_heads=2, num_kv_heads=2, head_dim=64,
                        block_size=block_size, q_dtype="f32", kv_dtype="f16", seed=seed,
                        num_blocks=64, notes={"lens": "uniform[1,64]; seq 3 forks seq 2"})


def _7b(seed: int, block_size: int, num_seqs: int = 64, num_q_tokens: int = 1, fp8: bool = False) -> Workload:
    rng = np.random.default_rng([seed, _S_LENS])
    L = np.maximum(rng.integers(128, 2049, size=num_seqs), num_q_tokens)
    kw = dict(num_q_heads=32, num_kv_heads=32, head_dim=128, block_size=block_size, q_dtype="bf16",
              kv_dtype="bf16", seed=seed, notes={"lens": "uniform[128,2048]"})
    return independent("7b", L, num_q_tokens, **_fp8_kw(kw, fp8))


def _13b(seed: int, block_size: int, num_seqs: int = 128, num_q_tokens: int = 1, fp8: bool = False) -> Workload:
    rng = np.random.default_rng([seed, _S_LENS])
    L = np.maximum(rng.integers(16, 2049, size=num_seqs), num_q_tokens)
    kw = dict(num_q_heads=40, num_kv_heads=40, head_dim=128, block_size=block_size, q_dtype="f16",
              kv_dtype="f16", seed=seed, notes={"lens": "uniform[16,2048]"})
    return independent(f"13b-bs{block_size}", L, num_q_tokens, **_fp8_kw(kw, fp8))


def lognormal_lengths(rng: np.random.Generator, n: int, median: float = 1024.0, sigma: float = 1.0,
                      lo: int = 32, hi: int = 8192) -> np.ndarray:
    z = rng.standard_normal(n)
    return np.clip(np.rint(np.exp(math.log(median) + sigma * z)), lo, hi).astype(np.int64)


def _8b(seed: int, block_size: int, num_seqs: int = 256, num_q_tokens: int = 1, fp8: bool = False,
        uniform_lens: Optional[Tuple[int, int]] = None) -> Workload:
    # uniform_lens=(lo, hi): the same shapes with lengths uniform in [lo, hi] (e.g. thousands of short
    # or empty sequences, for the plan kernel's scaling) instead of the lognormal mix
    rng = np.random.default_rng([seed, _S_LENS])
    if uniform_lens is None:
        L = np.maximum(lognormal_lengths(rng, num_seqs), num_q_tokens)
        lens = "lognormal(median 1024, sigma 1.0) clipped to [32, 8192]"
    else:
        lo, hi = uniform_lens
        L = rng.integers(lo, hi + 1, size=num_seqs)
        L = np.where(L > 0, np.maximum(L, num_q_tokens), 0)
        lens = f"uniform[{lo},{hi}]"
    kw = dict(num_q_heads=32, num_kv_heads=8, head_dim=128, block_size=block_size, q_dtype="bf16",
              kv_dtype="bf16", seed=seed, notes={"lens": lens})
    return independent("8b", L, num_q_tokens, **_fp8_kw(kw, fp8))


STEPS_70B = ("decode", "fork")


def _70b(seed: int, block_size: int, num_groups: int = 64, samples: int = 4,
         prefix: int = 4096, long_len: int = 32768, num_long: int = 4, step: str = "decode",
         fp8: bool = False) -> Workload:
    # 64 groups x 4 samples.  Each group's parent holds prefix + r_g tokens, r_g uniform in
    # [1, bs-1], so its last shared block is partial; the samples fork from it and each has a
    # divergent suffix of uniform [1, 512] tokens: the first three writers into the shared
    # partial block copy it, the fourth writes in place.  Four standalone 32768-token
    # sequences ride in the same batch.
    #   step "decode": one decode step of every sequence -- each stores one new token (256 + 4
    #     new tokens); a sample's earlier suffix tokens, and the copy-on-write of its first
    #     write, precede the step (a sample whose suffix is that one token copies in the step);
    #   step "fork": every sample's whole suffix is stored in the step, so all 192 copies
    #     (64 groups x 3) are part of it.
    if step not in STEPS_70B:
        raise ValueError(f"step must be one of {STEPS_70B}")
    rng = np.random.default_rng([seed, _S_LENS])
    groups = []
    for _ in range(num_groups):
        r = int(rng.integers(1, block_size))
        suffix = [int(x) for x in rng.integers(1, 513, size=samples)]
        if step == "fork":
            groups.append(Group(prefix + r, suffix))
        else:
            groups.append(Group(prefix + r, [1] * samples, own_history=[n - 1 for n in suffix]))
    groups += [Group(long_len - 1, [1]) for _ in range(num_long)]
    stored = "one token per sequence" if step == "decode" else "each sample's whole suffix"
    kw = dict(num_q_heads=64, num_kv_heads=8, head_dim=128, block_size=block_size, q_dtype="bf16",
              kv_dtype="bf16", seed=seed,
              notes={"lens": "64 groups x 4 samples: prefix 4096+r (r in [1,bs-1]) + suffix uniform[1,512]; "
                             "plus 4 x 32768", "step": f"{step}: the step stores {stored}"})
    return build_groups("70b" if step == "decode" else "70b-fork", groups, **_fp8_kw(kw, fp8))


_BUILDERS = {"tiny": _tiny, "7b": _7b, "13b": _13b, "8b": _8b, "70b": _70b}
_DEFAULT_BS = {"tiny": 16, "7b": 16, "13b": 16, "8b": 16, "70b": 16}


def make_config(name: str, block_size: Optional[int] = None, seed: Optional[int] = None,
                kv_dtype: Optional[str] = None, **overrides) -> Workload:
    """Build one of the named decode configs ("tiny", "7b", "13b", "8b", "70b").

    kv_dtype="e4m3" gives the same config over an FP8 cache (head_dim 128 configs): the
    history is stored as FP8 codes, the step's new tokens stay in the config's dtype.
    num_q_tokens=T ("7b", "13b", "8b") gives the multi-token step: the same lengths (raised to T
    where shorter), the last T tokens of every sequence stored in the step and attended to
    causally by T queries.  step="fork" ("70b") stores every sample's whole suffix in the step
    instead of one token per sequence.
    """
    if name not in _BUILDERS:
        raise KeyError(f"unknown config {name!r}; choose from {CONFIG_NAMES}")
    if kv_dtype not in (None, "e4m3"):
        raise ValueError("kv_dtype is None (the config's own) or 'e4m3'")
    bs = block_size or _DEFAULT_BS[name]
    return _BUILDERS[name](config_seed(name) if seed is None else seed, bs, fp8=kv_dtype == "e4m3", **overrides)


def apply_step_host(w: Workload) -> Tuple[np.ndarray, np.ndarray]:
    """The post-step caches computed with plain numpy indexing (no kernel, no oracle).

    Used only to give tests an independent expectation of the cache state.  Not defined for
    an FP8 cache, whose step quantises the new tokens.
    """
    if w.kv_dtype == "e4m3":
        raise ValueError("the post-step state of an FP8 cache needs the quantising store")
    kc, vc = w.k_cache.copy(), w.v_cache.copy()
    for s, d in w.copy_pairs:
        kc[d] = kc[s]
        vc[d] = vc[s]
    NB, bs, Hkv, D = kc.shape
    keep = w.slot_mapping >= 0
    kc.reshape(NB * bs, Hkv, D)[w.slot_mapping[keep]] = w.new_k[keep]
    vc.reshape(NB * bs, Hkv, D)[w.slot_mapping[keep]] = w.new_v[keep]
    return kc, vc
