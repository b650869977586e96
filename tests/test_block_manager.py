"""Host block manager and workload generator (CPU only).

Pins: ceil(num_tokens / block_size) blocks per table and the exhausted-pool error
("vLLM 深度解读", section 2); fork shares blocks and copy-on-write copies only a
block whose refcount exceeds 1, then drops one reference from it ("详解vLLM推理引擎架构",
"Copy-on-Write 与内存共享"); the seeded free list gives a shuffled placement.
"""
import numpy as np
import pytest
from paged_kv_cache_327_b200 import block_manager as BM

from paged_kv_cache_327_b200 import workload as W
from paged_kv_cache_327_b200.block_manager import (BlockAllocator, BlockTable, NoFreeBlocksError,
                                                   tables_to_array)


def test_required_blocks_is_ceil():
    t = BlockTable(16)
    assert [t.get_num_required_blocks(n) for n in (0, 1, 15, 16, 17, 32, 33)] == [0, 1, 1, 1, 2, 2, 3]
    t32 = BlockTable(32)
    assert t32.get_num_required_blocks(33) == 2


def test_allocator_exhaustion_raises_and_free_returns():
    a = BlockAllocator(3, 16, seed=1)
    got = [a.allocate() for _ in range(3)]
    assert sorted(got) == [0, 1, 2]
    with pytest.raises(NoFreeBlocksError):
        a.allocate()
    a.free(got[1])
    assert a.get_num_free_blocks() == 1
    assert a.allocate() == got[1]


def test_seeded_placement_is_shuffled_and_reproducible():
    a = [BlockAllocator(64, 16, seed=7).allocate() for _ in range(1)]
    b1 = BlockAllocator(64, 16, seed=7)
    b2 = BlockAllocator(64, 16, seed=7)
    s1 = [b1.allocate() for _ in range(64)]
    s2 = [b2.allocate() for _ in range(64)]
    assert s1 == s2 and sorted(s1) == list(range(64)) and s1 != list(range(64))
    assert a[0] == s1[0]


def test_append_slots_allocates_when_block_full():
    a = BlockAllocator(10, 4, seed=None)
    t = BlockTable(4)
    slots = t.append_tokens(9, a)
    assert len(t) == 3 and t.num_tokens == 9
    blocks = t.get_physical_blocks()
    assert list(slots) == [blocks[j // 4] * 4 + j % 4 for j in range(9)]
    # token-at-a-time gives the same slots
    a2 = BlockAllocator(10, 4, seed=None)
    t2 = BlockTable(4)
    assert [t2.append_token(a2) for _ in range(9)] == list(slots)


def test_fork_and_copy_on_write_counts():
    a = BlockAllocator(16, 4, seed=3)
    parent = BlockTable(4)
    parent.append_tokens(6, a)                      # 2 blocks, last one half full
    kids = []
    for _ in range(3):
        c = BlockTable(4)
        c.fork_from(parent, a)
        kids.append(c)
    last = parent.get_block_number(1)
    assert a.get_refcount(last) == 4 and a.get_refcount(parent.get_block_number(0)) == 4
    # writers 1..3 copy (refcount 4 -> 3 -> 2 -> 1), the last one writes in place
    for t in [parent] + kids:
        t.append_token(a)
    pairs = a.take_pending_copies()
    assert len(pairs) == 3 and all(p[0] == last for p in pairs)
    assert len({int(p[1]) for p in pairs}) == 3 and last not in {int(p[1]) for p in pairs}
    assert a.get_refcount(last) == 1
    assert kids[-1].get_block_number(1) == last
    # the full first block stays shared
    assert a.get_refcount(parent.get_block_number(0)) == 4


def test_write_to_unshared_block_copies_nothing():
    a = BlockAllocator(4, 4, seed=0)
    t = BlockTable(4)
    t.append_tokens(2, a)
    t.write_to_block(0, a)
    assert len(a.take_pending_copies()) == 0


def test_refcount_underflow_raises():
    a = BlockAllocator(2, 4)
    b = a.allocate()
    a.free(b)
    with pytest.raises(ValueError):
        a.free(b)


def test_tables_to_array_pads():
    a = BlockAllocator(8, 4, seed=2)
    t1, t2 = BlockTable(4), BlockTable(4)
    t1.append_tokens(9, a)
    t2.append_tokens(1, a)
    arr = tables_to_array([t1, t2])
    assert arr.shape == (2, 3) and arr.dtype == np.int32 and list(arr[1, 1:]) == [-1, -1]


def test_tiny_config_has_one_cow_pair_and_poisoned_pool():
    w = W.make_config("tiny")
    assert w.num_seqs == 4 and w.num_blocks == 64 and len(w.copy_pairs) == 1
    assert w.q.dtype == np.float32 and w.kv_dtype == "f16"
    assert all(1 <= L <= 64 for L in w.seq_lens)
    assert w.seq_lens[2] == w.seq_lens[3]
    # the CoW destination is unwritten (NaN) before the step
    dst = int(w.copy_pairs[0, 1])
    assert np.all(w.k_cache[dst] == W.NAN_BITS["f16"])
    # after copy + store, every position a sequence reads is finite
    kc, vc = W.apply_step_host(w)
    for i in range(w.num_seqs):
        L = int(w.seq_lens[i])
        for j in range(L):
            phys = w.block_tables[i, j // 16]
            assert np.all(np.isfinite(W.storage_to_f32(kc[phys, j % 16], "f16")))


def test_workload_draws_do_not_depend_on_block_size():
    a = W.independent("x", [40, 3, 77], num_q_heads=4, num_kv_heads=2, head_dim=64, block_size=16,
                      q_dtype="bf16", kv_dtype="bf16", seed=9)
    b = W.independent("x", [40, 3, 77], num_q_heads=4, num_kv_heads=2, head_dim=64, block_size=32,
                      q_dtype="bf16", kv_dtype="bf16", seed=9)
    assert np.array_equal(a.q, b.q) and np.array_equal(a.new_k, b.new_k)
    for w in (a, b):
        kc, _ = W.apply_step_host(w)
        flat = kc.reshape(-1, 2, 64)
        w.__dict__["_logical"] = np.concatenate(
            [flat[w.block_tables[i, np.arange(L) // w.block_size] * w.block_size + np.arange(L) % w.block_size]
             for i, L in enumerate(w.seq_lens)])
    assert np.array_equal(a._logical, b._logical)


def test_bf16_rounding_is_nearest_even():
    x = np.array([1.0, 1.0 + 2**-8, 1.0 + 3 * 2**-8, 1.0 + 2**-9, -2.5, 3.0e-39], np.float32)
    got = W.bf16_bits_to_f32(W.f32_to_bf16_bits(x))
    import torch
    ref = torch.from_numpy(x).to(torch.bfloat16).float().numpy()
    assert np.array_equal(got, ref)


@pytest.mark.parametrize("name", ["7b", "13b", "8b", "70b"])
def test_named_config_shapes(name):
    w = W.make_config(name)
    G = {"7b": 1, "13b": 1, "8b": 4, "70b": 8}[name]
    assert w.group_size == G and w.head_dim == 128
    L = w.seq_lens
    if name == "7b":
        assert w.num_seqs == 64 and L.min() >= 128 and L.max() <= 2048
    if name == "13b":
        assert w.num_seqs == 128 and L.min() >= 16 and L.max() <= 2048
    if name == "8b":
        assert w.num_seqs == 256 and L.min() >= 32 and L.max() <= 8192
        assert 700 < np.median(L) < 1400
    if name == "70b":
        # one decode step: one new token per sequence; the 64 x 3 copy-on-write copies of the
        # samples' first writes precede it (a sample whose whole suffix is the step's token
        # copies in the step)
        assert w.num_seqs == 260 and len(w.slot_mapping) == 260
        assert len(w.copy_pairs) + w.notes["cow_pairs_before_step"] == 192
        assert sorted(L)[-4:] == [32768] * 4
        assert w.kv_bytes_unique() < w.kv_bytes_logical() / 2
    assert w.num_blocks >= int(np.ceil(1.25 * w.notes["blocks_needed"]))
    # no block is referenced by two different sequences unless it is a shared prefix block
    if name != "70b":
        used = np.concatenate([w.block_tables[i, :-(-int(l) // w.block_size)] for i, l in enumerate(L)])
        assert len(np.unique(used)) == len(used)


def test_70b_fork_step_stores_every_suffix():
    """The fork-step variant of the 70B batch: the same sequences, but every sample's whole
    suffix (and so every copy-on-write) lies in the step."""
    a = W.make_config("70b")
    b = W.make_config("70b", step="fork")
    assert np.array_equal(a.seq_lens, b.seq_lens)
    assert len(b.copy_pairs) == 192 and b.notes["cow_pairs_before_step"] == 0
    # a group's samples store their suffixes (1..512 tokens each), a long sequence one token
    assert 256 + 4 < len(b.slot_mapping) <= 256 * 512 + 4
    # the step's tokens of the decode variant are the last token of every sequence; in the fork
    # variant each sample stores its whole suffix, which ends with that token
    assert a.kv_bytes_unique() == b.kv_bytes_unique()
    with pytest.raises(ValueError):
        W.make_config("70b", step="prefill")


def test_fp8_configs_are_reentrant():
    """An FP8 config build leaves no state behind: the next plain build is the plain config."""
    f = W.make_config("8b", kv_dtype="e4m3", num_seqs=4)
    p = W.make_config("8b", num_seqs=4)
    assert f.kv_dtype == "e4m3" and f.new_kv_dtype == "bf16"
    assert p.kv_dtype == "bf16" and p.new_kv_dtype == "bf16"
    with pytest.raises(ValueError):
        W.make_config("tiny", kv_dtype="e4m3")


def test_swap_out_and_in_move_groups_and_keep_sharing():
    from paged_kv_cache_327_b200.block_manager import swap_in, swap_out
    gpu = BlockAllocator(16, 4, seed=11)
    cpu = BlockAllocator(8, 4, seed=12)
    parent = BlockTable(4)
    parent.append_tokens(9, gpu)                      # 3 blocks
    child = BlockTable(4)
    child.fork_from(parent, gpu)
    child.append_token(gpu)                           # copy-on-write of the partial block
    gpu.take_pending_copies()
    before_free = gpu.get_num_free_blocks()
    old = (parent.get_physical_blocks(), child.get_physical_blocks())
    pairs = swap_out([parent, child], gpu, cpu)
    # 2 shared full blocks + 2 private last blocks = 4 distinct blocks move once each
    assert len(pairs) == 4 and len(set(pairs[:, 0])) == 4 and len(set(pairs[:, 1])) == 4
    assert gpu.get_num_free_blocks() == before_free + 4
    m = {int(a): int(b) for a, b in pairs}
    assert parent.get_physical_blocks() == [m[b] for b in old[0]]
    assert child.get_physical_blocks() == [m[b] for b in old[1]]
    assert cpu.get_refcount(parent.get_block_number(0)) == 2          # still shared on the CPU side
    back = swap_in([parent, child], cpu, gpu)
    assert len(back) == 4 and cpu.get_num_free_blocks() == 8
    assert gpu.get_refcount(parent.get_block_number(0)) == 2
    assert parent.get_block_number(0) == child.get_block_number(0)


# ---------------------------------------------------------------------------------------------
# prefix groups (input of pa_decode_prefix)
# ---------------------------------------------------------------------------------------------
def test_prefix_groups_of_the_70b_batch():
    from paged_kv_cache_327_b200 import workload as W
    w = W.make_config("70b")
    g = BM.find_prefix_groups(w.block_tables, w.seq_lens, w.block_size)
    # 64 parents of 4096 + r tokens (r < 16) forked into 4 samples; the partial block is
    # copied on write, so exactly the 256 full blocks are shared; the long sequences stand alone
    assert g.shape == (64, 3)
    assert np.array_equal(g[:, 0], np.arange(0, 256, 4)) and np.all(g[:, 1] == 4) and np.all(g[:, 2] == 4096)
    for first, m, S in g:
        nb = S // w.block_size
        for k in range(1, m):
            assert np.array_equal(w.block_tables[first + k, :nb], w.block_tables[first, :nb])
        # the next block is no longer shared by all members
        assert len({int(w.block_tables[first + k, nb]) for k in range(m)}) > 1


def test_prefix_groups_edge_cases():
    bs = 16
    bt = np.array([[7, 8, 9, -1],      # 0: leader
                   [7, 8, 3, -1],      # 1: shares 2 blocks with 0
                   [7, 8, 9, 4],       # 2: shares 3 with 0, but the run's common part is 2 blocks
                   [5, 6, -1, -1],     # 3: alone
                   [1, 2, -1, -1],     # 4: shares block 1 only partly filled by 5
                   [1, 2, -1, -1],     # 5
                   [10, -1, -1, -1],   # 6: shares a block 7 does not fill
                   [10, -1, -1, -1],   # 7
                   [11, 12, -1, -1],   # 8: same table as 9 but not next to it in order
                   [13, -1, -1, -1],   # 9
                   [11, 12, -1, -1]],  # 10
                  np.int32)
    lens = np.array([40, 40, 60, 20, 32, 20, 16, 10, 30, 5, 30], np.int32)
    g = BM.find_prefix_groups(bt, lens, bs)
    assert g.tolist() == [[0, 3, 32], [4, 2, 16]]


def test_prefix_groups_of_forks_built_by_the_allocator():
    bs = 16
    alloc = BM.BlockAllocator(64, bs, seed=4)
    parent = BM.BlockTable(bs)
    parent.append_tokens(40, alloc)           # 2 full blocks + 8 tokens
    kids = []
    for _ in range(3):
        k = BM.BlockTable(bs)
        k.fork_from(parent, alloc)
        kids.append(k)
    for t in [parent] + kids:
        t.append_tokens(5, alloc)             # copy-on-write of the partial third block
    tables = [parent] + kids
    g = BM.find_prefix_groups(BM.tables_to_array(tables), np.array([t.num_tokens for t in tables]), bs)
    assert g.tolist() == [[0, 4, 32]]
