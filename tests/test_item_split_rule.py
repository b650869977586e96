"""Invariants of the work-item split rule (PA_OPT_ITEM_SPLIT), on the CPU.

tests/test_item_split_gpu.py restates the plan kernel's rule in Python and compares the kernel's
work list with it word for word on the GPU.  Here the same restatement runs over many random
batches and pipeline counts, and the properties the host side relies on are checked:

  * every sequence's own tokens are covered once, in order, by its pieces;
  * every piece but a sequence's last holds whole partitions, at most four and at most 128 blocks;
  * a sequence never has more pieces than ceil(L / P): the partial results fit the workspace that
    pa_decode_workspace_size() reserves;
  * the list holds all long pieces, then the middle ones, then the tails, and no tail is longer
    than a middle piece, so the items that end a launch are the short ones;
  * PA_SPLIT_FIXED gives pieces of exactly P tokens (and a shorter tail).
"""
import math
import types

import numpy as np
import pytest

import tests.test_item_split_gpu as rule

P = rule.P


def batch(rng, n, max_len, bs=16, hkv=8):
    lens = rng.integers(0, max_len + 1, size=n)
    return types.SimpleNamespace(num_seqs=n, num_kv_heads=hkv, block_size=bs, seq_lens=lens)


@pytest.mark.parametrize("fixed", [False, True])
@pytest.mark.parametrize("rings", [148, 592, 1184])
def test_rule_invariants_on_random_batches(rings, fixed):
    rng = np.random.default_rng(3270 + rings + fixed)
    for trial in range(40):
        n = int(rng.integers(1, 600))
        w = batch(rng, n, int(rng.choice([40, 700, 4096, 32768])), bs=int(rng.choice([16, 32])))
        items, parts, (_, Pb, Pm) = rule.expected_list(w, rings, fixed, 1)
        mmax = 1 if fixed else min(4 * P, 128 * w.block_size) // P
        assert P <= Pm <= Pb <= mmax * P and Pb % P == 0 and Pm % P == 0
        if fixed:
            assert Pb == Pm == P
        for i in range(n):
            rows = items[items[:, 0] == i]
            L = int(w.seq_lens[i])
            # covered once, in order
            assert rows.shape[0] == 0 if L == 0 else rows[0, 1] == 0
            if L:
                assert np.array_equal(rows[1:, 1], rows[:-1, 2]) and rows[-1, 2] == L
            sizes = rows[:, 2] - rows[:, 1]
            # whole partitions (at most four, at most 128 blocks) but the last piece
            assert np.all(sizes[:-1] % P == 0) and np.all(sizes <= mmax * P)
            # the workspace holds every partial result
            assert rows.shape[0] <= max(1, math.ceil(L / P))
            assert parts[i] == (-1 if L == 0 else 0 if rows.shape[0] == 1 else rows.shape[0])
            # partial-result numbers run 0 .. count - 1
            assert np.array_equal(rows[:, 3] & 0xffff, np.arange(rows.shape[0]))
        # long pieces (Pb, when longer than Pm), then middle ones (Pm), then tails (shorter than Pm):
        # along the list the class never goes back
        sizes = items[:, 2] - items[:, 1]
        cls = np.where((sizes == Pb) & (Pb > Pm), 0, np.where(sizes == Pm, 1, 2))
        assert np.all(np.diff(cls) >= 0)
        assert np.all(sizes[cls == 2] < Pm)
