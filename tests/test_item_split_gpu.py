"""How the decode calls cut sequences into work items (PA_OPT_ITEM_SPLIT), read back from the
plan kernel's work list.

The plan kernel leaves its work list in the caller's workspace: a 256-byte header whose second
32-bit word is the item count, three per-sequence int32 arrays (partial-result count, shared
tokens, members led), each padded to 256 bytes, then the items, eight int32 words each:
(sequence, first token, end token, partial result | members << 16 | direct << 30, first query
token, query tokens, 0, 0).  These white-box tests rebuild that list from the rule that
include/pa.h states and compare the two word for word:

  * counted at one partition (P tokens) each, the call's own items come to n per page pipeline
    (SMs x 4 rings, x 8 with an FP8 cache, x 1 on the tensor-core kernel), its shared items to
    n_sh; shared items take min(4, n_sh / 2) partitions, a sequence's leading own tokens
    min(4, n / 2), the following ones min(4, n / 8), then its ragged tail;
  * the list holds shared items, then long, then middle own items, then tails, each kind in
    sequence order; a sequence with no shared tokens and one item writes `out` directly;
  * PA_SPLIT_FIXED keeps every piece at P tokens, so a sequence's output is the same bits in
    every batch, which the last test checks on the full 8B-shaped batch.

The attention these lists lead to is checked against the oracle by the parity tests, with the
adaptive split in force at every full-size batch.
"""
import numpy as np
import pytest
import torch

from paged_kv_cache_327_b200 import binding as B
from paged_kv_cache_327_b200 import block_manager as BM
from paged_kv_cache_327_b200 import workload as W

pytestmark = pytest.mark.gpu

P = 512
DIRECT = 1 << 30


@pytest.fixture(scope="module", autouse=True)
def _require_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    B.load_library()


@pytest.fixture(autouse=True)
def _restore_options():
    yield
    B.set_item_split("adaptive")
    B.set_wide_kernel("auto")


def align256(n):
    return (n + 255) // 256 * 256


def work_list(ws, num_seqs):
    """(items [n, 8], seq_parts, seq_shared, seq_sub) from a workspace after a call."""
    t = ws.tensor
    n = int(t[:8].view(torch.int32)[1].item())
    a = align256(num_seqs * 4)
    arrays = [t[256 + k * a:256 + k * a + num_seqs * 4].view(torch.int32).cpu().numpy() for k in range(3)]
    off = 256 + 3 * a
    items = t[off:off + 32 * n].view(torch.int32).reshape(n, 8).cpu().numpy()
    return items, arrays[0], arrays[1], arrays[2]


def expected_list(w, rings, fixed, T, seq_shared=None, seq_sub=None):
    """The work list the stated rule gives (one column group: T query tokens per item)."""
    N, hkv, bs = w.num_seqs, w.num_kv_heads, w.block_size
    L = np.asarray(w.seq_lens, dtype=np.int64)
    S = np.zeros(N, np.int64) if seq_shared is None else seq_shared.astype(np.int64)
    sub = np.zeros(N, np.int64) if seq_sub is None else seq_sub.astype(np.int64)
    mmax = 1 if fixed else min(4 * P, 128 * bs) // P
    n_sh = int(sum((S[i] + P - 1) // P for i in range(N) if sub[i] > 0)) * hkv
    n_own = int(sum((L[i] - S[i] + P - 1) // P for i in range(N))) * hkv
    Ps = max(1, min(mmax, n_sh // (2 * rings))) * P
    Pb = max(1, min(mmax, n_own // (2 * rings))) * P
    Pm = max(1, min(mmax, n_own // (8 * rings))) * P
    shared, long_, mid, tail, parts = [], [], [], [], np.zeros(N, np.int64)
    for i in range(N):
        s, own = int(S[i]), int(L[i] - S[i])
        nps = (s + Ps - 1) // Ps
        if sub[i] > 0:
            for k in range(nps):
                shared.append([i, k * Ps, min(s, (k + 1) * Ps), k | (int(sub[i]) << 16), 0, 1, 0, 0])
        nb = own // Pb if Pb > Pm else 0
        nm = (own - nb * Pb) // Pm
        nt = 1 if (own - nb * Pb) % Pm else 0
        n_parts = nps + nb + nm + nt
        direct = s == 0 and n_parts == 1
        parts[i] = -1 if L[i] == 0 else 0 if direct else n_parts
        flag = DIRECT if direct else 0
        tok, part = s, nps
        for dst, count, size in ((long_, nb, Pb), (mid, nm, Pm)):
            for _ in range(count):
                dst.append([i, tok, tok + size, part | (1 << 16) | flag, 0, T, 0, 0])
                tok, part = tok + size, part + 1
        if nt:
            tail.append([i, tok, int(L[i]), part | (1 << 16) | flag, 0, T, 0, 0])
    items = np.array(shared + long_ + mid + tail, dtype=np.int64).reshape(-1, 8)
    return items, parts, (Ps, Pb, Pm)


def run_call(w):
    """One step (the step's tokens stored, then decode) with a fresh workspace."""
    dw = B.device_workload(w)
    ws = B.DecodeWorkspace.for_workload(dw)
    out = torch.empty(tuple(dw.q.shape), dtype=torch.bfloat16, device="cuda")
    B.run_step(dw, out, ws)
    torch.cuda.synchronize()
    assert B.pa_get_device_error() == B.PA_DEV_OK
    return dw, ws, out


# (name, config overrides, pipelines per SM, expect pieces longer than P under the adaptive rule)
CASES = [
    ("8b", dict(), 4, True),
    ("8b_small", dict(num_seqs=8), 4, False),
    ("8b_T8", dict(num_q_tokens=8), 4, True),
    ("8b_T16_tcgen05", dict(num_q_tokens=16), 1, True),
    ("8b_e4m3", dict(kv_dtype="e4m3"), 8, True),
]


@pytest.mark.parametrize("split", ["adaptive", "fixed"])
@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_work_list_follows_the_rule(case, split):
    name, kw, per_sm, longer = case
    w = W.make_config("8b", **kw)
    B.set_item_split(split)
    dw, ws, out = run_call(w)
    assert torch.isfinite(out.float()).all()
    sm = torch.cuda.get_device_properties(0).multi_processor_count
    got, parts, _, _ = work_list(ws, w.num_seqs)
    want, want_parts, (_, Pb, Pm) = expected_list(w, sm * per_sm, split == "fixed", w.num_q_tokens)
    assert got.shape == want.shape, f"{name}: {got.shape[0]} items, the rule gives {want.shape[0]}"
    assert np.array_equal(got, want), f"{name}: work list differs from the rule at item " \
                                      f"{int(np.argmax((got != want).any(axis=1)))}"
    assert np.array_equal(parts, want_parts)
    assert (Pb > P) == (longer and split == "adaptive"), (Pb, Pm)
    # every sequence's tokens are covered once, in order
    for i in range(w.num_seqs):
        rows = got[got[:, 0] == i]
        rows = rows[np.argsort(rows[:, 1])]
        ends = np.concatenate([[0], rows[:, 2]])
        assert np.array_equal(rows[:, 1], ends[:-1]) and ends[-1] == w.seq_lens[i]


def test_prefix_work_list_follows_the_rule():
    """The 70B shared-prefix batch: shared items of up to four partitions per leader, then the
    members' and the long sequences' own items."""
    w = W.make_config("70b")
    dw = B.device_workload(w)
    ws = B.DecodeWorkspace.for_workload(dw)
    out = torch.empty(tuple(dw.q.shape), dtype=torch.bfloat16, device="cuda")
    g = torch.from_numpy(BM.find_prefix_groups(w.block_tables, w.seq_lens, w.block_size)).cuda()
    mm = B.max_prefix_members(w.num_q_heads, w.num_kv_heads)
    B.pa_decode_prefix(out, dw.q, dw.k_cache, dw.v_cache, dw.block_tables, dw.seq_lens, w.scale, ws.tensor, g, mm)
    torch.cuda.synchronize()
    assert B.pa_get_device_error() == B.PA_DEV_OK
    got, parts, shared, sub = work_list(ws, w.num_seqs)
    assert (sub > 0).sum() == g.shape[0] and shared.max() > 0
    sm = torch.cuda.get_device_properties(0).multi_processor_count
    want, want_parts, (Ps, Pb, Pm) = expected_list(w, sm * 4, False, 1, shared, sub)
    assert Ps > P
    assert np.array_equal(got, want)
    assert np.array_equal(parts, want_parts)


def test_fixed_split_is_batch_invariant_at_full_size():
    """Under PA_SPLIT_FIXED the longest sequence of the full 8B-shaped batch (which the adaptive
    split cuts into longer pieces) decodes to the same bits alone as in the batch."""
    w = W.make_config("8b")
    B.set_item_split("fixed")
    dw, _, a = run_call(w)
    assert torch.isfinite(a.float()).all()
    i = int(np.argmax(w.seq_lens))
    one = torch.empty((1,) + tuple(a.shape[1:]), dtype=a.dtype, device="cuda")
    ws1 = B.DecodeWorkspace(1, w.num_q_heads, w.head_dim, w.max_blocks_per_seq * w.block_size)
    B.pa_decode(one, dw.q[i:i + 1].contiguous(), dw.k_cache, dw.v_cache, dw.block_tables[i:i + 1].contiguous(),
                dw.seq_lens[i:i + 1].contiguous(), w.scale, ws1.tensor)
    torch.cuda.synchronize()
    assert torch.equal(one[0], a[i])
    B.set_item_split("adaptive")
    _, _, b = run_call(w)
    assert (a.float() - b.float()).abs().max().item() < 2e-2  # two splits of the same attention
