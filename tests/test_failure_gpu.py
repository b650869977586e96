"""Failure detection on the GPU without a fault (needs a B200).

Every wait in the library's kernels is bounded: after its poll limit it records PA_DEV_TIMEOUT
in the device error word and the kernel returns.  pa_selftest_wait_timeout runs that same wait
on a barrier nothing ever completes; the test checks that the status reaches the host and that
the context stays usable (a decode afterwards is correct).  Data-dependent faults (bad block
ids, lengths, slots, pairs, prefix groups) are covered beside their operations.
"""
import time

import numpy as np
import pytest
import torch

import oracle
from paged_kv_cache_327_b200 import binding as B
from paged_kv_cache_327_b200 import workload as W

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _require_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    B.load_library()


@pytest.mark.parametrize("polls", [1, 4096])
def test_bounded_wait_gives_up_and_reports(polls):
    assert B.pa_get_device_error() in (B.PA_DEV_OK, B.PA_DEV_TIMEOUT)  # clear the word
    t0 = time.perf_counter()
    B.pa_selftest_wait_timeout(polls)
    assert B.pa_get_device_error() == B.PA_DEV_TIMEOUT
    assert time.perf_counter() - t0 < 5.0, "each poll sleeps at most 1 us"
    assert B.pa_get_device_error() == B.PA_DEV_OK, "reading the word clears it"


def test_context_is_usable_after_a_timeout():
    B.pa_selftest_wait_timeout(64)
    assert B.pa_get_device_error() == B.PA_DEV_TIMEOUT
    w = W.make_config("tiny")
    dw = B.device_workload(w)
    out = torch.empty((w.num_seqs, w.num_q_heads, w.head_dim), device="cuda")
    B.run_step(dw, out, B.DecodeWorkspace.for_workload(dw))
    torch.cuda.synchronize()
    assert B.pa_get_device_error() == B.PA_DEV_OK
    kc, vc = w.k_cache.copy(), w.v_cache.copy()
    oracle.copy_blocks(kc, vc, w.copy_pairs)
    oracle.reshape_and_cache(w.new_k, w.new_v, kc, vc, w.slot_mapping, w.kv_dtype)
    ref = oracle.decode(w.q, w.q_dtype, kc, vc, w.kv_dtype, w.block_tables, w.seq_lens, w.scale)
    assert np.max(np.abs(out.cpu().numpy() - ref)) < 2e-3
