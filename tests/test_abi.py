"""The C ABI on a machine without a GPU: the library loads, exports every entry point
that include/pa.h declares, and rejects invalid arguments on the host before any CUDA
call (no compute is launched here)."""
import ctypes
import os
import re

import numpy as np
import pytest

from paged_kv_cache_327_b200 import binding as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "pa.h")


def declared_symbols():
    text = open(HEADER, encoding="utf-8").read()
    return re.findall(r"^PA_API\s+[\w\s\*]+?\b(pa_\w+)\s*\(", text, flags=re.M)


@pytest.fixture(scope="module")
def lib():
    from paged_kv_cache_327_b200 import build
    build.build()
    return B.load_library()


def test_header_declares_the_entry_points():
    names = declared_symbols()
    assert set(names) == set(B.EXPORTED), names


def test_library_exports_every_declared_symbol(lib):
    for name in declared_symbols():
        assert hasattr(lib, name), f"{name} not exported"


def test_version_and_strerror(lib):
    assert lib.pa_version() == 101
    for st in (B.PA_OK, B.PA_ERR_INVALID, B.PA_ERR_UNSUPPORTED, B.PA_ERR_WORKSPACE, B.PA_ERR_CUDA):
        assert len(B.pa_strerror(st)) > 5
    assert "unknown" in B.pa_strerror(12345)


def test_workspace_size(lib):
    ws = B.pa_decode_workspace_size
    assert ws(0, 1, 128, 0) > 0
    assert ws(-1, 32, 128, 100) == 0 and ws(4, 0, 128, 100) == 0
    a = ws(256, 32, 128, 8192)
    # 16 partitions of 512 per sequence: the fp32 partial outputs dominate
    assert a >= 256 * 16 * 32 * 128 * 4
    assert ws(256, 32, 128, 8192, 256) > a
    assert ws(256, 32, 128, 8193) > a


FAKE = 0x10000  # a 16-byte aligned non-null address that is never dereferenced


def decode_call(lib, **kw):
    a = dict(out=FAKE, q=FAKE, k=FAKE, v=FAKE, bt=FAKE, sl=FAKE, N=4, Hq=8, Hkv=2, D=128, bs=16, scale=0.1,
             MB=8, NB=64, qd=2, kd=2, od=0, P=0, ws=FAKE, wsb=0, stream=0)
    a.update(kw)
    V = ctypes.c_void_p
    return lib.pa_decode(V(a["out"]), V(a["q"]), V(a["k"]), V(a["v"]), V(a["bt"]), V(a["sl"]), a["N"], a["Hq"],
                         a["Hkv"], a["D"], a["bs"], ctypes.c_float(a["scale"]), a["MB"], a["NB"], a["qd"], a["kd"],
                         a["od"], a["P"], V(a["ws"]), a["wsb"], V(a["stream"]))


def test_decode_argument_validation(lib):
    assert decode_call(lib, N=0) == B.PA_OK                      # nothing to do, no CUDA call
    assert decode_call(lib, Hq=6, Hkv=4) == B.PA_ERR_INVALID     # heads not a multiple
    assert decode_call(lib, Hq=32, Hkv=2) == B.PA_ERR_UNSUPPORTED  # G = 16
    assert decode_call(lib, D=96) == B.PA_ERR_UNSUPPORTED
    assert decode_call(lib, bs=8) == B.PA_ERR_UNSUPPORTED
    assert decode_call(lib, kd=0, qd=0) == B.PA_ERR_UNSUPPORTED  # fp32 cache
    assert decode_call(lib, qd=1) == B.PA_ERR_UNSUPPORTED        # f16 q with bf16 cache
    assert decode_call(lib, od=7) == B.PA_ERR_UNSUPPORTED
    assert decode_call(lib, P=24) == B.PA_ERR_UNSUPPORTED        # not a multiple of the block size
    assert decode_call(lib, P=1024) == B.PA_ERR_UNSUPPORTED      # more than 32 blocks per partition
    assert decode_call(lib, scale=float("nan")) == B.PA_ERR_INVALID
    assert decode_call(lib, q=0) == B.PA_ERR_INVALID
    assert decode_call(lib, k=FAKE + 8) == B.PA_ERR_INVALID      # misaligned cache
    assert decode_call(lib, wsb=100) == B.PA_ERR_WORKSPACE
    # the size query bounds every decode entry point (prefix groups need one more partition per
    # sequence than plain decode); a workspace well below it is refused
    need = B.pa_decode_workspace_size(4, 8, 128, 8 * 16)
    assert decode_call(lib, wsb=need // 2) == B.PA_ERR_WORKSPACE
    assert decode_call(lib, ws=FAKE + 16, wsb=need) == B.PA_ERR_INVALID   # workspace not 256-aligned


def test_cache_op_argument_validation(lib):
    V = ctypes.c_void_p
    r = lib.pa_reshape_and_cache
    assert r(V(FAKE), V(FAKE), V(FAKE), V(FAKE), V(FAKE), 0, 8, 128, 16, 10, 2, 0, 0, V(0)) == B.PA_OK
    assert r(V(FAKE), V(FAKE), V(FAKE), V(FAKE), V(FAKE), 3, 8, 128, 16, 10, 2, 100, 0, V(0)) == B.PA_ERR_INVALID
    assert r(V(FAKE), V(FAKE), V(FAKE), V(FAKE), V(FAKE), 3, 1, 4, 16, 10, 2, 0, 0, V(0)) == B.PA_ERR_UNSUPPORTED
    assert r(V(0), V(FAKE), V(FAKE), V(FAKE), V(FAKE), 3, 8, 128, 16, 10, 2, 0, 0, V(0)) == B.PA_ERR_INVALID
    c = lib.pa_copy_blocks
    assert c(V(FAKE), V(FAKE), V(FAKE), 0, 10, 4096, V(0), V(0)) == B.PA_OK
    assert c(V(FAKE), V(FAKE), V(FAKE), 1, 10, 4008, V(0), V(0)) == B.PA_ERR_INVALID   # not a multiple of 16
    for bad in ([[1, 2], [3, 2]], [[1, 2], [2, 3]], [[1, 10]], [[4, 4]], [[-1, 2]]):
        hp = np.asarray(bad, np.int32)
        assert c(V(FAKE), V(FAKE), V(FAKE), len(hp), 10, 4096, V(hp.ctypes.data), V(0)) == B.PA_ERR_INVALID, bad


def test_missing_library_fails_loudly(tmp_path):
    with pytest.raises(ImportError):
        B.load_library(str(tmp_path / "libpa.so"))


def multi_call(lib, **kw):
    a = dict(out=FAKE, q=FAKE, k=FAKE, v=FAKE, bt=FAKE, sl=FAKE, N=4, T=4, Hq=8, Hkv=2, D=128, bs=16, scale=0.1,
             MB=8, NB=64, qd=2, kd=2, od=0, P=0, ws=FAKE, wsb=0, stream=0)
    a.update(kw)
    V = ctypes.c_void_p
    return lib.pa_decode_multi(V(a["out"]), V(a["q"]), V(a["k"]), V(a["v"]), V(a["bt"]), V(a["sl"]), a["N"],
                               a["T"], a["Hq"], a["Hkv"], a["D"], a["bs"], ctypes.c_float(a["scale"]), a["MB"],
                               a["NB"], a["qd"], a["kd"], a["od"], a["P"], V(a["ws"]), a["wsb"], V(a["stream"]))


def test_multi_argument_validation(lib):
    assert multi_call(lib, N=0) == B.PA_OK
    assert multi_call(lib, T=0) == B.PA_ERR_INVALID
    assert multi_call(lib, T=9) == B.PA_ERR_WORKSPACE              # 36 rows: two column groups of tokens
    assert multi_call(lib, T=100000) == B.PA_ERR_UNSUPPORTED       # more than 65536 query tokens
    assert multi_call(lib, D=64) == B.PA_ERR_WORKSPACE             # head_dim 64: groups of 8 rows
    assert multi_call(lib, qd=0) == B.PA_ERR_UNSUPPORTED           # several tokens need q_dtype == kv_dtype
    assert multi_call(lib, kd=3) == B.PA_ERR_UNSUPPORTED           # FP8 cache
    assert multi_call(lib, T=2, qd=0) == B.PA_ERR_UNSUPPORTED      # several tokens: q_dtype == kv_dtype
    assert multi_call(lib, T=1, qd=0) == B.PA_ERR_WORKSPACE        # one token: pa_decode's dtype pairs
    assert multi_call(lib, T=2, D=64) == B.PA_ERR_WORKSPACE        # 8 rows: head_dim 64 too
    # the workspace is pa_decode's for T * Hq heads
    need = B.pa_decode_workspace_size(4, 4 * 8, 128, 8 * 16)
    assert need > B.pa_decode_workspace_size(4, 8, 128, 8 * 16)
    assert multi_call(lib, wsb=need // 2) == B.PA_ERR_WORKSPACE
    assert multi_call(lib, ws=FAKE + 16, wsb=need) == B.PA_ERR_INVALID  # passes the size check, not 256-aligned


def prefix_call(lib, **kw):
    a = dict(out=FAKE, q=FAKE, k=FAKE, v=FAKE, bt=FAKE, sl=FAKE, N=4, Hq=16, Hkv=2, D=128, bs=16, scale=0.1,
             MB=8, NB=64, qd=2, kd=2, od=0, P=0, groups=FAKE, ng=1, mm=4, ws=FAKE, wsb=0, stream=0)
    a.update(kw)
    V = ctypes.c_void_p
    return lib.pa_decode_prefix(V(a["out"]), V(a["q"]), V(a["k"]), V(a["v"]), V(a["bt"]), V(a["sl"]), a["N"],
                                a["Hq"], a["Hkv"], a["D"], a["bs"], ctypes.c_float(a["scale"]), a["MB"], a["NB"],
                                a["qd"], a["kd"], a["od"], a["P"], V(a["groups"]), a["ng"], a["mm"], V(a["ws"]),
                                a["wsb"], V(a["stream"]))


def test_prefix_argument_validation(lib):
    assert prefix_call(lib, N=0) == B.PA_OK
    assert prefix_call(lib, ng=-1) == B.PA_ERR_INVALID
    assert prefix_call(lib, mm=0) == B.PA_ERR_INVALID
    assert prefix_call(lib, groups=0) == B.PA_ERR_INVALID          # groups promised, none given
    assert prefix_call(lib, ng=5) == B.PA_ERR_INVALID              # more groups than sequences
    # 5 members x 8 heads = 40 rows: beyond the warp-MMA kernel's 32, within the tensor-core
    # kernel's 64 (which the default option takes for it); 9 members: beyond both
    assert prefix_call(lib, mm=5) == B.PA_ERR_WORKSPACE
    assert prefix_call(lib, mm=9) == B.PA_ERR_UNSUPPORTED
    B.set_wide_kernel("mma")
    try:
        assert prefix_call(lib, mm=5) == B.PA_ERR_UNSUPPORTED
    finally:
        B.set_wide_kernel("auto")
    assert prefix_call(lib, kd=3) == B.PA_ERR_UNSUPPORTED           # FP8 cache
    assert prefix_call(lib, qd=0) == B.PA_ERR_UNSUPPORTED           # 32 rows need q_dtype == kv_dtype
    assert prefix_call(lib, Hq=512, Hkv=256) == B.PA_ERR_UNSUPPORTED  # more than 255 KV heads
    assert prefix_call(lib, mm=1, qd=0) == B.PA_ERR_WORKSPACE       # 8 rows: any dtype pair
    assert prefix_call(lib, ng=0, mm=99, qd=0) == B.PA_ERR_WORKSPACE  # no groups: max_members unused
    need = B.pa_decode_workspace_size(4, 16, 128, 8 * 16)
    assert prefix_call(lib, wsb=need - 1) == B.PA_ERR_WORKSPACE       # prefix calls need the full bound
    assert prefix_call(lib, ws=FAKE + 16, wsb=need) == B.PA_ERR_INVALID
    assert B.max_prefix_members(64, 8) == 4 and B.max_prefix_members(32, 8) == 8 and B.max_prefix_members(8, 8) == 32


def test_selftest_argument_checks(lib):
    assert lib.pa_selftest_wait_timeout(0, ctypes.c_void_p(0)) == B.PA_ERR_INVALID
    assert lib.pa_selftest_wait_timeout((1 << 20) + 1, ctypes.c_void_p(0)) == B.PA_ERR_INVALID


def test_set_option(lib):
    """The wide-kernel option takes its three values, the item-split option its two, and both
    reject others (no GPU needed)."""
    assert lib.pa_set_option(B.PA_OPT_WIDE_KERNEL, 1) == B.PA_OK
    assert lib.pa_set_option(B.PA_OPT_WIDE_KERNEL, 0) == B.PA_OK
    assert lib.pa_set_option(B.PA_OPT_WIDE_KERNEL, 2) == B.PA_OK
    assert lib.pa_set_option(B.PA_OPT_WIDE_KERNEL, 3) == B.PA_ERR_INVALID
    assert lib.pa_set_option(B.PA_OPT_WIDE_KERNEL, -1) == B.PA_ERR_INVALID
    assert lib.pa_set_option(0, 0) == B.PA_ERR_INVALID
    with pytest.raises(ValueError):
        B.set_wide_kernel("wgmma")
    B.set_wide_kernel("tcgen05")
    B.set_wide_kernel("mma")
    B.set_wide_kernel("auto")
    assert lib.pa_set_option(B.PA_OPT_ITEM_SPLIT, 1) == B.PA_OK
    assert lib.pa_set_option(B.PA_OPT_ITEM_SPLIT, 0) == B.PA_OK
    assert lib.pa_set_option(B.PA_OPT_ITEM_SPLIT, 2) == B.PA_ERR_INVALID
    assert lib.pa_set_option(B.PA_OPT_ITEM_SPLIT, -1) == B.PA_ERR_INVALID
    assert lib.pa_set_option(3, 0) == B.PA_ERR_INVALID
    with pytest.raises(ValueError):
        B.set_item_split("longest")
    B.set_item_split("fixed")
    B.set_item_split("adaptive")


def test_workspace_reserves_every_work_item(lib):
    """Every multi-token shape that the library accepts fits its work list in the workspace that
    pa_decode_workspace_size() advertises.  The library refuses (PA_ERR_WORKSPACE) a call whose
    plan could write more work items than the layout reserved, so a call that passes every host
    check reaches the device lookup, which fails here without a GPU (PA_ERR_CUDA).  The grid
    includes the shapes whose column groups hold only 5 to 8 query rows (head_dim 64, few KV
    heads), the worst case for the reservation."""
    checked = 0
    for wide in ("mma", "tcgen05", "auto"):  # the tensor-core kernel's items hold up to 64 rows
        B.set_wide_kernel(wide)
        try:
            checked += _reservation_grid(lib)
        finally:
            B.set_wide_kernel("auto")
    assert checked == 3 * 6192


def _reservation_grid(lib):
    checked = 0
    for D in (64, 128):
        for Hkv in (1, 2, 3):
            for G in range(1, 9):
                for T in list(range(1, 41)) + [64, 100, 1000]:
                    for N, MB in ((1, 1), (3, 8), (64, 130)):
                        need = B.pa_decode_workspace_size(N, T * G * Hkv, D, MB * 16)
                        rc = multi_call(lib, N=N, T=T, Hq=G * Hkv, Hkv=Hkv, D=D, MB=MB, NB=64, qd=2, kd=2,
                                        ws=0x100000, wsb=need)
                        assert rc == B.PA_ERR_CUDA, (D, Hkv, G, T, N, MB, rc)
                        checked += 1
    return checked
