"""The C ABI on a host without a GPU: the library loads, exports every entry point
that include/twell.h declares, and its host-only checks answer as documented.
None of these calls reaches the GPU (they return before any CUDA call)."""

import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "twell.h")


@pytest.fixture(scope="module")
def tw():
    from activation_sparse_ffn_gemm_b200 import build

    build.build()
    import activation_sparse_ffn_gemm_b200 as tw

    return tw


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(twell_[a-z_0-9]+)\s*\(", text)))


def test_header_declares_the_entry_points():
    names = declared_functions()
    for n in ("twell_pack", "twell_ffn_fwd", "twell_ffn_bwd", "twell_workspace_bytes", "twell_status_read"):
        assert n in names


def test_library_exports_every_declared_symbol(tw):
    L = tw.lib()
    for name in declared_functions():
        assert hasattr(L, name), f"{name} is declared in twell.h but not exported"
    # nothing else is exported with the twell_ prefix besides the declared API
    out = os.popen(f"nm -D --defined-only {tw.LIB_PATH}").read()
    exported = set(re.findall(r"\bT (twell_[a-z_0-9]+)\b", out))
    assert exported == set(declared_functions())


def test_hybrid_struct_matches_header(tw, tmp_path):
    # six int32 fields, eleven pointers
    assert ctypes.sizeof(tw.TwellHybrid) == 24 + 11 * 8
    assert tw.TwellHybrid.dense_min.offset == 20
    assert tw.TwellHybrid.count.offset == 24
    assert tw.TwellHybrid.row_plan.offset == 24 + 10 * 8
    # the header's own layout, as a C compiler sees it
    src = tmp_path / "layout.c"
    src.write_text('#include <stdio.h>\n#include <stddef.h>\n#include "twell.h"\n'
                   'int main(void) { printf("%zu", sizeof(twell_hybrid)); '
                   'printf(" %zu %zu %zu %zu\\n", offsetof(twell_hybrid, ovf_cap), offsetof(twell_hybrid, dense_min), '
                   'offsetof(twell_hybrid, count), offsetof(twell_hybrid, row_plan)); return 0; }\n')
    exe = tmp_path / "layout"
    rc = os.system(f"gcc -std=c11 -I{os.path.join(ROOT, 'include')} -o {exe} {src}")
    assert rc == 0
    got = [int(v) for v in os.popen(str(exe)).read().split()]
    fields = dict(tw.TwellHybrid._fields_)
    assert got == [ctypes.sizeof(tw.TwellHybrid), tw.TwellHybrid.ovf_cap.offset, tw.TwellHybrid.dense_min.offset,
                   tw.TwellHybrid.count.offset, tw.TwellHybrid.row_plan.offset]
    assert "dense_min" in fields


def test_plan_ints(tw):
    L = tw.lib()
    # 4 + 2 M + 2 * (M + max(65536, ceil(M * T * K / 256))), rounded up to 4 ints,
    # then the routing scratch: 512 blocks x (4 int64 + 2 int32)
    def expect(core):
        return (core + 3) // 4 * 4 + 512 * 10
    assert L.twell_plan_ints(4096, 8192, 128, 8) == expect(4 + 2 * 4096 + 2 * (4096 + 65536))
    big = 65536 * 112 * 64 // 256
    assert L.twell_plan_ints(65536, 14336, 128, 64) == expect(4 + 2 * 65536 + 2 * (65536 + big))
    assert L.twell_plan_ints(0, 8192, 128, 8) == expect(4 + 2 * 65536)
    assert L.twell_plan_ints(1, 8192, 128, 8) == expect(4 + 2 + 2 * (1 + 65536))
    assert L.twell_plan_ints(16, 8192, 64, 8) == 0


def test_query_support(tw):
    ok = tw.query_support
    assert ok(4096, 2048, 8192, 128, 8, 4096) == 0
    assert ok(0, 2048, 8192, 128, 8, 0) == 0
    assert ok(16384, 4096, 14336, 128, 64, 100) == 0
    assert ok(4096, 2048, 8192, 64, 8, 0) == 2      # T_n must be 128
    assert ok(4096, 2048, 8192, 128, 12, 0) == 2    # K not in {8,16,32,64}
    assert ok(4096, 2000, 8192, 128, 8, 0) == 2     # d_model % 64
    assert ok(4096, 2048, 8000, 128, 8, 0) == 2     # d_ff % 128
    assert ok(4096, 2048, 32768, 128, 8, 0) == 2    # d_ff too wide
    assert ok(10, 2048, 8192, 128, 8, 11) == 2      # ovf_cap > M
    assert ok(-1, 2048, 8192, 128, 8, 0) == 1
    assert tw.lib().twell_status_string(6).decode().startswith("workspace")


def test_workspace_sizes(tw):
    M, d, f, K = 4096, 2048, 8192, 8
    pack = tw.workspace_bytes(tw.OP_PACK, M, d, f, 128, K, M)
    fwd = tw.workspace_bytes(tw.OP_FWD, M, d, f, 128, K, M)
    bwd = tw.workspace_bytes(tw.OP_BWD, M, d, f, 128, K, M)
    assert pack >= M * f * 2 and fwd > pack and bwd > f * d * 2
    assert tw.workspace_bytes(tw.OP_FWD, M, d, f, 64, K, M) == 0
    assert tw.workspace_bytes(7, M, d, f, 128, K, M) == 0


def test_host_side_errors(tw):
    L = tw.lib()
    h = tw.TwellHybrid(64, 1024, 128, 8, 64, 0, *([None] * 11))
    # null descriptor, null arrays, unsupported shape, missing workspace
    assert L.twell_pack(None, None, None, 256, None, None, None, 0, None) == 1
    assert L.twell_pack(None, None, None, 256, ctypes.byref(h), None, None, 0, None) == 1
    bad = tw.TwellHybrid(64, 1024, 64, 8, 64, 0, *([None] * 11))
    assert L.twell_pack(None, None, None, 256, ctypes.byref(bad), None, None, 0, None) == 2
    fake = 1 << 20  # aligned non-null addresses; never dereferenced by these checks
    h2 = tw.TwellHybrid(64, 1024, 128, 8, 64, 0, *([fake] * 11))
    p = ctypes.c_void_p(fake)
    assert L.twell_pack(p, p, p, 256, ctypes.byref(h2), None, None, 0, None) == 6
    assert L.twell_pack(p, p, p, 256, ctypes.byref(h2), None, ctypes.c_void_p(fake + 8), 1 << 30, None) == 6
    mis = ctypes.c_void_p(fake + 2)
    assert L.twell_ffn_fwd(mis, p, p, p, p, None, 256, p, ctypes.byref(h2), None, None, 0, None) == 1
    # empty batch forward: nothing to do, nothing touched
    h0 = tw.TwellHybrid(0, 1024, 128, 8, 0, 0, *([None] * 11))
    assert L.twell_ffn_fwd(None, None, None, None, None, None, 256, None, ctypes.byref(h0), None, None, 0, None) == 0
    assert L.twell_transpose_wd(None, 256, 1024, None, None) == 1
    # a negative row threshold is refused before anything is enqueued
    hn = tw.TwellHybrid(64, 1024, 128, 8, 64, -1, *([fake] * 11))
    assert L.twell_pack(p, p, p, 256, ctypes.byref(hn), None, p, 1 << 30, None) == 1
    assert L.twell_pack_noalloc(p, p, p, 256, ctypes.byref(hn), None, None) == 1
    # count statistics: null or misaligned outputs, bad threshold, unsupported shape
    assert L.twell_count_stats(ctypes.byref(h2), None, p, p, None) == 1
    assert L.twell_count_stats(ctypes.byref(h2), p, ctypes.c_void_p(fake + 4), p, None) == 1
    assert L.twell_count_stats(ctypes.byref(hn), p, p, p, None) == 1
    assert L.twell_count_stats(ctypes.byref(bad), p, p, p, None) == 2
    assert L.twell_count_stats(None, p, p, p, None) == 1
    # the sparse-kernel schedule: unknown modes and negative budgets are refused;
    # the default is put back
    assert L.twell_set_sparse_schedule(3, 0) == 1
    assert L.twell_set_sparse_schedule(-1, 0) == 1
    assert L.twell_set_sparse_schedule(tw.SCHED_PASSES, -5) == 1
    assert L.twell_set_sparse_schedule(tw.SCHED_FUSED, 1 << 20) == 0
    assert L.twell_set_sparse_schedule(tw.SCHED_AUTO, 0) == 0
    assert L.twell_set_overlap(3) == 1 and L.twell_set_overlap(-1) == 1
    assert L.twell_set_overlap(tw.OVERLAP_OFF) == 0 and L.twell_set_overlap(tw.OVERLAP_AUTO) == 0


def test_missing_library_fails_loudly(tw, monkeypatch):
    monkeypatch.setattr(tw, "_libs", {})
    monkeypatch.setattr(tw, "LIB_PATH", os.path.join(ROOT, "does_not_exist", "libtwell.so"))
    with pytest.raises(RuntimeError, match="missing"):
        tw.lib()


def test_bounds_checked_library_exports_the_same_symbols(tw):
    """libtwell_bounds.so (the -DTWELL_BOUNDS build) exports exactly the header's
    entry points too, and bounds_checked() routes the binding to it."""
    out = os.popen(f"nm -D --defined-only {tw.BOUNDS_LIB_PATH}").read()
    assert set(re.findall(r"\bT (twell_[a-z_0-9]+)\b", out)) == set(declared_functions())
    plain = tw.lib()
    with tw.bounds_checked() as L:
        assert L is not plain and tw.lib() is L
        assert tw.query_support(64, 256, 1024, 128, 8, 64) == 0
    assert tw.lib() is plain
    assert tw.STATUS_BOUNDS == 1 << 7


def test_pair_list_bound(tw):
    """The weight gradients' pair list has 32-bit positions: a backward whose list
    could pass 2^31 - 1 entries is refused before anything is enqueued, and its
    workspace size is reported as 0 (the forward is unaffected)."""
    L = tw.lib()
    M, d, f, K = 1 << 18, 2048, 14336, 8
    assert (M - M) * (f // 128) * K + M * f > 2 ** 31 - 1
    assert tw.workspace_bytes(tw.OP_BWD, M, d, f, 128, K, M) == 0
    assert tw.workspace_bytes(tw.OP_FWD, M, d, f, 128, K, M) > 0
    assert tw.workspace_bytes(tw.OP_BWD, M, d, f, 128, K, 0) > 0  # 2^18 * 112 * 8 entries fit
    assert tw.workspace_bytes(tw.OP_BWD, 65536, 4096, 14336, 128, 8, 65536) > 0  # the sweep's largest
    fake = 1 << 20
    p = ctypes.c_void_p(fake)
    h = tw.TwellHybrid(M, f, 128, K, M, 0, *([fake] * 11))
    assert L.twell_ffn_bwd(p, p, p, p, None, d, ctypes.byref(h), p, ctypes.c_float(0.0), p, p, p, p, None, p,
                           1 << 40, None) == 2
