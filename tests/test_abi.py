"""C-ABI checks that need no GPU: the library loads, exports what include/mr.h declares, sizes its
workspaces, and rejects invalid calls on the host before any launch."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "mr.h")


@pytest.fixture(scope="module")
def mr():
    from cross_model_attention_mr_b200 import mr as m
    return m


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(mr_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for want in ("mr_compress", "mr_retrieve", "mr_dense_ref", "mr_sync_status", "mr_bsr_export",
                 "mr_status_string", "mr_compress_workspace_bytes", "mr_retrieve_workspace_bytes"):
        assert want in names


def test_library_exports_every_declared_symbol(mr):
    lib = ctypes.CDLL(mr.LIB_PATH)
    missing = [n for n in declared_functions() if not hasattr(lib, n)]
    assert not missing, missing
    # the binding declares a prototype for each of them
    assert set(declared_functions()) <= set(mr.EXPORTS)


def test_checked_build_exports_the_same_symbols(mr):
    """libmr_checked.so (compiled with -DMR_CHECKED) is a drop-in twin of libmr.so."""
    path = os.path.join(os.path.dirname(mr.LIB_PATH), "libmr_checked.so")
    assert os.path.exists(path), "build it with __graft_entry__.build()"
    lib = ctypes.CDLL(path)
    missing = [n for n in declared_functions() if not hasattr(lib, n)]
    assert not missing, missing
    lib.mr_checked_build.restype = ctypes.c_int
    assert lib.mr_checked_build() == 1


def test_library_variant_matches_environment(mr):
    """MR_LIBRARY=checked loads the bounds-checked build; anything else the normal one."""
    assert mr.LIB.mr_checked_build() == (1 if os.environ.get("MR_LIBRARY") == "checked" else 0)


def test_bench_traffic_is_tied_to_its_workload_and_sources():
    """The bench line's DRAM traffic comes from the committed capture only for the workload it was
    scaled to, and only while the kernel sources it was taken on are unchanged."""
    import json
    import sys
    sys.path.insert(0, ROOT)
    import bench
    d = json.load(open(os.path.join(ROOT, "profiles", "traffic.json")))
    wl = d["workload"]
    for kernel in ("mr_compress_tc", "mr_emit_tc", "mr_retrieve_tc"):
        ent = d[kernel]
        fresh = bench.source_hash(ent["sources"]) == ent["source_hash"]
        got = bench.traffic_for(kernel, wl)
        assert (got == ent["bytes_per_launch"]) if fresh else got is None
        assert bench.traffic_for(kernel, wl + "+fp8") is None
        assert bench.traffic_for(kernel, "L8192_32to64_d128_bf16_B128") is None


def test_bench_work_of_the_config_lines():
    """The --config lines average the per-layer algorithmic work and keep its labels (which
    head-mixing path the retrieval takes) as they are."""
    import importlib.util
    spec = importlib.util.spec_from_file_location("bench", os.path.join(ROOT, "bench.py"))
    bench = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(bench)
    from cross_model_attention_mr_b200.workloads import config
    c2, c4 = config(2), config(4)
    assert bench.algorithmic(c2, 100, 50)["mix_path"] == "cuda_core"       # 64-key blocks
    assert bench.algorithmic(c4, 100, 50)["mix_path"] == "tensor"          # bf16, 128-key blocks, 32 heads
    assert bench.algorithmic(c4, 100, 50, fp8=True)["mix_path"] == "cuda_core"
    assert bench.algorithmic(c4, 100, 50, n_req=4)["mix_path"] == "cuda_core"
    layers = [bench.algorithmic(c2, nnz, un) for nnz, un in ((100, 50), (300, 70))]
    m = bench.mean_work(layers)
    assert m["mix_path"] == "cuda_core"
    assert m["map_bytes"] == (layers[0]["map_bytes"] + layers[1]["map_bytes"]) / 2
    assert m["compress_flops"] == layers[0]["compress_flops"]


def test_status_strings(mr):
    for code in range(8):
        s = mr.LIB.mr_status_string(code)
        assert isinstance(s, bytes) and len(s) > 0
    assert mr.LIB.mr_version() >= 100


def test_workspace_sizes(mr):
    assert mr.compress_workspace_bytes(32, 32768, 128, 128) > 32 * 32768 * 4
    assert mr.compress_workspace_bytes(32, 32768, 96, 128) == 0       # unsupported head dim
    assert mr.compress_workspace_bytes(32, 1000, 128, 64) == 0        # L not a multiple of the block
    assert mr.compress_workspace_bytes(32, 64 * 257, 128, 64) == 0    # more than 256 key blocks
    assert mr.max_tiles(32, 32768, 128) == 32 * 256 * 257 // 2
    assert mr.max_tiles(4, 512, 64) == 4 * 8 * 9 // 2


def _bsr(mr, H=4, L=512, B=64, dt=0, cap=100, fake=0x1000):
    return mr.BSR(H, L, B, dt, cap, fake, fake, fake, fake, fake, None, None, fake)


def test_compress_rejects_bad_arguments_without_launching(mr):
    lib = mr.LIB
    fake = 0x1000  # never dereferenced: every call below must fail validation first
    ws_bytes = mr.compress_workspace_bytes(4, 512, 64, 64)
    b = _bsr(mr)
    call = lambda **kw: lib.mr_compress(kw.get("Q", fake), kw.get("K", fake), kw.get("dt", 0), kw.get("H", 4),
                                        kw.get("L", 512), kw.get("d", 64), kw.get("scale", 0.125),
                                        kw.get("p", 0.9), None, ctypes.byref(kw.get("b", b)), kw.get("ws", fake),
                                        kw.get("wsb", ws_bytes), None)
    assert call(Q=None) == mr.MR_ERR_INVALID_ARG
    assert call(ws=None) == mr.MR_ERR_INVALID_ARG
    assert call(dt=7) == mr.MR_ERR_INVALID_ARG
    assert call(p=0.0) == mr.MR_ERR_INVALID_ARG
    assert call(p=float("nan")) == mr.MR_ERR_INVALID_ARG
    assert call(scale=float("inf")) == mr.MR_ERR_INVALID_ARG
    assert call(d=96) == mr.MR_ERR_UNSUPPORTED
    assert call(H=65, b=_bsr(mr, H=65)) == mr.MR_ERR_UNSUPPORTED
    assert call(b=_bsr(mr, B=32)) == mr.MR_ERR_UNSUPPORTED
    assert call(b=_bsr(mr, H=3)) == mr.MR_ERR_INVALID_ARG           # descriptor disagrees with H
    assert call(b=_bsr(mr, dt=1)) == mr.MR_ERR_UNSUPPORTED          # vals dtype differs from inputs
    assert call(b=_bsr(mr, cap=-1)) == mr.MR_ERR_INVALID_ARG
    assert call(wsb=16) == mr.MR_ERR_INVALID_ARG
    bad_bias = mr.LogitBias(0, 0.0, 0, 0.0, fake, 0, 8)             # kb table without a block size
    assert lib.mr_compress(fake, fake, 0, 4, 512, 64, 0.125, 0.9, ctypes.byref(bad_bias), ctypes.byref(b),
                           fake, ws_bytes, None) == mr.MR_ERR_INVALID_ARG
    # query-block range of mr_compress_blocks: 0 <= begin < end <= L / block (= 8 here)
    blk = lambda q0, q1: lib.mr_compress_blocks(fake, fake, 0, 4, 512, 64, 0.125, 0.9, None, q0, q1,
                                                ctypes.byref(b), fake, ws_bytes, None)
    for q0, q1 in ((0, 0), (4, 4), (5, 3), (-1, 2), (0, 9)):
        assert blk(q0, q1) == mr.MR_ERR_INVALID_ARG


def test_retrieve_and_dense_reject_bad_arguments(mr):
    lib = mr.LIB
    fake = 0x1000
    b = _bsr(mr)
    full = 5 * 512 * 64  # elements of [5][512][64] values

    def r(**kw):
        o = kw.get("opts")
        return lib.mr_retrieve(ctypes.byref(kw.get("b", b)), kw.get("W", fake), kw.get("H_r", 5), fake,
                               kw.get("ve", full), fake, kw.get("dt", 0), kw.get("dv", 64), kw.get("n", 1), None,
                               kw.get("rs", 0), kw.get("hs", 512 * 64), ctypes.byref(o) if o else None, fake,
                               kw.get("wsb", 4096 + 256), None)
    assert r(W=None) == mr.MR_ERR_INVALID_ARG
    assert r(dv=80) == mr.MR_ERR_UNSUPPORTED
    assert r(H_r=0) == mr.MR_ERR_INVALID_ARG
    assert r(n=0) == mr.MR_ERR_INVALID_ARG
    assert r(hs=10) == mr.MR_ERR_INVALID_ARG
    assert r(dt=1) == mr.MR_ERR_UNSUPPORTED
    # the values must fit inside the stated allocation: heads x rows, and every request
    assert r(ve=0) == mr.MR_ERR_INVALID_ARG
    assert r(ve=full - 1) == mr.MR_ERR_INVALID_ARG
    assert r(n=2, rs=full, ve=2 * full - 64) == mr.MR_ERR_INVALID_ARG
    # options: query-block range inside the map, value groups dividing the receiver heads
    assert r(opts=mr.RetrieveOpts(3, 3, 1)) == mr.MR_ERR_INVALID_ARG
    assert r(opts=mr.RetrieveOpts(0, 9, 1)) == mr.MR_ERR_INVALID_ARG      # 512 / 64 = 8 query blocks
    assert r(opts=mr.RetrieveOpts(-1, 4, 1)) == mr.MR_ERR_INVALID_ARG
    assert r(opts=mr.RetrieveOpts(0, 0, 2)) == mr.MR_ERR_INVALID_ARG      # 5 heads, groups of 2
    assert r(opts=mr.RetrieveOpts(0, 0, -1)) == mr.MR_ERR_INVALID_ARG
    # paged values: pages of a positive multiple of 64 rows that cover the map's L = 512 rows
    assert r(opts=mr.RetrieveOpts(0, 0, 1, fake, 32, 16)) == mr.MR_ERR_INVALID_ARG
    assert r(opts=mr.RetrieveOpts(0, 0, 1, fake, 64, 7)) == mr.MR_ERR_INVALID_ARG      # 448 < 512 rows
    assert r(opts=mr.RetrieveOpts(0, 0, 1, fake, 128, 0)) == mr.MR_ERR_INVALID_ARG
    assert r(ve=64 * 64 * 5 - 1, opts=mr.RetrieveOpts(0, 0, 1, fake, 64, 8)) == mr.MR_ERR_INVALID_ARG  # no page fits
    # the workspace holds the status header and one progress counter per CTA (up to 1024)
    need = lib.mr_retrieve_workspace_bytes(ctypes.byref(b), 5, 64, 1)
    assert need == 256 + 1024 * 4
    assert r(wsb=need - 1) == mr.MR_ERR_INVALID_ARG  # rejected before anything is launched
    assert r(wsb=256) == mr.MR_ERR_INVALID_ARG
    d = lambda **kw: lib.mr_dense_ref(fake, fake, fake, fake, kw.get("dt", 0), 4, kw.get("d", 64), 64,
                                      kw.get("cu", fake), fake, None, 2, 100, 100, 0.125, None, fake, 4096, None)
    assert d(cu=None) == mr.MR_ERR_INVALID_ARG
    assert d(d=32) == mr.MR_ERR_UNSUPPORTED
    assert d(dt=3) == mr.MR_ERR_INVALID_ARG


def test_debug_hook_validates_and_resets(mr):
    lib = mr.LIB
    assert lib.mr_debug_set(0, 2) == mr.MR_ERR_INVALID_ARG
    assert lib.mr_debug_set(1000, 1) == mr.MR_OK
    assert lib.mr_debug_set(0, 0) == mr.MR_OK
