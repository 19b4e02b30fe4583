"""mr_compress_noalloc: the allocation-free compression entry point, checked against mr_compress.

Callers that cannot allocate device memory (code inside a framework whose pool already owns the
GPU, plug-ins with a fixed memory budget, serving loops that must not call the allocator) cannot
give mr_compress a workspace; mr_compress_noalloc takes its scratch from a fixed array inside
libmr instead.  These tests call it through the C-ABI and require the same map as mr_compress on
the same inputs, for two calls in a row (the array is shared and keeps the previous call's
contents), within the tolerances the other parity tests use.

This file sorts last so that a run stopping at the first failure has already run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

from cross_model_attention_mr_b200.workloads import config, draw_layers, shrink

from parity import MASS_ATOL, VAL_TOL, dev, p32

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def mr():
    from cross_model_attention_mr_b200 import mr as m
    assert torch.cuda.is_available()
    return m


def _noalloc(mr, Q, K, spec, bias, out):
    return mr.LIB.mr_compress_noalloc(Q.data_ptr(), K.data_ptr(), mr._dt(Q), spec.H_s, spec.L, spec.d,
                                      float(spec.scale), p32(spec.p), mr._bias_ptr(bias), ctypes.byref(out.c),
                                      torch.cuda.current_stream().cuda_stream)


def _same_map(mr, spec, a, b):
    torch.cuda.synchronize()
    n = a.nnz_host()
    assert b.nnz_host() == n
    assert torch.equal(a.row_ptr.cpu(), b.row_ptr.cpu())
    assert torch.equal(a.kept_bits.cpu(), b.kept_bits.cpu())
    assert torch.equal(a.col_idx[:n].cpu(), b.col_idx[:n].cpu())
    assert float((a.kept_mass - b.kept_mass).abs().max()) <= MASS_ATOL
    va, vb = a.export().double(), b.export().double()
    rtol, atol = VAL_TOL[spec.dtype]
    assert bool(((va - vb).abs() <= rtol * vb.abs() + atol).all())


def test_noalloc_matches_workspace_entry_point_twice_in_a_row(mr):
    specs = [shrink(config(2), L=1024, H_s=8, H_r=4), shrink(config(4), L=2048, H_s=4, H_r=4)]
    for spec in specs + specs[:1]:          # two different shapes, then the first again
        lay = draw_layers(spec)[0]
        Q, K = dev(lay.Q, spec.dtype), dev(lay.K, spec.dtype)
        bias = mr.Bias.from_spec(lay.bias)
        ref = mr.compress(Q, K, p32(spec.p), spec.block, bias=bias, scale=spec.scale)
        assert ref.ws.sync_status() == mr.MR_OK
        cap = mr.max_tiles(spec.H_s, spec.L, spec.block)
        out = mr.Map(spec.H_s, spec.L, spec.block, mr._dt(Q), cap, "cuda")
        assert _noalloc(mr, Q, K, spec, bias, out) == mr.MR_OK
        assert mr.compress_noalloc_status() == mr.MR_OK   # the device-side status of that call
        _same_map(mr, spec, out, ref)
        # a second call into the same (already used) scratch gives the same map again
        out2 = mr.Map(spec.H_s, spec.L, spec.block, mr._dt(Q), cap, "cuda")
        assert _noalloc(mr, Q, K, spec, bias, out2) == mr.MR_OK
        assert mr.compress_noalloc_status() == mr.MR_OK
        _same_map(mr, spec, out2, ref)


def test_noalloc_fp32_workload(mr):
    spec = config(1)
    lay = draw_layers(spec)[0]
    Q, K = dev(lay.Q, "f32"), dev(lay.K, "f32")
    bias = mr.Bias.from_spec(lay.bias)
    ref = mr.compress(Q, K, p32(spec.p), spec.block, bias=bias, scale=spec.scale)
    out = mr.Map(spec.H_s, spec.L, spec.block, mr.MR_F32, mr.max_tiles(spec.H_s, spec.L, spec.block), "cuda")
    assert _noalloc(mr, Q, K, spec, bias, out) == mr.MR_OK
    assert mr.compress_noalloc_status() == mr.MR_OK
    _same_map(mr, spec, out, ref)


def test_noalloc_status_reports_capacity_overflow(mr):
    """The status word of the fixed scratch is readable: a map that outgrows its capacity reports
    MR_ERR_CAPACITY there, and the next call that fits reports MR_OK again."""
    spec = shrink(config(2), L=512, H_s=2, H_r=2)
    lay = draw_layers(spec)[0]
    Q, K = dev(lay.Q, spec.dtype), dev(lay.K, spec.dtype)
    bias = mr.Bias.from_spec(lay.bias)
    small = mr.Map(spec.H_s, spec.L, spec.block, mr.MR_BF16, 5, "cuda")
    assert _noalloc(mr, Q, K, spec, bias, small) == mr.MR_OK
    assert mr.compress_noalloc_status() == mr.MR_ERR_CAPACITY
    big = mr.Map(spec.H_s, spec.L, spec.block, mr.MR_BF16, mr.max_tiles(spec.H_s, spec.L, spec.block), "cuda")
    assert _noalloc(mr, Q, K, spec, bias, big) == mr.MR_OK
    assert mr.compress_noalloc_status() == mr.MR_OK


def test_noalloc_rejects_shapes_beyond_its_scratch(mr):
    # 64 heads x 32768 tokens needs 8 MiB of row normalisers, more than the fixed array holds
    spec = shrink(config(4), H_s=64)
    need = mr.compress_workspace_bytes(spec.H_s, spec.L, spec.d, spec.block)
    assert need > 256 + 4194304 + 65536
    fake = torch.empty(1, device="cuda")
    out = mr.BSR(spec.H_s, spec.L, spec.block, mr.MR_BF16, 1, fake.data_ptr(), fake.data_ptr(), fake.data_ptr(),
                 fake.data_ptr(), fake.data_ptr(), None, None, fake.data_ptr())
    st = mr.LIB.mr_compress_noalloc(fake.data_ptr(), fake.data_ptr(), mr.MR_BF16, spec.H_s, spec.L, spec.d,
                                    0.088, 0.9, None, ctypes.byref(out), None)
    assert st == mr.MR_ERR_UNSUPPORTED
    # the largest workload of the benchmark fits
    big = config(4)
    assert mr.compress_workspace_bytes(big.H_s, big.L, big.d, big.block) <= 256 + 4194304 + 65536
