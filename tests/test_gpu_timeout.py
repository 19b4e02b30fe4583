"""A bounded device wait that runs out, on the GPU, without any fault.

The test hook mr_debug_set shortens the tensor-core dense kernel's protocol waits to 1 ms and makes
its softmax warpgroup withhold the arrive that tells the MMA warp the first P tile is ready.  The
MMA warp's wait then runs out: the call must record MR_ERR_TIMEOUT with that wait's code in the
workspace, drain, free Tensor Memory and return, and the next call on the same workspace must run
cleanly and give the right result.
"""
import numpy as np
import pytest
import torch

from cross_model_attention_mr_b200.workloads import round_to_bf16

from parity import OUT_TOL, dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def mr():
    from cross_model_attention_mr_b200 import mr as m
    assert torch.cuda.is_available()
    return m


def test_dense_wait_runs_out_then_next_call_is_clean(mr):
    import oracle
    H, d, lq, lk = 1, 128, 64, 256          # one 64-row query tile over two 128-key tiles: one CTA
    rng = np.random.default_rng(3)
    Q = round_to_bf16(rng.standard_normal((H, lq, d), dtype=np.float32) * np.float32(0.35))
    K = round_to_bf16(rng.standard_normal((H, lk, d), dtype=np.float32) * np.float32(0.35))
    V = round_to_bf16(rng.standard_normal((H, lk, d), dtype=np.float32))
    cu_q = torch.tensor([0, lq], dtype=torch.int32, device="cuda")
    cu_k = torch.tensor([0, lk], dtype=torch.int32, device="cuda")
    off = torch.tensor([lk - lq], dtype=torch.int32, device="cuda")
    ws = mr.Workspace(int(mr.LIB.mr_dense_ref_workspace_bytes(1)))
    args = (dev(Q, "bf16"), dev(K, "bf16"), dev(V, "bf16"), cu_q, cu_k, off, lq, lk)
    assert mr.LIB.mr_debug_set(1_000_000, 1) == mr.MR_OK
    try:
        mr.dense_ref(*args, ws=ws)
        st = ws.sync_status()
        hdr = torch.empty(2, dtype=torch.int32)
        hdr.copy_(ws.buf[(ws.ptr - ws.buf.data_ptr()):(ws.ptr - ws.buf.data_ptr()) + 8].view(torch.int32))
    finally:
        assert mr.LIB.mr_debug_set(0, 0) == mr.MR_OK
    assert st == mr.MR_ERR_TIMEOUT
    assert int(hdr[1]) == 0x913               # the MMA warp's wait for the first P tile
    # the context is usable and the next call on the same workspace is clean and right
    O = mr.dense_ref(*args, ws=ws)
    assert ws.sync_status() == mr.MR_OK
    want = oracle.dense_rows(Q, K, V, 1.0 / np.sqrt(d), np.arange(lq), lk - lq, None)
    assert np.max(np.abs(O.float().cpu().numpy() - want)) <= OUT_TOL["bf16"] * float(np.abs(V).max())
