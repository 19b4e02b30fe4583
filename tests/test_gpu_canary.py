"""NaN canaries around and inside the output buffers (MapFlow section 5.4 retrieval, section 5.2
compression, and the dense causal path): every call writes exactly the elements it owns.

Each output is a view into a larger buffer filled with a NaN bit pattern.  After the call the guard
regions before and after the view, the rows outside a query-block range, the map tiles past the
stored count and their column indices must still hold the pattern, bit for bit, while the written
part matches the oracle.
"""
import numpy as np
import pytest
import torch

from cross_model_attention_mr_b200.workloads import config, draw_layers, round_to_bf16, shrink

from parity import OUT_TOL, dev, p32

pytestmark = pytest.mark.gpu

NAN_BF16 = 0x7FC1        # a quiet NaN no kernel writes by accident
GUARD = 4096             # elements before and after each view


@pytest.fixture(scope="module")
def mr():
    from cross_model_attention_mr_b200 import mr as m
    assert torch.cuda.is_available()
    return m


def _canary(n: int) -> torch.Tensor:
    buf = torch.empty(n + 2 * GUARD, dtype=torch.int16, device="cuda")
    buf.fill_(NAN_BF16)
    return buf


def _untouched(x: torch.Tensor) -> bool:
    return bool(torch.all(x.view(torch.int16) == NAN_BF16).item())


def test_retrieve_writes_only_its_query_blocks(mr):
    import oracle
    spec = shrink(config(4), L=1024, H_s=4, H_r=6)
    lay = draw_layers(spec)[0]
    B, L, H_r, d_v = spec.block, spec.L, spec.H_r, spec.d_v
    m = mr.compress(dev(lay.Q, "bf16"), dev(lay.K, "bf16"), p32(spec.p), B, bias=mr.Bias.from_spec(lay.bias),
                    scale=spec.scale)
    assert m.ws.sync_status() == mr.MR_OK
    n = H_r * L * d_v
    buf = _canary(n)
    out = buf[GUARD:GUARD + n].view(torch.bfloat16).view(1, H_r, L, d_v)
    qb0, qb1 = 2, 5
    ws = mr.Workspace(mr.retrieve_workspace_bytes(m, H_r, d_v, 1))
    mr.retrieve(m, torch.from_numpy(lay.W).cuda(), dev(lay.V, "bf16"), out=out, ws=ws, blocks=(qb0, qb1))
    assert ws.sync_status() == mr.MR_OK
    assert _untouched(buf[:GUARD]) and _untouched(buf[GUARD + n:])
    r0, r1 = qb0 * B, qb1 * B
    assert _untouched(out[:, :, :r0]) and _untouched(out[:, :, r1:])
    assert bool(torch.isfinite(out[:, :, r0:r1].float()).all().item())
    rows = np.array([r0, r0 + 1, (r0 + r1) // 2, r1 - 1])
    want = oracle.retrieve_rows(lay.Q, lay.K, spec.scale, B, m.kept_bits_host(), lay.W, lay.V, rows, lay.bias)
    got = out[:, :, rows].float().cpu().numpy()
    assert np.max(np.abs(got - want)) <= OUT_TOL["bf16"] * float(np.abs(lay.V).max())


def test_dense_writes_exactly_the_packed_rows(mr):
    import oracle
    H, d = 2, 128
    lens_q, offs = [200, 77], [0, 300]                   # a ragged tile in each sequence
    lens_k = [lq + o for lq, o in zip(lens_q, offs)]
    rng = np.random.default_rng(11)
    tq, tk = sum(lens_q), sum(lens_k)
    Q = round_to_bf16(rng.standard_normal((H, tq, d), dtype=np.float32) * np.float32(0.3))
    K = round_to_bf16(rng.standard_normal((H, tk, d), dtype=np.float32) * np.float32(0.3))
    V = round_to_bf16(rng.standard_normal((H, tk, d), dtype=np.float32))
    cu_q = torch.tensor(np.concatenate([[0], np.cumsum(lens_q)]), dtype=torch.int32, device="cuda")
    cu_k = torch.tensor(np.concatenate([[0], np.cumsum(lens_k)]), dtype=torch.int32, device="cuda")
    off = torch.tensor(offs, dtype=torch.int32, device="cuda")
    n = H * tq * d
    buf = _canary(n)
    out = buf[GUARD:GUARD + n].view(torch.bfloat16).view(H, tq, d)
    ws = mr.Workspace(int(mr.LIB.mr_dense_ref_workspace_bytes(2)))
    mr.dense_ref(dev(Q, "bf16"), dev(K, "bf16"), dev(V, "bf16"), cu_q, cu_k, off, tq, tk, out=out, ws=ws)
    assert ws.sync_status() == mr.MR_OK
    assert _untouched(buf[:GUARD]) and _untouched(buf[GUARD + n:])
    assert bool(torch.isfinite(out.float()).all().item())
    scale = 1.0 / np.sqrt(d)
    for s in range(2):
        q0, k0 = int(cu_q[s]), int(cu_k[s])
        rows = np.array([0, lens_q[s] // 2, lens_q[s] - 1])
        want = oracle.dense_rows(Q[:, q0:q0 + lens_q[s]], K[:, k0:k0 + lens_k[s]], V[:, k0:k0 + lens_k[s]], scale,
                                 rows, offs[s], None)
        got = out[:, q0 + rows].float().cpu().numpy()
        assert np.max(np.abs(got - want)) <= OUT_TOL["bf16"] * float(np.abs(V).max())


@pytest.mark.parametrize("map_dtype", ["bf16", "fp8"])
def test_compress_leaves_unused_capacity_untouched(mr, map_dtype):
    spec = shrink(config(4), L=1024, H_s=4, H_r=4)
    lay = draw_layers(spec)[0]
    B = spec.block
    dt = mr.MR_BF16 if map_dtype == "bf16" else mr.MR_FP8_E4M3
    # room for every causal tile and some more, so the unused tail is never empty
    m = mr.Map(spec.H_s, spec.L, B, dt, mr.max_tiles(spec.H_s, spec.L, B) + 37, "cuda")
    if map_dtype == "bf16":
        m.vals.view(torch.int16).fill_(NAN_BF16)
    else:
        m.vals.view(torch.uint8).fill_(0x7F)              # e4m3 NaN
        m.tile_scale.fill_(float("nan"))
    m.col_idx.fill_(-7)
    mr.compress(dev(lay.Q, "bf16"), dev(lay.K, "bf16"), p32(spec.p), B, bias=mr.Bias.from_spec(lay.bias),
                scale=spec.scale, out=m)
    assert m.ws.sync_status() == mr.MR_OK
    nnz = m.nnz_host()
    assert 0 < nnz < m.capacity
    assert bool((m.col_idx[nnz:] == -7).all().item()) and bool((m.col_idx[:nnz] >= 0).all().item())
    if map_dtype == "bf16":
        assert _untouched(m.vals[nnz:])
        assert not bool(torch.isnan(m.vals[:nnz].float()).any().item())
    else:
        assert bool((m.vals.view(torch.uint8)[nnz:] == 0x7F).all().item())
        assert bool(torch.isnan(m.tile_scale[nnz:]).all().item())
        assert bool(torch.isfinite(m.tile_scale[:nnz]).all().item())
