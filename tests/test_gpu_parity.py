"""GPU parity: the CUDA path through the C-ABI against the fp64 oracle on the same seeded inputs.

Reduced sizes run the oracle on every unit and row; full-size cases (the benchmark's shapes and
launch configuration) compare sampled units and rows.  Tolerances are defined in tests/parity.py.
"""
import numpy as np
import pytest
import torch

from cross_model_attention_mr_b200.workloads import config, draw_batch, draw_layers, shrink

from parity import compare_compress, compare_retrieve, dev, p32, OUT_TOL

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def mr():
    from cross_model_attention_mr_b200 import mr as m
    assert torch.cuda.is_available()
    assert m.LIB.mr_device_supported() == 1
    return m


def run_layer(mr, spec, lay, capacity=None, p=None):
    Q, K = dev(lay.Q, spec.dtype), dev(lay.K, spec.dtype)
    bias = mr.Bias.from_spec(lay.bias)
    m = mr.compress(Q, K, p32(spec.p if p is None else p), spec.block, bias=bias, scale=spec.scale,
                    capacity=capacity, store_mass=True, store_lse=True)
    st = m.ws.sync_status()
    W = torch.from_numpy(lay.W).cuda()
    V = dev(lay.V, spec.dtype)
    ws_r = mr.Workspace(mr.retrieve_workspace_bytes(m, spec.H_r, spec.d_v, 1))
    O = mr.retrieve(m, W, V, ws=ws_r)
    torch.cuda.synchronize()
    check_retrieve_status(mr, ws_r, st)
    return m, O, st


def check_retrieve_status(mr, ws_r, st_compress=0):
    """The retrieval's own status word: OK, or CAPACITY when the map it reads overflowed."""
    st = ws_r.sync_status()
    allowed = (mr.MR_OK, mr.MR_ERR_CAPACITY) if st_compress == mr.MR_ERR_CAPACITY else (mr.MR_OK,)
    assert st in allowed, mr.LIB.mr_status_string(st)


CASES = {
    "toy_full": (1, {}),
    "c2_small": (2, dict(L=1024, H_s=8, H_r=10)),
    "c3_small": (3, dict(L=1024, H_s=8, H_r=7, n_layers=2)),
    "c4_small": (4, dict(L=2048, H_s=4, H_r=8)),
    "c5_prefix_small": (5, dict(L=512, H_s=4, H_r=4)),
}


@pytest.mark.parametrize("name", list(CASES))
def test_reduced_configs_all_units(mr, name):
    n, kw = CASES[name]
    spec = shrink(config(n), **kw) if kw else config(n)
    layers = draw_layers(spec) if n != 5 else draw_layers(spec, [0])
    for lay in layers:
        m, O, st = run_layer(mr, spec, lay)
        assert st == mr.MR_OK
        nqb = spec.L // spec.block
        stats = compare_compress(spec, lay, m, list(range(spec.H_s * nqb)))
        rel = compare_retrieve(spec, lay, m, O, np.arange(spec.L))
        print(name, stats, "out_err/max|V|", rel)


@pytest.mark.parametrize("L,block", [(64, 64), (128, 64), (128, 128), (256, 128)])
def test_tiny_lengths(mr, L, block):
    spec = shrink(config(4), L=L, block=block, H_s=2, H_r=3)
    lay = draw_layers(spec)[0]
    m, O, st = run_layer(mr, spec, lay)
    assert st == mr.MR_OK
    compare_compress(spec, lay, m, list(range(spec.H_s * (L // block))))
    compare_retrieve(spec, lay, m, O, np.arange(L))


@pytest.mark.parametrize("p", [1.0, 0.05])
def test_extreme_thresholds(mr, p):
    spec = shrink(config(2), L=512, H_s=3, H_r=4, p=p)
    lay = draw_layers(spec)[0]
    m, O, st = run_layer(mr, spec, lay)
    assert st == mr.MR_OK
    nqb = spec.L // spec.block
    kept = m.kept_bits_host()
    if p >= 1:
        assert np.array_equal(kept, np.tril(np.ones((nqb, nqb), np.uint8))[None].repeat(3, 0))
        assert m.nnz_host() == mr.max_tiles(3, 512, 64)
    compare_compress(spec, lay, m, list(range(spec.H_s * nqb)))
    compare_retrieve(spec, lay, m, O, np.arange(spec.L))


def test_single_sender_head_identity_map(mr):
    """H_s = H_r = 1, W = [1], p = 1: retrieval is exact causal attention (the dense reference)."""
    spec = shrink(config(2), L=640, H_s=1, H_r=1, p=1.0)
    lay = draw_layers(spec)[0]
    lay.W = np.ones((1, 1), np.float32)
    m, O, st = run_layer(mr, spec, lay)
    cu = torch.tensor([0, spec.L], dtype=torch.int32, device="cuda")
    Q, K, V = dev(lay.Q, "bf16"), dev(lay.K, "bf16"), dev(lay.V, "bf16")
    D = mr.dense_ref(Q, K, V, cu, cu, None, spec.L, spec.L, mr.Bias.from_spec(lay.bias), spec.scale)
    err = (D.float() - O[0].float()).abs().max().item()
    assert err <= OUT_TOL["bf16"] * float(np.abs(lay.V).max())


@pytest.mark.parametrize("n,H_s,H_r", [(2, 1, 1), (2, 1, 5), (4, 1, 4), (4, 2, 3)])
def test_one_or_two_sender_heads_long_units(mr, n, H_s, H_r):
    """One or two kept heads per key block: sub-steps of one or two panels, many per unit, so the
    retrieval's page ring, register queue and double-buffered V run far ahead of the MMAs."""
    spec = shrink(config(n), L=1536, H_s=H_s, H_r=H_r)
    lay = draw_layers(spec)[0]
    m, O, st = run_layer(mr, spec, lay)
    assert st == mr.MR_OK
    compare_retrieve(spec, lay, m, O, np.arange(0, spec.L, 7))


def _retrieve_requests(mr, spec, lay, V_req):
    """Compress once, retrieve n_req strided value sets [n_req][H_r][L][d_v] in one launch."""
    Q, K = dev(lay.Q, spec.dtype), dev(lay.K, spec.dtype)
    m = mr.compress(Q, K, p32(spec.p), spec.block, bias=mr.Bias.from_spec(lay.bias), scale=spec.scale)
    assert m.ws.sync_status() == mr.MR_OK
    n_req = V_req.shape[0]
    ws_r = mr.Workspace(mr.retrieve_workspace_bytes(m, spec.H_r, spec.d_v, n_req))
    O = mr.retrieve(m, torch.from_numpy(lay.W).cuda(), dev(V_req, spec.dtype), ws=ws_r)
    torch.cuda.synchronize()
    check_retrieve_status(mr, ws_r)
    return m, O


@pytest.mark.parametrize("n_req", [2, 4, 5])
def test_request_groups_strided_values(mr, n_req):
    """2 requests: 2 heads x 2 requests per CTA; 4 or 5: 1 head x 4 requests (the 5th request in
    a partial request group).  Values strided per request."""
    from cross_model_attention_mr_b200.workloads import Layer
    spec = shrink(config(2), L=768, H_s=4, H_r=3)
    lay = draw_layers(spec)[0]
    rng = np.random.default_rng(77 + n_req)
    V_req = rng.standard_normal((n_req, spec.H_r, spec.L, spec.d_v), dtype=np.float32)
    V_req = V_req.astype(np.float32)
    from cross_model_attention_mr_b200.workloads import round_to_bf16
    V_req = round_to_bf16(V_req)
    m, O = _retrieve_requests(mr, spec, lay, V_req)
    rows = np.array([0, 1, 63, 64, 129, 383, 500, 767])
    for q in range(n_req):
        lq = Layer(Q=lay.Q, K=lay.K, V=np.ascontiguousarray(V_req[q]), W=lay.W, bias=lay.bias)
        compare_retrieve(spec, lq, m, O[q:q + 1], rows)


def test_ungrouped_schedule_many_receiver_heads(mr):
    """160 receiver heads x 4 requests: one row block needs 160 CTAs, more than the SMs, so the
    retrieval falls back to the ungrouped schedule."""
    from cross_model_attention_mr_b200.workloads import Layer, round_to_bf16
    spec = shrink(config(4), L=512, H_s=2, H_r=160)
    lay = draw_layers(spec)[0]
    rng = np.random.default_rng(91)
    V_req = round_to_bf16(rng.standard_normal((4, spec.H_r, spec.L, spec.d_v), dtype=np.float32))
    m, O = _retrieve_requests(mr, spec, lay, V_req)
    rows = np.array([0, 127, 128, 300, 511])
    for q in (0, 3):
        lq = Layer(Q=lay.Q, K=lay.K, V=np.ascontiguousarray(V_req[q]), W=lay.W, bias=lay.bias)
        compare_retrieve(spec, lq, m, O[q:q + 1], rows)


def test_capacity_overflow_is_reported(mr):
    spec = shrink(config(2), L=512, H_s=2, H_r=2)
    lay = draw_layers(spec)[0]
    full, _, _ = run_layer(mr, spec, lay)
    nnz = full.nnz_host()
    cap = nnz // 3
    m, _, st = run_layer(mr, spec, lay, capacity=cap)
    assert st == mr.MR_ERR_CAPACITY
    assert m.nnz_host() == nnz
    a = m.export(cap).cpu()
    b = full.export(cap).cpu()
    assert torch.equal(a, b)
    assert torch.equal(m.col_idx[:cap].cpu(), full.col_idx[:cap].cpu())


def test_multi_request_and_packed_values(mr):
    """n_req value sets read through per-request offsets into one packed buffer."""
    spec = shrink(config(5), L=512, H_s=4, H_r=4)
    b = draw_batch(shrink(spec, n_req=3, suffix_min=64, suffix_max=200))
    import oracle  # noqa: F401  (oracle used through parity helpers)
    from cross_model_attention_mr_b200.workloads import Layer
    P = spec.L
    lens = [P + r.suffix for r in b.requests]
    cu = np.concatenate([[0], np.cumsum(lens)])
    Vp = np.concatenate([r.V for r in b.requests], axis=1)  # [H_r][total][d_v]
    Qs, Ks = dev(b.Qs, "bf16"), dev(b.Ks, "bf16")
    m = mr.compress(Qs, Ks, p32(spec.p), spec.block, bias=mr.Bias.from_spec(b.bias), scale=spec.scale)
    Vd = dev(Vp, "bf16")
    off = torch.tensor(cu[:-1] * spec.d_v, dtype=torch.int64, device="cuda")
    ws_r = mr.Workspace(mr.retrieve_workspace_bytes(m, spec.H_r, spec.d_v, 3))
    O = mr.retrieve(m, torch.from_numpy(b.W).cuda(), Vd, v_req_off=off, v_head_stride=int(cu[-1]) * spec.d_v,
                    n_req=3, ws=ws_r)
    torch.cuda.synchronize()
    check_retrieve_status(mr, ws_r)
    rows = np.array([0, 1, 63, 64, 300, 511])
    for q in range(3):
        lay = Layer(Q=b.Qs, K=b.Ks, V=np.ascontiguousarray(b.requests[q].V[:, :P]), W=b.W, bias=b.bias)
        compare_retrieve(spec, lay, m, O[q:q + 1], rows)


def test_dense_varlen_suffix(mr):
    """Receiver suffix rows: dense causal attention over prefix + own suffix, ragged lengths."""
    import oracle
    spec = shrink(config(5), L=512, H_s=4, H_r=4, n_req=3, suffix_min=70, suffix_max=200)
    b = draw_batch(spec)
    P = spec.L
    lens_k = [P + r.suffix for r in b.requests]
    lens_q = [r.suffix for r in b.requests]
    cu_k = np.concatenate([[0], np.cumsum(lens_k)]).astype(np.int32)
    cu_q = np.concatenate([[0], np.cumsum(lens_q)]).astype(np.int32)
    Qp = np.concatenate([r.Q[:, P:] for r in b.requests], axis=1)
    Kp = np.concatenate([r.K for r in b.requests], axis=1)
    Vp = np.concatenate([r.V for r in b.requests], axis=1)
    bias = mr.Bias(b.bias.sink_len, b.bias.sink_bias, b.bias.window, b.bias.window_bias)
    O = mr.dense_ref(dev(Qp, "bf16"), dev(Kp, "bf16"), dev(Vp, "bf16"), torch.from_numpy(cu_q).cuda(),
                     torch.from_numpy(cu_k).cuda(), torch.full((3,), P, dtype=torch.int32, device="cuda"),
                     int(cu_q[-1]), int(cu_k[-1]), bias, spec.scale)
    torch.cuda.synchronize()
    Oh = O.float().cpu().numpy()
    from cross_model_attention_mr_b200.workloads import Bias as SpecBias
    sb = SpecBias(b.bias.sink_len, b.bias.sink_bias, b.bias.window, b.bias.window_bias)
    for q, r in enumerate(b.requests):
        rows = np.arange(r.suffix)
        want = oracle.dense_rows(r.Q[:, P:], r.K, r.V, spec.scale, rows, P, sb)
        got = Oh[:, cu_q[q]:cu_q[q + 1]]
        assert np.max(np.abs(got - want)) <= OUT_TOL["bf16"] * float(np.abs(r.V).max())


def test_dense_fp32_toy(mr):
    import oracle
    spec = config(1)
    lay = draw_layers(spec)[0]
    cu = torch.tensor([0, spec.L], dtype=torch.int32, device="cuda")
    O = mr.dense_ref(dev(lay.Q, "f32"), dev(lay.K, "f32"), dev(lay.V, "f32"), cu, cu, None, spec.L, spec.L,
                     mr.Bias.from_spec(lay.bias), spec.scale)
    torch.cuda.synchronize()
    want = oracle.dense_rows(lay.Q, lay.K, lay.V, spec.scale, np.arange(spec.L), 0, lay.bias)
    assert np.max(np.abs(O.cpu().numpy() - want)) <= OUT_TOL["f32"] * float(np.abs(lay.V).max())


# ------------------------------------------------------------------------------------------------
# Full benchmark sizes: sampled units and rows (oracle cost per unit grows with its query block).
# ------------------------------------------------------------------------------------------------
def _sample_units(spec, n, seed):
    nqb = spec.L // spec.block
    rng = np.random.default_rng(seed)
    Is = sorted(set([0, 1, nqb // 2, nqb - 1] + rng.integers(0, nqb, size=n).tolist()))
    hs = rng.integers(0, spec.H_s, size=len(Is))
    return [int(h) * nqb + I for h, I in zip(hs, Is)]


@pytest.mark.parametrize("n", [2, 4])
def test_full_size_sampled(mr, n):
    spec = config(n)
    lay = draw_layers(spec)[0]
    m, O, st = run_layer(mr, spec, lay)
    assert st == mr.MR_OK
    stats = compare_compress(spec, lay, m, _sample_units(spec, 4, n), n_tiles=6)
    rows = np.array([0, 5, spec.L // 2 + 17, spec.L - 1])
    rel = compare_retrieve(spec, lay, m, O, rows)
    print(spec.name, stats, rel)
