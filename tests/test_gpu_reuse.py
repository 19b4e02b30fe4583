"""Prefix reuse across requests and receivers (MapFlow section 5.3 "Block Manager", section 1
"prefix-hash indexing and overlapping retrieval with partial recomputation") on the GPU.

A sender compresses request A once.  Request B shares A's first k blocks of tokens: the block
manager finds them, and two receivers retrieve B's first k query blocks from A's stored maps on
two streams, while B's remaining rows are recomputed with dense causal attention on a third
stream.  Every output row is checked against the fp64 oracle.
"""
import numpy as np
import pytest
import torch

from cross_model_attention_mr_b200.workloads import Bias as SpecBias, config, draw_layers, round_to_bf16, shrink

from parity import OUT_TOL, dev, p32

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def mr():
    from cross_model_attention_mr_b200 import mr as m
    assert torch.cuda.is_available()
    return m


def test_prefix_reuse_two_receivers_and_dense_suffix_on_streams(mr):
    import oracle
    spec = shrink(config(5), L=1024, H_s=4, H_r=4)
    B, L = spec.block, spec.L
    lay = draw_layers(spec)[0]                        # request A: sender Q, K over L tokens
    rng = np.random.default_rng(8)
    tok_a = rng.integers(0, 32000, size=L).astype(np.int32)
    shared = 10                                       # blocks of tokens B has in common with A
    tok_b = np.concatenate([tok_a[: shared * B], rng.integers(0, 32000, size=L - shared * B)]).astype(np.int32)

    m_a = mr.compress(dev(lay.Q, "bf16"), dev(lay.K, "bf16"), p32(spec.p), B, bias=mr.Bias.from_spec(lay.bias),
                      scale=spec.scale)
    assert m_a.ws.sync_status() == mr.MR_OK
    bm = mr.BlockManager(B)
    e_a = bm.insert(tok_a, [m_a])
    bm.release(e_a)
    k, e = bm.lookup(tok_b)
    assert (k, e) == (shared, e_a)
    m = bm.map(e, 0)

    # two receivers of request B (own W and V each), and B's own receiver Q, K, V for the rest
    std = np.float32(spec.qk_std)
    Ws = [np.ascontiguousarray(lay.W), np.ascontiguousarray(lay.W[::-1])]
    Vs = [round_to_bf16(rng.standard_normal((spec.H_r, L, spec.d_v), dtype=np.float32)) for _ in range(2)]
    Qb = round_to_bf16(rng.standard_normal((spec.H_r, L, spec.d), dtype=np.float32) * std)
    Kb = round_to_bf16(rng.standard_normal((spec.H_r, L, spec.d), dtype=np.float32) * std)
    P = k * B
    streams = [torch.cuda.Stream() for _ in range(3)]
    outs = []
    for r in range(2):
        with torch.cuda.stream(streams[r]):
            outs.append(mr.retrieve(m, torch.from_numpy(Ws[r]).cuda(), dev(Vs[r], "bf16"), blocks=(0, k),
                                    stream=streams[r]))
    sb = SpecBias(lay.bias.sink_len, lay.bias.sink_bias, lay.bias.window, lay.bias.window_bias)
    with torch.cuda.stream(streams[2]):
        cu_q = torch.tensor([0, L - P], dtype=torch.int32, device="cuda")
        cu_k = torch.tensor([0, L], dtype=torch.int32, device="cuda")
        off = torch.tensor([P], dtype=torch.int32, device="cuda")
        Od = mr.dense_ref(dev(Qb[:, P:], "bf16"), dev(Kb, "bf16"), dev(Vs[0], "bf16"), cu_q, cu_k, off, L - P, L,
                          mr.Bias.from_spec(sb), spec.scale, stream=streams[2])
    torch.cuda.synchronize()
    rows = np.array([0, 1, 63, 64, 300, P - 1])
    for r in range(2):
        from cross_model_attention_mr_b200.workloads import Layer
        lr = Layer(Q=lay.Q, K=lay.K, V=Vs[r], W=Ws[r], bias=lay.bias)
        want = oracle.retrieve_rows(lr.Q, lr.K, spec.scale, B, m.kept_bits_host(), lr.W, lr.V, rows, lr.bias)
        got = outs[r][:, :, rows].float().cpu().numpy()
        assert np.max(np.abs(got - want)) <= OUT_TOL["bf16"] * float(np.abs(Vs[r]).max())
    srows = np.array([0, 17, L - P - 1])
    want = oracle.dense_rows(Qb[:, P:], Kb, Vs[0], spec.scale, srows, P, sb)
    got = Od[:, srows].float().cpu().numpy()
    assert np.max(np.abs(got - want)) <= OUT_TOL["bf16"] * float(np.abs(Vs[0]).max())
    st = bm.stats()
    assert st["hits"] == 1 and st["hit_blocks"] == shared
    bm.release(e)
