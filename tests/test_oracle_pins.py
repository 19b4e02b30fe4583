"""Pins for the fp64 oracle against things other than itself (CPU only).

Each test ties one oracle step to a fact the mathematics fixes independently of the oracle's own
code: closed forms, exhaustive search on tiny inputs, invariants of the definitions, and torch's
float64 scaled-dot-product attention as an independent library routine.  Together they are chosen
so that a dropped term, a wrong sign, index or normalisation, or a transposed operand in the
oracle fails at least one of them.

Definitions pinned (page "Accelerating Cross-Model LLM Inference via Attention Map Reuse"):
row-softmax attention map (s2.1), block-level top-p over per-(head, query-block) block masses
(s4, s5.2), simplex head mapping applied to the sparse maps and the receiver's values (s3.3, s5.4).
"""
import itertools
import math
from fractions import Fraction

import numpy as np
import pytest
import torch

from cross_model_attention_mr_b200.workloads import Bias, config, draw_layers, shrink

pytestmark = pytest.mark.filterwarnings("ignore::UserWarning")


def _sdpa(Q, K, V, bias_mask):
    """torch float64 SDPA (math path) with an additive mask; Q,K,V: [H][L][d]."""
    q = torch.from_numpy(np.asarray(Q, np.float64))[None]
    k = torch.from_numpy(np.asarray(K, np.float64))[None]
    v = torch.from_numpy(np.asarray(V, np.float64))[None]
    m = torch.from_numpy(bias_mask)[None]
    with torch.nn.attention.sdpa_kernel(torch.nn.attention.SDPBackend.MATH):
        o = torch.nn.functional.scaled_dot_product_attention(q, k, v, attn_mask=m)
    return o[0].numpy()


def _mask_from_rule(H, Lq, Lk, bias: Bias, q_offset=0):
    """Additive [H][Lq][Lk] mask: -inf above the causal diagonal, else the max-of-applicable bias.

    Written from the bias rule stated in the workload generator's docstring, with numpy
    broadcasting rather than the oracle's per-element loop."""
    i = np.arange(Lq)[:, None] + q_offset
    j = np.arange(Lk)[None, :]
    cand = []
    if bias.sink_len > 0:
        cand.append(np.where(j < bias.sink_len, bias.sink_bias, -np.inf) + 0 * i)
    if bias.window > 0:
        cand.append(np.where(i - j < bias.window, bias.window_bias, -np.inf) + 0 * j)
    out = np.zeros((H, Lq, Lk))
    for h in range(H):
        c = list(cand)
        if bias.kb_bias is not None:
            kb = bias.kb_bias[h].astype(np.float64)[j // bias.kb_block]
            c.append(np.broadcast_to(kb, (Lq, Lk)))
        if c:
            best = np.max(np.stack([np.broadcast_to(x, (Lq, Lk)) for x in c]), axis=0)
            best = np.where(np.isfinite(best), best, 0.0)
        else:
            best = np.zeros((Lq, Lk))
        out[h] = np.where(j <= i, best, -np.inf)
    return out


def _small(n=2, **kw):
    base = dict(L=512, H_s=4, H_r=5)
    base.update(kw)
    return shrink(config(n), **base)


# ---------------------------------------------------------------------------------------------
# s2.1: the map rows are a softmax -> each row sums to 1; the block masses sum to 1 per row-block.
# ---------------------------------------------------------------------------------------------
def test_map_rows_sum_to_one(oracle_mod):
    spec = _small(2, L=256)
    lay = draw_layers(spec)[0]
    B = spec.block
    for I in (0, 1, 3):
        tiles = [oracle_mod.tile_probs(lay.Q, lay.K, spec.scale, B, 1, I, J, lay.bias) for J in range(I + 1)]
        rows = np.concatenate(tiles, axis=1).sum(axis=1)
        assert np.max(np.abs(rows - 1.0)) < 1e-12
        # tiles above the diagonal are empty, the diagonal tile is lower-triangular
        up = oracle_mod.tile_probs(lay.Q, lay.K, spec.scale, B, 1, I, I + 1, lay.bias)
        assert np.all(up == 0)
        assert np.all(np.triu(tiles[-1], 1) == 0)


def test_block_masses_sum_to_one(oracle_mod):
    spec = _small(4, L=1024, block=128)
    lay = draw_layers(spec)[0]
    r = oracle_mod.compress(lay.Q, lay.K, spec.scale, spec.p, spec.block, lay.bias)
    tot = r.mass.sum(axis=2)
    assert np.max(np.abs(tot - 1.0)) < 1e-12
    nb = spec.L // spec.block
    assert np.all(r.mass[:, np.triu_indices(nb, 1)[0], np.triu_indices(nb, 1)[1]] == 0)


# ---------------------------------------------------------------------------------------------
# Closed form: Q = 0 and no bias give A_ij = 1/(i+1).  Every off-diagonal block of a row-block
# then has exactly the same mass, which also pins the tie-break (smaller J first).
# ---------------------------------------------------------------------------------------------
@pytest.mark.parametrize("p", [0.3, 0.6, 0.9, 0.999, 1.0])
def test_zero_query_closed_form(oracle_mod, p):
    H, L, d, B = 2, 96, 8, 8
    Q = np.zeros((H, L, d), np.float32)
    K = np.random.default_rng(1).standard_normal((H, L, d)).astype(np.float32)
    r = oracle_mod.compress(Q, K, 1 / math.sqrt(d), p, B, None)
    nb = L // B
    for I in range(nb):
        exact = []
        for J in range(I + 1):
            m = Fraction(0)
            for i in range(I * B, I * B + B):
                lo, hi = J * B, min(J * B + B - 1, i)
                if hi >= lo:
                    m += Fraction(hi - lo + 1, i + 1)
            exact.append(m / B)
        assert abs(sum(exact) - 1) == 0
        got = r.mass[0, I, : I + 1]
        assert np.max(np.abs(got - np.array([float(x) for x in exact]))) < 1e-14
        # canonical set: order by exact mass desc, index asc; shortest prefix reaching p
        order = sorted(range(I + 1), key=lambda J: (-exact[J], J))
        k, cum = 0, Fraction(0)
        if p >= 1:
            k = I + 1
        else:
            while k < I + 1:
                cum += exact[order[k]]
                k += 1
                if cum >= Fraction(p):
                    break
        want = np.zeros(nb, np.uint8)
        want[order[:k]] = 1
        for h in range(H):
            assert np.array_equal(r.kept[h, I], want), (h, I, p)
            assert r.count[h, I] == k


# ---------------------------------------------------------------------------------------------
# Exhaustive search: the selected set has the least size among sets reaching p and, among those,
# the largest mass; with ties, it is the set the (mass desc, index asc) order picks.
# ---------------------------------------------------------------------------------------------
def _brute(mass, p):
    """All minimum-size subsets reaching p with the largest mass, in exact rational arithmetic.

    Returns (sets, near): ``near`` is True when some subset sum lies within 1e-12 of p, where the
    oracle's sequential fp64 sum may legitimately decide the other way."""
    n = len(mass)
    fm = [Fraction(float(x)) for x in mass]
    fp = Fraction(float(p))
    if p >= 1:
        return [set(range(n))], False
    near = False
    for k in range(1, n + 1):
        best, best_sets = None, []
        for c in itertools.combinations(range(n), k):
            s = sum((fm[t] for t in c), Fraction(0))
            if abs(s - fp) < Fraction(1, 10**12):
                near = True
            if s >= fp:
                if best is None or s > best:
                    best, best_sets = s, [set(c)]
                elif s == best:
                    best_sets.append(set(c))
        if best is not None:
            return best_sets, near
    return [set(range(n))], near


def test_select_brute_force(oracle_mod):
    rng = np.random.default_rng(7)
    cases = []
    # masses of real rows (tiny oracle runs, up to 12 blocks)
    spec = _small(2, L=768, H_s=2)
    lay = draw_layers(spec)[0]
    r = oracle_mod.compress(lay.Q, lay.K, spec.scale, 0.9, spec.block, lay.bias)
    for h in range(2):
        for I in range(12):
            cases.append(r.mass[h, I, : I + 1])
    # random simplex rows, some with exact ties
    for n in range(1, 12):
        x = rng.dirichlet(np.ones(n))
        cases.append(x)
        t = np.round(x * 8) / 8.0
        if t.sum() > 0:
            cases.append(t / t.sum())
    for mass in cases:
        for p in (0.25, 0.5, 0.8, 0.9, 0.95, 1.0):
            kept, k, km = oracle_mod.select(mass, p)
            S = set(np.nonzero(kept)[0].tolist())
            assert len(S) == k
            sets, near = _brute(list(mass), p)
            if near:
                continue
            assert len(S) == len(sets[0])
            best = math.fsum(mass[t] for t in sets[0])
            assert abs(math.fsum(mass[t] for t in S) - best) <= 1e-12
            if p < 1:
                # minimal: dropping the smallest kept block falls below p
                assert km >= p - 1e-15
                assert km - min(mass[t] for t in S) < p
            # canonical among ties: exactly the (mass desc, index asc) prefix
            order = sorted(range(len(mass)), key=lambda J: (-mass[J], J))
            assert S == set(order[: len(S)])


# ---------------------------------------------------------------------------------------------
# Library routine: p = 1 and W = I reduce retrieval to exact causal attention; compare with
# torch float64 SDPA (with the bias rule as an additive mask).  A general W with p = 1 reduces
# to a W-weighted sum of per-(sender, receiver) SDPA outputs, which pins W's orientation.
# ---------------------------------------------------------------------------------------------
def test_p1_identity_matches_sdpa(oracle_mod):
    spec = _small(2, L=256, H_s=3, H_r=3)
    lay = draw_layers(spec)[0]
    nb = spec.L // spec.block
    kept = np.tril(np.ones((nb, nb), np.uint8))[None].repeat(spec.H_s, 0)
    rows = np.array([0, 1, 63, 64, 130, 255])
    O = oracle_mod.retrieve_rows(lay.Q, lay.K, spec.scale, spec.block, kept,
                                 np.eye(3, dtype=np.float32), lay.V, rows, lay.bias)[0]
    mask = _mask_from_rule(3, spec.L, spec.L, lay.bias)
    ref = _sdpa(lay.Q, lay.K, lay.V, mask)
    assert np.max(np.abs(O - ref[:, rows])) < 1e-12
    # the dense oracle is the same function
    D = oracle_mod.dense_rows(lay.Q, lay.K, lay.V, spec.scale, rows, 0, lay.bias)
    assert np.max(np.abs(D - ref[:, rows])) < 1e-12


def test_p1_general_W_matches_sdpa_mix(oracle_mod):
    spec = _small(4, L=512, block=128, H_s=3, H_r=4)
    lay = draw_layers(spec)[0]
    nb = spec.L // spec.block
    kept = np.tril(np.ones((nb, nb), np.uint8))[None].repeat(spec.H_s, 0)
    rows = np.array([5, 127, 128, 300, 511])
    O = oracle_mod.retrieve_rows(lay.Q, lay.K, spec.scale, spec.block, kept, lay.W, lay.V, rows,
                                 lay.bias)[0]
    mask = _mask_from_rule(spec.H_s, spec.L, spec.L, lay.bias)
    ref = np.zeros_like(O)
    for r in range(spec.H_r):
        for s in range(spec.H_s):
            o = _sdpa(lay.Q[s:s + 1], lay.K[s:s + 1], lay.V[r:r + 1], mask[s:s + 1])[0]
            ref[r] += float(lay.W[r, s]) * o[rows]
    assert np.max(np.abs(O - ref)) < 1e-12


def test_single_head_sparse_matches_masked_sdpa(oracle_mod):
    """H_s = 1, W = [1]: O = (kept row mass) x (softmax restricted to the kept blocks) . V."""
    spec = _small(2, L=512, H_s=1, H_r=1)
    lay = draw_layers(spec)[0]
    r = oracle_mod.compress(lay.Q, lay.K, spec.scale, 0.6, spec.block, lay.bias)
    B = spec.block
    rows = np.arange(spec.L)
    O = oracle_mod.retrieve_rows(lay.Q, lay.K, spec.scale, B, r.kept, np.ones((1, 1), np.float32),
                                 lay.V, rows, lay.bias)[0, 0]
    mask = _mask_from_rule(1, spec.L, spec.L, lay.bias)
    keep = np.repeat(np.repeat(r.kept[0], B, axis=0), B, axis=1).astype(bool)
    masked = np.where(keep, mask[0], -np.inf)
    sub = _sdpa(lay.Q, lay.K, lay.V[:1], masked[None])[0]
    full = _sdpa(lay.Q, lay.K, np.ones((1, spec.L, 1)), mask)[0]  # = 1 (sanity)
    assert np.max(np.abs(full - 1)) < 1e-12
    # kept row mass from the (separately pinned) tile probabilities
    km = np.zeros(spec.L)
    for I in range(spec.L // B):
        for J in range(I + 1):
            if r.kept[0, I, J]:
                km[I * B:(I + 1) * B] += oracle_mod.tile_probs(lay.Q, lay.K, spec.scale, B, 0, I, J,
                                                               lay.bias).sum(axis=1)
    assert np.max(np.abs(O - km[:, None] * sub)) < 1e-12


# ---------------------------------------------------------------------------------------------
# Closed form: logits that are bias only (Q = K = 0) give A_ij = exp(b_ij) / sum_k exp(b_ik);
# the overlap of sink and window with different values pins the max (not sum) rule.
# ---------------------------------------------------------------------------------------------
def test_bias_rule_closed_form(oracle_mod):
    H, L, d, B = 1, 8, 2, 4
    Q = np.zeros((H, L, d), np.float32)
    K = np.zeros((H, L, d), np.float32)
    kb = np.full((H, 2), -np.inf, np.float32)
    kb[0, 1] = 0.5
    bias = Bias(sink_len=2, sink_bias=1.0, window=3, window_bias=2.0, kb_bias=kb, kb_block=4)
    for I in range(2):
        for J in range(I + 1):
            t = oracle_mod.tile_probs(Q, K, 1.0, B, 0, I, J, bias)
            for a in range(B):
                i = I * B + a
                b = []
                for j in range(i + 1):
                    c = []
                    if j < 2:
                        c.append(1.0)
                    if i - j < 3:
                        c.append(2.0)
                    if j // 4 == 1:
                        c.append(0.5)
                    b.append(max(c) if c else 0.0)
                e = np.exp(np.array(b))
                want = e / e.sum()
                for c_ in range(B):
                    j = J * B + c_
                    exp_v = want[j] if j <= i else 0.0
                    assert abs(t[a, c_] - exp_v) < 1e-15


# ---------------------------------------------------------------------------------------------
# One-hot logits: with a huge logit on one key per row the map is a permutation-like 0/1 matrix
# and O = V of that key.
# ---------------------------------------------------------------------------------------------
def test_one_hot_logits(oracle_mod):
    H, L, d, B = 1, 64, 64, 16
    c = 30.0
    K = np.eye(L, d, dtype=np.float32) * c
    target = np.array([i // 2 for i in range(L)])
    Q = np.zeros((H, L, d), np.float32)
    Q[0, np.arange(L), target] = c
    V = np.random.default_rng(3).standard_normal((1, L, 4)).astype(np.float32)
    nb = L // B
    kept = np.tril(np.ones((nb, nb), np.uint8))[None]
    O = oracle_mod.retrieve_rows(Q, K[None], 1.0, B, kept, np.ones((1, 1), np.float32), V,
                                 np.arange(L), None)[0, 0]
    assert np.max(np.abs(O - V[0, target])) < 1e-12


# ---------------------------------------------------------------------------------------------
# Invariants of the translation (s3.3): linear in V; relabelling sender heads (with W's columns)
# changes nothing; V = 1 with p = 1 gives O = 1 because W's rows sum to 1.
# ---------------------------------------------------------------------------------------------
def test_translation_invariants(oracle_mod):
    spec = _small(3, L=512, H_s=4, H_r=3)
    lay = draw_layers(spec)[0]
    r = oracle_mod.compress(lay.Q, lay.K, spec.scale, spec.p, spec.block, lay.bias)
    rows = np.array([0, 70, 200, 511])
    f = lambda V, **kw: oracle_mod.retrieve_rows(kw.get("Q", lay.Q), kw.get("K", lay.K), spec.scale,
                                                  spec.block, kw.get("kept", r.kept),
                                                  kw.get("W", lay.W), V, rows,
                                                  kw.get("bias", lay.bias))[0]
    rng = np.random.default_rng(5)
    # values on a 1/8 grid so that the float32 combination below is exact
    V1 = (np.round(lay.V * 8) / 8).astype(np.float32)
    V2 = (np.round(rng.standard_normal(lay.V.shape) * 8) / 8).astype(np.float32)
    lin = f((2.0 * V1 - 0.5 * V2).astype(np.float32))
    assert np.max(np.abs(lin - (2.0 * f(V1) - 0.5 * f(V2)))) < 1e-11
    perm = np.array([2, 0, 3, 1])
    Op = f(lay.V, Q=lay.Q[perm], K=lay.K[perm], kept=r.kept[perm], W=lay.W[:, perm],
           bias=lay.bias.for_heads(perm))
    assert np.max(np.abs(Op - f(lay.V))) < 1e-12
    nb = spec.L // spec.block
    allk = np.tril(np.ones((nb, nb), np.uint8))[None].repeat(spec.H_s, 0)
    ones = f(np.ones_like(lay.V), kept=allk)
    assert np.max(np.abs(ones - 1.0)) < 1e-6  # W rows sum to 1 in float32


# ---------------------------------------------------------------------------------------------
# Dense attention with a query offset (suffix rows after a prefix) equals the same rows of the
# full-sequence computation.
# ---------------------------------------------------------------------------------------------
def test_dense_offset_rows(oracle_mod):
    spec = _small(5, L=256, H_s=2, H_r=2)
    lay = draw_layers(spec)[0]
    P = 192
    full = oracle_mod.dense_rows(lay.Q, lay.K, lay.V, spec.scale, np.arange(256), 0, lay.bias)
    suf = oracle_mod.dense_rows(lay.Q[:, P:], lay.K, lay.V, spec.scale, np.arange(64), P, lay.bias)
    assert np.max(np.abs(full[:, P:] - suf)) < 1e-13


def test_kept_mass_invariants(oracle_mod):
    spec = _small(4, L=1024, block=128)
    lay = draw_layers(spec)[0]
    for p in (0.5, 0.9, 0.99):
        r = oracle_mod.compress(lay.Q, lay.K, spec.scale, p, spec.block, lay.bias)
        nb = spec.L // spec.block
        for h in range(spec.H_s):
            for I in range(nb):
                S = np.nonzero(r.kept[h, I])[0]
                assert r.count[h, I] == len(S) and np.all(S <= I)
                km = r.mass[h, I, S].sum()
                assert abs(km - r.kept_mass[h, I]) < 1e-12
                assert km >= p - 1e-12 or len(S) == I + 1
                assert km - r.mass[h, I, S].min() < p


# ---------------------------------------------------------------------------------------------
# s2.1: the row log-normaliser the oracle stores next to the masses is log sum_j exp(s_ij) over
# the causal, biased logits.  Pinned to a closed form and to torch's float64 logsumexp over logits
# formed with a numpy matmul and the mask of the bias rule (not the oracle's own loops).
# ---------------------------------------------------------------------------------------------
def test_row_lse_zero_query_closed_form(oracle_mod):
    """Q = 0, no bias: every causal logit is 0, so the row normaliser is log(i + 1) exactly."""
    H, L, d, B = 2, 128, 16, 32
    Q = np.zeros((H, L, d), np.float32)
    K = np.random.default_rng(5).standard_normal((H, L, d)).astype(np.float32)
    r = oracle_mod.compress(Q, K, 1 / math.sqrt(d), 0.9, B, None)
    want = np.log(np.arange(1, L + 1, dtype=np.float64))
    assert np.max(np.abs(r.lse - want[None])) < 1e-13


@pytest.mark.parametrize("n,kw", [(2, dict(L=256, H_s=3)), (4, dict(L=512, H_s=2, block=128)),
                                  (3, dict(L=256, H_s=2))])
def test_row_lse_matches_torch_logsumexp(oracle_mod, n, kw):
    """Biased causal logits (sink, window and key-block terms, max rule) -> torch.logsumexp."""
    spec = _small(n, **kw)
    lay = draw_layers(spec)[0]
    r = oracle_mod.compress(lay.Q, lay.K, spec.scale, spec.p, spec.block, lay.bias)
    Q = lay.Q.astype(np.float64)
    K = lay.K.astype(np.float64)
    logits = spec.scale * np.einsum("hid,hjd->hij", Q, K) + _mask_from_rule(spec.H_s, spec.L, spec.L, lay.bias)
    want = torch.logsumexp(torch.from_numpy(logits), dim=-1).numpy()
    assert np.max(np.abs(r.lse - want)) < 1e-11


@pytest.mark.parametrize("n,kw", [(2, dict(L=256, H_s=3)), (4, dict(L=512, H_s=2, block=128))])
def test_row_block_probs_match_torch_softmax(oracle_mod, n, kw):
    """Whole query blocks of the map (s2.1) against torch's float64 softmax over the biased causal
    logits (numpy matmul + the bias-rule mask), and against the single-tile oracle entry."""
    spec = _small(n, **kw)
    lay = draw_layers(spec)[0]
    B, nqb = spec.block, spec.L // spec.block
    units = [0, nqb - 1, (spec.H_s - 1) * nqb + nqb // 2]
    got = oracle_mod.row_block_probs(lay.Q, lay.K, spec.scale, B, units, lay.bias)
    logits = spec.scale * np.einsum("hid,hjd->hij", lay.Q.astype(np.float64), lay.K.astype(np.float64))
    logits = logits + _mask_from_rule(spec.H_s, spec.L, spec.L, lay.bias)
    ref = torch.softmax(torch.from_numpy(logits), dim=-1).numpy()
    for t, u in enumerate(units):
        h, I = divmod(u, nqb)
        assert np.max(np.abs(got[t] - ref[h, I * B:(I + 1) * B])) < 1e-13
        J = I // 2
        tile = oracle_mod.tile_probs(lay.Q, lay.K, spec.scale, B, h, I, J, lay.bias)
        assert np.array_equal(got[t][:, J * B:(J + 1) * B], tile)


# ---------------------------------------------------------------------------------------------
# The renormalised variant (kept probabilities of each head's row rescaled to sum to 1): equal to
# torch's float64 softmax over the biased logits with every unkept key masked out.
# ---------------------------------------------------------------------------------------------
def test_renormalised_rows_are_the_masked_softmax(oracle_mod):
    spec = _small(2, L=512, H_s=3)
    lay = draw_layers(spec)[0]
    B, nqb = spec.block, spec.L // spec.block
    r = oracle_mod.compress(lay.Q, lay.K, spec.scale, 0.8, B, lay.bias)
    units = [0, nqb - 1, 1 * nqb + 5, 2 * nqb + 3]
    got = oracle_mod.row_block_probs(lay.Q, lay.K, spec.scale, B, units, lay.bias, renorm_kept=r.kept)
    logits = spec.scale * np.einsum("hid,hjd->hij", lay.Q.astype(np.float64), lay.K.astype(np.float64))
    logits = logits + _mask_from_rule(spec.H_s, spec.L, spec.L, lay.bias)
    for t, u in enumerate(units):
        h, I = divmod(u, nqb)
        keep_keys = np.repeat(r.kept[h, I], B).astype(bool)           # [L] kept keys of this row block
        lg = np.where(keep_keys[None, :], logits[h, I * B:(I + 1) * B], -np.inf)
        ref = torch.softmax(torch.from_numpy(lg), dim=-1).numpy()
        assert np.max(np.abs(got[t] - ref)) < 1e-13
        assert np.max(np.abs(got[t].sum(axis=1) - 1.0)) < 1e-12


def test_renormalised_retrieval_matches_masked_softmax_mix(oracle_mod):
    """O_r = (sum_s W[r,s] masked_softmax_s) V_r with torch; with every block kept it is the plain
    retrieval."""
    spec = _small(2, L=256, H_s=3, H_r=4)
    lay = draw_layers(spec)[0]
    B, nqb = spec.block, spec.L // spec.block
    r = oracle_mod.compress(lay.Q, lay.K, spec.scale, 0.7, B, lay.bias)
    rows = np.array([0, 70, 129, 255])
    got = oracle_mod.retrieve_rows(lay.Q, lay.K, spec.scale, B, r.kept, lay.W, lay.V, rows, lay.bias, renorm=True)
    logits = spec.scale * np.einsum("hid,hjd->hij", lay.Q.astype(np.float64), lay.K.astype(np.float64))
    logits = logits + _mask_from_rule(spec.H_s, spec.L, spec.L, lay.bias)
    keep = np.repeat(np.repeat(r.kept, B, axis=1), B, axis=2).astype(bool)   # [H][L][L]
    A = torch.softmax(torch.from_numpy(np.where(keep, logits, -np.inf)), dim=-1).numpy()
    At = np.einsum("rs,sij->rij", lay.W.astype(np.float64), A)
    want = np.einsum("rij,rjc->ric", At[:, rows], lay.V.astype(np.float64))
    assert np.max(np.abs(got[0] - want)) < 1e-12
    allk = np.tril(np.ones((nqb, nqb), np.uint8))[None].repeat(spec.H_s, 0)
    a = oracle_mod.retrieve_rows(lay.Q, lay.K, spec.scale, B, allk, lay.W, lay.V, rows, lay.bias, renorm=True)
    b = oracle_mod.retrieve_rows(lay.Q, lay.K, spec.scale, B, allk, lay.W, lay.V, rows, lay.bias)
    assert np.max(np.abs(a - b)) < 1e-13
