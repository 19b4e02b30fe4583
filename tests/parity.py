"""Shared helpers for the GPU parity tests: run the CUDA path through the C-ABI binding and compare it
with the fp64 oracle on the same seeded inputs.

Tolerances (stated once, used by every test):
  * selection: kept sets equal except blocks within BOUNDARY of the top-p boundary (see
    ``check_selection``), with the kept mass >= p - BOUNDARY and the set still minimal;
  * block masses: |M_gpu - M_oracle| <= MASS_ATOL (fp32 accumulation of fp32 probabilities);
  * stored probabilities: bf16 |P - A| <= 2^-8 |A| + 1e-6; fp32 |P - A| <= 3e-5 |A| + 1e-9;
  * outputs: max |O_gpu - O_oracle(GPU kept sets)| <= OUT_TOL[dtype] * max |V| (2e-2 bf16, 1e-4 fp32).
    For bf16 the path rounds the map values, the mixing weights (tensor-core mixing), X and O to bf16,
    each at most 2^-9 relative on non-negative terms of a row that sums to at most 1, so the error is
    at most 4 * 2^-9 max |V| < 8e-3 max |V|, inside the stated 2e-2.
  * fp8 (e4m3) maps: stored values |P - A| <= 2^-4 |A| + 3e-6 (half an e4m3 step relative, plus the
    subnormal step of a piece whose scale is at most 1/448); outputs within 7e-2 max |V|: each
    translated value is off by at most 2^-4 of itself, plus bf16 and half-precision rounding (< 2^-8)
    and the retrieval's bf16 copy of each piece's scale (2^-9), and a row's translated values sum to
    at most 1, so |dO| <= (2^-4 + 2^-8 + 2^-9) max |V| < 7e-2 max |V|.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
from cross_model_attention_mr_b200 import mr

BOUNDARY = 1e-5
MASS_ATOL = 2e-6
OUT_TOL = {"bf16": 2e-2, "f32": 1e-4, "fp8": 7e-2}
VAL_TOL = {"bf16": (2.0 ** -8, 1e-6), "f32": (3e-5, 1e-9), "fp8": (2.0 ** -4, 3e-6)}


def dev(x: np.ndarray, dtype: str) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    return t.to("cuda").to(torch.bfloat16 if dtype == "bf16" else torch.float32).contiguous()


def p32(p: float) -> float:
    """The threshold both sides use: the float32 value the C-ABI receives, widened exactly."""
    return float(np.float32(p))


def check_selection(M: np.ndarray, kept_o: np.ndarray, kept_g: np.ndarray, p: float):
    """Compare one row's kept sets.  M: oracle masses of the causal blocks (fp64).

    A block is exempt when swapping it across the boundary changes the kept mass by at most
    BOUNDARY (its mass is within BOUNDARY of the oracle's last kept block), or when the oracle's
    cumulative mass at the boundary is itself within BOUNDARY of p (then the last kept and the
    first dropped block are exempt).  Returns (ok, n_exempt_used, message)."""
    n = M.shape[0]
    So = set(np.nonzero(kept_o[:n])[0].tolist())
    Sg = set(np.nonzero(kept_g[:n])[0].tolist())
    if np.any(kept_g[n:]):
        return False, 0, "kept block above the diagonal"
    if So == Sg:
        return True, 0, ""
    if p >= 1.0:
        return False, 0, "p >= 1 must keep every block"
    order = sorted(range(n), key=lambda J: (-M[J], J))
    k = len(So)
    cum = np.cumsum([M[J] for J in order])
    m_k = M[order[k - 1]]
    exempt = {b for b in range(n) if abs(M[b] - m_k) <= BOUNDARY}
    near = abs(cum[k - 1] - p) <= BOUNDARY or (k >= 2 and abs(cum[k - 2] - p) <= BOUNDARY)
    if near:
        for t in (k - 1, k):
            if 0 <= t < n:
                mt = M[order[t]]
                exempt |= {b for b in range(n) if abs(M[b] - mt) <= BOUNDARY}
    diff = So ^ Sg
    if not diff <= exempt:
        return False, len(diff), f"non-exempt difference {sorted(diff - exempt)}"
    sg = sum(M[b] for b in Sg)
    if not (sg >= p - BOUNDARY or len(Sg) == n):
        return False, len(diff), f"kept mass {sg} below p"
    if Sg and sg - min(M[b] for b in Sg) >= p + BOUNDARY:
        return False, len(diff), "GPU set not minimal"
    return True, len(diff), ""


def compare_compress(spec, lay, m: mr.Map, units, n_tiles: int = 12, rng_seed: int = 0,
                     all_tiles: bool = False, val_kind: str = None, renorm: bool = False):
    """Check masses, selection, row normalisers and stored values of the given units (h*nqb + I)
    against the oracle: every tile both sides kept when ``all_tiles``, else ``n_tiles`` sampled ones
    (plus a diagonal tile and a J = 0 tile).  Returns a dict of statistics."""
    B = spec.block
    nqb = spec.L // B
    p = p32(spec.p)
    orc = oracle.compress(lay.Q, lay.K, spec.scale, p, B, lay.bias, units=units)
    kept_g = m.kept_bits_host()
    row_ptr = m.row_ptr.cpu().numpy()
    mass_g = m.mass.cpu().numpy().reshape(spec.H_s, nqb, nqb) if m.mass is not None else None
    lse_g = m.lse.cpu().numpy() if m.lse is not None else None
    kmass_g = m.kept_mass.cpu().numpy().reshape(spec.H_s, nqb)
    stats = {"units": len(units), "exempt": 0, "mass_err": 0.0, "lse_err": 0.0, "val_err": 0.0}
    for u in units:
        h, I = divmod(u, nqb)
        M = orc.mass[h, I, : I + 1]
        ok, nex, msg = check_selection(M, orc.kept[h, I], kept_g[h, I], p)
        assert ok, f"selection mismatch at head {h} block {I}: {msg}"
        stats["exempt"] += nex
        if mass_g is not None:
            e = float(np.max(np.abs(mass_g[h, I, : I + 1] - M)))
            stats["mass_err"] = max(stats["mass_err"], e)
            assert e <= MASS_ATOL, (h, I, e)
            assert np.all(mass_g[h, I, I + 1:] == 0)
        Sg = np.nonzero(kept_g[h, I, : I + 1])[0]
        assert abs(kmass_g[h, I] - M[Sg].sum()) <= 1e-5
        assert row_ptr[u + 1] - row_ptr[u] == len(Sg)
        if lse_g is not None:
            rows = slice(I * B, (I + 1) * B)
            e = float(np.max(np.abs(lse_g[h, rows] - orc.lse[h, rows])))
            stats["lse_err"] = max(stats["lse_err"], e)
            assert e <= 1e-4, (h, I, e)
    # stored probabilities: every tile kept by both sides (all_tiles), else a sample of them
    rng = np.random.default_rng(rng_seed)
    cand = []
    for u in units:
        h, I = divmod(u, nqb)
        for J in np.nonzero(kept_g[h, I, : I + 1] & orc.kept[h, I, : I + 1])[0]:
            cand.append((h, I, int(J)))
    if all_tiles:
        pick = cand
    else:
        pick = [cand[i] for i in rng.choice(len(cand), size=min(n_tiles, len(cand)), replace=False)] if cand else []
        # always include a diagonal tile and tile J = 0 when available
        for extra in ((lambda c: c[1] == c[2]), (lambda c: c[2] == 0)):
            sel = [c for c in cand if extra(c)]
            if sel:
                pick.append(sel[0])
    if pick:
        vals = m.export()
        vals_host = vals.cpu().numpy() if all_tiles else None  # reduced sizes: one host copy
        col = m.col_idx.cpu().numpy()
        rtol, atol = VAL_TOL[val_kind or spec.dtype]
        by_unit = {}
        for (h, I, J) in pick:
            by_unit.setdefault(h * nqb + I, []).append(J)
        ulist = sorted(by_unit)
        for c0 in range(0, len(ulist), 32):      # bounded memory: 32 row blocks of oracle rows at a time
            chunk = ulist[c0:c0 + 32]
            # a renormalised map divides each row by its kept mass over the GPU's own kept set
            slab = oracle.row_block_probs(lay.Q, lay.K, spec.scale, B, chunk, lay.bias,
                                          renorm_kept=kept_g if renorm else None)
            for k, u in enumerate(chunk):
                h, I = divmod(u, nqb)
                bits = kept_g[h, I]
                for J in by_unit[u]:
                    t = int(row_ptr[u] + bits[:J].sum())
                    if t >= m.capacity:
                        continue
                    # full sizes: one tile at a time (the whole export would not fit in host memory)
                    got = (vals_host[t] if all_tiles else vals[t].cpu().numpy()).astype(np.float64)
                    want = slab[k][:, J * B:(J + 1) * B]
                    err = np.abs(got - want)
                    assert np.all(err <= rtol * np.abs(want) + atol), (h, I, J, float(err.max()))
                    stats["val_err"] = max(stats["val_err"],
                                           float(np.max(err / (np.abs(want) + 1e-30) * (want > 1e-6))))
                    assert int(col[t]) == J
                    stats["tiles_checked"] = stats.get("tiles_checked", 0) + 1
    return stats


def compare_retrieve(spec, lay, m: mr.Map, O: torch.Tensor, rows, V=None, reqs=None, out_kind: str = None,
                     renorm: bool = False):
    """O [n_req][H_r][L][d_v] from the GPU vs the oracle on the GPU's own kept sets."""
    kept_g = m.kept_bits_host()
    V = lay.V if V is None else V
    want = oracle.retrieve_rows(lay.Q, lay.K, spec.scale, spec.block, kept_g, lay.W, V, rows, lay.bias,
                                renorm=renorm)
    got = O[:, :, rows].float().cpu().numpy() if reqs is None else O[reqs][:, :, rows].float().cpu().numpy()
    err = float(np.max(np.abs(got - want)))
    vmax = float(np.max(np.abs(V)))
    assert err <= OUT_TOL[out_kind or spec.dtype] * vmax, (err, vmax)
    return err / vmax
