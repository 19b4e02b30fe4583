"""fp64 CPU oracle for attention-map reuse: TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the benchmark's ``cpu_baseline`` / reference
leg may import this package.  The product path (``cross_model_attention_mr_b200``) never imports,
links or runs anything here, and this package never imports the product.

The arithmetic lives in ``mr_oracle.c`` (plain C, fp64, OpenMP over independent rows/units);
this module only marshals numpy arrays.  Each wrapper names the passage it follows:

  * ``compress``     -- block masses, block top-p selection, per-row normalisers
                        ("Accelerating Cross-Model LLM Inference via Attention Map Reuse", s4, s5.2)
  * ``select``       -- the top-p rule on one row of block masses (same sections)
  * ``tile_probs``   -- softmax probabilities of one map tile (s2.1)
  * ``row_block_probs`` -- the same softmax rows for whole query blocks (s2.1)
  * ``retrieve_rows``-- translated map times receiver values on given kept sets (s3.3, s5.4)
  * ``dense_rows``   -- exact causal attention ("AttnCache Guide", "The Quadratic Self-Attention Cost")
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional, Sequence

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "mr_oracle.c")
_OUT_DIR = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_OUT_DIR, "libmr_oracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (-O2, OpenMP, IEEE fp64: no fast-math)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        os.makedirs(_OUT_DIR, exist_ok=True)
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared",
                               "-fno-fast-math", "-ffp-contract=off", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        P = ctypes.c_void_p
        i32, i64, f64 = ctypes.c_int32, ctypes.c_int64, ctypes.c_double
        bias_args = [i32, f64, i32, f64, P, i32]
        lib.or_select.argtypes = [P, ctypes.c_int, f64, P, P]
        lib.or_select.restype = ctypes.c_int
        lib.or_compress.argtypes = [P, P, ctypes.c_int, ctypes.c_int, ctypes.c_int, f64, f64,
                                    ctypes.c_int] + bias_args + [P, P, P, P, P, P,
                                                                 ctypes.c_int, ctypes.c_int]
        lib.or_tile_probs.argtypes = [P, P, ctypes.c_int, ctypes.c_int, ctypes.c_int, f64,
                                      ctypes.c_int] + bias_args + [ctypes.c_int] * 3 + [P]
        lib.or_row_block_probs.argtypes = [P, P, ctypes.c_int, ctypes.c_int, ctypes.c_int, f64,
                                           ctypes.c_int] + bias_args + [P, ctypes.c_int, P, P, ctypes.c_int]
        lib.or_retrieve_rows.argtypes = [P, P, ctypes.c_int, ctypes.c_int, ctypes.c_int, f64,
                                         ctypes.c_int] + bias_args + [
            P, P, ctypes.c_int, P, ctypes.c_int, i64, ctypes.c_int, P, ctypes.c_int, ctypes.c_int, P,
            ctypes.c_int]
        lib.or_dense_rows.argtypes = [P, P, P] + [ctypes.c_int] * 5 + [i64, f64] + bias_args + [
            P, ctypes.c_int, P, ctypes.c_int]
        for name in ("or_compress", "or_tile_probs", "or_row_block_probs", "or_retrieve_rows",
                     "or_dense_rows"):
            getattr(lib, name).restype = ctypes.c_int
        _lib = lib
    return _lib


def _f32(a):
    return np.ascontiguousarray(a, dtype=np.float32)


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _bias_args(bias):
    if bias is None:
        return [0, 0.0, 0, 0.0, None, 0], None
    kb = None if bias.kb_bias is None else _f32(bias.kb_bias)
    return [int(bias.sink_len), float(bias.sink_bias), int(bias.window), float(bias.window_bias),
            _ptr(kb), int(bias.kb_block)], kb


def select(mass: Sequence[float], p: float):
    """Top-p rule on one row of block masses -> (kept mask uint8, count, kept mass)."""
    m = np.ascontiguousarray(mass, dtype=np.float64)
    kept = np.zeros(m.shape[0], np.uint8)
    km = ctypes.c_double(0.0)
    k = _load().or_select(_ptr(m), int(m.shape[0]), float(p), _ptr(kept), ctypes.byref(km))
    return kept, int(k), float(km.value)


class CompressResult:
    def __init__(self, mass, kept, count, kept_mass, lse):
        self.mass, self.kept, self.count, self.kept_mass, self.lse = mass, kept, count, kept_mass, lse


def compress(Q, K, sigma: float, p: float, B: int, bias=None, units: Optional[Sequence[int]] = None,
             n_threads: int = 0) -> CompressResult:
    """Block masses [H][nQB][nKB], kept [H][nQB][nKB], counts, kept masses and row log-normalisers.

    ``units`` restricts the work to unit ids h*nQB + I (other entries stay zero / -inf)."""
    Q, K = _f32(Q), _f32(K)
    H, L, d = Q.shape
    nb = L // B
    mass = np.zeros((H, nb, nb), np.float64)
    kept = np.zeros((H, nb, nb), np.uint8)
    count = np.zeros((H, nb), np.int32)
    kmass = np.zeros((H, nb), np.float64)
    lse = np.full((H, L), -np.inf, np.float64)
    ba, keep = _bias_args(bias)
    u = None if units is None else np.ascontiguousarray(units, dtype=np.int32)
    rc = _load().or_compress(_ptr(Q), _ptr(K), H, L, d, float(sigma), float(p), int(B), *ba,
                             _ptr(mass), _ptr(kept), _ptr(count), _ptr(kmass), _ptr(lse), _ptr(u),
                             0 if u is None else int(u.shape[0]), int(n_threads))
    if rc:
        raise ValueError("oracle compress rejected its arguments")
    return CompressResult(mass, kept, count, kmass, lse)


def tile_probs(Q, K, sigma: float, B: int, h: int, I: int, J: int, bias=None) -> np.ndarray:
    Q, K = _f32(Q), _f32(K)
    H, L, d = Q.shape
    out = np.zeros((B, B), np.float64)
    ba, keep = _bias_args(bias)
    rc = _load().or_tile_probs(_ptr(Q), _ptr(K), H, L, d, float(sigma), int(B), *ba, int(h), int(I),
                               int(J), _ptr(out))
    if rc:
        raise ValueError("oracle tile_probs rejected its arguments")
    return out


def row_block_probs(Q, K, sigma: float, B: int, units: Sequence[int], bias=None,
                    n_threads: int = 0, renorm_kept=None) -> np.ndarray:
    """Softmax rows of whole query blocks: [len(units)][B][L] for units u = h*nQB + I (s2.1).
    ``renorm_kept`` ([H][nQB][nKB] 0/1): the renormalised variant, kept blocks only, rows summing to 1."""
    Q, K = _f32(Q), _f32(K)
    H, L, d = Q.shape
    u = np.ascontiguousarray(units, dtype=np.int32)
    out = np.zeros((u.shape[0], B, L), np.float64)
    ba, keep = _bias_args(bias)
    kp = None if renorm_kept is None else np.ascontiguousarray(renorm_kept, dtype=np.uint8)
    rc = _load().or_row_block_probs(_ptr(Q), _ptr(K), H, L, d, float(sigma), int(B), *ba, _ptr(u),
                                    int(u.shape[0]), _ptr(kp), _ptr(out), int(n_threads))
    if rc:
        raise ValueError("oracle row_block_probs rejected its arguments")
    return out


def retrieve_rows(Q, K, sigma: float, B: int, kept, W, V, rows, bias=None, n_threads: int = 0,
                  renorm: bool = False):
    """O[q][r][t][:] for query rows ``rows`` (absolute positions), on the given kept sets
    (``renorm``: each sender head's kept row rescaled to sum to 1 first).

    V: [H_r][L][dv] or [n_req][H_r][L][dv]."""
    Q, K, W = _f32(Q), _f32(K), _f32(W)
    V = _f32(V)
    if V.ndim == 3:
        V = V[None]
    n_req, H_r, L, dv = V.shape
    H_s, Ls, d = Q.shape
    assert Ls == L
    kept = np.ascontiguousarray(kept, dtype=np.uint8)
    rows = np.ascontiguousarray(rows, dtype=np.int64)
    O = np.zeros((n_req, H_r, rows.shape[0], dv), np.float64)
    ba, keep = _bias_args(bias)
    rc = _load().or_retrieve_rows(_ptr(Q), _ptr(K), H_s, L, d, float(sigma), int(B), *ba,
                                  _ptr(kept), _ptr(W), H_r, _ptr(V), n_req, H_r * L * dv, dv,
                                  _ptr(rows), int(rows.shape[0]), 1 if renorm else 0, _ptr(O), int(n_threads))
    if rc:
        raise ValueError("oracle retrieve rejected its arguments")
    return O


def dense_rows(Q, K, V, sigma: float, rows, q_offset: int = 0, bias=None, n_threads: int = 0):
    """Exact causal attention for one sequence: O[h][t][:] for query rows ``rows`` (0-based in Q)."""
    Q, K, V = _f32(Q), _f32(K), _f32(V)
    H, Lq, d = Q.shape
    Lk = K.shape[1]
    dv = V.shape[2]
    rows = np.ascontiguousarray(rows, dtype=np.int64)
    O = np.zeros((H, rows.shape[0], dv), np.float64)
    ba, keep = _bias_args(bias)
    rc = _load().or_dense_rows(_ptr(Q), _ptr(K), _ptr(V), H, Lq, Lk, d, dv, int(q_offset),
                               float(sigma), *ba, _ptr(rows), int(rows.shape[0]), _ptr(O),
                               int(n_threads))
    if rc:
        raise ValueError("oracle dense rejected its arguments")
    return O
