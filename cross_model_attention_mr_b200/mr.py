"""Python binding of libmr (argument marshalling only; every step of the path runs in libmr's kernels).

The names follow the C-ABI in ``include/mr.h``: ``compress`` -> ``mr_compress``, ``retrieve`` ->
``mr_retrieve``, ``dense_ref`` -> ``mr_dense_ref``.  PyTorch is used for device memory and streams;
``send_map`` / ``recv_map`` move a compressed map between ranks with torch.distributed.
Importing this module loads ``libmr.so`` and raises ``ImportError`` if it has not been built:
there is no fallback implementation.
"""
from __future__ import annotations

import ctypes
import math
import os
from typing import Optional

import numpy as np
import torch

# MR_LIBRARY=checked selects the bounds-checked build (libmr_checked.so): same API and results,
# with every global store of the tensor-core kernels checked against its extent on the device.
LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)),
                        "libmr_checked.so" if os.environ.get("MR_LIBRARY") == "checked" else "libmr.so")

MR_OK, MR_ERR_INVALID_ARG, MR_ERR_UNSUPPORTED, MR_ERR_CAPACITY = 0, 1, 2, 3
MR_ERR_CUDA, MR_ERR_TIMEOUT, MR_ERR_DEVICE_CHECK, MR_ERR_RANGE = 4, 5, 6, 7
MR_BF16, MR_F32, MR_FP8_E4M3 = 0, 1, 2

_c_i32, _c_i64, _c_f32, _c_p, _c_sz = ctypes.c_int32, ctypes.c_int64, ctypes.c_float, ctypes.c_void_p, ctypes.c_size_t


class LogitBias(ctypes.Structure):
    _fields_ = [("sink_len", _c_i32), ("sink_bias", _c_f32), ("window", _c_i32), ("window_bias", _c_f32),
                ("kb_bias", _c_p), ("kb_block", _c_i32), ("n_kb", _c_i32)]


class RetrieveOpts(ctypes.Structure):
    _fields_ = [("qb_begin", _c_i32), ("qb_end", _c_i32), ("v_group", _c_i32), ("v_pages", _c_p),
                ("page_rows", _c_i32), ("pages_per_req", _c_i32)]


class BSR(ctypes.Structure):
    _fields_ = [("H_s", _c_i32), ("L", _c_i32), ("block", _c_i32), ("val_dtype", ctypes.c_int),
                ("capacity_tiles", _c_i64), ("row_ptr", _c_p), ("col_idx", _c_p), ("vals", _c_p),
                ("kept_mass", _c_p), ("kept_bits", _c_p), ("mass", _c_p), ("lse", _c_p), ("nnz", _c_p),
                ("tile_scale", _c_p), ("renormalised", _c_i32)]


EXPORTS = {
    "mr_version": ([], ctypes.c_int),
    "mr_status_string": ([ctypes.c_int], ctypes.c_char_p),
    "mr_device_supported": ([], ctypes.c_int),
    "mr_checked_build": ([], ctypes.c_int),
    "mr_compress_workspace_bytes": ([ctypes.c_int] * 4, _c_sz),
    "mr_bsr_max_tiles": ([ctypes.c_int] * 3, _c_i64),
    "mr_compress": ([_c_p, _c_p, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, _c_f32, _c_f32,
                     ctypes.POINTER(LogitBias), ctypes.POINTER(BSR), _c_p, _c_sz, _c_p], ctypes.c_int),
    "mr_compress_blocks": ([_c_p, _c_p, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, _c_f32, _c_f32,
                            ctypes.POINTER(LogitBias), ctypes.c_int, ctypes.c_int, ctypes.POINTER(BSR), _c_p, _c_sz,
                            _c_p], ctypes.c_int),
    "mr_compress_noalloc": ([_c_p, _c_p, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, _c_f32, _c_f32,
                             ctypes.POINTER(LogitBias), ctypes.POINTER(BSR), _c_p], ctypes.c_int),
    "mr_compress_noalloc_status": ([_c_p], ctypes.c_int),
    "mr_retrieve_workspace_bytes": ([ctypes.POINTER(BSR), ctypes.c_int, ctypes.c_int, ctypes.c_int], _c_sz),
    "mr_retrieve": ([ctypes.POINTER(BSR), _c_p, ctypes.c_int, _c_p, _c_i64, _c_p, ctypes.c_int, ctypes.c_int,
                     ctypes.c_int, _c_p, _c_i64, _c_i64, ctypes.POINTER(RetrieveOpts), _c_p, _c_sz, _c_p],
                    ctypes.c_int),
    "mr_dense_ref_workspace_bytes": ([ctypes.c_int], _c_sz),
    "mr_dense_ref": ([_c_p, _c_p, _c_p, _c_p, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                      _c_p, _c_p, _c_p, ctypes.c_int, ctypes.c_int, ctypes.c_int, _c_f32,
                      ctypes.POINTER(LogitBias), _c_p, _c_sz, _c_p], ctypes.c_int),
    "mr_sync_status": ([_c_p, _c_p], ctypes.c_int),
    "mr_bsr_nnz": ([ctypes.POINTER(BSR), ctypes.POINTER(_c_i64), _c_p], ctypes.c_int),
    "mr_bsr_export": ([ctypes.POINTER(BSR), _c_i64, _c_p, _c_p], ctypes.c_int),
    "mr_bm_create": ([ctypes.c_int, _c_i64], _c_p),
    "mr_bm_destroy": ([_c_p], None),
    "mr_bm_insert": ([_c_p, _c_p, ctypes.c_int, ctypes.POINTER(BSR), ctypes.c_int, _c_i64], _c_i64),
    "mr_bm_lookup": ([_c_p, _c_p, ctypes.c_int, ctypes.POINTER(_c_i64)], ctypes.c_int),
    "mr_bm_map": ([_c_p, _c_i64, ctypes.c_int, ctypes.POINTER(BSR)], ctypes.c_int),
    "mr_bm_release": ([_c_p, _c_i64], ctypes.c_int),
    "mr_bm_evicted": ([_c_p, ctypes.POINTER(_c_i64), ctypes.c_int], ctypes.c_int),
    "mr_bm_stats": ([_c_p, ctypes.POINTER(_c_i64)], ctypes.c_int),
    "mr_gather_probe": ([ctypes.POINTER(BSR), ctypes.c_int, ctypes.c_int, _c_p, _c_sz, _c_p], ctypes.c_int),
    "mr_debug_set": ([ctypes.c_uint64, ctypes.c_int], ctypes.c_int),
    "mr_profile_enable": ([ctypes.c_int], ctypes.c_int),
    "mr_profile_read": ([_c_p, _c_p, ctypes.c_int], ctypes.c_int),
    "mr_kernel_name": ([ctypes.c_int], ctypes.c_char_p),
    "mr_kernel_launches": ([], _c_i64),
}


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing; build it with __graft_entry__.build()")
    lib = ctypes.CDLL(LIB_PATH)
    for name, (args, res) in EXPORTS.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = res
    return lib


LIB = _load()


class MRError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {LIB.mr_status_string(code).decode()} (status {code})")


def check(code: int, where: str) -> None:
    if code != MR_OK:
        raise MRError(code, where)


def _dt(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return MR_BF16
    if t.dtype == torch.float32:
        return MR_F32
    raise TypeError(f"unsupported dtype {t.dtype}")


def _torch_dtype(dt: int):
    return {MR_BF16: torch.bfloat16, MR_F32: torch.float32, MR_FP8_E4M3: torch.uint8}[dt]


def fp8_scales_per_tile(block: int) -> int:
    """Scales of an fp8 tile: one per 32-row x 64-key piece."""
    return (block // 32) * (block // 64)


def _stream(stream) -> Optional[int]:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _need_cuda(*ts):
    for t in ts:
        if t is not None and (not t.is_cuda or not t.is_contiguous()):
            raise ValueError("tensors must be contiguous CUDA tensors")


class Workspace:
    """Device workspace (256-byte aligned torch allocation)."""

    def __init__(self, nbytes: int, device="cuda"):
        self.nbytes = max(256, int(nbytes))
        self.buf = torch.empty(self.nbytes + 256, dtype=torch.uint8, device=device)
        off = (-self.buf.data_ptr()) % 256
        self.ptr = self.buf.data_ptr() + off

    def sync_status(self, stream=None) -> int:
        return LIB.mr_sync_status(self.ptr, _stream(stream))


class Bias:
    """Device-side logit bias (holds the kb_bias tensor alive)."""

    def __init__(self, sink_len=0, sink_bias=0.0, window=0, window_bias=0.0, kb_bias=None,
                 kb_block=0, device="cuda"):
        self.kb = None
        if kb_bias is not None:
            kb = torch.as_tensor(np.ascontiguousarray(kb_bias, dtype=np.float32))
            self.kb = kb.to(device).contiguous()
        self.c = LogitBias(int(sink_len), float(sink_bias), int(window), float(window_bias),
                           self.kb.data_ptr() if self.kb is not None else None,
                           int(kb_block) if self.kb is not None else 0,
                           int(self.kb.shape[1]) if self.kb is not None else 0)

    @classmethod
    def from_spec(cls, b, device="cuda"):
        if b is None:
            return None
        return cls(b.sink_len, b.sink_bias, b.window, b.window_bias, b.kb_bias, b.kb_block, device)


def _bias_ptr(bias: Optional[Bias]):
    return ctypes.byref(bias.c) if bias is not None else None


class Map:
    """A compressed map: caller-owned device arrays described by an ``mr_bsr``."""

    def __init__(self, H_s: int, L: int, block: int, dtype: int, capacity: int, device="cuda",
                 store_mass: bool = False, store_lse: bool = False, renormalised: bool = False):
        self.H_s, self.L, self.block, self.dtype, self.capacity = H_s, L, block, dtype, int(capacity)
        self.nqb = L // block
        self.nkw = (self.nqb + 31) // 32
        n = H_s * self.nqb
        dev = device
        self.row_ptr = torch.zeros(n + 1, dtype=torch.int32, device=dev)
        self.col_idx = torch.zeros(max(1, self.capacity), dtype=torch.int32, device=dev)
        self.vals = torch.zeros((max(1, self.capacity), block, block), dtype=_torch_dtype(dtype), device=dev)
        self.kept_mass = torch.zeros(n, dtype=torch.float32, device=dev)
        self.kept_bits = torch.zeros((n, self.nkw), dtype=torch.int32, device=dev)
        self.mass = torch.zeros((n, self.nqb), dtype=torch.float32, device=dev) if store_mass else None
        self.lse = torch.zeros((H_s, L), dtype=torch.float32, device=dev) if store_lse else None
        self.nnz = torch.zeros(1, dtype=torch.int64, device=dev)
        self.tile_scale = (torch.zeros((max(1, self.capacity), fp8_scales_per_tile(block)), dtype=torch.float32,
                                       device=dev) if dtype == MR_FP8_E4M3 else None)
        self.c = BSR(H_s, L, block, dtype, self.capacity, self.row_ptr.data_ptr(), self.col_idx.data_ptr(),
                     self.vals.data_ptr(), self.kept_mass.data_ptr(), self.kept_bits.data_ptr(),
                     self.mass.data_ptr() if self.mass is not None else None,
                     self.lse.data_ptr() if self.lse is not None else None, self.nnz.data_ptr(),
                     self.tile_scale.data_ptr() if self.tile_scale is not None else None,
                     1 if renormalised else 0)

    def nnz_host(self, stream=None) -> int:
        v = _c_i64(0)
        check(LIB.mr_bsr_nnz(ctypes.byref(self.c), ctypes.byref(v), _stream(stream)), "mr_bsr_nnz")
        return int(v.value)

    def kept_bits_host(self) -> np.ndarray:
        """Kept flags [H_s][nqb][nkb] as uint8 (host copy)."""
        w = self.kept_bits.cpu().numpy().view(np.uint32).reshape(self.H_s, self.nqb, self.nkw)
        bits = ((w[..., :, None] >> np.arange(32, dtype=np.uint32)) & 1).astype(np.uint8)
        return bits.reshape(self.H_s, self.nqb, self.nkw * 32)[..., : self.nqb]

    def to(self, device) -> "Map":
        """A copy of this map on `device` (same capacity and flags), e.g. to move a received map
        from host memory onto the GPU that retrieves from it."""
        m = Map(self.H_s, self.L, self.block, self.dtype, max(1, self.capacity), device, self.mass is not None,
                self.lse is not None, bool(self.c.renormalised))
        m.capacity = self.capacity
        m.c.capacity_tiles = self.capacity
        pairs = [(m.row_ptr, self.row_ptr), (m.col_idx, self.col_idx), (m.vals, self.vals),
                 (m.kept_mass, self.kept_mass), (m.kept_bits, self.kept_bits), (m.nnz, self.nnz)]
        for opt in ("mass", "lse", "tile_scale"):
            if getattr(self, opt) is not None:
                pairs.append((getattr(m, opt), getattr(self, opt)))
        for dst, src in pairs:
            dst.copy_(src)
        return m

    def export(self, n_tiles: Optional[int] = None, stream=None) -> torch.Tensor:
        n = self.nnz_host(stream) if n_tiles is None else int(n_tiles)
        n = min(n, self.capacity)
        out = torch.empty((max(1, n), self.block, self.block), dtype=torch.float32, device=self.vals.device)
        check(LIB.mr_bsr_export(ctypes.byref(self.c), n, out.data_ptr(), _stream(stream)), "mr_bsr_export")
        return out[:n]


# ------------------------------------------------------------------------------------------------
# Moving a compressed map to another rank (MapFlow section 5.3: the sender's compressed maps are
# shipped to the receiver instance, which then runs the fused retrieval locally).
# torch.distributed point-to-point: NCCL between GPUs, gloo between CPU ranks.
# ------------------------------------------------------------------------------------------------
def _map_arrays(m: "Map", n_stored: int):
    arrays = [m.row_ptr, m.kept_bits, m.kept_mass]
    if n_stored > 0:
        # bf16 travels as its bit pattern, so every backend moves it unchanged
        vals = m.vals[:n_stored]
        arrays += [m.col_idx[:n_stored], vals.view(torch.int16) if vals.dtype == torch.bfloat16 else vals]
        if m.tile_scale is not None:
            arrays.append(m.tile_scale[:n_stored])
    return arrays


def send_map(m: "Map", dst: int, group=None) -> None:
    """Send the arrays the retrieval reads: row pointers, kept bits and masses, and the column
    indices and values of the stored tiles (min(kept tiles, capacity) of them)."""
    import torch.distributed as dist
    nnz = int(m.nnz.item())
    n = min(nnz, m.capacity)
    hdr = torch.tensor([m.H_s, m.L, m.block, m.dtype, nnz, n], dtype=torch.int64, device=m.row_ptr.device)
    dist.send(hdr, dst, group=group)
    for t in _map_arrays(m, n):
        dist.send(t.contiguous(), dst, group=group)


def recv_map(src: int, device="cuda", group=None) -> "Map":
    """Receive a map sent by send_map into a new Map on `device` whose capacity is the number of
    stored tiles; the kept-tile count is the sender's (tiles past the sender's capacity stay
    unstored, as they were)."""
    import torch.distributed as dist
    hdr = torch.empty(6, dtype=torch.int64, device=device)
    dist.recv(hdr, src, group=group)
    H_s, L, block, dtype, nnz, n = (int(x) for x in hdr.tolist())
    m = Map(H_s, L, block, dtype, max(1, n), device)
    m.capacity = n
    m.c.capacity_tiles = n
    for t in _map_arrays(m, n):
        dist.recv(t, src, group=group)
    m.nnz.fill_(nnz)
    return m


# ------------------------------------------------------------------------------------------------
# One sequence split across ranks by query-block range (MapFlow section 6: distributed settings).
# Compression units (head, query block) and retrieval rows are independent once every key and
# value row up to the range's end is present, so the only exchange is an all-gather of the
# ranks' K and V row shards; maps and outputs stay on their rank.
# ------------------------------------------------------------------------------------------------
def split_query_blocks(nqb: int, world: int, align: int = 1):
    """Contiguous ranges [(qb_begin, qb_end)] of the nqb query blocks, one per rank, balanced by
    causal work (query block I costs I + 1 key blocks).  Cuts fall on multiples of ``align``
    (2 for block 64, whose kernels work on pairs of query blocks); a rank may get an empty range
    when there are fewer aligned pieces than ranks."""
    if nqb < 1 or world < 1 or align < 1:
        raise ValueError("need nqb, world, align >= 1")
    cum = np.concatenate([[0.0], np.cumsum(np.arange(1, nqb + 1, dtype=np.float64))])  # work before cut c
    total = cum[-1]
    cands = sorted(set(list(range(0, nqb + 1, align)) + [nqb]))
    cuts = [0]
    for r in range(1, world):
        target = total * r / world
        # the aligned cut whose prefix work is closest to the target, never before the previous cut
        best = min((c for c in cands if c >= cuts[-1]), key=lambda c: abs(cum[c] - target))
        cuts.append(best)
    cuts.append(nqb)
    return [(cuts[r], cuts[r + 1]) for r in range(world)]


def row_shards(L: int, ranges, block: int):
    """Token rows [(row_begin, row_end)] of each rank's query-block range."""
    return [(q0 * block, q1 * block) for q0, q1 in ranges]


def gather_row_shards(local: torch.Tensor, shards, group=None) -> torch.Tensor:
    """All-gather of per-rank row shards [H][rows_r][d] into the full [H][L][d] on every rank
    (torch.distributed: NCCL between GPUs, gloo between CPU ranks).  Shards are padded to the
    longest one so every rank sends the same number of bytes."""
    import torch.distributed as dist
    H, _, d = local.shape
    longest = max(e - b for b, e in shards)
    L = shards[-1][1]
    pad = torch.zeros((H, longest, d), dtype=local.dtype, device=local.device)
    pad[:, : local.shape[1]] = local
    parts = [torch.empty_like(pad) for _ in shards]
    dist.all_gather(parts, pad.contiguous(), group=group)
    full = torch.empty((H, L, d), dtype=local.dtype, device=local.device)
    for (b, e), part in zip(shards, parts):
        full[:, b:e] = part[:, : e - b]
    return full


def max_tiles(H_s: int, L: int, block: int) -> int:
    return int(LIB.mr_bsr_max_tiles(H_s, L, block))


def compress_workspace_bytes(H_s, L, d, block) -> int:
    return int(LIB.mr_compress_workspace_bytes(H_s, L, d, block))


def compress(Q: torch.Tensor, K: torch.Tensor, p: float, block: int, bias: Optional[Bias] = None,
             scale: Optional[float] = None, capacity: Optional[int] = None, out: Optional[Map] = None,
             ws: Optional[Workspace] = None, store_mass=False, store_lse=False, stream=None,
             blocks: Optional[tuple] = None, map_dtype: Optional[int] = None,
             renormalised: bool = False) -> Map:
    """mr_compress: Q, K [H_s][L][d] (bf16 or fp32, CUDA) -> Map.  ``blocks=(qb_begin, qb_end)``
    calls mr_compress_blocks: only those query blocks, the other rows of the map left empty.
    ``map_dtype=MR_FP8_E4M3`` stores e4m3 values with per-piece scales (bf16 inputs);
    ``renormalised=True`` stores each row divided by its kept mass."""
    _need_cuda(Q, K)
    H, L, d = Q.shape
    dt = _dt(Q)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if out is None:
        cap = max_tiles(H, L, block) if capacity is None else capacity
        out = Map(H, L, block, dt if map_dtype is None else map_dtype, cap, Q.device, store_mass, store_lse,
                  renormalised)
    if ws is None:
        ws = Workspace(compress_workspace_bytes(H, L, d, block), Q.device)
    out.ws = ws
    if blocks is None:
        check(LIB.mr_compress(Q.data_ptr(), K.data_ptr(), dt, H, L, d, float(scale), float(p), _bias_ptr(bias),
                              ctypes.byref(out.c), ws.ptr, ws.nbytes, _stream(stream)), "mr_compress")
    else:
        check(LIB.mr_compress_blocks(Q.data_ptr(), K.data_ptr(), dt, H, L, d, float(scale), float(p),
                                     _bias_ptr(bias), int(blocks[0]), int(blocks[1]), ctypes.byref(out.c), ws.ptr,
                                     ws.nbytes, _stream(stream)), "mr_compress_blocks")
    return out


def retrieve_workspace_bytes(m: Map, H_r: int, d_v: int, n_req: int) -> int:
    return int(LIB.mr_retrieve_workspace_bytes(ctypes.byref(m.c), H_r, d_v, n_req))


def retrieve(m: Map, W: torch.Tensor, V: torch.Tensor, out: Optional[torch.Tensor] = None,
             v_req_off: Optional[torch.Tensor] = None, v_req_stride: Optional[int] = None,
             v_head_stride: Optional[int] = None, n_req: Optional[int] = None,
             ws: Optional[Workspace] = None, stream=None, blocks: Optional[tuple] = None,
             v_group: int = 1, v_elems: Optional[int] = None, v_pages: Optional[torch.Tensor] = None,
             page_rows: int = 0) -> torch.Tensor:
    """mr_retrieve: W [H_r][H_s] fp32; V [H_v][L][d_v] or [n_req][H_v][L][d_v] (or a packed buffer
    with explicit strides/offsets), H_v = H_r / v_group -> O [n_req][H_r][L][d_v].
    ``blocks=(qb_begin, qb_end)`` writes only those query blocks' rows of O; ``v_elems`` defaults to
    the number of elements of V.  ``v_pages`` [n_req][pages_per_req] (int32, device) reads V as a
    pool of pages [page][H_v][page_rows][d_v]."""
    _need_cuda(W, V, v_req_off, v_pages)
    H_r = W.shape[0]
    dt = _dt(V)
    d_v = V.shape[-1]
    if v_head_stride is None:
        v_head_stride = V.shape[-2] * d_v
    if n_req is None:
        n_req = V.shape[0] if V.dim() == 4 else 1
    if v_req_stride is None:
        v_req_stride = (H_r // max(1, v_group)) * v_head_stride
    if v_elems is None:
        v_elems = V.numel()
    if out is None:
        out = torch.empty((n_req, H_r, m.L, d_v), dtype=V.dtype, device=V.device)
    _need_cuda(out)
    if ws is None:
        ws = Workspace(retrieve_workspace_bytes(m, H_r, d_v, n_req), V.device)
    opts = None
    if blocks is not None or v_group != 1 or v_pages is not None:
        b = blocks if blocks is not None else (0, 0)
        opts = ctypes.byref(RetrieveOpts(int(b[0]), int(b[1]), int(v_group),
                                         v_pages.data_ptr() if v_pages is not None else None, int(page_rows),
                                         int(v_pages.shape[1]) if v_pages is not None else 0))
    check(LIB.mr_retrieve(ctypes.byref(m.c), W.data_ptr(), H_r, V.data_ptr(), int(v_elems), out.data_ptr(), dt,
                          d_v, n_req, v_req_off.data_ptr() if v_req_off is not None else None, int(v_req_stride),
                          int(v_head_stride), opts, ws.ptr, ws.nbytes, _stream(stream)), "mr_retrieve")
    return out


def dense_ref(Q: torch.Tensor, K: torch.Tensor, V: torch.Tensor, cu_q: torch.Tensor, cu_k: torch.Tensor,
              q_offset: Optional[torch.Tensor], total_q: int, total_k: int, bias: Optional[Bias] = None,
              scale: Optional[float] = None, out: Optional[torch.Tensor] = None,
              ws: Optional[Workspace] = None, stream=None) -> torch.Tensor:
    """mr_dense_ref: packed Q [H][total_q][d], K/V [H][total_k][d] -> O [H][total_q][d_v]."""
    _need_cuda(Q, K, V, cu_q, cu_k, q_offset)
    H, _, d = Q.shape
    d_v = V.shape[-1]
    n_seq = cu_q.shape[0] - 1
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty((H, total_q, d_v), dtype=V.dtype, device=V.device)
    if ws is None:
        ws = Workspace(int(LIB.mr_dense_ref_workspace_bytes(n_seq)), Q.device)
    check(LIB.mr_dense_ref(Q.data_ptr(), K.data_ptr(), V.data_ptr(), out.data_ptr(), _dt(Q), H, d, d_v,
                           cu_q.data_ptr(), cu_k.data_ptr(),
                           q_offset.data_ptr() if q_offset is not None else None, n_seq, int(total_q),
                           int(total_k), float(scale), _bias_ptr(bias), ws.ptr, ws.nbytes, _stream(stream)),
          "mr_dense_ref")
    return out


def gather_probe(m: "Map", readers: int, ws: Optional[Workspace] = None, stream=None, ring_slots: int = 8) -> None:
    """mr_gather_probe: the retrieval's map reads alone (measurement)."""
    if ws is None:
        ws = Workspace(256, m.vals.device)
    check(LIB.mr_gather_probe(ctypes.byref(m.c), int(readers), int(ring_slots), ws.ptr, ws.nbytes, _stream(stream)),
          "mr_gather_probe")


def profile_enable(on: bool = True) -> bool:
    return bool(LIB.mr_profile_enable(1 if on else 0))


def profile_read() -> dict:
    """{kernel name: (total ms, launches)} for kernels launched since profiling was enabled."""
    n = 64
    ms = (ctypes.c_double * n)()
    cnt = (_c_i64 * n)()
    k = LIB.mr_profile_read(ctypes.cast(ms, _c_p), ctypes.cast(cnt, _c_p), n)
    out = {}
    for i in range(min(k, n)):
        if cnt[i]:
            out[LIB.mr_kernel_name(i).decode()] = (float(ms[i]), int(cnt[i]))
    return out


def kernel_launches() -> int:
    return int(LIB.mr_kernel_launches())


def compress_noalloc(Q: torch.Tensor, K: torch.Tensor, p: float, out: Map, bias: Optional[Bias] = None,
                     scale: Optional[float] = None, stream=None) -> Map:
    """mr_compress_noalloc: as compress, with the library's fixed scratch instead of a workspace."""
    _need_cuda(Q, K)
    H, L, d = Q.shape
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    check(LIB.mr_compress_noalloc(Q.data_ptr(), K.data_ptr(), _dt(Q), H, L, d, float(scale), float(p),
                                  _bias_ptr(bias), ctypes.byref(out.c), _stream(stream)), "mr_compress_noalloc")
    return out


def compress_noalloc_status(stream=None) -> int:
    """mr_compress_noalloc_status: device status of the last allocation-free compression."""
    return int(LIB.mr_compress_noalloc_status(_stream(stream)))



class BlockManager:
    """mr_bm_*: prefix-hash index from token prefixes to stored maps (MapFlow section 5.3).

    ``insert(tokens, maps)`` registers the per-layer maps of one sequence (the Map objects are kept
    alive here until their entry is evicted and collected by ``collect_evicted``);
    ``lookup(tokens)`` returns (reusable query blocks, entry id); ``map(entry, layer)`` gives a Map
    view to pass to ``retrieve(..., blocks=(0, k))``."""

    def __init__(self, block: int, budget_bytes: int = 0):
        self.h = LIB.mr_bm_create(int(block), int(budget_bytes))
        if not self.h:
            raise MRError(MR_ERR_INVALID_ARG, "mr_bm_create")
        self.block = block
        self._maps = {}

    def __del__(self):
        if getattr(self, "h", None):
            LIB.mr_bm_destroy(self.h)
            self.h = None

    def insert(self, tokens, maps, map_bytes: Optional[int] = None) -> int:
        tok = np.ascontiguousarray(tokens, dtype=np.int32)
        arr = (BSR * len(maps))(*[m.c for m in maps])
        if map_bytes is None:
            map_bytes = sum(m.vals.numel() * m.vals.element_size() for m in maps)
        eid = int(LIB.mr_bm_insert(self.h, tok.ctypes.data_as(_c_p), int(tok.shape[0]), arr, len(maps),
                                   int(map_bytes)))
        if eid < 0:
            raise MRError(-eid, "mr_bm_insert")
        self._maps[eid] = list(maps)
        return eid

    def lookup(self, tokens):
        tok = np.ascontiguousarray(tokens, dtype=np.int32)
        e = _c_i64(-1)
        k = int(LIB.mr_bm_lookup(self.h, tok.ctypes.data_as(_c_p), int(tok.shape[0]), ctypes.byref(e)))
        if k < 0:
            raise MRError(-k, "mr_bm_lookup")
        return k, int(e.value)

    def map(self, entry: int, layer: int) -> "Map":
        d = BSR()
        check(LIB.mr_bm_map(self.h, int(entry), int(layer), ctypes.byref(d)), "mr_bm_map")
        m = self._maps[entry][layer]
        assert m.c.vals == d.vals  # the descriptor is the registered map's
        return m

    def release(self, entry: int) -> None:
        check(LIB.mr_bm_release(self.h, int(entry)), "mr_bm_release")

    def collect_evicted(self):
        """Ids evicted since the last call; their Map objects (device arrays) are dropped here."""
        ids = (_c_i64 * 64)()
        out = []
        while True:
            n = int(LIB.mr_bm_evicted(self.h, ids, 64))
            out += [int(ids[i]) for i in range(n)]
            if n < 64:
                break
        for i in out:
            self._maps.pop(i, None)
        return out

    def stats(self) -> dict:
        v = (_c_i64 * 5)()
        check(LIB.mr_bm_stats(self.h, v), "mr_bm_stats")
        return dict(zip(("entries", "bytes", "lookups", "hits", "hit_blocks"), [int(x) for x in v]))
