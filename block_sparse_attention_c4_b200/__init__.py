"""Python binding of ``libqsa.so``: one Qwen Sparse Attention (c4) layer on B200.

Thin argument marshalling over the C ABI in ``include/qsa.h`` (same names,
``qsa_`` prefix dropped).  Every step of the layer runs in the library's CUDA
kernels; PyTorch only provides device memory and the current stream.  There
is no fallback: if the library is missing or a call fails, an exception says
so.
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libqsa.so")

HEAD_DIM = 128
INDEX_HEADS = 4
Q_HEADS = 16
KV_HEADS = 2
BLOCK = 4
TOPK = 512
MAX_SEL = 2051
PAGE_SIZE = 64
MAX_DRAFT = 8

OP_INDEX_SCORE_TOPK, OP_SPARSE_GQA, OP_DECODE, OP_DECODE_INDEXSHARE, OP_COMPRESS_APPEND = 1, 2, 3, 4, 5
OP_PREFILL_SCORE_TOPK = 6
OP_DECODE_INDEXER, OP_DECODE_ATTEND, OP_SPLIT_SCORE = 7, 8, 9
PROJ_FEATURES = INDEX_HEADS * HEAD_DIM + HEAD_DIM + INDEX_HEADS  # 644

DEVERR_BITS = {1: "page", 2: "length", 4: "position", 8: "request", 16: "selection", 32: "timeout"}


class QsaError(RuntimeError):
    pass


class CacheStruct(ctypes.Structure):
    _fields_ = [
        ("k", ctypes.c_void_p), ("v", ctypes.c_void_p), ("cidx", ctypes.c_void_p), ("ring", ctypes.c_void_p),
        ("page_table", ctypes.c_void_p), ("num_slots", ctypes.c_int64), ("page_size", ctypes.c_int32),
        ("max_pages", ctypes.c_int32), ("batch", ctypes.c_int32), ("kv_stride", ctypes.c_int32),
        ("rope_theta", ctypes.c_double),
    ]


_lib = None
EXPORTS = [
    "qsa_workspace_bytes", "qsa_workspace_init", "qsa_compress_append", "qsa_index_score_topk",
    "qsa_expand_indices", "qsa_sparse_gqa", "qsa_decode", "qsa_decode_indexshare", "qsa_device_error",
    "qsa_set_profile_events", "qsa_decode_kernel_count", "qsa_status_string", "qsa_version",
    "qsa_prefill_score_topk", "qsa_sparse_gqa_noalloc", "qsa_check_bounded_wait", "qsa_last_error_string",
    "qsa_index_project", "qsa_decode_indexer", "qsa_decode_attend", "qsa_prefill_rescored_rows",
    "qsa_prefill_rotated_queries",
]


def lib():
    """Load libqsa.so (building it first if the sources are newer is the caller's job: see build.py)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise QsaError(f"{LIB_PATH} is missing: run `python -m block_sparse_attention_c4_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    vp, i32, i64, f32, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_float, ctypes.c_size_t
    cp = ctypes.POINTER(CacheStruct)
    L.qsa_workspace_bytes.argtypes = [i32, i32, i32]
    L.qsa_workspace_bytes.restype = sz
    L.qsa_workspace_init.argtypes = [vp, sz, vp]
    L.qsa_compress_append.argtypes = [cp, vp, vp, vp, i32, i32, vp]
    L.qsa_index_score_topk.argtypes = [cp, vp, vp, vp, vp, i32, i32, vp, vp, vp, sz, vp]
    L.qsa_expand_indices.argtypes = [vp, vp, vp, i32, vp, vp, vp]
    L.qsa_prefill_score_topk.argtypes = [cp, vp, vp, i32, i32, i32, vp, vp, vp, sz, vp]
    L.qsa_prefill_score_topk.restype = ctypes.c_int
    L.qsa_sparse_gqa.argtypes = [cp, vp, vp, vp, vp, i32, i32, i32, f32, vp, vp, vp, sz, vp]
    L.qsa_decode.argtypes = [cp, vp, vp, vp, vp, vp, i32, f32, vp, vp, vp, vp, vp, sz, vp]
    L.qsa_decode_indexshare.argtypes = [cp, vp, vp, i32, vp, i32, vp, f32, vp, vp, sz, vp]
    L.qsa_sparse_gqa_noalloc.argtypes = [cp, vp, vp, vp, vp, i32, i32, i32, f32, vp, vp, vp]
    L.qsa_sparse_gqa_noalloc.restype = ctypes.c_int
    L.qsa_index_project.argtypes = [vp, vp, i32, i32, vp, vp, vp, vp]
    L.qsa_decode_indexer.argtypes = [cp, vp, vp, i32, vp, i32, vp, vp, vp, sz, vp]
    L.qsa_decode_attend.argtypes = [cp, vp, vp, i32, vp, vp, f32, vp, vp, vp, sz, vp]
    for f in (L.qsa_index_project, L.qsa_decode_indexer, L.qsa_decode_attend):
        f.restype = ctypes.c_int
    L.qsa_prefill_score_topk_varlen.argtypes = [cp, vp, vp, i32, vp, vp, vp, i32, vp, vp, vp, sz, vp]
    L.qsa_prefill_score_topk_varlen.restype = ctypes.c_int
    L.qsa_split_score_topk.argtypes = [cp, vp, vp, vp, vp, vp, i32, vp, vp, vp, vp, sz, vp]
    L.qsa_split_merge.argtypes = [vp, vp, vp, i32, i32, vp, vp, vp]
    L.qsa_split_positions.argtypes = [vp, vp, vp, vp, vp, i32, vp, vp, vp]
    L.qsa_split_combine.argtypes = [vp, vp, i32, i32, vp, vp]
    for f in (L.qsa_split_score_topk, L.qsa_split_merge, L.qsa_split_positions, L.qsa_split_combine):
        f.restype = ctypes.c_int
    L.qsa_sparse_gqa_fp8.argtypes = [cp, f32, f32, vp, vp, vp, vp, i32, i32, i32, f32, vp, vp, vp, sz, vp]
    L.qsa_decode_fp8.argtypes = [cp, f32, f32, vp, vp, vp, vp, vp, i32, f32, vp, vp, vp, vp, vp, sz, vp]
    L.qsa_sparse_gqa_fp8.restype = ctypes.c_int
    L.qsa_decode_fp8.restype = ctypes.c_int
    L.qsa_prefill_rescored_rows.argtypes = [vp, i32, i32, vp]
    L.qsa_prefill_rescored_rows.restype = i32
    L.qsa_prefill_rotated_queries.argtypes = [vp, i32, i32, vp, vp]
    L.qsa_prefill_rotated_queries.restype = ctypes.c_int
    L.qsa_check_bounded_wait.argtypes = [cp, vp, vp, ctypes.c_uint64, vp, sz, vp]
    L.qsa_check_bounded_wait.restype = ctypes.c_int
    L.qsa_device_error.argtypes = [vp, i32, vp]
    L.qsa_device_error.restype = i32
    L.qsa_set_profile_events.argtypes = [ctypes.POINTER(vp), i32]
    L.qsa_set_profile_events.restype = None
    L.qsa_decode_kernel_count.argtypes = [i32]
    L.qsa_decode_kernel_count.restype = i32
    L.qsa_status_string.argtypes = [ctypes.c_int]
    L.qsa_status_string.restype = ctypes.c_char_p
    L.qsa_version.restype = ctypes.c_char_p
    L.qsa_last_error_string.restype = ctypes.c_char_p
    for name in ("qsa_workspace_init", "qsa_compress_append", "qsa_index_score_topk", "qsa_expand_indices",
                 "qsa_sparse_gqa", "qsa_decode", "qsa_decode_indexshare"):
        getattr(L, name).restype = ctypes.c_int
    _lib = L
    return L


def _check(status: int, what: str):
    if status != 0:
        detail = f" [{lib().qsa_last_error_string().decode()}]" if status == 4 else ""
        raise QsaError(f"{what} failed: {lib().qsa_status_string(status).decode()} (status {status}){detail}")


def _ptr(t):
    if t is None:
        return None
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _dev(t: torch.Tensor, dtype, name: str, shape=None):
    if not t.is_cuda:
        raise QsaError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise QsaError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise QsaError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise QsaError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    return t


def version() -> str:
    return lib().qsa_version().decode()


def workspace_bytes(op: int, rows: int, max_len: int) -> int:
    return int(lib().qsa_workspace_bytes(op, rows, max_len))


class Workspace:
    """Caller-owned scratch memory (a torch uint8 CUDA tensor), zeroed once."""

    def __init__(self, nbytes: int, device="cuda"):
        self.nbytes = max(int(nbytes), 256)
        self.buf = torch.empty(self.nbytes + 256, dtype=torch.uint8, device=device)
        off = (-self.buf.data_ptr()) % 256
        self.t = self.buf[off:off + self.nbytes]
        _check(lib().qsa_workspace_init(_ptr(self.t), self.nbytes, _stream()), "qsa_workspace_init")

    @property
    def ptr(self):
        return _ptr(self.t)

    def device_error(self, clear: bool = True) -> int:
        return int(lib().qsa_device_error(self.ptr, 1 if clear else 0, _stream()))


class LayerCache:
    """The layer's paged cache: raw K/V pool, compressed index keys, ring and page table.

    k, v: bf16 [num_slots, 2, 128] views; cidx: bf16 [num_slots/4, 128]; ring: bf16 [batch, 4, 128];
    page_table: int32 [batch, max_pages].
    kv_layout "interleaved" keeps each slot's K and V rows together (kv: [num_slots, 2, 2, 128], k and
    v its two halves), so the 4 slots of a compressed block are one 4 KiB run; "separate" allocates
    two arrays.  kv_dtype "fp8" stores K and V as E4M3 codes (uint8 tensors of the same shapes; strides
    counted in bytes) for the *_fp8 calls.
    """

    def __init__(self, num_slots: int, batch: int, max_pages: int, rope_theta: float = 1.0e7, device="cuda",
                 page_table: torch.Tensor | None = None, kv_layout: str = "interleaved", kv_dtype: str = "bf16"):
        if num_slots % PAGE_SIZE:
            raise QsaError("num_slots must be a multiple of 64")
        if kv_layout not in ("interleaved", "separate"):
            raise QsaError(f"kv_layout must be 'interleaved' or 'separate', got {kv_layout!r}")
        self.num_slots, self.batch, self.max_pages, self.rope_theta = num_slots, batch, max_pages, rope_theta
        if kv_dtype not in ("bf16", "fp8"):
            raise QsaError(f"kv_dtype must be 'bf16' or 'fp8', got {kv_dtype!r}")
        self.kv_layout, self.kv_dtype = kv_layout, kv_dtype
        dt = torch.bfloat16 if kv_dtype == "bf16" else torch.uint8
        if kv_layout == "interleaved":
            self.kv = torch.zeros(num_slots, 2, KV_HEADS, HEAD_DIM, dtype=dt, device=device)
            self.k, self.v = self.kv[:, 0], self.kv[:, 1]
            self.kv_stride = 2 * KV_HEADS * HEAD_DIM
        else:
            self.k = torch.zeros(num_slots, KV_HEADS, HEAD_DIM, dtype=dt, device=device)
            self.v = torch.zeros(num_slots, KV_HEADS, HEAD_DIM, dtype=dt, device=device)
            self.kv_stride = 0
        self.cidx = torch.zeros(num_slots // BLOCK, HEAD_DIM, dtype=torch.bfloat16, device=device)
        self.ring = torch.zeros(max(batch, 1), BLOCK, HEAD_DIM, dtype=torch.bfloat16, device=device)
        if page_table is None:
            page_table = torch.full((max(batch, 1), max_pages), -1, dtype=torch.int32, device=device)
        self.page_table = _dev(page_table, torch.int32, "page_table")

    def struct(self, batch: int | None = None) -> CacheStruct:
        return CacheStruct(self.k.data_ptr(), self.v.data_ptr(), self.cidx.data_ptr(), self.ring.data_ptr(),
                           self.page_table.data_ptr(), self.num_slots, PAGE_SIZE, self.max_pages,
                           self.batch if batch is None else batch, self.kv_stride, self.rope_theta)


def compress_append(cache: LayerCache, idx_k_new, cu_new, len_before, max_new: int, stream=None):
    c = cache.struct()
    total = int(idx_k_new.shape[0]) if idx_k_new is not None else 0
    if total:
        _dev(idx_k_new, torch.bfloat16, "idx_k_new", (total, HEAD_DIM))
    _dev(cu_new, torch.int32, "cu_new", (cache.batch + 1,))
    _dev(len_before, torch.int32, "len_before", (cache.batch,))
    _check(lib().qsa_compress_append(ctypes.byref(c), _ptr(idx_k_new) if total else None, _ptr(cu_new),
                                     _ptr(len_before), total, int(max_new), _stream(stream)), "qsa_compress_append")


def index_score_topk(cache: LayerCache, idx_q, w, q_req, q_pos, max_len: int, ws: Workspace, blocks=None,
                     nblocks=None, stream=None):
    nq = int(q_pos.shape[0])
    dev = q_pos.device
    if blocks is None:
        blocks = torch.full((nq, TOPK), -1, dtype=torch.int32, device=dev)
    if nblocks is None:
        nblocks = torch.zeros(nq, dtype=torch.int32, device=dev)
    c = cache.struct()
    _dev(blocks, torch.int32, "blocks", (nq, TOPK))
    _dev(nblocks, torch.int32, "nblocks", (nq,))
    _check(lib().qsa_index_score_topk(ctypes.byref(c), _ptr(_dev(idx_q, torch.bfloat16, "idx_q", (nq, INDEX_HEADS, HEAD_DIM))),
                                      _ptr(_dev(w, torch.float32, "w", (nq, INDEX_HEADS))),
                                      _ptr(_dev(q_req, torch.int32, "q_req", (nq,))),
                                      _ptr(_dev(q_pos, torch.int32, "q_pos", (nq,))), nq, int(max_len), _ptr(blocks),
                                      _ptr(nblocks), ws.ptr, ws.nbytes, _stream(stream)), "qsa_index_score_topk")
    return blocks, nblocks


def prefill_score_topk(cache: LayerCache, idx_q, w, req: int, pos0: int, ws: Workspace, blocks=None, nblocks=None,
                       stream=None):
    """Tensor-core scoring + top-512 of the causal chunk of queries at positions pos0 .. pos0+T-1."""
    T = int(idx_q.shape[0])
    dev = idx_q.device
    if blocks is None:
        blocks = torch.full((T, TOPK), -1, dtype=torch.int32, device=dev)
    if nblocks is None:
        nblocks = torch.zeros(T, dtype=torch.int32, device=dev)
    c = cache.struct()
    _dev(blocks, torch.int32, "blocks", (T, TOPK))
    _dev(nblocks, torch.int32, "nblocks", (T,))
    _check(lib().qsa_prefill_score_topk(ctypes.byref(c), _ptr(_dev(idx_q, torch.bfloat16, "idx_q", (T, INDEX_HEADS, HEAD_DIM))),
                                        _ptr(_dev(w, torch.float32, "w", (T, INDEX_HEADS))), int(req), int(pos0), T, _ptr(blocks),
                                        _ptr(nblocks), ws.ptr, ws.nbytes, _stream(stream)), "qsa_prefill_score_topk")
    return blocks, nblocks


def prefill_score_topk_varlen(cache: LayerCache, idx_q, w, seg_req, seg_pos0, cu_q, max_len: int, ws: Workspace,
                              blocks=None, nblocks=None, stream=None):
    """Tensor-core scoring + top-512 of a ragged batch of causal chunks: segment i is request seg_req[i],
    queries at positions seg_pos0[i] .. + (cu_q[i+1] - cu_q[i]) - 1, rows cu_q[i] .. cu_q[i+1]-1 of
    idx_q / w / blocks / nblocks.  seg_req, seg_pos0, cu_q are host sequences."""
    import numpy as np

    nseg = len(seg_req)
    req = np.ascontiguousarray(seg_req, dtype=np.int32)
    pos0 = np.ascontiguousarray(seg_pos0, dtype=np.int32)
    cu = np.ascontiguousarray(cu_q, dtype=np.int32)
    if len(pos0) != nseg or len(cu) != nseg + 1:
        raise QsaError("seg_req, seg_pos0 need nseg entries and cu_q nseg + 1")
    T = int(cu[-1])
    dev = idx_q.device
    blocks = torch.full((T, TOPK), -1, dtype=torch.int32, device=dev) if blocks is None else blocks
    nblocks = torch.zeros(T, dtype=torch.int32, device=dev) if nblocks is None else nblocks
    c = cache.struct()
    _dev(blocks, torch.int32, "blocks", (T, TOPK))
    _dev(nblocks, torch.int32, "nblocks", (T,))
    _check(lib().qsa_prefill_score_topk_varlen(
        ctypes.byref(c), _ptr(_dev(idx_q, torch.bfloat16, "idx_q", (T, INDEX_HEADS, HEAD_DIM))),
        _ptr(_dev(w, torch.float32, "w", (T, INDEX_HEADS))), nseg, req.ctypes.data_as(ctypes.c_void_p),
        pos0.ctypes.data_as(ctypes.c_void_p), cu.ctypes.data_as(ctypes.c_void_p), int(max_len), _ptr(blocks),
        _ptr(nblocks), ws.ptr, ws.nbytes, _stream(stream)), "qsa_prefill_score_topk_varlen")
    return blocks, nblocks


def prefill_rescored_rows(ws: Workspace, T: int, max_len: int, stream=None) -> int:
    """Rows of the last prefill_score_topk call on `ws` that were re-scored in full (synchronises)."""
    return int(lib().qsa_prefill_rescored_rows(ws.ptr, int(T), int(max_len), _stream(stream)))


def prefill_rotated_queries(ws: Workspace, T: int, max_len: int, stream=None):
    """The rotated index queries of the last prefill_score_topk call on `ws`: uint16 bf16 bits [T][4][128]
    (synchronises)."""
    import numpy as np

    out = np.empty((int(T), 4, 128), dtype=np.uint16)
    _check(lib().qsa_prefill_rotated_queries(ws.ptr, int(T), int(max_len), out.ctypes.data, _stream(stream)),
           "qsa_prefill_rotated_queries")
    return out


def expand_indices(blocks, nblocks, q_pos, pos=None, npos=None, stream=None):
    nq = int(q_pos.shape[0])
    dev = q_pos.device
    if pos is None:
        pos = torch.full((nq, MAX_SEL), -1, dtype=torch.int32, device=dev)
    if npos is None:
        npos = torch.zeros(nq, dtype=torch.int32, device=dev)
    _dev(blocks, torch.int32, "blocks", (nq, TOPK))
    _dev(nblocks, torch.int32, "nblocks", (nq,))
    _dev(q_pos, torch.int32, "q_pos", (nq,))
    _dev(pos, torch.int32, "pos", (nq, MAX_SEL))
    _dev(npos, torch.int32, "npos", (nq,))
    _check(lib().qsa_expand_indices(_ptr(blocks), _ptr(nblocks), _ptr(q_pos), nq, _ptr(pos), _ptr(npos),
                                    _stream(stream)), "qsa_expand_indices")
    return pos, npos


def sparse_gqa(cache: LayerCache, q, q_req, pos, npos, max_pos: int, ws: Workspace, scale: float | None = None,
               out=None, lse=None, stream=None):
    nq = int(q.shape[0])
    scale = HEAD_DIM ** -0.5 if scale is None else scale
    if out is None:
        out = torch.empty(nq, Q_HEADS, HEAD_DIM, dtype=torch.bfloat16, device=q.device)
    c = cache.struct()
    _dev(out, torch.bfloat16, "out", (nq, Q_HEADS, HEAD_DIM))
    if lse is not None:
        _dev(lse, torch.float32, "lse", (nq, Q_HEADS))
    _check(lib().qsa_sparse_gqa(ctypes.byref(c), _ptr(_dev(q, torch.bfloat16, "q", (nq, Q_HEADS, HEAD_DIM))),
                                _ptr(_dev(q_req, torch.int32, "q_req", (nq,))), _ptr(_dev(pos, torch.int32, "pos")),
                                _ptr(_dev(npos, torch.int32, "npos", (nq,))), int(pos.shape[1]), int(max_pos), nq,
                                float(scale), _ptr(out), _ptr(lse), ws.ptr, ws.nbytes, _stream(stream)),
           "qsa_sparse_gqa")
    return out


def _need_fp8(cache: LayerCache, name: str):
    if cache.kv_dtype != "fp8":
        raise QsaError(f"{name} needs a cache with kv_dtype='fp8'")


def sparse_gqa_fp8(cache: LayerCache, q, q_req, pos, npos, max_pos: int, ws: Workspace, k_scale: float,
                   v_scale: float, scale: float | None = None, out=None, lse=None, stream=None):
    """qsa_sparse_gqa over an FP8 (E4M3) K/V pool: value = code * k_scale (keys), code * v_scale (values)."""
    _need_fp8(cache, "sparse_gqa_fp8")
    nq = int(q.shape[0])
    scale = HEAD_DIM ** -0.5 if scale is None else scale
    out = torch.empty(nq, Q_HEADS, HEAD_DIM, dtype=torch.bfloat16, device=q.device) if out is None else out
    c = cache.struct()
    _dev(out, torch.bfloat16, "out", (nq, Q_HEADS, HEAD_DIM))
    if lse is not None:
        _dev(lse, torch.float32, "lse", (nq, Q_HEADS))
    _check(lib().qsa_sparse_gqa_fp8(ctypes.byref(c), float(k_scale), float(v_scale),
                                    _ptr(_dev(q, torch.bfloat16, "q", (nq, Q_HEADS, HEAD_DIM))),
                                    _ptr(_dev(q_req, torch.int32, "q_req", (nq,))), _ptr(_dev(pos, torch.int32, "pos")),
                                    _ptr(_dev(npos, torch.int32, "npos", (nq,))), int(pos.shape[1]), int(max_pos), nq,
                                    float(scale), _ptr(out), _ptr(lse), ws.ptr, ws.nbytes, _stream(stream)),
           "qsa_sparse_gqa_fp8")
    return out


def decode_fp8(cache: LayerCache, idx_k_new, idx_q, w, q, seq_len, max_len: int, ws: Workspace, k_scale: float,
               v_scale: float, scale: float | None = None, out=None, lse=None, blocks_out=None, nblocks_out=None,
               stream=None):
    """qsa_decode over an FP8 (E4M3) K/V pool."""
    _need_fp8(cache, "decode_fp8")
    B = cache.batch
    scale = HEAD_DIM ** -0.5 if scale is None else scale
    out = torch.empty(B, Q_HEADS, HEAD_DIM, dtype=torch.bfloat16, device=q.device) if out is None else out
    c = cache.struct()
    _dev(out, torch.bfloat16, "out", (B, Q_HEADS, HEAD_DIM))
    if lse is not None:
        _dev(lse, torch.float32, "lse", (B, Q_HEADS))
    if blocks_out is not None:
        _dev(blocks_out, torch.int32, "blocks_out", (B, TOPK))
        _dev(nblocks_out, torch.int32, "nblocks_out", (B,))
    _check(lib().qsa_decode_fp8(ctypes.byref(c), float(k_scale), float(v_scale),
                                _ptr(_dev(idx_k_new, torch.bfloat16, "idx_k_new", (B, HEAD_DIM))),
                                _ptr(_dev(idx_q, torch.bfloat16, "idx_q", (B, INDEX_HEADS, HEAD_DIM))),
                                _ptr(_dev(w, torch.float32, "w", (B, INDEX_HEADS))),
                                _ptr(_dev(q, torch.bfloat16, "q", (B, Q_HEADS, HEAD_DIM))),
                                _ptr(_dev(seq_len, torch.int32, "seq_len", (B,))), int(max_len), float(scale),
                                _ptr(out), _ptr(lse), _ptr(blocks_out), _ptr(nblocks_out), ws.ptr, ws.nbytes,
                                _stream(stream)), "qsa_decode_fp8")
    return out


def sparse_gqa_noalloc(cache: LayerCache, q, q_req, pos, npos, max_pos: int, scale: float | None = None,
                       out=None, lse=None, stream=None):
    """qsa_sparse_gqa without a workspace, for callers that cannot allocate device memory (a plugin that
    is handed only its input and output buffers, code running during CUDA-graph capture, a fixed
    device-memory budget).  Scratch is the library's own static device array (about 4.1 MiB per GPU);
    nq is limited to 4096; calls that overlap on the GPU share that array and race."""
    nq = int(q.shape[0])
    scale = HEAD_DIM ** -0.5 if scale is None else scale
    if out is None:
        out = torch.empty(nq, Q_HEADS, HEAD_DIM, dtype=torch.bfloat16, device=q.device)
    c = cache.struct()
    _dev(out, torch.bfloat16, "out", (nq, Q_HEADS, HEAD_DIM))
    if lse is not None:
        _dev(lse, torch.float32, "lse", (nq, Q_HEADS))
    _check(lib().qsa_sparse_gqa_noalloc(ctypes.byref(c), _ptr(_dev(q, torch.bfloat16, "q", (nq, Q_HEADS, HEAD_DIM))),
                                        _ptr(_dev(q_req, torch.int32, "q_req", (nq,))), _ptr(_dev(pos, torch.int32, "pos")),
                                        _ptr(_dev(npos, torch.int32, "npos", (nq,))), int(pos.shape[1]), int(max_pos), nq,
                                        float(scale), _ptr(out), _ptr(lse), _stream(stream)),
           "qsa_sparse_gqa_noalloc")
    return out


def decode(cache: LayerCache, idx_k_new, idx_q, w, q, seq_len, max_len: int, ws: Workspace,
           scale: float | None = None, out=None, lse=None, blocks_out=None, nblocks_out=None, stream=None):
    B = cache.batch
    scale = HEAD_DIM ** -0.5 if scale is None else scale
    if out is None:
        out = torch.empty(B, Q_HEADS, HEAD_DIM, dtype=torch.bfloat16, device=q.device)
    c = cache.struct()
    _dev(out, torch.bfloat16, "out", (B, Q_HEADS, HEAD_DIM))
    if lse is not None:
        _dev(lse, torch.float32, "lse", (B, Q_HEADS))
    if blocks_out is not None:
        _dev(blocks_out, torch.int32, "blocks_out", (B, TOPK))
        _dev(nblocks_out, torch.int32, "nblocks_out", (B,))
    _check(lib().qsa_decode(ctypes.byref(c), _ptr(_dev(idx_k_new, torch.bfloat16, "idx_k_new", (B, HEAD_DIM))),
                            _ptr(_dev(idx_q, torch.bfloat16, "idx_q", (B, INDEX_HEADS, HEAD_DIM))),
                            _ptr(_dev(w, torch.float32, "w", (B, INDEX_HEADS))),
                            _ptr(_dev(q, torch.bfloat16, "q", (B, Q_HEADS, HEAD_DIM))),
                            _ptr(_dev(seq_len, torch.int32, "seq_len", (B,))),
                            int(max_len), float(scale), _ptr(out), _ptr(lse), _ptr(blocks_out), _ptr(nblocks_out),
                            ws.ptr, ws.nbytes, _stream(stream)), "qsa_decode")
    return out


def decode_indexshare(cache: LayerCache, frozen_pos, frozen_n, len0, q, ws: Workspace, scale: float | None = None,
                      out=None, stream=None):
    B, n_plus_1 = int(q.shape[0]), int(q.shape[1])
    scale = HEAD_DIM ** -0.5 if scale is None else scale
    if out is None:
        out = torch.empty(B, n_plus_1, Q_HEADS, HEAD_DIM, dtype=torch.bfloat16, device=q.device)
    c = cache.struct()
    if B != cache.batch:
        raise QsaError(f"q must have one row per request ({cache.batch}), got {B}")
    _dev(out, torch.bfloat16, "out", (B, n_plus_1, Q_HEADS, HEAD_DIM))
    _check(lib().qsa_decode_indexshare(ctypes.byref(c), _ptr(_dev(frozen_pos, torch.int32, "frozen_pos")),
                                       _ptr(_dev(frozen_n, torch.int32, "frozen_n", (B,))), int(frozen_pos.shape[1]),
                                       _ptr(_dev(len0, torch.int32, "len0", (B,))), n_plus_1,
                                       _ptr(_dev(q, torch.bfloat16, "q")), float(scale), _ptr(out), ws.ptr,
                                       ws.nbytes, _stream(stream)), "qsa_decode_indexshare")
    return out


def index_project(x, w_proj, idx_q=None, idx_k=None, w=None, stream=None):
    """Hidden states x [n, hidden] -> (idx_q [n,4,128] bf16, idx_k [n,128] bf16, w [n,4] f32)."""
    n, hidden = int(x.shape[0]), int(x.shape[1])
    dev = x.device
    _dev(x, torch.bfloat16, "x", (n, hidden))
    _dev(w_proj, torch.bfloat16, "w_proj", (PROJ_FEATURES, hidden))
    idx_q = torch.empty(n, INDEX_HEADS, HEAD_DIM, dtype=torch.bfloat16, device=dev) if idx_q is None else idx_q
    idx_k = torch.empty(n, HEAD_DIM, dtype=torch.bfloat16, device=dev) if idx_k is None else idx_k
    w = torch.empty(n, INDEX_HEADS, dtype=torch.float32, device=dev) if w is None else w
    _dev(idx_q, torch.bfloat16, "idx_q", (n, INDEX_HEADS, HEAD_DIM))
    _dev(idx_k, torch.bfloat16, "idx_k", (n, HEAD_DIM))
    _dev(w, torch.float32, "w", (n, INDEX_HEADS))
    _check(lib().qsa_index_project(_ptr(x), _ptr(w_proj), n, hidden, _ptr(idx_q), _ptr(idx_k), _ptr(w),
                                   _stream(stream)), "qsa_index_project")
    return idx_q, idx_k, w


def decode_indexer(cache: LayerCache, x, w_proj, seq_len, max_len: int, ws: Workspace, blocks=None, nblocks=None,
                   stream=None):
    """Index phase of a decode step from the new tokens' hidden states: projection, append, scoring,
    top-512.  Returns (blocks [B,512], nblocks [B])."""
    B = cache.batch
    hidden = int(x.shape[1])
    dev = x.device
    blocks = torch.full((B, TOPK), -1, dtype=torch.int32, device=dev) if blocks is None else blocks
    nblocks = torch.zeros(B, dtype=torch.int32, device=dev) if nblocks is None else nblocks
    c = cache.struct()
    _dev(blocks, torch.int32, "blocks", (B, TOPK))
    _dev(nblocks, torch.int32, "nblocks", (B,))
    _check(lib().qsa_decode_indexer(ctypes.byref(c), _ptr(_dev(x, torch.bfloat16, "x", (B, hidden))),
                                    _ptr(_dev(w_proj, torch.bfloat16, "w_proj", (PROJ_FEATURES, hidden))), hidden,
                                    _ptr(_dev(seq_len, torch.int32, "seq_len", (B,))), int(max_len), _ptr(blocks),
                                    _ptr(nblocks), ws.ptr, ws.nbytes, _stream(stream)), "qsa_decode_indexer")
    return blocks, nblocks


def decode_attend(cache: LayerCache, q, seq_len, max_len: int, blocks, nblocks, ws: Workspace,
                  scale: float | None = None, out=None, lse=None, stream=None):
    """Attention phase of a decode step over the indexer's kept blocks plus each request's tail."""
    B = cache.batch
    scale = HEAD_DIM ** -0.5 if scale is None else scale
    out = torch.empty(B, Q_HEADS, HEAD_DIM, dtype=torch.bfloat16, device=q.device) if out is None else out
    c = cache.struct()
    _dev(out, torch.bfloat16, "out", (B, Q_HEADS, HEAD_DIM))
    if lse is not None:
        _dev(lse, torch.float32, "lse", (B, Q_HEADS))
    _check(lib().qsa_decode_attend(ctypes.byref(c), _ptr(_dev(q, torch.bfloat16, "q", (B, Q_HEADS, HEAD_DIM))),
                                   _ptr(_dev(seq_len, torch.int32, "seq_len", (B,))), int(max_len),
                                   _ptr(_dev(blocks, torch.int32, "blocks", (B, TOPK))),
                                   _ptr(_dev(nblocks, torch.int32, "nblocks", (B,))), float(scale), _ptr(out),
                                   _ptr(lse), ws.ptr, ws.nbytes, _stream(stream)), "qsa_decode_attend")
    return out


def check_bounded_wait(cache: LayerCache, q, out, limit_ns: int, ws: Workspace, stream=None):
    """Launch the decode attention for request 0 with a selection nothing publishes and a wait limit of
    `limit_ns`: the kernel gives up, records the timeout bit in ws's error word and writes zeros to `out`."""
    c = cache.struct()
    _dev(q, torch.bfloat16, "q", (Q_HEADS, HEAD_DIM))
    _dev(out, torch.bfloat16, "out", (Q_HEADS, HEAD_DIM))
    _check(lib().qsa_check_bounded_wait(ctypes.byref(c), _ptr(q), _ptr(out), int(limit_ns), ws.ptr, ws.nbytes,
                                        _stream(stream)), "qsa_check_bounded_wait")
    return out


def set_profile_events(events):
    """events: list of torch.cuda.Event (2 per kernel: start, end), or None to switch off."""
    if not events:
        lib().qsa_set_profile_events(None, 0)
        return
    arr = (ctypes.c_void_p * len(events))(*[e.cuda_event for e in events])
    lib().qsa_set_profile_events(arr, len(events) // 2)


def decode_kernel_count(batch: int) -> int:
    """Kernels one qsa_decode call launches for `batch` requests."""
    return int(lib().qsa_decode_kernel_count(int(batch)))


class PackedInputs:
    """A decode step's inputs as 256-byte-aligned views of one contiguous buffer, so that a step
    moves them host -> device with a single copy.  `views` maps each input name to its tensor."""

    ALIGN = 256

    def __init__(self, specs, device=None, pin_memory: bool = False):
        offs, off = {}, 0
        for name, shape, dtype in specs:
            nbytes = int(torch.Size(shape).numel()) * torch.empty((), dtype=dtype).element_size()
            offs[name] = (off, shape, dtype, nbytes)
            off += (nbytes + self.ALIGN - 1) // self.ALIGN * self.ALIGN
        self.nbytes = off
        self.buf = torch.empty(off, dtype=torch.uint8, device=device, pin_memory=pin_memory)
        self.views = {name: self.buf[o:o + n].view(dt).view(sh) for name, (o, sh, dt, n) in offs.items()}
        self.payload_bytes = sum(n for (_, _, _, n) in offs.values())

    def copy_from(self, other: "PackedInputs", non_blocking: bool = True):
        self.buf.copy_(other.buf, non_blocking=non_blocking)


class DecodeSession:
    """Decode steps fed from host memory: the call a serving loop makes once per step.

    step() copies the step's inputs from a pinned host buffer to a device staging buffer (one
    copy: both hold the inputs packed the same way), runs qsa_decode, and copies the attention
    output back to a pinned host tensor, all on one stream.
    """

    INPUTS = ("idx_k_new", "idx_q", "w", "q", "seq_len")

    @staticmethod
    def input_specs(B: int):
        bf = torch.bfloat16
        return [("idx_k_new", (B, HEAD_DIM), bf), ("idx_q", (B, INDEX_HEADS, HEAD_DIM), bf),
                ("w", (B, INDEX_HEADS), torch.float32), ("q", (B, Q_HEADS, HEAD_DIM), bf),
                ("seq_len", (B,), torch.int32)]

    def __init__(self, cache: LayerCache, max_len: int, device="cuda"):
        B = cache.batch
        self.cache, self.max_len = cache, int(max_len)
        self.ws = Workspace(workspace_bytes(OP_DECODE, B, self.max_len), device=device)
        self.staging = PackedInputs(self.input_specs(B), device=device)
        self.dev = self.staging.views
        self.out = torch.empty(B, Q_HEADS, HEAD_DIM, dtype=torch.bfloat16, device=device)
        self.host_out = torch.empty(B, Q_HEADS, HEAD_DIM, dtype=torch.bfloat16, pin_memory=True)

    @staticmethod
    def pinned_inputs(device_inputs: dict) -> PackedInputs:
        """The step's inputs packed into one pinned host buffer (what step() takes)."""
        B = int(device_inputs["seq_len"].shape[0])
        host = PackedInputs(DecodeSession.input_specs(B), pin_memory=True)
        for k in DecodeSession.INPUTS:
            host.views[k].copy_(device_inputs[k].cpu())
        return host

    def h2d_bytes(self) -> int:
        return self.staging.payload_bytes

    def d2h_bytes(self) -> int:
        return self.host_out.numel() * self.host_out.element_size()

    def step(self, host_inputs: PackedInputs, stream=None) -> torch.Tensor:
        """One step on `stream` (default: the current stream): both copies and the decode are enqueued
        on that one stream, in order.  The returned pinned tensor is valid once the stream is done."""
        if host_inputs.nbytes != self.staging.nbytes:
            raise QsaError("host inputs were packed for another batch size")
        st = torch.cuda.current_stream() if stream is None else stream
        with torch.cuda.stream(st):
            self.staging.copy_from(host_inputs)
            decode(self.cache, self.dev["idx_k_new"], self.dev["idx_q"], self.dev["w"], self.dev["q"],
                   self.dev["seq_len"], self.max_len, self.ws, out=self.out, stream=st)
            self.host_out.copy_(self.out, non_blocking=True)
        return self.host_out
