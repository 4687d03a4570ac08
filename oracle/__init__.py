"""CPU oracle for one QSA (c4) layer -- TEST INFRASTRUCTURE ONLY.

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product library never does, and the
two share no code; they meet only through the seeded inputs of ``qsa_gen``.

The arithmetic lives in ``qsa_oracle.cpp`` (plain C++, FP64 except the FP32
4-key average that the QSA description fixes); this module compiles it with
g++ and wraps it with numpy arrays.  See the header of the C++ file for the
method, its source sections and every reading taken where the text is silent.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "qsa_oracle.cpp")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lib = None

D, HI, HQ, HKV, C, TOPK = 128, 4, 16, 2, 4, 512
MAX_POS = TOPK * C + C - 1  # 2051
SCALE = 1.0 / np.sqrt(128.0)


def build(force: bool = False) -> str:
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["g++", "-O2", "-std=c++17", "-fPIC", "-shared", "-pthread", _SRC, "-o", tmp])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def threads() -> int:
    return max(1, os.cpu_count() or 1)


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB_PATH)
        vp, i64, i32, f64 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_double
        L.oracle_version.restype = ctypes.c_int
        L.oracle_f64_to_bf16.argtypes = [f64]
        L.oracle_f64_to_bf16.restype = ctypes.c_uint16
        L.oracle_rope_f64.argtypes = [vp, vp, i64, f64, vp]
        L.oracle_compress_block.argtypes = [vp, i64, f64, vp]
        L.oracle_compress.argtypes = [vp, i64, f64, vp, ctypes.c_int]
        L.oracle_append.argtypes = [vp, vp, vp, i64, f64]
        L.oracle_rotate_query.argtypes = [vp, ctypes.c_int, i64, f64, vp]
        L.oracle_block_scores.argtypes = [vp, vp, vp, i64, vp]
        L.oracle_select_topk.argtypes = [vp, i64, i32, vp]
        L.oracle_select_topk.restype = i32
        L.oracle_expand.argtypes = [vp, i32, i64, vp]
        L.oracle_expand.restype = i32
        L.oracle_sparse_gqa.argtypes = [vp, vp, vp, vp, i32, f64, vp, vp]
        L.oracle_select_query.argtypes = [vp, vp, vp, i64, f64, vp, vp, vp, vp]
        L.oracle_select_query.restype = i32
        L.oracle_decode_batch.argtypes = [i32, vp, vp, vp, vp, vp, vp, vp, vp, vp, f64, f64, vp, vp, vp, vp, vp,
                                          ctypes.c_int]
        L.oracle_prefill_rows.argtypes = [vp, i64, vp, vp, vp, vp, vp, vp, f64, f64, vp, vp, vp, vp, ctypes.c_int]
        L.oracle_indexshare.argtypes = [vp, i32, i64, i32, vp, vp, vp, f64, vp]
        L.oracle_e4m3_to_f64.argtypes = [ctypes.c_uint8]
        L.oracle_e4m3_to_f64.restype = f64
        L.oracle_sparse_gqa_fp8.argtypes = [vp, vp, vp, f64, f64, vp, i32, f64, vp, vp]
        L.oracle_sparse_gqa_fp8.restype = None
        L.oracle_index_project.argtypes = [vp, vp, i64, i64, vp, vp, vp, ctypes.c_int]
        for name in ("oracle_rope_f64", "oracle_compress_block", "oracle_compress", "oracle_append",
                     "oracle_rotate_query", "oracle_block_scores", "oracle_sparse_gqa", "oracle_decode_batch",
                     "oracle_prefill_rows", "oracle_indexshare", "oracle_index_project"):
            getattr(L, name).restype = None
        _lib = L
    return _lib


def _p(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return ctypes.c_void_p(a.ctypes.data)


def _u16(a) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=np.uint16)


# --- single steps --------------------------------------------------------------

def f64_to_bf16(x: float) -> int:
    return int(lib().oracle_f64_to_bf16(float(x)))


def rope(x: np.ndarray, pos, theta: float = 1e7) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float64).reshape(-1, D)
    pos = np.ascontiguousarray(np.broadcast_to(np.asarray(pos, dtype=np.float64), (x.shape[0],)))
    y = np.empty_like(x)
    lib().oracle_rope_f64(_p(x), _p(pos), x.shape[0], theta, _p(y))
    return y


def compress_block(raw4: np.ndarray, b: int, theta: float = 1e7) -> np.ndarray:
    raw4 = _u16(raw4).reshape(C, D)
    out = np.empty(D, dtype=np.uint16)
    lib().oracle_compress_block(_p(raw4), b, theta, _p(out))
    return out


def compress(raw: np.ndarray, theta: float = 1e7, nthreads: int | None = None) -> np.ndarray:
    raw = _u16(raw).reshape(-1, D)
    nb = raw.shape[0] // C
    out = np.empty((nb, D), dtype=np.uint16)
    if nb:
        lib().oracle_compress(_p(raw), raw.shape[0], theta, _p(out), nthreads or threads())
    return out


def append(ring: np.ndarray, comp: np.ndarray, key: np.ndarray, pos: int, theta: float = 1e7) -> None:
    """In place: ring [4,128] and comp [nb_cap,128] (uint16, C-contiguous)."""
    key = _u16(key).reshape(D)
    lib().oracle_append(_p(ring), _p(comp), _p(key), pos, theta)


def rotate_query(q: np.ndarray, pos: int, theta: float = 1e7) -> np.ndarray:
    q = _u16(q).reshape(-1, D)
    out = np.empty_like(q)
    lib().oracle_rotate_query(_p(q), q.shape[0], pos, theta, _p(out))
    return out


def block_scores(qrot: np.ndarray, w: np.ndarray, comp: np.ndarray, nb: int | None = None) -> np.ndarray:
    qrot = _u16(qrot).reshape(HI, D)
    w = np.ascontiguousarray(w, dtype=np.float32).reshape(HI)
    comp = _u16(comp).reshape(-1, D)
    nb = comp.shape[0] if nb is None else nb
    s = np.empty(max(nb, 1), dtype=np.float64)
    lib().oracle_block_scores(_p(qrot), _p(w), _p(comp), nb, _p(s))
    return s[:nb]


def select_topk(s: np.ndarray, k: int = TOPK) -> np.ndarray:
    s = np.ascontiguousarray(s, dtype=np.float64)
    out = np.empty(max(min(len(s), k), 1), dtype=np.int32)
    n = lib().oracle_select_topk(_p(s), len(s), k, _p(out))
    return out[:n]


def expand(blocks: np.ndarray, L: int) -> np.ndarray:
    blocks = np.ascontiguousarray(blocks, dtype=np.int32)
    out = np.empty(len(blocks) * C + C, dtype=np.int32)
    n = lib().oracle_expand(_p(blocks), len(blocks), L, _p(out))
    return out[:n]


def sparse_gqa(q: np.ndarray, K: np.ndarray, V: np.ndarray, pos: np.ndarray, scale: float = SCALE):
    """q [16,128] bf16 bits; K, V [T,2,128] bf16 bits (logical); pos int32 -> (out [16,128] f64, lse [16])."""
    q = _u16(q).reshape(HQ, D)
    K = _u16(K)
    V = _u16(V)
    pos = np.ascontiguousarray(pos, dtype=np.int32)
    out = np.empty((HQ, D), dtype=np.float64)
    lse = np.empty(HQ, dtype=np.float64)
    lib().oracle_sparse_gqa(_p(q), _p(K), _p(V), _p(pos), len(pos), scale, _p(out), _p(lse))
    return out, lse


def e4m3_to_f64(b: int) -> float:
    return float(lib().oracle_e4m3_to_f64(int(b)))


def sparse_gqa_fp8(q: np.ndarray, K8: np.ndarray, V8: np.ndarray, k_scale: float, v_scale: float, pos: np.ndarray,
                   scale: float = SCALE):
    """q [16,128] bf16 bits; K8, V8 [T,2,128] E4M3 bytes (uint8, logical); pos int32 -> (out [16,128] f64, lse [16])."""
    q = _u16(q).reshape(HQ, D)
    K8 = np.ascontiguousarray(K8, dtype=np.uint8)
    V8 = np.ascontiguousarray(V8, dtype=np.uint8)
    pos = np.ascontiguousarray(pos, dtype=np.int32)
    out = np.empty((HQ, D), dtype=np.float64)
    lse = np.empty(HQ, dtype=np.float64)
    lib().oracle_sparse_gqa_fp8(_p(q), _p(K8), _p(V8), float(k_scale), float(v_scale), _p(pos), len(pos), scale,
                                _p(out), _p(lse))
    return out, lse


def select_query(idx_q: np.ndarray, w: np.ndarray, comp: np.ndarray, L: int, theta: float = 1e7):
    """Selection of one query at position L-1 -> (blocks, positions, scores)."""
    idx_q = _u16(idx_q).reshape(HI, D)
    w = np.ascontiguousarray(w, dtype=np.float32).reshape(HI)
    comp = _u16(comp).reshape(-1, D)
    nb = L // C
    assert comp.shape[0] >= nb
    blocks = np.empty(TOPK, dtype=np.int32)
    nblocks = np.zeros(1, dtype=np.int32)
    pos = np.empty(MAX_POS, dtype=np.int32)
    scores = np.empty(max(nb, 1), dtype=np.float64)
    n = lib().oracle_select_query(_p(idx_q), _p(w), _p(comp), L, theta, _p(blocks), _p(nblocks), _p(pos), _p(scores))
    return blocks[:nblocks[0]].copy(), pos[:n].copy(), scores[:nb].copy()


# --- batched composites -----------------------------------------------------------

def _ptr_array(arrs):
    return (ctypes.c_void_p * len(arrs))(*[a.ctypes.data for a in arrs])


def decode_batch(L, ring, comp, new_key, idx_q, w, q, K, V, theta: float = 1e7, scale: float = SCALE,
                 nthreads: int | None = None):
    """One decode step over a batch.  Per-request lists of numpy arrays; ring/comp updated in place.
    Returns (out [B,16,128] f64, blocks list, positions list)."""
    B = len(L)
    Larr = np.ascontiguousarray(L, dtype=np.int64)
    ring = [_chk(a) for a in ring]
    comp = [_chk(a) for a in comp]
    new_key = [_u16(a) for a in new_key]
    idx_q = [_u16(a) for a in idx_q]
    w = [np.ascontiguousarray(a, dtype=np.float32) for a in w]
    q = [_u16(a) for a in q]
    K = [_u16(a) for a in K]
    V = [_u16(a) for a in V]
    out = [np.empty((HQ, D), dtype=np.float64) for _ in range(B)]
    blocks = [np.empty(TOPK, dtype=np.int32) for _ in range(B)]
    pos = [np.empty(MAX_POS, dtype=np.int32) for _ in range(B)]
    nblocks = np.zeros(max(B, 1), dtype=np.int32)
    npos = np.zeros(max(B, 1), dtype=np.int32)
    lib().oracle_decode_batch(B, _p(Larr), _ptr_array(ring), _ptr_array(comp), _ptr_array(new_key),
                              _ptr_array(idx_q), _ptr_array(w), _ptr_array(q), _ptr_array(K), _ptr_array(V), theta,
                              scale, _ptr_array(out), _ptr_array(blocks), _p(nblocks), _ptr_array(pos), _p(npos),
                              nthreads or threads())
    return (np.stack(out) if B else np.zeros((0, HQ, D)), [blocks[r][:nblocks[r]] for r in range(B)],
            [pos[r][:npos[r]] for r in range(B)])


def _chk(a: np.ndarray) -> np.ndarray:
    assert a.dtype == np.uint16 and a.flags["C_CONTIGUOUS"] and a.flags["WRITEABLE"]
    return a


def prefill_rows(rows, idx_q, w, q, comp, K, V, theta: float = 1e7, scale: float = SCALE, with_attention=True,
                 nthreads: int | None = None):
    """Rows (positions) of a causal prefill of one sequence -> (out [n,16,128] f64 | None, blocks list)."""
    rows = np.ascontiguousarray(rows, dtype=np.int64)
    n = len(rows)
    idx_q = _u16(idx_q)
    w = np.ascontiguousarray(w, dtype=np.float32)
    q = _u16(q) if with_attention else idx_q
    comp = _u16(comp)
    K = _u16(K) if with_attention else comp
    V = _u16(V) if with_attention else comp
    out = np.empty((max(n, 1), HQ, D), dtype=np.float64) if with_attention else None
    blocks = np.empty((max(n, 1), TOPK), dtype=np.int32)
    nblocks = np.zeros(max(n, 1), dtype=np.int32)
    npos = np.zeros(max(n, 1), dtype=np.int32)
    lib().oracle_prefill_rows(_p(rows), n, _p(idx_q), _p(w), _p(q), _p(comp), _p(K), _p(V), theta, scale,
                              _p(out) if out is not None else None, _p(blocks), _p(nblocks), _p(npos),
                              nthreads or threads())
    return (out[:n] if out is not None else None), [blocks[i, :nblocks[i]].copy() for i in range(n)]


PROJ_FEATURES = HI * D + D + HI  # 644


def index_project(x: np.ndarray, W: np.ndarray, nthreads: int | None = None):
    """x [n, hidden] and W [644, hidden] bf16 bits -> (idx_q [n,4,128] bits, idx_k [n,128] bits, w [n,4] f32)."""
    x = _u16(x)
    W = _u16(W)
    n, hidden = x.shape
    assert W.shape == (PROJ_FEATURES, hidden)
    idx_q = np.empty((n, HI, D), dtype=np.uint16)
    idx_k = np.empty((n, D), dtype=np.uint16)
    w = np.empty((n, HI), dtype=np.float32)
    if n:
        lib().oracle_index_project(_p(x), _p(W), n, hidden, _p(idx_q), _p(idx_k), _p(w), nthreads or threads())
    return idx_q, idx_k, w


def indexshare(frozen_pos: np.ndarray, L0: int, n_plus_1: int, q: np.ndarray, K: np.ndarray, V: np.ndarray,
               scale: float = SCALE) -> np.ndarray:
    frozen_pos = np.ascontiguousarray(frozen_pos, dtype=np.int32)
    q = _u16(q).reshape(n_plus_1, HQ, D)
    out = np.empty((n_plus_1, HQ, D), dtype=np.float64)
    lib().oracle_indexshare(_p(frozen_pos), len(frozen_pos), L0, n_plus_1, _p(q), _p(_u16(K)), _p(_u16(V)), scale,
                            _p(out))
    return out
