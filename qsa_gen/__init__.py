"""Seeded synthetic inputs for one QSA (c4) layer.

This package builds the inputs that both the CPU oracle and the CUDA path
consume.  It contains no arithmetic of the attention method: only the random
draws (see ``qsa_gen.c`` for the counter-based generator) and the recipes that
shape them like the workloads the QSA description talks about (paged BF16 K/V,
4 indexer heads x 128 dims, 16 query / 2 KV heads, contexts from 4K to 262K).

Every tensor of request ``r`` comes from its own counter stream
``(kind << 32) | r``, element ``i`` of the tensor from counter ``i``, so any
request (or any token range of it) can be regenerated alone, byte for byte.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass, field

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "qsa_gen.c")
_LIB_PATH = os.path.join(_HERE, "libqsagen.so")
_lib = None

HEAD_DIM = 128
INDEX_HEADS = 4
Q_HEADS = 16
KV_HEADS = 2
PAGE = 64

# stream kinds
K_IDXQ, K_W, K_IDXK, K_BIAS, K_Q, K_K, K_V, K_PAGES, K_LENS = 1, 2, 3, 4, 5, 6, 7, 8, 9
K_HIDDEN, K_WPROJ, K_K8, K_V8 = 10, 11, 12, 13


def _threads() -> int:
    return max(1, min(64, os.cpu_count() or 1))


def build(force: bool = False) -> str:
    """Compile the generator into ``libqsagen.so`` next to its source."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-D_GNU_SOURCE", "-fPIC", "-shared", "-pthread",
                               _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB_PATH)
        u64, i64, i32, f32, f64 = ctypes.c_uint64, ctypes.c_int64, ctypes.c_int, ctypes.c_float, ctypes.c_double
        vp = ctypes.c_void_p
        L.qsa_gen_normal_bf16.argtypes = [u64, u64, u64, i64, vp, i32]
        L.qsa_gen_normal_scaled_bf16.argtypes = [u64, u64, u64, i64, f64, vp, i32]
        L.qsa_gen_normal_scaled_bf16.restype = None
        L.qsa_gen_uniform_f32.argtypes = [u64, u64, u64, i64, f32, f32, vp]
        L.qsa_gen_uniform_i64.argtypes = [u64, u64, u64, i64, i64, i64, vp]
        L.qsa_gen_bernoulli_u8.argtypes = [u64, u64, u64, i64, f64, vp]
        L.qsa_gen_permutation_i32.argtypes = [u64, u64, i64, vp]
        L.qsa_gen_index_keys_bf16.argtypes = [u64, u64, u64, i64, i64, vp, f64, f64, vp, i32]
        L.qsa_gen_block_bias_u8.argtypes = [u64, u64, i64, i64, f64, vp]
        for f in (L.qsa_gen_normal_bf16, L.qsa_gen_uniform_f32, L.qsa_gen_uniform_i64, L.qsa_gen_bernoulli_u8,
                  L.qsa_gen_permutation_i32, L.qsa_gen_index_keys_bf16, L.qsa_gen_block_bias_u8):
            f.restype = None
        _lib = L
    return _lib


def stream(kind: int, r: int = 0) -> int:
    return (kind << 32) | r


def _ptr(a: np.ndarray):
    return ctypes.c_void_p(a.ctypes.data)


# --- primitives --------------------------------------------------------------

def normal_bf16(seed: int, strm: int, shape, offset: int = 0) -> np.ndarray:
    """N(0,1) values rounded once to bf16; returned as raw uint16 bits."""
    out = np.empty(shape, dtype=np.uint16)
    lib().qsa_gen_normal_bf16(seed, strm, offset, out.size, _ptr(out), _threads())
    return out


def normal_scaled_bf16(seed: int, strm: int, shape, std: float, offset: int = 0) -> np.ndarray:
    """N(0, std^2) values rounded once to bf16; raw uint16 bits."""
    out = np.empty(shape, dtype=np.uint16)
    lib().qsa_gen_normal_scaled_bf16(seed, strm, offset, out.size, float(std), _ptr(out), _threads())
    return out


def normal_fp8_e4m3(seed: int, strm: int, shape, std: float = 1.0, offset: int = 0) -> np.ndarray:
    """N(0, std^2) values of the stream (bf16 first), converted to E4M3 codes by torch's float8_e4m3fn
    conversion; raw uint8 codes."""
    import torch

    f = bf16_bits_to_f32(normal_scaled_bf16(seed, strm, shape, std, offset=offset))
    return torch.from_numpy(np.ascontiguousarray(f)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def uniform_f32(seed: int, strm: int, shape, lo: float = 0.0, hi: float = 1.0, offset: int = 0) -> np.ndarray:
    out = np.empty(shape, dtype=np.float32)
    lib().qsa_gen_uniform_f32(seed, strm, offset, out.size, lo, hi, _ptr(out))
    return out


def uniform_int(seed: int, strm: int, n: int, lo: int, hi: int) -> np.ndarray:
    out = np.empty(n, dtype=np.int64)
    lib().qsa_gen_uniform_i64(seed, strm, 0, n, lo, hi, _ptr(out))
    return out


def permutation(seed: int, strm: int, n: int) -> np.ndarray:
    out = np.empty(n, dtype=np.int32)
    lib().qsa_gen_permutation_i32(seed, strm, n, _ptr(out))
    return out


def index_keys_bf16(seed: int, r: int, n_tok: int, direction_bf16: np.ndarray | None, p: float = 0.05,
                    alpha: float = 0.5, tok0: int = 0) -> np.ndarray:
    """Raw index keys ``[n_tok, 128]`` (bf16 bits) of request ``r``, tokens tok0.., with the planted signal."""
    out = np.empty((n_tok, HEAD_DIM), dtype=np.uint16)
    d = None
    if direction_bf16 is not None:
        d = np.ascontiguousarray(direction_bf16, dtype=np.uint16).reshape(HEAD_DIM)
    lib().qsa_gen_index_keys_bf16(seed, stream(K_IDXK, r), stream(K_BIAS, r), tok0, n_tok,
                                  _ptr(d) if d is not None else None, p, alpha, _ptr(out), _threads())
    return out


def block_bias(seed: int, r: int, n_blocks: int, p: float = 0.05) -> np.ndarray:
    out = np.empty(n_blocks, dtype=np.uint8)
    lib().qsa_gen_block_bias_u8(seed, stream(K_BIAS, r), 0, n_blocks, p, _ptr(out))
    return out


def bf16_bits_to_f32(a: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bits to float32 (a bit shift, no rounding)."""
    return (a.astype(np.uint32) << 16).view(np.float32)


# --- workloads -----------------------------------------------------------------

@dataclass
class Workload:
    """A batch of requests of one QSA layer.

    ``lens[r]`` is the context length of request r *including* its newest
    token (decode: the query sits at position lens[r]-1).  ``extra[r]`` extra
    tokens of K/V exist after it (IndexShare draft positions).  ``nq[r]`` is
    the number of query tokens of request r: 1 for decode, lens[r] for a full
    prefill.  ``bias_from`` picks which query's head-0 index query is the planted
    direction of the index keys: "last" (the request's newest query).
    """

    name: str
    seed: int
    lens: np.ndarray
    kind: str = "decode"  # decode | prefill | indexshare
    extra: int = 0
    n_draft: int = 0
    p_bias: float = 0.05
    alpha: float = 0.5
    rope_theta: float = 1.0e7
    spare_pages: int = 0
    notes: str = ""
    _cache: dict = field(default_factory=dict, repr=False)

    @property
    def batch(self) -> int:
        return int(len(self.lens))

    def n_queries(self, r: int) -> int:
        return int(self.lens[r]) if self.kind == "prefill" else 1

    def tokens(self, r: int) -> int:
        """Tokens of K/V and raw index keys stored for request r."""
        return int(self.lens[r]) + self.extra

    # per-request tensors (bf16 bits as uint16 unless noted)
    def idx_q(self, r: int, q0: int = 0, n: int | None = None) -> np.ndarray:
        n = self.n_queries(r) if n is None else n
        return normal_bf16(self.seed, stream(K_IDXQ, r), (n, INDEX_HEADS, HEAD_DIM), offset=q0 * INDEX_HEADS * HEAD_DIM)

    def w(self, r: int, q0: int = 0, n: int | None = None) -> np.ndarray:
        n = self.n_queries(r) if n is None else n
        return uniform_f32(self.seed, stream(K_W, r), (n, INDEX_HEADS), offset=q0 * INDEX_HEADS)

    def q(self, r: int, q0: int = 0, n: int | None = None) -> np.ndarray:
        if n is None:
            n = self.n_queries(r) if self.kind != "indexshare" else self.n_draft + 1
        return normal_bf16(self.seed, stream(K_Q, r), (n, Q_HEADS, HEAD_DIM), offset=q0 * Q_HEADS * HEAD_DIM)

    def hidden(self, r: int, hidden: int, q0: int = 0, n: int | None = None) -> np.ndarray:
        """Hidden states [n, hidden] of request r's query tokens (bf16 bits, N(0,1)), the input of the
        index projection."""
        n = self.n_queries(r) if n is None else n
        return normal_bf16(self.seed, stream(K_HIDDEN, r), (n, hidden), offset=q0 * hidden)

    def k8(self, r: int, tok0: int = 0, n: int | None = None, std: float = 2.0) -> np.ndarray:
        """FP8 (E4M3) attention keys [n, 2, 128] of request r, N(0, std^2) in code units."""
        n = self.tokens(r) - tok0 if n is None else n
        return normal_fp8_e4m3(self.seed, stream(K_K8, r), (n, KV_HEADS, HEAD_DIM), std,
                               offset=tok0 * KV_HEADS * HEAD_DIM)

    def v8(self, r: int, tok0: int = 0, n: int | None = None, std: float = 4.0) -> np.ndarray:
        """FP8 (E4M3) attention values [n, 2, 128] of request r, N(0, std^2) in code units."""
        n = self.tokens(r) - tok0 if n is None else n
        return normal_fp8_e4m3(self.seed, stream(K_V8, r), (n, KV_HEADS, HEAD_DIM), std,
                               offset=tok0 * KV_HEADS * HEAD_DIM)

    def bias_direction(self, r: int) -> np.ndarray:
        nq = self.n_queries(r)
        return self.idx_q(r, q0=nq - 1, n=1)[0, 0]

    def idx_keys(self, r: int, tok0: int = 0, n: int | None = None) -> np.ndarray:
        n = self.tokens(r) - tok0 if n is None else n
        return index_keys_bf16(self.seed, r, n, self.bias_direction(r), self.p_bias, self.alpha, tok0=tok0)

    def k(self, r: int, tok0: int = 0, n: int | None = None) -> np.ndarray:
        n = self.tokens(r) - tok0 if n is None else n
        return normal_bf16(self.seed, stream(K_K, r), (n, KV_HEADS, HEAD_DIM), offset=tok0 * KV_HEADS * HEAD_DIM)

    def v(self, r: int, tok0: int = 0, n: int | None = None) -> np.ndarray:
        n = self.tokens(r) - tok0 if n is None else n
        return normal_bf16(self.seed, stream(K_V, r), (n, KV_HEADS, HEAD_DIM), offset=tok0 * KV_HEADS * HEAD_DIM)

    # paging
    def pages_needed(self, r: int) -> int:
        return (self.tokens(r) + PAGE - 1) // PAGE

    @property
    def max_pages(self) -> int:
        return max(self.pages_needed(r) for r in range(self.batch)) if self.batch else 0

    @property
    def total_pages(self) -> int:
        return sum(self.pages_needed(r) for r in range(self.batch)) + self.spare_pages

    def page_table(self) -> np.ndarray:
        """int32 [batch, max_pages]; logical page p of request r lives in physical page pt[r, p].
        Physical pages are a seeded permutation of all pages; unused entries are -1."""
        if "pt" not in self._cache:
            perm = permutation(self.seed, stream(K_PAGES), self.total_pages)
            pt = np.full((self.batch, max(1, self.max_pages)), -1, dtype=np.int32)
            off = 0
            for r in range(self.batch):
                n = self.pages_needed(r)
                pt[r, :n] = perm[off:off + n]
                off += n
            self._cache["pt"] = pt
        return self._cache["pt"]


PROJ_FEATURES = INDEX_HEADS * HEAD_DIM + HEAD_DIM + INDEX_HEADS  # 644


def projection_weights(seed: int, hidden: int) -> np.ndarray:
    """Index projection weights [644, hidden] ~ N(0, 1/hidden) (bf16 bits): rows 0..511 the 4 query
    heads, 512..639 the key, 640..643 the head weights."""
    return normal_scaled_bf16(seed, stream(K_WPROJ), (PROJ_FEATURES, hidden), hidden ** -0.5)


def _lens_uniform(seed: int, n: int, lo: int, hi: int) -> np.ndarray:
    return uniform_int(seed, stream(K_LENS), n, lo, hi).astype(np.int64)


def decode_small(seed: int = 0) -> Workload:
    """Decode, batch 4, contexts {4097, 6002, 8191, 8192} (tails 1, 2, 3, 0)."""
    return Workload("decode_b4_ctx4k-8k", seed, np.array([4097, 6002, 8191, 8192], dtype=np.int64))


def prefill_32k(seed: int = 1, L: int = 32768) -> Workload:
    """Prefill of one causal sequence of L tokens, every token a query."""
    return Workload(f"prefill_L{L}", seed, np.array([L], dtype=np.int64), kind="prefill")


def decode_128k(seed: int = 2, batch: int = 64) -> Workload:
    """Decode, batch 64, contexts uniform in [120000, 131072]: the memory-bound headline case."""
    return Workload(f"decode_b{batch}_ctx120k-128k", seed, _lens_uniform(seed, batch, 120000, 131072))


def indexshare_64k(seed: int = 3, batch: int = 16, n_draft: int = 3) -> Workload:
    """IndexShare draft step: capture at context L0 = 65536 + U[0,3], then n_draft+1 draft positions."""
    lens = _lens_uniform(seed, batch, 65536, 65539)
    return Workload(f"indexshare_b{batch}_ctx64k_n{n_draft}", seed, lens, kind="indexshare",
                    extra=n_draft + 1, n_draft=n_draft)


def long_262k(seed: int = 4) -> Workload:
    """Long context: one sequence of 262144 tokens plus 3 more (decode at 262144 and 262147)."""
    return Workload("long_L262144", seed, np.array([262147], dtype=np.int64), kind="prefill")


def custom_decode(seed: int, lens, extra: int = 0, p_bias: float = 0.05, alpha: float = 0.5,
                  spare_pages: int = 0) -> Workload:
    return Workload(f"decode_custom_{len(lens)}", seed, np.asarray(lens, dtype=np.int64), extra=extra,
                    p_bias=p_bias, alpha=alpha, spare_pages=spare_pages)


CONFIGS = {
    "decode_small": decode_small,
    "prefill_32k": prefill_32k,
    "decode_128k": decode_128k,
    "indexshare_64k": indexshare_64k,
    "long_262k": long_262k,
}
