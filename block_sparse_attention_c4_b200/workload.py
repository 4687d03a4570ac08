"""Put a synthetic workload into device memory in the layer's paged layout.

``wl`` is any object with the generator interface of ``qsa_gen.Workload``
(per-request numpy tensors as bf16 bits, a page table, lengths).  This module
only moves bytes: K/V rows go to their physical slots, and the compressed
index cache and ring are produced by the library's own ``qsa_compress_append``
(so a decode step starts from the state the layer itself builds).
"""
from __future__ import annotations

import numpy as np
import torch

from . import (BLOCK, HEAD_DIM, INDEX_HEADS, PAGE_SIZE, Q_HEADS, LayerCache, compress_append)


def bits_to_bf16(a: np.ndarray, device) -> torch.Tensor:
    """uint16 bf16 bits (numpy) -> torch.bfloat16 tensor on `device` (bit copy)."""
    t = torch.from_numpy(np.ascontiguousarray(a).view(np.int16))
    return t.to(device=device).view(torch.bfloat16)


def slots_of(page_table_row: np.ndarray, n_tok: int, tok0: int = 0) -> np.ndarray:
    t = np.arange(tok0, tok0 + n_tok, dtype=np.int64)
    return page_table_row[t // PAGE_SIZE].astype(np.int64) * PAGE_SIZE + (t % PAGE_SIZE)


def build_cache(wl, device="cuda", prefix_tokens=None, chunk_tokens: int = 1 << 16,
                kv_layout: str = "interleaved", kv_dtype: str = "bf16") -> LayerCache:
    """Allocate the cache of `wl`, fill K/V for every stored token, and append the raw index keys of
    the first `prefix_tokens[r]` tokens of each request (default: lens[r] - 1, the state before a
    decode step) through qsa_compress_append.  kv_dtype "fp8" fills K/V with the workload's E4M3
    codes (wl.k8 / wl.v8)."""
    pt = wl.page_table()
    B = wl.batch
    cache = LayerCache(wl.total_pages * PAGE_SIZE, B, pt.shape[1], rope_theta=wl.rope_theta, device=device,
                       page_table=torch.from_numpy(pt).to(device), kv_layout=kv_layout, kv_dtype=kv_dtype)
    if prefix_tokens is None:
        prefix_tokens = [int(wl.lens[r]) - 1 for r in range(B)]
    for r in range(B):
        n = wl.tokens(r)
        for t0 in range(0, n, chunk_tokens):
            m = min(chunk_tokens, n - t0)
            slots = torch.from_numpy(slots_of(pt[r], m, t0)).to(device)
            if kv_dtype == "fp8":
                cache.k.index_copy_(0, slots, torch.from_numpy(wl.k8(r, t0, m)).to(device))
                cache.v.index_copy_(0, slots, torch.from_numpy(wl.v8(r, t0, m)).to(device))
            else:
                cache.k.index_copy_(0, slots, bits_to_bf16(wl.k(r, t0, m), device))
                cache.v.index_copy_(0, slots, bits_to_bf16(wl.v(r, t0, m), device))
        append_tokens(cache, wl, r, 0, int(prefix_tokens[r]), chunk_tokens)
    return cache


def append_tokens(cache: LayerCache, wl, r: int, tok0: int, n: int, chunk_tokens: int = 1 << 16):
    """Append raw index keys tok0 .. tok0+n-1 of request r (in chunks) with qsa_compress_append."""
    B = cache.batch
    dev = cache.k.device
    for c0 in range(tok0, tok0 + n, chunk_tokens):
        m = min(chunk_tokens, tok0 + n - c0)
        keys = bits_to_bf16(wl.idx_keys(r, c0, m), dev)
        cu = np.zeros(B + 1, dtype=np.int32)
        cu[r + 1:] = m
        lb = np.zeros(B, dtype=np.int32)
        lb[r] = c0
        compress_append(cache, keys, torch.from_numpy(cu).to(dev), torch.from_numpy(lb).to(dev), m)


def decode_inputs(wl, device="cuda"):
    """Per-step inputs of a decode step: new index key, index queries, head weights, queries, lengths."""
    B = wl.batch
    knew = np.stack([wl.idx_keys(r, int(wl.lens[r]) - 1, 1)[0] for r in range(B)])
    idx_q = np.stack([wl.idx_q(r)[0] for r in range(B)])
    w = np.stack([wl.w(r)[0] for r in range(B)]).astype(np.float32)
    q = np.stack([wl.q(r)[0] for r in range(B)])
    return {
        "idx_k_new": bits_to_bf16(knew.reshape(B, HEAD_DIM), device),
        "idx_q": bits_to_bf16(idx_q.reshape(B, INDEX_HEADS, HEAD_DIM), device),
        "w": torch.from_numpy(w.reshape(B, INDEX_HEADS)).to(device),
        "q": bits_to_bf16(q.reshape(B, Q_HEADS, HEAD_DIM), device),
        "seq_len": torch.from_numpy(np.asarray(wl.lens, dtype=np.int32)).to(device),
    }


def ring_state(wl, r: int, L: int) -> np.ndarray:
    """Raw index keys in the ring of request r after L tokens have been appended ([4,128] bits; slots of
    positions >= L are zero)."""
    ring = np.zeros((BLOCK, HEAD_DIM), dtype=np.uint16)
    start = (L // BLOCK) * BLOCK
    if L > start:
        keys = wl.idx_keys(r, start, L - start)
        for i in range(L - start):
            ring[(start + i) % BLOCK] = keys[i]
    return ring
