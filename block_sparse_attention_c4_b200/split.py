"""Split-context decode: one request's context divided over several GPUs by page ranges.

Argument marshalling for the qsa_split_* entry points of ``include/qsa.h`` and the host side of a
step: which rank holds which pages, which rank holds the newest position (it appends the new index
key and attends to the tail), and the two exchanges (candidates, then attention partials), done
with ``torch.distributed`` all-gathers in rank order.  Every computation runs in the library's
kernels.

Rank r holds a contiguous range of each request's logical pages; ranks hold increasing ranges, so
the candidates gathered in rank order are in block order, which the exact merge relies on.
"""
from __future__ import annotations

import ctypes

import torch

from . import (HEAD_DIM, MAX_SEL, OP_SPARSE_GQA, OP_SPLIT_SCORE, PAGE_SIZE, Q_HEADS, TOPK, LayerCache, Workspace,
               _check, _dev, _ptr, _stream, compress_append, lib, sparse_gqa, workspace_bytes)


def partition_pages(n_pages: int, world: int):
    """Contiguous, balanced page ranges: rank r holds pages [lo[r], lo[r] + cnt[r])."""
    lo = [(r * n_pages) // world for r in range(world)]
    hi = lo[1:] + [n_pages]
    return lo, [h - l for l, h in zip(lo, hi)]


def holds_position(page_lo: int, page_cnt: int, pos: int) -> bool:
    """Whether the rank holding pages [page_lo, page_lo + page_cnt) holds position `pos`."""
    return page_lo * PAGE_SIZE <= pos < (page_lo + page_cnt) * PAGE_SIZE


def all_gather_stack(t: torch.Tensor, group=None) -> torch.Tensor:
    """[world, *t.shape]: every rank's `t`, in rank order (all ranks must call it)."""
    import torch.distributed as dist

    world = dist.get_world_size(group)
    out = torch.empty((world,) + tuple(t.shape), dtype=t.dtype, device=t.device)
    dist.all_gather(list(out.unbind(0)), t.contiguous(), group=group)
    return out


class SplitRank:
    """One rank's share of split-context decode.

    cache: this rank's LayerCache; its page-table rows are indexed by each request's logical page and
    map only the pages [page_lo[r], page_lo[r] + page_cnt[r]) the rank holds.  page_lo, page_cnt: host
    sequences (one entry per request of the cache)."""

    def __init__(self, cache: LayerCache, page_lo, page_cnt, max_len: int, device="cuda"):
        B = cache.batch
        self.cache, self.max_len = cache, int(max_len)
        self.page_lo_h, self.page_cnt_h = [int(x) for x in page_lo], [int(x) for x in page_cnt]
        self.page_lo = torch.tensor(self.page_lo_h, dtype=torch.int32, device=device)
        self.page_cnt = torch.tensor(self.page_cnt_h, dtype=torch.int32, device=device)
        self.ws_score = Workspace(workspace_bytes(OP_SPLIT_SCORE, B, self.max_len), device=device)
        self.ws_gqa = Workspace(workspace_bytes(OP_SPARSE_GQA, B, MAX_SEL), device=device)
        self.q_req = torch.arange(B, dtype=torch.int32, device=device)
        self.device = device

    def append(self, idx_k_new, seq_len_host):
        """Append each request's new index key (position L-1) if this rank holds that position."""
        B = self.cache.batch
        rows = [r for r in range(B) if holds_position(self.page_lo_h[r], self.page_cnt_h[r], int(seq_len_host[r]) - 1)]
        if not rows:
            return
        cu = [0] * (B + 1)
        for r in range(B):
            cu[r + 1] = cu[r] + (1 if r in rows else 0)
        lb = [int(seq_len_host[r]) - 1 if r in rows else 0 for r in range(B)]
        keys = idx_k_new[torch.tensor(rows, device=idx_k_new.device)].contiguous()
        compress_append(self.cache, keys, torch.tensor(cu, dtype=torch.int32, device=self.device),
                        torch.tensor(lb, dtype=torch.int32, device=self.device), 1)

    def score(self, idx_q, w, seq_len):
        """This rank's best min(512, its blocks) (key, block) per request: (keys int32 view, ids, n)."""
        B = self.cache.batch
        keys = torch.empty(B, TOPK, dtype=torch.int32, device=self.device)
        ids = torch.empty(B, TOPK, dtype=torch.int32, device=self.device)
        n = torch.empty(B, dtype=torch.int32, device=self.device)
        c = self.cache.struct()
        _check(lib().qsa_split_score_topk(ctypes.byref(c), _ptr(_dev(idx_q, torch.bfloat16, "idx_q", (B, 4, HEAD_DIM))),
                                          _ptr(_dev(w, torch.float32, "w", (B, 4))),
                                          _ptr(_dev(seq_len, torch.int32, "seq_len", (B,))), _ptr(self.page_lo),
                                          _ptr(self.page_cnt), self.max_len, _ptr(keys), _ptr(ids), _ptr(n),
                                          self.ws_score.ptr, self.ws_score.nbytes, _stream()), "qsa_split_score_topk")
        return keys, ids, n

    def attend(self, q, seq_len, blocks, nblocks):
        """Attention over the kept positions this rank holds (plus the tail if it holds L-1):
        (out bf16 [B,16,128], lse f32 [B,16])."""
        B = self.cache.batch
        pos = torch.empty(B, MAX_SEL, dtype=torch.int32, device=self.device)
        npos = torch.empty(B, dtype=torch.int32, device=self.device)
        _check(lib().qsa_split_positions(_ptr(seq_len), _ptr(self.page_lo), _ptr(self.page_cnt), _ptr(blocks),
                                         _ptr(nblocks), B, _ptr(pos), _ptr(npos), _stream()), "qsa_split_positions")
        lse = torch.empty(B, Q_HEADS, dtype=torch.float32, device=self.device)
        out = sparse_gqa(self.cache, q, self.q_req, pos, npos, MAX_SEL, self.ws_gqa, lse=lse)
        return out, lse

    def step(self, idx_k_new, idx_q, w, q, seq_len, seq_len_host, group=None):
        """One decode step of every request, this rank's part, with the two exchanges over `group`."""
        self.append(idx_k_new, seq_len_host)
        keys, ids, n = self.score(idx_q, w, seq_len)
        blocks, nblocks = merge(all_gather_stack(keys, group), all_gather_stack(ids, group),
                                all_gather_stack(n, group))
        out, lse = self.attend(q, seq_len, blocks, nblocks)
        return combine(all_gather_stack(out, group), all_gather_stack(lse, group))


def merge(keys, ids, n):
    """Exact top-512 of every request from the ranks' candidates stacked in rank order
    ([world, B, 512] keys (int32 view of the uint32 keys) and ids, [world, B] counts)."""
    world, B = int(n.shape[0]), int(n.shape[1])
    blocks = torch.empty(B, TOPK, dtype=torch.int32, device=n.device)
    nblocks = torch.empty(B, dtype=torch.int32, device=n.device)
    _check(lib().qsa_split_merge(_ptr(keys.contiguous()), _ptr(ids.contiguous()), _ptr(n.contiguous()), world, B,
                                 _ptr(blocks), _ptr(nblocks), _stream()), "qsa_split_merge")
    return blocks, nblocks


def combine(outs, lses):
    """LSE-weighted combination of the ranks' attention outputs ([world, B, 16, 128], [world, B, 16])."""
    world, B = int(outs.shape[0]), int(outs.shape[1])
    out = torch.empty(B, Q_HEADS, HEAD_DIM, dtype=torch.bfloat16, device=outs.device)
    _check(lib().qsa_split_combine(_ptr(outs.contiguous()), _ptr(lses.contiguous()), world, B, _ptr(out), _stream()),
           "qsa_split_combine")
    return out
