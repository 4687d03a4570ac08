"""Ragged (varlen) chunked prefill in one call, and a shared prefix scored from one copy.

* qsa_prefill_score_topk_varlen over several sequences (different requests, chunk starts and chunk
  sizes, an empty segment) gives, row for row, exactly what one qsa_prefill_score_topk call per
  sequence gives, and matches the oracle on sampled rows.
* Two requests whose page tables map the same physical pages for a 8192-token prefix: the prefix's
  compressed keys are appended once (by the first request); the second appends only its own tokens
  and its queries score the shared prefix through its page table (page-aligned full_slot / 4
  addressing).  Oracle: the second request's logical sequence is the shared prefix followed by its
  own keys.
"""
import numpy as np
import pytest
import torch

import oracle as O
import qsa_gen as G
from harness import bf16_tensor_to_bits, check_selection

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def Q():
    from block_sparse_attention_c4_b200 import build

    build.build()
    import block_sparse_attention_c4_b200 as Q

    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    Q.lib()
    return Q


@pytest.fixture(scope="module")
def W():
    import block_sparse_attention_c4_b200.workload as W

    return W


def _segments_inputs(wl, segs):
    idx_q = np.concatenate([wl.idx_q(r, q0=p0, n=T) for r, p0, T in segs if T > 0])
    w = np.concatenate([wl.w(r, q0=p0, n=T) for r, p0, T in segs if T > 0])
    cu = np.concatenate([[0], np.cumsum([T for _, _, T in segs])]).astype(np.int32)
    return idx_q, w, cu


def test_varlen_equals_one_call_per_sequence_and_the_oracle(Q, W):
    lens = [9000, 12000, 3000]
    wl = G.custom_decode(91, lens)
    cache = W.build_cache(wl, prefix_tokens=lens)
    segs = [(0, 1000, 3000), (1, 9000, 3000), (2, 0, 70), (1, 500, 0), (2, 2900, 100)]
    idx_q, w, cu = _segments_inputs(wl, segs)
    T = int(cu[-1])
    max_len = max(p0 + n for _, p0, n in segs)
    ws = Q.Workspace(Q.workspace_bytes(Q.OP_PREFILL_SCORE_TOPK, T, max_len))
    blocks, nblocks = Q.prefill_score_topk_varlen(cache, W.bits_to_bf16(idx_q, "cuda"), torch.from_numpy(w).cuda(),
                                                  [s[0] for s in segs], [s[1] for s in segs], cu, max_len, ws)
    torch.cuda.synchronize()
    assert ws.device_error() == 0
    bl, nbl = blocks.cpu().numpy(), nblocks.cpu().numpy()
    comps = {r: O.compress(wl.idx_keys(r)) for r in range(len(lens))}
    rng = np.random.default_rng(92)
    for i, (r, p0, n) in enumerate(segs):
        if n == 0:
            continue
        rows = slice(cu[i], cu[i + 1])
        ws1 = Q.Workspace(Q.workspace_bytes(Q.OP_PREFILL_SCORE_TOPK, n, p0 + n))
        b1, n1 = Q.prefill_score_topk(cache, W.bits_to_bf16(idx_q[rows], "cuda"), torch.from_numpy(w[rows]).cuda(),
                                      r, p0, ws1)
        torch.cuda.synchronize()
        assert ws1.device_error() == 0
        np.testing.assert_array_equal(n1.cpu().numpy(), nbl[rows])
        b1 = b1.cpu().numpy()
        for k in range(n):  # only the kept part of each row is defined
            np.testing.assert_array_equal(b1[k, :n1[k]], bl[cu[i] + k, :nbl[cu[i] + k]])
        for k in sorted({0, n - 1} | set(rng.integers(0, n, 6).tolist())):
            t = p0 + k
            g = cu[i] + k
            ob, _, s = O.select_query(idx_q[g], w[g], comps[r], t + 1)
            check_selection(bl[g, :nbl[g]], ob, s, (t + 1) // 4, what=f"segment {i} row {t}")


def test_shared_prefix_is_appended_once_and_scored_by_both_requests(Q, W):
    P = 8192  # shared prefix: 128 pages
    LA, LB = 20000, 15000
    wl = G.custom_decode(93, [LA, LB])
    pt = wl.page_table().copy()
    pt[1, :P // 64] = pt[0, :P // 64]  # request 1's prefix pages are request 0's pages
    cache = Q.LayerCache(wl.total_pages * 64, 2, pt.shape[1], rope_theta=wl.rope_theta,
                         page_table=torch.from_numpy(pt).cuda())
    keys_a = wl.idx_keys(0)
    keys_b = np.concatenate([keys_a[:P], wl.idx_keys(1)[P:LB]])  # request 1's logical sequence

    def append(r, t0, keys):
        cu = np.zeros(3, dtype=np.int32)
        cu[r + 1:] = len(keys)
        lb = np.zeros(2, dtype=np.int32)
        lb[r] = t0
        Q.compress_append(cache, W.bits_to_bf16(keys, "cuda"), torch.from_numpy(cu).cuda(),
                          torch.from_numpy(lb).cuda(), len(keys))

    append(0, 0, keys_a)          # request 0: every key, the shared prefix included
    append(1, P, keys_b[P:])      # request 1: only its own tokens after the prefix
    torch.cuda.synchronize()
    comp_a, comp_b = O.compress(keys_a), O.compress(keys_b)
    # one copy of the prefix: request 0's compressed keys are the oracle's, request 1 reads them too
    b = np.arange(LA // 4)
    ent_a = (pt[0][(4 * b) // 64].astype(np.int64) * 64 + (4 * b) % 64) // 4
    np.testing.assert_array_equal(bf16_tensor_to_bits(cache.cidx[torch.from_numpy(ent_a).cuda()]), comp_a)
    b = np.arange(LB // 4)
    ent_b = (pt[1][(4 * b) // 64].astype(np.int64) * 64 + (4 * b) % 64) // 4
    np.testing.assert_array_equal(bf16_tensor_to_bits(cache.cidx[torch.from_numpy(ent_b).cuda()]), comp_b)
    assert np.array_equal(ent_a[:P // 4], ent_b[:P // 4])
    # one ragged call scoring a chunk of each request
    segs = [(0, 12000, 2000), (1, 9000, 2000)]
    idx_q, w, cu = _segments_inputs(wl, segs)
    T = int(cu[-1])
    ws = Q.Workspace(Q.workspace_bytes(Q.OP_PREFILL_SCORE_TOPK, T, 14000))
    blocks, nblocks = Q.prefill_score_topk_varlen(cache, W.bits_to_bf16(idx_q, "cuda"), torch.from_numpy(w).cuda(),
                                                  [0, 1], [12000, 9000], cu, 14000, ws)
    torch.cuda.synchronize()
    assert ws.device_error() == 0
    bl, nbl = blocks.cpu().numpy(), nblocks.cpu().numpy()
    rng = np.random.default_rng(94)
    for i, (r, p0, n) in enumerate(segs):
        comp = comp_a if r == 0 else comp_b
        for k in sorted({0, n - 1} | set(rng.integers(0, n, 10).tolist())):
            t, g = p0 + k, cu[i] + k
            ob, _, s = O.select_query(idx_q[g], w[g], comp, t + 1)
            check_selection(bl[g, :nbl[g]], ob, s, (t + 1) // 4, what=f"request {r} row {t}")
