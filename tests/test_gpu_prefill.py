"""Parity of the tensor-core prefill scorer (qsa_prefill_score_topk) with the CPU oracle."""
import numpy as np
import pytest
import torch

import oracle as O
import qsa_gen as G
from harness import check_selection

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def Q():
    from block_sparse_attention_c4_b200 import build

    build.build()
    import block_sparse_attention_c4_b200 as Q

    Q.lib()
    return Q


@pytest.fixture(scope="module")
def W():
    import block_sparse_attention_c4_b200.workload as W

    return W


def _run(Q, W, wl, pos0, T, rows=None, w=None):
    """Append the first pos0+T index keys, score the chunk pos0 .. pos0+T-1 on the tensor cores, and check
    rows (default: all) against the oracle (head weights: the workload's, or `w`)."""
    cache = W.build_cache(wl, prefix_tokens=[pos0 + T])
    idx_q = wl.idx_q(0, q0=pos0, n=T)
    w = wl.w(0, q0=pos0, n=T) if w is None else w
    ws = Q.Workspace(Q.workspace_bytes(Q.OP_PREFILL_SCORE_TOPK, T, pos0 + T))
    blocks, nblocks = Q.prefill_score_topk(cache, W.bits_to_bf16(idx_q, "cuda"), torch.from_numpy(w).cuda(), 0,
                                           pos0, ws)
    torch.cuda.synchronize()
    assert ws.device_error() == 0
    print(f"prefill pos0={pos0} T={T}: {Q.prefill_rescored_rows(ws, T, pos0 + T)} rows re-scored in full")
    bl, nbl = blocks.cpu().numpy(), nblocks.cpu().numpy()
    comp = O.compress(wl.idx_keys(0, 0, pos0 + T))
    rows = range(T) if rows is None else rows
    for i in rows:
        t = pos0 + i
        nb = (t + 1) // 4
        ob, _, s = O.select_query(idx_q[i], w[i], comp, t + 1)
        assert nbl[i] == min(nb, 512), f"row {t}"
        check_selection(bl[i, :nbl[i]], ob, s, nb, what=f"prefill row {t}")
    return bl, nbl


@pytest.mark.parametrize("pos0,T", [(0, 3000), (0, 64), (0, 2100), (5000, 2000), (4097, 777), (9000, 33),
                                    (40000, 300), (32568, 400)])
def test_prefill_scorer_matches_oracle_every_row(Q, W, pos0, T):
    """(32568, 400): the chunk's first work tiles see at most 8192 blocks and write every score key, the
    later ones filter candidates."""
    wl = G.custom_decode(41 + T, [pos0 + T])
    _run(Q, W, wl, pos0, T)


@pytest.mark.parametrize("pos0,T", [(4000, 130), (40000, 130)])
def test_prefill_nonpositive_and_mixed_weights(Q, W, pos0, T):
    """Head weights of both signs (the projected weights can be negative): queries whose 4 weights are
    all <= 0 have no positive score bound, their scores are <= 0 and their best blocks are the least
    negative; queries with mixed signs keep a bound from their positive weights.  Every row against the
    oracle, for short (every key written) and long (filtered candidates) contexts."""
    wl = G.custom_decode(43 + pos0, [pos0 + T])
    rng = np.random.default_rng(pos0 + 7)
    w = rng.uniform(-1.0, 1.0, size=(T, 4)).astype(np.float32)
    w[::2] = -np.abs(w[::2])  # every other query: all weights <= 0
    w[4, :] = 0.0             # one query: every score exactly 0, all blocks tied
    _run(Q, W, wl, pos0, T, w=w)


def test_prefill_scorer_agrees_with_streaming_scorer(Q, W):
    wl = G.custom_decode(47, [6000])
    pos0, T = 0, 6000
    bl, nbl = _run(Q, W, wl, pos0, T, rows=range(0, T, 97))
    cache = W.build_cache(wl, prefix_tokens=[T])
    ws = Q.Workspace(Q.workspace_bytes(Q.OP_INDEX_SCORE_TOPK, T, T))
    b2, n2 = Q.index_score_topk(cache, W.bits_to_bf16(wl.idx_q(0, 0, T), "cuda"), torch.from_numpy(wl.w(0, 0, T)).cuda(),
                                torch.zeros(T, dtype=torch.int32).cuda(), torch.arange(T, dtype=torch.int32).cuda(),
                                T, ws)
    b2, n2 = b2.cpu().numpy(), n2.cpu().numpy()
    np.testing.assert_array_equal(nbl, n2)
    # the two scorers accumulate in different orders: they must agree exactly wherever the oracle's
    # 512th and 513th scores are not a near tie, and both must pass the parity rule everywhere
    comp = O.compress(wl.idx_keys(0, 0, T))
    idx_q, w = wl.idx_q(0, 0, T), wl.w(0, 0, T)
    clear = 0
    for i in range(0, T, 7):
        nb = (i + 1) // 4
        ob, _, s = O.select_query(idx_q[i], w[i], comp, i + 1)
        check_selection(b2[i, :n2[i]], ob, s, nb, what=f"streaming row {i}")
        check_selection(bl[i, :nbl[i]], ob, s, nb, what=f"tensor-core row {i}")
        if nb > 512:
            srt = np.sort(s)[::-1]
            if abs(srt[511] - srt[512]) > 1e-3 * abs(srt[511]):
                clear += 1
                np.testing.assert_array_equal(bl[i, :nbl[i]], b2[i, :n2[i]])
    assert clear > 20


@pytest.mark.parametrize("pos0,T", [(0, 3000), (200000, 64)])
def test_prefill_rotation_is_the_rounded_rope(Q, W, pos0, T):
    """Every rotated index query of the call is the oracle's rotation at the query's position (pinned to
    the complex-multiply definition), rounded once to bf16: bit for bit, at short and long positions."""
    wl = G.custom_decode(77 + T, [pos0 + T])
    cache = W.build_cache(wl, prefix_tokens=[pos0 + T])
    idx_q = wl.idx_q(0, q0=pos0, n=T)
    w = wl.w(0, q0=pos0, n=T)
    ws = Q.Workspace(Q.workspace_bytes(Q.OP_PREFILL_SCORE_TOPK, T, pos0 + T))
    Q.prefill_score_topk(cache, W.bits_to_bf16(idx_q, "cuda"), torch.from_numpy(w).cuda(), 0, pos0, ws)
    torch.cuda.synchronize()
    assert ws.device_error() == 0
    got = Q.prefill_rotated_queries(ws, T, pos0 + T)
    for i in range(T):
        ref = O.rotate_query(idx_q[i], pos0 + i, wl.rope_theta)
        np.testing.assert_array_equal(got[i].reshape(-1), ref.reshape(-1), err_msg=f"row {pos0 + i}")


def test_prefill_scorer_32k(Q, W):
    """The 32768-token prefill: every row's kept set is valid; sampled rows match the oracle."""
    wl = G.prefill_32k()
    rng = np.random.default_rng(5)
    rows = sorted({0, 2047, 2048, 2051, 4095, 8191, 16383, 32767} | set(rng.integers(0, 32768, 40).tolist()))
    bl, nbl = _run(Q, W, wl, 0, 32768, rows=rows)
    for i in range(32768):
        nb = (i + 1) // 4
        b = bl[i, :nbl[i]]
        assert nbl[i] == min(nb, 512)
        assert np.all(np.diff(b) > 0) and (nbl[i] == 0 or b[-1] < nb)


def test_prefill_heavy_ties(Q, W):
    """Thousands of bit-identical compressed keys: every query keeps the tied blocks with the lowest
    indices, for rows held in shared memory (3000 blocks) and rows read through L2 (20000 blocks)."""
    for nb in (3000, 20000):
        L = 4 * nb
        T = 40
        wl = G.custom_decode(31, [L])
        cache = W.build_cache(wl, prefix_tokens=[0])
        rng = np.random.default_rng(nb + 1)
        a = rng.standard_normal(128)
        b = 0.3 * a + rng.standard_normal(128)

        def bits(v):  # unit vector -> bf16 bits
            t = torch.from_numpy((v / np.linalg.norm(v)).astype(np.float32)).to(torch.bfloat16)
            return t.view(torch.int16).numpy().view(np.uint16)

        keys = np.empty((nb, 128), dtype=np.uint16)
        keys[:] = bits(b)
        keys[::50] = bits(a)
        pt = wl.page_table()[0]
        blk = np.arange(nb)
        entries = (pt[(4 * blk) // 64].astype(np.int64) * 64 + (4 * blk) % 64) // 4
        cache.cidx[torch.from_numpy(entries).cuda()] = W.bits_to_bf16(keys, "cuda")
        idx_q = np.repeat(np.repeat(bits(a)[None, :], 4, axis=0)[None], T, axis=0)
        w = np.tile(np.array([[0.5, 0.25, 0.125, 1.0]], dtype=np.float32), (T, 1))
        pos0 = L - T
        ws = Q.Workspace(Q.workspace_bytes(Q.OP_PREFILL_SCORE_TOPK, T, L))
        blocks, nblocks = Q.prefill_score_topk(cache, W.bits_to_bf16(idx_q, "cuda"), torch.from_numpy(w).cuda(), 0,
                                               pos0, ws)
        torch.cuda.synchronize()
        assert ws.device_error() == 0
        bl, nbl = blocks.cpu().numpy(), nblocks.cpu().numpy()
        for i in range(0, T, 3):
            t = pos0 + i
            ob, _, s = O.select_query(idx_q[i], w[i], keys[:(t + 1) // 4], t + 1)
            assert len(np.unique(s)) <= 2 and nbl[i] == 512
            np.testing.assert_array_equal(bl[i], ob)


def test_prefill_rows_the_candidates_cannot_settle(Q, W):
    """Blocks of the sampled M-tiles (every 8th run of 128 blocks) score high and every other block
    low, so each query's sampled threshold lets far fewer than 512 blocks through: every such row is
    re-scored in full, and the result is still the exact top 512.  (Contexts above 8192 blocks: shorter
    ones write every score key and never need the re-scoring.)"""
    nb = 12288
    L = 4 * nb
    T = 96
    wl = G.custom_decode(33, [L])
    cache = W.build_cache(wl, prefix_tokens=[0])
    rng = np.random.default_rng(9)
    a = rng.standard_normal(128)
    bdir = -a + 0.1 * rng.standard_normal(128)
    blk = np.arange(nb)
    sampled = (blk // 128) % 8 == 0
    vecs = np.where(sampled[:, None], a[None, :], bdir[None, :]) + 0.3 * rng.standard_normal((nb, 128))
    vecs /= np.linalg.norm(vecs, axis=1, keepdims=True)
    keys = torch.from_numpy(vecs.astype(np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    pt = wl.page_table()[0]
    entries = (pt[(4 * blk) // 64].astype(np.int64) * 64 + (4 * blk) % 64) // 4
    cache.cidx[torch.from_numpy(entries).cuda()] = W.bits_to_bf16(keys, "cuda")
    qa = torch.from_numpy((a / np.linalg.norm(a)).astype(np.float32)).to(torch.bfloat16)
    qa = qa.view(torch.int16).numpy().view(np.uint16)
    idx_q = np.repeat(np.repeat(qa[None, :], 4, axis=0)[None], T, axis=0)
    w = np.tile(np.array([[1.0, 0.5, 0.25, 0.125]], dtype=np.float32), (T, 1))
    pos0 = L - T
    ws = Q.Workspace(Q.workspace_bytes(Q.OP_PREFILL_SCORE_TOPK, T, L))
    blocks, nblocks = Q.prefill_score_topk(cache, W.bits_to_bf16(idx_q, "cuda"), torch.from_numpy(w).cuda(), 0,
                                           pos0, ws)
    torch.cuda.synchronize()
    assert ws.device_error() == 0
    assert Q.prefill_rescored_rows(ws, T, L) == T  # every row took the full re-scoring path
    bl, nbl = blocks.cpu().numpy(), nblocks.cpu().numpy()
    for i in range(0, T, 5):
        t = pos0 + i
        ob, _, s = O.select_query(idx_q[i], w[i], keys[:(t + 1) // 4], t + 1)
        check_selection(bl[i, :nbl[i]], ob, s, (t + 1) // 4, what=f"re-scored row {t}")
