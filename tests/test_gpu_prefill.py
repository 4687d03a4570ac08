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


def _run(Q, W, wl, pos0, T, rows=None):
    """Append the first pos0+T index keys, score the chunk pos0 .. pos0+T-1 on the tensor cores, and check
    rows (default: all) against the oracle."""
    cache = W.build_cache(wl, prefix_tokens=[pos0 + T])
    idx_q = wl.idx_q(0, q0=pos0, n=T)
    w = wl.w(0, q0=pos0, n=T)
    ws = Q.Workspace(Q.workspace_bytes(Q.OP_PREFILL_SCORE_TOPK, T, pos0 + T))
    blocks, nblocks = Q.prefill_score_topk(cache, W.bits_to_bf16(idx_q, "cuda"), torch.from_numpy(w).cuda(), 0,
                                           pos0, ws)
    torch.cuda.synchronize()
    assert ws.device_error() == 0
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


@pytest.mark.parametrize("pos0,T", [(0, 3000), (0, 64), (0, 2100), (5000, 2000), (4097, 777), (9000, 33)])
def test_prefill_scorer_matches_oracle_every_row(Q, W, pos0, T):
    wl = G.custom_decode(41 + T, [pos0 + T])
    _run(Q, W, wl, pos0, T)


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
