"""Parity at the full workload sizes, in the launch configuration the benchmark times.

The oracle checks sampled outputs (it computes any single query on its own),
plus properties that hold at any size for every output row: kept blocks are
512 distinct visible blocks (all of them when a row has at most 512), and
positions are causal, in range and distinct.
"""
import numpy as np
import pytest
import torch

import oracle as O
import qsa_gen as G
from harness import bf16_tensor_to_f32, check_attention, check_selection, oracle_decode_request

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


def _valid_rows(blocks, nblocks, nbs):
    for i, nb in enumerate(nbs):
        b = blocks[i, :nblocks[i]]
        assert nblocks[i] == min(nb, 512)
        assert np.all(np.diff(b) > 0) and (len(b) == 0 or (b[0] >= 0 and b[-1] < nb))
        if nb <= 512:
            np.testing.assert_array_equal(b, np.arange(nb))


def test_decode_128k_batch64_sampled(Q, W):
    """Decode, batch 64, contexts uniform in [120000, 131072] -- the benchmark's workload and call."""
    wl = G.decode_128k()
    cache = W.build_cache(wl)
    inp = W.decode_inputs(wl)
    B, max_len = wl.batch, int(max(wl.lens))
    ws = Q.Workspace(Q.workspace_bytes(Q.OP_DECODE, B, max_len))
    blocks = torch.full((B, 512), -1, dtype=torch.int32, device="cuda")
    nblocks = torch.zeros(B, dtype=torch.int32, device="cuda")
    out = Q.decode(cache, inp["idx_k_new"], inp["idx_q"], inp["w"], inp["q"], inp["seq_len"], max_len, ws,
                   blocks_out=blocks, nblocks_out=nblocks)
    torch.cuda.synchronize()
    assert ws.device_error() == 0
    out = bf16_tensor_to_f32(out)
    bl, nbl = blocks.cpu().numpy(), nblocks.cpu().numpy()
    _valid_rows(bl, nbl, [int(L) // 4 for L in wl.lens])
    assert np.all(np.isfinite(out))
    for r in (0, 17, 41, 63):
        o = oracle_decode_request(wl, r)
        L = o["L"]
        sel = check_selection(bl[r, :nbl[r]], o["blocks"], o["scores"], L // 4, what=f"request {r}")
        ref = o["out"] if np.array_equal(sel, o["blocks"]) else \
            O.sparse_gqa(wl.q(r)[0], o["K"], o["V"], O.expand(sel.astype(np.int32), L))[0]
        check_attention(out[r], ref, what=f"request {r} L={L}")


def _score_and_attend(Q, W, wl, cache, t_rows, max_len, dev="cuda"):
    """Score, expand and attend the queries at positions t_rows (one request) through the C ABI."""
    T = len(t_rows)
    t_rows = np.asarray(t_rows, dtype=np.int64)
    idx_q = np.concatenate([wl.idx_q(0, q0=int(t), n=1) for t in t_rows]) if T < 4096 else \
        wl.idx_q(0, q0=int(t_rows[0]), n=T)
    w = np.concatenate([wl.w(0, q0=int(t), n=1) for t in t_rows]) if T < 4096 else wl.w(0, q0=int(t_rows[0]), n=T)
    q = np.concatenate([wl.q(0, q0=int(t), n=1) for t in t_rows]) if T < 4096 else wl.q(0, q0=int(t_rows[0]), n=T)
    q_pos = torch.from_numpy(t_rows.astype(np.int32)).to(dev)
    q_req = torch.zeros(T, dtype=torch.int32, device=dev)
    ws = Q.Workspace(Q.workspace_bytes(Q.OP_INDEX_SCORE_TOPK, T, max_len))
    blocks, nblocks = Q.index_score_topk(cache, W.bits_to_bf16(idx_q, dev), torch.from_numpy(w).to(dev), q_req,
                                         q_pos, max_len, ws)
    pos, npos = Q.expand_indices(blocks, nblocks, q_pos)
    ws2 = Q.Workspace(Q.workspace_bytes(Q.OP_SPARSE_GQA, T, 2051))
    out = Q.sparse_gqa(cache, W.bits_to_bf16(q, dev), q_req, pos, npos, 2051, ws2)
    torch.cuda.synchronize()
    assert ws.device_error() == 0 and ws2.device_error() == 0
    bl, nbl = blocks.cpu().numpy(), nblocks.cpu().numpy()
    _valid_rows(bl, nbl, [(int(t) + 1) // 4 for t in t_rows])
    pp, npp = pos.cpu().numpy(), npos.cpu().numpy()
    for i in range(0, T, max(1, T // 64)):  # positions causal, in range and distinct on a spread of rows
        p = pp[i, :npp[i]]
        t = int(t_rows[i])
        assert np.all(np.diff(p) > 0) and p[0] >= 0 and p[-1] <= t
        assert np.sum(p >= 4 * ((t + 1) // 4)) == (t + 1) % 4  # exactly the tail of the query's own block
        if (t + 1) % 4:
            assert p[-1] == t
    o = bf16_tensor_to_f32(out)
    assert np.all(np.isfinite(o))
    return bl, nbl, o


def _check_rows(wl, results, L_keys):
    """Oracle check of prefill rows t -> (kept blocks, output)."""
    raw = wl.idx_keys(0, 0, L_keys)
    comp = O.compress(raw)
    K, V = wl.k(0, 0, L_keys), wl.v(0, 0, L_keys)
    for t in sorted(results):
        ob, opos, s = O.select_query(wl.idx_q(0, q0=t, n=1)[0], wl.w(0, q0=t, n=1)[0], comp, t + 1)
        gb, go = results[t]
        sel = check_selection(gb, ob, s, (t + 1) // 4, what=f"prefill row {t}")
        pos = opos if np.array_equal(sel, ob) else O.expand(sel.astype(np.int32), t + 1)
        ref, _ = O.sparse_gqa(wl.q(0, q0=t, n=1)[0], K, V, pos)
        check_attention(go, ref, what=f"prefill row {t}")


def test_prefill_32k_all_rows(Q, W):
    """Prefill of one sequence of 32768 tokens, every token a query; oracle check on chunk edges, the
    512-block boundary, ragged tails and seeded random rows; validity checks on every row."""
    wl = G.prefill_32k()
    cache = W.build_cache(wl, prefix_tokens=[32768])
    bl, nbl, o = _score_and_attend(Q, W, wl, cache, np.arange(32768), 32768)
    rng = np.random.default_rng(11)
    rows = {0, 1, 2, 3, 4, 2047, 2050, 2051, 2052, 2053, 4095, 4096, 8191, 16383, 32766, 32767}
    rows |= set(rng.integers(0, 32768, 48).tolist())
    _check_rows(wl, {t: (bl[t, :nbl[t]], o[t]) for t in rows}, 32768)


def test_long_context_262k(Q, W):
    """A 262144-token context: the prompt's index keys appended in causal chunks of 8192, sampled
    prefill rows scored against the history, then the decode steps at L = 262144 .. 262147 (the
    decode token at position 262143 is the 262144th; L = 262147 has a tail of 3)."""
    wl = G.long_262k()  # 262147 tokens of K/V and index keys
    cache = W.build_cache(wl, prefix_tokens=[0])
    for t0 in range(0, 262143, 8192):
        W.append_tokens(cache, wl, 0, t0, min(8192, 262143 - t0))
    rng = np.random.default_rng(12)
    rows = sorted({0, 8191, 8192, 131071, 262142} | set(rng.integers(0, 262143, 24).tolist()))
    bl, nbl, o = _score_and_attend(Q, W, wl, cache, rows, 262143)
    _check_rows(wl, {t: (bl[i, :nbl[i]], o[i]) for i, t in enumerate(rows)}, 262143)
    # decode steps: each appends its own token (positions 262143 .. 262146)
    ws = Q.Workspace(Q.workspace_bytes(Q.OP_DECODE, 1, 262147))
    raw = wl.idx_keys(0, 0, 262147)
    for L in (262144, 262145, 262146, 262147):
        t = L - 1
        blocks = torch.full((1, 512), -1, dtype=torch.int32, device="cuda")
        nblocks = torch.zeros(1, dtype=torch.int32, device="cuda")
        out = Q.decode(cache, W.bits_to_bf16(raw[t:t + 1], "cuda"), W.bits_to_bf16(wl.idx_q(0, q0=t, n=1), "cuda"),
                       torch.from_numpy(wl.w(0, q0=t, n=1)).cuda(), W.bits_to_bf16(wl.q(0, q0=t, n=1), "cuda"),
                       torch.tensor([L], dtype=torch.int32).cuda(), L, ws, blocks_out=blocks, nblocks_out=nblocks)
        torch.cuda.synchronize()
        assert ws.device_error() == 0
        if L in (262144, 262147):
            comp = O.compress(raw[:L])
            ob, opos, s = O.select_query(wl.idx_q(0, q0=t, n=1)[0], wl.w(0, q0=t, n=1)[0], comp, L)
            gb = blocks[0, :nblocks[0]].cpu().numpy()
            sel = check_selection(gb, ob, s, L // 4, what=f"decode L={L}")
            pos = opos if np.array_equal(sel, ob) else O.expand(sel.astype(np.int32), L)
            assert len(pos) == 2048 + L % 4
            ref, _ = O.sparse_gqa(wl.q(0, q0=t, n=1)[0], wl.k(0, 0, L), wl.v(0, 0, L), pos)
            check_attention(bf16_tensor_to_f32(out)[0], ref, what=f"decode L={L}")
    # the chunked appends left the same compressed cache as the oracle's bulk compression
    pt = wl.page_table()[0]
    b = np.arange(262147 // 4)
    entries = (pt[(4 * b) // 64].astype(np.int64) * 64 + (4 * b) % 64) // 4
    got = cache.cidx[torch.from_numpy(entries).cuda()].view(torch.int16).cpu().numpy().view(np.uint16)
    np.testing.assert_array_equal(got, O.compress(raw))


# ---------------------------------------------------------------------------------------------
# The tensor-core prefill scorer at full size, chained into expansion and sparse GQA
# ---------------------------------------------------------------------------------------------

def _prefill_chain(Q, W, wl, cache, pos0, T, check_rows, L_keys, comp=None):
    """qsa_prefill_score_topk over the causal chunk pos0 .. pos0+T-1 of request 0 (twice: bitwise the
    same kept blocks), then qsa_expand_indices and qsa_sparse_gqa over every query of the chunk.  Every
    row is validated;
    the rows in `check_rows` (positions) are checked against the oracle: kept blocks under the
    near-tie rule, attention against the oracle run on the GPU's own selection."""
    dev = "cuda"
    idx_q = W.bits_to_bf16(wl.idx_q(0, q0=pos0, n=T), dev)
    w = torch.from_numpy(wl.w(0, q0=pos0, n=T)).to(dev)
    q = W.bits_to_bf16(wl.q(0, q0=pos0, n=T), dev)
    ws = Q.Workspace(Q.workspace_bytes(Q.OP_PREFILL_SCORE_TOPK, T, pos0 + T))
    blocks, nblocks = Q.prefill_score_topk(cache, idx_q, w, 0, pos0, ws)
    # the same call again: the kept blocks are bitwise the same (the candidates' order in their lists
    # varies with scheduling, the selection does not)
    blocks2, nblocks2 = Q.prefill_score_topk(cache, idx_q, w, 0, pos0, ws)
    torch.cuda.synchronize()
    assert torch.equal(nblocks, nblocks2)
    keep = torch.arange(512, device=dev)[None, :] < nblocks[:, None]
    assert torch.equal(torch.where(keep, blocks, -1), torch.where(keep, blocks2, -1))
    del blocks2, nblocks2
    q_pos = torch.arange(pos0, pos0 + T, dtype=torch.int32, device=dev)
    pos, npos = Q.expand_indices(blocks, nblocks, q_pos)
    ws2 = Q.Workspace(Q.workspace_bytes(Q.OP_SPARSE_GQA, T, 2051))
    out = Q.sparse_gqa(cache, q, torch.zeros(T, dtype=torch.int32, device=dev), pos, npos, 2051, ws2)
    torch.cuda.synchronize()
    assert ws.device_error() == 0 and ws2.device_error() == 0
    del ws, ws2
    bl, nbl = blocks.cpu().numpy(), nblocks.cpu().numpy()
    t_all = np.arange(pos0, pos0 + T)
    _valid_rows(bl, nbl, [(int(t) + 1) // 4 for t in t_all])
    pp, npp = pos.cpu().numpy(), npos.cpu().numpy()
    assert np.all(npp == 4 * nbl + (t_all + 1) % 4)
    o = bf16_tensor_to_f32(out)
    assert np.all(np.isfinite(o))
    if comp is None:
        comp = O.compress(wl.idx_keys(0, 0, L_keys))
    K, V = wl.k(0, 0, L_keys), wl.v(0, 0, L_keys)
    for t in sorted(check_rows):
        i = t - pos0
        idx_q_t, w_t = wl.idx_q(0, q0=t, n=1)[0], wl.w(0, q0=t, n=1)[0]
        ob, opos, s = O.select_query(idx_q_t, w_t, comp, t + 1)
        sel = check_selection(bl[i, :nbl[i]], ob, s, (t + 1) // 4, what=f"tensor-core prefill row {t}")
        gpos = O.expand(sel.astype(np.int32), t + 1)
        np.testing.assert_array_equal(pp[i, :npp[i]], gpos)
        ref, _ = O.sparse_gqa(wl.q(0, q0=t, n=1)[0], K, V, gpos)
        check_attention(o[i], ref, what=f"tensor-core prefill row {t}")
    return bl, nbl


def test_prefill_32k_tensor_core_chain(Q, W):
    """Config 1 end to end on the tensor-core path: 32768 queries scored by qsa_prefill_score_topk,
    expanded, attended; every row validated, edge and seeded rows against the oracle."""
    wl = G.prefill_32k()
    cache = W.build_cache(wl, prefix_tokens=[32768])
    rng = np.random.default_rng(21)
    rows = {0, 1, 3, 4, 2047, 2050, 2051, 2052, 4095, 8191, 16384, 32766, 32767}
    rows |= set(rng.integers(0, 32768, 40).tolist())
    _prefill_chain(Q, W, wl, cache, 0, 32768, rows, 32768)


@pytest.fixture(scope="module")
def long_cache(Q, W):
    """The 262144-token context of config 4 with every index key appended in causal chunks of 8192."""
    wl = G.long_262k()
    cache = W.build_cache(wl, prefix_tokens=[0])
    for t0 in range(0, 262144, 8192):
        W.append_tokens(cache, wl, 0, t0, 8192)
    torch.cuda.synchronize()
    comp = O.compress(wl.idx_keys(0, 0, 262144))
    return wl, cache, comp


@pytest.mark.parametrize("pos0", [0, 131072, 253952])
def test_long_context_prefill_chunk_tensor_core(Q, W, long_cache, pos0):
    """Config 4's prefill: a causal chunk of 8192 queries at pos0 (up to 65,536 visible blocks per
    query) through the tensor-core scorer, chained into expansion and sparse GQA; every row
    validated, the chunk's first and last rows and seeded rows against the oracle."""
    wl, cache, comp = long_cache
    T = 8192
    rng = np.random.default_rng(pos0 + 7)
    rows = {pos0, pos0 + 1, pos0 + T // 2, pos0 + T - 2, pos0 + T - 1}
    rows |= set((pos0 + rng.integers(0, T, 20)).tolist())
    if pos0 == 0:
        rows |= {2047, 2050, 2051, 2052, 4095}
    _prefill_chain(Q, W, wl, cache, pos0, T, rows, pos0 + T, comp=comp[:(pos0 + T) // 4])
