"""GPU parity of each step of the layer against the CPU oracle, through the C ABI.

Inputs come from qsa_gen (byte-identical on both sides).  The CUDA path builds
its own cache with qsa_compress_append; the oracle recomputes everything from
the raw keys.
"""
import numpy as np
import pytest
import torch

import oracle as O
import qsa_gen as G
from harness import (bf16_tensor_to_bits, bf16_tensor_to_f32, check_attention, check_selection,
                     oracle_decode_request, oracle_state)

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


def cidx_of_request(cache, wl, r, nb):
    """Compressed keys of blocks 0..nb-1 of request r, read back through the page table (bits)."""
    pt = wl.page_table()[r]
    b = np.arange(nb)
    entries = (pt[(4 * b) // 64].astype(np.int64) * 64 + (4 * b) % 64) // 4
    return bf16_tensor_to_bits(cache.cidx[torch.from_numpy(entries).cuda()])


# ---------------------------------------------------------------------------------------------
# a1: ring append + compression
# ---------------------------------------------------------------------------------------------

def test_compress_append_bulk_matches_oracle(Q, W):
    wl = G.custom_decode(21, [1, 3, 4, 5, 63, 64, 65, 1027, 4097, 6002])
    cache = W.build_cache(wl, prefix_tokens=[int(x) for x in wl.lens])
    torch.cuda.synchronize()
    for r in range(wl.batch):
        L = int(wl.lens[r])
        raw = wl.idx_keys(r)
        got = cidx_of_request(cache, wl, r, L // 4)
        np.testing.assert_array_equal(got, O.compress(raw)[:L // 4], err_msg=f"request {r} L={L}")
        ring = bf16_tensor_to_bits(cache.ring[r])
        for p in range(4 * (L // 4), L):
            np.testing.assert_array_equal(ring[p % 4], raw[p])


def test_compress_append_chunked_and_token_by_token_are_bitwise_equal(Q, W):
    wl = G.custom_decode(22, [903, 1500])
    ref = W.build_cache(wl, prefix_tokens=[int(x) for x in wl.lens])
    # chunked: uneven chunk sizes that straddle blocks and pages
    chunked = W.build_cache(wl, prefix_tokens=[0, 0])
    rng = np.random.default_rng(0)
    for r in range(2):
        t = 0
        while t < wl.lens[r]:
            n = int(min(rng.integers(1, 200), wl.lens[r] - t))
            W.append_tokens(chunked, wl, r, t, n)
            t += n
    # token by token for the first request, through a batch call that appends to both requests at once
    tok = W.build_cache(wl, prefix_tokens=[0, 0])
    keys = [wl.idx_keys(r) for r in range(2)]
    for t in range(int(max(wl.lens))):
        rows, cu, lb = [], [0], []
        for r in range(2):
            if t < wl.lens[r]:
                rows.append(keys[r][t])
            cu.append(len(rows))
            lb.append(min(t, int(wl.lens[r])))
        Q.compress_append(tok, W.bits_to_bf16(np.stack(rows), "cuda"), torch.tensor(cu, dtype=torch.int32).cuda(),
                          torch.tensor(lb, dtype=torch.int32).cuda(), 1)
    torch.cuda.synchronize()
    for c in (chunked, tok):
        assert torch.equal(c.cidx.view(torch.int16), ref.cidx.view(torch.int16))
        for r in range(2):  # only the slots of the unfinished block are defined
            n = int(wl.lens[r]) % 4
            assert torch.equal(c.ring[r, :n].view(torch.int16), ref.ring[r, :n].view(torch.int16))


# ---------------------------------------------------------------------------------------------
# a2-a4: rotation, scoring, top-512 ; a5: expansion
# ---------------------------------------------------------------------------------------------

def _score_queries(Q, W, wl, q_req, q_pos, idx_q, w):
    cache = W.build_cache(wl, prefix_tokens=[int(x) for x in wl.lens])
    nq = len(q_pos)
    ws = Q.Workspace(Q.workspace_bytes(Q.OP_INDEX_SCORE_TOPK, nq, int(max(q_pos)) + 1))
    blocks, nblocks = Q.index_score_topk(cache, W.bits_to_bf16(idx_q, "cuda"), torch.from_numpy(w).cuda(),
                                         torch.tensor(q_req, dtype=torch.int32).cuda(),
                                         torch.tensor(q_pos, dtype=torch.int32).cuda(), int(max(q_pos)) + 1, ws)
    torch.cuda.synchronize()
    assert ws.device_error() == 0
    return cache, blocks.cpu().numpy(), nblocks.cpu().numpy()


def test_index_score_topk_matches_oracle(Q, W):
    # contexts around the 512-block boundary, ragged last pages, and several scorer chunks
    lens = [4, 2048, 2051, 2052, 2053, 2100, 4097, 6002, 8191, 8192, 20001, 70003]
    wl = G.custom_decode(23, lens)
    q_req, q_pos = [], []
    for r, L in enumerate(lens):
        for p in sorted({L - 1, max(0, L - 2), max(0, L // 2)}):
            q_req.append(r)
            q_pos.append(p)
    rng = np.random.default_rng(1)
    idx_q = G.normal_bf16(23, 1000, (len(q_pos), 4, 128))
    w = rng.random((len(q_pos), 4)).astype(np.float32)
    cache, blocks, nblocks = _score_queries(Q, W, wl, q_req, q_pos, idx_q, w)
    comps = {r: O.compress(wl.idx_keys(r)) for r in range(len(lens))}
    for i, (r, p) in enumerate(zip(q_req, q_pos)):
        ob, _, s = O.select_query(idx_q[i], w[i], comps[r], p + 1)
        nb = (p + 1) // 4
        assert nblocks[i] == min(nb, 512)
        check_selection(blocks[i, :nblocks[i]], ob, s, nb, what=f"query {i} (req {r}, pos {p})")


def test_topk_ties_keep_lower_block_index(Q, W):
    # zero head weights make every score exactly 0: the kept set must be blocks 0..511
    wl = G.custom_decode(24, [9000, 20000])
    q_req, q_pos = [0, 1], [8999, 19999]
    idx_q = G.normal_bf16(24, 1001, (2, 4, 128))
    w = np.zeros((2, 4), dtype=np.float32)
    _, blocks, nblocks = _score_queries(Q, W, wl, q_req, q_pos, idx_q, w)
    for i in range(2):
        assert nblocks[i] == 512
        np.testing.assert_array_equal(blocks[i], np.arange(512))
    # one head weight: many blocks have ReLU-zero scores, the rest are exact ties only by accident
    w = np.array([[1, 0, 0, 0], [0, 0, 0, 1]], dtype=np.float32)
    _, blocks, nblocks = _score_queries(Q, W, wl, q_req, q_pos, idx_q, w)
    for i, r in enumerate(q_req):
        comp = O.compress(wl.idx_keys(r))
        ob, _, s = O.select_query(idx_q[i], w[i], comp, q_pos[i] + 1)
        check_selection(blocks[i], ob, s, (q_pos[i] + 1) // 4, what=f"one-head query {i}")


def test_expand_indices_matches_oracle(Q, W):
    rng = np.random.default_rng(2)
    q_pos = np.array([0, 1, 2, 3, 4, 7, 2047, 2050, 2051, 5000, 8190, 131071], dtype=np.int32)
    nq = len(q_pos)
    blocks = np.full((nq, 512), -1, dtype=np.int32)
    nblocks = np.zeros(nq, dtype=np.int32)
    for i, p in enumerate(q_pos):
        nb = (int(p) + 1) // 4
        b = O.select_topk(rng.random(nb)) if nb else np.zeros(0, np.int32)
        blocks[i, :len(b)] = b
        nblocks[i] = len(b)
    pos, npos = Q.expand_indices(torch.from_numpy(blocks).cuda(), torch.from_numpy(nblocks).cuda(),
                                 torch.from_numpy(q_pos).cuda())
    pos, npos = pos.cpu().numpy(), npos.cpu().numpy()
    for i, p in enumerate(q_pos):
        ref = O.expand(blocks[i, :nblocks[i]], int(p) + 1)
        assert npos[i] == len(ref)
        np.testing.assert_array_equal(pos[i, :npos[i]], ref)


# ---------------------------------------------------------------------------------------------
# a6: sparse GQA over explicit positions
# ---------------------------------------------------------------------------------------------

@pytest.mark.parametrize("kv_layout", ["interleaved", "separate"])
def test_sparse_gqa_matches_oracle(Q, W, kv_layout):
    wl = G.custom_decode(25, [5000, 3000], extra=0)
    cache = W.build_cache(wl, prefix_tokens=[0, 0], kv_layout=kv_layout)
    rng = np.random.default_rng(3)
    cases = [(0, 0), (0, 1), (1, 17), (0, 2051), (1, 1000), (0, 33), (1, 2051), (0, 2048)]
    nq = len(cases)
    pos = np.full((nq, 2051), -1, dtype=np.int32)
    npos = np.zeros(nq, dtype=np.int32)
    for i, (r, n) in enumerate(cases):
        p = np.sort(rng.choice(int(wl.lens[r]), size=n, replace=False)).astype(np.int32)
        pos[i, :n] = p
        npos[i] = n
    q = G.normal_bf16(25, 2000, (nq, 16, 128))
    q_req = np.array([r for r, _ in cases], dtype=np.int32)
    ws = Q.Workspace(Q.workspace_bytes(Q.OP_SPARSE_GQA, nq, 2051))
    lse = torch.empty(nq, 16, dtype=torch.float32, device="cuda")
    out = Q.sparse_gqa(cache, W.bits_to_bf16(q, "cuda"), torch.from_numpy(q_req).cuda(), torch.from_numpy(pos).cuda(),
                       torch.from_numpy(npos).cuda(), 2051, ws, lse=lse)
    torch.cuda.synchronize()
    assert ws.device_error() == 0
    out = bf16_tensor_to_f32(out)
    lse = lse.cpu().numpy()
    KV = {r: (wl.k(r), wl.v(r)) for r in range(2)}
    for i, (r, n) in enumerate(cases):
        ro, rl = O.sparse_gqa(q[i], KV[r][0], KV[r][1], pos[i, :n])
        if n == 0:
            assert np.all(out[i] == 0) and np.all(np.isneginf(lse[i]))
            continue
        check_attention(out[i], ro, what=f"case {i} ({n} positions)")
        np.testing.assert_allclose(lse[i], rl, atol=2e-3, rtol=0)


# ---------------------------------------------------------------------------------------------
# the fused decode step
# ---------------------------------------------------------------------------------------------

def _run_decode(Q, W, wl, keep_cache=False, kv_layout="interleaved"):
    cache = W.build_cache(wl, kv_layout=kv_layout)
    inp = W.decode_inputs(wl)
    B = wl.batch
    max_len = int(max(wl.lens))
    ws = Q.Workspace(Q.workspace_bytes(Q.OP_DECODE, B, max_len))
    blocks = torch.full((B, 512), -1, dtype=torch.int32, device="cuda")
    nblocks = torch.zeros(B, dtype=torch.int32, device="cuda")
    lse = torch.empty(B, 16, dtype=torch.float32, device="cuda")
    out = Q.decode(cache, inp["idx_k_new"], inp["idx_q"], inp["w"], inp["q"], inp["seq_len"], max_len, ws,
                   lse=lse, blocks_out=blocks, nblocks_out=nblocks)
    torch.cuda.synchronize()
    assert ws.device_error() == 0
    res = dict(out=bf16_tensor_to_f32(out), blocks=blocks.cpu().numpy(), nblocks=nblocks.cpu().numpy(),
               lse=lse.cpu().numpy())
    if keep_cache:
        res.update(cache=cache, inputs=inp, ws=ws)
    return res


def _check_decode_request(wl, r, res, cache=None):
    o = oracle_decode_request(wl, r)
    L, nb = o["L"], o["L"] // 4
    gb = res["blocks"][r, :res["nblocks"][r]]
    sel = check_selection(gb, o["blocks"], o["scores"], nb, what=f"request {r} L={L}")
    if np.array_equal(sel, o["blocks"]):
        ref = o["out"]
    else:
        ref, _ = O.sparse_gqa(G.Workload.q(wl, r)[0], o["K"], o["V"], O.expand(sel.astype(np.int32), L))
    check_attention(res["out"][r], ref, what=f"request {r} L={L}")
    if cache is not None:  # the append left the cache as the oracle's
        np.testing.assert_array_equal(cidx_of_request(cache, wl, r, nb), o["comp"][:nb])
        ring = bf16_tensor_to_bits(cache.ring[r])
        for p in range(4 * nb, L):
            np.testing.assert_array_equal(ring[p % 4], o["ring"][p % 4])
    return o


@pytest.mark.parametrize("kv_layout", ["interleaved", "separate"])
def test_decode_small_batch_matches_oracle(Q, W, kv_layout):
    wl = G.decode_small()
    res = _run_decode(Q, W, wl, keep_cache=True, kv_layout=kv_layout)
    for r in range(wl.batch):
        _check_decode_request(wl, r, res, cache=res["cache"])


def test_decode_edge_lengths(Q, W):
    lens = [1, 2, 3, 4, 5, 8, 2047, 2048, 2051, 2052, 2053, 2055, 4096, 4099]
    wl = G.custom_decode(26, lens)
    res = _run_decode(Q, W, wl, keep_cache=True)
    for r in range(wl.batch):
        o = _check_decode_request(wl, r, res, cache=res["cache"])
        assert len(o["pos"]) == 4 * min(lens[r] // 4, 512) + lens[r] % 4


def test_decode_many_rows_front_end_kernel(Q, W):
    """More rows than the scorer keeps page offsets for in shared memory (> 512): the step runs the
    separate front-end kernel (append, rotation, page counts and their prefix) before the scorer and
    the sparse GQA.  Every row's selection is validated; edge and seeded rows against the oracle,
    including the appended key."""
    rng = np.random.default_rng(29)
    lens = rng.integers(1, 5000, 600)
    lens[:6] = [1, 4, 2051, 2052, 2055, 4999]
    wl = G.custom_decode(29, [int(x) for x in lens])
    assert Q.decode_kernel_count(wl.batch) == 3
    res = _run_decode(Q, W, wl, keep_cache=True)
    bl, nbl = res["blocks"], res["nblocks"]
    for r, L in enumerate(lens):
        nb = int(L) // 4
        assert nbl[r] == min(nb, 512), f"row {r}"
        if nbl[r]:
            b = bl[r, :nbl[r]]
            assert np.all(np.diff(b) > 0) and b[0] >= 0 and b[-1] < nb, f"row {r}"
    assert np.all(np.isfinite(res["out"]))
    for r in sorted({0, 1, 2, 3, 4, 5, 599} | set(rng.choice(600, 8, replace=False).tolist())):
        _check_decode_request(wl, r, res, cache=res["cache"])


def test_decode_is_idempotent(Q, W):
    wl = G.custom_decode(27, [4097, 9000])
    res = _run_decode(Q, W, wl, keep_cache=True)
    cache, inp, ws = res["cache"], res["inputs"], res["ws"]
    out2 = Q.decode(cache, inp["idx_k_new"], inp["idx_q"], inp["w"], inp["q"], inp["seq_len"], 9000, ws)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(bf16_tensor_to_f32(out2), res["out"])


def test_decode_reports_bad_page_without_faulting(Q, W):
    wl = G.custom_decode(28, [3000])
    cache = W.build_cache(wl)
    inp = W.decode_inputs(wl)
    cache.page_table[0, 5] = 10 ** 6  # outside the pool
    ws = Q.Workspace(Q.workspace_bytes(Q.OP_DECODE, 1, 3000))
    Q.decode(cache, inp["idx_k_new"], inp["idx_q"], inp["w"], inp["q"], inp["seq_len"], 3000, ws)
    torch.cuda.synchronize()
    assert ws.device_error() & 1  # QSA_DEVERR_PAGE
    # a length beyond the stated maximum is reported too
    cache2 = W.build_cache(wl)
    ws2 = Q.Workspace(Q.workspace_bytes(Q.OP_DECODE, 1, 3000))
    Q.decode(cache2, inp["idx_k_new"], inp["idx_q"], inp["w"], inp["q"], inp["seq_len"], 2999, ws2)
    torch.cuda.synchronize()
    assert ws2.device_error() & 2  # QSA_DEVERR_LENGTH


# ---------------------------------------------------------------------------------------------
# a7: IndexShare draft step
# ---------------------------------------------------------------------------------------------

def _indexshare_case(Q, W, wl):
    B = wl.batch
    n1 = wl.n_draft + 1
    cache = W.build_cache(wl)  # K/V for L0 + n1 tokens; index keys of the first L0-1 tokens
    inp = W.decode_inputs(wl)  # capture step at position L0-1
    max_len = int(max(wl.lens))
    ws = Q.Workspace(Q.workspace_bytes(Q.OP_DECODE, B, max_len))
    blocks = torch.full((B, 512), -1, dtype=torch.int32, device="cuda")
    nblocks = torch.zeros(B, dtype=torch.int32, device="cuda")
    Q.decode(cache, inp["idx_k_new"], inp["idx_q"], inp["w"], inp["q"], inp["seq_len"], max_len, ws,
             blocks_out=blocks, nblocks_out=nblocks)
    pos, npos = Q.expand_indices(blocks, nblocks, inp["seq_len"] - 1)
    q = np.stack([wl.q(r) for r in range(B)])  # [B, n1, 16, 128]
    ws2 = Q.Workspace(Q.workspace_bytes(Q.OP_DECODE_INDEXSHARE, B, max_len))
    out = Q.decode_indexshare(cache, pos, npos, inp["seq_len"], W.bits_to_bf16(q, "cuda"), ws2)
    torch.cuda.synchronize()
    assert ws.device_error() == 0 and ws2.device_error() == 0
    out = bf16_tensor_to_f32(out)
    pos, npos = pos.cpu().numpy(), npos.cpu().numpy()
    for r in range(B):
        L0 = int(wl.lens[r])
        o = oracle_decode_request(wl, r)
        gb = blocks[r, :nblocks[r]].cpu().numpy()
        sel = check_selection(gb, o["blocks"], o["scores"], L0 // 4, what=f"capture {r}")
        frozen = O.expand(sel.astype(np.int32), L0)
        np.testing.assert_array_equal(pos[r, :npos[r]], frozen)
        K, V = wl.k(r), wl.v(r)
        ref = O.indexshare(frozen, L0, n1, q[r], K, V)
        for i in range(n1):
            rows = np.concatenate([frozen, np.arange(L0, L0 + i + 1)])
            assert rows.max() == L0 + i and np.all(np.diff(rows) > 0)  # causal, in bounds, distinct
            check_attention(out[r, i], ref[i], what=f"request {r} draft {i}")


def test_indexshare_small(Q, W):
    wl = G.indexshare_64k(batch=4)
    wl.lens[:] = [8193, 8194, 8195, 8196]
    _indexshare_case(Q, W, wl)


def test_indexshare_full_config(Q, W):
    """Batch 16, capture context 65536 + U[0,3], 3 draft steps (4 drafted positions)."""
    _indexshare_case(Q, W, G.indexshare_64k())


def test_topk_heavy_ties_across_segments(Q, W):
    """Thousands of blocks with bit-identical compressed keys: the kept set must take the tied blocks
    with the lowest indices, inside every scorer segment and in the merge of the segments."""
    for nb in (3000, 20000):
        L = 4 * nb
        wl = G.custom_decode(29, [L])
        cache = W.build_cache(wl, prefix_tokens=[0])
        rng = np.random.default_rng(nb)
        a = rng.standard_normal(128)
        b = 0.3 * a + rng.standard_normal(128)
        keys = np.empty((nb, 128), dtype=np.uint16)

        def bits(v):  # unit vector -> bf16 bits
            t = torch.from_numpy((v / np.linalg.norm(v)).astype(np.float32)).to(torch.bfloat16)
            return t.view(torch.int16).numpy().view(np.uint16)

        keys[:] = bits(b)
        keys[::50] = bits(a)  # 400 (or 60) blocks tie at the top, the rest tie below
        pt = wl.page_table()[0]
        blk = np.arange(nb)
        entries = (pt[(4 * blk) // 64].astype(np.int64) * 64 + (4 * blk) % 64) // 4
        cache.cidx[torch.from_numpy(entries).cuda()] = W.bits_to_bf16(keys, "cuda")
        idx_q = np.repeat(bits(a)[None, :], 4, axis=0)[None]  # every head looks along a
        w = np.array([[0.5, 0.25, 0.125, 1.0]], dtype=np.float32)
        ws = Q.Workspace(Q.workspace_bytes(Q.OP_INDEX_SCORE_TOPK, 1, L))
        blocks, nblocks = Q.index_score_topk(cache, W.bits_to_bf16(idx_q, "cuda"), torch.from_numpy(w).cuda(),
                                             torch.zeros(1, dtype=torch.int32).cuda(),
                                             torch.tensor([L - 1], dtype=torch.int32).cuda(), L, ws)
        torch.cuda.synchronize()
        assert ws.device_error() == 0
        ob, _, s = O.select_query(idx_q[0], w[0], keys, L)
        assert len(np.unique(s)) <= 2 and nblocks.item() == 512
        np.testing.assert_array_equal(blocks[0].cpu().numpy(), ob)
