"""Index projection and the two-phase decode (indexer on a second stream) against the CPU oracle.

* qsa_index_project: projected index queries and keys within half a bf16 ulp of the exact projection
  plus a bound of the FP32 accumulation error (and at least 99% bit-equal to the oracle's), head
  weights within FP32 accumulation error.
* qsa_decode_indexer + qsa_decode_attend: the GPU's projections (the same kernel, read back through
  qsa_index_project) are checked against the oracle's; from those values on, the oracle appends the
  key, selects and attends, and the GPU's kept blocks and outputs must match it under the usual
  rules (near-tie rule for the blocks, 2e-2 / 5e-3 for attention on the GPU's own selection).
* The indexer on a second stream, overlapping the caller's main Q/K/V projection (a GEMM on the
  first stream), gives bit-identical results to both phases on one stream and to qsa_decode fed
  with the projected inputs.
"""
import numpy as np
import pytest
import torch

import oracle as O
import qsa_gen as G
from harness import bf16_tensor_to_bits, bf16_tensor_to_f32, check_attention, check_selection, oracle_state

pytestmark = pytest.mark.gpu

HIDDEN = 4096


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


def _check_projection(got_q, got_k, got_w, x, Wp, what=""):
    """Each GPU output against the exact (FP64) projection: within half a bf16 ulp of it plus the FP32
    accumulation error, bounded by 2^-18 * sum_j |x_j W_fj| (several dozen FP32 roundings of partial
    sums no larger than that); and at least 99% of the bf16 outputs bit-equal to the oracle's."""
    xf = G.bf16_bits_to_f32(x).astype(np.float64)
    wf = G.bf16_bits_to_f32(Wp).astype(np.float64)
    y = xf @ wf.T                                  # [n, 644] exact up to FP64 rounding
    bound = 2.0 ** -18 * (np.abs(xf) @ np.abs(wf).T)
    rq, rk, rw = O.index_project(x, Wp)
    n = x.shape[0]
    for got, ref, sl, name in ((got_q, rq, slice(0, 512), "idx_q"), (got_k, rk, slice(512, 640), "idx_k")):
        g = G.bf16_bits_to_f32(got.reshape(n, -1)).astype(np.float64)
        ye = y[:, sl]
        ulp = 2.0 ** (np.floor(np.log2(np.maximum(np.abs(ye), 1e-30))) - 7)
        err = np.abs(g - ye)
        assert np.all(err <= 0.5 * ulp + bound[:, sl]), f"{what} {name}: max excess {np.max(err - 0.5 * ulp - bound[:, sl])}"
        assert np.mean(got.reshape(n, -1) == ref.reshape(n, -1)) >= 0.99, f"{what} {name}: too few bit-exact"
    np.testing.assert_array_less(np.abs(got_w.astype(np.float64) - y[:, 640:]),
                                 np.abs(y[:, 640:]) * 2.0 ** -23 + bound[:, 640:] + 1e-30)
    np.testing.assert_allclose(got_w, rw, rtol=1e-4, atol=1e-5, err_msg=f"{what} w")


@pytest.mark.parametrize("n,hidden", [(1, 128), (70, 4096), (33, 2560)])
def test_index_project_matches_oracle(Q, W, n, hidden):
    x = G.normal_bf16(71, 1, (n, hidden))
    Wp = G.projection_weights(71, hidden)
    iq, ik, w = Q.index_project(W.bits_to_bf16(x, "cuda"), W.bits_to_bf16(Wp, "cuda"))
    torch.cuda.synchronize()
    _check_projection(bf16_tensor_to_bits(iq), bf16_tensor_to_bits(ik), w.cpu().numpy(), x, Wp,
                      what=f"n={n} hidden={hidden}")


def _projected_case(Q, W, lens, seed):
    wl = G.custom_decode(seed, lens, p_bias=0.0)
    B, max_len = wl.batch, int(max(lens))
    cache = W.build_cache(wl)  # K/V of every token, index keys of the first L-1 tokens
    x = np.stack([wl.hidden(r, HIDDEN)[0] for r in range(B)])
    Wp = G.projection_weights(seed, HIDDEN)
    xd, Wd = W.bits_to_bf16(x, "cuda"), W.bits_to_bf16(Wp, "cuda")
    seq_len = torch.tensor(lens, dtype=torch.int32, device="cuda")
    q = W.bits_to_bf16(np.stack([wl.q(r)[0] for r in range(B)]), "cuda")
    return wl, cache, x, Wp, xd, Wd, seq_len, q, max_len


def test_decode_indexer_and_attend_match_oracle(Q, W):
    lens = [3001, 4097, 8190, 20003]
    wl, cache, x, Wp, xd, Wd, seq_len, q, max_len = _projected_case(Q, W, lens, 72)
    B = wl.batch
    ws_i = Q.Workspace(Q.workspace_bytes(Q.OP_DECODE_INDEXER, B, max_len))
    ws_a = Q.Workspace(Q.workspace_bytes(Q.OP_DECODE_ATTEND, B, max_len))
    blocks, nblocks = Q.decode_indexer(cache, xd, Wd, seq_len, max_len, ws_i)
    out = Q.decode_attend(cache, q, seq_len, max_len, blocks, nblocks, ws_a)
    iq, ik, w = Q.index_project(xd, Wd)  # the projections the indexer used (same kernel)
    torch.cuda.synchronize()
    assert ws_i.device_error() == 0 and ws_a.device_error() == 0
    iq, ik, w = bf16_tensor_to_bits(iq), bf16_tensor_to_bits(ik), w.cpu().numpy()
    _check_projection(iq, ik, w, x, Wp, what="decode projection")
    bl, nbl = blocks.cpu().numpy(), nblocks.cpu().numpy()
    got = bf16_tensor_to_f32(out)
    for r, L in enumerate(lens):
        # the oracle from the GPU's projected values on: append the key, select, attend
        comp, ring, _ = oracle_state(wl, r, L - 1)
        O.append(ring, comp, ik[r], L - 1, wl.rope_theta)
        ob, opos, s = O.select_query(iq[r], w[r], comp, L, wl.rope_theta)
        sel = check_selection(bl[r, :nbl[r]], ob, s, L // 4, what=f"request {r} L={L}")
        pos = opos if np.array_equal(sel, ob) else O.expand(sel.astype(np.int32), L)
        ref, _ = O.sparse_gqa(wl.q(r)[0], wl.k(r), wl.v(r), pos)
        check_attention(got[r], ref, what=f"request {r} L={L}")
        # the appended key left the cache as the oracle's
        if L % 4 == 0:
            pt = wl.page_table()[r]
            b = L // 4 - 1
            e = (int(pt[(4 * b) // 64]) * 64 + (4 * b) % 64) // 4
            np.testing.assert_array_equal(bf16_tensor_to_bits(cache.cidx[e]), comp[b])
        else:
            np.testing.assert_array_equal(bf16_tensor_to_bits(cache.ring[r, (L - 1) % 4]), ik[r])


def test_indexer_on_second_stream_overlapping_main_projection(Q, W):
    lens = [120001, 125000, 131072, 9000]
    wl, cache, x, Wp, xd, Wd, seq_len, q, max_len = _projected_case(Q, W, lens, 73)
    B = wl.batch
    # the caller's main Q/K/V projection (16 query + 2 key + 2 value heads of 128) runs on the current
    # stream while the indexer runs on a second one
    w_qkv = torch.randn(HIDDEN, (16 + 4) * 128, device="cuda", dtype=torch.bfloat16) * HIDDEN ** -0.5
    ws_i = Q.Workspace(Q.workspace_bytes(Q.OP_DECODE_INDEXER, B, max_len))
    ws_a = Q.Workspace(Q.workspace_bytes(Q.OP_DECODE_ATTEND, B, max_len))
    torch.cuda.synchronize()
    main = torch.cuda.current_stream()
    side = torch.cuda.Stream()
    ready = torch.cuda.Event()
    side.wait_stream(main)
    blocks, nblocks = Q.decode_indexer(cache, xd, Wd, seq_len, max_len, ws_i, stream=side)
    ready.record(side)
    qkv = xd @ w_qkv  # stands in for the caller's projection (its outputs are not used here)
    main.wait_event(ready)
    out2 = Q.decode_attend(cache, q, seq_len, max_len, blocks, nblocks, ws_a)
    torch.cuda.synchronize()
    assert qkv.shape == (B, 20 * 128)
    assert ws_i.device_error() == 0 and ws_a.device_error() == 0
    # the same two phases on one stream
    b1, n1 = Q.decode_indexer(cache, xd, Wd, seq_len, max_len, ws_i)
    out1 = Q.decode_attend(cache, q, seq_len, max_len, b1, n1, ws_a)
    # qsa_decode fed with the projected inputs
    iq, ik, w = Q.index_project(xd, Wd)
    ws = Q.Workspace(Q.workspace_bytes(Q.OP_DECODE, B, max_len))
    b0 = torch.full((B, 512), -1, dtype=torch.int32, device="cuda")
    n0 = torch.zeros(B, dtype=torch.int32, device="cuda")
    out0 = Q.decode(cache, ik, iq, w, q, seq_len, max_len, ws, blocks_out=b0, nblocks_out=n0)
    torch.cuda.synchronize()
    assert ws.device_error() == 0
    assert torch.equal(blocks, b1) and torch.equal(nblocks, n1) and torch.equal(blocks, b0)
    assert torch.equal(out2.view(torch.int16), out1.view(torch.int16))
    assert torch.equal(out2.view(torch.int16), out0.view(torch.int16))
