"""FP8 (E4M3) K/V: qsa_sparse_gqa_fp8 and qsa_decode_fp8 against the CPU oracle.

The oracle decodes the same E4M3 codes from the format's definition and attends in FP64; the GPU's
outputs must match within 2e-2 max-abs / 5e-3 mean-abs (on the GPU's own selection for the decode
step, whose index path is the bf16 one of qsa_decode, checked under the near-tie rule).
"""
import numpy as np
import pytest
import torch

import oracle as O
import qsa_gen as G
from harness import bf16_tensor_to_f32, check_attention, check_selection, oracle_decode_request

pytestmark = pytest.mark.gpu

K_SCALE, V_SCALE = 0.5, 0.25


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


@pytest.mark.parametrize("kv_layout", ["interleaved", "separate"])
def test_sparse_gqa_fp8_matches_oracle(Q, W, kv_layout):
    wl = G.custom_decode(81, [5000, 3000])
    cache = W.build_cache(wl, prefix_tokens=[0, 0], kv_layout=kv_layout, kv_dtype="fp8")
    rng = np.random.default_rng(81)
    cases = [(0, 0), (0, 1), (1, 17), (0, 2051), (1, 1000), (0, 33), (1, 2051), (0, 2048)]
    nq = len(cases)
    pos = np.full((nq, 2051), -1, dtype=np.int32)
    npos = np.zeros(nq, dtype=np.int32)
    for i, (r, n) in enumerate(cases):
        pos[i, :n] = np.sort(rng.choice(int(wl.lens[r]), size=n, replace=False))
        npos[i] = n
    q = G.normal_bf16(81, 2000, (nq, 16, 128))
    q_req = np.array([r for r, _ in cases], dtype=np.int32)
    ws = Q.Workspace(Q.workspace_bytes(Q.OP_SPARSE_GQA, nq, 2051))
    lse = torch.empty(nq, 16, dtype=torch.float32, device="cuda")
    out = Q.sparse_gqa_fp8(cache, W.bits_to_bf16(q, "cuda"), torch.from_numpy(q_req).cuda(),
                           torch.from_numpy(pos).cuda(), torch.from_numpy(npos).cuda(), 2051, ws, K_SCALE, V_SCALE,
                           lse=lse)
    torch.cuda.synchronize()
    assert ws.device_error() == 0
    out = bf16_tensor_to_f32(out)
    lse = lse.cpu().numpy()
    KV = {r: (wl.k8(r), wl.v8(r)) for r in range(2)}
    for i, (r, n) in enumerate(cases):
        ro, rl = O.sparse_gqa_fp8(q[i], KV[r][0], KV[r][1], K_SCALE, V_SCALE, pos[i, :n])
        if n == 0:
            assert np.all(out[i] == 0) and np.all(np.isneginf(lse[i]))
            continue
        check_attention(out[i], ro, what=f"fp8 case {i} ({n} positions)")
        np.testing.assert_allclose(lse[i], rl, atol=2e-3, rtol=0)


def _decode_fp8(Q, W, wl):
    cache = W.build_cache(wl, kv_dtype="fp8")
    inp = W.decode_inputs(wl)
    B, max_len = wl.batch, int(max(wl.lens))
    ws = Q.Workspace(Q.workspace_bytes(Q.OP_DECODE, B, max_len))
    blocks = torch.full((B, 512), -1, dtype=torch.int32, device="cuda")
    nblocks = torch.zeros(B, dtype=torch.int32, device="cuda")
    out = Q.decode_fp8(cache, inp["idx_k_new"], inp["idx_q"], inp["w"], inp["q"], inp["seq_len"], max_len, ws,
                       K_SCALE, V_SCALE, blocks_out=blocks, nblocks_out=nblocks)
    torch.cuda.synchronize()
    assert ws.device_error() == 0
    return bf16_tensor_to_f32(out), blocks.cpu().numpy(), nblocks.cpu().numpy()


def _check_fp8_rows(wl, out, bl, nbl, rows):
    for r in rows:
        o = oracle_decode_request(wl, r)  # selection: the bf16 index path
        L = o["L"]
        sel = check_selection(bl[r, :nbl[r]], o["blocks"], o["scores"], L // 4, what=f"request {r}")
        pos = o["pos"] if np.array_equal(sel, o["blocks"]) else O.expand(sel.astype(np.int32), L)
        ref, _ = O.sparse_gqa_fp8(wl.q(r)[0], wl.k8(r, 0, L), wl.v8(r, 0, L), K_SCALE, V_SCALE, pos)
        check_attention(out[r], ref, what=f"fp8 decode request {r} L={L}")


def test_decode_fp8_small_batch_matches_oracle(Q, W):
    wl = G.decode_small()
    out, bl, nbl = _decode_fp8(Q, W, wl)
    _check_fp8_rows(wl, out, bl, nbl, range(wl.batch))


def test_decode_fp8_128k_batch64_sampled(Q, W):
    """The benchmark's workload with an FP8 K/V pool: every row valid, sampled rows against the oracle."""
    wl = G.decode_128k()
    out, bl, nbl = _decode_fp8(Q, W, wl)
    assert np.all(np.isfinite(out))
    for r in range(wl.batch):
        nb = int(wl.lens[r]) // 4
        b = bl[r, :nbl[r]]
        assert nbl[r] == min(nb, 512) and np.all(np.diff(b) > 0) and b[-1] < nb
    _check_fp8_rows(wl, out, bl, nbl, (0, 29, 63))
