"""Failure detection on the GPU without a fault, and the host-buffer session on a side stream.

* A bounded wait made to run out: the decode attention kernel is launched with a selection that
  nothing publishes and a 1 ms limit.  It must give up, record the timeout bit in the workspace's
  error word, write zeros, and leave the CUDA context usable (a normal decode step afterwards
  matches the oracle).  No wait here can hang: the limit ends it.
* DecodeSession.step on a stream other than the current one: both copies and the decode run on
  that stream, and the result matches the oracle.
"""
import time

import numpy as np
import pytest
import torch

import oracle as O
import qsa_gen as G
from harness import bf16_tensor_to_f32, check_attention, check_selection, oracle_decode_request

pytestmark = pytest.mark.gpu

TIMEOUT_BIT = 32


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


def _check_decode_output(wl, out, blocks, nblocks):
    """Kept blocks under the near-tie rule; attention against the oracle on the GPU's own selection."""
    for r in range(wl.batch):
        o = oracle_decode_request(wl, r)
        L = o["L"]
        sel = check_selection(blocks[r, :nblocks[r]], o["blocks"], o["scores"], L // 4, what=f"request {r}")
        ref = o["out"] if np.array_equal(sel, o["blocks"]) else \
            O.sparse_gqa(wl.q(r)[0], o["K"], o["V"], O.expand(sel.astype(np.int32), L))[0]
        check_attention(out[r], ref, what=f"request {r} L={L}")


def test_bounded_wait_gives_up_and_context_stays_usable(Q, W):
    wl = G.custom_decode(61, [3001, 4100])
    cache = W.build_cache(wl)
    ws = Q.Workspace(Q.workspace_bytes(Q.OP_DECODE, 1, 8))
    q = W.bits_to_bf16(wl.q(0)[0], "cuda")
    out = torch.full((16, 128), float("nan"), dtype=torch.bfloat16, device="cuda")
    t0 = time.perf_counter()
    Q.check_bounded_wait(cache, q, out, 1_000_000, ws)  # 1 ms
    torch.cuda.synchronize()
    elapsed = time.perf_counter() - t0
    assert ws.device_error() == TIMEOUT_BIT
    assert int(torch.count_nonzero(out.float())) == 0  # zeros, not NaN and not stale data
    assert elapsed < 1.5  # the wait ended at its limit, far below the default 2 s
    # a second run on the cleared workspace behaves the same
    Q.check_bounded_wait(cache, q, out, 3_000_000, ws)
    torch.cuda.synchronize()
    assert ws.device_error() == TIMEOUT_BIT
    # the context is intact: a normal decode step is correct
    inp = W.decode_inputs(wl)
    ws2 = Q.Workspace(Q.workspace_bytes(Q.OP_DECODE, wl.batch, 4100))
    blocks = torch.full((2, 512), -1, dtype=torch.int32, device="cuda")
    nblocks = torch.zeros(2, dtype=torch.int32, device="cuda")
    res = Q.decode(cache, inp["idx_k_new"], inp["idx_q"], inp["w"], inp["q"], inp["seq_len"], 4100, ws2,
                   blocks_out=blocks, nblocks_out=nblocks)
    torch.cuda.synchronize()
    assert ws2.device_error() == 0
    _check_decode_output(wl, bf16_tensor_to_f32(res), blocks.cpu().numpy(), nblocks.cpu().numpy())


def test_decode_session_on_side_stream_matches_oracle(Q, W):
    wl = G.custom_decode(62, [5003, 2100, 9000])
    cache = W.build_cache(wl)
    inp = W.decode_inputs(wl)
    sess = Q.DecodeSession(cache, int(max(wl.lens)))
    host_in = Q.DecodeSession.pinned_inputs(inp)
    side = torch.cuda.Stream()
    torch.cuda.synchronize()
    # keep the current stream busy so that work wrongly issued there would run out of order
    busy = torch.empty(1 << 28, dtype=torch.uint8, device="cuda")
    for _ in range(3):
        busy.zero_()
    host_out = sess.step(host_in, stream=side)
    side.synchronize()
    got = host_out.float().numpy()
    torch.cuda.synchronize()
    # the GPU's own selection for this step (decode is idempotent: the append was already made)
    ws = Q.Workspace(Q.workspace_bytes(Q.OP_DECODE, wl.batch, int(max(wl.lens))))
    blocks = torch.full((wl.batch, 512), -1, dtype=torch.int32, device="cuda")
    nblocks = torch.zeros(wl.batch, dtype=torch.int32, device="cuda")
    Q.decode(cache, inp["idx_k_new"], inp["idx_q"], inp["w"], inp["q"], inp["seq_len"], int(max(wl.lens)), ws,
             blocks_out=blocks, nblocks_out=nblocks)
    torch.cuda.synchronize()
    _check_decode_output(wl, got, blocks.cpu().numpy(), nblocks.cpu().numpy())
    # the same step on the current stream gives the same bytes
    again = sess.step(host_in).clone()
    torch.cuda.synchronize()
    assert torch.equal(again.view(torch.int16), host_out.view(torch.int16))
