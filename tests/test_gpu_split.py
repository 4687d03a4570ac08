"""Split-context decode over virtual ranks on one GPU, against qsa_decode and the CPU oracle.

The ranks of a step run one after another on the same GPU (no kernel of one rank waits on another;
the all-gathers become stacking in rank order).  Each rank has a cache of its own holding its page
range of the 262,147-token long-context request (K/V, compressed keys appended at their global
positions), the rank holding the newest position appends the new index key, and the step's kept
blocks must equal those of a single-GPU qsa_decode on the whole context (the same page scoring
arithmetic), with the attention output matching the oracle.
"""
import numpy as np
import pytest
import torch

import oracle as O
import qsa_gen as G
from harness import bf16_tensor_to_f32, check_attention, check_selection

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


@pytest.fixture(scope="module")
def long_wl():
    wl = G.long_262k()
    return wl, wl.idx_keys(0)


def _rank_cache(Q, W, wl, raw, lo, cnt, L):
    """Rank cache: pages [lo, lo + cnt) of request 0 at local physical pages 0..cnt-1, page-table row
    indexed by the request's logical page; K/V of its tokens; index keys of its positions < L - 1."""
    n_pages = wl.max_pages
    pt = np.full((1, n_pages), -1, dtype=np.int32)
    pt[0, lo:lo + cnt] = np.arange(cnt, dtype=np.int32)
    cache = Q.LayerCache(cnt * 64, 1, n_pages, rope_theta=wl.rope_theta, page_table=torch.from_numpy(pt).cuda())
    t0, t1 = lo * 64, min((lo + cnt) * 64, wl.tokens(0))
    slots = torch.arange(0, t1 - t0, device="cuda")
    cache.k.index_copy_(0, slots, W.bits_to_bf16(wl.k(0, t0, t1 - t0), "cuda"))
    cache.v.index_copy_(0, slots, W.bits_to_bf16(wl.v(0, t0, t1 - t0), "cuda"))
    a1 = min(t1, L - 1)
    if a1 > t0:
        keys = raw[t0:a1]
        Q.compress_append(cache, W.bits_to_bf16(keys, "cuda"), torch.tensor([0, a1 - t0], dtype=torch.int32).cuda(),
                          torch.tensor([t0], dtype=torch.int32).cuda(), a1 - t0)
    return cache


@pytest.mark.parametrize("world,L", [(2, 262144), (4, 262147), (3, 9001)])
def test_split_decode_matches_single_gpu_and_oracle(Q, W, long_wl, world, L):
    from block_sparse_attention_c4_b200 import split as SP

    wl, raw = long_wl
    t = L - 1
    n_pages = (L + 63) // 64
    lo, cnt = SP.partition_pages(n_pages, world)
    ranks = [SP.SplitRank(_rank_cache(Q, W, wl, raw, lo[r], cnt[r], L), [lo[r]], [cnt[r]], L) for r in range(world)]
    knew = W.bits_to_bf16(raw[t:t + 1], "cuda")
    idx_q = W.bits_to_bf16(wl.idx_q(0, q0=t, n=1), "cuda")
    w = torch.from_numpy(wl.w(0, q0=t, n=1)).cuda()
    q = W.bits_to_bf16(wl.q(0, q0=t, n=1), "cuda")
    seq_len = torch.tensor([L], dtype=torch.int32, device="cuda")
    # phase 1 on every rank, exchange, merge (identical on every rank), phase 2, exchange, combine
    for rk in ranks:
        rk.append(knew, [L])
    cands = [rk.score(idx_q, w, seq_len) for rk in ranks]
    stack = [torch.stack([c[i] for c in cands]) for i in range(3)]
    merged = [SP.merge(*stack) for _ in ranks]
    for b, n in merged[1:]:
        assert torch.equal(b, merged[0][0]) and torch.equal(n, merged[0][1])
    blocks, nblocks = merged[0]
    parts = [rk.attend(q, seq_len, blocks, nblocks) for rk in ranks]
    out = SP.combine(torch.stack([p[0] for p in parts]), torch.stack([p[1] for p in parts]))
    torch.cuda.synchronize()
    for rk in ranks:
        assert rk.ws_score.device_error() == 0 and rk.ws_gqa.device_error() == 0
    # single GPU, whole context
    full = W.build_cache(wl, prefix_tokens=[L - 1])
    ws = Q.Workspace(Q.workspace_bytes(Q.OP_DECODE, 1, L))
    b1 = torch.full((1, 512), -1, dtype=torch.int32, device="cuda")
    n1 = torch.zeros(1, dtype=torch.int32, device="cuda")
    out1 = Q.decode(full, knew, idx_q, w, q, seq_len, L, ws, blocks_out=b1, nblocks_out=n1)
    torch.cuda.synchronize()
    assert ws.device_error() == 0
    assert int(nblocks[0]) == int(n1[0]) == min(L // 4, 512)
    assert torch.equal(blocks[0, :nblocks[0]], b1[0, :n1[0]])
    # oracle
    comp = O.compress(raw[:L])
    ob, opos, s = O.select_query(wl.idx_q(0, q0=t, n=1)[0], wl.w(0, q0=t, n=1)[0], comp, L)
    sel = check_selection(blocks[0, :nblocks[0]].cpu().numpy(), ob, s, L // 4, what=f"split world={world}")
    pos = opos if np.array_equal(sel, ob) else O.expand(sel.astype(np.int32), L)
    ref, _ = O.sparse_gqa(wl.q(0, q0=t, n=1)[0], wl.k(0, 0, L), wl.v(0, 0, L), pos)
    check_attention(bf16_tensor_to_f32(out)[0], ref, what=f"split world={world} L={L}")
    check_attention(bf16_tensor_to_f32(out1)[0], ref, what=f"single GPU L={L}")
