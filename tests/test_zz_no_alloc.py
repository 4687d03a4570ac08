"""qsa_sparse_gqa_noalloc: sparse GQA for callers that cannot allocate device memory.

Some callers cannot give the library a workspace -- a plugin that its host
hands only input and output buffers, code that runs during CUDA-graph capture
(where cudaMalloc is not allowed), or a deployment with a device-memory budget
fixed at start-up.  For them the library keeps its split-K scratch in a static
device array.  These tests call that entry point through the C ABI and check
that it gives what the ordinary workspace entry point gives, on two calls in a
row (the array keeps the previous call's contents, so the second call shows
that nothing stale leaks through), check both against the oracle, run the
query counts where the array's capacity caps the split count (one split per
query above 256 queries, and the stated maximum of 4096 queries, which uses
every arrival counter), and check that sizes past the stated limit are
rejected.  The file sorts last so that a run stopping at the first failure has
already run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle as O
import qsa_gen as G
from harness import ATT_MAX_ABS, ATT_MEAN_ABS, bf16_tensor_to_f32, check_attention

pytestmark = pytest.mark.gpu


def setup_workload():
    return G.custom_decode(31, [6000, 2500, 9000])


@pytest.fixture(scope="module")
def setup():
    from block_sparse_attention_c4_b200 import build

    build.build()
    import block_sparse_attention_c4_b200 as Q
    import block_sparse_attention_c4_b200.workload as W

    assert torch.cuda.is_available(), "needs a CUDA device"
    wl = setup_workload()
    cache = W.build_cache(wl, prefix_tokens=[0, 0, 0])
    rng = np.random.default_rng(7)
    cases = [(0, 2051), (1, 1), (2, 700), (0, 0), (2, 2051), (1, 2048), (0, 37), (2, 1500)]
    nq = len(cases)
    pos = np.full((nq, 2051), -1, dtype=np.int32)
    npos = np.zeros(nq, dtype=np.int32)
    for i, (r, n) in enumerate(cases):
        pos[i, :n] = np.sort(rng.choice(int(wl.lens[r]), size=n, replace=False))
        npos[i] = n
    q = W.bits_to_bf16(G.normal_bf16(31, 3000, (nq, 16, 128)), "cuda")
    q_req = torch.tensor([r for r, _ in cases], dtype=torch.int32, device="cuda")
    return Q, cache, q, q_req, torch.from_numpy(pos).cuda(), torch.from_numpy(npos).cuda()


def close(a, b):
    d = np.abs(bf16_tensor_to_f32(a).astype(np.float64) - bf16_tensor_to_f32(b))
    return d.max() <= ATT_MAX_ABS and d.mean() <= ATT_MEAN_ABS


def test_noalloc_matches_workspace_entry_point_twice(setup):
    Q, cache, q, q_req, pos, npos = setup
    ws = Q.Workspace(Q.workspace_bytes(Q.OP_SPARSE_GQA, q.shape[0], 2051))
    lse_ref = torch.empty(q.shape[0], 16, dtype=torch.float32, device="cuda")
    ref = Q.sparse_gqa(cache, q, q_req, pos, npos, 2051, ws, lse=lse_ref)
    for call in range(2):
        lse = torch.full((q.shape[0], 16), float("nan"), dtype=torch.float32, device="cuda")
        out = torch.full_like(ref, float("nan"))
        Q.sparse_gqa_noalloc(cache, q, q_req, pos, npos, 2051, out=out, lse=lse)
        torch.cuda.synchronize()
        assert close(out, ref), f"call {call}: outputs differ from qsa_sparse_gqa"
        finite = torch.isfinite(lse_ref)
        assert torch.equal(finite, torch.isfinite(lse))
        assert torch.allclose(lse[finite], lse_ref[finite], atol=1e-3, rtol=0)


def test_noalloc_matches_oracle(setup):
    Q, cache, q, q_req, pos, npos = setup
    out = Q.sparse_gqa_noalloc(cache, q, q_req, pos, npos, 2051)
    torch.cuda.synchronize()
    got = bf16_tensor_to_f32(out)
    wl = setup_workload()
    qb = q.view(torch.int16).cpu().numpy().view(np.uint16)
    pp, nn, rr = pos.cpu().numpy(), npos.cpu().numpy(), q_req.cpu().numpy()
    for i in range(q.shape[0]):
        r = int(rr[i])
        ref, _ = O.sparse_gqa(qb[i], wl.k(r), wl.v(r), pp[i, :nn[i]])
        if nn[i] == 0:
            assert np.all(got[i] == 0)
        else:
            check_attention(got[i], ref, what=f"query {i}")


@pytest.mark.parametrize("nq", [300, 4096])
def test_noalloc_capped_splits_match_workspace_entry_point(setup, nq):
    """Many queries: the static array holds at most 512 (query, split) partials, so above 256 queries
    each query runs as one split (written directly), and 4096 queries use every arrival counter."""
    Q, cache, _, _, _, _ = setup
    wl = setup_workload()
    rng = np.random.default_rng(nq)
    reqs = rng.integers(0, 3, nq).astype(np.int32)
    counts = rng.integers(0, 2052, nq).astype(np.int32)
    counts[:4] = [0, 1, 2051, 2048]
    pos = np.full((nq, 2051), -1, dtype=np.int32)
    for i in range(nq):
        n = int(min(counts[i], wl.lens[reqs[i]]))
        counts[i] = n
        pos[i, :n] = np.sort(rng.choice(int(wl.lens[reqs[i]]), size=n, replace=False))
    q = torch.from_numpy(G.normal_bf16(31, 3100 + nq, (nq, 16, 128)).view(np.int16)).cuda().view(torch.bfloat16)
    q_req = torch.from_numpy(reqs).cuda()
    pos_d, npos_d = torch.from_numpy(pos).cuda(), torch.from_numpy(counts).cuda()
    ws = Q.Workspace(Q.workspace_bytes(Q.OP_SPARSE_GQA, nq, 2051))
    ref = Q.sparse_gqa(cache, q, q_req, pos_d, npos_d, 2051, ws)
    for call in range(2):
        out = torch.full_like(ref, float("nan"))
        Q.sparse_gqa_noalloc(cache, q, q_req, pos_d, npos_d, 2051, out=out)
        torch.cuda.synchronize()
        assert close(out, ref), f"nq={nq}, call {call}: outputs differ from qsa_sparse_gqa"
    # a few rows against the oracle as well
    got = bf16_tensor_to_f32(out)
    qb = q.view(torch.int16).cpu().numpy().view(np.uint16)
    for i in list(range(4)) + rng.integers(4, nq, 4).tolist():
        r = int(reqs[i])
        if counts[i] == 0:
            assert np.all(got[i] == 0)
            continue
        o, _ = O.sparse_gqa(qb[i], wl.k(r), wl.v(r), pos[i, :counts[i]])
        check_attention(got[i], o, what=f"nq={nq} query {i}")


def test_noalloc_rejects_too_many_queries(setup):
    Q, cache, q, q_req, pos, npos = setup
    c = cache.struct()
    nq = 4097  # one past the stated limit; rejected before anything is enqueued
    st = Q.lib().qsa_sparse_gqa_noalloc(ctypes.byref(c), ctypes.c_void_p(q.data_ptr()),
                                        ctypes.c_void_p(q_req.data_ptr()), ctypes.c_void_p(pos.data_ptr()),
                                        ctypes.c_void_p(npos.data_ptr()), 2051, 2051, nq, 0.088,
                                        ctypes.c_void_p(q.data_ptr()), None, None)
    assert st == 2  # QSA_ERR_UNSUPPORTED
