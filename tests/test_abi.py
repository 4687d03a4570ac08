"""CPU-only checks of the C ABI: the library builds for sm_100a, loads without a GPU, exports every
entry point that include/qsa.h declares, sizes workspaces, and rejects bad arguments before it
touches the GPU.  No compute call is made here."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def qsa():
    from block_sparse_attention_c4_b200 import build

    build.build()
    import block_sparse_attention_c4_b200 as Q

    Q.lib()
    return Q


def declared_functions():
    hdr = open(os.path.join(ROOT, "include", "qsa.h")).read()
    hdr = re.sub(r"/\*.*?\*/", "", hdr, flags=re.S)
    return sorted(set(re.findall(r"\b(qsa_[a-z0-9_]+)\s*\(", hdr)))


def test_header_declarations_are_exported(qsa):
    names = declared_functions()
    assert len(names) >= 13
    for n in names:
        assert hasattr(qsa.lib(), n), f"{n} declared in qsa.h but not exported"
    assert set(qsa.EXPORTS) <= set(names)


def test_version_and_status_strings(qsa):
    assert "sm_100a" in qsa.version()
    for s in range(5):
        assert qsa.lib().qsa_status_string(s)
    assert qsa.decode_kernel_count(64) == 2 and qsa.decode_kernel_count(512) == 2
    assert qsa.decode_kernel_count(513) == 3


def test_workspace_bytes(qsa):
    for op in (qsa.OP_INDEX_SCORE_TOPK, qsa.OP_SPARSE_GQA, qsa.OP_DECODE, qsa.OP_DECODE_INDEXSHARE,
               qsa.OP_COMPRESS_APPEND):
        n = qsa.workspace_bytes(op, 64, 131072)
        assert n > 0 and n % 256 == 0
    assert qsa.workspace_bytes(99, 4, 100) == 0
    assert qsa.workspace_bytes(qsa.OP_DECODE, -1, 100) == 0
    assert qsa.workspace_bytes(qsa.OP_DECODE, 4, (1 << 20) + 1) == 0
    # grows with the batch and with the context (candidate buffers)
    assert qsa.workspace_bytes(qsa.OP_DECODE, 64, 131072) > qsa.workspace_bytes(qsa.OP_DECODE, 4, 131072)
    assert qsa.workspace_bytes(qsa.OP_DECODE, 4, 262147) > qsa.workspace_bytes(qsa.OP_DECODE, 4, 8192)


def fake_cache(qsa, **kw):
    c = qsa.CacheStruct(0x1000, 0x2000, 0x3000, 0x4000, 0x5000, 64 * 100, 64, 10, 4, 0, 1e7)
    for k, v in kw.items():
        setattr(c, k, v)
    return c


def test_invalid_arguments_are_rejected_before_launch(qsa):
    L = qsa.lib()
    ws = ctypes.c_void_p(0x100000)
    big = 1 << 40
    INVALID, UNSUPPORTED, WORKSPACE = 1, 2, 3
    c = fake_cache(qsa)
    p = ctypes.c_void_p(0x10000)
    # null cache / null pool pointers
    assert L.qsa_decode(None, p, p, p, p, p, 100, 0.1, p, None, None, None, ws, big, None) == INVALID
    bad = fake_cache(qsa, k=None)
    assert L.qsa_decode(ctypes.byref(bad), p, p, p, p, p, 100, 0.1, p, None, None, None, ws, big, None) == INVALID
    # page size other than 64
    bad = fake_cache(qsa, page_size=32)
    assert L.qsa_decode(ctypes.byref(bad), p, p, p, p, p, 100, 0.1, p, None, None, None, ws, big, None) == UNSUPPORTED
    # num_slots not a multiple of the page
    bad = fake_cache(qsa, num_slots=100)
    assert L.qsa_decode(ctypes.byref(bad), p, p, p, p, p, 100, 0.1, p, None, None, None, ws, big, None) == INVALID
    # misaligned pool pointer
    bad = fake_cache(qsa, k=0x1002)
    assert L.qsa_decode(ctypes.byref(bad), p, p, p, p, p, 100, 0.1, p, None, None, None, ws, big, None) == INVALID
    # slot stride below the two KV heads' rows, or not a whole number of 16-byte chunks
    for stride in (128, 255, 260):
        bad = fake_cache(qsa, kv_stride=stride)
        assert L.qsa_decode(ctypes.byref(bad), p, p, p, p, p, 100, 0.1, p, None, None, None, ws, big, None) == INVALID
        assert L.qsa_sparse_gqa_noalloc(ctypes.byref(bad), p, p, p, p, 10, 10, 1, 0.1, p, None, None) == INVALID
    # max_len beyond the page table
    assert L.qsa_decode(ctypes.byref(c), p, p, p, p, p, 641, 0.1, p, None, None, None, ws, big, None) == INVALID
    # non-positive scale
    assert L.qsa_decode(ctypes.byref(c), p, p, p, p, p, 100, 0.0, p, None, None, None, ws, big, None) == INVALID
    # only one of blocks_out / nblocks_out
    assert L.qsa_decode(ctypes.byref(c), p, p, p, p, p, 100, 0.1, p, None, p, None, ws, big, None) == INVALID
    # workspace: null, misaligned, too small
    assert L.qsa_decode(ctypes.byref(c), p, p, p, p, p, 100, 0.1, p, None, None, None, None, big, None) == WORKSPACE
    assert L.qsa_decode(ctypes.byref(c), p, p, p, p, p, 100, 0.1, p, None, None, None,
                        ctypes.c_void_p(0x100010), big, None) == WORKSPACE
    assert L.qsa_decode(ctypes.byref(c), p, p, p, p, p, 100, 0.1, p, None, None, None, ws, 1024, None) == WORKSPACE
    # empty batch: nothing to do, nothing launched
    empty = fake_cache(qsa, batch=0)
    assert L.qsa_decode(ctypes.byref(empty), p, p, p, p, p, 100, 0.1, p, None, None, None, ws, 0, None) == 0
    # index scoring: nq == 0 is a no-op; negative nq or missing outputs are invalid
    assert L.qsa_index_score_topk(ctypes.byref(c), p, p, p, p, 0, 100, p, p, ws, big, None) == 0
    assert L.qsa_index_score_topk(ctypes.byref(c), p, p, p, p, -1, 100, p, p, ws, big, None) == INVALID
    assert L.qsa_index_score_topk(ctypes.byref(c), p, p, p, p, 4, 100, None, p, ws, big, None) == INVALID
    # sparse GQA: max_pos beyond the stride, zero queries
    assert L.qsa_sparse_gqa(ctypes.byref(c), p, p, p, p, 100, 200, 4, 0.1, p, None, ws, big, None) == INVALID
    assert L.qsa_sparse_gqa(ctypes.byref(c), p, p, p, p, 100, 100, 0, 0.1, p, None, ws, big, None) == 0
    # IndexShare: draft count outside 1..8
    for n in (0, 9):
        assert L.qsa_decode_indexshare(ctypes.byref(c), p, p, 2051, p, n, p, 0.1, p, ws, big, None) == UNSUPPORTED
    assert L.qsa_decode_indexshare(ctypes.byref(c), p, p, 3000, p, 4, p, 0.1, p, ws, big, None) == INVALID
    # expansion and append argument checks
    assert L.qsa_expand_indices(None, p, p, 4, p, p, None) == INVALID
    assert L.qsa_expand_indices(p, p, p, 0, p, p, None) == 0
    assert L.qsa_compress_append(ctypes.byref(c), p, p, p, -1, 0, None) == INVALID
    assert L.qsa_compress_append(ctypes.byref(c), p, p, p, 0, 0, None) == 0
    # a non-finite or non-positive scale is rejected by both sparse-GQA entry points alike
    for sc in (float("inf"), float("nan"), 0.0, -1.0):
        assert L.qsa_sparse_gqa(ctypes.byref(c), p, p, p, p, 100, 100, 4, sc, p, None, ws, big, None) == INVALID
        assert L.qsa_sparse_gqa_noalloc(ctypes.byref(c), p, p, p, p, 100, 100, 4, sc, p, None, None) == INVALID
        assert L.qsa_decode(ctypes.byref(c), p, p, p, p, p, 100, sc, p, None, None, None, ws, big, None) == INVALID
    # a pool too large for 32-bit page ids, rejected by both
    huge = fake_cache(qsa, num_slots=64 * (1 << 31))
    assert L.qsa_sparse_gqa(ctypes.byref(huge), p, p, p, p, 100, 100, 4, 0.1, p, None, ws, big, None) == UNSUPPORTED
    assert L.qsa_sparse_gqa_noalloc(ctypes.byref(huge), p, p, p, p, 100, 100, 4, 0.1, p, None, None) == UNSUPPORTED
    # bounded-wait check: limit in 1 ns .. 2 s, outputs present
    assert L.qsa_check_bounded_wait(ctypes.byref(c), p, p, 0, ws, big, None) == INVALID
    assert L.qsa_check_bounded_wait(ctypes.byref(c), p, p, 2_000_000_001, ws, big, None) == INVALID
    assert L.qsa_check_bounded_wait(ctypes.byref(c), p, None, 1000, ws, big, None) == INVALID
    assert L.qsa_check_bounded_wait(ctypes.byref(c), p, p, 1000, ws, 16, None) == WORKSPACE
    # workspace init rejects misaligned memory
    assert L.qsa_workspace_init(ctypes.c_void_p(0x100010), 1024, None) == WORKSPACE


def test_python_binding_fails_loudly_without_library(tmp_path, monkeypatch):
    import block_sparse_attention_c4_b200 as Q

    monkeypatch.setattr(Q, "LIB_PATH", str(tmp_path / "missing.so"))
    monkeypatch.setattr(Q, "_lib", None)
    with pytest.raises(Q.QsaError):
        Q.lib()


def test_decode_inputs_pack_into_one_buffer():
    """A decode step's host inputs are views of one contiguous buffer, so a step moves them with a
    single copy; the views keep their dtypes, shapes and 256-byte alignment, and a buffer-to-buffer
    copy carries every input (CPU tensors here; the session does the same host -> device)."""
    import torch

    import block_sparse_attention_c4_b200 as Q

    B = 5
    specs = Q.DecodeSession.input_specs(B)
    src = Q.PackedInputs(specs)
    dst = Q.PackedInputs(specs)
    g = torch.Generator().manual_seed(3)
    for name, shape, dtype in specs:
        v = src.views[name]
        assert v.shape == torch.Size(shape) and v.dtype == dtype and v.is_contiguous()
        assert (v.data_ptr() - src.buf.data_ptr()) % Q.PackedInputs.ALIGN == 0
        if dtype == torch.int32:
            v.copy_(torch.randint(0, 1 << 20, shape, generator=g, dtype=torch.int32))
        else:
            v.copy_(torch.randn(shape, generator=g).to(dtype))
    dst.copy_from(src, non_blocking=False)
    for name, _, _ in specs:
        assert torch.equal(dst.views[name], src.views[name])
    assert src.payload_bytes == B * (128 * 2 + 4 * 128 * 2 + 4 * 4 + 16 * 128 * 2 + 4)
    assert set(n for n, _, _ in specs) == set(Q.DecodeSession.INPUTS)
