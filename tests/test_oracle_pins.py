"""Pins of the CPU oracle against facts that do not come from the oracle itself.

Each test checks one step of the oracle against what the QSA description and
plain mathematics fix: printed structural numbers (tests/golden), closed forms,
invariants, special cases that reduce to a library routine (numpy, torch CPU in
float64), and brute force on tiny inputs.  Together they are chosen so that a
dropped term, a wrong sign or index, or swapped operands in any oracle step
fails at least one of them.
"""
import json
import os

import numpy as np
import pytest
import torch

import oracle as O
import qsa_gen as G

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "qsa_c4_structure.json")
THETA = 1.0e7


def f32(bits):
    return G.bf16_bits_to_f32(np.asarray(bits, dtype=np.uint16))


def bf16_ulp(x):
    """Spacing of bf16 numbers at |x| (normal range)."""
    e = np.floor(np.log2(np.maximum(np.abs(x), 1e-30)))
    return 2.0 ** (e - 7)


def to_bf16_bits_torch(x64):
    """float64 -> bf16 via torch, only for values exactly representable in float32."""
    t = torch.from_numpy(np.asarray(x64, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


# --- golden: the numbers the description prints ----------------------------------

def test_golden_structure(oracle_lib):
    facts = {f["name"]: f["value"] for f in json.load(open(GOLDEN))["facts"]}
    assert facts["compression_ratio"] == O.C
    assert facts["index_query_heads"] == O.HI
    assert facts["index_head_dim"] == O.D
    assert facts["kept_blocks"] == O.TOPK
    assert facts["max_positions"] == O.MAX_POS == O.TOPK * O.C + facts["tail_max"]
    # 512 kept blocks expand to exactly 2048 positions when there is no tail
    L = 4 * 5000
    s = np.random.default_rng(0).random(L // 4)
    blocks = O.select_topk(s)
    assert len(blocks) == facts["kept_blocks"]
    assert len(O.expand(blocks, L)) == facts["expanded_positions"]
    # the tail adds 0..3 tokens; the maximum number of positions is reached at L mod 4 == 3
    for tail in range(4):
        assert len(O.expand(blocks, L + tail)) == facts["expanded_positions"] + tail
    assert len(O.expand(blocks, L + 3)) == facts["max_positions"]
    # one compressed key per 4 tokens; the ring keeps 4 raw keys
    raw = G.normal_bf16(0, 99, (37, 128))
    assert O.compress(raw).shape[0] == int(37 * facts["compressed_keys_per_token"])
    ring = np.zeros((facts["ring_slots"], 128), dtype=np.uint16)
    comp = np.zeros((10, 128), dtype=np.uint16)
    for p in range(8):
        O.append(ring, comp, raw[p], p)
    assert np.array_equal(ring, raw[4:8])


# --- bf16 rounding ------------------------------------------------------------------

def test_bf16_rounding_matches_torch_on_float_values(oracle_lib):
    rng = np.random.default_rng(1)
    x = np.concatenate([rng.standard_normal(20000), rng.standard_normal(2000) * 1e-30,
                        rng.standard_normal(2000) * 1e30]).astype(np.float32).astype(np.float64)
    ours = np.array([O.f64_to_bf16(v) for v in x], dtype=np.uint16)
    assert np.array_equal(ours, to_bf16_bits_torch(x))


def test_bf16_rounding_ties_and_specials(oracle_lib):
    one = 0x3F80
    assert O.f64_to_bf16(1.0) == one
    assert O.f64_to_bf16(1.0 + 2.0 ** -8) == one                    # tie -> even (down)
    assert O.f64_to_bf16(1.0 + 3 * 2.0 ** -8) == one + 2             # tie -> even (up)
    assert O.f64_to_bf16(1.0 + 2.0 ** -8 + 2.0 ** -40) == one + 1    # just above the tie: FP64 bits matter
    assert O.f64_to_bf16(-2.0) == 0xC000
    assert O.f64_to_bf16(0.0) == 0 and O.f64_to_bf16(-0.0) == 0x8000
    assert O.f64_to_bf16(2.0 ** -133) == 0x0001                      # smallest bf16 subnormal
    assert O.f64_to_bf16(3.5e38) == 0x7F80                           # overflow -> inf


# --- RoPE -----------------------------------------------------------------------------

def test_rope_equals_complex_rotation(oracle_lib):
    """Pairs (i, i+64) rotate as complex numbers x_i + j x_{i+64} times exp(j * pos * theta^(-i/64))."""
    rng = np.random.default_rng(2)
    x = rng.standard_normal((6, 128))
    pos = np.array([0.0, 1.0, 7.0, 4096.0, 131071.0, 262146.0])
    y = O.rope(x, pos, THETA)
    z = x[:, :64] + 1j * x[:, 64:]
    freq = THETA ** (-np.arange(64) / 64.0)
    zr = z * np.exp(1j * pos[:, None] * freq[None, :])
    ref = np.concatenate([zr.real, zr.imag], axis=1)
    np.testing.assert_allclose(y, ref, rtol=0, atol=1e-12)


def test_rope_is_isometry_identity_at_zero_and_relative(oracle_lib):
    rng = np.random.default_rng(3)
    q = rng.standard_normal((4, 128))
    k = rng.standard_normal((4, 128))
    y = O.rope(q, 12345.0)
    np.testing.assert_allclose(np.linalg.norm(y, axis=1), np.linalg.norm(q, axis=1), rtol=1e-13)
    np.testing.assert_array_equal(O.rope(q, 0.0), q)
    for p, s, delta in [(100, 20, 7), (262146, 4, 1000), (4097, 4096, 65536)]:
        a = np.sum(O.rope(q, p) * O.rope(k, s), axis=1)
        b = np.sum(O.rope(q, p + delta) * O.rope(k, s + delta), axis=1)
        np.testing.assert_allclose(a, b, rtol=0, atol=1e-9)
    # the dot product depends on p - s, and not only on |p - s|: a sign error in the angle breaks this
    a = np.sum(O.rope(q, 50) * O.rope(k, 10), axis=1)
    b = np.sum(O.rope(q, 10) * O.rope(k, 50), axis=1)
    assert np.max(np.abs(a - b)) > 1e-3


# --- compression ------------------------------------------------------------------------

def test_compress_block_at_position_zero_is_normalized_mean(oracle_lib):
    """Block 0 rotates by angle 0: k^ = bf16(m / ||m||) with m the float32 mean of the 4 keys."""
    raw = G.normal_bf16(0, 11, (4, 128))
    m = f32(raw).astype(np.float32).sum(axis=0, dtype=np.float32) * np.float32(0.25)
    ref = m.astype(np.float64) / np.linalg.norm(m.astype(np.float64))
    got = f32(O.compress_block(raw, 0)).astype(np.float64)
    assert np.all(np.abs(got - ref) <= 0.5 * bf16_ulp(ref) * (1 + 1e-12))


def test_compress_block_general_position_closed_form(oracle_lib):
    """For any block b: undoing the rotation at 4b gives the normalized mean up to bf16 rounding,
    and the stored key is the nearest bf16 of the rotated normalized mean."""
    for b in [1, 17, 1023, 65535]:
        raw = G.normal_bf16(1, 12 + b, (4, 128))
        m = f32(raw).sum(axis=0, dtype=np.float32) * np.float32(0.25)
        unit = m.astype(np.float64) / np.linalg.norm(m.astype(np.float64))
        z = unit[:64] + 1j * unit[64:]
        zr = z * np.exp(1j * 4 * b * THETA ** (-np.arange(64) / 64.0))
        ref = np.concatenate([zr.real, zr.imag])
        got = f32(O.compress_block(raw, b)).astype(np.float64)
        assert np.all(np.abs(got - ref) <= 0.5 * bf16_ulp(ref) * (1 + 1e-9) + 1e-300)
        assert abs(np.linalg.norm(got) - 1.0) < 128 ** 0.5 * 2 ** -9
        back = O.rope(got, -4.0 * b)[0]
        np.testing.assert_allclose(back, unit, atol=2 ** -8)


def test_compress_invariances(oracle_lib):
    raw = G.normal_bf16(2, 13, (4, 128))
    # four copies of one key: the mean is that key
    same = np.repeat(raw[:1], 4, axis=0)
    k = f32(raw[0]).astype(np.float64)
    np.testing.assert_array_equal(O.compress_block(same, 0), O.compress_block(np.repeat(raw[:1], 4, 0), 0))
    got = f32(O.compress_block(same, 0)).astype(np.float64)
    assert np.all(np.abs(got - k / np.linalg.norm(k)) <= 0.5 * bf16_ulp(k / np.linalg.norm(k)) + 1e-300)
    # scaling every raw key by 2 (exact in bf16) leaves the normalized key unchanged
    doubled = to_bf16_bits_torch(f32(raw).astype(np.float64) * 2.0)
    np.testing.assert_array_equal(O.compress_block(doubled, 9), O.compress_block(raw, 9))
    # the order of the 4 keys does not matter up to FP32 rounding of the mean
    perm = raw[[3, 1, 0, 2]]
    a = f32(O.compress_block(perm, 5)).astype(np.float64)
    b = f32(O.compress_block(raw, 5)).astype(np.float64)
    assert np.max(np.abs(a - b)) <= np.max(bf16_ulp(b))
    # a block whose mean is zero stays zero (no NaN)
    zero = np.concatenate([raw[:2], to_bf16_bits_torch(-f32(raw[:2]).astype(np.float64))])
    assert np.all(f32(O.compress_block(zero, 3)) == 0.0)


def test_ring_appends_equal_bulk_compression(oracle_lib):
    n = 4 * 37 + 3
    raw = G.normal_bf16(3, 14, (n, 128))
    bulk = O.compress(raw)
    ring = np.zeros((4, 128), dtype=np.uint16)
    comp = np.zeros((n // 4, 128), dtype=np.uint16)
    for p in range(n):
        O.append(ring, comp, raw[p], p)
    np.testing.assert_array_equal(comp, bulk)
    np.testing.assert_array_equal(ring[:3], raw[n - 3:])
    # chunked (like chunked prefill): compress a prefix in bulk, then append the rest
    comp2 = np.zeros_like(comp)
    comp2[:20] = O.compress(raw[:80])
    ring2 = np.zeros((4, 128), dtype=np.uint16)
    for p in range(80, n):
        O.append(ring2, comp2, raw[p], p)
    np.testing.assert_array_equal(comp2, bulk)


# --- index query rotation and block scores ------------------------------------------------

def test_rotate_query_is_rounded_rope(oracle_lib):
    q = G.normal_bf16(4, 15, (4, 128))
    for pos in [0, 5, 131071, 262146]:
        got = f32(O.rotate_query(q, pos)).astype(np.float64)
        ref = O.rope(f32(q).astype(np.float64), float(pos))
        assert np.all(np.abs(got - ref) <= 0.5 * bf16_ulp(ref) * (1 + 1e-9) + 1e-300)


def test_block_scores_brute_force(oracle_lib):
    rng = np.random.default_rng(5)
    qrot = G.normal_bf16(5, 16, (4, 128))
    comp = G.normal_bf16(5, 17, (300, 128))
    w = rng.random(4).astype(np.float32)
    s = O.block_scores(qrot, w, comp)
    dots = f32(comp).astype(np.float64) @ f32(qrot).astype(np.float64).T      # [nb, 4]
    ref = (np.maximum(dots, 0.0) * w.astype(np.float64)[None, :]).sum(axis=1)
    np.testing.assert_allclose(s, ref, rtol=1e-12, atol=1e-12)
    # one-hot weights isolate one head; the ReLU clips negative dots to exactly zero
    for h in range(4):
        e = np.zeros(4, dtype=np.float32)
        e[h] = 1.0
        sh = O.block_scores(qrot, e, comp)
        np.testing.assert_allclose(sh, np.maximum(dots[:, h], 0.0), rtol=1e-12, atol=1e-12)
        assert np.all(sh[dots[:, h] < 0] == 0.0)
    # zero weights -> all scores zero
    assert np.all(O.block_scores(qrot, np.zeros(4, np.float32), comp) == 0.0)


# --- top-512 -----------------------------------------------------------------------------------

def test_topk_matches_lexsort(oracle_lib):
    rng = np.random.default_rng(6)
    for nb in [1, 511, 512, 513, 1000, 4096, 33000]:
        for quant in [None, 8]:
            s = rng.random(nb)
            if quant:
                s = np.floor(s * quant) / quant  # many exact ties
            got = O.select_topk(s)
            order = np.lexsort((np.arange(nb), -s))     # score desc, then index asc
            ref = np.sort(order[:512])
            np.testing.assert_array_equal(got, ref)


def test_topk_ties_prefer_lower_index(oracle_lib):
    s = np.zeros(2000)
    np.testing.assert_array_equal(O.select_topk(s), np.arange(512))
    s[1500:] = 1.0  # 500 strictly larger scores, then 12 zeros from the lowest indices
    np.testing.assert_array_equal(O.select_topk(s), np.concatenate([np.arange(12), np.arange(1500, 2000)]))


# --- expansion --------------------------------------------------------------------------------

def test_expand_invariants(oracle_lib):
    rng = np.random.default_rng(7)
    for L in [1, 2, 3, 4, 5, 2047, 2048, 2049, 2050, 2051, 2052, 2053, 4097, 6002, 8191, 8192, 131071, 262147]:
        nb = L // 4
        blocks = O.select_topk(rng.random(nb)) if nb else np.zeros(0, np.int32)
        pos = O.expand(blocks, L)
        assert len(pos) == 4 * min(nb, 512) + L % 4 <= 2051
        assert np.all(np.diff(pos) > 0)                         # sorted, distinct
        assert pos.min(initial=0) >= 0 and pos.max(initial=0) <= L - 1   # causal and in range
        assert np.sum(pos >= 4 * nb) == L % 4                    # exactly the tail tokens
        if nb <= 512:
            np.testing.assert_array_equal(pos, np.arange(L))      # short context: everything
        assert set(pos[pos < 4 * nb] // 4) == set(blocks.tolist())


# --- attention --------------------------------------------------------------------------------

def _sdpa_ref(q, K, V, pos):
    """torch float64 scaled_dot_product_attention with GQA over the gathered rows."""
    qt = torch.from_numpy(f32(q).astype(np.float64)).view(1, 16, 1, 128)
    kt = torch.from_numpy(f32(K[pos]).astype(np.float64)).permute(1, 0, 2).unsqueeze(0)  # [1,2,n,128]
    vt = torch.from_numpy(f32(V[pos]).astype(np.float64)).permute(1, 0, 2).unsqueeze(0)
    o = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, enable_gqa=True)
    s = (qt @ kt.repeat_interleave(8, dim=1).transpose(-1, -2)) / np.sqrt(128.0)
    return o.view(16, 128).numpy(), torch.logsumexp(s, dim=-1).view(16).numpy()


def test_sparse_gqa_matches_torch_sdpa(oracle_lib):
    rng = np.random.default_rng(8)
    T = 3000
    K = G.normal_bf16(8, 18, (T, 2, 128))
    V = G.normal_bf16(8, 19, (T, 2, 128))
    q = G.normal_bf16(8, 20, (16, 128))
    for n in [1, 7, 2051]:
        pos = np.sort(rng.choice(T, size=n, replace=False)).astype(np.int32)
        out, lse = O.sparse_gqa(q, K, V, pos)
        ro, rl = _sdpa_ref(q, K, V, pos)
        np.testing.assert_allclose(out, ro, rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(lse, rl, rtol=1e-12, atol=1e-12)
    # a KV head mix-up (h % 2 instead of h // 8) would change heads 1..7 and 8..14
    pos = np.arange(64, dtype=np.int32)
    out, _ = O.sparse_gqa(q, K, V, pos)
    K2 = K.copy()
    K2[:, 1] = K[:, 0]
    V2 = V.copy()
    V2[:, 1] = V[:, 0]
    out2, _ = O.sparse_gqa(q, K2, V2, pos)
    np.testing.assert_array_equal(out[:8], out2[:8])
    assert np.max(np.abs(out[8:] - out2[8:])) > 1e-3


# --- the whole layer ----------------------------------------------------------------------------

@pytest.mark.parametrize("L", [1, 3, 4, 5, 130, 2048, 2051])
def test_short_context_layer_is_dense_causal_gqa(oracle_lib, L):
    """With at most 512 complete blocks every position is attended: QSA == dense causal GQA."""
    wl = G.custom_decode(9, [L])
    raw = wl.idx_keys(0)
    K, V, q = wl.k(0), wl.v(0), wl.q(0)[0]
    comp = np.zeros((max(L // 4, 1), 128), dtype=np.uint16)
    comp[:(L - 1) // 4] = O.compress(raw[:L - 1])
    ring = np.zeros((4, 128), dtype=np.uint16)
    for p in range(4 * ((L - 1) // 4), L - 1):
        ring[p % 4] = raw[p]
    out, blocks, pos = O.decode_batch([L], [ring], [comp], [raw[L - 1]], [wl.idx_q(0)[0]], [wl.w(0)[0]], [q],
                                      [K], [V], nthreads=1)
    np.testing.assert_array_equal(pos[0], np.arange(L))
    ro, _ = _sdpa_ref(q, K, V, np.arange(L))
    np.testing.assert_allclose(out[0], ro, rtol=1e-10, atol=1e-12)
    # the decode append left the same compressed cache as a bulk compression of all L tokens
    np.testing.assert_array_equal(comp[:L // 4], O.compress(raw)[:L // 4])


def test_prefill_rows_short_context_is_dense_causal_attention(oracle_lib):
    """Prefill rows of one sequence: row t (position t, context t + 1) with at most 512 complete blocks
    attends to every position 0..t, i.e. textbook causal attention.  Reference: torch SDPA in FP64
    over the whole sequence with the causal mask j <= t, per KV group.  A context off by one (t or
    t + 2 tokens) or a row read at the wrong position fails it."""
    T = 2051
    wl = G.prefill_32k(seed=13, L=T)
    idx_q, w, q = wl.idx_q(0, 0, T), wl.w(0, 0, T), wl.q(0, 0, T)
    K, V = wl.k(0, 0, T), wl.v(0, 0, T)
    comp = O.compress(wl.idx_keys(0, 0, T))
    rows = np.array([0, 1, 2, 3, 4, 5, 130, 1023, 2047, 2048, 2049, 2050], dtype=np.int64)
    out, blocks = O.prefill_rows(rows, idx_q, w, q, comp, K, V, nthreads=4)
    qt = torch.from_numpy(f32(q[rows]).astype(np.float64)).permute(1, 0, 2).unsqueeze(0)  # [1,16,n,128]
    kt = torch.from_numpy(f32(K).astype(np.float64)).permute(1, 0, 2).unsqueeze(0)         # [1,2,T,128]
    vt = torch.from_numpy(f32(V).astype(np.float64)).permute(1, 0, 2).unsqueeze(0)
    mask = torch.from_numpy(np.arange(T)[None, :] <= rows[:, None])                      # [n, T]
    ref = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=mask, enable_gqa=True)
    ref = ref[0].permute(1, 0, 2).numpy()                                                # [n,16,128]
    np.testing.assert_allclose(out, ref, rtol=1e-10, atol=1e-12)
    for i, t in enumerate(rows):
        np.testing.assert_array_equal(blocks[i], np.arange((t + 1) // 4))


def test_prefill_rows_long_context_rows_follow_the_selection(oracle_lib):
    """Rows with more than 512 complete blocks: each row's kept blocks are the exact top-512 of
    brute-force scores at context t + 1 (numpy matmul, lexsort), and its output is torch SDPA over
    those blocks' positions plus the row's own unfinished block."""
    T = 2600
    wl = G.prefill_32k(seed=14, L=T)
    idx_q, w, q = wl.idx_q(0, 0, T), wl.w(0, 0, T), wl.q(0, 0, T)
    K, V = wl.k(0, 0, T), wl.v(0, 0, T)
    comp = O.compress(wl.idx_keys(0, 0, T))
    rows = np.array([2051, 2052, 2310, 2599], dtype=np.int64)
    out, blocks = O.prefill_rows(rows, idx_q, w, q, comp, K, V, nthreads=4)
    for i, t in enumerate(rows):
        L = int(t) + 1
        qrot = f32(O.rotate_query(idx_q[t], L - 1)).astype(np.float64)  # rotation: pinned above
        dots = f32(comp[:L // 4]).astype(np.float64) @ qrot.T
        s = (np.maximum(dots, 0) * w[t].astype(np.float64)).sum(axis=1)
        ref_blocks = np.sort(np.lexsort((np.arange(len(s)), -s))[:512])
        np.testing.assert_array_equal(blocks[i], ref_blocks)
        pos = np.concatenate([(4 * ref_blocks[:, None] + np.arange(4)).ravel(), np.arange(4 * (L // 4), L)])
        ro, _ = _sdpa_ref(q[t], K, V, pos.astype(np.int32))
        np.testing.assert_allclose(out[i], ro, rtol=1e-10, atol=1e-12)


def test_long_context_selection_is_exact_topk_of_brute_force_scores(oracle_lib):
    wl = G.custom_decode(10, [6002])
    L = 6002
    raw = wl.idx_keys(0)
    comp = O.compress(raw)
    idx_q, w = wl.idx_q(0)[0], wl.w(0)[0]
    blocks, pos, s = O.select_query(idx_q, w, comp, L)
    # independent brute force: rotation by complex numbers, scores by a matmul, order by lexsort
    qf = f32(idx_q).astype(np.float64)
    z = (qf[:, :64] + 1j * qf[:, 64:]) * np.exp(1j * (L - 1) * THETA ** (-np.arange(64) / 64.0))
    qrot_ref = np.concatenate([z.real, z.imag], axis=1)
    qrot = f32(O.rotate_query(idx_q, L - 1)).astype(np.float64)
    assert np.all(np.abs(qrot - qrot_ref) <= 0.5 * bf16_ulp(qrot_ref) + 1e-300)
    dots = f32(comp[:L // 4]).astype(np.float64) @ qrot.T
    ref_s = (np.maximum(dots, 0) * w.astype(np.float64)).sum(axis=1)
    np.testing.assert_allclose(s, ref_s, rtol=1e-12, atol=1e-12)
    ref_blocks = np.sort(np.lexsort((np.arange(len(ref_s)), -ref_s))[:512])
    np.testing.assert_array_equal(blocks, ref_blocks)
    assert len(pos) == 2048 + L % 4


# --- IndexShare -----------------------------------------------------------------------------------

def test_indexshare_rows_are_causal_and_match_explicit_union(oracle_lib):
    wl = G.indexshare_64k(batch=1)
    wl.lens[:] = 5003  # a short capture context keeps this CPU test fast
    L0 = int(wl.lens[0])
    raw = wl.idx_keys(0)
    K, V = wl.k(0), wl.v(0)
    comp = O.compress(raw[:L0])
    blocks, frozen, _ = O.select_query(wl.idx_q(0)[0], wl.w(0)[0], comp, L0)
    q = wl.q(0)
    out = O.indexshare(frozen, L0, 4, q, K, V)
    for i in range(4):
        rows = np.concatenate([frozen, np.arange(L0, L0 + i + 1, dtype=np.int32)])
        assert np.all(np.diff(rows) > 0) and rows.max() == L0 + i and len(rows) <= 2051 + 4
        ro, _ = O.sparse_gqa(q[i], K, V, rows)
        np.testing.assert_array_equal(out[i], ro)
        ref, _ = _sdpa_ref(q[i], K, V, rows)
        np.testing.assert_allclose(out[i], ref, rtol=1e-10, atol=1e-12)


def test_indexshare_short_context_equals_normal_path(oracle_lib):
    """With <=512 blocks the frozen row is every earlier position, so draft i sees 0..L0+i: the
    same rows (and output) as the normal decode path at that position."""
    L0 = 700
    wl = G.custom_decode(12, [L0], extra=4)
    raw = wl.idx_keys(0)
    K, V = wl.k(0), wl.v(0)
    q = G.normal_bf16(12, 77, (4, 16, 128))
    comp = O.compress(raw)
    _, frozen, _ = O.select_query(wl.idx_q(0)[0], wl.w(0)[0], comp, L0)
    out = O.indexshare(frozen, L0, 4, q, K, V)
    for i in range(4):
        _, pos_i, _ = O.select_query(wl.idx_q(0)[0], wl.w(0)[0], comp, L0 + i + 1)
        ro, _ = O.sparse_gqa(q[i], K, V, pos_i)
        np.testing.assert_array_equal(out[i], ro)


# --- index projection ---------------------------------------------------------------------------

def test_index_project_is_rounded_linear_map(oracle_lib):
    """Against a numpy float64 matmul of the decoded values: query heads are features 0..511 (head h,
    dim d at 128h + d), the key 512..639, the head weights 640..643; each bf16 output is the nearest
    bf16 of the exact product (within half an ulp), each weight its float rounding."""
    hidden, n = 512, 5
    x = G.normal_bf16(15, 1, (n, hidden))
    W = G.normal_scaled_bf16(15, 2, (O.PROJ_FEATURES, hidden), hidden ** -0.5)
    idx_q, idx_k, w = O.index_project(x, W, nthreads=2)
    y = f32(x).astype(np.float64) @ f32(W).astype(np.float64).T  # [n, 644]
    yq, yk, yw = y[:, :512].reshape(n, 4, 128), y[:, 512:640], y[:, 640:]
    for got, ref in ((idx_q, yq), (idx_k, yk)):
        g = f32(got).astype(np.float64)
        assert np.all(np.abs(g - ref) <= 0.5 * bf16_ulp(ref) * (1 + 1e-9) + 1e-300)
    np.testing.assert_allclose(w, yw.astype(np.float32), rtol=1e-6, atol=0)
    # swapping the roles of rows and features, or reading W transposed, changes the result
    assert not np.array_equal(idx_q[0, 0], idx_q[1, 0])
    x2 = x.copy()
    x2[:, 0] = x[:, 1]
    x2[:, 1] = x[:, 0]
    q2, _, _ = O.index_project(x2, W, nthreads=1)
    assert not np.array_equal(q2, idx_q)


# --- FP8 K/V ------------------------------------------------------------------------------------

def test_e4m3_decode_matches_torch_on_every_code(oracle_lib):
    """The oracle's E4M3 decode, written from the format's definition, against torch's
    float8_e4m3fn -> float32 conversion for all 256 codes (NaN codes included)."""
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float32).numpy().astype(np.float64)
    got = np.array([O.e4m3_to_f64(b) for b in range(256)])
    assert np.array_equal(np.isnan(got), np.isnan(ref))
    ok = ~np.isnan(ref)
    np.testing.assert_array_equal(got[ok], ref[ok])
    assert got[0x7E] == 448.0 and got[0x01] == 2.0 ** -9 and got[0x08] == 2.0 ** -6


def test_sparse_gqa_fp8_matches_torch_sdpa_on_dequantized_values(oracle_lib):
    rng = np.random.default_rng(16)
    T = 2500
    K8 = G.normal_fp8_e4m3(16, 1, (T, 2, 128), 2.0)
    V8 = G.normal_fp8_e4m3(16, 2, (T, 2, 128), 4.0)
    q = G.normal_bf16(16, 3, (16, 128))
    ks, vs = 0.5, 0.25
    Kd = torch.from_numpy(K8).view(torch.float8_e4m3fn).to(torch.float64).numpy() * ks
    Vd = torch.from_numpy(V8).view(torch.float8_e4m3fn).to(torch.float64).numpy() * vs
    for n in (1, 9, 2051):
        pos = np.sort(rng.choice(T, size=n, replace=False)).astype(np.int32)
        out, lse = O.sparse_gqa_fp8(q, K8, V8, ks, vs, pos)
        qt = torch.from_numpy(f32(q).astype(np.float64)).view(1, 16, 1, 128)
        kt = torch.from_numpy(Kd[pos]).permute(1, 0, 2).unsqueeze(0)
        vt = torch.from_numpy(Vd[pos]).permute(1, 0, 2).unsqueeze(0)
        ro = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, enable_gqa=True).view(16, 128).numpy()
        np.testing.assert_allclose(out, ro, rtol=1e-10, atol=1e-12)
        s = (qt @ kt.repeat_interleave(8, dim=1).transpose(-1, -2)) / np.sqrt(128.0)
        np.testing.assert_allclose(lse, torch.logsumexp(s, dim=-1).view(16).numpy(), rtol=1e-12, atol=1e-12)
    # the K scale and the V scale act where they should: swapping them changes the output
    pos = np.arange(64, dtype=np.int32)
    a, _ = O.sparse_gqa_fp8(q, K8, V8, ks, vs, pos)
    b, _ = O.sparse_gqa_fp8(q, K8, V8, vs, ks, pos)
    assert np.max(np.abs(a - b)) > 1e-3
