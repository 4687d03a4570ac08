"""Test helpers: oracle runs for generated workloads and the parity rules.

Parity rules (the layer's stated tolerances):
  * kept block sets are bit-exact, except when the oracle's 512th and 513th
    best scores lie within 1e-3 relative of each other; then the GPU's set must
    be a valid set of 512 distinct visible blocks whose oracle-score sum
    matches the oracle set's within 1e-4 relative;
  * attention outputs match within 2e-2 max-abs and 5e-3 mean-abs, against the
    oracle run on the GPU's own (validated) selection.
"""
from __future__ import annotations

import numpy as np

import oracle as O
import qsa_gen as G

NEAR_TIE_REL = 1e-3
SCORE_SUM_REL = 1e-4
ATT_MAX_ABS = 2e-2
ATT_MEAN_ABS = 5e-3


def bf16_tensor_to_f32(t) -> np.ndarray:
    import torch

    return t.detach().to(torch.float32).cpu().numpy()


def bf16_tensor_to_bits(t) -> np.ndarray:
    import torch

    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def oracle_state(wl, r: int, L_before: int, raw=None):
    """Oracle compressed cache and ring of request r after appending its first L_before keys."""
    raw = wl.idx_keys(r, 0, L_before + 1) if raw is None else raw
    comp = np.zeros((max((L_before + 1) // 4, 1), 128), dtype=np.uint16)
    nb0 = L_before // 4
    comp[:nb0] = O.compress(raw[:4 * nb0])
    ring = np.zeros((4, 128), dtype=np.uint16)
    for p in range(4 * nb0, L_before):
        ring[p % 4] = raw[p]
    return comp, ring, raw


def oracle_decode_request(wl, r: int):
    """Oracle decode step of request r of a decode workload (state = first L-1 keys appended)."""
    L = int(wl.lens[r])
    comp, ring, raw = oracle_state(wl, r, L - 1)
    O.append(ring, comp, raw[L - 1], L - 1, wl.rope_theta)
    blocks, pos, scores = O.select_query(wl.idx_q(r)[0], wl.w(r)[0], comp, L, wl.rope_theta)
    K, V = wl.k(r, 0, L), wl.v(r, 0, L)
    out, lse = O.sparse_gqa(wl.q(r)[0], K, V, pos)
    return dict(L=L, comp=comp, ring=ring, blocks=blocks, pos=pos, scores=scores, out=out, lse=lse, K=K, V=V)


def check_selection(gpu_blocks: np.ndarray, ora_blocks: np.ndarray, scores: np.ndarray, nb: int, what: str = ""):
    """Apply the kept-set parity rule.  Returns the selection the attention check must use."""
    gpu_blocks = np.asarray(gpu_blocks, dtype=np.int64)
    k = min(nb, 512)
    assert len(gpu_blocks) == k, f"{what}: kept {len(gpu_blocks)} blocks, expected {k}"
    if k:
        assert np.all(np.diff(gpu_blocks) > 0), f"{what}: kept blocks not strictly ascending"
        assert gpu_blocks[0] >= 0 and gpu_blocks[-1] < nb, f"{what}: kept block out of range"
    if np.array_equal(gpu_blocks, ora_blocks):
        return gpu_blocks
    assert nb > 512, f"{what}: with <= 512 blocks every block must be kept"
    srt = np.sort(scores)[::-1]
    s512, s513 = srt[511], srt[512]
    gap = abs(s512 - s513) / max(abs(s512), 1e-30)
    diff = len(set(gpu_blocks.tolist()) ^ set(ora_blocks.tolist())) // 2
    assert gap <= NEAR_TIE_REL, (f"{what}: kept sets differ in {diff} blocks but the 512th/513th oracle scores "
                                 f"{s512!r} / {s513!r} are not a near tie (rel gap {gap:.3g})")
    ssum_g = float(np.sum(scores[gpu_blocks]))
    ssum_o = float(np.sum(scores[ora_blocks]))
    assert abs(ssum_g - ssum_o) <= SCORE_SUM_REL * abs(ssum_o), \
        f"{what}: near-tie set score sum {ssum_g} vs oracle {ssum_o}"
    return gpu_blocks


def check_attention(gpu_out: np.ndarray, ora_out: np.ndarray, what: str = ""):
    d = np.abs(np.asarray(gpu_out, dtype=np.float64) - ora_out)
    assert np.all(np.isfinite(gpu_out)), f"{what}: non-finite outputs"
    mx, mean = float(d.max(initial=0.0)), float(d.mean()) if d.size else 0.0
    assert mx <= ATT_MAX_ABS and mean <= ATT_MEAN_ABS, f"{what}: max-abs {mx:.3g}, mean-abs {mean:.3g}"
    return mx, mean


def attention_on(wl_or_KV, q_bits, positions, K=None, V=None):
    return O.sparse_gqa(q_bits, K, V, np.asarray(positions, dtype=np.int32))
