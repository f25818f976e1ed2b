"""Helpers for GPU-vs-oracle parity tests (test infrastructure).

Acceptance rules (the bar for the CUDA path):
  * codes, magnitude indices, sign bits, weights, occupancy, q~, ||q||,
    bonus tables, collision scores S, the S histogram and threshold, and the
    candidate set: bit-exact;
  * 4-bit estimates: |gpu - oracle| <= 1e-5 * scale, where scale is the sum of
    the absolute values of all terms of the estimate, ||q|| sum_b |w_b|
    sum_j l_{t_j} |q~_j| (fp32 accumulation error is bounded by a multiple of
    it, and it does not vanish when the estimate cancels to ~0);
  * final Top-k: an index may differ from the oracle's only where the
    oracle's scores of the two sides differ by less than 1e-5 * scale;
  * attention: max-abs difference <= 2e-3 (bf16 inputs; the output is fp32).
"""
from __future__ import annotations

import numpy as np
import torch

import oracle

EST_REL = 1e-5
ATTN_ABS = 2e-3


def decode_records(rec: np.ndarray):
    """[n][128] u8 summary records -> (tidx [n][128] u16, neg [n][128] bool, w [n][16] f32).
    Record layout: 4 groups x (16 B of nibbles, 16 B of fp32 weights); the
    nibble of coordinate c is in byte c//2 of the concatenated nibble parts
    (low nibble for even c): bit 3 = negative sign, bits 0-2 = level index."""
    n = rec.shape[0]
    g = rec.reshape(n, 4, 32)
    nb = np.ascontiguousarray(g[:, :, :16]).reshape(n, 64)
    w = np.ascontiguousarray(g[:, :, 16:]).view(np.float32).reshape(n, 16)
    nib = np.empty((n, 128), np.uint8)
    nib[:, 0::2] = nb & 0xF
    nib[:, 1::2] = nb >> 4
    return (nib & 7).astype(np.uint16), (nib >> 3).astype(bool), w


def code_bits(codes: np.ndarray):
    """[n][16] codes -> [n][128] bool (bit j of block b = coordinate 8b + j negative)."""
    c = codes.astype(np.uint16)
    bits = (c[:, :, None] >> np.arange(8, dtype=np.uint16)[None, None, :]) & 1
    return bits.reshape(c.shape[0], 128).astype(bool)


def est_scale(enc: dict, cand: np.ndarray, qt: np.ndarray, qnorm: float):
    lev = enc["lev"].astype(np.float64)
    t = enc["tidx"][cand].astype(np.int64).reshape(-1, 16, 8)
    aq = np.abs(qt.astype(np.float64)).reshape(16, 8)
    per_block = (lev[t] * aq[None]).sum(-1)
    return float(qnorm) * (np.abs(enc["w"][cand].astype(np.float64)) * per_block).sum(-1)


def check_encoding(enc: dict, codes: np.ndarray, rec: np.ndarray, occ: np.ndarray):
    tidx, neg, w = decode_records(rec)
    assert np.array_equal(codes.astype(np.uint16), enc["codes"]), "codes differ"
    assert np.array_equal(tidx, enc["tidx"]), "magnitude indices differ"
    assert np.array_equal(neg, code_bits(enc["codes"])), "sign bits differ"
    assert np.array_equal(w.view(np.uint32), enc["w"].view(np.uint32)), "weights differ"
    assert np.array_equal(occ, enc["occ"]), "occupancy differs"


def check_topk(gpu_idx, gpu_score, orc: dict, enc: dict):
    """Final Top-k rule; returns the number of tolerated disagreements."""
    cand, est = orc["cand"], orc["est"]
    pos = {int(i): r for r, i in enumerate(cand)}
    scale = est_scale(enc, cand, orc["qt"], orc["qnorm"])
    k = len(orc["idx"])
    assert len(gpu_idx) == k and len(set(gpu_idx.tolist())) == k, "duplicate / missing ids"
    kth = orc["score"][-1]
    tol = EST_REL * float(scale.max())
    diff = set(gpu_idx.tolist()) ^ set(orc["idx"].tolist())
    for i in diff:
        assert i in pos, "id %d is not a candidate" % i
        assert abs(est[pos[i]] - kth) <= tol, "id %d: oracle score %.9g vs k-th %.9g" % (i, est[pos[i]], kth)
    # the GPU list is sorted by its own score, best first
    assert np.all(np.diff(gpu_score) <= 0)
    # scores of the ids agree with the oracle's estimate within tolerance
    for r, i in enumerate(gpu_idx.tolist()):
        assert abs(float(gpu_score[r]) - est[pos[i]]) <= EST_REL * scale[pos[i]] + 1e-30
    return len(diff) // 2


def check_search_pair(dbg: dict, p: int, orc: dict, enc: dict, n: int):
    """Compare the debug outputs of pair p with the oracle's intermediates."""
    assert np.array_equal(dbg["qt"][p].view(np.uint32), orc["qt"].view(np.uint32)), "q~ differs"
    assert dbg["qnorm"][p].view(np.uint32) == np.float32(orc["qnorm"]).view(np.uint32), "||q|| differs"
    assert np.array_equal(dbg["bonus"][p], orc["bonus"]), "bonus tables differ"
    assert np.array_equal(dbg["S"][p][:n], orc["S"]), "collision scores differ"
    hist = np.bincount(orc["S"], minlength=97)
    assert np.array_equal(dbg["hist"][p], hist), "score histogram differs"
    C = orc["C"]
    cum = np.cumsum(hist[::-1])[::-1]
    assert dbg["sstar"][p] == int(np.nonzero(cum >= C)[0].max()), "threshold differs"
    assert np.array_equal(dbg["cand"][p][:C], orc["cand"]), "candidate set differs"
    scale = est_scale(enc, orc["cand"], orc["qt"], orc["qnorm"])
    err = np.abs(dbg["cand_est"][p][:C].astype(np.float64) - orc["est"])
    assert np.all(err <= EST_REL * scale + 1e-30), "estimate error %.3g > tol" % float((err / scale).max())


def alloc_debug(BH: int, n: int, C: int, device="cuda"):
    return dict(
        qt=torch.empty(BH, 128, dtype=torch.float32, device=device),
        qnorm=torch.empty(BH, dtype=torch.float32, device=device),
        bonus=torch.empty(BH, 16, 256, dtype=torch.uint8, device=device),
        S=torch.empty(BH, n, dtype=torch.uint8, device=device),
        hist=torch.empty(BH, 97, dtype=torch.int32, device=device),
        sstar=torch.empty(BH, dtype=torch.int32, device=device),
        cand=torch.empty(BH, C, dtype=torch.int32, device=device),
        cand_est=torch.empty(BH, C, dtype=torch.float32, device=device),
    )


def to_np(d: dict):
    return {k: v.cpu().numpy() for k, v in d.items()}


def oracle_pair(K_np: np.ndarray, q_np: np.ndarray, topk: int, cand_budget: int, rot_seed: int = 0,
                collision_ratio: float = 0.0):
    enc = oracle.build_index(K_np, rot_seed=rot_seed)
    orc = oracle.search(enc, q_np, topk_k=topk, cand_budget=cand_budget, collision_ratio=collision_ratio)
    return enc, orc
