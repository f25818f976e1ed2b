"""Helpers for GPU-vs-oracle parity tests (test infrastructure).

Acceptance rules (the bar for the CUDA path):
  * codes, magnitude indices, sign bits, weights, occupancy, q~, ||q||,
    bonus tables, collision scores S, the S histogram and threshold, and the
    candidate set: bit-exact;
  * 4-bit estimates: |gpu - oracle| <= 1e-5 * den, with
        den = max(|est|, ||q|| sum_b |w_b <v_b, q~_b>|)
    computed in fp64 from the oracle's stored values: the estimate's own
    block terms, so a block whose 8-term dot cancels earns no slack, and the
    sum of the block terms' magnitudes survives an estimate that cancels to
    ~0 across blocks;
  * final Top-k: an id may be in one set and not the other only where its
    oracle score is within 1e-5 * den(k-th key) of the oracle's k-th score;
    at most MAX_SWAPS such ids per (sequence, KV head); the GPU order is
    (score desc, id asc) and, rank by rank, the oracle scores of the two
    lists agree within 1e-5 * den of the oracle's key at that rank;
  * attention: max-abs difference <= 2e-3 (bf16 inputs; the output is fp32).

Every check records its margin (largest error / tolerance, disagreements) in
STATS; tests/conftest.py prints them per test at the end of the run.
"""
from __future__ import annotations

import os

import numpy as np
import torch

import oracle

EST_REL = 1e-5
ATTN_ABS = 2e-3
MAX_SWAPS = 1             # tolerated Top-k disagreements per (sequence, KV head)

# test node id -> {"pairs": n, "swaps": n, "est": max err/tol, "attn": max err/tol}
STATS: dict = {}


def _record(kind: str, value: float, count: int = 0):
    test = os.environ.get("PYTEST_CURRENT_TEST", "(outside pytest)").split(" ")[0]
    s = STATS.setdefault(test, {"pairs": 0, "swaps": 0, "est": 0.0, "attn": 0.0})
    if kind == "topk":
        s["pairs"] += 1
        s["swaps"] += count
        s["est"] = max(s["est"], value)
    else:
        s[kind] = max(s[kind], value)


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


def est_denominator(enc: dict, cand: np.ndarray, qt: np.ndarray, qnorm: float, est: np.ndarray):
    """max(|est_i|, ||q|| sum_b |w_{i,b} <v_{i,b}, q~_b>|) for the ids cand (fp64)."""
    v = enc["v"][cand].reshape(-1, 16, 8)                 # signed levels sigma l_t, fp64
    dots = (v * qt.astype(np.float64).reshape(1, 16, 8)).sum(-1)
    blocks = np.abs(enc["w"][cand].astype(np.float64) * dots).sum(-1)
    return np.maximum(np.abs(np.asarray(est, np.float64)), float(qnorm) * blocks)


def check_encoding(enc: dict, codes: np.ndarray, rec: np.ndarray, occ: np.ndarray):
    tidx, neg, w = decode_records(rec)
    assert np.array_equal(codes.astype(np.uint16), enc["codes"]), "codes differ"
    assert np.array_equal(tidx, enc["tidx"]), "magnitude indices differ"
    assert np.array_equal(neg, code_bits(enc["codes"])), "sign bits differ"
    assert np.array_equal(w.view(np.uint32), enc["w"].view(np.uint32)), "weights differ"
    assert np.array_equal(occ, enc["occ"]), "occupancy differs"


def check_topk(gpu_idx, gpu_score, orc: dict, enc: dict):
    """Final Top-k rule.  Returns (disagreements, largest estimate error / tolerance)."""
    cand, est = orc["cand"], orc["est"]
    pos = {int(i): r for r, i in enumerate(cand)}
    gpu_idx = np.asarray(gpu_idx)
    gpu_score = np.asarray(gpu_score)
    k = len(orc["idx"])
    assert len(gpu_idx) == k and len(set(gpu_idx.tolist())) == k, "duplicate / missing ids"
    assert all(int(i) in pos for i in gpu_idx), "an id is not a candidate"
    rows = np.array([pos[int(i)] for i in gpu_idx])
    orows = np.array([pos[int(i)] for i in orc["idx"]])
    den_g = est_denominator(enc, cand[rows], orc["qt"], orc["qnorm"], est[rows])
    den_o = est_denominator(enc, cand[orows], orc["qt"], orc["qnorm"], est[orows])
    kth = float(orc["score"][-1])
    tol_kth = EST_REL * float(den_o[-1])
    diff = set(gpu_idx.tolist()) ^ set(orc["idx"].tolist())
    for i in diff:
        assert abs(est[pos[i]] - kth) <= tol_kth, \
            "id %d: oracle score %.9g vs k-th %.9g (tol %.3g)" % (i, est[pos[i]], kth, tol_kth)
    swaps = len(diff) // 2
    assert swaps <= MAX_SWAPS, "%d Top-k disagreements" % swaps
    # the GPU list is ordered by its own score, best first, ties by lower id
    g = gpu_score.astype(np.float32)
    assert np.all(np.diff(g) <= 0), "GPU scores not descending"
    tie = np.diff(g) == 0
    assert np.all(np.diff(gpu_idx.astype(np.int64))[tie] > 0), "ties not ordered by id"
    # the score of every returned id agrees with the oracle's estimate
    err = np.abs(g.astype(np.float64) - est[rows])
    ratio = err / (EST_REL * den_g + 1e-300)
    assert np.all(err <= EST_REL * den_g + 1e-30), "returned score error %.3g x tol" % float(ratio.max())
    # rank by rank, the two orders agree up to the tolerance
    gap = np.abs(est[rows] - orc["score"].astype(np.float64))
    assert np.all(gap <= EST_REL * np.maximum(den_o, den_g) + 1e-30), "order differs beyond tolerance"
    r = float(ratio.max()) if len(ratio) else 0.0
    _record("topk", r, swaps)
    return swaps, r


def check_search_pair(dbg: dict, p: int, orc: dict, enc: dict, n: int):
    """Compare the debug outputs of pair p with the oracle's intermediates.
    Returns the largest estimate error / tolerance over all candidates."""
    assert np.array_equal(dbg["qt"][p].view(np.uint32), orc["qt"].view(np.uint32)), "q~ differs"
    assert dbg["qnorm"][p].view(np.uint32) == np.float32(orc["qnorm"]).view(np.uint32), "||q|| differs"
    assert np.array_equal(dbg["bonus"][p], orc["bonus"]), "bonus tables differ"
    check_stage1(dbg, p, orc, n)
    C = orc["C"]
    den = est_denominator(enc, orc["cand"], orc["qt"], orc["qnorm"], orc["est"])
    err = np.abs(dbg["cand_est"][p][:C].astype(np.float64) - orc["est"])
    ratio = err / (EST_REL * den + 1e-300)
    assert np.all(err <= EST_REL * den + 1e-30), "estimate error %.3g x tol" % float(ratio.max())
    r = float(ratio.max()) if C else 0.0
    _record("est", r)
    return r


def check_stage1(dbg: dict, p: int, orc: dict, n: int):
    """Collision scores, their histogram, the threshold s* and the candidate
    set of pair p: bit-exact."""
    assert np.array_equal(dbg["S"][p][:n], orc["S"]), "collision scores differ"
    hist = np.bincount(orc["S"], minlength=97)
    assert np.array_equal(dbg["hist"][p], hist), "score histogram differs"
    C = orc["C"]
    cum = np.cumsum(hist[::-1])[::-1]
    assert dbg["sstar"][p] == int(np.nonzero(cum >= C)[0].max()), "threshold differs"
    assert np.array_equal(dbg["cand"][p][:C], orc["cand"]), "candidate set differs"


def check_attention(out: np.ndarray, ref: np.ndarray, tol: float = ATTN_ABS):
    err = float(np.abs(out - ref).max())
    assert err <= tol, "attention max-abs %.3g" % err
    _record("attn", err / tol)
    return err


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
