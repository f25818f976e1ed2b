"""CPU oracle for ParisKV retrieval -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The CUDA library never calls it, and it
never calls the CUDA library.

This module is a ctypes wrapper (argument marshalling with numpy) around the
plain-C oracle in ``pariskv_oracle.c``; the arithmetic lives there, each step
citing the page and equation it restates.  The helpers at the bottom only
compose those C steps in the order the method runs them.
"""
from __future__ import annotations

import ctypes as C
import functools

import numpy as np

from . import build as _build

_lib = C.CDLL(_build.build())

_p = C.c_void_p
_i64 = C.c_int64
_i32 = C.c_int
_f32 = C.c_float
_f64 = C.c_double
_u64 = C.c_uint64

_lib.or_splitmix64.restype = _u64
_lib.or_splitmix64.argtypes = [_u64]
_lib.or_srht_signs.argtypes = [_u64, _i32, _p]
_lib.or_magnitude_density.restype = _f64
_lib.or_magnitude_density.argtypes = [_i32, _f64]
_lib.or_lloyd_max.restype = _i32
_lib.or_lloyd_max.argtypes = [_i32, _i32, _p, _p]
_lib.or_levels_f32.restype = _i32
_lib.or_levels_f32.argtypes = [_i32, _i32, _p, _p]
_lib.or_rotate.restype = _f32
_lib.or_rotate.argtypes = [_p, _i32, _p, _p]
_lib.or_encode_keys.argtypes = [_p, _i64, _i32, _i32, _p, _p, _p, _i32, _i32,
                                _p, _p, _p, _p, _p, _p, _p]
_lib.or_bonus_from_qt.argtypes = [_p, _i32, _i32, _p, _i64, _p, _p]
_lib.or_query_prep.argtypes = [_p, _i32, _i32, _i32, _p, _p, _i64, _p, _p, _p, _p]
_lib.or_collision.argtypes = [_p, _i64, _i32, _i32, _p, _p]
_lib.or_candidates.restype = _i64
_lib.or_candidates.argtypes = [_p, _i64, _i64, _p]
_lib.or_dequantize.argtypes = [_p, _p, _p, _i64, _i32, _i32, _p]
_lib.or_rerank.argtypes = [_p, _i64, _p, _p, _i32, _i32, _p, _f32, _p]
_lib.or_topk.argtypes = [_p, _p, _i64, _i32, _p, _p]
_lib.or_attend.argtypes = [_p, _i32, _i32, _p, _p, _p, _i32, _f64, _p]
_lib.or_ratio_table.argtypes = [_i64, _p, _p]
_lib.or_resolve.argtypes = [_i64, _i64, _f32, _i32, _p, _p]


def _ptr(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return a.ctypes.data_as(_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


# ---------------------------------------------------------------- basics
def splitmix64(x: int) -> int:
    return int(_lib.or_splitmix64(x))


def srht_signs(seed: int, D: int) -> np.ndarray:
    s = np.empty(D, np.int8)
    _lib.or_srht_signs(seed, D, _ptr(s))
    return s


def magnitude_density(m: int, y: float) -> float:
    return float(_lib.or_magnitude_density(m, y))


@functools.lru_cache(maxsize=None)
def _lloyd_max_cached(m: int, L: int):
    lev = np.empty(L, np.float64)
    thr = np.empty(L - 1, np.float64)
    it = _lib.or_lloyd_max(m, L, _ptr(lev), _ptr(thr))
    lev.setflags(write=False)
    thr.setflags(write=False)
    return lev, thr, int(it)


def lloyd_max(m: int, L: int):
    """fp64 Lloyd-Max levels and midpoints of the magnitude prior."""
    return _lloyd_max_cached(m, L)


@functools.lru_cache(maxsize=None)
def _levels_f32_cached(m: int, L: int):
    lev = np.empty(L, np.float32)
    thr = np.empty(L - 1, np.float32)
    it = _lib.or_levels_f32(m, L, _ptr(lev), _ptr(thr))
    if it < 0:
        raise RuntimeError("oracle Lloyd-Max iteration did not converge")
    lev.setflags(write=False)
    thr.setflags(write=False)
    return lev, thr


def levels_f32(m: int = 8, L: int = 8):
    return _levels_f32_cached(m, L)


def rotate(x: np.ndarray, signs: np.ndarray):
    x = _c(x, np.float32)
    out = np.empty_like(x)
    nrm = _lib.or_rotate(_ptr(x), x.shape[-1], _ptr(_c(signs, np.int8)), _ptr(out))
    return out, np.float32(nrm)


# -------------------------------------------------------------- encoding
def encode_keys(K: np.ndarray, signs: np.ndarray, m: int = 8, L: int = 8,
                quantize: bool = True, debug: bool = False, levels=None):
    """Encode keys K[n][D] (fp32).  Returns a dict with codes [n][B] u16,
    tidx [n][D] u16, w [n][B] f32, occ [B][2^m] u32 (+ knorm, rb, u)."""
    K = _c(K, np.float32)
    n, D = K.shape
    B = D // m
    if levels is None:
        lev, thr = levels_f32(m, L)
    else:
        lev, thr = levels
    lev = _c(lev, np.float32)
    thr = _c(thr, np.float32)
    codes = np.zeros((n, B), np.uint16)
    tidx = np.zeros((n, D), np.uint16)
    w = np.zeros((n, B), np.float32)
    occ = np.zeros((B, 1 << m), np.uint32)
    knorm = np.zeros(n, np.float32) if debug else None
    rb = np.zeros((n, B), np.float32) if debug else None
    u = np.zeros((n, D), np.float32) if debug else None
    nul = None
    _lib.or_encode_keys(_ptr(K), n, D, m, _ptr(_c(signs, np.int8)), _ptr(lev), _ptr(thr),
                        len(lev), 1 if quantize else 0, _ptr(codes), _ptr(tidx), _ptr(w),
                        _ptr(occ), _ptr(knorm) if debug else nul, _ptr(rb) if debug else nul,
                        _ptr(u) if debug else nul)
    out = dict(codes=codes, tidx=tidx, w=w, occ=occ, lev=lev, thr=thr, m=m, D=D)
    if debug:
        out.update(knorm=knorm, rb=rb, u=u)
    return out


# --------------------------------------------------------------- Stage I
def bonus_from_qt(qt: np.ndarray, occ: np.ndarray, R: int, m: int = 8):
    qt = _c(qt, np.float32)
    D = qt.shape[-1]
    B = D // m
    lut = np.empty((B, 1 << m), np.float32)
    bonus = np.empty((B, 1 << m), np.uint8)
    _lib.or_bonus_from_qt(_ptr(qt), D, m, _ptr(_c(occ, np.uint32)), R, _ptr(lut), _ptr(bonus))
    return lut, bonus


def query_prep(q: np.ndarray, signs: np.ndarray, occ: np.ndarray, R: int, m: int = 8):
    """q [G][D] fp32 -> (qt [D] f32, qnorm f32, lut [B][2^m] f32, bonus [B][2^m] u8)."""
    q = _c(np.atleast_2d(q), np.float32)
    G, D = q.shape
    B = D // m
    qt = np.empty(D, np.float32)
    qn = np.empty(1, np.float32)
    lut = np.empty((B, 1 << m), np.float32)
    bonus = np.empty((B, 1 << m), np.uint8)
    _lib.or_query_prep(_ptr(q), G, D, m, _ptr(_c(signs, np.int8)), _ptr(_c(occ, np.uint32)), R,
                       _ptr(qt), _ptr(qn), _ptr(lut), _ptr(bonus))
    return qt, qn[0], lut, bonus


def collision(codes: np.ndarray, bonus: np.ndarray, D: int = 128, m: int = 8):
    codes = _c(codes, np.uint16)
    n = codes.shape[0]
    S = np.empty(n, np.uint8)
    _lib.or_collision(_ptr(codes), n, D, m, _ptr(_c(bonus, np.uint8)), _ptr(S))
    return S


def candidates(S: np.ndarray, C: int):
    S = _c(S, np.uint8)
    n = S.shape[0]
    C = min(int(C), n)
    cand = np.empty(max(C, 1), np.int32)
    got = _lib.or_candidates(_ptr(S), n, C, _ptr(cand))
    return cand[:got]


# -------------------------------------------------------------- Stage II
def dequantize(codes, tidx, lev, D: int = 128, m: int = 8):
    codes = _c(codes, np.uint16)
    tidx = _c(tidx, np.uint16)
    n = codes.shape[0]
    v = np.empty((n, D), np.float64)
    _lib.or_dequantize(_ptr(codes), _ptr(tidx), _ptr(_c(lev, np.float32)), n, D, m, _ptr(v))
    return v


def rerank(cand, v, w, qt, qnorm, m: int = 8):
    cand = _c(cand, np.int32)
    v = _c(v, np.float64)
    w = _c(w, np.float32)
    D = v.shape[1]
    est = np.empty(len(cand), np.float64)
    _lib.or_rerank(_ptr(cand), len(cand), _ptr(v), _ptr(w), D, m, _ptr(_c(qt, np.float32)),
                   float(qnorm), _ptr(est))
    return est


def topk(cand, est, k: int):
    cand = _c(cand, np.int32)
    est = _c(est, np.float64)
    k = min(int(k), len(cand))
    idx = np.empty(k, np.int32)
    score = np.empty(k, np.float64)
    _lib.or_topk(_ptr(cand), _ptr(est), len(cand), k, _ptr(idx), _ptr(score))
    return idx, score


def attend(q, K, V, idx, scale: float):
    """q [G][D], K/V [n][D] fp32 (bf16 values decoded exactly), idx [k]."""
    q = _c(np.atleast_2d(q), np.float32)
    K = _c(K, np.float32)
    V = _c(V, np.float32)
    idx = _c(idx, np.int32)
    G, D = q.shape
    o = np.empty((G, D), np.float64)
    _lib.or_attend(_ptr(q), G, D, _ptr(K), _ptr(V), _ptr(idx), len(idx), float(scale), _ptr(o))
    return o


def attend_union(q, K, V, idx, Kd, Vd, scale: float):
    """Attention of q [G][D] over the selected rows idx of (K, V) together
    with every row of the dense set (Kd, Vd) [m][D] -- the sink and local
    tokens kept on the GPU -- under one softmax (README, step 3: attention
    over sink, local and retrieved tokens; slides, Fig. 5).  The union of
    the two row sets is attended by `attend` above."""
    K = _c(K, np.float32)
    Kd = _c(np.reshape(Kd, (-1, K.shape[1])), np.float32)
    Vd = _c(np.reshape(Vd, (-1, K.shape[1])), np.float32)
    Ku = np.concatenate([K, Kd])
    Vu = np.concatenate([_c(V, np.float32), Vd])
    idx_u = np.concatenate([np.asarray(idx, np.int64), K.shape[0] + np.arange(Kd.shape[0])])
    return attend(q, Ku, Vu, idx_u, scale)


def ratio_table(n: int):
    b = np.empty(1, np.float64)
    r = np.empty(1, np.float64)
    _lib.or_ratio_table(n, _ptr(b), _ptr(r))
    return float(b[0]), float(r[0])


def resolve(n: int, cand_budget: int = 0, collision_ratio: float = 0.0, topk: int = 100):
    c = np.empty(1, np.int64)
    r = np.empty(1, np.int64)
    _lib.or_resolve(n, cand_budget, collision_ratio, topk, _ptr(c), _ptr(r))
    return int(c[0]), int(r[0])


# ------------------------------------------------- the steps, in order
def build_index(K: np.ndarray, rot_seed: int = 0, m: int = 8, L: int = 8):
    """Encode one (sequence, KV head): K [n][D] fp32."""
    D = K.shape[1]
    signs = srht_signs(rot_seed, D)
    enc = encode_keys(K, signs, m=m, L=L)
    enc["signs"] = signs
    enc["v"] = dequantize(enc["codes"], enc["tidx"], enc["lev"], D=D, m=m)
    return enc


def search(enc: dict, q: np.ndarray, topk_k: int = 100, cand_budget: int = 0,
           collision_ratio: float = 0.0):
    """One retrieval for one (sequence, KV head); q [G][D] fp32 (G query heads
    of the group).  Returns every intermediate of the path."""
    m, D = enc["m"], enc["D"]
    n = enc["codes"].shape[0]
    C, R = resolve(n, cand_budget, collision_ratio, topk_k)
    qt, qn, lut, bonus = query_prep(q, enc["signs"], enc["occ"], R, m=m)
    S = collision(enc["codes"], bonus, D=D, m=m)
    cand = candidates(S, C)
    est = rerank(cand, enc["v"], enc["w"], qt, qn, m=m)
    idx, score = topk(cand, est, topk_k)
    return dict(C=C, R=R, qt=qt, qnorm=qn, lut=lut, bonus=bonus, S=S, cand=cand,
                est=est, idx=idx, score=score)
