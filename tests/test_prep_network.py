"""The ranking network of the query-preparation kernel, emulated on the host.

The kernel ranks the 256 sign-pattern centres of a block by (score desc, id
asc) without sorting all 256 keys: flipping all 8 signs of a centre negates its
fp32 score exactly, so one warp sorts the 128 centres with bit 7 clear (4 keys
per lane, element 4*lane + i), appends the mirror key of each sorted key (a
descending run) and finishes with an 8-stage bitonic merge.  This test runs
that exact lane/register layout in Python and checks it against a plain sort
of all 256 keys, with exact ties (zero coordinates, coarse values) included.
It checks the design, not the CUDA code; the GPU parity tests check the
kernel's bonus tables against the oracle bit for bit.
"""
import struct

import numpy as np


def _ord(x):
    u = struct.unpack("<I", struct.pack("<f", np.float32(x)))[0]
    return (u ^ 0xFFFFFFFF) if (u >> 31) else (u | 0x80000000)


def _unord(k):
    u = (k & 0x7FFFFFFF) if (k >> 31) else (k ^ 0xFFFFFFFF)
    return np.float32(struct.unpack("<f", struct.pack("<I", u))[0])


def _key(L, c):
    L = np.float32(L + np.float32(0.0))          # +0 folds -0
    return ((~_ord(L) & 0xFFFFFFFF) << 8) | c


def _mirror(k):
    return _key(np.float32(-_unord((~(k >> 8)) & 0xFFFFFFFF)), (k & 0xFF) ^ 0xFF)


def _score(x, c):
    L = np.float32(0.0)
    for j in range(8):
        L = np.float32(L + (-x[j] if (c >> j) & 1 else x[j]))
    return L


def _network(x):
    v = [[_key(_score(x, 4 * lane + i), 4 * lane + i) for i in range(4)] + [0] * 4 for lane in range(32)]
    k = 2
    while k <= 128:                               # bitonic sort of the 128 keys
        j = k >> 1
        while j > 0:
            if j < 4:                             # inside a lane
                for lane in range(32):
                    for i in range(4):
                        if i & j == 0:
                            a, b = v[lane][i], v[lane][i | j]
                            lo, hi = min(a, b), max(a, b)
                            up = ((4 * lane + i) & k) == 0
                            v[lane][i], v[lane][i | j] = (lo, hi) if up else (hi, lo)
            else:                                 # across lanes: lane ^ j / 4
                nv = [row[:] for row in v]
                for lane in range(32):
                    for i in range(4):
                        o, e = v[lane ^ (j >> 2)][i], 4 * lane + i
                        take_min = ((e & j) == 0) == ((e & k) == 0)
                        nv[lane][i] = min(o, v[lane][i]) if take_min else max(o, v[lane][i])
                v = nv
            j >>= 1
        k <<= 1
    for lane in range(32):                        # positions 128 + 4 lane + i: mirrors
        for i in range(4):
            v[lane][4 + i] = _mirror(v[lane][i])
    for lane in range(32):                        # merge: stride 128 inside a lane
        for i in range(4):
            v[lane][i], v[lane][4 + i] = min(v[lane][i], v[lane][4 + i]), max(v[lane][i], v[lane][4 + i])
    j = 64
    while j >= 4:                                 # strides 64 .. 4 across lanes
        nv = [row[:] for row in v]
        for lane in range(32):
            lower = ((4 * lane) & j) == 0
            for i in range(8):
                o = v[lane ^ (j >> 2)][i]
                nv[lane][i] = min(o, v[lane][i]) if lower else max(o, v[lane][i])
        v = nv
        j >>= 1
    for lane in range(32):                        # strides 2, 1 inside a lane
        for h in (0, 4):
            for p, q in ((0, 2), (1, 3), (0, 1), (2, 3)):
                a, b = v[lane][h + p], v[lane][h + q]
                v[lane][h + p], v[lane][h + q] = min(a, b), max(a, b)
    return [v[lane][i] for lane in range(32) for i in range(4)] + \
           [v[lane][4 + i] for lane in range(32) for i in range(4)]


def test_mirror_score_is_exact_negation():
    rng = np.random.default_rng(5)
    for _ in range(200):
        x = rng.standard_normal(8).astype(np.float32) * np.float32(rng.uniform(1e-3, 1e3))
        for c in range(128):
            assert _score(x, c ^ 0xFF) == -_score(x, c)


def test_sort_mirror_merge_equals_full_sort():
    rng = np.random.default_rng(1)
    for trial in range(60):
        x = rng.standard_normal(8).astype(np.float32)
        if trial % 3 == 0:
            x[rng.integers(8)] = 0.0              # pairs of centres with equal scores
        if trial % 5 == 0:
            x = (np.round(x * 2) / 2).astype(np.float32)   # many equal scores
        ref = sorted(_key(_score(x, c), c) for c in range(256))
        assert _network(x) == ref, trial
