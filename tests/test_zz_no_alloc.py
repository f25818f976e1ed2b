"""The allocation-free candidate selection (pk_select_candidates_noalloc).

It serves callers that cannot allocate device memory when they need a
candidate set (work recorded into a CUDA graph, fully pre-reserved memory
pools, decode threads that must not touch the allocator).  Its result must be
the candidate set pk_search computes, bit for bit, on every call -- including
two calls in a row that share its static scratch array.  This file is
collected last so that a stop-at-first-failure run has run everything else.
"""
import numpy as np
import pytest
import torch

import workloads
from tests import parity

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def pk():
    from kv_cache_top_b200 import build
    build.build()
    import kv_cache_top_b200 as pk
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return pk


def test_noalloc_selection_matches_search_two_calls_in_a_row(pk):
    batch, H, G, n, topk = 1, 3, 2, 40007, 100
    w = workloads.llama_layer(batch, n, H=H, G=G, seed=21, device="cuda")
    p = pk.pk_default_params(batch=batch, n_kv_heads=H, group=G, topk=topk, kv_dtype=1)
    h = pk.pk_build_index(w["K"], w["V"], n, p)
    try:
        C, _ = pk.pk_resolve(n, 0, 0.0, topk)
        BH = batch * H
        idx = torch.empty(BH, topk, dtype=torch.int32, device="cuda")
        dbg = parity.alloc_debug(BH, n, C)
        pk.pk_search_debug(h, w["q"][0], topk, idx, None, dbg)
        torch.cuda.synchronize()
        want = dbg["cand"].cpu().numpy()
        S = dbg["S"]
        # two calls in a row on the same stream, sharing the scratch array
        outs = []
        for pair in (2, 0):
            cand = torch.full((C,), -1, dtype=torch.int32, device="cuda")
            pk.pk_select_candidates_noalloc(S[pair], n, C, cand)
            outs.append((pair, cand))
        torch.cuda.synchronize()
        for pair, cand in outs:
            assert np.array_equal(cand.cpu().numpy(), want[pair]), pair
        # a smaller budget on the same row: the lowest-index rule at the threshold
        C2 = 777
        cand = torch.full((C2,), -1, dtype=torch.int32, device="cuda")
        pk.pk_select_candidates_noalloc(S[1], n, C2, cand)
        s1 = S[1].cpu().numpy().astype(np.int64)
        ref = np.sort(np.lexsort((np.arange(n), -s1))[:C2])
        assert np.array_equal(cand.cpu().numpy(), ref)
    finally:
        pk.pk_free(h)


def test_noalloc_rejects_sizes_beyond_its_scratch(pk):
    S = torch.zeros(16, dtype=torch.uint8, device="cuda")
    cand = torch.zeros(16, dtype=torch.int32, device="cuda")
    with pytest.raises(pk.PkError) as e:
        pk.pk_select_candidates_noalloc(S, 4194305, 10, cand)
    assert e.value.status == 2
    with pytest.raises(pk.PkError) as e:
        pk.pk_select_candidates_noalloc(S, 16, 17, cand)
    assert e.value.status == 1


@pytest.mark.parametrize("n,C,hi", [
    (4194304, 300000, 256),   # the largest row (256 chunks), byte scores over the whole 0..255 range
    (1000003, 1000003, 256),  # C == n: every key
    (1000003, 123457, 4),     # four distinct scores: the threshold's ties span many chunks
    (65537, 1, 97),           # one candidate, ragged last chunk
])
def test_noalloc_synthetic_rows(pk, n, C, hi):
    """Synthetic score rows (not produced by a scan): the candidate set is the
    Top-C by (score desc, id asc) in ascending id order, on two calls in a row."""
    g = torch.Generator(device="cuda").manual_seed(n + C)
    S = torch.randint(0, hi, (n,), generator=g, device="cuda", dtype=torch.int32).to(torch.uint8)
    s = S.cpu().numpy().astype(np.int64)
    ref = np.sort(np.lexsort((np.arange(n), -s))[:C]).astype(np.int32)
    for _ in range(2):
        cand = torch.full((C,), -1, dtype=torch.int32, device="cuda")
        pk.pk_select_candidates_noalloc(S, n, C, cand)
        torch.cuda.synchronize()
        assert np.array_equal(cand.cpu().numpy(), ref)
