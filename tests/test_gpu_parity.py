"""GPU parity: the CUDA path through the C-ABI against the CPU oracle.

Every case compares the library's outputs with the oracle element by element
on the same seeded inputs (see tests/parity.py for the acceptance rules).
Sizes span several chunks and compaction windows with ragged tails; the full
8 x 128K and 1M workloads run in the launch configuration the benchmark
times and are checked on every (sequence, KV head) pair.
"""
import math
import os
from concurrent.futures import ThreadPoolExecutor

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


def _dt(dtype):
    return 1 if dtype == torch.bfloat16 else 0


def build(pk, K, V, n, batch, H, G, topk=100, cand_budget=0, collision_ratio=0.0, n_cap=0,
          kv_location=0, rot_seed=0):
    p = pk.pk_default_params(batch=batch, n_kv_heads=H, group=G, topk=topk, n_cap=n_cap,
                             cand_budget=cand_budget, collision_ratio=collision_ratio,
                             kv_dtype=_dt(K.dtype), kv_location=kv_location, rot_seed=rot_seed)
    return pk.pk_build_index(K, V, n, p)


def search_debug(pk, h, q, BH, n, C, topk):
    idx = torch.empty(BH, topk, dtype=torch.int32, device="cuda")
    score = torch.empty(BH, topk, dtype=torch.float32, device="cuda")
    dbg = parity.alloc_debug(BH, n, C)
    pk.pk_search_debug(h, q, topk, idx, score, dbg)
    torch.cuda.synchronize()
    return idx.cpu().numpy(), score.cpu().numpy(), parity.to_np(dbg)


def export(pk, h, BH, n):
    codes = torch.empty(BH, n, 16, dtype=torch.uint8, device="cuda")
    rec = torch.empty(BH, n, 128, dtype=torch.uint8, device="cuda")
    occ = torch.empty(BH, 16, 256, dtype=torch.int32, device="cuda")
    pk.pk_export_index(h, codes, rec, occ)
    torch.cuda.synchronize()
    return codes.cpu().numpy(), rec.cpu().numpy(), occ.cpu().numpy().view(np.uint32)


def oracle_pairs(K, V, q, pairs, H, G, n, topk, cand_budget=0, collision_ratio=0.0, workers=16):
    """Yield (p, K_np, V_np, qg, enc, orc) for every pair p: the oracle's
    build and search of that (sequence, KV head), run a few pairs at a time
    in a thread pool (the oracle's C calls release the GIL)."""
    W = max(1, min(len(pairs), os.cpu_count() or 1, workers))
    with ThreadPoolExecutor(W) as ex:
        for i0 in range(0, len(pairs), W):
            jobs = []
            for p in pairs[i0:i0 + W]:
                b, hh = divmod(p, H)
                K_np = workloads.to_np_f32(K[b, hh, :n])
                V_np = workloads.to_np_f32(V[b, hh, :n])
                qg = workloads.to_np_f32(q[b, hh * G:(hh + 1) * G])
                jobs.append((p, K_np, V_np, qg,
                             ex.submit(parity.oracle_pair, K_np, qg, topk, cand_budget, 0, collision_ratio)))
            for p, K_np, V_np, qg, fut in jobs:
                enc, orc = fut.result()
                yield p, K_np, V_np, qg, enc, orc


def check_pairs(pk, h, K, V, q, pairs, batch, H, G, n, topk, cand_budget=0, collision_ratio=0.0,
                attn_tol=parity.ATTN_ABS, check_encode=True, encode_pairs=None, workers=16):
    """Search + attend every pair through the C-ABI, then check the listed
    pairs against the oracle: bit-exact encoding (of encode_pairs, default
    all listed pairs, when check_encode), bit-exact q~, bonus tables, S,
    histogram, threshold and candidates, every candidate's estimate, the
    Top-k rule and the attention output."""
    BH = batch * H
    C, R = pk.pk_resolve(n, cand_budget, collision_ratio, topk)
    idx, score, dbg = search_debug(pk, h, q, BH, n, C, topk)
    out = torch.empty(batch, H * G, 128, dtype=torch.float32, device="cuda")
    pk.pk_attend(h, q, torch.from_numpy(idx).cuda(), topk, out)
    st, det = pk.pk_last_device_error(h)
    assert st == 0, (st, det)
    out = out.cpu().numpy()
    codes = rec = occ = None
    if check_encode:
        codes, rec, occ = export(pk, h, BH, n)
    enc_set = set(pairs if encode_pairs is None else encode_pairs)
    assert (idx >= 0).all() and (idx < n).all()
    for p, K_np, V_np, qg, enc, orc in oracle_pairs(K, V, q, pairs, H, G, n, topk, cand_budget,
                                                     collision_ratio, workers):
        b, hh = divmod(p, H)
        assert orc["C"] == C and orc["R"] == R
        if check_encode and p in enc_set:
            parity.check_encoding(enc, codes[p], rec[p], occ[p])
        parity.check_search_pair(dbg, p, orc, enc, n)
        parity.check_topk(idx[p], score[p], orc, enc)
        o_ref = parity.oracle.attend(qg, K_np, V_np, idx[p], 1.0 / math.sqrt(128))
        parity.check_attention(out[b, hh * G:(hh + 1) * G], o_ref, attn_tol)
    return idx


# ------------------------------------------------------------- configs
def test_tiny_single_head_config(pk):
    """1 KV head, n = 4096 fp32 keys with 4 outlier channels x8, 16 queries
    q = K[j] + N(0, 0.5^2), subspace dim 8, C = 512, Top-100."""
    w = workloads.tiny(seed=0, device="cuda")
    h = build(pk, w["K"], w["V"], 4096, 1, 1, 1, cand_budget=512)
    try:
        for qi in range(16):
            check_pairs(pk, h, w["K"], w["V"], w["q"][qi], [0], 1, 1, 1, 4096, 100,
                        cand_budget=512, attn_tol=1e-4, check_encode=(qi == 0))
    finally:
        pk.pk_free(h)


def test_llama_shaped_layer_config(pk):
    """batch 1, 32 query heads, 8 KV heads (G = 4), n = 32768 bf16 keys with
    LogNormal channel scales and RoPE; C = 2048; every pair checked."""
    w = workloads.llama_layer(1, 32768, H=8, G=4, seed=0, device="cuda", n_queries=2)
    h = build(pk, w["K"], w["V"], 32768, 1, 8, 4, cand_budget=2048)
    try:
        for qi in range(2):
            check_pairs(pk, h, w["K"], w["V"], w["q"][qi], list(range(8)), 1, 8, 4, 32768, 100,
                        cand_budget=2048, check_encode=(qi == 0))
    finally:
        pk.pk_free(h)


@pytest.mark.parametrize("n,cand,topk,batch,H,G", [
    (5000, 0, 100, 2, 2, 2),      # ratio table, ragged chunk tail, batch > 1
    (100, 0, 100, 1, 1, 1),       # n == topk: every key is a candidate and returned
    (1500, 1500, 37, 1, 2, 1),    # full budget C = n
    (16, 0, 16, 1, 1, 1),         # smallest index
    (3001, 0, 1, 1, 1, 3),        # topk = 1
    (70001, 0, 100, 1, 1, 4),     # many compaction windows, odd n
    (9000, 200, 200, 3, 1, 8),    # C == topk, G = 8
    (40000, 0, 256, 1, 2, 1),     # topk > 128 over several slices: shared-memory merge tree
    (60000, 0, 1024, 1, 2, 2),    # the largest topk: 1024-key selects and merges
    (70001, 70001, 100, 1, 2, 1), # every key a candidate (C = n)
    (400000, 0, 200, 1, 1, 1),    # 100 slices x 200 keys > the merge's 16384: rounds of radix select
])
def test_edge_and_ragged_sizes(pk, n, cand, topk, batch, H, G):
    w = workloads.llama_layer(batch, n, H=H, G=G, seed=n, device="cuda")
    h = build(pk, w["K"], w["V"], n, batch, H, G, topk=topk, cand_budget=cand)
    try:
        check_pairs(pk, h, w["K"], w["V"], w["q"][0], list(range(batch * H)), batch, H, G, n, topk,
                    cand_budget=cand)
    finally:
        pk.pk_free(h)


@pytest.mark.parametrize("beta,rho", [(0.02, 0.35), (0.2, 0.05)])
def test_explicit_budgets(pk, beta, rho):
    """Budgets away from the ratio table (the sweep's grid points): C =
    ceil(beta n) and R = ceil(rho n) reach the tiers, the threshold and the
    rerank unchanged."""
    n = 30000
    w = workloads.llama_layer(1, n, H=2, G=4, seed=int(1000 * beta + 100 * rho), device="cuda")
    C = math.ceil(beta * n)
    h = build(pk, w["K"], w["V"], n, 1, 2, 4, cand_budget=C, collision_ratio=rho)
    try:
        Cr, Rr = pk.pk_resolve(n, C, rho, 100)
        assert Cr == C and Rr == math.ceil(float(np.float32(rho)) * n)   # rho travels as fp32
        check_pairs(pk, h, w["K"], w["V"], w["q"][0], [0, 1], 1, 2, 4, n, 100, cand_budget=C,
                    collision_ratio=rho)
    finally:
        pk.pk_free(h)


def test_duplicate_keys_tie_rule(pk):
    """Many identical keys: equal scores everywhere, so the lower-id rule
    decides the candidate set and the Top-k, bit-exactly."""
    base = workloads.llama_layer(1, 64, H=1, G=1, seed=5, device="cuda")
    K = base["K"][:, :, :8].repeat(1, 1, 600, 1).contiguous()   # n = 4800, 8 distinct keys
    V = base["V"][:, :, :8].repeat(1, 1, 600, 1).contiguous()
    h = build(pk, K, V, 4800, 1, 1, 1, cand_budget=700)
    try:
        idx = check_pairs(pk, h, K, V, base["q"][0], [0], 1, 1, 1, 4800, 100, cand_budget=700)
        assert len(set(idx[0].tolist())) == 100
    finally:
        pk.pk_free(h)


@pytest.mark.parametrize("n,width", [(32768, 150), (262144, 150)])
def test_clustered_top_keys_merge(pk, n, width):
    """Keys n0..n0+width-1 are made close to the query, so the whole Top-k sits
    in one rerank slice: the per-slice lists are far from interleaved and the
    merge must leave its usual short-prefix case (the larger n also gives
    many slices and a weak prefix bound)."""
    w = workloads.llama_layer(1, n, H=1, G=1, seed=width + n, device="cuda")
    K = w["K"].clone()
    q = w["q"][0]
    n0 = n // 3
    K[0, 0, n0:n0 + width] = (3.0 * q[0, 0].float() + 0.2 * K[0, 0, n0:n0 + width].float()).to(K.dtype)
    h = build(pk, K, w["V"], n, 1, 1, 1)
    try:
        idx = check_pairs(pk, h, K, w["V"], q, [0], 1, 1, 1, n, 100)
        assert ((idx[0] >= n0) & (idx[0] < n0 + width)).sum() >= 90
    finally:
        pk.pk_free(h)


def test_append_matches_oracle(pk):
    """pk_append encodes new decode keys with the fixed codebook: the index
    after appends equals an index built over all keys at once."""
    w = workloads.llama_layer(1, 4200, H=2, G=2, seed=9, device="cuda")
    K, V = w["K"], w["V"]
    h = build(pk, K[:, :, :3000].contiguous(), V[:, :, :3000].contiguous(), 3000, 1, 2, 2,
              n_cap=4200)
    try:
        for i in range(3000, 3005):
            pk.pk_append(h, K[:, :, i:i + 1].contiguous(), V[:, :, i:i + 1].contiguous(), 1)
        pk.pk_append(h, K[:, :, 3005:4200].contiguous(), V[:, :, 3005:4200].contiguous(), 1195)
        assert pk.pk_get_info(h).n == 4200
        with pytest.raises(pk.PkError) as e:
            pk.pk_append(h, K[:, :, :1].contiguous(), V[:, :, :1].contiguous(), 1)
        assert e.value.status == 2
        check_pairs(pk, h, K, V, w["q"][0], [0, 1], 1, 2, 2, 4200, 100)
    finally:
        pk.pk_free(h)


def test_drift_stream_append_then_search(pk):
    """Drift config: prefill 65536 keys per KV head (8 heads, G = 1) from
    N(mu_0, diag sigma^2), then decode steps that each append one key drawn
    from a distribution whose mean moves towards mu_1 and search with a query
    from the same step law.  The codebook stays fixed; after 256 and 512
    steps the whole path (occupancy, tiers, candidates, rerank, Top-k,
    attention) still matches the oracle built over all keys at once."""
    n0, T, H = 65536, 512, 8
    w = workloads.drift_stream(n0, T, H=H, seed=7, device="cuda")
    h = build(pk, w["K"], w["V"], n0, 1, H, 1, n_cap=n0 + T)
    try:
        idx = torch.empty(H, 100, dtype=torch.int32, device="cuda")
        for t in range(T):
            pk.pk_append(h, w["k_new"][t], w["v_new"][t], 1)
            pk.pk_search(h, w["q"][t], 100, idx)
            if t + 1 in (256, 512):
                n = n0 + t + 1
                K = torch.cat([w["K"], w["k_new"][:t + 1, 0, :, 0].permute(1, 0, 2).unsqueeze(0)], dim=2)
                V = torch.cat([w["V"], w["v_new"][:t + 1, 0, :, 0].permute(1, 0, 2).unsqueeze(0)], dim=2)
                assert pk.pk_get_info(h).n == n
                check_pairs(pk, h, K, V, w["q"][t], [0, 5], 1, H, 1, n, 100, check_encode=(t + 1 == T))
    finally:
        pk.pk_free(h)


@pytest.mark.parametrize("kind,topk,dlen,kv_location", [
    ("llama", 100, 80, 0),      # 16 sink + 64 local rows beside the Top-100
    ("llama", 0, 80, 0),        # dense rows only
    ("llama", 100, 80, 1),      # index K/V in pinned host memory, dense rows on the GPU
    ("tiny", 100, 33, 0),       # fp32 rows, ragged dense count
])
def test_attend_with_dense_rows(pk, kind, topk, dlen, kv_location):
    """pk_attend_dense: the selected rows and the caller's dense (sink +
    local) rows under one softmax, against the oracle's attention over the
    union of the two row sets; with no dense rows it is pk_attend."""
    if kind == "tiny":
        w = workloads.tiny(seed=1, device="cuda")
        batch, H, G, n = 1, 1, 1, 4096
        q = w["q"][5]
        cand = 512
    else:
        batch, H, G, n = 2, 2, 4, 20000
        w = workloads.llama_layer(batch, n, H=H, G=G, seed=41, device="cuda")
        q = w["q"][0]
        cand = 0
    h = build(pk, w["K"], w["V"], n, batch, H, G, cand_budget=cand, kv_location=kv_location)
    try:
        BH = batch * H
        g = torch.Generator(device="cuda").manual_seed(5)
        dstride = dlen + 16
        dK = torch.randn(batch, H, dstride, 128, generator=g, device="cuda").to(w["K"].dtype)
        dV = torch.randn(batch, H, dstride, 128, generator=g, device="cuda").to(w["K"].dtype)
        idx = torch.empty(BH, 100, dtype=torch.int32, device="cuda")
        pk.pk_search(h, q, 100, idx)
        out = torch.full((batch, H * G, 128), float("nan"), dtype=torch.float32, device="cuda")
        pk.pk_attend_dense(h, q, idx if topk else None, topk, dK, dV, dlen, out)
        out0 = torch.empty_like(out)
        out1 = torch.empty_like(out)
        pk.pk_attend_dense(h, q, idx, 100, dK, dV, 0, out0)
        pk.pk_attend(h, q, idx, 100, out1)
        torch.cuda.synchronize()
        st, det = pk.pk_last_device_error(h)
        assert st == 0, (st, det)
        assert torch.equal(out0, out1)
        o = out.cpu().numpy()
        ids = idx.cpu().numpy()
        tol = 1e-4 if kind == "tiny" else parity.ATTN_ABS
        for p in range(BH):
            b, hh = divmod(p, H)
            qg = workloads.to_np_f32(q[b, hh * G:(hh + 1) * G])
            ref = parity.oracle.attend_union(qg, workloads.to_np_f32(w["K"][b, hh, :n]),
                                             workloads.to_np_f32(w["V"][b, hh, :n]), ids[p][:topk],
                                             workloads.to_np_f32(dK[b, hh, :dlen]),
                                             workloads.to_np_f32(dV[b, hh, :dlen]), 1.0 / math.sqrt(128))
            parity.check_attention(o[b, hh * G:(hh + 1) * G], ref, tol)
        with pytest.raises(pk.PkError):          # nothing to attend
            pk.pk_attend_dense(h, q, None, 0, dK, dV, 0, out)
        mis = torch.empty(dK.numel() + 8, dtype=dK.dtype, device="cuda")[1:1 + dK.numel()].view(dK.shape)
        with pytest.raises(pk.PkError):          # dense rows not 16-byte aligned
            pk.pk_attend_dense(h, q, idx, 100, mis, dV, dlen, out)
    finally:
        pk.pk_free(h)


@pytest.mark.parametrize("offload,async_reindex", [(False, False), (True, False), (False, True), (True, True)])
def test_decode_cache_sink_local_update(pk, offload, async_reindex):
    """The sink/local/update-buffer layout over 160 decode steps (sink 16,
    local 64, update 32; re-indexing every 32 steps): the retrieval zone
    grows by whole update buffers, the dense tail stays within
    (local, local + update] (up to 4 steps more while a batch is staged
    asynchronously, in 4 pieces),
    the Top-k over the zone matches the oracle's search of the zone, and the
    output is the oracle's attention over sink + tail + retrieved rows."""
    from kv_cache_top_b200.decode_cache import DecodeCache
    T0, steps, H, G = 4096, 160, 2, 2
    sink, local, update = 16, 64, 32
    w = workloads.llama_layer(1, T0 + steps, H=H, G=G, seed=77, device="cuda", n_queries=steps)
    K, V = w["K"], w["V"]
    cache = DecodeCache(K[:, :, :T0].contiguous(), V[:, :, :T0].contiguous(), group=G, sink=sink, local=local,
                        update=update, max_len=T0 + steps, offload=offload, async_reindex=async_reindex)
    lag = 4 if async_reindex else 0          # 4 staging pieces, published one step after the last
    try:
        for t in range(steps):
            out = cache.step(w["q"][t], K[:, :, T0 + t:T0 + t + 1].contiguous(),
                             V[:, :, T0 + t:T0 + t + 1].contiguous())
            if t not in (0, 31, 32, 33, 100, 129, steps - 1):
                continue
            torch.cuda.synchronize()
            T = T0 + t + 1
            z0, z1 = cache.zone
            assert z0 == sink and (z1 - (T0 - local)) % update == 0
            assert cache.info().n == z1 - z0 and cache.tail == T - z1 and local < cache.tail <= local + update + lag
            idx2 = torch.empty_like(cache.idx)
            sc2 = torch.empty(H, 100, dtype=torch.float32, device="cuda")
            pk.pk_search(cache.index, w["q"][t], 100, idx2, sc2)
            torch.cuda.synchronize()
            assert torch.equal(idx2, cache.idx)
            idx, sc, o = idx2.cpu().numpy(), sc2.cpu().numpy(), out.cpu().numpy()
            for p in range(H):
                Kz = workloads.to_np_f32(K[0, p, z0:z1])
                Vz = workloads.to_np_f32(V[0, p, z0:z1])
                qg = workloads.to_np_f32(w["q"][t][0, p * G:(p + 1) * G])
                enc, orc = parity.oracle_pair(Kz, qg, 100, 0)
                parity.check_topk(idx[p], sc[p], orc, enc)
                Kd = np.concatenate([workloads.to_np_f32(K[0, p, :sink]), workloads.to_np_f32(K[0, p, z1:T])])
                Vd = np.concatenate([workloads.to_np_f32(V[0, p, :sink]), workloads.to_np_f32(V[0, p, z1:T])])
                ref = parity.oracle.attend_union(qg, Kz, Vz, idx[p], Kd, Vd, 1.0 / math.sqrt(128))
                parity.check_attention(o[0, p * G:(p + 1) * G], ref)
        assert cache.reindexed == 4          # at steps 32, 64, 96 and 128
    finally:
        cache.close()


@pytest.mark.parametrize("batch,H,G,n,kv_location,dtype", [
    (1, 2, 4, 20000, 0, torch.bfloat16), (2, 1, 2, 9000, 1, torch.bfloat16),
    (1, 1, 6, 40000, 0, torch.bfloat16),   # two packed bonus words per centre, the second half full; 40 key chunks
    (1, 1, 8, 5000, 1, torch.bfloat16),    # the largest group: both words full
    (1, 2, 4, 9000, 1, torch.float32),     # fp32 K/V and query, rows gathered as a union over UVA
])
def test_per_query_head_search(pk, batch, H, G, n, kv_location, dtype):
    """pk_search_heads / pk_attend_heads: each query head searches its pair's
    index with its own query (the oracle's search with G = 1 on that head),
    and attends over its own rows; the aggregated search is unchanged."""
    w = workloads.llama_layer(batch, n, H=H, G=G, seed=n + 3, device="cuda", dtype=dtype)
    q = w["q"][0]
    h = build(pk, w["K"], w["V"], n, batch, H, G, kv_location=kv_location)
    try:
        U = batch * H * G
        idx = torch.empty(U, 100, dtype=torch.int32, device="cuda")
        sc = torch.empty(U, 100, dtype=torch.float32, device="cuda")
        out = torch.full((batch, H * G, 128), float("nan"), dtype=torch.float32, device="cuda")
        pk.pk_search_heads(h, q, 100, idx, sc)
        pk.pk_attend_heads(h, q, idx, 100, out)
        torch.cuda.synchronize()
        st, det = pk.pk_last_device_error(h)
        assert st == 0, (st, det)
        ids, scs, o = idx.cpu().numpy(), sc.cpu().numpy(), out.cpu().numpy()
        for u in range(U):
            b, j = divmod(u, H * G)
            hh = j // G
            K_np = workloads.to_np_f32(w["K"][b, hh, :n])
            V_np = workloads.to_np_f32(w["V"][b, hh, :n])
            qh = workloads.to_np_f32(q[b, j:j + 1])
            enc, orc = parity.oracle_pair(K_np, qh, 100, 0)
            parity.check_topk(ids[u], scs[u], orc, enc)
            ref = parity.oracle.attend(qh, K_np, V_np, ids[u], 1.0 / math.sqrt(128))
            parity.check_attention(o[b, j:j + 1], ref, 1e-4 if dtype == torch.float32 else parity.ATTN_ABS)
        # the aggregated path after the per-head workspace exists
        check_pairs(pk, h, w["K"], w["V"], q, [0], batch, H, G, n, 100, check_encode=False)
    finally:
        pk.pk_free(h)


@pytest.mark.parametrize("G,topk,kv_location,dtype", [
    (4, 100, 1, torch.bfloat16), (8, 100, 1, torch.bfloat16),   # K/V in host memory: the union gather
    (4, 100, 1, torch.float32),
    (4, 256, 1, torch.bfloat16),   # G x topk = 1024: the largest union the table takes
    (4, 1, 1, torch.bfloat16),     # one row per head
    (4, 100, 0, torch.bfloat16),   # K/V in HBM: one cluster per query head
    (8, 200, 1, torch.bfloat16),   # lists past the union table: one cluster per query head
])
def test_attend_heads_union_of_lists(pk, G, topk, kv_location, dtype):
    """pk_attend_heads on hand-made per-head lists: heavy overlap between the
    heads of a pair, one head's list equal to another's, an id repeated
    inside one list (union path only) and an out-of-range id.  Each head's
    output is the oracle's attention over the distinct valid ids of its own
    list."""
    batch, H, n = 1, 2, 5000
    w = workloads.llama_layer(batch, n, H=H, G=G, seed=17, device="cuda", dtype=dtype)
    q = w["q"][0]
    h = build(pk, w["K"], w["V"], n, batch, H, G, topk=topk, kv_location=kv_location)
    try:
        rng = np.random.default_rng(5)
        U = batch * H * G
        sel = np.empty((U, topk), np.int32)
        for pair in range(batch * H):
            pool = rng.choice(n, size=int(1.5 * topk), replace=False).astype(np.int32)
            for g in range(G):
                sel[pair * G + g] = rng.choice(pool, size=topk, replace=False)
            sel[pair * G + 1] = sel[pair * G + 0]           # two heads with the same list
            if kv_location == 1 and G * topk <= 1024:        # the union path takes a list as a set
                sel[pair * G + 2, -1] = sel[pair * G + 2, 0]    # an id twice in one list
        bad = n + 3
        if topk > 1:
            sel[G + 3, min(5, topk - 1)] = bad               # out of range: skipped and recorded
        sel_t = torch.from_numpy(sel).cuda()
        out = torch.full((batch, H * G, 128), float("nan"), dtype=torch.float32, device="cuda")
        pk.pk_attend_heads(h, q, sel_t, topk, out)
        torch.cuda.synchronize()
        st, det = pk.pk_last_device_error(h)
        assert (st, det) == ((6, bad) if topk > 1 else (0, 0)), (st, det)
        o = out.cpu().numpy()
        for u in range(U):
            b, j = divmod(u, H * G)
            hh = j // G
            K_np = workloads.to_np_f32(w["K"][b, hh, :n])
            V_np = workloads.to_np_f32(w["V"][b, hh, :n])
            qh = workloads.to_np_f32(q[b, j:j + 1])
            ids = np.unique(sel[u][(sel[u] >= 0) & (sel[u] < n)])
            ref = parity.oracle.attend(qh, K_np, V_np, ids, 1.0 / math.sqrt(128))
            parity.check_attention(o[b, j:j + 1], ref, 1e-4 if dtype == torch.float32 else parity.ATTN_ABS)
    finally:
        pk.pk_free(h)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_query_load_paths_agree(pk, dtype):
    """The query prep and the attention read q with 16-byte loads when its
    rows start on a 16-byte boundary and one element at a time otherwise
    (q shifted by one element here): ids, scores and outputs are bit-equal."""
    batch, H, G, n = 2, 2, 4, 6000
    w = workloads.llama_layer(batch, n, H=H, G=G, seed=23, device="cuda", dtype=dtype)
    h = build(pk, w["K"], w["V"], n, batch, H, G)
    try:
        q = w["q"][0].contiguous()
        buf = torch.empty(q.numel() + 8, dtype=dtype, device="cuda")
        q_odd = buf[1:1 + q.numel()].view_as(q)
        q_odd.copy_(q)
        assert q.data_ptr() % 16 == 0 and q_odd.data_ptr() % 16 != 0
        res = []
        for qq in (q, q_odd):
            idx = torch.empty(batch * H, 100, dtype=torch.int32, device="cuda")
            sc = torch.empty(batch * H, 100, dtype=torch.float32, device="cuda")
            out = torch.empty(batch, H * G, 128, dtype=torch.float32, device="cuda")
            pk.pk_search(h, qq, 100, idx, sc)
            pk.pk_attend(h, qq, idx, 100, out)
            torch.cuda.synchronize()
            res.append((idx.cpu(), sc.cpu(), out.cpu()))
        assert torch.equal(res[0][0], res[1][0])
        assert torch.equal(res[0][1].view(torch.int32), res[1][1].view(torch.int32))
        assert torch.equal(res[0][2].view(torch.int32), res[1][2].view(torch.int32))
        st, det = pk.pk_last_device_error(h)
        assert st == 0, (st, det)
    finally:
        pk.pk_free(h)


def test_host_pinned_kv_store(pk):
    """K/V kept in pinned host memory and read through UVA by the attention."""
    w = workloads.llama_layer(1, 20000, H=2, G=4, seed=3, device="cuda")
    h = build(pk, w["K"], w["V"], 20000, 1, 2, 4, kv_location=1)
    try:
        assert pk.pk_get_info(h).kv_location == 1
        check_pairs(pk, h, w["K"], w["V"], w["q"][0], [0, 1], 1, 2, 4, 20000, 100)
    finally:
        pk.pk_free(h)


def test_attend_out_of_range_ids_are_skipped_and_recorded(pk):
    w = workloads.llama_layer(1, 500, H=1, G=1, seed=4, device="cuda")
    h = build(pk, w["K"], w["V"], 500, 1, 1, 1)
    try:
        sel = torch.arange(100, dtype=torch.int32, device="cuda").view(1, 100)
        sel[0, 7] = 505
        out = torch.empty(1, 1, 128, dtype=torch.float32, device="cuda")
        pk.pk_attend(h, w["q"][0], sel, 100, out)
        st, det = pk.pk_last_device_error(h)
        assert st == 6 and det == 505
        assert torch.isfinite(out).all()
        keep = [i for i in range(100) if i != 7]
        ref = parity.oracle.attend(workloads.to_np_f32(w["q"][0, 0]), workloads.to_np_f32(w["K"][0, 0]),
                                   workloads.to_np_f32(w["V"][0, 0]), np.array(keep, np.int32),
                                   1.0 / math.sqrt(128))
        assert np.abs(out[0].cpu().numpy() - ref).max() <= parity.ATTN_ABS
        assert pk.pk_last_device_error(h)[0] == 0
    finally:
        pk.pk_free(h)


def test_append_stage_publish(pk):
    """Staged keys stay invisible to search until published; after publishing,
    the index equals one built over all keys at once (strided source rows,
    two staging calls, the staging on a side stream)."""
    w = workloads.llama_layer(2, 9000, H=2, G=2, seed=19, device="cuda")
    K, V = w["K"], w["V"]
    n0 = 8000
    h = build(pk, K[:, :, :n0].contiguous(), V[:, :, :n0].contiguous(), n0, 2, 2, 2, n_cap=9000)
    try:
        BH = 4
        idx0 = torch.empty(BH, 100, dtype=torch.int32, device="cuda")
        pk.pk_search(h, w["q"][0], 100, idx0)
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        # rows n0 .. n0+599 and n0+600 .. 8999 taken in place from the [batch][H][9000][D] arrays
        pk.pk_append_stage(h, K[:, :, n0:], V[:, :, n0:], 600, 9000, stream=side)
        pk.pk_append_stage(h, K[:, :, n0 + 600:], V[:, :, n0 + 600:], 400, 9000, stream=side)
        info = pk.pk_get_info(h)
        assert info.n == n0 and info.n_staged == 1000
        with pytest.raises(pk.PkError) as e:        # pk_append while keys are staged
            pk.pk_append(h, K[:, :, :1].contiguous(), V[:, :, :1].contiguous(), 1)
        assert e.value.status == 1
        idx1 = torch.empty_like(idx0)
        pk.pk_search(h, w["q"][0], 100, idx1)       # the decode stream: staged keys not visible
        torch.cuda.synchronize()
        assert torch.equal(idx0, idx1)
        pk.pk_append_publish(h)
        pk.pk_append_publish(h)                     # nothing left to publish
        assert pk.pk_get_info(h).n == 9000 and pk.pk_get_info(h).n_staged == 0
        check_pairs(pk, h, K, V, w["q"][0], list(range(BH)), 2, 2, 2, 9000, 100)
        with pytest.raises(pk.PkError) as e:        # past n_cap
            pk.pk_append_stage(h, K[:, :, :1], V[:, :, :1], 1, 9000)
        assert e.value.status == 2
    finally:
        pk.pk_free(h)


@pytest.mark.parametrize("kv_location", [0, 1])
def test_build_from_unaligned_kv(pk, kv_location):
    """K/V inputs aligned to their element size but not to 16 bytes take the
    copy path for unaligned sources into the interleaved K/V store; the
    index and the attention are the same."""
    w = workloads.llama_layer(1, 3000, H=2, G=2, seed=23, device="cuda")
    K, V = w["K"], w["V"]

    def shifted(x):                                   # same values at a 2-byte offset
        flat = torch.empty(x.numel() + 8, dtype=x.dtype, device="cuda")
        y = flat[1:1 + x.numel()].view(x.shape)
        y.copy_(x)
        assert y.data_ptr() % 16 != 0
        return y

    h = build(pk, shifted(K), shifted(V), 3000, 1, 2, 2, kv_location=kv_location)
    try:
        check_pairs(pk, h, K, V, w["q"][0], [0, 1], 1, 2, 2, 3000, 100)
    finally:
        pk.pk_free(h)


def test_search_rejects_bad_arguments(pk):
    w = workloads.llama_layer(1, 300, H=1, G=1, seed=6, device="cuda")
    h = build(pk, w["K"], w["V"], 300, 1, 1, 1)
    try:
        idx = torch.empty(1, 100, dtype=torch.int32, device="cuda")
        with pytest.raises(pk.PkError) as e:
            pk.pk_search(h, w["q"][0], 101, idx)
        assert e.value.status == 1
        host = np.zeros((1, 1, 128), np.float32)        # pageable host memory
        with pytest.raises(pk.PkError) as e:
            pk.pk_search(h, host.ctypes.data, 100, idx)
        assert e.value.status == 1
    finally:
        pk.pk_free(h)


def test_many_pairs_small_rerank_ctas(pk):
    """8 sequences x 8 KV heads (64 pairs), n = 40960, C = 4096: the rerank
    splits each pair's candidates over 128-thread CTAs (9 slices of 464; the
    256-thread split, 4 slices of 1024 on 256 CTAs, would load the busiest SM
    with 2048 records against 1856), so the merge combines 9 lists.  Four
    pairs checked element by element."""
    batch, n, H, G = 8, 40960, 8, 4
    w = workloads.llama_layer(batch, n, H=H, G=G, seed=12, device="cuda", n_queries=1)
    h = build(pk, w["K"], w["V"], n, batch, H, G, cand_budget=4096)
    try:
        idx = check_pairs(pk, h, w["K"], w["V"], w["q"][0], [0, 21, 42, 63], batch, H, G, n, 100,
                          cand_budget=4096)
        for p in range(batch * H):
            assert len(set(idx[p].tolist())) == 100
    finally:
        pk.pk_free(h)
        del w
        torch.cuda.empty_cache()


def test_compaction_large_chunks_every_key_a_candidate(pk):
    """40 pairs of n = 70000 with C = n: 14 chunks of ~5000 keys per pair, so
    a chunk holds more candidates than the compaction stages in shared memory
    and its threads store their ids directly.  Three pairs checked element by
    element."""
    batch, n, H, G = 40, 70000, 1, 1
    w = workloads.llama_layer(batch, n, H=H, G=G, seed=77, device="cuda", n_queries=1)
    h = build(pk, w["K"], w["V"], n, batch, H, G, cand_budget=n)
    try:
        assert pk.pk_get_info(h).nchunks <= 16
        check_pairs(pk, h, w["K"], w["V"], w["q"][0], [0, 17, 39], batch, H, G, n, 100, cand_budget=n,
                    check_encode=False)
    finally:
        pk.pk_free(h)
        del w
        torch.cuda.empty_cache()


# ------------------------------------------------- full-size workloads
def test_throughput_batch_full_size(pk):
    """8 sequences x n = 131072, 8 KV heads, 32 query heads, bf16, ratio-table
    budgets (C = 13108, R = 26215), K/V in HBM: the benchmark's workload and
    launch configuration.  All 64 (sequence, KV head) pairs are checked
    against the oracle (S, histogram, threshold and candidates bit-exact,
    every candidate's estimate, the Top-k rule and the attention output);
    the encoding is compared bit for bit on four of them."""
    batch, n, H, G = 8, 131072, 8, 4
    w = workloads.llama_layer(batch, n, H=H, G=G, seed=0, device="cuda")
    h = build(pk, w["K"], w["V"], n, batch, H, G)
    try:
        idx = check_pairs(pk, h, w["K"], w["V"], w["q"][0], list(range(batch * H)), batch, H, G, n, 100,
                          check_encode=True, encode_pairs=[0, 21, 45, 63])
        for p in range(batch * H):
            assert len(set(idx[p].tolist())) == 100
    finally:
        pk.pk_free(h)
        del w
        torch.cuda.empty_cache()


def test_million_token_offload_full_size(pk):
    """batch 1, n = 1048576, 8 KV heads, bf16, full K/V (4 GiB) in pinned host
    memory, codes + summaries on the GPU, Top-100 fetched through UVA.  All 8
    pairs are checked against the oracle; the encoding of one pair (1M keys)
    is compared bit for bit."""
    n, H, G = 1 << 20, 8, 4
    w = workloads.llama_layer(1, n, H=H, G=G, seed=1, device="cuda")
    h = build(pk, w["K"], w["V"], n, 1, H, G, kv_location=1)
    try:
        check_pairs(pk, h, w["K"], w["V"], w["q"][0], list(range(H)), 1, H, G, n, 100,
                    check_encode=True, encode_pairs=[5], workers=4)
    finally:
        pk.pk_free(h)
        del w
        torch.cuda.empty_cache()
