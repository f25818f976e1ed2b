"""C-ABI library: loads, exports every declared symbol, and its host logic
(argument checks, budgets, magnitude levels) agrees with the pages and the
oracle.  No kernel is launched and no GPU is needed."""
import ctypes as C
import os
import re

import numpy as np
import pytest

from tests.conftest import ROOT, read_golden


@pytest.fixture(scope="module")
def pk():
    from kv_cache_top_b200 import build
    build.build()
    import kv_cache_top_b200 as pk
    return pk


def _declared_functions():
    src = open(os.path.join(ROOT, "include", "pariskv.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(pk_[a-z_]+)\s*\(", src)))


def test_header_declares_the_boundary_calls():
    names = _declared_functions()
    for required in ("pk_build_index", "pk_append", "pk_search", "pk_attend"):
        assert required in names


def test_library_exports_every_declared_symbol(pk):
    names = _declared_functions()
    assert set(names) == set(pk._lib.EXPORTS)
    for name in names:
        assert hasattr(pk.lib, name), name


def test_library_is_sm100a_and_no_cpu_path(pk):
    out = os.popen("nm -D --defined-only %s" % pk._lib.LIB_PATH).read()
    for name in _declared_functions():
        assert re.search(r"\bT %s\b" % name, out), name


def test_status_strings(pk):
    assert pk.pk_status_str(0) == "ok"
    assert "capacity" in pk.pk_status_str(2)
    assert pk.pk_status_str(99) == "unknown status"


def test_default_params(pk):
    p = pk.pk_default_params()
    assert (p.head_dim, p.sub_dim, p.topk, p.group, p.n_kv_heads) == (128, 8, 100, 4, 8)
    assert p.kv_dtype == pk.PK_BF16 and p.kv_location == pk.PK_KV_DEVICE


def test_host_argument_checks_reject_before_any_launch(pk):
    h = C.c_void_p()
    p = pk.pk_default_params(head_dim=64)
    assert pk.lib.pk_build_index(None, None, 10, C.byref(p), None, C.byref(h)) == pk._lib.PK_ERR_UNSUPPORTED
    p = pk.pk_default_params(sub_dim=4)
    assert pk.lib.pk_build_index(None, None, 10, C.byref(p), None, C.byref(h)) == pk._lib.PK_ERR_UNSUPPORTED
    p = pk.pk_default_params(topk=5000)
    assert pk.lib.pk_build_index(None, None, 10, C.byref(p), None, C.byref(h)) == pk._lib.PK_ERR_UNSUPPORTED
    p = pk.pk_default_params(group=0)
    assert pk.lib.pk_build_index(None, None, 10, C.byref(p), None, C.byref(h)) == pk._lib.PK_ERR_INVALID_ARG
    p = pk.pk_default_params(batch=4096, n_kv_heads=8, group=4)       # 131072 query units
    assert pk.lib.pk_build_index(None, None, 10, C.byref(p), None, C.byref(h)) == pk._lib.PK_ERR_UNSUPPORTED
    p = pk.pk_default_params()
    assert pk.lib.pk_build_index(None, None, 10, C.byref(p), None, C.byref(h)) == pk._lib.PK_ERR_INVALID_ARG
    assert pk.lib.pk_build_index(None, None, 10, None, None, C.byref(h)) == pk._lib.PK_ERR_INVALID_ARG
    assert pk.lib.pk_search(None, None, 100, None, None, None) == pk._lib.PK_ERR_INVALID_ARG
    assert pk.lib.pk_attend(None, None, None, 100, None, None) == pk._lib.PK_ERR_INVALID_ARG
    assert pk.lib.pk_append(None, None, None, 1, None) == pk._lib.PK_ERR_INVALID_ARG
    assert pk.lib.pk_append_stage(None, None, None, 1, 0, None) == pk._lib.PK_ERR_INVALID_ARG
    assert pk.lib.pk_append_publish(None, None) == pk._lib.PK_ERR_INVALID_ARG
    pk.pk_free(None)


def test_resolve_matches_readme_ratio_table(pk):
    for ln in read_golden("ratio_table.txt"):
        lo, hi, beta, rho = ln.split()
        lo, hi, beta, rho = int(lo), int(hi), float(beta), float(rho)
        for n in [lo + 200, lo + 1000] + ([hi - 1] if hi > 0 else [1 << 20]):
            C_, R_ = pk.pk_resolve(n, 0, 0.0, 100)
            assert C_ == min(max(int(np.ceil(beta * n)), 100), n)
            assert R_ == int(np.ceil(rho * n))


def test_resolve_matches_oracle(pk):
    import oracle
    for args in [(4096, 512, 0.0, 100), (32768, 2048, 0.2, 100), (131072, 0, 0.0, 100),
                 (1 << 20, 0, 0.0, 100), (150, 10, 0.0, 100), (80, 0, 0.0, 100), (65536, 0, 0.37, 7)]:
        assert pk.pk_resolve(*args) == oracle.resolve(*args), args


def test_magnitude_levels_match_oracle_bit_exact(pk):
    """The library solves the Lloyd-Max fixed point with closed-form cell
    integrals; the oracle with adaptive quadrature.  Same fp32 levels."""
    import oracle
    for m, L in [(8, 8), (3, 8), (8, 4), (16, 8)]:
        lev, thr = pk.pk_magnitude_levels(m, L)
        olev, othr = oracle.levels_f32(m, L)
        assert np.array_equal(lev, olev), (m, L)
        assert np.array_equal(thr, othr), (m, L)


def test_magnitude_levels_reject_bad_arguments(pk):
    with pytest.raises(pk.PkError):
        pk.pk_magnitude_levels(2, 8)
