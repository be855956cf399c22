"""Host-side checks of the C-ABI library that need no GPU: it loads, exports every symbol that
include/tq.h declares, computes the codebook on the host like the oracle, and rejects bad
arguments before touching the device."""
import ctypes
import os
import re

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    from kv_cache_vector_06_b200.build import build
    build()
    from kv_cache_vector_06_b200 import tq
    return tq


def declared_functions():
    names = set()
    for f in os.listdir(os.path.join(ROOT, "include")):
        if f.endswith(".h"):
            src = open(os.path.join(ROOT, "include", f)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names |= set(re.findall(r"\b(tq_[a-z0-9_]+)\s*\(", src))
    return names


def test_exports_every_declared_symbol(lib):
    names = declared_functions()
    assert {"tq_make_codebook", "tq_encode_kv", "tq_scores", "tq_attend_decode", "tq_search_topk"} <= names
    raw = ctypes.CDLL(lib.LIB_PATH)
    for n in sorted(names):
        assert hasattr(raw, n), n


def test_library_is_built_for_sm100a_only(lib):
    # the build compiles every translation unit and links with exactly one target: sm_100a
    from kv_cache_vector_06_b200 import build
    assert build.ARCH == ["-gencode", "arch=compute_100a,code=sm_100a"]
    assert not any("compute_" in f or "sm_" in f for f in build.FLAGS)
    assert "sm_100a" in lib.version()


def test_search_k_range_checked_before_anything_else(lib):
    """k in [1, 1024] is supported (k > 32 takes the large-k scan); larger k is refused with
    TQ_EUNSUPPORTED and k < 1 with TQ_EINVAL, before the context is looked at."""
    from ctypes import byref, c_size_t
    L, b = lib.LIB, c_size_t()
    assert L.tq_search_workspace_size(None, 10, 5000, 1025, byref(b)) == 2
    assert b"at most 1024" in L.tq_last_error()
    assert L.tq_search_workspace_size(None, 10, 5000, 0, byref(b)) == 1
    for k in (1, 32, 33, 1024):  # accepted: the next check (the NULL context) answers
        assert L.tq_search_workspace_size(None, 10, 5000, k, byref(b)) == 1
        assert b"ctx is NULL" in L.tq_last_error()
    assert L.tq_search_topk(None, None, 0, 1, lib.PackedC(), 5000, 4096, None, None, None, 0, None) == 2
    assert L.tq_search_topk(None, None, 0, 1, lib.PackedC(), 5000, 1024, None, None, None, 0, None) == 1


def test_status_codes_match_the_header(lib):
    # the binding's status names follow tq.h's enum, TQ_ETIMEOUT included
    hdr = open(os.path.join(ROOT, "include", "tq.h")).read()
    for code, name in lib.STATUS.items():
        assert re.search(rf"\b{name}\s*=\s*{code}\b", hdr), name
    assert lib.TQ_ETIMEOUT == 5 and lib.STATUS[5] == "TQ_ETIMEOUT"


@pytest.mark.parametrize("d", [8, 16, 32, 64, 128, 256, 512, 1024])
@pytest.mark.parametrize("bits", [1, 2, 3, 4])
def test_host_codebook_matches_oracle(lib, d, bits):
    from oracle import codebook
    c, t, mse = lib.make_codebook(d, bits)
    co, to = codebook.codebook(d, bits)
    np.testing.assert_allclose(c, co, rtol=0, atol=1e-10)
    np.testing.assert_allclose(t, to, rtol=0, atol=1e-10)
    assert mse == pytest.approx(codebook.mse_per_coord(d, co, to), rel=1e-9)


def test_codebook_rejects_bad_sizes(lib):
    for d, b in [(100, 2), (4, 2), (2048, 2), (128, 0), (128, 5)]:
        with pytest.raises(lib.TqError) as e:
            lib.make_codebook(d, b)
        assert e.value.status == 2


def test_codebook_null_outputs_rejected(lib):
    st = lib.LIB.tq_make_codebook(128, 2, None, None, None)
    assert st == 1 and b"NULL" in lib.LIB.tq_last_error()


def test_ctx_create_validates_before_device(lib):
    import torch
    with pytest.raises(lib.TqError) as e:
        lib.Context(100, 2, 128, torch.ones(100, dtype=torch.int8), torch.zeros(128, 100))
    assert e.value.status == 2
    with pytest.raises(lib.TqError) as e:
        lib.Context(128, 2, 48, torch.ones(128, dtype=torch.int8), torch.zeros(48, 128))
    assert e.value.status == 2
    bad = torch.ones(128, dtype=torch.int8)
    bad[3] = 0
    with pytest.raises(lib.TqError) as e:
        lib.Context(128, 2, 0, bad)
    assert e.value.status == 1
    # norm storage: 32 (or 0) or 16 bits only
    with pytest.raises(lib.TqError) as e:
        lib.Context(128, 2, 0, torch.ones(128, dtype=torch.int8), norm_bits=8)
    assert e.value.status == 1 and "norm_bits" in str(e.value)


def test_null_arguments_rejected(lib):
    L = lib.LIB
    assert L.tq_ctx_destroy(None) == 0
    assert L.tq_ctx_layout(None, None, None) == 1
    assert L.tq_scores(None, None, 0, 1, lib.PackedC(), 1, None, None, 0, None) == 1
    assert L.tq_attend_decode(None, None, None, None, 0, None, None, 0, None) == 1
    assert L.tq_search_topk(None, None, 0, 1, lib.PackedC(), 1, 1, None, None, None, 0, None) == 1


@pytest.mark.parametrize("level", [1, 2, 3, 5, 7])
@pytest.mark.parametrize("bits", [1, 2, 3, 4])
def test_host_polar_codebook_matches_oracle(lib, level, bits):
    """The library's PolarQuant angle codebooks (host, fp64, Gauss-Legendre quadrature) against
    the oracle's (adaptive quadrature)."""
    from oracle import polar
    c, t = lib.make_polar_codebook(level, bits)
    co, to = polar.angle_codebook(level, bits)
    np.testing.assert_allclose(c, co, rtol=0, atol=1e-9)
    np.testing.assert_allclose(t, to, rtol=0, atol=1e-9)


def test_polar_codebook_rejects_bad_sizes(lib):
    for lv, b in [(0, 2), (11, 2), (3, 0), (3, 5)]:
        with pytest.raises(lib.TqError) as e:
            lib.make_polar_codebook(lv, b)
        assert e.value.status == 2
