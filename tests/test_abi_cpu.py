"""The C ABI library builds, loads and exports every entry point include/dsa.h declares; host-side
argument checks reject bad calls before anything touches CUDA.  No compute calls (no GPU here)."""
import ctypes
import os
import re

import pytest

import sparse_attention_06_b200 as dsa
from sparse_attention_06_b200 import build as dsa_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    dsa_build.build()
    return dsa.load_library()


def _declared():
    src = open(os.path.join(ROOT, "include", "dsa.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(dsa_[a-z0-9_]+)\s*\(", src)))


def test_every_declared_symbol_is_exported(lib):
    names = _declared()
    assert "dsa_indexer_scores" in names and "dsa_sparse_mla_prefill" in names
    for n in names:
        assert hasattr(lib, n), n
    assert set(dsa.EXPORTED) <= set(names)


def test_version_and_status_strings(lib):
    assert lib.dsa_abi_version() == 2
    assert lib.dsa_status_string(dsa.DSA_ERR_INVALID_ARG) == b"invalid argument"


def test_invalid_arguments_rejected_on_host(lib):
    # NULL batch
    st = lib.dsa_indexer_scores(None, 1, None, 64, 128, None, None, None, None, 0, None, None)
    assert st == dsa.DSA_ERR_INVALID_ARG
    assert b"batch" in lib.dsa_last_error_message()
    # k out of range / NULL pointers in the selection
    assert lib.dsa_topk_select(None, 10, None, 1, 5, None, None, None) == dsa.DSA_ERR_INVALID_ARG
    fake = ctypes.c_void_p(16)
    assert lib.dsa_topk_select(fake, 10, fake, 1, 0, fake, None, None) == dsa.DSA_ERR_INVALID_ARG
    assert lib.dsa_topk_select(fake, 10, fake, 1, 5000, fake, None, None) == dsa.DSA_ERR_INVALID_ARG
    # a histogram must be 16-byte aligned
    assert lib.dsa_topk_select(fake, 10, fake, 1, 5, fake, ctypes.c_void_p(20), None) == dsa.DSA_ERR_INVALID_ARG
    # query_group must divide num_queries
    b = dsa._Batch(6, 1, 16, 16, 16, 4, 256, 4, 0)
    kc = dsa._PagedCache(16, None, 4, 64, 128, dsa.DSA_BF16, 0)
    st = lib.dsa_indexer_scores(fake, 1, None, 64, 128, fake, ctypes.byref(kc), ctypes.byref(b), fake, 256, None, None)
    assert st == dsa.DSA_ERR_INVALID_ARG and b"query_group" in lib.dsa_last_error_message()
    # e4m3 queries without their per-head scale
    b1 = dsa._Batch(1, 1, 16, 16, 16, 4, 256, 1, 0)
    kc1 = dsa._PagedCache(16, 16, 4, 64, 128, dsa.DSA_E4M3, 0)
    st = lib.dsa_indexer_scores(fake, dsa.DSA_E4M3, None, 64, 128, fake, ctypes.byref(kc1), ctypes.byref(b1), fake,
                                256, None, None)
    assert st == dsa.DSA_ERR_INVALID_ARG and b"q_scale" in lib.dsa_last_error_message()
    # e4m3 cache without a scale
    b = dsa._Batch(1, 1, 16, 16, 16, 4, 256, 1, 0)
    kc = dsa._PagedCache(16, None, 4, 64, 128, dsa.DSA_E4M3, 0)
    st = lib.dsa_indexer_scores(fake, 1, None, 64, 128, fake, ctypes.byref(kc), ctypes.byref(b), fake, 256, None, None)
    assert st == dsa.DSA_ERR_INVALID_ARG and b"scale" in lib.dsa_last_error_message()
    # latent dim must be d_v + d_rope; scale must be positive
    lc = dsa._PagedCache(16, None, 4, 64, 500, dsa.DSA_BF16, 0)
    st = lib.dsa_sparse_mla_decode(fake, 1, 128, 512, 64, ctypes.byref(lc), ctypes.byref(b), fake, 2048,
                                   ctypes.c_float(0.07), fake, None, None, 0, None)
    assert st == dsa.DSA_ERR_INVALID_ARG
    lc = dsa._PagedCache(16, None, 4, 64, 576, dsa.DSA_BF16, 0)
    st = lib.dsa_sparse_mla_decode(fake, 1, 128, 512, 64, ctypes.byref(lc), ctypes.byref(b), fake, 2048,
                                   ctypes.c_float(-1.0), fake, None, None, 0, None)
    assert st == dsa.DSA_ERR_INVALID_ARG
    # the gather-rate diagnostic checks its shape and sizes on the host
    gc = dsa._PagedCache(16, None, 4, 64, 576, dsa.DSA_BF16, 0)
    assert lib.dsa_selftest_gather_rate(ctypes.byref(gc), None, 1, 1, fake, None) == dsa.DSA_ERR_INVALID_ARG
    assert lib.dsa_selftest_gather_rate(ctypes.byref(gc), fake, 0, 1, fake, None) == dsa.DSA_ERR_INVALID_ARG
    assert lib.dsa_selftest_gather_rate(ctypes.byref(gc), fake, 1, 2000, fake, None) == dsa.DSA_ERR_INVALID_ARG
    gc = dsa._PagedCache(16, None, 4, 64, 512, dsa.DSA_BF16, 0)
    assert lib.dsa_selftest_gather_rate(ctypes.byref(gc), fake, 1, 1, fake, None) == dsa.DSA_ERR_INVALID_ARG
    # max_blocks * block_size must cover max_context
    b = dsa._Batch(1, 1, 16, 16, 16, 2, 256, 1, 0)
    st = lib.dsa_sparse_mla_decode(fake, 1, 128, 512, 64, ctypes.byref(lc), ctypes.byref(b), fake, 2048,
                                   ctypes.c_float(0.07), fake, None, None, 0, None)
    assert st == dsa.DSA_ERR_INVALID_ARG


def test_empty_batch_is_a_noop(lib):
    b = dsa._Batch(0, 0, None, None, None, 0, 0, 1, 0)
    assert lib.dsa_indexer_scores(None, 1, None, 64, 128, None, None, ctypes.byref(b), None, 0, None, None) == dsa.DSA_OK
    assert lib.dsa_topk_select(None, 1, None, 0, 16, None, None, None) == dsa.DSA_OK


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    monkeypatch.setattr(dsa, "LIB_PATH", str(tmp_path / "nope.so"))
    monkeypatch.setattr(dsa, "_lib", None)
    with pytest.raises(dsa.DsaLibraryMissing):
        dsa.load_library()


def test_mla_split_plan_and_workspace(lib):
    # The decode plan of the tensor-core MLA: key splits per query chosen by the library's cost
    # model for a 148-SM B200 (the SM count the library assumes when no device answers), and the
    # workspace of their f32 partials: T * nsplit * 128 * (512 + 1) floats in two 256-byte aligned
    # parts.  A query alone spreads its 32 row tiles over 32 CTA pairs; a batch that already fills
    # the SMs takes no split (and needs no workspace).
    def ws(T, nsplit):
        o = T * nsplit * 128 * 512 * 4
        l = T * nsplit * 128 * 4
        return ((o + 255) // 256) * 256 + ((l + 255) // 256) * 256
    for T, nsplit in ((1, 32), (3, 16), (8, 8), (16, 4), (75, 2), (100, 2)):
        assert lib.dsa_mla_workspace_size(T, 128, 512, 2048) == ws(T, nsplit), T
    assert lib.dsa_mla_workspace_size(64, 128, 512, 2048) == 0
    assert lib.dsa_mla_workspace_size(2, 128, 512, 100) == 0   # two tiles per query: no split
    assert lib.dsa_mla_workspace_size(0, 128, 512, 2048) == 0
    # the GLM-5 shape (64 heads) takes the same plan, with half the partial rows
    def ws64(T, nsplit):
        o = T * nsplit * 64 * 512 * 4
        l = T * nsplit * 64 * 4
        return ((o + 255) // 256) * 256 + ((l + 255) // 256) * 256
    assert lib.dsa_mla_workspace_size(16, 64, 512, 2048) == ws64(16, 4)
    assert lib.dsa_mla_workspace_size(4, 32, 512, 2048) == 0    # not a tensor-core shape


def test_indexer_topk_workspace_size(lib):
    # one row of 4096 uint32 order-key digit counters per query
    assert lib.dsa_indexer_topk_workspace_size(1) == 4096 * 4
    assert lib.dsa_indexer_topk_workspace_size(64) == 64 * 4096 * 4
    assert lib.dsa_indexer_topk_workspace_size(0) == 0
