"""The allocation-free MLA decode entry point against the regular one.

dsa_sparse_mla_decode_noalloc serves callers that cannot call cudaMalloc (code running inside
another framework's memory pool, or on paths where allocation is not allowed): it keeps the
split-K partials in the library's fixed device scratch instead of a caller workspace.  This file
is collected last on purpose, so that a run stopping at the first failure has run every other
test first; it also passes when run alone in a fresh process.
"""
import ctypes

import pytest
import torch

import dsa_inputs as di
import sparse_attention_06_b200 as dsa
from _parity import TOL, cache_and_batch, check_mla, to_dev

pytestmark = pytest.mark.gpu


def _decode_case(lens, seed):
    spec = di.Spec("noalloc", lens=lens, q_req=list(range(len(lens))), q_pos=[L - 1 for L in lens], seed=seed)
    x = to_dev(di.generate(spec, "cpu"))
    keys, lat, batch, max_ctx = cache_and_batch(x)
    ld = (max_ctx + 3) // 4 * 4
    scores = torch.empty((spec.T, ld), dtype=torch.float32, device="cuda")
    idx = torch.empty((spec.T, spec.k), dtype=torch.int32, device="cuda")
    dsa.dsa_indexer_topk(x["q_idx"], x["w"], keys, batch, spec.k, scores, idx)
    return spec, x, lat, batch, idx


def test_noalloc_matches_workspace_entry_point_twice():
    # two queries: the regular entry point splits their rows across CTAs, so the scratch is used
    spec, x, lat, batch, idx = _decode_case([5000, 2900], seed=41)
    ws_bytes = dsa.dsa_mla_workspace_size(spec.T, spec.H, spec.d_v, spec.k)
    assert 0 < ws_bytes <= 32 << 20
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device="cuda")
    ref = torch.empty((spec.T, spec.H, spec.d_v), dtype=torch.bfloat16, device="cuda")
    ref_lse = torch.empty((spec.T, spec.H), dtype=torch.float32, device="cuda")
    dsa.dsa_clear_device_error()
    dsa.dsa_sparse_mla_decode(x["q_mla"], lat, batch, idx, spec.scale, ref, ref_lse, ws)
    lib = dsa.load_library()
    lc, bc = lat._c(), batch._c()
    for _ in range(2):  # the scratch keeps the previous call's contents; the result must not care
        out = torch.full((spec.T, spec.H, spec.d_v), float("nan"), dtype=torch.bfloat16, device="cuda")
        lse = torch.full((spec.T, spec.H), float("nan"), dtype=torch.float32, device="cuda")
        st = lib.dsa_sparse_mla_decode_noalloc(
            x["q_mla"].data_ptr(), dsa.DSA_BF16, spec.H, spec.d_v, spec.d_rope, ctypes.byref(lc),
            ctypes.byref(bc), idx.data_ptr(), spec.k, ctypes.c_float(spec.scale), out.data_ptr(),
            lse.data_ptr(), torch.cuda.current_stream().cuda_stream)
        assert st == dsa.DSA_OK, lib.dsa_last_error_message()
        torch.cuda.synchronize()
        check_mla(out.float().cpu(), lse.cpu(), ref.double().cpu().numpy(), ref_lse.double().cpu().numpy(),
                  TOL["bf16"])
    assert dsa.dsa_get_device_error() == 0


def test_noalloc_rejects_sizes_beyond_its_scratch():
    # the smallest decode batch whose split-K partials exceed the 32 MiB scratch on this GPU
    T = next((t for t in range(2, 1024) if dsa.dsa_mla_workspace_size(t, 128, 512, 2048) > 32 << 20), None)
    assert T is not None
    spec, x, lat, batch, idx = _decode_case([2100] * T, seed=42)
    need = dsa.dsa_mla_workspace_size(spec.T, spec.H, spec.d_v, spec.k)
    assert need > 32 << 20
    out = torch.empty((spec.T, spec.H, spec.d_v), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(dsa.DsaError) as e:
        dsa.dsa_sparse_mla_decode_noalloc(x["q_mla"], lat, batch, idx, spec.scale, out)
    assert e.value.status == dsa.DSA_ERR_INVALID_ARG and "scratch" in str(e.value)


def test_noalloc_generic_shape_needs_no_scratch():
    # f32 operands take the generic kernels, which use no split partials: a batch whose bf16
    # tensor-core plan would exceed the scratch is accepted and matches the workspace entry point
    T = next((t for t in range(2, 1024) if dsa.dsa_mla_workspace_size(t, 128, 512, 2048) > 32 << 20), None)
    spec = di.Spec("noalloc_f32", lens=[2100] * T, q_req=list(range(T)), q_pos=[2099] * T, act_dtype="f32",
                   key_dtype="f32", seed=43)
    x = to_dev(di.generate(spec, "cpu"))
    keys, lat, batch, max_ctx = cache_and_batch(x)
    idx = torch.empty((spec.T, spec.k), dtype=torch.int32, device="cuda")
    scores = torch.empty((spec.T, (max_ctx + 3) // 4 * 4), dtype=torch.float32, device="cuda")
    dsa.dsa_indexer_topk(x["q_idx"], x["w"], keys, batch, spec.k, scores, idx)
    ref = torch.empty((spec.T, spec.H, spec.d_v), dtype=torch.float32, device="cuda")
    dsa.dsa_sparse_mla_decode(x["q_mla"], lat, batch, idx, spec.scale, ref)
    out = torch.full_like(ref, float("nan"))
    dsa.dsa_sparse_mla_decode_noalloc(x["q_mla"], lat, batch, idx, spec.scale, out)
    torch.cuda.synchronize()
    assert torch.equal(out, ref)
