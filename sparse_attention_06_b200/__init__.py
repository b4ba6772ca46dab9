"""Python binding of the DSA hot-path library (``libdsa.so``, C ABI in ``include/dsa.h``).

Argument marshalling only: every function below takes torch CUDA tensors, checks that they are
laid out as the C ABI expects, and calls the C entry point of the same name.  Every step of the
path runs in the library's CUDA kernels; there is no Python or CPU fallback, and calling any
function without the built library raises ``DsaLibraryMissing``.

Build the library with ``python -m sparse_attention_06_b200.build`` (nvcc, sm_100a).
"""
from __future__ import annotations

import ctypes
import dataclasses
import os
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libdsa.so")

DSA_OK, DSA_ERR_INVALID_ARG, DSA_ERR_UNSUPPORTED, DSA_ERR_CUDA, DSA_ERR_DEVICE_FAULT = range(5)
DSA_F32, DSA_BF16, DSA_E4M3 = 0, 1, 2

DEVERR_BLOCK_ID = 1
DEVERR_INDEX = 2
DEVERR_REQUEST = 4
DEVERR_NAN_SCORE = 8
DEVERR_TIMEOUT = 16
DEVERR_QUERY_GROUP = 32

# Symbols the C ABI exports (checked by the CPU test suite).
EXPORTED = (
    "dsa_indexer_scores", "dsa_topk_select", "dsa_indexer_topk", "dsa_sparse_mla_decode",
    "dsa_sparse_mla_prefill", "dsa_mla_workspace_size", "dsa_get_device_error",
    "dsa_clear_device_error", "dsa_status_string", "dsa_last_error_message", "dsa_abi_version",
    "dsa_kernel_launch_count", "dsa_sparse_mla_decode_noalloc", "dsa_selftest_bounded_wait",
    "dsa_indexer_topk_workspace_size", "dsa_selftest_gather_rate",
)


class DsaLibraryMissing(RuntimeError):
    pass


class DsaError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__("%s (status %d)" % (message, status))
        self.status = status


class _PagedCache(ctypes.Structure):
    _fields_ = [("data", ctypes.c_void_p), ("scale", ctypes.c_void_p), ("num_blocks", ctypes.c_int64),
                ("block_size", ctypes.c_int32), ("dim", ctypes.c_int32), ("dtype", ctypes.c_int32),
                ("reserved", ctypes.c_int32)]


class _Batch(ctypes.Structure):
    _fields_ = [("num_queries", ctypes.c_int32), ("num_reqs", ctypes.c_int32),
                ("q_req", ctypes.c_void_p), ("q_pos", ctypes.c_void_p),
                ("block_table", ctypes.c_void_p), ("max_blocks", ctypes.c_int32),
                ("max_context", ctypes.c_int32), ("query_group", ctypes.c_int32),
                ("reserved", ctypes.c_int32)]


_lib = None


def load_library():
    """Load libdsa.so (raises DsaLibraryMissing if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise DsaLibraryMissing(
            "libdsa.so not found at %s; build it with `python -m sparse_attention_06_b200.build`" % LIB_PATH)
    lib = ctypes.CDLL(LIB_PATH)
    P, I32, I64, F = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_float
    PC, PB = ctypes.POINTER(_PagedCache), ctypes.POINTER(_Batch)
    sig = {
        "dsa_indexer_scores": [P, I32, P, I32, I32, P, PC, PB, P, I64, P, P],
        "dsa_topk_select": [P, I64, P, I32, I32, P, P, P],
        "dsa_indexer_topk": [P, I32, P, I32, I32, P, PC, PB, I32, P, I64, P, P, ctypes.c_size_t, P],
        "dsa_sparse_mla_decode": [P, I32, I32, I32, I32, PC, PB, P, I32, F, P, P, P, ctypes.c_size_t, P],
        "dsa_sparse_mla_prefill": [P, I32, I32, I32, I32, PC, PB, P, I32, F, P, P, P, ctypes.c_size_t, P],
        "dsa_sparse_mla_decode_noalloc": [P, I32, I32, I32, I32, PC, PB, P, I32, F, P, P, P],
        "dsa_get_device_error": [ctypes.POINTER(I32), P],
        "dsa_clear_device_error": [P],
        "dsa_selftest_bounded_wait": [I64, P],
        "dsa_selftest_gather_rate": [PC, P, I32, I32, P, P],
    }
    for name, args in sig.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = ctypes.c_int
    lib.dsa_mla_workspace_size.argtypes = [I32, I32, I32, I32]
    lib.dsa_mla_workspace_size.restype = ctypes.c_size_t
    lib.dsa_indexer_topk_workspace_size.argtypes = [I32]
    lib.dsa_indexer_topk_workspace_size.restype = ctypes.c_size_t
    lib.dsa_status_string.argtypes = [ctypes.c_int]
    lib.dsa_status_string.restype = ctypes.c_char_p
    lib.dsa_last_error_message.restype = ctypes.c_char_p
    lib.dsa_abi_version.restype = I32
    lib.dsa_kernel_launch_count.restype = I64
    _lib = lib
    return lib


def _check(status: int):
    if status != DSA_OK:
        lib = load_library()
        msg = (lib.dsa_last_error_message() or b"").decode() or lib.dsa_status_string(status).decode()
        raise DsaError(status, msg)


def _stream(stream) -> Optional[int]:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _dev_ptr(t: Optional[torch.Tensor], what: str):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("%s must be a CUDA tensor" % what)
    if not t.is_contiguous():
        raise ValueError("%s must be contiguous" % what)
    return t.data_ptr()


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return DSA_F32
    if t.dtype == torch.bfloat16:
        return DSA_BF16
    if t.dtype in (torch.uint8, torch.float8_e4m3fn):
        return DSA_E4M3
    raise ValueError("unsupported dtype %s" % t.dtype)


@dataclasses.dataclass
class PagedCache:
    """A paged per-token cache: data [num_blocks, block_size, dim] (f32 / bf16 / e4m3 codes as
    uint8), scale [num_blocks, block_size] f32 for e4m3."""
    data: torch.Tensor
    scale: Optional[torch.Tensor] = None

    def _c(self) -> _PagedCache:
        nb, bs, dim = self.data.shape
        return _PagedCache(_dev_ptr(self.data, "cache data"), _dev_ptr(self.scale, "cache scale"),
                           nb, bs, dim, _dtype_code(self.data), 0)


@dataclasses.dataclass
class Batch:
    """Queries of one call: q_req [T], q_pos [T] and block_table [B, max_blocks] int32 CUDA
    tensors; max_context bounds q_pos + 1 (host int); query_group as in dsa.h."""
    q_req: torch.Tensor
    q_pos: torch.Tensor
    block_table: torch.Tensor
    max_context: int
    query_group: int = 1

    def _c(self) -> _Batch:
        for n in ("q_req", "q_pos", "block_table"):
            if getattr(self, n).dtype != torch.int32:
                raise ValueError("%s must be int32" % n)
        B, mb = self.block_table.shape
        return _Batch(self.q_req.numel(), B, _dev_ptr(self.q_req, "q_req"), _dev_ptr(self.q_pos, "q_pos"),
                      _dev_ptr(self.block_table, "block_table"), mb, int(self.max_context),
                      int(self.query_group), 0)


def dsa_indexer_scores(q, w, keys: PagedCache, batch: Batch, scores, stream=None, q_scale=None, key_hist=None):
    """scores[t, s] = sum_h w[t,h] ReLU(qhat[t,h] . khat[s]) for s <= q_pos[t] (include/dsa.h);
    e4m3 queries (uint8 codes) come with q_scale [T, Hi] f32; key_hist [T, 4096] int32/uint32
    (optional) receives the scores' order-key digit counts."""
    lib = load_library()
    T, Hi, Di = q.shape
    kc, bc = keys._c(), batch._c()
    _check(lib.dsa_indexer_scores(_dev_ptr(q, "q"), _dtype_code(q), _dev_ptr(q_scale, "q_scale"), Hi, Di,
                                  _dev_ptr(w, "w"), ctypes.byref(kc), ctypes.byref(bc), _dev_ptr(scores, "scores"),
                                  scores.shape[1], _dev_ptr(key_hist, "key_hist"), _stream(stream)))
    return scores


def dsa_topk_select(scores, q_pos, k, idx, stream=None, key_hist=None):
    """idx[t] = the k best positions of scores[t, :q_pos[t]+1], ascending, -1 padded; key_hist
    (optional) places the threshold and is left zeroed (include/dsa.h)."""
    lib = load_library()
    _check(lib.dsa_topk_select(_dev_ptr(scores, "scores"), scores.shape[1], _dev_ptr(q_pos, "q_pos"),
                               q_pos.numel(), k, _dev_ptr(idx, "idx"), _dev_ptr(key_hist, "key_hist"),
                               _stream(stream)))
    return idx


def dsa_indexer_topk(q, w, keys: PagedCache, batch: Batch, k, scores, idx, stream=None, q_scale=None,
                     workspace=None):
    """Indexer scores fused with the top-K selection; workspace (optional, zero-filled before its
    first use, left zero-filled) holds the order-key digit histograms (include/dsa.h)."""
    lib = load_library()
    T, Hi, Di = q.shape
    kc, bc = keys._c(), batch._c()
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check(lib.dsa_indexer_topk(_dev_ptr(q, "q"), _dtype_code(q), _dev_ptr(q_scale, "q_scale"), Hi, Di,
                                _dev_ptr(w, "w"), ctypes.byref(kc), ctypes.byref(bc), k, _dev_ptr(scores, "scores"),
                                scores.shape[1], _dev_ptr(idx, "idx"), _dev_ptr(workspace, "workspace"), ws_bytes,
                                _stream(stream)))
    return idx


def dsa_indexer_topk_workspace_size(num_queries) -> int:
    return int(load_library().dsa_indexer_topk_workspace_size(num_queries))


def _mla(fn_name, q, latent: PagedCache, batch: Batch, idx, softmax_scale, out, lse, workspace, stream, k=None):
    lib = load_library()
    T, H, dqk = q.shape
    d_v = out.shape[-1]
    lc, bc = latent._c(), batch._c()
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    if k is None:
        k = idx.shape[1] if idx is not None else int(batch.max_context)
    _check(getattr(lib, fn_name)(_dev_ptr(q, "q"), _dtype_code(q), H, d_v, dqk - d_v, ctypes.byref(lc),
                                 ctypes.byref(bc), _dev_ptr(idx, "idx"), int(k), float(softmax_scale),
                                 _dev_ptr(out, "out"), _dev_ptr(lse, "lse"), _dev_ptr(workspace, "workspace"),
                                 ws_bytes, _stream(stream)))
    return out


def dsa_sparse_mla_decode(q, latent: PagedCache, batch: Batch, idx, softmax_scale, out, lse=None,
                          workspace=None, stream=None, k=None):
    """Sparse MQA-mode MLA over the selected latent rows, split-K across CTAs (include/dsa.h).
    ``idx=None`` is the dense case: every visible position, with k (default max_context) rows."""
    return _mla("dsa_sparse_mla_decode", q, latent, batch, idx, softmax_scale, out, lse, workspace, stream, k)


def dsa_sparse_mla_prefill(q, latent: PagedCache, batch: Batch, idx, softmax_scale, out, lse=None,
                           workspace=None, stream=None, k=None):
    return _mla("dsa_sparse_mla_prefill", q, latent, batch, idx, softmax_scale, out, lse, workspace, stream, k)


def dsa_sparse_mla_decode_noalloc(q, latent: PagedCache, batch: Batch, idx, softmax_scale, out, lse=None,
                                  stream=None):
    """dsa_sparse_mla_decode for callers that cannot allocate device memory: the split partials
    live in the library's fixed 32 MiB device scratch (see include/dsa.h)."""
    lib = load_library()
    T, H, dqk = q.shape
    d_v = out.shape[-1]
    lc, bc = latent._c(), batch._c()
    _check(lib.dsa_sparse_mla_decode_noalloc(_dev_ptr(q, "q"), _dtype_code(q), H, d_v, dqk - d_v,
                                             ctypes.byref(lc), ctypes.byref(bc), _dev_ptr(idx, "idx"),
                                             idx.shape[1], float(softmax_scale), _dev_ptr(out, "out"),
                                             _dev_ptr(lse, "lse"), _stream(stream)))
    return out


def dsa_mla_workspace_size(num_queries, H, d_v, k) -> int:
    return int(load_library().dsa_mla_workspace_size(num_queries, H, d_v, k))


def dsa_get_device_error(stream=None) -> int:
    """Synchronises the stream and returns the device error word (0 = no fault)."""
    code = ctypes.c_int32(0)
    st = load_library().dsa_get_device_error(ctypes.byref(code), _stream(stream))
    if st not in (DSA_OK, DSA_ERR_DEVICE_FAULT):
        _check(st)
    return int(code.value)


def dsa_kernel_launch_count() -> int:
    """Kernels the library has enqueued in this process so far."""
    return int(load_library().dsa_kernel_launch_count())


def dsa_selftest_bounded_wait(limit_cycles, stream=None):
    """Diagnostic: a kernel whose bounded wait on a phase that never completes gives up after
    ``limit_cycles`` SM cycles and sets DEVERR_TIMEOUT (include/dsa.h)."""
    _check(load_library().dsa_selftest_bounded_wait(int(limit_cycles), _stream(stream)))


def dsa_selftest_gather_rate(latent: PagedCache, rows, tiles_per_cta, num_ctas, cycles, stream=None):
    """Diagnostic: gathers latent pool rows with the sparse MLA's TMA pattern and nothing else;
    rows: int32 [num_ctas * tiles_per_cta * 64] pool row indices; cycles: int64 [num_ctas]
    receives each CTA's SM cycles (include/dsa.h)."""
    if rows.dtype != torch.int32 or rows.numel() < num_ctas * tiles_per_cta * 64:
        raise ValueError("rows must be int32 with num_ctas * tiles_per_cta * 64 entries")
    if cycles.dtype != torch.int64 or cycles.numel() < num_ctas:
        raise ValueError("cycles must be int64 with num_ctas entries")
    lc = latent._c()
    _check(load_library().dsa_selftest_gather_rate(ctypes.byref(lc), _dev_ptr(rows, "rows"), int(tiles_per_cta),
                                                   int(num_ctas), _dev_ptr(cycles, "cycles"), _stream(stream)))
    return cycles


def dsa_clear_device_error(stream=None):
    _check(load_library().dsa_clear_device_error(_stream(stream)))
