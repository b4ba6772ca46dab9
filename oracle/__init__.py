"""fp64 CPU oracle for the DeepSeek Sparse Attention hot path.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the benchmark's
``cpu_baseline`` leg (and its ``--impl reference`` arm) may import this package.  It shares no
code with the CUDA path in ``sparse_attention_06_b200`` and imports nothing from it.

The arithmetic lives in ``dsa_oracle.c`` (plain C, double precision, OpenMP over independent key positions, queries and heads); this
module only compiles it with gcc and marshals numpy / torch CPU arrays into it.  Every function
states the passage it follows in the C source.  Pins of the oracle against values fixed by the
pages and by mathematics are in ``tests/test_oracle_pins.py``.

Parity status: the pages print no worked numeric example of scores, selections or attention
outputs, so no function here is pinned to a printed value; each one is pinned instead to brute
force on tiny inputs, closed forms and invariants (see the tests).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "dsa_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

# dtype codes understood by the C oracle
F32, BF16, E4M3 = 0, 1, 2


def build(force: bool = False) -> str:
    """Compile dsa_oracle.c into liboracle.so next to it (gcc -O2 -fopenmp)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp%d" % os.getpid()
        subprocess.check_call(
            ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", _SRC, "-o", tmp, "-lm"]
        )
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            P, I, L, D = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_double
            lib.oracle_indexer_scores.argtypes = [I, P, I, P, I, I, P, P, I, P, I, P, I, P, P, P, L, I]
            lib.oracle_topk.argtypes = [I, P, L, P, I, P, I]
            lib.oracle_sparse_mla.argtypes = [I, P, I, I, I, I, P, I, I, P, I, P, P, I, D, P, P, I]
            lib.oracle_e4m3_to_double.argtypes = [ctypes.c_uint8]
            lib.oracle_e4m3_to_double.restype = D
            lib.oracle_bf16_to_double.argtypes = [ctypes.c_uint16]
            lib.oracle_bf16_to_double.restype = D
            lib.oracle_max_threads.restype = I
            _lib = lib
    return _lib


def max_threads() -> int:
    return _load().oracle_max_threads()


def _raw(x):
    """Return (contiguous numpy array, dtype code) for a torch CPU tensor or numpy array.

    bf16 and e4m3 tensors are passed as their raw bits; the C side decodes them.
    """
    try:
        import torch
    except ImportError:  # pragma: no cover
        torch = None
    if torch is not None and isinstance(x, torch.Tensor):
        x = x.detach().cpu().contiguous()
        if x.dtype == torch.bfloat16:
            return x.view(torch.int16).numpy().view(np.uint16), BF16
        if x.dtype == torch.float8_e4m3fn:
            return x.view(torch.uint8).numpy(), E4M3
        if x.dtype == torch.float32:
            return x.numpy(), F32
        if x.dtype in (torch.int32,):
            return x.numpy(), None
        if x.dtype == torch.uint8:
            return x.numpy(), E4M3
        if x.dtype == torch.float64:
            return x.numpy(), None
        raise TypeError("unsupported tensor dtype %s" % x.dtype)
    x = np.ascontiguousarray(x)
    if x.dtype == np.float32:
        return x, F32
    return x, None


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def indexer_scores(q, w, key_pool, key_scale, block_table, q_req, q_pos, ld=None, nthreads=0, q_scale=None):
    """Lightning-indexer scores in fp64 (page "How GLM5.3 Sparse Attention Affects HBM Memory
    Usage", section "Lightning Indexer").

    q [T, Hi, Di] (f32/bf16, or e4m3 codes with q_scale [T, Hi] f32), w [T, Hi] f32,
    key_pool [num_blocks, block_size, Di] (f32/bf16/e4m3), key_scale [num_blocks, block_size] f32
    or None, block_table [B, max_blocks] i32, q_req [T] i32, q_pos [T] i32.  Returns float64
    [T, ld]; entries past q_pos[t] are NaN.
    """
    qa, qdt = _raw(q)
    wa, _ = _raw(w)
    ka, kdt = _raw(key_pool)
    T, Hi, Di = qa.shape
    nblk, bs, Dk = ka.shape
    assert Dk == Di and wa.shape == (T, Hi) and wa.dtype == np.float32
    if qdt == E4M3:
        qsa = np.ascontiguousarray(_raw(q_scale)[0], dtype=np.float32)
        assert qsa.shape == (T, Hi)
    else:
        qsa = np.zeros(1, np.float32)
    if kdt == E4M3:
        sa, _ = _raw(key_scale)
        sa = np.ascontiguousarray(sa, dtype=np.float32)
        assert sa.shape == (nblk, bs)
    else:
        sa = np.zeros(1, np.float32)
    bt = np.ascontiguousarray(_raw(block_table)[0], dtype=np.int32)
    qr = np.ascontiguousarray(_raw(q_req)[0], dtype=np.int32)
    qp = np.ascontiguousarray(_raw(q_pos)[0], dtype=np.int32)
    if ld is None:
        ld = int(qp.max()) + 1 if T else 1
    out = np.full((T, ld), np.nan, dtype=np.float64)
    _load().oracle_indexer_scores(
        T, _ptr(qa), qdt, _ptr(qsa), Hi, Di, _ptr(wa), _ptr(ka), kdt, _ptr(sa), bs, _ptr(bt), bt.shape[1],
        _ptr(qr), _ptr(qp), _ptr(out), ld, nthreads,
    )
    return out


def topk(scores, q_pos, k, nthreads=0):
    """Top-K positions per query, ties to the lower position, ascending, -1 padded (page "How
    GLM5.3 Sparse Attention Affects HBM Memory Usage", section "Lightning Indexer": a query that
    sees fewer than K positions keeps them all).

    scores: [T, ld] float64 or float32 (float32 is widened exactly); returns int32 [T, k].
    """
    s = np.ascontiguousarray(_raw(scores)[0], dtype=np.float64)
    qp = np.ascontiguousarray(_raw(q_pos)[0], dtype=np.int32)
    T, ld = s.shape
    idx = np.empty((T, k), dtype=np.int32)
    _load().oracle_topk(T, _ptr(s), ld, _ptr(qp), k, _ptr(idx), nthreads)
    return idx


def sparse_mla(q, latent_pool, block_table, q_req, idx, d_v, scale, nthreads=0):
    """Sparse MLA in MQA mode over the selected latent rows, fp64 (same page, sections
    "Sparse MLA" and "MLA Modifications": P = Q K^T over the 576-wide latent row, O = P V with V
    its first d_v dims).

    q [T, H, Dqk], latent_pool [num_blocks, block_size, Dqk], idx [T, K] i32 (-1 = unused).
    Returns (out float64 [T, H, d_v], lse float64 [T, H]).
    """
    qa, qdt = _raw(q)
    la, ldt = _raw(latent_pool)
    T, H, Dqk = qa.shape
    nblk, bs, Dl = la.shape
    assert Dl == Dqk and 0 < d_v <= Dqk
    bt = np.ascontiguousarray(_raw(block_table)[0], dtype=np.int32)
    qr = np.ascontiguousarray(_raw(q_req)[0], dtype=np.int32)
    ix = np.ascontiguousarray(_raw(idx)[0], dtype=np.int32)
    K = ix.shape[1]
    out = np.empty((T, H, d_v), dtype=np.float64)
    lse = np.empty((T, H), dtype=np.float64)
    _load().oracle_sparse_mla(
        T, _ptr(qa), qdt, H, Dqk, d_v, _ptr(la), ldt, bs, _ptr(bt), bt.shape[1], _ptr(qr),
        _ptr(ix), K, float(scale), _ptr(out), _ptr(lse), nthreads,
    )
    return out, lse


def e4m3_to_double(code: int) -> float:
    return _load().oracle_e4m3_to_double(code)


def bf16_to_double(bits: int) -> float:
    return _load().oracle_bf16_to_double(bits)
