"""Helpers for the GPU parity tests: run the CUDA path through the binding, run the fp64 oracle on
the very same inputs, and compare with the stated tolerances.

Tolerances (written here once, used by every parity test):
  * indexer scores: |gpu - oracle| <= rtol * max(|oracle|, 1e-3 * max_s |oracle[t, s]|), with
    rtol 1e-3 for bf16 keys, 2e-2 for e4m3 keys and 1e-4 for the fp32 tiny layer (an f32 dot
    product of n = 32 terms is within n * 2^-24 * sum|q_i k_i| of exact; with cancellation up to
    ~50x that is 1e-4 of the score);
  * top-K positions: bit-exact against the oracle's selection applied to the GPU's own scores;
  * attention: max-abs <= 2e-2 and rel-L2 <= 1e-2 for bf16; 1e-4 / 1e-5 for the fp32 tiny layer;
    LSE: abs <= 2e-3 (bf16) or 1e-5 (fp32).
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
import sparse_attention_06_b200 as dsa

TOL = {
    "f32": dict(score_rtol=1e-4, mla_abs=1e-4, mla_rel=1e-5, lse_abs=1e-5),
    "bf16": dict(score_rtol=1e-3, mla_abs=2e-2, mla_rel=1e-2, lse_abs=2e-3),
    "e4m3": dict(score_rtol=2e-2, mla_abs=2e-2, mla_rel=1e-2, lse_abs=2e-3),
}


def to_dev(x, dev="cuda"):
    """The inputs dict with every tensor (also inside the IndexShare layers' list) on `dev`."""
    def mv(v):
        if isinstance(v, torch.Tensor):
            return v.to(dev)
        if isinstance(v, list):
            return [mv(e) for e in v]
        if isinstance(v, dict):
            return {k: mv(e) for k, e in v.items()}
        return v
    return {k: (mv(v) if k != "spec" else v) for k, v in x.items()}


def cache_and_batch(x):
    spec = x["spec"]
    keys = dsa.PagedCache(x["key_pool"], x.get("key_scale")) if "key_pool" in x else None
    lat = dsa.PagedCache(x["latent_pool"]) if "latent_pool" in x else None
    max_ctx = max(spec.q_pos) + 1
    batch = dsa.Batch(x["q_req"], x["q_pos"], x["block_table"], max_ctx, spec.query_group)
    return keys, lat, batch, max_ctx


def run_gpu(x, mla_entry="decode", fused=True):
    """Run indexer -> top-K -> sparse MLA through the C ABI on cuda tensors (by default the fused
    indexer-selection call with its histogram workspace, as the benchmark runs it; fused=False runs
    the two calls without a histogram).  Returns the device results; the histogram workspace must
    be all zeros again afterwards."""
    spec = x["spec"]
    keys, lat, batch, max_ctx = cache_and_batch(x)
    T = spec.T
    ld = (max_ctx + 3) // 4 * 4
    scores = torch.full((T, ld), float("nan"), dtype=torch.float32, device="cuda")
    idx = torch.empty((T, spec.k), dtype=torch.int32, device="cuda")
    dsa.dsa_clear_device_error()
    if fused:
        hist = torch.zeros(dsa.dsa_indexer_topk_workspace_size(T) // 4, dtype=torch.int32, device="cuda")
        dsa.dsa_indexer_topk(x["q_idx"], x["w"], keys, batch, spec.k, scores, idx, q_scale=x.get("q_idx_scale"),
                             workspace=hist)
        torch.cuda.synchronize()
        assert int(hist.abs().sum()) == 0, "the selection left its histogram workspace dirty"
    else:
        dsa.dsa_indexer_scores(x["q_idx"], x["w"], keys, batch, scores, q_scale=x.get("q_idx_scale"))
        dsa.dsa_topk_select(scores, x["q_pos"], spec.k, idx)
    out = torch.empty((T, spec.H, spec.d_v), dtype=x["q_mla"].dtype, device="cuda")
    lse = torch.empty((T, spec.H), dtype=torch.float32, device="cuda")
    ws_bytes = dsa.dsa_mla_workspace_size(T, spec.H, spec.d_v, spec.k)
    ws = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device="cuda") if ws_bytes else None
    fn = dsa.dsa_sparse_mla_decode if mla_entry == "decode" else dsa.dsa_sparse_mla_prefill
    fn(x["q_mla"], lat, batch, idx, spec.scale, out, lse, ws)
    err = dsa.dsa_get_device_error()
    torch.cuda.synchronize()
    return dict(scores=scores, idx=idx, out=out, lse=lse, err=err)


def parity_case(x, queries=None, kind="bf16", mla_entry="decode", e2e_min_overlap=0.999, topk_all_rows=False,
                fused=True):
    """Full parity of one workload ``x`` (tensors on cuda): GPU path vs the oracle on the queries
    listed (all by default).  With ``topk_all_rows`` the selection of every query (not only the
    listed ones) is checked bit-exactly against the oracle's selection from the GPU's own scores.
    Returns a dict of the measured errors."""
    spec = x["spec"]
    tol = TOL[kind]
    g = run_gpu(x, mla_entry, fused)
    assert g["err"] == 0, "device error word %d" % g["err"]
    if topk_all_rows:
        qpos_all = x["q_pos"].cpu().numpy()
        for r0 in range(0, spec.T, 64):  # rows in chunks: the f64 copy of all scores can be GBs
            r1 = min(spec.T, r0 + 64)
            check_topk(g["idx"][r0:r1].cpu(), g["scores"][r0:r1].cpu(), qpos_all[r0:r1], spec.k)
    qs = list(range(spec.T)) if queries is None else list(queries)
    sub = subset_cpu(x, qs)
    qpos = sub["q_pos"].numpy()
    ld = g["scores"].shape[1]
    ora_scores = oracle.indexer_scores(sub["q_idx"], sub["w"], sub["key_pool"], sub["key_scale"],
                                       sub["block_table"], sub["q_req"], sub["q_pos"], ld=ld,
                                       q_scale=sub.get("q_idx_scale"))
    qi = torch.tensor(qs, dtype=torch.long, device="cuda")
    gs = g["scores"][qi].cpu()
    gidx = g["idx"][qi].cpu()
    worst = check_scores(gs, ora_scores, qpos, tol["score_rtol"])
    check_topk(gidx, gs, qpos, spec.k)
    ora_out, ora_lse = oracle.sparse_mla(sub["q_mla"], sub["latent_pool"], sub["block_table"], sub["q_req"],
                                         gidx, spec.d_v, spec.scale)
    max_abs, rel_l2 = check_mla(g["out"][qi].float().cpu(), g["lse"][qi].cpu(), ora_out, ora_lse, tol)
    # end to end: the oracle's own selection (from its own scores) against the GPU's
    ora_idx = oracle.topk(ora_scores, qpos, spec.k)
    overlap = []
    for r in range(len(qs)):
        a = set(ora_idx[r][ora_idx[r] >= 0].tolist())
        b = set(gidx[r][gidx[r] >= 0].tolist())
        overlap.append(len(a & b) / max(1, len(a)))
    assert min(overlap) >= e2e_min_overlap, "end-to-end selection overlap %.5f" % min(overlap)
    return dict(score_rel=worst, mla_max_abs=max_abs, mla_rel_l2=rel_l2, overlap=min(overlap))


def subset_cpu(x, qs):
    import dsa_inputs as di
    return di.subset(x, qs)


def check_scores(gpu_scores, ora_scores, q_pos, rtol):
    """Element-wise score check with a per-row floor; returns the worst relative error."""
    worst = 0.0
    g = gpu_scores.double().numpy() if isinstance(gpu_scores, torch.Tensor) else gpu_scores
    for t in range(ora_scores.shape[0]):
        n = int(q_pos[t]) + 1
        o = ora_scores[t, :n]
        gg = g[t, :n]
        assert not np.isnan(gg).any(), "row %d has unwritten scores" % t
        floor = 1e-3 * np.abs(o).max() if n else 0.0
        denom = np.maximum(np.abs(o), floor)
        denom[denom == 0] = 1.0
        rel = np.abs(gg - o) / denom
        worst = max(worst, float(rel.max()))
        assert rel.max() <= rtol, "row %d: worst rel err %.3g > %.3g at s=%d" % (t, rel.max(), rtol, int(rel.argmax()))
    return worst


def check_topk(gpu_idx, gpu_scores, q_pos, k):
    """Bit-exact: the oracle's selection applied to the GPU's own scores."""
    ref = oracle.topk(gpu_scores.double().numpy(), np.asarray(q_pos, np.int32), k)
    got = gpu_idx.numpy()
    bad = np.where((ref != got).any(axis=1))[0]
    assert len(bad) == 0, "top-k mismatch in rows %s" % bad[:10].tolist()


def check_mla(gpu_out, gpu_lse, ora_out, ora_lse, tol):
    g = gpu_out.double().numpy()
    max_abs = float(np.abs(g - ora_out).max())
    rel_l2 = float(np.linalg.norm(g - ora_out) / max(np.linalg.norm(ora_out), 1e-300))
    assert max_abs <= tol["mla_abs"], "max-abs %.3g > %.3g" % (max_abs, tol["mla_abs"])
    assert rel_l2 <= tol["mla_rel"], "rel-L2 %.3g > %.3g" % (rel_l2, tol["mla_rel"])
    if gpu_lse is not None:
        lse_err = float(np.abs(gpu_lse.double().numpy() - ora_lse).max())
        assert lse_err <= tol["lse_abs"], "lse err %.3g" % lse_err
    return max_abs, rel_l2


def key_digit_hist(scores, q_pos):
    """Order-key digit histogram of each row's visible scores, as the indexer builds it for the
    selection (top 12 bits of the order key: larger score -> larger key, -0 as +0, NaN -> 0):
    int32 [T, 4096].  Only a hint for the selection's threshold; results never depend on it."""
    u = scores.contiguous().view(torch.int32).cpu().numpy().view(np.uint32)
    neg = (u & 0x80000000) != 0
    key = np.where(neg, ~u, u | 0x80000000).astype(np.uint32)
    key[u == 0x80000000] = 0x80000000
    nan = (u & 0x7FFFFFFF) > 0x7F800000
    key[nan] = 0
    out = np.zeros((u.shape[0], 4096), dtype=np.int32)
    for t in range(u.shape[0]):
        n = int(q_pos[t]) + 1
        out[t] = np.bincount(key[t, :n] >> 20, minlength=4096)
    return torch.from_numpy(out)
