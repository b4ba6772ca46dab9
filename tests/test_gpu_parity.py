"""GPU parity of the CUDA path against the fp64 oracle at sizes the oracle finishes in seconds:
several tiles, ragged tails, dense (n <= K) and sparse queries, bf16 and e4m3 keys, the tiny fp32
layer, and the device error word.  All calls go through the C ABI."""
import math

import numpy as np
import pytest
import torch

import dsa_inputs as di
import oracle
import sparse_attention_06_b200 as dsa
from _parity import TOL, cache_and_batch, check_mla, check_topk, key_digit_hist, parity_case, run_gpu, subset_cpu, to_dev

pytestmark = pytest.mark.gpu


def _spec(lens, key_dtype="bf16", k=2048, **kw):
    return di.Spec("t", lens=lens, q_req=list(range(len(lens))), q_pos=[L - 1 for L in lens],
                   key_dtype=key_dtype, k=k, **kw)


def test_tiny_fp32_layer():
    x = to_dev(di.generate(di.tiny(), "cpu"))
    r = parity_case(x, kind="f32")
    assert r["overlap"] == 1.0


@pytest.mark.parametrize("key_dtype", ["bf16", "e4m3"])
def test_decode_ragged_batch(key_dtype):
    # request 0 is dense (n <= K), the others span several 128-key tiles with ragged tails
    spec = _spec([300, 2049, 2100, 4133, 64], key_dtype=key_dtype, seed=11)
    x = to_dev(di.generate(spec, "cpu"))
    parity_case(x, kind=key_dtype)


@pytest.mark.parametrize("lens", [[6000], [3000, 2500, 7000]])
def test_decode_few_queries_many_splits(lens):
    # one or three queries at K = 2048: the rows of each query split across many CTAs (one 64-row
    # tile each), one unit per CTA with Q staged through shared memory, partials merged by the combine
    spec = _spec(lens, seed=15)
    x = to_dev(di.generate(spec, "cpu"))
    parity_case(x, kind="bf16")


def test_decode_split_partials_and_combine():
    # 75 decode queries of one request: more (query, split) units than SMs, so the splits leave
    # partials in the workspace and the combine kernel merges them
    ctx, n = 2200, 75
    spec = di.Spec("many", lens=[ctx], q_req=[0] * n, q_pos=[ctx - n + i for i in range(n)], seed=16)
    x = to_dev(di.generate(spec, "cpu"))
    assert dsa.dsa_mla_workspace_size(spec.T, spec.H, spec.d_v, spec.k) > 0
    parity_case(x, queries=range(0, n, 7), kind="bf16")  # the oracle on every 7th query


def test_decode_small_k_many_tiles():
    spec = _spec([1000, 777], k=100, seed=12)
    x = to_dev(di.generate(spec, "cpu"))
    parity_case(x, kind="bf16")


@pytest.mark.parametrize("entry,group", [("decode", 1), ("prefill", 4)])
def test_e4m3_queries_with_e4m3_keys(entry, group):
    # fp8 indexer queries with a per-(query, head) scale and fp8 keys: one e4m3 x e4m3 product per
    # key tile; one query per tile (decode) and four queries of one request per tile (prefill)
    if group == 1:
        spec = _spec([300, 2049, 4133, 9000, 130], key_dtype="e4m3", q_idx_dtype="e4m3", seed=51)
    else:
        ctx, chunk = 2990, 64
        spec = di.Spec("pq8", lens=[ctx + chunk], q_req=[0] * chunk, q_pos=[ctx + t for t in range(chunk)],
                       key_dtype="e4m3", q_idx_dtype="e4m3", query_group=4, seed=53)
    x = to_dev(di.generate(spec, "cpu"))
    assert x["q_idx"].dtype == torch.uint8 and x["q_idx_scale"].shape == (spec.T, 64)
    parity_case(x, kind="e4m3", mla_entry=entry)


@pytest.mark.parametrize("key_dtype", ["bf16", "e4m3"])
@pytest.mark.parametrize("magnitude", ["huge_and_tiny_heads", "all_tiny"])
def test_indexer_queries_of_any_bf16_magnitude(key_dtype, magnitude):
    # bf16 indexer queries far outside the f16 range: heads scaled up to 1e30 and down to 1e-30
    # (whose products overflow or vanish in f16), then every head around 2^-100; the e4m3-key path
    # carries each head at its own power-of-two scale, the bf16 path multiplies as stored
    spec = _spec([3000, 700, 2100], key_dtype=key_dtype, seed=52)
    x = di.generate(spec, "cpu")
    if magnitude == "huge_and_tiny_heads":
        mult = torch.tensor([1e30, 1e-30, 3e5, 1e-6, 1.0, 7e12, 2.0 ** -20, 1e20] * 8)
    else:
        mult = 2.0 ** (-100.0 + torch.arange(64).float() % 8)
    x["q_idx"] = (x["q_idx"].float() * mult[None, :, None]).to(torch.bfloat16)
    assert torch.isfinite(x["q_idx"].float()).all()
    parity_case(to_dev(x), kind=key_dtype)


@pytest.mark.parametrize("entry", ["decode", "prefill"])
def test_prefill_chunk_e4m3(entry):
    ctx, chunk = 1990, 96  # queries straddle the dense/sparse boundary at K = 2048
    spec = di.Spec("p", lens=[ctx + chunk], q_req=[0] * chunk, q_pos=[ctx + t for t in range(chunk)],
                   key_dtype="e4m3", query_group=4, seed=13)
    x = to_dev(di.generate(spec, "cpu"))
    parity_case(x, kind="e4m3", mla_entry=entry)


def test_prefill_chunk_bf16_two_requests():
    # two requests, 8 queries each, in groups of 4
    spec = di.Spec("p2", lens=[3000, 2500], q_req=[0] * 8 + [1] * 8,
                   q_pos=[2992 + t for t in range(8)] + [2492 + t for t in range(8)],
                   query_group=4, seed=14)
    x = to_dev(di.generate(spec, "cpu"))
    parity_case(x, kind="bf16", mla_entry="prefill")


# ---------------------------------------------------------------------------------------------
# standalone selection
# ---------------------------------------------------------------------------------------------

HIST_MODE = "none"  # set by test_topk_edge_cases_with_histograms


def _topk_gpu(scores, qpos, k, hist_mode=None):
    """The selection on the GPU.  hist_mode: "none" (threshold from a sample), "exact" (the rows'
    order-key digit histogram, as the indexer builds it), "garbage" (a histogram that does not
    match the scores): the result must be the same in every mode, and any histogram given must
    be zero afterwards."""
    mode = hist_mode or HIST_MODE
    s = scores.cuda()
    qp = torch.tensor(qpos, dtype=torch.int32, device="cuda")
    idx = torch.empty((len(qpos), k), dtype=torch.int32, device="cuda")
    hist = None
    if mode == "exact":
        hist = key_digit_hist(scores, qpos).cuda()
    elif mode == "garbage":
        g = torch.Generator().manual_seed(len(qpos) * 7919 + k)
        hist = torch.randint(0, 50, (len(qpos), 4096), generator=g, dtype=torch.int32).cuda()
    dsa.dsa_clear_device_error()
    dsa.dsa_topk_select(s, qp, k, idx, key_hist=hist)
    err = dsa.dsa_get_device_error()
    if hist is not None:
        assert int(hist.abs().sum()) == 0, "histogram left dirty"
    return idx.cpu(), err


def test_topk_planted_tail_long_rows():
    lens = [202752, 131072, 4096, 2049, 2048, 100]
    ld = 202752
    s = di.planted_scores(len(lens), ld, lens, seed=21)
    idx, err = _topk_gpu(s, [L - 1 for L in lens], 2048)
    assert err == 0
    check_topk(idx, s, [L - 1 for L in lens], 2048)


def test_topk_ties_and_signed_zeros():
    g = torch.Generator().manual_seed(5)
    T, ld = 6, 5000
    s = torch.randint(-3, 4, (T, ld), generator=g).float()     # heavy ties
    s[1] = 0.0
    s[1, ::2] = -0.0                                           # +0 / -0 mix, all equal
    s[2] = 7.5                                                 # all equal
    s[3, :] = torch.arange(ld).float() * 0                     # zeros
    s[4] = torch.randn(ld, generator=g).round(decimals=1)
    s[5] = -torch.arange(ld).float()                           # strictly decreasing
    qpos = [4999, 4999, 4000, 2500, 4999, 3000]
    for k in (1, 17, 2048, 4096):
        idx, err = _topk_gpu(s, qpos, k)
        assert err == 0
        check_topk(idx, s, qpos, k)
    idx, _ = _topk_gpu(s, qpos, 2048)
    assert idx[2].tolist() == list(range(2048))                # lower positions win the tie
    assert idx[5].tolist() == list(range(2048))


def test_topk_dense_boundary_and_padding():
    s = torch.randn(4, 3000)
    qpos = [0, 2046, 2047, 2048]      # n = 1, 2047, 2048 (dense) and 2049 (sparse)
    idx, err = _topk_gpu(s, qpos, 2048)
    assert err == 0
    assert idx[0, 0] == 0 and (idx[0, 1:] == -1).all()
    assert idx[1, :2047].tolist() == list(range(2047)) and idx[1, 2047] == -1
    assert idx[2].tolist() == list(range(2048))
    check_topk(idx, s, qpos, 2048)


def test_topk_cluster_shapes():
    # few rows (several CTAs per row), many rows (one CTA per row), take-all rows just below and
    # above the candidate capacity, a row stride that leaves most rows unaligned for vector loads
    g = torch.Generator().manual_seed(9)
    for T, ld, k in ((1, 32768, 2048), (1, 202752, 2048), (3, 9001, 2048), (40, 70000, 2048),
                     (160, 20000, 2048), (2, 8192, 2048), (5, 40001, 100), (1, 50000, 4096)):
        s = torch.randn(T, ld, generator=g) * 20 + 150
        qpos = [ld - 1 - (7 * t) % 1000 for t in range(T)]
        idx, err = _topk_gpu(s, qpos, k)
        assert err == 0
        check_topk(idx, s, qpos, k)


def test_topk_ties_straddle_slices():
    # the K-th score is shared by positions in every slice of a long row: the lowest positions win
    g = torch.Generator().manual_seed(10)
    n = 40000
    s = torch.randn(1, n, generator=g)
    perm = torch.randperm(n, generator=g)
    s[0, perm[:1000]] = 6.0
    s[0, perm[1000:4000]] = 5.0
    idx, err = _topk_gpu(s, [n - 1], 2048)
    assert err == 0
    check_topk(idx, s, [n - 1], 2048)
    fives = torch.sort(perm[1000:4000]).values[:1048]
    want = torch.sort(torch.cat([perm[:1000], fives])).values
    assert idx[0].tolist() == want.tolist()


def test_topk_skewed_and_equal_long_rows():
    g = torch.Generator().manual_seed(11)
    T, ld = 4, 120000
    s = torch.randn(T, ld, generator=g)
    s[0, :3000] += 10.0              # every selected score in the first slice
    s[1, -2500:] += 10.0             # ... in the last slice
    s[2] = 3.25                      # all equal: more ties than candidates fit
    s[3] = torch.randint(0, 3, (ld,), generator=g).float()  # three values, heavy ties
    qpos = [ld - 1, ld - 1, ld - 1, ld - 1]
    idx, err = _topk_gpu(s, qpos, 2048)
    assert err == 0
    check_topk(idx, s, qpos, 2048)
    assert idx[2].tolist() == list(range(2048))


def test_topk_small_tie_groups_in_last_bin():
    # scores on a coarse grid: the last radix bin of the K-th key holds a few keys, some equal,
    # and the K-th key may fall anywhere in such a group
    g = torch.Generator().manual_seed(12)
    for T, ld, grid in ((1, 32768, 2048.0), (1, 32768, 512.0), (4, 100000, 4096.0), (3, 9000, 256.0)):
        s = torch.round(torch.randn(T, ld, generator=g) * grid) / grid
        qpos = [ld - 1 - 13 * t for t in range(T)]
        for k in (2048, 1999):
            idx, err = _topk_gpu(s, qpos, k)
            assert err == 0
            check_topk(idx, s, qpos, k)


def test_topk_threshold_from_a_misleading_sample():
    # the strided sample (8-score chunks at multiples of n / 512) sees only large scores, so its
    # threshold leaves fewer than K candidates and the selection falls back to its exact path
    g = torch.Generator().manual_seed(13)
    n = 32768
    s = torch.randn(1, n, generator=g)
    pos = torch.arange(512).repeat_interleave(8) * (n // 512) + torch.arange(8).repeat(512)
    s[0, pos] = 10.0 + torch.rand(pos.numel(), generator=g)
    for k in (2048, 1000):
        idx, err = _topk_gpu(s, [n - 1], k)
        assert err == 0
        check_topk(idx, s, [n - 1], k)


def test_topk_nan_in_long_row():
    s = torch.randn(2, 100000)
    s[1, 77777] = float("nan")
    idx, err = _topk_gpu(s, [99999, 99999], 2048)
    assert err & dsa.DEVERR_NAN_SCORE
    check_topk(idx[:1], s[:1], [99999], 2048)


def test_topk_nan_sets_error_word():
    s = torch.randn(1, 5000)
    s[0, 77] = float("nan")
    idx, err = _topk_gpu(s, [4999], 2048)
    assert err & dsa.DEVERR_NAN_SCORE


# ---------------------------------------------------------------------------------------------
# device-detected faults: flagged, never trapped
# ---------------------------------------------------------------------------------------------

def test_bad_block_id_and_bad_index_flagged():
    spec = _spec([500], k=64, seed=31)
    x = to_dev(di.generate(spec, "cpu"))
    bt = x["block_table"].clone()
    bt[0, 3] = x["num_blocks"] + 5          # outside the pool
    keys = dsa.PagedCache(x["key_pool"], None)
    batch = dsa.Batch(x["q_req"], x["q_pos"], bt, 500)
    scores = torch.zeros((1, 500), dtype=torch.float32, device="cuda")
    dsa.dsa_clear_device_error()
    dsa.dsa_indexer_scores(x["q_idx"], x["w"], keys, batch, scores)
    assert dsa.dsa_get_device_error() & dsa.DEVERR_BLOCK_ID
    # a selected index beyond q_pos
    batch = dsa.Batch(x["q_req"], x["q_pos"], x["block_table"], 500)
    idx = torch.full((1, 64), -1, dtype=torch.int32, device="cuda")
    idx[0, 0] = 10
    idx[0, 1] = 600
    out = torch.empty((1, spec.H, spec.d_v), dtype=torch.bfloat16, device="cuda")
    dsa.dsa_clear_device_error()
    ws_bytes = dsa.dsa_mla_workspace_size(1, spec.H, spec.d_v, 64)
    ws = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device="cuda") if ws_bytes else None
    dsa.dsa_sparse_mla_decode(x["q_mla"], dsa.PagedCache(x["latent_pool"]), batch, idx, spec.scale, out,
                              None, ws)
    assert dsa.dsa_get_device_error() & dsa.DEVERR_INDEX
    # the valid row still gives the single-row closed form: O = V of row 10
    flat = x["latent_pool"].view(-1, spec.dqk)
    row = flat[int(x["block_table"][0, 0]) * 64 + 10, :spec.d_v].float()
    assert torch.allclose(out[0].float(), row.expand(spec.H, -1), atol=1e-2)
    dsa.dsa_clear_device_error()
    assert dsa.dsa_get_device_error() == 0


# ---------------------------------------------------------------------------------------------
# bounded waits: a wait that runs out sets the timeout bit and the kernel returns
# ---------------------------------------------------------------------------------------------

def test_bounded_wait_runs_out_and_context_stays_usable():
    dsa.dsa_clear_device_error()
    dsa.dsa_selftest_bounded_wait(2_000_000)  # about 1 ms of SM cycles; nothing completes the phase
    err = dsa.dsa_get_device_error()
    assert err & dsa.DEVERR_TIMEOUT
    dsa.dsa_clear_device_error()
    assert dsa.dsa_get_device_error() == 0
    # the context is still usable: a small layer passes parity afterwards
    spec = _spec([2300], seed=33)
    x = to_dev(di.generate(spec, "cpu"))
    parity_case(x, kind="bf16")


def test_gather_rate_diagnostic():
    # the sparse MLA's row gathers alone: every CTA reports its cycles, the implied rate is a
    # plausible number of bytes per SM cycle, and a row index outside the pool is flagged
    # (and read as zeros) without stopping the kernel
    g = torch.Generator().manual_seed(61)
    nblk, ctas, tiles = 40, 4, 8
    pool = torch.randn(nblk, 64, 576, generator=g).to(torch.bfloat16).cuda()
    lat = dsa.PagedCache(pool)
    rows = torch.randint(0, nblk * 64, (ctas * tiles * 64,), generator=g, dtype=torch.int32).cuda()
    cycles = torch.zeros(ctas, dtype=torch.int64, device="cuda")
    dsa.dsa_clear_device_error()
    dsa.dsa_selftest_gather_rate(lat, rows, tiles, ctas, cycles)
    assert dsa.dsa_get_device_error() == 0
    c = cycles.cpu()
    assert (c > 0).all()
    rate = tiles * 64 * 1152 / c.double()  # bytes per SM cycle of each CTA
    assert ((rate > 1.0) & (rate < 256.0)).all(), rate
    rows[5] = -1
    rows[77] = nblk * 64
    dsa.dsa_selftest_gather_rate(lat, rows, tiles, ctas, cycles)
    assert dsa.dsa_get_device_error() == dsa.DEVERR_INDEX
    assert (cycles.cpu() > 0).all()
    dsa.dsa_clear_device_error()
    with pytest.raises(dsa.DsaError):
        dsa.dsa_selftest_gather_rate(lat, rows, 0, ctas, cycles)


# ---------------------------------------------------------------------------------------------
# the dense case and IndexShare
# ---------------------------------------------------------------------------------------------

@pytest.mark.parametrize("entry", ["decode", "prefill"])
def test_dense_case_without_selection(entry):
    # every query sees at most K positions, so the method keeps them all: sparse MLA with no
    # selection (idx None) over the visible positions equals the oracle's attention over all of
    # them, and, bit for bit, the sparse path whose selection is then every position
    lens = [1500, 2048, 700, 64, 1999, 130]
    spec = _spec(lens, seed=17)
    x = to_dev(di.generate(spec, "cpu"))
    g = run_gpu(x, entry)
    assert g["err"] == 0
    keys, lat, batch, max_ctx = cache_and_batch(x)
    out = torch.full_like(g["out"], float("nan"))
    lse = torch.full_like(g["lse"], float("nan"))
    ws_bytes = dsa.dsa_mla_workspace_size(spec.T, spec.H, spec.d_v, spec.k)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device="cuda") if ws_bytes else None
    fn = dsa.dsa_sparse_mla_decode if entry == "decode" else dsa.dsa_sparse_mla_prefill
    dsa.dsa_clear_device_error()
    fn(x["q_mla"], lat, batch, None, spec.scale, out, lse, ws, k=spec.k)
    assert dsa.dsa_get_device_error() == 0
    assert torch.equal(out, g["out"]) and torch.equal(lse, g["lse"])
    j = np.arange(spec.k)[None, :]
    n = np.array(lens)[:, None]
    idx_all = np.where(j < n, j, -1).astype(np.int32)
    sub = subset_cpu(x, list(range(spec.T)))
    ora_out, ora_lse = oracle.sparse_mla(sub["q_mla"], sub["latent_pool"], sub["block_table"], sub["q_req"],
                                         idx_all, spec.d_v, spec.scale)
    check_mla(out.float().cpu(), lse.cpu(), ora_out, ora_lse, TOL["bf16"])


def test_dense_case_needs_k_covering_the_context():
    spec = _spec([3000], seed=19)
    x = to_dev(di.generate(spec, "cpu"))
    keys, lat, batch, max_ctx = cache_and_batch(x)
    out = torch.empty((1, spec.H, spec.d_v), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(dsa.DsaError) as e:
        dsa.dsa_sparse_mla_decode(x["q_mla"], lat, batch, None, spec.scale, out, k=2048)
    assert e.value.status == dsa.DSA_ERR_INVALID_ARG


def test_indexshare_layers_reuse_the_selection():
    # one full layer selects; the group's other layers (own queries and latent caches, same
    # requests and paging) attend over the cached selection
    spec = di.Spec("share", lens=[5000, 3000, 2100, 9000], q_req=[0, 1, 2, 3], q_pos=[4999, 2999, 2099, 8999],
                   share_layers=3, seed=18)
    x = to_dev(di.generate(spec, "cpu"))
    g = run_gpu(x)
    assert g["err"] == 0
    keys, lat, batch, max_ctx = cache_and_batch(x)
    ws_bytes = dsa.dsa_mla_workspace_size(spec.T, spec.H, spec.d_v, spec.k)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device="cuda") if ws_bytes else None
    sub = subset_cpu(x, list(range(spec.T)))
    assert len(x["shared"]) == 2
    for sh, sh_cpu in zip(x["shared"], sub["shared"]):
        out = torch.empty_like(g["out"])
        lse = torch.empty_like(g["lse"])
        dsa.dsa_clear_device_error()
        dsa.dsa_sparse_mla_decode(sh["q_mla"], dsa.PagedCache(sh["latent_pool"]), batch, g["idx"].cuda(),
                                  spec.scale, out, lse, ws)
        assert dsa.dsa_get_device_error() == 0
        ora_out, ora_lse = oracle.sparse_mla(sh_cpu["q_mla"], sh_cpu["latent_pool"], sub["block_table"],
                                             sub["q_req"], g["idx"].cpu(), spec.d_v, spec.scale)
        check_mla(out.float().cpu(), lse.cpu(), ora_out, ora_lse, TOL["bf16"])


@pytest.mark.parametrize("mode", ["exact", "garbage"])
def test_topk_edge_cases_with_histograms(mode):
    # every standalone selection case above again, with the threshold placed from a digit
    # histogram: the exact one the indexer builds, and one that does not describe the scores
    global HIST_MODE
    HIST_MODE = mode
    try:
        test_topk_planted_tail_long_rows()
        test_topk_ties_and_signed_zeros()
        test_topk_dense_boundary_and_padding()
        test_topk_cluster_shapes()
        test_topk_ties_straddle_slices()
        test_topk_skewed_and_equal_long_rows()
        test_topk_small_tie_groups_in_last_bin()
        test_topk_threshold_from_a_misleading_sample()
        test_topk_nan_in_long_row()
        test_topk_nan_sets_error_word()
    finally:
        HIST_MODE = "none"


def test_fused_indexer_topk_matches_unfused_and_reuses_workspace():
    # the fused call (histogram built by the indexer) against the two plain calls, twice in a row
    # on the same workspace; bf16 and e4m3 keys, several requests with ragged lengths
    for key_dtype, seed in (("bf16", 61), ("e4m3", 62)):
        spec = _spec([40000, 2049, 9000, 130000, 300], key_dtype=key_dtype, seed=seed)
        x = to_dev(di.generate(spec, "cpu"))
        keys, lat, batch, max_ctx = cache_and_batch(x)
        ld = (max_ctx + 3) // 4 * 4
        scores = torch.empty((spec.T, ld), dtype=torch.float32, device="cuda")
        ref = torch.empty((spec.T, spec.k), dtype=torch.int32, device="cuda")
        dsa.dsa_clear_device_error()
        dsa.dsa_indexer_topk(x["q_idx"], x["w"], keys, batch, spec.k, scores, ref)
        ws = torch.zeros(dsa.dsa_indexer_topk_workspace_size(spec.T) // 4, dtype=torch.int32, device="cuda")
        for _ in range(2):
            idx = torch.full_like(ref, -7)
            dsa.dsa_indexer_topk(x["q_idx"], x["w"], keys, batch, spec.k, scores, idx, workspace=ws)
            torch.cuda.synchronize()
            assert torch.equal(idx, ref)
            assert int(ws.abs().sum()) == 0
        assert dsa.dsa_get_device_error() == 0
        check_topk(ref.cpu(), scores.cpu(), [L - 1 for L in spec.lens], spec.k)


# ---------------------------------------------------------------------------------------------
# the GLM-5 attention shape: 64 heads, softmax scale 1/sqrt(256)
# ---------------------------------------------------------------------------------------------

@pytest.mark.parametrize("lens,entry", [
    ([6000], "decode"),                          # one query: 32 splits, one unit per CTA (staged Q)
    ([3000, 2500, 7000, 300], "decode"),         # few queries: splits and the combine kernel
    ([2100] * 80, "decode"),                     # more units than SMs: CTAs loop over units
    ([3000, 2500, 7000, 300], "prefill"),        # whole queries per CTA
])
def test_glm5_shape_64_heads(lens, entry):
    spec = di.Spec("glm5", lens=lens, q_req=list(range(len(lens))), q_pos=[L - 1 for L in lens], H=64,
                   scale=1.0 / math.sqrt(256.0), seed=71)
    x = to_dev(di.generate(spec, "cpu"))
    queries = None if len(lens) < 10 else list(range(0, len(lens), 9))
    parity_case(x, queries=queries, kind="bf16", mla_entry=entry)
