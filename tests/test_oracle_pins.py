"""Pins of the fp64 oracle against things other than itself: hand-worked examples from the
definitions (tests/golden), closed forms, invariants, brute force on tiny inputs, and special
cases that reduce to a library routine.  Each test is chosen so that a plausible slip in the
oracle (a dropped term, ReLU in the wrong place, a wrong tie direction, V taken over the RoPE
dims, a paging index error, a missing scale) fails at least one of them."""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch

import dsa_inputs as di
import oracle

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _single_block_table(n_rows, block=64):
    nb = -(-n_rows // block)
    return torch.arange(nb, dtype=torch.int32).view(1, nb), nb


def _pool_from_rows(rows, block=64):
    """Lay logical rows [n, D] into an identity-paged pool [nb, block, D] (zero-filled tail)."""
    n, D = rows.shape
    nb = -(-n // block)
    pool = torch.zeros((nb * block, D), dtype=rows.dtype)
    pool[:n] = rows
    return pool.view(nb, block, D)


# ------------------------------------------------------------------------------------------
# number formats: the decoders against torch's own conversions (a library routine)
# ------------------------------------------------------------------------------------------

def test_e4m3_decoder_matches_torch_all_codes():
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    for c in range(256):
        got = oracle.e4m3_to_double(c)
        if math.isnan(ref[c]):
            assert math.isnan(got), c
        else:
            assert got == ref[c], (c, got, ref[c])
    # spot values fixed by the format: max normal 448, min subnormal 2^-9
    assert oracle.e4m3_to_double(0x7E) == 448.0
    assert oracle.e4m3_to_double(0x01) == 2.0 ** -9


def test_bf16_decoder_matches_torch_sample():
    g = torch.Generator().manual_seed(3)
    bits = torch.randint(0, 1 << 16, (4096,), generator=g, dtype=torch.int32)
    bits = bits[((bits >> 7) & 0xFF) != 0xFF]  # skip inf/nan exponents
    ref = bits.to(torch.int16).view(torch.bfloat16).to(torch.float64).numpy()
    got = np.array([oracle.bf16_to_double(int(b) & 0xFFFF) for b in bits.tolist()])
    assert np.array_equal(got, ref)


# ------------------------------------------------------------------------------------------
# indexer
# ------------------------------------------------------------------------------------------

def test_indexer_hand_example():
    g = json.load(open(os.path.join(GOLD, "indexer_hand.json")))
    q = torch.tensor([g["q"]], dtype=torch.float32)
    w = torch.tensor([g["w"]], dtype=torch.float32)
    pool = _pool_from_rows(torch.tensor(g["keys"], dtype=torch.float32))
    bt, _ = _single_block_table(3)
    s = oracle.indexer_scores(q, w, pool, None, bt, torch.tensor([0], dtype=torch.int32),
                              torch.tensor([2], dtype=torch.int32))
    assert s[0].tolist() == g["scores"]
    assert oracle.topk(s, torch.tensor([2], dtype=torch.int32), 2)[0].tolist() == g["topk_k2"]
    assert oracle.topk(s, torch.tensor([2], dtype=torch.int32), 1)[0].tolist() == g["topk_k1"]


def test_indexer_hand_example_e4m3_scale():
    """The same hand example with keys stored as e4m3 codes and a per-token scale of 0.5: the
    codes hold 2x the keys (exactly representable), so the scores must be unchanged."""
    g = json.load(open(os.path.join(GOLD, "indexer_hand.json")))
    keys2 = torch.tensor(g["keys"], dtype=torch.float32) * 2.0
    codes = keys2.to(torch.float8_e4m3fn).view(torch.uint8)
    assert torch.equal(codes.view(torch.float8_e4m3fn).float(), keys2)
    pool = _pool_from_rows(codes)
    scale = torch.full((1, 64), 0.5, dtype=torch.float32)
    bt, _ = _single_block_table(3)
    s = oracle.indexer_scores(torch.tensor([g["q"]]), torch.tensor([g["w"]]), pool, scale, bt,
                              torch.tensor([0], dtype=torch.int32), torch.tensor([2], dtype=torch.int32))
    assert s[0].tolist() == g["scores"]


def test_indexer_single_head_reduces_to_matmul():
    """Hi = 1, w = 1 and keys chosen so every q.k > 0: the score is the plain product q k^T."""
    g = torch.Generator().manual_seed(5)
    Di, L = 16, 130
    q = torch.rand((1, 1, Di), generator=g) + 0.1
    keys = torch.rand((L, Di), generator=g) + 0.1
    pool = _pool_from_rows(keys)
    bt, _ = _single_block_table(L)
    s = oracle.indexer_scores(q, torch.ones((1, 1)), pool, None, bt, torch.tensor([0], dtype=torch.int32),
                              torch.tensor([L - 1], dtype=torch.int32))
    ref = (q[0].double() @ keys.double().T)[0].numpy()
    np.testing.assert_allclose(s[0], ref, rtol=1e-13)


def test_indexer_relu_is_per_head_and_weights_are_linear():
    """Linearity in w; ReLU applied to each head's logit (not to the weighted sum); homogeneity
    of degree 1 in a positive key scaling."""
    spec = di.tiny()
    x = di.generate(spec, "cpu", with_mla=False)
    args = (x["key_pool"], None, x["block_table"], x["q_req"], x["q_pos"])
    s = oracle.indexer_scores(x["q_idx"], x["w"], *args)
    w1 = torch.zeros_like(x["w"]); w1[:, 0] = 1.0
    w2 = x["w"] - w1
    s1 = oracle.indexer_scores(x["q_idx"], w1, *args)
    s2 = oracle.indexer_scores(x["q_idx"], w2, *args)
    np.testing.assert_allclose(s, s1 + s2, rtol=1e-12, atol=1e-12)
    # a single head with weight 1: score equals that head's ReLU'd logit, hence never negative
    assert (s1[0] >= 0).all()
    # flipping the sign of every query flips every logit: relu(x) + relu(-x) = |x|
    sn = oracle.indexer_scores(-x["q_idx"], w1, *args)
    L = spec.lens[0]
    rows = x["key_pool"].view(-1, spec.Di)[(x["block_table"][0].long().repeat_interleave(64) * 64
                                            + torch.arange(64).repeat(x["block_table"].shape[1]))[:L]]
    absdot = (x["q_idx"][0, 0].double() @ rows.double().T).abs().numpy()
    np.testing.assert_allclose(s1[0] + sn[0], absdot, rtol=1e-12, atol=1e-12)
    # keys scaled by 2 (exact in f32): scores double
    s2x = oracle.indexer_scores(x["q_idx"], x["w"], x["key_pool"] * 2, None, x["block_table"],
                                x["q_req"], x["q_pos"])
    np.testing.assert_allclose(s2x, 2 * s, rtol=1e-13)


def test_indexer_paging_invariance_and_causality():
    """Two different physical layouts of the same logical keys give identical scores; positions
    past q_pos are never written."""
    spec = di.tiny()
    x = di.generate(spec, "cpu", with_mla=False)
    bt = x["block_table"]
    pool = x["key_pool"]
    # build an alternative layout with the blocks in reverse physical order
    nb = pool.shape[0]
    perm = torch.arange(nb - 1, -1, -1)
    pool2 = pool[perm.argsort()]
    bt2 = bt.clone()
    valid = bt >= 0
    bt2[valid] = perm[bt[valid].long()].to(torch.int32)
    qp = torch.tensor([100], dtype=torch.int32)
    s1 = oracle.indexer_scores(x["q_idx"], x["w"], pool, None, bt, x["q_req"], qp, ld=256)
    s2 = oracle.indexer_scores(x["q_idx"], x["w"], pool2, None, bt2, x["q_req"], qp, ld=256)
    assert np.array_equal(s1, s2, equal_nan=True)
    assert np.isnan(s1[0, 101:]).all() and not np.isnan(s1[0, :101]).any()


# ------------------------------------------------------------------------------------------
# top-k
# ------------------------------------------------------------------------------------------

def _brute_topk(scores, n, K):
    """Enumerate every K-subset of 0..n-1 and return the unique one whose members all precede
    every non-member in the order (score desc, position asc)."""
    def before(a, b):
        return scores[a] > scores[b] or (scores[a] == scores[b] and a < b)
    found = []
    for sub in itertools.combinations(range(n), K):
        inside = set(sub)
        if all(before(a, b) for a in inside for b in range(n) if b not in inside):
            found.append(list(sub))
    assert len(found) == 1
    return found[0]


@pytest.mark.parametrize("seed", range(6))
def test_topk_brute_force_with_ties(seed):
    rng = np.random.default_rng(seed)
    n, K = 9, 4
    scores = rng.integers(0, 4, size=n).astype(np.float64)  # many ties
    scores[rng.integers(0, n)] = -0.0
    got = oracle.topk(scores[None, :], np.array([n - 1], np.int32), K)[0].tolist()
    assert got == _brute_topk(scores, n, K)


def test_topk_matches_library_lexsort_and_invariants():
    rng = np.random.default_rng(11)
    T, ld, K = 5, 700, 64
    scores = np.round(rng.normal(size=(T, ld)), 2)  # rounding forces ties
    qpos = np.array([699, 63, 64, 500, 0], np.int32)
    idx = oracle.topk(scores, qpos, K)
    for t in range(T):
        n = qpos[t] + 1
        sel = idx[t][idx[t] >= 0]
        assert len(sel) == min(n, K)
        assert (np.diff(sel) > 0).all()
        assert (idx[t][len(sel):] == -1).all()
        if n <= K:
            assert sel.tolist() == list(range(n))
            continue
        order = np.lexsort((np.arange(n), -scores[t, :n]))
        assert sorted(order[:K].tolist()) == sel.tolist()
        chosen = np.zeros(n, bool); chosen[sel] = True
        lo_sel = scores[t, :n][chosen].min()
        hi_rest = scores[t, :n][~chosen].max()
        assert lo_sel >= hi_rest
        if lo_sel == hi_rest:  # ties at the boundary: every chosen tie precedes every rejected one
            tie = scores[t, :n] == lo_sel
            assert np.where(tie & chosen)[0].max() < np.where(tie & ~chosen)[0].min()


def test_topk_lower_index_wins_all_equal():
    scores = np.zeros((1, 50))
    idx = oracle.topk(scores, np.array([49], np.int32), 7)
    assert idx[0].tolist() == list(range(7))


# ------------------------------------------------------------------------------------------
# sparse MLA
# ------------------------------------------------------------------------------------------

def test_mla_hand_example():
    g = json.load(open(os.path.join(GOLD, "mla_hand.json")))
    q = torch.tensor([g["q"]], dtype=torch.float32)           # [T=1, H=1, 2]
    pool = _pool_from_rows(torch.tensor(g["rows"], dtype=torch.float32))
    bt, _ = _single_block_table(2)
    out, lse = oracle.sparse_mla(q, pool, bt, torch.tensor([0], dtype=torch.int32),
                                 torch.tensor([[0, 1]], dtype=torch.int32), d_v=1, scale=1.0)
    assert abs(out[0, 0, 0] - g["out"][0]) < 1e-15
    assert abs(lse[0, 0] - g["lse"]) < 1e-14


def test_mla_dense_equals_library_sdpa_when_k_covers_context():
    """With K >= L every position is selected and sparse MLA is dense MQA attention: compare with
    torch's scaled_dot_product_attention in float64 (keys = full 80-wide latent rows, values =
    their first 64 dims)."""
    spec = di.tiny()
    x = di.generate(spec, "cpu", with_indexer=False)
    L = spec.lens[0]
    idx = torch.arange(L, dtype=torch.int32).view(1, L)
    out, lse = oracle.sparse_mla(x["q_mla"], x["latent_pool"], x["block_table"], x["q_req"], idx,
                                 spec.d_v, spec.scale)
    bt = x["block_table"][0].long()
    rows = x["latent_pool"].view(-1, spec.dqk)[(bt.repeat_interleave(64) * 64 + torch.arange(64).repeat(len(bt)))[:L]]
    qd = x["q_mla"][0].double().unsqueeze(0)                 # [1, H, Dqk]
    kd = rows.double().unsqueeze(0).unsqueeze(0).expand(1, spec.H, L, spec.dqk)
    vd = rows[:, :spec.d_v].double().unsqueeze(0).unsqueeze(0).expand(1, spec.H, L, spec.d_v)
    ref = torch.nn.functional.scaled_dot_product_attention(qd.unsqueeze(2), kd, vd, scale=spec.scale)
    np.testing.assert_allclose(out[0], ref[0, :, 0].numpy(), rtol=1e-10, atol=1e-12)
    logits = (qd[0] @ rows.double().T) * spec.scale
    np.testing.assert_allclose(lse[0], torch.logsumexp(logits, -1).numpy(), rtol=1e-12)


def test_mla_closed_forms():
    """q = 0 -> uniform weights: O is the mean of the selected value rows and LSE = log(n);
    one selected row -> O is that row's value part and LSE is its logit; -1 entries are skipped;
    the order of the selected positions does not matter."""
    spec = di.tiny()
    x = di.generate(spec, "cpu", with_indexer=False)
    bt = x["block_table"]
    flat = x["latent_pool"].view(-1, spec.dqk)
    def row(p):
        return flat[int(bt[0, p // 64]) * 64 + p % 64].double()
    sel = [3, 17, 64, 200, 255]
    idx = torch.tensor([sel + [-1] * 3], dtype=torch.int32)
    zero_q = torch.zeros_like(x["q_mla"])
    out, lse = oracle.sparse_mla(zero_q, x["latent_pool"], bt, x["q_req"], idx, spec.d_v, spec.scale)
    mean = torch.stack([row(p)[:spec.d_v] for p in sel]).mean(0).numpy()
    for h in range(spec.H):
        np.testing.assert_allclose(out[0, h], mean, rtol=1e-12, atol=1e-14)
        assert abs(lse[0, h] - math.log(len(sel))) < 1e-12
    one = torch.tensor([[-1, 200, -1]], dtype=torch.int32)
    out1, lse1 = oracle.sparse_mla(x["q_mla"], x["latent_pool"], bt, x["q_req"], one, spec.d_v, spec.scale)
    for h in range(spec.H):
        np.testing.assert_allclose(out1[0, h], row(200)[:spec.d_v].numpy(), rtol=1e-12)
        logit = spec.scale * float(x["q_mla"][0, h].double() @ row(200))
        assert abs(lse1[0, h] - logit) < 1e-12
    perm = torch.tensor([[255, -1, 3, 200, 17, 64, -1, -1]], dtype=torch.int32)
    a, la = oracle.sparse_mla(x["q_mla"], x["latent_pool"], bt, x["q_req"], idx, spec.d_v, spec.scale)
    b, lb = oracle.sparse_mla(x["q_mla"], x["latent_pool"], bt, x["q_req"], perm, spec.d_v, spec.scale)
    np.testing.assert_allclose(a, b, rtol=1e-12)
    np.testing.assert_allclose(la, lb, rtol=1e-12)
    none = torch.full((1, 4), -1, dtype=torch.int32)
    o0, l0 = oracle.sparse_mla(x["q_mla"], x["latent_pool"], bt, x["q_req"], none, spec.d_v, spec.scale)
    assert (o0 == 0).all() and np.isneginf(l0).all()


def test_mla_rope_dims_enter_logits_but_not_values():
    """Changing only the RoPE tail of a row changes the output (via the logits), while an output
    computed from rows whose RoPE tails are zeroed and queries whose RoPE tails are zeroed must
    equal the output for the 64-wide latent alone (d_rope = 0)."""
    spec = di.tiny()
    x = di.generate(spec, "cpu", with_indexer=False)
    idx = torch.tensor([[1, 5, 9, 77, 130]], dtype=torch.int32)
    pool0 = x["latent_pool"].clone(); pool0[..., spec.d_v:] = 0
    q0 = x["q_mla"].clone(); q0[..., spec.d_v:] = 0
    a, la = oracle.sparse_mla(q0, pool0, x["block_table"], x["q_req"], idx, spec.d_v, spec.scale)
    b, lb = oracle.sparse_mla(q0[..., :spec.d_v].contiguous(), pool0[..., :spec.d_v].contiguous(),
                              x["block_table"], x["q_req"], idx, spec.d_v, spec.scale)
    np.testing.assert_allclose(a, b, rtol=1e-12)
    c, _ = oracle.sparse_mla(x["q_mla"], x["latent_pool"], x["block_table"], x["q_req"], idx, spec.d_v, spec.scale)
    assert np.abs(c - a).max() > 1e-3


def test_indexer_e4m3_queries_dequantise_per_head():
    # e4m3 query codes with a per-(query, head) scale are the queries code * scale: with
    # power-of-two scales (exact in f32) the scores equal those of the f32 queries holding the same
    # values, and a head-index slip in the scale (distinct per head) would break the equality;
    # scores are degree-1 homogeneous in a common positive query scale
    x = di.generate(di.tiny(), "cpu")
    codes, _ = di.quantize_e4m3(x["q_idx"])
    T, Hi, Di = codes.shape
    scale = (2.0 ** torch.tensor([[-3.0, 0.0, 2.0, 5.0]])).expand(T, Hi).contiguous().float()
    qf = (codes.view(torch.float8_e4m3fn).float() * scale.unsqueeze(-1)).contiguous()
    args = (x["key_pool"], None, x["block_table"], x["q_req"], x["q_pos"])
    s_q8 = oracle.indexer_scores(codes, x["w"], *args, q_scale=scale)
    s_f = oracle.indexer_scores(qf, x["w"], *args)
    assert np.array_equal(s_q8, s_f)
    s_3 = oracle.indexer_scores(codes, x["w"], *args, q_scale=scale * 3.0)
    n = int(x["q_pos"][0]) + 1
    assert np.allclose(s_3[0, :n], 3.0 * s_q8[0, :n], rtol=1e-12, atol=0)


def test_planted_tail_calibration():
    # the long-context workload's planted keys are shifted by the beta that the committed
    # calibration script found with this oracle; on its draw the median planted score sits
    # 3 unplanted standard deviations above the unplanted mean
    import importlib.util
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "make_planted_beta.py")
    stored = json.load(open(os.path.join(os.path.dirname(path), "planted_beta.json")))
    assert di.PLANTED_BETA == stored["beta"] and di.long_decode().planted_sigma == stored["beta"]
    spec_ = importlib.util.spec_from_file_location("make_planted_beta", path)
    mod = importlib.util.module_from_spec(spec_)
    spec_.loader.exec_module(mod)
    spec = di.long_decode(B=1)
    q_idx, w, kraw, bt, _ = mod.draw_request(spec)
    L = spec.lens[0]
    rows = bt[0].long()[torch.arange(L) // di.BLOCK] * di.BLOCK + torch.arange(L) % di.BLOCK
    base = kraw[rows]
    planted = di.planted_positions(spec, 0)
    mask = torch.ones(L, dtype=torch.bool)
    mask[planted] = False
    unpl = mod.scores_of(base, q_idx, w)[mask.numpy()]
    got = mod.lift(stored["beta"], base, planted, di.plant_direction(q_idx[0], w[0]), q_idx, w,
                   float(unpl.mean()), float(unpl.std()))
    assert abs(got - 3.0) < 0.01
