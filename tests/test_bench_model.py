"""The benchmark's analytic model against values the article prints ("MLA Modifications" of "How
GLM5.3 Sparse Attention Affects HBM Memory Usage"): the MQA-mode MLA decode arithmetic intensity
2H(2d + r)/(b(d + r)) is about 2H for the V3.2 shape, 120.8 FLOP/B for GLM-5 (H = 64), and the
H800 ridge is 865 TFLOP/s / 3.35 TB/s = 258.2 FLOP/B, which puts H near 128."""
import pytest

import bench
import dsa_inputs as di


def test_printed_arithmetic_intensities():
    assert bench.mla_decode_arithmetic_intensity(64, 512, 64, 2) == pytest.approx(120.8, abs=0.1)
    for H in (16, 64, 128):
        assert bench.mla_decode_arithmetic_intensity(H, 512, 64, 2) == pytest.approx(2 * H, rel=0.06)
    r = bench.ridge(865.0, 3.35)
    assert r == pytest.approx(258.2, abs=0.05)
    # H at the H800 ridge: 2H(2d+r)/(b(d+r)) = 258.2  ->  H ~ 128 (the article's conclusion)
    H = r / bench.mla_decode_arithmetic_intensity(1, 512, 64, 2)
    assert H == pytest.approx(128, rel=0.07)


def test_work_model_decode_counts():
    spec = di.decode()
    m = bench.work_model(spec)
    assert m["key_tokens"] == 32768 and m["pairs"] == 32768 and m["mla_rows"] == 2048
    assert m["indexer_flops"] == 2 * 32768 * 64 * 128
    assert m["mla_flops"] == 2 * 128 * 2048 * (576 + 512)
    # keys 256 B/token + 4 B score per key + q and w once
    assert m["indexer_bytes"] == 32768 * (256 + 4) + 64 * (128 * 2 + 4)


def test_work_model_prefill_pairs():
    spec = di.prefill()
    m = bench.work_model(spec)
    assert m["pairs"] == sum(65537 + t for t in range(4096))
    assert m["indexer_flops"] == pytest.approx(4.54e12, rel=0.01)


def test_work_model_prefill_row_gather_hbm_bytes():
    # the 4096 queries of the prefill chunk select 4096 x 2048 rows, but they all come from one
    # request of 69632 positions: HBM serves each row at most once
    spec = di.prefill()
    m = bench.work_model(spec)
    assert m["mla_rows"] == 4096 * 2048
    assert m["mla_hbm_rows"] == 65536 + 4096
    dec = bench.work_model(di.batched_decode())
    assert dec["mla_hbm_rows"] == dec["mla_rows"] == 64 * 2048


def test_work_model_dense_and_indexshare():
    short = bench.work_model(di.short_decode())
    assert short["indexer_bytes"] == 0 and short["topk_bytes"] == 0      # the dense case: no indexer
    assert short["mla_rows"] == sum(L for L in di.short_decode().lens)   # every visible position
    one = bench.work_model(di.batched_decode())
    grp = bench.work_model(di.indexshare())
    assert grp["indexer_bytes"] == one["indexer_bytes"]                  # one indexer per group
    assert grp["mla_flops"] == 4 * one["mla_flops"] and grp["mla_bytes"] == 4 * one["mla_bytes"]


def test_mla_query_chunks_cover_the_batch_in_whole_groups():
    # the end-to-end step's MLA chunks: contiguous, covering every query once, whole query groups,
    # and only as many as keep each chunk at four or more units per SM
    for T, g, sms in ((4096, 4, 148), (64, 1, 148), (16, 1, 148), (1, 1, 148), (1200, 4, 148), (2000, 4, 148),
                      (1184, 1, 148), (4100, 4, 148)):
        ch = bench.mla_query_chunks(T, g, sms)
        assert ch[0][0] == 0 and ch[-1][1] == T
        assert all(a[1] == b[0] for a, b in zip(ch[:-1], ch[1:]))
        assert all(c0 % g == 0 for c0, _ in ch)
        if len(ch) > 1:
            assert all(2 * (c1 - c0) >= 4 * sms - 2 * g for c0, c1 in ch)
    assert len(bench.mla_query_chunks(4096, 4, 148)) == 4
    assert len(bench.mla_query_chunks(64, 1, 148)) == 1


def test_traffic_figures_follow_the_kernel_code(tmp_path, monkeypatch):
    # a committed DRAM-traffic figure stays valid across edits of comments and white space, and
    # is dropped (None) as soon as the kernel's code changes
    import json
    src = tmp_path / "k.cu"
    src.write_text("// header\n__global__ void k(int* a) { a[0] = 1; }  /* note */\n")
    d0 = bench.source_digest(str(src))
    src.write_text("// another header\n__global__ void k(int* a)\n{\n  a[0] = 1;   // same code\n}\n")
    assert bench.source_digest(str(src)) == d0
    (tmp_path / "profiles").mkdir()
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps(
        {"indexer@w": {"source": "k.cu", "source_digest": d0, "bytes_per_launch": 1234}}))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.ncu_traffic("indexer", "w") == 1234.0
    assert bench.ncu_traffic("indexer", "other") is None
    src.write_text("__global__ void k(int* a) { a[0] = 2; }\n")
    assert bench.source_digest(str(src)) != d0
    assert bench.ncu_traffic("indexer", "w") is None
