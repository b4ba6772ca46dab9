"""Parity at the full sizes of the five workloads, in the launch configuration the benchmark
times: the whole hot path runs on the GPU for every query; the fp64 oracle recomputes sampled
queries one by one (all scores of the sampled query, its selection from the GPU's scores, and its
attention output) and the end-to-end selection from the oracle's own scores must agree.  The
selection of every query of every workload is checked bit-exactly against the oracle's selection
applied to the GPU's own scores."""
import gc

import pytest
import torch

import dsa_inputs as di
from _parity import parity_case

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name,queries,kind,entry", [
    ("tiny", None, "f32", "decode"),
    ("decode", None, "bf16", "decode"),
    ("batched_decode", [0, 17, 38, 63], "bf16", "decode"),
    ("prefill", [0, 1, 2, 3, 1365, 2730, 4092, 4095], "e4m3", "prefill"),
    ("long_decode", [0, 9, 15], "e4m3", "decode"),
    ("long_decode_q8", [0, 15], "e4m3", "decode"),
    ("prefill_q8", [0, 2047, 4095], "e4m3", "prefill"),
    ("glm5_decode", [0, 31, 63], "bf16", "decode"),
])
def test_fullsize_sampled(name, queries, kind, entry):
    spec = di.WORKLOADS[name]()
    x = di.generate(spec, "cuda")
    try:
        r = parity_case(x, queries=queries, kind=kind, mla_entry=entry, topk_all_rows=True)
        print(name, r)
    finally:
        del x
        gc.collect()
        torch.cuda.empty_cache()
