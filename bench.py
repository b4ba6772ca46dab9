"""Benchmark of the DSA hot path (lightning indexer -> top-K -> sparse MLA) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME] [--impl dsa|reference]

One step is one pass of the whole hot path over one batch of synthetic, seeded input: indexer
scores fused with the top-K selection (dsa_indexer_topk with its histogram workspace) and sparse
MLA (dsa_sparse_mla_decode, or dsa_sparse_mla_prefill for the prefill chunk).  The default workload
is batched bf16 decode: 64 requests with context lengths uniform in [4096, 131072], paged in
64-token blocks with shuffled block tables (indexer 64 heads x 128, top-2048, MLA 128 heads over
512 + 64) -- the largest single-GPU workload by bytes.  Other workloads: tiny, decode (batch 1,
context 32768), prefill, long_decode (see dsa_inputs.py).

Timing: W untimed warm-up steps; then K steps, each bracketed by CUDA events on the launching
stream; when one copy of the workload's resident data fits in L2, the steps rotate over enough
identical copies of it (caches, queries, outputs) that every step's inputs are larger than L2
apart; barrier + synchronize on both sides; the max over ranks.  Rank 0 prints one
JSON line.  With --gpus N > 1 (torchrun) every rank runs an independent replica of the workload
(the path shards by request with no exchange step): value = all ranks' query tokens / max time.

--impl reference times the fp64 CPU oracle (the method's plain definition) on this host's cores
on a bounded sample of the same workload and prints the same line with "impl": "reference".
"""
from __future__ import annotations

import argparse
import json
import math
import os
import re
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "DSA layer µs and query-tokens/s; achieved HBM TB/s / tensor util vs B200 peak"
L2_BYTES = 126 * 1024 * 1024
GATE_CYCLES = 100_000_000  # ~50 ms spin at 2 GHz before the timed launches start

# ---------------------------------------------------------------------------------------------
# analytic model: algorithmic bytes and FLOPs of each step (method's own work, no re-reads)
# ---------------------------------------------------------------------------------------------


def mla_decode_arithmetic_intensity(H, d, r, b):
    """FLOP per byte of MQA-mode MLA decode for L >> H (page "How GLM5.3 Sparse Attention Affects
    HBM Memory Usage", section "MLA Modifications"): 2 H (2d + r) / (b (d + r))."""
    return 2.0 * H * (2 * d + r) / (b * (d + r))


def ridge(tflops, tbs):
    """Ridge point in FLOP/B of a machine with the given TFLOP/s and TB/s."""
    return tflops / tbs


def key_bytes_per_token(spec):
    return {"f32": 4, "bf16": 2, "e4m3": 1}[spec.key_dtype] * spec.Di + (4 if spec.key_dtype == "e4m3" else 0)


def work_model(spec):
    """Per-step algorithmic work of each kernel.  Units: bytes and FLOPs."""
    act = 4 if spec.act_dtype == "f32" else 2
    T = spec.T
    vis = [p + 1 for p in spec.q_pos]
    pairs = sum(vis)                                    # visible (query, key) pairs
    # keys each request must stream once (decode: one query per request)
    per_req = {}
    for t in range(T):
        r = spec.q_req[t]
        per_req[r] = max(per_req.get(r, 0), vis[t])
    key_tokens = sum(per_req.values())
    q_bytes = spec.Di + 4 if spec.q_idx_dtype == "e4m3" else spec.Di * act  # per head (+ its scale)
    idx_bytes = key_tokens * key_bytes_per_token(spec) + T * spec.Hi * (q_bytes + 4) + pairs * 4
    idx_flops = 2.0 * pairs * spec.Hi * spec.Di
    sel = [min(v, spec.k) for v in vis]
    topk_bytes = pairs * 4 + T * spec.k * 4
    mla_rows = sum(sel)
    # HBM bytes of the row gather: a row that several queries of one request select is read from
    # HBM once at best (the others hit L2), so a request costs at most its visible rows
    sel_req = {}
    for t in range(T):
        r = spec.q_req[t]
        sel_req[r] = sel_req.get(r, 0) + sel[t]
    mla_hbm_rows = sum(min(sel_req[r], per_req[r]) for r in sel_req)
    mla_bytes = mla_hbm_rows * spec.dqk * act + T * spec.H * (spec.dqk + spec.d_v) * act + T * spec.H * 4
    mla_flops = 2.0 * spec.H * mla_rows * (spec.dqk + spec.d_v)
    # rows the tensor-core MLA gathers into shared memory: whole 64-row tiles of each query's
    # selection slots (K of them; in the dense case its visible positions), by both value-half CTAs
    tc_mla = spec.act_dtype == "bf16" and spec.H in (64, 128) and spec.d_v == 512 and spec.dqk == 576
    dense = max(vis) <= spec.k
    slots = [min(v, spec.k) for v in vis] if dense else [spec.k] * T
    mla_gather_bytes = (2 * sum(-(-n // 64) * 64 for n in slots) * spec.dqk * act * spec.share_layers
                        if tc_mla else 0)
    if max(vis) <= spec.k:
        # the dense case: every query keeps all its positions, no indexer or selection runs
        idx_bytes = idx_flops = topk_bytes = 0
    # IndexShare: the group's other layers run sparse MLA on the same selection
    mla_bytes *= spec.share_layers
    mla_flops *= spec.share_layers
    return dict(indexer_bytes=idx_bytes, indexer_flops=idx_flops, topk_bytes=topk_bytes,
                mla_bytes=mla_bytes, mla_flops=mla_flops, key_tokens=key_tokens, pairs=pairs,
                mla_rows=mla_rows, mla_hbm_rows=mla_hbm_rows, mla_gather_bytes=mla_gather_bytes)


def resident_bytes(spec, x):
    tot = 0
    for k in ("key_pool", "key_scale", "latent_pool", "q_idx", "q_mla", "w"):
        v = x.get(k)
        if v is not None:
            tot += v.numel() * v.element_size()
    return tot


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return dict(hbm_gbs=d["hbm_gbs"], bf16_tflops=d["bf16_tflops"],
                    bf16_tflops_sustained=d.get("bf16_tflops_sustained", d["bf16_tflops"]), source="measured")
    return dict(hbm_gbs=6650.0, bf16_tflops=1590.0, bf16_tflops_sustained=1400.0, source="fallback")


def source_digest(path):
    """First 16 hex digits of the sha256 of a source file's code with comments and runs of white
    space removed: edits of comments alone keep the digest, any change of code changes it."""
    import hashlib
    src = open(path).read()
    src = re.sub(r"/\*.*?\*/", " ", src, flags=re.S)
    src = re.sub(r"//[^\n]*", " ", src)
    return hashlib.sha256(" ".join(src.split()).encode()).hexdigest()[:16]


def ncu_traffic(kernel, workload):
    """Per-launch DRAM bytes of `kernel` from the committed ncu summary, or None when there is
    none for this kernel and workload, or when the kernel's code changed since the capture."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    try:
        d = json.load(open(p))
        e = d.get("%s@%s" % (kernel, workload))
        if not e:
            return None
        if source_digest(os.path.join(ROOT, e["source"])) != e["source_digest"]:
            return None
        return float(e["bytes_per_launch"])
    except Exception:
        return None


# ---------------------------------------------------------------------------------------------
# clocks during the timed region
# ---------------------------------------------------------------------------------------------


class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        self.dev = device_index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.dev), "--query-gpu=" + self.FIELDS,
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if not self.proc:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                mx.append(float(parts[1]))
            except ValueError:
                continue
            for n, v in zip(names, parts[4:8]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


# ---------------------------------------------------------------------------------------------
# CUDA arm
# ---------------------------------------------------------------------------------------------


def _dist_env():
    return int(os.environ.get("RANK", 0)), int(os.environ.get("LOCAL_RANK", 0)), int(os.environ.get("WORLD_SIZE", 1))


def max_over_ranks(value, world, device=None):
    """Max of a per-rank float over all ranks (identity for a single process)."""
    if world == 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate(units_per_rank, max_time_s, world):
    """Whole-job throughput: all ranks' units over the slowest rank's time."""
    return units_per_rank * world / max_time_s


class Layer:
    """Buffers and calls of one hot-path step for a generated workload (all on the device)."""

    def __init__(self, x):
        import torch
        import sparse_attention_06_b200 as dsa
        self.dsa = dsa
        self.torch = torch
        self.x = x
        spec = x["spec"]
        self.spec = spec
        self.keys = dsa.PagedCache(x["key_pool"], x.get("key_scale"))
        self.lat = dsa.PagedCache(x["latent_pool"])
        self.max_ctx = max(spec.q_pos) + 1
        self.batch = dsa.Batch(x["q_req"], x["q_pos"], x["block_table"], self.max_ctx, spec.query_group)
        self.ld = (self.max_ctx + 3) // 4 * 4
        dev = x["key_pool"].device
        self.scores = torch.empty((spec.T, self.ld), dtype=torch.float32, device=dev)
        self.idx = torch.empty((spec.T, spec.k), dtype=torch.int32, device=dev)
        self.out = torch.empty((spec.T, spec.H, spec.d_v), dtype=x["q_mla"].dtype, device=dev)
        self.lse = torch.empty((spec.T, spec.H), dtype=torch.float32, device=dev)
        # end to end, a large batch's MLA runs in query chunks, so that the output of one chunk goes
        # back to the host while the next is computed: as many chunks (1, 2 or 4, whole query
        # groups) as keep every chunk at four or more (query, value half) units per SM
        sms = torch.cuda.get_device_properties(dev).multi_processor_count if dev.type == "cuda" else 148
        self.chunks = [(c0, c1, dsa.Batch(x["q_req"][c0:c1], x["q_pos"][c0:c1], x["block_table"], self.max_ctx,
                                          spec.query_group))
                       for c0, c1 in mla_query_chunks(spec.T, spec.query_group, sms)]
        self.chunk_done = [torch.cuda.Event() for _ in self.chunks] if dev.type == "cuda" else []
        self.back = torch.cuda.Event() if dev.type == "cuda" else None
        ws = max(dsa.dsa_mla_workspace_size(n, spec.H, spec.d_v, spec.k)
                 for n in {spec.T} | {c1 - c0 for c0, c1, _ in self.chunks})
        self.ws = torch.empty(ws, dtype=torch.uint8, device=dev) if ws else None
        self.prefill = spec.query_group > 1
        self.q_idx, self.w, self.q_mla = x["q_idx"], x["w"], x["q_mla"]
        self.q_scale = x.get("q_idx_scale")
        # the fused selection's histogram workspace: zero-filled once, every call leaves it zeroed
        self.khist = torch.zeros(dsa.dsa_indexer_topk_workspace_size(spec.T) // 4, dtype=torch.int32, device=dev)
        # every query sees at most K positions: the method keeps them all, so the layer is
        # attention over the whole context without indexer or selection (the dense case)
        self.dense = self.max_ctx <= spec.k
        # IndexShare: layers that reuse this layer's selection (own MLA queries and latent cache)
        self.shared = []
        for sh in x.get("shared", []):
            self.shared.append((sh["q_mla"], dsa.PagedCache(sh["latent_pool"]), torch.empty_like(self.out),
                                torch.empty_like(self.lse)))

    def _mla(self, q, lat, out, lse, idx):
        fn = self.dsa.dsa_sparse_mla_prefill if self.prefill else self.dsa.dsa_sparse_mla_decode
        fn(q, lat, self.batch, idx, self.spec.scale, out, lse, self.ws, k=self.spec.k)

    def _mla_first(self, idx, mla_ready, out_host, d2h_stream):
        """This layer's MLA (after its queries are in place); with out_host, its output goes back to
        the host on d2h_stream chunk by chunk, each copy overlapping the next chunk's MLA and the
        shared layers' MLAs; the compute stream waits for the copies at the end of the step."""
        torch = self.torch
        self._mla_inputs_ready(mla_ready)
        if out_host is None:
            self._mla(self.q_mla, self.lat, self.out, self.lse, idx)
            return None
        fn = self.dsa.dsa_sparse_mla_prefill if self.prefill else self.dsa.dsa_sparse_mla_decode
        cur = torch.cuda.current_stream()
        for (c0, c1, b), done in zip(self.chunks, self.chunk_done):
            fn(self.q_mla[c0:c1], self.lat, b, None if idx is None else idx[c0:c1], self.spec.scale,
               self.out[c0:c1], self.lse[c0:c1], self.ws, k=self.spec.k)
            done.record(cur)
            d2h_stream.wait_event(done)
            with torch.cuda.stream(d2h_stream):
                out_host[c0:c1].copy_(self.out[c0:c1], non_blocking=True)
        self.back.record(d2h_stream)
        return self.back

    def _mla_inputs_ready(self, ready):
        """The MLA reads queries that an end-to-end step copies on a side stream (None: resident)."""
        if ready is not None:
            self.torch.cuda.current_stream().wait_event(ready)

    def step_sparse(self, ev=None, mla_ready=None, out_host=None, d2h_stream=None):
        """Indexer fused with the top-K selection (the indexer builds each query's order-key digit
        histogram, the selection places its threshold from it and clears it) -> sparse MLA (and
        the shared layers' sparse MLA on the same selection).  With events (per-kernel breakdown)
        the two kernels of the fused call are enqueued by their own entry points, same arguments."""
        d = self.dsa
        if ev is None:
            d.dsa_indexer_topk(self.q_idx, self.w, self.keys, self.batch, self.spec.k, self.scores, self.idx,
                               q_scale=self.q_scale, workspace=self.khist)
        else:
            d.dsa_indexer_scores(self.q_idx, self.w, self.keys, self.batch, self.scores, q_scale=self.q_scale,
                                 key_hist=self.khist)
            ev[0].record()
            d.dsa_topk_select(self.scores, self.batch.q_pos, self.spec.k, self.idx, key_hist=self.khist)
            ev[1].record()
        back = self._mla_first(self.idx, mla_ready, out_host, d2h_stream)
        for q, lat, out, lse in self.shared:
            self._mla(q, lat, out, lse, self.idx)
        if back is not None:
            self.torch.cuda.current_stream().wait_event(back)

    def step_unfused(self):
        """The same layer with the selection sampling its threshold (no histogram from the
        indexer): the comparison for the fused indexer-selection path."""
        d = self.dsa
        d.dsa_indexer_scores(self.q_idx, self.w, self.keys, self.batch, self.scores, q_scale=self.q_scale)
        d.dsa_topk_select(self.scores, self.batch.q_pos, self.spec.k, self.idx)
        self._mla(self.q_mla, self.lat, self.out, self.lse, self.idx)
        for q, lat, out, lse in self.shared:
            self._mla(q, lat, out, lse, self.idx)

    def step(self, ev=None, mla_ready=None, out_host=None, d2h_stream=None):
        if not self.dense:
            return self.step_sparse(ev, mla_ready, out_host, d2h_stream)
        if ev is not None:
            ev[0].record()
            ev[1].record()
        back = self._mla_first(None, mla_ready, out_host, d2h_stream)
        if back is not None:
            self.torch.cuda.current_stream().wait_event(back)

    def step_full_layer(self):
        """One full layer alone (indexer, top-K, sparse MLA): the IndexShare comparison."""
        self.dsa.dsa_indexer_topk(self.q_idx, self.w, self.keys, self.batch, self.spec.k, self.scores, self.idx,
                                  q_scale=self.q_scale, workspace=self.khist)
        self._mla(self.q_mla, self.lat, self.out, self.lse, self.idx)


def mla_query_chunks(T, query_group, sms):
    """Query ranges [c0, c1) of an end-to-end step's MLA calls: 1, 2 or 4 chunks of whole query
    groups, as many as keep every chunk at four or more (query, value half) units per SM, so that
    each chunk still fills the GPU while the previous chunk's output goes back to the host."""
    nch = next(c for c in (4, 2, 1) if c == 1 or 2 * T // c >= 4 * sms)
    g = max(1, query_group)
    cuts = sorted({min(T, (T * i // nch) // g * g) for i in range(nch + 1)} | {T})
    return [(c0, c1) for c0, c1 in zip(cuts[:-1], cuts[1:]) if c1 > c0]


def gather_ceiling(dsa, lat, dev, tiles=32, seed=7):
    """Rate of the sparse MLA's row gathers alone on every SM (dsa_selftest_gather_rate): random
    rows of the latent pool, `tiles` 64-row tiles per CTA, one CTA per SM; GB/s over the launch
    (CUDA events) and the mean bytes per SM cycle of the CTAs."""
    import torch
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    pool_rows = lat.data.shape[0] * lat.data.shape[1]
    g = torch.Generator(device=dev).manual_seed(seed)
    rows = torch.randint(0, pool_rows, (sms * tiles * 64,), generator=g, device=dev, dtype=torch.int32)
    cycles = torch.zeros(sms, dtype=torch.int64, device=dev)
    dsa.dsa_selftest_gather_rate(lat, rows, tiles, sms, cycles)  # warm-up
    b = torch.cuda.Event(enable_timing=True)
    e = torch.cuda.Event(enable_timing=True)
    b.record()
    dsa.dsa_selftest_gather_rate(lat, rows, tiles, sms, cycles)
    e.record()
    torch.cuda.synchronize()
    tile_bytes = 64 * 1152
    gbs = sms * tiles * tile_bytes / (b.elapsed_time(e) / 1e3) / 1e9
    c = cycles.double().cpu()
    return {"gbs": gbs, "per_sm_cycle": float((tiles * tile_bytes / c[c > 0]).mean())}


def _time_steps(fn, K, stream, warmup=3):
    """Device time of K back-to-back calls of fn, after `warmup` untimed calls (so that a kernel
    no earlier pass ran is loaded and warm) and a stream gate (CUDA events, ms)."""
    import torch
    b = torch.cuda.Event(enable_timing=True)
    e = torch.cuda.Event(enable_timing=True)
    for i in range(warmup):
        fn(i)
    torch.cuda.synchronize()
    torch.cuda._sleep(GATE_CYCLES)
    b.record(stream)
    for i in range(K):
        fn(i)
    e.record(stream)
    torch.cuda.synchronize()
    return b.elapsed_time(e)


def run_cuda(args):
    import torch
    rank, local_rank, world = _dist_env()
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    import dsa_inputs as di
    import sparse_attention_06_b200 as dsa
    dsa.load_library()
    spec = di.WORKLOADS[args.config]()
    x = di.generate(spec, device=dev)
    model = work_model(spec)
    # inputs larger than L2 between uses: rotate over identical copies of the resident data
    ncopy = max(1, -(-2 * L2_BYTES // max(1, resident_bytes(spec, x))))
    def clone(v):
        if isinstance(v, torch.Tensor):
            return v.clone()
        if isinstance(v, list):
            return [clone(e) for e in v]
        if isinstance(v, dict):
            return {k: clone(e) for k, e in v.items()}
        return v
    copies = [x] + [{k: clone(v) for k, v in x.items() if k != "spec"} | {"spec": spec} for _ in range(ncopy - 1)]
    layers = [Layer(c) for c in copies]
    layer = layers[0]
    stream = torch.cuda.current_stream()

    dsa.dsa_clear_device_error()
    for i in range(args.warmup):
        layers[i % ncopy].step()
    torch.cuda.synchronize()
    err = dsa.dsa_get_device_error()
    if err:
        raise RuntimeError("device error word %d after warm-up" % err)

    K = args.steps
    sampler = ClockSampler(local_rank)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    launches0 = dsa.dsa_kernel_launch_count()
    sampler.start()
    # Headline pass: one event before and one after the K steps, nothing between the kernels (an
    # event between two kernels would keep the second from overlapping its launch with the first's
    # tail).  The stream is held for a moment first so that every timed launch is enqueued before
    # the device starts: the events then measure back-to-back device execution, not host gaps.
    t_beg = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    torch.cuda._sleep(GATE_CYCLES)
    t_beg.record(stream)
    for i in range(K):
        layers[i % ncopy].step()
    t_end.record(stream)
    torch.cuda.synchronize()
    launches = dsa.dsa_kernel_launch_count() - launches0
    # Breakdown pass (per-kernel rooflines only): the same K steps with events between kernels.
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(K)]
    torch.cuda._sleep(GATE_CYCLES)
    for i in range(K):
        e = evs[i]
        e[0].record(stream)
        layers[i % ncopy].step(ev=(e[1], e[2]))
        e[3].record(stream)
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    clocks = sampler.stop()
    idx_ms = [e[0].elapsed_time(e[1]) for e in evs]
    topk_ms = [e[1].elapsed_time(e[2]) for e in evs]
    mla_ms = [e[2].elapsed_time(e[3]) for e in evs]
    step_ms_sep = [e[0].elapsed_time(e[3]) for e in evs]
    total_s = max_over_ranks(t_beg.elapsed_time(t_end) / 1e3, world, dev)
    units = spec.T * K
    value = aggregate(units, total_s, world)
    ms_per_step = total_s * 1e3 / K

    # end to end through the public API: per-step query-side inputs from pinned host memory,
    # the KV caches resident in HBM (state), output read back every step.  The indexer's inputs
    # (and the batch description) are copied on the compute stream first; the MLA's queries,
    # which nothing reads before the selection is done, follow on a second stream that the compute
    # stream waits for just before the MLA, so that their copy overlaps the indexer and the
    # selection; the output goes back on a third stream, chunk by chunk when the MLA runs in query
    # chunks, or behind the shared layers' MLAs.  Small copies (under 1 MB of MLA queries; one
    # chunk and no shared layers) stay on the compute stream: there the extra stream hand-offs
    # would cost more than they hide.
    first = ("q_req", "q_pos", "block_table") + (() if layer.dense else ("q_idx", "w"))
    if not layer.dense and x.get("q_idx_scale") is not None:
        first += ("q_idx_scale",)

    def first_inputs(c):  # device tensors of one copy that the host supplies every step
        return [c[n] for n in first]

    def mla_inputs(c):
        return [c["q_mla"]] + [sh["q_mla"] for sh in c.get("shared", [])]
    host_first = [t.cpu().pin_memory() for t in first_inputs(x)]
    host_mla = [t.cpu().pin_memory() for t in mla_inputs(x)]
    dev_first = [first_inputs(c) for c in copies]
    dev_mla = [mla_inputs(c) for c in copies]
    host_out = torch.empty(layer.out.shape, dtype=layer.out.dtype).pin_memory()
    mla_bytes = sum(t.numel() * t.element_size() for t in host_mla)
    h2d = sum(t.numel() * t.element_size() for t in host_first) + mla_bytes
    d2h = host_out.numel() * host_out.element_size()
    side_in = mla_bytes >= (1 << 20)
    side_out = len(layer.chunks) > 1 or bool(layer.shared)
    e2e_ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(K)]
    copy_stream = torch.cuda.Stream()
    d2h_stream = torch.cuda.Stream()
    first_done = [torch.cuda.Event() for _ in range(K)]
    mla_ready = [torch.cuda.Event() for _ in range(K)]
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    for i in range(K):
        lay = layers[i % ncopy]
        torch.cuda.synchronize()  # end to end: every step starts from an idle device and host
        e2e_ev[i][0].record(stream)
        for dst, src in zip(dev_first[i % ncopy], host_first):
            dst.copy_(src, non_blocking=True)
        if side_in:
            first_done[i].record(stream)
            copy_stream.wait_event(first_done[i])  # after the indexer's inputs, inside the timed region
            with torch.cuda.stream(copy_stream):
                for dst, src in zip(dev_mla[i % ncopy], host_mla):
                    dst.copy_(src, non_blocking=True)
            mla_ready[i].record(copy_stream)
        else:
            for dst, src in zip(dev_mla[i % ncopy], host_mla):
                dst.copy_(src, non_blocking=True)
        if side_out:
            lay.step(mla_ready=mla_ready[i] if side_in else None, out_host=host_out, d2h_stream=d2h_stream)
        else:
            lay.step(mla_ready=mla_ready[i] if side_in else None)
            host_out.copy_(lay.out, non_blocking=True)
        e2e_ev[i][1].record(stream)
    torch.cuda.synchronize()
    e2e_s = max_over_ranks(sum(e[0].elapsed_time(e[1]) for e in e2e_ev) / 1e3, world, dev)
    e2e_value = aggregate(units, e2e_s, world)

    # roofline of every kernel; the line's "roofline" is the dominant (slowest) one.  A kernel's
    # bound is whichever of its algorithmic bytes / HBM peak and FLOPs / tensor peak is larger.
    peaks = load_peaks()
    tensor_peak = peaks["bf16_tflops_sustained"] if statistics.mean(step_ms_sep) > 50 else peaks["bf16_tflops"]
    roofs = {}
    # e4m3 x e4m3 indexer products run at twice the bf16 rate: their peak is the measured bf16
    # peak times the nominal fp8 / bf16 ratio (2)
    idx_peak_mult = 2.0 if spec.q_idx_dtype == "e4m3" else 1.0
    for name, ms_list, nbytes, flops, pmult in (
            ("indexer", idx_ms, model["indexer_bytes"], model["indexer_flops"], idx_peak_mult),
            ("topk", topk_ms, model["topk_bytes"], 0.0, 1.0),
            ("mla", mla_ms, model["mla_bytes"], model["mla_flops"], 1.0)):
        if nbytes == 0 and flops == 0:
            continue  # not run in this workload (the dense case has no indexer or selection)
        t = statistics.mean(ms_list) / 1e3
        t_hbm = nbytes / (peaks["hbm_gbs"] * 1e9)
        t_ten = flops / (pmult * tensor_peak * 1e12)
        if t_ten > t_hbm:
            pk = pmult * tensor_peak
            roofs[name] = {"bound": "tensor", "achieved": flops / t / 1e12, "peak": pk,
                           "unit": "TFLOP/s", "frac": flops / t / 1e12 / pk, "us": t * 1e6}
            if pmult != 1.0:
                roofs[name]["peak_note"] = "fp8: measured bf16 peak x 2 (nominal fp8/bf16 ratio)"
        else:
            roofs[name] = {"bound": "hbm", "achieved": nbytes / t / 1e9, "peak": peaks["hbm_gbs"],
                           "unit": "GB/s", "frac": nbytes / t / 1e9 / peaks["hbm_gbs"], "us": t * 1e6}
    dom = max(roofs, key=lambda n: roofs[n]["us"])
    roof = dict(roofs[dom])
    roof["kernel"] = dom
    roof["peak_source"] = peaks["source"]
    roof["traffic"] = ncu_traffic(dom, args.config)
    breakdown = {"layer_us": ms_per_step * 1e3, "layer_us_with_events_between_kernels": statistics.mean(step_ms_sep) * 1e3}
    for name, r in roofs.items():
        breakdown[name + "_us"] = r["us"]
        breakdown[name + "_frac"] = r["frac"]
        breakdown[name + "_bound"] = r["bound"]
    # The sparse MLA is bound by the rate at which the SMs gather its rows (TMA tile::gather4 of
    # 128-byte boxes), not by HBM or the tensor cores: its gathered bytes per second against that
    # rate, measured in this run by the library's gather diagnostic (the MLA's gathers alone) on
    # random rows of this workload's latent pool, over every SM.
    if model["mla_gather_bytes"] and mla_ms:
        ceil = gather_ceiling(dsa, layer.lat, dev)
        achieved = model["mla_gather_bytes"] / (statistics.mean(mla_ms) / 1e3) / 1e9
        breakdown["mla_gather"] = {"bytes": model["mla_gather_bytes"], "achieved_gbs": achieved,
                                   "ceiling_gbs": ceil["gbs"], "ceiling_bytes_per_sm_cycle": ceil["per_sm_cycle"],
                                   "frac": achieved / ceil["gbs"]}

    # comparisons on the same inputs: the sparse path where the dense case applies, and one full
    # layer alone where a group of layers shares one selection
    if layer.dense:
        sp_ms = _time_steps(lambda i: layers[i % ncopy].step_sparse(), K, stream) / K
        breakdown["sparse_path_us"] = sp_ms * 1e3
        breakdown["dense_saving"] = 1.0 - ms_per_step / sp_ms
    if not layer.dense:
        uf_ms = _time_steps(lambda i: layers[i % ncopy].step_unfused(), K, stream) / K
        breakdown["layer_us_selection_unfused"] = uf_ms * 1e3
    if layer.shared:
        fl_ms = _time_steps(lambda i: layers[i % ncopy].step_full_layer(), K, stream) / K
        n_l = 1 + len(layer.shared)
        breakdown["layers_per_group"] = n_l
        breakdown["full_layer_us"] = fl_ms * 1e3
        breakdown["full_layers_us"] = n_l * fl_ms * 1e3
        breakdown["group_saving"] = 1.0 - ms_per_step / (n_l * fl_ms)
    err = dsa.dsa_get_device_error()

    # the planted tail as the GPU's own scores show it (request 0): how far the median planted
    # score sits above the unplanted scores' mean, in their standard deviations
    planted = None
    if spec.planted_frac > 0 and not layer.dense:
        t0 = spec.q_req.index(0)
        row = layer.scores[t0, :spec.q_pos[t0] + 1].double().cpu()
        pos = di.planted_positions(spec, 0)
        mask = torch.ones(row.numel(), dtype=torch.bool)
        mask[pos] = False
        unpl = row[mask]
        planted = {"frac": spec.planted_frac, "beta": spec.planted_sigma,
                   "lift_sigma_measured": float((row[pos].median() - unpl.mean()) / unpl.std())}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(x, spec, budget_s=args.cpu_budget)

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "query-tokens/s", "n_gpus": world, "steps": K,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16" if spec.act_dtype == "bf16" else "f32",
            "data": "synthetic (seeded N(0,1) queries/keys/latent, U(0,1) head weights, shuffled 64-token pages)",
            "config": {"workload": spec.name, "queries_per_step": spec.T, "requests": spec.B,
                       "context": max(spec.lens), "indexer": "%dx%d %s keys" % (spec.Hi, spec.Di, spec.key_dtype),
                       "top_k": spec.k, "mla": "%d heads, %d+%d" % (spec.H, spec.d_v, spec.d_rope),
                       "l2": ("inputs larger than L2: steps rotate over %d identical copies" % ncopy
                              if ncopy > 1 else "inputs larger than L2"),
                       "parallelism": "replicas x%d" % world},
            "planted_tail": planted,
            "e2e": {"value": e2e_value, "unit": "query-tokens/s", "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h,
                    "note": ("query-side inputs copied from pinned host memory every step (MLA queries "
                             "%s, output read back %s); KV caches resident" % (
                                 "on a second stream, overlapping the indexer and the selection" if side_in
                                 else "in order", "on a third stream, per MLA query chunk (%d), overlapping "
                                 "the following work" % len(layer.chunks) if side_out else "at the end"))},
            "gpu_launches": launches,
            "roofline": roof,
            "breakdown": breakdown,
            "cpu_baseline": cpu,
            "clocks": clocks,
            "device_error": err,
        }
        print(json.dumps(line))
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()


# ---------------------------------------------------------------------------------------------
# CPU oracle: the cpu_baseline leg and the --impl reference arm
# ---------------------------------------------------------------------------------------------


def oracle_step(sub, spec, nthreads):
    """One pass of the oracle over the queries in `sub` (indexer, selection, sparse MLA)."""
    import numpy as np
    import oracle
    if int(sub["q_pos"].max()) + 1 <= spec.k:
        # the dense case, as the layer runs it: every visible position, no indexer or selection
        n = sub["q_pos"].numpy().astype(np.int64) + 1
        j = np.arange(spec.k)[None, :]
        idx = np.where(j < n[:, None], j, -1).astype(np.int32)
    else:
        s = oracle.indexer_scores(sub["q_idx"], sub["w"], sub["key_pool"], sub["key_scale"], sub["block_table"],
                                  sub["q_req"], sub["q_pos"], nthreads=nthreads, q_scale=sub.get("q_idx_scale"))
        idx = oracle.topk(s, sub["q_pos"], spec.k, nthreads=nthreads)
    oracle.sparse_mla(sub["q_mla"], sub["latent_pool"], sub["block_table"], sub["q_req"], idx, spec.d_v,
                      spec.scale, nthreads=nthreads)
    for sh in sub.get("shared", []):  # IndexShare: the other layers reuse the selection
        oracle.sparse_mla(sh["q_mla"], sh["latent_pool"], sub["block_table"], sub["q_req"], idx, spec.d_v,
                          spec.scale, nthreads=nthreads)


def oracle_macs(spec, t):
    """Multiply-adds of one oracle pass over query t (indexer unless dense, attention per layer)."""
    n = spec.q_pos[t] + 1
    dense = max(spec.q_pos) + 1 <= spec.k
    return (0 if dense else n * spec.Hi * spec.Di) + min(n, spec.k) * spec.H * (spec.dqk + spec.d_v) * spec.share_layers


def _sample_queries(spec, budget_macs):
    """Queries of a bounded sample: evenly spaced over the batch (at most 64), up to
    `budget_macs` multiply-adds of oracle work."""
    T = spec.T
    order = list(range(0, T, max(1, T // 64)))
    qs, macs = [], 0
    for t in order:
        qs.append(t)
        macs += oracle_macs(spec, t)
        if macs >= budget_macs:
            break
    return qs


def cpu_baseline(x, spec, budget_s=15.0, repeats=None):
    """Time the oracle (as it stands) on the host cores on a bounded sample of the workload."""
    import dsa_inputs as di
    import oracle
    cores = oracle.max_threads()
    # about 1e8 fp64 MAC/s per core in the oracle's loops: size the sample to the budget
    qs = _sample_queries(spec, budget_s * cores * 1e8)
    sub = di.subset(x, qs)
    threads = cores
    t0 = time.perf_counter()
    n = 0
    while True:
        oracle_step(sub, spec, threads)
        n += 1
        if repeats is not None and n >= repeats:
            break
        if repeats is None and (time.perf_counter() - t0 > budget_s / 3 or n >= 3):
            break
    dt = (time.perf_counter() - t0) / n
    return {"value": len(qs) / dt, "unit": "query-tokens/s", "cores": threads, "kind": "oracle",
            "sample": "%d of %d queries (%d visible key positions), %d pass(es), fp64" % (
                len(qs), spec.T, sum(spec.q_pos[t] + 1 for t in qs), n)}


def run_reference(args):
    rank, _, world = _dist_env()
    if rank != 0:
        return
    import torch
    import dsa_inputs as di
    spec = di.WORKLOADS[args.config]()
    # the same seeded draw as the CUDA arm (on the GPU when there is one, else on the host); only
    # the sampled queries' inputs go to the oracle
    x = di.generate(spec, device="cuda" if torch.cuda.is_available() else "cpu")
    budget = min(args.cpu_budget, 120.0 / max(1, args.steps + args.warmup))
    import oracle
    cores = oracle.max_threads()
    qs = _sample_queries(spec, budget * cores * 1e8)
    sub = di.subset(x, qs)
    threads = cores
    for _ in range(args.warmup):
        oracle_step(sub, spec, threads)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle_step(sub, spec, threads)
    total = time.perf_counter() - t0
    value = len(qs) * args.steps / total
    sample = "%d of %d queries per step (%d visible key positions), fp64" % (
        len(qs), spec.T, sum(spec.q_pos[t] + 1 for t in qs))
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "query-tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": total * 1e3 / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded)", "config": {"workload": spec.name, "sample": sample},
        "cpu_baseline": {"value": value, "unit": "query-tokens/s", "cores": threads, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "query-tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line))


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--config", default="batched_decode",
                    choices=["tiny", "decode", "batched_decode", "prefill", "long_decode", "short_decode",
                             "indexshare", "prefill_q8", "long_decode_q8", "glm5_decode", "profile_decode",
                             "profile_prefill", "profile_long", "profile_long_q8"])
    ap.add_argument("--impl", default="dsa", choices=["dsa", "reference"])
    ap.add_argument("--cpu-budget", type=float, default=15.0, help="seconds of oracle work for cpu_baseline")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        run_reference(args)
    else:
        run_cuda(args)


if __name__ == "__main__":
    main()
