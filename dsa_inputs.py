"""Seeded synthetic inputs for the DSA hot path, shared by the tests, the smoke check and the
benchmark.  This module only draws values and lays them out (paged pools, block tables,
positions); it holds none of the method's arithmetic and imports neither the CUDA path nor the
oracle.

Recipe (every tensor has its own generator seeded from (seed, tensor id, chunk)):
  * indexer queries q_idx [T, Hi, Di], MLA queries q_mla [T, H, Dqk], keys and latent rows:
    N(0, 1) rounded to the stored dtype (bf16 RNE, or f32 for the tiny workload);
  * indexer head weights w [T, Hi] ~ U(0, 1), f32;
  * e4m3 indexer keys: per-token scale = max_i |k_i| / 448 (f32), code = RNE(k / scale) clamped
    to +-448 -- the quantisation happens here, once; both sides read the same bytes; e4m3 indexer
    queries (the fp8-query workloads) are quantised the same way per (query, head);
  * paged pools of 64-token blocks; each request's logical blocks are mapped to a random
    permutation of the physical blocks (shuffled block tables), unused entries are -1;
  * planted heavy tail (long-context workload): a seeded 2% of each request's positions get their
    indexer key moved by PLANTED_BETA along the unit vector of sum_h w[h] q[h], before
    quantisation; PLANTED_BETA is calibrated (by the oracle, in a committed script) so that the
    median planted score sits 3 standard deviations above the unplanted scores' mean.
Values are drawn with torch generators on the requested device: CPU and CUDA draws differ, but
each is deterministic for a given seed, and parity checks always hand the oracle the very tensors
the GPU used.
"""
from __future__ import annotations

import dataclasses
import math
from typing import List, Optional

import torch

BLOCK = 64
E4M3_MAX = 448.0
_CHUNK_ROWS = 1 << 20  # rows per generator chunk (independent of device)


@dataclasses.dataclass
class Spec:
    name: str
    lens: List[int]            # cache length of each request (positions 0..len-1 exist)
    q_req: List[int]           # request of each query
    q_pos: List[int]           # position of each query (it sees 0..q_pos)
    Hi: int = 64
    Di: int = 128
    H: int = 128
    d_v: int = 512
    d_rope: int = 64
    k: int = 2048
    key_dtype: str = "bf16"    # "f32" | "bf16" | "e4m3"
    act_dtype: str = "bf16"    # dtype of q_idx, q_mla and the latent pool: "f32" | "bf16"
    scale: float = 1.0 / math.sqrt(192.0)
    planted_frac: float = 0.0
    planted_sigma: float = 0.0
    seed: int = 0x5EED
    query_group: int = 1       # queries come in runs of this many sharing one request
    share_layers: int = 1      # layers in an IndexShare group: one full layer, the rest reuse its selection
    q_idx_dtype: str = ""      # "" (act_dtype) or "e4m3": indexer queries quantised per (query, head)

    @property
    def T(self) -> int:
        return len(self.q_req)

    @property
    def B(self) -> int:
        return len(self.lens)

    @property
    def dqk(self) -> int:
        return self.d_v + self.d_rope


def _seed(seed: int, tid: int, chunk: int = 0) -> int:
    return (seed * 1_000_003 + tid * 7919 + chunk * 104_729) & 0x7FFF_FFFF_FFFF


def _gen(device, seed, tid, chunk=0):
    g = torch.Generator(device=device)
    g.manual_seed(_seed(seed, tid, chunk))
    return g


def _dt(name: str):
    return {"f32": torch.float32, "bf16": torch.bfloat16}[name]


def normal(shape, dtype, device, seed, tid):
    """N(0,1) of the given shape, drawn in row chunks so that large pools stay within memory."""
    shape = tuple(shape)
    rows = shape[0]
    inner = int(math.prod(shape[1:])) if len(shape) > 1 else 1
    out = torch.empty((rows, inner), dtype=dtype, device=device)
    step = max(1, _CHUNK_ROWS // max(1, inner // 64))
    for c, r0 in enumerate(range(0, rows, step)):
        r1 = min(rows, r0 + step)
        g = _gen(device, seed, tid, c)
        out[r0:r1] = torch.randn((r1 - r0, inner), generator=g, device=device, dtype=torch.float32).to(dtype)
    return out.view(shape)


def uniform01(shape, device, seed, tid):
    g = _gen(device, seed, tid)
    return torch.rand(tuple(shape), generator=g, device=device, dtype=torch.float32)


def quantize_e4m3(k: torch.Tensor):
    """Per-token e4m3 quantisation of keys [..., Di] -> (codes uint8 [..., Di], scale f32 [...])."""
    kf = k.float()
    amax = kf.abs().amax(dim=-1)
    scale = torch.where(amax > 0, amax / E4M3_MAX, torch.ones_like(amax))
    codes = (kf / scale.unsqueeze(-1)).clamp(-E4M3_MAX, E4M3_MAX).to(torch.float8_e4m3fn)
    return codes.view(torch.uint8), scale.float()


def make_block_table(lens, seed, device="cpu"):
    """Shuffled paging: returns (block_table int32 [B, max_blocks] with -1 padding, num_blocks)."""
    nblk = [max(1, -(-L // BLOCK)) for L in lens]
    total = sum(nblk)
    g = _gen("cpu", seed, 90)
    perm = torch.randperm(total, generator=g).to(torch.int32)
    mb = max(nblk)
    bt = torch.full((len(lens), mb), -1, dtype=torch.int32)
    off = 0
    for b, n in enumerate(nblk):
        bt[b, :n] = perm[off:off + n]
        off += n
    return bt.to(device), total


def generate(spec: Spec, device="cpu", with_mla=True, with_indexer=True):
    """Draw every input of one DSA layer step for ``spec`` on ``device``.

    Returns a dict of tensors: q_idx [T,Hi,Di], w [T,Hi], key_pool [nblk,64,Di] (f32/bf16, or
    uint8 e4m3 codes), key_scale [nblk,64] f32 (e4m3 only, else None), q_mla [T,H,Dqk],
    latent_pool [nblk,64,Dqk], block_table [B,mb] i32, q_req [T] i32, q_pos [T] i32.
    """
    dev = torch.device(device)
    bt, nblk = make_block_table(spec.lens, spec.seed, dev)
    rows = nblk * BLOCK
    act = _dt(spec.act_dtype)
    out = {
        "spec": spec,
        "block_table": bt,
        "num_blocks": nblk,
        "q_req": torch.tensor(spec.q_req, dtype=torch.int32, device=dev),
        "q_pos": torch.tensor(spec.q_pos, dtype=torch.int32, device=dev),
    }
    if with_indexer:
        q_idx = normal((spec.T, spec.Hi, spec.Di), act, dev, spec.seed, 1)
        w = uniform01((spec.T, spec.Hi), dev, spec.seed, 2)
        kraw = normal((rows, spec.Di), torch.float32, dev, spec.seed, 3)
        if spec.planted_frac > 0:
            _plant_tail(spec, kraw, q_idx, w, bt, dev)
        if spec.key_dtype == "e4m3":
            codes, scale = quantize_e4m3(kraw)
            out["key_pool"] = codes.view(nblk, BLOCK, spec.Di)
            out["key_scale"] = scale.view(nblk, BLOCK)
        else:
            out["key_pool"] = kraw.to(_dt(spec.key_dtype)).view(nblk, BLOCK, spec.Di)
            out["key_scale"] = None
        del kraw
        if spec.q_idx_dtype == "e4m3":
            codes, qscale = quantize_e4m3(q_idx)
            out["q_idx"] = codes
            out["q_idx_scale"] = qscale
        else:
            out["q_idx"] = q_idx
        out["w"] = w
    if with_mla:
        out["q_mla"] = normal((spec.T, spec.H, spec.dqk), act, dev, spec.seed, 4)
        out["latent_pool"] = normal((rows, spec.dqk), act, dev, spec.seed, 5).view(nblk, BLOCK, spec.dqk)
        # IndexShare: the other layers of the group have their own MLA queries and latent caches
        # (same requests, same paging) and no indexer inputs of their own
        out["shared"] = [
            {"q_mla": normal((spec.T, spec.H, spec.dqk), act, dev, spec.seed, 4 + 10 * l),
             "latent_pool": normal((rows, spec.dqk), act, dev, spec.seed, 5 + 10 * l).view(nblk, BLOCK, spec.dqk)}
            for l in range(1, spec.share_layers)]
    return out


def planted_positions(spec: Spec, b: int) -> torch.Tensor:
    """The seeded positions of request b whose indexer keys carry the planted tail (CPU int64)."""
    n_plant = int(round(spec.planted_frac * spec.lens[b]))
    g = _gen("cpu", spec.seed, 100 + b)
    return torch.randperm(spec.lens[b], generator=g)[:n_plant]


def plant_direction(q_idx_t, w_t):
    """Unit vector of sum_h w[h] q[h] for one query (float32 [Di]): the direction along which the
    planted keys are moved."""
    u = (w_t.float().unsqueeze(-1) * q_idx_t.float()).sum(0)
    return u / u.norm().clamp_min(1e-30)


def _plant_tail(spec, kraw, q_idx, w, bt, dev):
    """Move a seeded fraction of each request's indexer keys by planted_sigma along the unit
    vector of sum_h w[h] q[h] of that request's (first) query."""
    for b, L in enumerate(spec.lens):
        ts = [t for t, r in enumerate(spec.q_req) if r == b]
        if not ts:
            continue
        u = plant_direction(q_idx[ts[0]], w[ts[0]])
        pos = planted_positions(spec, b).to(dev)
        rows = bt[b].long()[pos // BLOCK] * BLOCK + pos % BLOCK
        kraw[rows] += spec.planted_sigma * u


def planted_scores(T, ld, lens, frac=0.02, lift=3.0, seed=0x5EED, device="cpu"):
    """Directly drawn indexer scores for the standalone selection check: N(0,1), plus ``lift`` on a
    seeded ``frac`` of each row's visible positions.  Entries past lens[t] are NaN."""
    s = normal((T, ld), torch.float32, device, seed, 20)
    for t in range(T):
        g = _gen("cpu", seed, 200 + t)
        n = int(round(frac * lens[t]))
        pos = torch.randperm(lens[t], generator=g)[:n].to(device)
        s[t, pos] += lift
        if lens[t] < ld:
            s[t, lens[t]:] = float("nan")
    return s


# ----------------------------------------------------------------------------------------------
# The five workloads (tiny, decode, batched decode, prefill chunk, long-context decode)
# ----------------------------------------------------------------------------------------------

def tiny(seed=0x5EED) -> Spec:
    """Tiny fp32 DSA layer: one decode query at L=256, indexer 4 heads x 32, top-32, MLA 8 heads,
    latent 64 + rope 16 (softmax scale 1/sqrt(80), the key width)."""
    return Spec("tiny_f32_L256", lens=[256], q_req=[0], q_pos=[255], Hi=4, Di=32, H=8, d_v=64,
                d_rope=16, k=32, key_dtype="f32", act_dtype="f32", scale=1 / math.sqrt(80.0),
                seed=seed)


def decode(L=32768, seed=0x5EED + 1) -> Spec:
    """bf16 decode, batch 1, context L: indexer 64x128, top-2048, MLA 128 heads, 512 + 64."""
    return Spec("decode_bf16_B1_L%d" % L, lens=[L], q_req=[0], q_pos=[L - 1], seed=seed)


def batched_decode(B=64, lo=4096, hi=131072, seed=0x5EED + 2) -> Spec:
    """bf16 batched decode: per-request lengths uniform in [lo, hi] (seeded)."""
    g = _gen("cpu", seed, 50)
    lens = torch.randint(lo, hi + 1, (B,), generator=g).tolist()
    return Spec("batched_decode_bf16_B%d" % B, lens=lens, q_req=list(range(B)),
                q_pos=[L - 1 for L in lens], seed=seed)


def prefill(ctx=65536, chunk=4096, seed=0x5EED + 3) -> Spec:
    """Prefill chunk: ``chunk`` causal queries appended to a ``ctx``-token context; e4m3 indexer
    keys with per-token f32 scale, bf16 queries and latent."""
    L = ctx + chunk
    return Spec("prefill_e4m3_%dq_ctx%d" % (chunk, ctx), lens=[L], q_req=[0] * chunk,
                q_pos=[ctx + t for t in range(chunk)], key_dtype="e4m3", seed=seed, query_group=4)


# Shift of the planted keys along plant_direction, in key-element units (about 3 element standard
# deviations, the keys being N(0, 1)): the value at which the
# median planted indexer score sits 3 standard deviations above the mean of the unplanted scores
# (the "2% of positions +3 sigma" tail).  Written by tests/golden/make_planted_beta.py, which
# finds it with the fp64 oracle on a draw of this workload (tests/golden/planted_beta.json).
PLANTED_BETA = 2.9541015625


def long_decode(B=16, L=202752, seed=0x5EED + 4) -> Spec:
    """Long-context decode: batch B at context L, e4m3 indexer keys, planted tail (2% of the
    positions lifted to a median of +3 score standard deviations)."""
    return Spec("long_decode_e4m3_B%d_L%d" % (B, L), lens=[L] * B, q_req=list(range(B)),
                q_pos=[L - 1] * B, key_dtype="e4m3", planted_frac=0.02, planted_sigma=PLANTED_BETA,
                seed=seed)


def short_decode(B=64, lo=1024, hi=2048, seed=0x5EED + 8) -> Spec:
    """bf16 batched decode at short contexts, uniform in [lo, hi] <= top-k: every query keeps all
    of its positions (the dense case), so the layer is attention over the whole context."""
    g = _gen("cpu", seed, 50)
    lens = torch.randint(lo, hi + 1, (B,), generator=g).tolist()
    return Spec("short_decode_bf16_B%d_L%d_%d" % (B, lo, hi), lens=lens, q_req=list(range(B)),
                q_pos=[L - 1 for L in lens], seed=seed)


def indexshare(B=64, lo=4096, hi=131072, layers=4, seed=0x5EED + 2) -> Spec:
    """IndexShare group over the batched-decode workload: one full DSA layer (indexer, top-K,
    sparse MLA) and ``layers - 1`` layers that reuse its selection (sparse MLA only)."""
    s = batched_decode(B, lo, hi, seed)
    s.name = "indexshare_x%d_batched_decode_bf16_B%d" % (layers, B)
    s.share_layers = layers
    return s


def prefill_q8(ctx=65536, chunk=4096, seed=0x5EED + 3) -> Spec:
    """The prefill chunk with e4m3 indexer queries (per-(query, head) scale) as well as e4m3 keys."""
    s = prefill(ctx, chunk, seed)
    s.name = "prefill_e4m3q_%dq_ctx%d" % (chunk, ctx)
    s.q_idx_dtype = "e4m3"
    return s


def long_decode_q8(B=16, L=202752, seed=0x5EED + 4) -> Spec:
    """Long-context decode with e4m3 indexer queries (per-(query, head) scale) and e4m3 keys."""
    s = long_decode(B, L, seed)
    s.name = "long_decode_e4m3q_B%d_L%d" % (B, L)
    s.q_idx_dtype = "e4m3"
    return s


def glm5_decode(B=64, lo=4096, hi=131072, seed=0x5EED + 9) -> Spec:
    """Batched decode with the GLM-5 attention shape: 64 MLA heads over the same 512 + 64 latent
    rows, softmax scale 1/sqrt(256) (its head dimension); indexer and selection as in the batched
    decode workload."""
    s = batched_decode(B, lo, hi, seed)
    s.name = "glm5_decode_bf16_B%d_H64" % B
    s.H = 64
    s.scale = 1.0 / math.sqrt(256.0)
    return s


def profile_decode(B=8, L=65536, seed=0x5EED + 5) -> Spec:
    """bf16 decode, batch B at context L: a profiling case larger than L2 (0.75 GB resident)."""
    return Spec("profile_decode_bf16_B%d_L%d" % (B, L), lens=[L] * B, q_req=list(range(B)),
                q_pos=[L - 1] * B, seed=seed)


def profile_long_q8(B=8, L=202752, seed=0x5EED + 7) -> Spec:
    """Long-context decode at batch 8 with e4m3 indexer keys and queries, for profiling captures."""
    s = profile_long(B, L, seed)
    s.name = "profile_long_e4m3q_B%d_L%d" % (B, L)
    s.q_idx_dtype = "e4m3"
    return s


def profile_prefill(ctx=16384, chunk=1024, seed=0x5EED + 6) -> Spec:
    """A smaller prefill chunk (e4m3 keys) for profiling captures."""
    return prefill(ctx=ctx, chunk=chunk, seed=seed)


def profile_long(B=8, L=202752, seed=0x5EED + 7) -> Spec:
    """Long-context e4m3 decode at batch 8 (about 2 GB resident) for profiling captures."""
    return Spec("profile_long_e4m3_B%d_L%d" % (B, L), lens=[L] * B, q_req=list(range(B)),
                q_pos=[L - 1] * B, key_dtype="e4m3", seed=seed)


WORKLOADS = {
    "tiny": tiny,
    "decode": decode,
    "batched_decode": batched_decode,
    "prefill": prefill,
    "long_decode": long_decode,
    "short_decode": short_decode,
    "indexshare": indexshare,
    "prefill_q8": prefill_q8,
    "long_decode_q8": long_decode_q8,
    "glm5_decode": glm5_decode,
    "profile_decode": profile_decode,
    "profile_prefill": profile_prefill,
    "profile_long": profile_long,
    "profile_long_q8": profile_long_q8,
}


def subset(inputs: dict, queries: List[int]) -> dict:
    """CPU copy of the inputs the given queries touch, with their requests' blocks gathered into a
    compact pool (so that the oracle can check sampled outputs of a full-size run)."""
    spec = inputs["spec"]
    bt = inputs["block_table"].cpu()
    reqs = sorted({spec.q_req[t] for t in queries})
    rmap = {r: i for i, r in enumerate(reqs)}
    blocks = []
    new_bt = torch.full((len(reqs), bt.shape[1]), -1, dtype=torch.int32)
    off = 0
    for r in reqs:
        n = max(1, -(-spec.lens[r] // BLOCK))
        new_bt[rmap[r], :n] = torch.arange(off, off + n, dtype=torch.int32)
        blocks.append(bt[r, :n].long())
        off += n
    ids = torch.cat(blocks)
    out = {
        "block_table": new_bt,
        "q_req": torch.tensor([rmap[spec.q_req[t]] for t in queries], dtype=torch.int32),
        "q_pos": torch.tensor([spec.q_pos[t] for t in queries], dtype=torch.int32),
    }
    qi = torch.tensor(queries, dtype=torch.long)
    for name in ("q_idx", "q_idx_scale", "w", "q_mla"):
        if name in inputs and inputs[name] is not None:
            out[name] = inputs[name][qi.to(inputs[name].device)].cpu()
    for name in ("key_pool", "key_scale", "latent_pool"):
        if name in inputs and inputs[name] is not None:
            out[name] = inputs[name][ids.to(inputs[name].device)].cpu()
        elif name in inputs:
            out[name] = None
    out["shared"] = [{"q_mla": sh["q_mla"][qi.to(sh["q_mla"].device)].cpu(),
                      "latent_pool": sh["latent_pool"][ids.to(sh["latent_pool"].device)].cpu()}
                     for sh in inputs.get("shared", [])]
    return out
