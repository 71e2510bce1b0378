"""Seeded synthetic inputs for MLA paged decoding.

This module only draws random numbers and lays them out in the storage formats
the decode path consumes. It holds none of the attention arithmetic, so the
fp64 oracle (``oracle/``) and the CUDA path can both be fed from it without
sharing any of the method's code.

Storage formats (DeepSeek MLA latent cache, 576 = 512 latent + 64 RoPE dims,
one row per token serving as K (all 576 dims) and V (first 512 dims); pages of
64 tokens reached through a block table):
  q            [B, s_q, h_q, 576]        bf16
  kcache bf16  [num_pages, 64, 1, 576]   bf16
  kcache fp8   [num_pages, 64, 656]      uint8 token records:
                 512 e4m3 latent codes | 4 fp32 scales (one per 128-element
                 tile, scale = amax/448) | 64 bf16 RoPE dims
  block_table  [B, max_pages]            int32, unused slots -1
  cache_seqlens[B]                       int32
  indices      [B, s_q, topk]            int32 token positions, -1 = ignored

Recipe: ``numpy.random.Generator(PCG64(seed))``; values drawn as fp32 N(0,1)
and rounded to bf16 (round-to-nearest-even) by torch; physical pages assigned
by a seeded permutation. The five named workloads mirror the shapes of the
paged-decode benchmarks: a tiny two-request case, a DeepSeek-V3-shaped
128-head batch, a variable-length two-token (MTP) causal batch, an FP8 latent
cache and a token-sparse batch.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import Optional

import numpy as np
import torch

PAGE = 64
D_QK = 576
D_V = 512
D_ROPE = D_QK - D_V
FP8_TILE = 128
FP8_RECORD_BYTES = D_V + 4 * (D_V // FP8_TILE) + 2 * D_ROPE  # 656
E4M3_MAX = 448.0
NVFP4_D = 512                 # NVFP4 rows: 512 values, the whole row is K and V
NVFP4_BLOCK = 16              # values per UE4M3 scale
E2M1_MAGNITUDES = (0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0)   # codes 0..7 (OCP MX FP4)


@dataclass
class Workload:
    name: str
    batch: int
    s_q: int
    h_q: int
    seqlens: list
    causal: bool
    kv: str = "bf16"            # "bf16" | "fp8" | "nvfp4"
    topk: int = 0               # >0: token-sparse decode
    neg_frac: float = 0.0       # fraction of index slots set to -1
    scale: float = 1.0 / math.sqrt(D_QK)
    seed: int = 0
    note: str = ""

    @property
    def rows(self) -> int:
        return self.s_q * self.h_q

    @property
    def d_qk(self) -> int:
        return NVFP4_D if self.kv == "nvfp4" else D_QK


def _mtp_seqlens(seed: int):
    rng = np.random.Generator(np.random.PCG64(seed + 7))
    lens = rng.integers(1024, 16384, size=128, endpoint=True).astype(np.int64)
    lens[0] = 65536
    return [int(x) for x in lens]


def named_workloads():
    """The five decode workloads (index i uses seed 20260 + i)."""
    return [
        Workload("tiny", 2, 1, 16, [70, 129], causal=False, seed=20260,
                 note="tiny BF16 paged decode, seqlens {70,129}, non-causal"),
        Workload("dsv3", 64, 1, 128, [4096] * 64, causal=False, seed=20261,
                 note="DeepSeek-V3-shaped BF16 decode, 128 heads, seqlen 4096"),
        Workload("mtp", 128, 2, 16, _mtp_seqlens(20262), causal=True, seed=20262,
                 note="variable-length BF16 decode, s_q=2 causal, U[1024,16384] + one 65536"),
        Workload("fp8", 64, 1, 64, [8192] * 64, causal=False, kv="fp8", seed=20263,
                 note="FP8-e4m3 latent cache (per-128 fp32 scales), 64 heads, seqlen 8192"),
        Workload("sparse", 32, 1, 128, [32768] * 32, causal=False, topk=2048,
                 neg_frac=0.05, seed=20264,
                 note="token-sparse BF16 decode, 32768-token caches, topk 2048, 5% -1"),
    ]


def extra_workloads():
    """Workloads of the rows built beyond the five (seeds 20265+): six query
    tokens per request at 64 heads (the FlashInfer README's DeepSeek-V4 decode
    geometry, q_len 6, here on the 576-dim BF16 latent rows), the token-sparse
    batch over the FP8 token-record cache, and the DeepSeek-V4 geometry on
    NVFP4 rows (512 values, query and cache E2M1 + UE4M3)."""
    return [
        Workload("mtp6", 64, 6, 64, [4096] * 64, causal=True, seed=20265,
                 note="q_len 6 x 64 heads (384 rows per request), causal, BF16, seqlen 4096"),
        Workload("fp8_sparse", 32, 1, 128, [32768] * 32, causal=False, kv="fp8", topk=2048,
                 neg_frac=0.05, seed=20266,
                 note="token-sparse FP8-record decode, 32768-token caches, topk 2048, 5% -1"),
        Workload("nvfp4", 32, 6, 64, [8192] * 32, causal=True, kv="nvfp4", scale=512 ** -0.5, seed=20267,
                 note="NVFP4 512-value rows (K = V) and query, q_len 6 x 64 heads, causal, seqlen 8192"),
    ]


def get_workload(name: str) -> Workload:
    for w in named_workloads() + extra_workloads():
        if w.name == name:
            return w
    raise KeyError(name)


def _rng(seed: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(seed))


def _normal_bf16(rng: np.random.Generator, shape, chunk_rows: int = 1 << 22) -> torch.Tensor:
    """fp32 N(0,1) draws rounded to bf16 (torch RNE), generated in chunks."""
    n = int(np.prod(shape))
    out = torch.empty(n, dtype=torch.bfloat16)
    step = chunk_rows * 8
    for s in range(0, n, step):
        e = min(n, s + step)
        x = rng.standard_normal(e - s, dtype=np.float32)
        out[s:e] = torch.from_numpy(x).to(torch.bfloat16)
    return out.view(*shape)


def _normal_f32(rng: np.random.Generator, shape) -> torch.Tensor:
    return torch.from_numpy(rng.standard_normal(int(np.prod(shape)), dtype=np.float32)).view(*shape)


@dataclass
class DecodeInputs:
    workload: Workload
    q: torch.Tensor                   # [B, s_q, h_q, 576] bf16
    kcache: torch.Tensor              # bf16 [P,64,1,576] or uint8 [P,64,656]
    block_table: torch.Tensor         # [B, max_pages] int32
    cache_seqlens: torch.Tensor       # [B] int32
    indices: Optional[torch.Tensor] = None   # [B, s_q, topk] int32
    extra: dict = field(default_factory=dict)
    sink: Optional[torch.Tensor] = None      # [h_q] fp32 per-head attention-sink logits
    q_scale: Optional[torch.Tensor] = None   # nvfp4: uint8 [B, s_q, h_q, 32] UE4M3 block scales
    kv_scale: Optional[torch.Tensor] = None  # nvfp4: uint8 [P, 64, 32] UE4M3 block scales

    @property
    def num_pages(self) -> int:
        return int(self.kcache.shape[0])


def quantize_fp8_records(src: torch.Tensor) -> torch.Tensor:
    """fp32 [P, 64, 576] source -> uint8 [P, 64, 656] token records.

    Per 128-element tile of the 512 latent dims: scale = amax/448 in fp32
    (1 if amax == 0); codes = e4m3(x/scale) round-to-nearest-even, clamped to
    +-448. The 64 RoPE dims are stored as bf16. This is data preparation (the
    cache is an input of the decode path), done with torch's fp8 conversion.
    """
    P = src.shape[0]
    lat = src[..., :D_V].reshape(P, PAGE, D_V // FP8_TILE, FP8_TILE)
    amax = lat.abs().amax(dim=-1)
    scale = torch.where(amax > 0, amax / E4M3_MAX, torch.ones_like(amax)).to(torch.float32)
    y = (lat / scale[..., None]).clamp(-E4M3_MAX, E4M3_MAX)
    codes = y.to(torch.float8_e4m3fn).view(torch.uint8).reshape(P, PAGE, D_V)
    rope = src[..., D_V:].to(torch.bfloat16).contiguous().view(torch.uint8).reshape(P, PAGE, 2 * D_ROPE)
    sc = scale.contiguous().view(torch.uint8).reshape(P, PAGE, 4 * (D_V // FP8_TILE))
    rec = torch.cat([codes, sc, rope], dim=-1).contiguous()
    assert rec.shape[-1] == FP8_RECORD_BYTES
    return rec


def quantize_nvfp4(src: torch.Tensor):
    """fp32 [..., 512] -> (uint8 [..., 256] packed E2M1, uint8 [..., 32] UE4M3).

    Per block of 16 values: scale = e4m3(amax / 6) by torch's fp8 conversion
    (round to nearest even; 0 when amax == 0); code = the E2M1 magnitude
    nearest |x| / scale (ties to the smaller magnitude, saturating at 6) with
    the sign of x; element 2i in the low nibble of byte i. This is data
    preparation: the decode path only reads codes and scales.
    """
    shp = src.shape
    blk = src.reshape(*shp[:-1], shp[-1] // NVFP4_BLOCK, NVFP4_BLOCK).to(torch.float32)
    amax = blk.abs().amax(dim=-1)
    sc8 = (amax / 6.0).to(torch.float8_e4m3fn)
    sc = sc8.to(torch.float32)
    y = torch.where(sc[..., None] > 0, blk / torch.where(sc > 0, sc, torch.ones_like(sc))[..., None],
                    torch.zeros_like(blk))
    mags = torch.tensor(E2M1_MAGNITUDES, dtype=torch.float32)
    idx = (y.abs()[..., None] - mags).abs().argmin(dim=-1)           # first minimum: smaller magnitude
    codes = (idx | torch.where(y < 0, 8, 0)).to(torch.uint8).reshape(*shp[:-1], shp[-1])
    packed = (codes[..., 0::2] | (codes[..., 1::2] << 4)).contiguous()
    return packed, sc8.view(torch.uint8).contiguous()


def make_inputs(w: Workload, *, poison_tail: bool = False, extra_pages: int = 0,
                seqlens_override=None) -> DecodeInputs:
    """Build the seeded host-side inputs of one workload.

    poison_tail: fill the unused tail tokens of every request's last page, and
    any extra never-referenced pages, with NaN (bf16) / NaN codes (fp8) so that
    a path reading them shows up in the output.
    """
    rng = _rng(w.seed)
    seqlens = list(seqlens_override) if seqlens_override is not None else list(w.seqlens)
    B = w.batch
    assert len(seqlens) == B
    q_scale = kv_scale = None
    if w.kv == "nvfp4":
        q, q_scale = quantize_nvfp4(_normal_f32(rng, (B, w.s_q, w.h_q, NVFP4_D)))
    else:
        q = _normal_bf16(rng, (B, w.s_q, w.h_q, D_QK))
    npages = [(L + PAGE - 1) // PAGE for L in seqlens]
    P_used = int(sum(npages))
    P = P_used + extra_pages
    perm = rng.permutation(P)
    max_pages = max(1, max(npages))
    bt = np.full((B, max_pages), -1, dtype=np.int32)
    off = 0
    for b in range(B):
        bt[b, :npages[b]] = perm[off:off + npages[b]]
        off += npages[b]
    if w.kv == "nvfp4":
        kc, kv_scale = quantize_nvfp4(_normal_f32(rng, (P, PAGE, NVFP4_D)))
        if poison_tail:   # UE4M3 0x7F is NaN: every value of a poisoned token is NaN
            for b in range(B):
                if npages[b] and seqlens[b] % PAGE:
                    kv_scale[int(bt[b, npages[b] - 1]), seqlens[b] % PAGE:] = 0x7F
            for p in perm[P_used:]:
                kv_scale[int(p)] = 0x7F
    elif w.kv == "bf16":
        kc = _normal_bf16(rng, (P, PAGE, 1, D_QK))
        if poison_tail:
            nan = torch.tensor(float("nan"), dtype=torch.bfloat16)
            for b in range(B):
                if npages[b] and seqlens[b] % PAGE:
                    kc[int(bt[b, npages[b] - 1]), seqlens[b] % PAGE:] = nan
            for p in perm[P_used:]:
                kc[int(p)] = nan
    else:
        src = _normal_f32(rng, (P, PAGE, D_QK))
        kc = quantize_fp8_records(src)
        if poison_tail:
            for b in range(B):
                if npages[b] and seqlens[b] % PAGE:
                    kc[int(bt[b, npages[b] - 1]), seqlens[b] % PAGE:, :D_V] = 0x7F  # e4m3 NaN
            for p in perm[P_used:]:
                kc[int(p), :, :D_V] = 0x7F
    idx = None
    if w.topk:
        idx = np.empty((B, w.s_q, w.topk), dtype=np.int32)
        n_neg = int(w.topk * w.neg_frac)
        for b in range(B):
            for i in range(w.s_q):
                sel = rng.choice(seqlens[b], size=min(w.topk, seqlens[b]), replace=False)
                row = np.full(w.topk, -1, dtype=np.int32)
                row[:sel.size] = sel
                if n_neg:
                    row[rng.choice(w.topk, size=n_neg, replace=False)] = -1
                idx[b, i] = row
        idx = torch.from_numpy(idx)
    return DecodeInputs(
        workload=w, q=q, kcache=kc, block_table=torch.from_numpy(bt),
        cache_seqlens=torch.tensor(seqlens, dtype=torch.int32), indices=idx,
        extra={"pages_per_request": npages}, q_scale=q_scale, kv_scale=kv_scale)


def make_sink(h_q: int, seed: int) -> torch.Tensor:
    """Per-head attention-sink logits [h_q] fp32, N(0, 1) + 1 (the scale of the
    scores scale * q.k with unit-variance q and k), seeded."""
    rng = np.random.Generator(np.random.PCG64(seed + 101))
    return torch.from_numpy((rng.standard_normal(h_q) + 1.0).astype(np.float32))


def with_sink(inp: "DecodeInputs", seed: int = 0) -> "DecodeInputs":
    """The same inputs with seeded per-head sink logits attached."""
    import dataclasses
    return dataclasses.replace(inp, sink=make_sink(inp.workload.h_q, seed))


def algorithmic_work(inp: DecodeInputs) -> dict:
    """FLOPs and bytes the method must do for one decode call.

    FLOPs = 2 * sum over (request, query row, head) of |key set| * (d_qk + 512)
    (d_qk 576, or 512 for NVFP4 rows), counting only unmasked, non-ignored
    keys. Bytes = distinct cache rows touched (1152 B bf16 / 656 B fp8 / 288 B
    nvfp4) + q + out + lse + block table, seqlens and indices read.
    """
    w = inp.workload
    seqlens = inp.cache_seqlens.tolist()
    row_bytes = {"bf16": 2 * D_QK, "fp8": FP8_RECORD_BYTES, "nvfp4": NVFP4_D // 2 + NVFP4_D // NVFP4_BLOCK}[w.kv]
    d_qk = w.d_qk
    q_bytes = 2 * D_QK if w.kv != "nvfp4" else NVFP4_D // 2 + NVFP4_D // NVFP4_BLOCK
    keys = 0
    touched = 0
    if w.topk:
        idx = inp.indices.numpy()
        for b in range(w.batch):
            valid_all = []
            for i in range(w.s_q):
                r = idx[b, i]
                v = r[(r >= 0) & (r < seqlens[b])]
                keys += v.size * w.h_q
                valid_all.append(v)
            touched += np.unique(np.concatenate(valid_all)).size
    else:
        for b in range(w.batch):
            L = seqlens[b]
            touched += L
            for i in range(w.s_q):
                lim = L - w.s_q + i + 1 if w.causal else L
                keys += max(0, min(L, lim)) * w.h_q
    flops = 2.0 * keys * (d_qk + D_V)
    rows = w.batch * w.s_q * w.h_q
    byts = touched * row_bytes + rows * (q_bytes + 2 * D_V + 4)
    if w.topk:
        byts += inp.indices.numel() * 4 + keys // max(1, w.h_q) * 4   # indices + one page lookup each
    else:
        byts += sum((L + PAGE - 1) // PAGE for L in seqlens) * 4       # block-table entries read
    byts += w.batch * 4                                               # cache_seqlens
    return {"flops": flops, "bytes": float(byts), "keys": keys, "tokens_touched": touched}


def restrict(inp: DecodeInputs, requests) -> DecodeInputs:
    """Sub-problem with only the given requests and only their pages (block
    table remapped). Each request's key set and values are unchanged, so a
    sampled check or a bounded CPU-baseline sample can run on it without
    touching the whole cache."""
    import dataclasses
    requests = list(requests)
    bt = inp.block_table.numpy()
    lens = inp.cache_seqlens.numpy()
    pages = []
    new_bt = np.full((len(requests), bt.shape[1]), -1, dtype=np.int32)
    for i, b in enumerate(requests):
        n = (int(lens[b]) + PAGE - 1) // PAGE
        for j in range(n):
            new_bt[i, j] = len(pages)
            pages.append(int(bt[b, j]))
    sub_lens = [int(lens[b]) for b in requests]
    w = dataclasses.replace(inp.workload, batch=len(requests), seqlens=sub_lens)
    return DecodeInputs(
        workload=w, q=inp.q[requests].clone(), kcache=inp.kcache[pages].clone(),
        block_table=torch.from_numpy(new_bt), cache_seqlens=torch.tensor(sub_lens, dtype=torch.int32),
        indices=None if inp.indices is None else inp.indices[requests].clone(),
        sink=inp.sink, q_scale=None if inp.q_scale is None else inp.q_scale[requests].clone(),
        kv_scale=None if inp.kv_scale is None else inp.kv_scale[pages].clone())


def rope_tables(cache_seqlens, s_q: int, base: float = 10000.0):
    """cos/sin [batch * s_q, 32] fp32 of the RoPE angles of every query token:
    the s_q queries of request b sit at positions seqlen_b - s_q + i (the
    request's last tokens), pair p turns by position * base^(-2p/64). Input
    data for the query pre-step and the output epilogue (the caller supplies
    the angles), not part of either computation."""
    lens = np.asarray(cache_seqlens, dtype=np.float64).reshape(-1)
    pos = lens[:, None] - s_q + np.arange(s_q)[None, :]
    inv = base ** (-2.0 * np.arange(32) / 64.0)
    ang = pos.reshape(-1, 1) * inv[None, :]
    return (torch.from_numpy(np.cos(ang).astype(np.float32)), torch.from_numpy(np.sin(ang).astype(np.float32)))


def norm_weight(d: int, seed: int) -> torch.Tensor:
    """A seeded per-dimension RMS-norm weight, U(0.5, 1.5), fp32 [d]."""
    return torch.from_numpy(_rng(seed).uniform(0.5, 1.5, size=d).astype(np.float32))
