"""fp64 CPU oracle for MLA decoding over a paged latent KV cache.

TEST INFRASTRUCTURE. Only ``tests/``, ``__graft_entry__.smoke()`` and
``bench.py``'s cpu_baseline / reference legs may import or run anything in this
directory. The CUDA path never calls it and shares no code with it.

What it computes (plain definition, no tiling, no online softmax). For request
b, query token i in [0, s_q) and head h:
  key set T  dense : { t : 0 <= t < seqlen_b }, and with the causal mask also
                     t <= seqlen_b - s_q + i (the s_q queries are the request's
                     last tokens);
             sparse: the multiset { indices[b, i, k] : entry != -1 }.
  row(t)   = cache[block_table[b, t // 64], t % 64, :]   (576 values)
  s_t      = scale * <q[b, i, h, :], row(t)>             (K = all 576 dims)
  m        = max_t s_t,   l = sum_t exp(s_t - m)
  out      = sum_t exp(s_t - m) * row(t)[:512] / l        (V = first 512 dims)
  lse      = m + ln(l)                                    (natural log)
  empty T  : out = 0, lse = -inf   (the pages say nothing; chosen reading)
  sink     : optional per-head logit sigma_h in the units of s_t; it joins the
             softmax denominator as one more key whose value vector is zero:
             m = max(max_t s_t, sigma), l = sum_t exp(s_t - m) + exp(sigma - m),
             out as above over this l, lse = m + ln(l); with an empty T,
             out = 0 and lse = sigma. (FlashInfer page, section 2: "an
             optional per-head attention sink", sinks [num_heads] float32;
             its exact use is not given, this is the plainest reading.)

Passages followed:
  * FlashMLA-ETAP (gist.science summary), "핵심 메커니즘" (core mechanism):
    S = Q K^T, P = softmax(S), O = P V.
  * "[flashinfer] FlashInfer, NVFP4를 활용한 DeepSeek-V4 디코딩 성능 최적화",
    section 2 (README of nvfp4_mla_decode): one latent row per token is both K
    and V, 64-token pages, causal mask inside the q_len block against the
    request's last tokens, natural-log FP32 LSE; tensor table (block_tables
    [batch, max_pages], seq_lens [batch], out [.., 512] bf16, lse fp32).
  * "Qu'est-ce que FlashMLA ?" (topnet.top), "Exécuter le décodage MLA": the
    decode call takes q, the paged cache, block_table, cache_seqlens, dv and
    causal.
  * deepseek-ai/FlashMLA (agentlenshq), "기술적 세부 사항": indices entries of
    -1 are ignored; FP8 cache = quantised values plus per-token scale factors.
  * DeepSeek MLA geometry (FlashMLA-ETAP summary, limitations paragraph): 576
    head dimension; the value part is the first 512 dims (dv = 512).

Readings where the pages are silent:
  * sparse indices are logical token positions of request b, resolved through
    the block table; valid range [0, seqlen_b); any other value except -1 is
    ignored and reported as out of range; duplicates count twice.
  * FP8 record = [512 e4m3 | 4 fp32 scales | 64 bf16 RoPE]; the dequantised
    value is bf16_RNE(fp32(e4m3) * scale) with the fp32 product rounded to
    nearest; the oracle then uses those values exactly in fp64.
  * NVFP4 ("[flashinfer] FlashInfer, NVFP4를 활용한 DeepSeek-V4 디코딩 성능
    최적화", section 2, the nvfp4_mla_decode README and its tensor table): the
    query and the cache rows are 512 values each (d_qk = d_v = 512: the whole
    row is K and V), E2M1 codes packed two per byte (256 bytes per row) with
    one UE4M3 scale per block of 16 values (32 bytes per row). Readings: byte
    i holds element 2i in its low nibble and 2i+1 in its high nibble; scale
    byte j applies to elements [16j, 16j+16); UE4M3 is E4M3 without the sign
    bit (bit 7 is not part of the format and is ignored); the value is
    e2m1(code) * ue4m3(scale), used exactly. The pages' kernel rounds P and a
    requantised V to FP8 on the way; the oracle is the attention of the
    dequantised values themselves.
"""
from __future__ import annotations

import numpy as np

PAGE = 64
D_QK = 576
D_V = 512
FP8_TILE = 128
FP8_RECORD_BYTES = 656


# --------------------------------------------------------------------------
# exact storage-format conversions
# --------------------------------------------------------------------------
def bf16_bits_to_f64(bits) -> np.ndarray:
    """bf16 bit patterns (uint16) -> fp64. bf16 is the top half of an fp32."""
    b = np.asarray(bits).astype(np.uint32) << np.uint32(16)
    return b.view(np.float32).astype(np.float64)


def torch_bf16_to_f64(t) -> np.ndarray:
    """A torch bfloat16 tensor -> fp64 numpy array, via its bit patterns."""
    import torch
    assert t.dtype == torch.bfloat16
    return bf16_bits_to_f64(t.contiguous().view(torch.int16).numpy().view(np.uint16))


def f32_round_to_bf16(x) -> np.ndarray:
    """fp32 -> nearest bf16 value (ties to even), returned as fp32.

    Round-to-nearest-even on the 16 dropped mantissa bits; NaN stays NaN.
    """
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32).astype(np.uint64)
    lsb = (u >> np.uint64(16)) & np.uint64(1)
    r = ((u + np.uint64(0x7FFF) + lsb) & np.uint64(0xFFFF0000)).astype(np.uint32)
    out = r.view(np.float32).copy()
    nan = np.isnan(x)
    out[nan] = np.nan
    return out


def e4m3_to_f64(codes) -> np.ndarray:
    """OCP FP8 E4M3 ("fn": no infinities) code -> value.

    sign bit 7, exponent bits 6..3 (bias 7), mantissa bits 2..0.
    exponent 0: subnormal, value = m/8 * 2^-6; exponent 15 with mantissa 7:
    NaN; otherwise (1 + m/8) * 2^(e-7). Largest finite magnitude 448.
    """
    c = np.asarray(codes).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = c & 0x7
    val = np.where(e == 0, (m / 8.0) * 2.0 ** -6, (1.0 + m / 8.0) * np.exp2(e - 7.0))
    val = sign * val
    return np.where((e == 15) & (m == 7), np.nan, val)


def e2m1_to_f64(codes) -> np.ndarray:
    """OCP FP4 E2M1 code (low 4 bits) -> value: sign bit 3, exponent bits 2..1
    (bias 1), mantissa bit 0; exponent 0 is subnormal (m * 0.5), otherwise
    2^(e-1) * (1 + m/2). Magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6."""
    c = np.asarray(codes).astype(np.int64) & 0xF
    sign = np.where(c & 0x8, -1.0, 1.0)
    e = (c >> 1) & 0x3
    m = c & 0x1
    mag = np.where(e == 0, 0.5 * m, np.exp2(e - 1.0) * (1.0 + 0.5 * m))
    return sign * mag


def ue4m3_to_f64(codes) -> np.ndarray:
    """UE4M3 scale byte -> value: the E4M3 value of the low 7 bits (no sign)."""
    return e4m3_to_f64(np.asarray(codes).astype(np.int64) & 0x7F)


NVFP4_BLOCK = 16


def dequant_nvfp4(packed, scales) -> np.ndarray:
    """uint8 packed E2M1 [..., n/2] and UE4M3 block scales [..., n/16] -> fp64
    [..., n]: element 2i is the low nibble of byte i, 2i+1 the high nibble;
    element d is scaled by scale byte d // 16."""
    pk = np.asarray(packed, dtype=np.uint8)
    codes = np.stack([pk & 0xF, pk >> 4], axis=-1).reshape(*pk.shape[:-1], 2 * pk.shape[-1])
    sc = ue4m3_to_f64(np.asarray(scales, dtype=np.uint8))
    return e2m1_to_f64(codes) * np.repeat(sc, NVFP4_BLOCK, axis=-1)


def dequant_fp8_records(records) -> np.ndarray:
    """uint8 [P, 64, 656] token records -> fp64 [P, 64, 576] dequantised rows.

    latent d (< 512): bf16_RNE(fp32(e4m3(code_d)) * scale[d // 128]) with the
    fp32 product rounded to nearest; RoPE dims 512..575: the stored bf16.
    """
    rec = np.ascontiguousarray(np.asarray(records, dtype=np.uint8))
    P = rec.shape[0]
    codes = rec[..., :D_V]
    scales = rec[..., D_V:D_V + 16].copy().view(np.float32)            # [P,64,4]
    rope_bits = rec[..., D_V + 16:].copy().view(np.uint16)               # [P,64,64]
    val = e4m3_to_f64(codes).astype(np.float32)                          # exact
    sc = np.repeat(scales, FP8_TILE, axis=-1)                            # [P,64,512]
    prod = (val * sc).astype(np.float32)                                 # fp32 RN product
    lat = f32_round_to_bf16(prod).astype(np.float64)
    out = np.empty((P, PAGE, D_QK), dtype=np.float64)
    out[..., :D_V] = lat
    out[..., D_V:] = bf16_bits_to_f64(rope_bits)
    return out


# --------------------------------------------------------------------------
# the attention definition
# --------------------------------------------------------------------------
def attend(q_rows, keys, scale, d_v=D_V, sink=None):
    """softmax(scale * q_rows @ keys^T) @ keys[:, :d_v] and its natural-log LSE.

    q_rows [R, d_qk], keys [T, d_qk] (T may be 0), sink None or [R] logits
    (an extra zero-value key per row). Returns (out [R, d_v], lse [R]).
    Empty key set: out 0, lse -inf (lse = sink with a sink).
    """
    q_rows = np.asarray(q_rows, dtype=np.float64)
    keys = np.asarray(keys, dtype=np.float64)
    R = q_rows.shape[0]
    sk = None if sink is None else np.asarray(sink, dtype=np.float64).reshape(R)
    if keys.shape[0] == 0:
        return np.zeros((R, d_v)), (np.full(R, -np.inf) if sk is None else sk.copy())
    s = scale * (q_rows @ keys.T)                        # [R, T]
    m = s.max(axis=1, keepdims=True)
    if sk is not None:
        m = np.maximum(m, sk[:, None])
    e = np.exp(s - m)
    l = e.sum(axis=1, keepdims=True)
    if sk is not None:
        l = l + np.exp(sk[:, None] - m)
    out = (e @ keys[:, :d_v]) / l
    lse = m[:, 0] + np.log(l[:, 0])
    return out, lse


def gather_rows(cache_f64, block_table_row, positions):
    """Rows of logical token positions of one request, through its block table.

    cache_f64 [P, 64, d_qk]; block_table_row [max_pages]; positions int array.
    """
    positions = np.asarray(positions, dtype=np.int64)
    pages = np.asarray(block_table_row, dtype=np.int64)[positions // PAGE]
    return cache_f64[pages, positions % PAGE]


def cache_to_f64(kcache) -> np.ndarray:
    """Decode the cache storage (torch bf16 [P,64,1,576] or uint8 fp8 records)."""
    import torch
    if isinstance(kcache, torch.Tensor) and kcache.dtype == torch.bfloat16:
        c = torch_bf16_to_f64(kcache)
        return c.reshape(c.shape[0], PAGE, -1)
    arr = kcache.numpy() if hasattr(kcache, "numpy") else np.asarray(kcache)
    if arr.dtype == np.uint8:
        return dequant_fp8_records(arr.reshape(arr.shape[0], PAGE, FP8_RECORD_BYTES))
    arr = np.asarray(arr, dtype=np.float64)
    return arr.reshape(arr.shape[0], PAGE, -1)


def decode_dense(q, cache_f64, block_table, cache_seqlens, scale, causal,
                 d_v=D_V, requests=None, sink=None):
    """Dense paged MLA decode. q [B, s_q, h_q, d_qk] (fp64 values).

    Returns out [B, s_q, h_q, d_v] and lse [B, s_q, h_q] (requests not in
    ``requests`` are left NaN when a subset is asked for).
    """
    q = np.asarray(q, dtype=np.float64)
    B, s_q, h_q, _ = q.shape
    bt = np.asarray(block_table)
    lens = np.asarray(cache_seqlens, dtype=np.int64)
    out = np.full((B, s_q, h_q, d_v), np.nan)
    lse = np.full((B, s_q, h_q), np.nan)
    for b in (range(B) if requests is None else requests):
        L = int(lens[b])
        keys_all = gather_rows(cache_f64, bt[b], np.arange(L))
        for i in range(s_q):
            n = L
            if causal:
                n = max(0, min(L, L - s_q + i + 1))
            o, l_ = attend(q[b, i], keys_all[:n], scale, d_v, sink)
            out[b, i], lse[b, i] = o, l_
    return out, lse


def sparse_key_positions(index_row, seqlen):
    """Kept positions of one indices row, and the slots that were ignored.

    -1 is ignored; any other value outside [0, seqlen) is ignored and counted
    as out of range. Returns (positions, ignored_slots, out_of_range_slots).
    """
    r = np.asarray(index_row, dtype=np.int64)
    valid = (r >= 0) & (r < seqlen)
    oob = ~valid & (r != -1)
    return r[valid], np.nonzero(~valid)[0], np.nonzero(oob)[0]


def decode_sparse(q, cache_f64, block_table, cache_seqlens, indices, scale,
                  d_v=D_V, requests=None, sink=None):
    """Token-sparse paged MLA decode; key set per (b, i) from indices[b, i]."""
    q = np.asarray(q, dtype=np.float64)
    B, s_q, h_q, _ = q.shape
    bt = np.asarray(block_table)
    lens = np.asarray(cache_seqlens, dtype=np.int64)
    idx = np.asarray(indices)
    out = np.full((B, s_q, h_q, d_v), np.nan)
    lse = np.full((B, s_q, h_q), np.nan)
    for b in (range(B) if requests is None else requests):
        for i in range(s_q):
            pos, _, _ = sparse_key_positions(idx[b, i], int(lens[b]))
            keys = gather_rows(cache_f64, bt[b], pos)
            o, l_ = attend(q[b, i], keys, scale, d_v, sink)
            out[b, i], lse[b, i] = o, l_
    return out, lse


def combine(o_parts, lse_parts, sink=None):
    """Merge attention results of disjoint key subsets (split-KV reduction).

    o_parts [n, R, d] (each normalised over its own subset), lse_parts [n, R].
    L = ln sum_s exp(lse_s); out = sum_s exp(lse_s - L) o_s. All parts empty:
    out 0, lse -inf. A sink [R] enters as one more part with lse = sink and
    a zero output.
    (FlashInfer PR #5443 analysis, section 3: a split-KV combine kernel merges
    the partial results of CTAs that split one request's KV.)
    """
    o_parts = np.asarray(o_parts, dtype=np.float64)
    lse_parts = np.asarray(lse_parts, dtype=np.float64)
    if sink is not None:
        sk = np.asarray(sink, dtype=np.float64).reshape(1, -1)
        o_parts = np.concatenate([o_parts, np.zeros((1,) + o_parts.shape[1:])], axis=0)
        lse_parts = np.concatenate([lse_parts, sk], axis=0)
    mx = lse_parts.max(axis=0)
    finite = np.isfinite(mx)
    mxs = np.where(finite, mx, 0.0)
    w = np.exp(lse_parts - mxs)                     # exp(-inf) = 0 for empty parts
    tot = w.sum(axis=0)
    L = np.where(finite, mxs + np.log(np.where(finite, tot, 1.0)), -np.inf)
    wn = np.where(finite, w / np.where(finite, tot, 1.0), 0.0)
    out = np.einsum("nr,nrd->rd", wn, o_parts)
    return out, L


def inputs_to_f64(inp):
    """(q fp64, cache fp64) from a workloads.DecodeInputs."""
    if inp.workload.kv == "nvfp4":
        return (dequant_nvfp4(inp.q.numpy(), inp.q_scale.numpy()),
                dequant_nvfp4(inp.kcache.numpy(), inp.kv_scale.numpy()))
    return torch_bf16_to_f64(inp.q), cache_to_f64(inp.kcache)


def reference_decode(inp, requests=None):
    """Run the oracle on a workloads.DecodeInputs; returns (out, lse) fp64."""
    w = inp.workload
    q, cache = inputs_to_f64(inp)
    sink = None if getattr(inp, "sink", None) is None else inp.sink.double().numpy()
    if w.topk:
        return decode_sparse(q, cache, inp.block_table.numpy(), inp.cache_seqlens.numpy(),
                             inp.indices.numpy(), w.scale, requests=requests, sink=sink)
    return decode_dense(q, cache, inp.block_table.numpy(), inp.cache_seqlens.numpy(),
                        w.scale, w.causal, requests=requests, sink=sink)


# --------------------------------------------------------------------------
# the steps around the attention: query norm + RoPE, output conjugate RoPE +
# FP8 cast ("deepseek-ai/FlashMLA" (agentlenshq), feature list: a fused kernel
# runs Q-norm, RoPE, the attention, the output-side conjugate RoPE and the
# final FP8 cast in one launch). The page gives the order of the steps only;
# the readings below are the plainest ones and are shared with the design doc:
#   * Q-norm = RMS normalisation of each query row (one head of one query
#     token) over all of its d_qk values, times a per-dimension weight gamma:
#     q / sqrt(mean(q^2) + eps) * gamma.
#   * RoPE acts on the last 64 dims of a row (the RoPE part of the 576-dim
#     latent row, or of a 512-dim NVFP4 row) and rotates consecutive pairs
#     (x[2i], x[2i+1]) by the angle theta_i of the query token's position:
#     (x0 cos - x1 sin, x0 sin + x1 cos). The caller gives cos/sin per query
#     token and pair, [B, s_q, 32].
#   * The output's RoPE part is the part of V that lies in those dims: none
#     for 576-dim rows (V = dims 0..511), dims 448..511 for 512-dim rows. It
#     is rotated back by the same angle (the conjugate rotation).
#   * FP8 cast: per 128-value tile of the 512-dim output row, scale =
#     amax / 448 (1 if amax = 0) and code = e4m3 round-to-nearest-even of
#     value / scale, saturated to +-448. These integer decisions are taken
#     in fp32 with every product, sum and quotient rounded once, the
#     precision of the kernel (the page fixes none).
# --------------------------------------------------------------------------
ROPE_DIMS = 64
E4M3_MAX = 448.0


def rms_norm(x, gamma, eps):
    """x / sqrt(mean(x^2, last axis) + eps) * gamma, in fp64."""
    x = np.asarray(x, dtype=np.float64)
    ms = np.mean(x * x, axis=-1, keepdims=True)
    return x / np.sqrt(ms + float(eps)) * np.asarray(gamma, dtype=np.float64)


def rope_rotate(x, cos, sin, conjugate=False):
    """Rotate consecutive pairs (x[..., 2i], x[..., 2i+1]) by theta_i, given
    cos/sin [..., n/2] (broadcast against x's leading axes); the conjugate
    rotation turns by -theta_i. fp64."""
    x = np.asarray(x, dtype=np.float64)
    c = np.asarray(cos, dtype=np.float64)
    s = np.asarray(sin, dtype=np.float64)
    if conjugate:
        s = -s
    x0, x1 = x[..., 0::2], x[..., 1::2]
    y = np.empty(np.broadcast(x, np.repeat(c, 2, axis=-1)).shape)
    y[..., 0::2] = x0 * c - x1 * s
    y[..., 1::2] = x0 * s + x1 * c
    return y


def q_norm_rope(q, gamma, eps, cos, sin):
    """q [B, s_q, h_q, d] -> RMS-normalised rows (weight gamma [d]) whose last
    ROPE_DIMS dims are rotated by the query token's angles (cos/sin
    [B, s_q, 32]). fp64."""
    y = rms_norm(q, gamma, eps)
    y[..., -ROPE_DIMS:] = rope_rotate(y[..., -ROPE_DIMS:], np.asarray(cos)[:, :, None, :],
                                      np.asarray(sin)[:, :, None, :])
    return y


def e4m3_encode(x) -> np.ndarray:
    """Value (fp64 or fp32) -> OCP E4M3 code: round to the nearest
    representable value, ties to the even code (mantissa bit 0 clear), with
    magnitudes beyond 448 saturated to 448; NaN -> 0x7F. The representable
    magnitudes are m/8 * 2^-6 (m < 8, subnormal) and (1 + m/8) * 2^(e-7)
    (e = 1..15, excluding e = 15, m = 7)."""
    x = np.asarray(x, dtype=np.float64)
    mags = np.array([(m / 8.0) * 2.0 ** -6 for m in range(8)] +
                    [(1.0 + m / 8.0) * 2.0 ** (e - 7) for e in range(1, 16) for m in range(8)
                     if not (e == 15 and m == 7)])          # index = code & 0x7F (0..126)
    a = np.minimum(np.abs(x), E4M3_MAX)
    hi = np.clip(np.searchsorted(mags, a, side="left"), 0, len(mags) - 1)   # first mag >= a
    lo = np.maximum(hi - 1, 0)
    dlo, dhi = a - mags[lo], mags[hi] - a
    pick_hi = (dhi < dlo) | ((dhi == dlo) & (hi % 2 == 0))
    code = np.where(pick_hi, hi, lo)
    code = np.where(a == mags[hi], hi, code).astype(np.int64)
    code = code | np.where(np.signbit(x), 0x80, 0)
    code = np.where(np.isnan(x), 0x7F, code)
    return code.astype(np.uint8)


def _f32(v):
    return np.asarray(v, dtype=np.float32)


def fp8_cast_rows(x, tile=128):
    """fp32 rows [..., n] -> (codes uint8 [..., n], scales fp32 [..., n/tile]).
    Per tile: amax = max |x|, scale = fp32(amax / 448) (1 if amax = 0),
    code = e4m3_encode(fp32(x / scale)); each division rounded once in fp32."""
    x = _f32(x)
    t = x.reshape(*x.shape[:-1], x.shape[-1] // tile, tile)
    amax = np.max(np.abs(t), axis=-1)
    scale = np.where(amax > 0, _f32(amax / np.float32(E4M3_MAX)), np.float32(1.0)).astype(np.float32)
    q = _f32(t / scale[..., None])
    return e4m3_encode(q).reshape(x.shape), scale


def out_rope_fp8(out, cos, sin, d_qk):
    """Output epilogue on [B, s_q, h_q, 512] output values (the bf16 results,
    exact in fp32): the output's RoPE part (dims d_qk-64..d_qk-1 that lie
    below 512: none for d_qk = 576, 448..511 for d_qk = 512) rotated back by
    the query token's angle, in fp32 with every product and sum rounded once
    ((x0 c + x1 s, x1 c - x0 s)), then fp8_cast_rows. Returns (codes, scales,
    rotated fp32 values)."""
    y = _f32(out).copy()
    lo = d_qk - ROPE_DIMS
    if lo < y.shape[-1]:
        c = _f32(cos)[:, :, None, :]
        s = _f32(sin)[:, :, None, :]
        x0 = y[..., lo::2].copy()
        x1 = y[..., lo + 1::2].copy()
        y[..., lo::2] = _f32(_f32(x0 * c) + _f32(x1 * s))
        y[..., lo + 1::2] = _f32(_f32(x1 * c) - _f32(x0 * s))
    codes, scales = fp8_cast_rows(y)
    return codes, scales, y
