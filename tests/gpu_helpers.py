"""Shared helpers for the GPU parity tests: move seeded inputs to the device,
run the decode through the C ABI, and compare with the fp64 oracle.

Tolerances (written here once, used by every parity test): output max-abs
1e-2, LSE max-abs 1e-3, cosine similarity of the flattened output >= 0.99999.
They follow from the arithmetic: scores are bf16 x bf16 products accumulated
in fp32 over 576 dims (relative error ~1e-6 of |q||k|), probabilities are
rounded to bf16 before the PV product (unit roundoff 2^-8 per term, averaging
out over many keys), and the output is rounded to bf16 (half an ulp: at most
2^-7 = 7.8e-3 for |out| < 4, which holds for N(0,1) data averaged over many
keys).
"""
from __future__ import annotations

import numpy as np
import torch

from head_latent_attention_get_b200 import DecodeRunner
from oracle import mla_oracle as O

OUT_ATOL = 1e-2
LSE_ATOL = 1e-3
COS_MIN = 0.99999

# Rows that attend to fewer than FEW_KEYS keys do not average the rounding of
# their probabilities out. There the bf16 arithmetic itself bounds the error
# (bf16 keeps 8 significant bits, unit roundoff u = 2^-8): each probability
# p_t enters the PV product rounded to bf16 (relative error <= u), so the
# normalised sum moves by <= u * max_t |v_t|, and the bf16 output adds
# <= u * |out|. Such a row is held to
#   max(OUT_ATOL, u * (|ref| + 1.01 * vmax) + 1e-4)
# per element, vmax = the largest |value| among its request's tokens (a bound
# on its keys' values). A CPU model of that rounding (fp32 scores, bf16
# probabilities, bf16 output) reproduces the kernel's error on a two-key row
# to the last bit: 0.0108 at |out| = 2.24, |v| <= 2.97.
FEW_KEYS = 16


def to_device(inp, dev="cuda"):
    return dict(
        q=inp.q.to(dev), kcache=inp.kcache.to(dev), block_table=inp.block_table.to(dev),
        cache_seqlens=inp.cache_seqlens.to(dev),
        indices=None if inp.indices is None else inp.indices.to(dev),
        sink=None if getattr(inp, "sink", None) is None else inp.sink.to(dev),
        q_scale=None if inp.q_scale is None else inp.q_scale.to(dev),
        kv_scale=None if inp.kv_scale is None else inp.kv_scale.to(dev))


def run_gpu(inp, runner_kwargs=None, dev_inputs=None):
    d = dev_inputs or to_device(inp)
    w = inp.workload
    r = DecodeRunner(d["q"], d["kcache"], d["block_table"], d["cache_seqlens"], softmax_scale=w.scale,
                     causal=w.causal, indices=d["indices"], sink=d.get("sink"), q_scale=d.get("q_scale"),
                     kv_scale=d.get("kv_scale"), **(runner_kwargs or {}))
    r.plan()
    out, lse = r.run()
    torch.cuda.synchronize()
    return out.float().cpu().numpy(), lse.cpu().numpy(), r


def few_key_bounds(inp, out_ref):
    """Per-element out bound [B, s_q, h_q, 512] (see FEW_KEYS)."""
    w = inp.workload
    lens = inp.cache_seqlens.numpy().astype(np.int64)
    B, s_q = w.batch, w.s_q
    if inp.indices is not None:
        idx = inp.indices.numpy()
        nkeys = ((idx >= 0) & (idx < lens[:, None, None])).sum(axis=2)
    elif w.causal:
        i = np.arange(s_q)[None, :]
        nkeys = np.clip(lens[:, None] - s_q + i + 1, 0, lens[:, None])
    else:
        nkeys = np.repeat(lens[:, None], s_q, axis=1)
    _, cache = O.inputs_to_f64(inp)
    bt = inp.block_table.numpy()
    vmax = np.zeros(B)
    for b in range(B):
        npg = (int(lens[b]) + 63) // 64
        if npg:
            rows = cache[bt[b, :npg]].reshape(npg * 64, -1)[:int(lens[b]), :512]
            vmax[b] = np.abs(rows).max()
    loose = 2.0 ** -8 * (np.abs(out_ref) + 1.01 * vmax[:, None, None, None]) + 1e-4
    few = (nkeys < FEW_KEYS)[:, :, None, None]
    return np.where(few, np.maximum(OUT_ATOL, loose), OUT_ATOL)


def compare(out_gpu, lse_gpu, out_ref, lse_ref, where="", inp=None):
    """Element-wise parity; rows with an empty key set must give out 0, lse -inf.
    With `inp`, rows of fewer than FEW_KEYS keys get the bf16 bound above;
    without it every element is held to OUT_ATOL."""
    out_gpu = np.asarray(out_gpu, dtype=np.float64)
    lse_gpu = np.asarray(lse_gpu, dtype=np.float64)
    assert out_gpu.shape == out_ref.shape, (out_gpu.shape, out_ref.shape)
    empty = np.isneginf(lse_ref)
    assert np.all(np.isneginf(lse_gpu[empty])), f"{where}: empty rows must have lse -inf"
    assert np.all(out_gpu[empty] == 0), f"{where}: empty rows must have out 0"
    assert np.all(np.isfinite(out_gpu)), f"{where}: non-finite output"
    if inp is not None:
        bound = few_key_bounds(inp, out_ref)
        over = np.abs(out_gpu - out_ref) - bound
        assert over.max(initial=-1.0) <= 0, f"{where}: out exceeds the few-key bound by {over.max()}"
        dense_rows = bound == OUT_ATOL
        err_o = np.abs(out_gpu - out_ref)[dense_rows].max(initial=0.0)
    else:
        err_o = np.abs(out_gpu - out_ref).max(initial=0.0)
    err_l = np.abs(lse_gpu[~empty] - lse_ref[~empty]).max(initial=0.0)
    a, b = out_gpu.ravel(), out_ref.ravel()
    cos = float(a @ b / (np.linalg.norm(a) * np.linalg.norm(b) + 1e-300)) if np.any(b) else 1.0
    info = {"out_maxabs": err_o, "lse_maxabs": err_l, "cos": cos}
    assert err_o <= OUT_ATOL, f"{where}: out max-abs {err_o} {info}"
    assert err_l <= LSE_ATOL, f"{where}: lse max-abs {err_l} {info}"
    assert cos >= COS_MIN, f"{where}: cosine {cos} {info}"
    return info


def oracle_for(inp, requests=None):
    return O.reference_decode(inp, requests=requests)


def compare_full(inp, out_gpu, lse_gpu, where, few_keys=False):
    """Every output row of the batch against the oracle (no sampling): the
    oracle runs on all requests, the comparison is element by element with
    the tolerances above (with few_keys, rows of fewer than FEW_KEYS keys get
    the bf16 bound)."""
    ref_o, ref_l = O.reference_decode(inp)
    assert not np.isnan(ref_l).any() and not np.isnan(ref_o).any(), "oracle left rows unset"
    return compare(out_gpu, lse_gpu, ref_o, ref_l, where, inp=inp if few_keys else None)


from workloads.mla_workloads import restrict  # noqa: E402,F401
