"""Shared helpers for the GPU parity tests: move seeded inputs to the device,
run the decode through the C ABI, and compare with the fp64 oracle.

Tolerances (written here once, used by every parity test): output max-abs
1e-2, LSE max-abs 1e-3, cosine similarity of the flattened output >= 0.99999.
They follow from the arithmetic: scores are bf16 x bf16 products accumulated
in fp32 over 576 dims (relative error ~1e-6 of |q||k|), probabilities are
rounded to bf16 before the PV product (relative 2^-9 per term, averaging out
over many keys), and the output is rounded to bf16 (relative 2^-9 of |out|,
|out| <= max |V| ~ 4 for N(0,1) data, i.e. <= 8e-3).
"""
from __future__ import annotations

import numpy as np
import torch

from head_latent_attention_get_b200 import DecodeRunner
from oracle import mla_oracle as O

OUT_ATOL = 1e-2
LSE_ATOL = 1e-3
COS_MIN = 0.99999


def to_device(inp, dev="cuda"):
    return dict(
        q=inp.q.to(dev), kcache=inp.kcache.to(dev), block_table=inp.block_table.to(dev),
        cache_seqlens=inp.cache_seqlens.to(dev),
        indices=None if inp.indices is None else inp.indices.to(dev),
        sink=None if getattr(inp, "sink", None) is None else inp.sink.to(dev))


def run_gpu(inp, runner_kwargs=None, dev_inputs=None):
    d = dev_inputs or to_device(inp)
    w = inp.workload
    r = DecodeRunner(d["q"], d["kcache"], d["block_table"], d["cache_seqlens"], softmax_scale=w.scale,
                     causal=w.causal, indices=d["indices"], sink=d.get("sink"), **(runner_kwargs or {}))
    r.plan()
    out, lse = r.run()
    torch.cuda.synchronize()
    return out.float().cpu().numpy(), lse.cpu().numpy(), r


def compare(out_gpu, lse_gpu, out_ref, lse_ref, where=""):
    """Element-wise parity; rows with an empty key set must give out 0, lse -inf."""
    out_gpu = np.asarray(out_gpu, dtype=np.float64)
    lse_gpu = np.asarray(lse_gpu, dtype=np.float64)
    assert out_gpu.shape == out_ref.shape, (out_gpu.shape, out_ref.shape)
    empty = np.isneginf(lse_ref)
    assert np.all(np.isneginf(lse_gpu[empty])), f"{where}: empty rows must have lse -inf"
    assert np.all(out_gpu[empty] == 0), f"{where}: empty rows must have out 0"
    assert np.all(np.isfinite(out_gpu)), f"{where}: non-finite output"
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


from workloads.mla_workloads import restrict  # noqa: E402,F401
