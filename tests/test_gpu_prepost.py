"""GPU parity of the steps around the attention: the query RMS-norm + RoPE
and the output conjugate RoPE + per-128 e4m3 cast, through the C ABI,
against the fp64 oracle (and, for the FP8 codes, its fp32 decision chain on
the same bf16 inputs: bit for bit)."""
import dataclasses

import numpy as np
import pytest
import torch

import head_latent_attention_get_b200 as M
from head_latent_attention_get_b200 import _capi as C
from oracle import mla_oracle as O
from tests import gpu_helpers as G
from workloads import mla_workloads as W

pytestmark = pytest.mark.gpu


def _bf16_close(gpu, ref):
    """bf16 result of an fp32 computation: within half a bf16 step of the
    exact value (2^-8 relative) plus the fp32 rounding of the norm and the
    rotation (a few 2^-24 of the row's largest magnitude, which also covers
    cancellation inside a rotated pair)."""
    err = np.abs(gpu - ref)
    bound = 2.0 ** -8 * np.abs(ref) + 2.0 ** -19 * np.max(np.abs(ref), axis=-1, keepdims=True)
    assert np.all(err <= bound), f"max excess {np.max(err - bound)}"


@pytest.mark.parametrize("d_qk,B,s_q,h_q,lens", [
    (576, 2, 1, 16, [70, 129]), (576, 8, 1, 128, [4096] * 8), (576, 5, 2, 16, [1024, 70, 5000, 129, 64]),
    (512, 3, 6, 64, [100, 200, 8192])])
def test_q_norm_rope_vs_oracle(d_qk, B, s_q, h_q, lens):
    rng = np.random.default_rng(7 + B)
    q = torch.from_numpy((rng.standard_normal((B, s_q, h_q, d_qk)) *
                          rng.uniform(0.05, 20, size=(B, s_q, h_q, 1))).astype(np.float32)).to(torch.bfloat16)
    cos, sin = W.rope_tables(lens, s_q)
    g = W.norm_weight(d_qk, seed=3)
    qd = q.cuda()
    qo = torch.empty_like(qd)
    M.mla_q_norm_rope(qd, qo, B, s_q, h_q, d_qk, g.cuda(), 1e-6, cos.cuda(), sin.cuda())
    M.mla_q_norm_rope(qd, qd, B, s_q, h_q, d_qk, g.cuda(), 1e-6, cos.cuda(), sin.cuda())  # in place
    torch.cuda.synchronize()
    assert torch.equal(qo, qd)
    ref = O.q_norm_rope(O.torch_bf16_to_f64(q), g.double().numpy(), 1e-6,
                        cos.double().numpy().reshape(B, s_q, 32), sin.double().numpy().reshape(B, s_q, 32))
    _bf16_close(O.torch_bf16_to_f64(qo.cpu()), ref)


@pytest.mark.parametrize("d_qk,rows", [(576, (2, 1, 16)), (512, (3, 2, 64)), (576, (64, 1, 128)),
                                       (512, (32, 6, 64))])
def test_out_rope_fp8_bit_exact(d_qk, rows):
    B, s_q, h_q = rows
    rng = np.random.default_rng(11 + B)
    out = torch.from_numpy((rng.standard_normal((B, s_q, h_q, 512)) *
                            rng.uniform(0.01, 3, size=(B, s_q, h_q, 1))).astype(np.float32)).to(torch.bfloat16)
    out[0, 0, 0, 128:256] = 0                      # an all-zero tile: scale 1, codes 0
    th = rng.uniform(-20, 20, size=(B * s_q, 32))
    cos = torch.from_numpy(np.cos(th).astype(np.float32))
    sin = torch.from_numpy(np.sin(th).astype(np.float32))
    o8 = torch.empty((B, s_q, h_q, 512), dtype=torch.uint8, device="cuda")
    sc = torch.empty((B, s_q, h_q, 4), dtype=torch.float32, device="cuda")
    M.mla_out_rope_fp8(out.cuda(), B, s_q, h_q, d_qk, cos.cuda(), sin.cuda(), o8, sc)
    torch.cuda.synchronize()
    codes, scales, _ = O.out_rope_fp8(O.torch_bf16_to_f64(out).astype(np.float32), cos.numpy().reshape(B, s_q, 32),
                                      sin.numpy().reshape(B, s_q, 32), d_qk)
    assert np.array_equal(sc.cpu().numpy().view(np.uint32), scales.view(np.uint32))
    assert np.array_equal(o8.cpu().numpy(), codes)


def test_chain_q_norm_rope_decode_out_fp8():
    """q -> RMS-norm + RoPE -> paged decode (CTA pairs, 128 heads) -> output
    cast, end to end against the oracle's chain in fp64: the dequantised FP8
    output within half an e4m3 step (2^-4 relative) plus the decode
    tolerance."""
    w = dataclasses.replace(W.get_workload("dsv3"), batch=4, seqlens=[300, 4096, 129, 1000], seed=91)
    inp = W.make_inputs(w, poison_tail=True)
    cos, sin = W.rope_tables(inp.cache_seqlens.numpy(), w.s_q)
    g = W.norm_weight(576, seed=5)
    d = G.to_device(inp)
    M.mla_q_norm_rope(d["q"], d["q"], w.batch, w.s_q, w.h_q, 576, g.cuda(), 1e-6, cos.cuda(), sin.cuda())
    r = M.DecodeRunner(d["q"], d["kcache"], d["block_table"], d["cache_seqlens"], softmax_scale=w.scale)
    r.plan()
    out, lse = r.run()
    o8 = torch.empty((w.batch, 1, w.h_q, 512), dtype=torch.uint8, device="cuda")
    sc = torch.empty((w.batch, 1, w.h_q, 4), dtype=torch.float32, device="cuda")
    M.mla_out_rope_fp8(out, w.batch, 1, w.h_q, 576, cos.cuda(), sin.cuda(), o8, sc)
    torch.cuda.synchronize()
    qn = O.q_norm_rope(O.torch_bf16_to_f64(inp.q), g.double().numpy(), 1e-6, cos.double().numpy().reshape(4, 1, 32),
                       sin.double().numpy().reshape(4, 1, 32))
    _, cache = O.inputs_to_f64(inp)
    ref_o, ref_l = O.decode_dense(qn, cache, inp.block_table.numpy(), inp.cache_seqlens.numpy(), w.scale, False)
    deq = O.e4m3_to_f64(o8.cpu().numpy()) * np.repeat(sc.cpu().numpy(), 128, axis=-1)
    tol = 2.0 ** -4 * np.abs(ref_o) + 2.0 ** -10 * np.repeat(sc.cpu().numpy(), 128, axis=-1) + 2e-2
    assert np.all(np.abs(deq - ref_o) <= tol)
    # the bf16 output of the same chain is within the decode tolerance
    G.compare(out.float().cpu().numpy(), lse.cpu().numpy(), ref_o, ref_l, "chain")
