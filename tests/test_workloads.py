"""Seeded input generators: structure and determinism (CPU only)."""
import dataclasses

import numpy as np
import torch

from workloads import mla_workloads as W
from oracle import mla_oracle as O


def test_named_workloads_shapes():
    ws = {w.name: w for w in W.named_workloads()}
    assert [w.seed for w in W.named_workloads()] == [20260 + i for i in range(5)]
    assert ws["tiny"].seqlens == [70, 129] and ws["tiny"].rows == 16
    assert ws["dsv3"].rows == 128 and set(ws["dsv3"].seqlens) == {4096}
    m = ws["mtp"]
    assert m.rows == 32 and m.causal and m.seqlens[0] == 65536
    assert all(1024 <= L <= 16384 for L in m.seqlens[1:])
    assert ws["fp8"].kv == "fp8" and ws["sparse"].topk == 2048


def test_tiny_inputs_deterministic_and_paged():
    w = W.get_workload("tiny")
    a = W.make_inputs(w)
    b = W.make_inputs(w)
    assert torch.equal(a.q.view(torch.int16), b.q.view(torch.int16))
    assert torch.equal(a.block_table, b.block_table)
    bt = a.block_table.numpy()
    used = bt[bt >= 0]
    assert sorted(used.tolist()) == list(range(a.num_pages))       # every page exactly once
    assert (bt[0, 2:] == -1).all() and bt.shape == (2, 3)


def test_poison_tail_marks_only_unused_tokens():
    w = W.get_workload("tiny")
    a = W.make_inputs(w, poison_tail=True, extra_pages=2)
    c = O.cache_to_f64(a.kcache)
    bt = a.block_table.numpy()
    assert np.isnan(c[bt[0, 1], 6:]).all() and not np.isnan(c[bt[0, 1], :6]).any()
    assert np.isnan(c[bt[1, 2], 1:]).all() and not np.isnan(c[bt[1, 2], :1]).any()
    assert a.num_pages == 7


def test_fp8_records_close_to_source_and_scaled():
    w = dataclasses.replace(W.get_workload("fp8"), batch=2, seqlens=[100, 64])
    a = W.make_inputs(w)
    assert a.kcache.dtype == torch.uint8 and a.kcache.shape[-1] == 656
    rec = a.kcache.numpy()
    scales = rec[..., 512:528].copy().view(np.float32)
    codes = O.e4m3_to_f64(rec[..., :512]).reshape(*rec.shape[:2], 4, 128)
    # every tile uses the full e4m3 range: max |code| hits 448 exactly
    assert np.allclose(np.abs(codes).max(-1), 448.0)
    assert (scales > 0).all()


def test_sparse_indices_distinct_with_holes():
    w = dataclasses.replace(W.get_workload("sparse"), batch=2, seqlens=[4096, 3000], topk=256)
    a = W.make_inputs(w)
    idx = a.indices.numpy()
    for b, L in enumerate([4096, 3000]):
        r = idx[b, 0]
        assert (r == -1).sum() == int(256 * 0.05)
        v = r[r >= 0]
        assert len(set(v.tolist())) == v.size and v.max() < L


def test_algorithmic_work_dsv3_formula():
    w = W.get_workload("tiny")
    a = W.make_inputs(w)
    work = W.algorithmic_work(a)
    assert work["flops"] == 2.0 * (70 + 129) * 16 * (576 + 512)


def test_nvfp4_encoder_round_trips_within_half_a_step():
    """The seeded NVFP4 encoder (data preparation) picks, per value, an E2M1
    code whose decoded value is within half an E2M1 step of x/scale (times the
    block scale), and the block maximum maps to 4..6 before saturation."""
    rng = np.random.default_rng(5)
    x = torch.from_numpy(rng.standard_normal((64, 512)).astype(np.float32))
    packed, scales = W.quantize_nvfp4(x)
    assert packed.shape == (64, 256) and scales.shape == (64, 32) and packed.dtype == torch.uint8
    dec = O.dequant_nvfp4(packed.numpy(), scales.numpy())
    sc = np.repeat(O.ue4m3_to_f64(scales.numpy()), 16, axis=-1)
    y = x.double().numpy() / sc
    # E2M1 magnitudes 0, .5, 1, 1.5, 2, 3, 4, 6: the gap to a neighbour is at most 2
    assert np.all(np.abs(dec / sc - np.clip(y, -6, 6)) <= 1.0 + 1e-12)
    blk_max = np.abs(dec).reshape(64, 32, 16).max(-1) / O.ue4m3_to_f64(scales.numpy())
    assert np.all((blk_max >= 4.0) | (blk_max == 0)) and np.all(blk_max <= 6.0)
    assert np.all(scales.numpy() < 0x7F)                               # finite, unsigned scales
