"""Plant plausible mistakes in the oracle (on the CPU) and check that at least
one pin catches each of them. This shows the pins are tight enough that a
dropped term, a wrong sign or index, or a transposed operand cannot pass."""
import numpy as np
import pytest

from oracle import mla_oracle as O
from tests import oracle_checks as C

real_attend = O.attend


def _attend_no_scale(q, k, scale, d_v=512):
    return real_attend(q, k, 1.0, d_v)


def _attend_neg(q, k, scale, d_v=512):
    return real_attend(q, k, -scale, d_v)


def _attend_shifted_v(q, k, scale, d_v=512):
    q = np.asarray(q, float)
    k = np.asarray(k, float)
    if k.shape[0] == 0:
        return np.zeros((q.shape[0], d_v)), np.full(q.shape[0], -np.inf)
    s = scale * q @ k.T
    m = s.max(1, keepdims=True)
    e = np.exp(s - m)
    v = np.roll(k, -1, axis=1)[:, :d_v]            # off-by-one value slice
    return (e @ v) / e.sum(1, keepdims=True), (m + np.log(e.sum(1, keepdims=True)))[:, 0]


def _attend_lse_is_max(q, k, scale, d_v=512):
    o, l = real_attend(q, k, scale, d_v)
    s = scale * np.asarray(q, float) @ np.asarray(k, float).T
    return o, (s.max(1) if s.shape[1] else l)


def _attend_log2(q, k, scale, d_v=512):
    o, l = real_attend(q, k, scale, d_v)
    return o, l / np.log(2.0)


def _attend_unnormalised(q, k, scale, d_v=512):
    o, l = real_attend(q, k, scale, d_v)
    s = scale * np.asarray(q, float) @ np.asarray(k, float).T
    if s.shape[1] == 0:
        return o, l
    return o * np.exp(s - s.max(1, keepdims=True)).sum(1, keepdims=True), l


ATTEND_MUTANTS = [_attend_no_scale, _attend_neg, _attend_shifted_v, _attend_lse_is_max,
                  _attend_log2, _attend_unnormalised]


def _fails(fn, *a):
    try:
        fn(*a)
    except AssertionError:
        return True
    return False


@pytest.mark.parametrize("mutant", ATTEND_MUTANTS, ids=lambda f: f.__name__)
def test_attend_mutants_caught(mutant, monkeypatch):
    caught = _fails(C.check_brute_force_attend, mutant)
    monkeypatch.setattr(O, "attend", mutant)
    caught = caught or _fails(C.check_single_token, O.decode_dense)
    caught = caught or _fails(C.check_lse_logsumexp, O.decode_dense)
    assert caught


def test_causal_off_by_one_caught(monkeypatch):
    def decode_dense_bad(q, cache, bt, lens, scale, causal, d_v=512, requests=None):
        # causal bound one token too short
        if causal:
            lens = np.asarray(lens)
            q = np.asarray(q, float)
            out, lse = O.decode_dense(q, cache, bt, lens, scale, False, d_v)
            for b in range(q.shape[0]):
                for i in range(q.shape[1]):
                    n = max(0, min(int(lens[b]), int(lens[b]) - q.shape[1] + i))
                    keys = O.gather_rows(cache, bt[b], np.arange(n))
                    out[b, i], lse[b, i] = O.attend(q[b, i], keys, scale, d_v)
            return out, lse
        return O.decode_dense(q, cache, bt, lens, scale, causal, d_v)
    assert _fails(C.check_brute_force_paged, decode_dense_bad, True)
    assert _fails(C.check_causal_row0, decode_dense_bad)


def test_page_lookup_mistake_caught(monkeypatch):
    def gather_bad(cache, bt_row, positions):
        positions = np.asarray(positions, dtype=np.int64)
        pages = np.asarray(bt_row)[positions % len(bt_row)]        # wrong page index
        return cache[pages, positions % 64]
    monkeypatch.setattr(O, "gather_rows", gather_bad)
    assert _fails(C.check_brute_force_paged, O.decode_dense, False)


def test_sparse_minus_one_mistake_caught(monkeypatch):
    def keys_bad(index_row, seqlen):
        r = np.asarray(index_row, dtype=np.int64)
        keep = r < seqlen                                   # -1 not excluded
        return np.where(r[keep] < 0, seqlen - 1, r[keep]), np.array([], int), np.array([], int)
    monkeypatch.setattr(O, "sparse_key_positions", keys_bad)
    assert _fails(C.check_sparse, O.decode_sparse, O.decode_dense)


def test_combine_mistake_caught():
    def combine_bad(o_parts, lse_parts):
        return np.asarray(o_parts).mean(0), np.asarray(lse_parts).max(0)
    assert _fails(C.check_combine, O.attend, combine_bad)


def test_e4m3_bias_mistake_caught():
    def e4m3_bad(codes):
        c = np.asarray(codes).astype(np.int64)
        e = (c >> 3) & 0xF
        m = c & 7
        v = np.where(e == 0, m / 8.0 * 2.0 ** -7, (1 + m / 8.0) * np.exp2(e - 8.0))
        return np.where(c & 0x80, -v, v)
    assert _fails(C.check_e4m3, e4m3_bad)


def test_bf16_truncation_caught():
    def trunc(x):
        x = np.ascontiguousarray(x, dtype=np.float32)
        return (x.view(np.uint32) & np.uint32(0xFFFF0000)).view(np.float32)
    assert _fails(C.check_bf16_rounding, trunc)


def test_fp8_scale_tile_mistake_caught(monkeypatch):
    monkeypatch.setattr(O, "FP8_TILE", 64)        # scales applied per 64 instead of 128
    def deq(rec):
        try:
            return O.dequant_fp8_records(rec)
        except ValueError:
            raise AssertionError("shape")
    assert _fails(C.check_fp8_record, deq)


def test_value_slice_mistake_caught():
    def decode_bad(q, cache, bt, lens, scale, causal, d_v=512, requests=None):
        shifted = np.concatenate([cache[..., 64:], cache[..., :64]], axis=-1)  # V = dims 64..575
        out, _ = O.decode_dense(q, shifted, bt, lens, scale, causal, d_v)
        _, lse = O.decode_dense(q, cache, bt, lens, scale, causal, d_v)
        return out, lse
    assert _fails(C.check_single_token, decode_bad)
    assert _fails(C.check_golden_two_tokens, decode_bad)


# ---------------------------------------------------------------- attention sink
def _sink_negated(q, k, scale, d_v=512, sink=None):
    return real_attend(q, k, scale, d_v, None if sink is None else -np.asarray(sink))


def _sink_scaled(q, k, scale, d_v=512, sink=None):
    return real_attend(q, k, scale, d_v, None if sink is None else scale * np.asarray(sink))


def _sink_lse_dropped(q, k, scale, d_v=512, sink=None):
    o, _ = real_attend(q, k, scale, d_v, sink)
    _, l = real_attend(q, k, scale, d_v)
    return o, l


def _sink_out_dropped(q, k, scale, d_v=512, sink=None):
    _, l = real_attend(q, k, scale, d_v, sink)
    o, _ = real_attend(q, k, scale, d_v)
    return o, l


def _sink_carries_value(q, k, scale, d_v=512, sink=None):
    """The sink key carries the first key's value instead of zero."""
    o, l = real_attend(q, k, scale, d_v, sink)
    k = np.asarray(k, float)
    if sink is None or k.shape[0] == 0:
        return o, l
    w = np.exp(np.asarray(sink, float) - l)[:, None]
    return o + w * k[0, :d_v], l


SINK_MUTANTS = [_sink_negated, _sink_scaled, _sink_lse_dropped, _sink_out_dropped, _sink_carries_value]


@pytest.mark.parametrize("mutant", SINK_MUTANTS, ids=lambda f: f.__name__)
def test_sink_mutants_caught(mutant, monkeypatch):
    caught = _fails(C.check_sink_brute_force, mutant)
    caught = caught or _fails(C.check_sink_single_token, mutant)
    monkeypatch.setattr(O, "attend", mutant)
    caught = caught or _fails(C.check_sink_as_extra_key, O.decode_dense)
    assert caught


def test_sink_in_every_split_caught():
    """A combine that adds the sink to each part instead of once."""
    real_combine = O.combine

    def per_part(o_parts, lse_parts, sink=None):
        if sink is None:
            return real_combine(o_parts, lse_parts)
        lse_parts = np.asarray(lse_parts, float)
        o_parts = np.asarray(o_parts, float)
        lp = np.logaddexp(lse_parts, np.asarray(sink, float)[None, :])
        op = o_parts * np.exp(lse_parts - lp)[..., None]
        return real_combine(op, lp)
    assert _fails(C.check_sink_reductions, O.decode_dense, O.decode_sparse, O.attend, per_part)


# ---------------------------------------------------------------- NVFP4
real_dequant_nvfp4 = O.dequant_nvfp4


def _nvfp4_nibbles_swapped(packed, scales):
    pk = np.asarray(packed, dtype=np.uint8)
    return real_dequant_nvfp4(((pk & 0xF) << 4) | (pk >> 4), scales)


def _nvfp4_block32(packed, scales):
    sc = np.asarray(scales, dtype=np.uint8)
    sc2 = np.repeat(sc[..., 0::2], 2, axis=-1)        # one scale per 32 values
    return real_dequant_nvfp4(packed, sc2)


def _nvfp4_scale_e8m0(packed, scales):
    pk = np.asarray(packed, dtype=np.uint8)
    codes = np.stack([pk & 0xF, pk >> 4], axis=-1).reshape(*pk.shape[:-1], 2 * pk.shape[-1])
    sc = np.exp2(np.asarray(scales, dtype=np.float64) - 127.0)
    return O.e2m1_to_f64(codes) * np.repeat(sc, 16, axis=-1)


def _e2m1_bias0(codes):
    c = np.asarray(codes).astype(np.int64) & 0xF
    e, m = (c >> 1) & 3, c & 1
    mag = np.where(e == 0, 0.5 * m, np.exp2(e * 1.0) * (1.0 + 0.5 * m))
    return np.where(c & 8, -mag, mag)


@pytest.mark.parametrize("mutant", [_nvfp4_nibbles_swapped, _nvfp4_block32, _nvfp4_scale_e8m0],
                         ids=lambda f: f.__name__)
def test_nvfp4_layout_mutants_caught(mutant, monkeypatch):
    caught = _fails(C.check_nvfp4_golden, mutant)
    monkeypatch.setattr(O, "dequant_nvfp4", mutant)
    caught = caught or _fails(C.check_nvfp4_decode_brute_force, O.reference_decode)
    assert caught


def test_e2m1_bias_mistake_caught():
    assert _fails(C.check_e2m1, _e2m1_bias0)
