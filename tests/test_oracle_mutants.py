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


# ---------------------------------------------------------------- query norm, RoPE, output FP8 cast
def _rms_sum_not_mean(x, gamma, eps):
    x = np.asarray(x, float)
    return x / np.sqrt(np.sum(x * x, axis=-1, keepdims=True) + eps) * gamma


def _rms_eps_outside(x, gamma, eps):
    x = np.asarray(x, float)
    return x / (np.sqrt(np.mean(x * x, axis=-1, keepdims=True)) + eps) * gamma


def _rms_no_gamma(x, gamma, eps):
    return O.rms_norm(x, np.ones(np.shape(x)[-1]), eps)


def _rms_no_sqrt(x, gamma, eps):
    x = np.asarray(x, float)
    return x / (np.mean(x * x, axis=-1, keepdims=True) + eps) * gamma


@pytest.mark.parametrize("mutant", [_rms_sum_not_mean, _rms_eps_outside, _rms_no_gamma, _rms_no_sqrt],
                         ids=lambda f: f.__name__)
def test_rms_norm_mutants_caught(mutant):
    assert _fails(C.check_rms_norm, mutant)


def _rope_half_split(x, cos, sin, conjugate=False):
    x = np.asarray(x, float)
    n = x.shape[-1] // 2
    s = -np.asarray(sin) if conjugate else np.asarray(sin)
    y = np.empty(np.broadcast(x, np.concatenate([cos, cos], axis=-1)).shape)
    y[..., :n] = x[..., :n] * cos - x[..., n:] * s
    y[..., n:] = x[..., :n] * s + x[..., n:] * cos
    return y


def _rope_sign_flipped(x, cos, sin, conjugate=False):
    return O.rope_rotate(x, cos, sin, not conjugate)


def _rope_sin_cos_swapped(x, cos, sin, conjugate=False):
    return O.rope_rotate(x, sin, cos, conjugate)


def _rope_conj_ignored(x, cos, sin, conjugate=False):
    return O.rope_rotate(x, cos, sin, False)


@pytest.mark.parametrize("mutant", [_rope_half_split, _rope_sign_flipped, _rope_sin_cos_swapped,
                                    _rope_conj_ignored], ids=lambda f: f.__name__)
def test_rope_mutants_caught(mutant):
    assert _fails(C.check_rope, mutant)


def _qnr_rotates_front(q, gamma, eps, cos, sin):
    y = O.rms_norm(q, gamma, eps)
    y[..., :64] = O.rope_rotate(y[..., :64], np.asarray(cos)[:, :, None, :], np.asarray(sin)[:, :, None, :])
    return y


def _qnr_rope_before_norm(q, gamma, eps, cos, sin):
    q = np.array(q, float)
    q[..., -64:] = O.rope_rotate(q[..., -64:], np.asarray(cos)[:, :, None, :], np.asarray(sin)[:, :, None, :])
    return O.rms_norm(q, gamma, eps) * 0 + O.q_norm_rope(q, gamma, eps, np.ones_like(cos), np.zeros_like(sin))


def _qnr_token0_angles(q, gamma, eps, cos, sin):
    c = np.repeat(np.asarray(cos)[:, :1], np.shape(cos)[1], axis=1)
    s = np.repeat(np.asarray(sin)[:, :1], np.shape(sin)[1], axis=1)
    return O.q_norm_rope(q, gamma, eps, c, s)


@pytest.mark.parametrize("mutant", [_qnr_rotates_front, _qnr_rope_before_norm, _qnr_token0_angles],
                         ids=lambda f: f.__name__)
def test_q_norm_rope_mutants_caught(mutant):
    assert _fails(C.check_q_norm_rope, mutant, O.rms_norm, O.rope_rotate)


def _enc_truncate(x):
    """round toward zero instead of to nearest"""
    x = np.asarray(x, float)
    v = O.e4m3_to_f64(np.arange(127))
    a = np.minimum(np.abs(x), 448.0)
    idx = np.searchsorted(v, a, side="right") - 1
    return (np.clip(idx, 0, 126) | np.where(np.signbit(x), 0x80, 0)).astype(np.uint8)


def _enc_ties_up(x):
    x = np.asarray(x, float)
    v = O.e4m3_to_f64(np.arange(127))
    a = np.minimum(np.abs(x), 448.0)
    hi = np.clip(np.searchsorted(v, a, side="left"), 0, 126)
    lo = np.maximum(hi - 1, 0)
    code = np.where(v[hi] - a <= a - v[lo], hi, lo)
    return (code | np.where(np.signbit(x), 0x80, 0)).astype(np.uint8)


def _enc_no_saturation(x):
    c = O.e4m3_encode(x)
    return np.where(np.abs(np.asarray(x, float)) > 448, 0x7F, c).astype(np.uint8)


@pytest.mark.parametrize("mutant", [_enc_truncate, _enc_ties_up, _enc_no_saturation], ids=lambda f: f.__name__)
def test_e4m3_encode_mutants_caught(mutant):
    assert _fails(C.check_e4m3_encode, mutant, O.e4m3_to_f64)


def _cast_scale_fp8max_240(x, tile=128):
    x = np.asarray(x, np.float32)
    t = x.reshape(*x.shape[:-1], -1, tile)
    amax = np.abs(t).max(-1)
    sc = np.where(amax > 0, amax / np.float32(240.0), 1).astype(np.float32)
    return O.e4m3_encode((t / sc[..., None]).astype(np.float32)).reshape(x.shape), sc


def _cast_tile_64(x, tile=128):
    return O.fp8_cast_rows(x, 64)


def _cast_no_scale(x, tile=128):
    x = np.asarray(x, np.float32)
    return O.e4m3_encode(x), np.ones((*x.shape[:-1], x.shape[-1] // tile), np.float32)


@pytest.mark.parametrize("mutant", [_cast_scale_fp8max_240, _cast_tile_64, _cast_no_scale],
                         ids=lambda f: f.__name__)
def test_fp8_cast_mutants_caught(mutant):
    assert _fails(C.check_fp8_cast_rows, mutant, O.e4m3_to_f64)


def _epi_rotates_forward(out, cos, sin, d_qk):
    return O.out_rope_fp8(out, cos, -np.asarray(sin), d_qk)


def _epi_rotates_576(out, cos, sin, d_qk):
    return O.out_rope_fp8(out, cos, sin, 512)


def _epi_wrong_dims(out, cos, sin, d_qk):
    y = np.array(out, np.float32)
    if d_qk == 512:
        r = O.rope_rotate(y[..., :64], np.asarray(cos)[:, :, None, :], np.asarray(sin)[:, :, None, :], True)
        y[..., :64] = r.astype(np.float32)
    c, s = O.fp8_cast_rows(y)
    return c, s, y


@pytest.mark.parametrize("mutant", [_epi_rotates_forward, _epi_rotates_576, _epi_wrong_dims],
                         ids=lambda f: f.__name__)
def test_out_epilogue_mutants_caught(mutant):
    assert _fails(C.check_out_rope_fp8, mutant, O.fp8_cast_rows, O.rope_rotate)
