"""Independent pins for the fp64 oracle.

Every check takes the oracle function(s) it exercises as arguments, so the
same check can be run against the real oracle (must pass) and against planted
mistakes (must fail; see test_oracle_mutants.py). None of the checks re-uses
the oracle's own formulas: they use 50-digit mpmath brute force, closed forms,
scipy's logsumexp, invariances, and torch's own fp8/bf16 conversions.
"""
from __future__ import annotations

import json
import math
import os

import mpmath
import numpy as np
import torch
from scipy.special import logsumexp

mpmath.mp.dps = 50
GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
PAGE = 64


# ---------------------------------------------------------------- helpers
def _mp_attend(q_rows, keys, scale, d_v):
    """Pure-Python 50-digit softmax attention (no numpy arithmetic)."""
    R = len(q_rows)
    outs, lses = [], []
    for r in range(R):
        s = [mpmath.mpf(scale) * mpmath.fsum(mpmath.mpf(float(a)) * mpmath.mpf(float(b))
                                             for a, b in zip(q_rows[r], k)) for k in keys]
        if not s:
            outs.append([0.0] * d_v)
            lses.append(-math.inf)
            continue
        m = max(s)
        e = [mpmath.exp(x - m) for x in s]
        l = mpmath.fsum(e)
        o = [mpmath.fsum(e[t] * mpmath.mpf(float(keys[t][d])) for t in range(len(keys))) / l
             for d in range(d_v)]
        outs.append([float(v) for v in o])
        lses.append(float(m + mpmath.log(l)))
    return np.array(outs), np.array(lses)


def _random_paged(rng, lens, d_qk, extra_pages=0):
    """Small paged cache with a random physical page order (fp64 values)."""
    npg = [(L + PAGE - 1) // PAGE for L in lens]
    P = sum(npg) + extra_pages
    perm = rng.permutation(P)
    bt = np.full((len(lens), max(1, max(npg))), -1, dtype=np.int64)
    off = 0
    for b, n in enumerate(npg):
        bt[b, :n] = perm[off:off + n]
        off += n
    cache = rng.standard_normal((P, PAGE, d_qk))
    return cache, bt


def _close(a, b, tol):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    assert a.shape == b.shape, (a.shape, b.shape)
    both_inf = np.isinf(a) & np.isinf(b) & (np.sign(a) == np.sign(b))
    err = np.where(both_inf, 0.0, np.abs(a - b) / (1.0 + np.abs(b)))
    assert np.all(np.isfinite(err)) and err.max(initial=0.0) <= tol, f"max rel err {err.max()}"


# ---------------------------------------------------------------- checks
def check_brute_force_attend(attend, seeds=range(6)):
    """attend() vs 50-digit brute force on tiny shapes (d_qk<=8, <=5 keys)."""
    for seed in seeds:
        rng = np.random.default_rng(seed)
        d_qk, d_v = int(rng.integers(2, 9)), 0
        d_v = int(rng.integers(1, d_qk + 1))
        T = int(rng.integers(1, 6))
        R = int(rng.integers(1, 4))
        q = rng.standard_normal((R, d_qk)) * 2
        k = rng.standard_normal((T, d_qk)) * 2
        scale = float(rng.uniform(0.1, 1.5))
        o, l = attend(q, k, scale, d_v)
        eo, el = _mp_attend(q.tolist(), k.tolist(), scale, d_v)
        _close(o, eo, 1e-13)
        _close(l, el, 1e-13)


def check_brute_force_paged(decode_dense, causal, seeds=range(3)):
    """decode_dense() vs brute force that walks token by token through pages."""
    for seed in seeds:
        rng = np.random.default_rng(100 + seed)
        d_qk, d_v = 6, 4
        s_q = 2 if causal else 1
        lens = [int(x) for x in rng.integers(1, 140, size=2)]
        cache, bt = _random_paged(rng, lens, d_qk, extra_pages=1)
        q = rng.standard_normal((2, s_q, 2, d_qk))
        scale = 0.7
        out, lse = decode_dense(q, cache, bt, np.array(lens), scale, causal, d_v=d_v)
        for b, L in enumerate(lens):
            for i in range(s_q):
                last = L - s_q + i if causal else L - 1
                keys = []
                for t in range(0, max(0, last + 1)):
                    page = bt[b][t // PAGE]
                    keys.append(list(cache[page][t % PAGE]))
                eo, el = _mp_attend(q[b, i].tolist(), keys, scale, d_v)
                _close(out[b, i], eo, 1e-13)
                _close(lse[b, i], el, 1e-13)


def check_single_token(decode_dense, d_v=512):
    """seqlen 1: out is that token's V row exactly; lse = scale * q.k."""
    rng = np.random.default_rng(7)
    d_qk = 576
    cache, bt = _random_paged(rng, [1], d_qk, extra_pages=2)
    q = rng.standard_normal((1, 1, 3, d_qk))
    out, lse = decode_dense(q, cache, bt, np.array([1]), 1 / 24, False, d_v=d_v)
    row = cache[bt[0][0], 0]
    for h in range(3):
        assert np.array_equal(out[0, 0, h], row[:d_v])
        _close(lse[0, 0, h], (1 / 24) * float(np.dot(q[0, 0, h], row)), 1e-14)


def check_constant_scores(decode_dense, d_v=512):
    """Equal scores for every key: out = mean of V rows, lse = s + ln n.

    q is zero on the first 512 dims, and every token shares the same RoPE part
    (dims 512..575) while its latent part differs, so all scores are equal
    but the V rows are not.
    """
    rng = np.random.default_rng(8)
    d_qk, n = 576, 131
    cache, bt = _random_paged(rng, [n], d_qk)
    rope = rng.standard_normal(d_qk - 512)
    cache[..., 512:] = rope
    q = np.zeros((1, 1, 2, d_qk))
    q[..., 512:] = rng.standard_normal((1, 1, 2, d_qk - 512))
    out, lse = decode_dense(q, cache, bt, np.array([n]), 0.5, False, d_v=d_v)
    rows = np.stack([cache[bt[0][t // PAGE], t % PAGE] for t in range(n)])
    for h in range(2):
        _close(out[0, 0, h], rows[:, :d_v].mean(axis=0), 1e-13)
        s = 0.5 * float(np.dot(q[0, 0, h, 512:], rope))
        _close(lse[0, 0, h], s + math.log(n), 1e-13)


def check_lse_logsumexp(decode_dense):
    """lse equals scipy's logsumexp of the explicit score vector."""
    rng = np.random.default_rng(9)
    d_qk = 576
    lens = [200, 64, 1]
    cache, bt = _random_paged(rng, lens, d_qk)
    q = rng.standard_normal((3, 1, 4, d_qk))
    _, lse = decode_dense(q, cache, bt, np.array(lens), 1 / 24, False)
    for b, L in enumerate(lens):
        for h in range(4):
            sc = [(1 / 24) * math.fsum(q[b, 0, h] * cache[bt[b][t // PAGE], t % PAGE])
                  for t in range(L)]
            _close(lse[b, 0, h], logsumexp(sc), 1e-13)


def check_page_permutation(decode_dense):
    """Moving physical pages (and the block table with them) changes no bit."""
    rng = np.random.default_rng(10)
    d_qk = 576
    lens = [70, 129, 5]
    cache, bt = _random_paged(rng, lens, d_qk, extra_pages=3)
    q = rng.standard_normal((3, 1, 2, d_qk))
    o1, l1 = decode_dense(q, cache, bt, np.array(lens), 1 / 24, False)
    P = cache.shape[0]
    perm = rng.permutation(P)                 # new location of old page p = perm[p]
    cache2 = np.empty_like(cache)
    cache2[perm] = cache
    bt2 = np.where(bt >= 0, perm[np.maximum(bt, 0)], -1)
    o2, l2 = decode_dense(q, cache2, bt2, np.array(lens), 1 / 24, False)
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)


def check_causal_row0(decode_dense):
    """s_q=2 causal: query 0 equals a non-causal run over seqlen-1 tokens,
    query 1 equals a non-causal run over all seqlen tokens."""
    rng = np.random.default_rng(11)
    d_qk = 576
    lens = [130, 65, 2]
    cache, bt = _random_paged(rng, lens, d_qk)
    q = rng.standard_normal((3, 2, 3, d_qk))
    oc, lc = decode_dense(q, cache, bt, np.array(lens), 1 / 24, True)
    o0, l0 = decode_dense(q[:, :1], cache, bt, np.array(lens) - 1, 1 / 24, False)
    o1, l1 = decode_dense(q[:, 1:], cache, bt, np.array(lens), 1 / 24, False)
    assert np.array_equal(oc[:, 0], o0[:, 0]) and np.array_equal(lc[:, 0], l0[:, 0])
    assert np.array_equal(oc[:, 1], o1[:, 0]) and np.array_equal(lc[:, 1], l1[:, 0])


def check_sparse(decode_sparse, decode_dense):
    """-1 slots contribute nothing; all positions in order equals dense;
    a shuffled index list gives the same result within fp64 rounding."""
    rng = np.random.default_rng(12)
    d_qk = 576
    lens = [300, 129]
    cache, bt = _random_paged(rng, lens, d_qk)
    q = rng.standard_normal((2, 1, 3, d_qk))
    # (a) -1 slots vs the compacted list (same order of kept entries)
    topk = 128
    idx = np.stack([rng.choice(L, size=topk, replace=False) for L in lens])[:, None, :]
    holes = idx.copy()
    holes[0, 0, rng.choice(topk, 17, replace=False)] = -1
    holes[1, 0, :5] = -1
    o_h, l_h = decode_sparse(q, cache, bt, np.array(lens), holes, 1 / 24)
    for b in range(2):
        kept = holes[b, 0][holes[b, 0] != -1]
        o_c, l_c = decode_sparse(q[b:b + 1], cache, bt[b:b + 1], np.array(lens[b:b + 1]),
                                 kept[None, None, :], 1 / 24)
        assert np.array_equal(o_h[b], o_c[0]) and np.array_equal(l_h[b], l_c[0])
    # (b) every position in order == dense
    L = 129
    allidx = np.arange(L)[None, None, :]
    o_s, l_s = decode_sparse(q[1:], cache, bt[1:], np.array([L]), allidx, 1 / 24)
    o_d, l_d = decode_dense(q[1:], cache, bt[1:], np.array([L]), 1 / 24, False)
    assert np.array_equal(o_s, o_d) and np.array_equal(l_s, l_d)
    # (c) order does not matter
    sh = idx.copy()
    for b in range(2):
        rng.shuffle(sh[b, 0])
    o1, l1 = decode_sparse(q, cache, bt, np.array(lens), idx, 1 / 24)
    o2, l2 = decode_sparse(q, cache, bt, np.array(lens), sh, 1 / 24)
    _close(o1, o2, 1e-13)
    _close(l1, l2, 1e-13)


def check_combine(attend, combine):
    """Combining any split of the key set reproduces the unsplit result."""
    rng = np.random.default_rng(13)
    d_qk, d_v, T = 576, 512, 300
    q = rng.standard_normal((4, d_qk))
    k = rng.standard_normal((T, d_qk))
    o_ref, l_ref = attend(q, k, 1 / 24, d_v)
    for cuts in ([0, 1, T], [0, 64, 64, 200, T], [0, 150, 299, T]):   # includes an empty part
        parts = [attend(q, k[a:b], 1 / 24, d_v) for a, b in zip(cuts[:-1], cuts[1:])]
        o, l = combine(np.stack([p[0] for p in parts]), np.stack([p[1] for p in parts]))
        _close(o, o_ref, 1e-13)
        _close(l, l_ref, 1e-13)
    o, l = combine(np.zeros((2, 4, d_v)), np.full((2, 4), -np.inf))
    assert np.all(o == 0) and np.all(np.isneginf(l))


def check_empty_key_sets(decode_dense, decode_sparse):
    """Chosen reading for an empty key set: out 0, lse -inf."""
    rng = np.random.default_rng(14)
    d_qk = 576
    cache, bt = _random_paged(rng, [64, 1], d_qk)
    q = rng.standard_normal((2, 2, 2, d_qk))
    out, lse = decode_dense(q, cache, bt, np.array([0, 1]), 1 / 24, True)
    assert np.all(out[0] == 0) and np.all(np.isneginf(lse[0]))     # seqlen 0
    assert np.all(out[1, 0] == 0) and np.all(np.isneginf(lse[1, 0]))  # causal row with no key
    assert np.all(np.isfinite(lse[1, 1]))
    idx = np.full((2, 2, 64), -1)
    o, l = decode_sparse(q, cache, bt, np.array([64, 1]), idx, 1 / 24)
    assert np.all(o == 0) and np.all(np.isneginf(l))


def check_e4m3(e4m3_to_f64):
    """All 256 codes vs torch's float8_e4m3fn decoding, plus closed forms."""
    codes = np.arange(256, dtype=np.uint8)
    mine = e4m3_to_f64(codes)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    nan_m, nan_r = np.isnan(mine), np.isnan(ref)
    assert np.array_equal(nan_m, nan_r)
    assert np.array_equal(mine[~nan_m], ref[~nan_r])
    fixed = {0x00: 0.0, 0x01: 2.0 ** -9, 0x07: 7 * 2.0 ** -9, 0x08: 2.0 ** -6, 0x38: 1.0,
             0xB8: -1.0, 0x7E: 448.0, 0xFE: -448.0, 0x40: 2.0, 0x3C: 1.5}
    for c, v in fixed.items():
        assert e4m3_to_f64(np.array([c], dtype=np.uint8))[0] == v, hex(c)
    assert np.isnan(e4m3_to_f64(np.array([0x7F, 0xFF], dtype=np.uint8))).all()


def check_bf16_rounding(f32_round_to_bf16):
    """fp32 -> bf16 round-to-nearest-even vs torch on random and tie values."""
    rng = np.random.default_rng(15)
    x = np.concatenate([rng.standard_normal(20000).astype(np.float32) * 10,
                        np.array([1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -(1.0 + 2 ** -8),
                                  3.0e38, 1e-40, 0.0, -0.0, 65504.0], dtype=np.float32)])
    mine = f32_round_to_bf16(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).to(torch.float32).numpy()
    assert np.array_equal(mine.view(np.uint32), ref.view(np.uint32))
    assert f32_round_to_bf16(np.array([1.0 + 2 ** -8], np.float32))[0] == 1.0          # tie -> even
    assert f32_round_to_bf16(np.array([1.0 + 3 * 2 ** -8], np.float32))[0] == 1.0 + 2 ** -6


def check_fp8_record(dequant_fp8_records):
    """A hand-built 656-byte record decodes to the hand-computed row."""
    rec = np.zeros((1, PAGE, 656), dtype=np.uint8)
    codes = np.array([0x38, 0xB8, 0x40, 0x7E], dtype=np.uint8)    # 1, -1, 2, 448
    scales = np.array([0.5, 3.0, 1.0 / 448.0, 7.0], dtype=np.float32)
    for t in range(4):
        rec[0, t, :512] = codes[t]
        rec[0, t, 512:528] = scales.view(np.uint8)
        rope = np.full(64, t + 0.25, dtype=np.float32)
        rec[0, t, 528:] = (rope.view(np.uint32) >> 16).astype(np.uint16).view(np.uint8)
    out = dequant_fp8_records(rec)
    vals = [1.0, -1.0, 2.0, 448.0]
    for t in range(4):
        for tile in range(4):
            prod = np.float32(vals[t]) * scales[tile]
            expect = float(torch.tensor(float(prod)).to(torch.bfloat16).float())
            assert np.all(out[0, t, 128 * tile:128 * (tile + 1)] == expect), (t, tile)
        assert np.all(out[0, t, 512:] == t + 0.25)


def check_golden_two_tokens(decode_dense):
    """Hand-derived closed form stored in tests/golden/two_token_closed_form.json."""
    with open(os.path.join(GOLDEN, "two_token_closed_form.json")) as f:
        g = json.load(f)
    d = 576
    cache = np.zeros((2, PAGE, d))
    for t, row in enumerate(g["key_rows_sparse"]):
        for k, v in row.items():
            cache[1, t, int(k)] = v
    q = np.zeros((1, 1, 1, d))
    for k, v in g["q_sparse"].items():
        q[0, 0, 0, int(k)] = v
    bt = np.array([[1]])
    out, lse = decode_dense(q, cache, bt, np.array([2]), g["scale"], False)
    for k, v in g["out_sparse"].items():
        _close(out[0, 0, 0, int(k)], v, 1e-15)
    nz = set(int(k) for k in g["out_sparse"])
    assert all(out[0, 0, 0, j] == 0 for j in range(512) if j not in nz)
    _close(lse[0, 0, 0], g["lse"], 1e-15)


# ---------------------------------------------------------------- attention sink
def _mp_attend_sink(q_rows, keys, scale, d_v, sink):
    """50-digit brute force with one extra logit per row that carries no value."""
    outs, lses = [], []
    for r in range(len(q_rows)):
        s = [mpmath.mpf(scale) * mpmath.fsum(mpmath.mpf(float(a)) * mpmath.mpf(float(b))
                                             for a, b in zip(q_rows[r], k)) for k in keys]
        sg = mpmath.mpf(float(sink[r]))
        m = max(s + [sg])
        e = [mpmath.exp(x - m) for x in s]
        l = mpmath.fsum(e) + mpmath.exp(sg - m)
        o = [mpmath.fsum(e[t] * mpmath.mpf(float(keys[t][d])) for t in range(len(keys))) / l
             for d in range(d_v)]
        outs.append([float(v) for v in o])
        lses.append(float(m + mpmath.log(l)))
    return np.array(outs), np.array(lses)


def check_sink_brute_force(attend, seeds=range(4)):
    """attend(..., sink) vs 50-digit brute force, including a sink that
    dominates every score and a key set of one."""
    for seed in seeds:
        rng = np.random.default_rng(300 + seed)
        d_qk = int(rng.integers(2, 9))
        d_v = int(rng.integers(1, d_qk + 1))
        T = int(rng.integers(1, 5))
        R = 3
        q = rng.standard_normal((R, d_qk)) * 2
        k = rng.standard_normal((T, d_qk)) * 2
        scale = float(rng.uniform(0.1, 1.5))
        sink = np.array([rng.standard_normal(), 40.0, -3.0])
        o, l = attend(q, k, scale, d_v, sink=sink)
        eo, el = _mp_attend_sink(q.tolist(), k.tolist(), scale, d_v, sink)
        _close(o, eo, 1e-13)
        _close(l, el, 1e-13)


def check_sink_single_token(attend):
    """One key of score s and a sink sigma: out = v / (1 + e^(sigma - s)),
    lse = ln(e^s + e^sigma) (closed form, computed here in 50 digits)."""
    rng = np.random.default_rng(301)
    d_qk, d_v = 576, 512
    q = rng.standard_normal((2, d_qk))
    k = rng.standard_normal((1, d_qk))
    sink = np.array([0.3, -1.7])
    o, l = attend(q, k, 1 / 24, d_v, sink=sink)
    for r in range(2):
        s = mpmath.mpf(1 / 24) * mpmath.fsum(mpmath.mpf(float(a)) * mpmath.mpf(float(b))
                                            for a, b in zip(q[r], k[0]))
        w = 1 / (1 + mpmath.exp(mpmath.mpf(float(sink[r])) - s))
        _close(o[r], k[0, :d_v] * float(w), 1e-14)
        _close(l[r], float(mpmath.log(mpmath.exp(s) + mpmath.exp(mpmath.mpf(float(sink[r]))))), 1e-14)


def check_sink_as_extra_key(decode_dense):
    """A per-head sink equals one more key whose value dims are zero and whose
    RoPE dims give score sigma_h with every head's query: the same decode
    without a sink over the longer key set. The key solves the h_q equations
    scale * q_h[512:] . k_rope = sigma_h (h_q <= 64 unknowns, exact)."""
    rng = np.random.default_rng(302)
    d_qk, h_q, scale = 576, 5, 1 / 24
    lens = [70, 1, 129]
    cache, bt = _random_paged(rng, lens, d_qk, extra_pages=3)
    sink = rng.standard_normal(h_q) + 1.0
    q = rng.standard_normal((len(lens), 1, h_q, d_qk))
    out, lse = decode_dense(q, cache, bt, np.array(lens), scale, False, sink=sink)
    for b, L in enumerate(lens):
        qb = q[b, 0]
        k_rope, *_ = np.linalg.lstsq(scale * qb[:, 512:], sink, rcond=None)
        extra = np.zeros(d_qk)
        extra[512:] = k_rope
        cb = cache.copy()
        n = (L + PAGE - 1) // PAGE
        bt_b = bt[b:b + 1].copy()
        if L % PAGE == 0:                       # the extra key opens a fresh page
            cb = np.concatenate([cb, np.zeros((1, PAGE, d_qk))])
            bt_b = np.concatenate([bt_b, np.full((1, 1), -1)], axis=1)
            bt_b[0, n] = cb.shape[0] - 1
        page = bt_b[0, L // PAGE]
        cb[page, L % PAGE] = extra
        o2, l2 = decode_dense(q[b:b + 1], cb, bt_b, np.array([L + 1]), scale, False)
        _close(out[b], o2[0], 1e-12)
        _close(lse[b], l2[0], 1e-12)


def check_sink_reductions(decode_dense, decode_sparse, attend, combine):
    """sigma = -inf leaves every bit unchanged; an empty key set gives out 0
    and lse = sigma; combining any split with the sink reproduces attend()
    with the sink (the sink joins once, in the combine)."""
    rng = np.random.default_rng(303)
    d_qk, h_q = 576, 3
    lens = [130, 0, 2]
    cache, bt = _random_paged(rng, lens, d_qk, extra_pages=1)
    q = rng.standard_normal((3, 2, h_q, d_qk))
    o0, l0 = decode_dense(q, cache, bt, np.array(lens), 1 / 24, True)
    o1, l1 = decode_dense(q, cache, bt, np.array(lens), 1 / 24, True, sink=np.full(h_q, -np.inf))
    assert np.array_equal(o0, o1) and np.array_equal(l0, l1)
    sink = np.array([0.5, -2.0, 7.0])
    o2, l2 = decode_dense(q, cache, bt, np.array(lens), 1 / 24, True, sink=sink)
    assert np.all(o2[1] == 0) and np.array_equal(l2[1, 0], sink) and np.array_equal(l2[1, 1], sink)
    assert np.all(o2[2, 0] != 0)                     # causal row 0 of a 2-token request sees 1 key
    idx = np.full((3, 2, 64), -1)
    o3, l3 = decode_sparse(q, cache, bt, np.array(lens), idx, 1 / 24, sink=sink)
    assert np.all(o3 == 0) and np.all(l3 == sink)
    k = rng.standard_normal((200, d_qk))
    qr = rng.standard_normal((h_q, d_qk))
    o_ref, l_ref = attend(qr, k, 1 / 24, 512, sink=sink)
    for cuts in ([0, 200], [0, 64, 64, 200], [0, 1, 199, 200]):
        parts = [attend(qr, k[a:b], 1 / 24, 512) for a, b in zip(cuts[:-1], cuts[1:])]
        o, l = combine(np.stack([p[0] for p in parts]), np.stack([p[1] for p in parts]), sink=sink)
        _close(o, o_ref, 1e-13)
        _close(l, l_ref, 1e-13)


# ---------------------------------------------------------------- NVFP4 (E2M1 + UE4M3 block 16)
OCP_E2M1 = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]   # OCP MX FP4 E2M1 magnitudes of codes 0..7


def check_e2m1(e2m1_to_f64):
    """All 16 codes against the OCP MX table; bit 3 is the sign."""
    got = e2m1_to_f64(np.arange(16))
    want = np.array(OCP_E2M1 + [-x for x in OCP_E2M1])
    assert np.array_equal(got, want), (got, want)
    assert np.signbit(got[8]) and not np.signbit(got[0])


def check_ue4m3(ue4m3_to_f64):
    """All 128 scale codes against torch's float8_e4m3fn; bit 7 is ignored."""
    codes = np.arange(128, dtype=np.uint8)
    want = torch.from_numpy(codes.copy()).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = ue4m3_to_f64(codes)
    fin = np.isfinite(want)
    assert np.array_equal(got[fin], want[fin]) and np.all(np.isnan(got[~fin]))
    assert np.array_equal(ue4m3_to_f64(codes[:127] | 0x80), got[:127])


def check_nvfp4_golden(dequant_nvfp4):
    """Hand-decoded two-block row stored in tests/golden/nvfp4_two_blocks.json."""
    with open(os.path.join(GOLDEN, "nvfp4_two_blocks.json")) as f:
        g = json.load(f)
    got = dequant_nvfp4(np.array([g["packed"]], np.uint8), np.array([g["scales"]], np.uint8))[0]
    want = np.array(g["values"])
    assert np.array_equal(got, want) and np.array_equal(np.signbit(got), np.signbit(want))


def check_nvfp4_products_exact():
    """Every E2M1 x UE4M3 product (finite scales) is exactly a bf16 and an f16
    value: a kernel that dequantises to bf16 loses nothing."""
    vals = np.array(OCP_E2M1 + [-x for x in OCP_E2M1])
    sc = torch.arange(127, dtype=torch.uint8).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    prod = (vals[:, None] * sc[None, :]).ravel()
    t = torch.from_numpy(prod)
    assert torch.equal(t.to(torch.bfloat16).to(torch.float64), t)
    assert torch.equal(t.to(torch.float16).to(torch.float64), t)


def _table_dequant(packed, scales):
    """Test-side NVFP4 decoder by table lookup (independent of the oracle's)."""
    tab = OCP_E2M1 + [-x for x in OCP_E2M1]
    e4m3 = torch.arange(256, dtype=torch.int32).to(torch.uint8).view(torch.float8_e4m3fn).to(torch.float64)
    out = []
    for i, byte in enumerate(packed):
        s = float(e4m3[int(scales[(2 * i) // 16]) & 0x7F])
        out += [tab[byte & 0xF] * s, tab[byte >> 4] * s]
    return out


def check_nvfp4_decode_brute_force(reference_decode):
    """A tiny NVFP4 decode (2 requests, causal s_q 2, d_qk = d_v = 512) against
    50-digit brute force over values decoded by table lookup."""
    import dataclasses
    from workloads import mla_workloads as W
    w = dataclasses.replace(W.get_workload("tiny"), kv="nvfp4", batch=2, seqlens=[3, 2], s_q=2, h_q=2,
                            causal=True, scale=512 ** -0.5, seed=41)
    inp = W.make_inputs(w)
    out, lse = reference_decode(inp)
    bt = inp.block_table.numpy()
    for b, L in enumerate([3, 2]):
        rows = []
        for t in range(L):
            pg, sl = bt[b, t // PAGE], t % PAGE
            rows.append(_table_dequant(inp.kcache[pg, sl].tolist(), inp.kv_scale[pg, sl].tolist()))
        for i in range(2):
            n = L - 2 + i + 1
            qs = [_table_dequant(inp.q[b, i, h].tolist(), inp.q_scale[b, i, h].tolist()) for h in range(2)]
            eo, el = _mp_attend(qs, rows[:n], 512 ** -0.5, 512)
            _close(out[b, i], eo, 1e-13)
            _close(lse[b, i], el, 1e-13)


# ---------------------------------------------------------------- query norm, RoPE, output FP8 cast
def check_rms_norm(rms_norm, seeds=range(3)):
    """Invariants of RMS normalisation: with gamma = 1 and eps = 0 every row
    has mean square exactly 1; the result does not change when a row is
    scaled; gamma multiplies per dimension; eps enters under the root, so the
    mean square becomes ms / (ms + eps)."""
    for sd in seeds:
        rng = np.random.default_rng(400 + sd)
        x = rng.standard_normal((5, 576)) * rng.uniform(0.1, 10, size=(5, 1))
        one = np.ones(576)
        y = rms_norm(x, one, 0.0)
        _close(np.mean(y * y, axis=1), np.ones(5), 1e-12)
        _close(rms_norm(3.5 * x, one, 0.0), y, 1e-12)
        g = rng.uniform(-2, 2, size=576)
        _close(rms_norm(x, g, 0.0), y * g, 1e-12)
        ms = np.mean(x * x, axis=1)
        eps = 0.37
        ye = rms_norm(x, one, eps)
        _close(np.mean(ye * ye, axis=1), ms / (ms + eps), 1e-12)


def check_rope(rope_rotate):
    """Rotation of consecutive pairs: angle 0 is the identity; a quarter turn
    maps (x0, x1) to (-x1, x0) with the pairs (2i, 2i+1) (so e_0 goes to e_1,
    not to e_32); every pair keeps its length; turning by a then b equals
    turning by a + b; the conjugate undoes the rotation."""
    rng = np.random.default_rng(410)
    x = rng.standard_normal((3, 64))
    z = np.zeros((3, 32))
    _close(rope_rotate(x, np.ones((3, 32)), z), x, 0)
    e0 = np.zeros(64)
    e0[0] = 1.0
    q = rope_rotate(e0, np.zeros(32), np.ones(32))
    want = np.zeros(64)
    want[1] = 1.0
    _close(q, want, 0)
    y = rope_rotate(x, np.zeros((3, 32)), np.ones((3, 32)))
    _close(y[:, 0::2], -x[:, 1::2], 0)
    _close(y[:, 1::2], x[:, 0::2], 0)
    a = rng.uniform(-7, 7, size=(3, 32))
    b = rng.uniform(-7, 7, size=(3, 32))
    ra = rope_rotate(x, np.cos(a), np.sin(a))
    _close(np.hypot(ra[:, 0::2], ra[:, 1::2]), np.hypot(x[:, 0::2], x[:, 1::2]), 1e-12)
    rab = rope_rotate(ra, np.cos(b), np.sin(b))
    _close(rab, rope_rotate(x, np.cos(a + b), np.sin(a + b)), 1e-12)
    _close(rope_rotate(ra, np.cos(a), np.sin(a), conjugate=True), x, 1e-12)


def check_q_norm_rope(q_norm_rope, rms_norm, rope_rotate):
    """Only the last 64 dims are rotated, each query token by its own angles
    (pinned through the two checks above and a per-token comparison)."""
    rng = np.random.default_rng(420)
    B, s_q, h, d = 2, 3, 4, 576
    q = rng.standard_normal((B, s_q, h, d))
    g = rng.uniform(0.5, 1.5, size=d)
    th = rng.uniform(-3, 3, size=(B, s_q, 32))
    y = q_norm_rope(q, g, 1e-6, np.cos(th), np.sin(th))
    n = rms_norm(q, g, 1e-6)
    _close(y[..., :d - 64], n[..., :d - 64], 0)
    for b in range(B):
        for i in range(s_q):
            for hh in range(h):
                r = rope_rotate(n[b, i, hh, d - 64:], np.cos(th[b, i]), np.sin(th[b, i]))
                _close(y[b, i, hh, d - 64:], r, 1e-12)
    # a zero angle leaves the normalised row unchanged
    y0 = q_norm_rope(q, g, 1e-6, np.ones((B, s_q, 32)), np.zeros((B, s_q, 32)))
    _close(y0, n, 0)


def check_e4m3_encode(e4m3_encode, e4m3_to_f64):
    """Every finite code decodes and re-encodes to itself; the midpoint of
    two neighbouring codes goes to the one with an even mantissa; values
    beyond 448 saturate; random in-range values match torch's float8_e4m3fn
    cast (round to nearest even)."""
    codes = np.arange(256)
    vals = e4m3_to_f64(codes)
    fin = ~np.isnan(vals)
    assert np.array_equal(e4m3_encode(vals[fin]), codes[fin].astype(np.uint8))
    pos = [c for c in range(0x7F) if c != 0x7F]
    for c in pos[:-1]:
        mid = 0.5 * (vals[c] + vals[c + 1])
        got = int(e4m3_encode(np.array([mid]))[0])
        assert got == (c if c % 2 == 0 else c + 1), (c, got)
        assert int(e4m3_encode(np.array([-mid]))[0]) == (got | 0x80)
    assert int(e4m3_encode(np.array([1e9]))[0]) == 0x7E
    assert int(e4m3_encode(np.array([-500.0]))[0]) == 0xFE
    x = np.random.default_rng(430).standard_normal(50000).astype(np.float32) * 60
    x = x[np.abs(x) < 448]
    t = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(e4m3_encode(x), t)


def check_fp8_cast_rows(fp8_cast_rows, e4m3_to_f64):
    """Per 128-value tile: the largest magnitude maps to +-448 exactly (code
    0x7E / 0xFE), the scale is amax/448, every dequantised value is within
    half an e4m3 step (2^-4 relative, or 2^-10 scale in the subnormal range)
    of the input, and an all-zero tile has scale 1 and zero codes."""
    rng = np.random.default_rng(440)
    x = (rng.standard_normal((7, 512)) * rng.uniform(1e-3, 30, size=(7, 1))).astype(np.float32)
    x[3, 128:256] = 0
    codes, sc = fp8_cast_rows(x)
    assert codes.shape == x.shape and sc.shape == (7, 4) and sc.dtype == np.float32
    assert np.all(sc[3, 1] == 1.0) and np.all(codes[3, 128:256] == 0)
    t = x.reshape(7, 4, 128)
    ct = codes.reshape(7, 4, 128)
    deq = e4m3_to_f64(ct) * sc[..., None]
    for r in range(7):
        for j in range(4):
            if r == 3 and j == 1:
                continue
            i = int(np.argmax(np.abs(t[r, j])))
            assert ct[r, j, i] in (0x7E, 0xFE)
            assert abs(sc[r, j] - np.max(np.abs(t[r, j])) / 448.0) <= 1e-7 * sc[r, j]
    bound = np.maximum(2.0 ** -4 * np.abs(t), 2.0 ** -10 * sc[..., None]) * (1 + 1e-6)
    assert np.all(np.abs(deq - t) <= bound)


def check_out_rope_fp8(out_rope_fp8, fp8_cast_rows, rope_rotate):
    """576-dim rows: the output has no RoPE part, so the epilogue is the
    plain cast. 512-dim rows: dims 448..511 are turned back by the query
    token's angle (the result matches the fp64 conjugate rotation to fp32
    rounding) and the other dims are untouched; a rotation then its
    epilogue returns the original values."""
    rng = np.random.default_rng(450)
    B, s_q, h = 2, 2, 3
    out = rng.standard_normal((B, s_q, h, 512)).astype(np.float32)
    th = rng.uniform(-3, 3, size=(B, s_q, 32))
    c, s = np.cos(th).astype(np.float32), np.sin(th).astype(np.float32)
    codes, sc, y = out_rope_fp8(out, c, s, 576)
    c2, s2 = fp8_cast_rows(out)
    assert np.array_equal(codes, c2) and np.array_equal(sc, s2) and np.array_equal(y, out)
    codes, sc, y = out_rope_fp8(out, c, s, 512)
    assert np.array_equal(y[..., :448], out[..., :448])
    ref = rope_rotate(out[..., 448:].astype(np.float64), c[:, :, None, :].astype(np.float64),
                      s[:, :, None, :].astype(np.float64), conjugate=True)
    _close(y[..., 448:], ref, 1e-5)
    rot = rope_rotate(out[..., 448:].astype(np.float64), c[:, :, None, :].astype(np.float64),
                      s[:, :, None, :].astype(np.float64))
    full = out.copy()
    full[..., 448:] = rot.astype(np.float32)
    _, _, back = out_rope_fp8(full, c, s, 512)
    _close(back[..., 448:], out[..., 448:], 1e-5)
