"""Pins for the oracle's score modifiers (softcap, local window), its
bfloat16 decoding and its rotary embedding, each checked against something
other than the oracle itself: a library's decoding of every bit pattern,
closed forms, limits, hand-computed rotations, the algebra of rotations and
an independent numpy dense reference.  CPU only."""
import math

import numpy as np
import pytest

import oracle
from test_oracle import _dense_to_paged, _random_problem


# ---------------------------------------------------------------- bfloat16

def test_bf16_decode_matches_torch_for_every_bit_pattern():
    import torch
    bits = np.arange(65536, dtype=np.uint16)
    ref = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).double().numpy()
    got = np.array([oracle.bf16_to_double(int(b)) for b in bits])
    nan = np.isnan(ref)
    assert np.array_equal(nan, np.isnan(got))
    assert np.array_equal(got[~nan], ref[~nan])


def test_bf16_attention_equals_attention_on_the_decoded_values():
    """The bf16 path reads each element as its exact value: the same problem
    given as bf16 bit patterns and as the float64 values they stand for
    gives the same output bit for bit."""
    import torch
    rng = np.random.default_rng(21)
    P = _random_problem(rng, [3, 5], [9, 0], 4, 2, 16, 4)

    def to_bf16_bits(a):
        t = torch.from_numpy(np.nan_to_num(a, nan=0.0)).to(torch.bfloat16)
        return t.view(torch.int16).numpy().view(np.uint16), t.double().numpy()

    qb, qd = to_bf16_bits(P["query"])
    kb, kd = to_bf16_bits(P["kc"])
    vb, vd = to_bf16_bits(P["vc"])
    got = oracle.attention(qb, kb, vb, P["table"], P["cu"], P["skv"], 0.25, bf16=True)
    ref = oracle.attention(qd, kd, vd, P["table"], P["cu"], P["skv"], 0.25)
    assert np.array_equal(got, ref)


# ---------------------------------------------------------------- dense references

def _dense_modified(q_seqs, k_seqs, v_seqs, scale, softcap=0.0, window=-1):
    """softmax(mod(Q K^T * scale) + M) V with an explicit causal + band mask,
    written independently of the oracle (numpy matrices per head)."""
    outs = []
    for q, k, v in zip(q_seqs, k_seqs, v_seqs):
        ql, qh, d = q.shape
        T, kvh, _ = k.shape
        g = qh // kvh
        pos = (T - ql) + np.arange(ql)
        j = np.arange(T)
        visible = j[None, :] <= pos[:, None]
        if window >= 0:
            visible &= j[None, :] >= (pos[:, None] - window)
        y = np.empty((ql, qh, d))
        for h in range(qh):
            s = q[:, h, :].astype(np.float64) @ k[:, h // g, :].astype(np.float64).T * scale
            if softcap > 0:
                s = softcap * np.tanh(s / softcap)
            s = np.where(visible, s, -np.inf)
            s = s - s.max(axis=1, keepdims=True)
            p = np.exp(s)
            p /= p.sum(axis=1, keepdims=True)
            y[:, h, :] = p @ v[:, h // g, :].astype(np.float64)
        outs.append(y)
    return np.concatenate(outs, axis=0)


MOD_CASES = [
    ([3, 1, 16], [20, 0, 40], 4, 2, 16, 4),
    ([8, 5], [0, 33], 2, 1, 32, 8),
]


@pytest.mark.parametrize("case", range(len(MOD_CASES)))
@pytest.mark.parametrize("softcap,window", [(5.0, -1), (0.0, 0), (0.0, 3), (0.0, 17), (2.5, 6)])
def test_modifiers_match_dense_reference(case, softcap, window):
    q_lens, past, qh, kvh, d, bs = MOD_CASES[case]
    rng = np.random.default_rng(300 + case)
    P = _random_problem(rng, q_lens, past, qh, kvh, d, bs)
    scale = 1.0 / math.sqrt(d)
    got = oracle.attention(P["query"], P["kc"], P["vc"], P["table"], P["cu"], P["skv"], scale,
                           softcap=softcap, window=window)
    ref = _dense_modified(P["q_seqs"], P["k_seqs"], P["v_seqs"], scale, softcap, window)
    np.testing.assert_allclose(got, ref.reshape(got.shape), atol=1e-12, rtol=1e-12)


# ---------------------------------------------------------------- softcap

def _two_key_problem(a, v1, v2):
    """One query row e0, keys a*e0 and 0 (scores a*scale and 0), causal q_len 1."""
    d = 4
    q = np.zeros((1, 1, d))
    q[0, 0, 0] = 1.0
    k = np.zeros((2, 1, d))
    k[0, 0, 0] = a
    v = np.stack([v1, v2])[:, None, :]
    kc, vc, table = _dense_to_paged([k], [v], 2, np.random.default_rng(0), extra_blocks=1)
    return q, kc, vc, table, np.array([0, 1], np.int32), np.array([2], np.int32)


def test_softcap_two_key_closed_form():
    """Scale chosen through atanh so that the capped first score is ln 3: the
    first key then carries weight 3/4.  Capping before the scale, or not
    capping, misses that weight."""
    c, a = 2.0, 1.5
    scale = c * math.atanh(math.log(3.0) / c) / a
    v1 = np.array([1.0, -2.0, 0.5, 4.0])
    v2 = np.array([-3.0, 1.0, 2.0, 0.0])
    q, kc, vc, table, cu, skv = _two_key_problem(a, v1, v2)
    got = oracle.attention(q, kc, vc, table, cu, skv, scale, softcap=c)[0, 0]
    np.testing.assert_allclose(got, 0.75 * v1 + 0.25 * v2, atol=1e-12)
    plain = oracle.attention(q, kc, vc, table, cu, skv, scale)[0, 0]
    assert np.abs(plain - got).max() > 1e-3


def test_softcap_saturates_at_plus_minus_cap():
    """Scores far beyond the cap sit at +c or -c (tanh's limits): two huge
    positive scores weigh e^c each, a huge negative one e^-c."""
    c = 1.0
    d = 4
    q = np.zeros((1, 1, d))
    q[0, 0, 0] = 1.0
    k = np.zeros((3, 1, d))
    k[:, 0, 0] = [1e6, 1e7, -1e6]
    v = np.random.default_rng(1).standard_normal((3, 1, d))
    kc, vc, table = _dense_to_paged([k], [v], 4, np.random.default_rng(2), extra_blocks=1)
    got = oracle.attention(q, kc, vc, table, np.array([0, 1], np.int32), np.array([3], np.int32),
                           1.0, softcap=c)[0, 0]
    w = np.array([math.e, math.e, 1 / math.e])
    np.testing.assert_allclose(got, (w[:, None] * v[:, 0, :]).sum(0) / w.sum(), atol=1e-12)


def test_huge_softcap_is_plain_attention():
    rng = np.random.default_rng(7)
    P = _random_problem(rng, [4, 2], [10, 30], 4, 2, 16, 8)
    a = oracle.attention(P["query"], P["kc"], P["vc"], P["table"], P["cu"], P["skv"], 0.25,
                         softcap=1e9)
    b = oracle.attention(P["query"], P["kc"], P["vc"], P["table"], P["cu"], P["skv"], 0.25)
    np.testing.assert_allclose(a, b, atol=1e-12)


# ---------------------------------------------------------------- local window

def test_window_zero_sees_only_its_own_key():
    rng = np.random.default_rng(8)
    q_lens, past = [3, 1, 5], [7, 0, 2]
    P = _random_problem(rng, q_lens, past, 4, 2, 16, 4)
    got = oracle.attention(P["query"], P["kc"], P["vc"], P["table"], P["cu"], P["skv"], 0.25,
                           window=0)
    t = 0
    for b, (ql, p) in enumerate(zip(q_lens, past)):
        for i in range(ql):
            for h in range(4):
                assert np.array_equal(got[t, h], P["v_seqs"][b][p + i, h // 2])
            t += 1


def test_window_covering_the_sequence_is_causal():
    rng = np.random.default_rng(9)
    P = _random_problem(rng, [6, 2], [10, 25], 4, 4, 16, 8)
    a = oracle.attention(P["query"], P["kc"], P["vc"], P["table"], P["cu"], P["skv"], 0.25,
                         window=40)
    b = oracle.attention(P["query"], P["kc"], P["vc"], P["table"], P["cu"], P["skv"], 0.25)
    assert np.array_equal(a, b)


# ---------------------------------------------------------------- rotary

def test_token_positions_match_loop():
    cu = np.array([0, 2, 2, 5, 6], np.int32)
    skv = np.array([9, 4, 3, 1], np.int32)
    assert list(oracle.token_positions(cu, skv)) == [7, 8, 0, 1, 2, 0]


def test_rotary_hand_values_tell_pairings_apart():
    """Pair 0 turned by 90 degrees, pair 1 by 0, on x = [1, 2, 3, 4]:
    split pairing rotates (x0, x2) -> (-3, 1); interleaved rotates
    (x0, x1) -> (-2, 1)."""
    x = np.array([[[1.0, 2.0, 3.0, 4.0]]])
    cos = np.array([[0.0, 1.0]])
    sin = np.array([[1.0, 0.0]])
    pos = np.array([0])
    split = oracle.rotary(x, pos, cos, sin, 4, interleaved=False)[0, 0]
    inter = oracle.rotary(x, pos, cos, sin, 4, interleaved=True)[0, 0]
    assert list(split) == [-3.0, 2.0, 1.0, 4.0]
    assert list(inter) == [-2.0, 1.0, 3.0, 4.0]


def _rope_cache(max_pos, rotary_dim, base=10000.0):
    m = np.arange(rotary_dim // 2)
    theta = base ** (-2.0 * m / rotary_dim)
    ang = np.arange(max_pos)[:, None] * theta[None, :]
    return np.cos(ang), np.sin(ang)


@pytest.mark.parametrize("interleaved", [False, True])
def test_rotary_pass_through_and_position_zero(interleaved):
    rng = np.random.default_rng(10)
    x = rng.standard_normal((5, 3, 32)).astype(np.float16)
    cos, sin = (c.astype(np.float16) for c in _rope_cache(64, 16))
    pos = np.array([0, 3, 9, 0, 63])
    y = oracle.rotary(x, pos, cos, sin, 16, interleaved)
    assert np.array_equal(y[:, :, 16:], x[:, :, 16:].astype(np.float64))
    assert np.array_equal(y[pos == 0], x[pos == 0].astype(np.float64))
    assert not np.allclose(y[1, :, :16], x[1, :, :16].astype(np.float64))


@pytest.mark.parametrize("interleaved", [False, True])
def test_rotary_is_a_rotation_group(interleaved):
    """fp64 caches of a standard RoPE: each pair keeps its norm, turning by a
    then by b equals turning by a + b, and a dot product of two rotated
    vectors depends only on their positions' difference."""
    rd, d = 32, 48
    cos, sin = _rope_cache(200, rd)
    rng = np.random.default_rng(11)
    x = rng.standard_normal((6, 2, d))
    a = np.array([0, 1, 5, 17, 40, 90])
    b = np.array([3, 8, 0, 60, 41, 9])
    ya = oracle.rotary(x, a, cos, sin, rd, interleaved)
    if interleaved:
        n0 = x[..., :rd:2] ** 2 + x[..., 1:rd:2] ** 2
        n1 = ya[..., :rd:2] ** 2 + ya[..., 1:rd:2] ** 2
    else:
        n0 = x[..., :rd // 2] ** 2 + x[..., rd // 2:rd] ** 2
        n1 = ya[..., :rd // 2] ** 2 + ya[..., rd // 2:rd] ** 2
    np.testing.assert_allclose(n1, n0, rtol=1e-12)
    yab = oracle.rotary(np.ascontiguousarray(ya), b, cos, sin, rd, interleaved)
    np.testing.assert_allclose(yab, oracle.rotary(x, a + b, cos, sin, rd, interleaved), atol=1e-9)
    q = rng.standard_normal((1, 1, d))
    k = rng.standard_normal((1, 1, d))
    dots = []
    for shift in (0, 7, 100):
        rq = oracle.rotary(q, np.array([30 + shift]), cos, sin, rd, interleaved)
        rk = oracle.rotary(k, np.array([12 + shift]), cos, sin, rd, interleaved)
        dots.append(float((rq * rk).sum()))
    np.testing.assert_allclose(dots, dots[0], rtol=1e-10)


def test_rotary_reads_strided_packed_rows():
    """Heads of a packed QKV row, read through the token stride, rotate like
    the same heads copied out densely."""
    rng = np.random.default_rng(12)
    qkv = rng.standard_normal((4, 2 + 2 * 1, 16)).astype(np.float16)
    cos, sin = (c.astype(np.float16) for c in _rope_cache(32, 16))
    pos = np.array([1, 2, 3, 30])
    k_view = qkv[:, 2:3, :]
    got = oracle.rotary(k_view, pos, cos, sin, 16, False)
    want = oracle.rotary(np.ascontiguousarray(k_view), pos, cos, sin, 16, False)
    assert np.array_equal(got, want)


# ---------------------------------------------------------------- INT4 cache

def test_int4_codes_round_trip_and_round_ties_to_even():
    for s in (1.0, 0.25, 4.0):
        for k in range(-8, 8):
            assert oracle.quantize_int4(k * s, s) == k
    # Ties: 2.5 -> 2 and 3.5 -> 4 (to even), -2.5 -> -2; half-away rounding gives 3, 4, -3.
    assert [oracle.quantize_int4(v, 0.5) for v in (1.25, 1.75, -1.25)] == [2, 4, -2]
    # Clamping at both ends, including a tie that rounds past 7.
    assert [oracle.quantize_int4(v, 1.0) for v in (100.0, 7.5, -8.5, -100.0)] == [7, 7, -8, -8]


def test_int4_packing_by_hand():
    """Codes (3, -2, 7, -8) of one head row pack into bytes 0xE3, 0x87 (low
    nibble = even channel), written at the token's slot only."""
    key = np.array([[[3.0, -2.0, 7.0, -8.0]]], dtype=np.float16)
    value = -key
    kc = np.zeros((2, 2, 1, 2), dtype=np.uint8)
    vc = np.zeros_like(kc)
    ones = np.ones((1, 4), dtype=np.float32)
    oracle.scatter_kv_int4(key, value, np.array([3], np.int32), ones, ones, kc, vc)
    assert list(kc.reshape(-1, 2)[3]) == [0xE3, 0x87]
    assert list(vc.reshape(-1, 2)[3]) == [0x2D, 0x79]      # codes (-3, 2, -7, 7): 8 clamps to 7
    assert not kc.reshape(-1, 2)[:3].any()
    deq = oracle.dequantize_int4(kc, np.full((1, 4), 0.5, np.float32))
    assert list(deq.reshape(-1, 4)[3]) == [1.5, -1.0, 3.5, -4.0]


def test_int4_error_bound_and_exact_grid():
    """Dequantised codes lie within half a scale step of in-range inputs, and
    inputs on the grid come back exactly."""
    rng = np.random.default_rng(13)
    kvh, d = 2, 16
    scale = rng.uniform(0.05, 0.5, size=(kvh, d)).astype(np.float32)
    x = (rng.uniform(-7.4, 7.4, size=(50, kvh, d)) * scale).astype(np.float16)
    kc = np.zeros((50, 1, kvh, d // 2), dtype=np.uint8)
    vc = np.zeros_like(kc)
    slots = np.arange(50, dtype=np.int32)
    oracle.scatter_kv_int4(x, x, slots, scale, scale, kc, vc)
    deq = oracle.dequantize_int4(kc, scale)[:, 0]
    assert (np.abs(deq - x.astype(np.float64)) <= scale.astype(np.float64) / 2 * (1 + 1e-6)).all()
    grid = (rng.integers(-8, 8, size=(50, kvh, d)) * 0.25).astype(np.float16)
    quarter = np.full((kvh, d), 0.25, np.float32)
    oracle.scatter_kv_int4(grid, grid, slots, quarter, quarter, kc, vc)
    assert np.array_equal(oracle.dequantize_int4(vc, quarter)[:, 0], grid.astype(np.float64))


def test_int4_attention_on_grid_values_equals_plain_attention():
    """Attention over an INT4 cache is attention over the values its codes
    stand for: with K and V on the quantisation grid, it equals the plain
    oracle on the f16 cache, bit for bit."""
    rng = np.random.default_rng(14)
    q_lens, past, qh, kvh, d, bs = [3, 1], [20, 9], 4, 2, 16, 8
    P = _random_problem(rng, q_lens, past, qh, kvh, d, bs, dtype=np.float16)
    s = np.float32(0.5)
    kc = (np.clip(np.rint(np.nan_to_num(P["kc"].astype(np.float32)) / s), -8, 7) * s).astype(np.float16)
    vc = (np.clip(np.rint(np.nan_to_num(P["vc"].astype(np.float32)) / s), -8, 7) * s).astype(np.float16)
    nb = kc.shape[0]
    slots = np.arange(nb * bs, dtype=np.int32)
    k4 = np.zeros((nb, bs, kvh, d // 2), np.uint8)
    v4 = np.zeros_like(k4)
    scale = np.full((kvh, d), s, np.float32)
    oracle.scatter_kv_int4(kc.reshape(-1, kvh, d), vc.reshape(-1, kvh, d), slots, scale, scale, k4, v4)
    want = oracle.attention(P["query"], kc, vc, P["table"], P["cu"], P["skv"], 0.25)
    got = oracle.attention(P["query"].astype(np.float64), oracle.dequantize_int4(k4, scale),
                           oracle.dequantize_int4(v4, scale), P["table"], P["cu"], P["skv"], 0.25)
    assert np.array_equal(got, want)


# ---------------------------------------------------------------- sparse (local + selected)

def _sel(T, kvh, rows):
    """selected [T, kvh, S] from per-(token, head) lists, -1 padded."""
    S = max(1, max((len(r) for r in rows.values()), default=1))
    a = np.full((T, kvh, S), -1, np.int32)
    for (t, h), r in rows.items():
        a[t, h, :len(r)] = r
    return a


def test_sparse_without_selections_is_the_local_window():
    rng = np.random.default_rng(15)
    P = _random_problem(rng, [3, 1, 5], [20, 9, 30], 4, 2, 16, 8)
    T = int(P["cu"][-1])
    for w in (0, 3, 100):
        a = oracle.sparse_attention(P["query"], P["kc"], P["vc"], P["table"], P["cu"], P["skv"],
                                    np.full((T, 2, 4), -1, np.int32), w, 0.25)
        b = oracle.attention(P["query"], P["kc"], P["vc"], P["table"], P["cu"], P["skv"], 0.25,
                             window=w)
        assert np.array_equal(a, b)


def test_sparse_selecting_every_earlier_key_is_causal_attention():
    rng = np.random.default_rng(16)
    P = _random_problem(rng, [2, 3], [12, 5], 4, 2, 16, 4)
    T = int(P["cu"][-1])
    every = np.broadcast_to(np.arange(40, dtype=np.int32), (T, 2, 40)).copy()
    a = oracle.sparse_attention(P["query"], P["kc"], P["vc"], P["table"], P["cu"], P["skv"],
                                every, 1, 0.25)
    b = oracle.attention(P["query"], P["kc"], P["vc"], P["table"], P["cu"], P["skv"], 0.25)
    assert np.array_equal(a, b)


def test_sparse_closed_forms_and_dense_reference():
    """Window 0 plus one selected key far back: the row averages exactly two
    value rows with softmax weights of their two scores; a duplicate or a
    future selection changes nothing; and a numpy dense reference with an
    explicit mask agrees on a random selection."""
    rng = np.random.default_rng(17)
    q_lens, past, qh, kvh, d = [2, 1], [30, 12], 4, 2, 16
    P = _random_problem(rng, q_lens, past, qh, kvh, d, 8)
    T = int(P["cu"][-1])
    sel = _sel(T, kvh, {(t, h): [3, 3, 50] for t in range(T) for h in range(kvh)})
    got = oracle.sparse_attention(P["query"], P["kc"], P["vc"], P["table"], P["cu"], P["skv"],
                                  sel, 0, 0.25)
    cu = P["cu"]
    for t in range(T):
        b = 0 if t < cu[1] else 1
        pos = past[b] + t - cu[b]
        for h in range(qh):
            k, v = P["k_seqs"][b][:, h // 2], P["v_seqs"][b][:, h // 2]
            s = np.array([P["query"][t, h] @ k[3], P["query"][t, h] @ k[pos]]) * 0.25
            w = np.exp(s - s.max())
            np.testing.assert_allclose(got[t, h], (w[0] * v[3] + w[1] * v[pos]) / w.sum(), atol=1e-12)
    # Random selections against a dense masked reference.
    sel = rng.integers(-1, 45, size=(T, kvh, 7)).astype(np.int32)
    got = oracle.sparse_attention(P["query"], P["kc"], P["vc"], P["table"], P["cu"], P["skv"],
                                  sel, 2, 0.25)
    for t in range(T):
        b = 0 if t < cu[1] else 1
        pos = past[b] + t - cu[b]
        for h in range(qh):
            keep = np.zeros(pos + 1, bool)
            keep[max(0, pos - 2):] = True
            for e in sel[t, h // 2]:
                if 0 <= e <= pos:
                    keep[e] = True
            k = P["k_seqs"][b][:pos + 1, h // 2][keep]
            v = P["v_seqs"][b][:pos + 1, h // 2][keep]
            s = k @ P["query"][t, h] * 0.25
            w = np.exp(s - s.max())
            np.testing.assert_allclose(got[t, h], w @ v / w.sum(), atol=1e-12)
