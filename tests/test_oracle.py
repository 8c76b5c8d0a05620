"""Pins for the fp64 oracle, checked against things other than itself:
the FlexAttention doc's printed worked examples, brute-force dense causal
attention written independently with numpy, closed forms, invariants and
the known-bad clamp variant the PagedAttention PR fixed.  CPU only."""
import math
import os

import numpy as np
import pytest

import oracle
import workloads

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _read_golden(name):
    arrays = {}
    with open(os.path.join(GOLDEN, name)) as f:
        lines = [ln.strip() for ln in f if ln.strip() and not ln.startswith("#")]
    for hdr, vals in zip(lines[0::2], lines[1::2]):
        parts = hdr.split()
        shape = tuple(int(x) for x in parts[1:])
        arrays[parts[0]] = np.array([float(v) for v in vals.split()], dtype=np.float64).reshape(shape)
    return arrays


def _dense_to_paged(k_seqs, v_seqs, block_size, rng, extra_blocks=3):
    """Place per-sequence contiguous K/V [T_b, kvh, d] into a pool of pages
    handed out by a random permutation.  Returns caches and block table."""
    kvh, d = k_seqs[0].shape[1:]
    pages = [-(-k.shape[0] // block_size) for k in k_seqs]
    nb = sum(pages) + extra_blocks
    order = rng.permutation(nb)
    maxb = max(1, max(pages))
    table = np.full((len(k_seqs), maxb), -1, dtype=np.int32)
    kc = np.full((nb, block_size, kvh, d), np.nan, dtype=k_seqs[0].dtype)
    vc = np.full_like(kc, np.nan)
    nxt = 0
    for b, (k, v) in enumerate(zip(k_seqs, v_seqs)):
        for p in range(pages[b]):
            blk = order[nxt]
            nxt += 1
            table[b, p] = blk
            rows = k[p * block_size:(p + 1) * block_size]
            kc[blk, :rows.shape[0]] = rows
            vc[blk, :rows.shape[0]] = v[p * block_size:(p + 1) * block_size]
    return kc, vc, table


def _dense_reference(q_seqs, k_seqs, v_seqs, scale, causal=True, clamp_max_q=None):
    """softmax(Q K^T * scale + M) V per sequence and head, with an explicit
    (q_len x T) mask; clamp_max_q reproduces the clamped-past variant."""
    outs = []
    for q, k, v in zip(q_seqs, k_seqs, v_seqs):
        ql, qh, d = q.shape
        T, kvh, _ = k.shape
        g = qh // kvh
        past = T - ql
        if clamp_max_q is not None:
            past = max(0, T - clamp_max_q)
        y = np.empty((ql, qh, d))
        for h in range(qh):
            s = q[:, h, :].astype(np.float64) @ k[:, h // g, :].astype(np.float64).T * scale
            if causal:
                mask = np.arange(T)[None, :] > (past + np.arange(ql))[:, None]
                s = np.where(mask, -np.inf, s)
            s = s - s.max(axis=1, keepdims=True)
            p = np.exp(s)
            p /= p.sum(axis=1, keepdims=True)
            y[:, h, :] = p @ v[:, h // g, :].astype(np.float64)
        outs.append(y)
    return np.concatenate(outs, axis=0) if outs else np.zeros((0,))


def _random_problem(rng, q_lens, past, qh, kvh, d, bs, dtype=np.float64):
    q_seqs, k_seqs, v_seqs = [], [], []
    for ql, p in zip(q_lens, past):
        T = ql + p
        q_seqs.append(rng.standard_normal((ql, qh, d)).astype(dtype))
        k_seqs.append(rng.standard_normal((T, kvh, d)).astype(dtype))
        v_seqs.append(rng.standard_normal((T, kvh, d)).astype(dtype))
    kc, vc, table = _dense_to_paged(k_seqs, v_seqs, bs, rng)
    query = np.concatenate(q_seqs, axis=0) if q_seqs else np.zeros((0, qh, d), dtype)
    cu = np.concatenate([[0], np.cumsum(q_lens)]).astype(np.int32)
    skv = (np.asarray(q_lens) + np.asarray(past)).astype(np.int32)
    return dict(q_seqs=q_seqs, k_seqs=k_seqs, v_seqs=v_seqs, query=query, kc=kc, vc=vc,
                table=table, cu=cu, skv=skv)


# ---------------------------------------------------------------- fp16 decode

def test_half_decode_matches_ieee_for_every_bit_pattern():
    bits = np.arange(65536, dtype=np.uint16)
    ref = bits.view(np.float16).astype(np.float64)
    got = np.array([oracle.half_to_double(int(b)) for b in bits])
    same = (got == ref) | (np.isnan(got) & np.isnan(ref))
    assert same.all()


# ------------------------------------------------ FlexAttention worked examples

def _flex_pin(name, block_size, seed):
    g = _read_golden(name)
    Q, K, V, Y = g["Q"][0], g["K"][0], g["V"][0], g["Y"][0]   # (heads, seq, d)
    qh, S, d = Q.shape
    kvh, L, _ = K.shape
    query = np.ascontiguousarray(Q.transpose(1, 0, 2))         # packed [token, head, d]
    k_seq = np.ascontiguousarray(K.transpose(1, 0, 2))         # [L, kvh, d]
    v_seq = np.ascontiguousarray(V.transpose(1, 0, 2))
    # The example's inputs are float32 values; take them to fp64 exactly.
    query = query.astype(np.float32).astype(np.float64)
    k_seq = k_seq.astype(np.float32).astype(np.float64)
    v_seq = v_seq.astype(np.float32).astype(np.float64)
    rng = np.random.default_rng(seed)
    kc, vc, table = _dense_to_paged([k_seq], [v_seq], block_size, rng)
    cu = np.array([0, S], dtype=np.int32)
    skv = np.array([L], dtype=np.int32)
    return query, kc, vc, table, cu, skv, Y.transpose(1, 0, 2), d


@pytest.mark.parametrize("name", ["flex_attention_basic.txt", "flex_attention_gqa.txt"])
@pytest.mark.parametrize("block_size,seed", [(1, 0), (2, 1), (4, 2)])
def test_flex_attention_worked_examples(name, block_size, seed):
    query, kc, vc, table, cu, skv, Y, d = _flex_pin(name, block_size, seed)
    got = oracle.attention(query, kc, vc, table, cu, skv, 1.0 / math.sqrt(d), causal=False)
    np.testing.assert_allclose(got, Y, atol=1e-6, rtol=0)


@pytest.mark.parametrize("name", ["flex_attention_basic.txt", "flex_attention_gqa.txt"])
def test_flex_examples_reject_wrong_scale(name):
    query, kc, vc, table, cu, skv, Y, d = _flex_pin(name, 2, 3)
    got = oracle.attention(query, kc, vc, table, cu, skv, 1.0, causal=False)
    assert np.abs(got - Y).max() > 1e-3


def test_gqa_example_pins_head_mapping():
    """The GQA example separates floor(h / group) from the other plausible
    mapping h % kv_heads: computing it that way misses the printed values."""
    g = _read_golden("flex_attention_gqa.txt")
    Q, K, V, Y = g["Q"][0], g["K"][0], g["V"][0], g["Y"][0]
    qh, kvh, d = Q.shape[0], K.shape[0], Q.shape[2]
    wrong = np.empty_like(Y)
    for h in range(qh):
        s = Q[h] @ K[h % kvh].T / math.sqrt(d)
        p = np.exp(s - s.max(axis=1, keepdims=True))
        wrong[h] = (p / p.sum(axis=1, keepdims=True)) @ V[h % kvh]
    assert np.abs(wrong - Y).max() > 1e-2


# ------------------------------------------------ brute-force dense causal

CASES = [
    # q_lens, past, q_heads, kv_heads, d, block_size
    ([1, 4], [7, 20], 2, 1, 16, 16),
    ([3, 1, 5, 2], [0, 9, 2, 30], 4, 2, 8, 4),
    ([6], [0], 3, 3, 4, 2),
    ([1, 1, 1], [5, 0, 17], 8, 2, 8, 8),
    ([2, 0, 3], [4, 6, 1], 4, 1, 8, 4),          # a zero-length sequence in the middle
    ([16, 4, 1], [16, 28, 63], 4, 4, 16, 16),
    ([1, 3, 2], [9, 0, 5], 64, 1, 8, 4),          # MQA, a group of 64
    ([2, 1], [3, 6], 96, 2, 8, 2),                # a group of 48
]


@pytest.mark.parametrize("case", range(len(CASES)))
@pytest.mark.parametrize("dtype", [np.float64, np.float16])
def test_oracle_matches_dense_causal_attention(case, dtype):
    q_lens, past, qh, kvh, d, bs = CASES[case]
    rng = np.random.default_rng(100 + case)
    P = _random_problem(rng, q_lens, past, qh, kvh, d, bs, dtype=dtype)
    scale = 1.0 / math.sqrt(d)
    got = oracle.attention(P["query"], P["kc"], P["vc"], P["table"], P["cu"], P["skv"], scale)
    ref = _dense_reference(P["q_seqs"], P["k_seqs"], P["v_seqs"], scale)
    assert got.shape == (sum(q_lens), qh, d)
    np.testing.assert_allclose(got, ref.reshape(got.shape), atol=1e-12, rtol=1e-12)


def test_clamped_past_variant_is_visible():
    """The clamp past = max(0, T - max_q) leaks future keys when q_len varies;
    the oracle must differ from it on such a batch and agree on a uniform one."""
    rng = np.random.default_rng(5)
    q_lens, past = [1, 6, 3], [10, 2, 0]
    P = _random_problem(rng, q_lens, past, 2, 1, 8, 4)
    scale = 1.0 / math.sqrt(8)
    got = oracle.attention(P["query"], P["kc"], P["vc"], P["table"], P["cu"], P["skv"], scale)
    bad = _dense_reference(P["q_seqs"], P["k_seqs"], P["v_seqs"], scale, clamp_max_q=6)
    assert np.abs(got - bad.reshape(got.shape)).max() > 1e-3
    q_lens, past = [4, 4], [0, 0]
    P = _random_problem(rng, q_lens, past, 2, 1, 8, 4)
    got = oracle.attention(P["query"], P["kc"], P["vc"], P["table"], P["cu"], P["skv"], scale)
    same = _dense_reference(P["q_seqs"], P["k_seqs"], P["v_seqs"], scale, clamp_max_q=4)
    np.testing.assert_allclose(got, same.reshape(got.shape), atol=1e-12)


# ------------------------------------------------ closed forms and invariants

def test_first_row_of_fresh_sequence_is_v0_exactly():
    rng = np.random.default_rng(9)
    P = _random_problem(rng, [5, 3], [0, 0], 4, 2, 16, 4, dtype=np.float16)
    got = oracle.attention(P["query"], P["kc"], P["vc"], P["table"], P["cu"], P["skv"], 0.25)
    for b, start in enumerate([0, 5]):
        for h in range(4):
            v0 = P["v_seqs"][b][0, h // 2].astype(np.float64)
            assert np.array_equal(got[start, h], v0)


def test_equal_keys_give_mean_of_visible_values():
    rng = np.random.default_rng(11)
    q_lens, past, d = [3, 2], [4, 7], 8
    k_seqs = [np.ones((ql + p, 1, d)) * 0.5 for ql, p in zip(q_lens, past)]
    v_seqs = [rng.standard_normal((ql + p, 1, d)) for ql, p in zip(q_lens, past)]
    q_seqs = [rng.standard_normal((ql, 2, d)) for ql in q_lens]
    kc, vc, table = _dense_to_paged(k_seqs, v_seqs, 4, rng)
    cu = np.array([0, 3, 5], dtype=np.int32)
    skv = np.array([7, 9], dtype=np.int32)
    got = oracle.attention(np.concatenate(q_seqs), kc, vc, table, cu, skv, 0.3)
    row = 0
    for b in range(2):
        for i in range(q_lens[b]):
            want = v_seqs[b][:past[b] + i + 1, 0].mean(axis=0)
            for h in range(2):
                np.testing.assert_allclose(got[row, h], want, atol=1e-13)
            row += 1


def test_single_query_sees_every_key():
    rng = np.random.default_rng(12)
    P = _random_problem(rng, [1, 1], [13, 6], 4, 2, 8, 4)
    s = 0.35
    causal = oracle.attention(P["query"], P["kc"], P["vc"], P["table"], P["cu"], P["skv"], s)
    full = oracle.attention(P["query"], P["kc"], P["vc"], P["table"], P["cu"], P["skv"], s,
                            causal=False)
    assert np.array_equal(causal, full)


def test_identity_table_reads_cache_as_contiguous_rows():
    """With blocks handed out in order, the pool reshaped to [rows, kvh, d] is
    the sequences' keys back to back: checks the layout without restating it."""
    rng = np.random.default_rng(13)
    bs, kvh, d = 4, 2, 8
    q_lens, past = [3, 2], [5, 6]           # T = 8 and 8: whole pages
    T = [8, 8]
    k = rng.standard_normal((16, kvh, d))
    v = rng.standard_normal((16, kvh, d))
    kc = k.reshape(4, bs, kvh, d).copy()
    vc = v.reshape(4, bs, kvh, d).copy()
    table = np.array([[0, 1], [2, 3]], dtype=np.int32)
    q = rng.standard_normal((5, 4, d))
    got = oracle.attention(q, kc, vc, table, np.array([0, 3, 5], np.int32),
                           np.array(T, np.int32), 0.4)
    ref = _dense_reference([q[:3], q[3:]], [k[:8], k[8:]], [v[:8], v[8:]], 0.4)
    np.testing.assert_allclose(got, ref, atol=1e-12)


def test_page_permutation_is_bit_identical():
    spec = workloads.custom([1, 5, 3, 2], [37, 0, 12, 50], 8, 2, 16, 8, num_blocks=40)
    a = workloads.generate(spec, fill=np.nan)
    rng = np.random.default_rng(3)
    b = workloads.generate(spec, fill=np.nan, block_order=rng.permutation(40))
    # Same logical contents under a different page placement.
    for name in ("key_cache", "value_cache"):
        b[name][:] = np.nan
        for s in range(spec.batch):
            for p in range(int(spec.pages_per_seq[s])):
                b[name][b["block_table"][s, p]] = a[name][a["block_table"][s, p]]
    args = ("cu_seqlens_q", "seqlens_kv")
    ya = oracle.attention(a["query"], a["key_cache"], a["value_cache"], a["block_table"],
                          a[args[0]], a[args[1]], 0.25)
    yb = oracle.attention(a["query"], b["key_cache"], b["value_cache"], b["block_table"],
                          a[args[0]], a[args[1]], 0.25)
    assert np.array_equal(ya, yb)
    assert np.isfinite(ya).all()


def test_row_subset_matches_full_computation():
    spec = workloads.custom([2, 1, 4], [3, 9, 0], 4, 2, 16, 4)
    x = workloads.generate(spec, fill=np.nan)
    full = oracle.attention(x["query"], x["key_cache"], x["value_cache"], x["block_table"],
                            x["cu_seqlens_q"], x["seqlens_kv"], 0.25)
    rows = np.array([[0, 0], [6, 3], [2, 1], [4, 2]], dtype=np.int64)
    sub = oracle.attention(x["query"], x["key_cache"], x["value_cache"], x["block_table"],
                           x["cu_seqlens_q"], x["seqlens_kv"], 0.25, rows=rows)
    for r, (t, h) in enumerate(rows):
        assert np.array_equal(sub[r], full[t, h])


# ------------------------------------------------ scatter and slot mapping

def _slots_by_loop(table, cu, skv, bs):
    out = []
    for b in range(len(skv)):
        ql = cu[b + 1] - cu[b]
        for i in range(ql):
            pos = skv[b] - ql + i
            out.append(table[b][pos // bs] * bs + pos % bs)
    return np.array(out, dtype=np.int32)


@pytest.mark.parametrize("cfg", [0, 1, 3, 4])
def test_slot_mapping_matches_loop(cfg):
    spec = workloads.CONFIGS[cfg]()
    rng = np.random.Generator(np.random.PCG64(spec.seed))
    # Only the metadata is needed: draw the block table the way generate() does.
    pages = spec.pages_per_seq
    order = rng.permutation(spec.num_blocks)
    table = np.full((spec.batch, int(pages.max())), -1, np.int32)
    n = 0
    for b in range(spec.batch):
        table[b, :pages[b]] = order[n:n + pages[b]]
        n += pages[b]
    cu = np.concatenate([[0], np.cumsum(spec.q_lens)]).astype(np.int32)
    skv = spec.seqlens_kv.astype(np.int32)
    got = oracle.slot_mapping(table, cu, skv, spec.block_size)
    assert np.array_equal(got, _slots_by_loop(table, cu, skv, spec.block_size))
    assert len(set(got.tolist())) == got.size


def test_slot_mapping_skips_zero_length_sequences():
    table = np.array([[3, 1], [0, -1], [2, 4]], dtype=np.int32)
    cu = np.array([0, 2, 2, 5], dtype=np.int32)
    skv = np.array([5, 3, 7], dtype=np.int32)
    got = oracle.slot_mapping(table, cu, skv, 4)
    # seq 0: positions 3,4 -> block 3 row 3, block 1 row 0; seq 2: positions 4,5,6 -> block 4.
    assert got.tolist() == [15, 4, 16, 17, 18]


def test_scatter_matches_loop_and_skips_negative_slots():
    rng = np.random.default_rng(21)
    nb, bs, kvh, d, T = 6, 4, 2, 8, 7
    key = rng.standard_normal((T, kvh, d)).astype(np.float16)
    value = rng.standard_normal((T, kvh, d)).astype(np.float16)
    slots = np.array([5, 0, -1, 23, 12, 7, -3], dtype=np.int32)
    kc = rng.standard_normal((nb, bs, kvh, d)).astype(np.float16)
    vc = rng.standard_normal((nb, bs, kvh, d)).astype(np.float16)
    kc_ref, vc_ref = kc.copy(), vc.copy()
    for t, s in enumerate(slots):
        if s >= 0:
            kc_ref.reshape(nb * bs, kvh, d)[s] = key[t]
            vc_ref.reshape(nb * bs, kvh, d)[s] = value[t]
    oracle.scatter_kv(key, value, slots, kc, vc)
    assert np.array_equal(kc.view(np.uint16), kc_ref.view(np.uint16))
    assert np.array_equal(vc.view(np.uint16), vc_ref.view(np.uint16))


def test_scatter_then_attention_reads_new_tokens():
    """Tokens written by the scatter are the ones attention reads at
    positions [past, T): the last query of a sequence with past 0 and all-equal
    keys averages exactly the new values."""
    spec = workloads.custom([3], [0], 2, 1, 8, 4)
    x = workloads.generate(spec, fill=np.nan)
    x["key"][:] = 0.5
    slots = oracle.slot_mapping(x["block_table"], x["cu_seqlens_q"], x["seqlens_kv"], 4)
    oracle.scatter_kv(x["key"], x["value"], slots, x["key_cache"], x["value_cache"])
    y = oracle.attention(x["query"], x["key_cache"], x["value_cache"], x["block_table"],
                         x["cu_seqlens_q"], x["seqlens_kv"], 0.3)
    want = x["value"][:, 0].astype(np.float64).mean(axis=0)
    np.testing.assert_allclose(y[2, 0], want, atol=1e-12)
    np.testing.assert_allclose(y[2, 1], want, atol=1e-12)


def test_kv_slots_matches_loop():
    table = np.array([[2, 0], [1, 3]], dtype=np.int32)
    skv = np.array([5, 2], dtype=np.int32)
    got = oracle.kv_slots(table, skv, 4)
    assert got.tolist() == [8, 9, 10, 11, 0, 4, 5]


def test_empty_batch():
    spec = workloads.custom([0, 0], [3, 0], 2, 1, 8, 4)
    x = workloads.generate(spec)
    y = oracle.attention(x["query"], x["key_cache"], x["value_cache"], x["block_table"],
                         x["cu_seqlens_q"], x["seqlens_kv"], 0.3)
    assert y.shape == (0, 2, 8)
    assert oracle.slot_mapping(x["block_table"], x["cu_seqlens_q"], x["seqlens_kv"], 4).size == 0
