"""GPU parity of sparse paged attention (local window plus selected
positions) against the fp64 oracle, through the C ABI."""
import math

import numpy as np
import pytest

import oracle
import workloads
from pa_harness import (MAX_ABS, MAX_ABS_BF16, MEAN_ABS, MEAN_ABS_BF16, assert_close,
                        host_bits, poison_unused, to_dev)

pytestmark = pytest.mark.gpu


def _selections(spec, x, num_selected, rng, extra_past=True):
    """Per (token, KV head): a sorted, duplicate-free sample of positions in
    [0, P] (some inside the window, some -- when extra_past -- beyond P),
    -1 padded to num_selected."""
    pos = oracle.token_positions(x["cu_seqlens_q"], x["seqlens_kv"])
    T = spec.token_count
    sel = np.full((T, spec.kv_heads, max(1, num_selected)), -1, np.int32)
    for t in range(T):
        for h in range(spec.kv_heads):
            hi = int(pos[t]) + (40 if extra_past else 1)
            k = int(rng.integers(0, min(num_selected, hi) + 1))
            sel[t, h, :k] = np.sort(rng.choice(hi, size=k, replace=False))
    return sel


def _run(spec, x, sel, window):
    import torch
    import scatter_kv_b200 as pa
    dv = to_dev(x)
    dims = pa.make_dims(batch=spec.batch, token_count=spec.token_count, q_heads=spec.q_heads,
                        kv_heads=spec.kv_heads, head_size=spec.head_size,
                        num_blocks=spec.num_blocks, block_size=spec.block_size,
                        max_blocks_per_seq=x["block_table"].shape[1],
                        dtype=pa.PA_DTYPE_BF16 if spec.elem == "bf16" else pa.PA_DTYPE_F16)
    bufs = pa.allocate(dims)
    pa.pa_compute_slot_mapping(dv["block_table"], dv["cu_seqlens_q"], dv["seqlens_kv"],
                               bufs.slot_mapping, dims, bufs.status)
    pa.pa_scatter_kv(dv["key"], dv["value"], bufs.slot_mapping, dv["key_cache"],
                     dv["value_cache"], dims, bufs.status)
    seld = torch.from_numpy(sel).cuda()
    pa.pa_sparse_attention(dv["query"], dv["key_cache"], dv["value_cache"], dv["block_table"],
                           dv["cu_seqlens_q"], dv["seqlens_kv"], seld, sel.shape[2], window, 0.0,
                           bufs.out, dims, bufs.status)
    torch.cuda.synchronize()
    return host_bits(bufs.out, spec.elem), int(bufs.status[0].item())


def _want(spec, x, sel, window):
    bf16 = spec.elem == "bf16"
    kc, vc = x["key_cache"].copy(), x["value_cache"].copy()
    slots = oracle.slot_mapping(x["block_table"], x["cu_seqlens_q"], x["seqlens_kv"],
                                spec.block_size)
    oracle.scatter_kv(x["key"], x["value"], slots, kc, vc)
    return oracle.sparse_attention(x["query"], kc, vc, x["block_table"], x["cu_seqlens_q"],
                                   x["seqlens_kv"], sel, window,
                                   1.0 / math.sqrt(spec.head_size), bf16=bf16)


CASES = [
    # q_lens, past, qh, kvh, d, bs, num_selected, window, elem
    ([1, 1, 1, 1], [700, 3000, 45, 2000], 32, 8, 128, 16, 64, 16, "f16"),
    ([1, 5, 2], [1500, 300, 4000], 16, 4, 128, 256, 200, 0, "f16"),
    ([3, 1], [900, 60], 8, 8, 64, 32, 33, 100, "f16"),
    ([1, 2, 1], [2500, 800, 90], 64, 8, 128, 128, 500, 64, "f16"),
    ([4, 1], [100, 5000], 16, 2, 32, 16, 0, 7, "f16"),
    ([1, 1, 3], [3000, 700, 64], 32, 8, 128, 16, 64, 16, "bf16"),
    ([2, 1], [1000, 3000], 12, 4, 16, 16, 20, 3, "f16"),
]


@pytest.mark.parametrize("case", CASES, ids=[f"c{i}" for i in range(len(CASES))])
def test_sparse_matches_oracle(case):
    q_lens, past, qh, kvh, d, bs, S, window, elem = case
    spec = workloads.custom(q_lens, past, qh, kvh, d, bs, seed=S + window, elem=elem)
    x = workloads.generate(spec)
    poison_unused(spec, x)
    sel = _selections(spec, x, S, np.random.default_rng(S))
    got, status = _run(spec, x, sel, window)
    want = _want(spec, x, sel, window)
    assert status == 0
    mx, mn = (MAX_ABS_BF16, MEAN_ABS_BF16) if elem == "bf16" else (MAX_ABS, MEAN_ABS)
    assert_close(got, want, mx, mn, what=f"sparse {case}", elem=elem)
    again, _ = _run(spec, x, sel, window)
    assert np.array_equal(got, again)


def test_sparse_long_selection():
    """2048 selections and a 128-key window over sequences up to 9000 keys."""
    spec = workloads.custom([1, 1, 2], [9000, 4000, 2500], 32, 8, 128, 16, seed=99)
    x = workloads.generate(spec)
    poison_unused(spec, x)
    sel = _selections(spec, x, 2048, np.random.default_rng(3), extra_past=False)
    got, status = _run(spec, x, sel, 128)
    assert status == 0
    assert_close(got, _want(spec, x, sel, 128), what="sparse long selection")


def test_sparse_flags_an_unsorted_selection():
    """A selection that is not strictly increasing zeroes that (token, KV
    head)'s rows and sets the status bit; the other rows are unaffected."""
    import scatter_kv_b200 as pa
    spec = workloads.custom([1, 1], [500, 600], 8, 2, 64, 16, seed=4)
    x = workloads.generate(spec)
    sel = _selections(spec, x, 8, np.random.default_rng(4), extra_past=False)
    sel[1, 1, :3] = [30, 20, 40]
    got, status = _run(spec, x, sel, 4)
    assert status & pa.PA_DEV_BAD_SELECTION
    assert not got[1, 4:8].any()
    want = _want(spec, x, sel, 4)
    assert_close(got[0], want[0], what="token 0")
    assert_close(got[1, :4], want[1, :4], what="token 1, KV head 0")
