"""GPU parity of the attention variants against the fp64 oracle, through the
C ABI: bfloat16 inputs, the softcap and local-window score modifiers (the
features the PagedAttention PR's first version rejects), head sizes that are
multiples of 8 up to 128, and query-head groups that are not powers of two.
Each case runs both attention paths (split-KV decode and the tcgen05 prefill
kernel) and, where it matters, both producer paths (16-key pages through
cp.async, pages of 128 keys or more through TMA)."""
import numpy as np
import pytest

import workloads
from pa_harness import assert_close, oracle_step, poison_unused, run_gpu, tolerances

pytestmark = pytest.mark.gpu

DECODE_AND_PREFILL = [
    ([1, 3, 2, 4], [900, 40, 3000, 130]),           # decode: one and several splits
    ([9, 130, 300, 1], [0, 17, 700, 5000]),         # prefill: ragged tiles, long past, decode too
]


def _check(spec, softcap=0.0, window=None, hints=True):
    x = workloads.generate(spec)
    poison_unused(spec, x)
    got, _, status, _ = run_gpu(spec, x, hints=hints, softcap=softcap, window=window)
    want, _, _, _ = oracle_step(spec, x, softcap=softcap, window=window)
    assert status == 0
    mx, mn = tolerances(spec)
    assert_close(got, want, mx, mn, what=spec.name, elem=spec.elem)
    return got


@pytest.mark.parametrize("bs", [16, 256])
@pytest.mark.parametrize("lens", DECODE_AND_PREFILL)
@pytest.mark.parametrize("heads", [(8, 2), (16, 16)])
def test_bf16(bs, lens, heads):
    q, past = lens
    spec = workloads.custom(q, past, heads[0], heads[1], 128, bs, seed=bs + heads[0], elem="bf16")
    got = _check(spec)
    # Deterministic, as the f16 path.
    x = workloads.generate(spec)
    poison_unused(spec, x)
    outs, _, _, _ = run_gpu(spec, x, repeat=2)
    assert np.array_equal(outs[0], outs[1])


@pytest.mark.parametrize("softcap", [5.0, 30.0])
@pytest.mark.parametrize("bs", [16, 128])
@pytest.mark.parametrize("lens", DECODE_AND_PREFILL)
def test_softcap(softcap, bs, lens):
    q, past = lens
    spec = workloads.custom(q, past, 16, 4, 128, bs, seed=int(softcap) + bs)
    _check(spec, softcap=softcap)


@pytest.mark.parametrize("window", [0, 1, 17, 128, 300, 2500])
@pytest.mark.parametrize("bs", [16, 256])
@pytest.mark.parametrize("lens", DECODE_AND_PREFILL)
def test_local_window(window, bs, lens):
    q, past = lens
    spec = workloads.custom(q, past, 16, 4, 128, bs, seed=window + bs)
    _check(spec, window=window)


def test_window_softcap_bf16_together():
    spec = workloads.custom([1, 200, 4, 513], [4000, 900, 77, 0], 32, 8, 128, 16, seed=31,
                            elem="bf16")
    _check(spec, softcap=20.0, window=333)


def test_window_covering_everything_matches_no_window():
    spec = workloads.custom([1, 200, 3], [700, 100, 2000], 16, 4, 128, 16, seed=5)
    x = workloads.generate(spec)
    a, _, _, _ = run_gpu(spec, x)
    b, _, _, _ = run_gpu(spec, x, window=10 ** 6)
    assert np.array_equal(a.view(np.uint16), b.view(np.uint16))


@pytest.mark.parametrize("head_size", [8, 24, 40, 48, 80, 96, 112, 120])
@pytest.mark.parametrize("bs", [16, 128])
def test_head_sizes_padded(head_size, bs):
    q, past = [1, 3, 70, 200], [600, 33, 0, 301]
    spec = workloads.custom(q, past, 8, 2, head_size, bs, seed=head_size + bs)
    _check(spec)


@pytest.mark.parametrize("qh,kvh", [(3, 1), (6, 2), (10, 2), (12, 2), (24, 1), (20, 4)])
@pytest.mark.parametrize("bs", [16, 256])
def test_groups_not_powers_of_two(qh, kvh, bs):
    q, past = [1, 2, 4, 45, 160, 300], [1200, 30, 7, 0, 500, 64]
    spec = workloads.custom(q, past, qh, kvh, 128, bs, seed=qh * 10 + kvh + bs)
    _check(spec)


def test_group_of_three_without_hints():
    spec = workloads.custom([1, 77, 3], [4000, 10, 500], 24, 8, 64, 16, seed=9)
    _check(spec, hints=False)


@pytest.mark.parametrize("bs", [16, 32, 64])
@pytest.mark.parametrize("heads,d", [((32, 8), 128), ((16, 16), 64), ((8, 2), 32)])
def test_cp_async_page_sizes(bs, heads, d):
    """Pages smaller than the prefill kernel's 128-key tile take its cp.async
    producers: whole tiles by 16-row units (one page each), the tile holding
    the sequence end row by row.  Long pasts give many whole tiles."""
    q, past = [300, 1, 700, 129, 2], [1000, 4000, 0, 517, 60]
    spec = workloads.custom(q, past, heads[0], heads[1], d, bs, seed=bs + d)
    _check(spec)


@pytest.mark.parametrize("qh,kvh", [(48, 1), (64, 1), (128, 2), (96, 1), (128, 1)])
@pytest.mark.parametrize("bs", [16, 256])
def test_groups_above_32(qh, kvh, bs):
    """Groups of more than 32 query heads per KV head (MQA with many heads):
    every sequence, decode ones included, runs in the prefill kernel (query
    tiles of 128 / group tokens)."""
    q, past = [1, 3, 2, 45, 160], [1200, 30, 0, 500, 64]
    spec = workloads.custom(q, past, qh, kvh, 128, bs, seed=qh + kvh + bs)
    _check(spec)
    _check(spec, hints=False)
