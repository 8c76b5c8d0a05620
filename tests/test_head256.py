"""GPU parity of attention at head sizes 136 .. 256 against the fp64 oracle,
through the C ABI.  Head sizes up to 256 run the split-KV decode kernel at
256 columns and the tcgen05 prefill kernel that holds one 128-row query
tile per CTA (S double-buffered in tensor memory, O in 256 columns, 64-key
tiles); smaller head sizes in that range are padded to 256.  Pages of 16 and
32 keys take the cp.async producers, pages of 64 keys or more the TMA ones."""
import numpy as np
import pytest

import workloads
from pa_harness import assert_close, oracle_step, poison_unused, run_gpu, tolerances

pytestmark = pytest.mark.gpu

LENS = [
    ([1, 3, 2, 4], [900, 40, 3000, 130]),            # decode only: one and several splits
    ([9, 130, 300, 1, 64], [0, 17, 700, 2500, 63]),  # prefill with ragged tiles, and a decode row
]


def _check(spec, softcap=0.0, window=None, hints=True, x=None, repeat=1):
    if x is None:
        x = workloads.generate(spec)
        poison_unused(spec, x)
    got, _, status, _ = run_gpu(spec, x, hints=hints, softcap=softcap, window=window, repeat=repeat)
    outs = got if repeat > 1 else [got]
    want, _, _, _ = oracle_step(spec, x, softcap=softcap, window=window)
    assert status == 0
    mx, mn = tolerances(spec)
    assert_close(outs[0], want, mx, mn, what=spec.name, elem=spec.elem)
    for o in outs[1:]:
        assert np.array_equal(o.view(np.uint16), outs[0].view(np.uint16))
    return outs[0]


@pytest.mark.parametrize("elem", ["f16", "bf16"])
@pytest.mark.parametrize("bs", [16, 32, 64, 256])
@pytest.mark.parametrize("lens", LENS, ids=["decode", "mixed"])
def test_head256(elem, bs, lens):
    q, past = lens
    spec = workloads.custom(q, past, 16, 4, 256, bs, seed=bs + len(q), elem=elem)
    _check(spec, repeat=2)


@pytest.mark.parametrize("head_size", [136, 144, 192, 200, 248])
@pytest.mark.parametrize("bs", [16, 128])
def test_head_sizes_padded_to_256(head_size, bs):
    q, past = [1, 3, 70, 200], [600, 33, 0, 301]
    spec = workloads.custom(q, past, 8, 2, head_size, bs, seed=head_size + bs)
    _check(spec)


@pytest.mark.parametrize("bs", [16, 128])
def test_head256_softcap_and_window(bs):
    spec = workloads.custom([1, 200, 4, 300], [4000, 900, 77, 0], 16, 4, 256, bs, seed=bs,
                            elem="bf16")
    _check(spec, softcap=30.0)
    _check(spec, window=100)
    _check(spec, softcap=20.0, window=333)


@pytest.mark.parametrize("qh,kvh", [(6, 2), (10, 2), (8, 8), (32, 1), (64, 1)])
def test_head256_groups(qh, kvh):
    q, past = [1, 2, 45, 160], [1200, 30, 0, 500]
    spec = workloads.custom(q, past, qh, kvh, 256, 16, seed=qh * 10 + kvh)
    _check(spec)


@pytest.mark.parametrize("bs", [16, 256])
def test_head256_growing_keys(bs):
    """Key magnitudes that grow along each sequence: the running row maximum
    keeps rising, so the softmax rescales O between key tiles."""
    spec = workloads.custom([150, 1, 40], [2000, 3000, 600], 8, 2, 256, bs, seed=17 + bs)
    x = workloads.generate(spec)
    poison_unused(spec, x)
    kc = x["key_cache"].astype(np.float32)
    for s in range(spec.batch):
        for p in range(int(spec.pages_per_seq[s])):
            kc[x["block_table"][s, p]] *= 1.0 + 0.05 * p * bs / 16
    x["key_cache"] = kc.astype(np.float16)
    x["key"] = (x["key"].astype(np.float32) * 3.0).astype(np.float16)
    _check(spec, x=x)


def test_head256_long_prefill_without_hints():
    spec = workloads.custom([700, 513], [1500, 0], 16, 2, 256, 128, seed=3)
    _check(spec, hints=False)


def test_head256_full_size_prefill_sampled_rows_and_bit_identity():
    """The head-256 causal prefill workload at full size (8 x 2048 tokens,
    16/16 heads, 256-key pages): 2048 sampled rows (every sequence's first
    and last token included) against the oracle, with unused cache rows
    poisoned, and the same bits on a second run."""
    from pa_harness import sample_rows
    spec = workloads.spec_prefill_mha_d256()
    x = workloads.generate(spec)
    poison_unused(spec, x)
    outs, _, status, _ = run_gpu(spec, x, repeat=2)
    assert status == 0
    assert np.array_equal(outs[0].view(np.uint16), outs[1].view(np.uint16))
    rows = sample_rows(spec, 2048, seed=7)
    want, _, _, _ = oracle_step(spec, x, rows=rows)
    got = outs[0][rows[:, 0], rows[:, 1]]
    mx, mn = tolerances(spec)
    assert_close(got, want, mx, mn, what="head-256 prefill, sampled rows")
