"""Repetition tests: the same step launched many times back to back (its
kernels overlapping through programmatic dependent launch) must keep the
status word clear and give the same bits every time.  A race between the
warps of a kernel shows up here as a timed-out wait, a non-finite value or a
changed bit long before a single-run parity test would catch it."""
import numpy as np
import pytest

import workloads
from pa_harness import dims_for, host_bits, poison_unused, to_dev

pytestmark = pytest.mark.gpu


def _repeat(spec, reps):
    import torch
    import scatter_kv_b200 as pa
    x = workloads.generate(spec)
    poison_unused(spec, x)
    dv = to_dev(x)
    dims = dims_for(spec, x)
    bufs = pa.allocate(dims)
    outs = []
    for i in range(reps):
        pa.step(dv["query"], dv["key"], dv["value"], dv["key_cache"], dv["value_cache"],
                dv["block_table"], dv["cu_seqlens_q"], dv["seqlens_kv"], 0.0, dims, bufs)
        if i % 10 == 9:
            outs.append(bufs.out.clone())
    torch.cuda.synchronize()
    assert int(bufs.status[0].item()) == 0
    ref = host_bits(outs[0], spec.elem)
    assert np.isfinite(ref.astype(np.float64)).all()
    for o in outs[1:]:
        assert np.array_equal(host_bits(o, spec.elem).view(np.uint16), ref.view(np.uint16))


@pytest.mark.parametrize("which", ["prefill_d256", "prefill_d256_bs16", "mixed", "causal_bs128",
                                   "long_decode_small"])
def test_repeated_steps(which):
    if which == "prefill_d256":
        spec = workloads.spec_prefill_mha_d256()
    elif which == "prefill_d256_bs16":
        spec = workloads.custom([600, 1, 900, 300], [1000, 3000, 0, 2000], 16, 4, 256, 16, seed=71)
    elif which == "mixed":
        spec = workloads.spec_mixed()
    elif which == "causal_bs128":
        spec = workloads.custom([2048, 2048, 700], [0, 0, 300], 16, 16, 128, 128, seed=72)
    else:
        ld = workloads.spec_long_decode()
        spec = workloads.custom(ld.q_lens[:4], ld.past[:4] // 4, 64, 8, 128, 256, seed=73)
    _repeat(spec, 200)


def test_repeated_int4_decode():
    """INT4 caches: 200 back-to-back quantising scatters and decode calls
    (two-row-tile build, short and long sequences)."""
    import torch
    import scatter_kv_b200 as pa
    from test_int4 import _dims, _int4_problem
    spec, x, ks, vs = _int4_problem([1, 4, 2, 3], [9000, 2000, 4100, 600], 64, 8, 128, 256, "f16",
                                    seed=81)
    dv = to_dev(x)
    ksd, vsd = (torch.from_numpy(a).cuda() for a in (ks, vs))
    dims = _dims(spec, x)
    bufs = pa.allocate(dims)
    outs = []
    for i in range(200):
        pa.pa_compute_slot_mapping(dv["block_table"], dv["cu_seqlens_q"], dv["seqlens_kv"],
                                   bufs.slot_mapping, dims, bufs.status)
        pa.pa_scatter_kv_int4(dv["key"], dv["value"], bufs.slot_mapping, ksd, vsd, dv["key_cache"],
                              dv["value_cache"], dims, bufs.status)
        pa.pa_attention_int4(dv["query"], dv["key_cache"], dv["value_cache"], ksd, vsd,
                             dv["block_table"], dv["cu_seqlens_q"], dv["seqlens_kv"], 0.0,
                             bufs.out, dims, bufs.workspace, None, bufs.status)
        if i % 10 == 9:
            outs.append(bufs.out.clone())
    torch.cuda.synchronize()
    assert int(bufs.status[0].item()) == 0
    ref = host_bits(outs[0], spec.elem)
    assert np.isfinite(ref.astype(np.float64)).all()
    for o in outs[1:]:
        assert np.array_equal(host_bits(o, spec.elem).view(np.uint16), ref.view(np.uint16))


def test_repeated_sparse():
    """Sparse attention: 200 back-to-back calls over one selection."""
    import torch
    import scatter_kv_b200 as pa
    from test_sparse import _selections
    spec = workloads.custom([1, 1, 3, 1], [3000, 700, 2000, 5000], 32, 8, 128, 16, seed=82)
    x = workloads.generate(spec)
    poison_unused(spec, x)
    sel = _selections(spec, x, 256, np.random.default_rng(82))
    dv = to_dev(x)
    dims = pa.make_dims(batch=spec.batch, token_count=spec.token_count, q_heads=spec.q_heads,
                        kv_heads=spec.kv_heads, head_size=spec.head_size,
                        num_blocks=spec.num_blocks, block_size=spec.block_size,
                        max_blocks_per_seq=x["block_table"].shape[1])
    bufs = pa.allocate(dims)
    seld = torch.from_numpy(sel).cuda()
    outs = []
    for i in range(200):
        pa.pa_sparse_attention(dv["query"], dv["key_cache"], dv["value_cache"], dv["block_table"],
                               dv["cu_seqlens_q"], dv["seqlens_kv"], seld, sel.shape[2], 64, 0.0,
                               bufs.out, dims, bufs.status)
        if i % 10 == 9:
            outs.append(bufs.out.clone())
    torch.cuda.synchronize()
    assert int(bufs.status[0].item()) == 0
    ref = host_bits(outs[0], spec.elem)
    assert np.isfinite(ref.astype(np.float64)).all()
    for o in outs[1:]:
        assert np.array_equal(host_bits(o, spec.elem).view(np.uint16), ref.view(np.uint16))
