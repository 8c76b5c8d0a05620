"""pa_attention_noalloc: the variant of pa_attention for callers that cannot
allocate device memory (a host runtime that gives them a fixed budget and no
workspace, or a path that must not call cudaMalloc).  Its split-KV scratch is
a fixed array inside the library.  This file is collected last on purpose, so
that a run stopping at the first failure has run every other test first; it
also passes on its own in a fresh process."""
import numpy as np
import pytest

import workloads
from pa_harness import (MAX_ABS, MEAN_ABS, assert_close, dims_for, oracle_step,
                        poison_unused, to_dev)

pytestmark = pytest.mark.gpu


def _spec():
    # Decode sequences long enough to need several splits (so the scratch is
    # used), plus one prefill sequence; its scratch need stays under 8 MiB.
    return workloads.custom([1, 2, 4, 1, 1, 3, 1, 40], [2900, 1500, 600, 2000, 90, 2500, 3000, 70],
                            16, 4, 128, 16, seed=404)


def test_noalloc_matches_workspace_entry_point_twice():
    import torch
    import scatter_kv_b200 as pa
    spec = _spec()
    x = workloads.generate(spec)
    poison_unused(spec, x)
    dv = to_dev(x)
    dims = dims_for(spec, x)
    need = pa.pa_attention_workspace_size(dims)
    assert 0 < need <= pa.NOALLOC_SCRATCH_BYTES
    bufs = pa.allocate(dims)
    pa.pa_compute_slot_mapping(dv["block_table"], dv["cu_seqlens_q"], dv["seqlens_kv"],
                               bufs.slot_mapping, dims, bufs.status)
    pa.pa_scatter_kv(dv["key"], dv["value"], bufs.slot_mapping, dv["key_cache"],
                     dv["value_cache"], dims, bufs.status)
    # Reference: the existing entry point with a caller-owned workspace.  Both
    # run the same kernels on the same split plan and differ only in where the
    # split-KV scratch lives, so their outputs must agree bit for bit.
    pa.pa_attention(dv["query"], dv["key_cache"], dv["value_cache"], dv["block_table"],
                    dv["cu_seqlens_q"], dv["seqlens_kv"], 0.0, bufs.out, dims, bufs.workspace,
                    None, bufs.status)
    assert pa.pa_get_status(bufs.status) == 0
    ref = bufs.out.cpu().numpy().copy()
    want, _, _, _ = oracle_step(spec, x)
    for call in range(2):
        out = torch.full_like(bufs.out, float("nan"))
        pa.pa_attention_noalloc(dv["query"], dv["key_cache"], dv["value_cache"],
                                dv["block_table"], dv["cu_seqlens_q"], dv["seqlens_kv"], 0.0,
                                out, dims, bufs.status)
        assert pa.pa_get_status(bufs.status) == 0, f"device status after noalloc call {call}"
        got = out.cpu().numpy()
        assert np.array_equal(got.view(np.uint16), ref.view(np.uint16)), f"noalloc call {call}"
        assert_close(got, want, MAX_ABS, MEAN_ABS, what=f"noalloc call {call} vs oracle")


def test_noalloc_rejects_dims_beyond_its_scratch():
    import scatter_kv_b200 as pa
    dims = pa.make_dims(batch=256, token_count=256, q_heads=32, kv_heads=8, head_size=128,
                        num_blocks=100000, block_size=16, max_blocks_per_seq=4096)
    assert pa.pa_attention_workspace_size(dims) > pa.NOALLOC_SCRATCH_BYTES
    with pytest.raises(pa.PagedAttentionError) as e:
        pa.pa_attention_noalloc(1 << 20, 1 << 20, 1 << 20, 1 << 20, 1 << 20, 1 << 20, 0.0,
                                1 << 20, dims, None, 0)
    assert e.value.status == pa.PA_ERR_INVALID_ARGUMENT
    assert "pa_attention_noalloc" in str(e.value)
