"""GPU parity of the scatter and the slot mapping: bit-exact against the
oracle, through the C ABI."""
import numpy as np
import pytest

import oracle
import workloads
from pa_harness import dims_for, to_dev

pytestmark = pytest.mark.gpu


def _gpu_slots(spec, x):
    import torch
    import scatter_kv_b200 as pa
    dv = to_dev(x)
    dims = dims_for(spec, x)
    slots = torch.full((max(spec.token_count, 1),), -7, dtype=torch.int32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    pa.pa_compute_slot_mapping(dv["block_table"], dv["cu_seqlens_q"], dv["seqlens_kv"], slots,
                               dims, status)
    torch.cuda.synchronize()
    return slots[:spec.token_count].cpu().numpy(), int(status.item()), dv, dims


@pytest.mark.parametrize("cfg", [0, 1, 2, 3, 4])
def test_slot_mapping_bit_exact(cfg):
    spec = workloads.CONFIGS[cfg]()
    # Only the metadata matters here: same lengths, pool and seed, tiny heads.
    meta = workloads.custom(spec.q_lens, spec.past, 1, 1, 16, spec.block_size,
                            num_blocks=spec.num_blocks, seed=spec.seed)
    x = workloads.generate(meta)
    got, status, _, _ = _gpu_slots(meta, x)
    want = oracle.slot_mapping(x["block_table"], x["cu_seqlens_q"], x["seqlens_kv"],
                               spec.block_size)
    assert status == 0
    assert np.array_equal(got, want)


def test_slot_mapping_zero_length_sequences():
    spec = workloads.custom([3, 0, 0, 5, 0, 1], [2, 9, 0, 0, 4, 30], 2, 1, 16, 16, num_blocks=12)
    x = workloads.generate(spec)
    got, status, _, _ = _gpu_slots(spec, x)
    want = oracle.slot_mapping(x["block_table"], x["cu_seqlens_q"], x["seqlens_kv"], 16)
    assert status == 0 and np.array_equal(got, want)


@pytest.mark.parametrize("cfg", [0, 1, 2, 3, 4])
def test_scatter_bit_exact(cfg):
    import torch
    import scatter_kv_b200 as pa
    spec = workloads.CONFIGS[cfg]()
    x = workloads.generate(spec)
    slots = oracle.slot_mapping(x["block_table"], x["cu_seqlens_q"], x["seqlens_kv"],
                                spec.block_size)
    dv = to_dev(x)
    dims = dims_for(spec, x)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    pa.pa_scatter_kv(dv["key"], dv["value"], torch.from_numpy(slots).cuda(), dv["key_cache"],
                     dv["value_cache"], dims, status)
    torch.cuda.synchronize()
    kc, vc = x["key_cache"].copy(), x["value_cache"].copy()
    oracle.scatter_kv(x["key"], x["value"], slots, kc, vc)
    assert int(status.item()) == 0
    assert np.array_equal(dv["key_cache"].cpu().numpy().view(np.uint16), kc.view(np.uint16))
    assert np.array_equal(dv["value_cache"].cpu().numpy().view(np.uint16), vc.view(np.uint16))


def test_scatter_skips_negative_and_flags_out_of_range_slots():
    import torch
    import scatter_kv_b200 as pa
    spec = workloads.custom([6], [10], 4, 2, 64, 16, num_blocks=4)
    x = workloads.generate(spec)
    nslots = spec.num_blocks * spec.block_size
    slots = np.array([3, -1, nslots, 40, -5, nslots + 100], dtype=np.int32)
    dv = to_dev(x)
    dims = dims_for(spec, x)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    pa.pa_scatter_kv(dv["key"], dv["value"], torch.from_numpy(slots).cuda(), dv["key_cache"],
                     dv["value_cache"], dims, status)
    torch.cuda.synchronize()
    kc, vc = x["key_cache"].copy(), x["value_cache"].copy()
    ok = np.where(slots < nslots, slots, -1).astype(np.int32)
    oracle.scatter_kv(x["key"], x["value"], ok, kc, vc)
    assert int(status.item()) == pa.PA_DEV_BAD_SLOT
    assert np.array_equal(dv["key_cache"].cpu().numpy().view(np.uint16), kc.view(np.uint16))
    assert np.array_equal(dv["value_cache"].cpu().numpy().view(np.uint16), vc.view(np.uint16))


@pytest.mark.parametrize("head_size,kv_heads", [(16, 1), (32, 3), (64, 2), (128, 8)])
def test_scatter_head_shapes(head_size, kv_heads):
    import torch
    import scatter_kv_b200 as pa
    spec = workloads.custom([5, 1, 33], [0, 7, 2], kv_heads, kv_heads, head_size, 16)
    x = workloads.generate(spec)
    slots = oracle.slot_mapping(x["block_table"], x["cu_seqlens_q"], x["seqlens_kv"], 16)
    dv = to_dev(x)
    pa.pa_scatter_kv(dv["key"], dv["value"], torch.from_numpy(slots).cuda(), dv["key_cache"],
                     dv["value_cache"], dims_for(spec, x))
    torch.cuda.synchronize()
    kc, vc = x["key_cache"].copy(), x["value_cache"].copy()
    oracle.scatter_kv(x["key"], x["value"], slots, kc, vc)
    assert np.array_equal(dv["key_cache"].cpu().numpy().view(np.uint16), kc.view(np.uint16))
    assert np.array_equal(dv["value_cache"].cpu().numpy().view(np.uint16), vc.view(np.uint16))
