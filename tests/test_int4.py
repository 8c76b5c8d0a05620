"""GPU parity of the INT4 KV cache through the C ABI: the quantising scatter
bit for bit against the oracle's (codes, packing, untouched slots, status
bits), and decode attention over INT4 pages against the oracle's attention
over the values the codes stand for (fp64), within the attention tolerance
of the query's type."""
import math

import numpy as np
import pytest

import oracle
import workloads
from pa_harness import (MAX_ABS, MAX_ABS_BF16, MEAN_ABS, MEAN_ABS_BF16, as_float64,
                        assert_close, host_bits, to_dev)

pytestmark = pytest.mark.gpu


def _scales(rng, kvh, d):
    return (rng.uniform(0.1, 0.3, size=(kvh, d)).astype(np.float32),
            rng.uniform(0.1, 0.3, size=(kvh, d)).astype(np.float32))


def _int4_problem(q_lens, past, qh, kvh, d, bs, elem, seed):
    """A seeded decode batch with INT4 caches: page codes drawn uniformly,
    the new tokens' K/V drawn as 16-bit values (the scatter quantises them)."""
    spec = workloads.custom(q_lens, past, qh, kvh, d, bs, seed=seed, elem=elem)
    x = workloads.generate(spec)
    rng = np.random.default_rng(seed)
    ks, vs = _scales(rng, kvh, d)
    shape = (spec.num_blocks, bs, kvh, d // 2)
    x["key_cache"] = rng.integers(0, 256, size=shape, dtype=np.uint8)
    x["value_cache"] = rng.integers(0, 256, size=shape, dtype=np.uint8)
    return spec, x, ks, vs


def _dims(spec, x):
    import scatter_kv_b200 as pa
    return pa.make_dims(batch=spec.batch, token_count=spec.token_count, q_heads=spec.q_heads,
                        kv_heads=spec.kv_heads, head_size=spec.head_size,
                        num_blocks=spec.num_blocks, block_size=spec.block_size,
                        max_blocks_per_seq=x["block_table"].shape[1],
                        max_seqlen_q=int(spec.q_lens.max()),
                        max_seqlen_kv=int(spec.seqlens_kv.max()),
                        dtype=pa.PA_DTYPE_BF16 if spec.elem == "bf16" else pa.PA_DTYPE_F16)


def _gpu_step(spec, x, ks, vs, repeat=1):
    import torch
    import scatter_kv_b200 as pa
    dv = to_dev(x)
    ksd, vsd = (torch.from_numpy(a).cuda() for a in (ks, vs))
    dims = _dims(spec, x)
    bufs = pa.allocate(dims)
    pa.pa_compute_slot_mapping(dv["block_table"], dv["cu_seqlens_q"], dv["seqlens_kv"],
                               bufs.slot_mapping, dims, bufs.status)
    pa.pa_scatter_kv_int4(dv["key"], dv["value"], bufs.slot_mapping, ksd, vsd, dv["key_cache"],
                          dv["value_cache"], dims, bufs.status)
    outs = []
    for _ in range(repeat):
        pa.pa_attention_int4(dv["query"], dv["key_cache"], dv["value_cache"], ksd, vsd,
                             dv["block_table"], dv["cu_seqlens_q"], dv["seqlens_kv"], 0.0,
                             bufs.out, dims, bufs.workspace, None, bufs.status)
        torch.cuda.synchronize()
        outs.append(host_bits(bufs.out, spec.elem))
    return outs, dv, int(bufs.status[0].item())


def _oracle(spec, x, ks, vs):
    bf16 = spec.elem == "bf16"
    kc, vc = x["key_cache"].copy(), x["value_cache"].copy()
    slots = oracle.slot_mapping(x["block_table"], x["cu_seqlens_q"], x["seqlens_kv"],
                                spec.block_size)
    oracle.scatter_kv_int4(x["key"], x["value"], slots, ks, vs, kc, vc, bf16=bf16)
    q = as_float64(x["query"], spec.elem)
    y = oracle.attention(q, oracle.dequantize_int4(kc, ks), oracle.dequantize_int4(vc, vs),
                         x["block_table"], x["cu_seqlens_q"], x["seqlens_kv"],
                         1.0 / math.sqrt(spec.head_size))
    return y, kc, vc


@pytest.mark.parametrize("elem", ["f16", "bf16"])
@pytest.mark.parametrize("bs", [16, 256])
def test_int4_scatter_bit_exact(elem, bs):
    import torch
    import scatter_kv_b200 as pa
    spec, x, ks, vs = _int4_problem([1, 3, 40, 0, 2], [100, 7, 300, 5, 900], 16, 4, 128, bs,
                                    elem, seed=bs)
    # Exact ties (x = (k + 1/2) * s with s a power of two) in the first token.
    ks[:, :16] = 0.25
    tie = ((np.arange(16) % 15) - 7.5) * 0.25
    if elem == "bf16":
        x["key"][0, :, :16] = workloads._to_bf16_bits(np.broadcast_to(tie, (4, 16)).astype(np.float32))
    else:
        x["key"][0, :, :16] = tie.astype(np.float16)
    dv = to_dev(x)
    ksd, vsd = (torch.from_numpy(a).cuda() for a in (ks, vs))
    dims = _dims(spec, x)
    slots = oracle.slot_mapping(x["block_table"], x["cu_seqlens_q"], x["seqlens_kv"], bs)
    slots[1] = -1                                       # a skipped token
    sd = torch.from_numpy(slots).cuda()
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    pa.pa_scatter_kv_int4(dv["key"], dv["value"], sd, ksd, vsd, dv["key_cache"], dv["value_cache"],
                          dims, st)
    torch.cuda.synchronize()
    kc, vc = x["key_cache"].copy(), x["value_cache"].copy()
    oracle.scatter_kv_int4(x["key"], x["value"], slots, ks, vs, kc, vc, bf16=elem == "bf16")
    assert int(st.item()) == 0
    assert np.array_equal(dv["key_cache"].cpu().numpy(), kc)
    assert np.array_equal(dv["value_cache"].cpu().numpy(), vc)


def test_int4_scatter_flags_out_of_range_slot():
    import torch
    import scatter_kv_b200 as pa
    spec, x, ks, vs = _int4_problem([2], [3], 8, 2, 64, 16, "f16", seed=1)
    dv = to_dev(x)
    ksd, vsd = (torch.from_numpy(a).cuda() for a in (ks, vs))
    slots = torch.tensor([spec.num_blocks * 16, 0], dtype=torch.int32, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    kc0 = dv["key_cache"].clone()
    pa.pa_scatter_kv_int4(dv["key"], dv["value"], slots, ksd, vsd, dv["key_cache"], dv["value_cache"],
                          _dims(spec, x), st)
    torch.cuda.synchronize()
    assert int(st.item()) & pa.PA_DEV_BAD_SLOT
    assert torch.equal(dv["key_cache"].view(-1, 64)[2:], kc0.view(-1, 64)[2:])


CASES = [
    # q_lens, past, qh, kvh, d, bs, elem
    ([1, 1, 1, 1], [700, 3000, 45, 9000], 32, 8, 128, 16, "f16"),
    ([1, 2, 3, 4], [1200, 33, 5000, 260], 16, 4, 128, 256, "f16"),
    ([1, 4, 2], [2000, 100, 4100], 64, 8, 128, 32, "f16"),
    ([2, 1, 3], [500, 6000, 77], 16, 2, 64, 16, "f16"),
    ([1, 3], [999, 64], 8, 8, 32, 128, "f16"),
    ([1, 1, 2, 4], [700, 3000, 45, 9000], 32, 8, 128, 16, "bf16"),
    # head size 256 (the pages' INT4 XQA kernels are built for it)
    ([1, 2, 4, 1], [2500, 300, 6000, 33], 16, 2, 256, 16, "f16"),
    ([3, 1], [4100, 900], 32, 4, 256, 256, "bf16"),
    ([1, 1, 1], [1500, 70, 8000], 8, 8, 256, 64, "f16"),
]


@pytest.mark.parametrize("case", CASES, ids=[f"c{i}" for i in range(len(CASES))])
def test_int4_decode_matches_oracle(case):
    q_lens, past, qh, kvh, d, bs, elem = case
    spec, x, ks, vs = _int4_problem(q_lens, past, qh, kvh, d, bs, elem, seed=sum(past) % 1000)
    outs, dv, status = _gpu_step(spec, x, ks, vs, repeat=2)
    want, kc, vc = _oracle(spec, x, ks, vs)
    assert status == 0
    assert np.array_equal(dv["key_cache"].cpu().numpy(), kc)
    assert np.array_equal(outs[0], outs[1])              # deterministic
    mx, mn = (MAX_ABS_BF16, MEAN_ABS_BF16) if elem == "bf16" else (MAX_ABS, MEAN_ABS)
    assert_close(outs[0], want, mx, mn, what=f"int4 {case}", elem=elem)


def test_int4_long_context_shape_and_page_permutation():
    """Two sequences of the long-context decode shape (64/8 heads, 256-key
    pages): the oracle's result, and the same bits under another placement
    of the pages."""
    spec, x, ks, vs = _int4_problem([1, 4], [20000, 9000], 64, 8, 128, 256, "f16", seed=44)
    outs, _, status = _gpu_step(spec, x, ks, vs)
    want, _, _ = _oracle(spec, x, ks, vs)
    assert status == 0
    assert_close(outs[0], want, what="int4 long context")
    rng = np.random.default_rng(5)
    y = workloads.generate(spec, block_order=rng.permutation(spec.num_blocks))
    for name in ("key_cache", "value_cache"):
        y[name] = np.zeros_like(x[name])
        for s in range(spec.batch):
            for p in range(int(spec.pages_per_seq[s])):
                y[name][y["block_table"][s, p]] = x[name][x["block_table"][s, p]]
    for name in ("query", "key", "value"):
        y[name] = x[name]
    outs2, _, status2 = _gpu_step(spec, y, ks, vs)
    assert status2 == 0
    assert np.array_equal(outs[0], outs2[0])


def test_int4_rejects_prefill_batches_and_unbuilt_heads():
    import scatter_kv_b200 as pa
    spec, x, ks, vs = _int4_problem([1, 9], [10, 10], 16, 4, 128, 16, "f16", seed=2)
    d = _dims(spec, x)
    with pytest.raises(pa.PagedAttentionError) as e:
        pa.pa_attention_int4(1 << 20, 1 << 20, 1 << 20, 1 << 20, 1 << 20, 1 << 20, 1 << 20,
                             1 << 20, 0.0, 1 << 20, d, None, 0, None, 0)
    assert e.value.status == pa.PA_ERR_NOT_IMPLEMENTED and "decode" in str(e.value)
    d.max_seqlen_q_hint = 1
    d.head_size = 80
    with pytest.raises(pa.PagedAttentionError) as e:
        pa.pa_attention_int4(1 << 20, 1 << 20, 1 << 20, 1 << 20, 1 << 20, 1 << 20, 1 << 20,
                             1 << 20, 0.0, 1 << 20, d, None, 0, None, 0)
    assert e.value.status == pa.PA_ERR_NOT_IMPLEMENTED
