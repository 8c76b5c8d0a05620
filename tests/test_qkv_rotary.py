"""GPU parity of pa_split_qkv_rotary_scatter (split of packed QKV, rotary
embedding of Q and K, scatter of K and V into the paged cache, one kernel)
against the fp64 oracle, through the C ABI.

Rotated values: the kernel rounds x1 cos - x2 sin once in fp32 (the
products of two 16-bit floats are exact there) and then to the 16-bit type;
the oracle's value is exact in fp64 and rounded once.  The two agree except
where the fp32 rounding lands on a 16-bit tie, so the bar is at most one ulp
apart everywhere and bit-equal on all but a small fraction.  V and the slot
mapping are bit-exact."""
import numpy as np
import pytest

import oracle
import workloads
from pa_harness import assert_close, poison_unused, to_dev

pytestmark = pytest.mark.gpu


def _rope_cache(max_pos, rotary_dim, base=10000.0):
    m = np.arange(rotary_dim // 2)
    theta = base ** (-2.0 * m / rotary_dim)
    ang = np.arange(max_pos)[:, None] * theta[None, :]
    return np.cos(ang), np.sin(ang)


def _to_bits(a64, bf16):
    """fp64 -> 16-bit pattern, rounded to nearest-even (numpy for f16, torch
    for bf16)."""
    if not bf16:
        return a64.astype(np.float16).view(np.uint16)
    import torch
    t = torch.from_numpy(np.ascontiguousarray(a64)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def _ordered(bits):
    b = bits.astype(np.int64)
    return np.where(b & 0x8000, -(b & 0x7FFF), b)


def _assert_rounded(got_bits, want64, bf16, what):
    want_bits = _to_bits(want64, bf16)
    dist = np.abs(_ordered(got_bits) - _ordered(want_bits))
    assert dist.max() <= 1, f"{what}: {int(dist.max())} ulp apart"
    assert (dist == 0).mean() >= 0.995, f"{what}: only {(dist == 0).mean():.4f} bit-equal"


CASES = [
    # q_lens, past, qh, kvh, d, bs, rotary_dim, interleaved, packed, bf16
    ([1, 4, 0, 37], [20, 7, 3, 100], 8, 2, 128, 16, 128, False, True, False),
    ([1, 4, 0, 37], [20, 7, 3, 100], 8, 2, 128, 16, 128, True, True, False),
    ([300, 2], [0, 900], 16, 16, 128, 256, 64, False, False, False),
    ([5, 70], [33, 0], 32, 8, 64, 32, 32, True, True, False),
    ([5, 70], [33, 0], 32, 8, 64, 32, 0, False, True, False),
    ([9, 1, 64], [0, 4000, 128], 8, 1, 128, 128, 128, False, True, True),
    ([9, 1, 64], [0, 4000, 128], 8, 1, 128, 128, 64, True, False, True),
    ([16], [48], 4, 4, 16, 16, 16, False, True, False),
]


def _run(case):
    import torch
    import scatter_kv_b200 as pa
    q_lens, past, qh, kvh, d, bs, rd, inter, packed, bf16 = case
    spec = workloads.custom(q_lens, past, qh, kvh, d, bs, seed=sum(q_lens) + rd)
    x = workloads.generate(spec)
    poison_unused(spec, x)
    T = spec.token_count
    rng = np.random.default_rng(len(q_lens) + d)
    qkv64 = rng.standard_normal((T, qh + 2 * kvh, d))
    maxpos = int(spec.seqlens_kv.max()) + 3
    cos64, sin64 = _rope_cache(maxpos, max(rd, 2))
    tdt = torch.bfloat16 if bf16 else torch.float16
    qkv_bits = _to_bits(qkv64, bf16)
    cos_bits, sin_bits = _to_bits(cos64, bf16), _to_bits(sin64, bf16)
    kc_bits = x["key_cache"].view(np.uint16).copy()
    vc_bits = x["value_cache"].view(np.uint16).copy()
    dv = to_dev({k: x[k] for k in ("block_table", "cu_seqlens_q", "seqlens_kv")})
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda().view(tdt)
    qkv_d = dev(qkv_bits)
    kc_d, vc_d = dev(kc_bits), dev(vc_bits)
    cos_d, sin_d = dev(cos_bits), dev(sin_bits)
    dims = pa.make_dims(batch=spec.batch, token_count=T, q_heads=qh, kv_heads=kvh, head_size=d,
                        num_blocks=spec.num_blocks, block_size=bs,
                        max_blocks_per_seq=x["block_table"].shape[1],
                        dtype=pa.PA_DTYPE_BF16 if bf16 else pa.PA_DTYPE_F16)
    q_out = torch.full((T, qh, d), float("nan"), dtype=tdt, device="cuda")
    slots = torch.full((max(T, 1),), -7, dtype=torch.int32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    rot = pa.pa_rotary()
    rot.rotary_dim, rot.interleaved, rot.max_position = rd, int(inter), maxpos
    if packed:
        qp, kp, vp, stride = pa.packed_qkv_views(qkv_d, dims)
        pa.pa_split_qkv_rotary_scatter(qp, kp, vp, stride, stride, cos_d, sin_d, rot,
                                       dv["block_table"], dv["cu_seqlens_q"], dv["seqlens_kv"],
                                       q_out, kc_d, vc_d, slots, dims, status)
    else:
        qd = qkv_d[:, :qh].contiguous()
        kd = qkv_d[:, qh:qh + kvh].contiguous()
        vd = qkv_d[:, qh + kvh:].contiguous()
        pa.pa_split_qkv_rotary_scatter(qd, kd, vd, 0, 0, cos_d, sin_d, rot, dv["block_table"],
                                       dv["cu_seqlens_q"], dv["seqlens_kv"], q_out, kc_d, vc_d,
                                       slots, dims, status)
    torch.cuda.synchronize()
    host = lambda t: t.view(torch.int16).cpu().numpy().view(np.uint16)
    return dict(spec=spec, x=x, qkv_bits=qkv_bits, cos_bits=cos_bits, sin_bits=sin_bits,
                kc0=kc_bits, vc0=vc_bits, q_out=host(q_out), kc=host(kc_d), vc=host(vc_d),
                slots=slots[:T].cpu().numpy(), status=int(status.item()), dims=dims,
                q_out_dev=q_out, kc_dev=kc_d, vc_dev=vc_d, dv=dv)


def _oracle_rotated(r, case):
    q_lens, past, qh, kvh, d, bs, rd, inter, packed, bf16 = case
    x = r["x"]
    pos = oracle.token_positions(x["cu_seqlens_q"], x["seqlens_kv"])
    qkv = r["qkv_bits"] if bf16 else r["qkv_bits"].view(np.float16)
    cc = r["cos_bits"] if bf16 else r["cos_bits"].view(np.float16)
    sc = r["sin_bits"] if bf16 else r["sin_bits"].view(np.float16)
    if rd == 0:
        cc, sc = cc[:, :0], sc[:, :0]
    q = oracle.rotary(qkv[:, :qh], pos, cc, sc, rd, inter, bf16=bf16)
    k = oracle.rotary(qkv[:, qh:qh + kvh], pos, cc, sc, rd, inter, bf16=bf16)
    return q, k, pos


@pytest.mark.parametrize("case", CASES, ids=[f"c{i}" for i in range(len(CASES))])
def test_split_qkv_rotary_scatter_matches_oracle(case):
    q_lens, past, qh, kvh, d, bs, rd, inter, packed, bf16 = case
    r = _run(case)
    x, spec = r["x"], r["spec"]
    assert r["status"] == 0
    want_slots = oracle.slot_mapping(x["block_table"], x["cu_seqlens_q"], x["seqlens_kv"], bs)
    assert np.array_equal(r["slots"], want_slots)
    q, k, _ = _oracle_rotated(r, case)
    _assert_rounded(r["q_out"], q, bf16, "rotated Q")
    # Cache: rotated K and copied V at the slots, every other row untouched.
    kc = r["kc"].reshape(-1, kvh, d)
    vc = r["vc"].reshape(-1, kvh, d)
    _assert_rounded(kc[want_slots], k, bf16, "rotated K in the cache")
    assert np.array_equal(vc[want_slots], r["qkv_bits"][:, qh + kvh:])
    others = np.setdiff1d(np.arange(kc.shape[0]), want_slots)
    assert np.array_equal(kc[others], r["kc0"].reshape(-1, kvh, d)[others])
    assert np.array_equal(vc[others], r["vc0"].reshape(-1, kvh, d)[others])
    if rd < d:   # pass-through elements are copies
        assert np.array_equal(r["q_out"][:, :, rd:], r["qkv_bits"][:, :qh, rd:])


def test_rotated_batch_then_attention():
    """The fused pass followed by attention equals the oracle's attention on
    the oracle's own rotated Q and cache."""
    import scatter_kv_b200 as pa
    import torch
    case = CASES[0]
    q_lens, past, qh, kvh, d, bs, rd, inter, packed, bf16 = case
    r = _run(case)
    spec, x = r["spec"], r["x"]
    dims = r["dims"]
    dims.max_seqlen_q_hint = int(spec.q_lens.max())
    ws = torch.empty(max(pa.pa_attention_workspace_size(dims), 16), dtype=torch.uint8, device="cuda")
    out = torch.empty_like(r["q_out_dev"])
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    pa.pa_attention(r["q_out_dev"], r["kc_dev"], r["vc_dev"], r["dv"]["block_table"],
                    r["dv"]["cu_seqlens_q"], r["dv"]["seqlens_kv"], 0.0, out, dims, ws, None, st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    # Oracle side: its own rotation, rounded to f16, scattered by its own slots.
    q, k, _ = _oracle_rotated(r, case)
    q16 = q.astype(np.float16)
    kc = r["kc0"].view(np.float16).copy()
    vc = r["vc0"].view(np.float16).copy()
    slots = oracle.slot_mapping(x["block_table"], x["cu_seqlens_q"], x["seqlens_kv"], bs)
    oracle.scatter_kv(k.astype(np.float16), r["qkv_bits"][:, qh + kvh:].view(np.float16).copy(),
                      slots, kc, vc)
    want = oracle.attention(q16, kc, vc, x["block_table"], x["cu_seqlens_q"], x["seqlens_kv"],
                            1.0 / np.sqrt(d))
    assert_close(out.cpu().numpy(), want, what="attention after the fused pass")


def test_position_past_the_caches_is_flagged():
    import scatter_kv_b200 as pa
    import torch
    spec = workloads.custom([3, 2], [1, 10], 4, 2, 64, 16, seed=3)
    x = workloads.generate(spec)
    dv = to_dev(x)
    dims = pa.make_dims(batch=2, token_count=5, q_heads=4, kv_heads=2, head_size=64,
                        num_blocks=spec.num_blocks, block_size=16,
                        max_blocks_per_seq=x["block_table"].shape[1])
    rot = pa.pa_rotary()
    rot.rotary_dim, rot.interleaved, rot.max_position = 64, 0, 8   # sequence 1 reaches 11
    cos = torch.ones((8, 32), dtype=torch.float16, device="cuda")
    sin = torch.zeros((8, 32), dtype=torch.float16, device="cuda")
    q_out = torch.full((5, 4, 64), float("nan"), dtype=torch.float16, device="cuda")
    kc0 = dv["key_cache"].clone()
    slots = torch.empty(5, dtype=torch.int32, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    pa.pa_split_qkv_rotary_scatter(dv["query"], dv["key"], dv["value"], 0, 0, cos, sin, rot,
                                   dv["block_table"], dv["cu_seqlens_q"], dv["seqlens_kv"], q_out,
                                   dv["key_cache"], dv["value_cache"], slots, dims, st)
    torch.cuda.synchronize()
    assert int(st.item()) & pa.PA_DEV_BAD_POSITION
    s = slots.cpu().numpy()
    assert (s[:3] >= 0).all() and (s[3:] == -1).all()
    qo = q_out.cpu().numpy()
    assert np.array_equal(qo[:3], x["query"][:3])          # cos 1, sin 0: identity
    assert (qo[3:] == 0).all()
    kc = dv["key_cache"].view(-1, 2, 64)
    untouched = np.setdiff1d(np.arange(kc.shape[0]), s[:3])
    assert torch.equal(kc[untouched].view(torch.int16), kc0.view(-1, 2, 64)[untouched].view(torch.int16))


@pytest.mark.parametrize("cfg", [1, 3])
def test_scatter_only_pass_equals_slot_mapping_then_scatter(cfg):
    """Without a query output the fused pass is slot mapping plus scatter in
    one kernel: the step built on it gives the same slots, caches and
    attention output, bit for bit, as pa_compute_slot_mapping followed by
    pa_scatter_kv."""
    spec = workloads.CONFIGS[cfg]()
    x = workloads.generate(spec)
    from pa_harness import run_gpu
    a, dva, sa, slots_a = run_gpu(spec, x, fused=True)
    b, dvb, sb, slots_b = run_gpu(spec, x, fused=False)
    assert sa == sb == 0
    assert np.array_equal(slots_a, slots_b)
    assert np.array_equal(a.view(np.uint16), b.view(np.uint16))
    import torch
    for name in ("key_cache", "value_cache"):
        assert torch.equal(dva[name].view(torch.int16), dvb[name].view(torch.int16))
