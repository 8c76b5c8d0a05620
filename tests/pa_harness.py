"""Shared helpers of the GPU parity tests: move a seeded batch to the GPU, run
the library through its C ABI, and run the fp64 oracle on the same inputs."""
from __future__ import annotations

import math

import numpy as np

import oracle
import workloads

MAX_ABS = 4e-3       # attention tolerance vs the fp64 oracle (f16 out, fp32 accumulate)
MEAN_ABS = 3e-4
# bf16 keeps 8 significant bits instead of f16's 11: half an ulp of an output
# in [2, 4) is 2^-7 (7.8e-3), and P rounded to bf16 before P V adds at most
# 2^-9 times the largest |V| (about 4 here) -- together 1.6e-2.  Typical
# outputs are well below 1, where the same two terms average a few 1e-4.
MAX_ABS_BF16 = 1.6e-2
MEAN_ABS_BF16 = 1.5e-3


def tolerances(spec):
    return (MAX_ABS_BF16, MEAN_ABS_BF16) if spec.elem == "bf16" else (MAX_ABS, MEAN_ABS)


def as_float64(a, elem):
    """Output or input array (f16 values, or bf16 bit patterns) as float64."""
    a = np.asarray(a)
    if elem == "bf16":
        import torch
        return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).double().numpy()
    return a.astype(np.float64)


def to_dev(x: dict):
    """numpy arrays -> device tensors (bf16 bit patterns travel as int16)."""
    import torch
    return {k: torch.from_numpy(np.ascontiguousarray(v.view(np.int16) if v.dtype == np.uint16 else v))
            .cuda() for k, v in x.items()}


def host_bits(t, elem):
    """A 16-bit device tensor back on the host: float16 values, or bf16 bit
    patterns as uint16."""
    import torch
    if elem == "bf16":
        return t.view(torch.int16).cpu().numpy().view(np.uint16).copy()
    return t.cpu().numpy().copy()


def dims_for(spec: workloads.Spec, x: dict, hints: bool = True, softcap: float = 0.0,
             window=None):
    import scatter_kv_b200 as pa
    return pa.make_dims(
        batch=spec.batch, token_count=spec.token_count, q_heads=spec.q_heads,
        kv_heads=spec.kv_heads, head_size=spec.head_size, num_blocks=spec.num_blocks,
        block_size=spec.block_size, max_blocks_per_seq=x["block_table"].shape[1],
        max_seqlen_q=int(spec.q_lens.max()) if hints and spec.batch else 0,
        max_seqlen_kv=int(spec.seqlens_kv.max()) if hints and spec.batch else 0,
        dtype=pa.PA_DTYPE_BF16 if spec.elem == "bf16" else pa.PA_DTYPE_F16,
        softcap=softcap, window=window)


def run_gpu(spec: workloads.Spec, x: dict, hints: bool = True, scale: float | None = None,
            repeat: int = 1, softcap: float = 0.0, window=None, fused: bool = False):
    """Slot mapping + scatter + attention on the GPU.  Returns (out as numpy
    float16 -- bf16 bit patterns as uint16 for bf16 inputs --, device tensors
    dict, status word, slot mapping as numpy)."""
    import torch
    import scatter_kv_b200 as pa
    dv = to_dev(x)
    dims = dims_for(spec, x, hints, softcap, window)
    bufs = pa.allocate(dims)
    sc = 0.0 if scale is None else scale    # 0: the library's 1 / sqrt(head_size)
    outs = []
    for _ in range(repeat):
        pa.step(dv["query"], dv["key"], dv["value"], dv["key_cache"], dv["value_cache"],
                dv["block_table"], dv["cu_seqlens_q"], dv["seqlens_kv"], sc, dims, bufs,
                fused=fused)
        torch.cuda.synchronize()
        outs.append(host_bits(bufs.out, spec.elem))
    status = int(bufs.status[0].item())
    slots = bufs.slot_mapping[:spec.token_count].cpu().numpy().copy()
    return (outs if repeat > 1 else outs[0]), dv, status, slots


def oracle_step(spec: workloads.Spec, x: dict, rows=None, scale: float | None = None,
                softcap: float = 0.0, window=None):
    """The oracle's slot mapping, scatter (on copies of the caches) and attention."""
    kc = x["key_cache"].copy()
    vc = x["value_cache"].copy()
    slots = oracle.slot_mapping(x["block_table"], x["cu_seqlens_q"], x["seqlens_kv"],
                                spec.block_size)
    oracle.scatter_kv(x["key"], x["value"], slots, kc, vc)
    sc = 1.0 / math.sqrt(spec.head_size) if scale is None else scale
    y = oracle.attention(x["query"], kc, vc, x["block_table"], x["cu_seqlens_q"], x["seqlens_kv"],
                         sc, rows=rows, softcap=softcap, window=-1 if window is None else window,
                         bf16=spec.elem == "bf16")
    return y, kc, vc, slots


def assert_close(got, want, max_abs=MAX_ABS, mean_abs=MEAN_ABS, what="", elem="f16"):
    got = as_float64(got, elem)
    want = np.asarray(want, dtype=np.float64)
    assert got.shape == want.shape, (got.shape, want.shape)
    if got.size == 0:
        return
    assert np.isfinite(got).all(), f"{what}: non-finite output"
    err = np.abs(got - want)
    i = int(np.argmax(err))
    assert err.max() <= max_abs, f"{what}: max abs err {err.max():.3g} at flat {i} (got {got.flat[i]}, want {want.flat[i]})"
    assert err.mean() <= mean_abs, f"{what}: mean abs err {err.mean():.3g}"


def sample_rows(spec: workloads.Spec, n: int, seed: int = 0) -> np.ndarray:
    """n (token, head) pairs: every sequence's first and last token plus random ones."""
    rng = np.random.default_rng(seed)
    cu = np.concatenate([[0], np.cumsum(spec.q_lens)])
    picks = []
    for b in range(spec.batch):
        if spec.q_lens[b] == 0:
            continue
        for t in {int(cu[b]), int(cu[b + 1] - 1)}:
            picks.append((t, int(rng.integers(spec.q_heads))))
    while len(picks) < n and spec.token_count:
        picks.append((int(rng.integers(spec.token_count)), int(rng.integers(spec.q_heads))))
    return np.array(picks[:max(n, len(picks))], dtype=np.int64)


def poison_unused(spec: workloads.Spec, x: dict):
    """NaN into every cache row that no sequence's keys [0, seqlens_kv) map to."""
    used = oracle.kv_slots(x["block_table"], x["seqlens_kv"], spec.block_size)
    for name in ("key_cache", "value_cache"):
        flat = x[name].reshape(spec.num_blocks * spec.block_size, spec.kv_heads, spec.head_size)
        keep = flat[used].copy()
        flat[:] = workloads.fill_value(spec.elem, np.nan)
        flat[used] = keep
