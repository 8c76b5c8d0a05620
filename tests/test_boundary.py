"""Device-side metadata checks: invalid sequences are flagged in the status
word and get all-zero output rows; valid sequences in the same batch are
unaffected.  Every case is built so that no kernel reads outside its buffers
(the checks run before any page is touched)."""
import numpy as np
import pytest

import scatter_kv_b200 as pa
import workloads
from pa_harness import assert_close, oracle_step, run_gpu

pytestmark = pytest.mark.gpu


def _spec():
    # seq 0 decode, seq 1 prefill, seq 2 decode with several splits, seq 3 prefill.
    return workloads.custom([1, 40, 2, 150], [600, 20, 3000, 10], 16, 4, 128, 16, seed=21)


def _rows(spec, b):
    cu = np.concatenate([[0], np.cumsum(spec.q_lens)])
    return slice(int(cu[b]), int(cu[b + 1]))


def _check(spec, x, bad_seq, bit, hints=True, want_x=None):
    got, _, status, _ = run_gpu(spec, x, hints=hints)
    assert status & bit, f"status {status:#x} lacks {bit:#x}"
    assert not got[_rows(spec, bad_seq)].any(), "rows of the invalid sequence must be zero"
    want, _, _, _ = oracle_step(spec, want_x if want_x is not None else x)
    for b in range(spec.batch):
        if b != bad_seq:
            assert_close(got[_rows(spec, b)], want[_rows(spec, b)], what=f"seq {b}")


@pytest.mark.parametrize("where", ["first", "last"])
@pytest.mark.parametrize("bad_seq", [0, 1, 2, 3])
def test_out_of_range_block_id(bad_seq, where):
    # "last" puts the bad id in the sequence's last page, which for sequence 2
    # belongs to its last split rather than the first.
    spec = _spec()
    x = workloads.generate(spec)
    ref = {k: v.copy() for k, v in x.items()}
    page = 0 if where == "first" else (int(spec.seqlens_kv[bad_seq]) - 1) // spec.block_size
    x["block_table"][bad_seq, page] = spec.num_blocks + 5 if where == "first" else -1
    _check(spec, x, bad_seq, pa.PA_DEV_BAD_BLOCK, want_x=ref)


def test_bad_id_past_sequence_end_ignored():
    # Block-table entries past a sequence's last page are never read.
    spec = _spec()
    x = workloads.generate(spec)
    for b in range(spec.batch):
        npages = int(spec.pages_per_seq[b])
        x["block_table"][b, npages:] = -7
    got, _, status, _ = run_gpu(spec, x)
    assert status == 0, f"status {status:#x}"
    want, _, _, _ = oracle_step(spec, x)
    assert_close(got, want)


@pytest.mark.parametrize("bad_seq", [0, 1])
def test_q_len_longer_than_kv(bad_seq):
    spec = _spec()
    x = workloads.generate(spec)
    ref = {k: v.copy() for k, v in x.items()}
    x["seqlens_kv"][bad_seq] = spec.q_lens[bad_seq] - 1
    _check(spec, x, bad_seq, pa.PA_DEV_QLEN_GT_KV, want_x=ref)


def test_kv_longer_than_block_table():
    spec = _spec()
    x = workloads.generate(spec)
    ref = {k: v.copy() for k, v in x.items()}
    x["seqlens_kv"][3] = x["block_table"].shape[1] * spec.block_size + 1
    _check(spec, x, 3, pa.PA_DEV_KV_TOO_LONG, want_x=ref)


def test_hint_exceeded():
    spec = _spec()
    x = workloads.generate(spec)
    ref = {k: v.copy() for k, v in x.items()}
    x["seqlens_kv"][2] += 0       # unchanged data; the hint below is one short of seq 2
    import pa_harness
    orig = pa_harness.dims_for

    def short_hint(s, xx, hints=True, *args, **kwargs):
        d = orig(s, xx, hints, *args, **kwargs)
        d.max_seqlen_kv_hint = int(s.seqlens_kv[2]) - 1
        return d
    pa_harness.dims_for = short_hint
    try:
        _check(spec, x, 2, pa.PA_DEV_HINT_EXCEEDED, want_x=ref)
    finally:
        pa_harness.dims_for = orig


def test_bad_cu_seqlens_flagged():
    spec = _spec()
    x = workloads.generate(spec)
    x["cu_seqlens_q"][-1] -= 1       # last sequence ends before token_count
    got, _, status, _ = run_gpu(spec, x)
    assert status & pa.PA_DEV_BAD_CU_SEQLENS


@pytest.mark.gpu
def test_side_stream_from_two_host_threads():
    """Mixed batches (decode and prefill sequences, so the decode part forks
    to the library's side stream) from two host threads on two streams at
    once, 20 calls each: every result equals the serial one bit for bit."""
    import threading

    import torch
    import scatter_kv_b200 as pa
    from pa_harness import dims_for, host_bits, to_dev

    specs = [workloads.custom([1, 3, 90, 1, 200], [700, 2000, 30, 5, 400], 16, 4, 128, 16, seed=61),
             workloads.custom([2, 150, 1], [3000, 0, 900], 32, 8, 128, 16, seed=62)]
    runs = []
    for spec in specs:
        x = workloads.generate(spec)
        dv = to_dev(x)
        dims = dims_for(spec, x)
        bufs = pa.allocate(dims)
        pa.step(dv["query"], dv["key"], dv["value"], dv["key_cache"], dv["value_cache"],
                dv["block_table"], dv["cu_seqlens_q"], dv["seqlens_kv"], 0.0, dims, bufs)
        torch.cuda.synchronize()
        runs.append((spec, dv, dims, bufs, host_bits(bufs.out, spec.elem)))
    errors = []

    def worker(i):
        try:
            spec, dv, dims, bufs, ref = runs[i]
            s = torch.cuda.Stream()
            outs = []
            with torch.cuda.stream(s):
                for _ in range(20):
                    pa.pa_attention(dv["query"], dv["key_cache"], dv["value_cache"], dv["block_table"],
                                    dv["cu_seqlens_q"], dv["seqlens_kv"], 0.0, bufs.out, dims,
                                    bufs.workspace, None, bufs.status, s)
                    outs.append(bufs.out.clone())
            s.synchronize()
            for o in outs:
                if not np.array_equal(host_bits(o, spec.elem).view(np.uint16), ref.view(np.uint16)):
                    errors.append(f"thread {i}: result differs")
                    break
            if int(bufs.status[0].item()) != 0:
                errors.append(f"thread {i}: status {int(bufs.status[0].item()):#x}")
        except Exception as e:          # noqa: BLE001 -- reported below
            errors.append(f"thread {i}: {e!r}")

    threads = [threading.Thread(target=worker, args=(i,)) for i in range(2)]
    for t in threads:
        t.start()
    for t in threads:
        t.join()
    assert not errors, errors
