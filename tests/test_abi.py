"""The C-ABI library builds for sm_100a, loads, exports every symbol the
header declares, and rejects bad arguments on the host before any launch
(none of these calls reaches a GPU)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def pa():
    import scatter_kv_b200
    return scatter_kv_b200


def _declared_functions():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names |= set(re.findall(r"\b(pa_[a-z0-9_]+)\s*\(", src))
    return sorted(names)


def test_library_exports_every_declared_function(pa):
    declared = _declared_functions()
    assert "pa_attention" in declared and "pa_scatter_kv" in declared
    lib = ctypes.CDLL(pa.LIB_PATH)
    for name in declared:
        assert hasattr(lib, name), f"{name} declared in include/ but not exported"
    assert set(pa.EXPORTS) == set(declared)


def test_library_is_built_for_sm100a():
    from scatter_kv_b200 import build
    assert "arch=compute_100a,code=sm_100a" in " ".join(build.ARCH)


def _dims(pa, **kw):
    base = dict(batch=2, token_count=5, q_heads=8, kv_heads=2, head_size=128, num_blocks=16,
                block_size=16, max_blocks_per_seq=4)
    base.update(kw)
    return pa.make_dims(**base)


FAKE = 1 << 20          # aligned non-null address; never dereferenced (calls fail first)


@pytest.mark.parametrize("kw,status", [
    (dict(q_heads=6, kv_heads=4), 1),            # not a multiple
    (dict(q_heads=256, kv_heads=1), 2),          # group 256: not built (prefill rows <= 128)
    (dict(head_size=20), 1),                     # not a multiple of 8
    (dict(head_size=264), 1),                    # beyond 256
    (dict(softcap=-1.0), 1),
    (dict(window=-2), 1),
    (dict(block_size=24), 1),
    (dict(block_size=512), 1),
    (dict(num_blocks=1 << 28, block_size=16), 1),  # slots overflow int32
    (dict(token_count=-1), 1),
])
def test_dims_rejected_before_launch(pa, kw, status):
    d = _dims(pa, **kw)
    with pytest.raises(pa.PagedAttentionError) as e:
        pa.pa_attention(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 0.0, FAKE, d, None, 0, None, 0)
    assert e.value.status == status


def _rotary(pa, rd, inter=0, maxpos=64):
    r = pa.pa_rotary()
    r.rotary_dim, r.interleaved, r.max_position = rd, inter, maxpos
    return r


@pytest.mark.parametrize("rd,maxpos,qs,status,text", [
    (15, 64, 0, 1, "rotary_dim"),        # odd
    (136, 64, 0, 1, "rotary_dim"),       # beyond head_size
    (24, 64, 0, 2, "multiples of 16"),   # even, valid per the pages, not built
    (64, 0, 0, 1, "max_position"),
    (64, 64, 8 * 128 - 8, 1, "strides"),  # stride shorter than the query heads
    (64, 64, 8 * 128 + 4, 1, "strides"),  # not a multiple of 8 elements
])
def test_split_qkv_rotary_rejects_bad_arguments(pa, rd, maxpos, qs, status, text):
    d = _dims(pa)
    with pytest.raises(pa.PagedAttentionError) as e:
        pa.pa_split_qkv_rotary_scatter(FAKE, FAKE, FAKE, qs, 0, FAKE, FAKE, _rotary(pa, rd, 0, maxpos),
                                       FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, d, None, 0)
    assert e.value.status == status
    assert text in str(e.value)


def test_split_qkv_rotary_needs_caches_only_with_rotation(pa):
    d = _dims(pa)
    with pytest.raises(pa.PagedAttentionError) as e:
        pa.pa_split_qkv_rotary_scatter(FAKE, FAKE, FAKE, 0, 0, None, FAKE, _rotary(pa, 64), FAKE,
                                       FAKE, FAKE, FAKE, FAKE, FAKE, None, d, None, 0)
    assert "cos_cache" in str(e.value)
    # Without a query output the query may be NULL (scatter only); the other
    # tensors may not.
    with pytest.raises(pa.PagedAttentionError) as e:
        pa.pa_split_qkv_rotary_scatter(None, None, FAKE, 0, 0, None, None, None, FAKE, FAKE, FAKE,
                                       None, FAKE, FAKE, None, d, None, 0)
    assert "key" in str(e.value)
    # token_count 0: nothing to do, nothing read.
    pa.pa_split_qkv_rotary_scatter(None, None, None, 0, 0, None, None, None, None, None, None,
                                   None, None, None, None, _dims(pa, token_count=0), None, 0)


def test_null_and_misaligned_pointers(pa):
    d = _dims(pa)
    with pytest.raises(pa.PagedAttentionError) as e:
        pa.pa_scatter_kv(None, FAKE, FAKE, FAKE, FAKE, d, None, 0)
    assert e.value.status == pa.PA_ERR_INVALID_ARGUMENT and "key" in str(e.value)
    with pytest.raises(pa.PagedAttentionError) as e:
        pa.pa_attention(FAKE + 8, FAKE, FAKE, FAKE, FAKE, FAKE, 0.0, FAKE, d, None, 0, None, 0)
    assert "aligned" in str(e.value)
    with pytest.raises(pa.PagedAttentionError):
        pa.pa_compute_slot_mapping(FAKE, FAKE + 2, FAKE, FAKE, d, None, 0)


def test_bad_scale_rejected(pa):
    d = _dims(pa)
    for sc in (-1.0, float("inf"), float("nan")):
        with pytest.raises(pa.PagedAttentionError):
            pa.pa_attention(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, sc, FAKE, d, None, 0, None, 0)


def test_empty_batch_is_a_noop(pa):
    d = _dims(pa, token_count=0)
    pa.pa_scatter_kv(None, None, None, None, None, d, None, 0)
    pa.pa_compute_slot_mapping(None, None, None, None, d, None, 0)
    pa.pa_attention(None, None, None, None, None, None, 0.0, None, d, None, 0, None, 0)


def test_workspace_size_and_undersized_workspace(pa):
    d = _dims(pa, max_blocks_per_seq=512, block_size=16)
    n = pa.pa_attention_workspace_size(d)
    assert n > 0 and n % 256 == 0
    with pytest.raises(pa.PagedAttentionError) as e:
        pa.pa_attention(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 0.0, FAKE, d, FAKE, n - 256, None, 0)
    assert "workspace" in str(e.value)
    # A short maximum length needs a single split and no workspace at all.
    assert pa.pa_attention_workspace_size(_dims(pa, max_blocks_per_seq=2)) == 0
    # Groups above 32 run no decode kernel, so they need no split workspace.
    assert pa.pa_attention_workspace_size(_dims(pa, q_heads=64, kv_heads=1, max_blocks_per_seq=512)) == 0
    assert pa.pa_attention_workspace_size(_dims(pa, q_heads=128, kv_heads=1, max_blocks_per_seq=512)) == 0


def test_int4_and_sparse_reject_groups_above_32(pa):
    d = _dims(pa, q_heads=64, kv_heads=1, head_size=128, max_seqlen_q=1)
    with pytest.raises(pa.PagedAttentionError) as e:
        pa.pa_attention_int4(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 0.0, FAKE, d, None, 0,
                             None, 0)
    assert e.value.status == pa.PA_ERR_NOT_IMPLEMENTED
    with pytest.raises(pa.PagedAttentionError) as e:
        pa.pa_sparse_attention(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 4, 8, 0.0, FAKE, d, None, 0)
    assert e.value.status == pa.PA_ERR_NOT_IMPLEMENTED


def test_status_strings(pa):
    assert pa.lib.pa_status_string(0) == b"PA_OK"
    assert pa.lib.pa_status_string(2) == b"PA_ERR_NOT_IMPLEMENTED"
    assert pa.lib.pa_kernel_name(pa.PA_KERNEL_PREFILL) == b"prefill_tcgen05"
