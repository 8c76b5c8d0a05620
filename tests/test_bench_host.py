"""Host logic of bench.py that needs no GPU: the kernel-source hash that ties a
committed ncu summary (its DRAM traffic figure) to the code it measured."""
import bench


def test_strip_comments_keeps_code_and_literals():
    src = ('int a = 1;  // trailing\n'
           '/* block\n   comment */ const char* s = "// not a comment";\n'
           "char q = '\"'; int b; /* x */\n"
           '\n\n'
           'asm("add.rn.f32x2 %0, %1;");\n')
    out = bench._strip_comments(src)
    assert out == ('int a = 1;\n'
                   ' const char* s = "// not a comment";\n'
                   "char q = '\"'; int b;\n"
                   'asm("add.rn.f32x2 %0, %1;");')


def test_source_hash_ignores_comments_but_not_code(tmp_path, monkeypatch):
    csrc = tmp_path / "scatter_kv_b200" / "csrc"
    csrc.mkdir(parents=True)
    (csrc / "k.cu").write_text("__global__ void k(int* p) { p[0] = 1; }  // one\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    h0 = bench.kernel_source_hash()
    (csrc / "k.cu").write_text("// header\n__global__ void k(int* p) { p[0] = 1; }  /* other */\n")
    assert bench.kernel_source_hash() == h0
    (csrc / "k.cu").write_text("__global__ void k(int* p) { p[0] = 2; }\n")
    assert bench.kernel_source_hash() != h0
    (csrc / "k.cu").write_text("__global__ void k(int* p) { p[0] = 1; }\n")
    (csrc / "k2.cuh").write_text("#define X 1\n")
    assert bench.kernel_source_hash() != h0


def test_algorithmic_counts_split_between_kernels():
    import workloads
    # GQA 4 (decode cut-off 4): two decode sequences, one prefill chunk.
    spec = workloads.custom([1, 4, 10], [100, 20, 5], 8, 2, 16, 16)
    c = bench.algorithmic_counts(spec)
    kv = lambda t: t * 2 * 16 * 2 * 2          # K and V rows of 2 KV heads, f16
    q = lambda n: n * 8 * 16 * 2                # query (or output) rows of 8 heads
    assert c["kv_bytes"] == kv(101) + kv(24) + kv(15)
    assert c["decode_bytes"] == kv(101) + kv(24) + q(1) + q(4)
    assert c["prefill_bytes"] == kv(15) + 2 * q(10)
    # visible keys: 101 for the first sequence; 21..24; 6..15
    assert c["flops"] == 4 * 8 * 16 * (101 + sum(range(21, 25)) + sum(range(6, 16)))
    assert c["prefill_flops"] == 4 * 8 * 16 * sum(range(6, 16))
    assert not c["decode"] and bench.unit_of(spec) == "TFLOP/s"
    assert bench.unit_of(workloads.custom([1, 3], [9, 9], 8, 2, 16, 16)) == "GB/s"


def test_profile_hash_covers_only_the_kernels_sources(tmp_path, monkeypatch):
    csrc = tmp_path / "scatter_kv_b200" / "csrc"
    csrc.mkdir(parents=True)
    for n in ("pa_decode.cu", "pa_common.cuh", "pa_internal.h", "pa_prefill.cu"):
        (csrc / n).write_text(f"int {n.split('.')[0]};\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    files = bench.KERNEL_SOURCES["decode_split_kv"]
    h0 = bench.kernel_source_hash(files)
    (csrc / "pa_prefill.cu").write_text("int changed;\n")
    assert bench.kernel_source_hash(files) == h0
    (csrc / "pa_common.cuh").write_text("int changed;\n")
    assert bench.kernel_source_hash(files) != h0
