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


def test_committed_profiles_are_well_formed():
    """Every ncu summary under profiles/ names a kernel the bench reports,
    records the source hash and the DRAM traffic the bench reads, and gives
    commands with --clock-control none.  (Whether the hash still matches the
    kernel's sources is the bench's business: it reports no traffic then.)"""
    import os
    import re
    pdir = os.path.join(bench.ROOT, "profiles")
    names = sorted(f for f in os.listdir(pdir) if f.endswith(".md"))
    assert names
    for f in names:
        assert any(f.startswith(k + "_") for k in bench.KERNEL_SOURCES if "@" not in k), f
        text = open(os.path.join(pdir, f)).read()
        assert re.search(r"source_hash:\s*[0-9a-f]{16}", text), f
        assert re.search(r"traffic_bytes_per_launch:\s*[0-9.]+", text), f
        for line in text.splitlines():
            if line.startswith("ncu "):
                assert "--clock-control none" in line, (f, line)


def test_head256_profiles_hash_the_head256_kernel(tmp_path, monkeypatch):
    csrc = tmp_path / "scatter_kv_b200" / "csrc"
    csrc.mkdir(parents=True)
    for n in ("pa_prefill.cu", "pa_prefill256.cu", "pa_common.cuh", "pa_internal.h"):
        (csrc / n).write_text(f"int {n.split('.')[0]};\n")
    pdir = tmp_path / "profiles"
    pdir.mkdir()
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    h = bench.kernel_source_hash(bench.KERNEL_SOURCES["prefill_tcgen05@d256"])
    (pdir / "prefill_tcgen05_prefill_d256.md").write_text(
        f"source_hash: {h}\ntraffic_bytes_per_launch: 123\n")
    assert bench.profiled_traffic("prefill_tcgen05", "prefill_d256") == 123.0
    (csrc / "pa_prefill.cu").write_text("int changed;\n")          # the 128-wide kernel: no effect
    assert bench.profiled_traffic("prefill_tcgen05", "prefill_d256") == 123.0
    (csrc / "pa_prefill256.cu").write_text("int changed;\n")
    assert bench.profiled_traffic("prefill_tcgen05", "prefill_d256") is None


def test_part_option_is_parsed():
    seen = {}

    def fake_run_gpu(args, spec, rank, world, local):
        seen["part"], seen["only"], seen["workload"] = args.part, args.only, args.workload

    orig = bench.run_gpu
    bench.run_gpu = fake_run_gpu
    try:
        bench.main(["--only", "--part", "d256", "--workload", "prefill", "--steps", "1"])
    finally:
        bench.run_gpu = orig
    assert seen == {"part": "d256", "only": True, "workload": "prefill"}
