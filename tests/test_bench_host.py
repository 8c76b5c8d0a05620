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
