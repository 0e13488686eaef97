"""Host logic of bench.py that needs no GPU: the source hash that keeps committed ncu traffic
figures attached to the kernel code they were measured on."""


def test_code_sha_ignores_comments_but_not_code(tmp_path):
    import bench

    a = tmp_path / "a.cu"
    a.write_text("// header\n__global__ void k(int* p) {\n  p[0] = 1;  /* store */\n}\n")
    b = tmp_path / "b.cu"
    b.write_text("// a reworded header\n/* block\n comment */\n__global__ void k(int* p) {\n\n  p[0] = 1;\n}\n")
    c = tmp_path / "c.cu"
    c.write_text("// header\n__global__ void k(int* p) {\n  p[0] = 2;  /* store */\n}\n")
    assert bench.code_sha(str(a)) == bench.code_sha(str(b))
    assert bench.code_sha(str(a)) != bench.code_sha(str(c))

