"""Host logic of bench.py that needs no GPU: the source hash that keeps committed ncu traffic
figures attached to the kernel code they were measured on, and the count of the library's kernels
per prefill step."""


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



def test_prefill_launch_count_follows_the_library_indexer_form():
    """bench.py counts the prefill step's kernels from the indexer form the automatic score path
    resolves to (stream-K: sample, scan, stream, select; else one launch).  The library's choice is
    visible on the host through the workspace size, which differs between the two forms: check
    that the bench's geometry rule agrees with it on the prefill workloads."""
    import bench
    import learned_block_sparse_qsa_b200 as q
    from qsa_synth import CONFIGS

    for name in ("C2", "C4"):
        c = CONFIGS[name]
        b = q.QsaBatch(c.batch, c.num_q, c.max_pages, c.num_pages, c.ctx - 1, 0x1000, 0x1000, 0x1000,
                       0x1000)
        size = {}
        for path in (0, 1, 5):  # auto, stream-K form, single-launch form
            cfg = q.QsaConfig.make(c.Hq, c.Hkv, c.D, c.Di, topk=c.topk, score_path=path)
            size[path] = q.qsa_workspace_size(cfg, b, q.QSA_OP_INDEX_SCORE_TOPK)
        assert size[1] != size[5]
        stream = size[0] == size[1]
        assert size[0] == (size[1] if stream else size[5])
        assert bench.prefill_launches_per_step(c) == (7 if stream else 4), name
    assert bench.prefill_launches_per_step(CONFIGS["C4"]) == 7
