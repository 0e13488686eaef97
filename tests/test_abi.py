"""CPU checks of the C-ABI boundary: the libraries load, export every declared symbol, and the
host-side argument checks answer with the documented status codes (no kernel is launched)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared(header):
    text = open(os.path.join(ROOT, "include", header)).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b((?:qsa|qsyn)_[a-z_0-9]+)\s*\(", text)))


@pytest.mark.parametrize("header,lib", [("qsa.h", "learned_block_sparse_qsa_b200/libqsa.so"),
                                        ("qsa_synth.h", "qsa_synth/libqsa_synth.so")])
def test_library_exports_every_declared_symbol(header, lib):
    names = declared(header)
    assert len(names) >= 2
    so = ctypes.CDLL(os.path.join(ROOT, lib))
    missing = [n for n in names if not hasattr(so, n)]
    assert not missing, missing


def test_qsa_header_declares_the_layer_entry_points():
    names = declared("qsa.h")
    for n in ["qsa_index_compress", "qsa_index_score_topk", "qsa_sparse_attn_prefill",
              "qsa_sparse_attn_decode", "qsa_dense_attn_prefill", "qsa_dense_attn_decode",
              "qsa_workspace_size", "qsa_status_string"]:
        assert n in names


import learned_block_sparse_qsa_b200 as q  # noqa: E402


def mk_batch(num_q=16, batch=1, max_pages=4, num_pages=4, max_pos=255, ptr=0x1000):
    return q.QsaBatch(batch, num_q, max_pages, num_pages, max_pos, ptr, ptr, ptr, ptr)


def test_status_strings_and_version():
    assert q.qsa_status_string(0) == "ok"
    assert "workspace" in q.qsa_status_string(3)
    assert q.qsa_version() >= 100


def test_workspace_sizes_are_host_computable():
    cfg = q.QsaConfig.make(32, 4, 128, 128)
    b = mk_batch(num_q=16384, max_pages=16384, num_pages=16384, max_pos=1048575)
    n_stream = q.qsa_workspace_size(cfg, b, q.QSA_OP_INDEX_SCORE_TOPK)
    assert n_stream >= 16384 * 2048 * 8           # streaming path: >= 2048 candidate slots per row
    b = mk_batch(num_q=16, batch=4, max_pages=16384, num_pages=65536, max_pos=1048575)
    assert q.qsa_workspace_size(cfg, b, q.QSA_OP_INDEX_SCORE_TOPK) > 0
    cfg_mat = q.QsaConfig.make(32, 4, 128, 128, score_path=2)
    n_mat = q.qsa_workspace_size(cfg_mat, b, q.QSA_OP_INDEX_SCORE_TOPK)
    assert n_mat >= 16 * 262144 * 12              # materialised path: scores + boundary keys
    assert q.qsa_workspace_size(cfg, b, q.QSA_OP_SPARSE_ATTN_DECODE, 1) == 0
    assert q.qsa_workspace_size(cfg, b, q.QSA_OP_SPARSE_ATTN_DECODE, 8) >= 16 * 8 * 32 * 129 * 4


@pytest.mark.parametrize("field,value,status", [
    ("block_tokens", 8, q.QSA_ERR_UNSUPPORTED), ("idx_heads", 2, q.QSA_ERR_UNSUPPORTED),
    ("head_dim", 96, q.QSA_ERR_UNSUPPORTED), ("topk_blocks", 0, q.QSA_ERR_UNSUPPORTED),
    ("topk_blocks", 513, q.QSA_ERR_UNSUPPORTED), ("num_q_heads", 6, q.QSA_ERR_INVALID_ARG),
    ("page_tokens", 32, q.QSA_ERR_UNSUPPORTED), ("score_path", 6, q.QSA_ERR_INVALID_ARG)])
def test_invalid_config_rejected_before_launch(field, value, status):
    cfg = q.QsaConfig.make(32, 4, 128, 128)
    setattr(cfg, field, value)
    with pytest.raises(q.QsaError) as e:
        q.qsa_workspace_size(cfg, mk_batch(), q.QSA_OP_INDEX_SCORE_TOPK)
    assert e.value.status == status


def test_invalid_arguments_rejected_before_launch():
    cfg = q.QsaConfig.make(4, 1, 64, 32)
    b = mk_batch()
    with pytest.raises(q.QsaError) as e:   # n_new not a multiple of 4
        q.qsa_index_compress(cfg, b, 0x1000, 0x1000, 0x1000, 6, 0x1000, stream=0)
    assert e.value.status == q.QSA_ERR_INVALID_ARG
    with pytest.raises(q.QsaError) as e:   # misaligned key pointer
        q.qsa_index_compress(cfg, b, 0x1002, 0x1000, 0x1000, 8, 0x1000, stream=0)
    assert e.value.status == q.QSA_ERR_INVALID_ARG
    with pytest.raises(q.QsaError) as e:   # no workspace
        q.qsa_index_score_topk(cfg, b, 0x1000, 0x1000, 0x1000, 0x1000, 0x1000, None, None, 0, stream=0)
    assert e.value.status == q.QSA_ERR_WORKSPACE
    with pytest.raises(q.QsaError) as e:   # missing page table
        bad = mk_batch()
        bad.page_table = None
        q.qsa_sparse_attn_prefill(cfg, bad, 0x1000, 0x1000, 0x1000, 0x1000, 0x1000, 0x1000, stream=0)
    assert e.value.status == q.QSA_ERR_INVALID_ARG
    with pytest.raises(q.QsaError) as e:   # decode with splits but no workspace
        q.qsa_sparse_attn_decode(cfg, b, 0x1000, 0x1000, 0x1000, 0x1000, 0x1000, 0x1000, None, 12,
                                 None, 0, stream=0)
    assert e.value.status == q.QSA_ERR_WORKSPACE


def test_redo_flags_live_in_the_score_workspace():
    """The redo-flag query is host arithmetic on the workspace address: flags for the tensor-core
    and split-list paths, none for the materialised and plain streaming paths."""
    b = mk_batch(num_q=16384, max_pages=16384, num_pages=16384, max_pos=1048575)
    ws = 1 << 40
    for path, has in [(1, True), (2, False), (4, False), (5, True)]:
        cfg = q.QsaConfig.make(32, 4, 128, 128, score_path=path)
        n = q.qsa_workspace_size(cfg, b, q.QSA_OP_INDEX_SCORE_TOPK)
        p = q.qsa_index_score_redo_flags(cfg, b, ws, n)
        assert (p is not None) == has
        if has:
            assert ws <= p and p + 16384 * 4 <= ws + n
    dec = mk_batch(num_q=16, batch=4, max_pages=16384, num_pages=65536, max_pos=1048575)
    cfg = q.QsaConfig.make(32, 4, 128, 128)
    n = q.qsa_workspace_size(cfg, dec, q.QSA_OP_INDEX_SCORE_TOPK)
    p = q.qsa_index_score_redo_flags(cfg, dec, ws, n)
    assert p is not None and ws <= p and p + 16 * 4 <= ws + n
    with pytest.raises(q.QsaError) as e:
        q.qsa_index_score_redo_flags(cfg, dec, ws, n - 256)
    assert e.value.status == q.QSA_ERR_WORKSPACE
    c32 = q.QsaConfig.make(4, 1, 64, 32, score_path=1)
    assert q.qsa_index_score_redo_flags(c32, b, ws, 1 << 40) is None


def test_selftest_rejects_limits_outside_range_before_launch():
    with pytest.raises(q.QsaError) as e:
        q.qsa_selftest_wait_timeout(0x1000, 10, stream=0)
    assert e.value.status == q.QSA_ERR_INVALID_ARG
    with pytest.raises(q.QsaError) as e:
        q.qsa_selftest_wait_timeout(None, 1_000_000, stream=0)
    assert e.value.status == q.QSA_ERR_INVALID_ARG


def test_distill_workspace_contract():
    """The distillation call's workspace: block masses and indexer scores of every row (fp32,
    candidates rounded up to 4 per row) in the tensor-core form (head_dim 128, 8 query heads per
    KV head); none in the other forms.  Without it the tensor-core form refuses to launch."""
    b = mk_batch(num_q=1024, max_pages=1024, num_pages=1024, max_pos=65535)
    cfg = q.QsaConfig.make(32, 4, 128, 128)
    ld = ((65535 // 4 + 1) + 3) // 4 * 4
    assert q.qsa_workspace_size(cfg, b, q.QSA_OP_DISTILL_KL) == 2 * 1024 * ld * 4
    for hq, hkv, d in ((32, 4, 64), (32, 2, 128), (8, 8, 128)):  # head_dim 64; 16 and 1 per KV head
        assert q.qsa_workspace_size(q.QsaConfig.make(hq, hkv, d, 128), b, q.QSA_OP_DISTILL_KL) == 0
    with pytest.raises(q.QsaError) as e:
        q.qsa_index_distill_kl(cfg, b, 0x1000, 0x1000, 0x1000, 0x1000, 0x1000, 0x1000, stream=0)
    # QSA_ERR_WORKSPACE, or QSA_ERR_UNSUPPORTED where the driver has no tensor-map encoder (no GPU)
    assert e.value.status in (q.QSA_ERR_WORKSPACE, q.QSA_ERR_UNSUPPORTED)


def test_decode_score_workspace_holds_the_exact_path_keys():
    """The split-list decode indexer (score_path 3, and auto for a few rows) runs the exact
    selection of a row its lists cannot settle inside the merge launch; the workspace must hold
    that path's keys: (max_pos/4 + 1) 8-byte keys for every row."""
    b = mk_batch(num_q=16, batch=4, max_pages=16384, num_pages=65536, max_pos=1048575)
    for path in (0, 3):
        cfg = q.QsaConfig.make(32, 4, 128, 128, score_path=path)
        assert q.qsa_workspace_size(cfg, b, q.QSA_OP_INDEX_SCORE_TOPK) >= 16 * (1048575 // 4 + 1) * 8


def test_noalloc_automatic_split_count_fits_the_scratch():
    """qsa_sparse_attn_decode_noalloc with an automatic split count lowers the count until the
    partials fit its 4 MiB scratch; an explicit count that does not fit is refused.  A shape whose
    automatic workspace exceeds 4 MiB (64 rows x 64 query heads): the explicit count gets
    QSA_ERR_WORKSPACE before anything else, the automatic one passes that point and, on a host
    with no GPU, stops at the launch (QSA_ERR_CUDA).  Host-only: the pointers are not real, so
    the test never runs where a GPU could launch on them."""
    torch = pytest.importorskip("torch")
    if torch.cuda.is_available():
        pytest.skip("host-only: would launch on placeholder pointers")
    b = mk_batch(num_q=64, max_pages=16384, num_pages=16384, max_pos=1048575)
    cfg = q.QsaConfig.make(64, 8, 128, 128)
    assert q.qsa_workspace_size(cfg, b, q.QSA_OP_SPARSE_ATTN_DECODE, 0) > 4 << 20
    args = (cfg, b, 0x1000, 0x1000, 0x1000, 0x1000, 0x1000, 0x1000, None)
    with pytest.raises(q.QsaError) as e:
        q.qsa_sparse_attn_decode_noalloc(*args, 64, stream=0)
    assert e.value.status == q.QSA_ERR_WORKSPACE
    with pytest.raises(q.QsaError) as e:
        q.qsa_sparse_attn_decode_noalloc(*args, 0, stream=0)
    assert e.value.status == q.QSA_ERR_CUDA
