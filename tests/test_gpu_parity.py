"""GPU parity: the CUDA path (through the C-ABI) against the fp64 oracle on the same seeded inputs.

Bars: bit-exact compressed keys; on integer inputs (exact fp32 scores) identical selections and
scores; on N(0,1)-like inputs, indexer scores within 1e-3 relative to max(|s|, |s_512|), selection
differences only for blocks within that tolerance of the 512th score, attention within
atol 2e-2 + rtol 1e-2 of the oracle run on the GPU's own selection.
"""
import numpy as np
import pytest

from oracle import qsa_oracle as orc
from qsa_synth import CONFIGS
from tests.qsa_testlib import (Run, check_attention, check_selection, host, host_kcomp,
                               oracle_attend_row, oracle_dense_row, oracle_select_row, sample_rows,
                               score_bound)

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)


def kcomp_blocks(run: Run, s: int) -> np.ndarray:
    """GPU compressed keys of sequence s in block order, bf16 bits [n_pages*16, Di]."""
    pt = run.di.page_table[s].long()
    kc = run.di.kcomp_pool[pt].reshape(-1, run.c.Di)
    return kc.view(torch.int16).cpu().numpy().view(np.uint16)


@pytest.fixture(scope="module", params=[False, True], ids=["random", "int"])
def c1(request):
    return Run(CONFIGS["C1"], integer=request.param).step()


# ------------------------------------------------------------------------------------ C1, full

def test_compress_bit_exact_c1(c1):
    got = kcomp_blocks(c1, 0)[: c1.c.ctx // 4]
    want = host_kcomp(c1.c, c1.di.host.integer, 0)
    assert np.array_equal(got, want)


def test_selection_c1_all_rows(c1):
    o = c1.numpy()
    c, integer = c1.c, c1.di.host.integer
    h = host(c, integer)
    q_seq, q_pos = h.rows()
    kc = host_kcomp(c, integer, 0)
    iq, iw = h.idx_q(np.arange(c.num_q)), h.idx_w(np.arange(c.num_q))
    ndiff = 0
    for r in range(c.num_q):
        t = int(q_pos[r])
        ref_sel, ref_s = orc.qsa_select(kc, iq[r], iw[r], t, c.topk)
        ndiff += check_selection(o["sel"][r], o["n_sel"][r], o["sel_scores"][r], ref_sel, ref_s, t,
                                 c.topk, exact=integer, bound=score_bound(kc, iq[r], iw[r], t // 4))
    assert ndiff <= c.num_q // 100


def test_attention_c1_all_rows(c1):
    o = c1.numpy()
    c, integer = c1.c, c1.di.host.integer
    for r in range(0, c.num_q, 7 if not integer else 13):
        n = o["n_sel"][r]
        ref_o, ref_lse = oracle_attend_row(c, integer, r, o["sel"][r][:n])
        check_attention(o["out"][r], o["lse"][r], ref_o, ref_lse)


@pytest.mark.parametrize("path", [1, 2], ids=["streaming", "materialised"])
def test_score_paths_agree_c1(path):
    """Both selection algorithms give identical selections on exact (integer) inputs."""
    run = Run(CONFIGS["C1"], integer=True, score_path=path).step()
    o = run.numpy()
    c = run.c
    kc = host_kcomp(c, True, 0)
    h = host(c, True)
    q_seq, q_pos = h.rows()
    rows = list(range(0, 64)) + list(range(2040, 2060)) + list(range(4032, 4096))
    for r in rows:
        t = int(q_pos[r])
        ref_sel, ref_s = orc.qsa_select(kc, h.idx_q([r])[0], h.idx_w([r])[0], t, c.topk)
        check_selection(o["sel"][r], o["n_sel"][r], o["sel_scores"][r], ref_sel, ref_s, t, c.topk, True)


def test_scores_dump_c1():
    run = Run(CONFIGS["C1"], integer=False)
    from learned_block_sparse_qsa_b200 import qsa_index_compress, qsa_index_scores

    c = run.c
    d = run.di
    qsa_index_compress(run.cfg, run.b, d.idx_k_new, d.new_seq, d.new_pos, c.num_q, d.kcomp_pool)
    ld = c.ctx // 4
    scores = torch.full((c.num_q, ld), float("nan"), dtype=torch.float32, device="cuda")
    qsa_index_scores(run.cfg, run.b, d.idx_q, d.idx_w, d.kcomp_pool, scores, ld)
    torch.cuda.synchronize()
    g = scores.cpu().numpy()
    h = host(c, False)
    kc = host_kcomp(c, False, 0)
    _, q_pos = h.rows()
    for r in range(0, c.num_q, 5):
        t = int(q_pos[r])
        n = t // 4
        ref = orc.block_scores(kc, h.idx_q([r])[0], h.idx_w([r])[0], n)
        if n:
            sk = np.sort(ref)[-min(512, n)]
            eb = score_bound(kc, h.idx_q([r])[0], h.idx_w([r])[0], n)
            assert np.all(np.abs(g[r, :n] - ref) <= 1e-3 * np.maximum(np.abs(ref), abs(sk)) + eb)
        assert np.all(np.isnan(g[r, n:]))  # entries past the candidates are left untouched


def test_edge_rows_c1(c1):
    """t < 4 (only the tail block), the budget boundary, and t % 4 == 3."""
    o = c1.numpy()
    for r in range(4):
        assert o["n_sel"][r] == 1 and o["sel"][r][0] == 0 and np.all(o["sel"][r][1:] == -1)
    for t in (2047, 2048, 2051, 2052, 2055, 4095):
        n = min(512, t // 4) + 1
        assert o["n_sel"][t] == n and o["sel"][t][n - 1] == t // 4
        assert len(orc.expand(o["sel"][t][:n], t)) == min(t + 1, 2048 + t % 4 + 1)


def test_sparse_equals_dense_below_budget_c1(c1):
    """For t <= 2051 the selection covers every earlier block: QSA output == dense output."""
    c = c1.c
    d = c1.di
    dense = torch.empty_like(c1.out)
    c1.runner.dense(c1.b, q=d.q, k_pool=d.k_pool, v_pool=d.v_pool, out=dense)
    torch.cuda.synchronize()
    a = c1.out[:2052].float()
    b = dense[:2052].float()
    assert torch.allclose(a, b, atol=2e-2, rtol=1e-2)


def test_dense_prefill_c1_sampled(c1):
    c = c1.c
    d = c1.di
    dense = torch.empty_like(c1.out)
    lse = torch.empty_like(c1.lse)
    c1.runner.dense(c1.b, q=d.q, k_pool=d.k_pool, v_pool=d.v_pool, out=dense, lse=lse)
    torch.cuda.synchronize()
    g = dense.view(torch.int16).cpu().numpy().view(np.uint16)
    gl = lse.cpu().numpy()
    for r in sample_rows(c, 24):
        ref_o, ref_lse = oracle_dense_row(c, c1.di.host.integer, r)
        check_attention(g[r], gl[r], ref_o, ref_lse)


# ------------------------------------------------------------------------------------ small topk

@pytest.mark.parametrize("path", [1, 2], ids=["streaming", "materialised"])
@pytest.mark.parametrize("topk", [1, 4, 37])
def test_small_budget_exact(path, topk):
    """Budgets below the article's 512 exercise many compactions and ragged tiles."""
    c = CONFIGS["C1"].replace(ctx=1000, n_new=1000)
    run = Run(c, integer=True, score_path=path, topk=topk).step()
    o = run.numpy()
    h = host(run.c, True)
    kc = host_kcomp(run.c, True, 0)
    _, q_pos = h.rows()
    for r in range(0, c.num_q, 3):
        t = int(q_pos[r])
        ref_sel, ref_s = orc.qsa_select(kc, h.idx_q([r])[0], h.idx_w([r])[0], t, topk)
        check_selection(o["sel"][r], o["n_sel"][r], o["sel_scores"][r], ref_sel, ref_s, t, topk, True)
        ref_o, ref_lse = orc.attend(h.q([r])[0], *h.kv(0, orc.expand(ref_sel, t)))
        check_attention(o["out"][r], o["lse"][r], ref_o, ref_lse)


# ------------------------------------------------------------------------------------ decode C3

@pytest.fixture(scope="module", params=[False, True], ids=["random", "int"])
def c3(request):
    return Run(CONFIGS["C3"], integer=request.param).step()


def test_decode_c3_all_rows(c3):
    o = c3.numpy()
    c, integer = c3.c, c3.di.host.integer
    _, q_pos = host(c, integer).rows()
    for r in range(c.num_q):
        t = int(q_pos[r])
        ref_sel, ref_s, eb = oracle_select_row(c, integer, r)
        check_selection(o["sel"][r], o["n_sel"][r], o["sel_scores"][r], ref_sel, ref_s, t, c.topk, integer, eb)
        ref_o, ref_lse = oracle_attend_row(c, integer, r, o["sel"][r][: o["n_sel"][r]])
        check_attention(o["out"][r], o["lse"][r], ref_o, ref_lse)


@pytest.mark.parametrize("splits", [1, 2, 7, 33])
def test_decode_splits_agree(c3, splits):
    ref = c3.out.float().clone()
    c3.step(splits=splits)
    assert torch.allclose(c3.out.float(), ref, atol=1e-2, rtol=1e-2)


def test_decode_streaming_path_agrees_c3():
    """The streaming selection (many-row algorithm) on the decode workload, integer inputs."""
    a = Run(CONFIGS["C3"], integer=True, score_path=1).step().numpy()
    b = Run(CONFIGS["C3"], integer=True, score_path=2).step().numpy()
    assert np.array_equal(a["sel"], b["sel"]) and np.array_equal(a["n_sel"], b["n_sel"])


def test_dense_decode_c3_sampled(c3):
    c = c3.c
    d = c3.di
    dense = torch.empty_like(c3.out)
    lse = torch.empty_like(c3.lse)
    c3.runner.dense(c3.b, q=d.q, k_pool=d.k_pool, v_pool=d.v_pool, out=dense, lse=lse, decode=True)
    torch.cuda.synchronize()
    g = dense.view(torch.int16).cpu().numpy().view(np.uint16)
    gl = lse.cpu().numpy()
    r = 5
    h = host(c, c3.di.host.integer)
    q_seq, q_pos = h.rows()
    s, t = int(q_seq[r]), int(q_pos[r])
    # one KV head group of one row: regenerate only what head group 0 reads
    pos = np.arange(t + 1)
    starts = (s * c.ctx + pos) * (c.Hkv * c.D)
    k0 = h._lin(2, h.dist["k"], starts, c.D).reshape(-1, 1, c.D)
    v0 = h._lin(3, h.dist["v"], starts, c.D).reshape(-1, 1, c.D)
    qh = h.q([r])[0][: c.Hq // c.Hkv]
    ref_o, ref_lse = orc.dense_causal(qh, k0, v0, t)
    check_attention(g[r][: c.Hq // c.Hkv], gl[r][: c.Hq // c.Hkv], ref_o, ref_lse)


# ------------------------------------------------------------------------------------ C2 / C4 / C5

@pytest.mark.parametrize("name,nrows", [("C2", 48), ("C4", 128), ("C5", 16)])
def test_full_size_sampled(name, nrows):
    """The full-size workloads in the launch configuration the bench times: sampled rows against
    the oracle, properties on every row, and no row handed from the fast indexer kernel
    (tensor-core prefill, split-list decode) to the exact streaming kernel."""
    c = CONFIGS[name]
    run = Run(c, integer=False).step()
    redo = run.redo_flags()
    assert redo is not None and not redo.any(), int(redo.sum())
    o = run.numpy()
    _, q_pos = host(c, False).rows()
    for r in sample_rows(c, nrows):
        t = int(q_pos[r])
        ref_sel, ref_s, eb = oracle_select_row(c, False, r)
        check_selection(o["sel"][r], o["n_sel"][r], o["sel_scores"][r], ref_sel, ref_s, t, c.topk, False, eb)
        ref_o, ref_lse = oracle_attend_row(c, False, r, o["sel"][r][: o["n_sel"][r]])
        check_attention(o["out"][r], o["lse"][r], ref_o, ref_lse)
    # properties at every row: constant budget, tail last, causality
    assert np.all(o["n_sel"] == 513)
    assert np.all(o["sel"][:, 512] == q_pos // 4)
    assert np.all(np.diff(o["sel"], axis=1) > 0)
    assert run.runner.error_bits() == 0


def test_needle_recall_c2():
    """Sanity (not parity): rows that carry a planted needle select the needle block."""
    c = CONFIGS["C2"]
    run = Run(c, integer=False).step()
    o = run.numpy()
    nd = host(c, False).needles()
    hits = total = 0
    for r, j in nd["q_rows"].items():
        blk = int(nd["blocks"][0][j])
        total += 1
        hits += blk in set(o["sel"][r][:512].tolist())
    assert total > 1000 and hits / total > 0.99


# ------------------------------------------------------------------------------------ robustness

def test_bad_page_id_sets_flag_without_fault():
    c = CONFIGS["C1"].replace(ctx=512, n_new=512)
    run = Run(c, integer=True)
    run.di.page_table[0, 3] = 10_000  # outside the pool
    run.step()
    assert run.runner.error_bits() & 4


def test_bad_selection_entry_sets_flag():
    c = CONFIGS["C1"].replace(ctx=512, n_new=512)
    run = Run(c, integer=True).step()
    from learned_block_sparse_qsa_b200 import qsa_sparse_attn_prefill

    run.sel[100, 0] = 99999
    run.runner.clear_error()
    qsa_sparse_attn_prefill(run.cfg, run.b, run.di.q, run.di.k_pool, run.di.v_pool, run.sel,
                            run.n_sel, run.out, run.lse)
    torch.cuda.synchronize()
    assert run.runner.error_bits() & 16
    assert torch.isfinite(run.out.float()).all()


def test_empty_batch_is_a_no_op():
    from learned_block_sparse_qsa_b200 import QsaBatch, qsa_index_score_topk, qsa_sparse_attn_prefill

    c = CONFIGS["C1"].replace(ctx=512, n_new=512)
    run = Run(c, integer=True)
    b = QsaBatch(1, 0, c.max_pages, c.num_pages, 511, 0, 0, run.di.page_table.data_ptr(),
                 run.runner.err.data_ptr())
    qsa_index_score_topk(run.cfg, b, run.di.idx_q, run.di.idx_w, run.di.kcomp_pool, run.sel,
                         run.n_sel, None, None, 0)
    qsa_sparse_attn_prefill(run.cfg, b, run.di.q, run.di.k_pool, run.di.v_pool, run.sel, run.n_sel,
                            run.out)
    torch.cuda.synchronize()
    assert run.runner.error_bits() == 0


def test_device_generator_matches_host():
    c = CONFIGS["C3"]
    run = Run(c, integer=False)
    h = host(c, False)
    rng = np.random.default_rng(0)
    pt = h.page_table()
    for s in range(c.batch):
        pos = rng.integers(0, c.ctx, 64)
        k, v = h.kv(s, pos)
        phys = pt[s, pos // 64]
        gk = run.di.k_pool[torch.from_numpy(phys).long(), torch.from_numpy(pos % 64).long()]
        assert np.array_equal(gk.view(torch.int16).cpu().numpy().view(np.uint16), k)
    assert np.array_equal(run.di.q.view(torch.int16).cpu().numpy().view(np.uint16), h.q(np.arange(c.num_q)))
    assert np.array_equal(run.di.idx_q.view(torch.int16).cpu().numpy().view(np.uint16),
                          h.idx_q(np.arange(c.num_q)))
