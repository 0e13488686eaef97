"""GPU parity of the tensor-core (tcgen05) indexer path: exact on integer inputs on both of its
branches (rows of at most 4,096 candidates keep every key; longer rows -- every row of a long-
context chunk -- keep the keys at or above a threshold taken from a sample of tiles), ragged
multi-sequence row tiles, and the exact fallback for rows the fast kernel cannot settle.  The
redo flags the score call leaves in its workspace show which kernel produced each checked row.
Path 1 runs the tensor-core kernels in their stream-K form (every SM takes an equal share of the
row tiles' key tiles); path 5 runs the single-launch form (one CTA per 128-row tile); the two must
give identical selections."""
import numpy as np
import pytest

from oracle import qsa_oracle as orc
from qsa_synth import CONFIGS, Config
from tests.qsa_testlib import (Run, check_attention, check_selection, host, host_kcomp,
                               positive_int_weights, sample_rows, score_bound, tc_redo_model)

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

TC_PREFILL = Config("tc_prefill_T8192_di128", "prefill", 1, 8192, 8192, 8, 2, 64, 4, 128, seed=0x7C01)


def check_rows(run, rows, integer, topk=None, w_bits=None, model=False):
    """Selections of the given rows against the oracle.  w_bits: head weights [num_q, 4] that
    replaced the generator's.  model=True (integer inputs only): also compare the row's redo flag
    with tc_redo_model; returns the number of checked rows the fast kernel settled itself."""
    o = run.numpy()
    c = run.c
    topk = c.topk if topk is None else topk
    h = host(c, integer)
    q_seq, q_pos = h.rows()
    redo = run.redo_flags() if model else None
    settled = 0
    for r in rows:
        s, t = int(q_seq[r]), int(q_pos[r])
        kc = host_kcomp(c, integer, s)
        iq = h.idx_q([r])[0]
        iw = h.idx_w([r])[0] if w_bits is None else w_bits[r]
        ref_sel, ref_s = orc.qsa_select(kc, iq, iw, t, topk)
        check_selection(o["sel"][r], o["n_sel"][r], o["sel_scores"][r], ref_sel, ref_s, t, topk,
                        integer, score_bound(kc, iq, iw, t // 4))
        if model:
            tile = r // 128
            last = min(c.num_q, tile * 128 + 128) - 1  # rows of one sequence, positions ascending
            ntile = (int(q_pos[last]) // 4 + 127) // 128  # the CTA's tiles: its longest row
            nsamp = (ntile + 31) // 32
            want = tc_redo_model(ref_s, topk, nsamp)
            assert bool(redo[r]) == want, (r, t, int(redo[r]), want)
            settled += not want
    return settled if model else o


def run_positive_weights(c, score_path=1, **kw):
    """Integer inputs with head weights in {1, 2, 3} (positive, as in the pages' workloads)."""
    run = Run(c, integer=True, score_path=score_path, **kw)
    w = positive_int_weights(host(c, True).idx_w(np.arange(c.num_q)))
    run.di.idx_w.copy_(torch.from_numpy(w.view(np.int16)).view(torch.bfloat16))
    return run.step(), w


@pytest.mark.parametrize("path", [1, 5], ids=["stream_k", "single_launch"])
def test_tc_prefill_integer_exact_all_rows(path):
    """Rows of at most 2,048 candidates: the keep-every-key branch, no row handed over."""
    run = Run(TC_PREFILL, integer=True, score_path=path).step()
    check_rows(run, range(TC_PREFILL.num_q), True)
    assert run.runner.error_bits() == 0
    assert not run.redo_flags().any()


SAMPLED = Config("tc_sampled_chunk4096_ctx65536", "prefill", 1, 65536, 4096, 8, 2, 64, 4, 128,
                 shuffle_pages=True, seed=0x7C04)


@pytest.mark.parametrize("path", [1, 5], ids=["stream_k", "single_launch"])
def test_tc_sampled_threshold_integer_exact_all_rows(path):
    """A 4,096-token chunk at 65,536 tokens of context: every row has 15,360-16,383 candidates,
    so every row takes the sampled-threshold branch.  All rows bit-exact against the oracle, and
    each row's redo flag equals the model of the branch, which settles every row here: the
    checked selections are the tensor-core kernel's own."""
    run, w = run_positive_weights(SAMPLED, score_path=path)
    settled = check_rows(run, range(SAMPLED.num_q), True, w_bits=w, model=True)
    assert settled == SAMPLED.num_q
    assert run.runner.error_bits() == 0


def test_tc_sampled_threshold_generator_weights_exact():
    """The same chunk with the generator's weights in [-3, 3]: rows whose weights are all <= 0
    have mostly tied scores and are handed to the exact kernel; every row is still exact and
    every redo flag matches the model."""
    run = Run(SAMPLED, integer=True, score_path=1).step()
    rows = list(range(0, SAMPLED.num_q, 3)) + [SAMPLED.num_q - 1]
    settled = check_rows(run, rows, True, model=True)
    assert 0 < settled < len(rows)


KEEP_ALL_EDGE = Config("tc_keepall_chunk4096_ctx16384", "prefill", 1, 16384, 4096, 8, 2, 64, 4, 128,
                       shuffle_pages=True, seed=0x7C05)


@pytest.mark.parametrize("path", [1, 5], ids=["stream_k", "single_launch"])
def test_tc_keep_all_rows_on_both_sides_of_the_staging_limit(path):
    """Rows of 3,072-4,095 candidates keep every key.  The single-launch form's final select
    stages a row's keys in shared memory when they fit (3,456 keys) and reads them in place
    otherwise; the stream-K form stages every row.  Every row bit-exact and settled by the
    tensor-core kernels."""
    run, w = run_positive_weights(KEEP_ALL_EDGE, score_path=path)
    _, q_pos = host(KEEP_ALL_EDGE, True).rows()
    lim = q_pos // 4
    assert (lim <= 3456).any() and (lim > 3456).any()
    settled = check_rows(run, range(KEEP_ALL_EDGE.num_q), True, w_bits=w, model=True)
    assert settled == KEEP_ALL_EDGE.num_q
    assert run.runner.error_bits() == 0


def test_tc_c2_integer_sampled_rows():
    """The C2 chunk (16,384 tokens at 131,072) on integer inputs with positive weights: 256 rows
    across the chunk bit-exact, each settled by the tensor-core kernel, and no row of the chunk
    handed over."""
    c = CONFIGS["C2"]
    run, w = run_positive_weights(c)
    rows = sample_rows(c, 256)
    assert check_rows(run, rows, True, w_bits=w, model=True) == len(rows)
    assert not run.redo_flags().any()
    assert run.runner.error_bits() == 0


def test_tc_prefill_random_sampled_rows_and_attention():
    run = Run(TC_PREFILL, integer=False, score_path=1).step()
    rows = list(range(0, 8192, 97)) + [8191]
    o = check_rows(run, rows, False)
    h = host(run.c, False)
    _, q_pos = h.rows()
    for r in rows[::4]:
        t = int(q_pos[r])
        n = o["n_sel"][r]
        ref_o, ref_lse = orc.attend(h.q([r])[0], *h.kv(0, orc.expand(o["sel"][r][:n], t)))
        check_attention(o["out"][r], o["lse"][r], ref_o, ref_lse)


@pytest.mark.parametrize("path", [1, 5], ids=["stream_k", "single_launch"])
def test_tc_two_sequences_in_one_row_tile(path):
    c = Config("tc_ragged_b3", "prefill", 3, 4096, 100, 8, 2, 64, 4, 128, shuffle_pages=True, seed=0x7C02)
    run = Run(c, integer=True, score_path=path).step()
    check_rows(run, range(c.num_q), True)


def test_tc_small_budget_exact():
    run = Run(TC_PREFILL.replace(ctx=3000, n_new=3000), integer=True, score_path=1, topk=37).step()
    check_rows(run, range(0, 3000, 7), True, topk=37)


@pytest.mark.parametrize("ctx,n_new", [(4096, 4096), (32768, 2048)], ids=["short_rows", "sampled_rows"])
def test_tc_fallback_on_decreasing_scores(ctx, n_new):
    """Scores that fall with the block index: rows of up to 4,096 candidates keep every key and
    need no fallback; longer rows defeat the sampled threshold (the sample's best blocks are the
    first ones) and go to the exact fallback.  Both must be exact."""
    c = TC_PREFILL.replace(ctx=ctx, n_new=n_new)
    run = Run(c, integer=True, score_path=1)
    nb = c.ctx // 4
    vals = np.zeros((c.ctx, c.Di), dtype=np.float32)
    blk = np.arange(c.ctx) // 4
    vals[:, 0] = (nb - blk) // 256
    vals[:, 1] = (nb - blk) % 256
    kbits = torch.tensor(vals).to(torch.bfloat16)
    run.di.idx_k[0] = kbits.cuda()
    run.di.idx_k_new.copy_(run.di.idx_k[0, c.ctx_start:])
    if c.ctx_start > 0:  # the prefix's compressed keys, from the keys planted above
        run.di.kcomp_pool.zero_()
        run.setup_prefix()
    q = np.zeros((c.num_q, 4, c.Di), dtype=np.float32)
    q[:, :, 0] = 256
    q[:, :, 1] = 1
    run.di.idx_q.copy_(torch.tensor(q).to(torch.bfloat16).cuda())
    run.di.idx_w.fill_(1.0)
    run.step()
    o = run.numpy()
    kc = orc.compress(kbits.view(torch.int16).numpy().view(np.uint16))
    qb = torch.tensor(q[0]).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    wb = torch.ones(4).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    _, q_pos = host(c, True).rows()
    redo = run.redo_flags()
    for r in list(range(0, c.num_q, 11)) + [c.num_q - 1]:
        t = int(q_pos[r])
        ref_sel, ref_s = orc.qsa_select(kc, qb, wb, t, c.topk)
        check_selection(o["sel"][r], o["n_sel"][r], o["sel_scores"][r], ref_sel, ref_s, t, c.topk, True)
        if t // 4 > 512:
            assert list(ref_sel[:-1]) == list(range(512))  # the earliest blocks win
        assert bool(redo[r]) == (t // 4 > 4096)  # only the sampled branch is defeated


@pytest.mark.parametrize("path", [1, 5], ids=["stream_k", "single_launch"])
def test_tc_decode_shaped_tile_with_four_sequences(path):
    """4 sequences x 4 positions share one 128-row tile: four segments processed in turn."""
    c = Config("tc_decode_b4x4", "decode", 4, 8192, 4, 8, 2, 64, 4, 128, shuffle_pages=True, seed=0x7C03)
    run = Run(c, integer=True, score_path=path).step()
    check_rows(run, range(c.num_q), True)


def test_tc_stream_k_equals_single_launch_c2_random():
    """The C2 chunk on random inputs: the stream-K form and the single-launch form select the
    same blocks with the same scores on every row."""
    c = CONFIGS["C2"]
    a = Run(c, integer=False, score_path=1).step()
    sel1, n1, sc1 = a.sel.cpu(), a.n_sel.cpu(), a.sel_scores.cpu().numpy()
    r1 = a.redo_flags()
    b = Run(c, integer=False, score_path=5).step()
    assert torch.equal(n1, b.n_sel.cpu()) and torch.equal(sel1, b.sel.cpu())
    assert np.array_equal(np.nan_to_num(sc1, nan=-1.0), np.nan_to_num(b.sel_scores.cpu().numpy(), nan=-1.0))
    assert not r1.any() and not b.redo_flags().any()
