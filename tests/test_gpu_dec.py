"""GPU parity of the split-list indexer path (score_path 3, decode-sized batches): exact on integer
inputs, row tiles shared by several sequences, short contexts, small budgets, and the exact
fallback for rows whose best blocks crowd into one chunk."""
import numpy as np
import pytest

from oracle import qsa_oracle as orc
from qsa_synth import CONFIGS, Config
from tests.qsa_testlib import Run, check_attention, check_selection, host, host_kcomp, score_bound

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

# 5 sequences x 3 positions = 15 rows: 4-row tiles hold rows of two sequences.  The 3 new tokens
# of a sequence do not fill a block (and their block is only ever the tail), so steps on this
# workload skip the compress call.
RAGGED = Config("dec_b5x3_ctx65536", "decode", 5, 65536, 3, 32, 4, 128, 4, 128, needles=8,
                shuffle_pages=True, seed=0xDEC1)


def check_rows(run, rows, integer, topk=None):
    o = run.numpy()
    c = run.c
    topk = c.topk if topk is None else topk
    h = host(c, integer)
    q_seq, q_pos = h.rows()
    for r in rows:
        s, t = int(q_seq[r]), int(q_pos[r])
        kc = host_kcomp(c, integer, s)
        iq, iw = h.idx_q([r])[0], h.idx_w([r])[0]
        ref_sel, ref_s = orc.qsa_select(kc, iq, iw, t, topk)
        check_selection(o["sel"][r], o["n_sel"][r], o["sel_scores"][r], ref_sel, ref_s, t, topk,
                        integer, score_bound(kc, iq, iw, t // 4))
    return o


@pytest.mark.parametrize("integer", [True, False], ids=["int", "random"])
def test_split_lists_c3_all_rows(integer):
    run = Run(CONFIGS["C3"], integer=integer, score_path=3).step()
    o = check_rows(run, range(run.c.num_q), integer)
    assert run.runner.error_bits() == 0
    if integer:  # same exact answer as the materialised path
        m = Run(CONFIGS["C3"], integer=True, score_path=2).step().numpy()
        assert np.array_equal(o["sel"], m["sel"]) and np.array_equal(o["n_sel"], m["n_sel"])


@pytest.mark.parametrize("integer", [True, False], ids=["int", "random"])
def test_split_lists_tiles_shared_by_sequences(integer):
    run = Run(RAGGED, integer=integer, score_path=3).step(compress=False)
    o = check_rows(run, range(RAGGED.num_q), integer)
    h = host(RAGGED, integer)
    for r in (0, 3, 7, 14):
        t = int(h.rows()[1][r])
        n = o["n_sel"][r]
        ref_o, ref_lse = orc.attend(h.q([r])[0], *h.kv(int(h.rows()[0][r]), orc.expand(o["sel"][r][:n], t)))
        check_attention(o["out"][r], o["lse"][r], ref_o, ref_lse)
    assert run.runner.error_bits() == 0


@pytest.mark.parametrize("ctx,topk", [(1000, 512), (3000, 512), (65536, 37), (65536, 1)])
def test_split_lists_short_contexts_and_small_budgets(ctx, topk):
    c = RAGGED.replace(ctx=ctx, needles=0)
    run = Run(c, integer=True, score_path=3, topk=topk).step(compress=False)
    check_rows(run, range(c.num_q), True, topk=topk)


def test_split_lists_fallback_on_crowded_chunk():
    """Scores that fall with the block index put the whole top 512 into the first chunks, so the
    lists drop keys that beat the merged threshold; the rows must go to the exact fallback."""
    c = Config("dec_b4x4_ctx65536_decreasing", "decode", 4, 65536, 4, 32, 4, 128, 4, 128, seed=0xDEC2)
    run = Run(c, integer=True, score_path=3)
    nb = c.ctx // 4
    blk = np.arange(c.ctx) // 4
    vals = np.zeros((c.ctx, c.Di), dtype=np.float32)
    vals[:, 0] = (nb - blk) // 256
    vals[:, 1] = (nb - blk) % 256
    kbits = torch.tensor(vals).to(torch.bfloat16)
    for s in range(c.batch):
        run.di.idx_k[s] = kbits.cuda()
    run.di.idx_k_new.copy_(torch.cat([run.di.idx_k[s, c.ctx_start:] for s in range(c.batch)]))
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
    for r in range(c.num_q):
        t = int(q_pos[r])
        ref_sel, ref_s = orc.qsa_select(kc, qb, wb, t, c.topk)
        check_selection(o["sel"][r], o["n_sel"][r], o["sel_scores"][r], ref_sel, ref_s, t, c.topk, True)
        assert list(ref_sel[:-1]) == list(range(512))
    assert run.runner.error_bits() == 0


def test_split_lists_invalid_position_row():
    """A row whose position lies beyond max_pos gets an empty selection and a device flag."""
    import learned_block_sparse_qsa_b200 as q

    run = Run(CONFIGS["C3"], integer=True, score_path=3)
    run.di.q_pos[5] = run.c.ctx + 100
    run.runner.clear_error()
    run.step(compress=False)
    o = run.numpy()
    assert o["n_sel"][5] == 0 and np.all(o["sel"][5] == -1)
    assert run.runner.error_bits() & q.DEVERR["POS"]
    ok = [r for r in range(run.c.num_q) if r != 5]
    check_rows(run, ok[::5], True)


def test_split_lists_many_rows_warp_lists():
    """64 rows (16 sequences x 4 positions): fewer chunks per tile, so the merge takes the warps'
    16-key lists directly (no CTA-level fold), and those lists drop keys."""
    c = Config("dec_b16x4_ctx65536", "decode", 16, 65536, 4, 32, 4, 128, 4, 128, needles=4,
               shuffle_pages=True, seed=0xDEC3)
    run = Run(c, integer=True, score_path=3).step()
    check_rows(run, range(c.num_q), True)
    assert run.runner.error_bits() == 0


@pytest.mark.parametrize("positions", [1, 2, 8])
def test_multi_token_decode_widths(positions):
    """1 to 8 query positions per sequence (multi-token-prediction verify widths): row tiles of
    four hold one sequence's rows, parts of two sequences, or one sequence over two tiles."""
    c = Config(f"dec_b3x{positions}_ctx65536", "decode", 3, 65536, positions, 32, 4, 128, 4, 128,
               needles=4, shuffle_pages=True, seed=0xDEC4 + positions)
    run = Run(c, integer=True, score_path=3).step(compress=positions % 4 == 0)
    o = check_rows(run, range(c.num_q), True)
    h = host(c, True)
    q_seq, q_pos = h.rows()
    for r in sorted({0, c.num_q - 1}):
        t, n = int(q_pos[r]), o["n_sel"][r]
        ref_o, ref_lse = orc.attend(h.q([r])[0], *h.kv(int(q_seq[r]), orc.expand(o["sel"][r][:n], t)))
        check_attention(o["out"][r], o["lse"][r], ref_o, ref_lse)
    assert run.runner.error_bits() == 0
