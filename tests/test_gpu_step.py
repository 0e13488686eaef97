"""GPU parity of the fused one-launch decode step (qsa_decode_step): compress + select + split-K
attention in one cooperative kernel.  Its results must equal, bit for bit, the three separate
calls (qsa_index_compress, qsa_index_score_topk, qsa_sparse_attn_decode) -- the same arithmetic
in the same order -- and, through them, the oracle.  Covered: the C3 and C5 decode workloads,
multi-token-prediction widths 1, 2 and 8 (at width 8 a block compressed in the same launch is a
candidate of the step's later rows), rows whose best blocks crowd into one chunk (the exact path
inside the launch), an invalid row, and two calls in a row on one workspace (its synchronisation
words come back to zero)."""
import numpy as np
import pytest

from oracle import qsa_oracle as orc
from qsa_synth import CONFIGS, Config
from tests.qsa_testlib import Run, check_selection, host, host_kcomp, score_bound

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)


def fused(run: Run, ws=None, splits=0):
    from learned_block_sparse_qsa_b200 import QSA_OP_DECODE_STEP, qsa_decode_step, qsa_workspace_size

    c, d = run.c, run.di
    n = qsa_workspace_size(run.cfg, run.b, QSA_OP_DECODE_STEP, splits)
    if ws is None:
        ws = torch.zeros(n, dtype=torch.uint8, device="cuda")
    sel = torch.full_like(run.sel, -7)
    n_sel = torch.full_like(run.n_sel, -7)
    sc = torch.full_like(run.sel_scores, 7.0)
    out = torch.full_like(run.out, float("nan"))
    lse = torch.full_like(run.lse, float("nan"))
    n_new = d.new_seq.numel() if c.n_new % 4 == 0 else 0
    qsa_decode_step(run.cfg, run.b, d.idx_k_new, d.new_seq, d.new_pos, n_new, d.kcomp_pool, d.idx_q,
                    d.idx_w, d.q, d.k_pool, d.v_pool, sel, n_sel, sc, out, lse, splits, ws, n)
    torch.cuda.synchronize()
    return dict(sel=sel.cpu(), n_sel=n_sel.cpu(), sc=sc.cpu(), out=out.view(torch.int16).cpu(),
                lse=lse.cpu()), ws


def same(a, run: Run, rows=None):
    rows = slice(None) if rows is None else rows
    assert torch.equal(a["n_sel"][rows], run.n_sel.cpu()[rows])
    assert torch.equal(a["sel"][rows], run.sel.cpu()[rows])
    assert np.array_equal(np.nan_to_num(a["sc"].numpy()[rows], nan=-1.0),
                          np.nan_to_num(run.sel_scores.cpu().numpy()[rows], nan=-1.0))
    assert torch.equal(a["out"][rows], run.out.view(torch.int16).cpu()[rows])
    assert torch.equal(a["lse"][rows], run.lse.cpu()[rows])


def kcomp_of_new_blocks(run: Run):
    c, d = run.c, run.di
    pt = d.page_table.long()
    got, want = [], []
    for s in range(c.batch):
        for b in range(c.ctx_start // 4, c.ctx // 4):
            got.append(d.kcomp_pool[pt[s, b // 16], b % 16].view(torch.int16).cpu().numpy().view(np.uint16))
            want.append(host_kcomp(c, run.di.host.integer, s)[b])
    return np.array(got), np.array(want)


@pytest.mark.parametrize("integer", [True, False], ids=["int", "random"])
def test_fused_step_equals_three_calls_c3(integer):
    run = Run(CONFIGS["C3"], integer=integer)
    a, ws = fused(run)                       # compresses the step's new blocks itself
    got, want = kcomp_of_new_blocks(run)
    assert np.array_equal(got, want)
    run.step()                               # the three calls on the same inputs
    same(a, run)
    b, _ = fused(run, ws)                    # the workspace's sync words came back to zero
    same(b, run)
    assert run.runner.error_bits() == 0


@pytest.mark.parametrize("positions", [1, 2, 8])
def test_fused_step_multi_token_widths(positions):
    c = Config(f"step_b3x{positions}_ctx65536", "decode", 3, 65536, positions, 32, 4, 128, 4, 128,
               needles=4, shuffle_pages=True, seed=0x57E0 + positions)
    run = Run(c, integer=True)
    a, _ = fused(run)
    run.step(compress=positions % 4 == 0)
    same(a, run)
    h = host(c, True)
    q_seq, q_pos = h.rows()
    for r in range(c.num_q):
        s, t = int(q_seq[r]), int(q_pos[r])
        kc = host_kcomp(c, True, s)
        iq, iw = h.idx_q([r])[0], h.idx_w([r])[0]
        ref_sel, ref_s = orc.qsa_select(kc, iq, iw, t, c.topk)
        check_selection(a["sel"][r].numpy(), int(a["n_sel"][r]), a["sc"][r].numpy(), ref_sel, ref_s, t,
                        c.topk, True, score_bound(kc, iq, iw, t // 4))
    assert run.runner.error_bits() == 0


def test_fused_step_exact_path_on_crowded_chunks():
    """Scores falling with the block index put the whole top 512 into the first chunks: the
    lists cannot settle these rows and the launch selects them on its exact path."""
    c = Config("step_b4x4_ctx65536_decreasing", "decode", 4, 65536, 4, 32, 4, 128, 4, 128, seed=0x57E9)
    run = Run(c, integer=True)
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
    a, _ = fused(run)
    kc = orc.compress(kbits.view(torch.int16).numpy().view(np.uint16))
    qb = torch.tensor(q[0]).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    wb = torch.ones(4).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    _, q_pos = host(c, True).rows()
    for r in range(c.num_q):
        t = int(q_pos[r])
        ref_sel, ref_s = orc.qsa_select(kc, qb, wb, t, c.topk)
        check_selection(a["sel"][r].numpy(), int(a["n_sel"][r]), a["sc"][r].numpy(), ref_sel, ref_s, t,
                        c.topk, True)
        assert list(ref_sel[:-1]) == list(range(512))
    run.step()
    same(a, run)                            # attention over the exact selection, too
    assert run.runner.error_bits() == 0


def test_fused_step_invalid_row():
    import learned_block_sparse_qsa_b200 as q

    run = Run(CONFIGS["C3"], integer=True)
    run.di.q_pos[5] = run.c.ctx + 100
    run.runner.clear_error()
    a, _ = fused(run)
    assert int(a["n_sel"][5]) == 0 and bool((a["sel"][5] == -1).all())
    assert run.runner.error_bits() & q.DEVERR["POS"]
    run.runner.clear_error()
    run.step()
    ok = [r for r in range(run.c.num_q) if r != 5]
    same(a, run, ok)


def test_fused_step_c5_full_size():
    run = Run(CONFIGS["C5"], integer=False)
    a, ws = fused(run)
    run.step()
    same(a, run)
    b, _ = fused(run, ws)
    same(b, run)
    assert run.runner.error_bits() == 0
