"""Prefill in chunks whose boundaries are not multiples of the 4-token block: each sequence's
unfinished block is carried to the next chunk (BlockCarry) and compressed once complete.  The
compressed keys must equal the oracle's compression of the whole context, bit for bit, and every
chunk's selections and attention must match the oracle."""
import numpy as np
import pytest

from oracle import qsa_oracle as orc
from qsa_synth import CONFIGS
from tests.qsa_testlib import (check_attention, check_selection, host, host_kcomp, qsa_config,
                               score_bound)

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

CHUNKS = [0, 1001, 1999, 2002, 3003, 4096]  # chunk boundaries of the 4,096-token prefill


@pytest.mark.parametrize("integer", [True, False], ids=["int", "random"])
def test_ragged_chunk_boundaries(integer):
    from learned_block_sparse_qsa_b200 import BlockCarry, QsaRunner
    from qsa_synth.device import DeviceInputs

    c = CONFIGS["C1"]
    d = DeviceInputs(c, integer)
    runner = QsaRunner(qsa_config(c))
    carry = BlockCarry()
    h = host(c, integer)
    kc_ref = host_kcomp(c, integer, 0)
    for c0, c1 in zip(CHUNKS[:-1], CHUNKS[1:]):
        n = c1 - c0
        b = runner.batch(batch=1, num_q=n, max_pages=c.max_pages, num_pages=c.num_pages,
                         max_pos=c1 - 1, q_seq=d.q_seq[c0:c1], q_pos=d.q_pos[c0:c1],
                         page_table=d.page_table)
        carry.compress_chunk(runner, b, 0, c0, d.idx_k[0, c0:c1], d.kcomp_pool)
        sel = torch.empty(n, c.topk + 1, dtype=torch.int32, device="cuda")
        n_sel = torch.empty(n, dtype=torch.int32, device="cuda")
        scores = torch.empty(n, c.topk + 1, dtype=torch.float32, device="cuda")
        out = torch.empty_like(d.q[c0:c1])
        lse = torch.empty(n, c.Hq, dtype=torch.float32, device="cuda")
        runner.prefill(b, q=d.q[c0:c1], idx_q=d.idx_q[c0:c1], idx_w=d.idx_w[c0:c1],
                       kcomp_pool=d.kcomp_pool, k_pool=d.k_pool, v_pool=d.v_pool, out=out,
                       sel=sel, n_sel=n_sel, lse=lse, sel_scores=scores)
        torch.cuda.synchronize()
        gs, gn, gsc = sel.cpu().numpy(), n_sel.cpu().numpy(), scores.cpu().numpy()
        go = out.view(torch.int16).cpu().numpy().view(np.uint16)
        gl = lse.cpu().numpy()
        rows = sorted({0, n - 1, *range(0, n, 37)})
        for i in rows:
            t = c0 + i
            iq, iw = h.idx_q([t])[0], h.idx_w([t])[0]
            ref_sel, ref_s = orc.qsa_select(kc_ref, iq, iw, t, c.topk)
            check_selection(gs[i], gn[i], gsc[i], ref_sel, ref_s, t, c.topk, integer,
                            score_bound(kc_ref, iq, iw, t // 4))
            if i % 3 == 0:
                ref_o, ref_lse = orc.attend(h.q([t])[0], *h.kv(0, orc.expand(gs[i][: gn[i]], t)))
                check_attention(go[i], gl[i], ref_o, ref_lse)
    # every block compressed once, when complete: equal to compressing the whole context
    pt = d.page_table[0].long()
    kc = d.kcomp_pool[pt].reshape(-1, c.Di)[: c.ctx // 4]
    assert np.array_equal(kc.view(torch.int16).cpu().numpy().view(np.uint16), kc_ref)
    assert runner.error_bits() == 0


# three sequences of different lengths, each cut at its own boundaries (most inside a block);
# every call carries one chunk of every sequence that still has tokens
RAGGED_LENS = [20001, 9002, 18003]
RAGGED_CUTS = [[0, 6001, 13002, 20001], [0, 3, 5001, 9002], [0, 8190, 16383, 18003]]


def test_ragged_batch_of_sequences_in_chunks():
    """A ragged batch through the block carry: per call, the next chunk of each of three
    sequences of different lengths, with the tensor-core indexer (Di = 128) on integer inputs
    with positive weights.  Rows past 16,388 tokens take the sampled-threshold branch.  The
    compressed keys of each sequence equal the oracle's whole-sequence compression bit for bit,
    and sampled rows of every call have exact selections and matching attention."""
    from learned_block_sparse_qsa_b200 import BlockCarry, QsaRunner
    from qsa_synth import Config
    from qsa_synth.device import DeviceInputs
    from tests.qsa_testlib import positive_int_weights

    ctx = 20480
    c = Config("ragged_b3_ctx20480", "prefill", 3, ctx, ctx, 8, 2, 64, 4, 128, shuffle_pages=True,
               seed=0x0C3A)
    d = DeviceInputs(c, True)
    h = host(c, True)
    w_all = positive_int_weights(h.idx_w(np.arange(c.num_q)))
    d.idx_w.copy_(torch.from_numpy(w_all.view(np.int16)).view(torch.bfloat16))
    runner = QsaRunner(qsa_config(c, score_path=1))
    carry = BlockCarry()
    checked = 0
    for k in range(3):
        pieces = [(s, cut[k], cut[k + 1]) for s, cut in enumerate(RAGGED_CUTS) if cut[k + 1] > cut[k]]
        rows = torch.cat([torch.arange(s * ctx + a, s * ctx + b) for s, a, b in pieces]).cuda()
        n = rows.numel()
        q_seq = d.q_seq[rows].contiguous()
        q_pos = d.q_pos[rows].contiguous()
        b = runner.batch(batch=c.batch, num_q=n, max_pages=c.max_pages, num_pages=c.num_pages,
                         max_pos=max(p1 for _, _, p1 in pieces) - 1, q_seq=q_seq, q_pos=q_pos,
                         page_table=d.page_table)
        for s, a, e in pieces:
            carry.compress_chunk(runner, b, s, a, d.idx_k[s, a:e], d.kcomp_pool)
        sel = torch.empty(n, c.topk + 1, dtype=torch.int32, device="cuda")
        n_sel = torch.empty(n, dtype=torch.int32, device="cuda")
        scores = torch.empty(n, c.topk + 1, dtype=torch.float32, device="cuda")
        out = torch.empty(n, c.Hq, c.D, dtype=torch.bfloat16, device="cuda")
        lse = torch.empty(n, c.Hq, dtype=torch.float32, device="cuda")
        runner.prefill(b, q=d.q[rows].contiguous(), idx_q=d.idx_q[rows].contiguous(),
                       idx_w=d.idx_w[rows].contiguous(), kcomp_pool=d.kcomp_pool, k_pool=d.k_pool,
                       v_pool=d.v_pool, out=out, sel=sel, n_sel=n_sel, lse=lse, sel_scores=scores)
        torch.cuda.synchronize()
        gs, gn, gsc = sel.cpu().numpy(), n_sel.cpu().numpy(), scores.cpu().numpy()
        go = out.view(torch.int16).cpu().numpy().view(np.uint16)
        gl = lse.cpu().numpy()
        grow = rows.cpu().numpy()
        for i in sorted({0, n - 1, *range(0, n, 41)}):
            r = int(grow[i])
            s, t = r // ctx, r % ctx
            kc = host_kcomp(c, True, s)
            iq, iw = h.idx_q([r])[0], w_all[r]
            ref_sel, ref_s = orc.qsa_select(kc, iq, iw, t, c.topk)
            check_selection(gs[i], gn[i], gsc[i], ref_sel, ref_s, t, c.topk, True)
            if i % 5 == 0:
                ref_o, ref_lse = orc.attend(h.q([r])[0], *h.kv(s, orc.expand(gs[i][: gn[i]], t)))
                check_attention(go[i], gl[i], ref_o, ref_lse)
            checked += 1
    assert checked > 1000
    for s, length in enumerate(RAGGED_LENS):
        pt = d.page_table[s].long()
        kc = d.kcomp_pool[pt].reshape(-1, c.Di)[: length // 4]
        want = host_kcomp(c, True, s)[: length // 4]
        assert np.array_equal(kc.view(torch.int16).cpu().numpy().view(np.uint16), want)
        # blocks past each sequence's length were never written
        rest = d.kcomp_pool[pt].reshape(-1, c.Di)[length // 4:]
        assert not rest.view(torch.int16).any()
    assert runner.error_bits() == 0
