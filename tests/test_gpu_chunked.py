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
