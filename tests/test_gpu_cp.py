"""GPU test of the context-parallel step on one device: the context split into R shards, each
"rank" run in turn with its own local page table over the same pools, the collectives replaced by
stacking the ranks' tensors.  The global selection must equal the single-GPU selection exactly
(integer inputs: exact fp32 scores), and the merged output must match the single-GPU output within
the attention tolerance.  Shards after a row's position, before it and containing it all occur."""
import numpy as np
import pytest

from qsa_synth import Config
from tests.qsa_testlib import ATTN_ATOL, ATTN_RTOL, Run, host, positive_int_weights

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)


def emulate(run: Run, nshards: int, decode: bool):
    from learned_block_sparse_qsa_b200.context_parallel import ContextParallelStep, Shard

    c, d = run.c, run.di
    L = c.ctx // nshards
    assert L % 64 == 0
    shards = [Shard(i * L, L) for i in range(nshards)]
    pt = d.page_table
    ranks = []
    for r in range(nshards):
        lpt = torch.cat([pt[:, r * L // 64:(r + 1) * L // 64], pt[:, :1]], dim=1).contiguous()
        cp = ContextParallelStep(run.cfg, shards, r)
        sel, sc = cp.select_local(batch=c.batch, q_seq=d.q_seq, q_pos=d.q_pos, local_page_table=lpt,
                                  num_pages=c.num_pages, idx_q=d.idx_q, idx_w=d.idx_w,
                                  kcomp_pool=d.kcomp_pool)
        ranks.append((cp, sel, sc))
    part_sel = torch.stack([s for _, s, _ in ranks])
    part_sc = torch.stack([x for _, _, x in ranks])
    parts = [cp.merge_and_attend(part_sel, part_sc, max_pos=c.ctx - 1, q=d.q, k_pool=d.k_pool,
                                 v_pool=d.v_pool, decode=decode) for cp, _, _ in ranks]
    out = torch.empty_like(d.q)
    lse = torch.empty(c.num_q, c.Hq, dtype=torch.float32, device="cuda")
    ranks[0][0].combine(torch.stack([o for o, _ in parts]), torch.stack([l for _, l in parts]), out, lse)
    torch.cuda.synchronize()
    for cp, _, _ in ranks:
        assert cp.ops.error_bits() == 0
    return [cp for cp, _, _ in ranks], out, lse


def positive(run: Run):
    c = run.c
    w = positive_int_weights(host(c, True).idx_w(np.arange(c.num_q)))
    run.di.idx_w.copy_(torch.from_numpy(w.view(np.int16)).view(torch.bfloat16))


@pytest.mark.parametrize("name,cfg,nshards,decode", [
    ("prefill_full_16384_x4", Config("cp_full", "prefill", 1, 16384, 16384, 8, 2, 64, 4, 128,
                                     shuffle_pages=True, seed=0xC901), 4, False),
    ("prefill_chunk1024_ctx32768_x4", Config("cp_chunk", "prefill", 1, 32768, 1024, 8, 2, 64, 4, 128,
                                             shuffle_pages=True, seed=0xC902), 4, False),
    ("decode_b4x4_ctx65536_x8", Config("cp_dec", "decode", 4, 65536, 4, 32, 4, 128, 4, 128,
                                       shuffle_pages=True, seed=0xC903), 8, True),
])
def test_context_parallel_equals_single_gpu(name, cfg, nshards, decode):
    run = Run(cfg, integer=True)
    positive(run)
    run.step()
    ref = run.numpy()
    cps, out, lse = emulate(run, nshards, decode)
    for cp in cps:
        assert torch.equal(cp.n_sel.cpu(), run.n_sel.cpu())
        assert torch.equal(cp.sel.cpu(), run.sel.cpu())
        got_sc = cp.sel_scores.cpu().numpy()
        assert np.array_equal(np.nan_to_num(got_sc, nan=-7.0), np.nan_to_num(ref["sel_scores"], nan=-7.0))
    assert torch.allclose(out.float(), run.out.float(), atol=ATTN_ATOL, rtol=ATTN_RTOL)
    assert torch.allclose(lse, run.lse, atol=ATTN_ATOL, rtol=ATTN_RTOL)


def test_context_parallel_random_decode_output():
    cfg = Config("cp_dec_rand", "decode", 4, 65536, 4, 32, 4, 128, 4, 128, needles=16,
                 shuffle_pages=True, seed=0xC904)
    run = Run(cfg, integer=False).step()
    cps, out, lse = emulate(run, 8, True)
    same = (cps[0].sel.cpu() == run.sel.cpu()).all(dim=1)
    assert same.float().mean() >= 0.9   # fp32 ties aside, the selection is the single-GPU one
    rows = torch.nonzero(same).flatten()
    assert torch.allclose(out[rows].float(), run.out[rows].float(), atol=ATTN_ATOL, rtol=ATTN_RTOL)
