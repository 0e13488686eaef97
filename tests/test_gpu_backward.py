"""GPU parity of the sparse attention backward (qsa_sparse_attn_backward) against the fp64 oracle in
oracle/qsa_backward.py, run on the GPU's own selection: dq of every row, and dk / dv of every
position of the sequence (summed over all the rows that selected it).

Tolerance, from the arithmetic: like the forward's P, the kernel feeds P and dS to the tensor
cores in bf16 (relative rounding 2^-9 per element) and accumulates in fp32, so each gradient
element carries an error of a few 1e-3 of the largest term it sums; 2e-2 of the tensor's largest
magnitude plus 2e-2 relative covers it."""
import numpy as np
import pytest

from oracle import qsa_backward as bwd
from oracle import qsa_oracle as orc
from qsa_synth import CONFIGS, Config
from tests.qsa_testlib import Run, host

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

CASES = {
    "C1_4q1kv_d64": CONFIGS["C1"].replace(ctx=2048, n_new=2048),
    "32q4kv_d128_chunk256": Config("bwd_32q4kv", "prefill", 1, 8192, 256, 32, 4, 128, 4, 128,
                                   needles=8, shuffle_pages=True, seed=0xB0A1),
    "8q8kv_d64_b2": Config("bwd_8q8kv", "prefill", 2, 3000, 200, 8, 8, 64, 4, 64,
                           shuffle_pages=True, seed=0xB0A2),
}


def close(got, want, what):
    tol = 2e-2 * max(float(np.max(np.abs(want))), 1e-6) + 2e-2 * np.abs(want)
    err = np.abs(got - want)
    assert np.all(err <= tol), (what, float(err.max()), float(np.max(np.abs(want))))


@pytest.mark.parametrize("name", list(CASES))
def test_sparse_backward_matches_oracle(name):
    from learned_block_sparse_qsa_b200 import qsa_sparse_attn_backward

    c = CASES[name]
    run = Run(c, integer=False).step()
    d = run.di
    gen = torch.Generator().manual_seed(0xD0)
    dout = torch.randn(c.num_q, c.Hq, c.D, generator=gen).to(torch.bfloat16)
    dq = torch.full((c.num_q, c.Hq, c.D), float("nan"), dtype=torch.float32, device="cuda")
    dk = torch.zeros(c.num_pages, 64, c.Hkv, c.D, dtype=torch.float32, device="cuda")
    dv = torch.zeros_like(dk)
    run.runner.clear_error()
    qsa_sparse_attn_backward(run.cfg, run.b, d.q, d.k_pool, d.v_pool, run.sel, run.n_sel, run.out,
                             run.lse, dout.cuda(), dq, dk, dv)
    torch.cuda.synchronize()
    assert run.runner.error_bits() == 0
    o = run.numpy()
    h = host(c, False)
    q_seq, q_pos = h.rows()
    do = dout.float().numpy().astype(np.float64)
    g_dq = dq.cpu().numpy()
    pt = h.page_table()
    for s in range(c.batch):
        rows = np.nonzero(q_seq == s)[0]
        sels = [o["sel"][r][: o["n_sel"][r]] for r in rows]
        ts = [int(q_pos[r]) for r in rows]
        k_all, v_all = h.kv(s, np.arange(c.ctx))
        want_dq, want_dk, want_dv = bwd.sparse_backward_rows(h.q(rows), k_all, v_all, sels, ts, do[rows])
        close(g_dq[rows], want_dq, "dq")
        # the sequence's positions in the gradient pools, through its page table
        phys = pt[s, np.arange(c.ctx) // 64]
        slot = np.arange(c.ctx) % 64
        got_dk = dk[torch.from_numpy(phys).long(), torch.from_numpy(slot).long()].cpu().numpy()
        got_dv = dv[torch.from_numpy(phys).long(), torch.from_numpy(slot).long()].cpu().numpy()
        close(got_dk, want_dk, "dk")
        close(got_dv, want_dv, "dv")
        untouched = np.ones(c.ctx, dtype=bool)
        for sel, t in zip(sels, ts):
            untouched[orc.expand(sel, t)] = False
        assert not np.any(got_dk[untouched]) and not np.any(got_dv[untouched])


def test_backward_unsupported_group_size_is_rejected():
    from learned_block_sparse_qsa_b200 import QSA_ERR_UNSUPPORTED, QsaError, qsa_sparse_attn_backward

    c = Config("bwd_g16", "prefill", 1, 512, 64, 16, 1, 64, 4, 32, seed=0xB0A3)
    run = Run(c, integer=False).step()
    d = run.di
    dq = torch.empty(c.num_q, c.Hq, c.D, dtype=torch.float32, device="cuda")
    dk = torch.zeros(c.num_pages, 64, c.Hkv, c.D, dtype=torch.float32, device="cuda")
    with pytest.raises(QsaError) as e:
        qsa_sparse_attn_backward(run.cfg, run.b, d.q, d.k_pool, d.v_pool, run.sel, run.n_sel,
                                 run.out, run.lse, run.out, dq, dk, dk)
    assert e.value.status == QSA_ERR_UNSUPPORTED
