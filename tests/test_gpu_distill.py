"""GPU parity of the indexer-distillation signal (qsa_index_distill_kl) against the fp64 oracle in
oracle/qsa_distill.py: per-row KL(teacher || indexer softmax), the teacher distribution and each
head's dense log-sum-exp, on rows spread over the context (including rows without candidates and
CTAs whose rows belong to two sequences), for several head layouts.

Tolerances, from the arithmetic: the kernel forms logits and indexer scores in fp32 from bf16
operands (relative error ~1e-6 of each dot product's magnitude) and exponentiates in fp32, so
teacher probabilities carry ~1e-5 relative error; the KL combines sums of magnitude up to the
largest score (~1e2 with planted needles), so 2e-3 absolute plus 2e-3 relative covers it."""
import numpy as np
import pytest

from oracle import qsa_distill as dst
from qsa_synth import CONFIGS, Config
from tests.qsa_testlib import Run, host, host_kcomp, sample_rows

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

KL_ATOL, KL_RTOL = 2e-3, 2e-3
P_ATOL, P_RTOL = 1e-6, 2e-3
LSE_ATOL, LSE_RTOL = 1e-3, 1e-4


def workspace(run):
    """The call's workspace (tensor-core form at head_dim 128 with 8 heads per KV head; none
    otherwise)."""
    from learned_block_sparse_qsa_b200 import QSA_OP_DISTILL_KL, qsa_workspace_size

    n = qsa_workspace_size(run.cfg, run.b, QSA_OP_DISTILL_KL)
    return (torch.empty(n, dtype=torch.uint8, device="cuda") if n else None), n


CASES = {
    "C1_4q1kv_d64_di32": CONFIGS["C1"],
    "b2_32q4kv_d128_di128": Config("distill_b2", "prefill", 2, 8192, 300, 32, 4, 128, 4, 128,
                                   needles=8, shuffle_pages=True, seed=0xD151),
    "g16_32q2kv_d64_di64": Config("distill_g16", "prefill", 1, 3000, 200, 32, 2, 64, 4, 64,
                                  shuffle_pages=True, seed=0xD152),
    "g1_8q8kv_d64_di128": Config("distill_g1", "prefill", 1, 2500, 152, 8, 8, 64, 4, 128,
                                 seed=0xD153),
}


@pytest.mark.parametrize("name", list(CASES))
def test_distill_kl_matches_oracle(name):
    from learned_block_sparse_qsa_b200 import qsa_index_distill_kl

    c = CASES[name]
    run = Run(c, integer=False).step()   # compresses the step's keys (and runs the layer)
    d = run.di
    ld = c.ctx // 4 + 1
    kl = torch.full((c.num_q,), float("nan"), dtype=torch.float32, device="cuda")
    lse = torch.full((c.num_q, c.Hq), float("nan"), dtype=torch.float32, device="cuda")
    teacher = torch.full((c.num_q, ld), float("nan"), dtype=torch.float32, device="cuda")
    ws, n = workspace(run)
    run.runner.clear_error()
    qsa_index_distill_kl(run.cfg, run.b, d.q, d.k_pool, d.idx_q, d.idx_w, d.kcomp_pool, kl, lse,
                         teacher, ld, ws, n)
    torch.cuda.synchronize()
    assert run.runner.error_bits() == 0
    g_kl, g_lse, g_p = kl.cpu().numpy(), lse.cpu().numpy(), teacher.cpu().numpy()
    assert np.all(np.isfinite(g_kl)) and np.all(g_kl >= -KL_ATOL)
    h = host(c, False)
    q_seq, q_pos = h.rows()
    rows = sorted(set(sample_rows(c, 24)) | {0, 1, 2, 3, 4, 5} & set(range(c.num_q)) |
                  ({c.n_new - 1, c.n_new} if c.batch > 1 else set()))
    for r in rows:
        s, t = int(q_seq[r]), int(q_pos[r])
        kc = host_kcomp(c, False, s)
        k, _ = h.kv(s, np.arange(t + 1))
        want_kl, want_p, _, want_lse = dst.distill_row(kc, h.idx_q([r])[0], h.idx_w([r])[0],
                                                       h.q([r])[0], k, t)
        assert abs(g_kl[r] - want_kl) <= KL_ATOL + KL_RTOL * abs(want_kl), (r, t, g_kl[r], want_kl)
        assert np.allclose(g_lse[r], want_lse, atol=LSE_ATOL, rtol=LSE_RTOL), r
        n = t // 4
        assert np.allclose(g_p[r, :n], want_p, atol=P_ATOL, rtol=P_RTOL), (r, t)
        if n:
            assert abs(g_p[r, :n].sum() - 1.0) < 1e-4
        assert np.all(np.isnan(g_p[r, n:]))   # entries b >= t/4 untouched


@pytest.mark.parametrize("base", ["C1", "d128_g8"])
def test_distill_invalid_rows_flagged_and_nan(base):
    from learned_block_sparse_qsa_b200 import qsa_index_distill_kl

    c = (CONFIGS["C1"] if base == "C1" else CASES["b2_32q4kv_d128_di128"]).replace(
        batch=1, ctx=512, n_new=512, needles=0)
    run = Run(c, integer=False).step()
    d = run.di
    run.di.q_pos[7] = 100000          # beyond the page table
    kl = torch.zeros(c.num_q, dtype=torch.float32, device="cuda")
    ws, n = workspace(run)
    run.runner.clear_error()
    qsa_index_distill_kl(run.cfg, run.b, d.q, d.k_pool, d.idx_q, d.idx_w, d.kcomp_pool, kl,
                         workspace=ws, ws_bytes=n)
    torch.cuda.synchronize()
    assert run.runner.error_bits() & 2
    g = kl.cpu().numpy()
    assert np.isnan(g[7]) and np.all(np.isfinite(np.delete(g, 7)))
