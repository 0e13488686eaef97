"""qsa_sparse_attn_decode_noalloc -- the decode attention for callers that cannot allocate device
memory at step time (its split-K scratch is a fixed array owned by the library) -- must give the
same output as qsa_sparse_attn_decode with a caller workspace, on two calls in a row.

Kept in its own file, collected last, so that a failure here leaves every other test already run;
it passes alone in a fresh process too (the library looks its scratch address up on first use)."""
import numpy as np
import pytest

from qsa_synth import Config
from tests.qsa_testlib import ATTN_ATOL, ATTN_RTOL, Run

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)


@pytest.mark.parametrize("splits", [0, 5])
def test_noalloc_decode_matches_workspace_form_twice(splits):
    import learned_block_sparse_qsa_b200 as q

    c = Config("noalloc_decode_b4x4", "decode", 4, 16384, 4, 32, 4, 128, 4, 128, needles=8,
               shuffle_pages=True, seed=0x0A11)
    run = Run(c, integer=False).step(splits=splits)  # selection + reference output (workspace form)
    ref = run.out.float().clone()
    ref_lse = run.lse.clone()
    d = run.di
    for _ in range(2):
        out = torch.full_like(run.out, float("nan"))
        lse = torch.full_like(run.lse, float("nan"))
        q.qsa_sparse_attn_decode_noalloc(run.cfg, run.b, d.q, d.k_pool, d.v_pool, run.sel, run.n_sel,
                                         out, lse, splits)
        torch.cuda.synchronize()
        assert torch.allclose(out.float(), ref, atol=ATTN_ATOL, rtol=ATTN_RTOL)
        assert torch.allclose(lse, ref_lse, atol=ATTN_ATOL, rtol=ATTN_RTOL)
    assert run.runner.error_bits() == 0


def test_noalloc_rejects_split_count_beyond_scratch():
    import learned_block_sparse_qsa_b200 as q

    c = Config("noalloc_many_rows", "decode", 64, 4096, 4, 32, 4, 128, 4, 128, seed=0x0A12)
    run = Run(c, integer=False).step()
    d = run.di
    # 256 rows x 64 splits x 32 heads x 129 floats = 270 MB of partials: far beyond 4 MiB
    with pytest.raises(q.QsaError) as e:
        q.qsa_sparse_attn_decode_noalloc(run.cfg, run.b, d.q, d.k_pool, d.v_pool, run.sel, run.n_sel,
                                         run.out, None, 64)
    assert e.value.status == q.QSA_ERR_WORKSPACE


def test_noalloc_auto_split_count_lowered_to_fit():
    """128 query heads of dim 128 (16 per KV head): the automatic split count of the workspace
    form would need more than the 4 MiB of library scratch, so the allocation-free form lowers it
    to the largest count that fits.  Its output must equal the workspace form run at that count
    (same kernels, same split: bit for bit), twice in a row."""
    import learned_block_sparse_qsa_b200 as q

    c = Config("noalloc_g16", "decode", 1, 8192, 4, 128, 8, 128, 4, 128, shuffle_pages=True,
               seed=0x0A13)
    run = Run(c, integer=False).step(splits=1)
    auto = q.qsa_workspace_size(run.cfg, run.b, q.QSA_OP_SPARSE_ATTN_DECODE, 0)
    assert auto > 4 << 20  # the automatic count does not fit: the lowering loop runs
    fit = max(s for s in range(1, 65)
              if q.qsa_workspace_size(run.cfg, run.b, q.QSA_OP_SPARSE_ATTN_DECODE, s) <= 4 << 20)
    assert fit > 1
    d = run.di
    ref = torch.empty_like(run.out)
    ref_lse = torch.empty_like(run.lse)
    ws, n = run.runner.workspace(run.b, q.QSA_OP_SPARSE_ATTN_DECODE, fit)
    q.qsa_sparse_attn_decode(run.cfg, run.b, d.q, d.k_pool, d.v_pool, run.sel, run.n_sel, ref,
                             ref_lse, fit, ws, n)
    for _ in range(2):
        out = torch.full_like(run.out, float("nan"))
        lse = torch.full_like(run.lse, float("nan"))
        q.qsa_sparse_attn_decode_noalloc(run.cfg, run.b, d.q, d.k_pool, d.v_pool, run.sel,
                                         run.n_sel, out, lse, 0)
        torch.cuda.synchronize()
        assert torch.equal(out.view(torch.int16), ref.view(torch.int16))
        assert torch.equal(lse, ref_lse)
    assert torch.allclose(run.out.float(), ref.float(), atol=ATTN_ATOL, rtol=ATTN_RTOL)
    assert run.runner.error_bits() == 0
