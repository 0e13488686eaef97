"""GPU parity of the dense paged-GQA baseline's prefill form on the tensor cores (head_dim 128)
against the oracle's dense causal attention: rows sampled over the chunk, query-head groups of 1,
4, 8 and 16, ragged batches whose sequences share a row tile, and cache slots after a sequence's
last position that hold NaN (never written): the output must be the attention over positions
0..t alone."""
import numpy as np
import pytest

from qsa_synth import Config
from tests.qsa_testlib import Run, check_attention, oracle_dense_row, sample_rows

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

CASES = {
    "g8_chunk512_ctx8192": Config("dense_g8", "prefill", 1, 8192, 512, 32, 4, 128, 4, 128,
                                  shuffle_pages=True, seed=0xDE01),
    "g4_ragged_b3": Config("dense_g4_b3", "prefill", 3, 3000, 200, 16, 4, 128, 4, 128,
                           shuffle_pages=True, seed=0xDE02),
    "g16_chunk300_ctx4100": Config("dense_g16", "prefill", 1, 4100, 300, 32, 2, 128, 4, 128,
                                   shuffle_pages=True, seed=0xDE03),
    "g1_chunk256_ctx2000": Config("dense_g1", "prefill", 1, 2000, 256, 4, 4, 128, 4, 128, seed=0xDE04),
}


def plant_nan_after_last_position(run: Run):
    """Fill the unwritten slots of each sequence's last page (positions >= ctx) with NaN."""
    c, d = run.c, run.di
    pt = d.page_table.cpu().numpy()
    if c.ctx % 64 == 0:
        return 0
    for s in range(c.batch):
        p = int(pt[s, c.ctx // 64])
        d.k_pool[p, c.ctx % 64:] = float("nan")
        d.v_pool[p, c.ctx % 64:] = float("nan")
    return c.batch


@pytest.mark.parametrize("name", list(CASES))
def test_dense_tc_prefill_matches_oracle(name):
    c = CASES[name]
    run = Run(c, integer=False)
    planted = plant_nan_after_last_position(run)
    d = run.di
    out = torch.full_like(run.out, float("nan"))
    lse = torch.full_like(run.lse, float("nan"))
    run.runner.clear_error()
    run.runner.dense(run.b, q=d.q, k_pool=d.k_pool, v_pool=d.v_pool, out=out, lse=lse)
    torch.cuda.synchronize()
    assert run.runner.error_bits() == 0
    g = out.view(torch.int16).cpu().numpy().view(np.uint16)
    gl = lse.cpu().numpy()
    assert np.isfinite(gl).all() and np.isfinite(out.float().cpu().numpy()).all()
    rows = sample_rows(c, 40)
    if c.batch > 1:  # rows on both sides of every sequence boundary
        rows = sorted(set(rows) | {k * c.n_new + o for k in range(c.batch) for o in (-1, 0) if 0 <= k * c.n_new + o < c.num_q})
    for r in rows:
        ref_o, ref_lse = oracle_dense_row(c, False, r)
        check_attention(g[r], gl[r], ref_o, ref_lse)
    assert planted or c.ctx % 64 == 0


DECODE_CASES = {
    # 4 sequences x 4 positions; the context ends inside a 32-position tile and a page
    "g8_b4x4_ctx2531": Config("dense_dec_g8", "decode", 4, 2531, 4, 32, 4, 128, 4, 128,
                              shuffle_pages=True, seed=0xDE11),
    "g4_d64_b2x8_ctx1111": Config("dense_dec_g4", "decode", 2, 1111, 8, 16, 4, 64, 4, 64,
                                  shuffle_pages=True, seed=0xDE12),
}


@pytest.mark.parametrize("splits", [1, 3, 7, 0])
@pytest.mark.parametrize("name", list(DECODE_CASES))
def test_dense_decode_all_rows(name, splits):
    """The decode form (split-K over half-page tiles, merged by log-sum-exp) on every row and head
    against the oracle; splits 0 is the automatic count that fills the GPU; NaN in the unwritten
    slots after the last position must not reach the output."""
    c = DECODE_CASES[name]
    run = Run(c, integer=False)
    plant_nan_after_last_position(run)
    d = run.di
    out = torch.empty_like(run.out)
    lse = torch.empty_like(run.lse)
    run.runner.clear_error()
    run.runner.dense(run.b, q=d.q, k_pool=d.k_pool, v_pool=d.v_pool, out=out, lse=lse, decode=True,
                     splits=splits)
    torch.cuda.synchronize()
    assert run.runner.error_bits() == 0
    g = out.view(torch.int16).cpu().numpy().view(np.uint16)
    gl = lse.cpu().numpy()
    for r in range(c.num_q):
        ref_o, ref_lse = oracle_dense_row(c, False, r)
        check_attention(g[r], gl[r], ref_o, ref_lse)
