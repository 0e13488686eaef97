"""Failure detection without a GPU fault: a bounded wait that runs out reports QSA_DEVERR_TIMEOUT
through the caller's error flag, the kernel returns, and the context stays usable."""
import pytest

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)


def test_bounded_wait_reports_timeout_and_context_survives():
    import learned_block_sparse_qsa_b200 as q
    from qsa_synth import CONFIGS
    from tests.qsa_testlib import Run

    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    q.qsa_selftest_wait_timeout(err, 2_000_000)  # about a millisecond of waiting
    torch.cuda.synchronize()
    assert int(err.item()) == q.DEVERR["TIMEOUT"]
    # the same context still runs the layer, exactly
    run = Run(CONFIGS["C1"].replace(ctx=1024, n_new=1024), integer=True).step()
    assert run.runner.error_bits() == 0
    o = run.numpy()
    assert (o["n_sel"] == [min(512, t // 4) + 1 for t in range(1024)]).all()
