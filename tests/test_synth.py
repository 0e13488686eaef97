"""CPU checks of the seeded input generator (qsa_synth): determinism, distribution shape, page
tables and the planted needles."""
import numpy as np

import qsa_synth as qs


def test_generator_is_deterministic_and_streams_differ():
    a = qs.values_bf16(7, 1, np.arange(1000), qs.NORMAL)
    b = qs.values_bf16(7, 1, np.arange(1000), qs.NORMAL)
    c = qs.values_bf16(7, 2, np.arange(1000), qs.NORMAL)
    d = qs.values_bf16(8, 1, np.arange(1000), qs.NORMAL)
    assert np.array_equal(a, b) and not np.array_equal(a, c) and not np.array_equal(a, d)
    # element-wise addressing: any subset regenerates the same bits
    idx = np.array([999, 3, 500])
    assert np.array_equal(qs.values_bf16(7, 1, idx, qs.NORMAL), a[idx])


def test_splitmix64_reference_values():
    # SplitMix64 seeded with 0: first outputs as published with the reference implementation
    with np.errstate(over="ignore"):
        st = np.array([0], dtype=np.uint64)
        outs = [int(qs._mix(st + np.uint64(i + 1) * qs.GAMMA)[0]) for i in range(3)]
    assert outs == [0xE220A8397B1DCDAF, 0x6E789E6AA1B965F4, 0x06C45D188009454F]


def test_distributions():
    n = 400000
    x = qs.values_f32(1, 1, np.arange(n), qs.NORMAL).astype(np.float64)
    assert abs(x.mean()) < 0.01 and abs(x.var() - 1) < 0.01 and np.abs(x).max() <= 3.47
    u = qs.values_f32(1, 2, np.arange(n), qs.UNIFORM).astype(np.float64)
    assert u.min() >= 0 and u.max() <= 1 and abs(u.mean() - 0.5) < 0.01
    i = qs.values_f32(1, 3, np.arange(n), qs.INT3)
    assert set(np.unique(i).tolist()) == {-3, -2, -1, 0, 1, 2, 3}
    assert np.all(np.abs(np.bincount((i + 3).astype(int)) / n - 1 / 7) < 0.01)


def test_page_table_is_a_permutation():
    c = qs.CONFIGS["C3"]
    h = qs.HostInputs(c)
    pt = h.page_table()
    assert pt.shape == (4, 4096)
    assert np.array_equal(np.sort(pt.reshape(-1)), np.arange(c.num_pages))
    assert not np.array_equal(pt.reshape(-1), np.arange(c.num_pages))
    owner = h.page_owner()
    assert np.array_equal(owner[pt.reshape(-1)], np.arange(c.num_pages))


def test_needles_have_cosine_point_eight():
    c = qs.CONFIGS["C3"]
    h = qs.HostInputs(c)
    nd = h.needles()
    assert len(nd["blocks"]) == 4 and all(len(set(b.tolist())) == 64 for b in nd["blocks"])
    assert all(b.max() < c.ctx // 4 - 1 for b in nd["blocks"])
    assert len(nd["q_rows"]) >= 1
    q_seq, _ = h.rows()
    for r, j in nd["q_rows"].items():
        u = nd["dirs"][q_seq[r], j]
        qv = qs.bf16_bits_to_f32(nd["q_vals"][r]).astype(np.float64)
        cos = qv @ u / np.linalg.norm(qv, axis=1)
        assert np.allclose(cos, 0.8, atol=0.01)
    # the needle block's 4 raw keys are identical, so its compressed key equals them
    s = 0
    blk = int(nd["blocks"][s][0])
    rows = h.idx_k(s, 4 * blk, 4 * blk + 4)
    assert np.all(rows == rows[0]) and np.array_equal(rows[0], nd["key_rows"][s][0])


def test_host_fill_equals_numpy_generator():
    """The C++ host fill of libqsa_synth.so returns the numpy generator's bits, for every
    distribution and for rows starting at arbitrary indices."""
    if qs._host_lib() is None:
        import pytest

        pytest.skip("libqsa_synth.so not built")
    rng = np.random.default_rng(5)
    starts = rng.integers(0, 1 << 40, 300)
    for dist in (qs.NORMAL, qs.UNIFORM, qs.INT3):
        got = qs.rows_bf16(11, 4, starts, 129, dist)
        idx = starts[:, None] + np.arange(129)[None, :]
        assert np.array_equal(got, qs.values_bf16(11, 4, idx.reshape(-1), dist).reshape(300, 129))
