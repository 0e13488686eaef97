"""A host model of the decode indexer's exact top-k by split lists, checked against the oracle's
selection on CPU.

The decode kernels keep, per chunk of consecutive blocks, the best 16 keys and a bound above
every key the chunk dropped. Groups of 8 chunks then fold into the best 32 keys and the larger
bound. The merge keeps the keys at or above the need-th largest kept key (tau) when no bound
exceeds tau, and otherwise hands the row to the exact path.

The property the kernels rely on is tested here on random, tied and adversarial score orders:
whenever the model keeps a row, its answer is the oracle's. A key is the fp32 score mapped onto
an order-preserving uint32 (with -0 folded onto +0) in the high word and 0xFFFFFFFF - block in
the low word, so that the lower block wins ties.
"""
import numpy as np
import pytest

from oracle import qsa_oracle as orc

LIST_KEYS, FOLD_KEYS, FOLD_GROUP = 16, 32, 8


def make_keys(scores32: np.ndarray) -> np.ndarray:
    bits = (scores32.astype(np.float32) + np.float32(0.0)).view(np.uint32).astype(np.uint64)
    neg = (bits >> np.uint64(31)) == 1
    ordered = np.where(neg, np.uint64(0xFFFFFFFF) - bits, bits | np.uint64(0x80000000))
    blocks = np.arange(scores32.shape[0], dtype=np.uint64)
    return (ordered << np.uint64(32)) | (np.uint64(0xFFFFFFFF) - blocks)


def chunk_lists(keys: np.ndarray, chunk_blocks: int, nchunks: int):
    """Per chunk (block range [c*chunk_blocks, (c+1)*chunk_blocks)): its best LIST_KEYS keys and
    the bound (its smallest kept key when it had more candidates than that, else 0)."""
    lists, bounds = [], []
    for c in range(nchunks):
        k = np.sort(keys[c * chunk_blocks:(c + 1) * chunk_blocks])[::-1]
        lists.append(k[:LIST_KEYS])
        bounds.append(int(k[LIST_KEYS - 1]) if k.shape[0] > LIST_KEYS else 0)
    return lists, bounds


def fold(lists, bounds):
    """Groups of FOLD_GROUP consecutive lists -> their best FOLD_KEYS keys; the bound is the
    largest member bound, raised to the group's smallest kept key when the fold dropped keys."""
    out_l, out_b = [], []
    for g in range(0, len(lists), FOLD_GROUP):
        k = np.sort(np.concatenate(lists[g:g + FOLD_GROUP]))[::-1]
        b = max(bounds[g:g + FOLD_GROUP])
        if k.shape[0] > FOLD_KEYS:
            b = max(b, int(k[FOLD_KEYS - 1]))
        out_l.append(k[:FOLD_KEYS])
        out_b.append(b)
    return out_l, out_b


def merge(lists, bounds, need: int):
    """The row's selection (ascending blocks) or None when the exact path must redo it."""
    keys = np.concatenate(lists) if lists else np.zeros(0, dtype=np.uint64)
    if keys.shape[0] < need:
        return None
    if need == 0:
        return np.zeros(0, dtype=np.int64)
    tau = int(np.sort(keys)[::-1][need - 1])
    if max(bounds, default=0) > tau:
        return None
    kept = keys[keys >= np.uint64(tau)]
    assert kept.shape[0] == need  # keys are unique
    return np.sort((np.uint64(0xFFFFFFFF) - (kept & np.uint64(0xFFFFFFFF))).astype(np.int64))


def model_select(scores32: np.ndarray, warps: int, topk: int = 512):
    """Warps split the row's pages evenly (16 blocks a page); lists fold in groups when there are
    at least 512 warps, as the kernels do."""
    n = scores32.shape[0]
    need = min(topk, n)
    pages = (n + 15) // 16
    chunk_pages = (pages + warps - 1) // warps
    lists, bounds = chunk_lists(make_keys(scores32), chunk_pages * 16, warps)
    if warps >= 512:
        lists, bounds = fold(lists, bounds)
    return merge(lists, bounds, need)


def oracle_select(scores32: np.ndarray, topk: int = 512) -> np.ndarray:
    n = scores32.shape[0]
    t = 4 * n  # a position whose candidates are exactly blocks 0..n-1
    return orc.select_blocks(scores32.astype(np.float64), t, topk)[:-1]


@pytest.mark.parametrize("warps", [128, 592])
@pytest.mark.parametrize("seed", range(3))
def test_random_scores_are_exact_and_need_no_redo(warps, seed):
    rng = np.random.default_rng(seed)
    s = rng.standard_normal(65536).astype(np.float32)
    got = model_select(s, warps)
    assert got is not None
    assert np.array_equal(got, oracle_select(s))


@pytest.mark.parametrize("warps", [128, 592])
def test_tied_integer_scores_break_ties_by_lower_block(warps):
    rng = np.random.default_rng(7)
    s = rng.integers(-3, 4, 65536).astype(np.float32)  # thousands of ties at the boundary
    got = model_select(s, warps)
    if got is not None:
        assert np.array_equal(got, oracle_select(s))


def test_signed_zeros_map_to_one_key_and_tie_by_block():
    z = np.array([0.0, -0.0, 1.0, -1.0], dtype=np.float32)
    k = make_keys(z) >> np.uint64(32)
    assert k[0] == k[1] and k[2] > k[0] > k[3]
    # zeros of both signs spread through random scores: a kept row still matches the oracle
    rng = np.random.default_rng(11)
    s = rng.standard_normal(65536).astype(np.float32)
    s[rng.integers(0, 65536, 3000)] = np.float32(0.0)
    s[rng.integers(0, 65536, 3000)] = np.float32(-0.0)
    got = model_select(s, 592)
    assert got is not None and np.array_equal(got, oracle_select(s))


def test_equal_scores_crowd_the_first_chunks_and_are_handed_over():
    """All-equal scores: the lower-block tie-break puts the whole top 512 into the first chunks,
    which keep only 16 keys each; the row must go to the exact path."""
    assert model_select(np.zeros(4096, dtype=np.float32), 128) is None
    assert np.array_equal(oracle_select(np.zeros(4096, dtype=np.float32)), np.arange(512))


def test_crowded_chunks_are_handed_to_the_exact_path():
    """Scores that fall with the block index put the whole top 512 into the first chunks: the
    lists drop keys above tau, and the model must refuse the row rather than answer wrongly."""
    s = (65536 - np.arange(65536)).astype(np.float32)
    assert model_select(s, 592) is None
    assert model_select(s, 128) is None


def mixed_case(seed: int):
    """Noise with planted clusters of high scores and plateaus of equal scores, on a random
    number of warps and budget."""
    rng = np.random.default_rng(100 + seed)
    n = int(rng.integers(600, 20000))
    s = rng.standard_normal(n).astype(np.float32)
    for _ in range(int(rng.integers(0, 6))):  # clusters of high scores in one region
        a = int(rng.integers(0, n))
        s[a:a + int(rng.integers(1, 400))] += np.float32(rng.uniform(2, 6))
    if rng.random() < 0.5:  # a plateau of equal scores
        a = int(rng.integers(0, n))
        s[a:a + 300] = np.float32(1.5)
    return s, int(rng.choice([8, 64, 128, 512, 592])), int(rng.choice([1, 37, 512]))


@pytest.mark.parametrize("seed", range(20))
def test_whenever_a_row_is_kept_the_answer_is_exact(seed):
    s, warps, topk = mixed_case(seed)
    got = model_select(s, warps, topk)
    if got is not None:
        assert np.array_equal(got, oracle_select(s, topk))


def test_mixed_cases_are_mostly_kept():
    """Guards the test above against passing by handing every row over."""
    kept = sum(model_select(*mixed_case(seed)) is not None for seed in range(20))
    assert kept >= 8


def test_short_rows_keep_every_candidate():
    s = np.random.default_rng(3).standard_normal(300).astype(np.float32)
    got = model_select(s, 128)
    assert got is not None and np.array_equal(got, np.arange(300))


# --------------------------------------------------------------------------------------------
# The prefill indexer's sampled threshold.  The tile sequence is first every 32nd tile of 128
# blocks (the sample), then all tiles.  Each half-row (blocks 64h..64h+63 of every tile) keeps its
# 24 best sampled scores.  The row threshold is the smaller of the two halves' 24th best (minus
# infinity when the row has no more candidates than the budget or than the two half-row buffers
# hold, or when a half sampled fewer than 24).
# Every key at or above it is kept, and the exact select runs over the kept keys.  The row is
# handed to the exact path when fewer than need keys were kept, or a half-row kept more than its
# 2,048 slots.

TILE, SAMPLE_EVERY, SAMPLE_KEEP, HALF_CAP = 128, 32, 24, 2048


def sampled_select(scores32: np.ndarray, topk: int = 512):
    n = scores32.shape[0]
    need = min(topk, n)
    keys = make_keys(scores32)
    blocks = np.arange(n)
    half = (blocks % TILE) // (TILE // 2)
    sampled = (blocks // TILE) % SAMPLE_EVERY == 0
    if n <= topk or n <= 2 * HALF_CAP:
        tau_key = np.uint64(0)
    else:
        taus = []
        for h in (0, 1):
            s = np.sort(keys[sampled & (half == h)])[::-1]
            taus.append(int(s[SAMPLE_KEEP - 1]) >> 32 if s.shape[0] >= SAMPLE_KEEP else 0)
        tau_key = np.uint64(min(taus) << 32)  # a score threshold: every block at that score
    kept = keys[keys >= tau_key]
    if kept.shape[0] < need or any(np.sum((keys >= tau_key) & (half == h)) > HALF_CAP for h in (0, 1)):
        return None
    top = np.sort(kept)[::-1][:need]
    return np.sort((np.uint64(0xFFFFFFFF) - (top & np.uint64(0xFFFFFFFF))).astype(np.int64))


@pytest.mark.parametrize("n,seed", [(262144, 0), (262144, 1), (32768, 2), (32768, 3)])
def test_sampled_threshold_is_exact_without_redo_at_chunk_scale(n, seed):
    """Rows of the C4 and C2 prefill chunks (about 262,144 and 32,768 candidates)."""
    s = np.random.default_rng(seed).standard_normal(n).astype(np.float32)
    got = sampled_select(s)
    assert got is not None
    assert np.array_equal(got, oracle_select(s))


@pytest.mark.parametrize("seed", range(12))
def test_sampled_threshold_kept_rows_are_exact(seed):
    s, _, topk = mixed_case(seed)
    got = sampled_select(s, topk)
    if got is not None:
        assert np.array_equal(got, oracle_select(s, topk))


def test_sampled_threshold_keeps_every_key_of_rows_the_buffers_hold():
    """Just above 512 candidates a one-tile sample would keep about half of the row (fewer than
    512 keys, a redo); rows of up to 4,096 candidates keep every key instead, and are exact."""
    for n, seed in ((700, 5), (1024, 6), (4096, 7), (6000, 8)):
        s = np.random.default_rng(seed).standard_normal(n).astype(np.float32)
        got = sampled_select(s)
        assert got is not None and np.array_equal(got, oracle_select(s))
