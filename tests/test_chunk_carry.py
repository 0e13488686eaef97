"""Host logic of prefill chunks whose boundaries are not multiples of the 4-token block: which
keys form whole blocks now and which are carried to the next chunk (CPU; no library calls)."""
import pytest

from learned_block_sparse_qsa_b200.runner import compress_split


def test_aligned_chunk_compresses_everything():
    assert compress_split(0, 0, 0, 4096) == (0, 4096, 4096, 0)


def test_unaligned_end_carries_the_tail():
    assert compress_split(0, 0, 0, 1001) == (0, 1000, 1000, 1)


def test_carry_is_prepended_and_completed():
    # carried position 1000; the chunk 1001..1998 completes block 250 and ends inside block 499
    assert compress_split(1000, 1, 1001, 998) == (1000, 996, 1996, 3)


def test_short_chunk_inside_one_block_compresses_nothing():
    assert compress_split(1996, 2, 1998, 1) == (1996, 0, 1996, 3)


def test_chain_of_ragged_chunks_covers_every_block_once():
    sizes = [1001, 998, 3, 1, 1003, 1090]
    carry_pos, carry_len, pos, done = 0, 0, 0, []
    for n in sizes:
        start, k, carry_pos, carry_len = compress_split(carry_pos, carry_len, pos, n)
        assert start % 4 == 0 and k % 4 == 0
        done += list(range(start // 4, (start + k) // 4))
        pos += n
    assert done == list(range(pos // 4)) and carry_len == pos % 4


@pytest.mark.parametrize("args", [(0, 0, 2, 5), (1000, 1, 1002, 4), (1001, 1, 1002, 4)])
def test_gaps_and_misaligned_carries_are_rejected(args):
    with pytest.raises(ValueError):
        compress_split(*args)
