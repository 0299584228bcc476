"""The BF16 layer policy of the NVFP4 recipe (section 2B.1 of the NVFP4 page):
the first two and the last eight blocks keep BF16 linear layers.  CPU only."""
import pytest

from nvfp4_bit_microscaled_b200.api import block_uses_bf16


def test_first_two_and_last_eight_blocks_stay_bf16():
    n = 62
    bf16 = [b for b in range(n) if block_uses_bf16(b, n)]
    assert bf16 == [0, 1] + list(range(54, 62))
    assert not block_uses_bf16(2, n) and not block_uses_bf16(53, n)


def test_share_of_bf16_blocks_is_about_the_pages_sixteen_percent():
    # ten BF16 blocks out of the 62 of a 12B-class stack: ~16 %
    n = 62
    share = sum(block_uses_bf16(b, n) for b in range(n)) / n
    assert abs(share - 0.16) < 0.01


def test_small_stacks_and_bounds():
    assert all(block_uses_bf16(b, 10) for b in range(10))      # 2 + 8 covers everything
    assert [block_uses_bf16(b, 12) for b in range(12)] == [True, True, False, False] + [True] * 8
    with pytest.raises(ValueError):
        block_uses_bf16(12, 12)
