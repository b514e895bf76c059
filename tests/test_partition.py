"""CPU check of the prologue's work partition (no GPU).

Pass 1 cuts the (row block) x (64-wide K tile) grid into one contiguous run of
tiles per CTA, CTA c taking [c T / G, (c + 1) T / G), and sizes its partial-sum
workspace for max_segs runs meeting one row block.  This mirrors the
library's integer rules (the grid G from the tile count, the run bound) and
checks the bound against a direct count of the owners of every row block's
tiles, over a sweep of token counts and channel counts."""
import pytest


def grid_for(total, sms=148):
    by_work = (total + 3) // 4
    floor_ctas = min(total, 32)
    return min(max(by_work, floor_ctas), sms)


def max_segs(kt2, total, grid):
    run = total // grid
    return (kt2 - 2) // run + 2


def owners_per_block(m_blocks, kt2, grid):
    total = m_blocks * kt2
    worst = 0
    for mb in range(m_blocks):
        first, last = mb * kt2, mb * kt2 + kt2 - 1
        o_first = ((first + 1) * grid - 1) // total
        o_last = ((last + 1) * grid - 1) // total
        worst = max(worst, o_last - o_first + 1)
    return worst


@pytest.mark.parametrize("sms", [148, 132, 2])
def test_segment_bound_holds(sms):
    checked = 0
    for M in list(range(1, 2100, 37)) + [4096, 4608, 32760]:
        m_blocks = ((M + 255) // 256 * 256) // 128
        for K in (8, 64, 72, 136, 256, 1000, 3072, 5120, 12288, 16384):
            kt2 = 2 * ((K + 127) // 128)
            total = m_blocks * kt2
            grid = grid_for(total, sms)
            assert 1 <= grid <= min(total, sms)
            assert owners_per_block(m_blocks, kt2, grid) <= max_segs(kt2, total, grid), (M, K, sms)
            checked += m_blocks
    assert checked > 8000


def test_grid_rule_examples():
    assert grid_for(4) == 4            # tiny: a CTA per tile
    assert grid_for(192) == 48         # M = 512, K = 3072: four tiles a CTA
    assert grid_for(1536) == 148       # qkv: every SM
    assert grid_for(40) == 32          # small: at least 32 CTAs
