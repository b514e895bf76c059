"""CPU check of the library's work split (no GPU), through rtlynx_schedule_info.

Pass 1 of the prologue cuts the (row block) x (64-wide K tile) grid into one
contiguous run of tiles per CTA, CTA c taking [c T / G, (c + 1) T / G), and
sizes its partial-sum workspace for prologue_max_segs runs meeting one row
block.  The test takes the library's own G and bound and counts, from that
partition rule, the CTAs that really meet every row block.  The GEMM's split
of its last wave is checked against the invariants the kernel relies on."""
import pytest

import activation_sparse_gemm_b200 as rl
from activation_sparse_gemm_b200 import build as rl_build


@pytest.fixture(scope="module", autouse=True)
def _built():
    rl_build.build()


def owners_per_block(m_blocks, kt2, grid):
    total = m_blocks * kt2
    worst = 0
    for mb in range(m_blocks):
        first, last = mb * kt2, mb * kt2 + kt2 - 1
        o_first = ((first + 1) * grid - 1) // total   # CTA c holds tile t iff c T / G <= t < (c+1) T / G
        o_last = ((last + 1) * grid - 1) // total
        worst = max(worst, o_last - o_first + 1)
    return worst


def test_owner_rule_matches_the_partition():
    # the closed-form owner above is the inverse of c -> [c T / G, (c + 1) T / G)
    for total in (1, 7, 48, 1536, 20480):
        for grid in {1, min(total, 3), min(total, 32), min(total, 148)}:
            for c in range(grid):
                for t in range(c * total // grid, (c + 1) * total // grid):
                    assert ((t + 1) * grid - 1) // total == c


@pytest.mark.parametrize("sms", [148, 132, 2])
def test_segment_bound_holds(sms):
    checked = 0
    for M in list(range(1, 2100, 37)) + [4096, 4608, 32760]:
        for K in (8, 64, 72, 136, 256, 1000, 3072, 5120, 12288, 16384):
            s = rl.rtlynx_schedule_info(M, K, 64, 64, sms)
            assert s.row_blocks == (M + 255) // 256 * 2
            assert s.k_tiles_per_block == 2 * ((K + 127) // 128)
            assert s.prologue_tiles == s.row_blocks * s.k_tiles_per_block
            assert 1 <= s.prologue_ctas <= min(s.prologue_tiles, sms)
            assert owners_per_block(s.row_blocks, s.k_tiles_per_block, s.prologue_ctas) <= s.prologue_max_segs, \
                (M, K, sms)
            checked += s.row_blocks
    assert checked > 8000


def test_prologue_grid_examples():
    def grid(M, K):
        return rl.rtlynx_schedule_info(M, K, 64, 0, 148).prologue_ctas
    assert grid(128, 128) == 4      # tiny: a CTA per tile (2 row blocks x 2 K tiles)
    assert grid(512, 3072) == 48    # four tiles a CTA
    assert grid(4096, 3072) == 148  # qkv: every SM
    assert grid(256, 1280) == 32    # 40 tiles: at least 32 CTAs


@pytest.mark.parametrize("M,K,N,R", [(4096, 3072, 9216, 64), (4608, 3072, 12288, 64), (4608, 12288, 3072, 64),
                                     (32760, 5120, 13824, 64), (128, 256, 256, 64), (2560, 2048, 1920, 64),
                                     (2560, 256, 1920, 256), (1, 64, 8, 8), (5000, 136, 264, 16)])
def test_gemm_tail_split_invariants(M, K, N, R):
    s = rl.rtlynx_schedule_info(M, K, N, R, 148)
    assert s.gemm_tiles == (M + 255) // 256 * ((N + 239) // 240)
    assert s.gemm_pairs == min(s.gemm_tiles, 74)
    rem = s.gemm_tiles % s.gemm_pairs
    n_iter = s.k_stages + s.lora_stages
    if s.tail_units == 0:
        assert s.tail_full == s.gemm_tiles and s.tail_split == 1
    else:
        # only the partial last wave is split; one part per pair, 3 to 6 parts a
        # tile, each part at least two stages long
        assert s.tail_full == s.gemm_tiles - rem
        assert 3 <= s.tail_split <= 6
        assert s.tail_units == rem * s.tail_split <= s.gemm_pairs
        assert n_iter // s.tail_split >= 2
    r_pad = (R + 63) // 64 * 64
    assert s.lora_stages in ((0,) if R == 0 else (r_pad // 64, r_pad // 32))  # 64- or 32-wide LoRA stages


def test_workloads_examples():
    qkv = rl.rtlynx_schedule_info(4096, 3072, 9216, 64, 148)
    assert (qkv.gemm_tiles, qkv.tail_units) == (624, 0)      # 8 whole waves and 32 tiles: too few parts to split
    video = rl.rtlynx_schedule_info(32760, 5120, 13824, 64, 148)
    assert (video.gemm_tiles, video.tail_split, video.tail_units) == (7424, 3, 72)
    down = rl.rtlynx_schedule_info(4608, 12288, 3072, 64, 148)
    assert (down.gemm_tiles, down.tail_split, down.tail_units) == (234, 6, 72)


def test_schedule_rejects_bad_arguments():
    with pytest.raises(rl.RtlynxError):
        rl.rtlynx_schedule_info(0, 64, 64, 0, 148)
    with pytest.raises(rl.RtlynxError):
        rl.rtlynx_schedule_info(16, 60, 64, 0, 148)
    with pytest.raises(rl.RtlynxError):
        rl.rtlynx_schedule_info(16, 64, 64, 0, 1)


def test_small_path_selection():
    """The one-kernel small path: the output is one wave of 256 x 240 tiles
    (at most one CTA pair per two SMs), D_in <= 256 and R <= 64; anything
    else takes the general three-kernel path."""
    def small(M, K, N, R, sms=148):
        return rl.rtlynx_schedule_info(M, K, N, R, sms).small_path

    assert small(128, 256, 256, 64) == 1          # the tiny workload
    assert small(4096, 3072, 9216, 64) == 0       # qkv
    assert small(128, 264, 256, 64) == 0          # D_in past 256
    assert small(128, 256, 256, 72) == 0          # R past 64
    assert small(128, 256, 256, 0) == 1           # no LoRA
    assert small(1, 8, 8, 8) == 1
    # one wave: 74 pairs on 148 SMs (row pairs of 256 tokens x column tiles of 240)
    assert small(256 * 74, 256, 240, 16) == 1
    assert small(256 * 74 + 1, 256, 240, 16) == 0
    assert small(256 * 37, 256, 480, 16) == 1
    assert small(256 * 37, 256, 488, 16) == 0
    assert small(256 * 37, 256, 480, 16, sms=72) == 0
    # the ABI's launch count follows the same rule (148 SMs where no GPU is present)
    if rl.rtlynx_schedule_info(128, 256, 256, 64, 148).small_path == 1 and not _has_gpu():
        assert rl.rtlynx_kernel_launches(128, 256, 256, 64, rl.MODE_SPARSE) == 1
        assert rl.rtlynx_kernel_launches(4096, 3072, 9216, 64, rl.MODE_SPARSE) == 3


def _has_gpu():
    try:
        import torch
        return torch.cuda.is_available()
    except Exception:
        return False
