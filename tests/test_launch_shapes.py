"""The launch shapes the library picks, asked through the C ABI on the host
(no device needed): the GEMM tile shape per problem size and the quantizers'
tile height.  The GPU tests that target one tile shape assert it the same
way, so they keep covering the shape they are written for."""
import pytest

import nvfp4_block_scaled_12_b200 as F

SMS = 148  # B200


@pytest.mark.parametrize("m,n,want,why", [
    (4608, 12288, (2, 256, 1), "FLUX MLP-up: 18 x 48 wide tiles, far more than 74 CTA pairs"),
    (4608, 3072, (2, 256, 1), "attention projection at 4608 tokens: 216 wide tiles"),
    (2304, 2304, (2, 256, 1), "81 wide tiles: one per CTA pair and more"),
    (1000, 2880, (2, 192, 2), "48 wide tiles leave pairs idle; 92 tiles of 128 would need two waves"),
    (1024, 3072, (2, 192, 2), "48 wide, 64 of 192, 96 of 128: 192 fills most pairs in one wave"),
    (512, 3072, (2, 128, 2), "24 wide, 32 of 192, 48 of 128: the narrowest tiles put the most pairs to work"),
    (128, 12288, (1, 192, 2), "M <= 128: one CTA per 128-row tile"),
    (1, 8, (1, 192, 2), "a single row"),
    (129, 8, (2, 128, 2), "just past one 128-row tile"),
])
def test_gemm_tile_shape_table(m, n, want, why):
    assert F.nvfp4_gemm_tile_shape(m, n, SMS) == want, why


def test_gemm_takes_wide_tiles_from_one_wave_of_pairs_on():
    # for a fixed width, more tokens never move the GEMM off the wide tiles
    # once it has taken them, and it takes them exactly at one tile per pair
    for n in (3072, 12288, 15360, 2056):
        wide = [m for m in range(129, 20000, 61) if F.nvfp4_gemm_tile_shape(m, n, SMS) == (2, 256, 1)]
        assert wide and all(F.nvfp4_gemm_tile_shape(m, n, SMS) == (2, 256, 1) for m in range(wide[0], 20000, 61))
        first = wide[0]
        assert ((first + 255) // 256) * ((n + 255) // 256) >= SMS // 2
        prev = first - 61
        assert ((prev + 255) // 256) * ((n + 255) // 256) < SMS // 2 or prev <= 128


def test_gemm_tile_shape_depends_on_the_sm_count():
    # a device with fewer SMs reaches one tile per pair sooner
    assert F.nvfp4_gemm_tile_shape(1024, 3072, 148) == (2, 192, 2)
    assert F.nvfp4_gemm_tile_shape(1024, 3072, 80) == (2, 256, 1)


def test_gemm_tile_shape_rejects_bad_arguments():
    for args in ((0, 64, SMS), (16, 4, SMS), (16, 64, 1), (1 << 30, 64, SMS)):
        with pytest.raises(F.NVFP4Error) as e:
            F.nvfp4_gemm_tile_shape(*args)
        assert e.value.status == F.NVFP4_EINVAL


@pytest.mark.parametrize("m,k,want", [
    (4608, 12288, 256),   # the standalone quantize workload: 18 x 192 = 3456 tiles of 256 rows
    (4608, 3072, 128),    # the MLP-up activations: 864 tiles of 256 rows, under 8 per SM
    (4608, 15360, 256),
    (512, 3072, 128),
    (9216, 2048, 128),    # 36 x 32 = 1152 < 8 x 148
    (9217, 2048, 256),    # 37 x 32 = 1184: eight per SM
])
def test_quantize_tile_rows(m, k, want):
    assert F.nvfp4_quantize_tile_rows(m, k, SMS) == want


def test_quantize_tile_rows_is_zero_for_invalid_sizes():
    assert F.nvfp4_quantize_tile_rows(0, 64, SMS) == 0
    assert F.nvfp4_quantize_tile_rows(4, 96, SMS) == 0
    assert F.nvfp4_quantize_tile_rows(4, 64, 0) == 0


@pytest.mark.parametrize("m,n,k,w16,want,why", [
    (100, 3072, 3072, 0, (1, 192, 2, 4), "16 tiles of 128 x 192: four CTAs share each tile, 12 k-tiles -> 3 each"),
    (100, 3072, 3072, 1, (1, 192, 2, 4), "W4A16: 48 k-tiles of 64 -> 12 a CTA"),
    (512, 3072, 3072, 0, (2, 128, 2, 1), "12 k-tiles: a split would save less than its own work"),
    (512, 3072, 3072, 1, (2, 192, 2, 2), "W4A16, 48 k-tiles: 32 pair tiles of 192 split in two"),
    (1024, 3072, 3072, 0, (2, 192, 2, 1), "64 pair tiles already fill the pairs"),
    (4608, 12288, 3072, 0, (2, 256, 1, 1), "wide tiles never split"),
    (128, 256, 256, 0, (1, 192, 2, 1), "one k-tile: nothing to split"),
    (300, 520, 1088, 1, (2, 128, 2, 2), "two CTA pairs (4 CTAs) to a cluster at most"),
    (16, 3072, 15360, 0, (1, 192, 2, 4), "4 CTAs to a cluster at most"),
    (300, 520, 15360, 0, (2, 128, 2, 2), "a long K splits over CTA pairs too"),
])
def test_gemm_plan_table(m, n, k, w16, want, why):
    assert F.nvfp4_gemm_plan(m, n, k, SMS, w16) == want, why


def test_gemm_plan_keeps_every_cluster_within_4_ctas_resident_at_once():
    for m in (1, 37, 128, 129, 300, 512, 777, 1024, 2000):
        for n in (8, 192, 1000, 3072, 12288):
            for k in (64, 256, 320, 3072, 15360):
                for w16 in (0, 1):
                    cg, bn, acc, ks = F.nvfp4_gemm_plan(m, n, k, SMS, w16)
                    num_kt = k // 64 if w16 else (k // 2 + 127) // 128
                    assert ks in (1, 2, 4) and cg * ks <= 4 and ks <= num_kt
                    tiles = ((m + 128 * cg - 1) // (128 * cg)) * ((n + bn - 1) // bn)
                    assert ks == 1 or tiles * ks * cg * 8 <= SMS * 7  # every split cluster resident at once
                    if ks > 1:
                        assert (cg, bn) != (2, 256)  # the wide tiles never split
                        assert (num_kt + ks - 1) // ks + 6 < num_kt  # the split saves more than it costs
