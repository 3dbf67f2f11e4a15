"""Memory-footprint accounting (host only): the counts follow the stored-
parameter formula the oracle pins, and the byte sizes match what the library
actually stores and builds."""
import math

import pytest

from oracle import bfmoe_oracle as O
from ternary_butterfly_experts_b200 import footprint as F


@pytest.mark.parametrize("d,N", [(4, 1), (64, 8), (512, 64), (512, 256), (2048, 1024)])
def test_counts_match_the_parameter_formula(d, N):
    f = F.footprint(d, N)
    n_ternary, n_angles = O.param_count(d, N)
    assert f.n_angles == n_angles
    assert f.base_bytes * 8 == 2 * n_ternary or d < 16   # 2 bits per weight
    assert f.angle_total_bytes == 4 * n_angles
    assert f.dense_total_bytes == 4 * N * d * d
    assert f.stored_bytes == f.base_bytes + 4 + f.angle_total_bytes
    assert math.isclose(f.base_ideal_bytes, d * d * math.log2(3) / 8)


def test_headline_point_and_ratios():
    f = F.footprint(512, 256)
    # 2-bit base 64 KiB, 2 * 256 * 256 * 9 float32 angles
    assert f.base_bytes == 65536
    assert f.angle_total_bytes == 2 * 256 * 256 * 9 * 4
    assert f.stored_bytes == 65536 + 4 + 4718592
    assert abs(f.ratio - 256 * 512 * 512 * 4 / (65536 + 4 + 4718592)) < 1e-9
    # bf16 angles halve the angle bytes
    assert F.footprint(512, 256, angle_bytes=2).angle_total_bytes == f.angle_total_bytes // 2


def test_ratio_grows_with_experts_towards_the_angle_bound():
    # dense N d^2 against N d log d angles: the ratio tends to d / log2(d)
    # (float32 both) as the shared base becomes negligible
    r = [F.footprint(512, n).ratio for n in (8, 64, 256, 4096)]
    assert r == sorted(r)
    assert r[-1] < 512 / 9 < r[-1] * 1.01


def test_packed_size_matches_the_library_layout():
    from ternary_butterfly_experts_b200 import words_per_row
    for d in (4, 16, 512, 4096):
        assert F.footprint(d, 1).base_bytes == d * words_per_row(d) * 4


def test_cli_prints_a_table(capsys):
    assert F.main(["--d", "512", "--experts", "8", "64", "256"]) == 0
    out = capsys.readouterr().out
    assert "| 256 |" in out and "dense / stored" in out
