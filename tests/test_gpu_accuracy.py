"""The premise of the method, measured end to end through the library: on keys with
outlier channels, rotating by the block-diagonal Hadamard transform before token-wise INT4
lowers the attention-output error against exact attention on the unquantised rows
(wispaper.ai blog on SAW-INT4, section 2: rotation spreads channel outliers so one
token-wise scale fits; the paper's abstract: near-lossless INT4 with BDR).  The BF16 cache
is the lossless reference of the pages' comparisons."""
import pytest
import torch

import bench

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def study():
    w = bench.Workload("batch16", 0, torch.device("cuda"))
    return bench.accuracy_study(w, torch.device("cuda"))


def test_bf16_cache_is_nearly_exact(study):
    assert study["bf16"]["max_rel"] < 5e-3


def test_rotation_lowers_int4_error(study):
    """Every block size lowers the mean row error; the worst row (a noisy statistic over one
    batch) is checked for the block size the pages recommend, 128."""
    naive = study["int4"]
    for b in (16, 32, 64, 128):
        rot = study[f"bdr{b}_k"]
        assert rot["mean_rel"] < 0.5 * naive["mean_rel"], (b, rot, naive)
    assert study["bdr128_k"]["max_rel"] < 0.5 * naive["max_rel"]


def test_wider_blocks_spread_outliers_further(study):
    assert study["bdr128_k"]["mean_rel"] < study["bdr16_k"]["mean_rel"]


def test_rotating_values_too_does_not_hurt(study):
    for b in (16, 32, 64, 128):
        assert study[f"bdr{b}_kv"]["mean_rel"] <= study[f"bdr{b}_k"]["mean_rel"] * 1.05
