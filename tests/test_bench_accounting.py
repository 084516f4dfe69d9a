"""bench.py's work accounting on CPU: the closed-form FLOP count of a step
against the step's GEMMs listed one by one, the figures the design notes quote
for one 1540x1540 image, and the exponential-unit arithmetic of attention."""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from vision_language_model_b200 import vlm  # noqa: E402


@pytest.fixture(scope="module")
def cfg():
    if not os.path.exists(vlm.lib_path()):
        from vision_language_model_b200 import build
        build.build()
    return vlm.preset("mistral3")


def _listed_gemm_flops(T, Tm, d=1024, f=4096, e=5120, p=14, layers=24):
    """Every GEMM of a step as (M, N, K), 2 FLOPs per multiply-add."""
    shapes = [(T, d, 3 * p * p)]                                    # patch embed (K = 3 p^2, unpadded)
    for _ in range(layers):
        shapes += [(T, 3 * d, d), (T, d, d), (T, 2 * f, d), (T, d, f)]  # QKV, O, gate/up, down
    shapes += [(Tm, d, 4 * d), (Tm, e, d), (Tm, e, e)]              # merge linear, W1, W2
    return sum(2.0 * m * n * k for m, n, k in shapes)


def test_step_flops_match_the_listed_gemms_and_attention(cfg):
    fl = bench.flops_breakdown(cfg, [(1540, 1540)])
    assert (fl["T"], fl["Tm"]) == (12100, 3025)
    assert fl["gemm"] == _listed_gemm_flops(12100, 3025)
    # attention: q k^T and p v over the image's own 12,100^2 pairs, 16 heads x 64
    assert fl["attn_per_launch"] == 2 * (2.0 * 12100 * 12100 * 64) * 16
    assert fl["total"] == fl["gemm"] + 24 * fl["attn_per_launch"]
    # the figures quoted for this workload
    assert round(fl["total"] / 1e13, 3) == 2.437
    assert round(fl["attn"] / fl["total"], 3) == 0.591
    # of the tower alone (the 24 blocks: attention plus their four GEMMs) it is 59.6%
    tower = fl["attn"] + 24 * 2.0 * 12100 * (3 * 1024 ** 2 + 1024 ** 2 + 2 * 4096 * 1024 + 4096 * 1024)
    assert round(tower / 1e13, 3) == 2.414 and round(fl["attn"] / tower, 3) == 0.596


def test_packed_images_count_attention_per_block(cfg):
    sizes = [(224, 224), (112, 168)]
    fl = bench.flops_breakdown(cfg, sizes)
    lens = [16 * 16, 8 * 12]
    assert fl["T"] == sum(lens)
    assert fl["attn_per_launch"] == sum(4.0 * n * n * 1024 for n in lens)  # no cross-image pairs


def test_exp_unit_line_arithmetic():
    # 256 FLOPs per score at head_dim 64; 7 in 8 exponentials on the MUFU pipe
    got = bench.exp_unit_line(256e9, 1.0, {"sm_mhz": 1000.0}, 100)
    assert got["scores_per_s"] == pytest.approx(1e12)
    assert got["mufu_ex2_per_s"] == pytest.approx(0.875e12)
    assert got["peak_mufu_ex2_per_s"] == pytest.approx(16 * 100 * 1e9)
    assert got["frac"] == pytest.approx(0.875e12 / 1.6e12)
    none = bench.exp_unit_line(256e9, 1.0, None, 100)
    assert none["peak_mufu_ex2_per_s"] is None and none["frac"] is None


def test_job_throughput_adds_ranks_over_the_slowest_time():
    assert bench.job_throughput(12100, 4, 10, 500.0) == pytest.approx(12100 * 4 * 10 / 0.5)
