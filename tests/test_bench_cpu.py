"""The benchmark's algorithmic work figures, checked against the operand
sizes written out by hand (no GPU): these are the numerators of every
roofline fraction bench.py reports."""

import pytest


def test_up_proj_work():
    import bench
    M, K, N = 4096, 2560, 6912
    w = bench.stage_work(M, N, K, w_bytes=2)
    # W bf16 read once (35.39 MB), codes written (4.42 MB), gamma (4 B),
    # x bf16 read (20.97 MB), xq written (10.49 MB), s_x written (16 KB)
    assert w["quantize"]["bytes"] == 35_389_440 + 4_423_680 + 4 + 20_971_520 + 10_485_760 + 16_384
    assert w["forward"]["ops"] == 144_955_146_240          # 2 M N K
    assert w["backward"]["ops"] == 2 * 144_955_146_240     # dX and dW, 2 M N K each
    assert w["forward"]["bound"] == w["backward"]["bound"] == "tensor"
    assert w["quantize"]["bound"] == "hbm"


def test_f32_masters_read_four_bytes_per_weight():
    import bench
    a = bench.stage_work(32, 256, 128, w_bytes=4)["quantize"]["bytes"]
    b = bench.stage_work(32, 256, 128, w_bytes=2)["quantize"]["bytes"]
    assert a - b == 256 * 128 * 2


@pytest.mark.parametrize("name", ["up_proj", "down_proj", "tiny"])
def test_workloads_have_the_documented_shapes(name):
    from workloads import WORKLOADS
    shapes = {"up_proj": (4096, 2560, 6912), "down_proj": (2048, 6912, 2560), "tiny": (32, 128, 256)}
    wl = WORKLOADS[name]
    assert (wl.M, wl.K, wl.N) == shapes[name]
    assert wl.K % 32 == 0
