"""The seeded generators are deterministic and produce the advertised shapes and dtypes."""

import numpy as np

from synth import make_workload, make_case, to_bf16, WORKLOADS


def test_tiny_workload_shape_and_recipe():
    a = make_workload("tiny_16x256x128_int4")
    b = make_workload("tiny_16x256x128_int4")
    assert a.x.shape == (16, 256) and a.W.shape == (256, 128) and a.scale.shape == (256,)
    assert np.array_equal(a.x, b.x) and np.array_equal(a.W, b.W) and np.array_equal(a.scale, b.scale)
    assert a.x_dtype == "f32" and a.rank == 16 and a.bits == 4
    assert list(a.notes["outlier_idx"]) == [3, 77, 140, 201]
    col = np.abs(a.x).max(0)
    assert np.median(col[[3, 77, 140, 201]]) > 10 * np.median(col)
    assert np.all(a.scale > 0) and np.all(np.isfinite(a.scale))
    s = np.sqrt(np.abs(a.x.astype(np.float64)).max(0)) / np.sqrt(np.abs(a.W.astype(np.float64)).max(1))
    np.testing.assert_allclose(a.scale, s.astype(np.float32), rtol=1e-7)


def test_bf16_case_values_are_representable():
    wl = make_case(33, 64, 48, rank=4, seed=5, bias=True)
    assert np.array_equal(to_bf16(wl.x), wl.x)
    assert np.array_equal(to_bf16(wl.W), wl.W)
    assert np.array_equal(to_bf16(wl.bias), wl.bias)


def test_named_workloads_exist():
    for n in ("dit_attn_4096x3072x3072_int4", "dit_mlp_4096x3072x12288_nvfp4",
              "decode_128x4096x4096_int4", "decode_128x4096x4096_nvfp4",
              "large_8192x12288x3072_nvfp4_r128", "large_8192x12288x3072_int8_r32"):
        assert n in WORKLOADS
