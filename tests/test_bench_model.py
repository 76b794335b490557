"""The bench's roofline arithmetic (host logic, no GPU): algorithmic bytes and
operation counts of a step against the per-workload table worked out by hand
from the measurement definition (x bf16 read once; weight codes at 0.5 / 1 byte
per element, plus 1/16 byte of ue4m3 scale for NVFP4 or 1/32 byte of E8M0
scale for MXFP4; bf16 ld and lu; fp32 scale; bf16 bias and Y; ops 2BMN
residual + 2Br(M+N) low-rank)."""

import pytest

import bench


@pytest.mark.parametrize("B,M,N,r,fmt,bits,bias,mb", [
    (4096, 3072, 3072, 32, "int", 4, False, 55.46),      # DiT attention, INT4
    (4096, 3072, 12288, 32, "nvfp4", 4, True, 148.08),   # DiT MLP, NVFP4, bias
    (1, 4096, 4096, 32, "int", 4, False, 8.95),          # decode B = 1
    (16, 4096, 4096, 32, "int", 4, False, 9.19),
    (128, 4096, 4096, 32, "int", 4, False, 11.03),
    (1, 4096, 4096, 32, "nvfp4", 4, False, 9.99),
    (128, 4096, 4096, 32, "nvfp4", 4, False, 12.08),
    (8192, 12288, 3072, 32, "int", 4, False, 271.56),    # large, INT4 r 32 / 128, INT8, NVFP4
    (8192, 12288, 3072, 128, "int", 4, False, 274.51),
    (8192, 12288, 3072, 32, "int", 8, False, 290.44),
    (8192, 12288, 3072, 32, "nvfp4", 4, False, 273.92),
])
def test_algorithmic_bytes_match_the_worked_table(B, M, N, r, fmt, bits, bias, mb):
    assert bench.alg_bytes(B, M, N, r, fmt, bits, bias) / 1e6 == pytest.approx(mb, abs=0.01)


def test_mxfp4_scale_bytes_are_half_of_nvfp4():
    M, N = 3072, 12288
    nv = bench.alg_bytes(4096, M, N, 32, "nvfp4", 4, True)
    mx = bench.alg_bytes(4096, M, N, 32, "mxfp4", 4, True)
    assert nv - mx == M * N / 32


def test_operation_counts():
    assert bench.workload_ops(4096, 3072, 3072, 32) == 2 * 4096 * 3072 * 3072 + 2 * 4096 * 32 * 6144
    assert bench.gemm_alg_ops(4096, 3072, 3072, 32) == 2 * 4096 * 3072 * 3072 + 2 * 4096 * 32 * 3072
