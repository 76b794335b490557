"""The C-ABI library builds, loads and exports every function include/svdq.h declares;
its host-side argument checks work without a GPU (no kernel is launched here)."""

import ctypes

import pytest

import rank_bit_residual_b200 as rb
from rank_bit_residual_b200 import build as rbuild


@pytest.fixture(scope="module")
def lib():
    rbuild.build()
    return rb.load_library()


def test_every_declared_function_is_exported(lib):
    names = rb.header_functions()
    assert len(names) >= 14
    for n in names:
        assert hasattr(lib, n), f"{n} declared in include/svdq.h but not exported"
        assert n in rb._SIGS, f"{n} has no binding signature"


def test_version_and_status_strings(lib):
    assert lib.svdq_version().decode().count(".") == 2
    for s in range(7):
        assert len(lib.svdq_status_string(s)) >= 2


def _sizes(lib, M, N, r, fmt):
    sizes = (ctypes.c_size_t * 7)()
    st = lib.svdq_weight_buffer_sizes(M, N, r, rb.parse_fmt(fmt), sizes)
    return st, list(sizes)


def test_weight_buffer_sizes(lib):
    st, s = _sizes(lib, 3072, 3072, 32, "int4")
    assert st == rb.SVDQ_OK
    assert s == [3072 * 3072, 0, 4, 32 * 3072 * 2, 32 * 3072 * 4, 3072 * 64 * 2, 3072 * 3072 // 2]
    assert _sizes(lib, 3072, 3072, 32, "int8")[1][6] == 0      # no packed copy above 4 bits
    st, s = _sizes(lib, 256, 3216, 20, "nvfp4")
    assert st == rb.SVDQ_OK
    assert s[0] == 3216 * 128 and s[1] == 3328 * 16   # rows padded to 128, 16 scale columns
    assert s[3] == 32 * 256 * 2
    assert s[6] == 0
    st, s = _sizes(lib, 288, 3216, 20, "mxfp4")
    assert st == rb.SVDQ_OK
    assert s[0] == 3216 * 144 and s[1] == 3328 * 12   # 9 scale columns padded to 12
    assert s[6] == 0
    assert _sizes(lib, 64, 32, 1, (2, 8))[0] == rb.SVDQ_EINVAL   # MXFP4 has 4 bits only
    assert _sizes(lib, 64, 32, 1, (3, 4))[0] == rb.SVDQ_EINVAL   # no fourth kind


def test_host_checks_follow_the_page_contract(lib):
    # "_check_rank": rank in [0, min(M, N)]
    assert _sizes(lib, 64, 32, 33, "int4")[0] == rb.SVDQ_ERANK
    assert _sizes(lib, 64, 32, -1, "int4")[0] == rb.SVDQ_ERANK
    assert _sizes(lib, 64, 32, 32, "int4")[0] == rb.SVDQ_OK
    assert _sizes(lib, 64, 32, 0, "int4")[0] == rb.SVDQ_OK
    # "_check_smoothing": nonempty
    assert _sizes(lib, 0, 32, 0, "int4")[0] == rb.SVDQ_EINVAL
    # grid: 2 <= bits <= 8
    assert _sizes(lib, 64, 32, 1, (0, 1))[0] == rb.SVDQ_EINVAL
    assert _sizes(lib, 64, 32, 1, (0, 9))[0] == rb.SVDQ_EINVAL
    assert _sizes(lib, 64, 32, 1, (1, 8))[0] == rb.SVDQ_EINVAL
    # this library's limits
    assert _sizes(lib, 48, 32, 1, "int4")[0] == rb.SVDQ_EUNSUPPORTED
    assert _sizes(lib, 64, 40, 1, "int4")[0] == rb.SVDQ_EUNSUPPORTED
    assert _sizes(lib, 512, 512, 257, "int4")[0] == rb.SVDQ_EUNSUPPORTED


def test_workspace_queries(lib):
    b = ctypes.c_size_t()
    assert lib.svdq_quantize_act_workspace_size(4096, 3072, rb.parse_fmt("int4"), 32, ctypes.byref(b)) == 0
    assert b.value > 0
    assert lib.svdq_quantize_act_workspace_size(4096, 3072, rb.parse_fmt("int4"), 20, ctypes.byref(b)) \
        == rb.SVDQ_EINVAL
    assert lib.svdq_quantize_residual_workspace_size(3072, 3072, rb.parse_fmt("nvfp4"), ctypes.byref(b)) == 0
    assert lib.svdq_prepare_workspace_size(3072, 3072, 32, rb.parse_fmt("int4"), 0, ctypes.byref(b)) == 0


def test_python_binding_rejects_non_int_rank():
    import torch
    W = torch.zeros(64, 32)
    s = torch.ones(64)
    for r in (True, 1.0, "1"):
        with pytest.raises(ValueError):
            rb.svdq_prepare(W, s, r)
    with pytest.raises(ValueError):      # CPU tensors are refused, never computed on the host
        rb.svdq_prepare(W, s, 1)


def test_linear_ex_rejects_unknown_flags(lib):
    """Checked before anything touches the device."""
    w = rb.SvdqWeight()
    st = lib.svdq_linear_ex(ctypes.byref(w), None, 0, 1, 64, None, None, None, 0, 64, None, 0,
                            ctypes.c_uint32(2), None)
    assert st == rb.SVDQ_EINVAL


def test_quantize_act_rejects_unaligned_outputs(lib):
    """The codes (8-byte stores) and the down tile (8- and 16-byte stores) must be
    16-byte aligned; checked on the host, before anything touches the device (the
    pointers here are never dereferenced)."""
    x, scale, ld, act_scale = 0x10000, 0x20000, 0x30000, 0x40000
    fmt = rb.parse_fmt("int4")

    def call(codes, down):
        return lib.svdq_quantize_act(x, rb.SVDQ_BF16, 256, 64, 64, scale, fmt, None, None, ld, 32,
                                     codes, None, act_scale, down, None, 0, None)

    assert call(0x50008, 0x60000) == rb.SVDQ_EUNSUPPORTED     # codes off by 8 bytes
    assert call(0x50000, 0x60004) == rb.SVDQ_EUNSUPPORTED     # down off by 4 bytes
    assert call(0x50000, None) == rb.SVDQ_EINVAL             # ld given without down


def test_weight_outputs_must_be_aligned(lib):
    """svdq_prepare and svdq_quantize_residual write the weight's buffers in 8- and
    16-byte pieces; a buffer off a 16-byte boundary is refused on the host (the
    pointers here are never dereferenced)."""
    W, scale, ws, R = 0x10000, 0x20000, 0x30000, 0x40000
    fmt = rb.parse_fmt("nvfp4")

    def weight(**off):
        w = rb.SvdqWeight()
        for i, f in enumerate(("codes", "sf", "w_scale", "ld", "lu", "ld32")):
            setattr(w, f, 0x100000 * (i + 1) + off.get(f, 0))
        return w

    for field in ("codes", "sf", "ld", "lu", "ld32"):
        w = weight(**{field: 8})
        st = lib.svdq_prepare(W, rb.SVDQ_BF16, 64, 32, 32, scale, 4, fmt, 0, 0, 0, ws, 1 << 30,
                              ctypes.byref(w), None)
        assert st == rb.SVDQ_EUNSUPPORTED, field
    st = lib.svdq_quantize_residual(R, 64, 32, 32, fmt, 0x50008, 0x60000, 0x70000, ws, 1 << 30, None)
    assert st == rb.SVDQ_EUNSUPPORTED


def test_no_cpu_path():
    """Every operator call takes CUDA tensors only: host tensors raise instead of
    being computed on the CPU, and a missing library raises on load."""
    import torch
    x = torch.zeros((4, 64), dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        rb.svdq_quantize_act(x, torch.ones(64), "mxfp4")
    with pytest.raises(ValueError):
        rb.svdq_smooth_scale(x, torch.zeros((64, 32)), 0.5)
    with pytest.raises(ValueError):
        rb.svdq_prepare(torch.zeros((64, 32)), torch.ones(64), 4, "nvfp4")
    saved = rb._lib
    try:
        rb._lib = None
        with pytest.raises(ImportError):
            rb.load_library("/nonexistent/libsvdq.so")
    finally:
        rb._lib = saved
