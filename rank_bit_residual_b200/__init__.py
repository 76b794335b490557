"""Python binding of libsvdq (include/svdq.h): the SVDQuant inference linear on B200.

Argument marshalling only. Every step of the operator runs in the CUDA library;
torch supplies device memory and the current stream. There is no CPU path: if
libsvdq.so is missing or no GPU is present, the calls raise.

    w = svdq_prepare(W, scale, rank, fmt="int4")          # one-time split on the GPU
    y = svdq_linear(w, x, bias=None, out_dtype=torch.bfloat16)
    y = svdq_linear_chain([w1, w2], x)                     # consecutive layers, PDL-chained

Formats: "int2" .. "int8" (per-tensor grid), "nvfp4" (ue4m3 scales per 16
elements and an fp32 global scale), "mxfp4" (E8M0 scales per 32 elements).

Conventions follow "SVDQuant Smoothing, Low-rank and Residual Quantization":
x[B, M] @ W[M, N], positive finite scale[M], rank a Python int in
[0, min(M, N)]; invalid layouts, scales and ranks raise ValueError.
"""

from __future__ import annotations

import ctypes
import os
import re
from dataclasses import dataclass
from typing import Optional

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libsvdq.so")
HEADER_PATH = os.path.join(os.path.dirname(_PKG), "include", "svdq.h")

SVDQ_OK, SVDQ_EINVAL, SVDQ_ERANK, SVDQ_EUNSUPPORTED, SVDQ_ECUDA, SVDQ_ETIMEOUT, SVDQ_EWORKSPACE = range(7)
SVDQ_F32, SVDQ_BF16 = 0, 1
KIND_INT, KIND_NVFP4, KIND_MXFP4 = 0, 1, 2
SVDQ_LINEAR_PDL = 1

c_i32, c_i64, c_u64, c_sz, c_vp = ctypes.c_int32, ctypes.c_int64, ctypes.c_uint64, ctypes.c_size_t, ctypes.c_void_p


class SvdqFmt(ctypes.Structure):
    _fields_ = [("kind", c_i32), ("bits", c_i32)]


class SvdqWeight(ctypes.Structure):
    _fields_ = [("M", c_i64), ("N", c_i64), ("rank", c_i32), ("rank_pad", c_i32),
                ("fmt", SvdqFmt), ("codes", c_vp), ("sf", c_vp), ("w_scale", c_vp),
                ("ld", c_vp), ("ld32", c_vp), ("lu", c_vp), ("scale", c_vp), ("codes4", c_vp)]


_SIGS = {
    "svdq_version": (ctypes.c_char_p, []),
    "svdq_smooth_scale": (c_i32, [c_vp, c_i32, c_i64, c_i64, c_i64, c_vp, c_i32, c_i64, c_i64, ctypes.c_float,
                                  c_vp, c_vp, c_sz, c_vp]),
    "svdq_fold_scale": (c_i32, [c_vp, c_i32, c_i64, c_i64, c_i64, c_vp, c_i32, c_i64, c_i64, c_i32,
                                c_vp, c_vp, c_sz, c_vp]),
    "svdq_fold_scale_workspace_size": (c_i32, [c_i64, c_i64, ctypes.POINTER(c_sz)]),
    "svdq_status_string": (ctypes.c_char_p, [c_i32]),
    "svdq_weight_buffer_sizes": (c_i32, [c_i64, c_i64, c_i32, SvdqFmt, ctypes.POINTER(c_sz)]),
    "svdq_prepare_workspace_size": (c_i32, [c_i64, c_i64, c_i32, SvdqFmt, c_i32, ctypes.POINTER(c_sz)]),
    "svdq_prepare": (c_i32, [c_vp, c_i32, c_i64, c_i64, c_i64, c_vp, c_i32, SvdqFmt, c_u64,
                             c_i32, c_i32, c_vp, c_sz, ctypes.POINTER(SvdqWeight), c_vp]),
    "svdq_quantize_residual": (c_i32, [c_vp, c_i64, c_i64, c_i64, SvdqFmt, c_vp, c_vp, c_vp,
                                       c_vp, c_sz, c_vp]),
    "svdq_quantize_residual_workspace_size": (c_i32, [c_i64, c_i64, SvdqFmt, ctypes.POINTER(c_sz)]),
    "svdq_quantize_act": (c_i32, [c_vp, c_i32, c_i64, c_i64, c_i64, c_vp, SvdqFmt, c_vp, c_vp, c_vp,
                                  c_i32, c_vp, c_vp, c_vp, c_vp, c_vp, c_sz, c_vp]),
    "svdq_quantize_act_workspace_size": (c_i32, [c_i64, c_i64, SvdqFmt, c_i32, ctypes.POINTER(c_sz)]),
    "svdq_linear": (c_i32, [ctypes.POINTER(SvdqWeight), c_vp, c_i32, c_i64, c_i64, c_vp, c_vp,
                            c_vp, c_i32, c_i64, c_vp, c_sz, c_vp]),
    "svdq_linear_ex": (c_i32, [ctypes.POINTER(SvdqWeight), c_vp, c_i32, c_i64, c_i64, c_vp, c_vp,
                               c_vp, c_i32, c_i64, c_vp, c_sz, ctypes.c_uint32, c_vp]),
    "svdq_linear_workspace_size": (c_i32, [ctypes.POINTER(SvdqWeight), c_i64, ctypes.POINTER(c_sz)]),
    "svdq_residual_product_i32": (c_i32, [ctypes.POINTER(SvdqWeight), c_vp, c_i64, c_vp, c_i64, c_vp]),
    "svdq_residual_linear": (c_i32, [ctypes.POINTER(SvdqWeight), c_vp, c_vp, c_vp, c_vp, c_i64, c_vp,
                                     c_vp, c_i32, c_i64, c_vp]),
    "svdq_quantize_act_noalloc": (c_i32, [c_vp, c_i32, c_i64, c_i64, c_i64, c_vp, SvdqFmt, c_vp, c_vp,
                                          c_vp, c_i32, c_vp, c_vp, c_vp, c_vp, c_vp]),
    "svdq_pack_int4": (c_i32, [c_vp, c_i64, c_i64, c_vp, c_vp]),
    "svdq_check_status": (c_i32, [c_vp]),
    "svdq_selftest_wait_timeout": (c_i32, [c_i64, c_vp]),
}

_lib = None


def load_library(path: str = LIB_PATH):
    """Load libsvdq.so (raises if it has not been built) and set the signatures."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise ImportError(f"libsvdq.so not built at {path}; run python -m rank_bit_residual_b200.build")
    lib = ctypes.CDLL(path)
    for name, (res, args) in _SIGS.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


def header_functions(path: str = HEADER_PATH):
    """Names of the functions include/svdq.h declares."""
    text = open(path).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(svdq_[a-z0-9_]+)\s*\(", text)))


class SvdqError(RuntimeError):
    def __init__(self, status: int, what: str):
        lib = load_library()
        super().__init__(f"{what}: {lib.svdq_status_string(status).decode()} (status {status})")
        self.status = status


def _check(status: int, what: str):
    if status == SVDQ_OK:
        return
    if status in (SVDQ_EINVAL, SVDQ_ERANK):
        lib = load_library()
        raise ValueError(f"{what}: {lib.svdq_status_string(status).decode()}")
    raise SvdqError(status, what)


def parse_fmt(fmt) -> SvdqFmt:
    """'int4' / 'int8' / ... / 'nvfp4' / 'mxfp4', or (kind, bits)."""
    if isinstance(fmt, SvdqFmt):
        return fmt
    if isinstance(fmt, tuple):
        return SvdqFmt(*fmt)
    m = re.fullmatch(r"int([2-8])", str(fmt))
    if m:
        return SvdqFmt(KIND_INT, int(m.group(1)))
    if str(fmt) == "nvfp4":
        return SvdqFmt(KIND_NVFP4, 4)
    if str(fmt) == "mxfp4":
        return SvdqFmt(KIND_MXFP4, 4)
    raise ValueError(f"unknown format {fmt!r}")


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _dt(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return SVDQ_BF16
    if t.dtype == torch.float32:
        return SVDQ_F32
    raise ValueError(f"unsupported dtype {t.dtype}")


def _rows_ready(t: torch.Tensor) -> torch.Tensor:
    """A row-major view with unit inner stride and a 16-byte aligned pitch (copy if not)."""
    if t.dim() != 2:
        raise ValueError("expected a matrix")
    es = t.element_size()
    if t.stride(1) == 1 and (t.stride(0) * es) % 16 == 0 and t.data_ptr() % 16 == 0 and t.stride(0) >= t.shape[1]:
        return t
    return t.contiguous()


def _ptr(t: Optional[torch.Tensor]):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else ctypes.c_void_p(0)


def _require_cuda(*ts):
    for t in ts:
        if t is not None and not t.is_cuda:
            raise ValueError("tensors must live on a CUDA device")


def _check_rank_arg(rank):
    if isinstance(rank, bool) or not isinstance(rank, int):
        raise ValueError("rank must be a Python int")


@dataclass
class PreparedWeight:
    """The svdq_weight descriptor plus the torch buffers that back it."""
    desc: SvdqWeight
    codes: torch.Tensor
    sf: Optional[torch.Tensor]
    w_scale: torch.Tensor
    ld: torch.Tensor
    ld32: torch.Tensor
    lu: torch.Tensor
    scale: torch.Tensor
    codes4: Optional[torch.Tensor] = None

    @property
    def M(self):
        return self.desc.M

    @property
    def N(self):
        return self.desc.N

    @property
    def rank(self):
        return self.desc.rank

    @property
    def rank_pad(self):
        return self.desc.rank_pad

    @property
    def fmt(self):
        return (self.desc.fmt.kind, self.desc.fmt.bits)


def weight_buffer_sizes(M: int, N: int, rank: int, fmt):
    lib = load_library()
    sizes = (c_sz * 7)()
    _check(lib.svdq_weight_buffer_sizes(M, N, rank, parse_fmt(fmt), sizes), "svdq_weight_buffer_sizes")
    return list(sizes)


def allocate_weight(M: int, N: int, rank: int, fmt, scale: torch.Tensor) -> PreparedWeight:
    """Allocate (torch) the buffers of a prepared weight and fill the descriptor's pointers."""
    f = parse_fmt(fmt)
    sizes = weight_buffer_sizes(M, N, rank, f)
    dev = scale.device
    rp = (rank + 15) // 16 * 16
    codes = torch.empty(sizes[0], dtype=torch.uint8, device=dev)
    sf = torch.zeros(max(sizes[1], 1), dtype=torch.uint8, device=dev) if f.kind != KIND_INT else None
    w_scale = torch.zeros(4, dtype=torch.float32, device=dev)
    ld = torch.zeros((max(rp, 1), M), dtype=torch.bfloat16, device=dev)
    ld32 = torch.zeros((max(rp, 1), M), dtype=torch.float32, device=dev)
    lu = torch.zeros((N, max(2 * rp, 1)), dtype=torch.bfloat16, device=dev)
    codes4 = torch.empty(sizes[6], dtype=torch.uint8, device=dev) if sizes[6] else None
    d = SvdqWeight(M=M, N=N, rank=rank, rank_pad=rp, fmt=f,
                   codes=codes.data_ptr(), sf=sf.data_ptr() if sf is not None else None,
                   w_scale=w_scale.data_ptr(), ld=ld.data_ptr(), ld32=ld32.data_ptr(),
                   lu=lu.data_ptr(), scale=scale.data_ptr(),
                   codes4=codes4.data_ptr() if codes4 is not None else None)
    return PreparedWeight(d, codes, sf, w_scale, ld, ld32, lu, scale, codes4)


def weight_from_buffers(M, N, rank, fmt, codes, sf, w_scale, ld, ld32, lu, scale,
                        codes4=None) -> PreparedWeight:
    """Wrap caller-made device buffers (layouts of svdq_weight in include/svdq.h)."""
    f = parse_fmt(fmt)
    rp = (rank + 15) // 16 * 16
    d = SvdqWeight(M=M, N=N, rank=rank, rank_pad=rp, fmt=f, codes=codes.data_ptr(),
                   sf=sf.data_ptr() if sf is not None else None, w_scale=w_scale.data_ptr(),
                   ld=ld.data_ptr(), ld32=ld32.data_ptr() if ld32 is not None else None,
                   lu=lu.data_ptr(), scale=scale.data_ptr(),
                   codes4=codes4.data_ptr() if codes4 is not None else None)
    return PreparedWeight(d, codes, sf, w_scale, ld, ld32, lu, scale, codes4)


def svdq_pack_int4(codes: torch.Tensor) -> torch.Tensor:
    """INT codes int8 [N, M] -> the packed copy uint8 [N, M // 2] (svdq_weight.codes4)."""
    lib = load_library()
    _require_cuda(codes)
    N, M = codes.shape
    c = codes.contiguous()
    out = torch.empty((N, M // 2), dtype=torch.uint8, device=codes.device)
    _check(lib.svdq_pack_int4(_ptr(c), N, M, _ptr(out), _stream()), "svdq_pack_int4")
    return out


def svdq_prepare(W: torch.Tensor, scale: torch.Tensor, rank: int, fmt="int4", seed: int = 0,
                 oversample: int = 0, power_iters: int = 0) -> PreparedWeight:
    """One-time weight split (svdq_prepare in include/svdq.h). Synchronises the stream."""
    lib = load_library()
    _check_rank_arg(rank)
    _require_cuda(W, scale)
    if W.dim() != 2 or scale.dim() != 1:
        raise ValueError("W must be [M, N] and scale [M]")
    M, N = W.shape
    f = parse_fmt(fmt)
    W = _rows_ready(W)
    scale = scale.to(torch.float32).contiguous()
    wsz = c_sz()
    _check(lib.svdq_prepare_workspace_size(M, N, rank, f, oversample, ctypes.byref(wsz)),
           "svdq_prepare_workspace_size")
    w = allocate_weight(M, N, rank, f, scale)
    ws = torch.empty(wsz.value, dtype=torch.uint8, device=W.device)
    st = lib.svdq_prepare(_ptr(W), _dt(W), M, N, W.stride(0), _ptr(scale), rank, f, seed,
                          oversample, power_iters, _ptr(ws), wsz.value, ctypes.byref(w.desc), _stream())
    _check(st, "svdq_prepare")
    return w


def svdq_quantize_residual(R: torch.Tensor, fmt="int4"):
    """Quantise a residual R[M, N] (fp32): returns (codes, sf or None, w_scale)."""
    lib = load_library()
    _require_cuda(R)
    f = parse_fmt(fmt)
    R = _rows_ready(R.to(torch.float32))
    M, N = R.shape
    sizes = weight_buffer_sizes(M, N, 0, f)
    codes = torch.empty(sizes[0], dtype=torch.uint8, device=R.device)
    sf = torch.empty(max(sizes[1], 1), dtype=torch.uint8, device=R.device) if f.kind != KIND_INT else None
    w_scale = torch.zeros(1, dtype=torch.float32, device=R.device)
    wsz = c_sz()
    _check(lib.svdq_quantize_residual_workspace_size(M, N, f, ctypes.byref(wsz)), "workspace")
    ws = torch.empty(wsz.value, dtype=torch.uint8, device=R.device)
    _check(lib.svdq_quantize_residual(_ptr(R), M, N, R.stride(0), f, _ptr(codes), _ptr(sf),
                                      _ptr(w_scale), _ptr(ws), wsz.value, _stream()),
           "svdq_quantize_residual")
    if f.kind == KIND_INT:
        codes = codes.view(torch.int8).view(N, M)
    else:
        codes = codes.view(N, M // 2)
    return codes, sf, w_scale


def _act_buffers(B, M, f, rp, dev):
    if f.kind == KIND_INT:
        codes = torch.empty((B, M), dtype=torch.int8, device=dev)
        sf = None
    else:
        codes = torch.empty((B, M // 2), dtype=torch.uint8, device=dev)
        block = 32 if f.kind == KIND_MXFP4 else 16
        sf = torch.empty(max(((B + 127) // 128 * 128) * ((M // block + 3) // 4 * 4), 1),
                         dtype=torch.uint8, device=dev)
    act_scale = torch.zeros(1, dtype=torch.float32, device=dev)
    down = torch.empty((B, 2 * rp), dtype=torch.bfloat16, device=dev) if rp else None
    return codes, sf, act_scale, down


_act_ws = {}


def svdq_quantize_act_into(x: torch.Tensor, scale: torch.Tensor, fmt, ld: Optional[torch.Tensor],
                           codes: torch.Tensor, sf: Optional[torch.Tensor], act_scale: torch.Tensor,
                           down: Optional[torch.Tensor], act_global_scale: Optional[torch.Tensor] = None,
                           w_global_scale: Optional[torch.Tensor] = None):
    """svdq_quantize_act writing into caller buffers (shapes as returned by svdq_quantize_act)."""
    lib = load_library()
    f = parse_fmt(fmt)
    x = _rows_ready(x)
    B, M = x.shape
    rp = ld.shape[0] if ld is not None else 0
    key = (x.device, B, M, f.kind, rp)
    ws = _act_ws.get(key)
    if ws is None:
        wsz = c_sz()
        _check(lib.svdq_quantize_act_workspace_size(B, M, f, rp, ctypes.byref(wsz)), "workspace")
        ws = torch.empty(max(wsz.value, 1), dtype=torch.uint8, device=x.device)
        _act_ws[key] = ws
    _check(lib.svdq_quantize_act(_ptr(x), _dt(x), B, M, x.stride(0), _ptr(scale), f,
                                 _ptr(act_global_scale), _ptr(w_global_scale), _ptr(ld), rp,
                                 _ptr(codes), _ptr(sf),
                                 _ptr(act_scale), _ptr(down), _ptr(ws), ws.numel(), _stream()),
           "svdq_quantize_act")


def svdq_quantize_act(x: torch.Tensor, scale: torch.Tensor, fmt="int4", ld: Optional[torch.Tensor] = None,
                      act_global_scale: Optional[torch.Tensor] = None,
                      w_global_scale: Optional[torch.Tensor] = None):
    """Fused activation pass: returns (codes, sf or None, act_scale, down or None).

    ld is the [rank_pad, M] down factor (bf16 for bf16 x, fp32 for fp32 x); down is
    bf16 [B, 2 * rank_pad] (hi | lo). For NVFP4, down is multiplied by gs_x (and by
    w_global_scale when given), the units the NVFP4 GEMM accumulates in. MXFP4 has
    no global scales: act_scale is 1 and down is unscaled.
    """
    _require_cuda(x, scale)
    f = parse_fmt(fmt)
    x = _rows_ready(x)
    B, M = x.shape
    rp = ld.shape[0] if ld is not None else 0
    bufs = _act_buffers(B, M, f, rp, x.device)
    svdq_quantize_act_into(x, scale.contiguous(), f, ld, *bufs, act_global_scale=act_global_scale,
                           w_global_scale=w_global_scale)
    return bufs


def svdq_quantize_act_noalloc(x: torch.Tensor, scale: torch.Tensor, fmt="int4",
                              ld: Optional[torch.Tensor] = None,
                              act_global_scale: Optional[torch.Tensor] = None,
                              w_global_scale: Optional[torch.Tensor] = None):
    """The activation pass through svdq_quantize_act_noalloc.

    For callers whose runtime gives them no way to allocate device memory on the
    request path: the library passes no workspace and allocates nothing, using a
    fixed scratch array of its own (8 MiB per GPU, shared by all calls, so calls
    that overlap on the GPU must not be issued). Only the outputs are allocated
    here, on the caller's side. Returns (codes, sf or None, act_scale, down or None)
    like svdq_quantize_act.
    """
    lib = load_library()
    _require_cuda(x, scale)
    f = parse_fmt(fmt)
    x = _rows_ready(x)
    B, M = x.shape
    rp = ld.shape[0] if ld is not None else 0
    codes, sf, act_scale, down = _act_buffers(B, M, f, rp, x.device)
    _check(lib.svdq_quantize_act_noalloc(_ptr(x), _dt(x), B, M, x.stride(0), _ptr(scale.contiguous()), f,
                                         _ptr(act_global_scale), _ptr(w_global_scale), _ptr(ld), rp,
                                         _ptr(codes), _ptr(sf), _ptr(act_scale), _ptr(down), _stream()),
           "svdq_quantize_act_noalloc")
    return codes, sf, act_scale, down


class LinearWorkspace:
    """Reusable scratch for svdq_linear (one per stream in flight)."""

    def __init__(self):
        self.buf = None

    def get(self, nbytes: int, device) -> torch.Tensor:
        if self.buf is None or self.buf.numel() < nbytes or self.buf.device != device:
            self.buf = torch.empty(max(nbytes, 1), dtype=torch.uint8, device=device)
        return self.buf


_default_ws = LinearWorkspace()


def linear_workspace_size(w: PreparedWeight, B: int) -> int:
    lib = load_library()
    wsz = c_sz()
    _check(lib.svdq_linear_workspace_size(ctypes.byref(w.desc), B, ctypes.byref(wsz)), "workspace")
    return wsz.value


def svdq_linear(w: PreparedWeight, x: torch.Tensor, bias: Optional[torch.Tensor] = None,
                out_dtype=torch.bfloat16, act_global_scale: Optional[torch.Tensor] = None,
                out: Optional[torch.Tensor] = None, workspace: Optional[LinearWorkspace] = None,
                pdl: bool = False):
    """Y[B, N] = x ld^T lu^T + alpha Q(X_hat) Q(R) (+ bias) on the current stream.

    pdl=True (svdq_linear_ex with SVDQ_LINEAR_PDL): the activation pass starts as a
    programmatic dependent of the kernel queued before it (the previous linear's
    GEMM, whose output is x) and reads x only once that kernel has finished. w's
    buffers and the bias must not be written by work still in flight on the stream.
    """
    lib = load_library()
    _require_cuda(x)
    x = _rows_ready(x)
    B, M = x.shape
    if M != w.M:
        raise ValueError("x[B, M] does not match the prepared weight's M")
    if bias is not None:
        _require_cuda(bias)
        bias = bias.to(torch.bfloat16).contiguous()
        if bias.shape != (w.N,):
            raise ValueError("bias must be [N]")
    y = out if out is not None else torch.empty((B, w.N), dtype=out_dtype, device=x.device)
    nbytes = linear_workspace_size(w, B)
    ws = (workspace or _default_ws).get(nbytes, x.device)
    if pdl:
        _check(lib.svdq_linear_ex(ctypes.byref(w.desc), _ptr(x), _dt(x), B, x.stride(0), _ptr(bias),
                                  _ptr(act_global_scale), _ptr(y), _dt(y), y.stride(0), _ptr(ws),
                                  ws.numel(), SVDQ_LINEAR_PDL, _stream()), "svdq_linear_ex")
    else:
        _check(lib.svdq_linear(ctypes.byref(w.desc), _ptr(x), _dt(x), B, x.stride(0), _ptr(bias),
                               _ptr(act_global_scale), _ptr(y), _dt(y), y.stride(0), _ptr(ws), ws.numel(),
                               _stream()), "svdq_linear")
    return y


def svdq_linear_chain(weights, x: torch.Tensor, biases=None, out_dtype=torch.bfloat16,
                      pdl: bool = True, workspace: Optional[LinearWorkspace] = None,
                      outs=None) -> torch.Tensor:
    """Consecutive linears y_i = linear(w_i, y_{i-1}) (y_0 = x) on the current stream,
    every call after the first chained to the one before with PDL (pdl=True). Each
    intermediate y is in out_dtype (bf16 by default); ``outs`` may hold
    preallocated outputs, one per linear."""
    biases = biases if biases is not None else [None] * len(weights)
    ws = workspace or LinearWorkspace()
    y = x
    for i, (w, b) in enumerate(zip(weights, biases)):
        y = svdq_linear(w, y, bias=b, out_dtype=out_dtype, workspace=ws, pdl=pdl and i > 0,
                        out=outs[i] if outs is not None else None)
    return y


def svdq_residual_linear(w: PreparedWeight, act_codes: torch.Tensor, act_sf: Optional[torch.Tensor],
                         act_scale: torch.Tensor, down: Optional[torch.Tensor],
                         bias: Optional[torch.Tensor] = None, out_dtype=torch.bfloat16,
                         out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """GEMM stage alone: Y from the outputs of svdq_quantize_act (current stream)."""
    lib = load_library()
    _require_cuda(act_codes, act_scale)
    B = act_codes.shape[0]
    y = out if out is not None else torch.empty((B, w.N), dtype=out_dtype, device=act_codes.device)
    if bias is not None:
        bias = bias.to(torch.bfloat16).contiguous()
    _check(lib.svdq_residual_linear(ctypes.byref(w.desc), _ptr(act_codes), _ptr(act_sf), _ptr(act_scale),
                                    _ptr(down), B, _ptr(bias), _ptr(y), _dt(y), y.stride(0), _stream()),
           "svdq_residual_linear")
    return y


def svdq_residual_product_i32(w: PreparedWeight, act_codes: torch.Tensor) -> torch.Tensor:
    """Exact int32 product act_codes[B, M] . codes[N, M]^T of the INT residual branch."""
    lib = load_library()
    _require_cuda(act_codes)
    a = act_codes.contiguous()
    B = a.shape[0]
    acc = torch.empty((B, w.N), dtype=torch.int32, device=a.device)
    _check(lib.svdq_residual_product_i32(ctypes.byref(w.desc), _ptr(a), B, _ptr(acc), w.N, _stream()),
           "svdq_residual_product_i32")
    return acc


def svdq_smooth_scale(x: torch.Tensor, W: torch.Tensor, alpha: float = 0.5) -> torch.Tensor:
    """Per-channel smoothing scale max|x[:, j]|^alpha / max|W[j, :]|^(1 - alpha) (fp32 [M])."""
    lib = load_library()
    _require_cuda(x, W)
    if x.dim() != 2 or W.dim() != 2 or x.shape[1] != W.shape[0]:
        raise ValueError("x must be [B, M] and W [M, N]")
    x = _rows_ready(x)
    W = _rows_ready(W)
    M, N = W.shape
    scale = torch.empty(M, dtype=torch.float32, device=W.device)
    ws = torch.empty(8 * M, dtype=torch.uint8, device=W.device)
    _check(lib.svdq_smooth_scale(_ptr(x), _dt(x), x.shape[0], M, x.stride(0), _ptr(W), _dt(W), N, W.stride(0),
                                 float(alpha), _ptr(scale), _ptr(ws), ws.numel(), _stream()), "svdq_smooth_scale")
    return scale


def svdq_fold_scale(x: torch.Tensor, W: torch.Tensor, bits: int = 4) -> torch.Tensor:
    """Per-channel smoothing scale of the optimal diagonal fold of x @ W under per-tensor
    INT grids of `bits` (the geometric program of svdq_fold_scale; fp32 [M])."""
    lib = load_library()
    _require_cuda(x, W)
    if x.dim() != 2 or W.dim() != 2 or x.shape[1] != W.shape[0]:
        raise ValueError("x must be [B, M] and W [M, N]")
    x = _rows_ready(x)
    W = _rows_ready(W)
    B, M = x.shape
    N = W.shape[1]
    nb = c_sz(0)
    _check(lib.svdq_fold_scale_workspace_size(B, M, ctypes.byref(nb)), "svdq_fold_scale_workspace_size")
    scale = torch.empty(M, dtype=torch.float32, device=W.device)
    ws = torch.empty(nb.value, dtype=torch.uint8, device=W.device)
    _check(lib.svdq_fold_scale(_ptr(x), _dt(x), B, M, x.stride(0), _ptr(W), _dt(W), N, W.stride(0), int(bits),
                               _ptr(scale), _ptr(ws), ws.numel(), _stream()), "svdq_fold_scale")
    return scale


def svdq_check_status() -> int:
    """Synchronise the current stream and return (and clear) the device status word."""
    return load_library().svdq_check_status(_stream())


def svdq_selftest_wait_timeout(limit_us: int = 1000) -> int:
    """Run a bounded wait on a flag nothing sets; returns the status (SVDQ_ETIMEOUT expected)."""
    return load_library().svdq_selftest_wait_timeout(limit_us, _stream())


__all__ = [
    "svdq_prepare", "svdq_quantize_act", "svdq_quantize_act_into", "svdq_quantize_act_noalloc",
    "svdq_quantize_residual", "svdq_linear", "svdq_linear_chain", "svdq_pack_int4", "svdq_fold_scale",
    "svdq_residual_product_i32", "svdq_residual_linear", "svdq_check_status", "svdq_selftest_wait_timeout",
    "svdq_smooth_scale",
    "PreparedWeight", "LinearWorkspace", "allocate_weight", "weight_from_buffers",
    "weight_buffer_sizes", "load_library", "header_functions", "parse_fmt",
]
