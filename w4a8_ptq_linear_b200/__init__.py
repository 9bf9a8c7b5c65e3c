"""Python binding of the rotated, quantized linear layer's C ABI (include/oq.h).

This module only marshals arguments: it turns torch tensors into device pointers and the
current CUDA stream into a ``cudaStream_t``, allocates outputs with torch, and calls the
shared library ``lib/liboq.so``. Every step of the layer runs in the library's kernels.
There is no CPU fallback: if the library is missing, importing works but every compute
call raises ``OQError``.

The function names follow the C ABI: ``rotate_quantize``, ``prepare_weights``,
``gemm_w4a8``, ``gemm_w4a4``, ``gemm_w4a2``, ``linear`` (oq_rotate_quantize, oq_prepare_weights, ...).
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import numpy as np

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "lib", "liboq.so")
# the bounds-checked build (python -m w4a8_ptq_linear_b200.build --checked)
LIB_CHECKED_PATH = os.path.join(_PKG, "lib", "liboq_checked.so")

OQ_OK, OQ_ERR_INVALID_ARG, OQ_ERR_UNSUPPORTED, OQ_ERR_MISALIGNED = 0, 1, 2, 3
OQ_ERR_CUDA, OQ_ERR_DEVICE_TIMEOUT, OQ_ERR_NOMEM = 4, 5, 6
ACT_KINDS = {"int8_absmax": 0, "int4_absmax": 1, "int4_lloydmax": 2, "int4_percentile": 3,
             "int4_lloydmax_width": 4, "int8_lloydmax": 5, "int2_percentile": 6}
OUT_BF16, OUT_ACC = 0, 1

# (name, restype, argtypes) of every exported entry point
_P, _I, _I64, _U64, _SZ, _D = (ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_uint64,
                               ctypes.c_size_t, ctypes.c_double)
SIGNATURES = [
    ("oq_status_string", ctypes.c_char_p, [_I]),
    ("oq_last_error", ctypes.c_char_p, []),
    ("oq_device_status", _I, [_I, ctypes.POINTER(_U64)]),
    ("oq_default_block", _I, [_I]),
    ("oq_default_rounds", _I, [_I]),
    ("oq_rpbh_tables", _I, [_I, _I, _U64, _P, _P]),
    ("oq_lloyd_max_codebook", _I, [_P, _P]),
    ("oq_lloyd_max_codebook_width", _I, [_I, _P, _P]),
    ("oq_lloyd_max_codebook_8bit", _I, [_P, _P]),
    ("oq_plan_create", _I, [ctypes.POINTER(_P), _I, _I, _I, _U64, _I, _I]),
    ("oq_plan_destroy", None, [_P]),
    ("oq_plan_get_rpbh", _I, [_P, _I, _P, _P]),
    ("oq_plan_get_codebook", _I, [_P, _I, _P, _P]),
    ("oq_rotate_quantize", _I, [_P, _P, _I64, _I64, _P, _P, _P, _P, _P]),
    ("oq_prepare_weights", _I, [_P, _P, _I64, _I64, _P, _P, _P, _P]),
    ("oq_gemm_w4a8", _I, [_P, _P, _P, _P, _P, _P, _P, _I64, _I64, _I64, _I, _P, _P]),
    ("oq_gemm_w4a4", _I, [_P, _I, _P, _P, _P, _P, _P, _P, _P, _I64, _I64, _I64, _I, _P, _P]),
    ("oq_gemm_w4a2", _I, [_P, _P, _P, _P, _P, _P, _P, _I64, _I64, _I64, _I, _P, _P]),
    ("oq_gemm_w4a8_lloydmax", _I, [_P, _P, _P, _P, _P, _P, _P, _P, _I64, _I64, _I64, _I, _P, _P]),
    ("oq_linear_workspace_bytes", _SZ, [_P, _I64]),
    ("oq_linear", _I, [_P, _P, _I64, _I64, _P, _P, _P, _P, _I64, _P, _P, _SZ, _P]),
    ("oq_debug_wait_timeout", _I, [_U64, _P]),
    ("oq_prepare_weights_g64", _I, [_P, _P, _I64, _I64, _P, _P, _P, _P, _P]),
    ("oq_gemm_w4a4_g64", _I, [_I, _P, _P, _P, _P, _P, _P, _P, _P, _I64, _I64, _I64, _I, _P, _P]),
    ("oq_linear_g64", _I, [_P, _P, _I64, _I64, _P, _P, _P, _P, _P, _I64, _P, _P, _SZ, _P]),
    ("oq_linear_fused", _I, [_P, _P, _I64, _I64, _P, _P, _P, _P, _I64, _P, _P, _SZ, _P]),
    ("oq_linear_static_scratch", _I, [_P, _P, _I64, _I64, _P, _P, _P, _P, _I64, _P, _P]),
    ("oq_mma_peak_loop", _I, [_I, _I64, _P, _P]),
    ("oq_debug_pair_layout", _I, [_I, _I, _U64, _P]),
]


class OQError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"{_status_name(status)}: {msg}")
        self.status = status


_lib = None


def _status_name(s: int) -> str:
    names = {0: "OQ_OK", 1: "OQ_ERR_INVALID_ARG", 2: "OQ_ERR_UNSUPPORTED",
             3: "OQ_ERR_MISALIGNED", 4: "OQ_ERR_CUDA", 5: "OQ_ERR_DEVICE_TIMEOUT",
             6: "OQ_ERR_NOMEM"}
    return names.get(s, f"status {s}")


def load(path: str):
    """A ctypes handle on a build of the library at `path`, with every signature set."""
    if not os.path.exists(path):
        raise OQError(OQ_ERR_UNSUPPORTED,
                      f"{path} is not built: run python -m w4a8_ptq_linear_b200.build")
    L = ctypes.CDLL(path)
    for name, res, args in SIGNATURES:
        f = getattr(L, name)
        f.restype = res
        f.argtypes = args
    return L


def lib():
    """The loaded ctypes library; raises OQError if it is not built."""
    global _lib
    if _lib is None:
        _lib = load(LIB_PATH)
    return _lib


class using:
    """Within the block, every call of this module goes to the library build `handle` (for
    example ``load(LIB_CHECKED_PATH)``); plans must be created and used inside one build."""

    def __init__(self, handle):
        self.handle = handle

    def __enter__(self):
        global _lib
        self.saved = lib()
        _lib = self.handle
        return self.handle

    def __exit__(self, *exc):
        global _lib
        _lib = self.saved


def _check(status: int):
    if status != OQ_OK:
        raise OQError(status, lib().oq_last_error().decode())


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    import torch
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def device_status(clear: bool = True):
    """(status, code) of the device error word; synchronizes the current device."""
    code = ctypes.c_uint64(0)
    st = lib().oq_device_status(1 if clear else 0, ctypes.byref(code))
    return st, code.value


def default_block(d: int) -> int:
    return lib().oq_default_block(d)


def default_rounds(h: int) -> int:
    return lib().oq_default_rounds(h)


def rpbh_tables(d: int, round_: int, seed: int):
    """Host RPBH tables of one round: (signs int8[d], perm int32[d])."""
    s = np.empty(d, np.int8)
    p = np.empty(d, np.int32)
    _check(lib().oq_rpbh_tables(d, round_, seed, s.ctypes.data, p.ctypes.data))
    return s, p


def lloyd_max_codebook():
    """The library's Newton-solved N(0,1) codebook: (centroids[16], thresholds[15])."""
    c = np.empty(16, np.float64)
    t = np.empty(15, np.float64)
    _check(lib().oq_lloyd_max_codebook(c.ctypes.data, t.ctypes.data))
    return c, t


def lloyd_max_codebook_8bit():
    """The library's Newton-solved 256-level N(0,1) codebook: (centroids, thresholds)."""
    c = np.empty(256, np.float64)
    t = np.empty(255, np.float64)
    _check(lib().oq_lloyd_max_codebook_8bit(c.ctypes.data, t.ctypes.data))
    return c, t


def lloyd_max_codebook_width(d: int):
    """The library's Newton-solved codebook of the width-d marginal: (centroids, thresholds)."""
    c = np.empty(16, np.float64)
    t = np.empty(15, np.float64)
    _check(lib().oq_lloyd_max_codebook_width(d, c.ctypes.data, t.ctypes.data))
    return c, t


@dataclass
class Plan:
    """An RPBH plan on the current CUDA device (oq_plan_create / oq_plan_destroy)."""
    d: int
    h: int
    rounds: int
    seed: int = 0
    center: bool = False
    act: str = "int8_absmax"

    def __post_init__(self):
        h = ctypes.c_void_p()
        _check(lib().oq_plan_create(ctypes.byref(h), self.d, self.h, self.rounds, self.seed,
                                    1 if self.center else 0, ACT_KINDS[self.act]))
        self._h = h

    @property
    def handle(self):
        return self._h

    def close(self):
        if getattr(self, "_h", None) and self._h.value:
            lib().oq_plan_destroy(self._h)
            self._h = ctypes.c_void_p()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def __enter__(self):
        return self

    def __exit__(self, *exc):
        self.close()

    def rpbh(self, round_: int):
        s = np.empty(self.d, np.int8)
        p = np.empty(self.d, np.int32)
        _check(lib().oq_plan_get_rpbh(self._h, round_, s.ctypes.data, p.ctypes.data))
        return s, p

    def codebook(self):
        """The plan's Lloyd-Max codebook (oq_plan_get_codebook): (centroids, thresholds),
        16 or 256 levels by the plan's activation kind."""
        levels = 256 if self.act == "int8_lloydmax" else 16
        c = np.empty(levels, np.float64)
        t = np.empty(levels - 1, np.float64)
        _check(lib().oq_plan_get_codebook(self._h, levels, c.ctypes.data, t.ctypes.data))
        return c, t

    @property
    def packed(self) -> bool:
        return self.act not in ("int8_absmax", "int8_lloydmax")

    @property
    def code_row_bytes(self) -> int:
        """Bytes of one token's codes: d (8-bit kinds), d/2 (4-bit) or d/4 (2-bit)."""
        if not self.packed:
            return self.d
        return self.d // 4 if self.act == "int2_percentile" else self.d // 2

    def workspace_bytes(self, T: int) -> int:
        return int(lib().oq_linear_workspace_bytes(self._h, T))


def rotate_quantize(plan: Plan, x, *, codes=None, scale=None, mean=None, rotated=False,
                    stream=None):
    """oq_rotate_quantize on a bf16 [T, d] CUDA tensor.

    Returns (codes, scale, mean or None, rotated float32 [T, d] or None)."""
    import torch
    T, ldx = x.shape[0], x.stride(0)
    dev = x.device
    if codes is None:
        codes = torch.empty((T, plan.code_row_bytes),
                            dtype=torch.int8 if plan.act == "int8_absmax" else torch.uint8,
                            device=dev)
    if scale is None:
        scale = torch.empty(T, dtype=torch.float32, device=dev)
    if plan.center and mean is None:
        mean = torch.empty(T, dtype=torch.float32, device=dev)
    rot = torch.empty((T, plan.d), dtype=torch.float32, device=dev) if rotated else None
    _check(lib().oq_rotate_quantize(plan.handle, _ptr(x), T, ldx, _ptr(codes), _ptr(scale),
                                    _ptr(mean) if plan.center else None, _ptr(rot),
                                    _stream(stream)))
    return codes, scale, (mean if plan.center else None), rot


def prepare_weights(plan: Plan, w, *, stream=None):
    """oq_prepare_weights on a bf16 [n_out, d] CUDA tensor: (w_packed, w_scale, w_rowsum)."""
    import torch
    n = w.shape[0]
    wp = torch.empty((n, plan.d // 2), dtype=torch.uint8, device=w.device)
    ws = torch.empty(n, dtype=torch.float32, device=w.device)
    w1 = torch.empty(n, dtype=torch.float32, device=w.device)
    _check(lib().oq_prepare_weights(plan.handle, _ptr(w), n, w.stride(0), _ptr(wp), _ptr(ws),
                                    _ptr(w1), _stream(stream)))
    return wp, ws, w1


def _out(T, N, out_kind, acc_dtype, dev, out):
    import torch
    if out is not None:
        return out
    dt = torch.bfloat16 if out_kind == OUT_BF16 else acc_dtype
    return torch.empty((T, N), dtype=dt, device=dev)


def gemm_w4a8(a, a_scale, w_packed, w_scale, *, mean=None, w_rowsum=None, bias=None,
              out_kind=OUT_BF16, out=None, stream=None):
    """oq_gemm_w4a8: int8 [T, K] codes x packed INT4 [N, K/2] weights."""
    import torch
    T, K = a.shape
    N = w_packed.shape[0]
    out = _out(T, N, out_kind, torch.int32, a.device, out)
    _check(lib().oq_gemm_w4a8(_ptr(a), _ptr(a_scale), _ptr(mean), _ptr(w_packed), _ptr(w_scale),
                              _ptr(w_rowsum), _ptr(bias), T, K, N, out_kind, _ptr(out),
                              _stream(stream)))
    return out


def gemm_w4a4(plan, kind, a_packed, a_scale, w_packed, w_scale, *, mean=None, w_rowsum=None,
              bias=None, out_kind=OUT_BF16, out=None, stream=None):
    """oq_gemm_w4a4: packed 4-bit [T, K/2] codes (absmax or Lloyd-Max) x packed INT4."""
    import torch
    T, K = a_packed.shape[0], a_packed.shape[1] * 2
    N = w_packed.shape[0]
    acc_dt = torch.float32 if kind.startswith("int4_lloydmax") else torch.int32
    out = _out(T, N, out_kind, acc_dt, a_packed.device, out)
    _check(lib().oq_gemm_w4a4(plan.handle if plan is not None else None, ACT_KINDS[kind],
                              _ptr(a_packed), _ptr(a_scale), _ptr(mean), _ptr(w_packed),
                              _ptr(w_scale), _ptr(w_rowsum), _ptr(bias), T, K, N, out_kind,
                              _ptr(out), _stream(stream)))
    return out


def gemm_w4a2(a_packed, a_scale, w_packed, w_scale, *, mean=None, w_rowsum=None, bias=None,
              out_kind=OUT_BF16, out=None, stream=None):
    """oq_gemm_w4a2: 2-bit codes [T, K/4] (four per byte) x packed INT4 [N, K/2] weights."""
    import torch
    T, K = a_packed.shape[0], a_packed.shape[1] * 4
    N = w_packed.shape[0]
    out = _out(T, N, out_kind, torch.int32, a_packed.device, out)
    _check(lib().oq_gemm_w4a2(_ptr(a_packed), _ptr(a_scale), _ptr(mean), _ptr(w_packed),
                              _ptr(w_scale), _ptr(w_rowsum), _ptr(bias), T, K, N, out_kind,
                              _ptr(out), _stream(stream)))
    return out


def gemm_w4a8_lloydmax(plan, codes, sigma, w_packed, w_scale, *, mean=None, w_rowsum=None,
                       bias=None, out_kind=OUT_BF16, out=None, stream=None):
    """oq_gemm_w4a8_lloydmax: uint8 [T, K] 8-bit Lloyd-Max codes x packed INT4."""
    import torch
    T, K = codes.shape
    N = w_packed.shape[0]
    out = _out(T, N, out_kind, torch.float32, codes.device, out)
    _check(lib().oq_gemm_w4a8_lloydmax(plan.handle, _ptr(codes), _ptr(sigma), _ptr(mean),
                                       _ptr(w_packed), _ptr(w_scale), _ptr(w_rowsum), _ptr(bias),
                                       T, K, N, out_kind, _ptr(out), _stream(stream)))
    return out


def linear(plan: Plan, x, w_packed, w_scale, w_rowsum=None, bias=None, *, workspace=None,
           out=None, stream=None):
    """oq_linear: the whole layer on a bf16 [T, d] CUDA tensor -> bf16 [T, N]."""
    import torch
    T = x.shape[0]
    N = w_packed.shape[0]
    need = plan.workspace_bytes(T)
    if workspace is None:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=x.device)
    if out is None:
        out = torch.empty((T, N), dtype=torch.bfloat16, device=x.device)
    _check(lib().oq_linear(plan.handle, _ptr(x), T, x.stride(0), _ptr(w_packed), _ptr(w_scale),
                           _ptr(w_rowsum), _ptr(bias), N, _ptr(out), _ptr(workspace),
                           workspace.numel() * workspace.element_size(), _stream(stream)))
    return out


def linear_fused(plan: Plan, x, w_packed, w_scale, w_rowsum=None, bias=None, *, workspace=None,
                 out=None, stream=None):
    """oq_linear_fused: the whole layer in one launch (T <= 256; INT8 absmax, INT4 absmax and
    INT4 percentile plans)."""
    import torch
    T = x.shape[0]
    N = w_packed.shape[0]
    need = plan.workspace_bytes(T)
    if workspace is None:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=x.device)
    if out is None:
        out = torch.empty((T, N), dtype=torch.bfloat16, device=x.device)
    _check(lib().oq_linear_fused(plan.handle, _ptr(x), T, x.stride(0), _ptr(w_packed),
                                 _ptr(w_scale), _ptr(w_rowsum), _ptr(bias), N, _ptr(out),
                                 _ptr(workspace), workspace.numel() * workspace.element_size(),
                                 _stream(stream)))
    return out


def prepare_weights_g64(plan: Plan, w, *, stream=None):
    """oq_prepare_weights_g64 on a bf16 [n_out, d] CUDA tensor: asymmetric INT4 groups of 64.

    Returns (w_packed uint8 [n, d/2]: Q - 8 nibbles in the GEMM layout, K order 0, 2, 1, 3
    inside every four columns; w_sz int32 [d/64, n] of fp16 (sigma, z) pairs; w_scale float32
    [n] (ones); w_rowsum float32 [n])."""
    import torch
    n = w.shape[0]
    wp = torch.empty((n, plan.d // 2), dtype=torch.uint8, device=w.device)
    wsz = torch.empty((plan.d // 64, n), dtype=torch.int32, device=w.device)
    ws = torch.empty(n, dtype=torch.float32, device=w.device)
    w1 = torch.empty(n, dtype=torch.float32, device=w.device)
    _check(lib().oq_prepare_weights_g64(plan.handle, _ptr(w), n, w.stride(0), _ptr(wp), _ptr(wsz),
                                        _ptr(ws), _ptr(w1), _stream(stream)))
    return wp, wsz, ws, w1


def gemm_w4a4_g64(kind, a_packed, a_scale, w_packed, w_sz, w_scale, *, mean=None, w_rowsum=None,
                  bias=None, out_kind=OUT_BF16, out=None, stream=None):
    """oq_gemm_w4a4_g64: packed INT4 [T, K/2] codes x asymmetric grouped INT4 weights."""
    import torch
    T, K = a_packed.shape[0], a_packed.shape[1] * 2
    N = w_packed.shape[0]
    out = _out(T, N, out_kind, torch.float32, a_packed.device, out)
    _check(lib().oq_gemm_w4a4_g64(ACT_KINDS[kind], _ptr(a_packed), _ptr(a_scale), _ptr(mean),
                                  _ptr(w_packed), _ptr(w_sz), _ptr(w_scale), _ptr(w_rowsum),
                                  _ptr(bias), T, K, N, out_kind, _ptr(out), _stream(stream)))
    return out


def linear_g64(plan: Plan, x, w_packed, w_sz, w_scale, w_rowsum=None, bias=None, *,
               workspace=None, out=None, stream=None):
    """oq_linear_g64: the whole layer against asymmetric grouped weights -> bf16 [T, N]."""
    import torch
    T = x.shape[0]
    N = w_packed.shape[0]
    need = plan.workspace_bytes(T)
    if workspace is None:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=x.device)
    if out is None:
        out = torch.empty((T, N), dtype=torch.bfloat16, device=x.device)
    _check(lib().oq_linear_g64(plan.handle, _ptr(x), T, x.stride(0), _ptr(w_packed), _ptr(w_sz),
                               _ptr(w_scale), _ptr(w_rowsum), _ptr(bias), N, _ptr(out),
                               _ptr(workspace), workspace.numel() * workspace.element_size(),
                               _stream(stream)))
    return out


def linear_static_scratch(plan: Plan, x, w_packed, w_scale, w_rowsum=None, bias=None, *,
                          out=None, stream=None):
    """oq_linear_static_scratch: the whole layer without a caller workspace.

    For callers that cannot allocate device scratch (plug-ins inside a framework that owns all
    device memory, or paths that may not call cudaMalloc). The scratch is a 16 MiB array inside
    the library, shared by every call on the device; calls that overlap on the GPU race on it.
    T is limited to what fits that array. Make the first call on a device before any capture.
    """
    import torch
    T = x.shape[0]
    N = w_packed.shape[0]
    if out is None:
        out = torch.empty((T, N), dtype=torch.bfloat16, device=x.device)
    _check(lib().oq_linear_static_scratch(plan.handle, _ptr(x), T, x.stride(0), _ptr(w_packed),
                                          _ptr(w_scale), _ptr(w_rowsum), _ptr(bias), N,
                                          _ptr(out), _stream(stream)))
    return out


def mma_peak_loop(kind: str, iters: int, stream=None) -> int:
    """oq_mma_peak_loop: launches the tensor-core peak loop (kind "i8", "f16", or "i8_serial":
    each group of four MMAs waited for before the next) on the stream; returns the number of
    CTA pairs, from which the operation count follows."""
    pairs = ctypes.c_int(0)
    _check(lib().oq_mma_peak_loop({"i8": 0, "f16": 1, "i8_serial": 2}[kind], iters,
                                  ctypes.byref(pairs), _stream(stream)))
    return pairs.value


def debug_pair_layout(d: int, h: int, seed: int = 0):
    """oq_debug_pair_layout: the word of every channel in the two-token kernel's
    interleaved row (int32[d])."""
    w = np.empty(d, np.int32)
    _check(lib().oq_debug_pair_layout(d, h, seed, w.ctypes.data))
    return w


def debug_wait_timeout(timeout_ns: int, stream=None):
    """Launch a kernel whose bounded wait must give up (tests the error path)."""
    _check(lib().oq_debug_wait_timeout(timeout_ns, _stream(stream)))
