"""Python binding of the w4a16 C-ABI library (libw4a16.so, sm_100a).

Argument marshalling only: every entry point checks dtypes, shapes and
contiguity of the torch tensors it is given, then calls the C function of the
same name with raw device pointers and the current CUDA stream.  All compute
runs in the library's CUDA kernels; there is no CPU path.  If the shared
library is missing, ``load()`` raises -- build it with
``python -m weight_only_int4_linear_b200.build``.

Tensor conventions (torch dtypes standing in for the C types):
  X, Y, scales, W_hat : torch.bfloat16      (uint16_t bit patterns in C)
  qweight             : torch.int32 holding uint32 words (8 codes each, low nibble = lowest k)
  zeros               : torch.int32
  W                   : torch.float32
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libw4a16.so")
GROUP = 128

OK = 0
ERR_ARG = 1
ERR_ALIGN = 2
ERR_SHAPE = 3
ERR_DEVICE = 4
ERR_WORKSPACE = 5
ERR_CUDA = 6
ERR_NONFINITE = 7
ERR_ZERO_RANGE = 8

PATH_AUTO = 0
PATH_DECODE = 1
PATH_PREFILL = 2

_lib = None

# C signatures: name -> (restype, argtypes)
_i64, _vp, _int, _sz = ctypes.c_int64, ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
SIGNATURES = {
    "w4a16_status_string": (ctypes.c_char_p, [_int]),
    "w4a16_version": (_int, []),
    "w4a16_quantize_pack": (_int, [_vp, _i64, _i64, _vp, _vp, _vp, _vp, _vp]),
    "w4a16_quantize_pack_sym": (_int, [_vp, _i64, _i64, _vp, _vp, _vp, _vp, _vp]),
    "w4a16_workspace_bytes": (_sz, [_i64, _i64, _i64]),
    "w4a16_workspace_init": (_int, [_vp, _sz, _vp]),
    "w4a16_linear": (_int, [_vp, _i64, _i64, _vp, _vp, _vp, _i64, _vp, _vp, _sz, _vp]),
    "w4a16_linear_path": (_int, [_vp, _i64, _i64, _vp, _vp, _vp, _i64, _vp, _vp, _sz, _int, _vp]),
    "w4a16_linear_awq": (_int, [_vp, _vp, _i64, _i64, _vp, _vp, _vp, _i64, _vp, _vp, _sz, _int, _vp]),
    "w4a16_quantize_pack_awq": (_int, [_vp, _vp, _i64, _i64, _vp, _vp, _vp, _vp, _vp]),
    "w4a16_quantize_pack_g": (_int, [_vp, _i64, _i64, _int, _int, _vp, _vp, _vp, _vp, _vp]),
    "w4a16_workspace_bytes_g": (_sz, [_i64, _i64, _i64, _int]),
    "w4a16_linear_g": (_int, [_vp, _i64, _i64, _int, _vp, _vp, _vp, _i64, _vp, _vp, _sz, _vp]),
    "w8a16_quantize": (_int, [_vp, _i64, _i64, _vp, _vp, _vp, _vp]),
    "w8a16_dequant": (_int, [_vp, _vp, _i64, _i64, _vp, _vp]),
    "w8a16_workspace_bytes": (_sz, [_i64, _i64, _i64]),
    "w8a16_linear": (_int, [_vp, _i64, _i64, _vp, _vp, _i64, _vp, _vp, _sz, _vp]),
    "w4a16_linear_host": (_int, [_vp, _vp, _i64, _i64, _vp, _vp, _vp, _i64, _vp, _vp, _vp, _sz, _vp]),
    "w4a16_unpack": (_int, [_vp, _i64, _i64, _vp, _vp]),
    "w4a16_dequant": (_int, [_vp, _vp, _vp, _i64, _i64, _vp, _vp]),
    "w4a16_dequant_codes": (_int, [_vp, _vp, _vp, _i64, _i64, _vp, _vp]),
    "w4a16_renorm_rows": (_int, [_vp, _i64, _i64, _vp, _vp]),
    "w4a16_device_fault": (_int, []),
    "w4a16_selftest_wait": (_int, [_i64, _vp]),
    "w4a16_linear_noalloc": (_int, [_vp, _i64, _i64, _vp, _vp, _vp, _i64, _vp, _vp]),
    "w4a16_noalloc_scratch_bytes": (_sz, []),
}


class W4A16Error(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        super().__init__(f"{fn}: {status_string(status)} (status {status})")


def load():
    """Load libw4a16.so (raises if it is missing: there is no fallback)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"CUDA library not built: {LIB_PATH} is missing "
                               "(run python -m weight_only_int4_linear_b200.build)")
        lib = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
    return _lib


def status_string(status: int) -> str:
    return load().w4a16_status_string(status).decode()


def version() -> int:
    return int(load().w4a16_version())


def _check(fn: str, st: int) -> None:
    if st != OK:
        raise W4A16Error(fn, st)


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _dev(t: torch.Tensor, name: str, dtype, shape=None) -> int:
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    return t.data_ptr()


def quantize_pack(W: torch.Tensor, qweight: torch.Tensor, scales: torch.Tensor, zeros: torch.Tensor,
                  dev_status: torch.Tensor, stream=None, symmetric: bool = False) -> None:
    """w4a16_quantize_pack (w4a16_quantize_pack_sym when symmetric): W fp32 [N, K] ->
    qweight int32 [N, K/8], scales bf16 [N, K/128], zeros int32 [N, K/128];
    dev_status int32 [1] receives device-detected data errors."""
    N, K = W.shape
    name = "w4a16_quantize_pack_sym" if symmetric else "w4a16_quantize_pack"
    st = getattr(load(), name)(
        _dev(W, "W", torch.float32), N, K,
        _dev(qweight, "qweight", torch.int32, (N, K // 8)),
        _dev(scales, "scales", torch.bfloat16, (N, K // GROUP)),
        _dev(zeros, "zeros", torch.int32, (N, K // GROUP)),
        _dev(dev_status, "dev_status", torch.int32, (1,)), _stream(stream))
    _check(name, st)


def workspace_bytes(M: int, N: int, K: int) -> int:
    return int(load().w4a16_workspace_bytes(M, N, K))


def workspace_init(workspace: torch.Tensor, stream=None) -> None:
    st = load().w4a16_workspace_init(_dev(workspace, "workspace", torch.uint8), workspace.numel(), _stream(stream))
    _check("w4a16_workspace_init", st)


def linear(X: torch.Tensor, qweight: torch.Tensor, scales: torch.Tensor, zeros: torch.Tensor, Y: torch.Tensor,
           workspace: torch.Tensor | None = None, path: int = PATH_AUTO, stream=None) -> None:
    """w4a16_linear_path: Y[M, N] = X[M, K] . W_hat^T (BF16 out, FP32 accumulation)."""
    M, K = X.shape
    N = qweight.shape[0]
    ws_ptr, ws_bytes = None, 0
    if workspace is not None:
        ws_ptr = _dev(workspace, "workspace", torch.uint8)
        ws_bytes = workspace.numel()
    st = load().w4a16_linear_path(
        _dev(X, "X", torch.bfloat16), M, K,
        _dev(qweight, "qweight", torch.int32, (N, K // 8)),
        _dev(scales, "scales", torch.bfloat16, (N, K // GROUP)),
        _dev(zeros, "zeros", torch.int32, (N, K // GROUP)), N,
        _dev(Y, "Y", torch.bfloat16, (M, N)), ws_ptr, ws_bytes, path, _stream(stream))
    _check("w4a16_linear", st)


def linear_awq(X: torch.Tensor, inv_s: torch.Tensor, qweight: torch.Tensor, scales: torch.Tensor,
               zeros: torch.Tensor, Y: torch.Tensor, workspace: torch.Tensor | None = None, path: int = PATH_AUTO,
               stream=None) -> None:
    """w4a16_linear_awq: Y = bf16(X * inv_s) . W_hat'^T, the activation scaling formed where the
    kernels prepare X; qweight/scales/zeros from quantize_pack_awq."""
    M, K = X.shape
    N = qweight.shape[0]
    ws_ptr, ws_bytes = None, 0
    if workspace is not None:
        ws_ptr = _dev(workspace, "workspace", torch.uint8)
        ws_bytes = workspace.numel()
    st = load().w4a16_linear_awq(
        _dev(X, "X", torch.bfloat16), _dev(inv_s, "inv_s", torch.float32, (K,)), M, K,
        _dev(qweight, "qweight", torch.int32, (N, K // 8)),
        _dev(scales, "scales", torch.bfloat16, (N, K // GROUP)),
        _dev(zeros, "zeros", torch.int32, (N, K // GROUP)), N,
        _dev(Y, "Y", torch.bfloat16, (M, N)), ws_ptr, ws_bytes, path, _stream(stream))
    _check("w4a16_linear_awq", st)


def quantize_pack_awq(W: torch.Tensor, s: torch.Tensor, qweight: torch.Tensor, scales: torch.Tensor,
                      zeros: torch.Tensor, dev_status: torch.Tensor, stream=None) -> None:
    """w4a16_quantize_pack_awq: quantise and pack fp32(W * s) (s per input channel, [K])."""
    N, K = W.shape
    st = load().w4a16_quantize_pack_awq(
        _dev(W, "W", torch.float32), _dev(s, "s", torch.float32, (K,)), N, K,
        _dev(qweight, "qweight", torch.int32, (N, K // 8)),
        _dev(scales, "scales", torch.bfloat16, (N, K // GROUP)),
        _dev(zeros, "zeros", torch.int32, (N, K // GROUP)),
        _dev(dev_status, "dev_status", torch.int32, (1,)), _stream(stream))
    _check("w4a16_quantize_pack_awq", st)


def quantize_pack_g(W: torch.Tensor, group: int, qweight: torch.Tensor, scales: torch.Tensor,
                    zeros: torch.Tensor, dev_status: torch.Tensor, symmetric: bool = False, stream=None) -> None:
    """w4a16_quantize_pack_g: groups of `group` (32, 64, 128) weights; scales/zeros [N, K/group]."""
    N, K = W.shape
    st = load().w4a16_quantize_pack_g(
        _dev(W, "W", torch.float32), N, K, group, int(symmetric),
        _dev(qweight, "qweight", torch.int32, (N, K // 8)),
        _dev(scales, "scales", torch.bfloat16, (N, K // group)),
        _dev(zeros, "zeros", torch.int32, (N, K // group)),
        _dev(dev_status, "dev_status", torch.int32, (1,)), _stream(stream))
    _check("w4a16_quantize_pack_g", st)


def workspace_bytes_g(M: int, N: int, K: int, group: int) -> int:
    return int(load().w4a16_workspace_bytes_g(M, N, K, group))


def linear_g(X: torch.Tensor, group: int, qweight: torch.Tensor, scales: torch.Tensor, zeros: torch.Tensor,
             Y: torch.Tensor, workspace: torch.Tensor | None = None, stream=None) -> None:
    """w4a16_linear_g: the layer on weights packed with groups of `group`."""
    M, K = X.shape
    N = qweight.shape[0]
    ws_ptr, ws_bytes = None, 0
    if workspace is not None:
        ws_ptr = _dev(workspace, "workspace", torch.uint8)
        ws_bytes = workspace.numel()
    st = load().w4a16_linear_g(
        _dev(X, "X", torch.bfloat16), M, K, group, _dev(qweight, "qweight", torch.int32, (N, K // 8)),
        _dev(scales, "scales", torch.bfloat16, (N, K // group)), _dev(zeros, "zeros", torch.int32, (N, K // group)),
        N, _dev(Y, "Y", torch.bfloat16, (M, N)), ws_ptr, ws_bytes, _stream(stream))
    _check("w4a16_linear_g", st)


def w8_quantize(W: torch.Tensor, qweight: torch.Tensor, scales: torch.Tensor, dev_status: torch.Tensor,
                stream=None) -> None:
    """w8a16_quantize: W fp32 [N, K] -> qweight int8 [N, K], scales bf16 [N] (symmetric per row)."""
    N, K = W.shape
    st = load().w8a16_quantize(
        _dev(W, "W", torch.float32), N, K, _dev(qweight, "qweight", torch.int8, (N, K)),
        _dev(scales, "scales", torch.bfloat16, (N,)), _dev(dev_status, "dev_status", torch.int32, (1,)),
        _stream(stream))
    _check("w8a16_quantize", st)


def w8_dequant(qweight: torch.Tensor, scales: torch.Tensor, W_hat: torch.Tensor, stream=None) -> None:
    N, K = qweight.shape
    st = load().w8a16_dequant(_dev(qweight, "qweight", torch.int8, (N, K)),
                              _dev(scales, "scales", torch.bfloat16, (N,)), N, K,
                              _dev(W_hat, "W_hat", torch.bfloat16, (N, K)), _stream(stream))
    _check("w8a16_dequant", st)


def w8_workspace_bytes(M: int, N: int, K: int) -> int:
    return int(load().w8a16_workspace_bytes(M, N, K))


def w8_linear(X: torch.Tensor, qweight: torch.Tensor, scales: torch.Tensor, Y: torch.Tensor,
              workspace: torch.Tensor, stream=None) -> None:
    """w8a16_linear: Y[M, N] = X[M, K] . (q s)^T (BF16 out, FP32 accumulation)."""
    M, K = X.shape
    N = qweight.shape[0]
    st = load().w8a16_linear(
        _dev(X, "X", torch.bfloat16), M, K, _dev(qweight, "qweight", torch.int8, (N, K)),
        _dev(scales, "scales", torch.bfloat16, (N,)), N, _dev(Y, "Y", torch.bfloat16, (M, N)),
        _dev(workspace, "workspace", torch.uint8), workspace.numel(), _stream(stream))
    _check("w8a16_linear", st)


class PackedW8:
    """Device buffers of one INT8 weight matrix (plumbing: allocation via torch)."""

    def __init__(self, N: int, K: int, device="cuda"):
        self.N, self.K = N, K
        self.qweight = torch.empty((N, K), dtype=torch.int8, device=device)
        self.scales = torch.empty((N,), dtype=torch.bfloat16, device=device)

    @classmethod
    def from_float(cls, W: torch.Tensor, stream=None) -> "PackedW8":
        N, K = W.shape
        pw = cls(N, K, device=W.device)
        pw.status = torch.zeros(1, dtype=torch.int32, device=W.device)
        w8_quantize(W, pw.qweight, pw.scales, pw.status, stream)
        return pw


def _host(t: torch.Tensor, name: str, shape) -> int:
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.is_cuda:
        raise ValueError(f"{name} must be a host tensor")
    if t.dtype not in (torch.bfloat16, torch.int16):
        raise TypeError(f"{name} must hold BF16 bits (bfloat16 or int16), got {t.dtype}")
    if not t.is_contiguous() or tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must be contiguous with shape {tuple(shape)}")
    return t.data_ptr()


def linear_host(X_host: torch.Tensor, X_dev: torch.Tensor, qweight: torch.Tensor, scales: torch.Tensor,
                zeros: torch.Tensor, Y_dev: torch.Tensor, Y_host: torch.Tensor,
                workspace: torch.Tensor | None = None, stream=None) -> None:
    """w4a16_linear_host: copy X_host to X_dev, run the layer into Y_dev, copy it to Y_host, all
    enqueued on the stream by one library call (host tensors should be pinned for the copies to be
    asynchronous; Y_host is valid once the stream has passed this call)."""
    M, K = X_dev.shape
    N = qweight.shape[0]
    ws_ptr, ws_bytes = None, 0
    if workspace is not None:
        ws_ptr = _dev(workspace, "workspace", torch.uint8)
        ws_bytes = workspace.numel()
    st = load().w4a16_linear_host(
        _host(X_host, "X_host", (M, K)), _dev(X_dev, "X_dev", torch.bfloat16), M, K,
        _dev(qweight, "qweight", torch.int32, (N, K // 8)),
        _dev(scales, "scales", torch.bfloat16, (N, K // GROUP)),
        _dev(zeros, "zeros", torch.int32, (N, K // GROUP)), N,
        _dev(Y_dev, "Y_dev", torch.bfloat16, (M, N)), _host(Y_host, "Y_host", (M, N)), ws_ptr, ws_bytes,
        _stream(stream))
    _check("w4a16_linear_host", st)


def linear_noalloc(X: torch.Tensor, qweight: torch.Tensor, scales: torch.Tensor, zeros: torch.Tensor,
                   Y: torch.Tensor, stream=None) -> None:
    """w4a16_linear_noalloc: the decode-path linear layer using the library's built-in
    device scratch array instead of a workspace (for callers that cannot allocate)."""
    M, K = X.shape
    N = qweight.shape[0]
    st = load().w4a16_linear_noalloc(
        _dev(X, "X", torch.bfloat16), M, K,
        _dev(qweight, "qweight", torch.int32, (N, K // 8)),
        _dev(scales, "scales", torch.bfloat16, (N, K // GROUP)),
        _dev(zeros, "zeros", torch.int32, (N, K // GROUP)), N,
        _dev(Y, "Y", torch.bfloat16, (M, N)), _stream(stream))
    _check("w4a16_linear_noalloc", st)


def noalloc_scratch_bytes() -> int:
    return int(load().w4a16_noalloc_scratch_bytes())


def unpack(qweight: torch.Tensor, K: int, codes: torch.Tensor, stream=None) -> None:
    N = qweight.shape[0]
    st = load().w4a16_unpack(_dev(qweight, "qweight", torch.int32, (N, K // 8)), N, K,
                             _dev(codes, "codes", torch.uint8, (N, K)), _stream(stream))
    _check("w4a16_unpack", st)


def dequant(qweight: torch.Tensor, scales: torch.Tensor, zeros: torch.Tensor, K: int, W_hat: torch.Tensor,
            stream=None) -> None:
    N = qweight.shape[0]
    st = load().w4a16_dequant(_dev(qweight, "qweight", torch.int32, (N, K // 8)),
                              _dev(scales, "scales", torch.bfloat16, (N, K // GROUP)),
                              _dev(zeros, "zeros", torch.int32, (N, K // GROUP)), N, K,
                              _dev(W_hat, "W_hat", torch.bfloat16, (N, K)), _stream(stream))
    _check("w4a16_dequant", st)


def dequant_codes(codes: torch.Tensor, scales: torch.Tensor, zeros: torch.Tensor, W_hat: torch.Tensor,
                  stream=None) -> None:
    """w4a16_dequant_codes: W_hat bf16 [N, K] from unpacked codes uint8 [N, K] (unfused comparison)."""
    N, K = codes.shape
    st = load().w4a16_dequant_codes(_dev(codes, "codes", torch.uint8, (N, K)),
                                    _dev(scales, "scales", torch.bfloat16, (N, K // GROUP)),
                                    _dev(zeros, "zeros", torch.int32, (N, K // GROUP)), N, K,
                                    _dev(W_hat, "W_hat", torch.bfloat16, (N, K)), _stream(stream))
    _check("w4a16_dequant_codes", st)


def renorm_rows(y: torch.Tensor, out: torch.Tensor, stream=None) -> None:
    M, N = y.shape
    st = load().w4a16_renorm_rows(_dev(y, "y", torch.bfloat16), M, N,
                                  _dev(out, "out", torch.bfloat16, (M, N)), _stream(stream))
    _check("w4a16_renorm_rows", st)


def device_fault() -> int:
    """Synchronise, then read and clear the device fault word (0 = no bounded wait gave up)."""
    return int(load().w4a16_device_fault())


SELFTEST_SITE = 900


def selftest_wait(limit_cycles: int, stream=None) -> None:
    """w4a16_selftest_wait: one CTA's bounded wait on a barrier phase nothing completes; it gives up
    after limit_cycles, records SELFTEST_SITE in the fault word and returns."""
    _check("w4a16_selftest_wait", load().w4a16_selftest_wait(int(limit_cycles), _stream(stream)))


class PackedWeight:
    """Device buffers of one packed weight matrix (plumbing: allocation via torch)."""

    def __init__(self, N: int, K: int, device="cuda", group: int = GROUP):
        if K % GROUP:
            raise ValueError("K must be a multiple of 128")
        if group not in (32, 64, 128):
            raise ValueError("group must be 32, 64 or 128")
        self.N, self.K, self.group = N, K, group
        self.qweight = torch.empty((N, K // 8), dtype=torch.int32, device=device)
        self.scales = torch.empty((N, K // group), dtype=torch.bfloat16, device=device)
        self.zeros = torch.empty((N, K // group), dtype=torch.int32, device=device)

    @classmethod
    def from_float(cls, W: torch.Tensor, stream=None, symmetric: bool = False) -> "PackedWeight":
        """Pack W on `stream` (a torch.cuda.Stream, or None for the current one);
        the status word is cleared on that stream before the kernel runs.
        symmetric=True quantises without a zero point (stored zero points are 8)."""
        N, K = W.shape
        if stream is None:
            stream = torch.cuda.current_stream(W.device)
        if not isinstance(stream, torch.cuda.Stream):
            raise TypeError("stream must be a torch.cuda.Stream or None")
        with torch.cuda.stream(stream):
            pw = cls(N, K, device=W.device)
            status = torch.zeros(1, dtype=torch.int32, device=W.device)
            quantize_pack(W, pw.qweight, pw.scales, pw.zeros, status, stream, symmetric)
        pw.status = status
        return pw

    @property
    def nbytes(self) -> int:
        return self.qweight.numel() * 4 + self.scales.numel() * 2 + self.zeros.numel() * 4
