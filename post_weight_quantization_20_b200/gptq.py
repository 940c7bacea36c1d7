"""Python binding of libgptq.so (ctypes): argument marshalling only.

Every function named ``gptq_*`` mirrors the C call of the same name in
``include/gptq.h``; tensors are passed as device pointers and every step of the
solver runs in the library's CUDA kernels.  There is no CPU fallback: if the
library is missing or no CUDA device is present, the calls raise.

``quantize_layer`` strings the four calls together for one linear layer
(GPTQ量化算法深度解析 §3.1 steps 1-4) and allocates the outputs with PyTorch.
"""
from __future__ import annotations

import contextlib
import ctypes
import os
from dataclasses import dataclass

import torch

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "lib", "libgptq.so")

GPTQ_OK = 0
GPTQ_ERR_INVALID_ARG = 1
GPTQ_ERR_UNSUPPORTED = 2
GPTQ_ERR_WORKSPACE = 4
GPTQ_ERR_NOT_PD = 8
GPTQ_ERR_NONFINITE = 16
GPTQ_ERR_TIMEOUT = 32
GPTQ_ERR_CUDA = 64

GPTQ_F32, GPTQ_F16, GPTQ_BF16 = 0, 1, 2
GPTQ_ORDER_NATURAL, GPTQ_ORDER_DESC_DIAG, GPTQ_ORDER_GIVEN = 0, 1, 2
GPTQ_OP_PREPARE, GPTQ_OP_QUANTIZE = 1, 2

_DT = {torch.float32: GPTQ_F32, torch.float16: GPTQ_F16, torch.bfloat16: GPTQ_BF16}

# every symbol include/gptq.h declares
EXPORTS = ("gptq_workspace_size", "gptq_hessian_accumulate", "gptq_prepare",
           "gptq_quantize_layer", "gptq_pack", "gptq_status_string", "gptq_launch_count",
           "gptq_last_error", "gptq_prepare_static", "gptq_selftest_timeout",
           "gptq_repack_sweep_order", "gptq_dequant_matmul", "gptq_debug_set_wait_limit")
GPTQ_SELFTEST_MBARRIER, GPTQ_SELFTEST_GRID_BARRIER = 0, 1

GPTQ_STATIC_MAX_COLS = 1024


class GPTQError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = int(code)
        super().__init__(f"{where}: {status_names(code)}")


def status_names(code: int) -> str:
    if code == 0:
        return "GPTQ_OK"
    names = ["INVALID_ARG", "UNSUPPORTED", "WORKSPACE", "NOT_PD", "NONFINITE", "TIMEOUT", "CUDA"]
    return "|".join("GPTQ_ERR_" + n for i, n in enumerate(names) if code & (1 << i))


class gptq_config(ctypes.Structure):
    _fields_ = [("bits", ctypes.c_int), ("group_size", ctypes.c_int), ("sym", ctypes.c_int),
                ("act_order", ctypes.c_int), ("damp", ctypes.c_float),
                ("block_size", ctypes.c_int)]


_lib = None


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libgptq.so (once) and declare the C signatures."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"{path} is not built; run `python -m post_weight_quantization_20_b200.build`")
    lib = ctypes.CDLL(path)
    vp, i64, i32, sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_size_t
    cfgp = ctypes.POINTER(gptq_config)
    lib.gptq_workspace_size.argtypes = [i32, i64, i64, cfgp]
    lib.gptq_workspace_size.restype = sz
    lib.gptq_hessian_accumulate.argtypes = [vp, ctypes.POINTER(i64), vp, i32, i64, i64, i64, vp, vp]
    lib.gptq_hessian_accumulate.restype = i32
    lib.gptq_prepare.argtypes = [vp, i64, cfgp, vp, vp, vp, sz, vp, vp]
    lib.gptq_prepare.restype = i32
    lib.gptq_quantize_layer.argtypes = [vp, i32, i64, i64, i64, vp, vp, cfgp, vp, vp, vp, vp, vp,
                                        vp, sz, vp, vp]
    lib.gptq_quantize_layer.restype = i32
    lib.gptq_pack.argtypes = [vp, i64, i64, i32, vp, vp]
    lib.gptq_pack.restype = i32
    lib.gptq_status_string.argtypes = [i32]
    lib.gptq_status_string.restype = ctypes.c_char_p
    lib.gptq_launch_count.argtypes = []
    lib.gptq_launch_count.restype = ctypes.c_uint64
    lib.gptq_prepare_static.argtypes = [vp, i64, cfgp, vp, vp, vp, vp]
    lib.gptq_prepare_static.restype = i32
    lib.gptq_selftest_timeout.argtypes = [i32, vp, vp]
    lib.gptq_selftest_timeout.restype = i32
    lib.gptq_last_error.argtypes = []
    lib.gptq_last_error.restype = ctypes.c_char_p
    lib.gptq_repack_sweep_order.argtypes = [vp, i64, i64, i32, vp, vp, vp]
    lib.gptq_repack_sweep_order.restype = i32
    lib.gptq_dequant_matmul.argtypes = [vp, i32, i64, i64, i64, vp, vp, vp, i32, i32, vp, vp,
                                        i64, i32, vp]
    lib.gptq_dequant_matmul.restype = i32
    lib.gptq_debug_set_wait_limit.argtypes = [ctypes.c_uint32]
    lib.gptq_debug_set_wait_limit.restype = ctypes.c_uint32
    _lib = lib
    return lib


def make_config(bits=4, group_size=128, sym=False, act_order=False, damp=0.01, block_size=128):
    order = act_order if isinstance(act_order, int) and not isinstance(act_order, bool) else \
        (GPTQ_ORDER_DESC_DIAG if act_order else GPTQ_ORDER_NATURAL)
    return gptq_config(int(bits), int(group_size), int(bool(sym)), int(order), float(damp),
                       int(block_size))


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _check(code: int, where: str):
    if code != GPTQ_OK:
        if code == GPTQ_ERR_CUDA:
            where = f"{where} [{gptq_last_error()}]"
        raise GPTQError(code, where)


def _need_cuda(*ts):
    devs = {t.device for t in ts if t is not None}
    if any(d.type != "cuda" for d in devs):
        raise ValueError("libgptq takes device tensors")
    if len(devs) > 1:
        raise ValueError(f"libgptq takes tensors on one device, got {sorted(map(str, devs))}")


def _expect(t, name, shape, dtypes, contiguous=True):
    """The library writes or reads exactly `shape` elements of `t`; check that `t`
    holds them (it cannot check buffer sizes itself)."""
    if t is None:
        raise ValueError(f"{name} is required")
    if t.numel() == 0 and 0 in tuple(shape):
        return                      # nothing is read or written through it
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if t.dtype not in dtypes:
        raise ValueError(f"{name} must be one of {dtypes}, got {t.dtype}")
    if contiguous and not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _expect_status(status):
    if status is not None and (status.dtype != torch.int32 or status.numel() < 1):
        raise ValueError("status must be an int32 tensor with at least one element")


def _expect_ws(ws):
    if ws.dtype != torch.uint8 or not ws.is_contiguous():
        raise ValueError("ws must be a contiguous uint8 tensor")


# --------------------------------------------------------------------------- the C calls
def gptq_workspace_size(op: int, rows: int, cols: int, cfg: gptq_config) -> int:
    return int(load_library().gptq_workspace_size(op, rows, cols, ctypes.byref(cfg)))


def gptq_hessian_accumulate(H: torch.Tensor, n_seen: int, X: torch.Tensor, status=None,
                            stream=None) -> int:
    """H (C x C fp32), X (m x C, row stride X.stride(0)); returns the new token count."""
    if X.dim() != 2 or X.stride(1) != 1:
        raise ValueError("X must be 2-D with unit column stride")
    if X.dtype not in _DT:
        raise ValueError(f"X must be float32, float16 or bfloat16, got {X.dtype}")
    C = X.shape[1]
    _expect(H, "H", (C, C), (torch.float32,))
    _expect_status(status)
    _need_cuda(H, X, status)
    n = ctypes.c_int64(int(n_seen))
    code = load_library().gptq_hessian_accumulate(
        _ptr(H), ctypes.byref(n), _ptr(X), _DT[X.dtype], X.shape[0], X.shape[1], X.stride(0),
        _ptr(status), _stream(stream))
    _check(code, "gptq_hessian_accumulate")
    return int(n.value)


def gptq_prepare(H, cfg, U, perm, ws, status=None, stream=None) -> None:
    C = H.shape[0]
    _expect(H, "H", (C, C), (torch.float32,))
    _expect(U, "U", (C, C), (torch.float32,))
    _expect(perm, "perm", (C,), (torch.int32,))
    _expect_ws(ws)
    _expect_status(status)
    _need_cuda(H, U, perm, ws, status)
    code = load_library().gptq_prepare(_ptr(H), H.shape[0], ctypes.byref(cfg), _ptr(U),
                                       _ptr(perm), _ptr(ws), ws.numel() * ws.element_size(),
                                       _ptr(status), _stream(stream))
    _check(code, "gptq_prepare")


def gptq_prepare_static(H, cfg, U, perm, status=None, stream=None) -> None:
    """gptq_prepare with the library's built-in scratch array instead of a workspace
    (for callers that cannot allocate; cols <= GPTQ_STATIC_MAX_COLS)."""
    C = H.shape[0]
    _expect(H, "H", (C, C), (torch.float32,))
    _expect(U, "U", (C, C), (torch.float32,))
    _expect(perm, "perm", (C,), (torch.int32,))
    _expect_status(status)
    _need_cuda(H, U, perm, status)
    code = load_library().gptq_prepare_static(_ptr(H), H.shape[0], ctypes.byref(cfg), _ptr(U),
                                              _ptr(perm), _ptr(status), _stream(stream))
    _check(code, "gptq_prepare_static")


def gptq_quantize_layer(W, U, perm, cfg, codes, scales, zeros, g_idx, losses, ws, status=None,
                        stream=None) -> None:
    if W.dim() != 2 or W.stride(1) != 1:
        raise ValueError("W must be 2-D with unit column stride")
    if W.dtype not in _DT:
        raise ValueError(f"W must be float32, float16 or bfloat16, got {W.dtype}")
    R, C = W.shape
    G = n_groups(C, cfg.group_size)
    _expect(U, "U", (C, C), (torch.float32,))
    _expect(perm, "perm", (C,), (torch.int32,))
    _expect(codes, "codes", (R, C), (torch.uint8,))
    _expect(scales, "scales", (R, G), (torch.float32,))
    _expect(zeros, "zeros", (R, G), (torch.float32,))
    _expect(g_idx, "g_idx", (C,), (torch.int32,))
    _expect(losses, "losses", (C,), (torch.float32,))
    _expect_ws(ws)
    _expect_status(status)
    _need_cuda(W, U, perm, codes, scales, zeros, g_idx, losses, ws, status)
    code = load_library().gptq_quantize_layer(
        _ptr(W), _DT[W.dtype], W.shape[0], W.shape[1], W.stride(0), _ptr(U), _ptr(perm),
        ctypes.byref(cfg), _ptr(codes), _ptr(scales), _ptr(zeros), _ptr(g_idx), _ptr(losses),
        _ptr(ws), ws.numel() * ws.element_size(), _ptr(status), _stream(stream))
    _check(code, "gptq_quantize_layer")


def gptq_pack(codes, bits, packed, stream=None) -> None:
    if codes.dim() != 2:
        raise ValueError("codes must be 2-D")
    R, C = codes.shape
    _expect(codes, "codes", (R, C), (torch.uint8,))
    _expect(packed, "packed", (R, packed_words(C, int(bits))), (torch.int32, torch.uint32))
    _need_cuda(codes, packed)
    code = load_library().gptq_pack(_ptr(codes), codes.shape[0], codes.shape[1], int(bits),
                                    _ptr(packed), _stream(stream))
    _check(code, "gptq_pack")


def gptq_status_string(code: int) -> str:
    return load_library().gptq_status_string(int(code)).decode()


def gptq_selftest_timeout(which: int, status: torch.Tensor, stream=None) -> None:
    """Launch the failure-detection self-test `which` (a bounded device wait that is
    made to run out); it ORs GPTQ_ERR_TIMEOUT into `status` on the device."""
    _expect_status(status)
    _need_cuda(status)
    _check(load_library().gptq_selftest_timeout(int(which), _ptr(status), _stream(stream)),
           "gptq_selftest_timeout")


def gptq_debug_set_wait_limit(polls: int) -> int:
    """Polls after which a tensor-core pipeline wait gives up (0 = the default);
    returns the previous limit.  For tests of the timeout path."""
    return int(load_library().gptq_debug_set_wait_limit(int(polls)))


def gptq_launch_count() -> int:
    return int(load_library().gptq_launch_count())


def gptq_last_error() -> str:
    return load_library().gptq_last_error().decode()


# --------------------------------------------------------------------------- stored form
def sweep_words(cols: int, bits: int) -> int:
    return cols // 32 * bits


def gptq_repack_sweep_order(packed, bits, perm, out, stream=None) -> None:
    """The packed codes (original column order) rewritten in the sweep order perm."""
    C = perm.shape[0]
    if C % 32:
        raise ValueError("cols must be a multiple of 32")
    R = packed.shape[0]
    _expect(packed, "packed", (R, packed_words(C, bits)), (torch.int32, torch.uint32))
    _expect(perm, "perm", (C,), (torch.int32,))
    _expect(out, "out", (R, sweep_words(C, bits)), (torch.int32, torch.uint32))
    _need_cuda(packed, perm, out)
    _check(load_library().gptq_repack_sweep_order(_ptr(packed), R, C, int(bits), _ptr(perm),
                                                  _ptr(out), _stream(stream)),
           "gptq_repack_sweep_order")


def gptq_dequant_matmul(X, qp, scales, zeros, bits, group_size, perm, Y, half_sums=False,
                        stream=None) -> None:
    """Y (m x rows fp32) = X (m x cols) Q^T from the sweep-order packed codes."""
    if X.dim() != 2 or X.stride(1) != 1:
        raise ValueError("X must be 2-D with unit column stride")
    if X.dtype not in _DT:
        raise ValueError(f"X must be float32, float16 or bfloat16, got {X.dtype}")
    M, C = X.shape
    R = qp.shape[0]
    G = n_groups(C, group_size)
    _expect(qp, "qp", (R, sweep_words(C, bits)), (torch.int32, torch.uint32))
    _expect(scales, "scales", (R, G), (torch.float32,))
    _expect(zeros, "zeros", (R, G), (torch.float32,))
    if perm is not None:
        _expect(perm, "perm", (C,), (torch.int32,))
    _expect(Y, "Y", (M, R), (torch.float32,))
    _need_cuda(X, qp, scales, zeros, perm, Y)
    _check(load_library().gptq_dequant_matmul(
        _ptr(X), _DT[X.dtype], M, C, X.stride(0), _ptr(qp), _ptr(scales), _ptr(zeros), int(bits),
        int(group_size), _ptr(perm), _ptr(Y), R, int(bool(half_sums)), _stream(stream)),
        "gptq_dequant_matmul")


# --------------------------------------------------------------------------- one layer
def packed_words(cols: int, bits: int) -> int:
    return (cols * bits + 31) // 32


def n_groups(cols: int, group_size: int) -> int:
    return (cols + group_size - 1) // group_size if group_size > 0 else 1


def alloc_workspace(op: int, rows: int, cols: int, cfg: gptq_config, device) -> torch.Tensor:
    nbytes = gptq_workspace_size(op, rows, cols, cfg)
    if nbytes == 0:
        raise GPTQError(GPTQ_ERR_INVALID_ARG, "gptq_workspace_size")
    # torch's caching allocator returns 512-byte aligned blocks
    return torch.empty(nbytes, dtype=torch.uint8, device=device)


@dataclass
class LayerResult:
    codes: torch.Tensor
    scales: torch.Tensor
    zeros: torch.Tensor
    g_idx: torch.Tensor
    losses: torch.Tensor
    perm: torch.Tensor
    packed: torch.Tensor
    H: torch.Tensor
    U: torch.Tensor
    n_tokens: int
    damp: float | None = None      # the relative damping the factor was formed with


def check_status(status: torch.Tensor, where: str = "device") -> None:
    code = int(status.item())
    if code:
        raise GPTQError(code, where)


def _on(stream):
    """Allocate on the stream the work runs on, so that the caching allocator reuses
    a buffer (a workspace released before its kernel has run) only in stream order."""
    return torch.cuda.stream(stream) if stream is not None else contextlib.nullcontext()


def _hessian(X, C: int, dev, status, chunk_tokens, stream, n_start: int = 0):
    """H of the tokens of X (a tensor or an iterable of chunks).  n_start > 0 starts
    the running mean as if n_start tokens of a zero Hessian had been seen already,
    so that the result is (2 / (n_start + n)) X^T X: a share of a Hessian whose
    tokens are split over several callers."""
    if n_start > 0:
        H = torch.zeros(C, C, dtype=torch.float32, device=dev)
    else:
        H = torch.empty(C, C, dtype=torch.float32, device=dev)
    n = int(n_start)
    chunks = [X] if isinstance(X, torch.Tensor) else X
    for Xc in chunks:
        if chunk_tokens:
            for t0 in range(0, Xc.shape[0], chunk_tokens):
                n = gptq_hessian_accumulate(H, n, Xc[t0:t0 + chunk_tokens], status, stream)
        else:
            n = gptq_hessian_accumulate(H, n, Xc, status, stream)
    return H, n


def _factor(H, cfg, perm, rows, dev, status, stream):
    C = H.shape[0]
    U = torch.empty(C, C, dtype=torch.float32, device=dev)
    if perm is None:
        perm = torch.empty(C, dtype=torch.int32, device=dev)
    ws = alloc_workspace(GPTQ_OP_PREPARE, rows, C, cfg, dev)
    gptq_prepare(H, cfg, U, perm, ws, status, stream)
    return U, perm


def _with_damp(cfg: gptq_config, damp: float) -> gptq_config:
    return gptq_config(cfg.bits, cfg.group_size, cfg.sym, cfg.act_order, float(damp),
                       cfg.block_size)


def _factor_retry(H, cfg, perm, rows, dev, status, stream, damp_retry):
    """Factor H; while the factorization reports a non-positive pivot (and nothing
    else) and larger damping values remain in `damp_retry`, factor again with the
    next one.  A near-singular Hessian from a small calibration set is stabilised
    by a larger damp_percent, e.g. 0.1 (GPTQ量化算法深度解析 §3.3).  Without retry
    values nothing is synchronised.  Returns (U, perm, the damp used)."""
    U, p = _factor(H, cfg, perm, rows, dev, status, stream)
    damp = float(cfg.damp)
    for d in damp_retry:
        code = int(status.item())
        if code != GPTQ_ERR_NOT_PD:
            break
        status.zero_()
        U, p = _factor(H, _with_damp(cfg, d), perm, rows, dev, status, stream)
        damp = float(d)
    return U, p, damp


def _sweep(W, U, perm, cfg, dev, status, stream):
    R, C = W.shape
    G = n_groups(C, cfg.group_size)
    codes = torch.empty(R, C, dtype=torch.uint8, device=dev)
    scales = torch.empty(R, G, dtype=torch.float32, device=dev)
    zeros = torch.empty(R, G, dtype=torch.float32, device=dev)
    g_idx = torch.empty(C, dtype=torch.int32, device=dev)
    losses = torch.empty(C, dtype=torch.float32, device=dev)
    ws = alloc_workspace(GPTQ_OP_QUANTIZE, R, C, cfg, dev)
    gptq_quantize_layer(W, U, perm, cfg, codes, scales, zeros, g_idx, losses, ws, status, stream)
    packed = torch.empty(R, packed_words(C, cfg.bits), dtype=torch.int32, device=dev)
    gptq_pack(codes, cfg.bits, packed, stream)
    return codes, scales, zeros, g_idx, losses, packed


def quantize_layer(W: torch.Tensor, X, cfg: gptq_config, perm: torch.Tensor | None = None,
                   chunk_tokens: int | None = None, stream=None, check: bool = True,
                   damp_retry=()) -> LayerResult:
    """Quantize one linear layer.  W (rows x cols) and X (tokens x cols, or an
    iterable of such chunks) are device tensors.  damp_retry: larger relative
    damping values to factor with, in turn, while the factorization reports a
    non-positive pivot (e.g. (0.1,)); each retry synchronises the stream once."""
    dev = W.device
    R, C = W.shape
    with _on(stream):
        status = torch.zeros(1, dtype=torch.int32, device=dev)
        H, n = _hessian(X, C, dev, status, chunk_tokens, stream)
        U, perm, damp = _factor_retry(H, cfg, perm, R, dev, status, stream, damp_retry)
        codes, scales, zeros, g_idx, losses, packed = _sweep(W, U, perm, cfg, dev, status, stream)
    if check:
        check_status(status, "quantize_layer")
    return LayerResult(codes, scales, zeros, g_idx, losses, perm, packed, H, U, n, damp)


def quantize_layers_shared(Ws, X, cfg: gptq_config, perm: torch.Tensor | None = None,
                           chunk_tokens: int | None = None, stream=None,
                           check: bool = True, damp_retry=()) -> list:
    """Quantize several linear layers that read the same input (the q/k/v or
    gate/up projections of one block): one Hessian and one factorization, then one
    sweep per weight.  Each W is rows_i x cols; the results are those of separate
    quantize_layer calls on the same X.  damp_retry as for quantize_layer."""
    Ws = list(Ws)
    if not Ws:
        return []
    dev = Ws[0].device
    C = Ws[0].shape[1]
    if any(W.shape[1] != C or W.device != dev for W in Ws):
        raise ValueError("the weights of a shared-input group need the same cols and device")
    out = []
    with _on(stream):
        status = torch.zeros(1, dtype=torch.int32, device=dev)
        H, n = _hessian(X, C, dev, status, chunk_tokens, stream)
        U, perm, damp = _factor_retry(H, cfg, perm, max(W.shape[0] for W in Ws), dev, status,
                                      stream, damp_retry)
        for W in Ws:
            codes, scales, zeros, g_idx, losses, packed = _sweep(W, U, perm, cfg, dev, status,
                                                                 stream)
            out.append(LayerResult(codes, scales, zeros, g_idx, losses, perm, packed, H, U, n,
                                   damp))
    if check:
        check_status(status, "quantize_layers_shared")
    return out


def quantize_rtn(W: torch.Tensor, cfg: gptq_config, stream=None, check: bool = True) -> LayerResult:
    """Round-to-nearest on the same grids, without error feedback: the sweep with
    U = I (every off-diagonal of U is zero, so no error is fed forward; the
    per-column losses are then (w - Q)^2 / 2 summed over rows).  Natural column
    order; act_order in cfg is ignored."""
    dev = W.device
    R, C = W.shape
    with _on(stream):
        status = torch.zeros(1, dtype=torch.int32, device=dev)
        U = torch.eye(C, dtype=torch.float32, device=dev)
        perm = torch.arange(C, dtype=torch.int32, device=dev)
        codes, scales, zeros, g_idx, losses, packed = _sweep(W, U, perm, cfg, dev, status, stream)
    if check:
        check_status(status, "quantize_rtn")
    return LayerResult(codes, scales, zeros, g_idx, losses, perm, packed, None, U, 0)


# --------------------------------------------------------------------------- host buffers
@dataclass
class HostResult:
    """Quantized layer copied back to (pinned) host memory."""
    packed: torch.Tensor
    scales: torch.Tensor
    zeros: torch.Tensor
    g_idx: torch.Tensor
    losses: torch.Tensor
    perm: torch.Tensor
    status: torch.Tensor

    @property
    def nbytes(self) -> int:
        return sum(t.numel() * t.element_size() for t in
                   (self.packed, self.scales, self.zeros, self.g_idx, self.losses, self.perm,
                    self.status))


_copy_streams: dict = {}


def _side_stream(dev) -> torch.cuda.Stream:
    key = torch.device(dev).index
    if key not in _copy_streams:
        _copy_streams[key] = torch.cuda.Stream(device=dev)
    return _copy_streams[key]


def quantize_layer_host(W_host: torch.Tensor, X_host: torch.Tensor, cfg: gptq_config, device=None,
                        chunk_tokens: int = 32768, stream=None) -> HostResult:
    """Quantize one layer whose W and X live in pinned host memory.

    X is uploaded in chunks on a side stream while the previous chunk is being
    accumulated into H on the compute stream (two device staging buffers); the
    packed codes, scales, zeros, g_idx, losses and perm are copied back into
    pinned host tensors.  Asynchronous: synchronize the stream before reading
    the result (result.status holds the device status word).  Every call returns
    its own pinned tensors (torch's caching host allocator hands a freed block out
    again only after the copies into it have completed), so results of several
    layers in flight never share memory.
    """
    dev = torch.device(device) if device is not None else torch.device("cuda")
    comp = stream if stream is not None else torch.cuda.current_stream(dev)
    side = _side_stream(dev)
    R, C = W_host.shape
    T = X_host.shape[0]
    # Every device buffer is allocated on the compute stream: the caching allocator
    # hands a freed block out again in that stream's order, and the side stream's
    # writes into W and the staging buffers are joined into it by events.
    with torch.cuda.stream(comp):
        W = torch.empty((R, C), dtype=W_host.dtype, device=dev)
        stage = [torch.empty((min(chunk_tokens, max(T, 1)), C), dtype=X_host.dtype, device=dev)
                 for _ in range(2)]
        H = torch.empty(C, C, dtype=torch.float32, device=dev)
        status = torch.zeros(1, dtype=torch.int32, device=dev)
    side.wait_stream(comp)          # the allocations above are ordered before the copies
    ready = [torch.cuda.Event(), torch.cuda.Event()]
    done = [torch.cuda.Event(), torch.cuda.Event()]
    with torch.cuda.stream(side):
        W.copy_(W_host, non_blocking=True)
    w_ready = torch.cuda.Event()
    w_ready.record(side)
    n = 0
    for k, t0 in enumerate(range(0, T, chunk_tokens)):
        m = min(chunk_tokens, T - t0)
        b = k % 2
        if k >= 2:
            side.wait_event(done[b])
        with torch.cuda.stream(side):
            stage[b][:m].copy_(X_host[t0:t0 + m], non_blocking=True)
        ready[b].record(side)
        comp.wait_event(ready[b])
        n = gptq_hessian_accumulate(H, n, stage[b][:m], status, comp)
        done[b].record(comp)
    comp.wait_event(w_ready)
    with torch.cuda.stream(comp):
        U = torch.empty(C, C, dtype=torch.float32, device=dev)
        perm = torch.empty(C, dtype=torch.int32, device=dev)
        wsp = alloc_workspace(GPTQ_OP_PREPARE, R, C, cfg, dev)
        gptq_prepare(H, cfg, U, perm, wsp, status, comp)
        Gn = n_groups(C, cfg.group_size)
        codes = torch.empty(R, C, dtype=torch.uint8, device=dev)
        scales = torch.empty(R, Gn, dtype=torch.float32, device=dev)
        zeros = torch.empty(R, Gn, dtype=torch.float32, device=dev)
        g_idx = torch.empty(C, dtype=torch.int32, device=dev)
        losses = torch.empty(C, dtype=torch.float32, device=dev)
        wsq = alloc_workspace(GPTQ_OP_QUANTIZE, R, C, cfg, dev)
        gptq_quantize_layer(W, U, perm, cfg, codes, scales, zeros, g_idx, losses, wsq, status, comp)
        packed = torch.empty(R, packed_words(C, cfg.bits), dtype=torch.int32, device=dev)
        gptq_pack(codes, cfg.bits, packed, comp)
        host = HostResult(*(torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in
                            (packed, scales, zeros, g_idx, losses, perm, status)))
        for dst, src in zip((host.packed, host.scales, host.zeros, host.g_idx, host.losses,
                             host.perm, host.status),
                            (packed, scales, zeros, g_idx, losses, perm, status)):
            dst.copy_(src, non_blocking=True)
    return host
