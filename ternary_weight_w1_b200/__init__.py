"""Python binding of libbitlinear, the BitLinear W1.58A8 matmul for B200.

Argument marshalling only: every step of the path runs in the CUDA library
(``libbitlinear.so``, built in-tree by ``ternary_weight_w1_b200.build``). The
functions carry the C ABI's names (see include/bitlinear.h for semantics and
layouts) and take torch tensors for device buffers; PyTorch supplies device
memory and streams. There is no CPU fallback: if the library is missing,
loading it raises.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libbitlinear.so")

BITLINEAR_OK = 0
BITLINEAR_ERR_ARG = 1
BITLINEAR_ERR_SHAPE = 2
BITLINEAR_ERR_ALIGN = 3
BITLINEAR_ERR_DTYPE = 4
BITLINEAR_ERR_CUDA = 5
BITLINEAR_ERR_TIMEOUT = 6
BITLINEAR_ERR_WORKSPACE = 7
BITLINEAR_ERR_SCRATCH_LIMIT = 8
BITLINEAR_ERR_HOST = 9
BITLINEAR_ERR_IO = 10
BITLINEAR_ERR_FORMAT = 11
BITLINEAR_STATIC_SCRATCH_BYTES = 16 << 20

BITLINEAR_BF16 = 0
BITLINEAR_FP32 = 1

PATH_AUTO = 0
PATH_GEMV = 1
PATH_TC = 2

# default eps of bitlinear_forward_rmsnorm: nn.RMSNorm's default for fp32
# inputs, the fp32 machine epsilon
RMSNORM_EPS = 2.0 ** -23

# Every symbol include/bitlinear.h declares.
EXPORTS = (
    "bitlinear_packed_bytes",
    "bitlinear_pack_weights",
    "bitlinear_packed_bytes_b3",
    "bitlinear_pack_weights_b3",
    "bitlinear_forward_b3",
    "bitlinear_save_packed",
    "bitlinear_read_packed_header",
    "bitlinear_load_packed",
    "bitlinear_quant_act",
    "bitlinear_workspace_bytes",
    "bitlinear_workspace_bytes_path",
    "bitlinear_forward",
    "bitlinear_forward_ex",
    "bitlinear_forward_rmsnorm",
    "bitlinear_get_fault",
    "bitlinear_status_string",
    "bitlinear_forward_inject_timeout",
    "bitlinear_forward_noalloc",
    "bitlinear_forward_grouped",
    "bitlinear_forward_grouped_host",
    "bitlinear_forward_grouped_b3",
    "bitlinear_workspace_bytes_grouped",
    "bitlinear_forward_grouped_ws",
    "bitlinear_forward_grouped_rmsnorm",
    "bitlinear_workspace_bytes_ffn",
    "bitlinear_ffn_forward",
)


class _Problem(ctypes.Structure):
    _fields_ = [("x_dev", ctypes.c_void_p), ("M", ctypes.c_int64), ("K", ctypes.c_int64),
                ("N", ctypes.c_int64), ("packed_dev", ctypes.c_void_p),
                ("gamma", ctypes.c_float), ("y_dev", ctypes.c_void_p)]

_lib = None


class BitLinearError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)} (status {status})")


def lib() -> ctypes.CDLL:
    """Load libbitlinear.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is missing: build it with "
                "`python -m ternary_weight_w1_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        i64, p, sz = ctypes.c_int64, ctypes.c_void_p, ctypes.c_size_t
        L.bitlinear_packed_bytes.restype = sz
        L.bitlinear_packed_bytes.argtypes = [i64, i64]
        L.bitlinear_pack_weights.restype = ctypes.c_int
        L.bitlinear_pack_weights.argtypes = [p, i64, i64, p, p]
        L.bitlinear_packed_bytes_b3.restype = sz
        L.bitlinear_packed_bytes_b3.argtypes = [i64, i64]
        L.bitlinear_pack_weights_b3.restype = ctypes.c_int
        L.bitlinear_pack_weights_b3.argtypes = [p, i64, i64, p, p]
        L.bitlinear_forward_b3.restype = ctypes.c_int
        L.bitlinear_forward_b3.argtypes = [p, ctypes.c_int, i64, i64, p, ctypes.c_float, i64, p,
                                           p, p, p, p]
        L.bitlinear_save_packed.restype = ctypes.c_int
        L.bitlinear_save_packed.argtypes = [ctypes.c_char_p, p, i64, i64, ctypes.c_float]
        L.bitlinear_read_packed_header.restype = ctypes.c_int
        L.bitlinear_read_packed_header.argtypes = [ctypes.c_char_p, p, p, p]
        L.bitlinear_load_packed.restype = ctypes.c_int
        L.bitlinear_load_packed.argtypes = [ctypes.c_char_p, p, sz, p, p, p]
        L.bitlinear_quant_act.restype = ctypes.c_int
        L.bitlinear_quant_act.argtypes = [p, ctypes.c_int, i64, i64, p, p, p]
        L.bitlinear_workspace_bytes.restype = sz
        L.bitlinear_workspace_bytes.argtypes = [i64, i64, i64]
        L.bitlinear_workspace_bytes_path.restype = sz
        L.bitlinear_workspace_bytes_path.argtypes = [i64, i64, i64, ctypes.c_int]
        fwd = [p, ctypes.c_int, i64, i64, p, ctypes.c_float, i64, p, p, sz, p, p, p, p]
        L.bitlinear_forward.restype = ctypes.c_int
        L.bitlinear_forward.argtypes = fwd
        L.bitlinear_forward_ex.restype = ctypes.c_int
        L.bitlinear_forward_ex.argtypes = fwd + [ctypes.c_int]
        L.bitlinear_forward_rmsnorm.restype = ctypes.c_int
        L.bitlinear_forward_rmsnorm.argtypes = (fwd[:4] + [p, ctypes.c_float] + fwd[4:] +
                                                [ctypes.c_int])
        L.bitlinear_forward_inject_timeout.restype = ctypes.c_int
        L.bitlinear_forward_inject_timeout.argtypes = fwd[:11] + [ctypes.c_int, ctypes.c_int]
        L.bitlinear_forward_noalloc.restype = ctypes.c_int
        L.bitlinear_forward_noalloc.argtypes = [p, ctypes.c_int, i64, i64, p, ctypes.c_float,
                                                i64, p, p]
        L.bitlinear_forward_grouped.restype = ctypes.c_int
        L.bitlinear_forward_grouped.argtypes = [p, ctypes.c_int, ctypes.c_int, p]
        L.bitlinear_forward_grouped_b3.restype = ctypes.c_int
        L.bitlinear_forward_grouped_b3.argtypes = [p, ctypes.c_int, ctypes.c_int, p]
        L.bitlinear_forward_grouped_host.restype = ctypes.c_int
        L.bitlinear_forward_grouped_host.argtypes = [p, ctypes.c_int, ctypes.c_int, p, p, p]
        L.bitlinear_workspace_bytes_grouped.restype = ctypes.c_size_t
        L.bitlinear_workspace_bytes_grouped.argtypes = [p, ctypes.c_int]
        L.bitlinear_forward_grouped_ws.restype = ctypes.c_int
        L.bitlinear_forward_grouped_ws.argtypes = [p, ctypes.c_int, ctypes.c_int, p,
                                                   ctypes.c_size_t, p]
        L.bitlinear_forward_grouped_rmsnorm.restype = ctypes.c_int
        L.bitlinear_forward_grouped_rmsnorm.argtypes = [p, p, ctypes.c_int, ctypes.c_float,
                                                        ctypes.c_int, p, sz, p]
        L.bitlinear_workspace_bytes_ffn.restype = sz
        L.bitlinear_workspace_bytes_ffn.argtypes = [i64, i64, i64]
        f32 = ctypes.c_float
        L.bitlinear_ffn_forward.restype = ctypes.c_int
        L.bitlinear_ffn_forward.argtypes = [p, ctypes.c_int, i64, i64, i64, p, f32, p, f32, p,
                                            f32, p, p, p, f32, p, p, p, sz, p, p, p]
        L.bitlinear_get_fault.restype = ctypes.c_int
        L.bitlinear_get_fault.argtypes = [p, p]
        L.bitlinear_status_string.restype = ctypes.c_char_p
        L.bitlinear_status_string.argtypes = [ctypes.c_int]
        _lib = L
    return _lib


def status_string(status: int) -> str:
    return lib().bitlinear_status_string(int(status)).decode()


def _check(rc: int, where: str) -> None:
    if rc != BITLINEAR_OK:
        raise BitLinearError(rc, where)


def _ptr(t) -> int | None:
    return None if t is None else t.data_ptr()


class _Args:
    """Device addresses of one call's tensors, after checking that the library
    can use them: contiguous CUDA tensors on the current device, of the dtype
    and shape given, with at least ``min_numel`` elements. A host tensor handed
    to a kernel would make it read host addresses, so it is refused here,
    before any library call. The current device is looked up once per call."""

    __slots__ = ("cur",)

    def __init__(self):
        self.cur = None

    def ptr(self, t, name: str, dtype=None, shape=None, min_numel: int = 0) -> int | None:
        if t is None:
            return None
        d = t.get_device()
        if d < 0:
            raise ValueError(f"{name} must be a CUDA tensor (got device {t.device})")
        if self.cur is None:
            import torch
            self.cur = torch.cuda.current_device()
        if d != self.cur:
            raise ValueError(f"{name} is on cuda:{d}, the current device is cuda:{self.cur}")
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
        if dtype is not None and t.dtype != dtype:
            raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
        if shape is not None and t.shape != shape:
            raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
        if min_numel and t.numel() < min_numel:
            raise ValueError(f"{name} holds {t.numel()} elements, {min_numel} needed")
        return t.data_ptr()

    def packed(self, packed, N: int, K: int) -> int | None:
        import torch
        # bitlinear_packed_bytes(N, K) for valid shapes (the library rejects
        # the others itself): ceil(N / 16) row blocks of 16 * K / 4 bytes
        need = (N + 15) // 16 * 16 * (K // 4) if N >= 1 and K >= 128 and K % 128 == 0 else 1
        return self.ptr(packed, "packed", torch.uint8, min_numel=need)




def _stream(stream) -> int | None:
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream


def _xdt(x) -> int:
    import torch
    if x.dtype == torch.bfloat16:
        return BITLINEAR_BF16
    if x.dtype == torch.float32:
        return BITLINEAR_FP32
    raise TypeError(f"x must be bf16 or fp32, got {x.dtype}")


# ---------------------------------------------------------------- packing

def bitlinear_packed_bytes(N: int, K: int) -> int:
    return int(lib().bitlinear_packed_bytes(N, K))


def bitlinear_pack_weights(W) -> tuple[np.ndarray, float]:
    """Ternarise and pack latent fp32 weights [N][K] on the host.
    Returns (packed bytes as a flat uint8 numpy array, gamma)."""
    W = np.ascontiguousarray(np.asarray(W, dtype=np.float32))
    if W.ndim != 2:
        raise ValueError("W must be 2-D [N][K]")
    N, K = W.shape
    nbytes = bitlinear_packed_bytes(N, K)
    if nbytes == 0:
        raise BitLinearError(BITLINEAR_ERR_SHAPE, "bitlinear_pack_weights")
    out = np.empty((nbytes,), dtype=np.uint8)
    gamma = ctypes.c_float(0.0)
    _check(lib().bitlinear_pack_weights(W.ctypes.data, N, K, out.ctypes.data,
                                        ctypes.addressof(gamma)),
           "bitlinear_pack_weights")
    return out, float(gamma.value)


def bitlinear_packed_bytes_b3(N: int, K: int) -> int:
    return int(lib().bitlinear_packed_bytes_b3(N, K))


def bitlinear_pack_weights_b3(W) -> tuple[np.ndarray, float]:
    """Ternarise and pack latent fp32 weights [N][K] into the base-3 layout
    (five codes per byte) on the host. Returns (packed bytes, gamma)."""
    W = np.ascontiguousarray(np.asarray(W, dtype=np.float32))
    if W.ndim != 2:
        raise ValueError("W must be 2-D [N][K]")
    N, K = W.shape
    nbytes = bitlinear_packed_bytes_b3(N, K)
    if nbytes == 0:
        raise BitLinearError(BITLINEAR_ERR_SHAPE, "bitlinear_pack_weights_b3")
    out = np.empty((nbytes,), dtype=np.uint8)
    gamma = ctypes.c_float(0.0)
    _check(lib().bitlinear_pack_weights_b3(W.ctypes.data, N, K, out.ctypes.data,
                                           ctypes.addressof(gamma)),
           "bitlinear_pack_weights_b3")
    return out, float(gamma.value)


def bitlinear_save_packed(path, packed, N: int, K: int, gamma: float) -> None:
    """Write packed weights (host uint8 array of bitlinear_packed_bytes(N, K)
    bytes, as bitlinear_pack_weights returns it) and gamma to a file."""
    packed = np.ascontiguousarray(packed, dtype=np.uint8)
    need = bitlinear_packed_bytes(N, K)
    if need and packed.size < need:
        raise ValueError(f"packed must hold {need} bytes, got {packed.size}")
    _check(lib().bitlinear_save_packed(os.fsencode(path), packed.ctypes.data, N, K,
                                       float(gamma)),
           "bitlinear_save_packed")


def bitlinear_read_packed_header(path) -> tuple[int, int, float]:
    """(N, K, gamma) from a packed-weight file's header."""
    n, k, g = ctypes.c_int64(0), ctypes.c_int64(0), ctypes.c_float(0.0)
    _check(lib().bitlinear_read_packed_header(os.fsencode(path), ctypes.addressof(n),
                                              ctypes.addressof(k), ctypes.addressof(g)),
           "bitlinear_read_packed_header")
    return n.value, k.value, float(g.value)


def bitlinear_load_packed(path) -> tuple[np.ndarray, int, int, float]:
    """(packed uint8 array, N, K, gamma) from a packed-weight file; the
    payload's hash is checked."""
    N, K, _ = bitlinear_read_packed_header(path)
    out = np.empty((bitlinear_packed_bytes(N, K),), dtype=np.uint8)
    n, k, g = ctypes.c_int64(0), ctypes.c_int64(0), ctypes.c_float(0.0)
    _check(lib().bitlinear_load_packed(os.fsencode(path), out.ctypes.data, out.size,
                                       ctypes.addressof(n), ctypes.addressof(k),
                                       ctypes.addressof(g)),
           "bitlinear_load_packed")
    return out, n.value, k.value, float(g.value)


# ------------------------------------------------- activation quantisation

def bitlinear_quant_act(x, xq=None, beta=None, stream=None):
    """x~ (int8 [M][K]) and beta (fp32 [M]) of device activations x."""
    a = _Args()
    import torch
    M, K = x.shape
    if xq is None:
        xq = torch.empty((M, K), dtype=torch.int8, device=x.device)
    if beta is None:
        beta = torch.empty((M,), dtype=torch.float32, device=x.device)
    _check(lib().bitlinear_quant_act(a.ptr(x, "x"), _xdt(x), M, K,
                                     a.ptr(xq, "xq", torch.int8, (M, K)),
                                     a.ptr(beta, "beta", torch.float32, (M,)), _stream(stream)),
           "bitlinear_quant_act")
    return xq, beta


# ---------------------------------------------------------------- forward

def bitlinear_workspace_bytes(M: int, N: int, K: int, path: int = PATH_AUTO) -> int:
    return int(lib().bitlinear_workspace_bytes_path(M, N, K, path))


def bitlinear_forward(x, packed, gamma: float, N: int, y=None, workspace=None,
                      stream=None, acc=None, xq=None, beta=None, path: int = PATH_AUTO):
    """y (bf16 [M][N]) = BitLinear(x) with device-resident packed weights.

    ``workspace`` is a device uint8 tensor of at least
    ``bitlinear_workspace_bytes(M, N, K, path)`` bytes (allocated here when
    omitted); ``acc``/``xq``/``beta`` are optional debug outputs of the
    integer stages."""
    a = _Args()
    import torch
    M, K = x.shape
    if y is None:
        y = torch.empty((M, N), dtype=torch.bfloat16, device=x.device)
    need = bitlinear_workspace_bytes(M, N, K, path)
    if need == ctypes.c_size_t(-1).value:
        raise BitLinearError(BITLINEAR_ERR_SHAPE, "bitlinear_workspace_bytes")
    if workspace is None and need > 0:
        workspace = torch.empty((need,), dtype=torch.uint8, device=x.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    args = (a.ptr(x, "x"), _xdt(x), M, K, a.packed(packed, N, K), float(gamma), N,
            a.ptr(y, "y", torch.bfloat16, (M, N)), a.ptr(workspace, "workspace"), ws_bytes,
            _stream(stream), a.ptr(acc, "acc", torch.int32, (M, N)),
            a.ptr(xq, "xq", torch.int8, (M, K)), a.ptr(beta, "beta", torch.float32, (M,)))
    if path == PATH_AUTO:
        rc = lib().bitlinear_forward(*args)
    else:
        rc = lib().bitlinear_forward_ex(*args, path)
    _check(rc, "bitlinear_forward")
    return y


def bitlinear_forward_b3(x, packed_b3, gamma: float, N: int, y=None, stream=None, acc=None,
                         xq=None, beta=None):
    """y (bf16 [M][N]) = BitLinear(x) with base-3 packed weights (the GEMV
    path: M <= 16); ``acc``/``xq``/``beta`` are optional debug outputs."""
    a = _Args()
    import torch
    M, K = x.shape
    if y is None:
        y = torch.empty((M, N), dtype=torch.bfloat16, device=x.device)
    need = bitlinear_packed_bytes_b3(N, K) if N >= 1 and K >= 128 and K % 128 == 0 else 1
    rc = lib().bitlinear_forward_b3(
        a.ptr(x, "x"), _xdt(x), M, K, a.ptr(packed_b3, "packed_b3", torch.uint8, min_numel=need),
        float(gamma), N, a.ptr(y, "y", torch.bfloat16, (M, N)), _stream(stream),
        a.ptr(acc, "acc", torch.int32, (M, N)), a.ptr(xq, "xq", torch.int8, (M, K)),
        a.ptr(beta, "beta", torch.float32, (M,)))
    _check(rc, "bitlinear_forward_b3")
    return y


def bitlinear_forward_rmsnorm(x, packed, gamma: float, N: int, norm_gain,
                              eps: float = RMSNORM_EPS, y=None, workspace=None, stream=None,
                              acc=None, xq=None, beta=None, path: int = PATH_AUTO):
    """y (bf16 [M][N]) = BitLinear(RMSNorm(x)): every token is normalised as
    (x * r) * g with r = 1 / sqrt(mean(x^2) + eps) and the fp32 gains
    ``norm_gain`` [K] before its quantisation, in the same launch. Other
    arguments as for ``bitlinear_forward``; ``xq``/``beta`` return the
    quantised normalised tokens."""
    a = _Args()
    import torch
    M, K = x.shape
    if y is None:
        y = torch.empty((M, N), dtype=torch.bfloat16, device=x.device)
    need = bitlinear_workspace_bytes(M, N, K, path)
    if need == ctypes.c_size_t(-1).value:
        raise BitLinearError(BITLINEAR_ERR_SHAPE, "bitlinear_workspace_bytes")
    if workspace is None and need > 0:
        workspace = torch.empty((need,), dtype=torch.uint8, device=x.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    rc = lib().bitlinear_forward_rmsnorm(
        a.ptr(x, "x"), _xdt(x), M, K, a.ptr(norm_gain, "norm_gain", torch.float32, (K,)),
        float(eps), a.packed(packed, N, K), float(gamma), N,
        a.ptr(y, "y", torch.bfloat16, (M, N)), a.ptr(workspace, "workspace"), ws_bytes,
        _stream(stream), a.ptr(acc, "acc", torch.int32, (M, N)),
        a.ptr(xq, "xq", torch.int8, (M, K)), a.ptr(beta, "beta", torch.float32, (M,)), path)
    _check(rc, "bitlinear_forward_rmsnorm")
    return y


def bitlinear_forward_inject_timeout(x, packed, gamma: float, N: int, timeout_us: int,
                                     y=None, workspace=None, stream=None,
                                     path: int = PATH_TC) -> int:
    """Run the GEMV (path=PATH_GEMV) or the tensor-core GEMM (PATH_TC) with
    one wait made to run out; returns the status the launch reported (the
    fault is read by bitlinear_get_fault)."""
    a = _Args()
    import torch
    M, K = x.shape
    if y is None:
        y = torch.empty((M, N), dtype=torch.bfloat16, device=x.device)
    need = bitlinear_workspace_bytes(M, N, K, path)
    if workspace is None:
        workspace = torch.empty((max(need, 1),), dtype=torch.uint8, device=x.device)
    return int(lib().bitlinear_forward_inject_timeout(
        a.ptr(x, "x"), _xdt(x), M, K, a.packed(packed, N, K), float(gamma), N,
        a.ptr(y, "y", torch.bfloat16, (M, N)), a.ptr(workspace, "workspace", torch.uint8),
        workspace.numel(), _stream(stream), int(path), int(timeout_us)))


def bitlinear_forward_grouped_rmsnorm(problems, gains, eps: float = RMSNORM_EPS,
                                      stream=None, workspace=None):
    """bitlinear_forward_grouped with each problem's tokens RMS-normalised by
    its own fp32 gains (``gains``: one [K] device tensor per problem).
    ``workspace`` (bitlinear_workspace_bytes_grouped bytes) is needed when
    any problem takes the tensor-core path. Returns the list of outputs."""
    import torch
    if not problems:
        return []
    if len(gains) != len(problems):
        raise ValueError("one gain tensor per problem")
    xdt = _xdt(problems[0][0])
    a = _Args()
    arr, outs = _problem_array(problems, alloc_y=True, a=a)
    gp = (ctypes.c_void_p * len(problems))(
        *[a.ptr(g, f"gains[{i}]", torch.float32, (problems[i][0].shape[1],))
          for i, g in enumerate(gains)])
    ws = None if workspace is None else a.ptr(workspace, "workspace", torch.uint8)
    ws_bytes = 0 if workspace is None else workspace.numel()
    _check(lib().bitlinear_forward_grouped_rmsnorm(ctypes.addressof(arr), ctypes.addressof(gp),
                                                   len(problems), float(eps), xdt, ws, ws_bytes,
                                                   _stream(stream)),
           "bitlinear_forward_grouped_rmsnorm")
    return outs


def bitlinear_workspace_bytes_ffn(M: int, K: int, F: int) -> int:
    return int(lib().bitlinear_workspace_bytes_ffn(M, K, F))


def bitlinear_ffn_forward(x, gate, up, down, gains=(None, None, None),
                          eps: float = RMSNORM_EPS, h=None, y=None, workspace=None,
                          stream=None, gate_y=None, up_y=None):
    """The feed-forward block: y = down(h), h = max(gate(x), 0)^2 * up(x) in
    fp32, for M decode tokens x [M][K]. ``gate``, ``up`` and ``down`` are
    (packed, gamma) pairs (gate/up F x K, down K x F); ``gains`` gives each
    BitLinear's RMSNorm gains (fp32 device tensors or None; gate and up
    together). Returns (y bf16 [M][K], h fp32 [M][F]); ``gate_y``/``up_y``
    optionally receive the bf16 gate and up outputs."""
    a = _Args()
    import torch
    M, K = x.shape
    (gp, gg), (upk, ug), (dp, dg) = gate, up, down
    F = _ffn_width(upk, K)
    if h is None:
        h = torch.empty((M, F), dtype=torch.float32, device=x.device)
    if y is None:
        y = torch.empty((M, K), dtype=torch.bfloat16, device=x.device)
    need = bitlinear_workspace_bytes_ffn(M, K, F)
    if need == ctypes.c_size_t(-1).value:
        raise BitLinearError(BITLINEAR_ERR_SHAPE, "bitlinear_workspace_bytes_ffn")
    if workspace is None and need > 0:
        workspace = torch.empty((need,), dtype=torch.uint8, device=x.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    g0, g1, g2 = gains
    rc = lib().bitlinear_ffn_forward(
        a.ptr(x, "x"), _xdt(x), M, K, F, a.packed(gp, F, K), float(gg), a.packed(upk, F, K),
        float(ug), a.packed(dp, K, F), float(dg),
        a.ptr(g0, "gate gain", torch.float32, (K,)), a.ptr(g1, "up gain", torch.float32, (K,)),
        a.ptr(g2, "down gain", torch.float32, (F,)), float(eps),
        a.ptr(h, "h", torch.float32, (M, F)), a.ptr(y, "y", torch.bfloat16, (M, K)),
        a.ptr(workspace, "workspace"), ws_bytes, _stream(stream),
        a.ptr(gate_y, "gate_y", torch.bfloat16, (M, F)),
        a.ptr(up_y, "up_y", torch.bfloat16, (M, F)))
    _check(rc, "bitlinear_ffn_forward")
    return y, h


def _ffn_width(packed, K: int) -> int:
    """F of an F x K packed matrix whose F is a multiple of 16 (as every d_ff
    the feed-forward call accepts, a multiple of 128, is)."""
    return packed.numel() // (K // 4)


def bitlinear_get_fault(stream=None) -> tuple[int, int]:
    """(status, fault word); synchronises the stream and clears the word."""
    word = ctypes.c_int(0)
    rc = lib().bitlinear_get_fault(ctypes.addressof(word), _stream(stream))
    return int(rc), int(word.value)


def bitlinear_forward_noalloc(x, packed, gamma: float, N: int, y=None, stream=None):
    """y = BitLinear(x) on the tensor-core path with the library's static
    scratch instead of a workspace, for callers that cannot allocate device
    memory (see include/bitlinear.h for the size limit and the sharing rules).
    Pass ``y`` to keep this wrapper from allocating the output."""
    a = _Args()
    import torch
    M, K = x.shape
    if y is None:
        y = torch.empty((M, N), dtype=torch.bfloat16, device=x.device)
    _check(lib().bitlinear_forward_noalloc(a.ptr(x, "x"), _xdt(x), M, K, a.packed(packed, N, K),
                                           float(gamma), N, a.ptr(y, "y", torch.bfloat16, (M, N)),
                                           _stream(stream)),
           "bitlinear_forward_noalloc")
    return y


def _problem_array(problems, alloc_y, a=None, b3=False):
    import torch
    arr = (_Problem * len(problems))()
    outs = []
    for i, (x, packed, gamma, N, y) in enumerate(problems):
        M, K = x.shape
        if y is None and alloc_y:
            y = torch.empty((M, N), dtype=torch.bfloat16, device=x.device)
        outs.append(y)
        if alloc_y:
            if b3:
                need = (bitlinear_packed_bytes_b3(N, K)
                        if N >= 1 and K >= 128 and K % 128 == 0 else 1)
                pk = a.ptr(packed, f"problems[{i}].packed_b3", torch.uint8, min_numel=need)
            else:
                pk = a.packed(packed, N, K)
            arr[i] = _Problem(a.ptr(x, f"problems[{i}].x"), M, K, N, pk, float(gamma),
                              a.ptr(y, f"problems[{i}].y", torch.bfloat16, (M, N)))
        else:                              # sizing only: shapes, no pointers
            arr[i] = _Problem(None, M, K, N, None, float(gamma), None)
    return arr, outs


def bitlinear_workspace_bytes_grouped(problems) -> int:
    """Workspace bytes of ``bitlinear_forward_grouped(problems, workspace=...)``
    for a list of (x, packed, gamma, N, y) (only the shapes are read)."""
    arr, _ = _problem_array(problems, alloc_y=False)
    return lib().bitlinear_workspace_bytes_grouped(ctypes.addressof(arr), len(problems))


def bitlinear_forward_grouped(problems, stream=None, workspace=None):
    """Several independent BitLinear matmuls in one launch (pair). ``problems``
    is a list of (x, packed, gamma, N, y) with device tensors (y may be None to
    allocate it here); all x share one dtype. Without ``workspace`` every
    problem must fit the GEMV (one launch); with it any batch size is accepted
    (``bitlinear_forward_grouped_ws``). Returns the list of outputs."""
    import torch
    if not problems:
        return []
    xdt = _xdt(problems[0][0])
    a = _Args()
    arr, outs = _problem_array(problems, alloc_y=True, a=a)
    if workspace is None:
        _check(lib().bitlinear_forward_grouped(ctypes.addressof(arr), len(problems), xdt,
                                               _stream(stream)),
               "bitlinear_forward_grouped")
    else:
        _check(lib().bitlinear_forward_grouped_ws(ctypes.addressof(arr), len(problems), xdt,
                                                  a.ptr(workspace, "workspace", torch.uint8),
                                                  workspace.numel(), _stream(stream)),
               "bitlinear_forward_grouped_ws")
    return outs


def bitlinear_forward_grouped_b3(problems, stream=None):
    """bitlinear_forward_grouped with base-3 packed weights (one GEMV
    launch). ``problems`` is a list of (x, packed_b3, gamma, N, y) with device
    tensors (y may be None). Returns the list of outputs."""
    if not problems:
        return []
    xdt = _xdt(problems[0][0])
    a = _Args()
    arr, outs = _problem_array(problems, alloc_y=True, a=a, b3=True)
    _check(lib().bitlinear_forward_grouped_b3(ctypes.addressof(arr), len(problems), xdt,
                                              _stream(stream)),
           "bitlinear_forward_grouped_b3")
    return outs


def _host_buffer(t, name: str, dtype, numel: int) -> int:
    if t.device.type != "cpu":
        raise ValueError(f"{name} must be a host tensor (got device {t.device})")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if t.numel() != numel:
        raise ValueError(f"{name} holds {t.numel()} elements, {numel} expected")
    return t.data_ptr()


class GroupedHostCall:
    """bitlinear_forward_grouped_host with its problem list checked and
    marshalled once. ``problems`` is a list of (x_dev, packed, gamma, N,
    y_dev): the device staging buffers for the tokens and outputs (allocated
    back to back, one copy serves all of them), the packed weights and gamma.
    Each call takes a host tensor of every problem's tokens in problem order
    (sum of M*K elements of x's dtype) and a host bf16 tensor for every
    problem's outputs (sum of M*N elements), and makes one library call:
    copy in, grouped launch, copy out, enqueued on ``stream`` (the current
    stream when None). Pinned host tensors keep the copies asynchronous;
    ``y_host`` holds the results once the stream has synchronised. The
    object holds references to the problems' tensors, so their memory stays
    theirs for as long as the prepared call exists."""

    __slots__ = ("_arr", "_count", "_xdt", "_x_dtype", "_x_numel", "_y_numel", "_stream",
                 "_tensors")

    def __init__(self, problems, stream=None):
        if not problems:
            raise ValueError("at least one problem")
        if any(pr[4] is None for pr in problems):
            raise ValueError("every problem needs its device output buffer y_dev")
        self._xdt = _xdt(problems[0][0])
        self._x_dtype = problems[0][0].dtype
        self._arr, _ = _problem_array(problems, alloc_y=True, a=_Args())
        self._tensors = [(pr[0], pr[1], pr[4]) for pr in problems]
        self._count = len(problems)
        self._x_numel = sum(pr[0].numel() for pr in problems)
        self._y_numel = sum(pr[0].shape[0] * pr[3] for pr in problems)
        self._stream = _stream(stream)

    def __call__(self, x_host, y_host):
        import torch
        _check(lib().bitlinear_forward_grouped_host(
                   ctypes.addressof(self._arr), self._count, self._xdt,
                   _host_buffer(x_host, "x_host", self._x_dtype, self._x_numel),
                   _host_buffer(y_host, "y_host", torch.bfloat16, self._y_numel), self._stream),
               "bitlinear_forward_grouped_host")
        return y_host


def bitlinear_forward_grouped_host(problems, x_host, y_host, stream=None):
    """One grouped decode call with host tokens and outputs (see
    GroupedHostCall, which prepares the problem list once for repeated
    calls). Returns ``y_host``, valid after the stream synchronises."""
    return GroupedHostCall(problems, stream)(x_host, y_host)
