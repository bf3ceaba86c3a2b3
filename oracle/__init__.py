"""CPU oracle for the BitLinear W1.58A8 matmul -- TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package. The CUDA library never imports, links or
runs it, and the oracle shares no code with the library.

The arithmetic lives in ``bitlinear_oracle.c`` (plain C, built with gcc into
``liboracle.so`` next to it); this module only compiles it on demand and
marshals numpy arrays through ctypes. Every function cites the passage of
"BitNet b1.58 2B4T Guide: Scaling Native 1-Bit LLMs" it follows in the C file.

Functions:
    absmean_gamma(W)            gamma = max(mean|W|, 1e-5)
    ternarize(W, gamma)         W~ = clip(round(W / gamma), -1, 1)  (int8)
    bf16_to_f32(bits)           exact widening of bf16 bit patterns
    rmsnorm(x, g, eps)          (x * r) * g per token, r = 1/sqrt(mean x^2 + eps)
    quant_act(x)                (x~ int8 [M][K], beta fp32 [M])
    matmul_i32(xq, Wq)          acc = x~ W~^T in int32
    matmul_i32_pairs(xq, Wq, ms, ns)   acc at sampled (m, n) pairs
    f32_to_bf16(f)              RNE rounding to bf16 bit patterns (uint16)
    rescale_bf16(acc, beta, gamma)     y bf16 bits [M][N]
    pack_codes(Wq)              the 2-bit packed layout (flat uint8)
    pack_codes_b3(Wq)           the base-3 layout, 5 codes per byte (flat uint8)
    relu2_glu(gate, up)         h = max(gate, 0)^2 * up (fp32, elementwise)
    forward(x, W)               the whole path, returning every stage
    ffn(x, W_gate, W_up, W_down)   gate/up -> gated ReLU^2 -> down, every stage
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "bitlinear_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
# the same source built with -fopenmp: the benchmark's all-core CPU baseline
_OMP_LIB_PATH = os.path.join(_HERE, "liboracle_omp.so")
CFLAGS = ["-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off",
          "-fno-fast-math", "-Wall", "-Wextra"]

# nn.RMSNorm's default eps for fp32 inputs: the fp32 machine epsilon
RMSNORM_EPS = float(np.finfo(np.float32).eps)

_lock = threading.Lock()
_lib = None


def build(src: str = _SRC, out: str = _LIB_PATH, extra_flags=()) -> str:
    """Compile the C oracle with gcc. Returns the path of the shared object."""
    cmd = ["gcc", *CFLAGS, *extra_flags, src, "-o", out, "-lm"]
    subprocess.run(cmd, check=True, capture_output=True, text=True)
    return out


def _declare(lib):
    c_i64 = ctypes.c_int64
    p = ctypes.c_void_p
    lib.oracle_absmean_gamma.restype = ctypes.c_float
    lib.oracle_absmean_gamma.argtypes = [p, c_i64, c_i64]
    lib.oracle_ternarize.restype = None
    lib.oracle_ternarize.argtypes = [p, c_i64, c_i64, ctypes.c_float, p]
    lib.oracle_bf16_to_f32.restype = None
    lib.oracle_bf16_to_f32.argtypes = [p, c_i64, p]
    lib.oracle_rmsnorm.restype = None
    lib.oracle_rmsnorm.argtypes = [p, c_i64, c_i64, p, ctypes.c_float, p]
    lib.oracle_quant_act.restype = None
    lib.oracle_quant_act.argtypes = [p, c_i64, c_i64, p, p]
    lib.oracle_matmul_i32.restype = None
    lib.oracle_matmul_i32.argtypes = [p, p, c_i64, c_i64, c_i64, p]
    lib.oracle_matmul_i32_pairs.restype = None
    lib.oracle_matmul_i32_pairs.argtypes = [p, p, c_i64, p, p, c_i64, p]
    lib.oracle_f32_to_bf16.restype = ctypes.c_uint16
    lib.oracle_f32_to_bf16.argtypes = [ctypes.c_float]
    lib.oracle_f32_to_bf16_array.restype = None
    lib.oracle_f32_to_bf16_array.argtypes = [p, c_i64, p]
    lib.oracle_rescale_bf16.restype = None
    lib.oracle_rescale_bf16.argtypes = [p, p, ctypes.c_float, c_i64, c_i64, p]
    lib.oracle_relu2_glu.restype = None
    lib.oracle_relu2_glu.argtypes = [p, p, c_i64, p]
    lib.oracle_pack_codes.restype = ctypes.c_int
    lib.oracle_pack_codes.argtypes = [p, c_i64, c_i64, p]
    lib.oracle_pack_codes_b3.restype = ctypes.c_int
    lib.oracle_pack_codes_b3.argtypes = [p, c_i64, c_i64, p]
    return lib


def build_omp() -> str:
    """The same C source compiled with -fopenmp (integer products over all
    cores). The benchmark's all-core CPU baseline and the full-size parity
    tests use it; the CPU tests check that it gives the single-threaded
    build's results."""
    return build(_SRC, _OMP_LIB_PATH, extra_flags=("-fopenmp",))


_omp_lib = None


def load_omp():
    """Load (building first if needed) the OpenMP build of the oracle."""
    global _omp_lib
    with _lock:
        if _omp_lib is None:
            if (not os.path.exists(_OMP_LIB_PATH) or
                    os.path.getmtime(_OMP_LIB_PATH) < os.path.getmtime(_SRC)):
                build_omp()
            _omp_lib = _declare(ctypes.CDLL(_OMP_LIB_PATH))
    return _omp_lib


def load(path: str | None = None):
    """Load (building first if needed) and return the ctypes library.

    With ``path`` given, load that shared object instead of the default one
    (used by the tests that plant mistakes in a modified copy)."""
    global _lib
    if path is not None:
        return _declare(ctypes.CDLL(path))
    with _lock:
        if _lib is None:
            stale = (not os.path.exists(_LIB_PATH) or
                     os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC))
            if stale:
                build()
            _lib = _declare(ctypes.CDLL(_LIB_PATH))
    return _lib


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


class Oracle:
    """Thin numpy front end over one loaded copy of the C oracle."""

    def __init__(self, lib=None):
        self.lib = lib if lib is not None else load()

    def absmean_gamma(self, W) -> np.float32:
        W = _c(W, np.float32)
        N, K = W.shape
        return np.float32(self.lib.oracle_absmean_gamma(_ptr(W), N, K))

    def ternarize(self, W, gamma) -> np.ndarray:
        W = _c(W, np.float32)
        out = np.empty(W.shape, dtype=np.int8)
        self.lib.oracle_ternarize(_ptr(W), W.shape[0], W.shape[1],
                                  float(np.float32(gamma)), _ptr(out))
        return out

    def bf16_to_f32(self, bits) -> np.ndarray:
        bits = _c(bits, np.uint16)
        out = np.empty(bits.shape, dtype=np.float32)
        self.lib.oracle_bf16_to_f32(_ptr(bits), bits.size, _ptr(out))
        return out

    def rmsnorm(self, x, g=None, eps=RMSNORM_EPS) -> np.ndarray:
        """RMS-normalised rows of fp32 x [M][K] with gain g [K] (ones when
        omitted)."""
        x = _c(x, np.float32)
        M, K = x.shape
        g = np.ones((K,), dtype=np.float32) if g is None else _c(g, np.float32)
        assert g.shape == (K,)
        out = np.empty((M, K), dtype=np.float32)
        self.lib.oracle_rmsnorm(_ptr(x), M, K, _ptr(g), float(np.float32(eps)),
                                _ptr(out))
        return out

    def quant_act(self, x):
        x = _c(x, np.float32)
        M, K = x.shape
        xq = np.empty((M, K), dtype=np.int8)
        beta = np.empty((M,), dtype=np.float32)
        self.lib.oracle_quant_act(_ptr(x), M, K, _ptr(xq), _ptr(beta))
        return xq, beta

    def matmul_i32(self, xq, Wq) -> np.ndarray:
        xq = _c(xq, np.int8)
        Wq = _c(Wq, np.int8)
        M, K = xq.shape
        N, K2 = Wq.shape
        assert K == K2
        acc = np.empty((M, N), dtype=np.int32)
        self.lib.oracle_matmul_i32(_ptr(xq), _ptr(Wq), M, N, K, _ptr(acc))
        return acc

    def matmul_i32_pairs(self, xq, Wq, ms, ns) -> np.ndarray:
        xq = _c(xq, np.int8)
        Wq = _c(Wq, np.int8)
        ms = _c(ms, np.int64)
        ns = _c(ns, np.int64)
        assert ms.shape == ns.shape and xq.shape[1] == Wq.shape[1]
        acc = np.empty(ms.shape, dtype=np.int32)
        self.lib.oracle_matmul_i32_pairs(_ptr(xq), _ptr(Wq), xq.shape[1],
                                         _ptr(ms), _ptr(ns), ms.size,
                                         _ptr(acc))
        return acc

    def f32_to_bf16(self, f) -> np.ndarray:
        f = _c(f, np.float32)
        out = np.empty(f.shape, dtype=np.uint16)
        self.lib.oracle_f32_to_bf16_array(_ptr(f), f.size, _ptr(out))
        return out

    def rescale_bf16(self, acc, beta, gamma) -> np.ndarray:
        acc = _c(acc, np.int32)
        beta = _c(beta, np.float32)
        M, N = acc.shape
        y = np.empty((M, N), dtype=np.uint16)
        self.lib.oracle_rescale_bf16(_ptr(acc), _ptr(beta),
                                     float(np.float32(gamma)), M, N, _ptr(y))
        return y

    def pack_codes(self, Wq) -> np.ndarray:
        """The packed layout as a flat uint8 array of
        ceil(N/16) * 16 * K/4 bytes."""
        Wq = _c(Wq, np.int8)
        N, K = Wq.shape
        out = np.empty(((N + 15) // 16) * 16 * (K // 4), dtype=np.uint8)
        rc = self.lib.oracle_pack_codes(_ptr(Wq), N, K, _ptr(out))
        if rc != 0:
            raise ValueError("oracle_pack_codes: K % 128 != 0 or non-ternary")
        return out

    def pack_codes_b3(self, Wq) -> np.ndarray:
        """The base-3 layout (5 codes per byte, K padded to a multiple of
        160) of int8 ternary weights [N][K]."""
        Wq = _c(Wq, np.int8)
        N, K = Wq.shape
        Kp = (K + 159) // 160 * 160
        out = np.empty(((N + 15) // 16 * 16 * Kp // 5,), dtype=np.uint8)
        rc = self.lib.oracle_pack_codes_b3(_ptr(Wq), N, K, _ptr(out))
        if rc != 0:
            raise ValueError("oracle_pack_codes_b3: K % 128 != 0 or non-ternary")
        return out

    def relu2_glu(self, gate, up) -> np.ndarray:
        """h = max(gate, 0)^2 * up elementwise on fp32 arrays of one shape."""
        gate = _c(gate, np.float32)
        up = _c(up, np.float32)
        assert gate.shape == up.shape
        h = np.empty(gate.shape, dtype=np.float32)
        self.lib.oracle_relu2_glu(_ptr(gate), _ptr(up), gate.size, _ptr(h))
        return h

    def forward(self, x, W, gamma=None, norm_gain=None, norm_eps=RMSNORM_EPS):
        """The whole path on the CPU. ``x`` is fp32 [M][K] or bf16 bit
        patterns (uint16); ``W`` is the fp32 latent [N][K]. ``gamma`` may be
        supplied (e.g. the packer's) instead of recomputed. With ``norm_gain``
        (fp32 [K]) the tokens are RMS-normalised before quantisation (the
        listing's BitLinear.forward step 1). Returns a dict with gamma, Wq,
        xq, beta, acc and y (bf16 bit patterns)."""
        x = np.asarray(x)
        xf = self.bf16_to_f32(x) if x.dtype == np.uint16 else _c(x, np.float32)
        if norm_gain is not None:
            xf = self.rmsnorm(xf, norm_gain, norm_eps)
        g = self.absmean_gamma(W) if gamma is None else np.float32(gamma)
        Wq = self.ternarize(W, g)
        xq, beta = self.quant_act(xf)
        acc = self.matmul_i32(xq, Wq)
        y = self.rescale_bf16(acc, beta, g)
        return {"gamma": g, "Wq": Wq, "xq": xq, "beta": beta, "acc": acc,
                "y": y}

    def ffn(self, x, W_gate, W_up, W_down, gammas=(None, None, None),
            gains=(None, None, None), norm_eps=RMSNORM_EPS):
        """The feed-forward chain on the CPU: the gate and up BitLinears of
        the tokens x, the gated ReLU^2 of their bf16 outputs in fp32, and the
        down BitLinear of that fp32 h. ``gammas`` may supply each matrix's
        gamma (e.g. the packer's); ``gains`` gives each BitLinear's RMSNorm
        gains (None: no normalisation), the down projection's being the one
        ahead of its quantisation. Returns the three forward dicts and h."""
        rg = self.forward(x, W_gate, gammas[0], gains[0], norm_eps)
        ru = self.forward(x, W_up, gammas[1], gains[1], norm_eps)
        h = self.relu2_glu(self.bf16_to_f32(rg["y"]), self.bf16_to_f32(ru["y"]))
        rd = self.forward(h, W_down, gammas[2], gains[2], norm_eps)
        return {"gate": rg, "up": ru, "h": h, "down": rd}


_default = None


def default() -> Oracle:
    global _default
    if _default is None:
        _default = Oracle()
    return _default
