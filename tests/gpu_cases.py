"""Shared machinery of the GPU parity tests: build one BitLinear problem from
the seeded generators, run the CUDA library through its C ABI, run the
oracle on the same inputs, and compare stage by stage.

Bar (see the design notes): x~, beta and acc bit-exact; y within relative
error 1e-2 elementwise (y_oracle == 0 requires y == 0). The kernels follow
the oracle's operation order, so y is also expected to be bit-identical and
the helpers report how many elements are.
"""
from __future__ import annotations

import numpy as np

import oracle
import workloads
import ternary_weight_w1_b200 as bl

Y_REL_TOL = 1e-2


def bf16_bits_to_tensor(bits: np.ndarray, device="cuda"):
    import torch
    return torch.from_numpy(bits.view(np.int16).copy()).view(torch.bfloat16).to(device)


def tensor_to_bf16_bits(t) -> np.ndarray:
    import torch
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def bf16_value(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << 16).view(np.float32)


class Guarded:
    """An output tensor inside a larger buffer whose PAD_BYTES before and
    after it, and the output itself, start filled with a canary bit pattern
    no correct result holds. After a launch, check() fails if a kernel wrote
    past either end of the output (the interior is compared with the oracle,
    so an element left unwritten shows there)."""

    PAD_BYTES = 256
    RAW = {1: "int8", 2: "int16", 4: "int32"}

    def __init__(self, shape, dtype, device, canary: int):
        import torch
        esz = torch.empty((), dtype=dtype).element_size()
        self.pad = self.PAD_BYTES // esz
        self.n = int(np.prod(shape))
        self.canary = canary
        self.raw = torch.full((2 * self.pad + self.n,), canary,
                              dtype=getattr(torch, self.RAW[esz]), device=device)
        self.t = self.raw[self.pad:self.pad + self.n].view(dtype).view(*shape)

    def check(self, name: str = "output"):
        import torch
        head = self.raw[:self.pad]
        tail = self.raw[self.pad + self.n:]
        assert bool(torch.all(head == self.canary)), f"write before the start of {name}"
        assert bool(torch.all(tail == self.canary)), f"write past the end of {name}"


# canaries: a bf16 NaN, an accumulator far beyond 127 * 65536, an x~ of -128
# (|x~| <= 127) and an fp32 NaN
CANARY_Y = 0x7FA5
CANARY_ACC = 0x5A5A5A5A
CANARY_XQ = -128
CANARY_BETA = 0x7FC0A5A5


def guarded_outputs(M, N, K, device, debug=True):
    """Guarded y (bf16 [M][N]) and, with `debug`, acc, xq and beta."""
    import torch
    out = {"y": Guarded((M, N), torch.bfloat16, device, CANARY_Y)}
    if debug:
        out["acc"] = Guarded((M, N), torch.int32, device, CANARY_ACC)
        out["xq"] = Guarded((M, K), torch.int8, device, CANARY_XQ)
        out["beta"] = Guarded((M,), torch.float32, device, CANARY_BETA)
    return out


def read_guarded(g) -> dict:
    """Checks every canary and returns the outputs as numpy arrays (y as
    bf16 bit patterns)."""
    for name, v in g.items():
        v.check(name)
    out = {"y": tensor_to_bf16_bits(g["y"].t)}
    for name in ("acc", "xq", "beta"):
        if name in g:
            out[name] = g[name].t.cpu().numpy()
    return out


class Case:
    """One problem: inputs, the packed weights and the oracle's view of them."""

    def __init__(self, M, K, N, w_seed=1, x_seed=2, x_dtype="bf16", outliers=True,
                 W=None, x=None):
        self.M, self.K, self.N = M, K, N
        self.W = workloads.latent_weights(N, K, w_seed) if W is None else W
        xf = workloads.activations_f32(M, K, x_seed, outliers) if x is None else x
        self.x_dtype = x_dtype
        if x_dtype == "bf16":
            self.x_bits = workloads.to_bf16_bits(xf)
            self.orc = oracle.default()
            self.xf = self.orc.bf16_to_f32(self.x_bits)
        else:
            self.orc = oracle.default()
            self.xf = np.ascontiguousarray(xf, dtype=np.float32)
        self.packed, self.gamma = bl.bitlinear_pack_weights(self.W)
        # the oracle ternarises with the packer's gamma (checked separately)
        self.Wq = self.orc.ternarize(self.W, np.float32(self.gamma))
        self.xq, self.beta = self.orc.quant_act(self.xf)

    def x_tensor(self):
        import torch
        if self.x_dtype == "bf16":
            return bf16_bits_to_tensor(self.x_bits)
        return torch.from_numpy(self.xf).cuda()

    def packed_tensor(self):
        import torch
        return torch.from_numpy(self.packed).cuda()

    def run(self, path=bl.PATH_AUTO, debug=True):
        import torch
        x = self.x_tensor()
        packed = self.packed_tensor()
        g = guarded_outputs(self.M, self.N, self.K, x.device, debug)
        dbg = {k: g[k].t for k in ("acc", "xq", "beta")} if debug else {}
        bl.bitlinear_forward(x, packed, self.gamma, self.N, y=g["y"].t, path=path, **dbg)
        torch.cuda.synchronize()
        return read_guarded(g)

    # ---------------------------------------------------------- checks

    def oracle_full(self, orc=None):
        """acc and y of the whole problem; ``orc`` may name another copy of
        the oracle for the integer products (the OpenMP build, whose results
        equal the single-threaded build's, for the full-size cases)."""
        acc = (orc or self.orc).matmul_i32(self.xq, self.Wq)
        y = self.orc.rescale_bf16(acc, self.beta, np.float32(self.gamma))
        return acc, y

    def check_quant(self, got):
        np.testing.assert_array_equal(got["beta"], self.beta)
        np.testing.assert_array_equal(got["xq"], self.xq)

    def check_full(self, got, orc=None):
        self.check_quant(got)
        acc, y = self.oracle_full(orc)
        np.testing.assert_array_equal(got["acc"], acc)
        return check_y(got["y"], y)

    def sample_pairs(self, count, seed=0, full_rows=2, full_cols=2):
        r = np.random.Generator(np.random.PCG64(seed))
        ms = [r.integers(0, self.M, count)]
        ns = [r.integers(0, self.N, count)]
        for m in r.integers(0, self.M, full_rows):
            ms.append(np.full(self.N, m))
            ns.append(np.arange(self.N))
        for n in r.integers(0, self.N, full_cols):
            ms.append(np.arange(self.M))
            ns.append(np.full(self.M, n))
        ms.append(np.array([self.M - 1])); ns.append(np.array([self.N - 1]))
        return np.concatenate(ms).astype(np.int64), np.concatenate(ns).astype(np.int64)

    def check_sampled(self, got, count=20000, seed=0):
        self.check_quant(got)
        ms, ns = self.sample_pairs(count, seed)
        acc = self.orc.matmul_i32_pairs(self.xq, self.Wq, ms, ns)
        np.testing.assert_array_equal(got["acc"][ms, ns], acc)
        # the oracle's rescale, one sampled output per "row"
        y_ref = self.orc.rescale_bf16(acc.reshape(-1, 1), self.beta[ms],
                                      np.float32(self.gamma))[:, 0]
        return check_y(got["y"][ms, ns], y_ref)


# Half-integer band of the normalised forms: an x~ whose oracle value
# n * 127 / beta lies this close to a tie may round to either neighbour.
TIE_BAND = 1e-4


class NormCase(Case):
    """A Case whose tokens go through the RMS normalisation first
    (bitlinear_forward_rmsnorm against the oracle's rmsnorm + forward).

    The device adds a token's squares in another order than the oracle (both
    in double), so its fp32 mean can differ in the last bit when the two sums
    straddle an fp32 rounding boundary; every normalised value then moves by
    at most an ulp. Hence beta is compared within 2 ulps and x~ exactly
    except within TIE_BAND of a half-integer, and acc and y exactly against
    the oracle applied to the kernel's own x~ and beta."""

    def __init__(self, M, K, N, g_seed=7, eps=bl.RMSNORM_EPS, gain=None, **kw):
        super().__init__(M, K, N, **kw)
        self.eps = eps
        self.gain = workloads.norm_gains(K, g_seed) if gain is None else gain
        self.xn = self.orc.rmsnorm(self.xf, self.gain, eps)
        self.xq, self.beta = self.orc.quant_act(self.xn)

    def run(self, path=bl.PATH_AUTO, debug=True):
        import torch
        x = self.x_tensor()
        gain = torch.from_numpy(self.gain).to(x.device)
        g = guarded_outputs(self.M, self.N, self.K, x.device, True)
        bl.bitlinear_forward_rmsnorm(x, self.packed_tensor(), self.gamma, self.N, gain,
                                     eps=self.eps, y=g["y"].t, acc=g["acc"].t, xq=g["xq"].t,
                                     beta=g["beta"].t, path=path)
        torch.cuda.synchronize()
        return read_guarded(g)

    def check_norm_quant(self, got) -> int:
        """x~ and beta of the normalised tokens (see the class docstring);
        returns how many x~ differ from the oracle's."""
        b_or = self.beta.astype(np.float64)
        assert np.all(np.abs(got["beta"].astype(np.float64) - b_or) <=
                      2 * np.spacing(self.beta).astype(np.float64))
        v = self.xn.astype(np.float64) * 127.0 / b_or[:, None]
        near_tie = np.abs(np.abs(v - np.floor(v)) - 0.5) < TIE_BAND
        diff = got["xq"].astype(np.int32) - self.xq.astype(np.int32)
        assert np.all(np.abs(diff) <= 1)
        assert np.all(near_tie[diff != 0])
        return int(np.count_nonzero(diff))

    def check_norm_full(self, got) -> int:
        ndiff = self.check_norm_quant(got)
        acc = self.orc.matmul_i32(got["xq"], self.Wq)
        np.testing.assert_array_equal(got["acc"], acc)
        np.testing.assert_array_equal(
            got["y"], self.orc.rescale_bf16(acc, got["beta"], np.float32(self.gamma)))
        return ndiff

    def check_norm_sampled(self, got, count=20000, seed=0) -> int:
        ndiff = self.check_norm_quant(got)
        ms, ns = self.sample_pairs(count, seed)
        acc = self.orc.matmul_i32_pairs(got["xq"], self.Wq, ms, ns)
        np.testing.assert_array_equal(got["acc"][ms, ns], acc)
        y_ref = self.orc.rescale_bf16(acc.reshape(-1, 1), got["beta"][ms],
                                      np.float32(self.gamma))[:, 0]
        np.testing.assert_array_equal(got["y"][ms, ns], y_ref)
        return ndiff


def check_y(y_bits: np.ndarray, y_ref_bits: np.ndarray) -> float:
    """Relative-error check of bf16 outputs; returns the fraction of
    bit-identical elements."""
    y = bf16_value(y_bits).astype(np.float64)
    r = bf16_value(y_ref_bits).astype(np.float64)
    assert np.all(np.isfinite(y))
    zero = r == 0
    assert np.all(y[zero] == 0)
    rel = np.abs(y[~zero] - r[~zero]) / np.abs(r[~zero])
    assert rel.size == 0 or rel.max() <= Y_REL_TOL, float(rel.max())
    return float(np.mean(y_bits == y_ref_bits))
