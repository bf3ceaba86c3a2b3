"""Pins for the CPU oracle: checks against facts fixed by the pages and by
mathematics, independent of the oracle's own code.

Each ``pin_*`` function takes an ``oracle.Oracle`` and raises AssertionError
when the oracle disagrees with the pinned fact. ``tests/test_oracle_pins.py``
runs them on the oracle; ``tests/test_oracle_mutants.py`` runs them on copies
of the oracle with a planted mistake and expects at least one to fail.

What pins what (pages: "BitNet b1.58 2B4T Guide: Scaling Native 1-Bit LLMs"
unless stated):
  * hand-worked examples under tests/golden/ (sections "Ternary Weight
    Quantization", "8-Bit Activation Quantization", "Matrix Multiplication as
    Pure Integer Addition");
  * brute force of the add/ignore/subtract form of the product (same section,
    the sum over W~ = +1 minus the sum over W~ = -1), written as Python loops;
  * library routines: torch.nn.functional.linear in float64 (exact for these
    integer sums), torch's fp32 -> bf16 conversion, numpy's float64 mean;
  * closed forms and invariants: constant and zero inputs, identity weights,
    +-a weights, the Gaussian zero fraction (about 31%, which the bitnet.xin
    guide's "Core Architecture" section quotes as about 32% zero entries),
    |x~| <= 127 with the per-token maximum reaching 127, the rounding bound
    |x~ - x*127/beta| <= 1/2, invariance under power-of-two scaling, and the
    bf16 rounding bound of the output;
  * the exact widening of every bf16 bit pattern against torch's conversion;
  * for the RMS normalisation ahead of quantisation (the listing's
    nn.RMSNorm member of BitLinear): torch's rms_norm in float64 within the
    fp32 error bound, constant rows in closed form, exact invariance under
    power-of-two scaling at eps = 0, and the gain applied last;
  * for the gated ReLU^2 of the feed-forward chain: exact products on bf16
    operands (float64 reference), closed forms, and the roles of the gate and
    up projections in the whole chain.
"""
from __future__ import annotations

import math
import os

import numpy as np

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


# ------------------------------------------------------------------ fixtures

def _parse_values(text: str):
    rows = [r.split() for r in text.split(";")]
    return [[float(v) for v in r] for r in rows if r]


def load_golden(name: str) -> dict:
    out = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, _, val = line.partition("=")
            out[key.strip()] = _parse_values(val)
    return out


def load_pack_cases(name: str = "pack_words.txt") -> list:
    """(name, N, K, [(row, k, value)], {offset: byte}, size) per golden case."""
    cases = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line.startswith("case"):
                continue
            head, _, rest = line.partition(":")
            shape, weights, bytes_part, size = [x.strip() for x in rest.split(";")]
            N = int(shape.split()[0].split("=")[1])
            K = int(shape.split()[1].split("=")[1])
            ws = []
            for item in weights.split("=")[1].split():
                r, k, v = item.split(",")
                ws.append((int(r), int(k), int(v)))
            by = {}
            for item in bytes_part.split("=")[1].split():
                off, val = item.split(":")
                by[int(off)] = int(val, 16)
            cases.append((head.split()[1], N, K, ws, by, int(size.split("=")[1])))
    return cases


def _f32(v):
    return np.asarray(v, dtype=np.float32)


def _bf16_value(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << 16).view(np.float32)


# ---------------------------------------------------------------- the pins

def pin_hand_example(orc):
    g = load_golden("hand_example.txt")
    W = _f32(g["W"])
    x = _f32(g["x"])
    r = orc.forward(x, W)
    gamma_ref = np.float32(g["gamma"][0][0])
    assert abs(float(r["gamma"]) - float(gamma_ref)) <= 2 * np.spacing(gamma_ref), r["gamma"]
    np.testing.assert_array_equal(r["Wq"], np.array(g["Wq"], dtype=np.int8))
    assert float(r["beta"][0]) == g["beta"][0][0]
    np.testing.assert_array_equal(r["xq"], np.array(g["xq"], dtype=np.int8))
    np.testing.assert_array_equal(r["acc"], np.array(g["acc"], dtype=np.int32))
    np.testing.assert_array_equal(_bf16_value(r["y"]), _f32(g["y"]))


def pin_weight_ties_even(orc):
    g = load_golden("weight_ties.txt")
    W = _f32(g["W"])
    gamma = orc.absmean_gamma(W)
    assert float(gamma) == g["gamma"][0][0]
    np.testing.assert_array_equal(orc.ternarize(W, gamma),
                                  np.array(g["Wq"], dtype=np.int8))


def pin_activation_ties_even(orc):
    g = load_golden("activation_ties.txt")
    xq, beta = orc.quant_act(_f32(g["x"]))
    assert float(beta[0]) == g["beta"][0][0]
    np.testing.assert_array_equal(xq, np.array(g["xq"], dtype=np.int8))


def pin_pack_words(orc):
    for name, N, K, ws, by, size in load_pack_cases():
        Wq = np.zeros((N, K), dtype=np.int8)
        for r, k, v in ws:
            Wq[r, k] = v
        got = orc.pack_codes(Wq)
        want = np.full(size, 0x55, dtype=np.uint8)
        for off, val in by.items():
            want[off] = val
        assert got.shape == want.shape, (name, got.shape)
        np.testing.assert_array_equal(got, want, err_msg=name)


def decode_packed_spec(packed: np.ndarray, N: int, K: int) -> np.ndarray:
    """Independent decoder of the 2-bit layout, bit by bit from its spec:
    row n = 16 blk + r; its weights k = 128 g + 16 w + 4 j + b sit in the
    32-bit little-endian word at byte blk*16*K/4 + 512 g + 32 r + 4 w, in
    bits 8b + 2j, as the code W~ + 1. Padding rows must decode to zeros."""
    packed = np.asarray(packed).reshape(-1)
    blocks = (N + 15) // 16
    assert packed.size == blocks * 16 * K // 4
    out = np.zeros((blocks * 16, K), dtype=np.int8)
    for blk in range(blocks):
        for r in range(16):
            for g in range(K // 128):
                for w in range(8):
                    base = blk * 16 * K // 4 + 512 * g + 32 * r + 4 * w
                    word = 0
                    for q in range(4):
                        word |= int(packed[base + q]) << (8 * q)
                    for j in range(4):
                        for b in range(4):
                            code = (word >> (8 * b + 2 * j)) & 3
                            assert code != 3
                            out[16 * blk + r, 128 * g + 16 * w + 4 * j + b] = code - 1
    assert np.all(out[N:] == 0)
    return out[:N]


def pin_pack_roundtrip(orc):
    r = np.random.Generator(np.random.PCG64(7))
    Wq = r.integers(-1, 2, size=(21, 256), dtype=np.int8)
    packed = orc.pack_codes(Wq)
    assert packed.size == 32 * 256 // 4
    np.testing.assert_array_equal(decode_packed_spec(packed, 21, 256), Wq)


def pin_pack_b3_bytes(orc):
    for name, N, K, ws, by, size in load_pack_cases("pack_b3_bytes.txt"):
        Wq = np.zeros((N, K), dtype=np.int8)
        for r, k, v in ws:
            Wq[r, k] = v
        got = orc.pack_codes_b3(Wq)
        want = np.full(size, 121, dtype=np.uint8)
        for off, val in by.items():
            want[off] = val
        assert got.shape == want.shape, (name, got.shape)
        np.testing.assert_array_equal(got, want, err_msg=name)


def decode_packed_b3_spec(packed: np.ndarray, N: int, K: int) -> np.ndarray:
    """Independent decoder of the base-3 layout from its spec: byte B of row
    n = 16 blk + r, group g sits at blk*16*Kp/5 + 512 g + 32 r + B and holds
    the base-3 digits of stream positions p = 5B + i (digit i is worth 3^i);
    position p = 16 w + 4 b + j is the weight k = 160 g + 16 w + 4 j + b.
    Padding rows and padding columns (k >= K) must decode to zeros."""
    packed = np.asarray(packed).reshape(-1)
    Kp = (K + 159) // 160 * 160
    blocks = (N + 15) // 16
    assert packed.size == blocks * 16 * Kp // 5
    out = np.zeros((blocks * 16, Kp), dtype=np.int8)
    for blk in range(blocks):
        for r in range(16):
            for g in range(Kp // 160):
                for B in range(32):
                    v = int(packed[blk * 16 * Kp // 5 + 512 * g + 32 * r + B])
                    assert v < 243
                    for i in range(5):
                        code = v % 3
                        v //= 3
                        p = 5 * B + i
                        w, b, j = p // 16, (p % 16) // 4, p % 4
                        out[16 * blk + r, 160 * g + 16 * w + 4 * j + b] = code - 1
    assert np.all(out[N:] == 0) and np.all(out[:, K:] == 0)
    return out[:N, :K]


def pin_pack_b3_roundtrip(orc):
    """Random ternary weights, ragged rows and a K that is not a multiple of
    160, decode back to themselves; both layouts decode to the same weights."""
    r = np.random.Generator(np.random.PCG64(8))
    for N, K in [(21, 384), (5, 128), (16, 640)]:
        Wq = r.integers(-1, 2, size=(N, K), dtype=np.int8)
        packed = orc.pack_codes_b3(Wq)
        assert packed.size == (N + 15) // 16 * 16 * ((K + 159) // 160 * 160) // 5
        np.testing.assert_array_equal(decode_packed_b3_spec(packed, N, K), Wq)
        np.testing.assert_array_equal(decode_packed_spec(orc.pack_codes(Wq), N, K), Wq)


def pin_constant_token(orc):
    for c in (0.75, -3.0, 1e-3):
        x = np.full((1, 40), c, dtype=np.float32)
        xq, beta = orc.quant_act(x)
        assert float(beta[0]) == abs(np.float32(c))
        assert np.all(xq == (127 if c > 0 else -127))


def pin_zero_inputs(orc):
    xq, beta = orc.quant_act(np.zeros((2, 32), dtype=np.float32))
    assert np.all(beta == np.float32(1e-5)) and np.all(xq == 0)
    W = np.zeros((8, 32), dtype=np.float32)
    gamma = orc.absmean_gamma(W)
    assert gamma == np.float32(1e-5)
    assert np.all(orc.ternarize(W, gamma) == 0)
    r = orc.forward(np.ones((2, 32), dtype=np.float32), W)
    assert np.all(r["acc"] == 0) and np.all(r["y"] == 0)


def pin_tiny_scale_epsilon(orc):
    # |x| below the epsilon: beta is clamped to 1e-5, so x~ = x * 127 / 1e-5.
    # 4e-6 * 127 / 1e-5 = 50.8, -2.6e-6 -> -33.02, 1e-6 -> 12.7 (no ties nearby)
    x = _f32([[4e-6, -2.6e-6, 0.0, 1e-6]])
    xq, beta = orc.quant_act(x)
    assert beta[0] == np.float32(1e-5)
    np.testing.assert_array_equal(xq[0], np.array([51, -33, 0, 13], np.int8))


def pin_identity_weights(orc):
    K = 48
    W = np.eye(K, dtype=np.float32)          # mean |W| = 1/K, diagonal -> K -> clip 1
    x = np.random.Generator(np.random.PCG64(3)).standard_normal((3, K)).astype(np.float32)
    r = orc.forward(x, W)
    np.testing.assert_array_equal(r["Wq"], np.eye(K, dtype=np.int8))
    np.testing.assert_array_equal(r["acc"], r["xq"].astype(np.int32))


def pin_plus_minus_a(orc):
    r = np.random.Generator(np.random.PCG64(11))
    W = np.where(r.random((16, 64)) < 0.5, -0.25, 0.25).astype(np.float32)
    gamma = orc.absmean_gamma(W)
    assert gamma == np.float32(0.25)
    np.testing.assert_array_equal(orc.ternarize(W, gamma), np.sign(W).astype(np.int8))
    Wc = np.full((3, 16), -0.125, dtype=np.float32)
    assert orc.absmean_gamma(Wc) == np.float32(0.125)
    assert np.all(orc.ternarize(Wc, np.float32(0.125)) == -1)


def pin_gamma_vs_numpy_mean(orc):
    W = np.random.Generator(np.random.PCG64(5)).standard_normal((64, 96)).astype(np.float32) * np.float32(0.02)
    ref = np.float32(np.mean(np.abs(W.astype(np.float64))))
    got = orc.absmean_gamma(W)
    assert abs(float(got) - float(ref)) <= np.spacing(ref), (got, ref)


def pin_zero_fraction(orc):
    # Gaussian latent: zero iff |W| < gamma/2 with gamma = sigma*sqrt(2/pi), so
    # P(0) = P(|Z| < sqrt(2/pi)/2) = erf(sqrt(2/pi)/2/sqrt(2)) ~ 0.310 and
    # P(+1) = P(-1) ~ 0.345.
    W = np.random.Generator(np.random.PCG64(0)).standard_normal((256, 256)).astype(np.float32) * np.float32(0.02)
    Wq = orc.ternarize(W, orc.absmean_gamma(W))
    p0 = math.erf(math.sqrt(2 / math.pi) / 2 / math.sqrt(2))
    frac0 = float(np.mean(Wq == 0))
    assert abs(frac0 - p0) < 0.01, (frac0, p0)
    assert abs(float(np.mean(Wq == 1)) - (1 - p0) / 2) < 0.01
    assert abs(float(np.mean(Wq == -1)) - (1 - p0) / 2) < 0.01
    assert set(np.unique(Wq).tolist()) <= {-1, 0, 1}


def pin_bruteforce_add_subtract(orc):
    r = np.random.Generator(np.random.PCG64(21))
    for (M, K, N) in ((1, 4, 1), (2, 7, 3), (4, 64, 16), (3, 33, 5)):
        xq = r.integers(-127, 128, size=(M, K), dtype=np.int8)
        Wq = r.integers(-1, 2, size=(N, K), dtype=np.int8)
        acc = orc.matmul_i32(xq, Wq)
        for m in range(M):
            for n in range(N):
                plus = sum(int(xq[m, k]) for k in range(K) if Wq[n, k] == 1)
                minus = sum(int(xq[m, k]) for k in range(K) if Wq[n, k] == -1)
                assert int(acc[m, n]) == plus - minus, (M, K, N, m, n)


def pin_exhaustive_single_term(orc):
    xq = np.arange(-128, 128, dtype=np.int8).reshape(256, 1)
    Wq = np.array([[-1], [0], [1]], dtype=np.int8)
    acc = orc.matmul_i32(xq, Wq)
    for i, v in enumerate(range(-128, 128)):
        assert acc[i].tolist() == [-v, 0, v]


def pin_matmul_vs_linear(orc):
    import torch
    r = np.random.Generator(np.random.PCG64(31))
    xq = r.integers(-127, 128, size=(6, 512), dtype=np.int8)
    Wq = r.integers(-1, 2, size=(40, 512), dtype=np.int8)
    acc = orc.matmul_i32(xq, Wq)
    ref = torch.nn.functional.linear(torch.from_numpy(xq.astype(np.float64)),
                                     torch.from_numpy(Wq.astype(np.float64)))
    np.testing.assert_array_equal(acc.astype(np.float64), ref.numpy())
    # sampled pairs agree with the full product
    ms = np.array([0, 5, 3, 2]); ns = np.array([0, 39, 17, 3])
    np.testing.assert_array_equal(orc.matmul_i32_pairs(xq, Wq, ms, ns), acc[ms, ns])


def pin_quant_act_invariants(orc):
    r = np.random.Generator(np.random.PCG64(41))
    x = r.standard_normal((16, 300)).astype(np.float32)
    x[:, r.choice(300, 3, replace=False)] *= 50
    x[3] *= 1e-3
    xq, beta = orc.quant_act(x)
    np.testing.assert_array_equal(beta, np.max(np.abs(x), axis=1))
    assert np.all(np.abs(xq.astype(np.int32)) <= 127)
    assert np.all(np.max(np.abs(xq.astype(np.int32)), axis=1) == 127)
    exact = x.astype(np.float64) * 127.0 / beta.astype(np.float64)[:, None]
    assert np.max(np.abs(xq - exact)) <= 0.5 + 1e-4
    assert np.all(np.sign(xq) * np.sign(x) >= 0)
    for m in range(x.shape[0]):
        order = np.argsort(x[m], kind="stable")
        assert np.all(np.diff(xq[m][order].astype(np.int32)) >= 0)


def pin_quant_act_pow2_invariance(orc):
    r = np.random.Generator(np.random.PCG64(43))
    x = r.standard_normal((4, 128)).astype(np.float32)
    base, _ = orc.quant_act(x)
    for e in (-7, -1, 3, 12):
        xq, _ = orc.quant_act(x * np.float32(2.0 ** e))
        np.testing.assert_array_equal(xq, base)


def pin_bf16_rounding_vs_torch(orc):
    import torch
    r = np.random.Generator(np.random.PCG64(51))
    f = (r.standard_normal(20000) * np.exp(r.uniform(-60, 60, 20000))).astype(np.float32)
    base = (r.integers(0, 2 ** 31, 4000, dtype=np.int64).astype(np.uint32) & np.uint32(0x7fff0000))
    ties = (base | np.uint32(0x8000)).view(np.float32)          # exact halfway cases
    near = (base | np.uint32(0x7fff)).view(np.float32)
    specials = np.array([0.0, -0.0, np.inf, -np.inf, 3.3895314e38, -3.3895314e38,
                         1e-40, -1e-45, 1.0, 2.359375], dtype=np.float32)
    allf = np.concatenate([f, ties, -ties, near, specials]).astype(np.float32)
    allf = allf[np.isfinite(allf) | np.isinf(allf)]
    got = orc.f32_to_bf16(allf)
    ref = torch.from_numpy(allf).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(got, ref)
    nan_bits = orc.f32_to_bf16(np.array([np.nan], dtype=np.float32))
    assert np.isnan(_bf16_value(nan_bits))[0]


def pin_bf16_widening_vs_torch(orc):
    """Every one of the 65,536 bf16 bit patterns widens to the fp32 value
    torch's bf16 -> fp32 conversion gives, bit for bit (NaNs by class: any
    NaN for a NaN). The listing's quantiser takes the activations in their
    input dtype, so this widening is where every bf16 token enters the path."""
    import torch
    bits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    got = orc.bf16_to_f32(bits)
    ref = torch.from_numpy(bits.view(np.int16).copy()).view(torch.bfloat16).float().numpy()
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    np.testing.assert_array_equal(got[~nan].view(np.uint32), ref[~nan].view(np.uint32))
    # a few values by hand: 1.0, -2.0, the smallest subnormal, -0, +inf
    hand = np.array([0x3F80, 0xC000, 0x0001, 0x8000, 0x7F80], dtype=np.uint16)
    want = np.array([1.0, -2.0, 2.0 ** -133, -0.0, np.inf], dtype=np.float32)
    np.testing.assert_array_equal(orc.bf16_to_f32(hand).view(np.uint32), want.view(np.uint32))


def pin_rescale_bound(orc):
    r = np.random.Generator(np.random.PCG64(61))
    acc = r.integers(-3_000_000, 3_000_000, size=(5, 70)).astype(np.int32)
    beta = np.abs(r.standard_normal(5)).astype(np.float32) * 40 + np.float32(0.1)
    gamma = np.float32(0.0159)
    y = _bf16_value(orc.rescale_bf16(acc, beta, gamma)).astype(np.float64)
    exact = acc.astype(np.float64) * beta.astype(np.float64)[:, None] * float(gamma) / 127.0
    rel = np.abs(y - exact) / np.maximum(np.abs(exact), 1e-30)
    assert np.all(rel <= 2.0 ** -8 + 1e-6), float(rel.max())
    assert np.all(np.sign(y) == np.sign(exact))


def pin_listing_semantics_torch(orc):
    """The page's PyTorch listing, restated with torch CPU primitives
    (mean/abs/clamp/round/linear) on fp32 tensors, gives the same integer
    stages and the same bf16 output as the oracle on small random cases."""
    import torch
    r = np.random.Generator(np.random.PCG64(71))
    for (M, K, N) in ((4, 256, 256), (3, 96, 40)):
        W = (r.standard_normal((N, K)) * 0.02).astype(np.float32)
        x = r.standard_normal((M, K)).astype(np.float32)
        res = orc.forward(x, W)
        Wt = torch.from_numpy(W)
        g = Wt.abs().mean().clamp(min=1e-5)
        assert abs(float(g) - float(res["gamma"])) <= 2 * np.spacing(res["gamma"])
        g = torch.tensor(float(res["gamma"]), dtype=torch.float32)
        wq = (Wt / g).round().clamp(-1.0, 1.0)
        xt = torch.from_numpy(x)
        b = xt.abs().amax(dim=-1, keepdim=True).clamp(min=1e-5)
        xq = (xt * (127.0 / b)).round().clamp(-128.0, 127.0)
        acc = torch.nn.functional.linear(xq.double(), wq.double())
        y = (acc.float() * ((b * g) / 127.0)).to(torch.bfloat16)
        np.testing.assert_array_equal(res["Wq"], wq.numpy().astype(np.int8))
        np.testing.assert_array_equal(res["xq"], xq.numpy().astype(np.int8))
        np.testing.assert_array_equal(res["beta"], b.numpy()[:, 0])
        np.testing.assert_array_equal(res["acc"], acc.numpy().astype(np.int32))
        np.testing.assert_array_equal(
            res["y"], y.view(torch.int16).numpy().view(np.uint16))


# ------------------------------------------------------------------- RMSNorm
#
# The listing's BitLinear normalises each token with nn.RMSNorm(in_features)
# before quantising it: out = x / sqrt(mean(x^2) + eps) * g.

def _rms_rows(r):
    """Four token rows of 384 channels at very different scales (the second
    so small that eps moves the result), with a few large channels."""
    x = r.standard_normal((4, 384))
    x[:, ::97] *= 50.0
    x *= np.array([1.0, 1e-4, 3e-2, 7.0])[:, None]
    return x.astype(np.float32)


def pin_rmsnorm_vs_torch_f64(orc):
    """torch.nn.functional.rms_norm in float64 on the same fp32 inputs is
    within the fp32 error bound of the oracle: six correctly rounded steps
    (mean, + eps, sqrt, divide, * r, * g), so 8 units of 2^-24 relative."""
    import torch
    r = np.random.Generator(np.random.PCG64(81))
    x = _rms_rows(r)
    g = r.uniform(0.5, 1.5, size=384).astype(np.float32)
    for eps in (2.0 ** -23, 1e-6):
        got = orc.rmsnorm(x, g, eps).astype(np.float64)
        ref = torch.nn.functional.rms_norm(
            torch.from_numpy(x.astype(np.float64)), (384,),
            weight=torch.from_numpy(g.astype(np.float64)), eps=float(np.float32(eps))).numpy()
        rel = np.abs(got - ref) / np.maximum(np.abs(ref), 1e-30)
        assert np.all(rel <= 8 * 2.0 ** -24), float(rel.max())


def pin_rmsnorm_constant_rows(orc):
    """A constant row c normalises to c / sqrt(c^2 + eps) (closed form in
    float64; 1 for |c| >> sqrt(eps), about 0.28 at c = 1e-4 where eps is
    comparable to c^2), and a zero row stays exactly zero."""
    eps = 2.0 ** -23
    cs = np.array([1.0, -3.0, 1e-3, 1e-4, 0.0], dtype=np.float32)
    x = np.repeat(cs[:, None], 256, axis=1)
    got = orc.rmsnorm(x, None, eps).astype(np.float64)
    c = cs.astype(np.float64)
    ref = c / np.sqrt(c * c + np.float64(np.float32(eps)))
    for i in range(len(cs)):
        assert np.all(got[i] == got[i, 0])
        assert abs(got[i, 0] - ref[i]) <= 4 * 2.0 ** -24 * abs(ref[i]), (cs[i], got[i, 0], ref[i])
    assert np.all(got[-1] == 0.0)
    assert abs(got[3, 0] - 0.278) < 1e-3


def pin_rmsnorm_pow2_invariance(orc):
    """With eps = 0 the normalisation is exactly invariant under scaling a
    row by a power of two: every step scales exactly or cancels."""
    r = np.random.Generator(np.random.PCG64(82))
    x = r.standard_normal((3, 256)).astype(np.float32)
    g = r.uniform(0.5, 1.5, size=256).astype(np.float32)
    base = orc.rmsnorm(x, g, 0.0)
    for j in (-20, -3, 5, 30):
        np.testing.assert_array_equal(orc.rmsnorm(x * np.float32(2.0 ** j), g, 0.0), base)


def pin_rmsnorm_gain_applied_last(orc):
    """The gain multiplies the normalised value, channel by channel:
    out(x, g)[m, k] is the fp32 product of out(x, 1)[m, k] and g[k]."""
    r = np.random.Generator(np.random.PCG64(83))
    x = _rms_rows(r)
    g = r.uniform(0.25, 4.0, size=384).astype(np.float32)
    unit = orc.rmsnorm(x, None, 2.0 ** -23)
    np.testing.assert_array_equal(orc.rmsnorm(x, g, 2.0 ** -23), unit * g[None, :])


# ---------------------------------------------------------------- FFN chain
#
# ReLU^2 replaces SwiGLU in the feed-forward block (winbuzzer.com release
# article, "Under the Hood"): h = max(gate, 0)^2 * up on the BitLinear outputs.

def _bf16_round(x):
    import torch
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(
        torch.bfloat16).float().numpy()


def pin_relu2_glu_exact_on_bf16(orc):
    """On bf16 operands every product has at most 24 significant bits, so
    the fp32 result equals the exact product (computed in float64)."""
    r = np.random.Generator(np.random.PCG64(91))
    scale = 10.0 ** r.uniform(-6, 4, size=4096)
    g = _bf16_round(r.standard_normal(4096) * scale)
    u = _bf16_round(r.standard_normal(4096) * scale[::-1])
    h = orc.relu2_glu(g, u).astype(np.float64)
    exact = np.maximum(g.astype(np.float64), 0.0) ** 2 * u.astype(np.float64)
    assert np.all(h == exact)
    assert np.count_nonzero(h) > 1500          # about half the gates are positive


def pin_relu2_glu_closed_forms(orc):
    g = np.array([2.0, -1.0, 0.0, 0.5, 1.0, 3.0, -1e-3], dtype=np.float32)
    u = np.array([-3.0, 5.0, 7.0, 2.0, -0.75, 1.0, 4.0], dtype=np.float32)
    h = orc.relu2_glu(g, u)
    np.testing.assert_array_equal(h, np.array([-12.0, 0.0, 0.0, 0.5, -0.75, 9.0, 0.0],
                                              dtype=np.float32))


def pin_ffn_gate_and_up_roles(orc):
    """With every gate output negative the block's output is exactly zero
    (h = 0, so the down projection quantises a zero token); swapping the
    gate and up weights then gives a non-zero output."""
    K, F, N = 256, 64, 48
    x = np.ones((2, K), dtype=np.float32)
    neg = np.full((F, K), -0.02, dtype=np.float32)       # ternarises to all -1
    pos = np.full((F, K), 0.02, dtype=np.float32)        # all +1
    Wd = (np.random.Generator(np.random.PCG64(92)).standard_normal((N, F)) * 0.02).astype(
        np.float32)
    off = orc.ffn(x, neg, pos, Wd)
    assert np.all(off["h"] == 0.0) and np.all(off["down"]["y"] == 0)
    on = orc.ffn(x, pos, neg, Wd)
    assert np.all(on["h"] < 0.0) and np.count_nonzero(on["down"]["y"]) > N


ALL_PINS = [
    pin_hand_example,
    pin_weight_ties_even,
    pin_activation_ties_even,
    pin_pack_words,
    pin_pack_roundtrip,
    pin_pack_b3_bytes,
    pin_pack_b3_roundtrip,
    pin_constant_token,
    pin_zero_inputs,
    pin_tiny_scale_epsilon,
    pin_identity_weights,
    pin_plus_minus_a,
    pin_gamma_vs_numpy_mean,
    pin_zero_fraction,
    pin_bruteforce_add_subtract,
    pin_exhaustive_single_term,
    pin_matmul_vs_linear,
    pin_quant_act_invariants,
    pin_quant_act_pow2_invariance,
    pin_bf16_rounding_vs_torch,
    pin_bf16_widening_vs_torch,
    pin_rescale_bound,
    pin_listing_semantics_torch,
    pin_rmsnorm_vs_torch_f64,
    pin_rmsnorm_constant_rows,
    pin_rmsnorm_pow2_invariance,
    pin_rmsnorm_gain_applied_last,
    pin_relu2_glu_exact_on_bf16,
    pin_relu2_glu_closed_forms,
    pin_ffn_gate_and_up_roles,
]


def failing_pins(orc) -> list:
    """Names of the pins the given oracle fails (an exception counts)."""
    failed = []
    for pin in ALL_PINS:
        try:
            pin(orc)
        except Exception:  # noqa: BLE001 - any failure is a caught mistake
            failed.append(pin.__name__)
    return failed
