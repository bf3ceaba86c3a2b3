"""The feed-forward chain (bitlinear_ffn_forward) against the CPU oracle's
Oracle.ffn: gate and up BitLinears of the same tokens, the gated squared
ReLU h = max(gate, 0)^2 * up in fp32, and the down BitLinear of h.

Without RMS normalisation every stage is compared bit for bit: the gate and
up outputs, h (fp32) and the down projection's output. With each
BitLinear's own RMSNorm (the listing's per-BitLinear nn.RMSNorm) the
device adds a token's squares in another order than the oracle, so a
normalised value sitting on a rounding tie may quantise to either
neighbour (the same bar as the other normalised forms): the gate, up and
down outputs are then held to the relative tolerance and must be
bit-identical almost everywhere, while h must equal the gated ReLU^2 of the
kernel's own gate and up outputs exactly, and y the oracle's down
projection of the kernel's own h within the tolerance.
"""

import numpy as np
import pytest

import oracle
import workloads
import ternary_weight_w1_b200 as bl
from tests.gpu_cases import Guarded, bf16_bits_to_tensor, check_y, tensor_to_bf16_bits

pytestmark = pytest.mark.gpu

CANARY_H = 0x7FC0A5A5          # an fp32 NaN: no finite h holds it
CANARY_Y = 0x7FA5


@pytest.fixture(scope="module", autouse=True)
def cuda():
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    bl.lib()
    return torch


class FfnCase:
    """Seeded gate (F x K), up (F x K) and down (K x F) latents, bf16 (or
    fp32) tokens [M][K], optional RMSNorm gains for each BitLinear, packed by
    the library's packer; the oracle runs the chain with the packer's
    gammas."""

    def __init__(self, M, K, F, seed, norm=False, x_dtype="bf16"):
        self.M, self.K, self.F = M, K, F
        self.orc = oracle.default()
        Wg = workloads.latent_weights(F, K, seed)
        Wu = workloads.latent_weights(F, K, seed + 1)
        Wd = workloads.latent_weights(K, F, seed + 2)
        xf = workloads.activations_f32(M, K, seed + 3)
        self.x_dtype = x_dtype
        if x_dtype == "bf16":
            self.x_in = workloads.to_bf16_bits(xf)
        else:
            self.x_in = np.ascontiguousarray(xf, dtype=np.float32)
        self.packed = [bl.bitlinear_pack_weights(W) for W in (Wg, Wu, Wd)]
        self.gains = ((workloads.norm_gains(K, seed + 4), workloads.norm_gains(K, seed + 5),
                       workloads.norm_gains(F, seed + 6)) if norm else (None, None, None))
        self.norm = norm
        self.Wd = Wd
        self.ref = self.orc.ffn(self.x_in, Wg, Wu, Wd,
                                gammas=tuple(np.float32(g) for _, g in self.packed),
                                gains=self.gains)

    def run(self):
        import torch
        dev = "cuda"
        x = (bf16_bits_to_tensor(self.x_in) if self.x_dtype == "bf16"
             else torch.from_numpy(self.x_in).to(dev))
        mats = [(torch.from_numpy(pk).to(dev), g) for pk, g in self.packed]
        gains = tuple(None if g is None else torch.from_numpy(g).to(dev) for g in self.gains)
        out = {"y": Guarded((self.M, self.K), torch.bfloat16, dev, CANARY_Y),
               "h": Guarded((self.M, self.F), torch.float32, dev, CANARY_H),
               "gate": Guarded((self.M, self.F), torch.bfloat16, dev, CANARY_Y),
               "up": Guarded((self.M, self.F), torch.bfloat16, dev, CANARY_Y)}
        bl.bitlinear_ffn_forward(x, mats[0], mats[1], mats[2], gains=gains, h=out["h"].t,
                                 y=out["y"].t, gate_y=out["gate"].t, up_y=out["up"].t)
        torch.cuda.synchronize()
        for name, g in out.items():
            g.check(name)
        return {"y": tensor_to_bf16_bits(out["y"].t), "h": out["h"].t.cpu().numpy(),
                "gate": tensor_to_bf16_bits(out["gate"].t),
                "up": tensor_to_bf16_bits(out["up"].t)}


# M <= 6 takes the fused GEMV launch; larger batches the tensor-core route
# (grouped gate/up GEMM, the h kernel, then the down projection)
PLAIN = [(1, 2560, 6912), (3, 2560, 6912), (6, 512, 1024), (12, 2560, 6912), (16, 384, 896),
         (2, 128, 128), (7, 1280, 2560), (40, 2560, 6912), (300, 512, 1024)]


@pytest.mark.parametrize("M,K,F", PLAIN)
def test_ffn_matches_oracle_bit_for_bit(M, K, F):
    c = FfnCase(M, K, F, seed=M * 7 + K + F)
    got = c.run()
    np.testing.assert_array_equal(got["gate"], c.ref["gate"]["y"])
    np.testing.assert_array_equal(got["up"], c.ref["up"]["y"])
    np.testing.assert_array_equal(got["h"].view(np.uint32), c.ref["h"].view(np.uint32))
    np.testing.assert_array_equal(got["y"], c.ref["down"]["y"])


def test_ffn_fp32_tokens():
    c = FfnCase(2, 512, 1024, seed=77, x_dtype="fp32")
    got = c.run()
    np.testing.assert_array_equal(got["h"].view(np.uint32), c.ref["h"].view(np.uint32))
    np.testing.assert_array_equal(got["y"], c.ref["down"]["y"])


@pytest.mark.parametrize("M,K,F", [(1, 2560, 6912), (5, 1024, 2048), (16, 2560, 6912),
                                   (24, 1024, 2048)])
def test_ffn_normalised_matches_oracle(M, K, F):
    c = FfnCase(M, K, F, seed=M * 11 + K + F, norm=True)
    got = c.run()
    for name in ("gate", "up"):
        exact = check_y(got[name], c.ref[name]["y"])
        assert exact >= 0.99, (name, exact)
    # h is the gated ReLU^2 of the kernel's own gate and up outputs, exactly
    h_ref = c.orc.relu2_glu(c.orc.bf16_to_f32(got["gate"]), c.orc.bf16_to_f32(got["up"]))
    np.testing.assert_array_equal(got["h"].view(np.uint32), h_ref.view(np.uint32))
    # the down projection of the kernel's own h
    down = c.orc.forward(got["h"], c.Wd, gamma=np.float32(c.packed[2][1]),
                         norm_gain=c.gains[2])
    exact = check_y(got["y"], down["y"])
    assert exact >= 0.99, exact


def test_ffn_2b_decode_step_with_zero_and_negative_gates():
    """An all-zero token (beta clamps to 1e-5, everything is zero) next to
    ordinary ones: h and y stay exact."""
    c = FfnCase(3, 2560, 6912, seed=5)
    c.x_in[1, :] = 0
    c.ref = c.orc.ffn(c.x_in, workloads.latent_weights(6912, 2560, 5),
                      workloads.latent_weights(6912, 2560, 6), c.Wd,
                      gammas=tuple(np.float32(g) for _, g in c.packed))
    got = c.run()
    assert np.all(got["h"][1] == 0)
    np.testing.assert_array_equal(got["h"].view(np.uint32), c.ref["h"].view(np.uint32))
    np.testing.assert_array_equal(got["y"], c.ref["down"]["y"])
    assert bl.bitlinear_get_fault() == (bl.BITLINEAR_OK, 0)
