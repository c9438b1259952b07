"""The seeded input generator shared by the kernels' tests and the oracle.

It holds no layer arithmetic, only storage encodings and random draws, so it
is pinned against library conversions and brute force: bf16 rounding against
torch's float32 -> bfloat16, the NVFP4 encoder against an exhaustive
nearest-code search and torch's e4m3, and the counter streams against
regeneration of any single tensor."""
import numpy as np
import pytest
import torch

from mixture_experts_layer_sqrt_b200 import synth

E2M1 = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


def test_bf16_rounding_matches_torch():
    g = np.random.default_rng(7)
    a = np.concatenate([g.standard_normal(100000).astype(np.float32) * 10.0 ** g.integers(-20, 20, 100000),
                        # exact halfway cases between bf16 neighbours, both parities
                        np.array([1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, -(1.0 + 2.0 ** -8), 0.0, -0.0],
                                 dtype=np.float32)]).astype(np.float32)
    ours = synth.f32_to_bf16_bits(a)
    ref = torch.from_numpy(a).to(torch.bfloat16).view(torch.uint16).numpy()
    np.testing.assert_array_equal(ours, ref)


def _nearest_code(v: float) -> int:
    """Brute force: the e2m1 magnitude nearest to |v| (ties to the even code), saturating at 6."""
    a = abs(v)
    best = min(range(8), key=lambda c: (abs(E2M1[c] - a), c & 1))
    return (8 if (v < 0 and best != 0) else 0) | best


def test_nvfp4_encoder_is_the_nearest_code_of_each_scaled_weight():
    g = np.random.default_rng(11)
    w = (g.standard_normal((6, 64)) * 0.05).astype(np.float32)
    w[0, :16] = 0.0                                  # an all-zero block: scale 0, codes 0
    w[1, 16:32] *= 1e-6                              # tiny block: e4m3 subnormal scale
    packed, scales = synth.quantize_nvfp4(w)
    assert packed.shape == (6, 32) and scales.shape == (6, 4)
    sval = torch.from_numpy(scales).view(torch.float8_e4m3fn).float().numpy()
    blocks = w.reshape(6, 4, 16)
    amax = np.abs(blocks).max(axis=-1)
    ref_scale = torch.from_numpy((amax / np.float32(6.0)).astype(np.float32)).to(torch.float8_e4m3fn)
    np.testing.assert_array_equal(scales, ref_scale.view(torch.uint8).numpy())
    codes = np.stack([packed & 0xF, packed >> 4], axis=-1).reshape(6, 64)
    for r in range(6):
        for c in range(64):
            s = sval[r, c // 16]
            want = _nearest_code(float(np.float32(w[r, c]) / np.float32(s))) if s > 0 else 0
            assert codes[r, c] == want, (r, c)


def test_counter_streams_regenerate_any_tensor_alone():
    p = synth.PROBLEMS["tiny_f32"]
    a = synth.generate(p)
    b = synth.generate(p)
    for k, v in a.items():
        if v is None:
            assert b[k] is None
        else:
            np.testing.assert_array_equal(v, b[k])
    only_x = synth.generate(p, experts=False)
    np.testing.assert_array_equal(only_x["x"], a["x"])
    other = synth.generate(p.with_(seed=p.seed + 1))
    assert not np.array_equal(other["x"], a["x"])
    np.testing.assert_array_equal(synth.gen_expert_weights(p, "w_up", 3), a["w_up"][3])


@pytest.mark.parametrize("name", ["tiny_f32", "sqrt_fp4"])
def test_storage_shapes_and_types(name):
    p = synth.PROBLEMS[name]
    if name == "sqrt_fp4":
        p = p.with_(T=32, D=256, F=128, E=4, k=2, Fs=64)
    a = synth.generate(p)
    assert a["x"].shape == (p.T, p.D) and a["w_router"].shape == (p.E, p.D)
    if p.wdtype == "nvfp4":
        assert a["w_gate"].shape == (p.E, p.F, p.D // 2) and a["w_gate"].dtype == np.uint8
        assert a["w_gate_scale"].shape == (p.E, p.F, p.D // 16)
        assert a["w_down"].shape == (p.E, p.D, p.F // 2)
        assert a["sh_gate"].shape == (p.Fs, p.D) and a["x"].dtype == np.uint16
        assert a["image_mask"].shape == (p.T,) and a["bias"].shape == (p.E,)
    else:
        assert a["w_gate"].shape == (p.E, p.F, p.D) and a["w_gate"].dtype == np.float32
        assert a["sh_gate"] is None
