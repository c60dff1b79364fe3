"""Host-side checks of the seeded input recipe (CPU only)."""
import torch

from weight_linear_attention_ttt_b200 import inputs as inp


def test_dual_recipe_shapes_dtypes_and_determinism():
    w = inp.WORKLOADS["dual_bf16_B8H12T2048_d64C16"]
    a = inp.make_inputs(w, "cpu", B=1, H=2, T=64)
    b = inp.make_inputs(w, "cpu", B=1, H=2, T=64)
    for k in ("Q", "K", "V"):
        assert a[k].shape == (1, 2, 64, 64) and a[k].dtype == torch.bfloat16
        assert torch.equal(a[k], b[k])
    assert a["eta"].shape == (1, 2, 64) and a["eta"].dtype == torch.float32
    assert torch.equal(a["eta"], b["eta"])
    # eta = sigmoid(z)/d lies in (0, 1/d)
    assert float(a["eta"].min()) > 0 and float(a["eta"].max()) < 1.0 / 64
    # K and V are normalised per token before rounding; Q is not
    kn = a["K"].float().norm(dim=-1)
    assert torch.allclose(kn, torch.ones_like(kn), atol=1e-2)
    assert float((a["Q"].float().norm(dim=-1) - 1).abs().max()) > 0.1
    assert a["W0"].dtype == torch.float32 and a["W0"].shape == (1, 2, 64, 64)
    assert 0.015 < float(a["W0"].std()) < 0.025


def test_fp32_tiny_recipe():
    w = inp.WORKLOADS["dual_f32_B1H2T256_d32C16"]
    a = inp.make_inputs(w, "cpu")
    assert a["Q"].dtype == torch.float32 and a["eta"] is None and a["eta_scalar"] == 0.1
    assert float(a["W0"].abs().max()) == 0.0
    assert 0.14 < float(a["Q"].std()) < 0.21  # N(0, 1/32)


def test_assoc_and_inplace_recipes():
    w = inp.WORKLOADS["assoc_bf16_B4H16T65536_d128C64"]
    a = inp.make_inputs(w, "cpu", B=1, H=1, T=128)
    assert a["eta"].shape == (1, 1, 128) and float(a["eta"].max()) < 1.0
    qn = a["Q"].float().norm(dim=-1)
    assert torch.allclose(qn, torch.ones_like(qn), atol=1e-2)
    assert float(a["W0"].abs().max()) == 0.0
    w = inp.WORKLOADS["inplace_bf16_T32768_Dff9728_D2560_C1024"]
    z = inp.make_inputs(w, "cpu", T=64, Dff=96, D=32)
    assert z["Z"].shape == (64, 96) and z["Vhat"].shape == (64, 32) and z["W0"].shape == (96, 32)
    assert z["Z"].dtype == torch.bfloat16 and z["eta"] == 1e-3


def test_seed_changes_values():
    w = inp.WORKLOADS["dual_bf16_B8H12T2048_d64C16"]
    a = inp.make_inputs(w, "cpu", B=1, H=1, T=16)
    b = inp.make_inputs(w, "cpu", B=1, H=1, T=16, seed=5)
    assert not torch.equal(a["Q"], b["Q"])
