"""Host-side checks of the nn.Module front end (no GPU): buffers, serialisation of the
quantised state, argument checks, and the layer-replacement walk."""
import io

import pytest
import torch

from bit_matmul_decomposition_b200 import linear as L


def test_buffers_and_shapes():
    m = L.Linear8bitLt(64, 48, bias=True, threshold=6.0)
    sd = m.state_dict()
    assert set(sd) == {"CB", "SCB", "bias"}
    assert sd["CB"].dtype == torch.int8 and tuple(sd["CB"].shape) == (48, 64)
    assert sd["SCB"].dtype == torch.float32 and tuple(sd["SCB"].shape) == (48,)
    assert sd["bias"].dtype == torch.float16 and tuple(sd["bias"].shape) == (48,)
    assert set(L.Linear8bitLt(64, 48, bias=False).state_dict()) == {"CB", "SCB"}


def test_in_features_must_be_a_multiple_of_16():
    with pytest.raises(ValueError):
        L.Linear8bitLt(40, 8)


def test_state_dict_round_trip():
    """CB / SCB serialisation: the quantised state saves and restores exactly."""
    g = torch.Generator().manual_seed(3)
    m = L.Linear8bitLt(32, 16)
    m.CB.copy_(torch.randint(-127, 128, (16, 32), generator=g, dtype=torch.int8))
    m.SCB.copy_(torch.rand(16, generator=g) + 0.25)
    m.bias.copy_(torch.randn(16, generator=g).half())
    buf = io.BytesIO()
    torch.save(m.state_dict(), buf)
    buf.seek(0)
    m2 = L.Linear8bitLt(32, 16)
    m2.load_state_dict(torch.load(buf))
    assert torch.equal(m2.CB, m.CB) and torch.equal(m2.SCB, m.SCB) and torch.equal(m2.bias, m.bias)
    # the dequantised weight comes from the library's kernel: not on a CPU module
    with pytest.raises(ValueError):
        m.dequantized_weight()


def test_forward_rejects_other_dtypes_before_any_call():
    m = L.Linear8bitLt(32, 8)
    with pytest.raises(TypeError):
        m(torch.zeros(2, 32))
    with pytest.raises(ValueError):
        m(torch.zeros(2, 16, dtype=torch.float16))


def test_replace_walk(monkeypatch):
    made = []

    def fake_from_linear(linear, threshold=6.0, has_fp16_weights=False, outlier_cache_cols=0,
                         code_format="int8"):
        made.append((linear.in_features, linear.out_features, threshold, outlier_cache_cols))
        return torch.nn.Identity()

    monkeypatch.setattr(L.Linear8bitLt, "from_linear", staticmethod(fake_from_linear))
    model = torch.nn.Sequential(torch.nn.Linear(32, 64), torch.nn.GELU(),
                                torch.nn.Sequential(torch.nn.Linear(64, 32)))
    model.lm_head = torch.nn.Linear(32, 10)
    L.replace_linear_with_int8(model, threshold=5.0, outlier_cache_cols=64)
    assert made == [(32, 64, 5.0, 64), (64, 32, 5.0, 64)]
    assert isinstance(model[0], torch.nn.Identity) and isinstance(model[2][0], torch.nn.Identity)
    assert isinstance(model.lm_head, torch.nn.Linear)


def test_training_mode_holds_fp16_parameters():
    m = L.Linear8bitLt(64, 32, bias=True, has_fp16_weights=True)
    assert {n for n, _ in m.named_parameters()} == {"weight", "bias"}
    assert m.weight.dtype == torch.float16 and m.weight.requires_grad
    assert {n for n, _ in m.named_buffers()} == {"CB", "SCB"}
    assert set(m.state_dict()) == {"weight", "bias", "CB", "SCB"}
    assert {n for n, _ in L.Linear8bitLt(64, 32).named_parameters()} == set()


def test_outlier_cache_option():
    m = L.Linear8bitLt(64, 32, outlier_cache_cols=128)
    assert "outlier_cache_cols=128" in repr(m)
    assert set(m.state_dict()) == {"CB", "SCB", "bias"}    # the cache is not saved
    m.load_state_dict(m.state_dict())                      # no cache allocated yet: no-op
    with pytest.raises(ValueError):
        L.Linear8bitLt(64, 32, outlier_cache_cols=-1)
    with pytest.raises(ValueError):
        L.Linear8bitLt(64, 32, outlier_cache_cols=64, has_fp16_weights=True)


def test_e4m3_code_format_option():
    m = L.Linear8bitLt(64, 32, code_format="e4m3")
    assert m.CB.dtype == torch.uint8 and "code_format=e4m3" in repr(m)
    with pytest.raises(ValueError):
        L.Linear8bitLt(64, 32, code_format="int4")
    with pytest.raises(ValueError):
        L.Linear8bitLt(64, 32, code_format="e4m3", outlier_cache_cols=64)
