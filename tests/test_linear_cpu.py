"""CompressedLinear on the host (no GPU): construction from an nn.Linear with the host encoder, storage, and the
state_dict round trip of the blob (README_zh, section 使用 Compressed Linear: from_linear, compressed_bits)."""
import pytest
import torch

import synth


@pytest.fixture(scope="module")
def ep():
    import decode_ep_b200 as m
    m.lib()
    return m


def make_linear(out_f=96, in_f=256, seed=3):
    lin = torch.nn.Linear(in_f, out_f, bias=True, dtype=torch.bfloat16)
    with torch.no_grad():
        lin.weight.copy_(synth.dit_layer(seed, shape=(out_f, in_f)))
        lin.bias.copy_(torch.linspace(-0.1, 0.1, out_f))
    return lin


def test_from_linear_storage_and_state_dict(ep, orc):
    lin = make_linear()
    layer = ep.CompressedLinear.from_linear(lin, 4.0)
    assert (layer.out_features, layer.in_features) == (96, 256)
    assert layer.weight_dtype == torch.bfloat16
    assert layer.compressed_bits == 8 * layer.blob.numel()
    assert abs(layer.compressed_bits / (96 * 256) - layer.actual_bpp) < 1e-12
    # the blob is the host encoder's, and the oracle accepts it
    blob = bytes(layer.blob.numpy().tobytes())
    assert blob == ep.compress(lin.weight.detach(), 4.0).blob
    assert orc.blob_info(blob)["rows"] == 96
    sd = layer.state_dict()
    assert set(sd) == {"blob", "bias", "weight_scale"}
    again = ep.CompressedLinear.from_state_dict(sd)
    assert torch.equal(again.blob, layer.blob) and torch.equal(again.bias, layer.bias)
    # load_state_dict into a layer of another size takes the stored blob as it is
    other = ep.CompressedLinear.from_linear(make_linear(32, 64, seed=4), 3.0)
    other.load_state_dict(sd)
    assert (other.out_features, other.in_features) == (96, 256) and torch.equal(other.blob, layer.blob)


def test_from_linear_fp8_codes(ep, orc):
    lin = make_linear(64, 512, seed=5)
    layer = ep.CompressedLinear.from_linear(lin, 5.0, container="fp8")
    assert layer.weight_dtype == torch.float8_e4m3fn
    w = lin.weight.detach().float()
    assert float(layer.weight_scale) == pytest.approx(float(w.abs().max()) / 448.0)
    info = orc.blob_info(bytes(layer.blob.numpy().tobytes()))
    assert info["dtype"] == 4
    with pytest.raises(ep.EntroPackError):
        layer.decode_weight()  # the blob is still on the host
