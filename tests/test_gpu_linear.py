"""CompressedLinear on the GPU (README_zh, section 使用 Compressed Linear; section 预量化模型 for FP8 codes).

- The weight a layer decodes for its GEMM equals the oracle's decode of the layer's blob, bit for bit, in both
  format versions and in FP8 e4m3.
- layer(x) matches x @ W^T + b computed in float32 from the oracle-decoded weight. The GEMM runs in BF16 (or
  FP8 with BF16 output) with float32 accumulation in cuBLAS, so the bound is on BF16 output rounding and the
  library's reduction order: |y - ref| <= 2^-6 max |ref| (a wrong weight is off by O(max |ref|)).
- A state_dict round trip, and a chain of layers whose decodes are prefetched on a second stream, give the
  same outputs bit for bit as a lone layer decoding in its own forward.
"""
import numpy as np
import pytest
import torch

import synth

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA GPU", allow_module_level=True)

import decode_ep_b200 as ep  # noqa: E402

TOL = 2.0 ** -6


def make_linear(out_f, in_f, seed, dtype=torch.bfloat16):
    lin = torch.nn.Linear(in_f, out_f, bias=True, dtype=dtype)
    with torch.no_grad():
        lin.weight.copy_(synth.dit_layer(seed, shape=(out_f, in_f)).to(dtype))
        lin.bias.copy_(torch.linspace(-0.05, 0.05, out_f).to(dtype))
    return lin.cuda()


def oracle_weight(orc, layer):
    """The oracle's decode of the layer's blob, as float32 (scaled by s_w for FP8 codes)."""
    out = orc.decompress(bytes(layer.blob.cpu().numpy().tobytes()))
    if layer.weight_dtype == torch.bfloat16:
        w = torch.from_numpy(out.view(np.int16)).view(torch.bfloat16).float()
    elif layer.weight_dtype == torch.float16:
        w = torch.from_numpy(out.view(np.int16)).view(torch.float16).float()
    elif layer.weight_dtype == torch.float8_e4m3fn:
        w = torch.from_numpy(out.view(np.uint8)).view(torch.float8_e4m3fn).float() * float(layer.weight_scale)
    else:
        w = torch.from_numpy(out.copy())
    return w, out


def bits(t):
    t = t.cpu()
    if t.dtype in (torch.bfloat16, torch.float16):
        return t.view(torch.int16).numpy().view(np.uint16)
    if t.dtype == torch.float8_e4m3fn:
        return t.view(torch.uint8).numpy()
    return t.numpy()


@pytest.mark.parametrize("version", [2, 1])
def test_bf16_layer_weight_bit_exact_and_output(orc, version):
    lin = make_linear(384, 512, seed=11)
    layer = ep.CompressedLinear.from_linear(lin, ep.EntroPackLossyConfig(4.0, format_version=version))
    assert layer.blob.is_cuda and layer.compressed_bits <= 4.05 * 384 * 512
    w_ref, raw = oracle_weight(orc, layer)
    assert np.array_equal(bits(layer.decode_weight()), raw)
    x = torch.randn(64, 512, generator=torch.Generator().manual_seed(1)).to(torch.bfloat16).cuda()
    y = layer(x)
    assert y.dtype == torch.bfloat16 and y.shape == (64, 384)
    ref = x.float().cpu() @ w_ref.T + lin.bias.float().cpu()
    assert float((y.float().cpu() - ref).abs().max()) <= TOL * float(ref.abs().max())
    assert ep.device_status() == 0


def test_state_dict_round_trip_and_prefetch_chain(orc):
    lins = [make_linear(256, 256, seed=20 + i) for i in range(4)]
    layers = [ep.CompressedLinear.from_linear(l, 3.5) for l in lins]
    x = torch.randn(32, 256, generator=torch.Generator().manual_seed(2)).to(torch.bfloat16).cuda()

    def run(ls):
        h = x
        for l in ls:
            h = l(h)
        return h

    plain = run(layers)
    # the same layers rebuilt from their state_dicts
    again = [ep.CompressedLinear.from_state_dict(l.state_dict()) for l in layers]
    assert torch.equal(run(again).view(torch.int16), plain.view(torch.int16))
    # decodes prefetched on the workspace's decode stream, into the other buffer, while each GEMM runs
    ep.link_prefetch(layers)
    for _ in range(3):
        assert torch.equal(run(layers).view(torch.int16), plain.view(torch.int16))
    ep.link_prefetch([])
    for l in layers:
        l.next_layer = None
    # and the decoded weights themselves are the oracle's
    for l in layers:
        assert np.array_equal(bits(l.decode_weight()), oracle_weight(orc, l)[1])
    assert ep.device_status() == 0


def test_fp8_layer_codes_bit_exact_and_output(orc):
    lin = make_linear(512, 1024, seed=30)
    layer = ep.CompressedLinear.from_linear(lin, 5.0, container="fp8")
    assert layer.weight_dtype == torch.float8_e4m3fn
    assert layer.compressed_bits <= 5.05 * 512 * 1024
    w_ref, raw = oracle_weight(orc, layer)
    assert np.array_equal(bits(layer.decode_weight()), raw)
    x = torch.randn(128, 1024, generator=torch.Generator().manual_seed(3)).to(torch.bfloat16).cuda()
    y = layer(x)
    assert y.dtype == torch.bfloat16 and y.shape == (128, 512)
    # the reference uses the same e4m3 activations the layer feeds the FP8 GEMM
    x8, sx = layer.quantize_input(x)
    assert float((x8.float() * sx - x.float()).abs().max()) <= 2.0 ** -3 * float(x.float().abs().max())
    ref = (x8.float() * sx).cpu() @ w_ref.T + lin.bias.float().cpu()
    assert float((y.float().cpu() - ref).abs().max()) <= TOL * float(ref.abs().max())
    # and FP8 codes decode to weights close to the original (5 bpp of 8-bit codes)
    rel = float((w_ref - lin.weight.float().cpu()).norm() / lin.weight.float().cpu().norm())
    assert rel < 0.08
    assert ep.device_status() == 0
