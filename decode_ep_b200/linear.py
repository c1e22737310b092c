"""CompressedLinear: a linear layer whose weight is kept EntroPack-compressed and decoded right before its GEMM.

The EntroPack README (section 使用 Compressed Linear) turns an ``nn.Linear`` into a compressed layer with
``from_linear(linear, config)``, calls it as ``layer(x)`` and reads its storage from ``compressed_bits``; the
paper page's abstract places the method on compute-heavy work (diffusion denoising, Transformer prefill),
where the decode time is small beside the GEMM. This module builds that on the library's C ABI:

- the weight is stored as one EPK1 blob (a ``uint8`` buffer, so ``state_dict()`` holds the blob and the bias);
- ``forward`` decodes the blob with the fused sm_100a kernel into a weight buffer owned by the library (one
  pair per device, shared by every compressed layer on it), then runs the GEMM (cuBLAS through
  ``torch.nn.functional.linear``, or cuBLASLt FP8 through ``torch._scaled_mm`` for FP8 weights);
- ``link_prefetch(layers)`` chains layers that run one after the other: while layer k's GEMM runs, layer
  k+1's weight decodes on a second stream into the other buffer of the pair.

FP8 weights (README_zh, section 预量化模型: FP8 codes stored at 5 bpp, FP8 GEMM at inference): with
``container="fp8"`` the layer keeps e4m3 codes of W / s_w (one scale s_w per tensor, max |W| / 448), the
blob decodes straight into e4m3, and the activations are cast to e4m3 with their own per-call scale before
``torch._scaled_mm``.

Every decode runs in the CUDA kernel; nothing here computes on the host except argument marshalling and
the FP8 scale of the weights at compression time.
"""
from __future__ import annotations

import threading

import torch
import torch.nn.functional as F

from . import (EP_FP8_E4M3, HEADER_BYTES, CompressedTensor, EntroPackError, EntroPackLossyConfig, blob_info, compress,
               lib, _check, _EP_TO_TORCH)

__all__ = ["CompressedLinear", "DecodeWorkspace", "link_prefetch"]

E4M3_MAX = 448.0


class DecodeWorkspace:
    """The library-owned weight buffers of one CUDA device: two slots used in turn, and a decode stream.

    A slot is a flat byte buffer, grown to the largest weight decoded into it. A layer's GEMM reads the
    slot its weight was decoded into; an event recorded after that GEMM marks the slot free again, and the
    next decode into the slot waits for it on the GPU (never on the host). Each stream that writes or reads
    a slot is recorded on its buffer, so a buffer given up when its slot grows is not reused by the
    allocator before that work is done. The slots' bookkeeping is host state: the layers of one device run
    their forwards one at a time (one thread), as a model's layers do."""

    _lock = threading.Lock()
    _by_device: dict = {}

    def __init__(self, device: torch.device):
        self.device = device
        self.buffers = [torch.empty(0, dtype=torch.uint8, device=device) for _ in range(2)]
        self.stream = torch.cuda.Stream(device)
        self.free = [None, None]      # event: the last GEMM that read the slot is done
        self.ready = [None, None]     # event: the decode into the slot is done
        self.holder = [None, None]    # the layer whose weight the slot holds (or is being decoded into it)
        self.turn = 0                 # the slot the next layer without a prefetch takes

    @classmethod
    def get(cls, device) -> "DecodeWorkspace":
        device = torch.device(device)
        with cls._lock:
            ws = cls._by_device.get(device.index)
            if ws is None:
                ws = cls._by_device[device.index] = DecodeWorkspace(device)
            return ws

    def _view(self, slot: int, layer: "CompressedLinear") -> torch.Tensor:
        n = layer.out_features * layer.in_features * torch.empty((), dtype=layer.weight_dtype).element_size()
        if self.buffers[slot].numel() < n:
            self.buffers[slot] = torch.empty(n, dtype=torch.uint8, device=self.device)
        return self.buffers[slot][:n].view(layer.weight_dtype).view(layer.out_features, layer.in_features)

    def decode(self, layer: "CompressedLinear", slot: int, stream) -> torch.Tensor:
        """Decodes layer's weight into `slot` on `stream` (after the slot's last reader is done)."""
        w = self._view(slot, layer)
        if self.free[slot] is not None:
            stream.wait_event(self.free[slot])
        layer.decode_weight(out=w, stream=stream)
        if self.buffers[slot].numel():
            self.buffers[slot].record_stream(stream)
        ev = torch.cuda.Event()
        ev.record(stream)
        self.ready[slot] = ev
        self.holder[slot] = layer
        return w

    def acquire(self, layer: "CompressedLinear", stream) -> tuple[int, torch.Tensor]:
        """The slot holding layer's decoded weight, ready for `stream`: the prefetched one, or a decode now."""
        for slot in (0, 1):
            if self.holder[slot] is layer and self.ready[slot] is not None:
                stream.wait_event(self.ready[slot])
                self.turn = 1 - slot
                return slot, self._view(slot, layer)
        slot = self.turn
        w = self.decode(layer, slot, stream)
        self.turn = 1 - slot
        return slot, w

    def release(self, slot: int, stream) -> None:
        """Marks the slot free once the work queued so far on `stream` (the GEMM) is done."""
        if self.buffers[slot].numel():
            self.buffers[slot].record_stream(stream)
        ev = torch.cuda.Event()
        ev.record(stream)
        self.free[slot] = ev

    def prefetch(self, layer: "CompressedLinear", busy_slot: int, stream) -> None:
        """Starts layer's decode on the decode stream into the slot other than `busy_slot`."""
        slot = 1 - busy_slot
        if self.holder[slot] is layer and self.ready[slot] is not None:
            return
        self.stream.wait_stream(stream)  # the blob and the previous contents are ordered before the decode
        self.decode(layer, slot, self.stream)


class CompressedLinear(torch.nn.Module):
    """y = x W^T + b with W stored as an EntroPack blob (README_zh, section 使用 Compressed Linear).

    The blob lives in the ``blob`` buffer (uint8), so ``state_dict()`` / ``load_state_dict()`` carry it with
    the bias; moving the module to a CUDA device moves the blob, which the decode reads in place. The decoded
    weight has the blob's container dtype (BF16, FP16, FP32 or FP8 e4m3); for e4m3, ``weight_scale`` holds
    the tensor scale s_w with W ~= s_w * codes."""

    def __init__(self, compressed: CompressedTensor, bias: torch.Tensor | None = None,
                 weight_scale: float | None = None):
        super().__init__()
        self.out_features, self.in_features = compressed.shape
        self.register_buffer("blob", torch.frombuffer(bytearray(compressed.blob), dtype=torch.uint8))
        self.bias = None if bias is None else torch.nn.Parameter(bias.detach().clone(), requires_grad=False)
        fp8 = compressed.dtype == torch.float8_e4m3fn
        if fp8 and weight_scale is None:
            raise EntroPackError(-1, "CompressedLinear: FP8 e4m3 weights need their weight_scale")
        self.register_buffer("weight_scale", torch.tensor(float(weight_scale if fp8 else 1.0), dtype=torch.float32))
        self.weight_dtype = compressed.dtype
        self.actual_bpp = compressed.actual_bpp
        self._header = compressed.blob[:HEADER_BYTES]
        self.next_layer = None  # set by link_prefetch; not a submodule

    # ------------------------------------------------------------------ construction

    @classmethod
    def from_linear(cls, linear: torch.nn.Linear, config: EntroPackLossyConfig | float,
                    container: str | None = None) -> "CompressedLinear":
        """Compresses ``linear.weight`` at ``config.target_bpp`` (README_zh, section 使用 Compressed Linear).

        container: None keeps the weight's own dtype (BF16, FP16 or FP32); "fp8" first turns the weight into
        FP8 e4m3 codes of W / s_w with s_w = max |W| / 448 (one scale per tensor), then compresses the codes
        (README_zh, section 预量化模型: FP8 codes at 5 bpp, FP8 GEMM)."""
        if not isinstance(config, EntroPackLossyConfig):
            config = EntroPackLossyConfig(float(config))
        w = linear.weight.detach()
        scale = None
        if container == "fp8":
            wf = w.float()
            amax = float(wf.abs().max())
            scale = amax / E4M3_MAX if amax > 0 else 1.0
            w = (wf / scale).clamp(-E4M3_MAX, E4M3_MAX).to(torch.float8_e4m3fn)
        elif container is not None:
            raise EntroPackError(-2, f"CompressedLinear.from_linear: unknown container {container!r}")
        if config.encoder == "cuda" and not w.is_cuda:
            w = w.cuda()
        layer = cls(compress(w, config), None if linear.bias is None else linear.bias.detach(), scale)
        return layer.to(linear.weight.device)

    @classmethod
    def from_state_dict(cls, state_dict: dict, prefix: str = "") -> "CompressedLinear":
        """A layer rebuilt from a state_dict that CompressedLinear.state_dict() wrote (on the blob's device)."""
        blob = state_dict[prefix + "blob"]
        info = blob_info(bytes(blob.cpu().numpy().tobytes()))
        comp = CompressedTensor(bytes(blob.cpu().numpy().tobytes()), (info["rows"], info["cols"]),
                                _EP_TO_TORCH[info["dtype"]], info["actual_bpp"])
        bias = state_dict.get(prefix + "bias")
        scale = float(state_dict[prefix + "weight_scale"]) if prefix + "weight_scale" in state_dict else None
        return cls(comp, bias, scale if comp.dtype == torch.float8_e4m3fn else None).to(blob.device)

    @classmethod
    def from_fp8(cls, codes: torch.Tensor, weight_scale: float, bias: torch.Tensor | None,
                 config: EntroPackLossyConfig | float) -> "CompressedLinear":
        """A layer from existing FP8 e4m3 weight codes and their tensor scale (W ~= weight_scale * codes)."""
        if codes.dtype != torch.float8_e4m3fn:
            raise EntroPackError(-2, "CompressedLinear.from_fp8: codes must be float8_e4m3fn")
        return cls(compress(codes, config), bias, weight_scale).to(codes.device)

    # ------------------------------------------------------------------ storage

    @property
    def compressed_bits(self) -> int:
        """Storage of the weight in bits, metadata included (README_zh, section 使用 Compressed Linear)."""
        return 8 * int(self.blob.numel())

    def _load_from_state_dict(self, state_dict, prefix, local_metadata, strict, missing_keys, unexpected_keys,
                              error_msgs):
        key = prefix + "blob"
        if key in state_dict:  # blobs differ in size from layer to layer: take the stored one as it is
            blob = state_dict[key]
            info = blob_info(bytes(blob.cpu().numpy().tobytes()))
            self.blob = blob.detach().clone().to(self.blob.device)
            self.out_features, self.in_features = info["rows"], info["cols"]
            self.weight_dtype = _EP_TO_TORCH[info["dtype"]]
            self.actual_bpp = info["actual_bpp"]
            self._header = bytes(blob[:HEADER_BYTES].cpu().numpy().tobytes())
            b = state_dict.get(prefix + "bias")
            if b is not None and (self.bias is None or self.bias.shape != b.shape):
                self.bias = torch.nn.Parameter(torch.empty_like(b, device=self.blob.device), requires_grad=False)
        super()._load_from_state_dict(state_dict, prefix, local_metadata, strict, missing_keys, unexpected_keys,
                                      error_msgs)

    def extra_repr(self) -> str:
        return (f"in_features={self.in_features}, out_features={self.out_features}, bias={self.bias is not None}, "
                f"weight={self.weight_dtype}, {self.actual_bpp:.3f} bpp")

    # ------------------------------------------------------------------ decode and forward

    def decode_weight(self, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
        """The decoded weight (out_features, in_features) in the blob's container dtype, written into `out`
        (a contiguous CUDA tensor of that shape and dtype) or a new tensor, on `stream` (default: current)."""
        if not self.blob.is_cuda:
            raise EntroPackError(-1, "CompressedLinear: move the layer to a CUDA device first")
        if out is None:
            out = torch.empty(self.out_features, self.in_features, dtype=self.weight_dtype, device=self.blob.device)
        if (not out.is_cuda or not out.is_contiguous() or out.dtype != self.weight_dtype
                or tuple(out.shape) != (self.out_features, self.in_features)):
            raise EntroPackError(-9, "CompressedLinear.decode_weight: out must be a contiguous CUDA tensor of the "
                                     "weight's shape and dtype")
        s = torch.cuda.current_stream(out.device) if stream is None else stream
        _check(lib().ep_decompress_into(self._header, self.blob.data_ptr(), int(self.blob.numel()), out.data_ptr(),
                                        out.numel() * out.element_size(), s.cuda_stream), "CompressedLinear decode")
        return out

    def weight_float(self) -> torch.Tensor:
        """The weight the layer computes with, in float32 (for checks; the layer itself never builds it)."""
        w = self.decode_weight().float()
        return w * self.weight_scale if self.weight_dtype == torch.float8_e4m3fn else w

    def forward(self, x: torch.Tensor, x_scale: torch.Tensor | None = None) -> torch.Tensor:
        """y = x W^T + b. For an FP8 layer, x may also be e4m3 activations already cast, with their float32
        scale x_scale (x ~= x_scale * x8), as quantize_input returns them."""
        if not x.is_cuda:
            raise EntroPackError(-1, "CompressedLinear: the input must be a CUDA tensor")
        stream = torch.cuda.current_stream(x.device)
        ws = DecodeWorkspace.get(x.device)
        slot, w = ws.acquire(self, stream)
        if self.next_layer is not None:  # the next layer decodes while this GEMM runs
            ws.prefetch(self.next_layer, slot, stream)
        y = self.forward_with(x, w, x_scale)
        ws.release(slot, stream)
        return y

    def forward_with(self, x: torch.Tensor, w: torch.Tensor, x_scale: torch.Tensor | None = None) -> torch.Tensor:
        """The layer's GEMM with a given decoded weight w (the container dtype, out_features x in_features)."""
        if self.weight_dtype == torch.float8_e4m3fn:
            return self._fp8_gemm(x, w, x_scale)
        return F.linear(x.to(self.weight_dtype), w, None if self.bias is None else self.bias.to(self.weight_dtype))

    @staticmethod
    def quantize_input(x2: torch.Tensor) -> tuple[torch.Tensor, torch.Tensor]:
        """FP8 e4m3 activations for the FP8 GEMM: x8 = e4m3(x * (448 / max |x|)) with the multiply in x's own
        dtype, and the scale s_x = max |x| / 448 (float32), so that x ~= s_x * x8."""
        amax = torch.amax(torch.abs(x2)).float().clamp_min(1e-12)
        x8 = (x2 * (E4M3_MAX / amax).to(x2.dtype)).to(torch.float8_e4m3fn)
        return x8, (amax / E4M3_MAX).reshape(())

    def _fp8_gemm(self, x: torch.Tensor, w8: torch.Tensor, x_scale: torch.Tensor | None) -> torch.Tensor:
        lead = x.shape[:-1]
        x2 = x.reshape(-1, x.shape[-1])
        if x.dtype == torch.float8_e4m3fn:
            if x_scale is None:
                raise EntroPackError(-1, "CompressedLinear: e4m3 activations need their x_scale")
            x8, sx = x2, x_scale.float().reshape(())
        else:
            x8, sx = self.quantize_input(x2)
        y = torch._scaled_mm(x8, w8.t(), scale_a=sx, scale_b=self.weight_scale.reshape(()), out_dtype=torch.bfloat16)
        if self.bias is not None:
            y = y + self.bias.to(y.dtype)
        return y.reshape(*lead, self.out_features)


def link_prefetch(layers) -> None:
    """Chains layers that run one after the other: each layer's forward starts the next one's decode on the
    workspace's decode stream, into the other weight buffer, while its own GEMM runs."""
    layers = list(layers)
    for a, b in zip(layers, layers[1:]):
        object.__setattr__(a, "next_layer", b)
    if layers:
        object.__setattr__(layers[-1], "next_layer", None)
