"""decode_ep_b200: EntroPack lossy weight compression with a fused sm_100a decode.

This is a thin ctypes binding over ``libentropack.so`` (C ABI in ``include/entropack.h``). Every
step of compression and decode runs in that library: the host encoder on the CPU, the decode in
the CUDA kernel. This module only moves arguments. PyTorch provides device memory and streams.
There is no CPU fallback. If the library is missing or cannot load, the import fails loudly.

API, after the EntroPack README (quick-start and Config sections):

    cfg = EntroPackLossyConfig(target_bpp=3.5)
    c = compress(tensor, cfg)                  # CompressedTensor; c.actual_bpp counts metadata
    w = decompress(c)                          # CUDA tensor, same shape and dtype
    decompress_into(c, out, stream=None)       # hot path: preallocated output, async on a stream
    layer = CompressedLinear.from_linear(linear, cfg)   # README, section 使用 Compressed Linear
"""
from __future__ import annotations

import ctypes
import math
import os
import threading
from dataclasses import dataclass, field

import torch

from . import build as _build

__all__ = ["EntroPackLossyConfig", "TileANSConfig", "CompressedTensor", "EntroPackError", "LayerBatch", "compress", "decompress",
           "decompress_into", "decompress_many", "decode_coords", "device_status", "blob_info", "plan_bitrates", "lib",
           "CompressedLinear", "DecodeWorkspace", "link_prefetch"]

EP_BF16, EP_FP16, EP_FP32, EP_FP8_E4M3, EP_INT8 = 1, 2, 3, 4, 5
_TORCH_TO_EP = {torch.bfloat16: EP_BF16, torch.float16: EP_FP16, torch.float32: EP_FP32,
                torch.float8_e4m3fn: EP_FP8_E4M3, torch.int8: EP_INT8}
_EP_TO_TORCH = {v: k for k, v in _TORCH_TO_EP.items()}
HEADER_BYTES = 64
TANS_HEADER_BYTES = 96  # lossless tile-ANS (EPL1) blobs


class EntroPackError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(message)
        self.status = status


class _Options(ctypes.Structure):
    _fields_ = [("rounds_per_tile", ctypes.c_uint32), ("sample_coords", ctypes.c_uint32),
                ("bisection_iters", ctypes.c_uint32), ("threads", ctypes.c_int32),
                ("format_version", ctypes.c_uint32)]


_lib = None
_lib_lock = threading.Lock()


def lib() -> ctypes.CDLL:
    """The loaded libentropack.so. The library is built in-tree if it is missing or out of date. Threads that
    ask for it at once wait for one build and load."""
    if _lib is None:
        with _lib_lock:
            if _lib is None:
                _load()
    return _lib


def _load() -> None:
    global _lib
    path = _build.LIB
    if not os.path.exists(path) or _build.stale():
        path = _build.build()
    L = ctypes.CDLL(path)
    c = ctypes
    L.ep_options_default.argtypes = [c.POINTER(_Options)]
    L.ep_compress.argtypes = [c.c_void_p, c.c_int, c.c_int, c.c_int64, c.c_int64, c.c_int64, c.c_double,
                              c.POINTER(_Options), c.POINTER(c.c_void_p), c.POINTER(c.c_size_t),
                              c.POINTER(c.c_double)]
    L.ep_compress_cuda.argtypes = [c.c_void_p, c.c_int, c.c_int64, c.c_int64, c.c_int64, c.c_double,
                                   c.POINTER(_Options), c.c_void_p, c.POINTER(c.c_void_p), c.POINTER(c.c_size_t),
                                   c.POINTER(c.c_double)]
    L.ep_compress_cuda_noalloc.argtypes = [c.c_void_p, c.c_int, c.c_int64, c.c_int64, c.c_int64, c.c_double,
                                           c.POINTER(_Options), c.c_void_p, c.c_void_p, c.c_size_t,
                                           c.POINTER(c.c_size_t), c.POINTER(c.c_double)]
    L.ep_compress_cuda_noalloc.restype = c.c_int
    L.ep_blob_free.argtypes = [c.c_void_p]
    L.ep_blob_info.argtypes = [c.c_void_p, c.c_size_t, c.POINTER(c.c_int), c.POINTER(c.c_int64),
                               c.POINTER(c.c_int64), c.POINTER(c.c_double)]
    for name in ("ep_decompress_into", "ep_decode_coords_into"):
        getattr(L, name).argtypes = [c.c_void_p, c.c_void_p, c.c_size_t, c.c_void_p, c.c_size_t, c.c_void_p]
    L.ep_decompress.argtypes = [c.c_void_p, c.c_void_p, c.c_size_t, c.POINTER(c.c_void_p), c.c_void_p]
    L.ep_decompress_many.argtypes = [c.c_int, c.POINTER(c.c_char_p), c.POINTER(c.c_void_p),
                                     c.POINTER(c.c_size_t), c.POINTER(c.c_void_p), c.POINTER(c.c_size_t),
                                     c.c_void_p]
    L.ep_get_device_status.argtypes = [c.c_void_p, c.POINTER(c.c_int32)]
    L.ep_plan_bitrates.argtypes = [c.c_int64, c.POINTER(c.c_int64), c.POINTER(c.c_int64), c.POINTER(c.c_double),
                                   c.c_double, c.c_double, c.c_double, c.POINTER(_Options), c.POINTER(c.c_double)]
    L.ep_status_string.restype = c.c_char_p
    L.ep_status_string.argtypes = [c.c_int]
    L.ep_last_error.restype = c.c_char_p
    L.ep_tans_compress.argtypes = [c.c_void_p, c.c_int, c.c_int, c.c_void_p, c.c_uint32, c.c_int,
                                   c.POINTER(c.c_void_p), c.POINTER(c.c_size_t)]
    L.ep_tans_info.argtypes = [c.c_void_p, c.c_size_t, c.POINTER(c.c_int), c.POINTER(c.c_int), c.c_void_p,
                               c.POINTER(c.c_uint32), c.POINTER(c.c_uint32)]
    L.ep_tans_decompress_into.argtypes = [c.c_void_p, c.c_void_p, c.c_size_t, c.c_void_p, c.c_size_t, c.c_void_p]
    for name in ("ep_compress", "ep_compress_cuda", "ep_blob_info", "ep_decompress_into", "ep_decode_coords_into", "ep_decompress",
                 "ep_get_device_status", "ep_decompress_many", "ep_plan_bitrates", "ep_tans_compress", "ep_tans_info",
                 "ep_tans_decompress_into"):
        getattr(L, name).restype = c.c_int
    _lib = L


def _check(st: int, what: str) -> None:
    if st != 0:
        L = lib()
        msg = L.ep_last_error().decode() or L.ep_status_string(st).decode()
        raise EntroPackError(st, f"{what}: {msg} (status {st})")


@dataclass
class EntroPackLossyConfig:
    """Lossy EntroPack configuration (README, Config table).

    target_bpp: finite, in [0.001, 11]. Fractional values are allowed. It counts metadata.
    rounds_per_tile: G. A tile is 32 lanes x G rounds x 8 coordinates. 0 (the default) means automatic:
    16 (4096 coordinates), or, for tensors of at least half a wave of tiles on a 148-SM B200, the G in
    [12, 24] that fills whole waves.
    encoder: "host" runs the multithreaded host encoder (ep_compress; CUDA inputs are copied to the host
    once). "cuda" runs the GPU encoder (ep_compress_cuda) on a CUDA input, on the current stream. Both
    write the same blob bytes.
    format_version: 2 (the default) writes 8-bit frequency tables with one rANS renormalisation per pair
    of symbols, the faster decode on B200; 1 writes 12-bit tables with one renormalisation per symbol.
    """
    target_bpp: float
    rounds_per_tile: int = 0
    sample_coords: int = 1 << 18
    bisection_iters: int = 40
    threads: int = 0
    encoder: str = "host"
    format_version: int = 2

    def _options(self) -> _Options:
        return _Options(self.rounds_per_tile, self.sample_coords, self.bisection_iters, self.threads,
                        self.format_version)


@dataclass
class TileANSConfig:
    """Lossless tile-ANS (README, Config table: TileANSConfig): exact restoration of BF16, FP16, FP32, FP8 and
    INT8 tensors of any shape (up to 8 dimensions); the ratio depends on the data. The elements' bytes are
    split into planes; clustered planes (sign and exponent bytes) are rANS-coded, the others stored as they
    are. elems_per_lane: K, a tile holds 32 x K elements (0 means 128). threads: host encoder threads (0: all
    cores)."""
    elems_per_lane: int = 0
    threads: int = 0


@dataclass
class CompressedTensor:
    """A compressed tensor: the blob bytes (EPK1 lossy, 2-D; or EPL1 lossless, any shape) plus a cached device
    copy per CUDA device."""
    blob: bytes
    shape: tuple
    dtype: torch.dtype
    actual_bpp: float
    _device_blobs: dict = field(default_factory=dict, repr=False)

    @property
    def lossless(self) -> bool:
        return self.blob[:4] == b"EPL1"

    @property
    def header(self) -> bytes:
        return self.blob[:TANS_HEADER_BYTES if self.lossless else HEADER_BYTES]

    @property
    def compressed_bits(self) -> int:
        return 8 * len(self.blob)

    def device_blob(self, device=None) -> torch.Tensor:
        """The blob as a uint8 CUDA tensor (cached). cudaMalloc alignment (256 B) meets the 16 B rule."""
        idx = None if device is None else torch.device(device).index
        dev = torch.device("cuda", torch.cuda.current_device() if idx is None else idx)
        t = self._device_blobs.get(dev.index)
        if t is None:
            host = torch.frombuffer(bytearray(self.blob), dtype=torch.uint8)
            t = host.to(dev)
            self._device_blobs[dev.index] = t
        return t

    def state_dict(self) -> dict:
        return {"blob": torch.frombuffer(bytearray(self.blob), dtype=torch.uint8)}

    @staticmethod
    def from_blob(blob: bytes) -> "CompressedTensor":
        info = blob_info(blob)
        return CompressedTensor(bytes(blob), info["shape"], _EP_TO_TORCH[info["dtype"]], info["actual_bpp"])


def blob_info(blob: bytes) -> dict:
    """Full host validation of a blob (header, tables, offsets, CRC) and its description. Lossy (EPK1) and
    lossless (EPL1) blobs both give dtype, shape and actual_bpp; lossy ones also rows and cols, lossless
    ones coded_mask (bit j: byte plane j is rANS-coded) and elems_per_lane."""
    c = ctypes
    if bytes(blob[:4]) == b"EPL1":
        dt, nd, mask, K = c.c_int(), c.c_int(), c.c_uint32(), c.c_uint32()
        dims = (c.c_int64 * 8)()
        _check(lib().ep_tans_info(blob, len(blob), c.byref(dt), c.byref(nd), dims, c.byref(mask), c.byref(K)),
               "blob_info")
        shape = tuple(dims[i] for i in range(nd.value))
        numel = math.prod(shape)
        return {"dtype": dt.value, "shape": shape, "coded_mask": mask.value, "elems_per_lane": K.value,
                "actual_bpp": 8 * len(blob) / numel if numel else 0.0}
    dt, M, N, bpp = c.c_int(), c.c_int64(), c.c_int64(), c.c_double()
    _check(lib().ep_blob_info(blob, len(blob), c.byref(dt), c.byref(M), c.byref(N), c.byref(bpp)), "blob_info")
    return {"dtype": dt.value, "rows": M.value, "cols": N.value, "shape": (M.value, N.value),
            "actual_bpp": bpp.value}


def _compress_lossless(tensor: torch.Tensor, config: TileANSConfig) -> CompressedTensor:
    if tensor.dtype not in _TORCH_TO_EP:
        raise EntroPackError(-2, f"compress: unsupported dtype {tensor.dtype}")
    if tensor.dim() > 8:
        raise EntroPackError(-3, "compress: tile-ANS takes tensors of at most 8 dimensions")
    host = tensor.detach().contiguous().cpu()
    dims = (ctypes.c_int64 * max(1, host.dim()))(*host.shape)
    blob_p, nbytes = ctypes.c_void_p(), ctypes.c_size_t()
    _check(lib().ep_tans_compress(host.data_ptr() if host.numel() else None, _TORCH_TO_EP[host.dtype], host.dim(),
                                  dims, int(config.elems_per_lane), int(config.threads), ctypes.byref(blob_p),
                                  ctypes.byref(nbytes)), "compress")
    try:
        blob = ctypes.string_at(blob_p.value, nbytes.value)
    finally:
        lib().ep_blob_free(blob_p)
    numel = host.numel()
    return CompressedTensor(blob, tuple(host.shape), tensor.dtype, 8 * len(blob) / numel if numel else 0.0)


def _rows_dense(t: torch.Tensor) -> torch.Tensor:
    """t itself when its rows are dense and do not overlap (the encoders take a row stride of at least cols),
    else a contiguous copy: transposed, expanded and other strided views."""
    return t if t.stride(1) == 1 and t.stride(0) >= t.shape[1] else t.contiguous()


def compress(tensor: torch.Tensor, config: EntroPackLossyConfig | TileANSConfig | float) -> CompressedTensor:
    """Compression of a tensor (CPU or CUDA). EntroPackLossyConfig (or a bare target in bits per parameter):
    lossy, 2-D tensors; the library runs rate control and encoding. TileANSConfig: lossless, any shape, on
    the host encoder."""
    if isinstance(config, TileANSConfig):
        return _compress_lossless(tensor, config)
    if not isinstance(config, EntroPackLossyConfig):
        config = EntroPackLossyConfig(float(config))
    if tensor.dim() != 2:
        raise EntroPackError(-3, "compress: EntroPack lossy mode takes 2-D tensors only")
    if tensor.dtype not in _TORCH_TO_EP:
        raise EntroPackError(-2, f"compress: unsupported dtype {tensor.dtype}")
    t = _rows_dense(tensor)
    rows, cols = t.shape
    blob_p, nbytes, actual = ctypes.c_void_p(), ctypes.c_size_t(), ctypes.c_double()
    opt = config._options()
    if config.encoder not in ("host", "cuda"):
        raise EntroPackError(-1, f"compress: unknown encoder {config.encoder!r}")
    if config.encoder == "cuda":
        if not t.is_cuda:
            raise EntroPackError(-1, "compress: the cuda encoder takes a CUDA tensor")
        with torch.cuda.device(t.device):
            st = lib().ep_compress_cuda(t.data_ptr(), _TORCH_TO_EP[t.dtype], rows, cols, t.stride(0),
                                        float(config.target_bpp), ctypes.byref(opt), torch.cuda.current_stream().cuda_stream,
                                        ctypes.byref(blob_p), ctypes.byref(nbytes), ctypes.byref(actual))
    elif t.is_cuda:
        with torch.cuda.device(t.device):
            torch.cuda.current_stream().synchronize()
            st = lib().ep_compress(t.data_ptr(), 1, _TORCH_TO_EP[t.dtype], rows, cols, t.stride(0),
                                   float(config.target_bpp), ctypes.byref(opt), ctypes.byref(blob_p),
                                   ctypes.byref(nbytes), ctypes.byref(actual))
    else:
        st = lib().ep_compress(t.data_ptr(), 0, _TORCH_TO_EP[t.dtype], rows, cols, t.stride(0),
                               float(config.target_bpp), ctypes.byref(opt), ctypes.byref(blob_p),
                               ctypes.byref(nbytes), ctypes.byref(actual))
    _check(st, "compress")
    try:
        blob = ctypes.string_at(blob_p.value, nbytes.value)
    finally:
        lib().ep_blob_free(blob_p)
    return CompressedTensor(blob, (rows, cols), tensor.dtype, actual.value)


def compress_cuda_noalloc(tensor: torch.Tensor, config: EntroPackLossyConfig | float) -> CompressedTensor:
    """ep_compress_cuda_noalloc on a CUDA tensor: the CUDA encoder with its device scratch in the
    library's fixed 64 MiB area (tensors up to about 4.5 M parameters), on the current stream."""
    if not isinstance(config, EntroPackLossyConfig):
        config = EntroPackLossyConfig(float(config))
    if tensor.dim() != 2 or not tensor.is_cuda:
        raise EntroPackError(-1, "compress_cuda_noalloc: takes a 2-D CUDA tensor")
    if tensor.dtype not in _TORCH_TO_EP:
        raise EntroPackError(-2, f"compress_cuda_noalloc: unsupported dtype {tensor.dtype}")
    t = _rows_dense(tensor)
    rows, cols = t.shape
    cap = 8 * rows * cols + 2 * rows + 4096
    buf = (ctypes.c_uint8 * cap)()
    nbytes, actual = ctypes.c_size_t(), ctypes.c_double()
    opt = config._options()
    with torch.cuda.device(t.device):
        st = lib().ep_compress_cuda_noalloc(t.data_ptr(), _TORCH_TO_EP[t.dtype], rows, cols, t.stride(0),
                                            float(config.target_bpp), ctypes.byref(opt),
                                            torch.cuda.current_stream().cuda_stream, buf, cap, ctypes.byref(nbytes),
                                            ctypes.byref(actual))
    _check(st, "compress_cuda_noalloc")
    return CompressedTensor(ctypes.string_at(buf, nbytes.value), (rows, cols), tensor.dtype, actual.value)


def plan_bitrates(shapes, weights, mean_bpp: float, min_bpp: float = 0.001, max_bpp: float = 11.0,
                  rounds_per_tile: int = 0, format_version: int = 2) -> list[float]:
    """ep_plan_bitrates: per-layer target bitrates that spend ``mean_bpp`` bits per parameter over the
    layers ``shapes`` [(rows, cols), ...], weighting layer i's squared error by ``weights[i]`` (the
    README's mixed-bitrate packs, which allocate bits by per-layer sensitivity). Each result is a
    target for ``compress``."""
    n = len(shapes)
    if n != len(weights) or n == 0:
        raise EntroPackError(-1, "plan_bitrates: need one weight per shape, and at least one layer")
    I64, F64 = ctypes.c_int64 * n, ctypes.c_double * n
    rows, cols = I64(*[int(r) for r, _ in shapes]), I64(*[int(c) for _, c in shapes])
    w, out = F64(*[float(x) for x in weights]), F64()
    opt = _Options()
    lib().ep_options_default(ctypes.byref(opt))
    opt.rounds_per_tile = int(rounds_per_tile)
    opt.format_version = int(format_version)
    _check(lib().ep_plan_bitrates(n, rows, cols, w, float(mean_bpp), float(min_bpp), float(max_bpp),
                                  ctypes.byref(opt), out), "plan_bitrates")
    return list(out)


def _stream_ptr(stream) -> int | None:
    s = torch.cuda.current_stream() if stream is None else stream
    return s.cuda_stream


def decompress_into(compressed: CompressedTensor, out: torch.Tensor, stream=None) -> torch.Tensor:
    """Decode into a preallocated CUDA tensor (contiguous, the blob's dtype and element count): the fused
    lossy decode (ep_decompress_into) or the lossless one (ep_tans_decompress_into). Asynchronous on
    ``stream`` (default: the current stream). It allocates nothing and does not synchronise."""
    if not out.is_cuda or not out.is_contiguous() or out.dtype != compressed.dtype:
        raise EntroPackError(-9, "decompress_into: out must be a contiguous CUDA tensor of the blob's dtype")
    dblob = compressed.device_blob(out.device)
    fn = lib().ep_tans_decompress_into if compressed.lossless else lib().ep_decompress_into
    _check(fn(compressed.header, dblob.data_ptr(), len(compressed.blob), out.data_ptr(),
              out.numel() * out.element_size(), _stream_ptr(stream)), "decompress_into")
    return out


class LayerBatch:
    """A fixed list of (compressed lossy tensor, output tensor) pairs, marshalled once. Each call to
    ``run()`` is one ``ep_decompress_many`` call on one stream: for version-2 blobs of one dtype, a table
    kernel and one persistent kernel over all the layers' tiles; otherwise one decode per blob, chained
    with programmatic dependent launch. Overlapping outputs end as if decoded in list order."""

    def __init__(self, pairs, stream=None):
        c = ctypes
        self.pairs = list(pairs)
        n = len(self.pairs)
        for comp, out in self.pairs:
            if not out.is_cuda or not out.is_contiguous() or out.dtype != comp.dtype:
                raise EntroPackError(-9, "LayerBatch: outputs must be contiguous CUDA tensors of the blobs' dtypes")
        self._keep = [comp.device_blob(out.device) for comp, out in self.pairs]
        self.n = n
        self.hdrs = (c.c_char_p * n)(*[comp.header for comp, _ in self.pairs])
        self.blobs = (c.c_void_p * n)(*[d.data_ptr() for d in self._keep])
        self.sizes = (c.c_size_t * n)(*[len(comp.blob) for comp, _ in self.pairs])
        self.dsts = (c.c_void_p * n)(*[out.data_ptr() for _, out in self.pairs])
        self.dst_sizes = (c.c_size_t * n)(*[out.numel() * out.element_size() for _, out in self.pairs])
        self.stream = stream

    def run(self, stream=None) -> None:
        s = _stream_ptr(stream if stream is not None else self.stream)
        _check(lib().ep_decompress_many(self.n, self.hdrs, self.blobs, self.sizes, self.dsts, self.dst_sizes, s),
               "decompress_many")


def decompress_many(pairs, stream=None) -> None:
    """Decodes each compressed tensor into its output tensor, in order, with one C call."""
    LayerBatch(pairs, stream).run()


def decompress(compressed: CompressedTensor, config=None, device=None, stream=None) -> torch.Tensor:
    """Decode to a new CUDA tensor of the original shape and dtype (README, quick-start section)."""
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    out = torch.empty(compressed.shape, dtype=compressed.dtype, device=dev)
    return decompress_into(compressed, out, stream)


def decode_coords(compressed: CompressedTensor, device=None, stream=None) -> torch.Tensor:
    """Lattice coordinates z = 2v (int32, shape of the tensor) as the CUDA decode produces them."""
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    out = torch.empty(compressed.shape, dtype=torch.int32, device=dev)
    dblob = compressed.device_blob(dev)
    _check(lib().ep_decode_coords_into(compressed.header, dblob.data_ptr(), len(compressed.blob), out.data_ptr(),
                                       out.numel() * 4, _stream_ptr(stream)), "decode_coords")
    return out


def device_status(stream=None) -> int:
    """Synchronises the stream, then reads and clears the device status word (EP_DEV_* bits). Decodes still
    running on other streams may set bits between the read and the clear: synchronise them first."""
    flags = ctypes.c_int32()
    _check(lib().ep_get_device_status(_stream_ptr(stream), ctypes.byref(flags)), "device_status")
    return flags.value


from .linear import CompressedLinear, DecodeWorkspace, link_prefetch  # noqa: E402  (uses the names above)
