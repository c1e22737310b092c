"""EntroPack oracle: a ctypes wrapper over the plain C encoder and decoder.

TEST INFRASTRUCTURE, NOT PRODUCT CODE. Only the test suite, the smoke check in
``__graft_entry__`` and the CPU-baseline leg of ``bench.py`` may import this
package. The product library (``decode_ep_b200``) never imports it and shares no
code with it. Where each part of the method comes from on the EntroPack pages is
written in ``entropack_oracle.c``.

Parity pins: ``tests/test_oracle_*.py`` check this oracle against brute force,
closed forms, library routines and the numbers the pages print. Every oracle
function has at least one pin.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "liboracle.so")
SRC_PATH = os.path.join(HERE, "entropack_oracle.c")
SOURCES = [SRC_PATH, os.path.join(HERE, "tileans_oracle.c")]

DTYPES = {"bf16": 1, "fp16": 2, "fp32": 3, "fp8_e4m3": 4, "int8": 5}
ELEM = {1: 2, 2: 2, 3: 4, 4: 1, 5: 1}
NP_CONTAINER = {1: np.uint16, 2: np.uint16, 3: np.float32, 4: np.uint8, 5: np.int8}


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (-O2, no FMA contraction)."""
    newest = max(os.path.getmtime(f) for f in SOURCES + [os.path.join(HERE, "entropack_oracle.h")])
    if force or not os.path.exists(LIB_PATH) or os.path.getmtime(LIB_PATH) < newest:
        cmd = ["gcc", "-O2", "-std=c11", "-Wall", "-ffp-contract=off", "-fPIC", "-shared",
               *SOURCES, "-o", LIB_PATH, "-lm"]
        subprocess.run(cmd, check=True)
    return LIB_PATH


_lib = None


def lib():
    global _lib
    if _lib is None:
        L = ctypes.CDLL(build())
        c = ctypes
        L.orc_crc32.restype = c.c_uint32
        L.orc_crc32.argtypes = [c.c_void_p, c.c_size_t]
        L.orc_e8_nearest.argtypes = [c.c_void_p, c.c_void_p, c.c_void_p]
        L.orc_normalize.argtypes = [c.c_void_p, c.c_int, c.c_void_p]
        L.orc_normalize_bits.argtypes = [c.c_void_p, c.c_int, c.c_int, c.c_void_p]
        L.orc_to_container.argtypes = [c.c_void_p, c.c_int64, c.c_int, c.c_void_p]
        L.orc_from_container.argtypes = [c.c_void_p, c.c_int64, c.c_int, c.c_void_p]
        L.orc_compress.argtypes = [c.c_void_p, c.c_int, c.c_int64, c.c_int64, c.c_double, c.c_int,
                                   c.c_double, c.c_int, c.POINTER(c.c_void_p), c.POINTER(c.c_size_t),
                                   c.POINTER(c.c_double)]
        L.orc_free.argtypes = [c.c_void_p]
        L.orc_estimate_bytes.restype = c.c_double
        L.orc_estimate_bytes.argtypes = [c.c_void_p, c.c_int, c.c_int64, c.c_int64, c.c_int, c.c_float, c.c_int]
        L.orc_blob_info.argtypes = [c.c_void_p, c.c_size_t, c.POINTER(c.c_int), c.POINTER(c.c_int64),
                                    c.POINTER(c.c_int64), c.POINTER(c.c_float), c.POINTER(c.c_int),
                                    c.POINTER(c.c_int), c.POINTER(c.c_uint32), c.POINTER(c.c_int)]
        L.orc_decode_tiles.argtypes = [c.c_void_p, c.c_size_t, c.c_uint32, c.c_uint32, c.c_void_p,
                                       c.c_void_p]
        L.orc_decompress.argtypes = [c.c_void_p, c.c_size_t, c.c_void_p, c.c_void_p]
        L.orc_quantize.argtypes = [c.c_void_p, c.c_int, c.c_int64, c.c_int64, c.c_float, c.c_void_p,
                                   c.c_void_p]
        L.orc_tans_compress.argtypes = [c.c_void_p, c.c_int, c.c_int, c.c_void_p, c.c_int, c.POINTER(c.c_void_p),
                                        c.POINTER(c.c_size_t)]
        L.orc_tans_info.argtypes = [c.c_void_p, c.c_size_t, c.POINTER(c.c_int), c.POINTER(c.c_int), c.c_void_p,
                                    c.POINTER(c.c_int), c.POINTER(c.c_uint32), c.POINTER(c.c_int)]
        L.orc_tans_decode_tiles.argtypes = [c.c_void_p, c.c_size_t, c.c_uint32, c.c_uint32, c.c_void_p]
        L.orc_tans_decompress.argtypes = [c.c_void_p, c.c_size_t, c.c_void_p]
        _lib = L
    return _lib


class OracleError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what}: oracle status {status}")
        self.status = status


def _check(st: int, what: str) -> None:
    if st != 0:
        raise OracleError(st, what)


def _ptr(a: np.ndarray) -> int:
    return a.ctypes.data


def crc32(data: bytes) -> int:
    buf = np.frombuffer(data, dtype=np.uint8)
    return int(lib().orc_crc32(_ptr(buf) if buf.size else None, buf.size))


def e8_nearest(x) -> tuple[int, np.ndarray]:
    """Nearest E8 point of x (8 floats): returns (b, u) with v = u + b/2."""
    xa = np.ascontiguousarray(x, dtype=np.float64)
    b = np.zeros(1, np.int32)
    u = np.zeros(8, np.int64)
    lib().orc_e8_nearest(_ptr(xa), _ptr(b), _ptr(u))
    return int(b[0]), u


def normalize(counts, bits: int = 12) -> np.ndarray:
    """Frequencies of `bits` bits (12: format version 1, 8: version 2) for the symbol counts."""
    c = np.ascontiguousarray(counts, dtype=np.uint64)
    f = np.zeros(c.size, np.uint32)
    _check(lib().orc_normalize_bits(_ptr(c), int(c.size), int(bits), _ptr(f)), "normalize")
    return f


def to_container(y, dtype: int) -> np.ndarray:
    ya = np.ascontiguousarray(y, dtype=np.float32).ravel()
    out = np.zeros(ya.size, NP_CONTAINER[dtype])
    lib().orc_to_container(_ptr(ya), ya.size, dtype, _ptr(out))
    return out


def from_container(a: np.ndarray, dtype: int) -> np.ndarray:
    a = np.ascontiguousarray(a).ravel()
    out = np.zeros(a.size, np.float32)
    _check(lib().orc_from_container(_ptr(a), a.size, dtype, _ptr(out)), "from_container")
    return out


def compress(data: np.ndarray, dtype: int, target_bpp: float, rounds_per_tile: int = 16,
             force_alpha: float = 0.0, prob_bits: int = 8) -> tuple[bytes, float]:
    """Compress a row-major 2-D container array (the raw container bit patterns). prob_bits 8 writes
    format version 2 (8-bit tables, pairs of symbols per renormalisation), 12 writes version 1."""
    a = np.ascontiguousarray(data)
    assert a.ndim == 2 and a.dtype.itemsize == ELEM.get(dtype, a.dtype.itemsize)
    blob = ctypes.c_void_p()
    nbytes = ctypes.c_size_t()
    actual = ctypes.c_double()
    st = lib().orc_compress(_ptr(a), dtype, a.shape[0], a.shape[1], float(target_bpp),
                            int(rounds_per_tile), float(force_alpha), int(prob_bits), ctypes.byref(blob),
                            ctypes.byref(nbytes), ctypes.byref(actual))
    _check(st, "compress")
    try:
        out = ctypes.string_at(blob.value, nbytes.value)
    finally:
        lib().orc_free(blob)
    return out, actual.value


def estimate_bytes(data: np.ndarray, dtype: int, alpha: float, rounds_per_tile: int = 16,
                   prob_bits: int = 8) -> float:
    a = np.ascontiguousarray(data)
    return float(lib().orc_estimate_bytes(_ptr(a), dtype, a.shape[0], a.shape[1], rounds_per_tile,
                                          float(alpha), int(prob_bits)))


def blob_info(blob: bytes) -> dict:
    c = ctypes
    dt, M, N, al, r, G, T = c.c_int(), c.c_int64(), c.c_int64(), c.c_float(), c.c_int(), c.c_int(), c.c_uint32()
    ver = c.c_int()
    st = lib().orc_blob_info(blob, len(blob), c.byref(dt), c.byref(M), c.byref(N), c.byref(al),
                             c.byref(r), c.byref(G), c.byref(T), c.byref(ver))
    _check(st, "blob_info")
    return {"dtype": dt.value, "rows": M.value, "cols": N.value, "alpha": al.value, "r": r.value,
            "G": G.value, "num_tiles": T.value, "version": ver.value}


def decompress(blob: bytes, with_coords: bool = False):
    """Decode the whole blob: returns the container array (and z = 2v if asked)."""
    info = blob_info(blob)
    M, N, dt = info["rows"], info["cols"], info["dtype"]
    out = np.zeros((M, N), NP_CONTAINER[dt])
    z = np.zeros((M, N), np.int32) if with_coords else None
    st = lib().orc_decompress(blob, len(blob), _ptr(out), _ptr(z) if z is not None else None)
    _check(st, "decompress")
    return (out, z) if with_coords else out


def decode_tiles(blob: bytes, t0: int, t1: int, out: np.ndarray, z: np.ndarray | None = None) -> None:
    """Decode tiles [t0, t1) into the full-size arrays out (and z)."""
    st = lib().orc_decode_tiles(blob, len(blob), t0, t1, _ptr(out), _ptr(z) if z is not None else None)
    _check(st, "decode_tiles")


def quantize(data: np.ndarray, dtype: int, alpha: float) -> tuple[np.ndarray, np.ndarray]:
    a = np.ascontiguousarray(data)
    M, N = a.shape
    z = np.zeros((M, N), np.int32)
    s = np.zeros(M, np.uint16)
    _check(lib().orc_quantize(_ptr(a), dtype, M, N, float(alpha), _ptr(z), _ptr(s)), "quantize")
    return z, s


# ------------------------------------------------------------------ lossless tile-ANS (EPL1)

TANS_NP = {1: np.uint16, 2: np.uint16, 3: np.uint32, 4: np.uint8, 5: np.uint8}


def tans_compress(bits: np.ndarray, dtype: int, K: int = 0) -> bytes:
    """Lossless tile-ANS blob of an array of raw bit patterns (``TANS_NP[dtype]``; any shape, ndim <= 8)."""
    a = np.asarray(bits)
    if not a.flags.c_contiguous:
        a = a.copy(order="C")  # (np.ascontiguousarray would turn a 0-d array into a 1-d one)
    if a.dtype != TANS_NP[dtype]:
        raise ValueError("tans_compress: bits must hold the dtype's raw patterns")
    dims = (ctypes.c_int64 * max(1, a.ndim))(*a.shape)
    p, n = ctypes.c_void_p(), ctypes.c_size_t()
    _check(lib().orc_tans_compress(a.ctypes.data if a.size else None, dtype, a.ndim, dims, K, ctypes.byref(p),
                                   ctypes.byref(n)), "tans_compress")
    try:
        return ctypes.string_at(p.value, n.value)
    finally:
        lib().orc_free(p)


def tans_info(blob: bytes) -> dict:
    c = ctypes
    dt, nd, K, T, mask = c.c_int(), c.c_int(), c.c_int(), c.c_uint32(), c.c_int()
    dims = (c.c_int64 * 8)()
    _check(lib().orc_tans_info(blob, len(blob), c.byref(dt), c.byref(nd), dims, c.byref(K), c.byref(T),
                               c.byref(mask)), "tans_info")
    return {"dtype": dt.value, "shape": tuple(dims[i] for i in range(nd.value)), "K": K.value,
            "num_tiles": T.value, "coded_mask": mask.value}


def tans_decompress(blob: bytes) -> np.ndarray:
    """The raw bit patterns, in the blob's shape."""
    info = tans_info(blob)
    out = np.zeros(info["shape"], TANS_NP[info["dtype"]])
    _check(lib().orc_tans_decompress(blob, len(blob), out.ctypes.data if out.size else None), "tans_decompress")
    return out


def tans_decode_tiles(blob: bytes, t0: int, t1: int, out: np.ndarray) -> None:
    """Decode tiles [t0, t1) into ``out`` (the whole tensor's array of raw bit patterns)."""
    _check(lib().orc_tans_decode_tiles(blob, len(blob), t0, t1, out.ctypes.data if out.size else None),
           "tans_decode_tiles")
