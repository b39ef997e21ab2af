"""Seeded, counter-based input generator shared by the oracle tests, the CUDA
parity tests and the benchmark.

It holds none of the attention method's arithmetic: it only maps
(seed, tensor id, flat index) to a reproducible pseudo-normal value, with
bit-identical implementations on the host (``rng_host.c``) and on the device
(``rng_device.cu``).  The definition is written out in ``rng_host.c``.

bf16 tensors are handled as uint16 bit patterns on the host; ``bf16_to_f32``
turns them into exactly-equal float32 values.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
HOST_SO = os.path.join(_HERE, "librng_host.so")
DEVICE_SO = os.path.join(_HERE, "librng_device.so")

_host = None
_device = None


def build(device: bool = True) -> None:
    """Compile the host generator with gcc and the device generator with nvcc (sm_100a)."""
    src = os.path.join(_HERE, "rng_host.c")
    subprocess.check_call(["gcc", "-O3", "-fopenmp", "-ffp-contract=off", "-fPIC", "-shared", src, "-o", HOST_SO])
    if device:
        dsrc = os.path.join(_HERE, "rng_device.cu")
        subprocess.check_call(["nvcc", "-O3", "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo",
                               "-fmad=false", "-Xcompiler", "-fPIC", "-shared", dsrc, "-o", DEVICE_SO])


def _load_host():
    global _host
    if _host is None:
        src = os.path.join(_HERE, "rng_host.c")
        if not os.path.exists(HOST_SO) or os.path.getmtime(HOST_SO) < os.path.getmtime(src):
            build(device=False)
        lib = ctypes.CDLL(HOST_SO)
        u64, i64, f32, vp = ctypes.c_uint64, ctypes.c_int64, ctypes.c_float, ctypes.c_void_p
        lib.rng_draw_u64.argtypes = [u64, u64, u64, i64, vp]
        lib.rng_normal_f32.argtypes = [u64, u64, u64, i64, f32, vp]
        lib.rng_normal_bf16.argtypes = [u64, u64, u64, i64, f32, vp]
        lib.rng_normal_rows_f32.argtypes = [u64, u64, i64, vp, i64, f32, vp]
        lib.rng_normal_rows_bf16.argtypes = [u64, u64, i64, vp, i64, f32, vp]
        lib.rng_splitmix64_from_state.argtypes = [u64, i64, vp]
        lib.rng_splitmix64_from_state.restype = None
        for f in (lib.rng_draw_u64, lib.rng_normal_f32, lib.rng_normal_bf16, lib.rng_normal_rows_f32,
                  lib.rng_normal_rows_bf16):
            f.restype = None
        _host = lib
    return _host


def _load_device():
    global _device
    if _device is None:
        if not os.path.exists(DEVICE_SO):
            raise RuntimeError(f"device generator not built: {DEVICE_SO} (run msa_inputs.rng.build())")
        lib = ctypes.CDLL(DEVICE_SO)
        lib.rng_fill_normal.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_uint64, ctypes.c_uint64,
                                        ctypes.c_uint64, ctypes.c_int64, ctypes.c_float, ctypes.c_void_p]
        lib.rng_fill_normal.restype = ctypes.c_int
        _device = lib
    return _device


# ----------------------------------------------------------------------------------------------
# bf16 <-> fp32 bit helpers (round-to-nearest-even, no NaN handling: the generator makes none)
# ----------------------------------------------------------------------------------------------
def f32_to_bf16(x: np.ndarray) -> np.ndarray:
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return u.astype(np.uint16)


def bf16_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def round_to(x: np.ndarray, dtype: str) -> np.ndarray:
    """float32 values rounded to the storage type and returned as float32."""
    x = np.asarray(x, dtype=np.float32)
    return bf16_to_f32(f32_to_bf16(x)) if dtype == "bf16" else x


def to_storage(x: np.ndarray, dtype: str) -> np.ndarray:
    """float32 array -> the array whose bytes are the storage form (fp32 or bf16 bits)."""
    return f32_to_bf16(x) if dtype == "bf16" else np.ascontiguousarray(x, dtype=np.float32)


# ----------------------------------------------------------------------------------------------
# host generation
# ----------------------------------------------------------------------------------------------
def splitmix64_stream(state: int, n: int) -> np.ndarray:
    """The plain SplitMix64 sequence started from `state` (for checking the generator itself)."""
    out = np.empty(n, dtype=np.uint64)
    _load_host().rng_splitmix64_from_state(state, n, out.ctypes.data)
    return out


def draw_u64(seed: int, tid: int, start: int, n: int) -> np.ndarray:
    out = np.empty(n, dtype=np.uint64)
    _load_host().rng_draw_u64(seed, tid, start, n, out.ctypes.data)
    return out


def normal(seed: int, tid: int, start: int, n: int, sigma: float = 1.0, dtype: str = "f32") -> np.ndarray:
    """float32 values of flat elements start..start+n-1 (bf16-rounded when dtype == 'bf16')."""
    lib = _load_host()
    if dtype == "bf16":
        bits = np.empty(n, dtype=np.uint16)
        lib.rng_normal_bf16(seed, tid, start, n, sigma, bits.ctypes.data)
        return bf16_to_f32(bits)
    out = np.empty(n, dtype=np.float32)
    lib.rng_normal_f32(seed, tid, start, n, sigma, out.ctypes.data)
    return out


def normal_rows(seed: int, tid: int, row_len: int, rows, sigma: float = 1.0, dtype: str = "f32") -> np.ndarray:
    """Selected rows of a [*, row_len] generated tensor, as float32 [len(rows), row_len]."""
    rows = np.ascontiguousarray(rows, dtype=np.int64)
    lib = _load_host()
    if dtype == "bf16":
        bits = np.empty((len(rows), row_len), dtype=np.uint16)
        lib.rng_normal_rows_bf16(seed, tid, row_len, rows.ctypes.data, len(rows), sigma, bits.ctypes.data)
        return bf16_to_f32(bits)
    out = np.empty((len(rows), row_len), dtype=np.float32)
    lib.rng_normal_rows_f32(seed, tid, row_len, rows.ctypes.data, len(rows), sigma, out.ctypes.data)
    return out


def uniform_int(seed: int, tid: int, n: int, hi: int) -> np.ndarray:
    """n integers in [0, hi) by the multiply-shift map (draw >> 32) * hi >> 32 (Lemire 2019)."""
    d = draw_u64(seed, tid, 0, n)
    return ((d >> np.uint64(32)) * np.uint64(hi)) >> np.uint64(32)


def distinct_ints(seed: int, tid: int, n: int, hi: int, exclude=()) -> np.ndarray:
    """n distinct integers in [0, hi), not in ``exclude``, taken in draw order."""
    got, seen, start = [], set(int(e) for e in exclude), 0
    free = hi - len({e for e in seen if 0 <= e < hi})
    if n > free:
        raise ValueError(f"distinct_ints: {n} distinct values asked from {free} available in [0, {hi})")
    while len(got) < n:
        d = draw_u64(seed, tid, start, 4 * n + 16)
        start += len(d)
        for v in ((d >> np.uint64(32)) * np.uint64(hi)) >> np.uint64(32):
            v = int(v)
            if v not in seen:
                seen.add(v)
                got.append(v)
                if len(got) == n:
                    break
    return np.array(got, dtype=np.int64)


# ----------------------------------------------------------------------------------------------
# device generation (torch tensors; torch is only the allocator here)
# ----------------------------------------------------------------------------------------------
def fill_device(t, seed: int, tid: int, start: int = 0, sigma: float = 1.0, stream=None) -> None:
    """Fill a contiguous CUDA tensor (float32 or bfloat16) with the generator's values."""
    import torch

    assert t.is_cuda and t.is_contiguous()
    dt = {torch.float32: 0, torch.bfloat16: 1}[t.dtype]
    s = stream if stream is not None else torch.cuda.current_stream()
    rc = _load_device().rng_fill_normal(t.data_ptr(), dt, seed, tid, start, t.numel(), sigma, s.cuda_stream)
    if rc != 0:
        raise RuntimeError(f"rng_fill_normal failed with CUDA error {rc}")
