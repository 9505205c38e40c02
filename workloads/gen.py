"""Counter-hash random inputs that are identical on the CPU and on the GPU.

Element ``i`` of a tensor drawn from stream ``k`` with seed ``s`` is

    N(0,1) sample = (pool[h1(i,k,s)] + pool[h2(i,k,s)]) / sqrt(2)

where ``pool`` is a fixed table of 2**24 standard normals drawn once from
torch's CPU generator, h1 is a 32-bit integer hash of the flat index
(Wellons' "lowbias32" mixer, keyed by seed and stream; the high 32 bits
of the index are mixed in only where they are non-zero) and h2 is one
more round of the mixer over h1.  The sum of two independent standard
normals divided by sqrt(2) is again standard normal.  Everything between
the index and the float is exact int64 arithmetic (products are split so
they never exceed 2**63), and the float part is one add and two multiplies
in float32, each correctly rounded, so CPU and CUDA produce bit-identical
values.  Uniform draws use the top 24 bits of one hash.

Any slice can be regenerated on its own (some rows, one expert), which is
what lets the CPU oracle check sampled outputs of layers whose weights
are tens of GB.
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess

import torch

_POOL_BITS = 24
_POOL_SEED = 0x5EED
_M32 = 0xFFFFFFFF
_pool_cache: dict = {}
_CHUNK_CPU = 1 << 20
_CHUNK_GPU = 1 << 26


def _chunk(device) -> int:
    return _CHUNK_CPU if torch.device(device).type == "cpu" else _CHUNK_GPU


def _pool(device) -> torch.Tensor:
    key = str(torch.device(device))
    p = _pool_cache.get(key)
    if p is None:
        if "cpu" not in _pool_cache:
            g = torch.Generator().manual_seed(_POOL_SEED)
            _pool_cache["cpu"] = torch.randn(1 << _POOL_BITS, generator=g,
                                             dtype=torch.float32)
        p = _pool_cache["cpu"].to(device)
        _pool_cache[key] = p
    return p


def _mul32(h: torch.Tensor, c: int) -> torch.Tensor:
    """(h * c) mod 2**32 for 0 <= h, c < 2**32 without int64 overflow."""
    lo = h * (c & 0xFFFF)
    hi = h * (c >> 16)
    hi &= 0xFFFF
    hi <<= 16
    lo += hi
    lo &= _M32
    return lo


def _mix32(h: torch.Tensor) -> torch.Tensor:
    h = h ^ (h >> 16)
    h = _mul32(h, 0x7FEB352D)
    h ^= h >> 15
    h = _mul32(h, 0x846CA68B)
    h ^= h >> 16
    return h


def _key(seed: int, stream: int, salt: int) -> int:
    v = torch.tensor([(seed * 0x3C6E + stream * 0x1B87 + salt * 0x5BD1) & _M32],
                     dtype=torch.int64)
    return int(_mix32(v)[0])


def _hash(flat: torch.Tensor, seed: int, stream: int) -> torch.Tensor:
    """32-bit hash of the flat index (both halves), keyed by seed and stream."""
    k = _key(seed, stream, 0)
    h = _mix32((flat & _M32) ^ k)
    hi = flat >> 32
    if flat.numel() and bool((hi > 0).any()):
        # element-wise, so a value never depends on how indices are chunked
        h = torch.where(hi > 0, _mix32(h ^ _mix32((hi + 0x68E31DA4) & _M32)), h)
    return h


def _flat_index(shape, device, rows=None, lead=None) -> list:
    """Chunks of flat int64 indices covering the requested slice."""
    shape = tuple(int(s) for s in shape)
    CH = _chunk(device)
    inner = 1
    for s in shape[1:]:
        inner *= s
    if rows is not None:
        rows = torch.as_tensor(rows, dtype=torch.int64, device=device)
        base = rows.reshape(-1, 1) * inner
        cols = torch.arange(inner, dtype=torch.int64, device=device)
        out_shape = (rows.numel(),) + shape[1:]
        total = rows.numel() * inner
        per = max(1, CH // max(inner, 1))
        chunks = [(base[i:i + per] + cols).reshape(-1)
                  for i in range(0, rows.numel(), per)]
        return chunks, out_shape, total
    if lead is not None:
        start = int(lead) * inner
        out_shape = shape[1:]
        total = inner
    else:
        start = 0
        out_shape = shape
        total = inner * shape[0]
    chunks = []
    for c0 in range(0, total, CH):
        n = min(CH, total - c0)
        chunks.append(torch.arange(start + c0, start + c0 + n,
                                   dtype=torch.int64, device=device))
    return chunks, out_shape, total


_clib = None
_CSRC = os.path.join(os.path.dirname(os.path.abspath(__file__)), "_gen.c")
_CSO = os.path.join(os.path.dirname(os.path.abspath(__file__)), "_gen.so")


def build_c(force: bool = False) -> str:
    """Compile the host generator (gcc, OpenMP); returns the .so path."""
    if force or not os.path.exists(_CSO) or (
            os.path.getmtime(_CSO) < os.path.getmtime(_CSRC)):
        tmp = _CSO + ".%d.tmp" % os.getpid()
        subprocess.run(["gcc", "-O2", "-fopenmp", "-ffp-contract=off",
                        "-shared", "-fPIC", _CSRC, "-o", tmp], check=True)
        os.replace(tmp, _CSO)
    return _CSO


def _c():
    global _clib
    if _clib is None:
        try:
            lib = ctypes.CDLL(build_c())
        except Exception:  # no compiler: fall back to the torch path
            _clib = False
            return None
        for fn in (lib.gen_normal_range, lib.gen_normal_at):
            fn.restype = None
        lib.gen_normal_range.argtypes = [
            ctypes.c_int64, ctypes.c_int64, ctypes.c_uint32, ctypes.c_void_p,
            ctypes.c_float, ctypes.c_float, ctypes.c_void_p]
        lib.gen_normal_at.argtypes = [
            ctypes.c_void_p, ctypes.c_int64, ctypes.c_uint32, ctypes.c_void_p,
            ctypes.c_float, ctypes.c_float, ctypes.c_void_p]
        _clib = lib
    return _clib or None


def _normal_cpu_c(lib, shape, seed, stream, std, rows, lead, dtype):
    pool = _pool("cpu")
    key = _key(seed, stream, 0)
    inv = float(torch.tensor(1.0 / math.sqrt(2.0), dtype=torch.float32))
    sd = float(torch.tensor(std, dtype=torch.float32))
    shape = tuple(int(s) for s in shape)
    inner = 1
    for s in shape[1:]:
        inner *= s
    if rows is not None:
        rows = torch.as_tensor(rows, dtype=torch.int64)
        flat = (rows.reshape(-1, 1) * inner
                + torch.arange(inner, dtype=torch.int64)).reshape(-1).contiguous()
        out = torch.empty(flat.numel(), dtype=torch.float32)
        lib.gen_normal_at(flat.data_ptr(), flat.numel(), key, pool.data_ptr(),
                          inv, sd, out.data_ptr())
        return out.reshape((rows.numel(),) + shape[1:]).to(dtype)
    start = int(lead) * inner if lead is not None else 0
    total = inner if lead is not None else inner * shape[0]
    out = torch.empty(total, dtype=torch.float32)
    lib.gen_normal_range(start, total, key, pool.data_ptr(), inv, sd,
                         out.data_ptr())
    return out.reshape(shape[1:] if lead is not None else shape).to(dtype)


def normal_at(shape, flat_index, seed: int, stream: int, std: float,
              dtype=torch.float32) -> torch.Tensor:
    """Samples at arbitrary flat indices of a tensor of `shape` (CPU)."""
    flat = torch.as_tensor(flat_index, dtype=torch.int64).reshape(-1).contiguous()
    lib = _c()
    if lib is not None:
        pool = _pool("cpu")
        inv = float(torch.tensor(1.0 / math.sqrt(2.0), dtype=torch.float32))
        sd = float(torch.tensor(std, dtype=torch.float32))
        out = torch.empty(flat.numel(), dtype=torch.float32)
        lib.gen_normal_at(flat.data_ptr(), flat.numel(), _key(seed, stream, 0),
                          pool.data_ptr(), inv, sd, out.data_ptr())
        return out.to(dtype)
    return _normal_torch(flat, seed, stream, std, "cpu").to(dtype)


def _normal_torch(flat, seed, stream, std, device):
    pool = _pool(device)
    mask = (1 << _POOL_BITS) - 1
    h = _hash(flat, seed, stream)
    i1 = h & mask
    i2 = _mix32(h ^ 0x9E3779B9) & mask
    v = pool[i1] + pool[i2]
    v = v * torch.tensor(1.0 / math.sqrt(2.0), dtype=torch.float32).to(device)
    v = v * torch.tensor(std, dtype=torch.float32).to(device)
    return v


def normal(shape, seed: int, stream: int, std: float, device="cpu", *,
           rows=None, lead=None, dtype=torch.float32,
           use_c: bool = True) -> torch.Tensor:
    """std * N(0,1) samples for `shape` (or its `rows` / `lead` slice)."""
    if torch.device(device).type == "cpu" and use_c:
        lib = _c()
        if lib is not None:
            return _normal_cpu_c(lib, shape, seed, stream, std, rows, lead,
                                 dtype)
    chunks, out_shape, total = _flat_index(shape, device, rows, lead)
    out = torch.empty(total, dtype=dtype, device=device)
    pos = 0
    for flat in chunks:
        v = _normal_torch(flat, seed, stream, std, device)
        out[pos:pos + flat.numel()] = v.to(dtype)
        pos += flat.numel()
    return out.reshape(out_shape)


def uniform(shape, seed: int, stream: int, lo: float, hi: float,
            device="cpu") -> torch.Tensor:
    """U(lo, hi) samples (float64 arithmetic, returned as float64)."""
    chunks, out_shape, total = _flat_index(shape, device)
    parts = []
    for flat in chunks:
        h = _mix32(_hash(flat, seed, stream) ^ 0x2545F491)
        u = (h >> 8).to(torch.float64) / float(1 << 24)
        parts.append(lo + (hi - lo) * u)
    return torch.cat(parts).reshape(out_shape)
