"""Seeded synthetic inputs, identical on the host and on the GPU.

This module is the only code that both the CUDA path's callers and the CPU
oracle's tests use. It draws numbers and lays them out; it performs none of
the method's arithmetic (no quantiser, score, selection or attention).

Generator: a counter-based splitmix64. Element i of stream s under seed S is
    z = mix(mix(S * G + s) + i * G)
with G = 0x9E3779B97F4A7C15 and mix() the splitmix64 finaliser (Steele, Lea
and Flood, "Fast splittable pseudorandom number generators", OOPSLA 2014).
All arithmetic is 64-bit two's complement in torch int64 tensors, so any
element can be drawn on any device and the CPU and GPU give the same bits.

Value maps, all table lookups so that no libm call decides a bit:
  * normal_bf16: the top 16 bits of z index a 65536-entry table of bf16
    values bf16(Phi^-1((j + 0.5) / 65536)), a discretised N(0, 1).
  * the same table rounded to E4M3 (via torch's float8_e4m3fn cast) for the
    FP8 sliding-window rows.
  * small integers in [lo, hi]: (z >>> 32) mod (hi - lo + 1) + lo, and their
    E4M3 bytes via a 17-entry table (integers in [-8, 8] are exact in E4M3).
"""
import torch

_G = 0x9E3779B97F4A7C15
_M1 = 0xBF58476D1CE4E5B9
_M2 = 0x94D049BB133111EB
_MASK64 = (1 << 64) - 1


def _s64(v: int) -> int:
    """Python int in [0, 2^64) -> the int64 with the same bits."""
    v &= _MASK64
    return v - (1 << 64) if v >= (1 << 63) else v


def _mix_int(z: int) -> int:
    z &= _MASK64
    z ^= z >> 30
    z = (z * _M1) & _MASK64
    z ^= z >> 27
    z = (z * _M2) & _MASK64
    z ^= z >> 31
    return z


def _lsr(z: torch.Tensor, k: int) -> torch.Tensor:
    """Logical right shift of int64 bits."""
    return (z >> k) & ((1 << (64 - k)) - 1)


def _mix(z: torch.Tensor) -> torch.Tensor:
    z = z ^ _lsr(z, 30)
    z = z * _s64(_M1)
    z = z ^ _lsr(z, 27)
    z = z * _s64(_M2)
    z = z ^ _lsr(z, 31)
    return z


def stream_base(seed: int, stream: int) -> int:
    return _mix_int(seed * _G + stream)


def raw_bits(seed: int, stream: int, start: int, count: int, device="cpu") -> torch.Tensor:
    """int64 tensor of the generator's 64-bit outputs for elements [start, start+count)."""
    base = _s64(stream_base(seed, stream))
    i = torch.arange(start, start + count, dtype=torch.int64, device=device)
    return _mix(base + i * _s64(_G))


def raw_bits_at(seed: int, stream: int, idx: torch.Tensor) -> torch.Tensor:
    """Generator outputs for arbitrary element indices (int64 tensor)."""
    base = _s64(stream_base(seed, stream))
    return _mix(base + idx.to(torch.int64) * _s64(_G))


# ---- value tables ---------------------------------------------------------------

_TABLES = {}


def _tables(device):
    key = str(device)
    if key not in _TABLES:
        j = torch.arange(65536, dtype=torch.float64)
        nrm = torch.special.ndtri((j + 0.5) / 65536.0)
        nrm_bf16 = nrm.to(torch.float32).to(torch.bfloat16)
        nrm_bits = nrm_bf16.view(torch.int16).to(torch.int32) & 0xFFFF
        nrm_e4m3 = nrm.to(torch.float32).to(torch.float8_e4m3fn).view(torch.uint8)
        ints = torch.arange(-8, 9, dtype=torch.float32)
        int_e4m3 = ints.to(torch.float8_e4m3fn).view(torch.uint8)
        _TABLES[key] = {
            "normal_bf16_bits": nrm_bits.to(device),
            "normal_e4m3": nrm_e4m3.to(device),
            "int_e4m3": int_e4m3.to(device),   # index v + 8 for v in [-8, 8]
        }
    return _TABLES[key]


def bf16_bits_to_tensor(bits_i32: torch.Tensor) -> torch.Tensor:
    """int32 tensor of bf16 bit patterns (0..65535) -> bfloat16 tensor."""
    return bits_i32.to(torch.int16).view(torch.bfloat16)


# ---- draws ----------------------------------------------------------------------

def normal_bf16(seed, stream, start, count, device="cpu", outlier_p=0.0, outlier_mul=1.0,
                outlier_stream=None):
    """bf16 tensor of discretised N(0,1) draws; optionally each element is, with
    probability outlier_p (decided by a second stream), multiplied by outlier_mul
    (the product rounded to bf16)."""
    t = _tables(device)
    z = raw_bits(seed, stream, start, count, device)
    bits = t["normal_bf16_bits"][_lsr(z, 48)]
    x = bf16_bits_to_tensor(bits)
    if outlier_p > 0.0:
        zo = raw_bits(seed, outlier_stream, start, count, device)
        u = _lsr(zo, 11).to(torch.float64) * (2.0 ** -53)
        sel = u < outlier_p
        x = torch.where(sel, (x.float() * outlier_mul).to(torch.bfloat16), x)
    return x


def normal_e4m3(seed, stream, start, count, device="cpu"):
    """uint8 tensor of E4M3 bytes of discretised N(0,1) draws."""
    t = _tables(device)
    z = raw_bits(seed, stream, start, count, device)
    return t["normal_e4m3"][_lsr(z, 48)]


def uniform_int(seed, stream, start, count, lo, hi, device="cpu"):
    """int64 tensor of integers uniform on [lo, hi]."""
    z = raw_bits(seed, stream, start, count, device)
    return _lsr(z, 32) % (hi - lo + 1) + lo


def int_e4m3(seed, stream, start, count, lo=-8, hi=8, device="cpu"):
    """uint8 tensor of E4M3 bytes of integers uniform on [lo, hi] (within [-8, 8])."""
    assert -8 <= lo <= hi <= 8
    t = _tables(device)
    v = uniform_int(seed, stream, start, count, lo, hi, device)
    return t["int_e4m3"][v + 8]


def permutation(seed, stream, n):
    """Fisher-Yates permutation of range(n) driven by the generator (host only)."""
    z = raw_bits(seed, stream, 0, max(n, 1), "cpu")
    r = _lsr(z, 32).tolist()
    perm = list(range(n))
    for i in range(n - 1, 0, -1):
        j = r[i] % (i + 1)
        perm[i], perm[j] = perm[j], perm[i]
    return torch.tensor(perm, dtype=torch.int32)
