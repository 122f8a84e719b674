"""Seeded, counter-based synthetic inputs (host side, numpy).

This module only draws numbers: it holds none of the method's arithmetic.
Both the CPU oracle's inputs and the device buffers the CUDA path reads come
from the generator defined here, so the two see identical bytes.

Generator definition (the device twin in ``gen_cuda.cu`` implements the same
definition and is tested bit-for-bit against this one):

* ``mix64`` is the SplitMix64 output finaliser (Steele, Lea & Flood,
  "Fast splittable pseudorandom number generators", OOPSLA 2014; constants of
  Vigna's ``splitmix64.c``): ``z ^= z>>30; z *= 0xBF58476D1CE4E5B9;
  z ^= z>>27; z *= 0x94D049BB133111EB; z ^= z>>31`` (all mod 2**64).
* Element ``i`` of the stream with 64-bit key ``s`` is
  ``x = mix64(s + (i + 1) * 0x9E3779B97F4A7C15)``.
* ``x`` is cut into four 16-bit fields; their sum minus its mean
  (``4 * 65535 / 2``) is an integer in [-131070, 131070] (Irwin-Hall of four
  uniform 16-bit integers), exactly representable in fp32.  Multiplying by the
  fp32 constant ``IH4_SCALE`` (1/std of that sum) gives an approximately
  standard-normal fp32 value bounded by +-sqrt(12) = 3.46.
* A code is ``fp16_rn(fp32_rn(normal * spectrum[j]))`` with ``spectrum`` an
  fp32 table.  Only IEEE round-to-nearest fp32 multiplies and an RN fp32->fp16
  conversion are involved, so host and device results are bit-identical.
"""
from __future__ import annotations

import numpy as np

GOLDEN = 0x9E3779B97F4A7C15
M1 = 0xBF58476D1CE4E5B9
M2 = 0x94D049BB133111EB
MASK64 = (1 << 64) - 1

# 1/std of the sum of four independent uniform integers on [0, 65535]:
# var = 4 * (65536**2 - 1) / 12.
IH4_SCALE = np.float32(1.0 / np.sqrt(4.0 * (65536.0 ** 2 - 1.0) / 12.0))
IH4_CENTER = 2 * 65535  # mean of the four-field sum


def mix64_int(z: int) -> int:
    """SplitMix64 finaliser on a Python int (mod 2**64)."""
    z &= MASK64
    z ^= z >> 30
    z = (z * M1) & MASK64
    z ^= z >> 27
    z = (z * M2) & MASK64
    z ^= z >> 31
    return z


def stream_key(*ids: int) -> int:
    """64-bit stream key from a tuple of small non-negative integers.

    Folds each id through the finaliser so that nearby tuples give unrelated
    streams.  Pure host-side integer work; the device generator receives the
    resulting key as a kernel argument.
    """
    s = 0x5DEECE66D
    for v in ids:
        s = mix64_int(s ^ ((int(v) + GOLDEN) & MASK64))
    return s


def _mix64_arr(z: np.ndarray) -> np.ndarray:
    z = z ^ (z >> np.uint64(30))
    z = z * np.uint64(M1)
    z = z ^ (z >> np.uint64(27))
    z = z * np.uint64(M2)
    z = z ^ (z >> np.uint64(31))
    return z


def normal_f32(key: int, n: int, offset: int = 0) -> np.ndarray:
    """Elements ``offset .. offset+n-1`` of stream ``key`` as fp32 ~N(0,1)."""
    with np.errstate(over="ignore"):
        i = np.arange(offset + 1, offset + n + 1, dtype=np.uint64)
        x = np.uint64(key) + i * np.uint64(GOLDEN)
        z = _mix64_arr(x)
    m16 = np.uint64(0xFFFF)
    s = ((z & m16) + ((z >> np.uint64(16)) & m16)
         + ((z >> np.uint64(32)) & m16) + (z >> np.uint64(48)))
    c = s.astype(np.int64) - IH4_CENTER
    return c.astype(np.float32) * IH4_SCALE


def spectrum_f32(n: int) -> np.ndarray:
    """Decaying spectrum s_i = i**-0.5 (i = 1..n), computed in fp64, stored fp32."""
    i = np.arange(1, n + 1, dtype=np.float64)
    return (i ** -0.5).astype(np.float32)


def codes_f16(key: int, n_rows: int, row_len: int, spectrum: np.ndarray | None,
              row_offset: int = 0) -> np.ndarray:
    """``[n_rows][row_len]`` fp16 codes: ``fp16(normal * spectrum[j % len])``.

    ``spectrum`` (fp32) is tiled along the row when shorter than ``row_len``
    (e.g. one K-rank spectrum repeated for every head).  ``None`` means all
    ones, i.e. plain fp16 ~N(0,1) draws.
    """
    z = normal_f32(key, n_rows * row_len, offset=row_offset * row_len)
    z = z.reshape(n_rows, row_len)
    if spectrum is not None:
        spec = np.asarray(spectrum, dtype=np.float32)
        reps = row_len // spec.shape[0]
        assert reps * spec.shape[0] == row_len
        z = z * np.tile(spec, reps)[None, :]
    return z.astype(np.float16)


def orthonormal_f64(seed: int, rows: int, cols: int) -> np.ndarray:
    """``rows x cols`` matrix with orthonormal columns: Q of a seeded Gaussian's QR."""
    g = np.random.default_rng(seed).standard_normal((rows, cols))
    q, r = np.linalg.qr(g)
    # Fix the sign convention so that diag(R) > 0 (unique Q).
    q = q * np.sign(np.diag(r))[None, :]
    return q
