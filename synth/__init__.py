"""Seeded synthetic inputs for the BenQ and MDBF quantized linear layers.

This module only *makes inputs*: random activations, BenQ weight tables and
codes, and MDBF sign matrices and envelopes.  It holds none of the forward
pass (no decode, no contraction); both the CUDA path and the CPU oracle take
its outputs as plain arrays.

Determinism: every tensor comes from ``numpy.random.Generator(PCG64(...))``
seeded from ``SeedSequence([seed, chunk])`` over fixed 256-row chunks, so the
bytes do not depend on how many threads build them.

Encoder rules (BenQ 6-bit model card, "What BenQ stores" and "Why equal-width
shells"): each output row gets 32 equal-width magnitude shells over
[0, max|w|]; a shell's level is the mean |w| of the weights that fall in it
(the shell midpoint when it is empty), rounded to bf16; the row's 64-entry
table holds the 32 levels negated in ascending value order, then the 32
positive levels; each weight takes the nearest level of its sign (the lower
tier on an exact distance tie, w == 0 counted as non-negative).  Codes are
packed 4 per 3 bytes as a little-endian bitstream: code j of a row occupies
bits [6j, 6j+6), bit q of the stream being bit q%8 of byte q//8.

MDBF (OneComp MDBF page, "Algorithm"): sign matrices are Bernoulli(1/2), one
bit per element packed LSB-first along each row, bit 1 meaning +1; the bytes
past the last column of a row (padding up to the row stride) hold random
garbage on purpose so that consumers are seen to ignore them.  Envelopes are
|N(0,1)| * 0.05 rounded to fp16.
"""
from __future__ import annotations

import os
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass

import numpy as np

CHUNK_ROWS = 256


def _rng(seed: int, chunk: int = 0) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([int(seed), int(chunk)])))


def _threads() -> int:
    return max(1, min(16, os.cpu_count() or 1))


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round float32 values to bf16 (round-to-nearest-even); returns uint16 bit patterns."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
    u = u + 0x7FFF + ((u >> 16) & 1)
    return (u >> 16).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def activations(B: int, K: int, seed: int) -> np.ndarray:
    """x ~ N(0,1) drawn in fp32, rounded to bf16.  Returns uint16 bits [B, K]."""
    x = _rng(seed).standard_normal((B, K), dtype=np.float32)
    return f32_to_bf16_bits(x)


# ----------------------------------------------------------------------------------------------
# BenQ
# ----------------------------------------------------------------------------------------------

@dataclass
class BenQWeights:
    codes: np.ndarray   # uint8 [N, 3K/4], packed 4 codes / 3 bytes
    lut: np.ndarray     # uint16 (bf16 bits) [N, 64]
    N: int
    K: int


def pack_codes(codes: np.ndarray) -> np.ndarray:
    """Pack uint8 codes [N, K] (values < 64, K % 4 == 0) into uint8 [N, 3K/4]."""
    N, K = codes.shape
    if K % 4:
        raise ValueError("K must be a multiple of 4")
    c = codes.reshape(N, K // 4, 4).astype(np.uint32)
    v = c[..., 0] | (c[..., 1] << 6) | (c[..., 2] << 12) | (c[..., 3] << 18)
    out = np.empty((N, K // 4, 3), dtype=np.uint8)
    out[..., 0] = v & 0xFF
    out[..., 1] = (v >> 8) & 0xFF
    out[..., 2] = (v >> 16) & 0xFF
    return out.reshape(N, 3 * K // 4)


def _benq_chunk(seed: int, chunk: int, rows: int, K: int):
    rng = _rng(seed, chunk)
    sigma = rng.uniform(0.01, 0.03, size=rows).astype(np.float32)
    w = rng.standard_normal((rows, K), dtype=np.float32) * sigma[:, None]
    a = np.abs(w)
    amax = a.max(axis=1).astype(np.float64)
    delta = amax / 32.0
    safe = np.where(delta > 0, delta, 1.0)
    band = np.minimum(np.floor(a / safe[:, None]), 31).astype(np.int64)      # [rows, K]
    flat = band + 32 * np.arange(rows, dtype=np.int64)[:, None]
    cnt = np.bincount(flat.ravel(), minlength=32 * rows).reshape(rows, 32)
    tot = np.bincount(flat.ravel(), weights=a.ravel().astype(np.float64),
                      minlength=32 * rows).reshape(rows, 32)
    mid = (np.arange(32)[None, :] + 0.5) * delta[:, None]
    level = np.where(cnt > 0, tot / np.maximum(cnt, 1), mid)                   # fp64
    lv_bits = f32_to_bf16_bits(level.astype(np.float32))                         # [rows, 32]
    lv = bf16_bits_to_f32(lv_bits).astype(np.float64)
    # nearest bf16 level; candidates band-2 .. band+2 suffice because every pre-rounding
    # level lies inside its own shell and bf16 rounding moves it by far less than a shell width
    a64 = a.astype(np.float64)
    best = np.clip(band - 2, 0, 31)
    bestd = np.abs(a64 - np.take_along_axis(lv, best, axis=1))
    for off in (-1, 0, 1, 2):
        cand = np.clip(band + off, 0, 31)
        d = np.abs(a64 - np.take_along_axis(lv, cand, axis=1))
        better = (d < bestd) | ((d == bestd) & (cand < best))
        best = np.where(better, cand, best)
        bestd = np.where(better, d, bestd)
    neg = np.signbit(w) & (w != 0)
    codes = np.where(neg, 31 - best, 32 + best).astype(np.uint8)
    lut = np.empty((rows, 64), dtype=np.uint16)
    lut[:, 32:] = lv_bits
    lut[:, :32] = lv_bits[:, ::-1] | np.uint16(0x8000)
    return pack_codes(codes), lut


def benq_weights(N: int, K: int, seed: int, threads: int | None = None) -> BenQWeights:
    """BenQ weights of an N x K (out x in) layer, built by the shell encoder described above."""
    if K % 4:
        raise ValueError("K must be a multiple of 4")
    nchunks = (N + CHUNK_ROWS - 1) // CHUNK_ROWS
    codes = np.empty((N, 3 * K // 4), dtype=np.uint8)
    lut = np.empty((N, 64), dtype=np.uint16)

    def work(c):
        r0 = c * CHUNK_ROWS
        rows = min(CHUNK_ROWS, N - r0)
        pc, pl = _benq_chunk(seed, c, rows, K)
        codes[r0:r0 + rows] = pc
        lut[r0:r0 + rows] = pl

    with ThreadPoolExecutor(threads or _threads()) as ex:
        list(ex.map(work, range(nchunks)))
    return BenQWeights(codes=codes, lut=lut, N=N, K=K)


# ----------------------------------------------------------------------------------------------
# MDBF
# ----------------------------------------------------------------------------------------------

def default_ld(cols: int) -> int:
    """Row stride in bytes for a packed sign matrix: ceil(cols/8) rounded up to 16."""
    return ((cols + 7) // 8 + 15) // 16 * 16


@dataclass
class MDBFPath:
    S_A: np.ndarray     # uint8 [n, ldSA]  packed signs of the n x r matrix
    S_B: np.ndarray     # uint8 [r, ldSB]  packed signs of the r x m matrix
    A_amp: np.ndarray   # uint16 (fp16 bits) [n, l]
    B_amp: np.ndarray   # uint16 (fp16 bits) [m, l]
    Q_U: np.ndarray     # uint16 (fp16 bits) [r, l]
    Q_V: np.ndarray     # uint16 (fp16 bits) [r, l]


def pack_signs(bits: np.ndarray, ld: int, rng: np.random.Generator | None = None) -> np.ndarray:
    """Pack a {0,1} matrix [rows, cols] LSB-first along rows into [rows, ld] bytes.

    Bits past ``cols`` and bytes past ceil(cols/8) are filled from ``rng`` (garbage) when given."""
    rows, cols = bits.shape
    nb = (cols + 7) // 8
    if ld < nb:
        raise ValueError("row stride too small")
    out = np.zeros((rows, ld), dtype=np.uint8)
    if rng is not None:
        out[:] = rng.integers(0, 256, size=(rows, ld), dtype=np.uint8)
    packed = np.packbits(bits.astype(np.uint8), axis=1, bitorder="little")
    if cols % 8:
        keep = np.uint8((1 << (cols % 8)) - 1)
        packed[:, -1] = (packed[:, -1] & keep) | (out[:, nb - 1] & ~keep)
    out[:, :nb] = packed
    return out


def _envelope(rng: np.random.Generator, shape) -> np.ndarray:
    v = np.abs(rng.standard_normal(shape, dtype=np.float32)) * np.float32(0.05)
    return v.astype(np.float16).view(np.uint16)


def _sign_rows(seed: int, tag: int, rows: int, cols: int, ld: int, threads: int | None) -> np.ndarray:
    out = np.empty((rows, ld), dtype=np.uint8)
    nchunks = (rows + CHUNK_ROWS - 1) // CHUNK_ROWS

    def work(c):
        r0 = c * CHUNK_ROWS
        rr = min(CHUNK_ROWS, rows - r0)
        rng = _rng(seed * 16 + tag, c)
        bits = rng.integers(0, 2, size=(rr, cols), dtype=np.uint8)
        out[r0:r0 + rr] = pack_signs(bits, ld, rng)

    with ThreadPoolExecutor(threads or _threads()) as ex:
        list(ex.map(work, range(nchunks)))
    return out


def mdbf_path(n: int, m: int, r: int, l: int, seed: int, ldSA: int | None = None,
              ldSB: int | None = None, threads: int | None = None) -> MDBFPath:
    """One MDBF path of an n x m (out x in) layer with rank r and envelope rank l."""
    ldSA = ldSA or default_ld(r)
    ldSB = ldSB or default_ld(m)
    rng = _rng(seed * 16 + 0)
    A = _envelope(rng, (n, l))
    Bm = _envelope(rng, (m, l))
    QU = _envelope(rng, (r, l))
    QV = _envelope(rng, (r, l))
    SA = _sign_rows(seed, 1, n, r, ldSA, threads)
    SB = _sign_rows(seed, 2, r, m, ldSB, threads)
    return MDBFPath(S_A=SA, S_B=SB, A_amp=A, B_amp=Bm, Q_U=QU, Q_V=QV)


def mdbf_paths(P: int, n: int, m: int, r: int, l: int, seed: int, **kw) -> list[MDBFPath]:
    return [mdbf_path(n, m, r, l, seed * 8 + p, **kw) for p in range(P)]
