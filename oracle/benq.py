"""BenQ 6-bit per-row lookup-table layer: CPU oracle (test infrastructure only).

Source: "Qwen3.8-27B -- BenQ 6-bit" model card, section "What BenQ stores".
Each weight is a 6-bit code (1 sign bit + 5 magnitude-tier bits) that indexes
its output row's own table of 64 signed bf16 magnitudes (32 negative ascending,
then 32 positive); decoding is exactly ``lut.gather(1, codes)``.  The card's
closing "Requires ~28 GB ... packing to 6-bit would bring this to ~21 GB"
remark is made concrete as 4 codes per 3 bytes: code k of a row is bits
[6k, 6k+6) of that row's little-endian bitstream (bit q = bit q%8 of byte q//8).

Shapes: W is N x K (out x in), x is B x K, y is B x N, y[b,n] = sum_k W[n,k] x[b,k].
"""
from __future__ import annotations

import numpy as np


def bf16_to_f32(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns -> float32 (exact: a bf16 is the top half of an fp32)."""
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def unpack_codes(packed: np.ndarray, K: int) -> np.ndarray:
    """Codes [N, K] (int64) from packed rows [N, >= 3K/4] bytes.

    Bits are expanded with numpy's little-endian unpack, grouped in sixes and
    read least significant bit first -- the bitstream definition, nothing more.
    """
    packed = np.ascontiguousarray(packed, dtype=np.uint8)
    N = packed.shape[0]
    nbytes = 6 * K // 8
    bits = np.unpackbits(packed[:, :nbytes], axis=1, bitorder="little")     # [N, 6K]
    fields = bits.reshape(N, K, 6).astype(np.int64)
    weights = np.array([1, 2, 4, 8, 16, 32], dtype=np.int64)
    return fields @ weights


def dequant_bits(packed: np.ndarray, lut_bits: np.ndarray, K: int) -> np.ndarray:
    """W as bf16 bit patterns [N, K]: W[n, k] = lut[n, code[n, k]] (the gather)."""
    codes = unpack_codes(packed, K)
    return np.take_along_axis(np.asarray(lut_bits, dtype=np.uint16), codes, axis=1)


def dequant(packed: np.ndarray, lut_bits: np.ndarray, K: int) -> np.ndarray:
    """W as float32 [N, K]."""
    return bf16_to_f32(dequant_bits(packed, lut_bits, K))


def linear(packed: np.ndarray, lut_bits: np.ndarray, x_bits: np.ndarray, K: int,
           rows: np.ndarray | None = None) -> np.ndarray:
    """y = x W^T in fp64, shape [B, N] (or [B, len(rows)] for a row subset).

    W is materialised (bf16 -> fp32, exact), then contracted in fp64: every
    product of two bf16 values is exact in fp64.
    """
    if rows is not None:
        rows = np.asarray(rows)
        packed = np.asarray(packed)[rows]
        lut_bits = np.asarray(lut_bits)[rows]
    W = dequant(packed, lut_bits, K).astype(np.float64)
    x = bf16_to_f32(x_bits).astype(np.float64).reshape(-1, K)
    return x @ W.T


# ---------------------------------------------------------------------------- gated MLP (gate, up)
# The card's model family computes its MLP as down(silu(gate(x)) * up(x)); the pages do not print
# it, so this is the plain definition of that gate: silu(v) = v * sigmoid(v) = v / (1 + e^-v).

def silu(v: np.ndarray) -> np.ndarray:
    """v / (1 + exp(-v)) in fp64, written in a form that does not overflow for large |v|."""
    v = np.asarray(v, dtype=np.float64)
    e = np.exp(-np.abs(v))                      # in (0, 1]
    sig = np.where(v >= 0, 1.0 / (1.0 + e), e / (1.0 + e))
    return v * sig


def mlp_gate_up(packed_g: np.ndarray, lut_g: np.ndarray, packed_u: np.ndarray, lut_u: np.ndarray,
                x_bits: np.ndarray, K: int, rows: np.ndarray | None = None) -> np.ndarray:
    """h = silu(x W_g^T) * (x W_u^T) in fp64, shape [B, N] (or [B, len(rows)]): both projections as
    ``linear``, the gate and the product taken in fp64."""
    g = linear(packed_g, lut_g, x_bits, K, rows)
    u = linear(packed_u, lut_u, x_bits, K, rows)
    return silu(g) * u


# ----------------------------------------------------------------------------------------- encoder
# Source: the BenQ card, sections "Why equal-width shells" and the calibration table note: 32
# magnitude tiers placed as equal-width shells of each row's range, a table refined Lloyd-style,
# and nearest-level assignment (the uncalibrated path; GPTQ needs calibration data).

def _bf16_rne_of_f32(v32: np.ndarray) -> np.ndarray:
    """bf16 bit patterns of float32 values, round to nearest even (finite inputs)."""
    u = np.asarray(v32, dtype=np.float32).view(np.uint32).astype(np.uint64)
    return ((u + 0x7FFF + ((u >> 16) & 1)) >> 16).astype(np.uint16)


def _shell_levels(a: np.ndarray, tier: np.ndarray, prev: np.ndarray) -> np.ndarray:
    """fp64 mean of the magnitudes in each tier (prev where a tier is empty), rounded fp64 -> fp32 -> bf16,
    returned as float64 values of the bf16 levels.  a, tier: [K]; prev: [32] float64."""
    cnt = np.bincount(tier, minlength=32)
    tot = np.bincount(tier, weights=a, minlength=32)
    mean = np.where(cnt > 0, tot / np.maximum(cnt, 1), prev)
    return bf16_to_f32(_bf16_rne_of_f32(mean.astype(np.float32))).astype(np.float64)


def _nearest(a: np.ndarray, levels: np.ndarray) -> np.ndarray:
    """Index of the level nearest to each magnitude; on an exact tie the lower index."""
    d = np.abs(a[:, None] - levels[None, :])                  # exact: differences of bf16 values in fp64
    return np.argmin(d, axis=1)                               # argmin keeps the first (lower) index


def encode(w_bits: np.ndarray, lloyd_iters: int = 0) -> tuple[np.ndarray, np.ndarray]:
    """BenQ codes (packed 4 per 3 bytes, [N, 3K/4]) and tables (bf16 bits [N, 64]) of a bf16 matrix [N, K].

    Per row: shell width D = max|w| / 32; tier t = min(floor(|w| / D), 31); level t = fp64 mean of the
    magnitudes in tier t (shell midpoint (t + 1/2) D when empty), rounded fp64 -> fp32 -> bf16; then
    lloyd_iters rounds of (assign every magnitude to its nearest level, lower tier on a tie; level =
    fp64 mean of its members, unchanged when it has none, rounded the same way).  Codes: nearest level
    t, written 32 + t for w >= 0 (zero included) and 31 - t for w < 0; table [-L31 .. -L0, L0 .. L31].
    An all-zero row gets zero levels and codes 32.
    """
    w = bf16_to_f32(np.asarray(w_bits, dtype=np.uint16)).astype(np.float64)
    N, K = w.shape
    if K % 4:
        raise ValueError("K must be a multiple of 4")
    codes = np.empty((N, K), dtype=np.uint8)
    lut = np.empty((N, 64), dtype=np.uint16)
    for n in range(N):
        a = np.abs(w[n])
        amax = a.max()
        if amax == 0.0:
            levels = np.zeros(32)
            t = np.zeros(K, dtype=np.int64)
        else:
            d = amax / 32.0
            tier = np.minimum(np.floor(a / d), 31).astype(np.int64)
            levels = _shell_levels(a, tier, (np.arange(32) + 0.5) * d)
            for _ in range(lloyd_iters):
                levels = _shell_levels(a, _nearest(a, levels), levels)
            t = _nearest(a, levels)
        neg = w[n] < 0
        codes[n] = np.where(neg, 31 - t, 32 + t)
        lv = _bf16_rne_of_f32(levels.astype(np.float32))
        lut[n, 32:] = lv
        lut[n, :32] = lv[::-1] | np.uint16(0x8000)
    return pack(codes), lut


def pack(codes: np.ndarray) -> np.ndarray:
    """Packs codes [N, K] (0..63) into rows of 3K/4 bytes: code k is bits [6k, 6k + 6) of the row's
    little-endian bitstream (bit q = bit q % 8 of byte q // 8)."""
    codes = np.asarray(codes, dtype=np.uint8)
    N, K = codes.shape
    bits = np.unpackbits(codes[:, :, None], axis=2, bitorder="little")[:, :, :6]     # [N, K, 6] LSB first
    return np.packbits(bits.reshape(N, 6 * K), axis=1, bitorder="little")
