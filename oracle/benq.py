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
