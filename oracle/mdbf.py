"""MDBF (multi-envelope double binary factorization) layer: CPU oracle (test infrastructure only).

Source: "MDBF (Multi-Envelope Double Binary Factorization)" (OneComp docs),
section "Algorithm":

    W ~= sum_{p=1..P} F_p G_p,
    F = S_A (.) (A_amp Q_U^T)        (n x r),
    G = S_B (.) (Q_V B_amp^T)        (r x m),

with S_A in {-1,+1}^{n x r}, S_B in {-1,+1}^{r x m} stored one bit per element
packed into uint8, and FP16 envelopes A_amp (n x l), B_amp (m x l), Q_U (r x l),
Q_V (r x l).  W is n x m (out x in) and multiplies x from the right:
y[b, a] = sum_j W[a, j] x[b, j].

Readings where the page is silent (each listed in the design notes):
* packing: bits run least significant first along each row, bit 1 = +1,
  rows padded to a byte stride ``ld``; padding bits are ignored;
* envelopes: E[a,k] = sum_i L[a,i] R[k,i] is formed in fp32, i ascending,
  starting from the first product (fp16 x fp16 products are exact in fp32);
* W: each element is the fp64 sum over p (outer) and k ascending (inner) of
  the exact fp64 products F_p[a,k] G_p[k,j], rounded once to fp32.
"""
from __future__ import annotations

import numpy as np


def f16_to_f32(bits: np.ndarray) -> np.ndarray:
    return np.asarray(bits, dtype=np.uint16).view(np.float16).astype(np.float32)


def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def unpack_signs(packed: np.ndarray, cols: int) -> np.ndarray:
    """{-1,+1} int8 matrix [rows, cols] from LSB-first packed bytes [rows, ld]."""
    bits = np.unpackbits(np.ascontiguousarray(packed, dtype=np.uint8), axis=1, bitorder="little")
    return (bits[:, :cols].astype(np.int8) * 2 - 1).astype(np.int8)


def envelope(Lbits: np.ndarray, Rbits: np.ndarray) -> np.ndarray:
    """E = L R^T in fp32 with the sum over the l envelope columns taken in ascending order."""
    L = f16_to_f32(Lbits)
    R = f16_to_f32(Rbits)
    E = L[:, 0][:, None] * R[:, 0][None, :]
    for i in range(1, L.shape[1]):
        E = E + L[:, i][:, None] * R[:, i][None, :]
    return E.astype(np.float32)


def factors(path, n: int, m: int, r: int):
    """(F, G) of one path as float32: F = S_A (.) (A_amp Q_U^T), G = S_B (.) (Q_V B_amp^T)."""
    SA = unpack_signs(path.S_A, r)
    SB = unpack_signs(path.S_B, m)
    F = (SA * envelope(path.A_amp, path.Q_U)).astype(np.float32)
    G = (SB * envelope(path.Q_V, path.B_amp)).astype(np.float32)
    assert F.shape == (n, r) and G.shape == (r, m)
    return F, G


def dequant(paths, n: int, m: int, r: int, return_f64: bool = False) -> np.ndarray:
    """W [n, m]: fp64 accumulation over p then k ascending, rounded to fp32.

    O(P r n m) numpy work; meant for small and medium shapes."""
    acc = np.zeros((n, m), dtype=np.float64)
    for path in paths:
        F, G = factors(path, n, m, r)
        F64 = F.astype(np.float64)
        G64 = G.astype(np.float64)
        for k in range(r):
            acc += F64[:, k][:, None] * G64[k][None, :]
    return acc if return_f64 else acc.astype(np.float32)


def dequant_at(paths, r: int, m: int, a_idx: np.ndarray, j_idx: np.ndarray) -> np.ndarray:
    """W[a_idx[t], j_idx[t]] for sampled coordinates, same arithmetic as ``dequant``."""
    a_idx = np.asarray(a_idx)
    j_idx = np.asarray(j_idx)
    acc = np.zeros(a_idx.shape[0], dtype=np.float64)
    for path in paths:
        SA = unpack_signs(path.S_A[a_idx], r)                             # [T, r]
        SBt = unpack_signs(path.S_B, m)[:, j_idx].T                        # [T, r]
        A = f16_to_f32(path.A_amp)[a_idx]                                   # [T, l]
        Bm = f16_to_f32(path.B_amp)[j_idx]                                  # [T, l]
        QU = f16_to_f32(path.Q_U)                                           # [r, l]
        QV = f16_to_f32(path.Q_V)
        l = QU.shape[1]
        EA = A[:, 0][:, None] * QU[:, 0][None, :]
        EB = QV[:, 0][None, :] * Bm[:, 0][:, None]
        for i in range(1, l):
            EA = EA + A[:, i][:, None] * QU[:, i][None, :]
            EB = EB + QV[:, i][None, :] * Bm[:, i][:, None]
        F = (SA * EA).astype(np.float32).astype(np.float64)
        G = (SBt * EB).astype(np.float32).astype(np.float64)
        prod = F * G                                                        # exact in fp64
        for k in range(r):
            acc += prod[:, k]
    return acc.astype(np.float32)


def linear_dense(paths, n: int, m: int, r: int, x_bits: np.ndarray) -> np.ndarray:
    """y [B, n] in fp64 from the materialised fp32 W (small and medium shapes)."""
    W = dequant(paths, n, m, r).astype(np.float64)
    x = bf16_to_f64(x_bits).reshape(-1, m)
    return x @ W.T


def linear_factored(paths, n: int, m: int, r: int, x_bits: np.ndarray,
                    rows: np.ndarray | None = None) -> np.ndarray:
    """y [B, n] (or [B, len(rows)]) in fp64 through the envelopes, any size.

    Expands F G x without forming W:
      z_i = B_amp[:, i] * x,  u_i = S_B z_i,  t = sum_i Q_V[:, i] * u_i,
      w_i = Q_U[:, i] * t,    v_i = S_A w_i,  y = sum_p sum_i A_amp[:, i] * v_i.
    All in fp64 from the stored fp16 / bf16 values (no intermediate rounding),
    so it equals the exact y up to fp64 rounding.
    """
    x = bf16_to_f64(x_bits).reshape(-1, m)                      # [B, m]
    nout = n if rows is None else len(rows)
    y = np.zeros((x.shape[0], nout), dtype=np.float64)
    for path in paths:
        SB = unpack_signs(path.S_B, m).astype(np.float64)       # [r, m]
        SA = unpack_signs(path.S_A if rows is None else path.S_A[rows], r).astype(np.float64)
        A = f16_to_f32(path.A_amp).astype(np.float64)
        if rows is not None:
            A = A[rows]
        Bm = f16_to_f32(path.B_amp).astype(np.float64)
        QU = f16_to_f32(path.Q_U).astype(np.float64)
        QV = f16_to_f32(path.Q_V).astype(np.float64)
        l = QU.shape[1]
        t = np.zeros((r, x.shape[0]), dtype=np.float64)
        for i in range(l):
            z = Bm[:, i][:, None] * x.T                             # [m, B]
            t += QV[:, i][:, None] * (SB @ z)                       # [r, B]
        for i in range(l):
            w = QU[:, i][:, None] * t                               # [r, B]
            y += (A[:, i][:, None] * (SA @ w)).T
    return y
