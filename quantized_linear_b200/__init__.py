"""Python binding of libqlinear.so: BenQ 6-bit and MDBF weight-only quantized linear layers on B200.

Argument marshalling only: every function here takes torch tensors (device
memory the caller owns), checks dtypes and shapes, passes raw pointers and the
current CUDA stream to the C ABI declared in ``include/qlinear.h``, and raises
``QLinearError`` on a non-OK status.  All arithmetic runs in the library's
sm_100a kernels; there is no fallback.  If ``libqlinear.so`` is missing, import
fails -- build it with ``python -m quantized_linear_b200.build``.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libqlinear.so")

_lib = None

QL_OK, QL_ERR_INVALID_ARG, QL_ERR_UNSUPPORTED, QL_ERR_ALIGNMENT, QL_ERR_CUDA, QL_ERR_TIMEOUT = range(6)
QL_OUT_F32, QL_OUT_BF16 = 0, 1
STATUS_NAMES = {0: "QL_OK", 1: "QL_ERR_INVALID_ARG", 2: "QL_ERR_UNSUPPORTED", 3: "QL_ERR_ALIGNMENT",
                4: "QL_ERR_CUDA", 5: "QL_ERR_TIMEOUT"}

_vp, _i, _sz, _d = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t, ctypes.c_double


class BenQLayerC(ctypes.Structure):
    _fields_ = [("codes", _vp), ("lut", _vp), ("y", _vp), ("N", _i)]


class MDBFPathC(ctypes.Structure):
    _fields_ = [("S_A", _vp), ("S_B", _vp), ("ldSA", _sz), ("ldSB", _sz),
                ("A_amp", _vp), ("B_amp", _vp), ("Q_U", _vp), ("Q_V", _vp)]


_SIGNATURES = {
    "benq_linear": (_i, [_vp, _vp, _vp, _vp, _i, _i, _i, _i, _vp]),
    "benq_linear_ws": (_i, [_vp, _vp, _vp, _vp, _i, _i, _i, _i, _vp, _sz, _vp]),
    "benq_linear_workspace_bytes": (_sz, [_i, _i, _i]),
    "benq_linear_multi": (_i, [ctypes.POINTER(BenQLayerC), _i, _vp, _i, _i, _i, _vp]),
    "benq_mlp_gate_up": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _vp, _sz, _vp]),
    "benq_mlp_workspace_bytes": (_sz, [_i, _i, _i]),
    "benq_encode": (_i, [_vp, _vp, _vp, _i, _i, _i, _vp]),
    "benq_dequant_debug": (_i, [_vp, _vp, _vp, _i, _i, _vp]),
    "benq_bits_per_weight": (_d, [_i]),
    "mdbf_workspace_bytes": (_sz, [_i, _i, _i, _i, _i, _i]),
    "mdbf_linear": (_i, [ctypes.POINTER(MDBFPathC), _i, _i, _i, _i, _i, _vp, _vp, _i, _i, _vp, _sz, _vp]),
    "mdbf_linear_multi": (_i, [ctypes.POINTER(MDBFPathC), _i, _i, _i, _i, _i, _i, _vp, ctypes.POINTER(_vp), _i, _i,
                               _vp, _sz, _vp]),
    "mdbf_dequant_debug": (_i, [ctypes.POINTER(MDBFPathC), _i, _i, _i, _i, _i, _vp, _vp, _vp, _vp]),
    "mdbf_linear_noalloc": (_i, [ctypes.POINTER(MDBFPathC), _i, _i, _i, _i, _i, _vp, _vp, _i, _i, _vp]),
    "mdbf_noalloc_scratch_bytes": (_sz, []),
    "mdbf_effective_bits": (_d, [_i, _i, _i, _i, _i, _i]),
    "mdbf_select_rank": (_i, [_i, _i, _i, _i, _i, _d, ctypes.POINTER(_i), ctypes.POINTER(_i)]),
    "ql_last_error": (ctypes.c_char_p, []),
    "ql_check": (_i, [_vp]),
    "ql_set_pdl": (_i, [_i]),
    "ql_selftest_timeout": (_i, [_vp]),
}


def lib() -> ctypes.CDLL:
    """The loaded libqlinear.so (loaded on first use; raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: run `python -m quantized_linear_b200.build` first")
        handle = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGNATURES.items():
            f = getattr(handle, name)
            f.restype = res
            f.argtypes = args
        _lib = handle
    return _lib


def _c(name):
    return getattr(lib(), name)

EXPORTS = ["benq_linear", "benq_linear_ws", "benq_linear_workspace_bytes", "benq_linear_multi", "benq_mlp_gate_up",
           "benq_mlp_workspace_bytes", "benq_encode", "benq_dequant_debug", "benq_bits_per_weight", "mdbf_workspace_bytes", "mdbf_linear",
           "mdbf_linear_multi", "mdbf_linear_noalloc", "mdbf_noalloc_scratch_bytes", "mdbf_dequant_debug", "mdbf_effective_bits",
           "mdbf_select_rank", "ql_last_error", "ql_check", "ql_set_pdl", "ql_selftest_timeout"]


class QLinearError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {msg}")
        self.status = status


def _check(status: int):
    if status != QL_OK:
        raise QLinearError(status, (_c("ql_last_error")() or b"").decode())


def _ptr(t):
    """Device address of a tensor argument (None and plain integers pass through unchanged).

    The library takes device pointers on the current device; a host tensor or one on another GPU
    is refused here, before any launch could read it as a device address."""
    if t is None:
        return None
    if isinstance(t, int):
        return t
    d = t.get_device()
    if d < 0:
        raise ValueError("tensor arguments must be CUDA tensors (got one on the host)")
    if d != torch.cuda.current_device():
        raise ValueError(f"tensor arguments must be on the current device cuda:{torch.cuda.current_device()}, "
                         f"got one on {t.device}")
    return t.data_ptr()


# the current stream's handle without building a torch.cuda.Stream object (a few microseconds per call)
_raw_stream = getattr(torch._C, "_cuda_getCurrentRawStream", None)


def _stream(stream=None):
    if stream is None:
        if _raw_stream is not None:
            return _raw_stream(torch.cuda.current_device())
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else stream


def _want(t, dtype, what):
    if t.dtype != dtype:
        raise TypeError(f"{what} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{what} must be contiguous")


def _ydt(y):
    if y.dtype == torch.float32:
        return QL_OUT_F32
    if y.dtype == torch.bfloat16:
        return QL_OUT_BF16
    raise TypeError("y must be float32 or bfloat16")


# ----------------------------------------------------------------------------------------------- BenQ

def benq_linear(codes, lut, x, y, stream=None, workspace=None):
    """y[B, N] = x[B, K] @ W^T with W[n, k] = lut[n, code(n, k)].

    codes uint8 [N, 3K/4]; lut bf16 (or int16 bit patterns) [N, 64]; x bf16 [B, K];
    y float32 or bf16 [B, N] (overwritten).  With a uint8 device `workspace` of at least
    benq_linear_workspace_bytes(B, N, K) bytes the GEMM splits its last wave along K
    (benq_linear_ws)."""
    N = codes.shape[0]
    B, K = x.shape
    _want(codes, torch.uint8, "codes")
    if codes.shape[1] != 3 * K // 4:
        raise ValueError("codes must be [N, 3K/4]")
    if lut.dtype not in (torch.bfloat16, torch.int16) or tuple(lut.shape) != (N, 64) or not lut.is_contiguous():
        raise TypeError("lut must be a contiguous bf16 [N, 64] tensor")
    _want(x, torch.bfloat16, "x")
    if tuple(y.shape) != (B, N) or not y.is_contiguous():
        raise ValueError("y must be contiguous [B, N]")
    if workspace is None:
        _check(_c("benq_linear")(_ptr(codes), _ptr(lut), _ptr(x), _ptr(y), _ydt(y), B, N, K, _stream(stream)))
    else:
        nbytes = workspace.numel() * workspace.element_size()
        _check(_c("benq_linear_ws")(_ptr(codes), _ptr(lut), _ptr(x), _ptr(y), _ydt(y), B, N, K, _ptr(workspace),
                                    nbytes, _stream(stream)))
    return y


def benq_linear_multi(layers, x, stream=None):
    """y_s = x @ W_s^T for several BenQ layers of the same K that read the same x (at batch 1 in one
    launch).  layers: list of (codes, lut, y) with codes uint8 [N_s, 3K/4], lut bf16 [N_s, 64] and y
    float32 or bf16 [B, N_s] (all the same dtype, overwritten)."""
    B, K = x.shape
    _want(x, torch.bfloat16, "x")
    if not 1 <= len(layers) <= 4:
        raise ValueError("benq_linear_multi takes 1 to 4 layers")
    ydt = _ydt(layers[0][2])
    arr = (BenQLayerC * len(layers))()
    for i, (codes, lut, y) in enumerate(layers):
        N = codes.shape[0]
        _want(codes, torch.uint8, "codes")
        if codes.shape[1] != 3 * K // 4:
            raise ValueError("codes must be [N, 3K/4]")
        if lut.dtype not in (torch.bfloat16, torch.int16) or tuple(lut.shape) != (N, 64) or not lut.is_contiguous():
            raise TypeError("lut must be a contiguous bf16 [N, 64] tensor")
        if tuple(y.shape) != (B, N) or not y.is_contiguous() or _ydt(y) != ydt:
            raise ValueError("each y must be contiguous [B, N] of the first y's dtype")
        arr[i] = BenQLayerC(_ptr(codes), _ptr(lut), _ptr(y), N)
    _check(_c("benq_linear_multi")(arr, len(layers), _ptr(x), ydt, B, K, _stream(stream)))
    return [y for _, _, y in layers]


def benq_linear_workspace_bytes(B: int, N: int, K: int) -> int:
    """Bytes of workspace the GEMM's split last wave uses for these sizes on the current device."""
    return int(_c("benq_linear_workspace_bytes")(B, N, K))


def benq_mlp_gate_up(codes_g, lut_g, codes_u, lut_u, x, h, workspace=None, stream=None):
    """h[B, N] = silu(x @ W_g^T) * (x @ W_u^T) for two BenQ layers of the same shape (codes and
    tables as for benq_linear); h float32 or bf16 [B, N] (overwritten).  `workspace`: uint8 device
    tensor of at least benq_mlp_workspace_bytes(B, N, K) bytes when that is non-zero."""
    N = codes_g.shape[0]
    B, K = x.shape
    for c, l, what in ((codes_g, lut_g, "gate"), (codes_u, lut_u, "up")):
        _want(c, torch.uint8, f"{what} codes")
        if tuple(c.shape) != (N, 3 * K // 4):
            raise ValueError(f"{what} codes must be [N, 3K/4]")
        if l.dtype not in (torch.bfloat16, torch.int16) or tuple(l.shape) != (N, 64) or not l.is_contiguous():
            raise TypeError(f"{what} lut must be a contiguous bf16 [N, 64] tensor")
    _want(x, torch.bfloat16, "x")
    if tuple(h.shape) != (B, N) or not h.is_contiguous():
        raise ValueError("h must be contiguous [B, N]")
    ws, nbytes = (None, 0) if workspace is None else (_ptr(workspace), workspace.numel() * workspace.element_size())
    _check(_c("benq_mlp_gate_up")(_ptr(codes_g), _ptr(lut_g), _ptr(codes_u), _ptr(lut_u), _ptr(x), _ptr(h), _ydt(h),
                                  B, N, K, ws, nbytes, _stream(stream)))
    return h


def benq_mlp_workspace_bytes(B: int, N: int, K: int) -> int:
    """Bytes of workspace benq_mlp_gate_up needs (0 when the fused batch-1 kernel runs)."""
    return int(_c("benq_mlp_workspace_bytes")(B, N, K))


def benq_encode(W, codes, lut, lloyd_iters=0, stream=None):
    """Quantizes W (bf16 [N, K]) to BenQ storage: codes uint8 [N, 3K/4] and lut bf16 [N, 64], both
    overwritten (equal-width shells, member-mean levels, lloyd_iters refinement rounds)."""
    N, K = W.shape
    if W.dtype not in (torch.bfloat16, torch.int16) or not W.is_contiguous():
        raise TypeError("W must be a contiguous bf16 [N, K] tensor")
    _want(codes, torch.uint8, "codes")
    if tuple(codes.shape) != (N, 3 * K // 4):
        raise ValueError("codes must be [N, 3K/4]")
    if lut.dtype not in (torch.bfloat16, torch.int16) or tuple(lut.shape) != (N, 64) or not lut.is_contiguous():
        raise TypeError("lut must be a contiguous bf16 [N, 64] tensor")
    _check(_c("benq_encode")(_ptr(W), _ptr(codes), _ptr(lut), N, K, int(lloyd_iters), _stream(stream)))
    return codes, lut


def benq_dequant_debug(codes, lut, W, stream=None):
    """W[n, k] = lut[n, code(n, k)] as bf16 [N, K]."""
    N, K = W.shape
    if codes.shape != (N, 3 * K // 4):
        raise ValueError("codes must be [N, 3K/4]")
    _check(_c("benq_dequant_debug")(_ptr(codes), _ptr(lut), _ptr(W), N, K, _stream(stream)))
    return W


def benq_bits_per_weight(K: int) -> float:
    return float(_c("benq_bits_per_weight")(int(K)))


# ----------------------------------------------------------------------------------------------- MDBF

def mdbf_paths_c(paths):
    """ctypes array of mdbf_path from a list of dicts / objects with S_A, S_B, A_amp, B_amp, Q_U, Q_V tensors
    (S_A, S_B uint8 [rows, ld]; envelopes fp16 [*, l]), or of entries of such arrays.  The array holds
    device addresses only: the tensors must outlive every call it is passed to.  mdbf_linear and
    mdbf_linear_multi take such arrays in place of the lists, which saves building them per call."""
    arr = (MDBFPathC * len(paths))()
    for i, p in enumerate(paths):
        if isinstance(p, MDBFPathC):   # an entry of an array made by an earlier call
            arr[i] = p
            continue
        g = (lambda k: p[k]) if isinstance(p, dict) else (lambda k: getattr(p, k))
        arr[i] = MDBFPathC(_ptr(g("S_A")), _ptr(g("S_B")), g("S_A").shape[1], g("S_B").shape[1],
                           _ptr(g("A_amp")), _ptr(g("B_amp")), _ptr(g("Q_U")), _ptr(g("Q_V")))
    return arr


def mdbf_workspace_bytes(P, n, m, r, l, B) -> int:
    return int(_c("mdbf_workspace_bytes")(P, n, m, r, l, B))


def mdbf_linear(paths, n, m, r, l, x, y, workspace, stream=None):
    """y[B, n] = x[B, m] @ (sum_p F_p G_p)^T without forming W.  workspace: uint8 CUDA tensor of at least
    mdbf_workspace_bytes(...) bytes, 256-byte aligned."""
    _want(x, torch.bfloat16, "x")
    B = x.shape[0]
    if x.shape[1] != m or tuple(y.shape) != (B, n) or not y.is_contiguous():
        raise ValueError("x must be [B, m] and y [B, n]")
    arr = paths if isinstance(paths, ctypes.Array) else mdbf_paths_c(paths)
    _check(_c("mdbf_linear")(arr, len(arr), n, m, r, l, _ptr(x), _ptr(y), _ydt(y), B, _ptr(workspace),
                        workspace.numel() * workspace.element_size(), _stream(stream)))
    return y


def mdbf_linear_multi(layers, n, m, r, l, x, ys, workspace, stream=None):
    """y_s[B, n] = x[B, m] @ W_s^T for S MDBF layers of the same sizes that read the same x (the gate and
    up projections of an MLP), bit for bit as mdbf_linear gives each; at decode batches the three
    launches cover all layers.  layers: S lists of P paths each (dicts / objects as for mdbf_linear);
    ys: S outputs [B, n] of one dtype; workspace: at least mdbf_workspace_bytes(S * P, n, m, r, l, B)
    bytes."""
    _want(x, torch.bfloat16, "x")
    B = x.shape[0]
    S = len(layers)
    if S != len(ys) or not 1 <= S <= 4:
        raise ValueError("mdbf_linear_multi takes 1 to 4 layers and one output per layer")
    P = len(layers[0])
    if any(len(lp) != P for lp in layers):
        raise ValueError("every layer must have the same number of paths")
    if x.shape[1] != m or any(tuple(y.shape) != (B, n) or not y.is_contiguous() for y in ys):
        raise ValueError("x must be [B, m] and every y [B, n]")
    if any(y.dtype != ys[0].dtype for y in ys):
        raise TypeError("all outputs must have one dtype")
    arr = mdbf_paths_c([p for lp in layers for p in lp])
    yp = (_vp * S)(*[_ptr(y) for y in ys])
    _check(_c("mdbf_linear_multi")(arr, S, P, n, m, r, l, _ptr(x), yp, _ydt(ys[0]), B, _ptr(workspace),
                                   workspace.numel() * workspace.element_size(), _stream(stream)))
    return ys


def mdbf_linear_noalloc(paths, n, m, r, l, x, y, stream=None):
    """mdbf_linear without a caller workspace, for callers that cannot allocate device memory.

    The scratch is a fixed array inside the library (mdbf_noalloc_scratch_bytes() bytes, shared by
    all calls: calls that overlap on the GPU race).  Make the first call on a device before any
    stream capture."""
    _want(x, torch.bfloat16, "x")
    B = x.shape[0]
    if x.shape[1] != m or tuple(y.shape) != (B, n) or not y.is_contiguous():
        raise ValueError("x must be [B, m] and y [B, n]")
    arr = paths if isinstance(paths, ctypes.Array) else mdbf_paths_c(paths)
    _check(_c("mdbf_linear_noalloc")(arr, len(arr), n, m, r, l, _ptr(x), _ptr(y), _ydt(y), B, _stream(stream)))
    return y


def mdbf_noalloc_scratch_bytes() -> int:
    return int(_c("mdbf_noalloc_scratch_bytes")())


def mdbf_dequant_debug(paths, n, m, r, l, W, F=None, G=None, stream=None):
    """W [n, m] fp32 (and optionally F [P, n, r], G [P, r, m]) materialised bit-reproducibly."""
    arr = paths if isinstance(paths, ctypes.Array) else mdbf_paths_c(paths)
    _check(_c("mdbf_dequant_debug")(arr, len(arr), n, m, r, l, _ptr(W), _ptr(F), _ptr(G), _stream(stream)))
    return W


def mdbf_effective_bits(n, m, r, P, l, scale_bits=16) -> float:
    return float(_c("mdbf_effective_bits")(n, m, r, P, l, scale_bits))


def mdbf_select_rank(n, m, P, l, scale_bits, target_bits):
    """(rank, clamped) for a target bits/weight; raises QLinearError when even rank 1 is too big."""
    r, c = _i(0), _i(0)
    _check(_c("mdbf_select_rank")(n, m, P, l, scale_bits, float(target_bits), ctypes.byref(r), ctypes.byref(c)))
    return r.value, bool(c.value)


def ql_check(stream=None):
    """Waits for the stream and raises QLinearError(QL_ERR_TIMEOUT) if a bounded device wait ran out."""
    _check(_c("ql_check")(_stream(stream)))


def ql_selftest_timeout(stream=None):
    """Launches the bounded-wait self-test: the next ql_check() on the stream raises QL_ERR_TIMEOUT."""
    _check(_c("ql_selftest_timeout")(_stream(stream)))


def ql_set_pdl(enable: bool) -> bool:
    """Enables or disables launch overlap (programmatic dependent launch) for every later call;
    returns the previous setting.  With overlap on, weights are read before the preceding kernel
    in the stream has finished, so they must not be written by that kernel."""
    return bool(_c("ql_set_pdl")(1 if enable else 0))
