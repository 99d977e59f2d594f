"""Python binding of libsage, the B200 (sm_100a) SAGE packed linear layer.

Argument marshalling only: every computation runs in the compiled library
(``libsage.so``, built in-tree by ``bit_vector_quantized_sage_b200.build``).
Function names mirror the C ABI declared in ``include/sage.h``.  There is no
fallback: if the library is missing or a CUDA device is absent the calls raise.

PyTorch is used only to own device memory and streams (``tensor.data_ptr()``
and ``torch.cuda.current_stream().cuda_stream`` are passed through).
"""
from __future__ import annotations

import ctypes as C
import os
from dataclasses import dataclass
from typing import List, Optional, Sequence

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libsage.so")

SAGE_OK = 0
SAGE_ERR_INVALID_ARGUMENT = 1
SAGE_ERR_UNSUPPORTED = 2
SAGE_ERR_MISALIGNED = 3
SAGE_ERR_WORKSPACE = 4
SAGE_ERR_CUDA = 5
SAGE_ERR_TIMEOUT = 6

SAGE_OP_GEMV, SAGE_OP_GEMM, SAGE_OP_MOE, SAGE_OP_GROUPED, SAGE_OP_ABS = 0, 1, 2, 3, 4

# Every extern "C" symbol declared in include/sage.h.
EXPORTS = (
    "sage_status_string", "sage_version", "sage_packed_sizes", "sage_pack", "sage_unpack",
    "sage_esg_permutation", "sage_encode", "sage_workspace_size", "sage_gemv", "sage_gemv_grouped",
    "sage_gemm", "sage_moe_gemv", "sage_dequant", "sage_unpack_device", "sage_permute_x",
    "sage_query_status", "sage_gemv_static", "sage_decoder_layer_workspace_size", "sage_decoder_layer_forward",
    "sage_qdq_forward", "sage_abs_error", "sage_abs_select", "sage_encode_rows", "sage_kmeans_workspace_size",
    "sage_kmeans", "sage_pack_device", "sage_encode_inputs", "sage_moe_combine",
)


class SageError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        super().__init__(f"{fn}: {status_string(status)} ({status})")


class sage_matrix(C.Structure):
    _fields_ = [
        ("d_out", C.c_int32), ("d_in", C.c_int32), ("log2K", C.c_int32),
        ("main", C.c_void_p), ("meta", C.c_void_p), ("codebook", C.c_void_p), ("perm", C.c_void_p),
    ]


class sage_decoder_layer(C.Structure):
    _fields_ = [(n, sage_matrix) for n in ("q", "k", "v", "o", "gate", "up", "down")] + [
        ("attn_norm", C.c_void_p), ("mlp_norm", C.c_void_p),
        ("n_heads", C.c_int32), ("n_kv_heads", C.c_int32), ("head_dim", C.c_int32), ("eps", C.c_float),
    ]


class sage_decoder_outputs(C.Structure):
    _fields_ = [(n, C.c_void_p) for n in ("q", "k", "v", "o", "gate", "up", "down", "h_out")]


_lib = None


def load(path: str = LIB_PATH):
    """Loads libsage.so and declares the argument types (raises if absent)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise OSError(f"libsage.so not built ({path}); run python -m bit_vector_quantized_sage_b200.build")
    L = C.CDLL(path)
    P, I, SZ = C.c_void_p, C.c_int, C.c_size_t
    MP = C.POINTER(sage_matrix)
    sig = {
        "sage_status_string": ([I], C.c_char_p),
        "sage_version": ([], C.c_char_p),
        "sage_packed_sizes": ([I, I, I, C.POINTER(SZ), C.POINTER(SZ)], I),
        "sage_pack": ([I, I, I, P, P, P, P, P, P, P], I),
        "sage_unpack": ([I, I, I, P, P, P, P, P, P, P], I),
        "sage_esg_permutation": ([I, P, P], I),
        "sage_encode": ([I, I, I, P, P, C.c_double, I, P, P, I, I, P, P, P, P, P, P, P], I),
        "sage_workspace_size": ([I, MP, I, I, C.POINTER(SZ)], I),
        "sage_gemv": ([MP, P, I, P, P, SZ, P], I),
        "sage_gemv_grouped": ([MP, I, P, P, I, P, SZ, P], I),
        "sage_gemm": ([MP, P, I, P, P, SZ, P], I),
        "sage_moe_gemv": ([MP, I, P, P, I, P, P, P, SZ, P], I),
        "sage_dequant": ([MP, P, P], I),
        "sage_unpack_device": ([MP, P, P, P, P, P, P], I),
        "sage_permute_x": ([P, P, I, I, P, P], I),
        "sage_query_status": ([P, P], I),
        "sage_gemv_static": ([MP, P, I, P, P], I),
        "sage_decoder_layer_workspace_size": ([C.POINTER(sage_decoder_layer), I, C.POINTER(SZ)], I),
        "sage_decoder_layer_forward": ([C.POINTER(sage_decoder_layer), P, I, C.POINTER(sage_decoder_outputs), P, SZ,
                                        P], I),
        "sage_qdq_forward": ([I, I, I, P, P, P, P, P, P, P, P], I),
        "sage_abs_error": ([MP, P, P, P, SZ, C.POINTER(C.c_double), P], I),
        "sage_abs_select": ([MP, I, P, P, P, SZ, C.POINTER(I), P, P], I),
        "sage_encode_rows": ([I, I, I, P, P, P, P, P, P, P, P, P, P], I),
        "sage_kmeans_workspace_size": ([I], C.c_size_t),
        "sage_pack_device": ([I, I, I, P, P, P, P, P, P, P, P], I),
        "sage_moe_combine": ([I, I, I, P, P, P, P], I),
        "sage_encode_inputs": ([I, I, P, P, C.c_double, I, P, P, P, P, P], I),
        "sage_kmeans": ([I, I, P, P, P, I, P, P, P, C.c_size_t, P], I),
    }
    for name, (args, res) in sig.items():
        f = getattr(L, name)
        f.argtypes = args
        f.restype = res
    _lib = L
    return L


def status_string(s: int) -> str:
    return load().sage_status_string(int(s)).decode()


def version() -> str:
    return load().sage_version().decode()


def _check(fn: str, rc: int):
    if rc != SAGE_OK:
        raise SageError(fn, rc)


def _np(a, dtype):
    a = np.ascontiguousarray(a, dtype=dtype)
    return a, a.ctypes.data_as(C.c_void_p)


def _ptr(t) -> Optional[int]:
    """Device pointer of a torch tensor (or None / int passthrough)."""
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream=None) -> Optional[int]:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


# ---------------------------------------------------------------------------
# Host entry points
# ---------------------------------------------------------------------------

def sage_packed_sizes(d_out: int, d_in: int, log2K: int):
    a, b = C.c_size_t(), C.c_size_t()
    _check("sage_packed_sizes", load().sage_packed_sizes(d_out, d_in, log2K, C.byref(a), C.byref(b)))
    return a.value, b.value


def sage_pack(d_out, d_in, log2K, signs, idx, q, mu, delta):
    """Packs fields (NumPy, storage order) into (main, meta) uint32 NumPy planes."""
    mb, tb = sage_packed_sizes(d_out, d_in, log2K)
    main = np.zeros(mb // 4, np.uint32)
    meta = np.zeros(tb // 4, np.uint32)
    s, ps = _np(signs, np.uint8)
    i, pi = _np(idx, np.uint16)
    qq, pq = _np(q, np.uint8)
    m, pm = _np(mu, np.uint16)
    d, pd = _np(delta, np.uint16)
    _check("sage_pack", load().sage_pack(d_out, d_in, log2K, ps, pi, pq, pm, pd,
                                          main.ctypes.data_as(C.c_void_p), meta.ctypes.data_as(C.c_void_p)))
    return main, meta


def sage_unpack(d_out, d_in, log2K, main, meta):
    S, G = d_in // 8, d_in // 128
    out = dict(signs=np.zeros((d_out, S), np.uint8), idx=np.zeros((d_out, S), np.uint16),
               q=np.zeros((d_out, S), np.uint8), mu=np.zeros((d_out, G), np.uint16),
               delta=np.zeros((d_out, G), np.uint16))
    mn, pmn = _np(main, np.uint32)
    mt, pmt = _np(meta, np.uint32)
    _check("sage_unpack", load().sage_unpack(d_out, d_in, log2K, pmn, pmt,
                                              *[out[k].ctypes.data_as(C.c_void_p)
                                                for k in ("signs", "idx", "q", "mu", "delta")]))
    return out


def sage_esg_permutation(energy) -> np.ndarray:
    e, pe = _np(energy, np.float64)
    perm = np.zeros(e.size, np.int32)
    _check("sage_esg_permutation", load().sage_esg_permutation(e.size, pe, perm.ctypes.data_as(C.c_void_p)))
    return perm


def sage_encode(W, energy, log2K: int, gamma: float, sample, init, iters: int, n_threads: int = 0):
    """CPU encoder (ESG, weighted k-means, Eq. 6, Eq. 14, Eq. 2) -> dict of fields + perm + codebook."""
    W, pW = _np(W, np.float64)
    e, pe = _np(energy, np.float64)
    sm, psm = _np(sample, np.int64)
    it, pit = _np(init, np.int64)
    d_out, d_in = W.shape
    K, S, G = 1 << log2K, d_in // 8, d_in // 128
    out = dict(perm=np.zeros(d_in, np.int32), codebook=np.zeros((K, 8), np.uint16),
               signs=np.zeros((d_out, S), np.uint8), idx=np.zeros((d_out, S), np.uint16),
               q=np.zeros((d_out, S), np.uint8), mu=np.zeros((d_out, G), np.uint16),
               delta=np.zeros((d_out, G), np.uint16))
    _check("sage_encode", load().sage_encode(
        d_out, d_in, log2K, pW, pe, float(gamma), sm.size, psm, pit, iters, n_threads,
        *[out[k].ctypes.data_as(C.c_void_p) for k in ("perm", "codebook", "signs", "idx", "q", "mu", "delta")]))
    return out


# ---------------------------------------------------------------------------
# Device-side packed matrices
# ---------------------------------------------------------------------------

@dataclass
class PackedMatrix:
    """A packed matrix resident on the device (torch tensors own the memory)."""
    d_out: int
    d_in: int
    log2K: int
    main: "object"
    meta: "object"
    codebook: "object"
    perm: "object" = None
    name: str = ""

    def desc(self) -> sage_matrix:
        return sage_matrix(self.d_out, self.d_in, self.log2K, _ptr(self.main), _ptr(self.meta),
                           _ptr(self.codebook), _ptr(self.perm) if self.perm is not None else None)

    @property
    def packed_bytes(self) -> int:
        return self.main.numel() * 4 + self.meta.numel() * 4

    @staticmethod
    def from_planes(d_out, d_in, log2K, main, meta, codebook, perm=None, device="cuda", name=""):
        import torch
        t = lambda a, dt: torch.from_numpy(np.ascontiguousarray(a).view(dt)).to(device)
        return PackedMatrix(d_out, d_in, log2K, t(main, np.int32), t(meta, np.int32),
                            t(np.asarray(codebook, np.uint16).reshape(-1), np.int16),
                            t(np.asarray(perm, np.int32), np.int32) if perm is not None else None, name)

    @staticmethod
    def from_fields(f, device="cuda"):
        main, meta = sage_pack(f.d_out, f.d_in, f.log2K, f.signs, f.idx, f.q, f.mu, f.delta)
        return PackedMatrix.from_planes(f.d_out, f.d_in, f.log2K, main, meta, f.codebook, f.perm, device, f.name)


def _mat_array(mats: Sequence[PackedMatrix]):
    arr = (sage_matrix * len(mats))(*[m.desc() for m in mats])
    return arr


def sage_workspace_size(op: int, mats, M: int) -> int:
    """Workspace bytes for one call of `op` over `mats` (one matrix, a grouped list or all experts)."""
    if isinstance(mats, PackedMatrix):
        mats = [mats]
    arr = _mat_array(mats)
    b = C.c_size_t()
    _check("sage_workspace_size", load().sage_workspace_size(op, arr, len(mats), M, C.byref(b)))
    return b.value


class Workspace:
    """Zero-initialised device workspace (status word + split-K scratch)."""

    def __init__(self, nbytes: int, device="cuda"):
        import torch
        self.nbytes = int(max(256, nbytes))
        self.buf = torch.zeros(self.nbytes, dtype=torch.uint8, device=device)

    @property
    def ptr(self) -> int:
        return self.buf.data_ptr()


def sage_gemv(A: PackedMatrix, x, M: int, y, ws: Workspace, stream=None):
    d = A.desc()
    _check("sage_gemv", load().sage_gemv(C.byref(d), _ptr(x), M, _ptr(y), ws.ptr, ws.nbytes, _stream(stream)))


def sage_gemv_static(A: PackedMatrix, x, M: int, y, stream=None):
    """sage_gemv with the library's built-in 4 MiB scratch instead of a workspace
    (for callers that cannot allocate; calls on one device must not overlap)."""
    d = A.desc()
    _check("sage_gemv_static", load().sage_gemv_static(C.byref(d), _ptr(x), M, _ptr(y), _stream(stream)))


def sage_gemm(A: PackedMatrix, x, M: int, y, ws: Workspace, stream=None):
    d = A.desc()
    _check("sage_gemm", load().sage_gemm(C.byref(d), _ptr(x), M, _ptr(y), ws.ptr, ws.nbytes, _stream(stream)))


class GroupedCall:
    """Pre-marshalled sage_gemv_grouped arguments (cheap to launch repeatedly)."""

    def __init__(self, mats: Sequence[PackedMatrix], xs, ys, M: int, ws: Workspace):
        self.n = len(mats)
        self.arr = _mat_array(mats)
        self.xs = (C.c_void_p * self.n)(*[_ptr(x) for x in xs])
        self.ys = (C.c_void_p * self.n)(*[_ptr(y) for y in ys])
        self.M = M
        self.ws = ws
        self.keep = (list(mats), list(xs), list(ys))

    def __call__(self, stream=None):
        _check("sage_gemv_grouped", load().sage_gemv_grouped(self.arr, self.n, self.xs, self.ys, self.M,
                                                             self.ws.ptr, self.ws.nbytes, _stream(stream)))


def sage_gemv_grouped(mats: Sequence[PackedMatrix], xs, ys, M: int, ws: Workspace, stream=None):
    GroupedCall(mats, xs, ys, M, ws)(stream)


def sage_moe_gemv(experts: Sequence[PackedMatrix], pair_expert, pair_xrow, n_pairs: int, x, y, ws: Workspace,
                  stream=None):
    arr = _mat_array(experts)
    _check("sage_moe_gemv", load().sage_moe_gemv(arr, len(experts), _ptr(pair_expert), _ptr(pair_xrow), n_pairs,
                                                 _ptr(x), _ptr(y), ws.ptr, ws.nbytes, _stream(stream)))


def sage_encode_rows(d_out: int, d_in: int, log2K: int, W, perm, omega, codebook, signs, idx, q, mu, delta,
                     stream=None):
    """The encoder's per-row stage on the GPU (device tensors: W fp64, perm int32, omega
    fp64 per storage column, codebook fp16 bits; outputs signs u8, idx int16/u16,
    q u8, mu/delta fp16 bits)."""
    _check("sage_encode_rows", load().sage_encode_rows(d_out, d_in, log2K, _ptr(W), _ptr(perm), _ptr(omega),
                                                       _ptr(codebook), _ptr(signs), _ptr(idx), _ptr(q), _ptr(mu),
                                                       _ptr(delta), _stream(stream)))


def sage_encode_inputs(W, energy, gamma: float, sample):
    """Host: ESG permutation, Eq. 4 weights per storage column and the sampled
    subvectors' magnitudes / weights -> dict(perm, omega, P, Wt) (numpy)."""
    W, pW = _np(W, np.float64)
    e, pe = _np(energy, np.float64)
    sm, psm = _np(sample, np.int64)
    d_out, d_in = W.shape
    n = sm.shape[0]
    out = dict(perm=np.zeros(d_in, np.int32), omega=np.zeros(d_in), P=np.zeros((n, 8)), Wt=np.zeros((n, 8)))
    _check("sage_encode_inputs", load().sage_encode_inputs(d_out, d_in, pW, pe, gamma, n, psm,
                                                           *(o.ctypes.data for o in out.values())))
    return out


def sage_moe_combine(T: int, topk: int, y_pairs, weights, y, stream=None):
    """Router-weighted combine (device tensors: y_pairs fp16 bits [T*topk][d_out],
    weights fp32 [T][topk], y fp16 bits [T][d_out])."""
    _check("sage_moe_combine", load().sage_moe_combine(T, topk, int(y.shape[-1]), _ptr(y_pairs), _ptr(weights),
                                                       _ptr(y), _stream(stream)))


def sage_kmeans_workspace_size(n: int) -> int:
    return int(load().sage_kmeans_workspace_size(n))


def sage_pack_device(d_out: int, d_in: int, log2K: int, signs, idx, q, mu, delta, stream=None):
    """The packer on the device (device field tensors) -> (main, meta) int32 device planes."""
    import torch
    mb, tb = C.c_size_t(), C.c_size_t()
    _check("sage_packed_sizes", load().sage_packed_sizes(d_out, d_in, log2K, C.byref(mb), C.byref(tb)))
    main = torch.empty(mb.value // 4, dtype=torch.int32, device=signs.device)
    meta = torch.empty(tb.value // 4, dtype=torch.int32, device=signs.device)
    _check("sage_pack_device", load().sage_pack_device(d_out, d_in, log2K, _ptr(signs), _ptr(idx), _ptr(q), _ptr(mu),
                                                       _ptr(delta), _ptr(main), _ptr(meta), _stream(stream)))
    return main, meta


def sage_kmeans(P, Wt, log2K: int, init, iters: int, ws: "Workspace | None" = None, stream=None):
    """Weighted spherical k-means on the GPU (device tensors: P, Wt fp64 [n][8],
    init int64 [K]) -> (codebook fp64 [K][8], codebook fp16 bits [K][8], workspace);
    asynchronous: sage_query_status(workspace) reports a bad init entry."""
    import torch
    n = int(P.shape[0])
    K = 1 << log2K
    cb = torch.empty((K, 8), dtype=torch.float64, device=P.device)
    cb16 = torch.empty((K, 8), dtype=torch.int16, device=P.device)
    if ws is None:
        ws = Workspace(sage_kmeans_workspace_size(n))
    _check("sage_kmeans", load().sage_kmeans(n, log2K, _ptr(P), _ptr(Wt), _ptr(init), iters, _ptr(cb), _ptr(cb16),
                                             ws.ptr, ws.nbytes, _stream(stream)))
    return cb, cb16, ws


def sage_abs_error(A: PackedMatrix, W, energy, ws: Workspace, stream=None) -> float:
    """Eq. 8 of packed matrix A against W (device fp32 [d_out][d_in], original
    channel order) with device fp32 channel energies (synchronous)."""
    d = A.desc()
    e = C.c_double()
    _check("sage_abs_error", load().sage_abs_error(C.byref(d), _ptr(W), _ptr(energy), ws.ptr, ws.nbytes, C.byref(e),
                                                   _stream(stream)))
    return e.value


def sage_abs_select(cands: Sequence[PackedMatrix], W, energy, ws: Workspace, stream=None):
    """Eq. 9 over candidate encodings of the same W: (index of the best, errors)."""
    arr = _mat_array(cands)
    best = C.c_int()
    errs = (C.c_double * len(cands))()
    _check("sage_abs_select", load().sage_abs_select(arr, len(cands), _ptr(W), _ptr(energy), ws.ptr, ws.nbytes,
                                                     C.byref(best), errs, _stream(stream)))
    return best.value, list(errs)


def sage_qdq_forward(d_out: int, d_in: int, log2K: int, alpha, rho, signs, idx, W, q=None, codebook=None,
                     stream=None):
    """Continuous-parameter decode (blockwise optimisation forward): device
    tensors alpha fp32 [K][7], rho fp32 [d_out][d_in/8], signs u8, idx int16/u16
    [d_out][d_in/8]; W fp32 [d_out][d_in] out; q u8 and codebook fp32 [K][8]
    optional outputs."""
    _check("sage_qdq_forward", load().sage_qdq_forward(d_out, d_in, log2K, _ptr(alpha), _ptr(rho), _ptr(signs),
                                                       _ptr(idx), _ptr(W), _ptr(q), _ptr(codebook),
                                                       _stream(stream)))


def sage_dequant(A: PackedMatrix, W, stream=None):
    d = A.desc()
    _check("sage_dequant", load().sage_dequant(C.byref(d), _ptr(W), _stream(stream)))


def sage_unpack_device(A: PackedMatrix, signs, idx, q, mu, delta, stream=None):
    d = A.desc()
    _check("sage_unpack_device", load().sage_unpack_device(C.byref(d), _ptr(signs), _ptr(idx), _ptr(q), _ptr(mu),
                                                           _ptr(delta), _stream(stream)))


def sage_permute_x(x, perm, M: int, d_in: int, x_perm, stream=None):
    _check("sage_permute_x", load().sage_permute_x(_ptr(x), _ptr(perm), M, d_in, _ptr(x_perm), _stream(stream)))


def sage_query_status(ws: Workspace, stream=None) -> int:
    return int(load().sage_query_status(ws.ptr, _stream(stream)))


# ---------------------------------------------------------------------------
# Fused decoder layer (one launch of the four dependent projection stages)
# ---------------------------------------------------------------------------

class DecoderLayer:
    """Pre-marshalled sage_decoder_layer_forward arguments.

    mats: dict name -> PackedMatrix for q, k, v, o, gate, up, down; attn_norm /
    mlp_norm: fp16 device tensors [hidden]; outputs: dict name -> fp16 device
    tensors for q, k, v, o, gate, up, down, h_out ([M][...])."""

    NAMES = ("q", "k", "v", "o", "gate", "up", "down")

    def __init__(self, mats, attn_norm, mlp_norm, n_heads: int, n_kv_heads: int, head_dim: int, eps: float,
                 outputs, M: int, ws: "Workspace" = None):
        self.L = sage_decoder_layer(*[mats[n].desc() for n in self.NAMES], _ptr(attn_norm), _ptr(mlp_norm),
                                    n_heads, n_kv_heads, head_dim, float(eps))
        self.out = sage_decoder_outputs(*[_ptr(outputs[n]) for n in self.NAMES + ("h_out",)])
        self.M = M
        self.ws = ws if ws is not None else Workspace(self.workspace_size())
        self.keep = (mats, attn_norm, mlp_norm, outputs)

    def workspace_size(self) -> int:
        b = C.c_size_t()
        _check("sage_decoder_layer_workspace_size",
               load().sage_decoder_layer_workspace_size(C.byref(self.L), self.M, C.byref(b)))
        return b.value

    def __call__(self, h, stream=None):
        _check("sage_decoder_layer_forward",
               load().sage_decoder_layer_forward(C.byref(self.L), _ptr(h), self.M, C.byref(self.out), self.ws.ptr,
                                                 self.ws.nbytes, _stream(stream)))
