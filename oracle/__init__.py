"""CPU oracle for the SAGE packed linear layer -- TEST INFRASTRUCTURE ONLY.

Only tests/, ``__graft_entry__.smoke()`` and the CPU-baseline leg of bench.py
may import this package.  The product library (bit_vector_quantized_sage_b200)
never imports it, and it imports nothing from the product.

The arithmetic lives in ``sage_oracle.c`` (plain C, fp64); this module compiles
it with gcc on first use and wraps it with ctypes/NumPy marshalling.
"""
from __future__ import annotations

import ctypes as C
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "sage_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile sage_oracle.c into liboracle.so (plain -O2, no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fno-fast-math",
                               "-ffp-contract=off", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def lib():
    global _lib
    with _lock:
        if _lib is None:
            # SAGE_ORACLE_LIB loads another build of sage_oracle.c (the mutation
            # check points it at a deliberately broken copy in a temp directory)
            L = C.CDLL(os.environ.get("SAGE_ORACLE_LIB") or build())
            P = C.c_void_p
            i32, u16, f64, i64, sz = C.c_int, C.c_uint16, C.c_double, C.c_int64, C.c_size_t
            L.oracle_half_to_double.argtypes = [u16]
            L.oracle_half_to_double.restype = f64
            L.oracle_double_to_half.argtypes = [f64]
            L.oracle_double_to_half.restype = u16
            L.oracle_unpack.argtypes = [i32, i32, i32, P, P, P, P, P, P, P]
            L.oracle_unpack.restype = i32
            L.oracle_pack.argtypes = [i32, i32, i32, P, P, P, P, P, P, sz, P, sz]
            L.oracle_pack.restype = i32
            L.oracle_dequant.argtypes = [i32, i32, i32, P, P, P, P, P, P, P]
            L.oracle_dequant.restype = None
            L.oracle_round_half.argtypes = [sz, P, P]
            L.oracle_round_half.restype = None
            L.oracle_gemv.argtypes = [i32, i32, i32, P, P, P, P, P]
            L.oracle_gemv.restype = None
            L.oracle_gemv_fields_rows.argtypes = [i32, i32, i32, i32, i32, P, P, P, P, P, P, i32, P, P, P, P]
            L.oracle_gemv_fields_rows.restype = None
            L.oracle_esg_perm.argtypes = [i32, P, P]
            L.oracle_esg_perm.restype = i32
            L.oracle_omega.argtypes = [P, f64, P]
            L.oracle_omega.restype = None
            L.oracle_assign.argtypes = [P, P, P, i32, P]
            L.oracle_assign.restype = i32
            L.oracle_grid.argtypes = [P, i32, P, P]
            L.oracle_grid.restype = None
            L.oracle_quantize.argtypes = [f64, u16, u16, i32]
            L.oracle_quantize.restype = i32
            L.oracle_kmeans.argtypes = [i32, P, P, i32, P, i32, P]
            L.oracle_kmeans.restype = None
            L.oracle_encode.argtypes = [i32, i32, i32, P, P, f64, i32, P, P, i32, P, P, P, P, P, P, P]
            L.oracle_encode.restype = i32
            L.oracle_bpw.argtypes = [i32, i32, i32, i32, i32, i32, f64]
            L.oracle_bpw.restype = f64
            L.oracle_rmsnorm.argtypes = [i32, i32, P, P, f64, P]
            L.oracle_rmsnorm.restype = None
            L.oracle_add.argtypes = [sz, P, P, P]
            L.oracle_add.restype = None
            L.oracle_silu_mul.argtypes = [sz, P, P, P]
            L.oracle_silu_mul.restype = None
            L.oracle_moe_combine.argtypes = [i32, i32, i32, P, P, P]
            L.oracle_moe_combine.restype = None
            L.oracle_attend_one_position.argtypes = [i32, i32, i32, i32, P, P]
            L.oracle_attend_one_position.restype = None
            L.oracle_qdq_angle.argtypes = [f64]
            L.oracle_qdq_angle.restype = f64
            L.oracle_softplus.argtypes = [f64]
            L.oracle_softplus.restype = f64
            L.oracle_codebook_from_angles.argtypes = [i32, P, P]
            L.oracle_codebook_from_angles.restype = None
            L.oracle_qdq_forward.argtypes = [i32, i32, i32, P, P, P, P, P, P, P]
            L.oracle_qdq_forward.restype = i32
            L.oracle_abs_error.argtypes = [i32, i32, i32, P, P, P, P, P, P, P, P, P]
            L.oracle_abs_error.restype = f64
            L.oracle_encode_rows.argtypes = [i32, i32, i32, P, P, P, P, P, P, P, P, P]
            L.oracle_encode_rows.restype = None
            _lib = L
    return _lib


def _p(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(C.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


# ---------------------------------------------------------------------------
# Scalar helpers
# ---------------------------------------------------------------------------

def half_to_double(h: int) -> float:
    return lib().oracle_half_to_double(int(h))


def double_to_half(x: float) -> int:
    return int(lib().oracle_double_to_half(float(x)))


def halves_to_double(h: np.ndarray) -> np.ndarray:
    f = np.vectorize(lambda v: lib().oracle_half_to_double(int(v)), otypes=[np.float64])
    return f(np.asarray(h, dtype=np.uint16))


# ---------------------------------------------------------------------------
# Packed layout and reconstruction
# ---------------------------------------------------------------------------

def unpack(d_out, d_in, log2K, main_plane, meta_plane):
    """Logical fields from the library's packed planes (format version 2)."""
    S, G = d_in // 8, d_in // 128
    main_plane = _c(main_plane, np.uint32).reshape(-1)
    meta_plane = _c(meta_plane, np.uint32).reshape(-1)
    signs = np.zeros((d_out, S), np.uint8)
    idx = np.zeros((d_out, S), np.uint16)
    q = np.zeros((d_out, S), np.uint8)
    mu = np.zeros((d_out, G), np.uint16)
    delta = np.zeros((d_out, G), np.uint16)
    rc = lib().oracle_unpack(d_out, d_in, log2K, _p(main_plane), _p(meta_plane),
                                _p(signs), _p(idx), _p(q), _p(mu), _p(delta))
    if rc:
        raise ValueError("oracle_unpack: unsupported shape")
    return dict(signs=signs, idx=idx, q=q, mu=mu, delta=delta)


def plane_words(d_out: int, d_in: int):
    """uint32 words of the main and meta planes (whole 256-row blocks; the last
    block holds only its ceil(d_out / 8) - 32 B octets)."""
    S, G, R8 = d_in // 8, d_in // 128, (d_out + 7) // 8
    return R8 * S * 4, R8 * G * 16


def pack(d_out, d_in, log2K, signs, idx, q, mu, delta):
    """Packed planes (main, meta) of the code fields: the inverse of unpack."""
    mw, tw = plane_words(d_out, d_in)
    main_plane = np.zeros(mw, np.uint32)
    meta_plane = np.zeros(tw, np.uint32)
    rc = lib().oracle_pack(d_out, d_in, log2K, _p(_c(signs, np.uint8)), _p(_c(idx, np.uint16)),
                           _p(_c(q, np.uint8)), _p(_c(mu, np.uint16)), _p(_c(delta, np.uint16)),
                           _p(main_plane), mw, _p(meta_plane), tw)
    if rc:
        raise ValueError(f"oracle_pack: rejected ({rc})")
    return main_plane, meta_plane


def dequant(f) -> np.ndarray:
    """fp64 reconstruction W[d_out, d_in] in storage (permuted) column order."""
    W = np.zeros((f.d_out, f.d_in), np.float64)
    lib().oracle_dequant(f.d_out, f.d_in, f.log2K, _p(_c(f.signs, np.uint8)), _p(_c(f.idx, np.uint16)),
                         _p(_c(f.q, np.uint8)), _p(_c(f.mu, np.uint16)), _p(_c(f.delta, np.uint16)),
                         _p(_c(f.codebook, np.uint16)), _p(W))
    return W


def round_half(W: np.ndarray) -> np.ndarray:
    W = _c(W, np.float64)
    out = np.zeros(W.shape, np.uint16)
    lib().oracle_round_half(W.size, _p(W), _p(out))
    return out


def gemv_dense(W: np.ndarray, x: np.ndarray, perm=None):
    """y = fp32(W) x_perm in fp64; returns (y[M, d_out], bound[M, d_out])."""
    W = _c(W, np.float64)
    x = _c(x, np.uint16)
    d_out, d_in = W.shape
    M = x.shape[0]
    y = np.zeros((M, d_out), np.float64)
    b = np.zeros((M, d_out), np.float64)
    pp = _c(perm, np.int32) if perm is not None else None
    lib().oracle_gemv(d_out, d_in, M, _p(W), _p(x), _p(pp) if pp is not None else None, _p(y), _p(b))
    return y, b


def gemv(f, x: np.ndarray, rows=None):
    """y = W_hat x for code fields f (SAGE Sec. 3.1 Eq. 1-2), fp64; optionally only rows[0]:rows[1]."""
    x = _c(x, np.uint16)
    M = x.shape[0]
    r0, r1 = (0, f.d_out) if rows is None else rows
    y = np.zeros((M, f.d_out), np.float64)
    b = np.zeros((M, f.d_out), np.float64)
    pp = _c(f.perm, np.int32) if f.perm is not None else None
    lib().oracle_gemv_fields_rows(f.d_out, f.d_in, f.log2K, r0, r1,
                                  _p(_c(f.signs, np.uint8)), _p(_c(f.idx, np.uint16)), _p(_c(f.q, np.uint8)),
                                  _p(_c(f.mu, np.uint16)), _p(_c(f.delta, np.uint16)),
                                  _p(_c(f.codebook, np.uint16)), M, _p(x),
                                  _p(pp) if pp is not None else None, _p(y), _p(b))
    return y, b


# ---------------------------------------------------------------------------
# Encoder steps
# ---------------------------------------------------------------------------

def esg_perm(energy: np.ndarray) -> np.ndarray:
    e = _c(energy, np.float64)
    perm = np.zeros(e.size, np.int32)
    if lib().oracle_esg_perm(e.size, _p(e), _p(perm)):
        raise ValueError("d_in must be a multiple of 8")
    return perm


def omega(e8, gamma: float) -> np.ndarray:
    e8 = _c(e8, np.float64)
    w = np.zeros(8, np.float64)
    lib().oracle_omega(_p(e8), float(gamma), _p(w))
    return w


def assign(p8, w8, cb: np.ndarray):
    p8, w8, cb = _c(p8, np.float64), _c(w8, np.float64), _c(cb, np.float64)
    r = np.zeros(1, np.float64)
    z = lib().oracle_assign(_p(p8), _p(w8), _p(cb), cb.shape[0], _p(r))
    return int(z), float(r[0])


def grid(r16, V: int):
    r16 = _c(r16, np.float64)
    mu = np.zeros(1, np.uint16)
    de = np.zeros(1, np.uint16)
    lib().oracle_grid(_p(r16), V, _p(mu), _p(de))
    return int(mu[0]), int(de[0])


def quantize(r: float, mu16: int, delta16: int, V: int) -> int:
    return int(lib().oracle_quantize(float(r), int(mu16), int(delta16), V))


def kmeans(P: np.ndarray, Wt: np.ndarray, K: int, init: np.ndarray, iters: int) -> np.ndarray:
    P, Wt = _c(P, np.float64), _c(Wt, np.float64)
    init = _c(init, np.int64)
    cb = np.zeros((K, 8), np.float64)
    lib().oracle_kmeans(P.shape[0], _p(P), _p(Wt), K, _p(init), iters, _p(cb))
    return cb


def encode(inp):
    """Per-matrix SAGE initialisation (ESG, weighted k-means, Eq. 6, Eq. 14, Eq. 2)."""
    W = _c(inp.W, np.float64)
    d_out, d_in = W.shape
    K, S, G = 1 << inp.log2K, d_in // 8, d_in // 128
    perm = np.zeros(d_in, np.int32)
    cb = np.zeros((K, 8), np.uint16)
    signs = np.zeros((d_out, S), np.uint8)
    idx = np.zeros((d_out, S), np.uint16)
    q = np.zeros((d_out, S), np.uint8)
    mu = np.zeros((d_out, G), np.uint16)
    delta = np.zeros((d_out, G), np.uint16)
    sample, init = _c(inp.sample, np.int64), _c(inp.init, np.int64)
    rc = lib().oracle_encode(d_out, d_in, inp.log2K, _p(W), _p(_c(inp.energies, np.float64)), float(inp.gamma),
                             sample.size, _p(sample), _p(init), inp.iters, _p(perm), _p(cb),
                             _p(signs), _p(idx), _p(q), _p(mu), _p(delta))
    if rc:
        raise ValueError("oracle_encode: unsupported shape")
    return dict(perm=perm, codebook=cb, signs=signs, idx=idx, q=q, mu=mu, delta=delta)


def bpw(v: int, B: int, G: int, bg: int, K: int, bc: int, N: float) -> float:
    return float(lib().oracle_bpw(v, B, G, bg, K, bc, float(N)))


# ---------------------------------------------------------------------------
# Decoder-layer operations around the packed projections (fp16 bits in / out)
# ---------------------------------------------------------------------------

def rmsnorm(x16: np.ndarray, g16: np.ndarray, eps: float) -> np.ndarray:
    """fp16(x * g / sqrt(mean(x^2) + eps)) per row of x ([M][d] fp16 bits)."""
    x = _c(np.atleast_2d(x16), np.uint16)
    g = _c(g16, np.uint16)
    out = np.zeros_like(x)
    lib().oracle_rmsnorm(x.shape[0], x.shape[1], _p(x), _p(g), float(eps), _p(out))
    return out


def add(a16: np.ndarray, b16: np.ndarray) -> np.ndarray:
    a, b = _c(a16, np.uint16), _c(b16, np.uint16)
    out = np.zeros_like(a)
    lib().oracle_add(a.size, _p(a), _p(b), _p(out))
    return out


def silu_mul(gate16: np.ndarray, up16: np.ndarray) -> np.ndarray:
    g, u = _c(gate16, np.uint16), _c(up16, np.uint16)
    out = np.zeros_like(g)
    lib().oracle_silu_mul(g.size, _p(g), _p(u), _p(out))
    return out


def moe_combine(y16: np.ndarray, w: np.ndarray) -> np.ndarray:
    """Router-weighted combine: y16 fp16 bits [T*topk][d], w [T][topk] -> fp16 bits [T][d]."""
    w = _c(np.atleast_2d(w), np.float64)
    T, topk = w.shape
    y = _c(y16, np.uint16).reshape(T * topk, -1)
    out = np.zeros((T, y.shape[1]), np.uint16)
    lib().oracle_moe_combine(T, topk, y.shape[1], _p(y), _p(w), _p(out))
    return out


def attend_one_position(v16: np.ndarray, n_heads: int, n_kv: int, hd: int) -> np.ndarray:
    v = _c(np.atleast_2d(v16), np.uint16)
    out = np.zeros((v.shape[0], n_heads * hd), np.uint16)
    lib().oracle_attend_one_position(v.shape[0], n_heads, n_kv, hd, _p(v), _p(out))
    return out


# ---------------------------------------------------------------------------
# Continuous-parameter decode (blockwise optimisation forward; Sec. 3.4,
# App. A.6, Eqs. 12-14 and Eq. 2)
# ---------------------------------------------------------------------------

def qdq_angle(alpha: float) -> float:
    """Eq. 13: theta = eps + (pi/2 - 2 eps) sigmoid(alpha), eps = 1e-4."""
    return lib().oracle_qdq_angle(float(alpha))


def softplus(rho: float) -> float:
    return lib().oracle_softplus(float(rho))


def codebook_from_angles(alpha) -> np.ndarray:
    """Eq. 12: unit nonnegative codewords [K][8] from angle logits [K][7] (fp32 in)."""
    alpha = _c(alpha, np.float32)
    K = alpha.shape[0]
    cb = np.zeros((K, 8), np.float64)
    lib().oracle_codebook_from_angles(K, _p(alpha), _p(cb))
    return cb


def qdq_forward(d_out, d_in, log2K, alpha, rho, signs, idx):
    """The forward pass: W [d_out][d_in] (fp64), q [d_out][d_in/8] and the
    unrounded grid positions t = (r~ - mu) / delta [d_out][d_in/8]."""
    S = d_in // 8
    W = np.zeros((d_out, d_in), np.float64)
    q = np.zeros((d_out, S), np.uint8)
    t = np.zeros((d_out, S), np.float64)
    rc = lib().oracle_qdq_forward(d_out, d_in, log2K, _p(_c(alpha, np.float32)), _p(_c(rho, np.float32)),
                                  _p(_c(signs, np.uint8)), _p(_c(idx, np.uint16)), _p(W), _p(q), _p(t))
    if rc:
        raise ValueError("oracle_qdq_forward: unsupported shape")
    return W, q, t


# ---------------------------------------------------------------------------
# Adaptive bit splitting (Sec. 3.3, Eqs. 7-9)
# ---------------------------------------------------------------------------

def abs_error(f, W: np.ndarray, energy: np.ndarray) -> float:
    """Eq. 8 for fields f against original weights W [d_out][d_in] (original channel
    order) with channel energies e [d_in]."""
    pp = _c(f.perm, np.int32) if f.perm is not None else None
    e = lib().oracle_abs_error(f.d_out, f.d_in, f.log2K, _p(_c(f.signs, np.uint8)), _p(_c(f.idx, np.uint16)),
                               _p(_c(f.q, np.uint8)), _p(_c(f.mu, np.uint16)), _p(_c(f.delta, np.uint16)),
                               _p(_c(f.codebook, np.uint16)), _p(pp) if pp is not None else None,
                               _p(_c(W, np.float64)), _p(_c(energy, np.float64)))
    if e < 0:
        raise ValueError("oracle_abs_error: unsupported shape or zero denominator")
    return e


def abs_select(candidates, W: np.ndarray, energy: np.ndarray):
    """Eq. 9: the candidate encoding (one per (K, V) split) with the smallest Eq. 8
    error; ties go to the earlier candidate.  Returns (index, errors)."""
    errs = [abs_error(f, W, energy) for f in candidates]
    return int(np.argmin(errs)), errs


def omega_columns(energy: np.ndarray, perm: np.ndarray, gamma: float) -> np.ndarray:
    """Eq. 4 weights per storage column: omega of subvector group j (storage
    columns 8j .. 8j + 7, original channels perm[8j + i])."""
    e = _c(energy, np.float64)
    perm = np.asarray(perm)
    out = np.zeros(e.size, np.float64)
    for j in range(e.size // 8):
        out[8 * j:8 * j + 8] = omega(e[perm[8 * j:8 * j + 8]], gamma)
    return out


def encode_rows(W: np.ndarray, perm: np.ndarray, omega_cols: np.ndarray, codebook: np.ndarray, log2K: int):
    """The encoder's per-row part for a given stored codebook (fp16 bits [K][8]):
    signs, Eq. 6 indices, Eq. 14 grid (fp16 bits), Eq. 2 codes."""
    W = _c(W, np.float64)
    d_out, d_in = W.shape
    S, G = d_in // 8, d_in // 128
    out = dict(signs=np.zeros((d_out, S), np.uint8), idx=np.zeros((d_out, S), np.uint16),
               q=np.zeros((d_out, S), np.uint8), mu=np.zeros((d_out, G), np.uint16),
               delta=np.zeros((d_out, G), np.uint16))
    lib().oracle_encode_rows(d_out, d_in, log2K, _p(W), _p(_c(perm, np.int32)), _p(_c(omega_cols, np.float64)),
                             _p(_c(codebook, np.uint16)), *[_p(out[k]) for k in ("signs", "idx", "q", "mu", "delta")])
    return out
