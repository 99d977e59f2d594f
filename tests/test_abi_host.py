"""Host-side checks of libsage (no GPU needed): the library builds and exports every
symbol include/sage.h declares, the host packer matches the oracle's independent
reading of the packed layout bit for bit, the ESG permutation and the CPU encoder
match the oracle, and argument errors are reported before anything is launched."""
import ctypes as C
import os
import re

import numpy as np
import pytest

import oracle
import synth
import bit_vector_quantized_sage_b200 as sage
from bit_vector_quantized_sage_b200 import build as sage_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    sage_build.build()
    return sage.load()


def _header_functions():
    txt = open(os.path.join(ROOT, "include", "sage.h")).read()
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w+\**\s+\**(sage_\w+)\s*\(", txt, re.M)))


def test_exports_every_declared_symbol(lib):
    declared = _header_functions()
    assert len(declared) >= 16
    assert sorted(sage.EXPORTS) == declared
    for name in declared:
        assert hasattr(lib, name), name
    assert "format v2" in sage.version()
    assert sage.status_string(sage.SAGE_ERR_TIMEOUT) == "SAGE_ERR_TIMEOUT"


@pytest.mark.parametrize("log2K", [4, 5, 6, 7, 8])
@pytest.mark.parametrize("d_out,d_in", [(1, 128), (13, 256), (64, 384), (257, 128), (520, 256)])
def test_pack_matches_oracle_unpack(lib, log2K, d_out, d_in):
    f = synth.random_fields(np.random.default_rng(log2K * 1000 + d_out), d_out, d_in, log2K)
    main, meta = sage.sage_pack(d_out, d_in, log2K, f.signs, f.idx, f.q, f.mu, f.delta)
    mb, tb = sage.sage_packed_sizes(d_out, d_in, log2K)
    assert main.nbytes == mb and meta.nbytes == tb
    R8 = (d_out + 7) // 8
    assert mb == d_in // 8 * R8 * 16 and tb == d_in // 128 * R8 * 64
    u = oracle.unpack(d_out, d_in, log2K, main, meta)
    for k in ("signs", "idx", "q", "mu", "delta"):
        assert np.array_equal(u[k], getattr(f, k)), k
    back = sage.sage_unpack(d_out, d_in, log2K, main, meta)
    for k in back:
        assert np.array_equal(back[k], getattr(f, k)), k
    om, ot = oracle.pack(d_out, d_in, log2K, f.signs, f.idx, f.q, f.mu, f.delta)
    assert np.array_equal(np.asarray(main).view(np.uint32).reshape(-1), om)
    assert np.array_equal(np.asarray(meta).view(np.uint32).reshape(-1), ot)


def test_pack_reproduces_hand_example(lib):
    import json
    for gx in json.load(open(os.path.join(ROOT, "tests", "golden", "format_example.json")))["examples"]:
        d_out, d_in, log2K = gx["d_out"], gx["d_in"], gx["log2K"]
        S, G = d_in // 8, d_in // 128
        signs = np.zeros((d_out, S), np.uint8)
        idx = np.zeros((d_out, S), np.uint16)
        q = np.zeros((d_out, S), np.uint8)
        mu = np.zeros((d_out, G), np.uint16)
        delta = np.zeros((d_out, G), np.uint16)
        for e in gx["fields_nonzero"]:
            signs[e["row"], e["j"]], idx[e["row"], e["j"]], q[e["row"], e["j"]] = e["signs"], e["idx"], e["q"]
        for e in gx["grid_nonzero"]:
            mu[e["row"], e["g"]], delta[e["row"], e["g"]] = int(e["mu"], 16), int(e["delta"], 16)
        main, meta = sage.sage_pack(d_out, d_in, log2K, signs, idx, q, mu, delta)
        exp_main = np.zeros(gx["main_words"], np.uint32)
        exp_meta = np.zeros(gx["meta_words"], np.uint32)
        for k, v in gx["main_nonzero"].items():
            exp_main[int(k)] = int(v, 16)
        for k, v in gx["meta_nonzero"].items():
            exp_meta[int(k)] = int(v, 16)
        assert np.array_equal(main, exp_main), d_out
        assert np.array_equal(meta, exp_meta), d_out


def test_pack_rejects_out_of_range_fields(lib):
    f = synth.random_fields(np.random.default_rng(0), 8, 128, 6)
    f.idx[3, 2] = 64
    with pytest.raises(sage.SageError) as e:
        sage.sage_pack(8, 128, 6, f.signs, f.idx, f.q, f.mu, f.delta)
    assert e.value.status == sage.SAGE_ERR_INVALID_ARGUMENT
    with pytest.raises(sage.SageError) as e:
        sage.sage_packed_sizes(8, 100, 6)
    assert e.value.status == sage.SAGE_ERR_UNSUPPORTED
    with pytest.raises(sage.SageError) as e:
        sage.sage_packed_sizes(8, 128, 9)
    assert e.value.status == sage.SAGE_ERR_UNSUPPORTED


def test_esg_matches_oracle(lib):
    import json
    for case in json.load(open(os.path.join(ROOT, "tests", "golden", "esg_tiny.json")))["cases"]:
        assert sage.sage_esg_permutation(np.array(case["energy"], float)).tolist() == case["perm"]
    for d_in in (128, 2560, 9728):
        e = np.random.default_rng(d_in).lognormal(0, 1.5, d_in)
        e[::17] = e[3]  # ties
        assert np.array_equal(sage.sage_esg_permutation(e), oracle.esg_perm(e))


def test_encoder_matches_oracle(lib):
    inp, _ = synth.config2(d_out=64, d_in=256, n_samples=1024, iters=5, log2K=5)
    a = oracle.encode(inp)
    b = sage.sage_encode(inp.W, inp.energies, inp.log2K, inp.gamma, inp.sample, inp.init, inp.iters, n_threads=4)
    for k in a:
        assert np.array_equal(a[k], b[k]), k


def test_host_argument_errors_before_launch(lib):
    """Every compute entry point validates on the host and returns an error code
    without touching the device (this runs on a machine without a GPU)."""
    L = lib
    ws = (C.c_uint8 * 4096)()
    wsp = C.cast(ws, C.c_void_p).value
    wsp16 = (wsp + 15) // 16 * 16
    good = dict(d_out=64, d_in=256, log2K=6, main=0x100000, meta=0x200000, codebook=0x300000, perm=None)

    def mat(**kw):
        d = dict(good, **kw)
        return sage.sage_matrix(d["d_out"], d["d_in"], d["log2K"], d["main"], d["meta"], d["codebook"], d["perm"])

    x, y = 0x400000, 0x500000
    A = mat()
    assert L.sage_gemv(C.byref(mat(main=None)), x, 1, y, wsp16, 4000, None) == sage.SAGE_ERR_INVALID_ARGUMENT
    assert L.sage_gemv(C.byref(mat(d_in=200)), x, 1, y, wsp16, 4000, None) == sage.SAGE_ERR_UNSUPPORTED
    assert L.sage_gemv(C.byref(mat(log2K=3)), x, 1, y, wsp16, 4000, None) == sage.SAGE_ERR_UNSUPPORTED
    assert L.sage_gemv(C.byref(mat(main=0x100004)), x, 1, y, wsp16, 4000, None) == sage.SAGE_ERR_MISALIGNED
    assert L.sage_gemv(C.byref(A), x + 2, 1, y, wsp16, 4000, None) == sage.SAGE_ERR_MISALIGNED
    assert L.sage_gemv(C.byref(A), x, 0, y, wsp16, 4000, None) == sage.SAGE_ERR_UNSUPPORTED
    assert L.sage_gemv(C.byref(A), x, 9, y, wsp16, 4000, None) == sage.SAGE_ERR_UNSUPPORTED
    assert L.sage_gemv(C.byref(A), None, 1, y, wsp16, 4000, None) == sage.SAGE_ERR_INVALID_ARGUMENT
    assert L.sage_gemv(C.byref(A), x, 1, y, None, 4000, None) == sage.SAGE_ERR_WORKSPACE
    assert L.sage_gemv(C.byref(A), x, 1, y, wsp16, 16, None) == sage.SAGE_ERR_WORKSPACE
    assert L.sage_gemm(C.byref(A), x, 300, y, wsp16, 4000, None) == sage.SAGE_ERR_UNSUPPORTED
    assert L.sage_dequant(C.byref(mat(codebook=None)), y, None) == sage.SAGE_ERR_INVALID_ARGUMENT
    assert L.sage_permute_x(x, None, 1, 100, y, None) == sage.SAGE_ERR_UNSUPPORTED
    pe = (C.c_int32 * 4)()
    arr = (sage.sage_matrix * 2)(mat(), mat(d_out=32))
    assert L.sage_moe_gemv(arr, 2, 0x600000, 0x700000, 4, x, y, wsp16, 1 << 20, None) == sage.SAGE_ERR_UNSUPPORTED
    # limits checked before the expert array is read: 256 experts, 4096 pairs
    assert L.sage_moe_gemv(arr, 257, 0x600000, 0x700000, 4, x, y, wsp16, 1 << 20, None) == sage.SAGE_ERR_UNSUPPORTED
    assert L.sage_moe_gemv(arr, 2, 0x600000, 0x700000, 4097, x, y, wsp16, 1 << 20, None) == sage.SAGE_ERR_UNSUPPORTED
    xs = (C.c_void_p * 2)(x, x)
    ys = (C.c_void_p * 2)(y, None)
    assert L.sage_gemv_grouped(arr, 2, xs, ys, 1, wsp16, 1 << 20, None) == sage.SAGE_ERR_INVALID_ARGUMENT
    b = C.c_size_t()
    assert L.sage_workspace_size(7, C.byref(A), 1, 1, C.byref(b)) == sage.SAGE_ERR_INVALID_ARGUMENT
    assert L.sage_workspace_size(sage.SAGE_OP_GEMV, C.byref(A), 0, 1, C.byref(b)) == sage.SAGE_ERR_INVALID_ARGUMENT
    assert L.sage_workspace_size(sage.SAGE_OP_GEMV, C.byref(A), 1, 1, C.byref(b)) == sage.SAGE_OK
    one = b.value
    assert one >= 256
    assert L.sage_workspace_size(sage.SAGE_OP_GROUPED, arr, 2, 1, C.byref(b)) == sage.SAGE_OK
    assert b.value >= one
    del pe


def test_packed_sizes_closed_form_up_to_int_max(lib):
    """Plane sizes are ceil(d_out / 8) octets x (d_in / 8) records of 16 B, and
    ceil(d_out / 8) x (d_in / 128) groups of 8 rows x 8 B, computed without
    overflow up to the largest int row count."""
    a, b = C.c_size_t(), C.c_size_t()
    for d_out, d_in in ((1, 128), (257, 2560), (2 ** 31 - 1, 128), (2 ** 31 - 8, 4096)):
        assert lib.sage_packed_sizes(d_out, d_in, 6, C.byref(a), C.byref(b)) == sage.SAGE_OK
        r8 = (d_out + 7) // 8
        assert a.value == r8 * (d_in // 8) * 16
        assert b.value == r8 * (d_in // 128) * 64


@pytest.mark.parametrize("d_out,d_in", [(2 ** 31 - 8, 9728), (2 ** 31 - 1, 2560), (900_000_000, 2560)])
def test_engine_rejects_unit_counts_beyond_int(lib, d_out, d_in):
    """A matrix whose block-column count (256-row blocks x d_in / 8) passes 2^30 is
    refused on the host before any device call: the pointers below are never
    dereferenced, and the unit arithmetic is 64-bit up to the check."""
    A = sage.sage_matrix(d_out, d_in, 6, 0x100000, 0x200000, 0x300000, None)
    need = C.c_size_t()
    assert lib.sage_workspace_size(sage.SAGE_OP_GEMV, C.byref(A), 1, 1, C.byref(need)) == sage.SAGE_OK
    blocks = ((d_out + 7) // 8 + 31) // 32
    assert need.value >= blocks * 4
    rc = lib.sage_gemv(C.byref(A), 0x400000, 1, 0x500000, 0x10000000, 1 << 45, None)
    assert rc == sage.SAGE_ERR_UNSUPPORTED


def test_qdq_forward_argument_errors(lib):
    """Refused on the host before any launch (the pointers are never dereferenced)."""
    a, r, s, i, w = 0x100000, 0x200000, 0x300000, 0x400000, 0x500000
    assert lib.sage_qdq_forward(8, 128, 6, None, r, s, i, w, None, None, None) == sage.SAGE_ERR_INVALID_ARGUMENT
    assert lib.sage_qdq_forward(8, 128, 6, a, r, s, i, None, None, None, None) == sage.SAGE_ERR_INVALID_ARGUMENT
    assert lib.sage_qdq_forward(8, 100, 6, a, r, s, i, w, None, None, None) == sage.SAGE_ERR_UNSUPPORTED
    assert lib.sage_qdq_forward(8, 128, 3, a, r, s, i, w, None, None, None) == sage.SAGE_ERR_UNSUPPORTED
    assert lib.sage_qdq_forward(0, 128, 6, a, r, s, i, w, None, None, None) == sage.SAGE_ERR_UNSUPPORTED
    assert lib.sage_qdq_forward(8, 128, 6, a, r, s, i, w + 4, None, None, None) == sage.SAGE_ERR_MISALIGNED


def test_abs_argument_errors(lib):
    """Refused on the host before any launch (the pointers are never dereferenced)."""
    A = sage.sage_matrix(64, 256, 6, 0x100000, 0x200000, 0x300000, None)
    e = C.c_double()
    need = C.c_size_t()
    assert lib.sage_workspace_size(sage.SAGE_OP_ABS, C.byref(A), 1, 1, C.byref(need)) == sage.SAGE_OK
    assert need.value >= 256 + 16
    ws = 0x10000000
    assert lib.sage_abs_error(C.byref(A), None, 0x500000, ws, need.value, C.byref(e), None) == sage.SAGE_ERR_INVALID_ARGUMENT
    assert lib.sage_abs_error(C.byref(A), 0x400000, 0x500000, None, need.value, C.byref(e), None) == sage.SAGE_ERR_WORKSPACE
    assert lib.sage_abs_error(C.byref(A), 0x400004, 0x500000, ws, need.value, C.byref(e), None) == sage.SAGE_ERR_MISALIGNED
    assert lib.sage_abs_error(C.byref(A), 0x400000, 0x500000, ws, 16, C.byref(e), None) == sage.SAGE_ERR_WORKSPACE
    B = (sage.sage_matrix * 2)(A, sage.sage_matrix(64, 512, 6, 0x100000, 0x200000, 0x300000, None))
    best = C.c_int()
    assert lib.sage_abs_select(B, 2, 0x400000, 0x500000, ws, need.value, C.byref(best), None, None) == sage.SAGE_ERR_UNSUPPORTED


def test_encode_rows_argument_errors(lib):
    a = [0x100000 * (i + 1) for i in range(10)]
    assert lib.sage_encode_rows(8, 128, 6, None, *a[1:10], None) == sage.SAGE_ERR_INVALID_ARGUMENT
    assert lib.sage_encode_rows(8, 100, 6, *a, None) == sage.SAGE_ERR_UNSUPPORTED
    assert lib.sage_encode_rows(8, 128, 9, *a, None) == sage.SAGE_ERR_UNSUPPORTED


def test_kmeans_argument_errors(lib):
    """Checks that return before any device work (no GPU here)."""
    n = 1000
    need = lib.sage_kmeans_workspace_size(n)
    assert need >= 64 * n and lib.sage_kmeans_workspace_size(0) == 0
    assert lib.sage_kmeans_workspace_size((1 << 30) + 1) == 0
    assert lib.sage_kmeans((1 << 30) + 1, 6, 0x100000, 0x200000, 0x300000, 3, 0x400000, None, 0x800000, 1 << 40,
                           None) == sage.SAGE_ERR_UNSUPPORTED
    a = [0x100000 * (i + 1) for i in range(4)]  # P, Wt, init, cb (never dereferenced)
    ws = 0x800000
    assert lib.sage_kmeans(n, 6, None, a[1], a[2], 3, a[3], None, ws, need, None) == sage.SAGE_ERR_INVALID_ARGUMENT
    assert lib.sage_kmeans(n, 6, a[0], a[1], a[2], 3, None, None, ws, need, None) == sage.SAGE_ERR_INVALID_ARGUMENT
    assert lib.sage_kmeans(0, 6, *a[:3], 3, a[3], None, ws, need, None) == sage.SAGE_ERR_UNSUPPORTED
    assert lib.sage_kmeans(n, 3, *a[:3], 3, a[3], None, ws, need, None) == sage.SAGE_ERR_UNSUPPORTED
    assert lib.sage_kmeans(n, 6, *a[:3], -1, a[3], None, ws, need, None) == sage.SAGE_ERR_UNSUPPORTED
    assert lib.sage_kmeans(n, 6, *a[:3], 3, a[3], None, None, need, None) == sage.SAGE_ERR_WORKSPACE
    assert lib.sage_kmeans(n, 6, *a[:3], 3, a[3], None, ws + 8, need, None) == sage.SAGE_ERR_MISALIGNED
    assert lib.sage_kmeans(n, 6, *a[:3], 3, a[3], None, ws, need - 1, None) == sage.SAGE_ERR_WORKSPACE


def test_encode_inputs_match_oracle():
    """The GPU encoder's host-side inputs: ESG permutation, Eq. 4 weights per
    storage column and the sampled subvectors' magnitudes / weights, against the
    oracle's definitions (bit for bit: the same fp64 operations)."""
    g = np.random.default_rng(17)
    d_out, d_in = 40, 256
    W = g.standard_normal((d_out, d_in))
    e = synth.lognormal_energies(g, d_in, 1.5)
    sample = np.sort(g.choice(d_out * d_in // 8, 300, replace=False)).astype(np.int64)
    r = sage.sage_encode_inputs(W, e, 0.75, sample)
    assert np.array_equal(r["perm"], oracle.esg_perm(e))
    om = oracle.omega_columns(e, r["perm"], 0.75)
    assert np.array_equal(r["omega"], om)
    S = d_in // 8
    o, j = sample // S, sample % S
    assert np.array_equal(r["P"], np.abs(W[o[:, None], r["perm"].reshape(S, 8)[j]]))
    assert np.array_equal(r["Wt"], om.reshape(S, 8)[j])
    with pytest.raises(sage.SageError):
        sage.sage_encode_inputs(W, e, 0.75, np.array([d_out * S], np.int64))
    with pytest.raises(sage.SageError) as err:
        sage.sage_encode_inputs(W[:, :200], e[:200], 0.75, sample[:4])
    assert err.value.status == sage.SAGE_ERR_UNSUPPORTED


def test_pack_device_argument_errors(lib):
    a = [0x100000 * (i + 1) for i in range(7)]
    assert lib.sage_pack_device(8, 128, 6, None, *a[1:], None) == sage.SAGE_ERR_INVALID_ARGUMENT
    assert lib.sage_pack_device(8, 100, 6, *a, None) == sage.SAGE_ERR_UNSUPPORTED
    assert lib.sage_pack_device(8, 128, 9, *a, None) == sage.SAGE_ERR_UNSUPPORTED
    assert lib.sage_pack_device(8, 128, 6, *a[:5], a[5] + 2, a[6], None) == sage.SAGE_ERR_MISALIGNED
    assert lib.sage_pack_device(8, 128, 6, *a[:6], a[6] + 4, None) == sage.SAGE_ERR_MISALIGNED
