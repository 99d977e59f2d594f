"""GPU parity of the encoder's per-row stage (sage_encode_rows: Eq. 6
assignment, Eq. 14 grid, Eq. 2 codes for a given stored codebook; Sec.
3.1-3.2): bit-exact against the oracle's stage and against the library's CPU
encoder at full size, through the C ABI (integer and fp16-bit outputs, so the
bar is equality)."""
import numpy as np
import pytest

import oracle
import synth
import bit_vector_quantized_sage_b200 as sage

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from bit_vector_quantized_sage_b200 import build
    build.build()
    sage.load()


def _dev(a):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def _gpu_rows(W, perm, om, codebook, log2K):
    import torch
    d_out, d_in = W.shape
    S, G = d_in // 8, d_in // 128
    out = dict(signs=torch.zeros((d_out, S), dtype=torch.uint8, device="cuda"),
               idx=torch.zeros((d_out, S), dtype=torch.int16, device="cuda"),
               q=torch.zeros((d_out, S), dtype=torch.uint8, device="cuda"),
               mu=torch.zeros((d_out, G), dtype=torch.int16, device="cuda"),
               delta=torch.zeros((d_out, G), dtype=torch.int16, device="cuda"))
    sage.sage_encode_rows(d_out, d_in, log2K, _dev(W), _dev(perm.astype(np.int32)), _dev(om),
                          _dev(codebook.view(np.int16)), out["signs"], out["idx"], out["q"], out["mu"], out["delta"])
    torch.cuda.synchronize()
    res = {k: v.cpu().numpy() for k, v in out.items()}
    for k in ("idx", "mu", "delta"):
        res[k] = res[k].view(np.uint16)
    return res


@pytest.mark.parametrize("log2K", [4, 5, 6, 7, 8])
def test_encode_rows_matches_oracle(log2K):
    """Random weights, energies, permutation and a random stored codebook; a few
    all-zero subvectors (the z = 0, r* = 0 rule) and a group of equal radii."""
    g = np.random.default_rng(60 + log2K)
    d_out, d_in = 77, 640
    W = g.standard_normal((d_out, d_in)) * 0.03
    perm = g.permutation(d_in).astype(np.int32)
    W[3, perm[:8]] = 0.0   # storage subvector 0 of row 3: all zero
    W[5, :] = 0.0          # every radius of row 5 is 0: delta = 0
    e = synth.lognormal_energies(g, d_in, 1.5)
    om = oracle.omega_columns(e, perm, 0.75)
    cb = synth.random_codebook(g, 1 << log2K)
    ref = oracle.encode_rows(W, perm, om, cb, log2K)
    got = _gpu_rows(W, perm, om, cb, log2K)
    for k in ref:
        assert np.array_equal(got[k], ref[k]), k


def test_encode_rows_matches_cpu_encoder_full_size():
    """The weight-derived 4096 x 4096 layer: given the CPU encoder's permutation,
    codebook (its k-means) and Eq. 4 weights, the GPU stage writes the CPU
    encoder's fields bit for bit."""
    inp, _ = synth.config2()
    r = sage.sage_encode(inp.W, inp.energies, inp.log2K, inp.gamma, inp.sample, inp.init, inp.iters)
    om = oracle.omega_columns(inp.energies, r["perm"], inp.gamma)
    got = _gpu_rows(inp.W, r["perm"], om, r["codebook"], inp.log2K)
    for k in ("signs", "idx", "q", "mu", "delta"):
        assert np.array_equal(got[k], r[k]), k
