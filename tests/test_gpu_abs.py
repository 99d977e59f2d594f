"""GPU parity of adaptive bit splitting (sage_abs_error / sage_abs_select;
Sec. 3.3, Eqs. 7-9) against the CPU oracle, through the C ABI.

The GPU rebuilds W^ in fp32 (r^ = mu + q delta, times the signed fp16
codeword) and sums e (w - w^)^2 in fp64; the oracle rebuilds W^ and sums in
fp64.  Bar: E within 1e-5 relative (each fp32 weight of W^ is within 2^-23
relative of the exact one, so E moves by about that times |w^| / |w - w^|,
a few times 1e-7 here), and the same Eq. 9 choice."""
import numpy as np
import pytest

import oracle
import synth
import bit_vector_quantized_sage_b200 as sage
from _util import workspace_for

pytestmark = pytest.mark.gpu

SPLITS = (4, 5, 6, 7, 8)  # log2 K of the five 18-bit splits (V = 10 - log2 K)


@pytest.fixture(scope="module", autouse=True)
def _built():
    from bit_vector_quantized_sage_b200 import build
    build.build()
    sage.load()


def _dev(a):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


@pytest.mark.parametrize("log2K", SPLITS)
@pytest.mark.parametrize("perm", [True, False])
def test_abs_error_matches_oracle(log2K, perm):
    g = np.random.default_rng(40 + log2K + (100 if perm else 0))
    d_out, d_in = 300, 1280
    f = synth.random_fields(g, d_out, d_in, log2K)
    if perm:
        f.perm = g.permutation(d_in).astype(np.int32)
    W = (g.standard_normal((d_out, d_in)) * 0.1).astype(np.float32)
    e = synth.lognormal_energies(g, d_in, 1.5).astype(np.float32)
    A = sage.PackedMatrix.from_fields(f)
    ws = workspace_for(sage.SAGE_OP_ABS, A, 1)
    err = sage.sage_abs_error(A, _dev(W), _dev(e), ws)
    ref = oracle.abs_error(f, W.astype(np.float64), e.astype(np.float64))
    assert abs(err - ref) <= 1e-5 * ref, (err, ref)
    assert sage.sage_abs_error(A, _dev(W), _dev(e), ws) == err  # deterministic


def _encodings(d_out, d_in, n_samples):
    """The five split encodings of one weight-derived W (the library's CPU encoder)."""
    fields = []
    for log2K in SPLITS:
        inp, _ = synth.config2(d_out=d_out, d_in=d_in, n_samples=n_samples, iters=5, log2K=log2K)
        r = sage.sage_encode(inp.W, inp.energies, log2K, inp.gamma, inp.sample, inp.init, inp.iters)
        fields.append(synth.Fields(d_out, d_in, log2K, r["signs"], r["idx"], r["q"], r["mu"], r["delta"],
                                   r["codebook"], r["perm"], f"K=2^{log2K}"))
    return inp, fields


@pytest.mark.parametrize("shape", [(256, 512, 8192), (4096, 4096, 65536)])
def test_abs_select_matches_oracle(shape):
    """Eq. 9 over the five encodings of a weight-derived layer (the 4096 x 4096
    one is the weight-derived configuration): the same split as the oracle's
    selection over the same encodings, every E within the bar."""
    d_out, d_in, n_samples = shape
    inp, fields = _encodings(d_out, d_in, n_samples)
    W32 = inp.W.astype(np.float32)
    e32 = inp.energies.astype(np.float32)
    packed = [sage.PackedMatrix.from_fields(f) for f in fields]
    ws = workspace_for(sage.SAGE_OP_ABS, packed[0], 1)
    best, errs = sage.sage_abs_select(packed, _dev(W32), _dev(e32), ws)
    # a workspace for all five: scored before one synchronisation, the same bits
    ws5 = workspace_for(sage.SAGE_OP_ABS, packed, 1)
    assert ws5.nbytes > ws.nbytes
    assert sage.sage_abs_select(packed, _dev(W32), _dev(e32), ws5) == (best, errs)
    ref_best, ref_errs = oracle.abs_select(fields, W32.astype(np.float64), e32.astype(np.float64))
    for a, b in zip(errs, ref_errs):
        assert abs(a - b) <= 1e-5 * b, (a, b)
    assert best == ref_best, (errs, ref_errs)
    assert 0.0 < min(errs) < 1.0


def _gpu_encoding(inp, log2K, x):
    """One split encoded on the GPU from the host-side inputs x (permutation,
    Eq. 4 weights, samples): k-means, row stage, device packer."""
    import torch
    d_out, d_in = inp.W.shape
    S, G = d_in // 8, d_in // 128
    _, cb16, ws = sage.sage_kmeans(_dev(x["P"]), _dev(x["Wt"]), log2K, _dev(inp.init), inp.iters)
    fl = dict(signs=torch.empty((d_out, S), dtype=torch.uint8, device="cuda"),
              idx=torch.empty((d_out, S), dtype=torch.int16, device="cuda"),
              q=torch.empty((d_out, S), dtype=torch.uint8, device="cuda"),
              mu=torch.empty((d_out, G), dtype=torch.int16, device="cuda"),
              delta=torch.empty((d_out, G), dtype=torch.int16, device="cuda"))
    sage.sage_encode_rows(d_out, d_in, log2K, _dev(inp.W), _dev(x["perm"]), _dev(x["omega"]), cb16, *fl.values())
    main, meta = sage.sage_pack_device(d_out, d_in, log2K, *fl.values())
    assert sage.sage_query_status(ws) == 0
    return sage.PackedMatrix(d_out, d_in, log2K, main, meta, cb16.reshape(-1), _dev(x["perm"]), f"K=2^{log2K}")


def test_abs_select_with_the_gpu_encoder():
    """Adaptive bit splitting end to end on the GPU: the five splits encoded by
    sage_kmeans + sage_encode_rows + sage_pack_device give the CPU encoder's
    planes and codebooks word for word, hence the same Eq. 8 errors (bit for
    bit) and the same Eq. 9 choice."""
    d_out, d_in, n_samples = 512, 1024, 8192
    inp, fields = _encodings(d_out, d_in, n_samples)
    x = sage.sage_encode_inputs(inp.W, inp.energies, inp.gamma, inp.sample)
    gpu, cpu = [], []
    for log2K, f in zip(SPLITS, fields):
        i2, _ = synth.config2(d_out=d_out, d_in=d_in, n_samples=n_samples, iters=5, log2K=log2K)
        A = _gpu_encoding(i2, log2K, x)
        B = sage.PackedMatrix.from_fields(f)
        assert np.array_equal(A.main.cpu().numpy(), B.main.cpu().numpy()), log2K
        assert np.array_equal(A.meta.cpu().numpy(), B.meta.cpu().numpy()), log2K
        assert np.array_equal(A.codebook.cpu().numpy(), B.codebook.cpu().numpy()), log2K
        gpu.append(A)
        cpu.append(B)
    W32, e32 = _dev(inp.W.astype(np.float32)), _dev(inp.energies.astype(np.float32))
    ws = workspace_for(sage.SAGE_OP_ABS, gpu[0], 1)
    assert sage.sage_abs_select(gpu, W32, e32, ws) == sage.sage_abs_select(cpu, W32, e32, ws)
