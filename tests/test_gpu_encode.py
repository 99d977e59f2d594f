"""GPU parity of the encoder (Sec. 3.1-3.2): its per-row stage
(sage_encode_rows: Eq. 6 assignment, Eq. 14 grid, Eq. 2 codes for a given
stored codebook) and its weighted spherical k-means (sage_kmeans), bit-exact
against the oracle and against the library's CPU encoder at full size, through
the C ABI (integer, fp16-bit and fp64 outputs computed with separately rounded
fp64 operations in the same order, so the bar is equality)."""
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


def _samples(W, perm, om, sample):
    """Magnitudes and Eq. 4 weights of the sampled subvectors (storage order)."""
    S = W.shape[1] // 8
    o, j = sample // S, sample % S
    cols = perm.reshape(S, 8)[j]                      # [n][8] original channels
    P = np.abs(W[o[:, None], cols])
    Wt = om.reshape(S, 8)[j]
    return np.ascontiguousarray(P), np.ascontiguousarray(Wt)


@pytest.mark.parametrize("log2K", [4, 5, 6, 7, 8])
def test_kmeans_matches_oracle(log2K):
    """Random samples with all-zero ones among them, an initial codeword on a
    zero sample (the 1/sqrt(8) direction) and a repeated initial pick (two equal
    codewords: the later one stays empty and keeps its codeword)."""
    g = np.random.default_rng(80 + log2K)
    n, K = 3000, 1 << log2K
    P = np.abs(g.standard_normal((n, 8))) * g.lognormal(0.0, 1.0, (n, 1))
    P[g.choice(n, 40, replace=False)] = 0.0
    Wt = g.lognormal(0.0, 0.7, (n, 8))
    init = g.choice(n, K, replace=False).astype(np.int64)
    zero = int(np.flatnonzero(P.sum(axis=1) == 0)[0])
    init[1] = zero
    init[K - 1] = init[2]
    ref = oracle.kmeans(P, Wt, K, init, 4)
    cb, cb16, ws = sage.sage_kmeans(_dev(P), _dev(Wt), log2K, _dev(init), 4)
    assert sage.sage_query_status(ws) == 0
    got = cb.cpu().numpy()
    assert np.array_equal(got.view(np.uint64), ref.view(np.uint64))
    want16 = np.array([oracle.double_to_half(float(v)) for v in ref.reshape(-1)], np.uint16).reshape(K, 8)
    assert np.array_equal(cb16.cpu().numpy().view(np.uint16), want16)
    # one round: the repeated pick's later cluster is empty (ties go to the smaller
    # index) and keeps its initial codeword; the zero sample's codeword starts uniform
    cb1, _, _ = sage.sage_kmeans(_dev(P), _dev(Wt), log2K, _dev(init), 1)
    ref0 = oracle.kmeans(P, Wt, K, init, 0)
    assert np.array_equal(cb1.cpu().numpy()[K - 1].view(np.uint64), ref0[K - 1].view(np.uint64))
    assert np.all(ref0[1] == 1.0 / np.sqrt(8.0))


def test_kmeans_zero_rounds_is_the_initialisation():
    g = np.random.default_rng(90)
    P = np.abs(g.standard_normal((100, 8)))
    Wt = np.ones((100, 8))
    init = np.arange(16, dtype=np.int64) * 3
    cb, _, _ = sage.sage_kmeans(_dev(P), _dev(Wt), 4, _dev(init), 0)
    ref = oracle.kmeans(P, Wt, 16, init, 0)
    assert np.array_equal(cb.cpu().numpy().view(np.uint64), ref.view(np.uint64))


def test_kmeans_rejects_init_outside_the_samples():
    """An init position >= n is found on the device (the kernel reads sample 0
    in its place) and reported through the workspace status word; the word is
    cleared by the query."""
    P = np.ones((50, 8))
    init = np.arange(16, dtype=np.int64)
    init[5] = 50
    _, _, ws = sage.sage_kmeans(_dev(P), _dev(P), 4, _dev(init), 2)
    assert sage.sage_query_status(ws) == sage.SAGE_ERR_INVALID_ARGUMENT
    assert sage.sage_query_status(ws) == 0


def test_gpu_encoder_matches_cpu_encoder_full_size():
    """The weight-derived 4096 x 4096 layer (65,536 samples): the GPU k-means on
    the CPU encoder's samples gives its codebook bit for bit, and the GPU row
    stage with that codebook gives every field."""
    inp, _ = synth.config2()
    r = sage.sage_encode(inp.W, inp.energies, inp.log2K, inp.gamma, inp.sample, inp.init, inp.iters)
    om = oracle.omega_columns(inp.energies, r["perm"], inp.gamma)
    P, Wt = _samples(inp.W, r["perm"], om, inp.sample)
    _, cb16, _ = sage.sage_kmeans(_dev(P), _dev(Wt), inp.log2K, _dev(inp.init), inp.iters)
    cb16 = cb16.cpu().numpy().view(np.uint16)
    assert np.array_equal(cb16, r["codebook"])
    got = _gpu_rows(inp.W, r["perm"], om, cb16, inp.log2K)
    for k in ("signs", "idx", "q", "mu", "delta"):
        assert np.array_equal(got[k], r[k]), k


@pytest.mark.parametrize("log2K", [4, 5, 6, 7, 8])
def test_pack_device_matches_host_packer(log2K):
    """Random fields on two storage blocks (the second one short: 300 rows are
    38 row octets) and a ragged last octet: the device planes equal the host
    packer's word for word."""
    g = np.random.default_rng(70 + log2K)
    d_out, d_in = 300, 384
    f = synth.random_fields(g, d_out, d_in, log2K)
    main, meta = sage.sage_pack(d_out, d_in, log2K, f.signs, f.idx, f.q, f.mu, f.delta)
    dm, dt = sage.sage_pack_device(d_out, d_in, log2K, _dev(f.signs), _dev(f.idx.view(np.int16)), _dev(f.q),
                                   _dev(f.mu.view(np.int16)), _dev(f.delta.view(np.int16)))
    assert np.array_equal(dm.cpu().numpy().view(np.uint32), np.asarray(main).view(np.uint32).reshape(-1))
    assert np.array_equal(dt.cpu().numpy().view(np.uint32), np.asarray(meta).view(np.uint32).reshape(-1))


def test_pack_device_masks_wide_fields():
    """Field values wider than their bits (idx >= K, q >= 2^V) are masked on the
    device, where the host packer rejects them: the planes equal the host
    packer's planes of the masked fields."""
    g = np.random.default_rng(77)
    d_out, d_in, log2K = 24, 128, 5
    f = synth.random_fields(g, d_out, d_in, log2K)
    wide_idx = (f.idx.astype(np.uint32) | (1 << log2K)).astype(np.uint16)
    wide_q = (f.q.astype(np.uint32) | (1 << (10 - log2K))).astype(np.uint8)
    main, meta = sage.sage_pack(d_out, d_in, log2K, f.signs, f.idx, f.q, f.mu, f.delta)
    dm, dt = sage.sage_pack_device(d_out, d_in, log2K, _dev(f.signs), _dev(wide_idx.view(np.int16)), _dev(wide_q),
                                   _dev(f.mu.view(np.int16)), _dev(f.delta.view(np.int16)))
    assert np.array_equal(dm.cpu().numpy().view(np.uint32), np.asarray(main).view(np.uint32).reshape(-1))
    assert np.array_equal(dt.cpu().numpy().view(np.uint32), np.asarray(meta).view(np.uint32).reshape(-1))
