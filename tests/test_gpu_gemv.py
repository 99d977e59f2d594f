"""GPU parity of the packed GEMV (batch 1..8), its grouped form and the device
hooks, against the CPU oracle, element by element, through the C ABI."""
import numpy as np
import pytest

import oracle
import synth
import bit_vector_quantized_sage_b200 as sage
from _util import REL, ABS, assert_within_bound, dev_u16, f16_to_f64, gemv, host_u16, workspace_for

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from bit_vector_quantized_sage_b200 import build
    build.build()
    sage.load()


def _fields(seed, d_out, d_in, log2K, perm=True):
    g = np.random.default_rng(seed)
    f = synth.random_fields(g, d_out, d_in, log2K)
    if perm:
        f.perm = g.permutation(d_in).astype(np.int32)
    return f


def test_config0_single_gemv():
    """256x512, (K,V) = (64,4), identity permutation, batch 1 (the small workload)."""
    f, x = synth.config0()
    y, _, _ = gemv(f, x)
    y_ref, B = oracle.gemv(f, x)
    r = assert_within_bound(y, y_ref, B, "config0")
    assert r < REL


@pytest.mark.parametrize("log2K", [4, 5, 6, 7, 8])
def test_all_splits_ragged_shapes(log2K):
    for n, (d_out, d_in) in enumerate([(1, 128), (9, 256), (200, 384), (257, 1280), (1000, 2560)]):
        f = _fields(100 * log2K + n, d_out, d_in, log2K)
        x = synth.activations(np.random.default_rng(n), 1, d_in)
        y, _, _ = gemv(f, x)
        y_ref, B = oracle.gemv(f, x)
        assert_within_bound(y, y_ref, B, f"K=2^{log2K} {d_out}x{d_in}")


@pytest.mark.parametrize("M", [1, 2, 3, 4, 5, 6, 7, 8])
def test_batches(M):
    f = _fields(M, 520, 1024, [4, 5, 6, 7, 8][M % 5])
    x = synth.activations(np.random.default_rng(77 + M), M, 1024)
    y, _, _ = gemv(f, x)
    y_ref, B = oracle.gemv(f, x)
    assert_within_bound(y, y_ref, B, f"M={M}")


def _heavy_inputs(kind, g, M, d_in, perm):
    """Heavy-tailed activations: N(0,1) scaled by sqrt of LogNormal(0, 1.5) channel
    energies (the energy model the ESG permutation is built from); a few channels at
    1e3..1e4; or one storage subvector whose four low-lane components (0, 2, 4, 6;
    one half2 accumulator) sit near 2^15, so that the power-of-two window prescale
    must act for the fp16 partial sums to stay finite."""
    x = g.standard_normal((M, d_in))
    if kind == "energy":
        x *= np.sqrt(synth.lognormal_energies(g, d_in, 1.5))[None, :]
    elif kind == "outliers":
        for m in range(M):
            c = g.choice(d_in, 6, replace=False)
            x[m, c] = g.choice([-1.0, 1.0], 6) * g.uniform(1e3, 1e4, 6)
    else:
        sv = 37
        for m in range(M):
            for i in (0, 2, 4, 6):
                x[m, perm[8 * sv + i]] = (1.0 if i % 4 == 0 else -1.0) * (29000.0 + 500.0 * i)
    return synth.f16_bits(x)


@pytest.mark.parametrize("kind", ["energy", "outliers", "near_2p15"])
@pytest.mark.parametrize("log2K", [4, 6, 8])
@pytest.mark.parametrize("M,entry", [(1, "gemv"), (3, "gemv"), (16, "gemm")])
def test_heavy_tailed_activations(kind, log2K, M, entry):
    g = np.random.default_rng(1000 * ("energy", "outliers", "near_2p15").index(kind) + 10 * log2K + M)
    f = synth.random_fields(g, 520, 2560, log2K)
    f.perm = g.permutation(2560).astype(np.int32)
    x = _heavy_inputs(kind, g, M, 2560, f.perm)
    y, _, _ = gemv(f, x, entry=entry)
    assert np.isfinite(f16_to_f64(y)).all()
    y_ref, B = oracle.gemv(f, x)
    assert_within_bound(y, y_ref, B, f"{kind} K=2^{log2K} M={M} {entry}")


def test_deterministic_and_status_clean():
    f = _fields(5, 3000, 2560, 6)
    x = synth.activations(np.random.default_rng(5), 2, 2560)
    y1, A, ws = gemv(f, x)
    y2, _, _ = gemv(f, x)
    assert np.array_equal(y1, y2)
    y_ref, B = oracle.gemv(f, x)
    assert_within_bound(y1, y_ref, B)


def test_special_cases():
    """Closed forms: a one-hot input selects a column; delta = 0 with a single
    codeword e_0 gives y = mu * sum_j s_j0 x_perm[8j]."""
    import torch
    f = _fields(9, 64, 256, 6)
    W = oracle.dequant(f)
    for c in (0, 255):
        x = np.zeros((1, 256))
        x[0, c] = 1.0
        xb = synth.f16_bits(x)
        y, _, _ = gemv(f, xb)
        p = int(np.nonzero(f.perm == c)[0][0])
        exp = W[:, p].astype(np.float32).astype(np.float16)
        assert np.array_equal(f16_to_f64(y[0]), exp.astype(np.float64))
    g = _fields(10, 32, 256, 4, perm=False)
    g.codebook[:] = 0
    g.codebook[:, 0] = 0x3C00
    g.delta[:] = 0
    x = synth.activations(np.random.default_rng(3), 1, 256)
    y, _, _ = gemv(g, x)
    mu = f16_to_f64(g.mu)
    xs = f16_to_f64(x[0])
    s0 = np.where(g.signs & 1, -1.0, 1.0)
    exp = np.array([sum(mu[o, j // 16] * s0[o, j] * xs[8 * j] for j in range(32)) for o in range(32)])
    assert np.allclose(f16_to_f64(y[0]), exp, rtol=2e-3, atol=1e-5)


def test_layer_grouped_stages():
    """The Qwen3-4B-shaped decoder layer: four stage launches (q|k|v, o, gate|up, down)."""
    import torch
    L = synth.config1()
    mats = {}
    for f in L.mats:
        f.perm = sage.sage_esg_permutation(L.energies[f.name])
        mats[f.name] = (f, sage.PackedMatrix.from_fields(f))
    for stage in synth.QWEN3_4B_STAGES:
        x_bits = L.xs[stage[0]]
        x = dev_u16(x_bits)
        ys = [torch.zeros((1, mats[n][0].d_out), dtype=torch.int16, device="cuda") for n in stage]
        ws = workspace_for(sage.SAGE_OP_GROUPED, [mats[n][1] for n in stage], 1)
        sage.sage_gemv_grouped([mats[n][1] for n in stage], [x] * len(stage), ys, 1, ws)
        torch.cuda.synchronize()
        assert sage.sage_query_status(ws) == sage.SAGE_OK
        for n, y in zip(stage, ys):
            y_ref, B = oracle.gemv(mats[n][0], x_bits)
            assert_within_bound(host_u16(y), y_ref, B, n)


def test_device_unpack_bit_exact():
    import torch
    for log2K in (4, 5, 6, 7, 8):
        f = _fields(log2K, 77, 384, log2K)
        A = sage.PackedMatrix.from_fields(f)
        S, G = 384 // 8, 3
        t = lambda shape, dt: torch.zeros(shape, dtype=dt, device="cuda")
        s, i, q = t((77, S), torch.uint8), t((77, S), torch.int16), t((77, S), torch.uint8)
        mu, de = t((77, G), torch.int16), t((77, G), torch.int16)
        sage.sage_unpack_device(A, s, i, q, mu, de)
        torch.cuda.synchronize()
        assert np.array_equal(s.cpu().numpy(), f.signs)
        assert np.array_equal(host_u16(i), f.idx)
        assert np.array_equal(q.cpu().numpy(), f.q)
        assert np.array_equal(host_u16(mu), f.mu)
        assert np.array_equal(host_u16(de), f.delta)


def test_device_dequant_within_one_ulp():
    import torch
    for log2K in (4, 5, 6, 7, 8):
        f = _fields(20 + log2K, 150, 512, log2K)
        A = sage.PackedMatrix.from_fields(f)
        W = torch.zeros((150, 512), dtype=torch.int16, device="cuda")
        sage.sage_dequant(A, W)
        torch.cuda.synchronize()
        got = host_u16(W).astype(np.int32)
        ref = oracle.round_half(oracle.dequant(f)).astype(np.int32)
        # ulp distance on the fp16 bit patterns (same sign; the codewords are nonnegative)
        same_sign = ((got ^ ref) & 0x8000) == 0
        dist = np.where(same_sign, np.abs(got - ref), np.abs((got & 0x7FFF) + (ref & 0x7FFF)))
        assert dist.max() <= 1, (log2K, dist.max())


def test_permute_x():
    import torch
    d_in, M = 1024, 3
    x = synth.activations(np.random.default_rng(1), M, d_in)
    perm = np.random.default_rng(2).permutation(d_in).astype(np.int32)
    xp = torch.zeros((M, d_in), dtype=torch.int16, device="cuda")
    sage.sage_permute_x(dev_u16(x), torch.from_numpy(perm).cuda(), M, d_in, xp)
    torch.cuda.synchronize()
    assert np.array_equal(host_u16(xp), x[:, perm])
