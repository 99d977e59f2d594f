"""GPU parity of the continuous-parameter decode (sage_qdq_forward; Sec. 3.4,
App. A.6, Eqs. 12-14 and Eq. 2) against the CPU oracle, through the C ABI.

The kernel computes in fp32, the oracle in fp64.  Bars:
  - radius codes q identical, except where the oracle's unrounded grid
    position (r~ - mu) / delta lies within 1e-4 of a rounding boundary k + 1/2
    (there both neighbours are correct roundings of the exact value; the
    fp32 and fp64 evaluations may legitimately pick either);
  - every weight of a subvector whose code agrees within 1e-5 x the group's
    largest radius of the oracle's (about 160 fp32 ulps of that radius: the
    chain is a sigmoid, a sin/cos pair and up to seven products per codeword
    component, a softplus, the grid and one multiply, each a few ulps);
  - the codebook within 1e-6 absolute (unit vectors)."""
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


def _run(f, want_q=True, want_cb=True):
    import torch
    K, S = 1 << f.log2K, f.d_in // 8
    W = torch.zeros((f.d_out, f.d_in), dtype=torch.float32, device="cuda")
    q = torch.zeros((f.d_out, S), dtype=torch.uint8, device="cuda") if want_q else None
    cb = torch.zeros((K, 8), dtype=torch.float32, device="cuda") if want_cb else None
    sage.sage_qdq_forward(f.d_out, f.d_in, f.log2K, _dev(f.alpha), _dev(f.rho), _dev(f.signs),
                          _dev(f.idx.view(np.int16)), W, q, cb)
    torch.cuda.synchronize()
    return (W.cpu().numpy(), q.cpu().numpy() if want_q else None, cb.cpu().numpy() if want_cb else None)


def _check(f, W, q, cb):
    W_ref, q_ref, t_ref = oracle.qdq_forward(f.d_out, f.d_in, f.log2K, f.alpha, f.rho, f.signs, f.idx)
    S, G = f.d_in // 8, f.d_in // 128
    if cb is not None:
        assert np.abs(cb - oracle.codebook_from_angles(f.alpha)).max() <= 1e-6
    ok = np.ones((f.d_out, S), bool)
    if q is not None:
        diff = q != q_ref
        if diff.any():
            lo = np.minimum(q, q_ref)[diff].astype(np.float64)
            assert np.all(np.abs(q.astype(int) - q_ref.astype(int))[diff] == 1)
            assert np.all(np.abs(t_ref[diff] - (lo + 0.5)) < 1e-4), "a radius code differs away from a tie"
            ok = ~diff
    r = np.vectorize(oracle.softplus)(f.rho.astype(np.float64))
    gmax = r.reshape(f.d_out, G, 16).max(axis=2)                       # [d_out][G]
    tol = 1e-5 * np.repeat(gmax, 16 * 8, axis=1)                       # per weight
    err = np.abs(W.astype(np.float64) - W_ref)
    bad = (err > tol) & np.repeat(ok, 8, axis=1)
    assert not bad.any(), f"{int(bad.sum())} weights outside the bar; worst {err[bad].max()} vs {tol[bad].min()}"
    return int((~ok).sum())


@pytest.mark.parametrize("log2K", [4, 5, 6, 7, 8])
def test_qdq_all_splits_ragged(log2K):
    for n, (d_out, d_in) in enumerate([(1, 128), (37, 256), (300, 1280)]):
        f = synth.qdq_inputs(10 * log2K + n, d_out, d_in, log2K)
        W, q, cb = _run(f)
        _check(f, W, q, cb)


def test_qdq_equal_radii_groups_and_optional_outputs():
    """Groups of coinciding radii reconstruct their common value (q = 0); the
    q and codebook outputs are optional."""
    f = synth.qdq_inputs(5, 64, 512, 6)
    f.rho[::3, :16] = -1.5
    f.rho[1::3, 32:48] = 0.25
    W, q, cb = _run(f)
    assert (q[::3, :16] == 0).all() and (q[1::3, 32:48] == 0).all()
    _check(f, W, q, cb)
    W2, _, _ = _run(f, want_q=False, want_cb=False)
    assert np.array_equal(W2, W)


def test_qdq_full_size_and_deterministic():
    """A 4096 x 4096 matrix at (K, V) = (64, 4), the configuration of the
    weight-derived layer; identical bits on a second run."""
    f = synth.qdq_inputs(7, 4096, 4096, 6)
    W, q, cb = _run(f)
    W2, q2, _ = _run(f)
    assert np.array_equal(W, W2) and np.array_equal(q, q2)
    ties = _check(f, W, q, cb)
    assert ties < 50  # ties within 1e-4 of a rounding boundary are rare
