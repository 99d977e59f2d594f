"""Pins for the CPU oracle: each check ties an oracle function to something other
than itself -- values the SAGE paper prints, hand-worked examples, closed forms,
invariants, library routines (NumPy, SciPy) and brute force on tiny inputs.

Citations refer to "SAGE: Pushing 2-Bit Vector-Quantized LLMs toward Real-World
Usability" by section / equation.
"""
import json
import os

import numpy as np
import pytest

import oracle
import synth

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _gold(name):
    with open(os.path.join(GOLD, name)) as fh:
        return json.load(fh)


def _fields(d_out, d_in, log2K, seed=0, **kw):
    return synth.random_fields(np.random.default_rng(seed), d_out, d_in, log2K, **kw)


# ---------------------------------------------------------------------------
# fp16 conversions (IEEE binary16), pinned to NumPy's float16
# ---------------------------------------------------------------------------

def test_half_to_double_all_patterns():
    h = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ref = h.view(np.float16).astype(np.float64)
    got = oracle.halves_to_double(h)
    finite = np.isfinite(ref)
    assert np.array_equal(got[finite], ref[finite])
    assert np.array_equal(np.isnan(got), np.isnan(ref))
    assert np.array_equal(np.isinf(got), np.isinf(ref))


def test_double_to_half_rne():
    g = np.random.default_rng(1)
    xs = np.concatenate([
        g.standard_normal(20000) * 10.0 ** g.integers(-9, 5, 20000),
        # exact ties between neighbouring fp16 values (round half to even)
        (np.arange(0, 2048, dtype=np.float64) + 0.5) * 2.0 ** -10,
        (np.arange(1024, 2048, dtype=np.float64) + 0.5) * 2.0 ** -24,
        [0.0, -0.0, 65504.0, 65519.99, 65520.0, 1e-9, -2.0 ** -25, 2.0 ** -25 * 1.0000001],
    ])
    with np.errstate(over="ignore"):
        ref = xs.astype(np.float16).view(np.uint16)
    got = np.array([oracle.double_to_half(v) for v in xs], dtype=np.uint16)
    assert np.array_equal(got, ref)


# ---------------------------------------------------------------------------
# Bit budget (Sec. 1, Sec. 3.1 Eq. 3, Sec. 3.3 Eq. 7, App. A.6 Eq. 15)
# ---------------------------------------------------------------------------

def test_budget_printed_values():
    gb = _gold("budget.json")
    ex = gb["example_split"]
    assert ex["signs"] + ex["index_bits"] + ex["radius_bits"] == gb["bits_per_subvector"]
    for K, V in list(synth.SPLITS) + [tuple(c) for c in gb["eq7_candidates"]]:
        assert int(np.log2(K)) + V == gb["eq7_index_plus_radius_bits"]
        assert 8 + int(np.log2(K)) + V == gb["bits_per_subvector"]
    N = 4096 * 4096
    # codebook term excluded (b_c = 0): payload + fp16 grid
    assert oracle.bpw(8, 18, 128, 0, 64, 16, N) == pytest.approx(gb["payload_bpw"] + 0.0, abs=1e-3)
    assert oracle.bpw(8, 18, 128, 0, 64, 0, N) == pytest.approx(gb["payload_bpw"])
    assert oracle.bpw(8, 18, 128, 16, 64, 0, N) == pytest.approx(gb["subtotal_bpw_before_codebook"])
    assert oracle.bpw(8, 18, 128, 16, 64, 0, N) - oracle.bpw(8, 18, 128, 0, 64, 0, N) == \
        pytest.approx(gb["fp16_grid_extra_bpw_at_G128"])
    # the codebook term: K v b_c bits for N weights; 64 fp16 codewords are 1 KiB
    cb_bits = (oracle.bpw(8, 18, 128, 16, 64, 16, N) - oracle.bpw(8, 18, 128, 16, 64, 0, N)) * N
    assert cb_bits / 8 == pytest.approx(gb["codebook_K64_fp16_bytes"])
    assert gb["group_size_G"] // 8 == gb["subvectors_per_group"]


# ---------------------------------------------------------------------------
# Packed layout (the library's own format, version 2)
# ---------------------------------------------------------------------------

def test_unpack_hand_example():
    for gx in _gold("format_example.json")["examples"]:
        main = np.zeros(gx["main_words"], np.uint32)
        meta = np.zeros(gx["meta_words"], np.uint32)
        for k, v in gx["main_nonzero"].items():
            main[int(k)] = int(v, 16)
        for k, v in gx["meta_nonzero"].items():
            meta[int(k)] = int(v, 16)
        f = oracle.unpack(gx["d_out"], gx["d_in"], gx["log2K"], main, meta)
        exp = {k: np.zeros_like(v) for k, v in f.items()}
        for e in gx["fields_nonzero"]:
            exp["signs"][e["row"], e["j"]] = e["signs"]
            exp["idx"][e["row"], e["j"]] = e["idx"]
            exp["q"][e["row"], e["j"]] = e["q"]
        for e in gx["grid_nonzero"]:
            exp["mu"][e["row"], e["g"]] = int(e["mu"], 16)
            exp["delta"][e["row"], e["g"]] = int(e["delta"], 16)
        for k in f:
            assert np.array_equal(f[k], exp[k]), (gx["d_out"], k)


@pytest.mark.parametrize("log2K", [4, 5, 6, 7, 8])
def test_unpack_is_a_bijection(log2K):
    """Every packed bit of a (record, meta entry) maps to exactly one field bit and
    every field bit is reached: flipping one packed bit changes one field bit."""
    d_out, d_in = 16, 128
    R8, S, G = 2, 16, 1
    V = 10 - log2K
    nmain, nmeta = S * R8 * 4, G * R8 * 8 * 2
    base = oracle.unpack(d_out, d_in, log2K, np.zeros(nmain, np.uint32), np.zeros(nmeta, np.uint32))
    for k in base:
        assert not base[k].any()
    hit = set()

    def field_bits(f):
        bits = set()
        for name, w in (("signs", 8), ("idx", log2K), ("q", V), ("mu", 16), ("delta", 16)):
            a = f[name].astype(np.uint32)
            for pos in zip(*np.nonzero(a)):
                for b in range(w):
                    if (int(a[pos]) >> b) & 1:
                        bits.add((name, pos, b))
        return bits

    # main record (j=3, b=1) and meta entry (g=0, b=1)
    for word in range(4):
        for bit in range(32):
            main = np.zeros(nmain, np.uint32)
            main[(3 * R8 + 1) * 4 + word] = np.uint32(1 << bit)
            fb = field_bits(oracle.unpack(d_out, d_in, log2K, main, np.zeros(nmeta, np.uint32)))
            assert len(fb) == 1, (word, bit, fb)
            hit |= fb
    for word in range(16):
        for bit in range(32):
            meta = np.zeros(nmeta, np.uint32)
            meta[(1 * 8) * 2 + word] = np.uint32(1 << bit)
            fb = field_bits(oracle.unpack(d_out, d_in, log2K, np.zeros(nmain, np.uint32), meta))
            assert len(fb) <= 1, (word, bit, fb)
            hit |= fb
    # 8 rows x (18 bits of subvector j=3) + 8 rows x 16 aux bits (only j=3's 2 counted) + grid
    sv_bits = {h for h in hit if h[0] in ("signs", "idx", "q") and h[1][1] == 3}
    assert len(sv_bits) == 8 * 18
    grid_bits = {h for h in hit if h[0] in ("mu", "delta")}
    assert len(grid_bits) == 8 * 32


@pytest.mark.parametrize("log2K", [4, 5, 6, 7, 8])
def test_pack_inverts_unpack(log2K):
    """oracle.pack is unpack's inverse both ways: fields -> planes -> fields, and
    every bit of random planes over whole octets survives planes -> fields -> planes
    (the format uses all 32 bits of a word: 2 x (log2K + V) = 20 code bits plus 12
    sign bits)."""
    f = synth.random_fields(np.random.default_rng(77 + log2K), 300, 384, log2K)
    main, meta = oracle.pack(f.d_out, f.d_in, log2K, f.signs, f.idx, f.q, f.mu, f.delta)
    u = oracle.unpack(f.d_out, f.d_in, log2K, main, meta)
    for k in ("signs", "idx", "q", "mu", "delta"):
        assert np.array_equal(u[k], getattr(f, k)), k
    d_out, d_in = 264, 256  # 33 octets: one whole block and a one-octet block
    mw, tw = oracle.plane_words(d_out, d_in)
    g = np.random.default_rng(5 + log2K)
    main = g.integers(0, 2**32, mw, dtype=np.uint64).astype(np.uint32)
    meta = g.integers(0, 2**32, tw, dtype=np.uint64).astype(np.uint32)
    u = oracle.unpack(d_out, d_in, log2K, main, meta)
    m2, t2 = oracle.pack(d_out, d_in, log2K, u["signs"], u["idx"], u["q"], u["mu"], u["delta"])
    assert np.array_equal(m2, main) and np.array_equal(t2, meta)


def test_pack_rejects_wide_fields():
    f = synth.random_fields(np.random.default_rng(3), 8, 128, 5)
    q = f.q.copy()
    q[0, 0] = 1 << 5  # V = 5: one bit too wide
    with pytest.raises(ValueError):
        oracle.pack(8, 128, 5, f.signs, f.idx, q, f.mu, f.delta)


def test_unpack_all_ones():
    for log2K in range(4, 9):
        V = 10 - log2K
        d_out, d_in = 8, 256
        f = oracle.unpack(d_out, d_in, log2K, np.full(32 * 4, 0xFFFFFFFF, np.uint32),
                             np.full(2 * 8 * 2, 0xFFFFFFFF, np.uint32))
        assert (f["signs"] == 255).all() and (f["idx"] == (1 << log2K) - 1).all()
        assert (f["q"] == (1 << V) - 1).all()
        assert (f["mu"] == 0xFFFF).all() and (f["delta"] == 0xFFFF).all()


# ---------------------------------------------------------------------------
# Reconstruction (Sec. 3.1 Eq. 1-2)
# ---------------------------------------------------------------------------

def _r_hat(f):
    mu = f.mu.view(np.float16).astype(np.float64)
    de = f.delta.view(np.float16).astype(np.float64)
    g = np.arange(f.d_in // 8) // 16
    return mu[:, g] + f.q.astype(np.float64) * de[:, g]


def test_dequant_hand_value():
    # mu = 0.125, delta = 2^-7, q = 14 -> r = 0.234375; c = 0.5; negative sign
    f = _fields(1, 128, 4, seed=3)
    f.mu[:] = 0x3000
    f.delta[:] = 0x2000
    f.q[:] = 14
    f.idx[:] = 0
    f.signs[:] = 0
    f.signs[0, 0] = 0b00000100
    f.codebook[0, :] = 0x3800
    W = oracle.dequant(f)
    assert W[0, 2] == -0.1171875
    assert W[0, 3] == 0.1171875


@pytest.mark.parametrize("log2K", [4, 6, 8])
def test_dequant_norm_equals_radius(log2K):
    """||w_hat|| = r_hat ||c_z|| for each subvector (signs do not change the norm),
    and the generated unit codewords have ||c|| within 2^-10 of 1 (fp16 rounding)."""
    f = _fields(24, 256, log2K, seed=log2K)
    W = oracle.dequant(f).reshape(24, 32, 8)
    cb = f.codebook.view(np.float16).astype(np.float64)
    cnorm = np.sqrt((cb * cb).sum(1))
    assert np.all(np.abs(cnorm - 1.0) <= 2.0 ** -10)
    got = np.sqrt((W * W).sum(2))
    exp = _r_hat(f) * cnorm[f.idx]
    assert np.allclose(got, exp, rtol=1e-15, atol=0)
    # magnitudes do not depend on the sign byte, and each sign bit flips one component
    f2 = synth.Fields(**{**f.__dict__, "signs": f.signs ^ np.uint8(0xFF)})
    W2 = oracle.dequant(f2).reshape(24, 32, 8)
    assert np.array_equal(W2, -W)


def test_dequant_zero_step_gives_common_radius():
    """App. A.6: if all radii in a group coincide the reconstruction is their common
    value; with delta = 0 every q decodes to mu."""
    f = _fields(4, 256, 5, seed=7)
    f.delta[:, 1] = 0
    W = oracle.dequant(f).reshape(4, 32, 8)
    mu = f.mu.view(np.float16).astype(np.float64)
    cb = f.codebook.view(np.float16).astype(np.float64)
    for o in range(4):
        for j in range(16, 32):
            assert np.linalg.norm(W[o, j]) == pytest.approx(mu[o, 1] * np.linalg.norm(cb[f.idx[o, j]]), rel=1e-15)


def test_dequant_single_codeword_closed_form():
    f = _fields(3, 128, 4, seed=11)
    f.codebook[:] = 0
    f.codebook[:, 0] = 0x3C00  # e_0 for every codeword
    W = oracle.dequant(f).reshape(3, 16, 8)
    s0 = np.where(f.signs & 1, -1.0, 1.0)
    assert np.array_equal(W[:, :, 0], s0 * _r_hat(f))
    assert not W[:, :, 1:].any()


# ---------------------------------------------------------------------------
# GEMV: y = W_hat x_perm (fp64), pinned to NumPy matmul and special cases
# ---------------------------------------------------------------------------

def test_gemv_matches_numpy_matmul():
    f = _fields(40, 384, 7, seed=5)
    f.perm = np.random.default_rng(9).permutation(384).astype(np.int32)
    x = synth.activations(np.random.default_rng(10), 3, 384)
    y, b = oracle.gemv(f, x)
    W32 = oracle.dequant(f).astype(np.float32).astype(np.float64)
    xp = x.view(np.float16).astype(np.float64)[:, f.perm]
    assert np.allclose(y, xp @ W32.T, rtol=1e-12, atol=1e-12)
    assert np.allclose(b, np.abs(xp) @ np.abs(W32).T, rtol=1e-12)
    assert np.all(np.abs(y) <= b * (1 + 1e-12))
    # dense entry point agrees with the fields entry point
    y2, b2 = oracle.gemv_dense(oracle.dequant(f), x, f.perm)
    assert np.array_equal(y, y2) and np.array_equal(b, b2)
    # row-subset evaluation agrees
    y3, _ = oracle.gemv(f, x, rows=(7, 19))
    assert np.array_equal(y3[:, 7:19], y[:, 7:19])


def test_gemv_permutation_direction():
    """Sec. 3.2/3.5: weights are stored in permuted column order and inference applies
    the permutation to the activations, x_perm[p] = x[perm[p]].  A one-hot input on
    original channel c selects the stored column p with perm[p] = c."""
    f = _fields(16, 128, 6, seed=2)
    f.perm = np.random.default_rng(4).permutation(128).astype(np.int32)
    W = oracle.dequant(f)
    for c in (0, 17, 127):
        x = np.zeros((1, 128), np.float64)
        x[0, c] = 1.0
        y, _ = oracle.gemv(f, synth.f16_bits(x))
        p = int(np.nonzero(f.perm == c)[0][0])
        assert np.array_equal(y[0], W[:, p].astype(np.float32).astype(np.float64))


# ---------------------------------------------------------------------------
# Encoder steps (Sec. 3.2-3.3, App. A.6)
# ---------------------------------------------------------------------------

def test_esg_hand_examples():
    for case in _gold("esg_tiny.json")["cases"]:
        assert oracle.esg_perm(np.array(case["energy"], float)).tolist() == case["perm"], case["name"]


@pytest.mark.parametrize("d_in", [128, 2560, 9728])
def test_esg_invariants(d_in):
    e = np.random.default_rng(d_in).lognormal(0, 1.5, d_in)
    perm = oracle.esg_perm(e)
    assert sorted(perm.tolist()) == list(range(d_in))
    m = d_in // 8
    rank = np.empty(d_in, int)
    rank[np.argsort(-e, kind="stable")] = np.arange(d_in)
    P = perm.reshape(m, 8)
    # position t of every subvector holds a channel of tier t (ranks [t m, (t+1) m))
    assert np.all(rank[P] // m == np.arange(8)[None, :])
    # energies decrease along the 8 positions of each subvector
    assert np.all(np.diff(e[P], axis=1) <= 0)


def test_omega_properties():
    """Eq. 4: weights normalised to unit mean; equal energies give omega = 1."""
    assert np.allclose(oracle.omega(np.full(8, 3.7), 0.75), 1.0, rtol=0, atol=1e-15)
    g = np.random.default_rng(3)
    for _ in range(20):
        e = g.lognormal(0, 1.5, 8)
        w = oracle.omega(e, 0.75)
        assert w.mean() == pytest.approx(1.0, rel=1e-14)
        assert np.allclose(w / w[0], (e / e[0]) ** 0.75, rtol=1e-12)
        assert np.array_equal(np.argsort(w, kind="stable"), np.argsort(e, kind="stable"))


def _unit_cb(g, K):
    c = np.abs(g.standard_normal((K, 8)))
    return c / np.linalg.norm(c, axis=1, keepdims=True)


def test_assign_uniform_weights_is_cosine_rule():
    """Sec. 3.1 / 3.2: with omega = 1 the assignment reduces to argmax_k d^T c_k and
    the radius to r~ = |w|^T c_z."""
    g = np.random.default_rng(5)
    cb = _unit_cb(g, 16)
    for _ in range(200):
        p = np.abs(g.standard_normal(8))
        z, r = oracle.assign(p, np.ones(8), cb)
        d = p / np.linalg.norm(p)
        assert z == int(np.argmax(cb @ d))
        assert r == pytest.approx(float(p @ cb[z]), rel=1e-12)


def test_error_decomposition_and_min_residual():
    """App. A.6 Eq. 11: ||p - r c||^2 = ||p||^2 - (p^T c)^2 + (r - p^T c)^2 for unit c;
    so the smallest continuous-radius residual is the largest cosine (both >= 0)."""
    g = np.random.default_rng(6)
    cb = _unit_cb(g, 32)
    for _ in range(100):
        p = np.abs(g.standard_normal(8))
        r = g.uniform(0, 3)
        c = cb[g.integers(32)]
        lhs = np.sum((p - r * c) ** 2)
        rhs = p @ p - (p @ c) ** 2 + (r - p @ c) ** 2
        assert lhs == pytest.approx(rhs, rel=1e-12, abs=1e-12)
        z, _ = oracle.assign(p, np.ones(8), cb)
        resid = [np.sum((p - (p @ ck) * ck) ** 2) for ck in cb]
        assert z == int(np.argmin(resid))


def test_weighted_assign_brute_force():
    """Eq. 6 against a numerical minimisation of Eq. 4 over the radius for every k."""
    from scipy.optimize import minimize_scalar
    g = np.random.default_rng(8)
    cb = _unit_cb(g, 16)
    for _ in range(60):
        p = np.abs(g.standard_normal(8))
        w = oracle.omega(g.lognormal(0, 1.5, 8), 0.75)
        best = []
        for ck in cb:
            res = minimize_scalar(lambda r: float(np.sum(w * (p - r * ck) ** 2)),
                                  bounds=(0.0, 10.0), method="bounded", options={"xatol": 1e-12})
            best.append((res.fun, res.x))
        losses = np.array([b[0] for b in best])
        z, r = oracle.assign(p, w, cb)
        if np.sort(losses)[1] - np.sort(losses)[0] > 1e-9:
            assert z == int(np.argmin(losses))
        assert r == pytest.approx(best[z][1], abs=1e-6)


def test_assign_zero_vector():
    z, r = oracle.assign(np.zeros(8), np.ones(8), _unit_cb(np.random.default_rng(1), 8))
    assert (z, r) == (0, 0.0)


def test_grid_and_quantize():
    """Eq. 14 grid and Eq. 2 codes: q in range, group extremes at the ends, and the
    decoded radius within half a step of the fitted one."""
    # hand example: mu = 0.125, delta = 2^-7
    assert oracle.quantize(0.2, 0x3000, 0x2000, 4) == 10       # 9.6 -> 10
    assert oracle.quantize(0.1, 0x3000, 0x2000, 4) == 0        # below the grid
    assert oracle.quantize(1.0, 0x3000, 0x2000, 4) == 15       # clipped
    assert oracle.quantize(0.125 + 2.5 * 2 ** -7, 0x3000, 0x2000, 4) == 3  # tie rounds up
    g = np.random.default_rng(12)
    for V in (2, 3, 4, 5, 6):
        for _ in range(50):
            r = g.uniform(0.01, 0.5, 16)
            mu16, de16 = oracle.grid(r, V)
            mu, de = np.uint16(mu16).view(np.float16).astype(float), np.uint16(de16).view(np.float16).astype(float)
            assert mu == pytest.approx(r.min(), rel=2 ** -11)
            assert de == pytest.approx((r.max() - r.min()) / (2 ** V - 1), rel=2 ** -11)
            q = np.array([oracle.quantize(x, mu16, de16, V) for x in r])
            assert q.min() >= 0 and q.max() <= 2 ** V - 1
            assert q[np.argmin(r)] == 0
            assert q[np.argmax(r)] >= 2 ** V - 2
            rec = mu + q * de
            inside = (r >= mu) & (r <= mu + (2 ** V - 1) * de)
            assert np.all(np.abs(rec - r)[inside] <= de / 2 * (1 + 1e-9) + 1e-12)
    mu16, de16 = oracle.grid(np.full(16, 0.3), 4)
    assert de16 == 0 and oracle.quantize(0.3, mu16, de16, 4) == 0


def test_kmeans_recovers_planted_directions():
    """With omega = 1 the update is spherical k-means; data drawn tightly around K
    well-separated nonnegative unit directions must give those directions back."""
    g = np.random.default_rng(13)
    K = 8
    centers = np.eye(8)
    lab = g.integers(0, K, 4000)
    P = np.abs(centers[lab] + 0.01 * g.standard_normal((4000, 8))) * g.uniform(0.5, 2, (4000, 1))
    init = np.array([int(np.nonzero(lab == k)[0][0]) for k in range(K)])
    cb = oracle.kmeans(P, np.ones_like(P), K, init, 10)
    assert np.allclose(np.linalg.norm(cb, axis=1), 1.0, atol=1e-12)
    assert (cb >= 0).all()
    # fixed point of spherical k-means: each codeword is the normalised sum of its
    # members' unit directions (the planted clusters are well separated)
    D = P / np.linalg.norm(P, axis=1, keepdims=True)
    exp = np.stack([D[lab == k].sum(0) for k in range(K)])
    exp /= np.linalg.norm(exp, axis=1, keepdims=True)
    assert np.allclose(cb, exp, rtol=0, atol=1e-12)
    assert np.allclose(cb, centers, atol=2e-2)


def test_kmeans_deterministic_and_optimal_assignment():
    inp, _ = synth.config2(d_out=32, d_in=256, n_samples=512, iters=4, log2K=4)
    a = oracle.encode(inp)
    b = oracle.encode(inp)
    for k in a:
        assert np.array_equal(a[k], b[k]), k
    assert np.array_equal(a["perm"], oracle.esg_perm(inp.energies))
    cb = a["codebook"].view(np.float16).astype(np.float64)
    assert (cb >= 0).all()
    assert np.allclose(np.linalg.norm(cb, axis=1), 1.0, atol=2 ** -9)
    # every stored index is Eq. 6-optimal for the stored codebook
    Wp = inp.W[:, a["perm"]]
    S = 256 // 8
    for o in range(0, 32, 7):
        for j in range(0, S, 5):
            w8 = oracle.omega(inp.energies[a["perm"][8 * j:8 * j + 8]], 0.75)
            p = np.abs(Wp[o, 8 * j:8 * j + 8])
            z, _ = oracle.assign(p, w8, cb)
            assert a["idx"][o, j] == z
            s = int(sum(1 << i for i in range(8) if Wp[o, 8 * j + i] < 0))
            assert a["signs"][o, j] == s
    assert a["q"].max() <= 2 ** 6 - 1


def _kmeans_case(seed=21, n=600, K=6):
    """Nonnegative subvector magnitudes with unequal per-channel weights."""
    g = np.random.default_rng(seed)
    P = np.abs(g.standard_normal((n, 8))) * g.uniform(0.2, 3.0, (n, 1))
    Wt = g.uniform(0.25, 4.0, (n, 8))
    init = g.choice(n, K, replace=False).astype(np.int64)
    return P, Wt, K, init


def test_kmeans_invariant_to_power_of_two_scaling():
    """Eq. 6 picks a direction, not a length: scaling every subvector, or every
    weight, by a power of two changes no assignment and no normalised
    centroid, so the codebook is bit-identical."""
    P, Wt, K, init = _kmeans_case()
    ref = oracle.kmeans(P, Wt, K, init, 5)
    assert np.array_equal(oracle.kmeans(P * 4.0, Wt, K, init, 5), ref)
    assert np.array_equal(oracle.kmeans(P * 0.125, Wt, K, init, 5), ref)
    assert np.array_equal(oracle.kmeans(P, Wt * 8.0, K, init, 5), ref)


def test_kmeans_single_cluster_is_a_fixed_point_after_one_step():
    """K = 1: every subvector joins the only cluster, so the first update is
    final and further iterations repeat it exactly."""
    P, Wt, _, init = _kmeans_case(K=1)
    one = oracle.kmeans(P, Wt, 1, init[:1], 1)
    assert np.array_equal(oracle.kmeans(P, Wt, 1, init[:1], 6), one)
    assert np.isclose(np.linalg.norm(one), 1.0, atol=1e-12) and (one >= 0).all()


def test_kmeans_equivariant_to_sample_order_and_channel_order():
    """Reordering the sampled subvectors (with the initial picks following them)
    leaves the codebook unchanged; permuting the 8 channels of every subvector
    and weight permutes the codebook's channels the same way (up to rounding
    of the reordered sums)."""
    P, Wt, K, init = _kmeans_case()
    ref = oracle.kmeans(P, Wt, K, init, 5)
    g = np.random.default_rng(5)
    order = g.permutation(P.shape[0])
    where = np.empty_like(order)
    where[order] = np.arange(order.size)
    got = oracle.kmeans(P[order], Wt[order], K, where[init], 5)
    assert np.allclose(got, ref, rtol=0, atol=1e-12)
    sigma = g.permutation(8)
    got = oracle.kmeans(P[:, sigma], Wt[:, sigma], K, init, 5)
    assert np.allclose(got, ref[:, sigma], rtol=0, atol=1e-12)


def test_kmeans_channel_without_weight_gets_zero_component():
    """The update weights each channel of a member's unit direction by that
    channel's omega (reading of Sec. 3.4 / App. A.7): a channel whose weight
    is zero in every sample contributes nothing, so after one step every
    codeword has a zero there."""
    P, Wt, K, init = _kmeans_case()
    Wt = Wt.copy()
    Wt[:, 3] = 0.0
    cb = oracle.kmeans(P, Wt, K, init, 2)
    assert np.all(cb[:, 3] == 0.0)
    assert np.allclose(np.linalg.norm(cb, axis=1), 1.0, atol=1e-12)


# ---------------------------------------------------------------------------
# The encoder's composition, hand-worked: Eq. 5 -> Eq. 4 -> Eq. 6 -> Eq. 14 -> Eq. 2
# ---------------------------------------------------------------------------

# Row 1 of the hand example: 16 unit directions exactly representable in fp16.
# k = 0..7 are the one-hot vectors e_k; k = 8..15 are half-vectors h_S = 1_S / 2
# over the listed four positions (norm 1, entries 0.5).
_HALVES = [(0, 1, 2, 3), (4, 5, 6, 7), (0, 1, 4, 5), (2, 3, 6, 7),
           (0, 2, 4, 6), (1, 3, 5, 7), (0, 1, 6, 7), (2, 3, 4, 5)]


def _direction(k):
    c = np.zeros(8)
    if k < 8:
        c[k] = 1.0
    else:
        c[list(_HALVES[k - 8])] = 0.5
    return c


def test_encode_composition_hand_worked():
    """A 2 x 128 layer encoded with K = 16 (V = 6), gamma = 1 and no k-means
    update (iters = 0, so the codebook is the directions of the initial
    samples), built so that every step has a closed form:

    * Eq. 5 (ESG): energies 3 for channels 0..31 and 1 for the rest are already
      sorted, so tier t holds channels 16t .. 16t + 15 and storage position
      8j + t holds channel 16t + j.
    * Eq. 4: every subvector has energies (3, 3, 1, 1, 1, 1, 1, 1) across its
      positions; gamma = 1, mean 1.5, so omega = (2, 2, 2/3, ..., 2/3).
    * Row 1 holds the 16 codeword directions, each scaled by 0.5 + n/16; it is
      the k-means sample and its subvector k initialises codeword k.
    * Eq. 6: a subvector parallel to codeword k scores sum(omega p^2) there and
      strictly less at every other codeword (weighted Cauchy-Schwarz), and its
      optimal radius is its length.  Row 0's subvector 1, p = (1, 1, 1/2, 1/2,
      0, 0, 0, 0), is parallel to no codeword: h_0123 scores
      (7/3)^2 / (4/3) = 49/12 (next best 3, at h_0145 and h_0167) with the
      weighted radius (7/3) / (4/3) = 7/4; the unweighted fit would be 3/2.
    * Eq. 14: row 0's radii span [1/2, 7/4], so mu = 1/2 and
      delta = (5/4) / 63 = 0.0198412..., stored in fp16 as 1300 / 65536
      (0x2514); row 1's span [1/2, 1/2 + 63/16] gives delta = 1/16 exactly.
    * Eq. 2 with the stored grid: row 0's subvector 2 has radius 1.1249, i.e.
      31.5027 fp16 steps (q = 32) but 31.4950 unrounded steps (31); the other
      radii are exact multiples of the stored step, or the ends of the group.
    """
    d_out, d_in, S = 2, 128, 16
    energies = np.where(np.arange(d_in) < 32, 3.0, 1.0)
    step16 = 1300.0 / 65536.0  # fp16 of 1.25 / 63
    # row 0: (codeword, radius) per subvector; subvector 1 is the non-parallel one
    row0 = [(3, 0.5), (None, None), (5, 1.1249), (10, 1.0), (0, 1.5)]
    fill_k = [1, 2, 4, 6, 7, 9, 11, 12, 13, 14, 15]
    fill_n = [3, 7, 12, 18, 22, 37, 41, 47, 55, 60, 62]
    row0 += [(k, 0.5 + n * step16) for k, n in zip(fill_k, fill_n)]
    n1 = [0, 5, 10, 15, 20, 25, 30, 35, 40, 45, 50, 55, 60, 62, 1, 63]
    P = np.zeros((d_out, S, 8))
    for t, (k, r) in enumerate(row0):
        P[0, t] = r * _direction(k) if k is not None else [1, 1, 0.5, 0.5, 0, 0, 0, 0]
    for k in range(S):
        P[1, k] = (0.5 + n1[k] / 16.0) * _direction(k)
    neg = np.zeros((d_out, S, 8), bool)
    for o in range(d_out):
        for j in range(S):
            for i in range(8):
                neg[o, j, i] = (o + j + i) % 2 == 1 and P[o, j, i] > 0
    W = np.zeros((d_out, d_in))
    for j in range(S):
        for i in range(8):
            W[:, 16 * i + j] = np.where(neg[:, j, i], -P[:, j, i], P[:, j, i])
    inp = synth.EncoderInputs(W, energies, np.arange(16, 32, dtype=np.int64), np.arange(16, dtype=np.int64),
                              1.0, 0, 4)
    out = oracle.encode(inp)

    assert np.array_equal(out["perm"], np.array([16 * t + j for j in range(S) for t in range(8)]))
    cb = out["codebook"].view(np.float16).astype(np.float64)
    assert np.array_equal(cb, np.stack([_direction(k) for k in range(16)]))
    assert out["idx"][0].tolist() == [3, 8, 5, 10, 0] + fill_k
    assert out["idx"][1].tolist() == list(range(16))
    assert out["mu"].tolist() == [[0x3800], [0x3800]]          # 1/2, both rows
    assert out["delta"].tolist() == [[0x2514], [0x2C00]]       # 1300/65536 and 1/16
    assert out["q"][0].tolist() == [0, 63, 32, 25, 50] + fill_n
    assert out["q"][1].tolist() == n1
    signs = (neg * (1 << np.arange(8))).sum(-1)
    assert np.array_equal(out["signs"], signs)


# ---------------------------------------------------------------------------
# Decoder-layer operations either side of the projections (Sec. 3.5 fuses the
# permutation with them): RMSNorm, residual add, SiLU * up, one-position attention
# ---------------------------------------------------------------------------

def _h(a):
    return np.asarray(a, np.float16).view(np.uint16)


def test_rmsnorm_constant_vector_and_scale_invariance():
    """RMSNorm of a constant vector c (eps = 0) is sign(c) * g exactly; scaling
    x by a power of two changes nothing; a hand-worked pair: x = (3, 4) has
    rms sqrt(12.5), so the outputs are 3 / sqrt(12.5) and 4 / sqrt(12.5)."""
    g = _h(np.linspace(-2, 3, 64))
    for c in (1.5, -0.25, 1000.0):
        out = oracle.rmsnorm(_h(np.full((1, 64), c)), g, 0.0)
        assert np.array_equal(out[0], _h(np.sign(c) * np.asarray(g.view(np.float16), np.float64)))
    x = _h(np.random.default_rng(3).standard_normal((2, 64)))
    x4 = _h(x.view(np.float16).astype(np.float64) * 4)
    assert np.array_equal(oracle.rmsnorm(x, g, 0.0), oracle.rmsnorm(x4, g, 0.0))
    out = oracle.rmsnorm(_h([[3.0, 4.0]]), _h([1.0, 1.0]), 0.0)
    assert np.array_equal(out[0], _h([3 / np.sqrt(12.5), 4 / np.sqrt(12.5)]))
    # eps enters under the root: x = (1, 1), eps = 3 -> 1 / 2
    assert np.array_equal(oracle.rmsnorm(_h([[1.0, 1.0]]), _h([1.0, 1.0]), 3.0)[0], _h([0.5, 0.5]))


def test_residual_add_matches_fp16_addition():
    g = np.random.default_rng(4)
    a = g.uniform(-8, 8, 1000).astype(np.float16)
    b = g.uniform(-8, 8, 1000).astype(np.float16)
    # operands within a few binades: their exact sum is an fp32 number, so
    # NumPy's fp16 addition (fp32 sum, one rounding) is the correctly rounded sum
    assert np.array_equal(oracle.add(a.view(np.uint16), b.view(np.uint16)), (a + b).view(np.uint16))


def test_silu_mul_closed_forms():
    """silu(0) = 0; silu(t) - silu(-t) = t (its odd part is t / 2); silu(ln 3)
    = (3/4) ln 3; silu(t) -> t for large t; the product is with `up`."""
    one = _h([1.0])
    assert oracle.silu_mul(_h([0.0]), one)[0] == 0
    ts = np.linspace(-6, 6, 97)
    pos = oracle.silu_mul(_h(ts), _h(np.ones_like(ts))).view(np.float16).astype(np.float64)
    neg = oracle.silu_mul(_h(-ts), _h(np.ones_like(ts))).view(np.float16).astype(np.float64)
    t16 = _h(ts).view(np.float16).astype(np.float64)
    assert np.all(np.abs((pos - neg) - t16) <= 2.0 ** -9 * np.maximum(1.0, np.abs(t16)))
    t = np.log(3.0)
    assert oracle.silu_mul(_h([t]), one)[0] == _h([0.75 * float(np.float16(t))])[0] or \
        abs(float(oracle.silu_mul(_h([t]), one).view(np.float16)[0]) - 0.75 * t) <= 2.0 ** -11
    assert oracle.silu_mul(_h([20.0]), _h([0.5]))[0] == _h([10.0])[0]
    assert oracle.silu_mul(_h([-2.0]), _h([-3.0]))[0] == _h([-2.0 / (1 + np.exp(2.0)) * -3.0])[0]


def test_attention_over_one_position_returns_the_kv_value_rows():
    """With a single cached key the softmax weight is 1: query head h reads the
    value row of key/value head h // (n_heads / n_kv)."""
    g = np.random.default_rng(5)
    n_heads, n_kv, hd = 8, 2, 16
    v = _h(g.standard_normal((3, n_kv * hd)))
    out = oracle.attend_one_position(v, n_heads, n_kv, hd)
    ref = np.repeat(v.reshape(3, n_kv, hd), n_heads // n_kv, axis=1).reshape(3, n_heads * hd)
    assert np.array_equal(out, ref)


# ---------------------------------------------------------------------------
# Continuous-parameter decode (Sec. 3.4, App. A.6, Eqs. 12-14, Eq. 2)
# ---------------------------------------------------------------------------

def test_codeword_angles_closed_form_at_zero_logits():
    """alpha = 0 puts every angle at exactly pi/4 (Eq. 13), so Eq. 12 gives
    c_j = 2^(-j/2) for j = 1..7 and c_8 = 2^(-7/2)."""
    cb = oracle.codebook_from_angles(np.zeros((1, 7), np.float32))[0]
    exp = np.array([2.0 ** (-j / 2) for j in range(1, 8)] + [2.0 ** -3.5])
    assert np.allclose(cb, exp, rtol=0, atol=1e-15)


def test_codeword_angles_unit_nonnegative_and_saturation():
    """Every codeword is a nonnegative unit vector (the map's purpose).  Saturated
    logits reach the boundaries kept eps = 1e-4 away: alpha -> -inf gives every
    angle eps, so c = (cos eps, sin eps cos eps, ...); alpha -> +inf gives
    pi/2 - eps, so the last component -> 1 and c_1 = sin eps."""
    a = np.random.default_rng(3).standard_normal((64, 7)).astype(np.float32) * 3
    cb = oracle.codebook_from_angles(a)
    assert (cb > 0).all()
    assert np.allclose(np.linalg.norm(cb, axis=1), 1.0, rtol=0, atol=1e-14)
    eps = 1e-4
    lo = oracle.codebook_from_angles(np.full((1, 7), -60.0, np.float32))[0]
    assert np.isclose(lo[0], np.cos(eps), rtol=1e-12) and np.isclose(lo[1], np.sin(eps) * np.cos(eps), rtol=1e-9)
    hi = oracle.codebook_from_angles(np.full((1, 7), 60.0, np.float32))[0]
    assert np.isclose(hi[0], np.sin(eps), rtol=1e-9) and np.isclose(hi[7], np.cos(eps) ** 7, rtol=1e-9)


def test_softplus_closed_forms():
    assert oracle.softplus(0.0) == np.log(2.0)
    assert np.isclose(oracle.softplus(40.0), 40.0, rtol=0, atol=1e-15)
    assert np.isclose(oracle.softplus(-40.0), np.exp(-40.0), rtol=1e-12, atol=0)
    assert np.isclose(oracle.softplus(1.0), np.log1p(np.e), rtol=1e-15)


def _qdq(seed=0, d_out=5, d_in=256, log2K=5):
    f = synth.qdq_inputs(seed, d_out, d_in, log2K)
    return f, oracle.qdq_forward(d_out, d_in, log2K, f.alpha, f.rho, f.signs, f.idx)


@pytest.mark.parametrize("log2K", [4, 6, 8])
def test_qdq_grid_invariants(log2K):
    """Per row group of 16 subvectors (Eq. 14, Eq. 2): the smallest fitted
    radius sits on code 0 and the largest on the top code 2^V - 1; every
    reconstructed radius is within half a grid step of its fitted radius; and
    the subvector norm |w^| is the reconstructed radius (unit codewords)."""
    f, (W, q, t) = _qdq(seed=log2K, log2K=log2K)
    V = 10 - log2K
    r = np.array([[oracle.softplus(v) for v in row] for row in f.rho.astype(np.float64)])
    S = f.d_in // 8
    for o in range(f.d_out):
        for g in range(f.d_in // 128):
            sl = slice(16 * g, 16 * g + 16)
            rr, qq = r[o, sl], q[o, sl].astype(int)
            assert qq[np.argmin(rr)] == 0 and qq[np.argmax(rr)] == (1 << V) - 1
            mu, delta = rr.min(), (rr.max() - rr.min()) / ((1 << V) - 1)
            rhat = mu + qq * delta
            assert np.all(np.abs(rhat - rr) <= delta / 2 + 1e-15)
            norms = np.linalg.norm(W[o].reshape(S, 8)[sl], axis=1)
            assert np.allclose(norms, rhat, rtol=1e-13, atol=0)


def test_qdq_equal_radii_and_signs():
    """A group whose radii coincide reconstructs their common value (delta = 0,
    q = 0); flipping one sign bit negates exactly that component."""
    f = synth.qdq_inputs(11, 2, 128, 6)
    f.rho[0, :] = -1.25
    W, q, _ = oracle.qdq_forward(2, 128, 6, f.alpha, f.rho, f.signs, f.idx)
    assert (q[0] == 0).all()
    cb = oracle.codebook_from_angles(f.alpha)
    r0 = oracle.softplus(-1.25)
    for j in range(16):
        s = np.where((f.signs[0, j] >> np.arange(8)) & 1, -1.0, 1.0)
        assert np.allclose(W[0, 8 * j:8 * j + 8], r0 * s * cb[f.idx[0, j]], rtol=1e-15, atol=0)
    s2 = f.signs.copy()
    s2[1, 3] ^= 1 << 5
    W2, _, _ = oracle.qdq_forward(2, 128, 6, f.alpha, f.rho, s2, f.idx)
    d = W2 != W
    assert d.sum() == 1 and d[1, 8 * 3 + 5] and W2[1, 29] == -W[1, 29]


# ---------------------------------------------------------------------------
# Adaptive bit splitting (Sec. 3.3, Eqs. 7-9)
# ---------------------------------------------------------------------------

def _abs_case(seed=0, d_out=24, d_in=256, log2K=5):
    g = np.random.default_rng(seed)
    f = synth.random_fields(g, d_out, d_in, log2K)
    f.perm = g.permutation(d_in).astype(np.int32)
    W = g.standard_normal((d_out, d_in)) * 0.1
    e = synth.lognormal_energies(g, d_in, 1.5)
    return f, W, e


def test_abs_error_exact_and_empty_reconstructions():
    """Eq. 8 is 0 when W is exactly the reconstruction (moved back to original
    channel order through the permutation) and 1 when the reconstruction is
    zero (all mu = delta = 0)."""
    f, _, e = _abs_case(1)
    Wh = oracle.dequant(f)                      # storage column order
    W = np.zeros_like(Wh)
    W[:, f.perm] = Wh                           # storage column p -> original channel perm[p]
    assert oracle.abs_error(f, W, e) == 0.0
    z = synth.Fields(f.d_out, f.d_in, f.log2K, f.signs, f.idx, f.q, np.zeros_like(f.mu), np.zeros_like(f.delta),
                     f.codebook, f.perm)
    assert oracle.abs_error(z, W + 0.5, e) == 1.0


def test_abs_error_single_channel_and_scale_invariance():
    """With all energy on one original channel c, Eq. 8 is that column's
    relative error, where W^'s column for c is storage column perm^-1(c); and it
    does not change when every energy is scaled by one constant."""
    f, W, e = _abs_case(2)
    Wh = oracle.dequant(f)
    c = 77
    p = int(np.nonzero(f.perm == c)[0][0])
    one = np.zeros(f.d_in)
    one[c] = 3.0
    exp = np.sum((W[:, c] - Wh[:, p]) ** 2) / np.sum(W[:, c] ** 2)
    assert np.isclose(oracle.abs_error(f, W, one), exp, rtol=1e-13)
    assert np.isclose(oracle.abs_error(f, W, e * 7.25), oracle.abs_error(f, W, e), rtol=1e-13)


def test_abs_select_picks_the_smallest_error():
    """Eq. 9 over candidate encodings of the same W: the exact encoding wins (E = 0);
    among equal errors the earlier candidate is kept."""
    f, _, e = _abs_case(3)
    Wh = oracle.dequant(f)
    W = np.zeros_like(Wh)
    W[:, f.perm] = Wh
    g1, _, _ = _abs_case(4)
    g2, _, _ = _abs_case(5)
    best, errs = oracle.abs_select([g1, f, g2], W, e)
    assert best == 1 and errs[1] == 0.0 and min(errs[0], errs[2]) > 0
    best, errs = oracle.abs_select([g1, g1, f, f], W, e)
    assert best == 2 and errs[0] == errs[1]


def test_encode_rows_is_the_encoders_row_part():
    """The per-row stage on its own (Eq. 6, Eq. 14, Eq. 2 for a given stored
    codebook) reproduces the full encoder's fields exactly when given the
    encoder's permutation, codebook and Eq. 4 weights."""
    for log2K in (4, 6, 8):
        inp, _ = synth.config2(d_out=96, d_in=256, n_samples=2048, iters=3, log2K=log2K)
        ref = oracle.encode(inp)
        om = oracle.omega_columns(inp.energies, ref["perm"], inp.gamma)
        rows = oracle.encode_rows(inp.W, ref["perm"], om, ref["codebook"], log2K)
        for k in rows:
            assert np.array_equal(rows[k], ref[k]), (log2K, k)


def test_moe_combine_closed_forms():
    """Router-weighted combine: one slot with weight 1 is the identity; equal
    slot outputs with weights summing to 1 give that output; a hand-worked
    token (exact in fp16 and fp64); the slots are those of their own token."""
    g = np.random.default_rng(5)
    y = _h(g.standard_normal((6, 32)))
    assert np.array_equal(oracle.moe_combine(y, np.ones((6, 1))), y)
    rows = np.repeat(y[:1], 4, axis=0)
    assert np.array_equal(oracle.moe_combine(rows, np.array([[0.125, 0.375, 0.25, 0.25]])), y[:1])
    # token 0: 0.25 * 1 + 0.75 * 2 = 1.75 ; token 1: 0.5 * -4 + 0.5 * 3 = -0.5
    y2 = _h([[1.0, 0.0], [2.0, 8.0], [-4.0, 1.0], [3.0, 1.0]])
    got = oracle.moe_combine(y2, np.array([[0.25, 0.75], [0.5, 0.5]])).view(np.float16)
    assert np.array_equal(got, np.array([[1.75, 6.0], [-0.5, 1.0]], np.float16))
    # against a direct fp64 sum with one rounding
    w = g.random((3, 2))
    want = _h((w[:, :, None] * y.view(np.float16).astype(np.float64).reshape(3, 2, 32)).sum(axis=1))
    assert np.array_equal(oracle.moe_combine(y, w), want)


def test_mutation_plants_apply_once():
    """Every planted mistake of oracle/mutation_check.py names a passage that
    occurs exactly once in the oracle's source, so the check plants what it
    says (a second copy of a line elsewhere would make the plant ambiguous)."""
    import importlib.util
    import os
    here = os.path.dirname(os.path.abspath(__file__))
    spec = importlib.util.spec_from_file_location("mutation_check", os.path.join(here, "..", "oracle", "mutation_check.py"))
    m = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(m)
    src = open(m.SRC).read()
    assert {n: src.count(a) for n, (a, _) in m.PLANTS.items() if src.count(a) != 1} == {}
