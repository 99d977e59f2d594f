"""Seeded synthetic inputs for the SAGE packed linear layer.

This module draws random numbers and nothing else: code fields, grid
parameters, codebooks, activations, channel energies, dense weights, routing
and sampling indices.  It contains none of the method's arithmetic (no ESG
permutation, no codeword selection, no radius grid, no packing, no
reconstruction); both the CUDA library's tests/benchmark and the CPU oracle
consume what it returns.

Every workload is identified by a config number; its generator is seeded with
``0x5A6E0000 + config`` (plus stream indices for independent sub-draws), using
NumPy's PCG64 through ``SeedSequence``.

Shapes follow the SAGE paper (SAGE: Pushing 2-Bit Vector-Quantized LLMs toward
Real-World Usability, Sec. 3.1 and App. A.6): subvectors of v = 8 consecutive
input channels, radius groups of G = 128 weights (16 subvectors of a row),
fp16 grid parameters and fp16 codebooks.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import Dict, List, Optional, Tuple

import numpy as np

SEED_BASE = 0x5A6E0000

# The five 18-bit splits (K, V) with log2 K + V = 10 (Sec. 3.3, Eq. 7 gives the
# last three; the remaining two keep the same 10-bit budget).
SPLITS: Tuple[Tuple[int, int], ...] = ((16, 6), (32, 5), (64, 4), (128, 3), (256, 2))

# Qwen3-4B decoder-layer linear shapes (d_out, d_in), hidden size 2560.
QWEN3_4B_LAYER: Tuple[Tuple[str, int, int], ...] = (
    ("q", 4096, 2560),
    ("k", 1024, 2560),
    ("v", 1024, 2560),
    ("o", 2560, 4096),
    ("gate", 9728, 2560),
    ("up", 9728, 2560),
    ("down", 2560, 9728),
)
# Dependency stages of one decoder layer: projections within a stage read the
# same input and can run as one grouped launch.
QWEN3_4B_STAGES: Tuple[Tuple[str, ...], ...] = (("q", "k", "v"), ("o",), ("gate", "up"), ("down",))

# Qwen3-30B-A3B MoE expert shapes (d_out, d_in).
MOE_EXPERTS = 128
MOE_TOPK = 8
MOE_PROJ: Tuple[Tuple[str, int, int], ...] = (("gate", 768, 2048), ("up", 768, 2048), ("down", 2048, 768))


def rng(config: int, *stream: int) -> np.random.Generator:
    """Independent, reproducible generator for (config, stream...)."""
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([SEED_BASE + config, *stream])))


def f16_bits(a) -> np.ndarray:
    """Round to IEEE fp16 (round-to-nearest-even) and return the uint16 bit patterns."""
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64).astype(np.float16).view(np.uint16))


@dataclass
class Fields:
    """Logical SAGE code fields of one matrix (storage / permuted column order).

    signs[o, j]  bit i set => component i of subvector j of row o is negative
    idx[o, j]    direction index z in [0, K)
    q[o, j]      radius code in [0, 2**V)
    mu[o, g], delta[o, g]  fp16 bit patterns of the per-group grid (g = j // 16)
    codebook[k, i]         fp16 bit patterns, K codewords of 8 components
    perm[p]      storage position p holds original input channel perm[p]; None = identity
    """

    d_out: int
    d_in: int
    log2K: int
    signs: np.ndarray
    idx: np.ndarray
    q: np.ndarray
    mu: np.ndarray
    delta: np.ndarray
    codebook: np.ndarray
    perm: Optional[np.ndarray] = None
    name: str = ""

    @property
    def K(self) -> int:
        return 1 << self.log2K

    @property
    def V(self) -> int:
        return 10 - self.log2K


def random_codebook(g: np.random.Generator, K: int) -> np.ndarray:
    """K codewords whose 8 components are |N(0,1)|, L2-normalised in fp64, stored fp16."""
    a = np.abs(g.standard_normal((K, 8)))
    a /= np.sqrt((a * a).sum(axis=1, keepdims=True))
    return f16_bits(a)


def random_fields(
    g: np.random.Generator,
    d_out: int,
    d_in: int,
    log2K: int,
    mu_range=(0.05, 0.2),
    delta_range=(0.005, 0.02),
    name: str = "",
) -> Fields:
    """Uniform random code fields: Bernoulli(1/2) signs, uniform z and q, uniform fp16 mu/delta."""
    assert d_in % 128 == 0 and 4 <= log2K <= 8
    S, G, V = d_in // 8, d_in // 128, 10 - log2K
    signs = g.integers(0, 256, size=(d_out, S), dtype=np.uint8)
    idx = g.integers(0, 1 << log2K, size=(d_out, S), dtype=np.uint16)
    q = g.integers(0, 1 << V, size=(d_out, S), dtype=np.uint8)
    mu = f16_bits(g.uniform(*mu_range, size=(d_out, G)))
    delta = f16_bits(g.uniform(*delta_range, size=(d_out, G)))
    cb = random_codebook(g, 1 << log2K)
    return Fields(d_out, d_in, log2K, signs, idx, q, mu, delta, cb, None, name)


def activations(g: np.random.Generator, M: int, d_in: int) -> np.ndarray:
    """fp16 N(0,1) activations of shape (M, d_in), as uint16 bit patterns."""
    return f16_bits(g.standard_normal((M, d_in)))


def lognormal_energies(g: np.random.Generator, d_in: int, sigma: float = 1.5) -> np.ndarray:
    """Synthetic channel energies e_c ~ LogNormal(0, sigma) (stand-in for E[x_c^2])."""
    return g.lognormal(0.0, sigma, size=d_in)


# ---------------------------------------------------------------------------
# Workloads
# ---------------------------------------------------------------------------


def config0() -> Tuple[Fields, np.ndarray]:
    """Single 256x512 matrix, (K,V) = (64,4), identity permutation, batch 1."""
    g = rng(0)
    f = random_fields(g, 256, 512, 6, name="cfg0")
    x = activations(g, 1, 512)
    return f, x


@dataclass
class LayerSpec:
    mats: List[Fields]
    energies: Dict[str, np.ndarray]
    xs: Dict[str, np.ndarray] = field(default_factory=dict)


def config1(M: int = 1, replica: int = 0) -> LayerSpec:
    """Qwen3-4B-shaped decoder layer: seven matrices, each with its own (K,V) split
    and channel energies e_c ~ LogNormal(0, 1.5) (from which the caller builds the
    ESG permutation).  ``replica`` selects an independent draw of codes."""
    mats, energies, xs = [], {}, {}
    g_split = rng(1, 0)
    splits = [SPLITS[int(i)] for i in g_split.integers(0, len(SPLITS), size=len(QWEN3_4B_LAYER))]
    for n, ((name, d_out, d_in), (K, _V)) in enumerate(zip(QWEN3_4B_LAYER, splits)):
        g = rng(1, 1 + n, replica)
        f = random_fields(g, d_out, d_in, int(K).bit_length() - 1, name=name)
        energies[name] = lognormal_energies(rng(1, 100 + n), d_in, 1.5)
        mats.append(f)
    for s, stage in enumerate(QWEN3_4B_STAGES):
        d_in = dict((nm, di) for nm, _, di in QWEN3_4B_LAYER)[stage[0]]
        xs[stage[0]] = activations(rng(1, 200 + s, replica), M, d_in)
    return LayerSpec(mats, energies, xs)


# Attention geometry of the Qwen3-4B-shaped layer: 32 query heads and 8
# key/value heads of dimension 128 (q 4096 = 32 x 128, k / v 1024 = 8 x 128).
QWEN3_4B_HEADS = (32, 8, 128)


@dataclass
class DecoderInputs:
    h: np.ndarray          # fp16 bits (M, hidden): the layer's input rows
    attn_norm: np.ndarray  # fp16 bits (hidden,)
    mlp_norm: np.ndarray   # fp16 bits (hidden,)
    eps: float


def decoder_inputs(config: int, M: int, hidden: int, replica: int = 0) -> DecoderInputs:
    """Inputs of a decoder layer around its projections: h ~ N(0, 1) and RMSNorm
    weights ~ U(0.5, 1.5), all fp16; eps = 1e-6."""
    g = rng(config, 300, replica)
    return DecoderInputs(f16_bits(g.standard_normal((M, hidden))), f16_bits(g.uniform(0.5, 1.5, hidden)),
                         f16_bits(g.uniform(0.5, 1.5, hidden)), 1e-6)


def small_layer(seed: int, hidden: int = 256, heads=(4, 2, 64), inter: int = 512) -> LayerSpec:
    """A small decoder layer with the Qwen3 structure (for fast parity tests):
    each projection draws its split from the five 18-bit splits."""
    nh, nkv, hd = heads
    shapes = (("q", nh * hd, hidden), ("k", nkv * hd, hidden), ("v", nkv * hd, hidden), ("o", hidden, nh * hd),
              ("gate", inter, hidden), ("up", inter, hidden), ("down", hidden, inter))
    g = np.random.default_rng(seed)
    mats, energies = [], {}
    for name, d_out, d_in in shapes:
        K, _V = SPLITS[int(g.integers(0, len(SPLITS)))]
        mats.append(random_fields(g, d_out, d_in, int(K).bit_length() - 1, name=name))
        energies[name] = lognormal_energies(g, d_in, 1.5)
    return LayerSpec(mats, energies, {})


@dataclass
class EncoderInputs:
    W: np.ndarray            # fp64 (d_out, d_in), original channel order
    energies: np.ndarray     # fp64 (d_in,)
    sample: np.ndarray       # int64 subvector ids (row-major over (d_out, d_in/8)), no repeats
    init: np.ndarray         # int64 positions into ``sample`` of the K initial codewords
    gamma: float
    iters: int
    log2K: int


def config2(d_out: int = 4096, d_in: int = 4096, n_samples: int = 65536, iters: int = 10,
            log2K: int = 6, seed_stream: int = 0) -> Tuple[EncoderInputs, np.ndarray]:
    """Weight-derived layer: W = N(0, 0.02) scaled per input channel by LogNormal(0, 0.5),
    energies LogNormal(0, 1.5), gamma = 0.75; plus the random draws the encoder needs
    (sampled subvector ids and initial-codeword picks)."""
    g = rng(2, seed_stream)
    scale = g.lognormal(0.0, 0.5, size=d_in)
    W = g.normal(0.0, 0.02, size=(d_out, d_in)) * scale[None, :]
    e = lognormal_energies(g, d_in, 1.5)
    n_sv = d_out * d_in // 8
    n_samples = min(n_samples, n_sv)
    sample = np.sort(g.choice(n_sv, size=n_samples, replace=False)).astype(np.int64)
    init = g.permutation(n_samples)[: 1 << log2K].astype(np.int64)
    x = activations(g, 1, d_in)
    return EncoderInputs(W, e, sample, init, 0.75, iters, log2K), x


def config3(M: int) -> Tuple[Fields, np.ndarray]:
    """Qwen3-8B-shaped MLP up-projection 4096 -> 12288, (K,V) = (32,5), batch M."""
    g = rng(3, 0)
    f = random_fields(g, 12288, 4096, 5, name="up8b")
    x = activations(rng(3, 1, M), M, 4096)
    return f, x


@dataclass
class MoESpec:
    T: int
    routes: np.ndarray                 # (T, 8) distinct expert ids per token
    x: np.ndarray                      # (T, 2048) fp16 bits, input of gate/up
    x_down: np.ndarray                 # (T*8, 768) fp16 bits, one fresh input per (token, slot)
    splits: np.ndarray                 # (128, 3) log2K per (expert, projection)

    def expert(self, e: int, proj: int) -> Fields:
        name, d_out, d_in = MOE_PROJ[proj]
        return random_fields(rng(4, 10 + e, proj), d_out, d_in, int(self.splits[e, proj]),
                             name=f"e{e}.{name}")

    def active(self) -> np.ndarray:
        return np.unique(self.routes)


def config4(T: int) -> MoESpec:
    """Qwen3-30B-A3B-shaped MoE layer: 128 experts (gate/up 2048->768, down 768->2048),
    top-8 routing drawn uniformly without replacement per token."""
    g = rng(4, 0)
    splits = np.array([[int(SPLITS[int(i)][0]).bit_length() - 1 for i in row]
                       for row in g.integers(0, len(SPLITS), size=(MOE_EXPERTS, 3))], dtype=np.int32)
    gt = rng(4, 1, T)
    routes = np.stack([gt.permutation(MOE_EXPERTS)[:MOE_TOPK] for _ in range(T)]).astype(np.int32)
    x = activations(gt, T, 2048)
    x_down = activations(gt, T * MOE_TOPK, 768)
    return MoESpec(T, routes, x, x_down, splits)


@dataclass
class QdqInputs:
    """Training state of one matrix for the continuous-parameter decode: codebook
    angle logits [K][7], radius logits [d_out][d_in/8] (r~ = softplus(rho)) and
    the retained discrete assignments (signs, codeword indices)."""
    d_out: int
    d_in: int
    log2K: int
    alpha: np.ndarray
    rho: np.ndarray
    signs: np.ndarray
    idx: np.ndarray


def qdq_inputs(seed: int, d_out: int, d_in: int, log2K: int) -> QdqInputs:
    """alpha ~ N(0, 1); rho ~ N(-2, 0.5), so that softplus(rho) ~ 0.13 with a
    spread, about the radius of an 8-weight subvector of N(0, 0.02^2) weights
    (0.02 x sqrt(8) = 0.057) to a few times it; Bernoulli(1/2) signs; uniform
    codeword indices."""
    g = rng(5, seed)
    S = d_in // 8
    K = 1 << log2K
    return QdqInputs(d_out, d_in, log2K,
                     g.standard_normal((K, 7)).astype(np.float32),
                     (g.standard_normal((d_out, S)) * 0.5 - 2.0).astype(np.float32),
                     g.integers(0, 256, (d_out, S), dtype=np.uint8),
                     g.integers(0, K, (d_out, S)).astype(np.uint16))
