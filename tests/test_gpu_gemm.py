"""GPU parity of the tensor-core path (sage_gemm, batch 9..256) against the CPU
oracle, element by element, through the C ABI."""
import numpy as np
import pytest

import oracle
import synth
import bit_vector_quantized_sage_b200 as sage
from _util import assert_within_bound, dev_u16, gemv, host_u16, workspace_for

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


@pytest.mark.parametrize("M", [9, 16, 33, 64, 128, 256])
def test_gemm_batches_ragged(M):
    """Ragged rows (a partial last 256-row block), several radius groups, permuted x."""
    f = _fields(1000 + M, 520, 1024, [4, 5, 6, 7, 8][M % 5])
    x = synth.activations(np.random.default_rng(M), M, 1024)
    y, _, _ = gemv(f, x, entry="gemm")
    y_ref, B = oracle.gemv(f, x)
    assert_within_bound(y, y_ref, B, f"M={M}")


@pytest.mark.parametrize("log2K", [4, 5, 6, 7, 8])
def test_gemm_all_splits(log2K):
    for n, (d_out, d_in, M) in enumerate([(8, 128, 16), (256, 256, 24), (1000, 2560, 40)]):
        f = _fields(50 * log2K + n, d_out, d_in, log2K, perm=(n != 1))
        x = synth.activations(np.random.default_rng(n + 7), M, d_in)
        y, _, _ = gemv(f, x, entry="gemm")
        y_ref, B = oracle.gemv(f, x)
        assert_within_bound(y, y_ref, B, f"K=2^{log2K} {d_out}x{d_in} M={M}")


def test_gemm_deterministic_and_status_clean():
    import torch
    f = _fields(3, 3000, 2048, 5)
    x_bits = synth.activations(np.random.default_rng(3), 48, 2048)
    y1, A, ws = gemv(f, x_bits, entry="gemm")
    x = dev_u16(x_bits)
    y = torch.zeros((48, 3000), dtype=torch.int16, device="cuda")
    sage.sage_gemm(A, x, 48, y, ws)
    torch.cuda.synchronize()
    assert sage.sage_query_status(ws) == sage.SAGE_OK
    assert np.array_equal(host_u16(y), y1)


@pytest.mark.parametrize("M,entry", [(1, "gemv"), (2, "gemv"), (4, "gemv"), (8, "gemv"), (16, "gemm"), (128, "gemm")])
def test_config3_full_rows(M, entry):
    """The 4096 -> 12288 up-projection at full size, every output row against the
    oracle: batch 1-8 through the GEMV engine, 16 and 128 through the tcgen05 path."""
    f, x = synth.config3(M)
    y, _, _ = gemv(f, x, entry=entry)
    y_ref, B = oracle.gemv(f, x)
    assert_within_bound(y, y_ref, B, f"config3 M={M} ({entry})")


def test_config3_back_to_back_replicas():
    """The launch form the benchmark times: a CUDA graph of the GEMV over copies of the
    planes back to back (programmatic dependent launch between them, one workspace).
    Each copy's output, captured in its own buffer, is bit-identical to an eager call."""
    import torch
    f, xb = synth.config3(1)
    A0 = sage.PackedMatrix.from_fields(f)
    As = [A0] + [sage.PackedMatrix(A0.d_out, A0.d_in, A0.log2K, A0.main.clone(), A0.meta.clone(),
                                   A0.codebook.clone(), None, "copy") for _ in range(3)]
    x = dev_u16(xb)
    ys = [torch.zeros((1, f.d_out), dtype=torch.int16, device="cuda") for _ in As]
    ws = workspace_for(sage.SAGE_OP_GEMV, A0, 1)
    s = torch.cuda.Stream()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        for A, y in zip(As, ys):
            sage.sage_gemv(A, x, 1, y, ws, s)
        s.synchronize()
        eager = [host_u16(y) for y in ys]
        for y in ys:
            y.zero_()
        with torch.cuda.graph(g, stream=s):
            for A, y in zip(As, ys):
                sage.sage_gemv(A, x, 1, y, ws, torch.cuda.current_stream())
        for _ in range(3):
            g.replay()
    torch.cuda.synchronize()
    assert sage.sage_query_status(ws) == sage.SAGE_OK
    for y, e in zip(ys, eager):
        assert np.array_equal(host_u16(y), e)
    y_ref, B = oracle.gemv(f, xb)
    assert_within_bound(eager[-1], y_ref, B, "config3 last copy")
    del g


@pytest.mark.parametrize("M", [16, 32, 64, 128])
def test_config3_sampled_rows(M):
    """Qwen3-8B-shaped up-projection 4096 -> 12288, (K,V) = (32,5), at full size;
    the oracle checks row ranges at the start, across block boundaries and at the end."""
    f, x = synth.config3(M)
    y, _, _ = gemv(f, x, entry="gemm")
    for r0, r1 in ((0, 40), (250, 262), (6140, 6160), (12230, 12288)):
        y_ref, B = oracle.gemv(f, x, rows=(r0, r1))
        assert_within_bound(y[:, r0:r1], y_ref[:, r0:r1], B[:, r0:r1], f"config3 M={M} rows {r0}:{r1}")


@pytest.mark.parametrize("log2K", [4, 6, 8])
def test_gemm_reconstruction_within_one_ulp(log2K):
    """The tensor-core path's own fp16 W_hat tiles, read back through one-hot
    inputs: batch row m selects original channel c_m, so y[m] is column
    pi^-1(c_m) of the tile-reconstructed W_hat times 1.0 summed in fp32 with
    zeros -- exactly its fp16 value.  Every such column is within 1 fp16 ulp
    of the oracle's W_hat rounded to fp16 (the bar for reconstructed
    weights), across all 256-row blocks and two radius groups."""
    g = np.random.default_rng(300 + log2K)
    d_out, d_in, M = 520, 256, 32
    f = synth.random_fields(g, d_out, d_in, log2K)
    f.perm = g.permutation(d_in).astype(np.int32)
    chans = g.choice(d_in, M, replace=False)
    x = np.zeros((M, d_in))
    x[np.arange(M), chans] = 1.0
    y, _, _ = gemv(f, synth.f16_bits(x), entry="gemm")
    ref16 = oracle.round_half(oracle.dequant(f))  # [d_out][storage position]
    pos = np.array([int(np.nonzero(f.perm == c)[0][0]) for c in chans])
    got = y.astype(np.int32)                      # [M][d_out]
    ref = ref16[:, pos].T.astype(np.int32)
    same_sign = ((got ^ ref) & 0x8000) == 0
    dist = np.where(same_sign, np.abs(got - ref), np.abs((got & 0x7FFF) + (ref & 0x7FFF)))
    assert dist.max() <= 1, (log2K, int(dist.max()))
