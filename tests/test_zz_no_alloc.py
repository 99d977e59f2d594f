"""sage_gemv_static (GEMV with the library's built-in scratch, no workspace)
against sage_gemv on the same inputs.  The file name sorts last so that its GPU
test runs after every other test in a full run; it passes on its own too."""
import ctypes as C

import numpy as np
import pytest

import oracle
import synth
import bit_vector_quantized_sage_b200 as sage
from _util import assert_within_bound, dev_u16, gemv, host_u16


@pytest.fixture(scope="module")
def lib():
    from bit_vector_quantized_sage_b200 import build
    build.build()
    return sage.load()


def test_static_rejects_shapes_beyond_its_scratch(lib):
    """A shape whose scratch exceeds 4 MiB is refused on the host, before any
    device call (the pointers below are never dereferenced)."""
    A = sage.sage_matrix(120_000_000, 128, 6, 0x100000, 0x200000, 0x300000, None)
    assert lib.sage_gemv_static(C.byref(A), 0x400000, 1, 0x500000, None) == sage.SAGE_ERR_WORKSPACE
    assert lib.sage_gemv_static(C.byref(A), 0x400000, 9, 0x500000, None) == sage.SAGE_ERR_UNSUPPORTED
    assert lib.sage_gemv_static(C.byref(A), 0x400002, 1, 0x500000, None) == sage.SAGE_ERR_MISALIGNED


def _split_ways(d_out, d_in, sms):
    """CTAs sharing the widest 256-row block under the engine's launch geometry:
    one CTA per SM (at most a quarter as many CTAs as block columns), the block
    columns of the launch split evenly over them."""
    units = ((d_out + 7) // 8 + 31) // 32 * (d_in // 8)
    n_cta = max(1, min(sms, units // 4))
    per_block = d_in // 8
    return min(n_cta, -(-per_block * n_cta // units) + 1)


@pytest.mark.gpu
@pytest.mark.parametrize("d_out,d_in,log2K,M", [(256, 512, 6, 1), (3000, 2560, 5, 1), (1500, 4096, 7, 4),
                                                (64, 9728, 6, 1), (200, 9728, 8, 2)])
def test_static_matches_workspace_entry_twice(lib, d_out, d_in, log2K, M):
    """Two calls in a row (the second relies on the first leaving the scratch's
    counters at zero) give the bits of sage_gemv, within the oracle's bound.  Every
    case splits a block over several CTAs, so the split-K counters and partial sums
    in the scratch are exercised (the last two over the whole GPU)."""
    import torch
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    assert _split_ways(d_out, d_in, sms) >= 2
    g = np.random.default_rng(d_out + M)
    f = synth.random_fields(g, d_out, d_in, log2K)
    f.perm = g.permutation(d_in).astype(np.int32)
    x_bits = synth.activations(g, M, d_in)
    y_ws, A, _ = gemv(f, x_bits)
    y_ref, B = oracle.gemv(f, x_bits)
    x = dev_u16(x_bits)
    for call in range(2):
        y = torch.full((M, d_out), -1, dtype=torch.int16, device="cuda")
        sage.sage_gemv_static(A, x, M, y)
        torch.cuda.synchronize()
        got = host_u16(y)
        assert_within_bound(got, y_ref, B, f"static call {call}")
        assert np.array_equal(got, y_ws), f"static call {call} differs from sage_gemv"
