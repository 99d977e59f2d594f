"""Shared helpers for the GPU parity tests (CUDA path through the C ABI vs the CPU oracle)."""
import numpy as np

import oracle
import bit_vector_quantized_sage_b200 as sage

# Acceptance bound per output element: |y - y_ref| <= REL * sum|w_hat||x| + ABS
REL, ABS = 1e-3, 1e-5


def dev_u16(a):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.uint16).view(np.int16)).cuda()


def host_u16(t):
    return t.cpu().numpy().view(np.uint16)


def f16_to_f64(a):
    return np.asarray(a, dtype=np.uint16).view(np.float16).astype(np.float64)


def assert_within_bound(y_gpu_bits, y_ref, bound, what=""):
    y = f16_to_f64(y_gpu_bits)
    err = np.abs(y - y_ref)
    lim = REL * bound + ABS
    bad = err > lim
    assert not bad.any(), (f"{what}: {int(bad.sum())} of {bad.size} outside bound; worst at "
                           f"{np.unravel_index(np.argmax(err - lim), err.shape)}: got {y.flat[np.argmax(err - lim)]}, "
                           f"ref {y_ref.flat[np.argmax(err - lim)]}, bound {lim.flat[np.argmax(err - lim)]}")
    return float(np.max(err / np.maximum(bound, 1e-30)))


def workspace_for(op, mats, M):
    return sage.Workspace(sage.sage_workspace_size(op, mats, M))


def gemv(f, x_bits, M=None, entry="gemv"):
    """Runs sage_gemv / sage_gemm on fields f (packed on the host) and returns y bits."""
    import torch
    M = x_bits.shape[0] if M is None else M
    A = sage.PackedMatrix.from_fields(f)
    x = dev_u16(x_bits)
    y = torch.zeros((M, f.d_out), dtype=torch.int16, device="cuda")
    op = sage.SAGE_OP_GEMV if entry == "gemv" else sage.SAGE_OP_GEMM
    ws = workspace_for(op, A, M)
    getattr(sage, "sage_" + entry)(A, x, M, y, ws)
    torch.cuda.synchronize()
    assert sage.sage_query_status(ws) == sage.SAGE_OK
    return host_u16(y), A, ws
