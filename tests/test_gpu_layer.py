"""The fused decoder layer (sage_decoder_layer_forward): one launch of the four
dependent projection stages with RMSNorm, single-position attention, residual
and SiLU * up fused around them (Sec. 3.5), checked stage by stage against the
oracle applied to the GPU's own previous-stage outputs, so that each stage is
held to the per-element bound on its own inputs."""
import numpy as np
import pytest

import oracle
import synth
import bit_vector_quantized_sage_b200 as sage
from _util import assert_within_bound, dev_u16, host_u16

NAMES = ("q", "k", "v", "o", "gate", "up", "down")


def _run_layer(spec, heads, M, config=9, replica=0):
    import torch
    nh, nkv, hd = heads
    mats, fields = {}, {}
    for f in spec.mats:
        f.perm = sage.sage_esg_permutation(spec.energies[f.name])
        fields[f.name] = f
        mats[f.name] = sage.PackedMatrix.from_fields(f)
    hidden = fields["q"].d_in
    inp = synth.decoder_inputs(config, M, hidden, replica)
    outs = {n: torch.zeros((M, fields[n].d_out), dtype=torch.int16, device="cuda") for n in NAMES}
    outs["h_out"] = torch.zeros((M, hidden), dtype=torch.int16, device="cuda")
    layer = sage.DecoderLayer(mats, dev_u16(inp.attn_norm), dev_u16(inp.mlp_norm), nh, nkv, hd, inp.eps, outs, M)
    h = dev_u16(inp.h)
    layer(h)
    torch.cuda.synchronize()
    assert sage.sage_query_status(layer.ws) == sage.SAGE_OK
    got = {n: host_u16(t) for n, t in outs.items()}
    return fields, inp, got, layer, h, outs


def _check_layer(fields, inp, got, heads):
    nh, nkv, hd = heads
    worst = {}
    x1 = oracle.rmsnorm(inp.h, inp.attn_norm, inp.eps)
    for n in ("q", "k", "v"):
        y, B = oracle.gemv(fields[n], x1)
        worst[n] = assert_within_bound(got[n], y, B, n)
    a = oracle.attend_one_position(got["v"], nh, nkv, hd)
    y, B = oracle.gemv(fields["o"], a)
    worst["o"] = assert_within_bound(got["o"], y, B, "o")
    r = oracle.add(inp.h, got["o"])
    x3 = oracle.rmsnorm(r, inp.mlp_norm, inp.eps)
    for n in ("gate", "up"):
        y, B = oracle.gemv(fields[n], x3)
        worst[n] = assert_within_bound(got[n], y, B, n)
    m = oracle.silu_mul(got["gate"], got["up"])
    y, B = oracle.gemv(fields["down"], m)
    worst["down"] = assert_within_bound(got["down"], y, B, "down")
    # the residual stream out is an exact fp16 sum of exact fp16 operands
    assert np.array_equal(got["h_out"], oracle.add(r, got["down"]))
    return worst


@pytest.mark.gpu
@pytest.mark.parametrize("M", [1, 3])
def test_small_layer_fused(M):
    heads = (4, 2, 64)
    spec = synth.small_layer(17 + M)
    fields, inp, got, *_ = _run_layer(spec, heads, M)
    _check_layer(fields, inp, got, heads)


@pytest.mark.gpu
def test_small_layer_deterministic_and_graph_replay():
    """Identical bits on a rerun and inside a CUDA graph (the way the bench
    times it), with the workspace counts restored between calls."""
    import torch
    heads = (4, 2, 64)
    fields, inp, got, layer, h, outs = _run_layer(synth.small_layer(5), heads, 1)
    for t in outs.values():
        t.zero_()
    s = torch.cuda.Stream()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        layer(h, s)  # warm-up on the capture stream
        s.synchronize()
        with torch.cuda.graph(g, stream=s):
            layer(h, torch.cuda.current_stream())
        for _ in range(3):
            g.replay()
    torch.cuda.synchronize()
    assert sage.sage_query_status(layer.ws) == sage.SAGE_OK
    for n, t in outs.items():
        assert np.array_equal(host_u16(t), got[n]), n
    del g


@pytest.mark.gpu
def test_qwen3_4b_layer_fused():
    """The bench's workload: the Qwen3-4B-shaped layer (config 1 codes) at batch 1."""
    spec = synth.config1()
    fields, inp, got, *_ = _run_layer(spec, synth.QWEN3_4B_HEADS, 1, config=1)
    _check_layer(fields, inp, got, synth.QWEN3_4B_HEADS)


@pytest.mark.gpu
def test_qwen3_4b_two_layers_chained_in_a_graph():
    """The launch form the benchmark times, with a real dependency between
    layers: two Qwen3-4B-shaped fused layers in one CUDA graph, the second
    reading the first's h_out (programmatic dependent launch between them, one
    workspace).  Every output is bit-identical to eager calls, and the second
    layer is held to the bound against the oracle on the first layer's GPU
    output."""
    import types
    import torch
    heads = synth.QWEN3_4B_HEADS
    nh, nkv, hd = heads
    layers, fields_by_layer = [], []
    inp = synth.decoder_inputs(1, 1, 2560)
    ws = None
    outs_all = []
    for replica in (0, 1):
        spec = synth.config1(1, replica)
        mats, fields = {}, {}
        for f in spec.mats:
            f.perm = sage.sage_esg_permutation(spec.energies[f.name])
            fields[f.name] = f
            mats[f.name] = sage.PackedMatrix.from_fields(f)
        outs = {n: torch.zeros((1, fields[n].d_out), dtype=torch.int16, device="cuda") for n in NAMES}
        outs["h_out"] = torch.zeros((1, 2560), dtype=torch.int16, device="cuda")
        lay = sage.DecoderLayer(mats, dev_u16(inp.attn_norm), dev_u16(inp.mlp_norm), nh, nkv, hd, inp.eps, outs, 1, ws)
        ws = lay.ws
        layers.append(lay)
        fields_by_layer.append(fields)
        outs_all.append(outs)
    h0 = dev_u16(inp.h)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        layers[0](h0, s)
        layers[1](outs_all[0]["h_out"], s)
        s.synchronize()
        eager = [{n: host_u16(t) for n, t in o.items()} for o in outs_all]
        for o in outs_all:
            for t in o.values():
                t.zero_()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s):
            layers[0](h0, torch.cuda.current_stream())
            layers[1](outs_all[0]["h_out"], torch.cuda.current_stream())
        for _ in range(2):
            g.replay()
    torch.cuda.synchronize()
    assert sage.sage_query_status(ws) == sage.SAGE_OK
    for o, e in zip(outs_all, eager):
        for n, t in o.items():
            assert np.array_equal(host_u16(t), e[n]), n
    _check_layer(fields_by_layer[0], inp, eager[0], heads)
    inp1 = types.SimpleNamespace(h=eager[0]["h_out"], attn_norm=inp.attn_norm, mlp_norm=inp.mlp_norm, eps=inp.eps)
    _check_layer(fields_by_layer[1], inp1, eager[1], heads)
    del g
