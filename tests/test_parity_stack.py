"""GPU parity of RMS normalisation and of chained MoE layers (the decode stack):
each layer normalises the running hidden state, routes and runs its experts,
and adds its output to the state.  Checked layer by layer with teacher
forcing: the oracle gets the GPU's own input to the layer, so every layer is
held to the single-layer tolerance instead of an accumulated one."""
import numpy as np
import pytest
import torch

import oracle
from quantised_expert_ffn_moe_b200 import moeq, synth

from moe_testutil import GpuLayer, assert_parity

pytestmark = pytest.mark.gpu

EPS = 1e-6


def _rmsnorm_ref(xb):
    """Oracle normalisation of bf16 rows (uint16 bits [T][H]) -> fp64."""
    return np.stack([oracle.rmsnorm(oracle.bf16_to_f64(r), EPS) for r in xb])


def _check_rmsnorm(x, y):
    """y (GPU bf16) is the oracle's fp64 result rounded to bf16: equal to the
    rounded value, or (only at a rounding tie within the fp64 rounding of the
    scale) one ulp from it; always within a bf16 half-ulp."""
    ref = _rmsnorm_ref(synth.to_np_bits(x))
    g = y.double().cpu().numpy()
    assert np.all(np.abs(g - ref) <= np.abs(ref) * 2.0 ** -8 * (1 + 1e-9) + 1e-30)
    exact = oracle.bf16_to_f64(oracle.f64_to_bf16(ref))
    assert np.mean(g == exact) > 0.9999


@pytest.mark.parametrize("T,H", [(1, 4096), (37, 4096), (5, 1000), (3, 8)])
def test_rmsnorm(T, H):
    g = torch.Generator(device="cuda").manual_seed(T * 7919 + H)
    x = (torch.randn((T, H), generator=g, device="cuda") * 3.0).to(torch.bfloat16)
    _check_rmsnorm(x, moeq.rmsnorm(x, EPS))


def test_rmsnorm_in_place_and_degenerate_rows():
    """out == x; a zero row (normalises to zero), a row of one repeated value
    (normalises to +-1 up to eps), a row with a single nonzero entry."""
    H = 512
    x = torch.randn((4, H), device="cuda").to(torch.bfloat16)
    x[0] = 0
    x[1] = -3.25
    x[2] = 0
    x[2, 17] = 100.0
    x0 = x.clone()
    moeq.rmsnorm(x, EPS, out=x)
    _check_rmsnorm(x0, x)
    assert torch.all(x[0] == 0)
    assert torch.all(x[1] == -1.0)
    assert x[2, 17].item() == pytest.approx(np.sqrt(H), rel=2 ** -8)
    moeq.rmsnorm(x[:0], EPS)  # no tokens: nothing launched


def test_rmsnorm_rejects_bad_sizes():
    x = torch.zeros((2, 12), device="cuda", dtype=torch.bfloat16)
    with pytest.raises(moeq.MoeError):
        moeq.rmsnorm(x, EPS)
    with pytest.raises(moeq.MoeError):
        moeq.rmsnorm(torch.zeros((2, 16), device="cuda", dtype=torch.bfloat16), -1.0)


@pytest.mark.parametrize("T", [1, 5, 64, 100])
def test_normed_entry_matches_rmsnorm_then_layer(T):
    """moe_layer_forward_normed (normalisation inside the router kernel at
    decode sizes, a kernel of its own from 64 tokens on) gives the very bits
    of moe_rmsnorm followed by moe_layer_forward."""
    shape = synth.LayerShape(hidden=2048, inter=256, n_experts=32, top_k=4)
    L = GpuLayer(shape, 71)
    ws = moeq.workspace(L.desc, T)
    h = synth.make_tokens(shape, T, 72, device="cuda", on_sphere=False) * 3
    xn = moeq.rmsnorm(h, EPS)
    out1, idx1, w1 = L.forward(xn, h, ws)
    xh = torch.empty_like(h)
    idx2 = torch.empty_like(idx1)
    w2 = torch.empty_like(w1)
    out2 = moeq.layer_forward_normed(L.desc, h, L.lay.router, L.slots, ws, EPS, shared_gate=L.lay.shared_gate,
                                     xhat_out=xh, topk_idx=idx2, topk_w=w2)
    assert torch.equal(xh, xn)
    assert torch.equal(idx1, idx2) and torch.equal(w1, w2)
    assert torch.equal(out1, out2)
    # in place (out = h), no x-hat copy
    h2 = h.clone()
    moeq.layer_forward_normed(L.desc, h2, L.lay.router, L.slots, ws, EPS, shared_gate=L.lay.shared_gate, out=h2)
    assert torch.equal(h2, out1)
    assert moeq.device_status(ws) == (0, 0)


def _run_stack_teacher_forced(shape, n_layers, T, seed, repeat_bias=False):
    layers = [GpuLayer(shape, seed + l) for l in range(n_layers)]
    ws = moeq.workspace(layers[0].desc, T)
    h0 = synth.make_tokens(shape, T, seed, device="cuda", on_sphere=False)
    bias = None
    if repeat_bias:
        bias = [torch.tensor(synth.repeat_logit_bias(shape.n_experts, shape.top_k, T, 0.27, seed + l)[0],
                             device="cuda") for l in range(n_layers)]
    spec = [(L.desc, L.lay.router, L.slots, L.lay.shared_gate) for L in layers]
    xhat, topk, states = [], [], [h0.clone()]
    h = h0.clone()
    # one layer at a time, keeping each layer's input state
    for l in range(n_layers):
        moeq.stack_forward(spec[l:l + 1], h, ws, EPS, None if bias is None else bias[l:l + 1],
                           xhat=xhat, topk=topk)
        states.append(h.clone())
    assert moeq.device_status(ws) == (0, 0)
    for l, L in enumerate(layers):
        _check_rmsnorm(states[l], xhat[l])
        ref = L.oracle_forward(xhat[l], states[l], logit_bias=None if bias is None else bias[l])
        assert_parity(states[l + 1], topk[l][0], topk[l][1], *ref[:3])
    # the whole chain in one call gives the same bits as the layer-by-layer run
    h2 = h0.clone()
    moeq.stack_forward(spec, h2, ws, EPS, bias)
    assert torch.equal(h2, states[-1])
    return states


def test_stack_decode_teacher_forced():
    """Four chained layers, three tokens (decode path), plain routing."""
    shape = synth.LayerShape(hidden=2048, inter=256, n_experts=64, top_k=6)
    _run_stack_teacher_forced(shape, 4, 3, 101)


def test_stack_decode_repeat_routing():
    """Three layers, eight consecutive tokens whose expert sets repeat 27% of
    the time from one token to the next (the decode-loop routing)."""
    shape = synth.LayerShape(hidden=2048, inter=256, n_experts=64, top_k=6)
    _run_stack_teacher_forced(shape, 3, 8, 202, repeat_bias=True)


def test_stack_prefill_teacher_forced():
    """Two chained layers over 64 tokens (the tensor-core path)."""
    shape = synth.LayerShape(hidden=2048, inter=256, n_experts=32, top_k=4)
    _run_stack_teacher_forced(shape, 2, 64, 303)


def test_stack_397b_16_layers_sampled():
    """The full decode stack: 16 layers of the hidden-4096, 512 + 1 expert,
    top-10, 4-bit shape (~58 GB resident), four consecutive tokens with 27%
    expert repeat.  Routing of every (layer, token) against the oracle on the
    GPU's own normalised inputs; outputs of sampled (layer, token) pairs
    teacher-forced against the oracle."""
    shape = synth.DECODE_397B
    n_layers, T = 16, 4
    layers = [GpuLayer(shape, 500 + l) for l in range(n_layers)]
    ws = moeq.workspace(layers[0].desc, 1)
    h = synth.make_tokens(shape, T, 17, device="cuda", on_sphere=False)
    bias = [torch.tensor(synth.repeat_logit_bias(shape.n_experts, shape.top_k, T, 0.27, 60 + l)[0],
                         device="cuda") for l in range(n_layers)]
    spec = [(L.desc, L.lay.router, L.slots, L.lay.shared_gate) for L in layers]
    states = [[None] * (n_layers + 1) for _ in range(T)]
    xhat = [[None] * n_layers for _ in range(T)]
    topk = [[None] * n_layers for _ in range(T)]
    for t in range(T):  # one token at a time through all layers (the decode loop)
        ht = h[t:t + 1].clone()
        states[t][0] = ht.clone()
        for l in range(n_layers):
            xs, tk = [], []
            moeq.stack_forward(spec[l:l + 1], ht, ws, EPS, [bias[l][t:t + 1]], xhat=xs, topk=tk)
            xhat[t][l], topk[t][l] = xs[0], tk[0]
            states[t][l + 1] = ht.clone()
    assert moeq.device_status(ws) == (0, 0)
    k = shape.top_k
    for l, L in enumerate(layers):
        wr = L.router_np()
        for t in range(T):
            _check_rmsnorm(states[t][l], xhat[t][l])
            xb = synth.to_np_bits(xhat[t][l])[0]
            lb = bias[l][t].cpu().numpy().astype(np.float64)
            _, ri, rw = oracle.route(oracle.bf16_to_f64(xb), wr, k, lb)
            assert np.array_equal(topk[t][l][0].cpu().numpy()[0], ri), (l, t)
            assert np.allclose(topk[t][l][1].cpu().numpy()[0], rw, rtol=1e-6, atol=1e-7)
    for l, t in [(0, 0), (0, 1), (7, 2), (15, 3)]:
        ref = layers[l].oracle_forward(xhat[t][l], states[t][l], logit_bias=bias[l][t:t + 1])
        assert_parity(states[t][l + 1], topk[t][l][0], topk[t][l][1], *ref[:3])
