"""GPU parity of the decode path (through the C ABI) against the fp64 CPU
oracle: top-k ids bit-exact, routing weights to fp32 precision, layer output
within relative L2 2e-3 per token."""
import numpy as np
import pytest
import torch

import oracle
from quantised_expert_ffn_moe_b200 import moeq, synth

from moe_testutil import GpuLayer, assert_parity, rel_l2, REL_L2_TOL

pytestmark = pytest.mark.gpu


def _ws(layer, T):
    return moeq.workspace(layer.desc, T)


def _tokens(shape, T, seed):
    return synth.make_tokens(shape, T, seed, device="cuda")


@pytest.mark.parametrize("seed", range(12))
def test_tiny_layer(seed):
    L = GpuLayer(synth.TINY, seed)
    ws = _ws(L, 1)
    x = _tokens(synth.TINY, 1, seed)
    out, idx, w = L.forward(x, x, ws)
    ref = L.oracle_forward(x, x)
    assert_parity(out, idx, w, *ref[:3])
    assert moeq.device_status(ws) == (0, 0)


@pytest.fixture(scope="module")
def decode_layer():
    return GpuLayer(synth.DECODE_397B, 1234)


def test_decode_397b_layer_single_tokens(decode_layer):
    L = decode_layer
    ws = _ws(L, 1)
    errs = []
    for s in range(3):
        x = _tokens(L.shape, 1, 100 + s)
        out, idx, w = L.forward(x, x, ws)
        errs.append(assert_parity(out, idx, w, *L.oracle_forward(x, x)[:3]))
    assert moeq.device_status(ws) == (0, 0)
    print("rel-L2", np.concatenate(errs))


def test_decode_397b_layer_multi_token_and_residual(decode_layer):
    L = decode_layer
    ws = _ws(L, 4)
    x = _tokens(L.shape, 3, 7)
    resid = synth.make_tokens(L.shape, 3, 8, device="cuda", on_sphere=False)
    out, idx, w = L.forward(x, resid, ws)
    assert_parity(out, idx, w, *L.oracle_forward(x, resid)[:3])


def test_decode_397b_routing_many_tokens(decode_layer):
    """moe_route alone over 256 tokens: ids bit-exact, weights to fp32."""
    L = decode_layer
    T = 256
    ws = _ws(L, T)
    x = _tokens(L.shape, T, 55)
    idx, w = moeq.route(L.desc, x, L.lay.router, ws)
    xb, wr = synth.to_np_bits(x), L.router_np()
    idx, w = idx.cpu().numpy(), w.cpu().numpy()
    for t in range(T):
        _, ri, rw = oracle.route(oracle.bf16_to_f64(xb[t]), wr, L.shape.top_k)
        assert np.array_equal(idx[t], ri), t
        assert np.allclose(w[t], rw, rtol=1e-6, atol=1e-7)


@pytest.mark.parametrize("shape", [synth.DECODE_2BIT, synth.DECODE_2BIT_K4], ids=["k3", "k4"])
def test_2bit_layer(shape):
    L = GpuLayer(shape, 77)
    ws = _ws(L, 2)
    x = _tokens(shape, 2, 5)
    out, idx, w = L.forward(x, x, ws)
    assert_parity(out, idx, w, *L.oracle_forward(x, x)[:3])


def test_split_entry_points_match_oracle(decode_layer):
    """moe_route -> moe_expert_ffn_q4 -> moe_combine_residual."""
    L = decode_layer
    ws = _ws(L, 2)
    x = _tokens(L.shape, 2, 31)
    idx, w = moeq.route(L.desc, x, L.lay.router, ws)
    y = moeq.expert_ffn_q4(L.desc, x, L.slots, idx, w, ws)
    out = moeq.combine_residual(L.desc, y, x, x, shared_gate=L.lay.shared_gate)
    ref_out, ref_idx, ref_w, _ = L.oracle_forward(x, x)
    assert_parity(out, idx, w, ref_out, ref_idx, ref_w)


# --------------------------------------------------------------- edge cases

EDGE_SHAPES = {
    "ragged_H320_I192": synth.LayerShape(hidden=320, inter=192, n_experts=8, top_k=2),
    "E40_not_mult_32": synth.LayerShape(hidden=256, inter=128, n_experts=40, top_k=5),
    "k1": synth.LayerShape(hidden=256, inter=256, n_experts=16, top_k=1, has_shared=False),
    "k_equals_E": synth.LayerShape(hidden=256, inter=128, n_experts=8, top_k=8),
    "no_shared_gate": synth.LayerShape(hidden=512, inter=256, n_experts=16, top_k=4, shared_gate=False),
    "q2_ragged": synth.LayerShape(hidden=448, inter=320, n_experts=12, top_k=3, bits=2),
    "k32_E1024": synth.LayerShape(hidden=256, inter=128, n_experts=1024, top_k=32),
    "wide_H8192": synth.LayerShape(hidden=8192, inter=512, n_experts=16, top_k=2),
    "deep_I4096": synth.LayerShape(hidden=512, inter=4096, n_experts=8, top_k=2, bits=2),
}


@pytest.mark.parametrize("name", list(EDGE_SHAPES))
def test_edge_shapes(name):
    shape = EDGE_SHAPES[name]
    L = GpuLayer(shape, 3)
    ws = _ws(L, 5)
    x = _tokens(shape, 5, 9)
    out, idx, w = L.forward(x, x, ws)
    assert_parity(out, idx, w, *L.oracle_forward(x, x)[:3])
    assert moeq.device_status(ws) == (0, 0)


def test_zero_tokens():
    L = GpuLayer(synth.TINY, 0)
    ws = _ws(L, 1)
    x = torch.empty((0, 256), dtype=torch.bfloat16, device="cuda")
    out = moeq.layer_forward(L.desc, x, x, L.lay.router, L.slots, ws)
    assert out.shape == (0, 256)


def test_all_tokens_to_one_expert():
    shape = synth.LayerShape(hidden=512, inter=256, n_experts=32, top_k=4)
    L = GpuLayer(shape, 4)
    T = 6
    ws = _ws(L, T)
    x = _tokens(shape, T, 2)
    bias = torch.zeros((T, 32), dtype=torch.float32, device="cuda")
    bias[:, 17] = 30.0
    out, idx, w = L.forward(x, x, ws, logit_bias=bias)
    assert (idx[:, 0] == 17).all()
    assert_parity(out, idx, w, *L.oracle_forward(x, x, logit_bias=bias)[:3])


def test_zero_scale_experts():
    shape = synth.LayerShape(hidden=512, inter=256, n_experts=8, top_k=2)
    tab = synth.make_experts(shape, 6, "cuda", scale_range=(0.0, 0.0))
    L = GpuLayer(shape, 6, experts=tab)
    ws = _ws(L, 2)
    x = _tokens(shape, 2, 1)
    out, idx, w = L.forward(x, x, ws)
    assert_parity(out, idx, w, *L.oracle_forward(x, x)[:3])


def test_workspace_reuse_across_token_counts(decode_layer):
    """Counters are left at zero by every call, whatever T the call used."""
    L = decode_layer
    ws = _ws(L, 5)
    for T in (3, 1, 5, 2):
        x = _tokens(L.shape, T, 200 + T)
        out, idx, w = L.forward(x, x, ws)
        ref = L.oracle_forward(x, x)
        assert np.array_equal(idx.cpu().numpy(), ref[1])
        assert np.all(rel_l2(out, ref[0]) <= REL_L2_TOL)


def test_deterministic(decode_layer):
    L = decode_layer
    ws = _ws(L, 2)
    x = _tokens(L.shape, 2, 3)
    o1 = L.forward(x, x, ws)[0].clone()
    for _ in range(5):
        assert torch.equal(L.forward(x, x, ws)[0], o1)


def test_bad_expert_id_sets_status_and_contributes_zero():
    shape = synth.LayerShape(hidden=256, inter=128, n_experts=8, top_k=2, has_shared=False)
    L = GpuLayer(shape, 2)
    ws = _ws(L, 1)
    x = _tokens(shape, 1, 0)
    idx = torch.tensor([[3, 99]], dtype=torch.int32, device="cuda")
    w = torch.tensor([[0.5, 0.5]], dtype=torch.float32, device="cuda")
    y = moeq.expert_ffn_q4(L.desc, x, L.slots, idx, w, ws)
    rc, st = moeq.device_status(ws)
    assert rc == moeq.MOE_ERR_DEVICE_FAULT and st & moeq.MOE_DEV_BAD_EXPERT_ID
    h, yref = oracle.expert_ffn(4, 64, 256, 128, L.host(3), oracle.bf16_to_f64(synth.to_np_bits(x)[0]))
    got = y[0, 0].double().cpu().numpy()
    assert np.linalg.norm(got - 0.5 * yref) <= 1e-3 * np.linalg.norm(0.5 * yref)
    assert moeq.device_status(ws) == (0, 0)  # cleared by the read


def test_null_slot_sets_status():
    shape = synth.LayerShape(hidden=256, inter=128, n_experts=8, top_k=2, has_shared=False)
    L = GpuLayer(shape, 2)
    L.slots.table.view(8, 9)[5].zero_()  # expert 5: all pointers NULL
    ws = _ws(L, 1)
    x = _tokens(shape, 1, 0)
    idx = torch.tensor([[5, 1]], dtype=torch.int32, device="cuda")
    w = torch.tensor([[0.25, 0.75]], dtype=torch.float32, device="cuda")
    y = moeq.expert_ffn_q4(L.desc, x, L.slots, idx, w, ws)
    rc, st = moeq.device_status(ws)
    assert st & moeq.MOE_DEV_BAD_SLOT
    _, yref = oracle.expert_ffn(4, 64, 256, 128, L.host(1), oracle.bf16_to_f64(synth.to_np_bits(x)[0]))
    got = y[0, 0].double().cpu().numpy()
    assert np.linalg.norm(got - 0.75 * yref) <= 1e-3 * np.linalg.norm(0.75 * yref)
