"""Pins of the fp64 CPU oracle against facts fixed outside it: the pages'
worked quantities (golden fixtures), closed forms, brute force on tiny inputs,
invariants, and library routines (numpy / torch float64) applied to the
materialised weights.  CPU only."""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from quantised_expert_ffn_moe_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


# ------------------------------------------------------------------ bf16 --

def test_bf16_widening_exact():
    # bf16 -> f64 against torch's own bf16 -> f32 widening (library routine)
    bits = np.arange(0, 1 << 16, 7, dtype=np.uint16)
    bits = bits[(bits & 0x7F80) != 0x7F80]  # finite values only
    ref = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).float().double().numpy()
    got = oracle.bf16_to_f64(bits)
    assert np.array_equal(got, ref)


def test_bf16_rounding_matches_torch_on_float_values():
    rng = np.random.default_rng(0)
    v = np.concatenate([rng.normal(0, 1, 4000), rng.normal(0, 1e-3, 1000),
                        rng.normal(0, 1e30, 500), [0.0, -0.0, 1.0, -2.5]]).astype(np.float32)
    # halfway cases: float values exactly between two bf16 neighbours
    base = rng.normal(0, 1, 500).astype(np.float32)
    half = (base.view(np.uint32) & np.uint32(0xFFFF0000)) | np.uint32(0x8000)
    v = np.concatenate([v, half.view(np.float32)])
    ref = torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = oracle.f64_to_bf16(v.astype(np.float64))
    assert np.array_equal(got, ref)


def test_bf16_rounding_is_nearest_from_double_brute_force():
    """For doubles not representable in float, the result is the nearest bf16
    (ties to even), checked against both neighbours by brute force; this
    catches rounding twice through float."""
    rng = np.random.default_rng(1)
    vals = list(rng.normal(0, 3, 3000))
    # just above / below exact halfway points, below float resolution
    for b in (1.0, 1.0 + 2 ** -7, 3.0, 1e-20, 5e10):
        e = math.frexp(b)[1]
        halfway = b + 2.0 ** (e - 9)
        vals += [halfway, halfway + 2.0 ** (e - 40), halfway - 2.0 ** (e - 40)]
    vals = np.array(vals)
    got = oracle.f64_to_bf16(vals)
    as_f = oracle.bf16_to_f64(got)
    for v, h, r in zip(vals, got, as_f):
        up = oracle.bf16_to_f64(np.array([h + 1], dtype=np.uint16))[0] if v >= 0 else None
        # neighbours in magnitude
        lo_bits = np.uint16(h - 1) if (h & 0x7FFF) else h
        hi_bits = np.uint16(h + 1)
        for nb in (lo_bits, hi_bits):
            n = oracle.bf16_to_f64(np.array([nb], dtype=np.uint16))[0]
            if np.isfinite(n) and np.sign(n) == np.sign(r):
                d_r, d_n = abs(v - r), abs(v - n)
                assert d_r <= d_n, (v, r, n)
                if d_r == d_n:
                    assert (h & 1) == 0  # tie goes to the even pattern
        del up
    # the double-rounding trap: 1 + 2^-8 + 2^-40 must round up to 1 + 2^-7
    assert oracle.f64_to_bf16(np.array([1 + 2 ** -8 + 2 ** -40]))[0] == 0x3F81
    assert oracle.f64_to_bf16(np.array([1 + 2 ** -8]))[0] == 0x3F80


# ---------------------------------------------------------------- format --

def test_pack_convention_golden():
    g = _golden("pack_convention.json")
    for case in g["cases"]:
        bits, word = case["bits"], int(case["word"], 16)
        codes = np.array(case["codes"], dtype=np.uint8)[None, :]
        assert oracle.pack(bits, codes)[0, 0] == word
        assert np.array_equal(oracle.unpack(bits, np.array([[word]], dtype=np.uint32), codes.shape[1]), codes)


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_pack_unpack_round_trip(bits):
    rng = np.random.default_rng(bits)
    rows, cols = 37, 256
    q = rng.integers(0, 1 << bits, size=(rows, cols), dtype=np.uint8)
    # every value at every bit position of a word (and straddling words, 3-bit)
    span = 32
    for v in range(1 << bits):
        q[v % rows, (v * span) % cols:(v * span) % cols + span] = v
    w = oracle.pack(bits, q)
    assert w.shape == (rows, cols * bits // 32)
    assert np.array_equal(oracle.unpack(bits, w, cols), q)
    # and words -> codes -> words
    w2 = rng.integers(0, 2 ** 32, size=(rows, cols * bits // 32), dtype=np.uint32)
    assert np.array_equal(oracle.pack(bits, oracle.unpack(bits, w2, cols)), w2)


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_pack_matches_bit_string_layout(bits):
    """Independent formulation of the packing: concatenate each row's codes
    as a string of bits, least significant bit of code 0 first, and cut it
    into 32-bit words read least significant bit first."""
    rng = np.random.default_rng(10 + bits)
    rows, cols = 5, 128
    q = rng.integers(0, 1 << bits, size=(rows, cols), dtype=np.uint8)
    w = oracle.pack(bits, q)
    for r in range(rows):
        stream = "".join(format(int(c), f"0{bits}b")[::-1] for c in q[r])
        words = [int(stream[32 * i:32 * i + 32][::-1], 2) for i in range(len(stream) // 32)]
        assert list(w[r]) == words


def test_pack_rejects_out_of_range_code():
    with pytest.raises(ValueError):
        oracle.pack(2, np.array([[4] * 16], dtype=np.uint8))


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_synth_words_unpack_to_uniform_codes(bits):
    """The generator's random words carry uniform codes under the oracle's
    own unpack (a distribution check on both conventions together)."""
    shp = synth.LayerShape(hidden=256, inter=128, n_experts=4, top_k=2, bits=bits)
    t = synth.make_experts(shp, seed=3)
    words = synth.to_np_bits(t.gate_codes).reshape(-1, shp.words_per_row_in)
    q = oracle.unpack(bits, words, 256)
    counts = np.bincount(q.ravel(), minlength=1 << bits)
    expect = q.size / (1 << bits)
    assert np.all(np.abs(counts - expect) < 6 * math.sqrt(expect))


def test_expert_size_pins_group_64():
    g = _golden("expert_size_q4.json")
    H, I, bits = g["hidden"], g["inter"], g["bits"]

    def expert_bytes(group):
        n = 0
        for rows, cols in ((I, H), (I, H), (H, I)):
            w = oracle.pack(bits, np.zeros((rows, cols), dtype=np.uint8))
            n += w.nbytes + 2 * g["scale_bias_bytes_each"] * rows * (cols // group)
        return n

    assert expert_bytes(64) == 7077888
    assert expert_bytes(64) / 2 ** 20 == g["stated_megabytes_per_expert"]
    assert expert_bytes(32) / 2 ** 20 == 7.5
    assert expert_bytes(128) / 2 ** 20 == 6.375
    assert synth.DECODE_397B.expert_bytes() == expert_bytes(64)


def test_expert_size_three_bit():
    """3-bit codes with the same group-64 bf16 scale and bias: 3 x 4096 x 1024
    codes x 3/8 bytes + 786,432 bytes = 5,505,024 bytes, 22% below the 4-bit
    expert (the pages quote 3-bit experts as about a quarter smaller)."""
    H, I = 4096, 1024
    n = 0
    for rows, cols in ((I, H), (I, H), (H, I)):
        n += oracle.pack(3, np.zeros((rows, cols), dtype=np.uint8)).nbytes + 2 * 2 * rows * (cols // 64)
    assert n == 5505024
    assert synth.LayerShape(hidden=H, inter=I, n_experts=512, top_k=10, bits=3).expert_bytes() == n
    assert abs(1 - n / 7077888 - 0.222) < 0.001


# ---------------------------------------------------------------- dequant --

def test_dequant_worked_example():
    g = _golden("dequant_worked_example.json")
    codes = np.array(g["codes"], dtype=np.uint8)[None, :]
    words = oracle.pack(4, codes)
    s = np.array([[int(g["scale_bf16"], 16)]], dtype=np.uint16)
    b = np.array([[int(g["bias_bf16"], 16)]], dtype=np.uint16)
    W = oracle.dequant(4, 64, words, s, b, 64)
    assert np.array_equal(W[0, :16], np.array(g["weights_first16"]))
    ones = np.ones(64)
    alt = np.array([1.0 if j % 2 == 0 else -1.0 for j in range(64)])
    for x, key in ((ones, "x_all_ones_dot"), (alt, "x_alternating_plus_minus_dot")):
        assert oracle.qmatvec(4, 64, words, s, b, x)[0] == g[key]
        assert oracle.qmatvec_grouped(4, 64, words, s, b, x)[0] == g[key]


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_two_formulations_agree(bits):
    """Literal (materialised W, then dot) vs the regrouped form
    s*sum(q x) + b*sum(x) per group: independent fp64 paths, 1e-12."""
    shp = synth.LayerShape(hidden=512, inter=192, n_experts=2, top_k=1, bits=bits)
    t = synth.make_experts(shp, seed=11)
    x = np.random.default_rng(5).normal(0, 1, 512)
    c, s, b = (synth.to_np_bits(a) for a in t.mats(0)["gate"])
    y1 = oracle.qmatvec(bits, 64, c, s, b, x)
    y2 = oracle.qmatvec_grouped(bits, 64, c, s, b, x)
    assert np.max(np.abs(y1 - y2)) <= 1e-12 * np.max(np.abs(y1))
    # and against numpy's matmul on the materialised weights (library routine)
    W = oracle.dequant(bits, 64, c, s, b, 512)
    assert np.max(np.abs(W @ x - y1)) <= 1e-12 * np.max(np.abs(y1))


def test_dequant_special_values():
    rng = np.random.default_rng(2)
    s = rng.uniform(0.005, 0.02, (3, 2))
    b = rng.uniform(-0.08, 0.08, (3, 2))
    s16 = oracle.f64_to_bf16(s)
    b16 = oracle.f64_to_bf16(b)
    sv, bv = oracle.bf16_to_f64(s16), oracle.bf16_to_f64(b16)
    for bits in (2, 4):
        qmax = (1 << bits) - 1
        for fill, expect in ((0, bv), (qmax, qmax * sv + bv)):
            q = np.full((3, 128), fill, dtype=np.uint8)
            W = oracle.dequant(bits, 64, oracle.pack(bits, q), s16, b16, 128)
            assert np.array_equal(W, np.repeat(expect, 64, axis=1))
        # zero scale: only the bias survives whatever the codes
        q = rng.integers(0, qmax + 1, (3, 128), dtype=np.uint8)
        W = oracle.dequant(bits, 64, oracle.pack(bits, q), np.zeros_like(s16), b16, 128)
        assert np.array_equal(W, np.repeat(bv, 64, axis=1))


# ------------------------------------------------------------------ route --

def test_topk_brute_force_tiny():
    """E=8, k=2: the selected pair is the one with the largest logit sum over
    all C(8,2) pairs; output in descending logit order; weights equal the
    two-way softmax closed form."""
    shp = synth.TINY
    for seed in range(40):
        lay = synth.make_layer(shp, seed)
        x = oracle.bf16_to_f64(synth.to_np_bits(synth.make_tokens(shp, 1, seed))[0])
        wr = synth.to_np_bits(lay.router)
        logits, idx, w = oracle.route(x, wr, 2)
        assert np.allclose(logits, wr.astype(np.float64) @ x, rtol=0, atol=1e-13)
        best = max(itertools.combinations(range(8), 2), key=lambda p: logits[p[0]] + logits[p[1]])
        assert sorted(best) == sorted(idx.tolist())
        assert logits[idx[0]] >= logits[idx[1]]
        assert abs(w[0] - 1.0 / (1.0 + math.exp(logits[idx[1]] - logits[idx[0]]))) < 1e-15
        assert abs(w.sum() - 1.0) < 1e-15


def test_topk_matches_torch_topk_large():
    shp = synth.DECODE_397B
    rng = np.random.default_rng(7)
    wr = oracle.f64_to_bf16(rng.normal(0, 0.02, (512, 512)))  # E=512 rows, short H for speed
    for t in range(20):
        x = oracle.bf16_to_f64(oracle.f64_to_bf16(rng.normal(0, 1, 512)))
        logits, idx, w = oracle.route(x, wr, shp.top_k)
        lt = torch.from_numpy(logits)
        tv, ti = torch.topk(lt, shp.top_k)
        assert ti.tolist() == idx.tolist()
        p = torch.softmax(lt, 0)[ti]
        assert np.allclose(w, (p / p.sum()).numpy(), rtol=1e-14, atol=0)
        assert np.all(np.diff(w) <= 0) and np.all(w > 0) and abs(w.sum() - 1) < 1e-14


def test_topk_ties_go_to_lower_index():
    E, H = 9, 64
    wr = np.zeros((E, H), dtype=np.uint16)  # bf16 zeros: logits = bias only
    bias = np.array([1, 3, 3, 2, 3, 0, 2, 3, -1], dtype=np.float64)
    _, idx, w = oracle.route(np.ones(H), wr, 5, logit_bias=bias)
    assert idx.tolist() == [1, 2, 4, 7, 3]
    e3, e2 = math.exp(0), math.exp(-1)
    z = 4 * e3 + e2
    assert np.allclose(w, [e3 / z] * 4 + [e2 / z], rtol=1e-15)


def test_topk_k_equals_E_is_full_softmax():
    rng = np.random.default_rng(3)
    wr = oracle.f64_to_bf16(rng.normal(0, 0.02, (16, 128)))
    x = rng.normal(0, 1, 128)
    logits, idx, w = oracle.route(x, wr, 16)
    assert sorted(idx.tolist()) == list(range(16))
    ref = torch.softmax(torch.from_numpy(logits), 0).numpy()[idx]
    assert np.allclose(w, ref, rtol=1e-14)


# ------------------------------------------------------------- FFN/layer --

def _host_expert(tab, e):
    m = tab.mats(e)
    return oracle.Expert(*[tuple(synth.to_np_bits(a) for a in m[k]) for k in ("gate", "up", "down")])


def _dense_expert(tab, e, bits):
    """Materialised fp64 weights (oracle dequant, pinned above)."""
    H, I = tab.shape.hidden, tab.shape.inter
    out = []
    for k, cols in (("gate", H), ("up", H), ("down", I)):
        c, s, b = (synth.to_np_bits(a) for a in tab.mats(e)[k])
        out.append(torch.from_numpy(oracle.dequant(bits, 64, c, s, b, cols)))
    return out


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_expert_ffn_against_torch_dense(bits):
    shp = synth.LayerShape(hidden=256, inter=128, n_experts=2, top_k=1, bits=bits)
    tab = synth.make_experts(shp, seed=21)
    x = oracle.bf16_to_f64(synth.to_np_bits(synth.make_tokens(shp, 1, 4))[0])
    h, y = oracle.expert_ffn(bits, 64, 256, 128, _host_expert(tab, 1), x)
    Wg, Wu, Wd = _dense_expert(tab, 1, bits)
    xt = torch.from_numpy(x)
    href = torch.nn.functional.silu(Wg @ xt) * (Wu @ xt)
    yref = Wd @ href
    assert torch.allclose(torch.from_numpy(h), href, rtol=1e-12, atol=1e-12)
    assert torch.allclose(torch.from_numpy(y), yref, rtol=1e-11, atol=1e-11)


def _layer_inputs(shp, seed, T=1):
    lay = synth.make_layer(shp, seed)
    x = synth.to_np_bits(synth.make_tokens(shp, T, seed))
    experts = {e: _host_expert(lay.experts, e) for e in range(shp.n_experts)}
    shared = _host_expert(lay.experts, shp.n_experts) if shp.has_shared else None
    sg = synth.to_np_bits(lay.shared_gate) if lay.shared_gate is not None else None
    return lay, x, experts, shared, sg


@pytest.mark.parametrize("with_gate,bits", [(False, 4), (True, 4), (True, 3), (True, 2)])
def test_layer_against_torch_composition(with_gate, bits):
    """Whole layer (routed + gated shared expert + residual) against a torch
    float64 composition: matmul, softmax, topk, silu, sigmoid."""
    shp = synth.LayerShape(hidden=256, inter=128, n_experts=8, top_k=3, has_shared=True,
                           shared_gate=with_gate, bits=bits)
    lay, x, experts, shared, sg = _layer_inputs(shp, 9, T=3)
    resid = synth.to_np_bits(synth.make_tokens(shp, 3, 99, on_sphere=False))
    wr = synth.to_np_bits(lay.router)
    out, idx, w, gamma = oracle.layer_forward(shp.desc(), x, resid, wr, experts, shared, sg)
    dense = {e: _dense_expert(lay.experts, e, bits) for e in range(shp.n_experts + 1)}
    for t in range(3):
        xt = torch.from_numpy(oracle.bf16_to_f64(x[t]))
        logits = torch.from_numpy(oracle.bf16_to_f64(wr)) @ xt
        tv, ti = torch.topk(logits, 3)
        assert ti.tolist() == idx[t].tolist()
        p = torch.softmax(logits, 0)[ti]
        p = p / p.sum()
        ref = torch.from_numpy(oracle.bf16_to_f64(resid[t])).clone()
        for e, we in zip(ti.tolist(), p):
            Wg, Wu, Wd = dense[e]
            ref += we * (Wd @ (torch.nn.functional.silu(Wg @ xt) * (Wu @ xt)))
        Wg, Wu, Wd = dense[shp.n_experts]
        g = torch.sigmoid(torch.from_numpy(oracle.bf16_to_f64(sg)) @ xt) if with_gate else torch.tensor(1.0, dtype=torch.float64)
        assert abs(gamma[t] - g.item()) < 1e-15
        ref += g * (Wd @ (torch.nn.functional.silu(Wg @ xt) * (Wu @ xt)))
        assert torch.allclose(torch.from_numpy(out[t]), ref, rtol=1e-11, atol=1e-9)


def test_one_hot_routing_reduces_to_dense_ffn():
    shp = synth.LayerShape(hidden=256, inter=128, n_experts=6, top_k=1, has_shared=False)
    lay, x, experts, _, _ = _layer_inputs(shp, 31)
    wr = synth.to_np_bits(lay.router)
    out, idx, w, _ = oracle.layer_forward(shp.desc(), x, x, wr, experts)
    assert w[0, 0] == 1.0
    xt = torch.from_numpy(oracle.bf16_to_f64(x[0]))
    e = int(np.argmax(oracle.bf16_to_f64(wr) @ xt.numpy()))
    assert idx[0, 0] == e
    Wg, Wu, Wd = _dense_expert(lay.experts, e, 4)
    ref = xt + Wd @ (torch.nn.functional.silu(Wg @ xt) * (Wu @ xt))
    assert torch.allclose(torch.from_numpy(out[0]), ref, rtol=1e-11, atol=1e-9)


def test_zero_scale_expert_closed_form():
    """All scales zero: W[r][j] = bias[r][group(j)], so gate_r = sum_g b_rg S_g(x),
    the same for up, and y_c = sum_g bd_cg S_g(h) with S_g the group sums."""
    shp = synth.LayerShape(hidden=256, inter=128, n_experts=1, top_k=1, has_shared=False)
    tab = synth.make_experts(shp, seed=41, scale_range=(0.0, 0.0))
    ex = _host_expert(tab, 0)
    x = oracle.bf16_to_f64(synth.to_np_bits(synth.make_tokens(shp, 1, 2))[0])
    h, y = oracle.expert_ffn(4, 64, 256, 128, ex, x)
    Sx = x.reshape(-1, 64).sum(1)
    bg = oracle.bf16_to_f64(ex.mats["gate"][2])
    bu = oracle.bf16_to_f64(ex.mats["up"][2])
    bd = oracle.bf16_to_f64(ex.mats["down"][2])
    g, u = bg @ Sx, bu @ Sx
    href = g / (1 + np.exp(-g)) * u
    assert np.allclose(h, href, rtol=1e-12, atol=1e-14)
    assert np.allclose(y, bd @ h.reshape(-1, 64).sum(1), rtol=1e-12, atol=1e-12)


def test_linearity_in_down_projection():
    """Doubling every down-projection scale and bias doubles the expert output
    (power-of-two scaling is exact in bf16 and fp64)."""
    shp = synth.LayerShape(hidden=256, inter=128, n_experts=1, top_k=1, has_shared=False)
    tab = synth.make_experts(shp, seed=8)
    ex = _host_expert(tab, 0)
    x = oracle.bf16_to_f64(synth.to_np_bits(synth.make_tokens(shp, 1, 1))[0])
    _, y1 = oracle.expert_ffn(4, 64, 256, 128, ex, x)
    c, s, b = ex.mats["down"]
    dbl = lambda a: oracle.f64_to_bf16(2 * oracle.bf16_to_f64(a))
    ex2 = oracle.Expert(ex.mats["gate"], ex.mats["up"], (c, dbl(s), dbl(b)))
    _, y2 = oracle.expert_ffn(4, 64, 256, 128, ex2, x)
    assert np.array_equal(y2, 2 * y1)


def test_expert_permutation_invariance():
    shp = synth.LayerShape(hidden=256, inter=128, n_experts=8, top_k=2, has_shared=False)
    lay, x, experts, _, _ = _layer_inputs(shp, 13, T=2)
    wr = synth.to_np_bits(lay.router)
    out, idx, w, _ = oracle.layer_forward(shp.desc(), x, x, wr, experts)
    perm = np.random.default_rng(0).permutation(8)  # new id of old expert e is perm[e]
    wr2 = np.zeros_like(wr)
    wr2[perm] = wr
    experts2 = {int(perm[e]): experts[e] for e in experts}
    out2, idx2, w2, _ = oracle.layer_forward(shp.desc(), x, x, wr2, experts2)
    assert np.array_equal(perm[idx], idx2)
    assert np.allclose(out, out2, rtol=0, atol=1e-12)


def test_rmsnorm_closed_form():
    rng = np.random.default_rng(4)
    x = rng.normal(0, 3, 4096)
    eps = 1e-6
    y = oracle.rmsnorm(x, eps)
    ms = np.mean(x * x)
    assert abs(np.mean(y * y) - ms / (ms + eps)) < 1e-14
    assert np.allclose(oracle.rmsnorm(5 * x, 0.0), oracle.rmsnorm(x, 0.0), rtol=1e-14)
