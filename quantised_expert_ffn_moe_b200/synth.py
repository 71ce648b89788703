"""Seeded synthetic inputs for the quantised MoE layer.

This module only draws random inputs with the shapes and value distributions
of the workloads (random code words, uniform scales/biases, normal router and
input vectors, harness-only routing skews).  It holds none of the layer's own
arithmetic, and both the CUDA path and the CPU oracle are fed from it.

Weights are drawn directly on the target device (a torch generator seeded per
tensor), so the large expert tables are generated in HBM; the oracle receives
host copies of the very same tensors.
"""
from dataclasses import dataclass, field
import math

import numpy as np
import torch


@dataclass(frozen=True)
class LayerShape:
    hidden: int
    inter: int
    n_experts: int
    top_k: int
    bits: int = 4
    group: int = 64
    has_shared: bool = True
    router_f32: bool = False  # the tiny layer uses an fp32 router
    shared_gate: bool = True  # bf16 [H] gate vector for the shared expert

    @property
    def words_per_row_in(self):  # gate/up rows (length hidden)
        return self.hidden * self.bits // 32

    @property
    def words_per_row_down(self):  # down rows (length inter)
        return self.inter * self.bits // 32

    def expert_bytes(self):
        """Bytes of one expert: codes + bf16 scale + bf16 bias of gate, up, down."""
        n = 3 * self.hidden * self.inter
        return n * self.bits // 8 + 2 * 2 * n // self.group

    def desc(self):
        return dict(hidden=self.hidden, inter=self.inter, n_experts=self.n_experts,
                    top_k=self.top_k, group_size=self.group, bits=self.bits,
                    has_shared=int(self.has_shared))


# Workloads.  Names say what they are.
TINY = LayerShape(hidden=256, inter=128, n_experts=8, top_k=2, has_shared=False,
                  router_f32=True, shared_gate=False)
DECODE_397B = LayerShape(hidden=4096, inter=1024, n_experts=512, top_k=10)
DECODE_2BIT = LayerShape(hidden=4096, inter=1024, n_experts=512, top_k=3, bits=2)
DECODE_2BIT_K4 = LayerShape(hidden=4096, inter=1024, n_experts=512, top_k=4, bits=2)


def _gen(device, seed):
    g = torch.Generator(device=device)
    g.manual_seed(int(seed) & 0x7FFFFFFFFFFFFFFF)
    return g


def _sub(seed, *tags):
    """Derive an independent seed from a base seed and integer tags."""
    h = (int(seed) * 0x9E3779B97F4A7C15) & 0xFFFFFFFFFFFFFFFF
    for t in tags:
        h ^= (int(t) + 0x632BE59BD9B4E019 + ((h << 6) & 0xFFFFFFFFFFFFFFFF) + (h >> 2))
        h &= 0xFFFFFFFFFFFFFFFF
    return h & 0x7FFFFFFFFFFFFFFF


def random_words(shape, gen, device):
    """uint32 words of uniform random bits (so every code is uniform), stored
    in an int32 tensor."""
    n = int(np.prod(shape))
    b = torch.randint(0, 256, (n * 4,), dtype=torch.uint8, generator=gen, device=device)
    return b.view(torch.int32).view(*shape)


def uniform_bf16(shape, lo, hi, gen, device):
    return (torch.rand(shape, generator=gen, device=device, dtype=torch.float32)
            * (hi - lo) + lo).to(torch.bfloat16)


def normal(shape, std, gen, device, dtype):
    return (torch.randn(shape, generator=gen, device=device, dtype=torch.float32) * std).to(dtype)


@dataclass
class ExpertTable:
    """All experts of one layer, stacked: index e < n_experts are routed
    experts, index n_experts (if present) is the shared expert.

    codes_*: int32 [n][rows][words]; scale_*/bias_*: bf16 [n][rows][rows_in/group]."""
    shape: LayerShape
    n: int
    gate_codes: torch.Tensor
    gate_scale: torch.Tensor
    gate_bias: torch.Tensor
    up_codes: torch.Tensor
    up_scale: torch.Tensor
    up_bias: torch.Tensor
    down_codes: torch.Tensor
    down_scale: torch.Tensor
    down_bias: torch.Tensor

    def mats(self, e):
        return {"gate": (self.gate_codes[e], self.gate_scale[e], self.gate_bias[e]),
                "up": (self.up_codes[e], self.up_scale[e], self.up_bias[e]),
                "down": (self.down_codes[e], self.down_scale[e], self.down_bias[e])}


def make_experts(shape: LayerShape, seed: int, device="cpu", n=None,
                 scale_range=(0.005, 0.02), bias_range=(-0.08, 0.08)) -> ExpertTable:
    """Codes uniform over [0, 2^bits); scale ~ U(0.005, 0.02) and bias ~
    U(-0.08, 0.08), both rounded to bf16."""
    if n is None:
        n = shape.n_experts + (1 if shape.has_shared else 0)
    H, I, G = shape.hidden, shape.inter, shape.group
    g = _gen(device, _sub(seed, 1))
    t = {}
    for m, rows, cols in (("gate", I, H), ("up", I, H), ("down", H, I)):
        t[m + "_codes"] = random_words((n, rows, cols * shape.bits // 32), g, device)
        t[m + "_scale"] = uniform_bf16((n, rows, cols // G), *scale_range, g, device)
        t[m + "_bias"] = uniform_bf16((n, rows, cols // G), *bias_range, g, device)
    return ExpertTable(shape=shape, n=n, **t)


@dataclass
class LayerInputs:
    shape: LayerShape
    experts: ExpertTable
    router: torch.Tensor            # [E][H] bf16 (or fp32 for the tiny layer)
    shared_gate: torch.Tensor = None  # bf16 [H] or None
    extra: dict = field(default_factory=dict)


def make_layer(shape: LayerShape, seed: int, device="cpu") -> LayerInputs:
    experts = make_experts(shape, seed, device)
    g = _gen(device, _sub(seed, 2))
    router = normal((shape.n_experts, shape.hidden), 0.02, g, device,
                    torch.float32 if shape.router_f32 else torch.bfloat16)
    sg = None
    if shape.has_shared and shape.shared_gate:
        sg = normal((shape.hidden,), 0.02, g, device, torch.bfloat16)
    return LayerInputs(shape=shape, experts=experts, router=router, shared_gate=sg)


def make_tokens(shape: LayerShape, T: int, seed: int, device="cpu", on_sphere=True):
    """bf16 [T][H] token vectors.  With on_sphere, each row is a normal vector
    scaled to Euclidean norm sqrt(H) (root-mean-square 1 before the bf16
    rounding), the distribution of an RMS-normalised input; otherwise plain
    N(0, 1)."""
    g = _gen(device, _sub(seed, 3))
    z = torch.randn((T, shape.hidden), generator=g, device=device, dtype=torch.float64)
    if on_sphere and T > 0:
        z = z * (math.sqrt(shape.hidden) / z.norm(dim=1, keepdim=True))
    return z.to(torch.bfloat16)


def zipf_logit_bias(n_experts: int, T: int, s: float, seed: int):
    """Harness-only routing skew: bias_e = log p_e with p_e proportional to
    rank(e)^-s, rank a seeded permutation of the experts.  fp32 [T][E] (the
    same row for every token)."""
    rng = np.random.default_rng(_sub(seed, 4))
    rank = rng.permutation(n_experts) + 1
    p = rank.astype(np.float64) ** (-s)
    p /= p.sum()
    b = np.log(p).astype(np.float32)
    return np.tile(b, (T, 1))


def repeat_logit_bias(n_experts: int, k: int, T: int, repeat: float, seed: int, boost=8.0):
    """Harness-only routing skew for a decode sequence: for token t a set of k
    experts gets +boost; each member of token t-1's set is kept with
    probability `repeat`, the rest of the set is drawn uniformly from the
    other experts.  Returns (bias fp32 [T][E], sets int [T][k])."""
    rng = np.random.default_rng(_sub(seed, 5))
    sets = np.zeros((T, k), dtype=np.int64)
    prev = rng.choice(n_experts, size=k, replace=False)
    for t in range(T):
        if t == 0:
            cur = prev
        else:
            keep = prev[rng.random(k) < repeat]
            rest = np.setdiff1d(np.arange(n_experts), keep)
            fresh = rng.choice(rest, size=k - keep.size, replace=False)
            cur = np.concatenate([keep, fresh])
        sets[t] = cur
        prev = cur
    bias = np.zeros((T, n_experts), dtype=np.float32)
    for t in range(T):
        bias[t, sets[t]] = boost
    return bias, sets


def to_np_bits(t: torch.Tensor):
    """Host numpy copy keeping raw bits: bf16 -> uint16, int32 words -> uint32,
    fp32 -> float32."""
    t = t.detach().contiguous().cpu()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    if t.dtype == torch.int32:
        return t.numpy().view(np.uint32)
    return t.numpy()
