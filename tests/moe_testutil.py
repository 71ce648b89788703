"""Shared helpers of the GPU parity tests: build a layer on the device from the
seeded generators, hand host copies of the very same tensors to the CPU
oracle, and compare."""
import numpy as np
import torch

import oracle
from quantised_expert_ffn_moe_b200 import moeq, synth

REL_L2_TOL = 2e-3   # output tolerance (bf16 outputs, fp32 accumulation)
WEIGHT_RTOL = 1e-6  # routing weights are fp32 of an fp64 softmax


def host_expert(table, e):
    m = table.mats(e)
    return oracle.Expert(*[tuple(synth.to_np_bits(a) for a in m[k]) for k in ("gate", "up", "down")])


class GpuLayer:
    def __init__(self, shape, seed, device="cuda", experts=None):
        self.shape = shape
        self.lay = synth.make_layer(shape, seed, device)
        if experts is not None:
            self.lay.experts = experts
        self.slots = moeq.DeviceSlots(self.lay.experts, shape.n_experts)
        self.desc = moeq.make_desc(shape)
        self._host = {}

    def host(self, e):
        if e not in self._host:
            self._host[e] = host_expert(self.lay.experts, e)
        return self._host[e]

    def router_np(self):
        return synth.to_np_bits(self.lay.router)

    def oracle_forward(self, x, resid, logit_bias=None):
        """x, resid: bf16 torch tensors [T][H] (any device)."""
        xb, rb = synth.to_np_bits(x), synth.to_np_bits(resid)
        wr = self.router_np()
        lb = None if logit_bias is None else logit_bias.detach().cpu().numpy().astype(np.float64)
        need = set()
        for t in range(xb.shape[0]):
            _, idx, _ = oracle.route(oracle.bf16_to_f64(xb[t]), wr, self.shape.top_k,
                                     None if lb is None else lb[t])
            need |= set(int(i) for i in idx)
        experts = {e: self.host(e) for e in need}
        shared = self.host(self.shape.n_experts) if self.shape.has_shared else None
        sg = synth.to_np_bits(self.lay.shared_gate) if self.lay.shared_gate is not None else None
        return oracle.layer_forward(self.shape.desc(), xb, rb, wr, experts, shared, sg, lb)

    def forward(self, x, resid, ws, logit_bias=None):
        T = x.shape[0]
        idx = torch.empty((T, self.shape.top_k), dtype=torch.int32, device=x.device)
        w = torch.empty((T, self.shape.top_k), dtype=torch.float32, device=x.device)
        out = moeq.layer_forward(self.desc, x, resid, self.lay.router, self.slots, ws,
                                 shared_gate=self.lay.shared_gate, logit_bias=logit_bias,
                                 topk_idx=idx, topk_w=w)
        return out, idx, w


def rel_l2(out_bf16, ref):
    """Per-token ||gpu - oracle|| / ||oracle||, gpu bf16 widened exactly."""
    g = out_bf16.detach().float().double().cpu().numpy()
    return np.linalg.norm(g - ref, axis=1) / np.linalg.norm(ref, axis=1)


def assert_parity(out, idx, w, ref_out, ref_idx, ref_w, tol=REL_L2_TOL):
    assert np.array_equal(idx.cpu().numpy(), ref_idx), (idx.cpu().numpy(), ref_idx)
    assert np.allclose(w.cpu().numpy(), ref_w, rtol=WEIGHT_RTOL, atol=1e-7)
    err = rel_l2(out, ref_out)
    assert np.all(err <= tol), err
    return err
