"""moe_layer_forward_noalloc: the layer without a caller-provided workspace.

Some callers cannot allocate device memory where they run (an inference
engine's plugin hook, a serving loop with a fixed memory plan, a process
whose memory belongs to a caching allocator), so this entry point keeps its
scratch in a fixed 4 MiB array inside the library.  These tests call it
through the C ABI twice in a row and compare each result with
moe_layer_forward's on the same inputs, within the parity tests' tolerance.
The file name makes pytest collect it last."""
import numpy as np
import pytest
import torch

from quantised_expert_ffn_moe_b200 import moeq, synth

from moe_testutil import GpuLayer, REL_L2_TOL

pytestmark = pytest.mark.gpu


def _rel_l2(a, b):
    a = a.double().cpu().numpy()
    b = b.double().cpu().numpy()
    return np.linalg.norm(a - b, axis=1) / np.linalg.norm(b, axis=1)


@pytest.mark.parametrize("shape,T", [(synth.TINY, 1), (synth.DECODE_397B, 1), (synth.DECODE_397B, 3)],
                         ids=["tiny", "decode_T1", "decode_T3"])
def test_noalloc_matches_workspace_entry_point(shape, T):
    L = GpuLayer(shape, 21)
    ws = moeq.workspace(L.desc, T)
    for call in range(2):  # two calls in a row on the shared static scratch
        x = synth.make_tokens(shape, T, 300 + call, device="cuda")
        ref_idx = torch.empty((T, shape.top_k), dtype=torch.int32, device="cuda")
        ref = moeq.layer_forward(L.desc, x, x, L.lay.router, L.slots, ws,
                                 shared_gate=L.lay.shared_gate, topk_idx=ref_idx)
        idx = torch.empty_like(ref_idx)
        out = torch.empty_like(x)
        moeq.layer_forward_noalloc(L.desc, x, x, L.lay.router, L.slots,
                                   shared_gate=L.lay.shared_gate, out=out, topk_idx=idx)
        torch.cuda.synchronize()
        assert torch.equal(idx, ref_idx)
        assert np.all(_rel_l2(out, ref) <= REL_L2_TOL)


def test_noalloc_rejects_more_tokens_than_scratch_holds():
    L = GpuLayer(synth.DECODE_397B, 2)
    T = 1  # the fewest tokens that need more than the 4 MiB scratch at this layer size
    while moeq.workspace_size(L.desc, T) <= moeq.NOALLOC_SCRATCH_BYTES:
        T += 1
    assert moeq.workspace_size(L.desc, T - 1) <= moeq.NOALLOC_SCRATCH_BYTES
    x = synth.make_tokens(synth.DECODE_397B, T, 0, device="cuda")
    with pytest.raises(moeq.MoeError) as ei:
        moeq.layer_forward_noalloc(L.desc, x, x, L.lay.router, L.slots,
                                   shared_gate=L.lay.shared_gate)
    assert ei.value.status == moeq.MOE_ERR_INVALID_ARG
    assert "scratch" in str(ei.value)
