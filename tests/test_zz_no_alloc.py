"""moe_expert_ffn_noalloc: the one-token expert FFN for callers that may not
allocate device memory (they run inside another program's memory budget, or
on a path where cudaMalloc could stall the device), so they cannot create a
context.  Its output must equal what moe_expert_ffn, which uses a context's
allocated scratch, gives for the same inputs, on two calls in a row (the
second call reuses the scratch the first one left behind), and the oracle's
sum of gate-weighted expert FFNs.  Its scratch is laid out once for the
largest shape it accepts, so smaller shapes (a scaled-down layer, a mid-size
one with fewer than 8 selections) run with other strides than the context
path and are checked too, as is a token that names one slot twice.

This file is collected last on purpose: if it fails, a run stopped at the
first failure has already run every other test."""
import numpy as np
import pytest
import torch

import oracle
from expert_streaming_decode_b200 import moe, synth
from gpu_data import TOL, Layer, bf16_tensor, rel_err

MID = synth.Dims(D=1536, E=32, K=6, F=256, FS=512, G=64, L=1, S=8)


def test_oversized_shapes_are_rejected_before_any_cuda_call():
    for d_model, d_ff, top_k in ((4096, 704, 8), (2816, 2816, 8), (2816, 704, 9), (2816, 700, 8)):
        rc = moe.lib.moe_expert_ffn_noalloc(d_model, d_ff, top_k, None, None, None, None, 0, 1, None, None,
                                            None, None)
        assert rc == moe.MOE_ERR_ARG, (d_model, d_ff, top_k)


def _oracle_combine(O, L, d, xb, slots, w, y_in):
    x = synth.bf16_bits_to_f32(xb).astype(np.float64)
    ref = np.zeros(d.D) if y_in is None else y_in.astype(np.float64)
    for k in range(len(slots)):
        ref = ref + float(w[k]) * O.expert_ffn(L.blobs[slots[k]], d.D, d.F, x)
    return ref


@pytest.mark.gpu
@pytest.mark.parametrize("d", [synth.GEMMA4_26B, synth.TINY, MID], ids=["full", "tiny", "mid-k6"])
def test_noalloc_matches_expert_ffn_and_oracle_on_two_calls(d):
    O = oracle.get()
    L = Layer(d, layer=3, seed=11, zipf_s=None, shared=False)
    ctx = moe.Ctx.from_dims(d, max_tokens=1)
    rng = np.random.default_rng(11)
    for call in range(2):
        xb = synth.hidden(11, call, 3, d.D)
        slots_np = rng.choice(d.E, d.K, replace=False).astype(np.int32)
        w_np = rng.uniform(0.05, 0.3, size=d.K).astype(np.float32)
        y_in_np = rng.standard_normal(d.D).astype(np.float32) if call else None
        slots = torch.from_numpy(slots_np[None]).cuda()
        w = torch.from_numpy(w_np[None]).cuda()
        y_in = None if y_in_np is None else torch.from_numpy(y_in_np[None]).cuda()
        y_ref = torch.empty((1, d.D), dtype=torch.float32, device="cuda")
        y_na = torch.full((1, d.D), float("nan"), dtype=torch.float32, device="cuda")
        moe.expert_ffn(ctx, bf16_tensor(xb[None]), 1, d.K, slots, w, L.experts_t, L.stride, d.E, d.F, y_in, y_ref)
        moe.expert_ffn_noalloc(d.D, d.F, d.K, bf16_tensor(xb[None]), slots, w, L.experts_t, L.stride, d.E, y_in,
                               y_na)
        torch.cuda.synchronize()
        ctx.sync()
        ref = _oracle_combine(O, L, d, xb, slots_np, w_np, y_in_np)
        got_na = y_na.cpu().numpy()[0].astype(np.float64)
        assert rel_err(got_na, y_ref.cpu().numpy()[0].astype(np.float64)) <= TOL, call
        assert rel_err(got_na, ref) <= TOL, call
    ctx.close()


@pytest.mark.gpu
def test_noalloc_slot_named_twice():
    """A token that names one slot twice: both selections count, each with its
    own weight, in both entry points and in the oracle's sum."""
    O = oracle.get()
    d = synth.TINY
    L = Layer(d, layer=0, seed=12, zipf_s=None, shared=False)
    ctx = moe.Ctx.from_dims(d, max_tokens=1)
    xb = synth.hidden(12, 0, 0, d.D)
    slots_np = np.array([5, 2, 5, 9][:d.K], dtype=np.int32)
    w_np = np.array([0.4, 0.1, 0.3, 0.2][:d.K], dtype=np.float32)
    slots = torch.from_numpy(slots_np[None]).cuda()
    w = torch.from_numpy(w_np[None]).cuda()
    y_ref = torch.empty((1, d.D), dtype=torch.float32, device="cuda")
    y_na = torch.empty((1, d.D), dtype=torch.float32, device="cuda")
    moe.expert_ffn(ctx, bf16_tensor(xb[None]), 1, d.K, slots, w, L.experts_t, L.stride, d.E, d.F, None, y_ref)
    moe.expert_ffn_noalloc(d.D, d.F, d.K, bf16_tensor(xb[None]), slots, w, L.experts_t, L.stride, d.E, None, y_na)
    torch.cuda.synchronize()
    ctx.sync()
    ref = _oracle_combine(O, L, d, xb, slots_np, w_np, None)
    assert rel_err(y_ref.cpu().numpy()[0], ref) <= TOL
    assert rel_err(y_na.cpu().numpy()[0], ref) <= TOL
    ctx.close()
