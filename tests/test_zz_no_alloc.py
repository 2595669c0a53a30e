"""moe_expert_ffn_noalloc: the one-token expert FFN for callers that may not
allocate device memory (they run inside another program's memory budget, or
on a path where cudaMalloc could stall the device), so they cannot create a
context.  Its output must equal what moe_expert_ffn, which uses a context's
allocated scratch, gives for the same inputs, on two calls in a row (the
second call reuses the scratch the first one left behind).

This file is collected last on purpose: if it fails, a run stopped at the
first failure has already run every other test."""
import numpy as np
import pytest
import torch

from expert_streaming_decode_b200 import moe, synth
from gpu_data import TOL, Layer, bf16_tensor, rel_err


def test_oversized_shapes_are_rejected_before_any_cuda_call():
    for d_model, d_ff, top_k in ((4096, 704, 8), (2816, 2816, 8), (2816, 704, 9), (2816, 700, 8)):
        rc = moe.lib.moe_expert_ffn_noalloc(d_model, d_ff, top_k, None, None, None, None, 0, 1, None, None,
                                            None, None)
        assert rc == moe.MOE_ERR_ARG, (d_model, d_ff, top_k)


@pytest.mark.gpu
def test_noalloc_matches_expert_ffn_on_two_calls():
    d = synth.GEMMA4_26B
    L = Layer(d, layer=3, seed=11, zipf_s=None, shared=False)
    ctx = moe.Ctx.from_dims(d, max_tokens=1)
    rng = np.random.default_rng(11)
    for call in range(2):
        xb = bf16_tensor(synth.hidden(11, call, 3, d.D)[None])
        slots = torch.from_numpy(rng.choice(d.E, d.K, replace=False).astype(np.int32)[None]).cuda()
        w = torch.from_numpy(rng.uniform(0.05, 0.3, size=(1, d.K)).astype(np.float32)).cuda()
        y_in = torch.from_numpy(rng.standard_normal((1, d.D)).astype(np.float32)).cuda() if call else None
        y_ref = torch.empty((1, d.D), dtype=torch.float32, device="cuda")
        y_na = torch.full((1, d.D), float("nan"), dtype=torch.float32, device="cuda")
        moe.expert_ffn(ctx, xb, 1, d.K, slots, w, L.experts_t, L.stride, d.E, d.F, y_in, y_ref)
        moe.expert_ffn_noalloc(d.D, d.F, d.K, xb, slots, w, L.experts_t, L.stride, d.E, y_in, y_na)
        torch.cuda.synchronize()
        ctx.sync()
        err = rel_err(y_na.cpu().numpy()[0], y_ref.cpu().numpy()[0].astype(np.float64))
        assert err <= TOL, (call, err)
    ctx.close()
