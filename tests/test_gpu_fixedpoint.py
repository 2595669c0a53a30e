"""The one-token expert kernels store each group of 64 inputs as a 16-bit
fixed-point image (scale = the group's largest magnitude / 32767) and take
integer dot products with the 4-bit weights.  That image is the kernels' own
approximation, not the pages' arithmetic ("TurboFieldfare: motor open source
...", section "Estructura de ejecucion para reducir memoria": 4-bit affine
weights, groups of 64), so these cases put inputs where it loses the most
precision and compare element by element with the oracle (fp64, no image):

  - one channel per group 1000 times its neighbours (the neighbours keep only
    about 5 significant bits of their own magnitude);
  - groups whose magnitudes differ by 2^10 (each group has its own scale);
  - all-zero groups (scale 0);
  - hidden states large enough that gelu(g) * u reaches about +-10^3, the
    down kernel's inputs;
  - an expert whose up row 5 is 1024 times larger than the rest, so one
    activation per token is ~10^3 times its group's others (an outlier in the
    down kernel's staged input).

Each case runs through moe_expert_ffn (one token, eight experts) and through
the one-token resident moe_layer_forward (router, shared expert, combine);
max|y - r| <= 2e-3 max|r| as everywhere else."""
import numpy as np
import pytest
import torch

import oracle
from expert_streaming_decode_b200 import moe, synth
from gpu_data import GATE_TOL, TOL, Layer, bf16_tensor, rel_err

pytestmark = pytest.mark.gpu

D = synth.GEMMA4_26B


@pytest.fixture(scope="module")
def O():
    return oracle.get()


@pytest.fixture(scope="module")
def layer():
    L = Layer(D, layer=2, seed=21, zipf_s=None)
    # expert 9: up row 5 scaled by 1024 (exact in binary16), bias kept at -8 * scale
    p = synth.draw_expert_parts(21, 2, 9, D.D, D.F)
    s = p["su"].astype(np.float32)
    s[5] *= 1024.0
    p["su"] = s.astype(np.float16)
    p["bu"] = (s * -8.0).astype(np.float16)
    blob = synth.pack_parts(p)
    L.host[9, :L.nb] = blob
    L.blobs[9] = L.host[9, :L.nb]
    L.experts_t[9].copy_(torch.from_numpy(L.host[9]))
    return L


def _inputs(case, rng):
    v = rng.standard_normal(D.D).astype(np.float32)
    g = v.reshape(-1, 64)
    if case == "outlier_per_group":
        pos = rng.integers(0, 64, g.shape[0])
        g[np.arange(g.shape[0]), pos] = 1000.0 * np.sign(rng.standard_normal(g.shape[0]))
    elif case == "group_scale_2e10":
        g[1::2] *= 1024.0
    elif case == "group_scale_2e-10":
        g[1::2] *= 1.0 / 1024.0
    elif case == "zero_groups":
        g[::3] = 0.0
    elif case == "large_activations":
        v *= 12.0
    return synth.to_bf16_bits(v)


CASES = ["outlier_per_group", "group_scale_2e10", "group_scale_2e-10", "zero_groups", "large_activations",
         "activation_outlier"]


def _h_max(O, L, e, x):
    """Largest |gelu(g) * u| of expert e on x (to check the case reaches its regime)."""
    g = O.dequant(L.blobs[e], D.D, D.F, 0) @ x
    u = O.dequant(L.blobs[e], D.D, D.F, 1) @ x
    gl = np.array([O.gelu_tanh(float(a)) for a in g])
    return np.abs(gl * u)


@pytest.mark.parametrize("case", CASES)
def test_expert_ffn_fixed_point_edges(O, layer, case):
    L = layer
    # the outlier case's seed is one where gelu(g_5) is large (asserted below)
    rng = np.random.default_rng(1000 if case == "activation_outlier" else CASES.index(case))
    xb = _inputs(case, rng)
    x = synth.bf16_bits_to_f32(xb).astype(np.float64)
    slots = rng.choice(D.E, D.K, replace=False).astype(np.int32)
    if case == "activation_outlier":
        others = rng.choice(np.delete(np.arange(D.E), 9), D.K - 1, replace=False)
        slots = np.concatenate([[9], others]).astype(np.int32)
        hm = _h_max(O, L, 9, x)
        assert hm[5] >= 100 * np.median(np.delete(hm, 5)), "the activation outlier case did not reach its regime"
    if case == "large_activations":
        assert _h_max(O, L, int(slots[0]), x).max() >= 300.0, "gelu(g) * u did not reach its regime"
    w = rng.uniform(0.05, 0.3, size=D.K).astype(np.float32)
    ctx = moe.Ctx.from_dims(D, max_tokens=1)
    y = torch.empty((1, D.D), dtype=torch.float32, device="cuda")
    moe.expert_ffn(ctx, bf16_tensor(xb[None]), 1, D.K, torch.from_numpy(slots[None]).cuda(),
                   torch.from_numpy(w[None]).cuda(), L.experts_t, L.stride, D.E, D.F, None, y)
    ctx.sync()
    ref = np.zeros(D.D)
    for k in range(D.K):
        ref = ref + float(w[k]) * O.expert_ffn(L.blobs[slots[k]], D.D, D.F, x)
    err = rel_err(y.cpu().numpy()[0], ref)
    assert err <= TOL, (case, err)
    ctx.close()


@pytest.mark.parametrize("kernel", ["split", "layer"])
@pytest.mark.parametrize("case", CASES)
def test_layer_forward_fixed_point_edges(O, layer, case, kernel, monkeypatch):
    """The whole one-token resident layer on the same inputs, through the
    separate router / GEMV kernels and through the one-launch layer kernel;
    the activation outlier case biases the router towards expert 9 so it is
    selected."""
    monkeypatch.setenv("MOE_LAYER_KERNEL", "1" if kernel == "layer" else "0")
    L = layer
    rng = np.random.default_rng(1001 if case == "activation_outlier" else 100 + CASES.index(case))
    xb = _inputs(case, rng)
    bias = None
    if case == "activation_outlier":
        bias = np.zeros(D.E, dtype=np.float32)
        bias[9] = 50.0
    ctx = moe.Ctx.from_dims(D, max_tokens=1)
    y = torch.empty((1, D.D), dtype=torch.float32, device="cuda")
    ids = torch.empty((1, D.K), dtype=torch.int32, device="cuda")
    gw = torch.empty((1, D.K), dtype=torch.float32, device="cuda")
    moe.layer_forward(ctx, L.weights(), None, bf16_tensor(xb[None]), 1, 0,
                      None if bias is None else torch.from_numpy(bias).cuda(), y, ids=ids, gate_w=gw)
    ctx.sync()
    want_ids, want_w, _, want_y = O.moe_token(D.as_dict(), xb, L.wq, L.ws, bias, L.shared, L.blobs)
    assert np.array_equal(ids.cpu().numpy()[0], want_ids)
    assert np.max(np.abs(gw.cpu().numpy()[0] - want_w)) <= GATE_TOL
    if case == "activation_outlier":
        assert 9 in want_ids
        hm = _h_max(O, L, 9, synth.bf16_bits_to_f32(xb).astype(np.float64))
        assert hm[5] >= 100 * np.median(np.delete(hm, 5)), "the activation outlier case did not reach its regime"
    err = rel_err(y.cpu().numpy()[0], want_y)
    assert err <= TOL, (case, err)
    ctx.close()
