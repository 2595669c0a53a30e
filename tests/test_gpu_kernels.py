"""GPU parity of each entry point against the CPU oracle (B200 only).

Router ids, cache plans and slot traces are compared bit for bit; expert FFN
outputs within max|y - r| <= 2e-3 * max|r| (fp32 accumulation against the
oracle's fp64); gate weights within 1e-5 absolute."""
import numpy as np
import pytest
import torch

import oracle
from expert_streaming_decode_b200 import moe, synth
from gpu_data import GATE_TOL, TOL, Layer, bf16_tensor, rel_err

pytestmark = pytest.mark.gpu

FULL = synth.GEMMA4_26B
TINY = synth.TINY


@pytest.fixture(scope="module")
def O():
    return oracle.get()


# ------------------------------------------------------------------ router
@pytest.mark.parametrize("d", [TINY, FULL], ids=["tiny", "full"])
@pytest.mark.parametrize("T", [1, 5, 32])
@pytest.mark.parametrize("with_bias", [True, False])
def test_router_ids_bit_exact(O, d, T, with_bias):
    ctx = moe.Ctx.from_dims(d, max_tokens=32)
    wq, ws = synth.router_weights(7, 2, d.E, d.D)
    bias = synth.zipf_bias(7, 2, d.E) if with_bias else None
    xb = synth.hidden_batch(7, range(T), 2, d.D)
    ids = torch.empty((T, d.K), dtype=torch.int32, device="cuda")
    gw = torch.empty((T, d.K), dtype=torch.float32, device="cuda")
    moe.router_topk(ctx, bf16_tensor(xb), torch.from_numpy(wq).cuda(), torch.from_numpy(ws.view(np.int16)).cuda(),
                    None if bias is None else torch.from_numpy(bias).cuda(), T, ids, gw)
    ctx.sync()
    ids, gw = ids.cpu().numpy(), gw.cpu().numpy()
    for t in range(T):
        lg = O.router_logits(xb[t], wq, ws, bias, d.E, d.D, d.G)
        want = O.topk(lg, d.K)
        assert np.array_equal(ids[t], want), (t, ids[t], want)
        assert np.max(np.abs(gw[t] - O.gate_weights(lg, want))) <= GATE_TOL


@pytest.mark.parametrize("D,E", [(8192, 256), (8192, 1024)], ids=["3-passes", "10-passes"])
def test_router_rows_in_passes(O, D, E):
    """Router rows that do not fit shared memory at once are staged in passes
    through two buffers (ragged last pass); ids stay bit-exact."""
    d = synth.Dims(D=D, E=E, K=8, F=64, FS=128, G=64, L=1, S=8)
    T = 3
    ctx = moe.Ctx.from_dims(d, max_tokens=T)
    wq, ws = synth.router_weights(11, 0, E, D)
    bias = synth.zipf_bias(11, 0, E)
    xb = synth.hidden_batch(11, range(T), 0, D)
    ids = torch.empty((T, d.K), dtype=torch.int32, device="cuda")
    gw = torch.empty((T, d.K), dtype=torch.float32, device="cuda")
    moe.router_topk(ctx, bf16_tensor(xb), torch.from_numpy(wq).cuda(), torch.from_numpy(ws.view(np.int16)).cuda(),
                    torch.from_numpy(bias).cuda(), T, ids, gw)
    ctx.sync()
    ids, gw = ids.cpu().numpy(), gw.cpu().numpy()
    for t in range(T):
        lg = O.router_logits(xb[t], wq, ws, bias, E, D, 64)
        want = O.topk(lg, d.K)
        assert np.array_equal(ids[t], want), (t, ids[t], want)
        assert np.max(np.abs(gw[t] - O.gate_weights(lg, want))) <= GATE_TOL


def test_router_ties_and_nan(O):
    d = TINY
    ctx = moe.Ctx.from_dims(d, max_tokens=4)
    wq = np.zeros((d.E, d.D), np.int8)          # every logit equals its bias
    ws = np.full((d.E, d.D // 64), 0x3C00, np.uint16)
    bias = np.zeros(d.E, np.float32)
    bias[[3, 9, 12]] = 1.0                       # three tied leaders, then 13 tied at 0
    xb = synth.hidden_batch(1, range(2), 0, d.D)
    ids = torch.empty((2, d.K), dtype=torch.int32, device="cuda")
    gw = torch.empty((2, d.K), dtype=torch.float32, device="cuda")
    args = (torch.from_numpy(wq).cuda(), torch.from_numpy(ws.view(np.int16)).cuda(), torch.from_numpy(bias).cuda())
    moe.router_topk(ctx, bf16_tensor(xb), *args, 2, ids, gw)
    ctx.sync()
    assert ids.cpu().numpy().tolist() == [[3, 9, 12, 0]] * 2
    xb[1, 5] = 0x7FC0                           # NaN in token 1 -> NaN logits only if weights touch it
    wq[:, 5] = 1
    moe.router_topk(ctx, bf16_tensor(xb), torch.from_numpy(wq).cuda(), *args[1:], 2, ids, gw)
    assert ctx.sync_status() == moe.MOE_ERR_NAN
    got = ids.cpu().numpy()
    assert got.min() >= 0 and got.max() < d.E
    assert ctx.sync_status() == moe.MOE_OK      # the status word was cleared


# -------------------------------------------------------------- cache plan
def _plan_sequence(O, d, S, T, steps, seed, zipf=True, policy=0, period=0):
    E, K = d.E, d.K
    ctx = moe.Ctx(d.D, E, K, d.F, d.FS, S, max_tokens=max(T, 1))
    state = torch.empty(ctx.state_words(), dtype=torch.int32, device="cuda")
    slots = torch.empty((S, 256), dtype=torch.uint8, device="cuda")  # plan only: slots never read
    cache = moe.slot_cache(slots, 256, state, policy=policy, decay_period=period)
    cache.slot_stride = synth.blob_bytes(d.D, d.F) + 255 & ~255
    moe.cache_reset(ctx, cache)
    ost = oracle.LfuState(E, S, policy, period)
    rng = np.random.default_rng(seed)
    zb = synth.zipf_bias(seed, 0, E) if zipf else np.zeros(E)
    ps = torch.empty((T, K), dtype=torch.int32, device="cuda")
    tr = moe.Trace(E)
    for step in range(steps):
        lg = rng.standard_normal((T, E)) + zb
        ids = np.argsort(-lg, axis=1, kind="stable")[:, :K].astype(np.int32)
        moe.cache_plan(ctx, cache, torch.from_numpy(ids).cuda(), T, step, ps, tr)
        got = tr.result()
        want = O.lfu_plan(ost, ids, step)
        for key in ("expert", "slot", "hit", "victim", "wave"):
            assert np.array_equal(got[key], want[key]), (step, key, got[key], want[key])
        assert got["waves"] == want["waves"] and got["misses"] == int((want["hit"] == 0).sum())
        assert got["h2d_bytes"] == 0   # no store: nothing copied
        assert np.array_equal(ps.cpu().numpy(), want["pair_slot"]), step
    ctx.sync()
    st = state.cpu().numpy()
    assert np.array_equal(st[:E].view(np.uint32), ost.count)
    assert np.array_equal(st[E:2 * E].view(np.uint32), ost.last_use)
    assert np.array_equal(st[2 * E:3 * E], ost.slot_of)
    assert np.array_equal(st[3 * E:], ost.expert_in)


@pytest.mark.parametrize("S,T,steps", [(16, 1, 300), (8, 1, 200), (64, 1, 200), (16, 4, 80), (16, 128, 6), (8, 32, 10)])
def test_cache_plan_trace_bit_exact(O, S, T, steps):
    _plan_sequence(O, FULL, S, T, steps, seed=S * 1000 + T)


@pytest.mark.parametrize("policy,period", [(moe.MOE_POLICY_LRU, 0), (moe.MOE_POLICY_LFU_DECAY, 16),
                                           (moe.MOE_POLICY_LFU_DECAY, 1), (moe.MOE_POLICY_LFU_IN_CACHE, 0)],
                         ids=["lru", "decay16", "decay1", "in-cache"])
@pytest.mark.parametrize("S,T,steps", [(16, 1, 300), (16, 128, 6)], ids=["decode", "prefill-waves"])
def test_cache_policy_traces_bit_exact(O, policy, period, S, T, steps):
    """Replacement-rule variants: traces, pair slots and the final state equal
    the oracle's bit for bit."""
    _plan_sequence(O, FULL, S, T, steps, seed=S * 1000 + T + 7 * policy, policy=policy, period=period)


def test_cache_policy_rejected_when_unknown():
    d = TINY
    ctx = moe.Ctx.from_dims(d, max_tokens=1)
    state = torch.empty(ctx.state_words(), dtype=torch.int32, device="cuda")
    slots = torch.empty((d.S, 256), dtype=torch.uint8, device="cuda")
    cache = moe.slot_cache(slots, 256, state, policy=7)
    cache.slot_stride = synth.blob_bytes(d.D, d.F) + 255 & ~255
    ids = torch.zeros((1, d.K), dtype=torch.int32, device="cuda")
    ps = torch.empty((1, d.K), dtype=torch.int32, device="cuda")
    with pytest.raises(moe.MoeError):
        moe.cache_plan(ctx, cache, ids, 1, 0, ps, None)


def test_cache_plan_tiny_uniform(O):
    _plan_sequence(O, TINY, 6, 3, 60, seed=5, zipf=False)


def test_cache_plan_rejects_bad_ids(O):
    d = TINY
    ctx = moe.Ctx.from_dims(d, max_tokens=1)
    state = torch.empty(ctx.state_words(), dtype=torch.int32, device="cuda")
    slots = torch.empty((d.S, synth.blob_bytes(d.D, d.F) + 255 & ~255), dtype=torch.uint8, device="cuda")
    cache = moe.slot_cache(slots, slots.shape[1], state)
    moe.cache_reset(ctx, cache)
    ids = torch.tensor([[0, 1, d.E + 5, 2]], dtype=torch.int32, device="cuda")
    ps = torch.empty((1, d.K), dtype=torch.int32, device="cuda")
    moe.cache_plan(ctx, cache, ids, 1, 0, ps)
    assert ctx.sync_status() == moe.MOE_ERR_RANGE
    assert ps.cpu().numpy().min() >= 0


# -------------------------------------------------------------- expert FFN
@pytest.mark.parametrize("d", [TINY, FULL], ids=["tiny", "full"])
@pytest.mark.parametrize("T", [1, 3, 11])
@pytest.mark.parametrize("with_yin", [False, True])
def test_expert_ffn_parity(O, d, T, with_yin):
    L = Layer(d, layer=1, seed=3, shared=False)
    ctx = moe.Ctx.from_dims(d, max_tokens=16)
    rng = np.random.default_rng(T)
    xb = synth.hidden_batch(3, range(T), 1, d.D)
    slots = np.stack([rng.choice(d.E, d.K, replace=False) for _ in range(T)]).astype(np.int32)
    w = rng.uniform(0.05, 0.3, size=(T, d.K)).astype(np.float32)
    y_in = rng.standard_normal((T, d.D)).astype(np.float32) if with_yin else None
    y = torch.empty((T, d.D), dtype=torch.float32, device="cuda")
    yb = torch.empty((T, d.D), dtype=torch.int16, device="cuda")
    moe.expert_ffn(ctx, bf16_tensor(xb), T, d.K, torch.from_numpy(slots).cuda(), torch.from_numpy(w).cuda(),
                   L.experts_t, L.stride, d.E, d.F, None if y_in is None else torch.from_numpy(y_in).cuda(), y, yb)
    ctx.sync()
    got = y.cpu().numpy()
    gotb = yb.cpu().numpy().view(np.uint16)
    for t in range(T):
        x = synth.bf16_bits_to_f32(xb[t]).astype(np.float64)
        ref = np.zeros(d.D) if y_in is None else y_in[t].astype(np.float64)
        for k in range(d.K):
            ref = ref + float(w[t, k]) * O.expert_ffn(L.blobs[slots[t, k]], d.D, d.F, x)
        assert rel_err(got[t], ref) <= TOL, (t, rel_err(got[t], ref))
        # bf16 output is the fp32 output rounded to nearest even
        assert np.array_equal(gotb[t], synth.to_bf16_bits(got[t]))


@pytest.mark.parametrize("d", [TINY, FULL], ids=["tiny", "full"])
def test_shared_width_expert_through_expert_ffn(O, d):
    """The shared expert (width FS) passed as top_k = 1, slot 0, weight 1."""
    ctx = moe.Ctx.from_dims(d, max_tokens=4)
    blob = synth.expert_blob(4, 0, 0, d.D, d.FS, shared=True)
    xb = synth.hidden_batch(4, range(2), 0, d.D)
    y = torch.empty((2, d.D), dtype=torch.float32, device="cuda")
    moe.expert_ffn(ctx, bf16_tensor(xb), 2, 1, torch.zeros((2, 1), dtype=torch.int32, device="cuda"),
                   torch.ones((2, 1), dtype=torch.float32, device="cuda"), torch.from_numpy(blob).cuda(),
                   0, 1, d.FS, None, y)
    ctx.sync()
    for t in range(2):
        ref = O.expert_ffn(blob, d.D, d.FS, synth.bf16_bits_to_f32(xb[t]).astype(np.float64))
        assert rel_err(y[t].cpu().numpy(), ref) <= TOL


def test_expert_ffn_argument_errors():
    d = TINY
    ctx = moe.Ctx.from_dims(d, max_tokens=4)
    x = torch.zeros((1, d.D), dtype=torch.int16, device="cuda")
    ps = torch.zeros((1, d.K), dtype=torch.int32, device="cuda")
    w = torch.zeros((1, d.K), dtype=torch.float32, device="cuda")
    y = torch.empty((1, d.D), dtype=torch.float32, device="cuda")
    blobs = torch.zeros((d.E, 256 * 256), dtype=torch.uint8, device="cuda")
    with pytest.raises(moe.MoeError) as ei:
        moe.expert_ffn(ctx, x, 0, d.K, ps, w, blobs, 256 * 256, d.E, d.F, None, y)     # T = 0
    assert ei.value.code == moe.MOE_ERR_ARG
    with pytest.raises(moe.MoeError):
        moe.expert_ffn(ctx, x, 1, d.K, ps, w, blobs, 1000, d.E, d.F, None, y)          # stride % 256
    with pytest.raises(moe.MoeError):
        moe.expert_ffn(ctx, x, 1, d.K, ps, w, blobs, 256 * 256, d.E, 100, None, y)     # unknown width


# ------------------------------------------------------------------ harness
@pytest.mark.parametrize("D", [512, 2816, 8192], ids=["512", "2816", "8192-looped"])
def test_residual_rmsnorm_harness(D):
    """The layer-chaining step of the benchmark: r += y exactly in fp32, and
    x_next = bf16(r / sqrt(mean(r^2) + 1e-6)) within one bf16 step of an
    fp64 evaluation (rows longer than the register path take the loop)."""
    d = synth.Dims(D=D, E=16, K=4, F=64, FS=128, G=64, L=1, S=6)
    T = 3
    ctx = moe.Ctx.from_dims(d, max_tokens=T)
    rng = np.random.default_rng(D)
    r0 = rng.standard_normal((T, D)).astype(np.float32)
    y0 = (0.3 * rng.standard_normal((T, D))).astype(np.float32)
    r = torch.from_numpy(r0).cuda()
    y = torch.from_numpy(y0).cuda()
    xn = torch.empty((T, D), dtype=torch.int16, device="cuda")
    moe.residual_rmsnorm(ctx, r, y, xn, T)
    ctx.sync()
    want_r = r0 + y0
    assert np.array_equal(r.cpu().numpy(), want_r)
    ref = want_r.astype(np.float64)
    ref = ref / np.sqrt(np.mean(ref * ref, axis=1, keepdims=True) + 1e-6)
    got = synth.bf16_bits_to_f32(xn.cpu().numpy().view(np.uint16)).astype(np.float64)
    assert np.all(np.abs(got - ref) <= np.abs(ref) * 2.0 ** -8 + 1e-30)
