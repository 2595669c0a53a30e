"""GPU parity of the whole layer (moe_layer_forward) against the CPU oracle on
the workloads of the pages' model shape: decode with every expert resident,
decode streaming from a pinned host store through the 16-slot LFU cache,
batched decode, and a 128-token prefill chunk with cold caches.

Inputs are seeded generator hidden states for every (token, layer), so the
oracle and the GPU see identical inputs; ids and cache traces must match bit
for bit, outputs within max|y - r| <= 2e-3 * max|r|."""
import os

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


def _check_token(O, L, xb, ids, gw, y):
    want_ids, want_w, _, want_y = L.oracle_token(O, xb)
    assert np.array_equal(ids, want_ids), (ids, want_ids)
    assert np.max(np.abs(gw - want_w)) <= GATE_TOL
    err = rel_err(y, want_y)
    assert err <= TOL, err
    return err


@pytest.mark.parametrize("kernel", ["layer", "split"])
@pytest.mark.parametrize("d", [TINY, FULL], ids=["tiny", "full"])
def test_decode_resident_single_layer(O, d, kernel, monkeypatch):
    """One layer, all experts resident, 16 sequential decode tokens: through the
    one-launch layer kernel and through the separate router / GEMV kernels."""
    monkeypatch.setenv("MOE_LAYER_KERNEL", "1" if kernel == "layer" else "0")
    L = Layer(d, layer=0, seed=0, zipf_s=None)
    ctx = moe.Ctx.from_dims(d, max_tokens=1)
    W = L.weights()
    y = torch.empty((1, d.D), dtype=torch.float32, device="cuda")
    ids = torch.empty((1, d.K), dtype=torch.int32, device="cuda")
    gw = torch.empty((1, d.K), dtype=torch.float32, device="cuda")
    for t in range(16):
        xb = synth.hidden(0, t, 0, d.D)
        moe.layer_forward(ctx, W, None, bf16_tensor(xb[None]), 1, t, None, y, ids=ids, gate_w=gw)
        ctx.sync()
        _check_token(O, L, xb, ids.cpu().numpy()[0], gw.cpu().numpy()[0], y.cpu().numpy()[0])


@pytest.mark.parametrize("kernel", ["layer", "split"])
@pytest.mark.parametrize("d", [TINY, FULL], ids=["tiny", "full"])
def test_decode_resident_with_next_layer(O, d, kernel, monkeypatch):
    """Two resident layers, the first called with the next layer named
    (moe_layer_forward_next, no cache: nothing to stage, exactly
    moe_layer_forward): results are the oracle's through either kernel path."""
    monkeypatch.setenv("MOE_LAYER_KERNEL", "1" if kernel == "layer" else "0")
    Ls = [Layer(d, layer=l, seed=4, zipf_s=None) for l in range(2)]
    ctx = moe.Ctx.from_dims(d, max_tokens=1)
    Ws = [L.weights() for L in Ls]
    nxt = moe.next_layer(Ws[1], None, Ls[1].bias_t)
    y = torch.empty((1, d.D), dtype=torch.float32, device="cuda")
    ids = torch.empty((1, d.K), dtype=torch.int32, device="cuda")
    gw = torch.empty((1, d.K), dtype=torch.float32, device="cuda")
    for t in range(6):
        for l, L in enumerate(Ls):
            xb = synth.hidden(4, t, l, d.D)
            if l == 0:
                moe.layer_forward_next(ctx, Ws[0], None, bf16_tensor(xb[None]), 1, t, None, y, nxt, ids=ids,
                                       gate_w=gw)
            else:
                moe.layer_forward(ctx, Ws[1], None, bf16_tensor(xb[None]), 1, t, None, y, ids=ids, gate_w=gw)
            ctx.sync()
            _check_token(O, L, xb, ids.cpu().numpy()[0], gw.cpu().numpy()[0], y.cpu().numpy()[0])


@pytest.mark.parametrize("d,T", [(TINY, 8), (FULL, 8), (FULL, 32)], ids=["tiny-8", "full-8", "full-32"])
def test_batched_decode_resident(O, d, T):
    L = Layer(d, layer=1, seed=2, zipf_s=None)
    ctx = moe.Ctx.from_dims(d, max_tokens=T)
    xb = synth.hidden_batch(2, range(T), 1, d.D)
    y = torch.empty((T, d.D), dtype=torch.float32, device="cuda")
    yb = torch.empty((T, d.D), dtype=torch.int16, device="cuda")
    ids = torch.empty((T, d.K), dtype=torch.int32, device="cuda")
    gw = torch.empty((T, d.K), dtype=torch.float32, device="cuda")
    moe.layer_forward(ctx, L.weights(), None, bf16_tensor(xb), T, 0, None, y, yb, ids, gw)
    ctx.sync()
    ids_h, gw_h, y_h = ids.cpu().numpy(), gw.cpu().numpy(), y.cpu().numpy()
    sample = range(T) if d is TINY else [0, 1, T // 2, T - 1]
    for t in sample:
        _check_token(O, L, xb[t], ids_h[t], gw_h[t], y_h[t])
    assert np.array_equal(yb.cpu().numpy().view(np.uint16), synth.to_bf16_bits(y_h))


def _streaming(O, d, layers, tokens, S, check_y_every=1, T=1, policy=0, period=0, file_dir=None, prefetch=0,
               same_x=False, stats=None, direct=False, counters=None, deep=False):
    Ls = [Layer(d, layer=l, seed=1, zipf_s=1.1, resident=False, pinned=True) for l in range(layers)]
    ctx = moe.Ctx.from_dims(d, max_tokens=T, S=S)
    caches, states, slotbufs = [], [], []
    fds = []
    for li, L in enumerate(Ls):
        state = torch.empty(ctx.state_words(), dtype=torch.int32, device="cuda")
        slots = torch.empty((S, L.stride), dtype=torch.uint8, device="cuda")
        if file_dir is not None:
            # the layer's experts in a file at a 4 KB-aligned stride, after a 4 KB header
            fstride = (L.nb + 4095) // 4096 * 4096
            path = os.path.join(file_dir, f"layer{li}.experts")
            with open(path, "wb") as f:
                f.write(b"\0" * 4096)
                for e in range(d.E):
                    f.write(L.blobs[e].tobytes() + b"\0" * (fstride - L.nb))
            fd = os.open(path, os.O_RDONLY)
            fds.append(fd)
            c = moe.slot_cache(slots, L.stride, state, None, fstride, policy=policy, decay_period=period,
                               store_fd=fd, store_file_offset=4096)
        else:
            c = moe.slot_cache(slots, L.stride, state, L.store_t, L.stride, policy=policy, decay_period=period,
                               direct=direct)
        moe.cache_reset(ctx, c)
        caches.append(c)
        states.append(state)
        slotbufs.append(slots)
    ost = [oracle.LfuState(d.E, S, policy, period) for _ in Ls]
    y = torch.empty((T, d.D), dtype=torch.float32, device="cuda")
    ids = torch.empty((T, d.K), dtype=torch.int32, device="cuda")
    gw = torch.empty((T, d.K), dtype=torch.float32, device="cuda")
    tr = moe.Trace(d.E)
    hits = misses = 0
    rep1 = rep2 = 0
    last_use = [np.zeros(d.E, dtype=np.int64) for _ in Ls]  # host copy, for the repeat counters
    ctx.stats_reset()
    if prefetch:
        moe.prefetch_configure(ctx, prefetch)
        # deep: layer l may also stage for layer l+2 when layer l+1 has nothing to stage
        after = [moe.next_layer(Ls[l + 2].weights(resident=False), caches[l + 2], Ls[l + 2].bias_t)
                 if deep and l + 2 < layers else None for l in range(layers)]
        nexts = [moe.next_layer(Ls[l + 1].weights(resident=False), caches[l + 1], Ls[l + 1].bias_t, after=after[l])
                 for l in range(layers - 1)] + [None]
        later_misses = 0  # misses of layers 1.. (the ones a prefetch can serve)
    for step in range(tokens):
        for l, L in enumerate(Ls):
            # same_x: every layer of a token sees one input, so the look-ahead
            # router predicts the next layer's experts exactly
            xb = synth.hidden_batch(1, range(step * T, step * T + T), 0 if same_x else l, d.D)
            if prefetch:
                moe.layer_forward_next(ctx, L.weights(resident=False), caches[l], bf16_tensor(xb), T, step,
                                       L.bias_t, y, nexts[l], ids=ids, gate_w=gw, trace=tr)
            else:
                moe.layer_forward(ctx, L.weights(resident=False), caches[l], bf16_tensor(xb), T, step, L.bias_t, y,
                                  ids=ids, gate_w=gw, trace=tr)
            ctx.sync()
            got = tr.result()
            ids_h = ids.cpu().numpy()
            oids = np.stack([O.topk(O.router_logits(xb[t], L.wq, L.ws, L.bias, d.E, d.D, d.G), d.K)
                             for t in range(T)])
            assert np.array_equal(ids_h, oids), (step, l)
            want = O.lfu_plan(ost[l], oids, step)
            for key in ("expert", "slot", "hit", "victim", "wave"):
                assert np.array_equal(got[key], want[key]), (step, l, key)
            nmiss = int((want["hit"] == 0).sum())
            assert got["misses"] == nmiss and got["h2d_bytes"] == nmiss * L.nb
            hits += int(want["hit"].sum())
            misses += nmiss
            for e in want["expert"]:
                lu = last_use[l][e]
                rep1 += int(lu != 0 and lu == step)
                rep2 += int(lu != 0 and lu + 1 >= step)
            last_use[l][want["expert"]] = step + 1
            if prefetch and l > 0:
                later_misses += nmiss
            if step % check_y_every == 0:
                for t in range(T):
                    _check_token(O, L, xb[t], ids_h[t], gw.cpu().numpy()[t], y.cpu().numpy()[t])
            # slot contents equal the store's blob of the expert the oracle placed there
            if step % 7 == 0:
                sl = slotbufs[l].cpu().numpy()
                for s_, e_ in enumerate(ost[l].expert_in):
                    if e_ >= 0:
                        assert np.array_equal(sl[s_, :L.nb], L.blobs[e_]), (step, l, s_, e_)
    for fd in fds:
        os.close(fd)
    # the device counters agree with the oracle's plans
    st = ctx.stats()
    assert st["calls"] == layers * tokens
    assert (st["hits"], st["misses"]) == (hits, misses)
    assert st["miss_bytes"] == misses * Ls[0].nb
    assert (st["repeat_prev"], st["repeat_prev2"], st["planned"]) == (rep1, rep2, hits + misses)
    if counters is not None:
        counters.update(st)
    if prefetch and stats is not None:
        stats["issued"], stats["used"] = moe.prefetch_stats(ctx)
        stats["later_misses"], stats["nb"] = later_misses, Ls[0].nb
    return hits, misses


def test_streaming_decode_tiny(O):
    _streaming(O, TINY, layers=3, tokens=40, S=6)


def test_streaming_decode_full(O):
    """Three layers of the real shape, 24 tokens, 16 slots, Zipf(1.1) router
    bias: traces bit-exact every token, outputs checked every 4th token."""
    h, m = _streaming(O, FULL, layers=3, tokens=24, S=16, check_y_every=4)
    assert h + m == 3 * 24 * 8


def test_streaming_batched_decode(O):
    _streaming(O, FULL, layers=1, tokens=4, S=16, check_y_every=2, T=4)


@pytest.mark.parametrize("S", [16, 8])
def test_prefill_chunk_cold_cache(O, S):
    """A 128-token chunk through a cold 16-slot (and 8-slot) cache: the
    distinct experts exceed the slots, so the plan runs in waves; traces must
    match and sampled tokens' outputs too."""
    d, T = FULL, 128
    L = Layer(d, layer=2, seed=5, zipf_s=1.1, resident=False, pinned=True)
    ctx = moe.Ctx.from_dims(d, max_tokens=T, S=S)
    state = torch.empty(ctx.state_words(), dtype=torch.int32, device="cuda")
    slots = torch.empty((S, L.stride), dtype=torch.uint8, device="cuda")
    cache = moe.slot_cache(slots, L.stride, state, L.store_t, L.stride)
    moe.cache_reset(ctx, cache)
    xb = synth.hidden_batch(5, range(T), 2, d.D)
    y = torch.empty((T, d.D), dtype=torch.float32, device="cuda")
    ids = torch.empty((T, d.K), dtype=torch.int32, device="cuda")
    gw = torch.empty((T, d.K), dtype=torch.float32, device="cuda")
    tr = moe.Trace(d.E)
    moe.layer_forward(ctx, L.weights(resident=False), cache, bf16_tensor(xb), T, 0, L.bias_t, y, ids=ids,
                      gate_w=gw, trace=tr)
    ctx.sync()
    got = tr.result()
    oids = np.stack([O.topk(O.router_logits(xb[t], L.wq, L.ws, L.bias, d.E, d.D, d.G), d.K) for t in range(T)])
    assert np.array_equal(ids.cpu().numpy(), oids)
    want = O.lfu_plan(oracle.LfuState(d.E, S), oids, 0)
    for key in ("expert", "slot", "hit", "victim", "wave"):
        assert np.array_equal(got[key], want[key]), key
    assert got["waves"] == want["waves"] > 1
    assert got["h2d_bytes"] == got["misses"] * L.nb == got["n_distinct"] * L.nb  # cold: every expert misses
    for t in (0, 1, 63, 127):
        _check_token(O, L, xb[t], ids.cpu().numpy()[t], gw.cpu().numpy()[t], y.cpu().numpy()[t])


def test_resident_no_shared_expert(O):
    d = TINY
    L = Layer(d, layer=0, seed=9, zipf_s=None, shared=False)
    L.shared = None
    ctx = moe.Ctx.from_dims(d, max_tokens=2)
    xb = synth.hidden_batch(9, range(2), 0, d.D)
    y = torch.empty((2, d.D), dtype=torch.float32, device="cuda")
    ids = torch.empty((2, d.K), dtype=torch.int32, device="cuda")
    gw = torch.empty((2, d.K), dtype=torch.float32, device="cuda")
    moe.layer_forward(ctx, L.weights(), None, bf16_tensor(xb), 2, 0, None, y, ids=ids, gate_w=gw)
    ctx.sync()
    for t in range(2):
        _check_token(O, L, xb[t], ids.cpu().numpy()[t], gw.cpu().numpy()[t], y.cpu().numpy()[t])


@pytest.mark.parametrize("policy,period", [(moe.MOE_POLICY_LRU, 0), (moe.MOE_POLICY_LFU_DECAY, 5),
                                           (moe.MOE_POLICY_LFU_IN_CACHE, 0)], ids=["lru", "decay5", "in-cache"])
def test_streaming_decode_policies(O, policy, period):
    """Whole streamed layers under the replacement-rule variants: traces,
    slot contents and outputs against the oracle."""
    _streaming(O, TINY, layers=2, tokens=30, S=6, policy=policy, period=period)


@pytest.mark.parametrize("d,layers,tokens,S,every", [(TINY, 3, 30, 6, 1), (FULL, 3, 8, 16, 4)],
                         ids=["tiny", "full"])
def test_streaming_decode_lookahead_exact(O, d, layers, tokens, S, every):
    """Look-ahead prefetch with one input per token for every layer: the
    prediction is then exact, so every miss of layers 1.. is filled from a
    staged blob and nothing staged is wasted; traces, slot contents and outputs
    are still those of the oracle."""
    st = {}
    _streaming(O, d, layers=layers, tokens=tokens, S=S, check_y_every=every, prefetch=d.K, same_x=True, stats=st)
    assert st["later_misses"] > 0
    assert st["issued"] == st["used"] == st["later_misses"] * st["nb"]


@pytest.mark.parametrize("d,layers,tokens,S,every", [(TINY, 4, 40, 6, 1), (FULL, 4, 10, 16, 3)], ids=["tiny", "full"])
def test_streaming_decode_lookahead_two_layers(O, d, layers, tokens, S, every):
    """One look-ahead buffer that may stage for the layer after next when the
    next layer is predicted to miss nothing (exact predictions: one input per
    token for every layer).  Traces, slots and outputs are the oracle's; every
    staged blob is used."""
    st = {}
    _streaming(O, d, layers=layers, tokens=tokens, S=S, check_y_every=every, prefetch=1, same_x=True, stats=st,
               deep=True)
    assert st["later_misses"] > 0 and st["issued"] > 0
    assert st["used"] == st["issued"]


def test_streaming_decode_lookahead_mispredicted(O):
    """Look-ahead prefetch with unrelated inputs per layer (mostly wrong
    guesses, fewer buffers than K): same traces, slots and outputs; the used
    bytes never exceed the issued ones."""
    st = {}
    _streaming(O, TINY, layers=3, tokens=30, S=6, prefetch=3, stats=st)
    assert 0 < st["issued"] and st["used"] <= st["issued"]
    assert st["used"] <= st["later_misses"] * st["nb"]


def test_streaming_decode_from_file(O, tmp_path):
    """Misses read from per-layer expert files with positional reads into
    pinned staging, then copied to the slots: traces, slot contents and
    outputs as with the pinned host store."""
    _streaming(O, TINY, layers=2, tokens=30, S=6, file_dir=str(tmp_path))
    _streaming(O, FULL, layers=1, tokens=6, S=16, check_y_every=3, file_dir=str(tmp_path))


def test_prefill_chunk_from_file(O, tmp_path):
    """A 4-token batch through the file store with waves (more distinct experts than slots)."""
    _streaming(O, TINY, layers=1, tokens=3, S=6, T=4, file_dir=str(tmp_path))


def test_file_store_short_file_is_an_io_error(tmp_path):
    d = TINY
    L = Layer(d, layer=0, seed=1, zipf_s=1.1, resident=False, pinned=False)
    ctx = moe.Ctx.from_dims(d, max_tokens=1, S=6)
    state = torch.empty(ctx.state_words(), dtype=torch.int32, device="cuda")
    slots = torch.empty((6, L.stride), dtype=torch.uint8, device="cuda")
    path = os.path.join(str(tmp_path), "short.experts")
    with open(path, "wb") as f:
        f.write(b"\1" * 4096)            # far shorter than E blobs
    fd = os.open(path, os.O_RDONLY)
    try:
        c = moe.slot_cache(slots, L.stride, state, None, L.stride, store_fd=fd)
        moe.cache_reset(ctx, c)
        x = bf16_tensor(synth.hidden(1, 0, 0, d.D)[None])
        y = torch.empty((1, d.D), dtype=torch.float32, device="cuda")
        with pytest.raises(moe.MoeError) as ei:
            moe.layer_forward(ctx, L.weights(resident=False), c, x, 1, 0, L.bias_t, y)
        assert ei.value.code == moe.MOE_ERR_IO
    finally:
        os.close(fd)
    ctx.sync()


def test_minimum_slots_equal_top_k(O):
    """S = K: every wave fills the whole cache; still bit-exact."""
    d = TINY
    _streaming(O, d, layers=1, tokens=30, S=d.K)


@pytest.mark.parametrize("d,T", [(TINY, 40), (TINY, 128), (FULL, 37), (FULL, 128)],
                         ids=["tiny-40", "tiny-128", "full-37", "full-128"])
def test_prefill_resident_tensor_core(O, d, T):
    """Batches run the tcgen05 grouped GEMM (tokens grouped per expert, fp16
    dequantised weight tiles, fp32 accumulation in tensor memory)."""
    L = Layer(d, layer=4, seed=13, zipf_s=1.1)
    ctx = moe.Ctx.from_dims(d, max_tokens=T)
    xb = synth.hidden_batch(13, range(T), 4, d.D)
    y = torch.empty((T, d.D), dtype=torch.float32, device="cuda")
    yb = torch.empty((T, d.D), dtype=torch.int16, device="cuda")
    ids = torch.empty((T, d.K), dtype=torch.int32, device="cuda")
    gw = torch.empty((T, d.K), dtype=torch.float32, device="cuda")
    moe.layer_forward(ctx, L.weights(), None, bf16_tensor(xb), T, 0, L.bias_t, y, yb, ids, gw)
    ctx.sync()
    ids_h, gw_h, y_h = ids.cpu().numpy(), gw.cpu().numpy(), y.cpu().numpy()
    sample = range(T) if d is TINY else [0, 1, T // 3, T // 2, T - 1]
    for t in sample:
        _check_token(O, L, xb[t], ids_h[t], gw_h[t], y_h[t])
    assert np.array_equal(yb.cpu().numpy().view(np.uint16), synth.to_bf16_bits(y_h))


@pytest.mark.parametrize("d,layers,tokens,S,every", [(TINY, 3, 40, 6, 1), (FULL, 3, 24, 16, 4)], ids=["tiny", "full"])
def test_streaming_decode_direct_fill(O, d, layers, tokens, S, every):
    """Misses read by the layer kernel straight from the pinned host store and
    written into their slots as it computes: traces, slot contents (the write
    back) and outputs against the oracle, and the device counters."""
    cnt = {}
    h, m = _streaming(O, d, layers=layers, tokens=tokens, S=S, check_y_every=every, direct=True, counters=cnt)
    assert m > 0 and h > 0
    assert h + m == layers * tokens * d.K


@pytest.mark.parametrize("policy,period", [(moe.MOE_POLICY_LRU, 0), (moe.MOE_POLICY_LFU_DECAY, 5),
                                           (moe.MOE_POLICY_LFU_IN_CACHE, 0)], ids=["lru", "decay5", "in-cache"])
def test_streaming_direct_fill_policies(O, policy, period):
    _streaming(O, TINY, layers=2, tokens=30, S=6, policy=policy, period=period, direct=True)


def test_direct_fill_with_batches_copies(O):
    """A direct-source cache given a 4-token batch: the plan runs in waves and
    the copy engine fills the slots, as for the pinned store."""
    _streaming(O, TINY, layers=1, tokens=3, S=6, T=4, direct=True)


def test_layer_kernel_nan_logits(O):
    """A NaN router logit: no order exists; the one-launch layer reports
    MOE_ERR_NAN and uses experts 0..K-1 with equal weights, like the router."""
    d = TINY
    L = Layer(d, layer=0, seed=3, zipf_s=None)
    ctx = moe.Ctx.from_dims(d, max_tokens=1)
    bias = np.zeros(d.E, dtype=np.float32)
    bias[5] = np.nan
    y = torch.empty((1, d.D), dtype=torch.float32, device="cuda")
    ids = torch.empty((1, d.K), dtype=torch.int32, device="cuda")
    gw = torch.empty((1, d.K), dtype=torch.float32, device="cuda")
    moe.layer_forward(ctx, L.weights(), None, bf16_tensor(synth.hidden(3, 0, 0, d.D)[None]), 1, 0,
                      torch.from_numpy(bias).cuda(), y, ids=ids, gate_w=gw)
    assert ctx.sync_status() == moe.MOE_ERR_NAN
    assert np.array_equal(ids.cpu().numpy()[0], np.arange(d.K))
    assert np.allclose(gw.cpu().numpy()[0], 1.0 / d.K)
    ctx.close()


def test_direct_fill_rejects_unpinned_store():
    d = TINY
    L = Layer(d, layer=0, seed=1, zipf_s=1.1, resident=False, pinned=False)
    ctx = moe.Ctx.from_dims(d, max_tokens=1, S=6)
    state = torch.empty(ctx.state_words(), dtype=torch.int32, device="cuda")
    slots = torch.empty((6, L.stride), dtype=torch.uint8, device="cuda")
    pageable = torch.from_numpy(L.host)  # not pinned: the kernel cannot read it
    c = moe.slot_cache(slots, L.stride, state, pageable, L.stride, direct=True)
    moe.cache_reset(ctx, c)
    y = torch.empty((1, d.D), dtype=torch.float32, device="cuda")
    with pytest.raises(moe.MoeError) as ei:
        moe.layer_forward(ctx, L.weights(resident=False), c, bf16_tensor(synth.hidden(1, 0, 0, d.D)[None]), 1, 0,
                          L.bias_t, y)
    assert ei.value.code == moe.MOE_ERR_ARG
    ctx.sync()
    ctx.close()


def test_missing_ready_word_times_out(O, monkeypatch):
    """Per-miss completion (MOE_PER_MISS=1): a one-token miss copied from
    pinned memory is announced by a stream memory write after its copy, and
    the routed experts' kernel waits for that word (bounded).  With the first write of a call left
    out on the host (MOE_INJECT_SKIP_READY=1) the wait runs out: the call
    reports MOE_ERR_TIMEOUT within seconds and the context stays usable (a
    resident call on it then matches the oracle)."""
    import time

    d = TINY
    S = 6
    monkeypatch.setenv("MOE_PER_MISS", "1")
    monkeypatch.setenv("MOE_INJECT_SKIP_READY", "1")
    L = Layer(d, layer=0, seed=1, zipf_s=1.1, resident=True, pinned=True)
    ctx = moe.Ctx.from_dims(d, max_tokens=1, S=S)
    monkeypatch.delenv("MOE_INJECT_SKIP_READY")
    monkeypatch.delenv("MOE_PER_MISS")
    state = torch.empty(ctx.state_words(), dtype=torch.int32, device="cuda")
    slots = torch.empty((S, L.stride), dtype=torch.uint8, device="cuda")
    c = moe.slot_cache(slots, L.stride, state, L.store_t, L.stride)
    moe.cache_reset(ctx, c)
    y = torch.empty((1, d.D), dtype=torch.float32, device="cuda")
    xb = synth.hidden(1, 0, 0, d.D)
    t0 = time.time()
    moe.layer_forward(ctx, L.weights(resident=False), c, bf16_tensor(xb[None]), 1, 0, L.bias_t, y)
    assert ctx.sync_status() == moe.MOE_ERR_TIMEOUT  # a cold cache: every selection misses
    assert time.time() - t0 < 15.0
    # the same context, resident experts (no copies): correct again
    moe.layer_forward(ctx, L.weights(), None, bf16_tensor(xb[None]), 1, 0, L.bias_t, y)
    assert ctx.sync_status() == 0
    want = L.oracle_token(O, xb)[3]
    assert rel_err(y.cpu().numpy()[0].astype(np.float64), want) <= TOL
    ctx.close()


@pytest.mark.parametrize("d,layers,tokens,S,every,prefetch", [(TINY, 3, 30, 6, 1, 0), (FULL, 2, 8, 16, 4, 0),
                                                              (FULL, 3, 8, 16, 4, 8)],
                         ids=["tiny", "full", "full-lookahead"])
def test_streaming_decode_per_miss_ready(O, monkeypatch, d, layers, tokens, S, every, prefetch):
    """Per-miss completion enabled (MOE_PER_MISS=1): list B starts before its
    blobs have landed and waits per blob; staged look-ahead blobs (device to
    device copies, which may run as kernels) are joined by event first.
    Traces, slot contents and outputs are the oracle's."""
    monkeypatch.setenv("MOE_PER_MISS", "1")
    _streaming(O, d, layers=layers, tokens=tokens, S=S, check_y_every=every, prefetch=prefetch,
               same_x=prefetch > 0)
