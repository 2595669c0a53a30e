"""GPU parity of the chained decode: the benchmark's own token loop
(bench.decode_token), where layer l+1's input is the residual stream after
layer l, RMS-normalised, so every layer's routing depends on the layers below
it, as in the pages' token loop ("TurboFieldfare: motor open source ...",
section "Proceso de generacion de tokens": the routed-layer loop repeats token
by token; "Gemma 4 26B en ~2 GB de RAM ...", section "Por que funciona").

The oracle is teacher-forced on the GPU's own bf16 input of every (token,
layer): its router, top-K, LFU plan (one state per layer, carried across the
tokens) and layer output are compared with the GPU's at every step, and its
chaining step (residual + RMS, fp64) with the harness kernel's.  Ids, gate
weights, plan traces and slot contents bit for bit (gate weights within 1e-5);
outputs within max|y - r| <= 2e-3 max|r|; the chained bf16 input within one
bf16 unit in the last place of the oracle's rounding of the fp64 value."""
import argparse
import gc

import numpy as np
import pytest
import torch

import bench
import oracle
from expert_streaming_decode_b200 import synth
from gpu_data import GATE_TOL, TOL, rel_err

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def O():
    return oracle.get()


def _args(layers, slots, prefetch, fill, seed=0):
    return argparse.Namespace(layers=layers, slots=slots, seed=seed, zipf=1.1, zipf_lambda=synth.ZIPF_LAMBDA,
                              policy="lfu", decay_period=0, store_file=None, direct=False, prefetch=prefetch,
                              fill=fill)


def _bf16_ulp_diff(a, b):
    """|a - b| in bf16 units in the last place (same-sign finite values)."""
    fa = synth.bf16_bits_to_f32(a).astype(np.float64)
    fb = synth.bf16_bits_to_f32(b).astype(np.float64)
    ulp = np.exp2(np.floor(np.log2(np.maximum(np.abs(fb), 2.0 ** -126))) - 7)
    return np.abs(fa - fb) / ulp


def _chain(O, d, layers, tokens, slots, prefetch, y_samples, fill="copy", slot_every=4):
    args = _args(layers, slots, prefetch, fill)
    model = bench.Model(args, synth.Dims(**{**d.as_dict(), "L": layers, "S": slots}), max_tokens=1, streaming=True)
    moe = model.moe
    nb = model.nb
    store = model.store.numpy()
    routers = [synth.router_weights(args.seed, l, d.E, d.D) for l in range(layers)]
    biases = [synth.zipf_bias(args.seed, l, d.E, s=args.zipf, lam=args.zipf_lambda) for l in range(layers)]
    shared = [synth.expert_blob(args.seed, l, 0, d.D, d.FS, shared=True) for l in range(layers)]
    ost = [oracle.LfuState(d.E, slots) for _ in range(layers)]
    dev = torch.device("cuda")
    x0 = torch.empty((1, d.D), dtype=torch.int16, device=dev)
    x = torch.empty((1, d.D), dtype=torch.int16, device=dev)
    r = torch.empty((1, d.D), dtype=torch.float32, device=dev)
    y = torch.empty((1, d.D), dtype=torch.float32, device=dev)
    ids = torch.empty((1, d.K), dtype=torch.int32, device=dev)
    gw = torch.empty((1, d.K), dtype=torch.float32, device=dev)
    tr = moe.Trace(d.E)
    acc = {"misses": 0, "distinct": 0, "h2d": 0}
    model.reset()
    stats = {"ids": 0, "plans": 0, "outputs": 0, "chained": 0, "slots": 0, "ulp1": 0, "misses": 0}
    for t in range(tokens):
        xb0 = synth.hidden(args.seed + 17, t, 0, d.D)
        x0.copy_(torch.from_numpy(xb0.view(np.int16)[None].copy()))
        prev = {}

        def on_layer(l, cur, y_t, r_t):
            torch.cuda.synchronize()
            model.ctx.sync()
            xl = cur.cpu().numpy().view(np.uint16)[0].copy()
            yl = y_t.cpu().numpy()[0].astype(np.float64)
            rl = r_t.cpu().numpy()[0].astype(np.float64)
            got_ids, got_w = ids.cpu().numpy()[0], gw.cpu().numpy()[0]
            plan = tr.result()
            # the chained input: layer 0 reads the token's state; layer l > 0
            # reads the oracle's chaining step applied to the GPU's r and y of l - 1
            if l == 0:
                assert np.array_equal(xl, xb0)
                assert np.array_equal(rl, synth.bf16_bits_to_f32(xb0).astype(np.float64))
            else:
                r_want, x_want = O.residual_rmsnorm(prev["r"], prev["y"])
                # fp32 residual add on the GPU: within half an fp32 ulp of the exact sum
                assert np.all(np.abs(rl - r_want) <= np.abs(r_want) * 2.0 ** -24 + 1e-30), (t, l)
                du = _bf16_ulp_diff(xl, x_want)
                assert du.max() <= 1.0, (t, l, du.max())
                stats["ulp1"] += int((du > 0).sum())
                stats["chained"] += 1
            wq, ws = routers[l]
            lg = O.router_logits(xl, wq, ws, biases[l], d.E, d.D, d.G)
            want_ids = O.topk(lg, d.K)
            assert np.array_equal(got_ids, want_ids), (t, l, got_ids, want_ids)
            assert np.max(np.abs(got_w - O.gate_weights(lg, want_ids))) <= GATE_TOL, (t, l)
            stats["ids"] += 1
            want = O.lfu_plan(ost[l], want_ids[None], t)
            for key in ("expert", "slot", "hit", "victim", "wave"):
                assert np.array_equal(plan[key], want[key]), (t, l, key)
            nmiss = int((want["hit"] == 0).sum())
            assert plan["misses"] == nmiss and plan["h2d_bytes"] == nmiss * nb, (t, l)
            stats["plans"] += 1
            stats["misses"] += nmiss
            if (t, l) in y_samples:
                _, _, _, want_y = O.moe_token(d.as_dict(), xl, wq, ws, biases[l], shared[l],
                                              [store[l, e, :nb] for e in range(d.E)])
                err = rel_err(yl, want_y)
                assert err <= TOL, (t, l, err)
                stats["outputs"] += 1
            if t % slot_every == slot_every - 1:
                sl = model.slots[l].cpu().numpy()
                for s_, e_ in enumerate(ost[l].expert_in):
                    if e_ >= 0:
                        assert np.array_equal(sl[s_, :nb], store[l, e_, :nb]), (t, l, s_, e_)
                stats["slots"] += 1
            prev["r"], prev["y"] = rl, yl

        bench.decode_token(model, x0, r, x, y, 1, t, tr=tr, trace_acc=acc, on_layer=on_layer, ids=ids, gate_w=gw)
    torch.cuda.synchronize()
    model.ctx.sync()
    if prefetch:
        issued, used = moe.prefetch_stats(model.ctx)
        stats["pf_issued"], stats["pf_used"] = issued, used
        assert used <= issued
    model.ctx.close()
    assert stats["ids"] == stats["plans"] == tokens * layers
    assert stats["chained"] == tokens * (layers - 1)
    assert stats["outputs"] == len(y_samples)
    return stats


@pytest.mark.parametrize("fill,prefetch", [("copy", 0), ("copy", 2), ("direct", 0)],
                         ids=["copy", "copy-lookahead-2", "direct"])
def test_chained_decode_tiny_30_layers(O, fill, prefetch):
    """30 chained layers of the scaled-down shape (6 slots), 24 tokens: every
    (token, layer) checked, outputs too."""
    d = synth.TINY
    samples = {(t, l) for t in range(24) for l in range(30)}
    st = _chain(O, d, layers=30, tokens=24, slots=6, prefetch=prefetch, y_samples=samples, fill=fill)
    assert st["misses"] > 0
    if prefetch:
        assert st["pf_used"] > 0


@pytest.mark.parametrize("fill,prefetch", [("copy", 0), ("copy", 1), ("direct", 0)],
                         ids=["copy", "copy-lookahead-1", "direct"])
def test_chained_decode_full_shape(O, fill, prefetch):
    """8 chained layers of the 26B-A4B shape, 16 slots, Zipf(1.1), 16 tokens:
    ids, gate weights, plans, chained inputs at every (token, layer), slot
    contents every 4th token, outputs on a sample spread over tokens and
    layers (the oracle's fp64 layer takes about a second each)."""
    d = synth.GEMMA4_26B
    samples = {(0, 0), (0, 7), (1, 3), (3, 1), (5, 6), (7, 2), (8, 5), (10, 0), (11, 4), (13, 7), (15, 1),
               (15, 6)}
    st = _chain(O, d, layers=8, tokens=16, slots=16, prefetch=prefetch, y_samples=samples, fill=fill)
    assert st["misses"] > 0
    if prefetch:
        assert st["pf_issued"] > 0


def test_chained_decode_headline_workload(O):
    """The benchmark's headline workload at its full size: 30 chained layers of
    the 26B-A4B shape, 16 slots, Zipf(1.1) at the default bias strength, misses
    copied by the copy engine with one look-ahead buffer, 25 tokens (the 5
    warm-up and 20 timed tokens of the round-end command).  Ids, gate weights,
    plans and chained inputs at every (token, layer); slot contents every 8th
    token; outputs on a sample spread over tokens and layers."""
    d = synth.GEMMA4_26B
    samples = {(0, 0), (2, 29), (6, 14), (11, 7), (15, 22), (19, 3), (22, 18), (24, 29)}
    st = _chain(O, d, layers=30, tokens=25, slots=16, prefetch=1, y_samples=samples, fill="copy", slot_every=8)
    assert st["misses"] > 0 and st["pf_issued"] > 0
    # the early tokens of the default workload miss in the pages' band
    hit = 1.0 - st["misses"] / (25 * 30 * d.K)
    assert 0.5 < hit < 0.8, hit


def _chain_batch(O, d, layers, T, slots, streaming, y_samples, seed=0, zipf=1.1):
    """One step of the benchmark's multi-token loop (a batched decode step on
    resident experts, or a prefill chunk through cold slot caches), with the
    oracle teacher-forced on every layer's bf16 input rows."""
    args = _args(layers, slots, 0, "copy", seed=seed)
    args.zipf = zipf  # 0: no popularity bias (the resident workload's uniform router)
    model = bench.Model(args, synth.Dims(**{**d.as_dict(), "L": layers, "S": slots}), max_tokens=T,
                        streaming=streaming)
    moe = model.moe
    nb = model.nb
    routers = [synth.router_weights(args.seed, l, d.E, d.D) for l in range(layers)]
    biases = [synth.zipf_bias(args.seed, l, d.E, s=args.zipf, lam=args.zipf_lambda) if zipf > 0 else None
              for l in range(layers)]
    shared = [synth.expert_blob(args.seed, l, 0, d.D, d.FS, shared=True) for l in range(layers)]
    dev = torch.device("cuda")
    x0 = torch.empty((T, d.D), dtype=torch.int16, device=dev)
    x = torch.empty((T, d.D), dtype=torch.int16, device=dev)
    r = torch.empty((T, d.D), dtype=torch.float32, device=dev)
    y = torch.empty((T, d.D), dtype=torch.float32, device=dev)
    ids = torch.empty((T, d.K), dtype=torch.int32, device=dev)
    gw = torch.empty((T, d.K), dtype=torch.float32, device=dev)
    tr = moe.Trace(d.E) if streaming else None
    acc = {"misses": 0, "distinct": 0, "h2d": 0}
    model.reset()
    xb0 = synth.hidden_batch(args.seed + 17, range(T), 0, d.D)
    x0.copy_(torch.from_numpy(xb0.view(np.int16).copy()))
    stats = {"layers": 0, "outputs": 0, "waves": 0, "misses": 0}
    prev = {}

    def blobs(l):
        if streaming:
            return [model.store.numpy()[l, e, :nb] for e in range(d.E)]
        return [model.experts[l, e, :nb].cpu().numpy() for e in range(d.E)]

    def on_layer(l, cur, y_t, r_t):
        torch.cuda.synchronize()
        model.ctx.sync()
        xl = cur.cpu().numpy().view(np.uint16).copy()
        yl = y_t.cpu().numpy().astype(np.float64)
        rl = r_t.cpu().numpy().astype(np.float64)
        got_ids, got_w = ids.cpu().numpy(), gw.cpu().numpy()
        if l == 0:
            assert np.array_equal(xl, xb0)
        else:
            for t in range(T):
                r_want, x_want = O.residual_rmsnorm(prev["r"][t], prev["y"][t])
                assert np.all(np.abs(rl[t] - r_want) <= np.abs(r_want) * 2.0 ** -24 + 1e-30), (t, l)
                assert _bf16_ulp_diff(xl[t], x_want).max() <= 1.0, (t, l)
        wq, ws = routers[l]
        lgs = [O.router_logits(xl[t], wq, ws, biases[l], d.E, d.D, d.G) for t in range(T)]
        want_ids = np.stack([O.topk(lg, d.K) for lg in lgs])
        assert np.array_equal(got_ids, want_ids), l
        for t in range(T):
            assert np.max(np.abs(got_w[t] - O.gate_weights(lgs[t], want_ids[t]))) <= GATE_TOL, (t, l)
        if streaming:
            plan = tr.result()
            want = O.lfu_plan(oracle.LfuState(d.E, slots), want_ids, 0)  # every chunk starts cold
            for key in ("expert", "slot", "hit", "victim", "wave"):
                assert np.array_equal(plan[key], want[key]), (l, key)
            assert plan["waves"] == want["waves"]
            stats["waves"] += plan["waves"]
            stats["misses"] += plan["misses"]
        rows = [t for (t, ll) in y_samples if ll == l]
        if rows:
            bl = blobs(l)
            for t in rows:
                _, _, _, want_y = O.moe_token(d.as_dict(), xl[t], wq, ws, biases[l], shared[l], bl)
                err = rel_err(yl[t], want_y)
                assert err <= TOL, (t, l, err)
                stats["outputs"] += 1
        stats["layers"] += 1
        prev["r"], prev["y"] = rl, yl

    bench.decode_token(model, x0, r, x, y, T, 0, tr=tr, trace_acc=acc if streaming else None, on_layer=on_layer,
                       ids=ids, gate_w=gw)
    torch.cuda.synchronize()
    model.ctx.sync()
    model.ctx.close()
    assert stats["layers"] == layers and stats["outputs"] == len(y_samples)
    return stats


@pytest.mark.parametrize("T", [8, 32])
def test_chained_batched_decode_resident_30_layers(O, T):
    """The resident batched-decode workload at full size: 30 chained layers
    of the 26B-A4B shape with every expert in HBM, a step of T tokens through
    the tensor-core grouped GEMM (uniform router, as the benchmark runs it).
    Ids and gate weights of every token at every layer, the chained inputs,
    and outputs on a sample of (token, layer)."""
    d = synth.GEMMA4_26B
    samples = {(0, 0), (T - 1, 4), (T // 2, 11), (1, 19), (T - 2, 25), (T // 3, 29)}
    torch.cuda.empty_cache()
    _chain_batch(O, d, layers=30, T=T, slots=16, streaming=False, y_samples=samples, zipf=0.0)
    gc.collect()
    torch.cuda.empty_cache()


def test_chained_prefill_chunk_30_layers(O):
    """The prefill workload at full size: a 128-token chunk through 30 chained
    layers of the 26B-A4B shape, every layer's 16-slot cache cold, the plan in
    waves, misses copied from the pinned host store; ids, gate weights, plans
    and chained inputs at every layer, outputs on a sample."""
    d = synth.GEMMA4_26B
    samples = {(0, 0), (127, 3), (64, 9), (5, 16), (100, 23), (31, 29)}
    torch.cuda.empty_cache()
    st = _chain_batch(O, d, layers=30, T=128, slots=16, streaming=True, y_samples=samples)
    assert st["waves"] > 30 and st["misses"] > 0
    gc.collect()
    torch.cuda.empty_cache()
