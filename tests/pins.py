"""Pins of the CPU oracle against facts fixed outside it: hand-derived golden
points, closed forms, exact small-integer cases, brute force, library routines
(numpy, scipy, torch) and a naive simulator.  Each pin takes the oracle object
so that tests/test_oracle_mutants.py can run the same pins against oracle
builds with a planted mistake and check that some pin fails.
"""
from __future__ import annotations

import math
import os
from fractions import Fraction

import numpy as np
import scipy.special
import torch

from expert_streaming_decode_b200 import synth
from naive_lfu import NaiveLfu

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")
TINY = synth.TINY


def _golden_rows(name):
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if line:
                yield line.split()


# ------------------------------------------------------------ number formats
def pin_binary16(O):
    """Golden binary16 values, then every one of the 65536 patterns against
    numpy's float16 (a library conversion)."""
    for h, v in _golden_rows("binary16_values.txt"):
        got = O.f16_to_f64(int(h, 16))
        want = float(v)
        assert got == want and math.copysign(1, got) == math.copysign(1, want), (h, got, want)
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ref = bits.view(np.float16).astype(np.float64)
    for b in range(0, 65536, 97):
        got = O.f16_to_f64(int(bits[b]))
        if math.isnan(ref[b]):
            assert math.isnan(got)
        else:
            assert got == ref[b], (hex(b), got, ref[b])


def pin_bf16(O):
    """bfloat16 -> float32 equals torch's conversion (library routine)."""
    rng = np.random.default_rng(5)
    bits = rng.integers(0, 65536, size=4000).astype(np.uint16)
    ref = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).float().numpy()
    for b, r in zip(bits, ref):
        got = O.bf16_to_f32(int(b))
        assert (math.isnan(got) and math.isnan(r)) or got == r, (hex(b), got, r)


# --------------------------------------------------------------- blob layout
def pin_layout_points(O):
    """Each hand-derived point: a blob holding a single nibble 9 with
    (scale 1, bias -2) in its group must dequantise to 7 at (n, k), -2 in the
    rest of that row's group, 0 everywhere else."""
    for D, F, m, n, k, qb, hi, sb in _golden_rows("blob_layout_points.txt"):
        D, F, m, n, k, qb, hi, sb = map(int, (D, F, m, n, k, qb, hi, sb))
        blob = np.zeros(O.blob_bytes(D, F), dtype=np.uint8)
        blob[qb] = (9 << 4) if hi else 9
        blob[sb:sb + 4] = [0x00, 0x3C, 0x00, 0xC0]
        W = O.dequant(blob, D, F, m)
        want = np.zeros_like(W)
        g0 = (k // 64) * 64
        want[n, g0:g0 + 64] = -2.0
        want[n, k] = 7.0
        assert np.array_equal(W, want), (D, F, m, n, k)


def pin_packer_points(_O=None):
    """The generator's packer puts the same hand-derived points in the same
    bytes (pins the input generator to the layout definition, too)."""
    for D, F, m, n, k, qb, hi, sb in _golden_rows("blob_layout_points.txt"):
        D, F, m, n, k, qb, hi, sb = map(int, (D, F, m, n, k, qb, hi, sb))
        qs = [np.zeros((F, D), np.uint8), np.zeros((F, D), np.uint8), np.zeros((D, F), np.uint8)]
        ss = [np.zeros((F, D // 64), np.float16), np.zeros((F, D // 64), np.float16),
              np.zeros((D, F // 64), np.float16)]
        bs = [a.copy() for a in ss]
        qs[m][n, k] = 9
        ss[m][n, k // 64] = 1.0
        bs[m][n, k // 64] = -2.0
        blob = synth.pack_expert(qs[0], qs[1], qs[2], ss[0], bs[0], ss[1], bs[1], ss[2], bs[2])
        want = np.zeros_like(blob)
        want[qb] = (9 << 4) if hi else 9
        want[sb:sb + 4] = [0x00, 0x3C, 0x00, 0xC0]
        assert np.array_equal(blob, want), (D, F, m, n, k, np.nonzero(blob != want)[0][:5])


def pin_dequant_random(O):
    """Random expert: oracle dequant equals s*q + b built by numpy from the
    generator's unpacked draw (exact)."""
    d = TINY
    for F in (d.F, d.FS):
        p = synth.draw_expert_parts(3, 1, 2, d.D, F)
        blob = synth.pack_parts(p)
        for m, key in enumerate("gud"):
            ref = (np.repeat(p["s" + key].astype(np.float64), 64, axis=1) * p["q" + key]
                   + np.repeat(p["b" + key].astype(np.float64), 64, axis=1))
            assert np.array_equal(O.dequant(blob, d.D, F, m), ref), (F, key)


# ------------------------------------------------------------------- router
def pin_router_exact(O):
    """Small integers and power-of-two scales make every partial sum exact, so
    the logits must equal the exact rational sum of s*q*x plus the bias."""
    rng = np.random.default_rng(11)
    E, D, G = 12, 512, 64
    x = rng.integers(-4, 5, size=D).astype(np.float32)
    xb = synth.to_bf16_bits(x)
    wq = rng.integers(-9, 10, size=(E, D)).astype(np.int8)
    exps = rng.integers(-6, 3, size=(E, D // G))
    ws = (2.0 ** exps).astype(np.float16).view(np.uint16)
    bias = (rng.integers(-8, 9, size=E) / 4.0).astype(np.float32)
    got = O.router_logits(xb, wq, ws, bias, E, D, G)
    for e in range(E):
        acc = Fraction(0)
        for g in range(D // G):
            sg = Fraction(2) ** int(exps[e, g])
            acc += sg * sum(int(wq[e, k]) * int(x[k]) for k in range(g * G, (g + 1) * G))
        acc += Fraction(float(bias[e]))
        assert Fraction(float(got[e])) == acc, (e, float(got[e]), float(acc))
    nob = O.router_logits(xb, wq, ws, None, E, D, G)
    assert np.array_equal(nob + bias, got)


def pin_router_random(O):
    """Random full-shape router row set: fp32 logits agree with an fp64 numpy
    matmul of the dequantised weights to fp32 accumulation accuracy."""
    d = synth.GEMMA4_26B
    wq, ws = synth.router_weights(0, 0, d.E, d.D)
    xb = synth.hidden(0, 0, 0, d.D)
    bias = synth.zipf_bias(0, 0, d.E)
    W = wq.astype(np.float64) * np.repeat(ws.view(np.float16).astype(np.float64), 64, axis=1)
    x = synth.bf16_bits_to_f32(xb).astype(np.float64)
    ref = W @ x + bias.astype(np.float64)
    got = O.router_logits(xb, wq, ws, bias, d.E, d.D, d.G).astype(np.float64)
    scale = np.abs(W * x).sum(axis=1)
    assert np.all(np.abs(got - ref) <= 1e-5 * scale), np.max(np.abs(got - ref))
    assert 0.5 < np.std(ref - bias) < 2.0  # unit-scale logits, as the recipe intends


def pin_topk(O):
    """Top-K equals a full lexicographic sort (logit descending, id ascending),
    including many exact ties; NaN logits are an error."""
    rng = np.random.default_rng(2)
    for trial in range(300):
        E = int(rng.integers(8, 130))
        K = int(rng.integers(1, min(E, 12) + 1))
        if trial % 3 == 0:
            lg = rng.integers(-3, 4, size=E).astype(np.float32)  # heavy ties
        else:
            lg = rng.standard_normal(E).astype(np.float32)
        want = np.lexsort((np.arange(E), -lg.astype(np.float64)))[:K]
        got = O.topk(lg, K)
        assert got is not None and np.array_equal(got, want), (trial, got, want)
    lg = np.zeros(16, np.float32)
    assert list(O.topk(lg, 4)) == [0, 1, 2, 3]
    lg[5] = np.nan
    assert O.topk(lg, 4) is None


def pin_gate_weights(O):
    """Softmax over the chosen K equals scipy's softmax over all E experts
    renormalised to the chosen ones; closed forms for equal and two logits."""
    rng = np.random.default_rng(4)
    for _ in range(50):
        E, K = 128, 8
        lg = (rng.standard_normal(E) * 3).astype(np.float32)
        ids = O.topk(lg, K)
        full = scipy.special.softmax(lg.astype(np.float64))
        want = full[ids] / full[ids].sum()
        got = O.gate_weights(lg, ids)
        assert np.allclose(got, want, rtol=1e-13, atol=0), (got, want)
        assert abs(got.sum() - 1.0) < 1e-14
        assert np.all(np.diff(got) <= 0)  # ids are in descending-logit order
    lg = np.full(8, 1.5, np.float32)
    assert np.allclose(O.gate_weights(lg, np.arange(8)), 1 / 8, rtol=1e-15)
    lg = np.array([0.75, -0.5], np.float32)
    w = O.gate_weights(lg, np.array([0, 1]))
    assert abs(w[0] - 1 / (1 + math.exp(-1.25))) < 1e-15 and abs(w[1] - 1 / (1 + math.exp(1.25))) < 1e-15


def pin_gelu(O):
    """GELU (tanh form) equals torch's gelu(approximate='tanh') in float64."""
    v = np.concatenate([np.linspace(-12, 12, 481), [0.0, 1e-8, -1e-8, 30.0, -30.0]])
    ref = torch.nn.functional.gelu(torch.from_numpy(v), approximate="tanh").numpy()
    for a, r in zip(v, ref):
        assert abs(O.gelu_tanh(a) - r) <= 1e-15 * max(1.0, abs(r)), (a, O.gelu_tanh(a), r)
    assert O.gelu_tanh(0.0) == 0.0
    assert abs(O.gelu_tanh(30.0) - 30.0) < 1e-12 and abs(O.gelu_tanh(-30.0)) < 1e-12


# --------------------------------------------------------------- expert FFN
def _numpy_ffn(p, x):
    """Unfused: dequantise whole matrices from the unpacked draw, then fp64
    matmuls and torch's tanh-GELU."""
    def W(key):
        return (np.repeat(p["s" + key].astype(np.float64), 64, axis=1) * p["q" + key]
                + np.repeat(p["b" + key].astype(np.float64), 64, axis=1))
    g = W("g") @ x
    u = W("u") @ x
    h = torch.nn.functional.gelu(torch.from_numpy(g), approximate="tanh").numpy() * u
    return W("d") @ h


def pin_ffn(O):
    d = TINY
    rng = np.random.default_rng(9)
    for F in (d.F, d.FS):
        p = synth.draw_expert_parts(1, 0, 5, d.D, F)
        blob = synth.pack_parts(p)
        x = rng.standard_normal(d.D)
        want = _numpy_ffn(p, x)
        got = O.expert_ffn(blob, d.D, F, x)
        assert np.allclose(got, want, rtol=1e-11, atol=1e-11 * np.abs(want).max()), F


def pin_layer(O):
    """Whole token: ids from the (pinned) router + top-K, then the combine
    y = y_shared + sum_i w_i y_{ids[i]} against the unfused numpy FFNs; and the
    special cases: zero shared blob, and K = 1 (gate weight exactly 1)."""
    d = TINY
    parts = [synth.draw_expert_parts(0, 0, e, d.D, d.F) for e in range(d.E)]
    blobs = [synth.pack_parts(p) for p in parts]
    sp = synth.draw_expert_parts(0, 0, 0, d.D, d.FS, shared=True)
    sblob = synth.pack_parts(sp)
    wq, ws = synth.router_weights(0, 0, d.E, d.D)
    bias = synth.zipf_bias(0, 0, d.E)
    dims = d.as_dict()
    for t in range(3):
        xb = synth.hidden(0, t, 0, d.D)
        x = synth.bf16_bits_to_f32(xb).astype(np.float64)
        ids, w, lg, y = O.moe_token(dims, xb, wq, ws, bias, sblob, blobs)
        assert np.array_equal(ids, O.topk(O.router_logits(xb, wq, ws, bias, d.E, d.D, d.G), d.K))
        want = _numpy_ffn(sp, x)
        for i, e in enumerate(ids):
            want = want + w[i] * _numpy_ffn(parts[e], x)
        assert np.allclose(y, want, rtol=1e-11, atol=1e-11 * np.abs(want).max())
        # zero shared expert: all scales and biases zero
        _, _, _, y0 = O.moe_token(dims, xb, wq, ws, bias, np.zeros_like(sblob), blobs)
        assert np.allclose(y0, want - _numpy_ffn(sp, x), rtol=1e-10, atol=1e-10 * np.abs(want).max())
        # K = 1: the single gate weight is exactly 1
        d1 = dict(dims, K=1)
        ids1, w1, _, y1 = O.moe_token(d1, xb, wq, ws, bias, None, blobs)
        assert w1[0] == 1.0
        assert np.allclose(y1, _numpy_ffn(parts[ids1[0]], x), rtol=1e-11,
                           atol=1e-11 * np.abs(y1).max())


# --------------------------------------------------------------------- LFU
def _lfu_trace(O, E, S, K, T, steps, seed, zipf=None, policy=0, period=0):
    import oracle
    st = oracle.LfuState(E, S, policy, period)
    sim = NaiveLfu(E, S, policy, period)
    rng = np.random.default_rng(seed)
    for step in range(steps):
        if zipf is not None:
            lg = rng.standard_normal((T, E)) + zipf
            ids = np.argsort(-lg, axis=1, kind="stable")[:, :K].astype(np.int32)
        else:
            ids = np.stack([rng.choice(E, K, replace=False) for _ in range(T)]).astype(np.int32)
        got = O.lfu_plan(st, ids, step)
        ps, ev = sim.plan(ids.tolist(), step)
        assert np.array_equal(got["pair_slot"], np.array(ps)), (step,)
        want = np.array(ev, dtype=np.int64).T
        for j, key in enumerate(("expert", "slot", "hit", "victim", "wave")):
            assert np.array_equal(got[key], want[j]), (step, key, got[key], want[j])
        # the state the oracle keeps matches the simulator's slots
        assert [(-1 if x is None else x) for x in sim.slots] == list(st.expert_in)
    return st


def pin_lfu_naive(O):
    """Identical traces to the naive history-rescanning simulator: decode
    (T=1), small batches, and prefill-like calls with several waves."""
    _lfu_trace(O, 16, 6, 4, 1, 120, 0)
    _lfu_trace(O, 32, 8, 4, 3, 60, 1)
    _lfu_trace(O, 24, 5, 3, 6, 25, 2)          # many waves per call
    _lfu_trace(O, 128, 16, 8, 1, 150, 3, zipf=synth.zipf_bias(0, 0, 128))


def pin_cache_policies_naive(O):
    """The LRU, decaying-LFU and in-cache-LFU variants give traces identical
    to the naive simulator, which recomputes each key from the full history
    (decay by replaying every call, in-cache frequency by scanning for the
    last eviction)."""
    import oracle
    for pol, per in ((oracle.POLICY_LRU, 0), (oracle.POLICY_LFU_DECAY, 7), (oracle.POLICY_LFU_DECAY, 1),
                     (oracle.POLICY_LFU_IN_CACHE, 0)):
        _lfu_trace(O, 16, 6, 4, 1, 100, 10 + pol, policy=pol, period=per)
        _lfu_trace(O, 24, 5, 3, 6, 20, 20 + pol, policy=pol, period=per)   # several waves per call
        _lfu_trace(O, 128, 16, 8, 1, 120, 30 + pol, zipf=synth.zipf_bias(0, 0, 128), policy=pol, period=per)


def pin_cache_policies_cases(O):
    """Hand-worked evictions that tell the variants apart (2 slots, 8 experts)."""
    import oracle

    def run(policy, calls, period=0):
        st = oracle.LfuState(8, 2, policy, period)
        r = None
        for step, ids in calls:
            r = O.lfu_plan(st, np.array([ids], np.int32), step)
        return st, r
    # expert 0 used three times long ago, expert 1 once recently: LFU evicts 1, LRU evicts 0
    calls = [(0, [0]), (1, [0]), (2, [0]), (3, [1]), (4, [2])]
    assert run(oracle.POLICY_LFU, calls)[1]["victim"][0] == 1
    assert run(oracle.POLICY_LRU, calls)[1]["victim"][0] == 0
    # halving at steps 2 and 4 (period 2): count0 = ((1 + 1) >> 1) + 1 = 2 after step 2, then
    # 1 at step 4; count1 = 1 after step 3, 0 at step 4; the victim is still 1
    st, r = run(oracle.POLICY_LFU_DECAY, calls, period=2)
    assert r["victim"][0] == 1 and st.count[0] == 1 and st.count[1] == 0
    # decay lets a once-hot expert go: counts 3 (expert 0) vs 2 (expert 1) under LFU; with
    # period 4 the only halving call is step 12, giving 1 vs 1, and the older last use loses
    calls = [(0, [0]), (1, [0]), (2, [0]), (10, [1]), (11, [1]), (12, [2])]
    assert run(oracle.POLICY_LFU, calls)[1]["victim"][0] == 1
    st, r = run(oracle.POLICY_LFU_DECAY, calls, period=4)
    assert r["victim"][0] == 0
    # in-cache: step 3 evicts 1 (count 1 vs 2) and its count restarts at 0; step 5 evicts 2
    calls = [(0, [0]), (1, [0]), (2, [1]), (3, [2]), (4, [0]), (5, [3])]
    assert run(oracle.POLICY_LFU, calls)[1]["victim"][0] == 2
    st, r = run(oracle.POLICY_LFU_IN_CACHE, calls)
    assert r["victim"][0] == 2 and st.count[1] == 0
    # in-cache: step 3 evicts 0 (count 1 vs 2), step 4 reloads 0 with count 1 and evicts 2
    # (count 1 vs 2); step 5 evicts 0 again (count 1 vs 2), while plain LFU (count0 = 2 at
    # step 4, a tie with 1 broken by recency) keeps 0 and evicts 1 at step 5
    calls = [(0, [0]), (1, [1]), (2, [1]), (3, [2]), (4, [0]), (5, [3])]
    st, r = run(oracle.POLICY_LFU_IN_CACHE, calls)
    assert r["victim"][0] == 0 and st.count[2] == 0
    assert run(oracle.POLICY_LFU, calls)[1]["victim"][0] == 1


def pin_lfu_invariants(O):
    import oracle
    rng = np.random.default_rng(7)
    # S >= E: every distinct expert misses exactly once, never an eviction
    st = oracle.LfuState(16, 16)
    seen, misses, total = set(), 0, 0
    for step in range(40):
        ids = np.stack([rng.choice(16, 4, replace=False)]).astype(np.int32)
        r = O.lfu_plan(st, ids, step)
        misses += int((r["hit"] == 0).sum())
        total += r["hit"].size
        assert np.all(r["victim"] == -1)
        seen |= set(ids.ravel().tolist())
    assert misses == len(seen)
    # hits + misses = number of distinct experts per call; cold start fills 0,1,2..
    st = oracle.LfuState(64, 8)
    r = O.lfu_plan(st, np.array([[40, 3, 9, 17]], np.int32), 0)
    assert list(r["expert"]) == [3, 9, 17, 40] and list(r["slot"]) == [0, 1, 2, 3]
    assert list(r["hit"]) == [0, 0, 0, 0]
    assert list(r["pair_slot"][0]) == [3, 0, 1, 2]
    # least frequently used goes first, then least recently used, then lower id
    st = oracle.LfuState(8, 2)
    O.lfu_plan(st, np.array([[0]], np.int32), 0)
    O.lfu_plan(st, np.array([[0]], np.int32), 1)
    O.lfu_plan(st, np.array([[1]], np.int32), 2)   # slots: 0 (count 2), 1 (count 1)
    r = O.lfu_plan(st, np.array([[2]], np.int32), 3)
    assert r["victim"][0] == 1 and r["slot"][0] == 1
    r = O.lfu_plan(st, np.array([[3]], np.int32), 4)   # 0: count 2; 2: count 1
    assert r["victim"][0] == 2
    O.lfu_plan(st, np.array([[3]], np.int32), 5)       # 3: count 2, last 6; 0: count 2, last 2
    r = O.lfu_plan(st, np.array([[4]], np.int32), 6)
    assert r["victim"][0] == 0                         # equal counts: older last use
    # an expert of the current wave is never the victim even when least used
    st = oracle.LfuState(8, 2)
    O.lfu_plan(st, np.array([[5, 6]], np.int32), 0)
    for s in range(1, 4):
        O.lfu_plan(st, np.array([[6]], np.int32), s)
    r = O.lfu_plan(st, np.array([[5, 7]], np.int32), 4)
    assert list(r["victim"]) == [-1, 6]


def pin_group_by_expert(O):
    rng = np.random.default_rng(1)
    for _ in range(20):
        T, K, E = int(rng.integers(1, 40)), 8, 128
        ids = np.stack([rng.choice(E, K, replace=False) for _ in range(T)]).astype(np.int32)
        off, pairs = O.group_by_expert(ids, E)
        flat = ids.ravel()
        want = np.argsort(flat, kind="stable")
        assert np.array_equal(pairs, want)
        assert np.array_equal(off, np.searchsorted(flat[want], np.arange(E + 1)))


# ------------------------------------------------------------ decode attention
def _attn_case(rng, Hq, Hkv, hd, cap):
    q = synth.to_bf16_bits(rng.standard_normal((Hq, hd)).astype(np.float32))
    k = rng.standard_normal((Hkv, cap, hd)).astype(np.float16).view(np.uint16)
    v = rng.standard_normal((Hkv, cap, hd)).astype(np.float16).view(np.uint16)
    return q, k, v


def _attn_torch(q, k, v, cap, n, scale):
    """torch's own attention routine on the attended rows, gathered by
    position (p = max(0, n - cap) .. n - 1 in slot p mod cap), in fp64, with
    each KV head repeated for its consecutive query heads."""
    Hq, Hkv = q.shape[0], k.shape[0]
    pos = np.arange(max(0, n - cap), n)
    kk = torch.from_numpy(k.view(np.float16)[:, pos % cap].astype(np.float64))
    vv = torch.from_numpy(v.view(np.float16)[:, pos % cap].astype(np.float64))
    qq = torch.from_numpy(synth.bf16_bits_to_f32(q).astype(np.float64))
    kk = kk.repeat_interleave(Hq // Hkv, dim=0)
    vv = vv.repeat_interleave(Hq // Hkv, dim=0)
    o = torch.nn.functional.scaled_dot_product_attention(qq[:, None, :], kk, vv, scale=scale)
    return o[:, 0, :].numpy()


def pin_attn_library(O):
    """Against torch's scaled_dot_product_attention on the explicitly gathered
    window: GQA head mapping, scale, window bounds, ring slots, normalisation."""
    rng = np.random.default_rng(11)
    for Hq, Hkv, hd, cap, n in [(4, 2, 8, 7, 1), (4, 2, 8, 7, 5), (4, 2, 8, 7, 7), (4, 2, 8, 7, 12),
                                (6, 3, 16, 5, 23), (8, 8, 4, 9, 9), (8, 1, 8, 4, 6), (4, 4, 32, 16, 100)]:
        q, k, v = _attn_case(rng, Hq, Hkv, hd, cap)
        scale = 1.0 / math.sqrt(hd) * float(rng.uniform(0.5, 2.0))
        got = O.attn_decode(q, k, v, cap, n, scale)
        want = _attn_torch(q, k, v, cap, n, scale)
        assert np.allclose(got, want, rtol=1e-12, atol=1e-12), (Hq, Hkv, hd, cap, n)


def pin_attn_closed_forms(O):
    rng = np.random.default_rng(12)
    Hq, Hkv, hd, cap = 4, 2, 8, 6
    q, k, v = _attn_case(rng, Hq, Hkv, hd, cap)
    vf = v.view(np.float16).astype(np.float64)
    kf = k.view(np.float16).astype(np.float64)
    qf = synth.bf16_bits_to_f32(q).astype(np.float64)
    # one position: the output is that value row, exactly
    o = O.attn_decode(q, k, v, cap, 1, 0.3)
    for h in range(Hq):
        assert np.array_equal(o[h], vf[h // 2, 0])
    # a zero query weighs every attended position equally: the mean of the rows
    z = np.zeros_like(q)
    o = O.attn_decode(z, k, v, cap, 4, 0.3)
    for h in range(Hq):
        assert np.allclose(o[h], vf[h // 2, :4].mean(axis=0), rtol=0, atol=1e-15)
    # two positions: weight of the newer one = logistic(scale * q . (k1 - k0))
    o = O.attn_decode(q, k, v, cap, 2, 0.3)
    for h in range(Hq):
        g = h // 2
        a = 1.0 / (1.0 + math.exp(-0.3 * float(qf[h] @ (kf[g, 1] - kf[g, 0]))))
        assert np.allclose(o[h], (1 - a) * vf[g, 0] + a * vf[g, 1], rtol=0, atol=1e-13)
    # a ring after wrap-around attends to exactly its cap newest positions: the
    # same result as a linear cache holding those positions in order
    n = 3 * cap + 2
    pos = np.arange(n - cap, n)
    k_lin = np.ascontiguousarray(k[:, pos % cap])
    v_lin = np.ascontiguousarray(v[:, pos % cap])
    ring = O.attn_decode(q, k, v, cap, n, 0.3)
    lin = O.attn_decode(q, k_lin, v_lin, cap, cap, 0.3)
    assert np.allclose(ring, lin, rtol=0, atol=1e-13)
    # one dominant key: its value row, up to exp(-gap)
    kk = np.zeros((Hkv, cap, hd), dtype=np.float16)
    kk[:, 2, 0] = 64.0
    qq = np.zeros((Hq, hd), dtype=np.float32)
    qq[:, 0] = 1.0
    o = O.attn_decode(synth.to_bf16_bits(qq), kk.view(np.uint16), v, cap, 5, 1.0)
    for h in range(Hq):
        assert np.allclose(o[h], vf[h // 2, 2], rtol=0, atol=1e-20 + 4 * math.exp(-64) * np.abs(vf).max())
    # sizes the definition rejects: no attended position, an empty cache
    try:
        O.attn_decode(q, k, v, cap, 0, 0.3)
    except ValueError:
        pass
    else:
        raise AssertionError("n < 1 accepted")
    assert O.lib.orc_attn_decode(None, None, None, Hq, Hkv, hd, 0, 1, 0.3, None) == -1


# ------------------------------------------------- layer chaining (harness)
def pin_bf16_round(O):
    """Rounding to bfloat16: hand-derived golden cases (ties to even,
    subnormals, overflow), then torch's float32 -> bfloat16 conversion (a
    library routine, round to nearest even) on random float32 values."""
    for v, bits in _golden_rows("bf16_round.txt"):
        got = O.f64_to_bf16(float.fromhex(v))
        assert got == int(bits, 16), (v, hex(got), bits)
    rng = np.random.default_rng(21)
    f = (rng.standard_normal(5000) * np.exp2(rng.integers(-30, 30, 5000))).astype(np.float32)
    ref = torch.from_numpy(f).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    for v, r in zip(f, ref):
        assert O.f64_to_bf16(float(v)) == int(r), (float(v), int(r))


def pin_residual_rmsnorm(O):
    """The chaining step r += y; x = bf16(r / sqrt(mean(r^2) + 1e-6)), pinned
    by cases whose result is fixed without evaluating that expression:
    the residual sum of float32 values is exact in double; a constant vector
    of 1e-3 has mean square equal to the 1e-6 term, so every output is
    1/sqrt(2) -> bf16 0x3F35; a large constant gives 1.0 exactly after
    rounding; a single non-zero entry 8 in 64 has mean square 1 (the mean, not
    the sum), so it maps to 8 -> 0x4100; the zero vector stays zero; negating
    the input flips only the sign bits; and for random rows the bf16 outputs
    have mean square 1 to within the rounding."""
    rng = np.random.default_rng(22)
    D = 512
    r0 = rng.standard_normal(D).astype(np.float32).astype(np.float64)
    y = rng.standard_normal(D).astype(np.float32).astype(np.float64)
    r1, x = O.residual_rmsnorm(r0, y)
    assert np.array_equal(r1, (r0.astype(np.float32) + y.astype(np.float32)).astype(np.float64)) or \
        np.array_equal(r1 - y, r0)
    assert np.array_equal(r1 - r0, y)
    _, x = O.residual_rmsnorm(np.zeros(D), np.full(D, 1e-3))
    assert np.all(x == 0x3F35), hex(int(x[0]))
    _, x = O.residual_rmsnorm(np.full(D, 1000.0), np.zeros(D))
    assert np.all(x == 0x3F80)
    one = np.zeros(64)
    one[5] = 8.0
    _, x = O.residual_rmsnorm(np.zeros(64), one)
    assert x[5] == 0x4100 and np.all(np.delete(x, 5) == 0), hex(int(x[5]))
    r_out, x = O.residual_rmsnorm(np.zeros(D), np.zeros(D))
    assert np.all(x == 0) and np.all(r_out == 0)
    v = rng.standard_normal(D) * 5
    _, xp = O.residual_rmsnorm(v, np.zeros(D))
    _, xn = O.residual_rmsnorm(-v, np.zeros(D))
    assert np.array_equal(xn, xp ^ np.uint16(0x8000))
    xf = synth.bf16_bits_to_f32(xp).astype(np.float64)
    assert abs(np.mean(xf * xf) - 1.0) < 2.0 ** -7


ALL_PINS = [pin_binary16, pin_bf16, pin_layout_points, pin_packer_points, pin_dequant_random,
            pin_router_exact, pin_router_random, pin_topk, pin_gate_weights, pin_gelu, pin_ffn,
            pin_layer, pin_lfu_naive, pin_cache_policies_naive, pin_cache_policies_cases, pin_lfu_invariants,
            pin_group_by_expert, pin_attn_library, pin_attn_closed_forms, pin_bf16_round,
            pin_residual_rmsnorm]
