"""Property-based pins of the oracle's cache plan: for random layer sizes,
batch shapes, replacement rules and selection sequences, the incremental plan
equals the naive simulator that recomputes every key from the whole history
(tests/naive_lfu.py), and the plan's invariants hold."""
import numpy as np
from hypothesis import given, settings, strategies as st

import oracle
from naive_lfu import NaiveLfu


@st.composite
def plan_case(draw):
    E = draw(st.integers(4, 40))
    K = draw(st.integers(1, min(6, E)))
    S = draw(st.integers(K, E))
    T = draw(st.integers(1, 5))
    steps = draw(st.integers(1, 25))
    policy = draw(st.sampled_from([oracle.POLICY_LFU, oracle.POLICY_LRU, oracle.POLICY_LFU_DECAY,
                                   oracle.POLICY_LFU_IN_CACHE]))
    period = draw(st.integers(1, 6)) if policy == oracle.POLICY_LFU_DECAY else 0
    seed = draw(st.integers(0, 2 ** 31 - 1))
    skew = draw(st.floats(0.0, 3.0))
    return E, K, S, T, steps, policy, period, seed, skew


@settings(max_examples=150, deadline=None)
@given(plan_case())
def test_plan_equals_naive_simulator(case):
    E, K, S, T, steps, policy, period, seed, skew = case
    O = oracle.get()
    rng = np.random.default_rng(seed)
    pop = -skew * np.log1p(rng.permutation(E))          # a popularity skew, as the router's bias gives
    st_ = oracle.LfuState(E, S, policy, period)
    sim = NaiveLfu(E, S, policy, period)
    step = 0
    for _ in range(steps):
        step += int(rng.integers(1, 3))                  # steps need not be consecutive
        lg = rng.standard_normal((T, E)) + pop
        ids = np.argsort(-lg, axis=1, kind="stable")[:, :K].astype(np.int32)
        got = O.lfu_plan(st_, ids, step)
        ps, ev = sim.plan(ids.tolist(), step)
        want = np.array(ev, dtype=np.int64).T
        for j, key in enumerate(("expert", "slot", "hit", "victim", "wave")):
            assert np.array_equal(got[key], want[j]), (key, got[key], want[j])
        assert np.array_equal(got["pair_slot"], np.array(ps))
        # invariants: every distinct expert once, waves of at most S, slots a consistent map
        assert np.array_equal(got["expert"], np.unique(ids))
        assert got["waves"] == (len(got["expert"]) + S - 1) // S
        res = st_.expert_in[st_.expert_in >= 0]
        assert len(set(res.tolist())) == len(res)
        for s_, e_ in enumerate(st_.expert_in):
            if e_ >= 0:
                assert st_.slot_of[e_] == s_
        assert (st_.slot_of >= 0).sum() == (st_.expert_in >= 0).sum()


@st.composite
def attn_case(draw):
    Hkv = draw(st.integers(1, 4))
    G = draw(st.sampled_from([1, 2, 3, 4]))
    hd = draw(st.integers(1, 40))
    cap = draw(st.integers(1, 30))
    n = draw(st.integers(1, 4 * cap + 3))
    scale = draw(st.floats(0.01, 3.0))
    seed = draw(st.integers(0, 2 ** 31 - 1))
    return Hkv * G, Hkv, hd, cap, n, scale, seed


@settings(max_examples=150, deadline=None)
@given(attn_case())
def test_attention_equals_library_routine(case):
    """Decode attention for random head counts, widths, ring capacities and
    token counts (wrapped or not) equals torch's attention routine applied to
    the explicitly gathered newest positions, and it is a convex combination
    of the attended value rows (each output lies within their range)."""
    import pins
    Hq, Hkv, hd, cap, n, scale, seed = case
    rng = np.random.default_rng(seed)
    q, k, v = pins._attn_case(rng, Hq, Hkv, hd, cap)
    O = oracle.get()
    got = O.attn_decode(q, k, v, cap, n, scale)
    want = pins._attn_torch(q, k, v, cap, n, scale)
    assert np.allclose(got, want, rtol=1e-11, atol=1e-11)
    pos = np.arange(max(0, n - cap), n) % cap
    vf = v.view(np.float16).astype(np.float64)[:, pos]
    for h in range(Hq):
        rows = vf[h // (Hq // Hkv)]
        assert (got[h] >= rows.min(axis=0) - 1e-12).all() and (got[h] <= rows.max(axis=0) + 1e-12).all()
