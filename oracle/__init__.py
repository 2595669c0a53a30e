"""CPU oracle for the routed-MoE layer with an LFU expert slot cache.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
package.  The product path (``expert_streaming_decode_b200``) never imports it.

The arithmetic lives in ``moe_oracle.c`` (plain C, fp64 except the router's
fp32 logits, which decide the top-8 ids).  This module only compiles it with
gcc and marshals numpy arrays through ctypes.  Every function cites its source
passage in the C file.
"""
from __future__ import annotations

import ctypes as C
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(_HERE, "moe_oracle.c")
LIB = os.path.join(_HERE, "liboracle.so")

CFLAGS = ["-std=c11", "-O2", "-Wall", "-ffp-contract=off", "-fPIC", "-shared"]


def build(src: str = SRC, out: str = LIB, extra=()) -> str:
    """Compile the oracle with gcc.  ``-ffp-contract=off`` keeps every fp
    operation as written (no silent FMA contraction), so the fp32 router
    logits follow exactly the FMA order stated in the source."""
    if (os.path.exists(out) and os.path.getmtime(out) >= os.path.getmtime(src)
            and not extra and src == SRC):
        return out
    cmd = ["gcc", *CFLAGS, *extra, "-I", _HERE, src, "-o", out, "-lm"]
    subprocess.run(cmd, check=True)
    return out


def _p(a):
    return a.ctypes.data_as(C.c_void_p)


class Oracle:
    """ctypes view of one compiled oracle library (the default one, or a
    planted-mistake variant built by the mutant test)."""

    def __init__(self, path: str | None = None):
        path = path or build()
        self.lib = C.CDLL(path)
        L = self.lib
        L.orc_f16_to_f64.restype = C.c_double
        L.orc_f16_to_f64.argtypes = [C.c_uint16]
        L.orc_bf16_to_f32.restype = C.c_float
        L.orc_bf16_to_f32.argtypes = [C.c_uint16]
        L.orc_gelu_tanh.restype = C.c_double
        L.orc_gelu_tanh.argtypes = [C.c_double]
        L.orc_blob_bytes.restype = C.c_size_t
        L.orc_blob_bytes.argtypes = [C.c_int, C.c_int]
        L.orc_weight.restype = C.c_double
        L.orc_weight.argtypes = [C.c_void_p, C.c_int, C.c_int, C.c_int, C.c_int, C.c_int]
        L.orc_dequant.restype = None
        L.orc_dequant.argtypes = [C.c_void_p, C.c_int, C.c_int, C.c_int, C.c_void_p]
        L.orc_expert_ffn.restype = None
        L.orc_expert_ffn.argtypes = [C.c_void_p, C.c_int, C.c_int, C.c_void_p, C.c_void_p]
        L.orc_router_logits.restype = None
        L.orc_router_logits.argtypes = [C.c_void_p] * 4 + [C.c_int] * 3 + [C.c_void_p]
        L.orc_topk.restype = C.c_int
        L.orc_topk.argtypes = [C.c_void_p, C.c_int, C.c_int, C.c_void_p]
        L.orc_gate_weights.restype = None
        L.orc_gate_weights.argtypes = [C.c_void_p, C.c_void_p, C.c_int, C.c_void_p]
        L.orc_moe_token.restype = C.c_int
        L.orc_moe_token.argtypes = [C.c_int] * 6 + [C.c_void_p] * 10
        L.orc_lfu_plan.restype = C.c_int
        L.orc_lfu_plan.argtypes = ([C.c_int, C.c_int] + [C.c_void_p] * 5
                                   + [C.c_int, C.c_int, C.c_uint32] + [C.c_void_p] * 7)
        L.orc_cache_plan.restype = C.c_int
        L.orc_cache_plan.argtypes = ([C.c_int, C.c_int, C.c_int, C.c_uint32] + [C.c_void_p] * 5
                                     + [C.c_int, C.c_int, C.c_uint32] + [C.c_void_p] * 7)
        L.orc_f64_to_bf16.restype = C.c_uint16
        L.orc_f64_to_bf16.argtypes = [C.c_double]
        L.orc_residual_rmsnorm.restype = None
        L.orc_residual_rmsnorm.argtypes = [C.c_void_p, C.c_void_p, C.c_int, C.c_void_p, C.c_void_p]
        L.orc_group_by_expert.restype = C.c_int
        L.orc_group_by_expert.argtypes = [C.c_void_p, C.c_int, C.c_int, C.c_int,
                                          C.c_void_p, C.c_void_p]
        L.orc_attn_decode.restype = C.c_int
        L.orc_attn_decode.argtypes = [C.c_void_p] * 3 + [C.c_int] * 5 + [C.c_double, C.c_void_p]

    # scalar helpers -------------------------------------------------------
    def f16_to_f64(self, h: int) -> float:
        return self.lib.orc_f16_to_f64(int(h))

    def bf16_to_f32(self, b: int) -> float:
        return self.lib.orc_bf16_to_f32(int(b))

    def gelu_tanh(self, v: float) -> float:
        return self.lib.orc_gelu_tanh(float(v))

    # expert blobs ---------------------------------------------------------
    def blob_bytes(self, D: int, F: int) -> int:
        return int(self.lib.orc_blob_bytes(D, F))

    def weight(self, blob: np.ndarray, D: int, F: int, m: int, n: int, k: int) -> float:
        blob = np.ascontiguousarray(blob, dtype=np.uint8)
        return self.lib.orc_weight(_p(blob), D, F, m, n, k)

    def dequant(self, blob: np.ndarray, D: int, F: int, m: int) -> np.ndarray:
        """m = 0 gate [F,D], 1 up [F,D], 2 down [D,F]; float64."""
        blob = np.ascontiguousarray(blob, dtype=np.uint8)
        shape = (D, F) if m == 2 else (F, D)
        W = np.empty(shape, dtype=np.float64)
        self.lib.orc_dequant(_p(blob), D, F, m, _p(W))
        return W

    def expert_ffn(self, blob: np.ndarray, D: int, F: int, x: np.ndarray) -> np.ndarray:
        blob = np.ascontiguousarray(blob, dtype=np.uint8)
        x = np.ascontiguousarray(x, dtype=np.float64)
        y = np.empty(D, dtype=np.float64)
        self.lib.orc_expert_ffn(_p(blob), D, F, _p(x), _p(y))
        return y

    # router ---------------------------------------------------------------
    def router_logits(self, x_bf16, wq, ws_f16, bias, E: int, D: int, G: int) -> np.ndarray:
        x_bf16 = np.ascontiguousarray(x_bf16, dtype=np.uint16)
        wq = np.ascontiguousarray(wq, dtype=np.int8)
        ws_f16 = np.ascontiguousarray(ws_f16, dtype=np.uint16)
        out = np.empty(E, dtype=np.float32)
        b = None if bias is None else np.ascontiguousarray(bias, dtype=np.float32)
        self.lib.orc_router_logits(_p(x_bf16), _p(wq), _p(ws_f16),
                                   None if b is None else _p(b), E, D, G, _p(out))
        return out

    def topk(self, logits, K: int):
        """Returns the K ids, or None when the oracle reports an error (NaN)."""
        logits = np.ascontiguousarray(logits, dtype=np.float32)
        ids = np.empty(K, dtype=np.int32)
        rc = self.lib.orc_topk(_p(logits), logits.size, K, _p(ids))
        return None if rc != 0 else ids

    def gate_weights(self, logits, ids) -> np.ndarray:
        logits = np.ascontiguousarray(logits, dtype=np.float32)
        ids = np.ascontiguousarray(ids, dtype=np.int32)
        w = np.empty(ids.size, dtype=np.float64)
        self.lib.orc_gate_weights(_p(logits), _p(ids), ids.size, _p(w))
        return w

    def moe_token(self, dims, x_bf16, wq, ws_f16, bias, shared_blob, expert_blobs):
        """One token through one layer.  ``expert_blobs``: list (or callable
        e -> blob) of E uint8 arrays.  Returns (ids, gate_w, logits, y)."""
        D, E, K, F, FS, G = (dims[k] for k in ("D", "E", "K", "F", "FS", "G"))
        x_bf16 = np.ascontiguousarray(x_bf16, dtype=np.uint16)
        wq = np.ascontiguousarray(wq, dtype=np.int8)
        ws_f16 = np.ascontiguousarray(ws_f16, dtype=np.uint16)
        b = None if bias is None else np.ascontiguousarray(bias, dtype=np.float32)
        blobs = [np.ascontiguousarray(expert_blobs[e], dtype=np.uint8) for e in range(E)]
        ptrs = (C.c_void_p * E)(*[bl.ctypes.data for bl in blobs])
        sh = None if shared_blob is None else np.ascontiguousarray(shared_blob, dtype=np.uint8)
        ids = np.empty(K, dtype=np.int32)
        w = np.empty(K, dtype=np.float64)
        lg = np.empty(E, dtype=np.float32)
        y = np.empty(D, dtype=np.float64)
        rc = self.lib.orc_moe_token(D, E, K, F, FS, G, _p(x_bf16), _p(wq), _p(ws_f16),
                                    None if b is None else _p(b),
                                    None if sh is None else _p(sh),
                                    C.cast(ptrs, C.c_void_p), _p(ids), _p(w), _p(lg), _p(y))
        if rc != 0:
            raise ValueError("oracle: NaN router logits")
        return ids, w, lg, y

    # LFU ------------------------------------------------------------------
    def lfu_plan(self, state: "LfuState", ids, step: int):
        """Plans one call (T tokens x K selections) against ``state`` (updated
        in place).  Returns dict with pair_slot [T,K] and per-distinct-expert
        arrays expert/slot/hit/victim/wave, and the number of waves."""
        ids = np.ascontiguousarray(ids, dtype=np.int32)
        T, K = ids.shape
        E = state.E
        pair_slot = np.full((T, K), -1, dtype=np.int32)
        ue, us, uh, uv, uw = (np.full(E, -1, dtype=np.int32) for _ in range(5))
        nu = C.c_int(0)
        if state.policy == POLICY_LFU and state.decay_period == 0:
            waves = self.lib.orc_lfu_plan(E, state.S, _p(state.count), _p(state.last_use),
                                          _p(state.slot_of), _p(state.expert_in),
                                          _p(ids), T, K, C.c_uint32(step), _p(pair_slot),
                                          _p(ue), _p(us), _p(uh), _p(uv), _p(uw), C.byref(nu))
        else:
            waves = self.lib.orc_cache_plan(E, state.S, state.policy, C.c_uint32(state.decay_period),
                                            _p(state.count), _p(state.last_use),
                                            _p(state.slot_of), _p(state.expert_in),
                                            _p(ids), T, K, C.c_uint32(step), _p(pair_slot),
                                            _p(ue), _p(us), _p(uh), _p(uv), _p(uw), C.byref(nu))
        if waves < 0:
            raise ValueError("oracle: expert id out of range")
        n = nu.value
        return dict(pair_slot=pair_slot, expert=ue[:n].copy(), slot=us[:n].copy(),
                    hit=uh[:n].copy(), victim=uv[:n].copy(), wave=uw[:n].copy(), waves=waves)

    # layer chaining (test and benchmark harness, not the MoE layer) ---------
    def f64_to_bf16(self, v: float) -> int:
        return int(self.lib.orc_f64_to_bf16(float(v)))

    def residual_rmsnorm(self, r_in, y):
        """(r_out fp64 [D], x_next bf16 bits [D]) for one token."""
        r_in = np.ascontiguousarray(r_in, dtype=np.float64)
        y = np.ascontiguousarray(y, dtype=np.float64)
        D = r_in.size
        r_out = np.empty(D, dtype=np.float64)
        x = np.empty(D, dtype=np.uint16)
        self.lib.orc_residual_rmsnorm(_p(r_in), _p(y), D, _p(r_out), _p(x))
        return r_out, x

    def group_by_expert(self, ids, E: int):
        ids = np.ascontiguousarray(ids, dtype=np.int32)
        T, K = ids.shape
        off = np.empty(E + 1, dtype=np.int32)
        pairs = np.empty(T * K, dtype=np.int32)
        rc = self.lib.orc_group_by_expert(_p(ids), T, K, E, _p(off), _p(pairs))
        if rc != 0:
            raise ValueError("oracle: expert id out of range")
        return off, pairs

    def attn_decode(self, q_bf16, k_f16, v_f16, cap: int, n: int, scale: float) -> np.ndarray:
        """Decode attention of one token: q bf16 bits [Hq][hd], k/v binary16
        bits [Hkv][cap][hd]; returns fp64 [Hq][hd]."""
        q = np.ascontiguousarray(q_bf16, dtype=np.uint16)
        k = np.ascontiguousarray(k_f16, dtype=np.uint16)
        v = np.ascontiguousarray(v_f16, dtype=np.uint16)
        Hq, hd = q.shape
        Hkv = k.shape[0]
        if k.shape != (Hkv, cap, hd) or v.shape != k.shape:
            raise ValueError("oracle: k/v must be [Hkv][cap][hd]")
        o = np.empty((Hq, hd), dtype=np.float64)
        if self.lib.orc_attn_decode(_p(q), _p(k), _p(v), Hq, Hkv, hd, cap, n, float(scale), _p(o)) != 0:
            raise ValueError("oracle: bad attention sizes")
        return o


POLICY_LFU, POLICY_LRU, POLICY_LFU_DECAY, POLICY_LFU_IN_CACHE = 0, 1, 2, 3


class LfuState:
    """Caller-owned cache state of one layer, cold start: counts 0, last_use 0,
    nothing resident, every slot empty.  `policy` selects the replacement
    rule (POLICY_*); `decay_period` is used by POLICY_LFU_DECAY."""

    def __init__(self, E: int, S: int, policy: int = POLICY_LFU, decay_period: int = 0):
        self.E, self.S = E, S
        self.policy, self.decay_period = policy, decay_period
        self.count = np.zeros(E, dtype=np.uint32)
        self.last_use = np.zeros(E, dtype=np.uint32)
        self.slot_of = np.full(E, -1, dtype=np.int32)
        self.expert_in = np.full(S, -1, dtype=np.int32)

    def copy(self) -> "LfuState":
        c = LfuState(self.E, self.S, self.policy, self.decay_period)
        for a in ("count", "last_use", "slot_of", "expert_in"):
            setattr(c, a, getattr(self, a).copy())
        return c


_default = None


def get() -> Oracle:
    """The default oracle library (built on first use)."""
    global _default
    if _default is None:
        _default = Oracle()
    return _default
