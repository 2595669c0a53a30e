"""Seeded synthetic inputs for the routed-MoE layer (both the CUDA path and the
CPU oracle consume these; this module holds none of the layer's arithmetic).

Every draw is keyed on (seed, kind, layer, index) through numpy's SeedSequence,
so any single expert blob, router or hidden state can be regenerated alone.

Distributions (the pages' model shape with synthetic values):
  expert q      uniform nibbles 0..15
  expert scale  binary16 of U(0.002, 0.02) per (row, group of 64); bias = -8*scale
                (exact in binary16)
  router q      int8 uniform in [-128, 127]
  router scale  binary16 of U(1.67e-4, 3.34e-4) per (expert, group of 64), which
                gives unit-variance logits for N(0,1) hidden states
  hidden state  bfloat16 (round to nearest even) of N(0, 1)
  Zipf bias     bias_e = -lam * s * ln(1 + pi(e)), pi a seeded per-layer
                permutation of 0..E-1 (popular experts repeat, as in decode)
  attention     decode query bfloat16 of N(0, 1) [Hq][hd]; KV cache binary16 of
                N(0, 1), [Hkv][capacity][hd] for keys and for values

Expert blob layout (the kernel-ready layout both sides read):
  an expert with width D and FFN width F is one contiguous blob of two sections
  of "chunks"; a chunk holds 32 matrix rows x KS inputs in 18*KS bytes:
    q part   (KS/32 word-quads) x (32 rows) x 16 bytes; within a row's 16
             bytes, input 32*wq + 8*word + j sits in byte 4*word + j//2, low
             nibble for even j, high nibble for odd j
    sb part  (KS/64 groups) x (32 rows) x (binary16 scale, binary16 bias)
  section 0 (gate/up): F/16 tiles x D/256 slices, KS = 256; tile t's rows 0..15
             are gate rows 16t.., rows 16..31 are up rows 16t..
  section 1 (down):    D/32 tiles x F/KS slices, KS = F if F <= 704 else 704;
             tile t's rows are down rows 32t..32t+31
"""
from __future__ import annotations

import concurrent.futures as cf
import dataclasses
import os

import numpy as np

# draw kinds (part of the seed key)
_ROUTED, _SHARED, _ROUTER, _HIDDEN, _ZIPF, _IDS, _ATTN = 1, 2, 3, 4, 5, 6, 7


@dataclasses.dataclass(frozen=True)
class Dims:
    D: int = 2816    # model width
    E: int = 128     # routed experts per layer
    K: int = 8       # experts selected per token
    F: int = 704     # routed expert FFN width
    FS: int = 2112   # shared expert FFN width
    G: int = 64      # quantisation group
    L: int = 30      # MoE layers
    S: int = 16      # LFU slots per layer

    def as_dict(self):
        return dataclasses.asdict(self)


GEMMA4_26B = Dims()
# small shape used by fast tests: every tile and slice rule still applies
TINY = Dims(D=512, E=16, K=4, F=64, FS=128, G=64, L=3, S=6)


def _rng(seed, kind, layer, index):
    return np.random.default_rng(np.random.SeedSequence([int(seed), kind, int(layer), int(index)]))


def down_ks(F: int) -> int:
    return F if F <= 704 else 704


def blob_bytes(D: int, F: int) -> int:
    ks = down_ks(F)
    return (F // 16) * (D // 256) * 18 * 256 + (D // 32) * (F // ks) * 18 * ks


def check_shape(D: int, F: int):
    ks = down_ks(F)
    if D % 256 or F % 64 or F % ks or ks % 64:
        raise ValueError(f"unsupported expert shape D={D} F={F}")


# ---------------------------------------------------------------- packing
def _pack_nibbles(q):
    """q [..., 8] nibbles -> [..., 4] bytes (even index low nibble)."""
    q = q.astype(np.uint8)
    return (q[..., 0::2] | (q[..., 1::2] << 4)).astype(np.uint8)


def _chunks(q_rows, s_rows, b_rows, ks):
    """q_rows [tiles, 32, Kin], s/b_rows [tiles, 32, Kin/64] (binary16) ->
    uint8 [tiles, Kin/ks, 18*ks]."""
    tiles, _, kin = q_rows.shape
    nsl = kin // ks
    q = q_rows.reshape(tiles, 32, nsl, ks // 32, 4, 8).transpose(0, 2, 3, 1, 4, 5)
    qb = _pack_nibbles(q).reshape(tiles, nsl, 16 * ks)
    sb = np.stack([s_rows.astype(np.float16).view(np.uint16),
                   b_rows.astype(np.float16).view(np.uint16)], axis=-1)  # [t,32,G,2]
    sb = sb.reshape(tiles, 32, nsl, ks // 64, 2).transpose(0, 2, 3, 1, 4)
    sbb = np.ascontiguousarray(sb).view(np.uint8).reshape(tiles, nsl, 2 * ks)
    return np.concatenate([qb, sbb], axis=2)


def pack_expert(qg, qu, qd, sg, bg, su, bu, sd, bd) -> np.ndarray:
    """Pack one expert from its unpacked parts: q* integer nibbles, s*/b*
    binary16 (np.float16) per group of 64.  qg, qu: [F, D]; qd: [D, F]."""
    F, D = qg.shape
    check_shape(D, F)
    gu_q = np.stack([qg.reshape(F // 16, 16, D), qu.reshape(F // 16, 16, D)], 1).reshape(F // 16, 32, D)
    gu_s = np.stack([sg.reshape(F // 16, 16, -1), su.reshape(F // 16, 16, -1)], 1).reshape(F // 16, 32, -1)
    gu_b = np.stack([bg.reshape(F // 16, 16, -1), bu.reshape(F // 16, 16, -1)], 1).reshape(F // 16, 32, -1)
    sec0 = _chunks(gu_q, gu_s, gu_b, 256)
    sec1 = _chunks(qd.reshape(D // 32, 32, F), sd.reshape(D // 32, 32, -1),
                   bd.reshape(D // 32, 32, -1), down_ks(F))
    out = np.concatenate([sec0.reshape(-1), sec1.reshape(-1)])
    assert out.size == blob_bytes(D, F)
    return out


def draw_expert_parts(seed, layer, expert, D, F, shared=False):
    """Unpacked random expert: dict of q (uint8 nibbles) and binary16 s, b."""
    r = _rng(seed, _SHARED if shared else _ROUTED, layer, expert)
    parts = {}
    for name, (n, kin) in (("g", (F, D)), ("u", (F, D)), ("d", (D, F))):
        parts["q" + name] = r.integers(0, 16, size=(n, kin), dtype=np.uint8)
        s = r.uniform(0.002, 0.02, size=(n, kin // 64)).astype(np.float16)
        parts["s" + name] = s
        parts["b" + name] = (s.astype(np.float32) * -8.0).astype(np.float16)
    return parts


def pack_parts(p) -> np.ndarray:
    return pack_expert(p["qg"], p["qu"], p["qd"], p["sg"], p["bg"], p["su"], p["bu"], p["sd"], p["bd"])


def fill_expert_blob(out: np.ndarray, seed, layer, expert, D, F, shared=False):
    """Full-size generator: writes a random expert blob straight into ``out``
    (uint8, blob_bytes(D, F)), without an unpacked copy.  Nibbles are iid
    uniform, so random bytes in the q parts have exactly the drawn
    distribution; the sb parts receive (scale, -8*scale) pairs."""
    check_shape(D, F)
    nb = blob_bytes(D, F)
    assert out.dtype == np.uint8 and out.size == nb
    r = _rng(seed, _SHARED if shared else _ROUTED, layer, expert)
    out[:] = r.integers(0, 256, size=nb, dtype=np.uint8)
    ks = down_ks(F)
    n0 = (F // 16) * (D // 256)
    sec0 = out[: n0 * 18 * 256].reshape(n0, 18 * 256)
    sec1 = out[n0 * 18 * 256:].reshape(-1, 18 * ks)
    for sec, k in ((sec0, 256), (sec1, ks)):
        npairs = sec.shape[0] * 32 * (k // 64)
        s = r.uniform(0.002, 0.02, size=npairs).astype(np.float16)
        b = (s.astype(np.float32) * -8.0).astype(np.float16)
        sb = np.stack([s.view(np.uint16), b.view(np.uint16)], axis=-1)
        sec[:, 16 * k:] = sb.view(np.uint8).reshape(sec.shape[0], 2 * k)
    return out


def expert_blob(seed, layer, expert, D, F, shared=False) -> np.ndarray:
    out = np.empty(blob_bytes(D, F), dtype=np.uint8)
    return fill_expert_blob(out, seed, layer, expert, D, F, shared)


def fill_store(store: np.ndarray, seed, dims: Dims, layers=None, threads=None):
    """Fill a [L, E, blob] uint8 store (pinned host memory in practice) with
    every routed expert of ``layers`` (default all)."""
    nb = blob_bytes(dims.D, dims.F)
    layers = range(dims.L) if layers is None else layers
    jobs = [(l, e) for l in layers for e in range(dims.E)]
    flat = store.reshape(-1, nb)

    def one(le):
        l, e = le
        fill_expert_blob(flat[l * dims.E + e], seed, l, e, dims.D, dims.F)

    with cf.ThreadPoolExecutor(threads or min(32, os.cpu_count() or 4)) as ex:
        list(ex.map(one, jobs))
    return store


# ----------------------------------------------------------------- router
def router_weights(seed, layer, E, D, G=64):
    """(wq int8 [E, D], ws binary16 bits uint16 [E, D/G])."""
    r = _rng(seed, _ROUTER, layer, 0)
    wq = r.integers(-128, 128, size=(E, D), dtype=np.int16).astype(np.int8)
    ws = r.uniform(1.67e-4, 3.34e-4, size=(E, D // G)).astype(np.float16).view(np.uint16)
    return wq, ws


# Strength of the popularity bias (see zipf_bias), calibrated on the chained
# 30-layer decode (residual stream between layers) with 16 LFU slots and
# Zipf s = 1.1 (a 256-token sequence from cold caches, measured on B200):
#   lambda 0.50: hit rate 0.60 over tokens 5-24, 0.67 over 0-255, repeats 34 % / 52 %
#   lambda 0.55: hit rate 0.63 over tokens 5-24, 0.70 over 0-255, repeats 37 % / 55 %
#   lambda 0.60: hit rate 0.66 over tokens 5-24, 0.73 over 0-255, repeats 39 % / 57 %
#   lambda 0.75: hit rate 0.76 over tokens 5-24, 0.80 over 0-255, repeats 47 % / 64 %
# 0.55 keeps both the early tokens and the whole sequence in the pages' 60-70 %
# band, with next-token / two-token repeats close to their 40 % / 57 %.
ZIPF_LAMBDA = 0.55
# The same band for independent hidden states per (token, layer) (no residual
# stream, so consecutive tokens route less alike): the router + LFU plan over
# such states give a 0.67 hit rate at 16 slots and Zipf 1.1 with lambda 0.75.
# The cache sweep and the plan-only tests draw their states this way.
ZIPF_LAMBDA_UNCHAINED = 0.75


def zipf_bias(seed, layer, E, s=1.1, lam=None):
    """Per-expert popularity bias, float32 [E]: -lam * s * ln(1 + pi(e))."""
    lam = ZIPF_LAMBDA if lam is None else lam
    r = _rng(seed, _ZIPF, layer, 0)
    rank = r.permutation(E).astype(np.float64) + 1.0
    return (-lam * s * np.log(rank)).astype(np.float32)


# ---------------------------------------------------------- hidden states
def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """float32 -> bfloat16 bits, round to nearest even (finite inputs)."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    u = u + 0x7FFF + ((u >> 16) & 1)
    return (u >> 16).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def hidden(seed, token, layer, D) -> np.ndarray:
    """bf16 bits [D] of N(0, 1) for (token, layer)."""
    r = _rng(seed, _HIDDEN, layer, token)
    return to_bf16_bits(r.standard_normal(D).astype(np.float32))


def hidden_batch(seed, tokens, layer, D) -> np.ndarray:
    return np.stack([hidden(seed, t, layer, D) for t in tokens])


def random_ids(seed, T, K, E, index=0) -> np.ndarray:
    """T rows of K distinct expert ids (for cache-plan tests)."""
    r = _rng(seed, _IDS, 0, index)
    return np.stack([r.choice(E, size=K, replace=False) for _ in range(T)]).astype(np.int32)


@dataclasses.dataclass(frozen=True)
class AttnDims:
    """Decode-attention shape.  The pages give the layer mix (25 sliding-window
    layers with a ring KV cache, 5 full-attention layers with linear storage,
    a 4K context) but no head counts; the head counts, head width and window
    here are chosen, not taken from the pages."""
    Hq: int = 16        # query heads
    Hkv: int = 8        # KV heads (query heads h*Hq/Hkv .. share KV head h)
    hd: int = 256       # head width
    window: int = 1024  # ring capacity of a sliding-window layer
    context: int = 4096  # tokens in the context (linear capacity of a full layer)
    sliding: int = 25
    full: int = 5


GEMMA4_ATTN = AttnDims()


def attn_query(seed, token, layer, Hq, hd) -> np.ndarray:
    """bf16 bits [Hq][hd] of N(0, 1)."""
    r = _rng(seed, _ATTN, layer, 2 * token)
    return to_bf16_bits(r.standard_normal((Hq, hd)).astype(np.float32))


def attn_kv(seed, layer, Hkv, cap, hd):
    """binary16 bits of N(0, 1): (k, v), each [Hkv][cap][hd]."""
    r = _rng(seed, _ATTN, layer, -1 & 0x7FFFFFFF)
    k = r.standard_normal((Hkv, cap, hd)).astype(np.float16).view(np.uint16)
    v = r.standard_normal((Hkv, cap, hd)).astype(np.float16).view(np.uint16)
    return k, v
