"""Python binding of libmoe.so (C ABI in include/moe.h).

Argument marshalling only: every function forwards torch tensors' device
pointers and the current CUDA stream to the C entry point of the same name and
raises MoeError on a non-zero status.  All arithmetic runs in the CUDA kernels
of libmoe.so; there is no fallback path.  Importing this module fails loudly
when the library has not been built (python -m expert_streaming_decode_b200.build).
"""
from __future__ import annotations

import ctypes as C
import os
import re

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoe.so")
HEADER = os.path.join(os.path.dirname(_HERE), "include", "moe.h")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"libmoe.so is not built ({LIB_PATH}); run `python -m expert_streaming_decode_b200.build`")
lib = C.CDLL(LIB_PATH)

MOE_OK, MOE_ERR_ARG, MOE_ERR_CUDA, MOE_ERR_TIMEOUT, MOE_ERR_STATE, MOE_ERR_NAN, MOE_ERR_RANGE = 0, -1, -2, -3, -4, -5, -6
MOE_ERR_IO = -7


class MoeError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {lib.moe_status_str(code).decode()} ({code})")


class moe_dims(C.Structure):
    _fields_ = [("d_model", C.c_int), ("n_experts", C.c_int), ("top_k", C.c_int), ("d_ff", C.c_int),
                ("d_ff_shared", C.c_int), ("group", C.c_int), ("n_slots", C.c_int), ("max_tokens", C.c_int)]


class moe_slot_cache(C.Structure):
    _fields_ = [("slots", C.c_void_p), ("slot_stride", C.c_size_t), ("state", C.c_void_p),
                ("store", C.c_void_p), ("store_stride", C.c_size_t), ("policy", C.c_int32),
                ("decay_period", C.c_uint32), ("source", C.c_int32), ("store_fd", C.c_int32),
                ("store_file_offset", C.c_uint64)]


MOE_SOURCE_HOST, MOE_SOURCE_FILE, MOE_SOURCE_HOST_DIRECT = 0, 1, 2
STAT_NAMES = ("calls", "hits", "misses", "miss_bytes", "repeat_prev", "repeat_prev2", "planned")
MOE_STATS = 8


MOE_POLICY_LFU, MOE_POLICY_LRU, MOE_POLICY_LFU_DECAY, MOE_POLICY_LFU_IN_CACHE = 0, 1, 2, 3


class moe_layer_weights(C.Structure):
    _fields_ = [("router_q", C.c_void_p), ("router_s", C.c_void_p), ("shared_blob", C.c_void_p),
                ("experts", C.c_void_p), ("expert_stride", C.c_size_t)]


_I32P = C.POINTER(C.c_int32)


class moe_next_layer(C.Structure):
    pass


moe_next_layer._fields_ = [("W", C.POINTER(moe_layer_weights)), ("cache", C.POINTER(moe_slot_cache)),
                           ("bias", C.c_void_p), ("after", C.POINTER(moe_next_layer))]


class moe_plan_trace(C.Structure):
    _fields_ = [("capacity", C.c_int32), ("n_distinct", C.c_int32), ("n_waves", C.c_int32),
                ("n_misses", C.c_int32), ("h2d_bytes", C.c_uint64), ("expert", _I32P), ("slot", _I32P),
                ("hit", _I32P), ("victim", _I32P), ("wave", _I32P)]


_vp, _i, _sz, _u32 = C.c_void_p, C.c_int, C.c_size_t, C.c_uint32
lib.moe_blob_bytes.restype = _sz
lib.moe_blob_bytes.argtypes = [_i, _i]
lib.moe_cache_state_words.restype = _sz
lib.moe_cache_state_words.argtypes = [C.POINTER(moe_dims)]
lib.moe_status_str.restype = C.c_char_p
lib.moe_status_str.argtypes = [_i]
lib.moe_ctx_create.restype = _i
lib.moe_ctx_create.argtypes = [C.POINTER(moe_dims), _i, C.POINTER(_vp)]
lib.moe_ctx_destroy.restype = _i
lib.moe_ctx_destroy.argtypes = [_vp]
lib.moe_ctx_sync.restype = _i
lib.moe_ctx_sync.argtypes = [_vp, _vp, _i]
lib.moe_ctx_launches.restype = C.c_uint64
lib.moe_ctx_launches.argtypes = [_vp]
lib.moe_gemm_min_tokens.restype = _i
lib.moe_gemm_min_tokens.argtypes = []
lib.moe_router_topk.restype = _i
lib.moe_router_topk.argtypes = [_vp, _vp, _vp, _vp, _vp, _i, _vp, _vp, _vp]
lib.moe_cache_reset.restype = _i
lib.moe_cache_reset.argtypes = [_vp, C.POINTER(moe_slot_cache), _vp]
lib.moe_cache_plan.restype = _i
lib.moe_cache_plan.argtypes = [_vp, C.POINTER(moe_slot_cache), _vp, _i, _u32, _vp, C.POINTER(moe_plan_trace), _vp]
lib.moe_expert_ffn.restype = _i
lib.moe_expert_ffn.argtypes = [_vp, _vp, _i, _i, _vp, _vp, _vp, _sz, _i, _i, _vp, _vp, _vp, _vp]
lib.moe_expert_ffn_noalloc.restype = _i
lib.moe_expert_ffn_noalloc.argtypes = [_i, _i, _i, _vp, _vp, _vp, _vp, _sz, _i, _vp, _vp, _vp, _vp]
lib.moe_layer_forward.restype = _i
lib.moe_layer_forward.argtypes = [_vp, C.POINTER(moe_layer_weights), C.POINTER(moe_slot_cache), _vp, _i, _u32,
                                  _vp, _vp, _vp, _vp, _vp, C.POINTER(moe_plan_trace), _vp]
lib.moe_layer_forward_next.restype = _i
lib.moe_layer_forward_next.argtypes = [_vp, C.POINTER(moe_layer_weights), C.POINTER(moe_slot_cache), _vp, _i, _u32,
                                       _vp, _vp, _vp, _vp, _vp, C.POINTER(moe_plan_trace), C.POINTER(moe_next_layer),
                                       _vp]
lib.moe_prefetch_configure.restype = _i
lib.moe_prefetch_configure.argtypes = [_vp, _i]
lib.moe_prefetch_stats.restype = _i
lib.moe_prefetch_stats.argtypes = [_vp, C.POINTER(C.c_uint64), C.POINTER(C.c_uint64)]
lib.moe_attn_workspace_bytes.restype = _sz
lib.moe_attn_workspace_bytes.argtypes = [_i, _i]
lib.moe_attn_decode.restype = _i
lib.moe_attn_decode.argtypes = [_vp, _vp, _vp, _i, _i, _i, _i, _i, C.c_float, _vp, _vp, _sz, _vp]
lib.moe_ctx_profile.restype = _i
lib.moe_ctx_profile.argtypes = [_vp, _i]
lib.moe_ctx_profile_read.restype = _i
lib.moe_ctx_profile_read.argtypes = [_vp, C.POINTER(C.c_double), C.POINTER(C.c_uint64)]
lib.moe_ctx_stats.restype = _i
lib.moe_ctx_stats.argtypes = [_vp, _vp, C.POINTER(C.c_uint64)]
lib.moe_ctx_stats_reset.restype = _i
lib.moe_ctx_stats_reset.argtypes = [_vp, _vp]
lib.moe_residual_rmsnorm.restype = _i
lib.moe_residual_rmsnorm.argtypes = [_vp, _vp, _vp, _vp, _i, _vp]
lib.moe_bf16_to_f32.restype = _i
lib.moe_bf16_to_f32.argtypes = [_vp, _vp, _vp, _sz, _vp]


def declared_symbols(header: str = HEADER) -> list[str]:
    """Entry points declared in include/moe.h."""
    src = open(header).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(moe_[a-z0-9_]+)\s*\(", src)))


def _check(code: int, where: str):
    if code != MOE_OK:
        raise MoeError(code, where)


def _ptr(t):
    return None if t is None else C.c_void_p(t.data_ptr())


def _stream(stream):
    import torch
    s = torch.cuda.current_stream() if stream is None else stream
    return C.c_void_p(s.cuda_stream)


def blob_bytes(d_model: int, d_ff: int) -> int:
    return int(lib.moe_blob_bytes(d_model, d_ff))


def status_str(code: int) -> str:
    return lib.moe_status_str(code).decode()


class Ctx:
    """A libmoe context (moe_ctx_create / moe_ctx_destroy)."""

    def __init__(self, D, E, K, F, FS, S, max_tokens, device=0, G=64):
        self.dims = moe_dims(D, E, K, F, FS, G, S, max_tokens)
        h = C.c_void_p()
        _check(lib.moe_ctx_create(C.byref(self.dims), device, C.byref(h)), "moe_ctx_create")
        self.h = h

    @classmethod
    def from_dims(cls, d, max_tokens, device=0, S=None):
        return cls(d.D, d.E, d.K, d.F, d.FS, d.S if S is None else S, max_tokens, device, d.G)

    def close(self):
        if self.h:
            lib.moe_ctx_destroy(self.h)
            self.h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def sync(self, stream=None, timeout_ms=20000):
        """moe_ctx_sync: raises MoeError with the first device-side error."""
        _check(lib.moe_ctx_sync(self.h, _stream(stream), timeout_ms), "moe_ctx_sync")

    def sync_status(self, stream=None, timeout_ms=20000) -> int:
        return int(lib.moe_ctx_sync(self.h, _stream(stream), timeout_ms))

    @property
    def launches(self) -> int:
        return int(lib.moe_ctx_launches(self.h))

    PROF_KINDS = ("router", "plan", "worklist", "gate_up", "down", "harness", "h2d", "layer")

    def profile(self, enable: bool):
        _check(lib.moe_ctx_profile(self.h, int(enable)), "moe_ctx_profile")

    def profile_read(self) -> dict:
        """{kind: (total_ms, intervals)} since the last read (synchronous)."""
        ms = (C.c_double * len(self.PROF_KINDS))()
        n = (C.c_uint64 * len(self.PROF_KINDS))()
        _check(lib.moe_ctx_profile_read(self.h, ms, n), "moe_ctx_profile_read")
        return {k: (ms[i], int(n[i])) for i, k in enumerate(self.PROF_KINDS)}

    def stats(self, stream=None) -> dict:
        """The device cache counters (moe_ctx_stats), by name."""
        out = (C.c_uint64 * MOE_STATS)()
        _check(lib.moe_ctx_stats(self.h, _stream(stream), out), "moe_ctx_stats")
        return {k: int(out[i]) for i, k in enumerate(STAT_NAMES)}

    def stats_reset(self, stream=None):
        _check(lib.moe_ctx_stats_reset(self.h, _stream(stream)), "moe_ctx_stats_reset")

    def state_words(self) -> int:
        return int(lib.moe_cache_state_words(C.byref(self.dims)))


def router_topk(ctx: Ctx, x, wq, ws, bias, T, ids, gate_w, stream=None):
    _check(lib.moe_router_topk(ctx.h, _ptr(x), _ptr(wq), _ptr(ws), _ptr(bias), T, _ptr(ids), _ptr(gate_w),
                               _stream(stream)), "moe_router_topk")


def slot_cache(slots, slot_stride, state, store=None, store_stride=0, policy=MOE_POLICY_LFU,
               decay_period=0, store_fd=None, store_file_offset=0, direct=False) -> moe_slot_cache:
    """moe_slot_cache for torch tensors.  The struct keeps references to the
    tensors, so their memory lives at least as long as the struct.  With
    store_fd (an open file descriptor) the misses are read from that file at
    store_file_offset + e * store_stride instead of the pinned `store`; with
    direct=True one-token layers read missed experts from the pinned `store`
    inside the layer kernel (MOE_SOURCE_HOST_DIRECT)."""
    src = MOE_SOURCE_HOST if store_fd is None else MOE_SOURCE_FILE
    if direct:
        if store_fd is not None:
            raise ValueError("direct reads need the pinned host store, not a file")
        src = MOE_SOURCE_HOST_DIRECT
    c = moe_slot_cache(slots.data_ptr(), slot_stride, state.data_ptr(),
                       None if store is None else store.data_ptr(), store_stride, policy, decay_period,
                       src, -1 if store_fd is None else store_fd, store_file_offset)
    c._keep = (slots, state, store)
    return c


def cache_reset(ctx: Ctx, cache: moe_slot_cache, stream=None):
    _check(lib.moe_cache_reset(ctx.h, C.byref(cache), _stream(stream)), "moe_cache_reset")


class Trace:
    """Host arrays receiving one call's plan (moe_plan_trace)."""

    def __init__(self, capacity: int):
        import numpy as np
        self.arrays = {k: np.full(capacity, -1, dtype=np.int32) for k in ("expert", "slot", "hit", "victim", "wave")}
        a = self.arrays
        self.c = moe_plan_trace(capacity, 0, 0, 0, 0, *[a[k].ctypes.data_as(_I32P)
                                                        for k in ("expert", "slot", "hit", "victim", "wave")])

    def result(self) -> dict:
        n = self.c.n_distinct
        out = {k: v[:n].copy() for k, v in self.arrays.items()}
        out.update(n_distinct=n, waves=self.c.n_waves, misses=self.c.n_misses, h2d_bytes=int(self.c.h2d_bytes))
        return out


def cache_plan(ctx: Ctx, cache: moe_slot_cache, ids, T, step, pair_slot, trace: Trace | None = None, stream=None):
    _check(lib.moe_cache_plan(ctx.h, C.byref(cache), _ptr(ids), T, step, _ptr(pair_slot),
                              None if trace is None else C.byref(trace.c), _stream(stream)), "moe_cache_plan")


def expert_ffn(ctx: Ctx, x, T, top_k, pair_slot, gate_w, slot_base, slot_stride, n_slot_range, d_ff, y_in, y,
               y_bf16=None, stream=None, slot_base_ptr=None):
    base = C.c_void_p(slot_base_ptr) if slot_base_ptr is not None else _ptr(slot_base)
    _check(lib.moe_expert_ffn(ctx.h, _ptr(x), T, top_k, _ptr(pair_slot), _ptr(gate_w), base, slot_stride,
                              n_slot_range, d_ff, _ptr(y_in), _ptr(y), _ptr(y_bf16), _stream(stream)),
           "moe_expert_ffn")


def expert_ffn_noalloc(d_model, d_ff, top_k, x, pair_slot, gate_w, slot_base, slot_stride, n_slot_range, y_in, y,
                       y_bf16=None, stream=None, slot_base_ptr=None):
    """moe_expert_ffn_noalloc: one token, no context and no device allocation."""
    base = C.c_void_p(slot_base_ptr) if slot_base_ptr is not None else _ptr(slot_base)
    _check(lib.moe_expert_ffn_noalloc(d_model, d_ff, top_k, _ptr(x), _ptr(pair_slot), _ptr(gate_w), base,
                                      slot_stride, n_slot_range, _ptr(y_in), _ptr(y), _ptr(y_bf16),
                                      _stream(stream)), "moe_expert_ffn_noalloc")


def layer_weights(router_q, router_s, shared_blob=None, experts=None, expert_stride=0) -> moe_layer_weights:
    """moe_layer_weights for torch tensors; keeps references to them (a struct
    of raw pointers alone would let the allocator reuse their memory)."""
    w = moe_layer_weights(router_q.data_ptr(), router_s.data_ptr(),
                          None if shared_blob is None else shared_blob.data_ptr(),
                          None if experts is None else experts.data_ptr(), expert_stride)
    w._keep = (router_q, router_s, shared_blob, experts)
    return w


def layer_forward(ctx: Ctx, W: moe_layer_weights, cache: moe_slot_cache | None, x, T, step, bias, y, y_bf16=None,
                  ids=None, gate_w=None, trace: Trace | None = None, stream=None):
    _check(lib.moe_layer_forward(ctx.h, C.byref(W), None if cache is None else C.byref(cache), _ptr(x), T, step,
                                 _ptr(bias), _ptr(y), _ptr(y_bf16), _ptr(ids), _ptr(gate_w),
                                 None if trace is None else C.byref(trace.c), _stream(stream)),
           "moe_layer_forward")


def next_layer(W: moe_layer_weights, cache: "moe_slot_cache | None", bias=None, after: "moe_next_layer | None" = None):
    """The layer after the one being run, for moe_layer_forward_next (keeps its
    structures alive with it); `after` is the layer after that, or None.  A
    next layer without a cache (resident experts) stages nothing."""
    n = moe_next_layer(C.pointer(W), C.pointer(cache) if cache is not None else None, _ptr(bias),
                       C.pointer(after) if after is not None else None)
    n._keep = (W, cache, bias, after)
    return n


def layer_forward_next(ctx: Ctx, W: moe_layer_weights, cache: "moe_slot_cache | None", x, T, step, bias, y,
                       next: moe_next_layer | None, y_bf16=None, ids=None, gate_w=None, trace: Trace | None = None,
                       stream=None):
    _check(lib.moe_layer_forward_next(ctx.h, C.byref(W), None if cache is None else C.byref(cache), _ptr(x), T, step,
                                      _ptr(bias), _ptr(y),
                                      _ptr(y_bf16), _ptr(ids), _ptr(gate_w),
                                      None if trace is None else C.byref(trace.c),
                                      None if next is None else C.byref(next), _stream(stream)),
           "moe_layer_forward_next")


def prefetch_configure(ctx: Ctx, n_buffers: int):
    _check(lib.moe_prefetch_configure(ctx.h, n_buffers), "moe_prefetch_configure")


def prefetch_stats(ctx: Ctx):
    """(issued_bytes, used_bytes) of the look-ahead prefetch so far."""
    a, b = C.c_uint64(0), C.c_uint64(0)
    _check(lib.moe_prefetch_stats(ctx.h, C.byref(a), C.byref(b)), "moe_prefetch_stats")
    return a.value, b.value


def attn_workspace_bytes(n_heads_q: int, head_dim: int) -> int:
    return int(lib.moe_attn_workspace_bytes(n_heads_q, head_dim))


def attn_decode(q, k_cache, v_cache, n_heads_q, n_heads_kv, head_dim, capacity, n_tokens, scale, o, workspace,
                stream=None):
    """Decode attention of one token (moe_attn_decode).  `workspace` is a
    zero-initialised device byte tensor of at least attn_workspace_bytes."""
    _check(lib.moe_attn_decode(_ptr(q), _ptr(k_cache), _ptr(v_cache), n_heads_q, n_heads_kv, head_dim, capacity,
                               n_tokens, float(scale), _ptr(o), _ptr(workspace),
                               0 if workspace is None else workspace.numel() * workspace.element_size(),
                               _stream(stream)),
           "moe_attn_decode")


def residual_rmsnorm(ctx: Ctx, r, y, x_next, T, stream=None):
    _check(lib.moe_residual_rmsnorm(ctx.h, _ptr(r), _ptr(y), _ptr(x_next), T, _stream(stream)),
           "moe_residual_rmsnorm")


def bf16_to_f32(ctx: Ctx, x, out, n, stream=None):
    _check(lib.moe_bf16_to_f32(ctx.h, _ptr(x), _ptr(out), n, _stream(stream)), "moe_bf16_to_f32")
