"""Seeded synthetic layers for the GPU parity tests: the same generator bytes
go to the CUDA path (device or pinned tensors) and to the oracle (numpy)."""
from __future__ import annotations

import numpy as np
import torch

from expert_streaming_decode_b200 import moe, synth


def stride_for(nbytes: int) -> int:
    return (nbytes + 255) // 256 * 256


class Layer:
    """One MoE layer's weights: router, shared blob, the E routed blobs
    (numpy), optionally uploaded as a resident device array and/or a pinned
    host store."""

    def __init__(self, d: synth.Dims, layer: int, seed: int = 0, zipf_s: float | None = 1.1,
                 resident: bool = True, pinned: bool = False, shared: bool = True):
        self.d, self.layer = d, layer
        self.nb = synth.blob_bytes(d.D, d.F)
        self.stride = stride_for(self.nb)
        self.wq, self.ws = synth.router_weights(seed, layer, d.E, d.D)
        self.bias = None if zipf_s is None else synth.zipf_bias(seed, layer, d.E, s=zipf_s)
        self.shared = synth.expert_blob(seed, layer, 0, d.D, d.FS, shared=True) if shared else None
        host = np.zeros((d.E, self.stride), dtype=np.uint8)
        for e in range(d.E):
            synth.fill_expert_blob(host[e, :self.nb], seed, layer, e, d.D, d.F)
        self.blobs = [host[e, :self.nb] for e in range(d.E)]
        self.host = host
        dev = torch.device("cuda")
        self.wq_t = torch.from_numpy(self.wq).to(dev)
        self.ws_t = torch.from_numpy(self.ws.view(np.int16)).to(dev)
        self.bias_t = None if self.bias is None else torch.from_numpy(self.bias).to(dev)
        self.shared_t = None if shared is False else torch.from_numpy(self.shared).to(dev)
        self.experts_t = torch.from_numpy(host).to(dev) if resident else None
        self.store_t = torch.from_numpy(host).pin_memory() if pinned else None

    def weights(self, resident=True):
        return moe.layer_weights(self.wq_t, self.ws_t, self.shared_t,
                                 self.experts_t if resident else None, self.stride if resident else 0)

    def oracle_token(self, O, xb):
        """(ids, gate_w, logits, y) for one token (bf16 bits)."""
        return O.moe_token(self.d.as_dict(), xb, self.wq, self.ws, self.bias, self.shared, self.blobs)


def bf16_tensor(bits: np.ndarray):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda()


def rel_err(y, r) -> float:
    """Max error relative to the reference vector's max magnitude (outputs
    cross zero, so elementwise relative error is meaningless)."""
    y = np.asarray(y, dtype=np.float64)
    r = np.asarray(r, dtype=np.float64)
    return float(np.max(np.abs(y - r)) / max(np.max(np.abs(r)), 1e-30))


TOL = 2e-3       # max |y - r| / max |r| per (token, layer)
GATE_TOL = 1e-5  # gate weights, absolute
