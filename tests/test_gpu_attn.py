"""GPU parity of decode attention (moe_attn_decode) against the CPU oracle.

Tolerance: |o - r| <= 1e-4 * a + 1e-7 per element, where r is the oracle's
fp64 result and a = sum_p w_p |v_p| is the same attention applied to |V| (the
oracle run on the values with their sign bits cleared).  The kernel's
rounding errors (fp32 dot products over head_dim terms, base-2 exponentials,
fp32 sums over the positions and over the merged parts) are all relative to
these absolute sums, not to |o|, which cancellation can make arbitrarily
small."""
import numpy as np
import pytest
import torch

import oracle
from expert_streaming_decode_b200 import moe, synth

pytestmark = pytest.mark.gpu

ATTN = synth.GEMMA4_ATTN
REL = 1e-4


@pytest.fixture(scope="module")
def O():
    return oracle.get()


def _dev(a):
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda()


def _ws(Hq, hd):
    return torch.zeros(moe.attn_workspace_bytes(Hq, hd), dtype=torch.uint8, device="cuda")


def _gpu(q, k, v, cap, n, scale, ws=None):
    Hq, hd = q.shape
    Hkv = k.shape[0]
    o = torch.full((Hq, hd), float("nan"), dtype=torch.float32, device="cuda")
    ws = _ws(Hq, hd) if ws is None else ws
    moe.attn_decode(_dev(q), _dev(k), _dev(v), Hq, Hkv, hd, cap, n, scale, o, ws)
    torch.cuda.synchronize()
    return o.cpu().numpy()


def _check(O, q, k, v, cap, n, scale, got):
    want = O.attn_decode(q, k, v, cap, n, scale)
    bound = O.attn_decode(q, k, v & np.uint16(0x7FFF), cap, n, scale)
    err = np.abs(got.astype(np.float64) - want)
    lim = REL * bound + 1e-7
    worst = float((err / lim).max())
    assert np.isfinite(got).all() and worst <= 1.0, f"error {worst:.3g} x the bound"
    return worst


def _case(seed, Hq, Hkv, hd, cap):
    q = synth.attn_query(seed, 0, 0, Hq, hd)
    k, v = synth.attn_kv(seed, 0, Hkv, cap, hd)
    return q, k, v


@pytest.mark.parametrize("Hq,Hkv,hd", [(4, 2, 64), (4, 4, 128), (8, 2, 256), (2, 1, 512), (16, 2, 64),
                                       (8, 1, 128), (4, 1, 256), (16, 8, 256)])
def test_attn_small(O, Hq, Hkv, hd):
    """Every head width and group size, a 37-slot cache: empty-ish, ragged,
    exactly full, and wrapped rings (n > capacity)."""
    cap = 37
    q, k, v = _case(3, Hq, Hkv, hd, cap)
    ws = _ws(Hq, hd)
    for n in (1, 2, 5, 36, 37, 38, 111):
        _check(O, q, k, v, cap, n, 1.0 / np.sqrt(hd), _gpu(q, k, v, cap, n, 1.0 / np.sqrt(hd), ws))


@pytest.mark.parametrize("cap,n", [(1000, 1000), (1000, 999), (257, 3000), (4096, 1), (5, 5)])
def test_attn_parts(O, cap, n):
    """Sizes whose parts end mid-batch and whose last part is short."""
    q, k, v = _case(4, 16, 8, 256, cap)
    _check(O, q, k, v, cap, n, 0.0625, _gpu(q, k, v, cap, n, 0.0625))


@pytest.mark.parametrize("kind", ["ring", "linear-full", "linear-partial"])
def test_attn_full_shape(O, kind):
    """The workload's layers: a 1024-slot ring after 4113 tokens, and a
    4096-slot linear cache full or partly filled; every output element."""
    cap, n = {"ring": (ATTN.window, ATTN.context + 17), "linear-full": (ATTN.context, ATTN.context),
              "linear-partial": (ATTN.context, 3001)}[kind]
    q, k, v = _case(5, ATTN.Hq, ATTN.Hkv, ATTN.hd, cap)
    scale = 1.0 / np.sqrt(ATTN.hd)
    _check(O, q, k, v, cap, n, scale, _gpu(q, k, v, cap, n, scale))


def test_attn_peaked_scores(O):
    """A large scale makes the softmax nearly one-hot (scores spread over
    hundreds): the running maximum must keep every exponential finite."""
    q, k, v = _case(6, 16, 8, 256, 500)
    for scale in (1.0, 4.0):
        _check(O, q, k, v, 500, 500, scale, _gpu(q, k, v, 500, 500, scale))


def test_attn_reproducible_and_workspace_reuse(O):
    """Parts merge in a fixed order: two calls agree bit for bit, and a
    workspace used for another shape in between still works."""
    q, k, v = _case(7, 16, 8, 256, 1024)
    ws = _ws(16, 256)
    a = _gpu(q, k, v, 1024, 2000, 0.0625, ws)
    q2, k2, v2 = _case(8, 4, 2, 64, 50)
    _check(O, q2, k2, v2, 50, 50, 0.125, _gpu(q2, k2, v2, 50, 50, 0.125, ws))
    b = _gpu(q, k, v, 1024, 2000, 0.0625, ws)
    assert np.array_equal(a.view(np.uint32), b.view(np.uint32))
    _check(O, q, k, v, 1024, 2000, 0.0625, a)


def test_attn_rejects_bad_arguments():
    Hq, Hkv, hd, cap = 4, 2, 64, 8
    q = torch.zeros((Hq, hd), dtype=torch.int16, device="cuda")
    k = torch.zeros((Hkv, cap, hd), dtype=torch.int16, device="cuda")
    o = torch.zeros((Hq, hd), dtype=torch.float32, device="cuda")
    ws = _ws(Hq, hd)
    nb = ws.numel()
    L = moe.lib

    def call(q_=q, hq=Hq, hkv=Hkv, hd_=hd, n=4, scale=0.1, wsb=nb):
        return L.moe_attn_decode(q_.data_ptr(), k.data_ptr(), k.data_ptr(), hq, hkv, hd_, cap, n, scale,
                                 o.data_ptr(), ws.data_ptr(), wsb, None)

    assert call() == moe.MOE_OK
    assert call(n=0) == moe.MOE_ERR_ARG                     # nothing to attend to
    assert call(hd_=96) == moe.MOE_ERR_ARG                  # unsupported head width
    assert call(hq=6, hkv=4) == moe.MOE_ERR_ARG             # heads not a multiple
    assert call(hq=32, hkv=2) == moe.MOE_ERR_ARG            # group of 16
    assert call(scale=0.0) == moe.MOE_ERR_ARG
    assert call(scale=float("nan")) == moe.MOE_ERR_ARG
    assert call(wsb=nb - 1) == moe.MOE_ERR_ARG              # workspace too small
    assert L.moe_attn_decode(q.data_ptr() + 2, k.data_ptr(), k.data_ptr(), Hq, Hkv, hd, cap, 4, 0.1,
                             o.data_ptr(), ws.data_ptr(), nb, None) == moe.MOE_ERR_ARG  # misaligned
    torch.cuda.synchronize()
