"""bench.py's argument rules, on CPU: the miss-fill and look-ahead defaults
and the combinations refused, and the attention workload's layer mix and
bytes."""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402
from expert_streaming_decode_b200 import synth  # noqa: E402


def _args(*argv):
    old = sys.argv
    sys.argv = ["bench.py", *argv]
    try:
        return bench.parse_args()
    finally:
        sys.argv = old


def test_fill_and_lookahead_defaults():
    """Misses are copied by the copy engine with one look-ahead buffer by
    default (the faster of the two fills on B200 today); the direct fill
    takes no look-ahead."""
    a = _args()
    assert a.fill == "copy" and a.prefetch == 1
    assert _args("--fill", "direct").prefetch == 0
    assert _args("--fill", "copy", "--prefetch", "0").prefetch == 0
    assert _args("--workload", "prefill").prefetch == 0
    assert _args("--workload", "decode_resident", "--batch", "8").prefetch == 0
    assert _args("--store-file", "/tmp/x").prefetch == 0
    assert _args("--workload", "attn_decode").prefetch == 0


@pytest.mark.parametrize("argv", [("--workload", "prefill", "--prefetch", "1"),
                                  ("--store-file", "/tmp/x", "--prefetch", "2"),
                                  ("--fill", "direct", "--prefetch", "1"),
                                  ("--prefetch", "17")])
def test_lookahead_refused_where_it_does_not_apply(argv):
    with pytest.raises(SystemExit):
        _args(*argv)


def test_attention_layer_mix_and_bytes():
    A = synth.GEMMA4_ATTN
    layers = bench._attn_layers(A)
    assert len(layers) == 30
    assert sum(c == A.context for c, _ in layers) == 5 and sum(c == A.window for c, _ in layers) == 25
    assert all(n == A.context for _, n in layers)
    # K and V rows of every KV head, plus the bf16 query and the fp32 output
    assert bench._attn_bytes(A, A.window, A.context) == 2 * 1024 * 8 * 256 * 2 + 16 * 256 * 6
    assert bench._attn_bytes(A, A.context, A.context) == 2 * 4096 * 8 * 256 * 2 + 16 * 256 * 6
    assert bench._attn_bytes(A, A.context, 100) == 2 * 100 * 8 * 256 * 2 + 16 * 256 * 6
