"""Parity at the workloads' full sizes, in the launch configuration bench.py
times: the whole workload is quantised (one kvq_quantize_append call) and
decoded (one kvq_decode_attention call) on the GPU; the float64 oracle then
checks a seeded sample of tiles and of (sequence, kv-head) outputs."""
import numpy as np
import pytest

from kv_cache_quantization_03_b200 import workloads as W

pytestmark = pytest.mark.gpu

from _parity import ATTN_TOL, CODE_FLIP_RATE, DecodeRun, QuantRun, attention_error, check_tiles  # noqa: E402


@pytest.mark.parametrize("name", ["rt1k", "gqa", "long", "prefill", "mla", "g128", "saw4", "hadonly", "gqa16",
                                  "kivi"])
def test_fullsize_sampled_parity(name):
    w = W.WORKLOADS[name]
    run = QuantRun(w)
    assert run.error_bits() == 0
    rng = np.random.default_rng(1234)
    n_tiles = w.n_tok // w.tile_tokens
    tiles = np.sort(rng.choice(n_tiles, size=min(n_tiles, 160), replace=False))
    layers = sorted(set(rng.integers(0, w.num_layers, size=3).tolist()))
    heads = sorted(set(rng.integers(0, w.num_kv_heads, size=2).tolist()))
    flips = ties = total = 0
    for which in (("k",) if w.mla else ("k", "v")):
        for layer in layers:
            for head in heads:
                f = check_tiles(run, which, layer, tiles, head, "%s %s L%d H%d" % (name, which, layer, head))
                flips, ties = flips + f.counted, ties + f.exact_ties
                total += len(tiles) * w.tile_tokens * w.head_dim
    print("%s: %d counted flips, %d exact ties in %d sampled codes" % (name, flips, ties, total))
    assert flips <= CODE_FLIP_RATE * total, "%d flips in %d sampled codes" % (flips, total)

    # (the prefill workload's step is quantise-append only; its decode is
    # checked too, for the range of its per-channel scales)
    dec = DecodeRun(run)
    o = dec()
    assert run.error_bits() == 0
    assert np.all(np.isfinite(o))
    G = w.group
    pairs = {(int(rng.integers(0, w.batch)), int(rng.integers(0, w.num_kv_heads))) for _ in range(3)}
    for b, h in sorted(pairs):
        err = attention_error(o[b, h * G:(h + 1) * G], dec.oracle(b, h))
        assert err <= ATTN_TOL, "%s seq %d kv-head %d: %g" % (name, b, h, err)
