"""Parity at the workloads' full sizes, in the launch configuration bench.py
times: the whole workload is quantised (one kvq_quantize_append call) and
decoded (one kvq_decode_attention call) on the GPU; the float64 oracle then
checks a seeded sample of tiles and of (sequence, kv-head) outputs."""
import numpy as np
import pytest

from kv_cache_quantization_03_b200 import workloads as W

pytestmark = pytest.mark.gpu

from _parity import (ATTN_TOL, CODE_FLIP_RATE, DecodeRun, QuantRun, attention_error, check_tiles,  # noqa: E402
                     compare_quantized, gpu_pages, mla_oracle_tail)


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


@pytest.mark.parametrize("name", ["long", "gqa", "g128", "mla"])
def test_fullsize_decode_fill_parity(name):
    """The decode step with quantise-on-fill that bench.py times at full size
    (decode_fill): sequences b with b % 16 == 0 have just filled their last
    page, which the call quantises from the tail buffer before the decode
    reads it; the others keep tails of tail_lens[b] < T tokens."""
    import torch

    import bench
    from kv_cache_quantization_03_b200 import kvq
    from oracle import kvarn_oracle as O

    w = W.WORKLOADS[name]
    run = QuantRun(w)
    tl, fill = bench.fill_state(w)
    dec = DecodeRun(run)
    kt = W.tail_inputs(w, "k")
    vt = W.tail_rope_inputs(w) if w.mla else W.tail_inputs(w, "v")
    dec.k_tail_bits, dec.v_tail_bits, dec.tl = kt, vt, tl
    kvq.kvq_decode_attention_fill(run.cfg, run.cache.view, 0, dec.q, dec.bt_d, dec.maxp, dec.sl_d,
                                  torch.from_numpy(kt.view(np.int16)).cuda(), torch.from_numpy(vt.view(np.int16)).cuda(),
                                  torch.from_numpy(tl).cuda(), torch.from_numpy(fill).cuda(), dec.batch, dec.hq,
                                  w.softmax_scale, dec.out, dec.ws, dec.ws_bytes, run.err)
    torch.cuda.synchronize()
    o = dec.out.cpu().numpy().astype(np.float64)
    assert run.error_bits() == 0
    rng = np.random.default_rng(4321)
    filled = np.nonzero(fill >= 0)[0]
    heads = sorted(set(rng.integers(0, w.num_kv_heads, size=2).tolist()))
    # the filled pages hold the quantised tails
    for b in filled[:2]:
        for which in (("k",) if w.mla else ("k", "v")):
            bits = w.bits_k if which == "k" else w.bits_v
            src = kt if which == "k" else vt
            for h in heads:
                x = W.half_bits_to_f64(src[0, b, :, h], w.in_dtype)[None]      # [1, T, d]
                ora = O.quantize_tiles(x, bits, w.sinkhorn_iters, w.block)
                compare_quantized(gpu_pages(run, which, 0, [fill[b]], h), ora, x, bits, w.sinkhorn_iters, w.block,
                                  "%s seq %d %s H%d" % (name, b, which, h), check_rate=False)
    # attention of a filled sequence and of two sequences with tails
    others = np.nonzero(fill < 0)[0]
    seqs = [int(filled[0])] + [int(b) for b in rng.choice(others, size=min(2, len(others)), replace=False)]
    for b in seqs:
        if w.mla:
            err = attention_error(o[b], mla_oracle_tail(dec, b))
            assert err <= ATTN_TOL, "%s seq %d (tail %d): %g" % (name, b, tl[b], err)
            continue
        h = int(rng.integers(0, w.num_kv_heads))
        G = w.group
        err = attention_error(o[b, h * G:(h + 1) * G], dec.oracle_tail(b, h, 0))
        assert err <= ATTN_TOL, "%s seq %d kv-head %d (tail %d): %g" % (name, b, h, tl[b], err)
