"""GPU parity of decode attention with an unquantised tail
(kvq_decode_attention_tail) and of quantise-on-fill (kvq_quantize_append over
a tail buffer with page -1 for the tails that are not full), against the
float64 oracle."""
import dataclasses

import numpy as np
import pytest
import torch

from kv_cache_quantization_03_b200 import kvq, workloads as W
from oracle import kvarn_oracle as O

pytestmark = pytest.mark.gpu

from _parity import (ATTN_TOL, CODE_FLIP_RATE, MLA_SHORT_ATTN_TOL, DecodeRun, QuantRun,  # noqa: E402
                     attention_error, compare_quantized, mla_oracle_tail)


def _check_tail(dec: DecodeRun, o: np.ndarray, layer=0, lens=None):
    w = dec.run.w
    G = dec.hq // w.num_kv_heads
    for b in range(dec.batch):
        for h in range(w.num_kv_heads):
            L = None if lens is None else lens[b]
            ref = dec.oracle_tail(b, h, layer, L)
            got = o[b, h * G:(h + 1) * G]
            if dec.sl[b] // w.tile_tokens == 0 and (L if L is not None else dec.tl[b]) == 0:
                assert np.all(got == 0)
                continue
            err = attention_error(got, ref)
            assert err <= ATTN_TOL, "seq %d kv-head %d: %g" % (b, h, err)


@pytest.mark.parametrize("name,kw,seq_lens", [
    ("gqa", dict(batch=4, seq_len=512), [512, 256, 0, 496]),
    ("g128", dict(batch=3, seq_len=1024), [1024, 0, 640]),
    ("rt1k", dict(batch=2, seq_len=256), [256, 16]),          # fp16 tail rows, one query head
    ("long", dict(batch=2, seq_len=512), [512, 128]),         # 8 query heads per kv-head, 3-bit keys
    ("saw4", dict(batch=2, seq_len=256), [256, 64]),          # block-diagonal rotation
])
def test_decode_with_tail_parity(name, kw, seq_lens):
    w = W.WORKLOADS[name].scaled(**kw)
    run = QuantRun(w)
    dec = DecodeRun(run, seq_lens=seq_lens)
    lens = W.tail_lens(w)
    lens[0] = w.tile_tokens - 1                                # the longest tail
    lens[-1] = 0                                               # no tail
    o = dec.with_tail(W.tail_inputs(w, "k"), W.tail_inputs(w, "v"), lens)
    assert run.error_bits() == 0
    assert np.all(np.isfinite(o))
    _check_tail(dec, o)


def test_tail_only_sequences_and_full_tail():
    # no cached page at all (seq_len 0), and a tail of T rows (full, not yet quantised)
    w = W.WORKLOADS["gqa"].scaled(batch=3, seq_len=256)
    run = QuantRun(w)
    dec = DecodeRun(run, seq_lens=[0, 0, 256])
    o = dec.with_tail(W.tail_inputs(w, "k"), W.tail_inputs(w, "v"), [7, w.tile_tokens, w.tile_tokens])
    assert run.error_bits() == 0
    _check_tail(dec, o)


def test_bad_tail_length_sets_error_and_ignores_tail():
    w = W.WORKLOADS["gqa"].scaled(batch=2, seq_len=256)
    run = QuantRun(w)
    dec = DecodeRun(run)
    o = dec.with_tail(W.tail_inputs(w, "k"), W.tail_inputs(w, "v"), [w.tile_tokens + 1, -3])
    assert run.error_bits() & kvq.KVQ_DEVERR_BAD_SEQ
    _check_tail(dec, o, lens=[0, 0])


def test_tail_of_a_later_layer():
    w = W.WORKLOADS["gqa"].scaled(batch=2, seq_len=256, num_layers=3)
    run = QuantRun(w)
    dec = DecodeRun(run)
    kt, vt = W.tail_inputs(w, "k"), W.tail_inputs(w, "v")
    for layer in (0, 2):
        bt = dec.bt_d
        kvq.kvq_decode_attention_tail(run.cfg, run.cache.view, layer, dec.q, bt, dec.maxp, dec.sl_d,
                                      torch.from_numpy(kt.view(np.int16)).cuda(),
                                      torch.from_numpy(vt.view(np.int16)).cuda(),
                                      torch.tensor([5, 12], dtype=torch.int32, device="cuda"), dec.batch, dec.hq,
                                      w.softmax_scale, dec.out, dec.ws, dec.ws_bytes, run.err)
        torch.cuda.synchronize()
        o = dec.out.cpu().numpy().astype(np.float64)
        dec.k_tail_bits, dec.v_tail_bits, dec.tl = kt, vt, np.array([5, 12], dtype=np.int32)
        G = dec.hq // w.num_kv_heads
        for b in range(2):
            for h in range(w.num_kv_heads):
                err = attention_error(o[b, h * G:(h + 1) * G], dec.oracle_tail(b, h, layer))
                assert err <= ATTN_TOL


@pytest.mark.parametrize("name", ["gqa", "g128"])
def test_quantize_on_fill_skips_partial_tails(name):
    # a tail buffer of 4 sequences x all layers: sequences 1 and 3 have full
    # tails and get pages 5 and 2; the others pass page -1 and are skipped
    w = W.WORKLOADS[name].scaled(batch=4, seq_len=W.WORKLOADS[name].tile_tokens, num_layers=2)
    run = QuantRun(w, quantize=False, num_pages=8)
    kt, vt = W.tail_inputs(w, "k"), W.tail_inputs(w, "v")      # [layers][4][T][H][d] = [layers][4 T][H][d]
    for which in ("k", "v"):
        run.cache.codes(which).fill_(0xA5)
    dst = torch.tensor([-1, 5, -1, 2], dtype=torch.int32, device="cuda")
    kvq.kvq_quantize_append(run.cfg, run.cache.view, torch.from_numpy(kt.view(np.int16)).cuda(),
                            torch.from_numpy(vt.view(np.int16)).cuda(), None, 4 * w.tile_tokens, dst, run.err)
    torch.cuda.synchronize()
    assert run.error_bits() == 0
    flips = total = 0
    for which, src in (("k", kt), ("v", vt)):
        bits = w.bits_k if which == "k" else w.bits_v
        codes = run.cache.codes(which)
        for pg in (0, 1, 3, 4, 6, 7):
            assert torch.all(codes[:, pg] == 0xA5)
        for layer in range(w.num_layers):
            for h in range(w.num_kv_heads):
                x = W.half_bits_to_f64(src[layer, [1, 3], :, h], w.in_dtype)      # [2, T, d]
                ora = O.quantize_tiles(x, bits, w.sinkhorn_iters, w.block)
                raw = codes[layer, [5, 2], h].cpu().numpy()
                tok = run.cache.tok_scale(which)[layer, [5, 2], h].cpu().numpy()
                ch = run.cache.chan_scale(which)[layer, [5, 2], h].cpu().numpy()
                gpu = O.QuantizedTiles(O.unpack_codes(raw, bits, w.tile_tokens, w.head_dim), tok[..., 0],
                                       tok[..., 1], ch)
                flips += compare_quantized(gpu, ora, x, bits, w.sinkhorn_iters, w.block,
                                           "%s L%d H%d" % (which, layer, h), check_rate=False).counted
                total += gpu.q.size
    assert flips <= CODE_FLIP_RATE * total, "%d tie flips in %d codes" % (flips, total)


def test_tail_entry_rejections():
    w = W.WORKLOADS["gqa"].scaled(batch=2, seq_len=256)
    run = QuantRun(w)
    dec = DecodeRun(run)
    kt = torch.zeros(1, w.batch, w.tile_tokens, w.num_kv_heads, w.head_dim, dtype=torch.int16, device="cuda")
    tl = torch.zeros(2, dtype=torch.int32, device="cuda")
    f = kvq.kvq_decode_attention_tail
    assert f(run.cfg, run.cache.view, 0, dec.q, dec.bt_d, dec.maxp, dec.sl_d, None, kt, tl, 2, dec.hq,
             w.softmax_scale, dec.out, dec.ws, dec.ws_bytes, run.err, raise_on_error=False) == kvq.KVQ_ERR_INVALID_ARG
    assert f(run.cfg, run.cache.view, 0, dec.q, dec.bt_d, dec.maxp, dec.sl_d, kt.data_ptr() + 2, kt, tl, 2, dec.hq,
             w.softmax_scale, dec.out, dec.ws, dec.ws_bytes, run.err, raise_on_error=False) == kvq.KVQ_ERR_INVALID_ARG
    g = kvq.kvq_decode_attention_fill
    assert g(run.cfg, run.cache.view, 0, dec.q, dec.bt_d, dec.maxp, dec.sl_d, kt, kt, tl, None, 2, dec.hq,
             w.softmax_scale, dec.out, dec.ws, dec.ws_bytes, run.err, raise_on_error=False) == kvq.KVQ_ERR_INVALID_ARG
    assert g(run.cfg, run.cache.view, 3, dec.q, dec.bt_d, dec.maxp, dec.sl_d, kt, kt, tl, tl, 2, dec.hq,
             w.softmax_scale, dec.out, dec.ws, dec.ws_bytes, run.err, raise_on_error=False) == kvq.KVQ_ERR_INVALID_ARG
    assert g(run.cfg, run.cache.view, 0, dec.q, dec.bt_d, dec.maxp, dec.sl_d, kt, kt, tl, tl, 2, dec.hq,
             w.softmax_scale, dec.out, dec.ws, 16, run.err, raise_on_error=False) == kvq.KVQ_ERR_WORKSPACE_TOO_SMALL
    torch.cuda.synchronize()
    assert run.error_bits() == 0                               # nothing was launched


@pytest.mark.parametrize("kw,seq_lens,lens", [(dict(batch=3, seq_len=256), [256, 0, 112], [15, 9, 0]),
                                              (dict(batch=2, seq_len=64, num_q_heads=16), [64, 32], [16, 3])])
def test_mla_decode_with_tail_parity(kw, seq_lens, lens):
    # latent and rope tail rows merged in the MLA combine; a sequence with no
    # cached page, a full tail and an empty one
    nq = kw.pop("num_q_heads", None)
    w = W.WORKLOADS["mla"].scaled(**kw)
    if nq:
        w = dataclasses.replace(w, num_q_heads=nq)
    run = QuantRun(w)
    dec = DecodeRun(run, seq_lens=seq_lens)
    o = dec.with_tail(W.tail_inputs(w, "k"), W.tail_rope_inputs(w), lens)
    assert run.error_bits() == 0
    assert np.all(np.isfinite(o))
    for b in range(dec.batch):
        err = attention_error(o[b], mla_oracle_tail(dec, b))
        assert err <= MLA_SHORT_ATTN_TOL, "seq %d: %g" % (b, err)


@pytest.mark.parametrize("name,layer", [("gqa", 0), ("gqa", 1), ("g128", 1), ("mla", 1), ("kivi", 0), ("gqa16", 1)])
def test_decode_with_fill_parity(name, layer):
    # kvq_decode_attention_fill: sequences 0 and 2 have full tails in `layer`,
    # quantised into spare pages by the call, then attention runs over the
    # cache (with those pages) and the other sequences' partial tails
    w = W.WORKLOADS[name].scaled(batch=3, seq_len=2 * W.WORKLOADS[name].tile_tokens, num_layers=2)
    T = w.tile_tokens
    run = QuantRun(w, num_pages=w.num_pages + 3)             # three spare pages past the appended ones
    bt = np.zeros((w.batch, w.tiles_per_seq + 1), dtype=np.int32)
    bt[:, :w.tiles_per_seq] = W.block_table(w)
    fill = np.array([w.num_pages + 1, -1, w.num_pages + 2], dtype=np.int32)
    seq = np.full(w.batch, w.seq_len, dtype=np.int32)
    tl = np.array([0, 5, 0], dtype=np.int32)
    for b in (0, 2):
        bt[b, w.tiles_per_seq] = fill[b]
        seq[b] += T
    dec = DecodeRun(run, seq_lens=seq, block_table=bt)
    kt = W.tail_inputs(w, "k")
    vt = W.tail_rope_inputs(w) if w.mla else W.tail_inputs(w, "v")
    dec.k_tail_bits, dec.v_tail_bits, dec.tl = kt, vt, tl
    kvq.kvq_decode_attention_fill(run.cfg, run.cache.view, layer, dec.q, dec.bt_d, dec.maxp, dec.sl_d,
                                  torch.from_numpy(kt.view(np.int16)).cuda(), torch.from_numpy(vt.view(np.int16)).cuda(),
                                  torch.from_numpy(tl).cuda(), torch.from_numpy(fill).cuda(), dec.batch, dec.hq,
                                  w.softmax_scale, dec.out, dec.ws, dec.ws_bytes, run.err)
    torch.cuda.synchronize()
    o = dec.out.cpu().numpy().astype(np.float64)
    assert run.error_bits() == 0
    from _parity import gpu_pages
    # the filled pages hold the quantised tails (oracle on the same rows)
    for b in (0, 2):
        for which in (("k",) if w.mla else ("k", "v")):
            bits = w.bits_k if which == "k" else w.bits_v
            for h in range(w.num_kv_heads):
                src = kt if which == "k" else vt
                x = W.half_bits_to_f64(src[layer, b, :, h], w.in_dtype)[None]      # [1, T, d]
                if which == "k" and w.k_per_channel:
                    ora = O.quantize_tiles_per_channel(x, bits, w.block)
                else:
                    ora = O.quantize_tiles(x, bits, w.sinkhorn_iters, w.block, meta="f16" if w.meta_f16 else "f32")
                compare_quantized(gpu_pages(run, which, layer, [fill[b]], h), ora, x, bits, w.sinkhorn_iters,
                                  w.block, "seq %d %s H%d" % (b, which, h), check_rate=False)
        if w.mla:   # the rope rows of the filled page
            rope_all = run.cache["rope"].view(w.num_layers, -1, T, w.rope_dim)
            got = rope_all[layer, int(fill[b])].cpu().view(torch.int16).numpy()
            assert np.array_equal(got, vt[layer, b].view(np.int16))
    # attention over the cache with the filled pages and the remaining tails
    for b in range(w.batch):
        if w.mla:   # 32..48-token contexts
            err = attention_error(o[b], mla_oracle_tail(dec, b, layer))
            assert err <= MLA_SHORT_ATTN_TOL, "seq %d: %g" % (b, err)
            continue
        G = dec.hq // w.num_kv_heads
        for h in range(w.num_kv_heads):
            err = attention_error(o[b, h * G:(h + 1) * G], dec.oracle_tail(b, h, layer))
            assert err <= ATTN_TOL, "seq %d kv-head %d: %g" % (b, h, err)



@pytest.mark.parametrize("name", ["gqa", "long", "g128"])
def test_decode_with_fill_of_a_first_page(name):
    # The fill's pages are read by the decode kernel as soon as its grid
    # completes: sequence 0's only page is the one being filled (its tiles
    # are the first copies of their warps), sequence 1 has no page and a
    # tail, sequence 2 two cached pages and then its filled one.
    w = W.WORKLOADS[name].scaled(batch=3, seq_len=2 * W.WORKLOADS[name].tile_tokens)
    T = w.tile_tokens
    run = QuantRun(w, num_pages=w.num_pages + 2)
    bt = np.full((w.batch, w.tiles_per_seq + 1), -1, dtype=np.int32)
    bt[:, :w.tiles_per_seq] = W.block_table(w)
    fill = np.array([w.num_pages, -1, w.num_pages + 1], dtype=np.int32)
    bt[0, 0], bt[0, 1:] = fill[0], -1
    bt[2, w.tiles_per_seq] = fill[2]
    seq = np.array([T, 0, w.seq_len + T], dtype=np.int32)
    tl = np.array([0, 7, 0], dtype=np.int32)
    dec = DecodeRun(run, seq_lens=seq, block_table=bt)
    kt, vt = W.tail_inputs(w, "k"), W.tail_inputs(w, "v")
    dec.k_tail_bits, dec.v_tail_bits, dec.tl = kt, vt, tl
    kvq.kvq_decode_attention_fill(run.cfg, run.cache.view, 0, dec.q, dec.bt_d, dec.maxp, dec.sl_d,
                                  torch.from_numpy(kt.view(np.int16)).cuda(), torch.from_numpy(vt.view(np.int16)).cuda(),
                                  torch.from_numpy(tl).cuda(), torch.from_numpy(fill).cuda(), dec.batch, dec.hq,
                                  w.softmax_scale, dec.out, dec.ws, dec.ws_bytes, run.err)
    torch.cuda.synchronize()
    o = dec.out.cpu().numpy().astype(np.float64)
    assert run.error_bits() == 0
    G = dec.hq // w.num_kv_heads
    for b in range(w.batch):
        for h in range(w.num_kv_heads):
            err = attention_error(o[b, h * G:(h + 1) * G], dec.oracle_tail(b, h, 0))
            assert err <= ATTN_TOL, "seq %d kv-head %d: %g" % (b, h, err)
