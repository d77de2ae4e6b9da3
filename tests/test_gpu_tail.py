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

from _parity import (ATTN_TOL, CODE_FLIP_RATE, DecodeRun, QuantRun, attention_error,  # noqa: E402
                     compare_quantized)


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
    m = dataclasses.replace(W.WORKLOADS["mla"].scaled(batch=1, seq_len=32))
    mrun = QuantRun(m)
    assert f(mrun.cfg, mrun.cache.view, 0, dec.q, dec.bt_d, dec.maxp, dec.sl_d, kt, kt, tl, 1, 128,
             m.softmax_scale, dec.out, dec.ws, dec.ws_bytes, run.err, raise_on_error=False) == kvq.KVQ_ERR_UNSUPPORTED
