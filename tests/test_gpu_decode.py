"""GPU parity of kvq_decode_attention against the oracle run on the GPU's
stored codes and scales (tolerance 2e-3 max relative error per head)."""
import dataclasses

import numpy as np
import pytest
import torch

from kv_cache_quantization_03_b200 import kvq, workloads as W

pytestmark = pytest.mark.gpu

from _parity import ATTN_TOL, DecodeRun, QuantRun, attention_error  # noqa: E402


def _check(dec: DecodeRun, o: np.ndarray, pairs=None):
    w = dec.run.w
    G = dec.hq // w.num_kv_heads
    worst = 0.0
    pairs = [(b, h) for b in range(dec.batch) for h in range(w.num_kv_heads)] if pairs is None else pairs
    for b, h in pairs:
        ref = dec.oracle(b, h)
        got = o[b, h * G:(h + 1) * G]
        if dec.sl[b] // w.tile_tokens == 0:
            assert np.all(got == 0)
            continue
        err = attention_error(got, ref)
        worst = max(worst, err)
        assert err <= ATTN_TOL, "seq %d kv-head %d: %g" % (b, h, err)
    return worst


@pytest.mark.parametrize("name,kw", [
    ("rt1k", {}),
    ("gqa", dict(batch=3, seq_len=512)),
    ("long", dict(batch=2, seq_len=2048)),
    ("g128", dict(batch=3, seq_len=1024)),
    ("saw4", dict(batch=3, seq_len=512)),
    ("prefill", dict(seq_len=1024, num_layers=2)),   # per-channel scales over two decades
    ("gqa16", dict(batch=3, seq_len=512)),            # a, z, c as IEEE half
    ("kivi", dict(batch=3, seq_len=512)),             # keys per channel, no rotation
    ("hadonly", dict(batch=3, seq_len=512)),          # full rotation, no normalisation
])
def test_decode_parity_small(name, kw):
    w = W.WORKLOADS[name]
    w = w.scaled(**kw) if kw else w
    run = QuantRun(w)
    dec = DecodeRun(run)
    o = dec()
    assert run.error_bits() == 0
    assert np.all(np.isfinite(o))
    _check(dec, o)


def _pow2(bits: np.ndarray, dtype: str, e: int) -> np.ndarray:
    """bf16/fp16 bit patterns times the exact power of two 2^e."""
    return W._round_to((W.half_bits_to_f64(bits, dtype) * 2.0 ** e).astype(np.float32), dtype)


@pytest.mark.parametrize("kv_exp,q_exp", [(20, 0), (-20, 0), (0, 8), (0, -8), (20, -8), (-20, 8)])
@pytest.mark.parametrize("name", ["gqa", "long", "g128"])
def test_decode_parity_input_magnitudes(name, kv_exp, q_exp):
    # u = q~ c_K and w = p a_V / max(a_V) travel as f16 hi + lo pairs: the
    # result must hold when keys, values and queries are far from unit scale
    w = W.WORKLOADS[name].scaled(batch=2, seq_len=1024)
    kb = _pow2(W.kv_inputs(w, "k"), w.in_dtype, kv_exp)
    vb = _pow2(W.kv_inputs(w, "v"), w.in_dtype, -kv_exp)
    run = QuantRun(w, inputs=(kb, vb))
    dec = DecodeRun(run, q_bits=_pow2(W.queries(w), "bf16", q_exp))
    o = dec()
    assert run.error_bits() == 0
    assert np.all(np.isfinite(o))
    _check(dec, o)


@pytest.mark.parametrize("lat_exp", [12, 14, 20, -12, -8])
def test_mla_decode_parity_latent_magnitudes(lat_exp):
    # The latent tiles meet the tensor cores as f16 operands: a chunk whose
    # dequantised latent would pass the f16 range is scaled down by a power of
    # two first (and the rope keys with it), and small latents keep f16's
    # relative precision down to 2^-14.  The query's latent part is scaled the
    # other way, so the logits stay at the workload's scale: with single f16
    # operands the score carries ~2^-12 relative error, which the 2e-3
    # tolerance absorbs only while |logits| stay of order ten (log2 units).
    w = W.WORKLOADS["mla"].scaled(batch=2, seq_len=512)
    kb = _pow2(W.kv_inputs(w, "k"), w.in_dtype, lat_exp)
    run = QuantRun(w, inputs=(kb, None))
    qb = W.queries(w).copy()
    qb[..., : w.head_dim] = _pow2(qb[..., : w.head_dim], "bf16", -lat_exp)
    dec = DecodeRun(run, q_bits=qb)
    o = dec()
    assert run.error_bits() == 0
    assert np.all(np.isfinite(o))
    _check(dec, o)


@pytest.mark.parametrize("kw", [dict(batch=2, seq_len=512), dict(batch=3, seq_len=304)])
def test_mla_decode_parity(kw):
    w = W.WORKLOADS["mla"].scaled(**kw)
    run = QuantRun(w)
    dec = DecodeRun(run)
    o = dec()
    assert run.error_bits() == 0
    assert np.all(np.isfinite(o))
    _check(dec, o)


def test_mla_decode_fewer_heads_ragged():
    w = dataclasses.replace(W.WORKLOADS["mla"].scaled(batch=3, seq_len=256), num_q_heads=16)
    run = QuantRun(w)
    dec = DecodeRun(run, seq_lens=[256, 48, 0])
    o = dec()
    assert run.error_bits() == 0
    _check(dec, o)


@pytest.mark.parametrize("name,kw", [("long", dict(batch=2, seq_len=1024)), ("g128", dict(batch=3, seq_len=1024)),
                                     ("mla", dict(batch=2, seq_len=512))])
def test_decode_parity_half_metadata(name, kw):
    # the half-precision layout through both decode kernels (one and two
    # kv-heads per CTA, 128-token pages, the MLA latent)
    w = dataclasses.replace(W.WORKLOADS[name].scaled(**kw), meta_f16=True)
    run = QuantRun(w)
    dec = DecodeRun(run)
    o = dec()
    assert run.error_bits() == 0
    assert np.all(np.isfinite(o))
    _check(dec, o)


@pytest.mark.parametrize("group,bits,block,meta16", [(8, 4, 1, False), (4, 8, 128, True), (1, 2, 32, False),
                                                 (2, 4, 1, True)])
def test_decode_parity_per_channel_keys(group, bits, block, meta16):
    # KIVI-style axes through one and two kv-heads per CTA, with and without a rotation
    w = dataclasses.replace(W.WORKLOADS["kivi"].scaled(batch=2, seq_len=768), num_q_heads=8 * group, bits_k=bits,
                            bits_v=bits, hadamard_block=block, meta_f16=meta16)
    run = QuantRun(w)
    dec = DecodeRun(run, seq_lens=[768, 400 // 16 * 16])
    o = dec()
    assert run.error_bits() == 0
    _check(dec, o)


def test_decode_ragged_and_empty_sequences():
    w = W.WORKLOADS["gqa"].scaled(batch=4, seq_len=1024)
    run = QuantRun(w)
    dec = DecodeRun(run, seq_lens=[1024, 16, 0, 1008])
    o = dec()
    assert run.error_bits() == 0
    _check(dec, o)


@pytest.mark.parametrize("group,bits", [(1, (4, 4)), (2, (2, 8)), (8, (8, 2)), (8, (3, 4)), (4, (2, 2))])
def test_decode_group_sizes_and_bit_widths(group, bits):
    w = dataclasses.replace(W.WORKLOADS["gqa"].scaled(batch=2, seq_len=768), num_q_heads=8 * group,
                            bits_k=bits[0], bits_v=bits[1])
    run = QuantRun(w)
    dec = DecodeRun(run)
    _check(dec, dec())


def test_decode_long_pages_ragged_and_empty():
    # 128-token pages read as eight 16-token tiles; a split may start mid-page
    w = W.WORKLOADS["g128"].scaled(batch=4, seq_len=2048)
    run = QuantRun(w)
    dec = DecodeRun(run, seq_lens=[2048, 128, 0, 1920])
    o = dec()
    assert run.error_bits() == 0
    _check(dec, o)


@pytest.mark.parametrize("tile,group,bits", [(32, 8, (3, 4)), (64, 4, (3, 2)), (128, 1, (8, 8)), (64, 2, (2, 4))])
def test_decode_tile_lengths(tile, group, bits):
    # 3-bit keys come from the two planes of the page; one or two kv-heads per CTA
    w = dataclasses.replace(W.WORKLOADS["gqa"].scaled(batch=2, seq_len=1024), tile_tokens=tile,
                            num_q_heads=8 * group, bits_k=bits[0], bits_v=bits[1])
    run = QuantRun(w)
    dec = DecodeRun(run)
    o = dec()
    assert run.error_bits() == 0
    _check(dec, o)


@pytest.mark.parametrize("block,group,bits", [(1, 4, (4, 4)), (2, 8, (3, 4)), (4, 2, (4, 2)), (8, 4, (4, 4)),
                                             (16, 8, (3, 4)), (64, 1, (2, 2)), (32, 2, (8, 8))])
def test_decode_block_diagonal_rotation(block, group, bits):
    # query rotation and output un-rotation by blocks; one or two kv-heads per CTA
    w = dataclasses.replace(W.WORKLOADS["saw4"].scaled(batch=2, seq_len=512), hadamard_block=block,
                            num_q_heads=8 * group, bits_k=bits[0], bits_v=bits[1])
    run = QuantRun(w)
    dec = DecodeRun(run)
    o = dec()
    assert run.error_bits() == 0
    _check(dec, o)


def test_decode_long_pages_bad_page_and_partial():
    w = W.WORKLOADS["g128"].scaled(batch=2, seq_len=512)
    run = QuantRun(w)
    bt = W.block_table(w).copy()
    bt[1, 2] = w.num_pages + 3
    dec = DecodeRun(run, block_table=bt, seq_lens=[500, 512])
    o = dec()
    bits = run.error_bits()
    assert bits & 0x1 and bits & 0x2          # bad page in sequence 1, partial page in sequence 0
    assert np.all(np.isfinite(o))
    _check(dec, o, pairs=[(0, h) for h in range(w.num_kv_heads)])   # sequence 0: its three whole pages


def test_decode_bad_page_sets_error():
    w = W.WORKLOADS["gqa"].scaled(batch=2, seq_len=256)
    run = QuantRun(w)
    bt = W.block_table(w).copy()
    bt[1, 3] = w.num_pages + 5
    dec = DecodeRun(run, block_table=bt)
    o = dec()
    assert run.error_bits() & 0x1
    assert np.all(np.isfinite(o))
    _check(dec, o, pairs=[(0, h) for h in range(w.num_kv_heads)])


def test_decode_partial_tile_flag_and_host_errors():
    w = W.WORKLOADS["gqa"].scaled(batch=2, seq_len=256)
    run = QuantRun(w)
    dec = DecodeRun(run, seq_lens=[256, 250])
    o = dec()
    assert run.error_bits() & 0x2
    # host-side rejections: workspace too small, group > 8, partial append
    st = kvq.kvq_decode_attention(run.cfg, run.cache.view, 0, dec.q, dec.bt_d, dec.maxp, dec.sl_d, 2, 32,
                                  0.1, dec.out, dec.ws, 16, run.err, raise_on_error=False)
    assert st == kvq.KVQ_ERR_WORKSPACE_TOO_SMALL
    st = kvq.kvq_decode_attention(run.cfg, run.cache.view, 0, dec.q, dec.bt_d, dec.maxp, dec.sl_d, 2, 8 * 16,
                                  0.1, dec.out, dec.ws, dec.ws_bytes, run.err, raise_on_error=False)
    assert st == kvq.KVQ_ERR_UNSUPPORTED
    st = kvq.kvq_quantize_append(run.cfg, run.cache.view, run.k, run.v, None, 24, run.dst, run.err,
                                 raise_on_error=False)
    assert st == kvq.KVQ_ERR_PARTIAL_TILE


def test_decode_deterministic():
    w = W.WORKLOADS["gqa"].scaled(batch=2, seq_len=1024)
    run = QuantRun(w)
    dec = DecodeRun(run)
    a = dec()
    b = dec()
    assert np.array_equal(a, b)


def test_decode_wait_timeout_reports_and_recovers():
    # A bounded device wait that runs out (the testing hook makes every CTA
    # wait 2 ms on a flag nothing sets) raises KVQ_DEVERR_TIMEOUT, the call
    # still returns with nothing in flight, and the next call is correct.
    w = W.WORKLOADS["gqa"].scaled(batch=2, seq_len=512)
    run = QuantRun(w)
    dec = DecodeRun(run)
    kvq.kvq_set_test_wait(2_000_000)
    try:
        o = dec()
    finally:
        kvq.kvq_set_test_wait(0)
    st, bits = kvq.kvq_read_error(run.err)
    assert st == kvq.KVQ_ERR_TIMEOUT and bits & kvq.KVQ_DEVERR_TIMEOUT
    assert np.all(o == 0)
    o2 = dec()
    assert run.error_bits() == 0
    _check(dec, o2)
