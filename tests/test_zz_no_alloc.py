"""kvq_decode_attention_noalloc: decode attention for callers that cannot
allocate device memory when they decode (a plug-in whose host owns every
device allocation, a deployment that forbids allocation after start-up).

Its split-KV scratch is the library's own fixed array, so it must give the
same result as kvq_decode_attention with a caller workspace, call after call
(the array keeps the previous call's contents), whatever shape came before.
This file is collected last on purpose and needs nothing from the other
tests."""
import numpy as np
import pytest
import torch

from kv_cache_quantization_03_b200 import kvq, workloads as W

pytestmark = pytest.mark.gpu

from _parity import ATTN_TOL, DecodeRun, QuantRun, attention_error  # noqa: E402


def _noalloc(dec: DecodeRun):
    w = dec.run.w
    out = torch.full_like(dec.out, float("nan"))
    kvq.kvq_decode_attention_noalloc(dec.run.cfg, dec.run.cache.view, 0, dec.q, dec.bt_d, dec.maxp, dec.sl_d,
                                     dec.batch, dec.hq, w.softmax_scale, out, dec.run.err)
    torch.cuda.synchronize()
    return out.cpu().numpy().astype(np.float64)


def _same_as_workspace_entry(dec: DecodeRun):
    ref = dec()
    for _ in range(2):
        got = _noalloc(dec)
        assert np.all(np.isfinite(got))
        assert attention_error(got, ref) <= ATTN_TOL
        assert np.array_equal(got, ref)          # same kernels and split plan: bit-identical
    assert dec.run.error_bits() == 0


def test_noalloc_matches_workspace_entry_point_twice():
    w = W.WORKLOADS["gqa"].scaled(batch=3, seq_len=1024)
    _same_as_workspace_entry(DecodeRun(QuantRun(w), seq_lens=[1024, 512, 16]))


def test_noalloc_after_a_larger_call_with_more_splits():
    # a large call fills much of the array; a smaller one (fewer splits,
    # shorter sequences) must not see its leftovers
    big = W.WORKLOADS["long"].scaled(batch=2, seq_len=8192)
    _same_as_workspace_entry(DecodeRun(QuantRun(big)))
    small = W.WORKLOADS["gqa"].scaled(batch=2, seq_len=256)
    _same_as_workspace_entry(DecodeRun(QuantRun(small), seq_lens=[256, 32]))


def test_noalloc_mla_cache():
    # the MLA path also keeps its prepared queries in the scratch array
    w = W.WORKLOADS["mla"].scaled(batch=2, seq_len=256)
    _same_as_workspace_entry(DecodeRun(QuantRun(w), seq_lens=[256, 112]))


def test_noalloc_rejects_shapes_beyond_its_scratch():
    w = W.WORKLOADS["gqa"].scaled(batch=2, seq_len=256)
    run = QuantRun(w)
    dec = DecodeRun(run)
    big_batch = 4096                              # needs far more than the fixed scratch
    need = kvq.kvq_decode_workspace_bytes(run.cfg, big_batch, dec.hq, dec.maxp * w.tile_tokens)
    assert need > 8 << 20
    f = kvq.kvq_decode_attention_noalloc
    st = f(run.cfg, run.cache.view, 0, dec.q, dec.bt_d, dec.maxp, dec.sl_d, big_batch, dec.hq, w.softmax_scale,
           dec.out, run.err, raise_on_error=False)
    assert st == kvq.KVQ_ERR_WORKSPACE_TOO_SMALL
    # a bad argument is reported as such, whatever the size
    st = f(run.cfg, run.cache.view, 5, dec.q, dec.bt_d, dec.maxp, dec.sl_d, big_batch, dec.hq, w.softmax_scale,
           dec.out, run.err, raise_on_error=False)
    assert st == kvq.KVQ_ERR_INVALID_ARG            # layer outside the cache
    st = f(run.cfg, run.cache.view, 0, dec.q, dec.bt_d, dec.maxp, dec.sl_d, big_batch, dec.hq + 1,
           w.softmax_scale, dec.out, run.err, raise_on_error=False)
    assert st == kvq.KVQ_ERR_INVALID_ARG            # query heads not a multiple of the kv-heads
    torch.cuda.synchronize()
    assert run.error_bits() == 0                    # nothing was launched
