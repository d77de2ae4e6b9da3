"""kvq_decode_attention_noalloc: decode attention for callers that cannot
allocate device memory when they decode (a plug-in whose host owns every
device allocation, a deployment that forbids allocation after start-up).

Its split-KV scratch is the library's own fixed array, so it must give the
same result as kvq_decode_attention with a caller workspace, call after call
(the array keeps the previous call's contents).  This file is collected last
on purpose and needs nothing from the other tests.
"""
import numpy as np
import pytest
import torch

from kv_cache_quantization_03_b200 import kvq, workloads as W

pytestmark = pytest.mark.gpu

from _parity import ATTN_TOL, DecodeRun, QuantRun, attention_error  # noqa: E402


def _noalloc(dec: DecodeRun, out):
    w = dec.run.w
    kvq.kvq_decode_attention_noalloc(dec.run.cfg, dec.run.cache.view, 0, dec.q, dec.bt_d, dec.maxp, dec.sl_d,
                                     dec.batch, dec.hq, w.softmax_scale, out, dec.run.err)
    torch.cuda.synchronize()
    return out.cpu().numpy().astype(np.float64)


def test_noalloc_matches_workspace_entry_point_twice():
    w = W.WORKLOADS["gqa"].scaled(batch=3, seq_len=1024)
    run = QuantRun(w)
    dec = DecodeRun(run, seq_lens=[1024, 512, 16])
    ref = dec()
    for _ in range(2):
        out = torch.full_like(dec.out, float("nan"))
        got = _noalloc(dec, out)
        assert np.all(np.isfinite(got))
        assert attention_error(got, ref) <= ATTN_TOL
        assert np.array_equal(got, ref)          # same kernels and split plan: bit-identical
    assert run.error_bits() == 0


def test_noalloc_rejects_shapes_beyond_its_scratch():
    w = W.WORKLOADS["gqa"].scaled(batch=2, seq_len=256)
    run = QuantRun(w)
    dec = DecodeRun(run)
    big_batch = 4096                              # needs far more than the fixed scratch
    need = kvq.kvq_decode_workspace_bytes(run.cfg, big_batch, dec.hq, dec.maxp * w.tile_tokens)
    assert need > 8 << 20
    st = kvq.kvq_decode_attention_noalloc(run.cfg, run.cache.view, 0, dec.q, dec.bt_d, dec.maxp, dec.sl_d,
                                          big_batch, dec.hq, w.softmax_scale, dec.out, run.err,
                                          raise_on_error=False)
    assert st == kvq.KVQ_ERR_WORKSPACE_TOO_SMALL
