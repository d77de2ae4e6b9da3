"""The C ABI under CUDA graph capture: a quantize-append and a decode step
captured once and replayed give bit-identical caches and outputs to the same
calls made eagerly.  Every entry point is asynchronous on the caller's stream
and never synchronises, so a serving loop can replay a captured step instead
of paying the host-side launch cost per kernel."""
import numpy as np
import pytest
import torch

from kv_cache_quantization_03_b200 import kvq, workloads as W
from kv_cache_quantization_03_b200.cache import NAMES

pytestmark = pytest.mark.gpu

from _parity import DecodeRun, QuantRun  # noqa: E402


def _arrays(run):
    return {n: run.cache[n].clone() for n in NAMES if run.cache[n] is not None}


def _step(run, dec):
    w = run.w
    kvq.kvq_quantize_append(run.cfg, run.cache.view, run.k, run.v, run.rope, w.n_tok, run.dst, run.err)
    kvq.kvq_decode_attention(run.cfg, run.cache.view, 0, dec.q, dec.bt_d, dec.maxp, dec.sl_d, dec.batch, dec.hq,
                             w.softmax_scale, dec.out, dec.ws, dec.ws_bytes, run.err)


@pytest.mark.parametrize("name,kw", [
    ("rt1k", {}),
    ("gqa", dict(batch=3, seq_len=512)),
    ("long", dict(batch=2, seq_len=1024)),
    ("g128", dict(batch=2, seq_len=512)),
    ("mla", dict(batch=2, seq_len=256)),
])
def test_graph_replay_matches_eager(name, kw):
    w = W.WORKLOADS[name]
    w = w.scaled(**kw) if kw else w
    eager = QuantRun(w)
    dec = DecodeRun(eager)
    o_eager = dec()
    ref = _arrays(eager)
    assert eager.error_bits() == 0

    run = QuantRun(w, quantize=False)   # a fresh, zeroed cache
    dg = DecodeRun(run)
    g = torch.cuda.CUDAGraph()
    cap = torch.cuda.Stream()
    cap.wait_stream(torch.cuda.current_stream())
    with torch.cuda.graph(g, stream=cap, capture_error_mode="relaxed"):
        _step(run, dg)                   # recorded, not run
    torch.cuda.synchronize()
    assert all(int(run.cache[n].view(torch.uint8).count_nonzero()) == 0 for n in ref)
    for _ in range(3):                   # a replayed step is idempotent
        dg.out.fill_(float("nan"))
        g.replay()
        torch.cuda.synchronize()
        for n, a in ref.items():
            assert torch.equal(run.cache[n].view(torch.uint8), a.view(torch.uint8)), n
        assert np.array_equal(dg.out.cpu().numpy().astype(np.float64), o_eager)
    assert run.error_bits() == 0
    del g
