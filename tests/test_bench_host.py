"""Host logic of bench.py that needs no GPU: the byte counts behind the
reported bandwidths, the decode-with-fill state, and the traffic lookup."""
import dataclasses
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from kv_cache_quantization_03_b200 import workloads as W  # noqa: E402


def test_algorithmic_bytes_match_the_cache_layout():
    # gqa at 4/4 bits: per row 256 B in, 64 B of codes + 8 B of (a, z) + 512 / 16 B of c out; decode
    # reads 208 B per token per kv-head plus the queries and outputs
    w = W.WORKLOADS["gqa"]
    q, d = bench.algorithmic_bytes(w)
    rows = w.n_tok * w.num_kv_heads
    assert q == rows * 2 * 256 + rows * 2 * (64 + 8 + 32)
    assert d == w.batch * w.seq_len * w.num_kv_heads * 208 + w.batch * w.num_q_heads * 128 * 6
    # half metadata halves (a, z) and c: 168 B per token per kv-head
    w16 = W.WORKLOADS["gqa16"]
    _, d16 = bench.algorithmic_bytes(w16)
    assert d16 == w16.batch * w16.seq_len * w16.num_kv_heads * 168 + w16.batch * w16.num_q_heads * 128 * 6
    # per-channel keys: codes + (s, m) per channel of a 16-token tile
    wk = W.WORKLOADS["kivi"]
    _, dk = bench.algorithmic_bytes(wk)
    k_row = 128 * 2 / 8 + 128 * 2 * 4 / 16
    v_row = 128 * 2 / 8 + 8 + 128 * 4 / 16
    assert dk == wk.batch * wk.seq_len * wk.num_kv_heads * (k_row + v_row) + wk.batch * wk.num_q_heads * 128 * 6


def test_fill_state_marks_every_sixteenth_sequence():
    w = dataclasses.replace(W.WORKLOADS["gqa"], batch=40, seq_len=64)
    tl, fill = bench.fill_state(w)
    bt = W.block_table(w)
    assert tl.dtype == np.int32 and fill.dtype == np.int32
    for b in range(w.batch):
        if b % 16 == 0:
            assert tl[b] == 0 and fill[b] == bt[b, w.tiles_per_seq - 1]
        else:
            assert fill[b] == -1 and 0 <= tl[b] < w.tile_tokens
    assert np.array_equal(tl[np.arange(w.batch) % 16 != 0], W.tail_lens(w)[np.arange(w.batch) % 16 != 0])


def test_fill_bytes_count_the_filled_pages_and_the_tails():
    w = W.WORKLOADS["gqa"]
    # one filled 16-token page: 16 rows x 8 kv-heads of K and V in (256 B each) and out (104 B each);
    # 10 tail tokens read as K and V rows
    assert bench.fill_bytes(w, 1, 10) == 16 * 8 * (2 * 256 + 2 * 104) + 10 * 8 * 2 * 256
    assert bench.fill_bytes(w, 0, 0) == 0
    m = W.WORKLOADS["mla"]
    lat_row = 512 * 4 / 8 + 8 + 512 * 4 / 16
    assert bench.fill_bytes(m, 1, 0) == 16 * (1024 + 128 + lat_row + 128)


def test_traffic_lookup_needs_the_matching_source_hash(tmp_path, monkeypatch):
    prof = tmp_path / "profiles"
    src = tmp_path / "kv_cache_quantization_03_b200" / "csrc"
    prof.mkdir()
    src.mkdir(parents=True)
    (src / "k.cu").write_text("kernel source\n")
    import hashlib
    sha = hashlib.sha256(b"kernel source\n").hexdigest()[:16]
    (prof / "p.md").write_text("traffic_bytes_per_call: 12345 source_sha256_16: %s\n" % sha)
    (prof / "q.md").write_text("traffic_bytes_per_call: 12345 source_sha256_16: 0000000000000000\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.traffic_from_profile("k.cu", "p.md") == 12345.0
    assert bench.traffic_from_profile("k.cu", "q.md") is None      # the kernel changed since the capture
    assert bench.traffic_from_profile("k.cu", "missing.md") is None



def test_algorithmic_bytes_of_the_benched_configs():
    # the totals behind the reported bandwidths, from the per-row byte counts of the cache format
    lng = W.WORKLOADS["long"]          # 3-bit K: 48 B codes + 8 B (a, z) + 32 B of c; 4-bit V: 64 + 8 + 32
    q, d = bench.algorithmic_bytes(lng)
    rows = lng.n_tok * lng.num_kv_heads
    assert q == rows * 2 * 256 + rows * (88 + 104) == 2952790016
    assert d == lng.batch * lng.seq_len * 8 * 192 + lng.batch * 64 * 128 * 6 == 805502976
    mla = W.WORKLOADS["mla"]           # latent 256 B codes + 8 B (a, z) + 128 B of c, rope 128 B in and out
    q, d = bench.algorithmic_bytes(mla)
    assert q == mla.n_tok * (1024 + 128) + mla.n_tok * (392 + 128) == 3506438144
    assert d == mla.batch * mla.seq_len * 520 + mla.batch * 128 * (576 * 2 + 512 * 4) == 1116733440
    g = W.WORKLOADS["g128"]            # 128-token pages: 4-bit K 64 + 8 + 4, 2-bit V 32 + 8 + 4 = 120 B
    q, d = bench.algorithmic_bytes(g)
    rows = g.n_tok * g.num_kv_heads
    assert q == rows * 2 * 256 + rows * 120
    assert d == g.batch * g.seq_len * 8 * 120 + g.batch * 32 * 128 * 6
