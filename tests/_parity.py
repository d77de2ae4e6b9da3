"""Helpers of the parity tests: run the CUDA path through the C ABI, run the
float64 oracle on the same seeded inputs, compare with the stated tolerances.

Tolerances (readings as stated in the oracle's header):
* codes: identical, except +-1 flips where the oracle's (y - m) / s lies within
  1e-4 of a half-integer (a rounding tie the float32 kernel may resolve the
  other way); such flips on at most 1e-5 of the elements, not counting flips
  at exact ties, where both codes are equally near and either is acceptable.
  A tie is exact when (y - m) / s is a half-integer in real arithmetic; that
  is decided with integer arithmetic on the (dyadic) input values, and can
  only happen without normalisation rounds (with them y involves square
  roots).  Counted flips and exact ties are reported separately;
* a, z, c: |gpu - oracle| <= 1e-6 |oracle| (purely relative, so it holds at
  any magnitude; a zero must be an exact zero); with half-precision metadata
  the stored half must equal the oracle's, or be its neighbour where the
  oracle's float64 value lies within 1e-6 (relative) of the midpoint between
  the two (the kernel rounds its float32 value, the oracle the exact one);
* attention: per (sequence, head) max_j |o_j - o'_j| / max_j |o'_j| <= 2e-3,
  with the oracle run on the GPU's stored codes and scales.
"""
from __future__ import annotations

import math
from fractions import Fraction
from typing import NamedTuple

import numpy as np
import torch

from kv_cache_quantization_03_b200 import kvq, workloads as W
from kv_cache_quantization_03_b200.cache import QuantizedCache
from oracle import kvarn_oracle as O

CODE_TIE_BAND = 1e-4
CODE_FLIP_RATE = 1e-5
SCALE_RTOL = 1e-6
ATTN_TOL = 2e-3
# MLA decode on short contexts (tens of tokens, outside the MLA workload):
# its 128-head contraction runs on single-f16 operands, and the query's f16
# rounding shifts every token's score the same way, so it does not average
# out over a few tokens.  A CPU emulation of that rounding (f16 query, f16
# latent chunk, f16 P, fp32 accumulation) on 32..256-token contexts of the
# mla distribution gives up to 2.7e-3 max relative error over 128 heads
# (1.65e-3 at 4096 tokens; 5.9e-4 with an exact query).  The MLA workload
# itself is checked at ATTN_TOL.
MLA_SHORT_ATTN_TOL = 3.5e-3


def config_for(w: W.Workload, num_pages=None) -> kvq.kvq_config:
    return kvq.make_config(head_dim=w.head_dim, num_kv_heads=w.num_kv_heads, tile_tokens=w.tile_tokens,
                           bits_k=w.bits_k, bits_v=w.bits_v, sinkhorn_iters=w.sinkhorn_iters, mla=w.mla,
                           rope_dim=w.rope_dim, num_layers=w.num_layers,
                           num_pages=w.num_pages if num_pages is None else num_pages, in_dtype=w.in_dtype,
                           hadamard_block=w.hadamard_block or None, meta_f16=w.meta_f16,
                           k_per_channel=w.k_per_channel)


class QuantRun:
    """Inputs of a workload on the GPU, quantised into a fresh cache."""

    def __init__(self, w: W.Workload, quantize=True, inputs=None, pages=None, num_pages=None):
        self.w = w
        self.cfg = config_for(w, num_pages)
        self.cache = QuantizedCache(self.cfg)
        if inputs is None:
            self.k_bits = W.kv_inputs(w, "k")
            self.v_bits = None if w.mla else W.kv_inputs(w, "v")
        else:
            self.k_bits, self.v_bits = inputs
        self.pages = W.page_assignment(w) if pages is None else np.asarray(pages, dtype=np.int32)
        self.k = torch.from_numpy(self.k_bits.view(np.int16)).cuda()
        self.v = None if w.mla else torch.from_numpy(self.v_bits.view(np.int16)).cuda()
        self.rope_bits = W.rope_inputs(w) if (w.mla and w.rope_dim) else None
        self.rope = None if self.rope_bits is None else torch.from_numpy(self.rope_bits.view(np.int16)).cuda()
        self.dst = torch.from_numpy(self.pages).cuda()
        self.err = torch.zeros(1, dtype=torch.int32, device="cuda")
        if quantize:
            self.quantize()

    def quantize(self):
        kvq.kvq_quantize_append(self.cfg, self.cache.view, self.k, self.v, self.rope, self.w.n_tok, self.dst,
                                self.err)
        torch.cuda.synchronize()

    def error_bits(self):
        st, bits = kvq.kvq_read_error(self.err)
        return bits

    def gpu_tiles(self, which: str, layer: int, tiles, head: int):
        """Stored codes (unpacked with the oracle's unpack) and scales of tiles (append order)."""
        return gpu_pages(self, which, layer, self.pages[np.asarray(tiles)], head)

    def input_tiles(self, which: str, layer: int, tiles, head: int) -> np.ndarray:
        w = self.w
        src = self.k_bits if which == "k" else self.v_bits
        idx = (np.asarray(tiles)[:, None] * w.tile_tokens + np.arange(w.tile_tokens)[None, :])
        return W.half_bits_to_f64(src[layer, idx, head, :], w.in_dtype)   # [n, T, d]


def oracle_fraction(x: np.ndarray, bits: int, n_iter: int, block=None, per_channel=False) -> np.ndarray:
    """The oracle's (y - m) / s of every element (to locate rounding ties);
    the groups are token rows, or channels with per_channel."""
    y, _, _ = O.sinkhorn_normalize(O.rotate(x, block), n_iter)
    ax = -2 if per_channel else -1
    m = y.min(ax, keepdims=True)
    s = (y.max(ax, keepdims=True) - m) / ((1 << bits) - 1)
    return (y - m) / np.where(s > 0, s, 1.0)


def exact_half_ties(x: np.ndarray, bits: int, n_iter: int, block, idx, per_channel=False) -> np.ndarray:
    """Whether the codes at idx (index arrays into tiles x: [n, T, d]) sit at
    an exact rounding tie: (y - m) / s a half-integer in real arithmetic.

    With normalisation rounds y carries square roots of sums of squares, so
    an exact tie has probability zero and none is granted.  Without them y is
    x H / sqrt(b), and (y - m) / s = (2^bits - 1) (y - m) / (max - m), in
    which the 1/sqrt(b) cancels: with the inputs scaled to integers (they are
    dyadic), the test is integer arithmetic on x H."""
    n = len(idx[0])
    if n_iter > 0 or n == 0:
        return np.zeros(n, dtype=bool)
    d = x.shape[-1]
    h = O.block_hadamard_matrix(d, block or d).astype(object)
    qmax = (1 << bits) - 1
    tiles = {}
    out = np.zeros(n, dtype=bool)
    for e, (i, t, j) in enumerate(zip(*idx)):
        if i not in tiles:   # the whole tile, exactly: den * sqrt(b) * y as integers
            fr = [[Fraction(float(v)) for v in row] for row in x[i]]
            den = max(f.denominator for row in fr for f in row)   # a power of two
            ints = np.array([[f.numerator * (den // f.denominator) for f in row] for row in fr], dtype=object)
            tiles[i] = ints.dot(h)
        y = tiles[i]
        grp = y[:, j] if per_channel else y[t, :]        # the RTN group of the element
        lo, hi = min(grp), max(grp)
        if hi == lo:
            continue
        num = 2 * qmax * (y[t, j] - lo)                    # 2 (y - m) / s = num / (hi - lo)
        out[e] = num % (hi - lo) == 0 and (num // (hi - lo)) % 2 == 1
    return out


class Flips(NamedTuple):
    counted: int      # flips that count toward the 1e-5 rate
    exact_ties: int   # flips at exact ties (both codes correct)


def compare_quantized(gpu, ora, x: np.ndarray, bits: int, n_iter: int, block=None, label="",
                      check_rate=True) -> Flips:
    """Asserts the code and scale tolerances of quantised tiles against the
    oracle's on the same inputs x: [n, T, d]; returns the flip counts.

    With check_rate=False the caller aggregates the counted flips over
    several comparisons and checks the 1e-5 rate itself."""
    per_channel = isinstance(ora, O.ChannelQuantizedTiles)
    diff = gpu.q != ora.q
    counted = ties = 0
    if diff.any():
        assert np.all(np.abs(gpu.q[diff] - ora.q[diff]) == 1), label + ": code off by more than 1"
        frac = oracle_fraction(x, bits, n_iter, block, per_channel)
        f = frac[diff]
        dist = np.abs(f - np.floor(f) - 0.5)
        assert np.all(dist <= CODE_TIE_BAND), "%s: flip away from a tie (distance %g)" % (label, dist.max())
        exact = exact_half_ties(x, bits, n_iter, block, np.nonzero(diff), per_channel)
        ties = int(exact.sum())
        counted = int(diff.sum()) - ties
    if check_rate:
        assert counted <= CODE_FLIP_RATE * gpu.q.size, "%s: %d flips in %d codes" % (label, counted, gpu.q.size)
    if per_channel:   # the per-channel step and minimum
        for name in ("s", "m"):
            g = getattr(gpu, name).astype(np.float64)
            o = getattr(ora, name).astype(np.float64)
            tol = (2.0 ** -10 if np.asarray(getattr(gpu, name)).dtype == np.float16 else SCALE_RTOL) * np.abs(o)
            assert np.all(np.abs(g - o) <= tol), "%s: %s off by %g relative" % (
                label, name, float(np.max(np.abs(g - o) / np.maximum(np.abs(o), 1e-300))))
        return Flips(counted, ties)
    if np.asarray(gpu.a).dtype == np.float16:
        _, a64, z64, c64 = O.quantize_stages(x, bits, n_iter, block)
        for name, exact in (("a", a64), ("z", z64), ("c", c64)):
            g16, o16 = np.asarray(getattr(gpu, name), np.float16), np.asarray(getattr(ora, name), np.float16)
            g, o = g16.astype(np.float64), o16.astype(np.float64)
            gb, ob = g16.view(np.uint16).astype(np.int64), o16.view(np.uint16).astype(np.int64)
            neighbour = (np.abs(gb - ob) == 1) & ((gb ^ ob) & 0x8000 == 0)
            at_mid = np.abs(exact - (g + o) / 2) <= SCALE_RTOL * np.abs(exact)
            ok = (gb == ob) | (neighbour & at_mid)
            assert np.all(ok), "%s: half %s differs from the oracle's (%d values)" % (label, name, int((~ok).sum()))
        return Flips(counted, ties)
    for name in ("a", "z", "c"):
        g = getattr(gpu, name).astype(np.float64)
        o = getattr(ora, name).astype(np.float64)
        err = np.abs(g - o) - SCALE_RTOL * np.abs(o)
        assert np.all(err <= 0), "%s: %s off by %g relative" % (
            label, name, float(np.max(np.abs(g - o) / np.maximum(np.abs(o), 1e-300))))
    return Flips(counted, ties)


def check_tiles(run, which: str, layer: int, tiles, head: int, label="", check_rate=False) -> Flips:
    """Oracle against the GPU's stored tiles of one (layer, kv-head, K/V)."""
    w = run.w
    bits = w.bits_k if which == "k" else w.bits_v
    x = run.input_tiles(which, layer, tiles, head)
    if which == "k" and w.k_per_channel:
        ora = O.quantize_tiles_per_channel(x, bits, w.block)
    else:
        ora = O.quantize_tiles(x, bits, w.sinkhorn_iters, w.block, meta="f16" if w.meta_f16 else "f32")
    gpu = run.gpu_tiles(which, layer, tiles, head)
    return compare_quantized(gpu, ora, x, bits, w.sinkhorn_iters, w.block, label, check_rate)


def attention_error(o_gpu: np.ndarray, o_ref: np.ndarray) -> float:
    """max over heads of max_j |o - o'| / max_j |o'|."""
    num = np.max(np.abs(o_gpu - o_ref), axis=-1)
    den = np.maximum(np.max(np.abs(o_ref), axis=-1), 1e-30)
    return float(np.max(num / den))


def seq_tiles(w: W.Workload, b: int) -> np.ndarray:
    return b * w.tiles_per_seq + np.arange(w.tiles_per_seq)


def gpu_pages(run: QuantRun, which: str, layer: int, pages, head: int):
    """Stored tiles of the given physical pages (unpacked with the oracle)."""
    w = run.w
    bits = w.bits_k if which == "k" else w.bits_v
    pg = torch.as_tensor(np.asarray(pages, dtype=np.int64)).cuda()
    raw = run.cache.codes(which)[layer, pg, head].cpu().numpy()
    tok = run.cache.tok_scale(which)[layer, pg, head].cpu().numpy()
    q = O.unpack_codes(raw, bits, w.tile_tokens, w.head_dim)
    if which == "k" and w.k_per_channel:       # (s, m) per channel
        return O.ChannelQuantizedTiles(q=q, s=tok[..., 0], m=tok[..., 1])
    ch = run.cache.chan_scale(which)[layer, pg, head].cpu().numpy()
    return O.QuantizedTiles(q=q, a=tok[..., 0], z=tok[..., 1], c=ch)


class DecodeRun:
    """One decode step through kvq_decode_attention on a quantised cache."""

    def __init__(self, run: QuantRun, q_bits=None, seq_lens=None, block_table=None, num_q_heads=None):
        w = run.w
        self.run = run
        self.hq = w.num_q_heads if num_q_heads is None else num_q_heads
        self.q_bits = W.queries(w) if q_bits is None else q_bits
        self.bt = W.block_table(w) if block_table is None else np.asarray(block_table, dtype=np.int32)
        self.sl = W.seq_lens(w) if seq_lens is None else np.asarray(seq_lens, dtype=np.int32)
        self.batch = self.sl.shape[0]
        self.maxp = self.bt.shape[1]
        self.q = torch.from_numpy(self.q_bits.view(np.int16)).cuda()
        self.bt_d = torch.from_numpy(np.ascontiguousarray(self.bt)).cuda()
        self.sl_d = torch.from_numpy(self.sl).cuda()
        self.out = torch.full((self.batch, self.hq, w.head_dim), float("nan"), device="cuda")
        self.ws_bytes = kvq.kvq_decode_workspace_bytes(run.cfg, self.batch, self.hq, self.maxp * w.tile_tokens)
        self.ws = torch.empty(max(self.ws_bytes, 256), dtype=torch.uint8, device="cuda")

    def __call__(self):
        w = self.run.w
        kvq.kvq_decode_attention(self.run.cfg, self.run.cache.view, 0, self.q, self.bt_d, self.maxp, self.sl_d,
                                 self.batch, self.hq, w.softmax_scale, self.out, self.ws, self.ws_bytes,
                                 self.run.err)
        torch.cuda.synchronize()
        return self.out.cpu().numpy().astype(np.float64)

    def with_tail(self, k_tail_bits, v_tail_bits, tail_lens, layer=0):
        """kvq_decode_attention_tail with the given tail buffers; returns the output."""
        w = self.run.w
        self.k_tail_bits, self.v_tail_bits = k_tail_bits, v_tail_bits
        self.tl = np.asarray(tail_lens, dtype=np.int32)
        kt = torch.from_numpy(k_tail_bits.view(np.int16)).cuda()
        vt = torch.from_numpy(v_tail_bits.view(np.int16)).cuda()
        tl = torch.from_numpy(self.tl).cuda()
        kvq.kvq_decode_attention_tail(self.run.cfg, self.run.cache.view, layer, self.q, self.bt_d, self.maxp,
                                      self.sl_d, kt, vt, tl, self.batch, self.hq, w.softmax_scale, self.out,
                                      self.ws, self.ws_bytes, self.run.err)
        torch.cuda.synchronize()
        return self.out.cpu().numpy().astype(np.float64)

    def oracle_tail(self, b: int, kvh: int, layer=0, tail_len=None) -> np.ndarray:
        """Oracle output with the tail rows of (layer, sequence b, kv-head kvh): [G, d]."""
        w = self.run.w
        G = self.hq // w.num_kv_heads
        n = int(self.sl[b]) // w.tile_tokens
        L = int(self.tl[b]) if tail_len is None else tail_len
        q = W.half_bits_to_f64(self.q_bits[b, kvh * G:(kvh + 1) * G], "bf16")
        kt = W.half_bits_to_f64(self.k_tail_bits[layer, b, :L, kvh], w.in_dtype)
        vt = W.half_bits_to_f64(self.v_tail_bits[layer, b, :L, kvh], w.in_dtype)
        k = v = None
        if n:
            pages = self.bt[b, :n]
            k = gpu_pages(self.run, "k", layer, pages, kvh)
            v = gpu_pages(self.run, "v", layer, pages, kvh)
        return O.decode_attention_with_tail(q, k, v, kt, vt, w.softmax_scale, block=w.block)

    def oracle(self, b: int, kvh: int) -> np.ndarray:
        """Oracle output of the query heads of (sequence b, kv-head kvh): [G, d]."""
        w = self.run.w
        G = self.hq // w.num_kv_heads
        n = int(self.sl[b]) // w.tile_tokens
        if w.mla:
            q = W.half_bits_to_f64(self.q_bits[b], "bf16")
            if n == 0:
                return np.zeros((G, w.head_dim))
            pages = self.bt[b, :n]
            lat = gpu_pages(self.run, "k", 0, pages, 0)
            rope_all = self.run.cache["rope"].view(w.num_layers, -1, w.tile_tokens, w.rope_dim)
            pg = torch.as_tensor(np.asarray(pages, dtype=np.int64)).cuda()
            rope = rope_all[0, pg].float().cpu().numpy().astype(np.float64).reshape(-1, w.rope_dim)
            return O.mla_decode_attention(q, lat, rope, w.softmax_scale)
        q = W.half_bits_to_f64(self.q_bits[b, kvh * G:(kvh + 1) * G], "bf16")
        if n == 0:
            return np.zeros((G, w.head_dim))
        pages = self.bt[b, :n]
        kt = gpu_pages(self.run, "k", 0, pages, kvh)
        vt = gpu_pages(self.run, "v", 0, pages, kvh)
        return O.decode_attention(q, kt, vt, w.softmax_scale, block=w.block)


def mla_oracle_tail(dec: "DecodeRun", b: int, layer=0) -> np.ndarray:
    """Oracle MLA attention of sequence b over its cached pages (the GPU's
    stored latents and rope rows) and its unquantised tail (dec.tl[b] rows of
    dec.k_tail_bits / dec.v_tail_bits)."""
    w = dec.run.w
    n = int(dec.sl[b]) // w.tile_tokens
    L = int(dec.tl[b])
    q = W.half_bits_to_f64(dec.q_bits[b], "bf16")
    lt = W.half_bits_to_f64(dec.k_tail_bits[layer, b, :L].reshape(L, w.head_dim), w.in_dtype)
    rt = W.half_bits_to_f64(dec.v_tail_bits[layer, b, :L], "bf16")
    lat = rope = None
    if n:
        pages = dec.bt[b, :n]
        lat = gpu_pages(dec.run, "k", layer, pages, 0)
        rope_all = dec.run.cache["rope"].view(w.num_layers, -1, w.tile_tokens, w.rope_dim)
        pg = torch.as_tensor(np.asarray(pages, dtype=np.int64)).cuda()
        rope = rope_all[layer, pg].float().cpu().numpy().astype(np.float64).reshape(-1, w.rope_dim)
    return O.mla_decode_attention_with_tail(q, lat, rope, lt, rt, w.softmax_scale)
