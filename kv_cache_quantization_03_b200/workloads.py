"""Seeded synthetic workloads for KVarN-style KV-cache quantization.

This module only draws random numbers and lays out buffers.  It holds none of
the method's arithmetic (no rotation, normalisation, quantisation or
attention), so both the CUDA path and the float64 oracle can be fed from it
without sharing any code that computes a result.

The five workloads mirror the shapes the KVarN pages talk about (the open-radar
project page "KVarN", Key Features; the 16K burst and the MLA capacity claims)
with synthetic data in place of the model activations the pages use:

=====  ==================================================================
name   shape and distribution
=====  ==================================================================
rt1k   1 seq x 1024 tok, H_kv = H_q = 1, d = 128, fp16 N(0,1) with channels
       3, 17, 64, 101 scaled x20 (before the cast); 4/4-bit, 4 iterations
gqa    32 seq x 8192 tok, H_kv = 8, H_q = 32, d = 128, bf16 N(0,1) plus
       round(0.02*128) = 3 outlier channels x15 per kv-head; 4/4-bit
long   4 seq x 131072 tok, H_kv = 8, H_q = 64, d = 128; K Student-t(nu=4),
       V N(0,1), bf16; 3-bit K, 4-bit V, 6 iterations
prefill 16384 tok x 32 layers x 8 kv-heads, d = 128, bf16 N(0,1) times a
       per-(layer, head, channel) scale log-uniform in [0.1, 10]; 4-bit
mla    64 seq x 32768 tok, latent 512 (4-bit) + rope 64 (bf16), 128
       absorbed query heads, bf16 N(0,1) latents with round(0.01*512) = 5
       outlier dims x25
g128   the shipped preset kvarn_k4v2_g128 on the gqa shapes and
       distribution: 4-bit K, 2-bit V, 128-token tiles (= pages)
gqa16  gqa (same seed and inputs) with a, z, c stored as IEEE half
kivi   ablation on gqa's inputs: KIVI-style axes (keys per channel, values
       per token), 2-bit codes, no rotation, no normalisation
saw4   ablation on the gqa shapes and distribution: block-diagonal
       Hadamard (32-channel blocks) and per-token INT4, no normalisation
=====  ==================================================================

All draws use numpy's PCG64 with the seed of the workload; the values are
cast to bf16/fp16 with round-to-nearest-even.
"""
from __future__ import annotations

import dataclasses
import math
import os
from concurrent.futures import ThreadPoolExecutor
from typing import Dict, Optional

import numpy as np


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    batch: int            # sequences
    seq_len: int          # tokens per sequence (multiple of tile_tokens)
    num_kv_heads: int
    num_q_heads: int
    head_dim: int         # d (MLA: latent width)
    bits_k: int
    bits_v: int
    sinkhorn_iters: int
    seed: int
    in_dtype: str = "bf16"          # "bf16" or "fp16"
    tile_tokens: int = 16
    num_layers: int = 1
    mla: bool = False
    rope_dim: int = 0
    hadamard_block: int = 0         # channels per block of a block-diagonal rotation; 0 = full head_dim
    meta_f16: bool = False          # a, z, c stored as IEEE half (the compact layout)
    k_per_channel: bool = False     # keys quantised per channel (the KIVI-style axes ablation)
    description: str = ""

    @property
    def block(self) -> Optional[int]:
        """The rotation's block for the oracle (None = full width)."""
        return self.hadamard_block or None

    @property
    def group(self) -> int:
        return self.num_q_heads // self.num_kv_heads

    @property
    def n_tok(self) -> int:
        """Tokens appended in one quantize-append call (all sequences)."""
        return self.batch * self.seq_len

    @property
    def tiles_per_seq(self) -> int:
        return self.seq_len // self.tile_tokens

    @property
    def num_pages(self) -> int:
        return self.batch * self.tiles_per_seq

    @property
    def softmax_scale(self) -> float:
        dot = self.head_dim + (self.rope_dim if self.mla else 0)
        return 1.0 / math.sqrt(dot)

    def scaled(self, batch: Optional[int] = None, seq_len: Optional[int] = None,
               num_layers: Optional[int] = None, name: Optional[str] = None) -> "Workload":
        """Same distribution and format at a smaller size (parity cases)."""
        return dataclasses.replace(
            self, batch=batch or self.batch, seq_len=seq_len or self.seq_len,
            num_layers=num_layers or self.num_layers, name=name or self.name + "-small")


WORKLOADS: Dict[str, Workload] = {
    "rt1k": Workload("rt1k", 1, 1024, 1, 1, 128, 4, 4, 4, 0, in_dtype="fp16",
                     description="round trip + decode, 1 x 1024 tokens, 1 head, fp16"),
    "gqa": Workload("gqa", 32, 8192, 8, 32, 128, 4, 4, 4, 2,
                    description="Llama-3-8B-shaped GQA decode, one layer, 32 x 8192 ctx"),
    "long": Workload("long", 4, 131072, 8, 64, 128, 3, 4, 6, 3,
                     description="long-context decode, 4 x 131072 ctx, K3/V4"),
    "prefill": Workload("prefill", 1, 16384, 8, 8, 128, 4, 4, 4, 4, num_layers=32,
                        description="prefill append, 16384 tokens x 32 layers x 8 kv-heads"),
    "mla": Workload("mla", 64, 32768, 1, 128, 512, 4, 4, 4, 5, mla=True, rope_dim=64,
                    description="MLA latent cache, 64 x 32768 ctx, latent 512 + rope 64"),
    "g128": Workload("g128", 32, 8192, 8, 32, 128, 4, 2, 4, 6, tile_tokens=128,
                     description="preset kvarn_k4v2_g128 (4-bit K, 2-bit V, 128-token pages), gqa shapes"),
    "saw4": Workload("saw4", 32, 8192, 8, 32, 128, 4, 4, 0, 9, hadamard_block=32,
                     description="ablation: block-diagonal Hadamard (32-channel blocks) + per-token INT4, "
                                 "no normalisation rounds, gqa shapes"),
    "gqa16": Workload("gqa16", 32, 8192, 8, 32, 128, 4, 4, 4, 2, meta_f16=True,
                      description="gqa with the compact layout: a, z, c as IEEE half (same inputs as gqa)"),
    "hadonly": Workload("hadonly", 32, 8192, 8, 32, 128, 4, 4, 0, 2,
                        description="ablation: full Hadamard rotation + per-token 4-bit RTN, no normalisation "
                                    "(same inputs as gqa)"),
    "kivi": Workload("kivi", 32, 8192, 8, 32, 128, 2, 2, 0, 2, hadamard_block=1, k_per_channel=True,
                     description="ablation: KIVI-style axes, 2-bit keys per channel and values per token, "
                                 "no rotation, no normalisation (same inputs as gqa)"),
}


def _rng(seed: int, stream: int) -> np.random.Generator:
    # Independent PCG64 streams per tensor of one workload.
    return np.random.Generator(np.random.PCG64([seed, stream]))


def _round_to(x32: np.ndarray, dtype: str) -> np.ndarray:
    """Round float32 values to bf16 / fp16 (nearest-even); returns uint16 bit patterns."""
    if dtype == "fp16":
        return x32.astype(np.float16).view(np.uint16)
    if dtype != "bf16":
        raise ValueError(dtype)
    u = np.ascontiguousarray(x32, dtype=np.float32).view(np.uint32)
    # round-to-nearest-even on the upper 16 bits (inputs here are finite)
    lsb = (u >> 16) & 1
    r = (u + 0x7FFF + lsb) >> 16
    return r.astype(np.uint16)


def half_bits_to_f64(bits: np.ndarray, dtype: str) -> np.ndarray:
    """Exact widening of bf16 / fp16 bit patterns to float64."""
    bits = np.asarray(bits, dtype=np.uint16)
    if dtype == "fp16":
        return bits.view(np.float16).astype(np.float64)
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def outlier_channels(w: Workload, layer: int, head: int, which: str) -> np.ndarray:
    """Seeded outlier channel set of one (layer, kv-head, K/V); fixed across tokens."""
    if _base_name(w) == "rt1k":
        return np.array([3, 17, 64, 101])
    if w.mla:
        n = round(0.01 * w.head_dim)
    elif _base_name(w) in ("gqa", "g128", "saw4", "gqa16", "kivi", "hadonly"):
        n = round(0.02 * w.head_dim)
    else:
        return np.zeros(0, dtype=np.int64)
    r = _rng(w.seed, 1000 + 2 * (layer * max(w.num_kv_heads, 1) + head) + (which == "v"))
    return np.sort(r.choice(w.head_dim, size=n, replace=False))


def _base_name(w: Workload) -> str:
    for k in WORKLOADS:
        if w.name == k or w.name.startswith(k + "-"):
            return k
    return w.name


CHUNK_TOKENS = 4096


def kv_inputs(w: Workload, which: str, tokens: Optional[slice] = None) -> np.ndarray:
    """New K (which="k") or V (which="v") rows: uint16 bits [layers][n_tok][H_kv][d].

    For MLA, which="k" gives the latent [layers][n_tok][1][d]; "v" is unused.
    Values are drawn per chunk of CHUNK_TOKENS tokens from its own PCG64 stream,
    so any token range can be regenerated alone (``tokens`` must then start and
    stop on chunk boundaries, or on n_tok).
    """
    base = _base_name(w)
    L, N, H, d = w.num_layers, w.n_tok, w.num_kv_heads, w.head_dim
    t0, t1 = (0, N) if tokens is None else (tokens.start or 0, tokens.stop if tokens.stop is not None else N)
    if t0 % CHUNK_TOKENS or (t1 % CHUNK_TOKENS and t1 != N):
        raise ValueError("token range must be chunk aligned")
    out = np.empty((L, t1 - t0, H, d), dtype=np.uint16)
    kind = 1 if which == "k" else 2
    scale = None
    if base == "prefill":
        r = _rng(w.seed, 10 * kind)
        scale = np.exp(r.uniform(math.log(0.1), math.log(10.0), size=(L, 1, H, d))).astype(np.float32)
    outl = None
    if base in ("rt1k", "gqa", "mla", "g128", "saw4", "gqa16", "kivi", "hadonly"):
        factor = {"rt1k": 20.0, "gqa": 15.0, "mla": 25.0, "g128": 15.0, "saw4": 15.0, "gqa16": 15.0, "kivi": 15.0,
                  "hadonly": 15.0}[base]
        outl = np.ones((L, 1, H, d), dtype=np.float32)
        for layer in range(L):
            for h in range(H):
                ch = outlier_channels(dataclasses.replace(w, name=base), layer, h, which)
                outl[layer, 0, h, ch] = factor
    def chunk(layer: int, c0: int) -> None:
        c1 = min(c0 + CHUNK_TOKENS, t1)
        r = _rng(w.seed, (kind << 40) | (layer << 24) | (c0 // CHUNK_TOKENS))
        if base == "long" and which == "k":
            x = r.standard_t(4.0, size=(c1 - c0, H, d)).astype(np.float32)
        else:
            x = r.standard_normal(size=(c1 - c0, H, d), dtype=np.float32)
        if outl is not None:
            x *= outl[layer]
        if scale is not None:
            x *= scale[layer]
        out[layer, c0 - t0:c1 - t0] = _round_to(x, w.in_dtype)

    # every chunk has its own stream, so the chunks may be drawn in any order
    # (numpy's generators release the GIL: threads draw them in parallel)
    jobs = [(layer, c0) for layer in range(L) for c0 in range(t0, t1, CHUNK_TOKENS)]
    if len(jobs) <= 2:
        for j in jobs:
            chunk(*j)
    else:
        with ThreadPoolExecutor(min(16, os.cpu_count() or 1)) as ex:
            list(ex.map(lambda j: chunk(*j), jobs))
    return out


def rope_inputs(w: Workload) -> np.ndarray:
    """MLA rope keys: uint16 bf16 bits [layers][n_tok][rope_dim]."""
    r = _rng(w.seed, 3)
    x = r.standard_normal(size=(w.num_layers, w.n_tok, w.rope_dim), dtype=np.float32)
    return _round_to(x, "bf16")


def queries(w: Workload) -> np.ndarray:
    """Decode queries: uint16 bf16 bits [B][H_q][d (+ rope_dim for MLA)], N(0,1)."""
    r = _rng(w.seed, 4)
    width = w.head_dim + (w.rope_dim if w.mla else 0)
    x = r.standard_normal(size=(w.batch, w.num_q_heads, width), dtype=np.float32)
    return _round_to(x, "bf16")


def tail_inputs(w: Workload, which: str) -> np.ndarray:
    """Unquantised tail buffer: uint16 bits [layers][B][T][H_kv][d] in the
    workload's input dtype, N(0,1) (only rows below each tail length are read)."""
    r = _rng(w.seed, 6 if which == "k" else 7)
    x = r.standard_normal(size=(w.num_layers, w.batch, w.tile_tokens, w.num_kv_heads, w.head_dim),
                          dtype=np.float32)
    return _round_to(x, w.in_dtype)


def tail_rope_inputs(w: Workload) -> np.ndarray:
    """Unquantised rope keys of an MLA tail buffer: uint16 bf16 bits
    [layers][B][T][rope_dim], N(0,1)."""
    r = _rng(w.seed, 9)
    x = r.standard_normal(size=(w.num_layers, w.batch, w.tile_tokens, w.rope_dim), dtype=np.float32)
    return _round_to(x, "bf16")


def tail_lens(w: Workload) -> np.ndarray:
    """Tail length of every sequence: int32 [B], uniform in [0, T)."""
    r = _rng(w.seed, 8)
    return r.integers(0, w.tile_tokens, size=w.batch).astype(np.int32)


def page_assignment(w: Workload) -> np.ndarray:
    """Physical page of every tile, in append order (sequence-major): int32 [n_tok / T].

    A seeded permutation, so pages of one sequence are scattered through the pool.
    """
    r = _rng(w.seed, 5)
    return r.permutation(w.num_pages).astype(np.int32)


def block_table(w: Workload) -> np.ndarray:
    """int32 [B][tiles_per_seq]: the pages of each sequence, in token order."""
    return page_assignment(w).reshape(w.batch, w.tiles_per_seq)


def seq_lens(w: Workload) -> np.ndarray:
    return np.full(w.batch, w.seq_len, dtype=np.int32)
