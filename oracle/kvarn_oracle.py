"""Float64 CPU oracle of KVarN-style variance-normalised KV-cache quantisation.

TEST INFRASTRUCTURE ONLY.  This module is the plain, slow, obviously correct
statement of what the CUDA path computes.  Only ``tests/``,
``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` may import
it; the library (``kv_cache_quantization_03_b200``) never does, and this module
imports nothing from the library.  It shares no code, table or constant
generator with the kernels.

What it follows
---------------
The KVarN pipeline as the pages describe it, one tile (T tokens x d channels
of one layer / kv-head, keys or values alone) at a time:

1. a Hadamard rotation along head_dim that spreads channel outliers
   (KVarN project page on open-radar, Key Features, "Variance-Normalized
   Quantization Pipeline"; KV-Cache tag page on baguaai.com, KVarN item:
   rotation combined with dual-axis variance normalisation);
2. an iterative Sinkhorn-like normalisation that equalises the variance of
   the tile's rows (tokens) and columns (channels), computed per tile with no
   calibration (same page, "Calibration-Free Operation");
3. asymmetric round-to-nearest quantisation (same pages; the KV-Cache tag
   page names RTN);
4. packing of the codes into the paged cache, one tile per cache block
   (KVarN project page, "4-bit Keys, 2-bit Values Preset": the tile equals
   the serving engine's block).

and the consumer: decode attention over the quantised cache with the query
rotated by the same orthogonal Hadamard, plus the MLA variant in which one
quantised latent serves as both key and value next to an unquantised rope
key (KVarN project page, "MLA Model Support").

Readings where the pages are silent (each is a declared choice):

* "variance" is the uncentred second moment (mean of squares); with it the
  normalisation is Sinkhorn-Knopp scaling of the positive matrix Z*Z, which
  converges, whereas the centred form does not settle;
* each iteration normalises the rows first, then the columns; a row or
  column whose second moment is exactly 0 is left as it is (factor 1);
* the Hadamard matrix is Sylvester's, of full width d, scaled by 1/sqrt(d);
* quantisation groups are token rows of the normalised tile: zero point
  m = row min (a float), step s = (max - min) / (2^b - 1), codes
  rint((y - m) / s) with ties to even, clamped to [0, 2^b - 1]; s = 0 gives
  code 0;
* the row and column factors are folded into what is stored: per token
  a = r * s and z = r * m, per channel c, all float32 (round to nearest);
  dequantisation in the rotated domain is (a * q + z) * c;
* the pages fix no scale layout, and (a, z, c) is only defined up to moving
  a factor between c and (a, z).  The stored tile is balanced by a power of
  two: with k the integer for which max_j c_j (as float32) lies in
  (2^(k-1), 2^k], c is stored times 2^-k and a, z times 2^k.  The scaling is
  exact, so the dequantised tile is unchanged, and every stored c is <= 1
  (a consumer can bound a dequantised row by max(|z|, |a (2^b - 1) + z|));
* metadata format: float32 by default; the compact layout stores a, z, c
  as IEEE half precision (round to nearest even from the balanced float64
  values).  Codes do not depend on it;
* codes are packed little-endian inside each byte, lowest channel in the
  lowest bits, token rows one after the other; 3-bit codes are two planes
  per tile: all rows' low 2 bits (2-bit packing), then all rows' high bit
  (1-bit packing).

All arithmetic is float64 except the rounding of the stored a, z, c to the
metadata format.
Parity of every function here is pinned in tests/test_oracle_pins.py against
closed forms, library routines, brute force and hand-worked fixtures.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import numpy as np

SUPPORTED_BITS = (2, 3, 4, 8)


# --------------------------------------------------------------------------
# 1. Hadamard rotation
# --------------------------------------------------------------------------
def hadamard_matrix(n: int) -> np.ndarray:
    """Sylvester Hadamard matrix of order n (a power of two), int64 entries +-1.

    H_1 = [1];  H_2k = [[H_k, H_k], [H_k, -H_k]].  Unnormalised: H H^T = n I.
    """
    if n < 1 or n & (n - 1):
        raise ValueError("order must be a power of two")
    h = np.ones((1, 1), dtype=np.int64)
    while h.shape[0] < n:
        h = np.block([[h, h], [h, -h]])
    return h


def block_hadamard_matrix(d: int, block: int) -> np.ndarray:
    """Block-diagonal Hadamard of order d: d / block copies of H_block on the
    diagonal, int64 (the "block-diagonal Hadamard rotation" of the SAW-INT4
    entry on the Hugging Face paper listing; blocks are runs of consecutive
    channels).  block == d gives the full Sylvester matrix."""
    if d % block:
        raise ValueError("block must divide d")
    return np.kron(np.eye(d // block, dtype=np.int64), hadamard_matrix(block))


def rotate(x: np.ndarray, block: Optional[int] = None) -> np.ndarray:
    """x H / sqrt(b) along the last axis (float64), H the Sylvester matrix of
    the full width d (block None or d) or the block-diagonal one of order d
    with blocks of b channels.

    H / sqrt(b) is symmetric and orthogonal, so the same call undoes itself:
    rotate(rotate(x)) == x up to rounding.  Dense product, no fast transform.
    """
    x = np.asarray(x, dtype=np.float64)
    d = x.shape[-1]
    b = d if block is None else block
    return (x @ block_hadamard_matrix(d, b).astype(np.float64)) / math.sqrt(b)


# --------------------------------------------------------------------------
# 2. Sinkhorn-like dual-axis variance normalisation
# --------------------------------------------------------------------------
def sinkhorn_normalize(z: np.ndarray, n_iter: int, history: Optional[list] = None):
    """Normalise the second moments of rows and columns of each tile.

    z: [..., T, d] float64 (rotated tile(s)).  Returns (y, r, c) with
    y: [..., T, d], r: [..., T], c: [..., d] such that z = diag(r) y diag(c).

    Each of the n_iter rounds divides every row by its root-mean-square
    (over d channels) and multiplies that factor into r, then divides every
    column by its root-mean-square (over T tokens) and multiplies it into c.
    A zero root-mean-square leaves its row or column unchanged.  If
    ``history`` is a list, (y, r, c) after every half-step is appended.
    """
    y = np.array(z, dtype=np.float64, copy=True)
    r = np.ones(y.shape[:-1], dtype=np.float64)
    c = np.ones(y.shape[:-2] + y.shape[-1:], dtype=np.float64)
    for _ in range(n_iter):
        sigma = np.sqrt(np.mean(y * y, axis=-1))            # row RMS, [..., T]
        f = np.where(sigma > 0, sigma, 1.0)
        y = y / f[..., :, None]
        r = r * f
        if history is not None:
            history.append((y.copy(), r.copy(), c.copy()))
        tau = np.sqrt(np.mean(y * y, axis=-2))              # column RMS, [..., d]
        g = np.where(tau > 0, tau, 1.0)
        y = y / g[..., None, :]
        c = c * g
        if history is not None:
            history.append((y.copy(), r.copy(), c.copy()))
    return y, r, c


# --------------------------------------------------------------------------
# 3. Asymmetric round-to-nearest quantisation (per token row)
# --------------------------------------------------------------------------
def rtn_rows(y: np.ndarray, bits: int):
    """Asymmetric RTN of every row of y: [..., T, d] -> (q int64, m, s).

    m = row min, s = (row max - m) / (2^bits - 1),
    q = clamp(rint((y - m) / s), 0, 2^bits - 1)  (rint rounds half to even);
    rows with s == 0 get q = 0.
    """
    if bits not in SUPPORTED_BITS:
        raise ValueError("bits must be one of %s" % (SUPPORTED_BITS,))
    qmax = (1 << bits) - 1
    m = np.min(y, axis=-1)
    s = (np.max(y, axis=-1) - m) / qmax
    safe = np.where(s > 0, s, 1.0)
    t = (y - m[..., None]) / safe[..., None]
    q = np.clip(np.rint(t), 0, qmax).astype(np.int64)
    q = np.where((s > 0)[..., None], q, 0)
    return q, m, s


@dataclasses.dataclass
class QuantizedTiles:
    """What one or more quantised tiles store: logical codes and folded scales."""
    q: np.ndarray   # int64 [..., T, d]   codes in [0, 2^bits - 1]
    a: np.ndarray   # float32 [..., T]    a = r * s * 2^k
    z: np.ndarray   # float32 [..., T]    z = r * m * 2^k
    c: np.ndarray   # float32 [..., d]    column factor * 2^-k (max in (1/2, 1])


def balance_exponent(c32: np.ndarray) -> np.ndarray:
    """The integer k with max_j c_j in (2^(k-1), 2^k] of each tile's float32
    column factors c32: [..., d] (positive).  Exact: from the binary exponent."""
    cmax = np.max(np.asarray(c32, dtype=np.float64), axis=-1)
    mant, e = np.frexp(cmax)                  # cmax = mant * 2^e, mant in [1/2, 1)
    return np.where(mant == 0.5, e - 1, e).astype(np.int64)


def quantize_stages(x: np.ndarray, bits: int, n_iter: int, block: Optional[int] = None):
    """The pipeline up to storage: rotate, normalise, RTN, balance.

    Returns (q, a, z, c) with a, z, c in float64, already balanced by the
    power of two 2^k (k decided on the float32 column factors, the precision
    in which the stored c lives).  quantize_tiles rounds them for storage."""
    z = rotate(x, block)
    y, r, c = sinkhorn_normalize(z, n_iter)
    q, m, s = rtn_rows(y, bits)
    k = balance_exponent(c.astype(np.float32))
    return q, np.ldexp(r * s, k[..., None]), np.ldexp(r * m, k[..., None]), np.ldexp(c, -k[..., None])


def quantize_tiles(x: np.ndarray, bits: int, n_iter: int, block: Optional[int] = None,
                   meta: str = "f32") -> QuantizedTiles:
    """Rotate, normalise and quantise tiles x: [..., T, d] (any float dtype).

    The tiles are independent; leading axes only batch them.  block: the
    rotation's block (None = full width).  The stored scales are balanced
    by a power of two (max c in (1/2, 1]; see the module notes) and rounded
    to nearest in the metadata format: meta "f32" (float32) or "f16" (IEEE
    half: the compact layout, same codes, scales to 11 significant bits).
    """
    q, a, z, c = quantize_stages(x, bits, n_iter, block)
    if meta == "f32":
        # the unbalanced float32 values times an exact power of two
        return QuantizedTiles(q=q, a=a.astype(np.float32), z=z.astype(np.float32), c=c.astype(np.float32))
    if meta == "f16":
        return QuantizedTiles(q=q, a=a.astype(np.float16), z=z.astype(np.float16), c=c.astype(np.float16))
    raise ValueError("meta must be 'f32' or 'f16'")


@dataclasses.dataclass
class ChannelQuantizedTiles:
    """Keys quantised along the other axis: one (step, minimum) per channel."""
    q: np.ndarray   # int64 [..., T, d]   codes in [0, 2^bits - 1]
    s: np.ndarray   # float32 [..., d]    step of each channel
    m: np.ndarray   # float32 [..., d]    minimum of each channel


def quantize_tiles_per_channel(x: np.ndarray, bits: int, block: Optional[int] = None) -> ChannelQuantizedTiles:
    """KIVI-style key quantisation (the KIVI entry of the Hugging Face paper
    listing: keys quantised per channel, values per token, asymmetric,
    tuning-free), as the ablation of the dual-axis normalisation: the tile
    is rotated (block 1 = no rotation, as in KIVI), not normalised, and every
    channel (a column of the tile: its T tokens) is one asymmetric RTN group
    with its own minimum m_j and step s_j = (max_j - m_j) / (2^b - 1).
    Dequantised (rotated domain): s_j q_tj + m_j."""
    z = rotate(x, block)
    qt, m, st = rtn_rows(np.swapaxes(z, -1, -2), bits)     # the channels as the groups
    return ChannelQuantizedTiles(q=np.swapaxes(qt, -1, -2), s=st.astype(np.float32), m=m.astype(np.float32))


def dequantize_channel_tiles(t: ChannelQuantizedTiles, unrotate: bool = True,
                             block: Optional[int] = None) -> np.ndarray:
    """s_j q_tj + m_j (float64), then optionally un-rotated."""
    zh = np.asarray(t.s, np.float64)[..., None, :] * np.asarray(t.q, np.float64) + \
        np.asarray(t.m, np.float64)[..., None, :]
    return rotate(zh, block) if unrotate else zh


def _rotated_rows(t) -> np.ndarray:
    """Dequantised rows, rotated domain, of either kind of quantised tiles."""
    if isinstance(t, ChannelQuantizedTiles):
        return dequantize_channel_tiles(t, unrotate=False)
    return dequantize_tiles(t.q, t.a, t.z, t.c, unrotate=False)


def dequantize_tiles(q, a, z, c, unrotate: bool = True, block: Optional[int] = None) -> np.ndarray:
    """(a q + z) c in the rotated domain (float64), then optionally un-rotated."""
    a = np.asarray(a, dtype=np.float64)
    z = np.asarray(z, dtype=np.float64)
    c = np.asarray(c, dtype=np.float64)
    zh = (a[..., :, None] * np.asarray(q, dtype=np.float64) + z[..., :, None]) * c[..., None, :]
    return rotate(zh, block) if unrotate else zh


# --------------------------------------------------------------------------
# 4. Packing into the cache's byte format
# --------------------------------------------------------------------------
def tile_code_bytes(bits: int, tile_tokens: int, head_dim: int) -> int:
    return tile_tokens * head_dim * bits // 8


def _pack_fields(v: np.ndarray, width: int) -> np.ndarray:
    """Pack [..., n] small ints of `width` bits, 8/width per byte, low bits first."""
    per = 8 // width
    v = v.reshape(v.shape[:-1] + (v.shape[-1] // per, per)).astype(np.uint16)
    out = np.zeros(v.shape[:-1], dtype=np.uint16)
    for i in range(per):
        out |= v[..., i] << (width * i)
    return out.astype(np.uint8)


def _unpack_fields(b: np.ndarray, width: int) -> np.ndarray:
    per = 8 // width
    b = b.astype(np.uint16)
    mask = (1 << width) - 1
    parts = [(b >> (width * i)) & mask for i in range(per)]
    return np.stack(parts, axis=-1).reshape(b.shape[:-1] + (b.shape[-1] * per,)).astype(np.int64)


def pack_codes(q: np.ndarray, bits: int) -> np.ndarray:
    """Logical codes [..., T, d] -> bytes [..., T * d * bits / 8] of one tile each."""
    q = np.asarray(q)
    lead, (T, d) = q.shape[:-2], q.shape[-2:]
    if bits in (2, 4, 8):
        return _pack_fields(q, bits).reshape(lead + (T * d * bits // 8,))
    if bits == 3:
        lo = _pack_fields(q & 3, 2).reshape(lead + (T * d // 4,))
        hi = _pack_fields(q >> 2, 1).reshape(lead + (T * d // 8,))
        return np.concatenate([lo, hi], axis=-1)
    raise ValueError("bits")


def unpack_codes(buf: np.ndarray, bits: int, tile_tokens: int, head_dim: int) -> np.ndarray:
    """Inverse of pack_codes: bytes [..., nbytes] -> int64 codes [..., T, d]."""
    buf = np.asarray(buf, dtype=np.uint8)
    lead = buf.shape[:-1]
    T, d = tile_tokens, head_dim
    if bits in (2, 4, 8):
        return _unpack_fields(buf.reshape(lead + (T, d * bits // 8)), bits)
    if bits == 3:
        lo = _unpack_fields(buf[..., : T * d // 4].reshape(lead + (T, d // 4)), 2)
        hi = _unpack_fields(buf[..., T * d // 4:].reshape(lead + (T, d // 8)), 1)
        return lo | (hi << 2)
    raise ValueError("bits")


# --------------------------------------------------------------------------
# 5. Decode attention over the quantised cache
# --------------------------------------------------------------------------
def _softmax(s: np.ndarray) -> np.ndarray:
    e = np.exp(s - np.max(s, axis=-1, keepdims=True))
    return e / np.sum(e, axis=-1, keepdims=True)


def decode_attention(q: np.ndarray, k: QuantizedTiles, v: QuantizedTiles,
                     softmax_scale: float, block: Optional[int] = None) -> np.ndarray:
    """One decode step of the G query heads that share one kv-head.

    q: [G, d] (float, un-rotated).  k, v: the kv-head's tiles in token order,
    q/a/z/c with leading tile axis [n_tiles, T, ...].  Returns o: [G, d]
    float64, un-rotated.  The query is rotated with the same H as the cache,
    attention runs in the rotated domain on the dequantised tiles, and the
    output is rotated back.
    """
    d = q.shape[-1]
    kh = _rotated_rows(k).reshape(-1, d)      # keys: per-token tiles, or per-channel (KIVI-style axes)
    vh = _rotated_rows(v).reshape(-1, d)
    qr = rotate(q, block)
    p = _softmax(softmax_scale * (qr @ kh.T))
    return rotate(p @ vh, block)


def decode_attention_with_tail(q: np.ndarray, k: Optional[QuantizedTiles], v: Optional[QuantizedTiles],
                               k_tail: np.ndarray, v_tail: np.ndarray, softmax_scale: float,
                               block: Optional[int] = None) -> np.ndarray:
    """Decode step over a sequence whose newest tokens do not fill a tile yet.

    The cache holds the sequence's whole tiles; the last L < T tokens (the
    tail) are kept at input precision until their tile fills (the pages say
    nothing on this; the reading: a serving engine appends token by token,
    so the tokens past the last whole tile stay unquantised, and attention
    runs over all of the sequence's keys).

    q: [G, d] un-rotated; k, v: the kv-head's quantised tiles in token order
    (or None for none); k_tail, v_tail: [L, d] tail rows.  Written in the
    input basis: the tiles are dequantised and rotated back, the tail rows
    join them as they are, then plain softmax attention.  Returns [G, d].
    """
    q = np.asarray(q, dtype=np.float64)
    d = q.shape[-1]
    keys = [np.asarray(k_tail, dtype=np.float64).reshape(-1, d)]
    vals = [np.asarray(v_tail, dtype=np.float64).reshape(-1, d)]
    if k is not None and k.q.shape[0] > 0:
        keys.insert(0, rotate(_rotated_rows(k), block).reshape(-1, d))
        vals.insert(0, dequantize_tiles(v.q, v.a, v.z, v.c, unrotate=True, block=block).reshape(-1, d))
    kk = np.concatenate(keys, 0)
    vv = np.concatenate(vals, 0)
    if kk.shape[0] == 0:
        return np.zeros((q.shape[0], d))
    p = _softmax(softmax_scale * (q @ kk.T))
    return p @ vv


def mla_decode_attention(q: np.ndarray, lat: QuantizedTiles, rope: np.ndarray,
                         softmax_scale: float) -> np.ndarray:
    """MLA decode step: one quantised latent serves as key and value.

    q: [H, d + rope_dim] (latent part un-rotated, rope part as is).
    lat: the latent tiles [n_tiles, T, d]; rope: [n_tiles * T, rope_dim] keys.
    Score of token t: scale * (rotate(q_lat) . latent_t + q_rope . rope_t);
    output: rotate back (sum_t p_t latent_t): [H, d] float64.
    """
    d = lat.q.shape[-1]
    ch = dequantize_tiles(lat.q, lat.a, lat.z, lat.c, unrotate=False).reshape(-1, d)
    q = np.asarray(q, dtype=np.float64)
    qr = rotate(q[:, :d])
    s = qr @ ch.T + q[:, d:] @ np.asarray(rope, dtype=np.float64).T
    p = _softmax(softmax_scale * s)
    return rotate(p @ ch)


def mla_decode_attention_with_tail(q: np.ndarray, lat: Optional[QuantizedTiles], rope: Optional[np.ndarray],
                                   lat_tail: np.ndarray, rope_tail: np.ndarray, softmax_scale: float) -> np.ndarray:
    """MLA decode step over a sequence whose newest tokens do not fill a tile.

    Same reading as decode_attention_with_tail: the last L < T tokens stay
    unquantised (latent row and rope key as given) and attention runs over
    all of the sequence's tokens.  Written in the input basis: the cached
    latent tiles are dequantised and rotated back, the tail rows join them
    as they are; score = scale * (q_lat . latent + q_rope . rope), output =
    sum p latent.  q: [H, d + rope_dim]; lat: [n_tiles, T, d] quantised (or
    None); rope: [n_tiles * T, rope_dim]; lat_tail: [L, d]; rope_tail:
    [L, rope_dim].  Returns [H, d].
    """
    q = np.asarray(q, dtype=np.float64)
    d = np.asarray(lat_tail).shape[-1]
    rd = q.shape[-1] - d
    keys = [np.asarray(lat_tail, dtype=np.float64).reshape(-1, d)]
    ropes = [np.asarray(rope_tail, dtype=np.float64).reshape(-1, rd)]
    if lat is not None and lat.q.shape[0] > 0:
        keys.insert(0, dequantize_tiles(lat.q, lat.a, lat.z, lat.c, unrotate=True).reshape(-1, d))
        ropes.insert(0, np.asarray(rope, dtype=np.float64).reshape(-1, rd))
    kk, rr = np.concatenate(keys, 0), np.concatenate(ropes, 0)
    if kk.shape[0] == 0:
        return np.zeros((q.shape[0], d))
    p = _softmax(softmax_scale * (q[:, :d] @ kk.T + q[:, d:] @ rr.T))
    return p @ kk

