"""GPU parity of kvq_quantize_append (and kvq_dequantize) against the oracle."""
import numpy as np
import pytest
import torch

from kv_cache_quantization_03_b200 import workloads as W
from oracle import kvarn_oracle as O

pytestmark = pytest.mark.gpu

from _parity import CODE_FLIP_RATE, QuantRun, check_tiles  # noqa: E402

SMALL = {
    "rt1k": {},
    "gqa": dict(batch=2, seq_len=512),
    "long": dict(batch=1, seq_len=1024),
    "prefill": dict(seq_len=256, num_layers=3),
    "mla": dict(batch=2, seq_len=256),
    "g128": dict(batch=2, seq_len=512),
    "saw4": dict(batch=2, seq_len=512),
    "hadonly": dict(batch=2, seq_len=512),
    "kivi": dict(batch=2, seq_len=512),
}


def _check_all(run: QuantRun, tiles=None, heads=None, layers=None):
    w = run.w
    tiles = np.arange(w.n_tok // w.tile_tokens) if tiles is None else np.asarray(tiles)
    flips = ties = total = 0
    for which in (("k",) if w.mla else ("k", "v")):
        for layer in (range(w.num_layers) if layers is None else layers):
            for head in (range(w.num_kv_heads) if heads is None else heads):
                f = check_tiles(run, which, layer, tiles, head, "%s L%d H%d" % (which, layer, head))
                flips, ties = flips + f.counted, ties + f.exact_ties
                total += len(tiles) * w.tile_tokens * w.head_dim
    assert flips <= CODE_FLIP_RATE * total, "%d tie flips in %d codes (%d more at exact ties)" % (flips, total, ties)
    return flips, ties, total


@pytest.mark.parametrize("name", list(SMALL))
def test_quantize_parity_small(name):
    w = W.WORKLOADS[name]
    w = w.scaled(**SMALL[name]) if SMALL[name] else w
    run = QuantRun(w)
    assert run.error_bits() == 0
    _check_all(run)


@pytest.mark.parametrize("bits", [(2, 8), (8, 2), (3, 3), (4, 2)])
def test_quantize_parity_other_bit_widths(bits):
    import dataclasses
    w = dataclasses.replace(W.WORKLOADS["gqa"].scaled(batch=1, seq_len=256), bits_k=bits[0], bits_v=bits[1])
    run = QuantRun(w)
    _check_all(run)


@pytest.mark.parametrize("iters", [0, 1, 9, 64])
@pytest.mark.parametrize("name", ["gqa", "g128"])
def test_quantize_parity_iteration_counts(name, iters):
    import dataclasses
    w = dataclasses.replace(W.WORKLOADS[name].scaled(batch=1, seq_len=256), sinkhorn_iters=iters)
    _check_all(QuantRun(w))


@pytest.mark.parametrize("block,iters,bits,tile", [(1, 4, (4, 4), 16), (2, 0, (4, 4), 16), (4, 4, (3, 2), 16),
                                                    (8, 0, (4, 4), 16), (16, 4, (3, 2), 16), (32, 0, (4, 4), 16),
                                                    (64, 6, (2, 8), 16), (32, 4, (4, 2), 128)])
def test_quantize_parity_block_diagonal_rotation(block, iters, bits, tile):
    # SAW-INT4-style ablation: blocks of 1..64 channels (1: no rotation), with and without the normalisation
    import dataclasses
    w = dataclasses.replace(W.WORKLOADS["saw4"].scaled(batch=1, seq_len=512), hadamard_block=block,
                            sinkhorn_iters=iters, bits_k=bits[0], bits_v=bits[1], tile_tokens=tile)
    run = QuantRun(w)
    assert run.error_bits() == 0
    _check_all(run)


@pytest.mark.parametrize("tile,bits", [(32, (3, 4)), (64, (4, 8)), (128, (3, 2)), (128, (8, 4))])
def test_quantize_parity_tile_lengths(tile, bits):
    # 2, 4 or 8 warps share a tile's column sums; 3-bit planes span the whole page
    import dataclasses
    w = dataclasses.replace(W.WORKLOADS["gqa"].scaled(batch=1, seq_len=512), tile_tokens=tile, bits_k=bits[0],
                            bits_v=bits[1])
    run = QuantRun(w)
    assert run.error_bits() == 0
    _check_all(run)


def _special_tiles():
    """Degenerate tiles: zeros, a single nonzero, constant rows, a +-1
    checkerboard, a huge outlier channel, a zero row and a zero column."""
    T, d = 16, 128
    rng = np.random.default_rng(21)
    tiles = []
    tiles.append(np.zeros((T, d)))
    t = np.zeros((T, d)); t[5, 17] = 3.0; tiles.append(t)
    tiles.append(np.repeat(rng.standard_normal((T, 1)), d, axis=1))
    tiles.append(np.where((np.arange(T)[:, None] + np.arange(d)[None, :]) % 2 == 0, 1.0, -1.0))
    t = rng.standard_normal((T, d)); t[:, 40] *= 1000.0; tiles.append(t)
    t = rng.standard_normal((T, d)); t[7, :] = 0.0; tiles.append(t)
    t = rng.standard_normal((T, d)) * 1e-3; tiles.append(t)
    t = rng.standard_normal((T, d)) * 1e4; tiles.append(t)
    x = np.concatenate(tiles, 0).astype(np.float32)        # [n*T, d]
    return x


@pytest.mark.parametrize("tile", [16, 128])
def test_quantize_parity_degenerate_tiles(tile):
    # at 128 tokens the eight blocks form one tile: zero rows, a constant block,
    # a huge outlier column and a 1e7 spread of magnitudes in one normalisation
    import dataclasses
    x = _special_tiles()
    n_tok = x.shape[0]
    w = dataclasses.replace(W.WORKLOADS["gqa"], batch=1, seq_len=n_tok, num_kv_heads=1, num_q_heads=1,
                            name="special", tile_tokens=tile)
    kb = W._round_to(x, "bf16").reshape(1, n_tok, 1, 128)
    vb = W._round_to(-x[::-1].copy(), "bf16").reshape(1, n_tok, 1, 128)
    run = QuantRun(w, inputs=(kb, vb), pages=np.arange(n_tok // tile, dtype=np.int32))
    assert run.error_bits() == 0
    _check_all(run)
    if tile == 16:
        zero = run.gpu_tiles("k", 0, [0], 0)
        assert np.all(zero.q == 0) and np.all(zero.a == 0) and np.all(zero.z == 0) and np.all(zero.c == 1)


def _scaled(w, which, row_exp):
    """The workload's inputs with token row i of every tile scaled by the exact
    power of two 2^row_exp[i % T], rounded back to the input format (exact for
    normal values)."""
    x = W.half_bits_to_f64(W.kv_inputs(w, which), w.in_dtype)
    e = np.asarray(row_exp, dtype=np.float64)
    f = np.exp2(np.tile(e, x.shape[1] // e.size))[None, :, None, None]
    return W._round_to((x * f).astype(np.float32), w.in_dtype)


# exponent of every token row of a tile: unit rows, single rows far from the
# others, and whole tiles near the ends of the bf16 range (kept in its normal
# range: elements below 2^-126 would be subnormal inputs)
ROW_SCALES = {
    "one_row_2^-64": [0] * 5 + [-64] + [0] * 10,
    "rows_2^-100_to_2^100": [0, -100, 60, 0, -30, 30, 0, -64, 0, 64, 0, 0, -96, 0, 100, 0],
    "tile_2^-100": [-100] * 16,
    "tile_2^+100": [100] * 16,
}


@pytest.mark.parametrize("scales", list(ROW_SCALES))
@pytest.mark.parametrize("name,iters", [("gqa", 4), ("gqa", 0), ("long", 6), ("g128", 4), ("mla", 4)])
def test_quantize_parity_dynamic_range(name, iters, scales):
    # The method is invariant to a power-of-two scale of a token row (codes
    # and column factors unchanged, a and z scaled): the kernel must follow
    # the float64 oracle across the bf16 exponent range, including tiles whose
    # rows differ by 2^200.
    import dataclasses
    w = dataclasses.replace(W.WORKLOADS[name].scaled(batch=1, seq_len=256), sinkhorn_iters=iters)
    e = ROW_SCALES[scales]
    e = (e * (w.tile_tokens // 16))[: w.tile_tokens] if w.tile_tokens > 16 else e
    kb = _scaled(w, "k", e)
    vb = None if w.mla else _scaled(w, "v", e[::-1])
    run = QuantRun(w, inputs=(kb, vb))
    assert run.error_bits() == 0
    flips, ties, total = _check_all(run)
    assert flips + ties <= 1e-3 * total


@pytest.mark.parametrize("name", ["gqa16", "long", "g128", "mla", "prefill"])
def test_quantize_parity_half_metadata(name):
    # a, z, c stored as IEEE half: the codes are the float32 layout's, bit for
    # bit (the format does not enter the code decision), and each half is the
    # oracle's rounding of the exact value (or its neighbour at a midpoint)
    import dataclasses
    w = W.WORKLOADS[name]
    w = dataclasses.replace(w.scaled(batch=1, seq_len=256, num_layers=2 if w.num_layers > 1 else None),
                            meta_f16=True)
    run = QuantRun(w)
    assert run.error_bits() == 0
    _check_all(run)
    ref = QuantRun(dataclasses.replace(w, meta_f16=False))
    for which in (("k",) if w.mla else ("k", "v")):
        assert torch.equal(run.cache.codes(which), ref.cache.codes(which)), which


@pytest.mark.parametrize("bits,block,meta16", [(4, 1, False), (8, 1, False), (2, 32, False), (4, 128, True),
                                           (2, 1, True)])
def test_quantize_parity_per_channel_keys(bits, block, meta16):
    # KIVI-style axes: keys per channel (with and without a rotation, either
    # metadata format), values per token
    import dataclasses
    w = dataclasses.replace(W.WORKLOADS["kivi"].scaled(batch=2, seq_len=256), bits_k=bits, bits_v=bits,
                            hadamard_block=block, meta_f16=meta16)
    run = QuantRun(w)
    assert run.error_bits() == 0
    _check_all(run)


def test_quantize_bad_page_sets_error_and_skips_tile():
    w = W.WORKLOADS["gqa"].scaled(batch=1, seq_len=64)
    pages = np.array([0, 7, 2, 3], dtype=np.int32)        # pool of 4 pages: 7 is out of range
    run = QuantRun(w, quantize=False, pages=pages, num_pages=4)
    canary = run.cache.codes("k")[0, 1].clone()
    run.cache.codes("k")[0, 1].fill_(0xA5)
    run.cache.codes("v")[0, 1].fill_(0xA5)
    run.quantize()
    assert run.error_bits() & 0x1
    assert torch.all(run.cache.codes("k")[0, 1] == 0xA5) and torch.all(run.cache.codes("v")[0, 1] == 0xA5)
    del canary
    _check_all(run, tiles=[0, 2, 3])


@pytest.mark.parametrize("name", ["rt1k", "mla", "g128"])
def test_quantize_single_tile(name):
    # One tile per call: at head_dim 128 three of the CTA's four warps have no
    # tile and go straight to the CTA's final barrier; at 512 one CTA works;
    # a 128-token tile is one CTA of eight warps.
    w = W.WORKLOADS[name]
    w = w.scaled(batch=1, seq_len=w.tile_tokens)
    run = QuantRun(w)
    assert run.error_bits() == 0
    _check_all(run)


def test_long_tile_bad_page_sets_error_and_skips_tile():
    # 128-token tiles: the eight warps of a tile leave it together on a bad page
    w = W.WORKLOADS["g128"].scaled(batch=1, seq_len=512)
    pages = np.array([0, 1, 6, 3], dtype=np.int32)        # pool of 4 pages: 6 is out of range
    run = QuantRun(w, quantize=False, pages=pages, num_pages=4)
    run.cache.codes("k")[0, 2].fill_(0xA5)
    run.cache.codes("v")[0, 2].fill_(0xA5)
    run.quantize()
    assert run.error_bits() & 0x1
    assert torch.all(run.cache.codes("k")[0, 2] == 0xA5) and torch.all(run.cache.codes("v")[0, 2] == 0xA5)
    _check_all(run, tiles=[0, 1, 3])


def test_mla_quantize_bad_page_sets_error_and_skips_tile():
    # head_dim 512: the four warps of a tile leave it together on a bad page
    w = W.WORKLOADS["mla"].scaled(batch=1, seq_len=64)
    pages = np.array([0, 9, 2, 3], dtype=np.int32)        # pool of 4 pages: 9 is out of range
    run = QuantRun(w, quantize=False, pages=pages, num_pages=4)
    run.cache.codes("k")[0, 1].fill_(0xA5)
    run.quantize()
    assert run.error_bits() & 0x1
    assert torch.all(run.cache.codes("k")[0, 1] == 0xA5)
    _check_all(run, tiles=[0, 2, 3])


def test_mla_rope_rows_copied_to_their_pages():
    w = W.WORKLOADS["mla"].scaled(batch=2, seq_len=128)
    run = QuantRun(w)
    assert run.error_bits() == 0
    rope = run.cache["rope"].view(w.num_layers, w.num_pages, 16, w.rope_dim).cpu().view(torch.int16).numpy()
    src = run.rope_bits.view(np.int16).reshape(w.num_layers, -1, 16, w.rope_dim)
    for tile, page in enumerate(run.pages):
        assert np.array_equal(rope[0, page], src[0, tile])


def test_quantize_deterministic():
    w = W.WORKLOADS["gqa"].scaled(batch=1, seq_len=512)
    run = QuantRun(w)
    first = {n: t.clone() for n, t in run.cache.arrays.items() if t is not None}
    run.quantize()
    for n, t in first.items():
        assert torch.equal(run.cache.arrays[n], t), n


@pytest.mark.parametrize("name", ["long", "mla", "g128", "saw4", "hadonly", "gqa16", "kivi"])
def test_dequantize_matches_oracle_on_stored_codes(name):
    from kv_cache_quantization_03_b200 import kvq
    w = W.WORKLOADS[name].scaled(batch=1, seq_len=256)
    run = QuantRun(w)
    pages = torch.arange(w.num_pages, dtype=torch.int32, device="cuda")
    for unrot in (0, 1):
        ko = torch.empty(w.num_pages, w.num_kv_heads, w.tile_tokens, w.head_dim, device="cuda")
        vo = torch.empty_like(ko)
        kvq.kvq_dequantize(run.cfg, run.cache.view, 0, pages, w.num_pages, unrot, ko, None if w.mla else vo,
                           run.err)
        torch.cuda.synchronize()
        for which, out in ((("k", ko),) if w.mla else (("k", ko), ("v", vo))):
            for h in range(w.num_kv_heads):
                inv = np.argsort(run.pages)                      # page -> tile
                g = run.gpu_tiles(which, 0, inv, h)              # tiles in page order
                if isinstance(g, O.ChannelQuantizedTiles):
                    ref = O.dequantize_channel_tiles(g, unrotate=bool(unrot), block=w.block)
                else:
                    ref = O.dequantize_tiles(g.q, g.a, g.z, g.c, unrotate=bool(unrot), block=w.block)
                got = out[:, h].cpu().numpy().astype(np.float64)
                scale = np.max(np.abs(ref), axis=(-1, -2), keepdims=True)
                assert np.max(np.abs(got - ref) / scale) < 2e-6
