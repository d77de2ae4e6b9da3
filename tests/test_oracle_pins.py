"""Pins of the float64 oracle against things other than itself.

Closed forms, library routines (scipy's Hadamard, torch's scaled-dot-product
attention in float64), brute force on tiny inputs, invariants of the method and
hand-worked fixtures under tests/golden/.  Each test is chosen so that a
plausible slip in the oracle (a dropped term, a wrong sign or axis, a
transposed operand, a wrong rounding rule) fails it.
"""
import json
import math
import os

import numpy as np
import pytest

from oracle import kvarn_oracle as O
from kv_cache_quantization_03_b200 import workloads as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


# ---------------------------------------------------------------- Hadamard
@pytest.mark.parametrize("n", [1, 2, 4, 8, 16, 128, 512])
def test_hadamard_orthogonal_exact(n):
    h = O.hadamard_matrix(n)
    assert h.dtype == np.int64
    assert np.array_equal(h @ h.T, n * np.eye(n, dtype=np.int64))
    assert np.array_equal(h, h.T)


def test_hadamard_small_cases_and_scipy():
    import scipy.linalg
    assert np.array_equal(O.hadamard_matrix(2), [[1, 1], [1, -1]])
    assert np.array_equal(O.hadamard_matrix(4), [[1, 1, 1, 1], [1, -1, 1, -1],
                                                 [1, 1, -1, -1], [1, -1, -1, 1]])
    for n in (8, 64, 128, 512):
        assert np.array_equal(O.hadamard_matrix(n), scipy.linalg.hadamard(n))


def test_hadamard_entry_formula():
    # Sylvester entries: (-1)^popcount(i & j)
    n = 128
    h = O.hadamard_matrix(n)
    i, j = np.meshgrid(np.arange(n), np.arange(n), indexing="ij")
    pc = np.vectorize(lambda v: bin(v).count("1"))(i & j)
    assert np.array_equal(h, np.where(pc % 2 == 0, 1, -1))


@pytest.mark.parametrize("block", [8, 16, 32, 64, 128])
def test_block_hadamard_orthogonal_and_block_local(block):
    B = O.block_hadamard_matrix(128, block)
    assert np.array_equal(B @ B.T, block * np.eye(128, dtype=np.int64))
    # a spike in channel 37 spreads over its own block of channels only
    e = np.zeros(128); e[37] = 1.0
    r = O.rotate(e, block)
    lo = 37 // block * block
    assert np.allclose(np.abs(r[lo:lo + block]), 1 / math.sqrt(block), rtol=0, atol=1e-15)
    assert np.all(r[:lo] == 0) and np.all(r[lo + block:] == 0)
    x = np.random.default_rng(40).standard_normal((3, 128))
    assert np.max(np.abs(O.rotate(O.rotate(x, block), block) - x)) < 1e-12


@pytest.mark.parametrize("block", [8, 32])
def test_full_rotation_factors_through_the_block_rotation(block):
    # Sylvester: H_d = H_(d/b) (x) H_b = (H_(d/b) (x) I_b)(I_(d/b) (x) H_b), so the
    # full rotation is the block rotation followed by H_(d/b) across the blocks
    x = np.random.default_rng(41).standard_normal((4, 128))
    across = np.kron(O.hadamard_matrix(128 // block), np.eye(block)) / math.sqrt(128 // block)
    assert np.max(np.abs(O.rotate(x, block) @ across - O.rotate(x))) < 1e-12
    assert np.array_equal(O.block_hadamard_matrix(128, 128), O.hadamard_matrix(128))


def test_block_rotation_attention_matches_plain_attention_on_dequantised_rows():
    # decode with a block rotation equals plain attention on the rows the cache
    # decodes to (dequantised and rotated back with the same blocks)
    rng = np.random.default_rng(42)
    x = rng.standard_normal((2, 3, 16, 128))
    k = O.quantize_tiles(x[0], 4, 0, block=32)
    v = O.quantize_tiles(x[1], 4, 0, block=32)
    q = rng.standard_normal((4, 128))
    o = O.decode_attention(q, k, v, 0.1, block=32)
    kk = O.dequantize_tiles(k.q, k.a, k.z, k.c, block=32).reshape(-1, 128)
    vv = O.dequantize_tiles(v.q, v.a, v.z, v.c, block=32).reshape(-1, 128)
    s = 0.1 * q @ kk.T
    p = np.exp(s - s.max(-1, keepdims=True))
    p /= p.sum(-1, keepdims=True)
    assert np.max(np.abs(o - p @ vv)) < 1e-12


def test_rotate_roundtrip_and_parseval():
    rng = np.random.default_rng(1)
    x = rng.standard_normal((5, 16, 128)) * 7.0
    y = O.rotate(x)
    assert np.max(np.abs(O.rotate(y) - x)) <= 1e-12 * np.max(np.abs(x))
    assert np.allclose(np.sum(y * y, -1), np.sum(x * x, -1), rtol=1e-12, atol=0)
    # a single basis vector spreads evenly over all channels (outlier spreading)
    e = np.zeros(128); e[17] = 1.0
    assert np.allclose(np.abs(O.rotate(e)), 1 / math.sqrt(128), rtol=0, atol=1e-15)


# ---------------------------------------------------------------- Sinkhorn
@pytest.mark.parametrize("T", [16, 128])
def test_sinkhorn_closed_form_rank_one_scaling(T):
    # Z = diag(u) S diag(v) with S = +-1 reaches Y = S after one round,
    # with r_i c_j = u_i v_j.
    rng = np.random.default_rng(2)
    d = 128
    u = np.exp(rng.uniform(-2, 2, T))
    v = np.exp(rng.uniform(-2, 2, d))
    s = np.where(rng.random((T, d)) < 0.5, -1.0, 1.0)
    z = u[:, None] * s * v[None, :]
    for n in (1, 4):
        y, r, c = O.sinkhorn_normalize(z, n)
        assert np.max(np.abs(y - s)) < 1e-12
        assert np.max(np.abs(np.outer(r, c) / np.outer(u, v) - 1)) < 1e-12


def test_sinkhorn_golden_rank1():
    fx = _golden("tile_t2_d4_rank1.json")
    z = np.array(fx["z_rotated"])
    y, r, c = O.sinkhorn_normalize(z, fx["n_iter"])
    assert np.allclose(c, fx["c_normalisation"], rtol=1e-14, atol=0)   # before the stored balance
    s = np.array([[1, -1, 1, 1], [-1, 1, 1, -1]], dtype=float)
    assert np.allclose(y, s, rtol=0, atol=1e-14)


def test_sinkhorn_invariant_every_half_step():
    rng = np.random.default_rng(3)
    z = rng.standard_normal((16, 128)) * np.exp(rng.uniform(-3, 3, 128))
    hist = []
    O.sinkhorn_normalize(z, 5, history=hist)
    assert len(hist) == 10
    for y, r, c in hist:
        assert np.max(np.abs(r[:, None] * y * c[None, :] - z)) <= 1e-12 * np.max(np.abs(z))


def test_sinkhorn_uncentred_second_moment_not_variance():
    # rows with a large mean: the reading normalises the mean of squares,
    # so a centred variance would differ from 1 while the RMS is 1.
    rng = np.random.default_rng(4)
    z = rng.standard_normal((16, 128)) + 3.0
    y, _, _ = O.sinkhorn_normalize(z, 60)
    rms_rows = np.sqrt(np.mean(y * y, -1))
    assert np.max(np.abs(rms_rows - 1)) < 1e-9
    assert np.max(np.abs(np.var(y, -1) - 1)) > 0.5


def test_sinkhorn_order_rows_then_columns():
    # After any number of rounds the column step came last, so the columns are
    # exactly normalised while the rows are only close.
    rng = np.random.default_rng(5)
    z = rng.standard_normal((16, 128)) * np.exp(rng.uniform(-2, 2, (16, 1)))
    y, _, _ = O.sinkhorn_normalize(z, 2)
    assert np.max(np.abs(np.sqrt(np.mean(y * y, 0)) - 1)) < 1e-13
    assert np.max(np.abs(np.sqrt(np.mean(y * y, 1)) - 1)) > 1e-6


@pytest.mark.parametrize("name", ["rt1k", "gqa", "long", "prefill", "mla", "g128"])
def test_sinkhorn_converges_on_workload_distributions(name):
    # Row and column second moments equal 1 within 1e-6 after convergence,
    # on tiles drawn from each workload's distribution (with its tile length).
    w = W.WORKLOADS[name]
    small = w.scaled(batch=1, seq_len=max(w.tile_tokens, 64 if not w.mla else 32), num_layers=1)
    x = W.half_bits_to_f64(W.kv_inputs(small, "k"), w.in_dtype)      # [1, n, H, d]
    tiles = x[0].reshape(-1, w.tile_tokens, small.num_kv_heads, w.head_dim).transpose(0, 2, 1, 3)
    y, _, _ = O.sinkhorn_normalize(O.rotate(tiles), 50)
    assert np.max(np.abs(np.mean(y * y, -1) - 1)) < 1e-6
    assert np.max(np.abs(np.mean(y * y, -2) - 1)) < 1e-6


def test_sinkhorn_zero_rows_and_columns_untouched():
    z = np.zeros((16, 8))
    z[3, :] = np.arange(1, 9)
    y, r, c = O.sinkhorn_normalize(z, 4)
    assert np.all(np.isfinite(y))
    assert np.array_equal(np.delete(r, 3), np.ones(15))
    y0, r0, c0 = O.sinkhorn_normalize(np.zeros((16, 8)), 4)
    assert np.all(y0 == 0) and np.all(r0 == 1) and np.all(c0 == 1)


# ---------------------------------------------------------------- RTN
def test_rtn_golden_ties_to_even():
    fx = _golden("rtn_ties.json")
    q, m, s = O.rtn_rows(np.array(fx["y"]), fx["bits"])
    assert np.array_equal(q, fx["q"])
    assert np.array_equal(m, fx["m"]) and np.array_equal(s, fx["s"])


@pytest.mark.parametrize("bits", [2, 3, 4, 8])
def test_rtn_is_nearest_level_brute_force(bits):
    rng = np.random.default_rng(6 + bits)
    y = rng.standard_normal((64, 16))
    q, m, s = O.rtn_rows(y, bits)
    levels = np.arange(1 << bits)
    recon = m[:, None, None] + s[:, None, None] * levels[None, None, :]
    err = np.abs(y[:, :, None] - recon)
    best = np.argmin(err, axis=-1)            # first minimum; no exact ties here
    assert np.array_equal(q, best)
    assert np.all(np.abs(y - (m[:, None] + s[:, None] * q)) <= s[:, None] / 2 * (1 + 1e-12))
    assert np.all(q[np.arange(64), np.argmin(y, 1)] == 0)
    assert np.all(q[np.arange(64), np.argmax(y, 1)] == (1 << bits) - 1)


# ---------------------------------------------------------------- tiles
def test_quantize_golden_identity_tile():
    fx = _golden("tile_t2_d2_identity.json")
    qt = O.quantize_tiles(np.array(fx["x"]), fx["bits"], fx["n_iter"])
    assert np.array_equal(qt.q, fx["q"])
    for k in ("a", "z", "c"):
        assert np.array_equal(getattr(qt, k), np.array(fx[k], dtype=np.float32)), k
    xr = O.dequantize_tiles(qt.q, qt.a, qt.z, qt.c)
    assert np.max(np.abs(xr - np.array(fx["x"]))) < 1e-7


def test_quantize_golden_rank1_tile():
    fx = _golden("tile_t2_d4_rank1.json")
    x = O.rotate(np.array(fx["z_rotated"]))
    qt = O.quantize_tiles(x, fx["bits"], fx["n_iter"])
    assert np.array_equal(qt.q, fx["q"])
    for k in ("a", "z", "c"):
        assert np.allclose(getattr(qt, k), np.array(fx[k], dtype=np.float32), rtol=2e-7, atol=0), k


def test_quantize_homogeneity_and_token_permutation():
    rng = np.random.default_rng(7)
    x = rng.standard_normal((16, 128)) * np.exp(rng.uniform(-1, 1, 128))
    base = O.quantize_tiles(x, 4, 4)
    sc = O.quantize_tiles(x * 8.0, 4, 4)        # power of two: exact scaling
    assert np.array_equal(sc.q, base.q)
    assert np.array_equal(sc.a, base.a * 8) and np.array_equal(sc.z, base.z * 8)
    assert np.array_equal(sc.c, base.c)
    perm = rng.permutation(16)
    pm = O.quantize_tiles(x[perm], 4, 4)
    assert np.array_equal(pm.q, base.q[perm])
    assert np.allclose(pm.a, base.a[perm], rtol=1e-6) and np.allclose(pm.z, base.z[perm], rtol=1e-6)
    assert np.allclose(pm.c, base.c, rtol=1e-6)


def test_stored_scales_balanced_by_a_power_of_two():
    # The stored (a, z, c) are the textbook (r s, r m, c) with an exact power
    # of two 2^k moved from c into a and z, k chosen so that max c lies in
    # (1/2, 1]; the dequantised tile is bit-for-bit the unbalanced one.
    rng = np.random.default_rng(31)
    x = rng.standard_normal((40, 16, 128)) * np.exp(rng.uniform(-3, 3, (40, 1, 128)))
    x[:4] *= np.exp2(rng.integers(-40, 40, (4, 1, 1)))
    for n_iter in (0, 1, 4):
        qt = O.quantize_tiles(x, 4, n_iter)
        cmax = qt.c.max(-1).astype(np.float64)
        assert np.all(cmax > 0.5) and np.all(cmax <= 1.0)
        # unbalanced, from the pipeline's steps taken one by one
        y, r, c = O.sinkhorn_normalize(O.rotate(x), n_iter)
        q, m, st = O.rtn_rows(y, 4)
        a0, z0, c0 = (r * st).astype(np.float32), (r * m).astype(np.float32), c.astype(np.float32)
        assert np.array_equal(q, qt.q)
        k = np.log2(c0.max(-1).astype(np.float64) / cmax)
        assert np.array_equal(k, np.round(k))                      # a power of two per tile
        assert np.array_equal(O.dequantize_tiles(qt.q, qt.a, qt.z, qt.c, unrotate=False),
                              O.dequantize_tiles(q, a0, z0, c0, unrotate=False))
    # no normalisation: c = 1, already balanced (k = 0)
    qt = O.quantize_tiles(x, 4, 0)
    assert np.all(qt.c == 1.0)


def _f16_neighbours(v16):
    """The fp16 values just below and just above each fp16 value (brute force on the bit patterns)."""
    b = v16.astype(np.float16).view(np.uint16).astype(np.int64)
    up = np.where(b & 0x8000, b - 1, b + 1)           # toward +inf
    dn = np.where(b & 0x8000, b + 1, b - 1)           # toward -inf
    dn = np.where(b == 0, 0x8001, dn)                 # below +0: the smallest negative subnormal
    return up.astype(np.uint16).view(np.float16).astype(np.float64), dn.astype(np.uint16).view(np.float16).astype(np.float64)


def test_fp16_metadata_is_the_nearest_half_and_leaves_codes_alone():
    rng = np.random.default_rng(33)
    x = rng.standard_normal((24, 16, 128)) * np.exp(rng.uniform(-2, 2, (24, 1, 128)))
    for n_iter, bits in ((4, 4), (0, 3), (6, 2)):
        f32 = O.quantize_tiles(x, bits, n_iter)
        f16 = O.quantize_tiles(x, bits, n_iter, meta="f16")
        assert f16.a.dtype == np.float16 and f16.c.dtype == np.float16
        assert np.array_equal(f16.q, f32.q)                       # codes do not see the format
        _, a64, z64, c64 = O.quantize_stages(x, bits, n_iter)
        for got, exact in ((f16.a, a64), (f16.z, z64), (f16.c, c64)):
            g = got.astype(np.float64)
            up, dn = _f16_neighbours(got)
            err = np.abs(g - exact)
            assert np.all(err <= np.abs(up - exact)) and np.all(err <= np.abs(dn - exact))   # nearest half
        assert np.all(f16.c.astype(np.float64) <= 1.0) and np.all(f16.c.max(-1).astype(np.float64) >= 0.5)
        # dequantised with half scales: within 2^-10 (relative, per element bound) of the float32 ones
        d32 = O.dequantize_tiles(f32.q, f32.a, f32.z, f32.c, unrotate=False)
        d16 = O.dequantize_tiles(f16.q, f16.a, f16.z, f16.c, unrotate=False)
        bound = 2.0 ** -10 * (np.abs(f32.a)[..., None] * f32.q + np.abs(f32.z)[..., None] + 1e-30) * \
            f32.c.astype(np.float64)[..., None, :] * 1.5
        assert np.all(np.abs(d16 - d32) <= bound)


# ---------------------------------------------------------------- KIVI-style axes (ablation)
def test_block_one_rotation_is_the_identity():
    x = np.random.default_rng(41).standard_normal((3, 16, 128))
    assert np.array_equal(O.rotate(x, 1), x)
    assert np.array_equal(O.block_hadamard_matrix(128, 1), np.eye(128, dtype=np.int64))


def test_per_channel_golden():
    fx = _golden("tile_per_channel.json")
    t = O.quantize_tiles_per_channel(np.array(fx["x"]), fx["bits"], block=1)
    assert np.array_equal(t.q, fx["q"])
    assert np.allclose(t.s, np.array(fx["s"], np.float32), rtol=0, atol=0)
    assert np.array_equal(t.m, np.array(fx["m"], np.float32))
    assert np.allclose(O.dequantize_channel_tiles(t, unrotate=False, block=1), fx["x"], rtol=0, atol=1e-7)


@pytest.mark.parametrize("bits,block", [(2, 1), (4, 1), (3, 32), (8, 128)])
def test_per_channel_rtn_is_nearest_level_brute_force(bits, block):
    rng = np.random.default_rng(42)
    x = rng.standard_normal((6, 16, 128)) * np.exp(rng.uniform(-2, 2, (6, 1, 128)))
    t = O.quantize_tiles_per_channel(x, bits, block)
    z = O.rotate(x, block)
    s, m = t.s.astype(np.float64), t.m.astype(np.float64)
    levels = np.arange(1 << bits)
    # every code is the nearest level of its own channel's grid (the stored
    # float32 step and minimum reproduce it to float32 rounding)
    recon = m[..., None, :, None] + s[..., None, :, None] * levels
    best = np.argmin(np.abs(z[..., None] - recon), axis=-1)
    assert np.mean(best == t.q) > 0.9999
    assert np.all(np.abs(z - (m[..., None, :] + s[..., None, :] * t.q)) <= s[..., None, :] / 2 * (1 + 1e-5) + 1e-12)
    lo, hi = np.argmin(z, axis=-2), np.argmax(z, axis=-2)          # per channel
    assert np.all(np.take_along_axis(t.q, lo[..., None, :], -2) == 0)
    assert np.all(np.take_along_axis(t.q, hi[..., None, :], -2) == (1 << bits) - 1)


def test_attention_with_per_channel_keys_matches_torch_sdpa():
    torch = pytest.importorskip("torch")
    rng = np.random.default_rng(43)
    x = rng.standard_normal((2, 5, 16, 128))
    k = O.quantize_tiles_per_channel(x[0], 2, block=1)
    v = O.quantize_tiles(x[1], 2, 0, block=1)
    q = rng.standard_normal((4, 128))
    got = O.decode_attention(q, k, v, 0.1, block=1)
    kk = torch.from_numpy(O.dequantize_channel_tiles(k, unrotate=True, block=1).reshape(-1, 128))
    vv = torch.from_numpy(O.dequantize_tiles(v.q, v.a, v.z, v.c, unrotate=True, block=1).reshape(-1, 128))
    ref = torch.nn.functional.scaled_dot_product_attention(torch.from_numpy(q)[None], kk[None], vv[None],
                                                           scale=0.1)[0].numpy()
    assert np.max(np.abs(got - ref)) < 1e-12


def test_quantize_row_scale_invariance():
    # Scaling one token row by a power of two scales that row's a and z by it
    # and changes no code and no column factor: the row step divides it out
    # before any column step sees it.  Holds across the float range the input
    # formats reach.
    rng = np.random.default_rng(32)
    x = rng.standard_normal((16, 128)) * np.exp(rng.uniform(-1, 1, 128))
    base = O.quantize_tiles(x, 4, 4)
    f = np.ones(16)
    f[3], f[7], f[11] = 2.0 ** -64, 2.0 ** 60, 2.0 ** -100
    sc = O.quantize_tiles(x * f[:, None], 4, 4)
    assert np.array_equal(sc.q, base.q) and np.array_equal(sc.c, base.c)
    assert np.array_equal(sc.a, (base.a * f).astype(np.float32))
    assert np.array_equal(sc.z, (base.z * f).astype(np.float32))


@pytest.mark.parametrize("bits", [2, 3, 4, 8])
def test_dequantize_error_bound(bits):
    # In the rotated domain each element is off by at most half a step, times
    # the row and column factors (plus float32 rounding of a, z, c).
    rng = np.random.default_rng(8)
    x = rng.standard_normal((4, 16, 128)) * np.exp(rng.uniform(-1, 1, (4, 1, 128)))
    z = O.rotate(x)
    y, r, c = O.sinkhorn_normalize(z, 4)
    qt = O.quantize_tiles(x, bits, 4)
    zh = O.dequantize_tiles(qt.q, qt.a, qt.z, qt.c, unrotate=False)
    bound = (qt.a.astype(np.float64)[..., None] / 2 + 1e-6 * (np.abs(qt.a)[..., None] * (1 << bits) + np.abs(qt.z)[..., None])) \
        * qt.c.astype(np.float64)[..., None, :]
    assert np.all(np.abs(zh - z) <= bound)
    assert np.allclose(O.dequantize_tiles(qt.q, qt.a, qt.z, qt.c), O.rotate(zh), rtol=0, atol=1e-12)


def test_normalisation_does_not_hurt_on_outlier_rows():
    # Sanity of the method, not of parity: on tiles whose tokens have very
    # different scales the dual-axis normalisation keeps the error no worse
    # than rotation + RTN alone.
    rng = np.random.default_rng(9)
    x = rng.standard_t(4.0, (64, 16, 128)) * np.exp(rng.uniform(-2, 2, (64, 16, 1)))
    full = O.quantize_tiles(x, 4, 4)
    rot = O.quantize_tiles(x, 4, 0)
    e_full = np.mean((O.dequantize_tiles(full.q, full.a, full.z, full.c) - x) ** 2)
    e_rot = np.mean((O.dequantize_tiles(rot.q, rot.a, rot.z, rot.c) - x) ** 2)
    assert e_full <= 1.05 * e_rot


# ---------------------------------------------------------------- packing
def test_packing_golden():
    fx = _golden("packing.json")
    for case in fx["cases"]:
        q = np.array(case["q"])
        b = O.pack_codes(q, case["bits"])
        assert list(b) == case["bytes"], case["bits"]
        assert np.array_equal(O.unpack_codes(b, case["bits"], q.shape[0], q.shape[1]), q)


@pytest.mark.parametrize("T", [16, 128])
@pytest.mark.parametrize("bits", [2, 3, 4, 8])
def test_pack_unpack_roundtrip(bits, T):
    rng = np.random.default_rng(10)
    q = rng.integers(0, 1 << bits, size=(3, T, 128))
    b = O.pack_codes(q, bits)
    assert b.shape == (3, O.tile_code_bytes(bits, T, 128)) and b.dtype == np.uint8
    assert np.array_equal(O.unpack_codes(b, bits, T, 128), q)


def test_packing_three_bit_planes_span_the_page():
    # 128-token page, code 5 = 0b101 at token 127, channel 9: its low bits
    # sit in the low-bit plane's last row, its high bit in the high-bit plane
    # that starts after all 128 rows of the low plane (128 * 32 bytes).
    q = np.zeros((128, 128), dtype=np.int64)
    q[127, 9] = 5
    b = O.pack_codes(q, 3)
    nz = np.flatnonzero(b)
    assert list(nz) == [127 * 32 + 2, 128 * 32 + 127 * 16 + 1]
    assert b[127 * 32 + 2] == 0b01 << 2 and b[128 * 32 + 127 * 16 + 1] == 1 << 1


# ---------------------------------------------------------------- attention
def _random_cache(rng, n_tiles, d, bits_k=4, bits_v=4):
    xk = rng.standard_normal((n_tiles, 16, d)) * 2
    xv = rng.standard_normal((n_tiles, 16, d))
    return O.quantize_tiles(xk, bits_k, 4), O.quantize_tiles(xv, bits_v, 4)


def test_attention_matches_torch_sdpa_float64():
    import torch
    rng = np.random.default_rng(11)
    k, v = _random_cache(rng, 5, 128, 3, 4)
    q = rng.standard_normal((4, 128))
    scale = 1 / math.sqrt(128)
    o = O.decode_attention(q, k, v, scale)
    kh = O.dequantize_tiles(k.q, k.a, k.z, k.c).reshape(-1, 128)     # un-rotated
    vh = O.dequantize_tiles(v.q, v.a, v.z, v.c).reshape(-1, 128)
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q)[None, :, None, :], torch.from_numpy(kh)[None, None].expand(1, 4, -1, -1),
        torch.from_numpy(vh)[None, None].expand(1, 4, -1, -1), scale=scale)[0, :, 0, :].numpy()
    assert np.max(np.abs(o - ref)) <= 1e-12 * np.max(np.abs(ref))


def test_attention_single_token_and_identical_keys():
    rng = np.random.default_rng(12)
    k, v = _random_cache(rng, 1, 128)
    q = rng.standard_normal((2, 128))
    vh = O.dequantize_tiles(v.q, v.a, v.z, v.c).reshape(-1, 128)
    one = O.QuantizedTiles(k.q[:, :1], k.a[:, :1], k.z[:, :1], k.c)
    onev = O.QuantizedTiles(v.q[:, :1], v.a[:, :1], v.z[:, :1], v.c)
    assert np.allclose(O.decode_attention(q, one, onev, 0.1), vh[:1].repeat(2, 0), rtol=0, atol=1e-12)
    same = O.QuantizedTiles(np.repeat(k.q[:, :1], 16, 1), np.repeat(k.a[:, :1], 16, 1),
                            np.repeat(k.z[:, :1], 16, 1), k.c)
    o = O.decode_attention(q, same, v, 0.3)
    assert np.allclose(o, vh.mean(0)[None].repeat(2, 0), rtol=0, atol=1e-12)


def test_tail_attention_reduces_to_cache_attention_without_tail():
    # two formulations: rotated-domain attention on the cache vs the input-basis
    # attention with an empty tail
    rng = np.random.default_rng(31)
    k, v = _random_cache(rng, 5, 128, 3, 2)
    q = rng.standard_normal((4, 128))
    a = O.decode_attention(q, k, v, 1 / math.sqrt(128))
    b = O.decode_attention_with_tail(q, k, v, np.zeros((0, 128)), np.zeros((0, 128)), 1 / math.sqrt(128))
    assert np.max(np.abs(a - b)) < 1e-12


def test_tail_attention_matches_torch_sdpa_on_tail_only():
    import torch
    rng = np.random.default_rng(32)
    kt, vt = rng.standard_normal((11, 128)), rng.standard_normal((11, 128))
    q = rng.standard_normal((8, 128))
    o = O.decode_attention_with_tail(q, None, None, kt, vt, 0.09)
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q)[None, :, None], torch.from_numpy(kt)[None, None].expand(1, 8, 11, 128),
        torch.from_numpy(vt)[None, None].expand(1, 8, 11, 128), scale=0.09)[0, :, 0].numpy()
    assert np.max(np.abs(o - ref)) < 1e-12
    assert np.all(O.decode_attention_with_tail(q, None, None, np.zeros((0, 128)), np.zeros((0, 128)), 0.09) == 0)


def test_tail_attention_tokens_may_move_between_cache_and_tail():
    # the last tile's dequantised rows given as tail rows change nothing: the
    # result depends on the set of keys only
    rng = np.random.default_rng(33)
    k, v = _random_cache(rng, 4, 128)
    q = rng.standard_normal((2, 128))
    full = O.decode_attention_with_tail(q, k, v, np.zeros((0, 128)), np.zeros((0, 128)), 0.1)
    head = O.QuantizedTiles(k.q[:3], k.a[:3], k.z[:3], k.c[:3]), O.QuantizedTiles(v.q[:3], v.a[:3], v.z[:3], v.c[:3])
    kt = O.dequantize_tiles(k.q[3:], k.a[3:], k.z[3:], k.c[3:], unrotate=True)[0]
    vt = O.dequantize_tiles(v.q[3:], v.a[3:], v.z[3:], v.c[3:], unrotate=True)[0]
    moved = O.decode_attention_with_tail(q, head[0], head[1], kt, vt, 0.1)
    assert np.max(np.abs(full - moved)) < 1e-12


def test_mla_attention_matches_torch_sdpa_float64():
    import torch
    rng = np.random.default_rng(13)
    d, rd, H = 512, 64, 8
    lat = O.quantize_tiles(rng.standard_normal((3, 16, d)), 4, 4)
    rope = rng.standard_normal((48, rd))
    q = rng.standard_normal((H, d + rd))
    scale = 1 / math.sqrt(d + rd)
    o = O.mla_decode_attention(q, lat, rope, scale)
    ch = O.dequantize_tiles(lat.q, lat.a, lat.z, lat.c).reshape(-1, d)     # un-rotated latent
    key = np.concatenate([ch, rope], 1)
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q)[None, :, None, :], torch.from_numpy(key)[None, None].expand(1, H, -1, -1),
        torch.from_numpy(ch)[None, None].expand(1, H, -1, -1), scale=scale)[0, :, 0, :].numpy()
    assert np.max(np.abs(o - ref)) <= 1e-12 * np.max(np.abs(ref))


def test_mla_tail_attention_pins():
    # an empty tail gives the cache-only formula (rotated domain, 1e-12); no
    # cached tiles gives SDPA over the tail rows; moving the last tile's
    # dequantised rows into the tail changes nothing
    torch = pytest.importorskip("torch")
    rng = np.random.default_rng(44)
    d, rd, H = 512, 64, 8
    lat = O.quantize_tiles(rng.standard_normal((3, 16, d)), 4, 4)
    rope = rng.standard_normal((48, rd))
    q = rng.standard_normal((H, d + rd))
    base = O.mla_decode_attention(q, lat, rope, 0.04)
    got = O.mla_decode_attention_with_tail(q, lat, rope, np.zeros((0, d)), np.zeros((0, rd)), 0.04)
    assert np.max(np.abs(got - base)) < 1e-12
    lt, rt = rng.standard_normal((7, d)), rng.standard_normal((7, rd))
    only = O.mla_decode_attention_with_tail(q, None, None, lt, rt, 0.04)
    kk = torch.from_numpy(np.concatenate([lt, rt], 1))[None]
    ref = torch.nn.functional.scaled_dot_product_attention(torch.from_numpy(q)[None], kk,
                                                           torch.from_numpy(lt)[None], scale=0.04)[0].numpy()
    assert np.max(np.abs(only - ref)) < 1e-12
    rows = O.dequantize_tiles(lat.q[2], lat.a[2], lat.z[2], lat.c[2], unrotate=True)
    two = O.QuantizedTiles(lat.q[:2], lat.a[:2], lat.z[:2], lat.c[:2])
    moved = O.mla_decode_attention_with_tail(q, two, rope[:32], np.concatenate([rows, lt]),
                                             np.concatenate([rope[32:], rt]), 0.04)
    whole = O.mla_decode_attention_with_tail(q, lat, rope, lt, rt, 0.04)
    assert np.max(np.abs(moved - whole)) < 1e-12

