"""Host-side checks of the C ABI: the library loads without a GPU, exports
every function include/kvq.h declares, and rejects bad arguments before any
launch (these calls never reach the device)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def kvq():
    from kv_cache_quantization_03_b200 import build
    build.build()
    from kv_cache_quantization_03_b200 import kvq as k
    return k


def _declared():
    txt = open(os.path.join(ROOT, "include", "kvq.h")).read()
    return sorted(set(re.findall(r"^\s*(?:const\s+)?[\w\s\*]*?\b(kvq_\w+)\s*\(", txt, re.M)))


def test_every_declared_symbol_is_exported(kvq):
    names = _declared()
    assert len(names) >= 9
    for n in names:
        assert hasattr(kvq.lib, n), n
    assert set(names) == set(kvq.EXPORTED)


def test_status_strings_and_version(kvq):
    assert kvq.status_string(kvq.KVQ_OK) == "KVQ_OK"
    assert kvq.status_string(kvq.KVQ_ERR_WORKSPACE_TOO_SMALL) == "KVQ_ERR_WORKSPACE_TOO_SMALL"
    assert kvq.kvq_version().count(".") == 2


def test_config_from_string(kvq):
    c = kvq.make_config()
    kvq.kvq_config_from_string("kvarn_k4v2_g128", c)
    assert (c.bits_k, c.bits_v, c.tile_tokens) == (4, 2, 128)
    for bad in ("kvarn_k5v2_g128", "kvarn_k4v2_g100", "kvarn_k4v2", "k4v2_g128", "kvarn_k4v2_g128x"):
        assert kvq.kvq_config_from_string(bad, c, raise_on_error=False) == kvq.KVQ_ERR_INVALID_ARG


def test_cache_layout_sizes(kvq):
    c = kvq.make_config(num_kv_heads=8, num_layers=2, num_pages=10, bits_k=3, bits_v=4)
    sizes = kvq.kvq_cache_layout(c)
    n = 2 * 10 * 8
    assert sizes == [n * 16 * 128 * 3 // 8, n * 16 * 2 * 4, n * 128 * 4, n * 16 * 128 * 4 // 8,
                     n * 16 * 2 * 4, n * 128 * 4, 0]
    m = kvq.make_config(head_dim=512, num_kv_heads=1, mla=True, rope_dim=64, num_pages=4)
    s = kvq.kvq_cache_layout(m)
    assert s[3:6] == [0, 0, 0] and s[6] == 4 * 16 * 64 * 2 and s[0] == 4 * 16 * 512 // 2
    # half-precision metadata: a, z, c take two bytes each, codes unchanged
    h = kvq.make_config(num_kv_heads=8, num_layers=2, num_pages=10, bits_k=3, bits_v=4, meta_f16=True)
    assert kvq.kvq_cache_layout(h) == [n * 16 * 128 * 3 // 8, n * 16 * 2 * 2, n * 128 * 2, n * 16 * 128 * 4 // 8,
                                       n * 16 * 2 * 2, n * 128 * 2, 0]
    bad = kvq.make_config(num_pages=4)
    bad.meta_f16 = 2
    with pytest.raises(kvq.KvqError):
        kvq.kvq_cache_layout(bad)
    # per-channel keys (KIVI-style axes): (s, m) per channel, no key c
    kc = kvq.make_config(num_kv_heads=8, num_layers=2, num_pages=10, bits_k=2, bits_v=2, sinkhorn_iters=0,
                         hadamard_block=1, k_per_channel=True)
    assert kvq.kvq_cache_layout(kc) == [n * 16 * 128 * 2 // 8, n * 128 * 2 * 4, 0, n * 16 * 128 * 2 // 8,
                                        n * 16 * 2 * 4, n * 128 * 4, 0]
    for kw in (dict(sinkhorn_iters=4), dict(mla=True, head_dim=512, num_kv_heads=1, rope_dim=64)):
        bad = kvq.make_config(num_pages=4, k_per_channel=True, **kw)
        with pytest.raises(kvq.KvqError):
            kvq.kvq_cache_layout(bad)


def test_invalid_configs_rejected(kvq):
    for kw in (dict(head_dim=96), dict(bits_k=5), dict(bits_v=1), dict(num_kv_heads=0),
               dict(tile_tokens=12), dict(sinkhorn_iters=-1), dict(in_dtype=7)):
        c = kvq.make_config(num_pages=4, **kw)
        with pytest.raises(kvq.KvqError):
            kvq.kvq_cache_layout(c)
    out = (ctypes.c_size_t * 7)()
    for blk, want in ((64, kvq.KVQ_OK), (8, kvq.KVQ_OK), (4, kvq.KVQ_OK), (1, kvq.KVQ_OK),
                      (48, kvq.KVQ_ERR_INVALID_ARG), (256, kvq.KVQ_ERR_INVALID_ARG), (0, kvq.KVQ_ERR_INVALID_ARG)):
        c = kvq.make_config(num_pages=4, hadamard_block=blk)
        assert kvq.lib.kvq_cache_layout(ctypes.byref(c), out) == want, blk
    m = kvq.make_config(head_dim=512, num_kv_heads=1, mla=True, rope_dim=64, num_pages=4, hadamard_block=128)
    assert kvq.lib.kvq_cache_layout(ctypes.byref(m), out) == kvq.KVQ_ERR_UNSUPPORTED  # the latent rotates in full


def test_host_rejections_before_launch(kvq):
    c = kvq.make_config(num_kv_heads=2, num_pages=8)
    fake = 1 << 20                       # aligned non-null "device" pointers; never dereferenced
    view = kvq.make_view([fake] * 6 + [None])
    f = kvq.kvq_quantize_append
    assert f(c, view, fake, fake, None, 17, fake, fake, 0, raise_on_error=False) == kvq.KVQ_ERR_PARTIAL_TILE
    assert f(c, view, None, fake, None, 16, fake, fake, 0, raise_on_error=False) == kvq.KVQ_ERR_INVALID_ARG
    assert f(c, view, fake + 2, fake, None, 16, fake, fake, 0, raise_on_error=False) == kvq.KVQ_ERR_INVALID_ARG
    bad_view = kvq.make_view([fake, None] + [fake] * 4 + [None])
    assert f(c, bad_view, fake, fake, None, 16, fake, fake, 0, raise_on_error=False) == kvq.KVQ_ERR_INVALID_ARG
    d512 = kvq.make_config(head_dim=256, num_kv_heads=2, num_pages=8)
    assert f(d512, view, fake, fake, None, 16, fake, fake, 0, raise_on_error=False) == kvq.KVQ_ERR_UNSUPPORTED
    assert f(c, view, fake, fake, None, 0, fake, fake, 0, raise_on_error=False) == kvq.KVQ_OK
    # tile ids are 32-bit in the kernel: 2 kinds x 2 kv-heads x 2^29 tiles = 2^31 tiles is refused
    assert f(c, view, fake, fake, None, 1 << 33, fake, fake, 0, raise_on_error=False) == kvq.KVQ_ERR_UNSUPPORTED
    dec = kvq.kvq_decode_attention
    ws = kvq.kvq_decode_workspace_bytes(c, 4, 8, 1024)
    assert ws > 0
    assert dec(c, view, 0, fake, fake, 64, fake, 4, 8, 0.1, fake, fake, ws - 1, fake, 0,
               raise_on_error=False) == kvq.KVQ_ERR_WORKSPACE_TOO_SMALL
    ws18 = kvq.kvq_decode_workspace_bytes(c, 4, 18, 1024)
    assert dec(c, view, 0, fake, fake, 64, fake, 4, 18, 0.1, fake, fake, ws18, fake, 0,
               raise_on_error=False) == kvq.KVQ_ERR_UNSUPPORTED       # group 9 > 8
    assert dec(c, view, 0, fake, fake, 64, fake, 4, 5, 0.1, fake, fake, ws, fake, 0,
               raise_on_error=False) == kvq.KVQ_ERR_INVALID_ARG       # 5 q heads over 2 kv heads
    assert dec(c, view, 0, fake, fake, 64, fake, 4, 8, 0.1, fake + 4, fake, ws, fake, 0,
               raise_on_error=False) == kvq.KVQ_ERR_INVALID_ARG       # out not 16-byte aligned
    assert dec(c, view, 0, fake, fake, 64, fake, 4, 8, float("nan"), fake, fake, ws, fake, 0,
               raise_on_error=False) == kvq.KVQ_ERR_INVALID_ARG
    assert dec(c, view, 1, fake, fake, 64, fake, 4, 8, 0.1, fake, fake, ws, fake, 0,
               raise_on_error=False) == kvq.KVQ_ERR_INVALID_ARG       # layer out of range
    assert dec(c, view, 0, fake, fake, 64, fake, 0, 8, 0.1, fake, fake, ws, fake, 0,
               raise_on_error=False) == kvq.KVQ_OK                    # empty batch: nothing to do
    # per-channel keys: no key c array needed; 16-token tiles and 2/4/8-bit keys only
    kc = kvq.make_config(num_kv_heads=2, num_pages=8, bits_k=2, bits_v=2, sinkhorn_iters=0, hadamard_block=1,
                         k_per_channel=True)
    no_kc = kvq.make_view([fake, fake, None, fake, fake, fake, None])
    assert f(kc, no_kc, fake, fake, None, 0, fake, fake, 0, raise_on_error=False) == kvq.KVQ_OK
    for kw in (dict(tile_tokens=32), dict(bits_k=3)):
        k2 = kvq.make_config(num_kv_heads=2, num_pages=8, bits_v=2, sinkhorn_iters=0, k_per_channel=True,
                             **dict(dict(bits_k=2), **kw))
        assert f(k2, no_kc, fake, fake, None, 32, fake, fake, 0, raise_on_error=False) == kvq.KVQ_ERR_UNSUPPORTED


def test_tile_lengths_accepted_and_rejected(kvq):
    # head_dim 128 caches take 16..128-token tiles; the MLA latent 16 only
    fake = 1 << 20
    view = kvq.make_view([fake] * 6 + [None])
    f = kvq.kvq_quantize_append
    for T, want in ((8, kvq.KVQ_ERR_UNSUPPORTED), (16, kvq.KVQ_OK), (32, kvq.KVQ_OK), (128, kvq.KVQ_OK),
                    (256, kvq.KVQ_ERR_UNSUPPORTED)):
        c = kvq.make_config(num_kv_heads=2, num_pages=8, tile_tokens=T)
        assert f(c, view, fake, fake, None, 0, fake, fake, 0, raise_on_error=False) == want, T
        assert f(c, view, fake, fake, None, T // 2, fake, fake, 0, raise_on_error=False) == kvq.KVQ_ERR_PARTIAL_TILE
    m = kvq.make_config(head_dim=512, num_kv_heads=1, mla=1, rope_dim=64, num_pages=8, tile_tokens=128)
    mview = kvq.make_view([fake] * 3 + [None] * 3 + [fake])
    assert f(m, mview, fake, None, fake, 0, fake, fake, 0, raise_on_error=False) == kvq.KVQ_ERR_UNSUPPORTED


def test_tail_entry_host_rejections(kvq):
    # checked before any launch: missing or misaligned tail buffers, MLA caches
    fake = 1 << 20
    c = kvq.make_config(num_kv_heads=2, num_pages=8)
    view = kvq.make_view([fake] * 6 + [None])
    ws = kvq.kvq_decode_workspace_bytes(c, 4, 8, 1024)
    f = kvq.kvq_decode_attention_tail
    args = (0, fake, fake, 64, fake)
    assert f(c, view, *args, None, fake, fake, 4, 8, 0.1, fake, fake, ws, fake, 0,
             raise_on_error=False) == kvq.KVQ_ERR_INVALID_ARG
    assert f(c, view, *args, fake, fake, None, 4, 8, 0.1, fake, fake, ws, fake, 0,
             raise_on_error=False) == kvq.KVQ_ERR_INVALID_ARG
    assert f(c, view, *args, fake + 8, fake, fake, 4, 8, 0.1, fake, fake, ws, fake, 0,
             raise_on_error=False) == kvq.KVQ_ERR_INVALID_ARG
    assert f(c, view, *args, fake, fake, fake, 4, 8, 0.1, fake, fake, ws - 1, fake, 0,
             raise_on_error=False) == kvq.KVQ_ERR_WORKSPACE_TOO_SMALL
    assert f(c, view, *args, None, None, None, 0, 8, 0.1, fake, fake, ws, fake, 0,
             raise_on_error=False) == kvq.KVQ_OK                     # empty batch: nothing to do
    # MLA caches take a tail too (latent rows + rope keys); their checks run before any launch
    m = kvq.make_config(head_dim=512, num_kv_heads=1, mla=True, rope_dim=64, num_pages=8)
    mview = kvq.make_view([fake] * 3 + [None] * 3 + [fake])
    assert f(m, mview, *args, fake, fake + 8, fake, 4, 128, 0.1, fake, fake, 1 << 30, fake, 0,
             raise_on_error=False) == kvq.KVQ_ERR_INVALID_ARG          # misaligned rope tail
    assert f(m, mview, *args, fake, fake, fake, 4, 128, 0.1, fake, fake, 16, fake, 0,
             raise_on_error=False) == kvq.KVQ_ERR_WORKSPACE_TOO_SMALL
    g = kvq.kvq_decode_attention_fill    # the fill call: every check before the fill's launch
    for mm, vv, heads in ((c, view, 8), (m, mview, 128)):
        assert g(mm, vv, *args, fake, fake, fake, None, 4, heads, 0.1, fake, fake, 1 << 30, fake, 0,
                 raise_on_error=False) == kvq.KVQ_ERR_INVALID_ARG      # no fill pages
        assert g(mm, vv, *args, fake, fake, fake, fake, 4, heads, 0.1, fake, fake, 16, fake, 0,
                 raise_on_error=False) == kvq.KVQ_ERR_WORKSPACE_TOO_SMALL
    assert g(c, view, 0, fake, fake, 64, fake, fake, fake, fake, fake, 0, 8, 0.1, fake, fake, 0, fake, 0,
             raise_on_error=False) == kvq.KVQ_OK                       # empty batch


def test_decode_workspace_counts_16_token_tiles(kvq):
    # decode works on 16-token tiles whatever the page length, so the split
    # plan (and the workspace) depends on the context length only
    for seq in (128, 1024, 8192, 131072):
        sizes = {T: kvq.kvq_decode_workspace_bytes(kvq.make_config(num_kv_heads=8, num_pages=8, tile_tokens=T),
                                                   32, 32, seq) for T in (16, 32, 64, 128)}
        assert len(set(sizes.values())) == 1, (seq, sizes)


def test_decode_split_plan(kvq):
    # The split count, read back from the workspace size (batch x kv-heads x
    # splits x 8 head slots x (d + 2) floats), on a 148-SM sizing (no device
    # here): a short sequence spreads its tiles down to one per warp, the
    # combine's share per split stops it at two per warp for 4096 tokens,
    # and once the grid is full the wave count decides.
    import torch
    if torch.cuda.is_available() and torch.cuda.get_device_properties(0).multi_processor_count != 148:
        pytest.skip("split plans are sized by the SM count")

    def splits(batch, seq, kv, hq, T=16):
        c = kvq.make_config(num_kv_heads=kv, num_pages=8, tile_tokens=T)
        return kvq.kvq_decode_workspace_bytes(c, batch, hq, seq) / (batch * kv * 8 * 130 * 4)

    assert splits(1, 64, 1, 1) == 1            # 4 tiles: one per warp of one CTA
    assert splits(1, 1024, 1, 1) == 16         # 64 tiles: one per warp
    assert splits(1, 4096, 1, 1) == 32         # 256 tiles: two per warp
    assert splits(3, 512, 8, 32) == 8          # 12 kv-head pairs (two per CTA), 32 tiles each
    assert splits(32, 8192, 8, 32) == 4        # 128 kv-head pairs x 4 = 512 CTAs of 592 slots
    assert splits(32, 8192, 8, 32, T=128) == 4  # 128-token pages: the same 16-token tiles
    assert splits(4, 131072, 8, 64) == 18      # 32 kv-heads (one per CTA) x 18 = 576 CTAs of 592


def test_binding_fails_loudly_without_library(tmp_path):
    # the product path has no CPU fallback: without libkvq.so the binding refuses to import
    import shutil
    import subprocess
    import sys
    pkg = tmp_path / "kv_cache_quantization_03_b200"
    pkg.mkdir()
    src = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "kv_cache_quantization_03_b200")
    for name in ("__init__.py", "kvq.py"):
        shutil.copy(os.path.join(src, name), pkg / name)
    r = subprocess.run([sys.executable, "-c", "import kv_cache_quantization_03_b200.kvq"], cwd=tmp_path,
                       capture_output=True, text=True)
    assert r.returncode != 0 and "ImportError" in r.stderr and "libkvq.so is not built" in r.stderr


def test_header_is_plain_c_and_links(tmp_path, kvq):
    # include/kvq.h compiles as C99 and a C program calls the library through it (host-only calls)
    import shutil
    import subprocess
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("no C compiler")
    src = tmp_path / "abi.c"
    src.write_text(r"""
#include <stdio.h>
#include <string.h>
#include "kvq.h"
int main(void) {
  kvq_config c;
  size_t sizes[7];
  memset(&c, 0, sizeof c);
  c.head_dim = 128; c.num_kv_heads = 8; c.sinkhorn_iters = 4; c.hadamard_block = 128;
  c.num_layers = 2; c.num_pages = 10; c.in_dtype = KVQ_BF16;
  if (kvq_config_from_string("kvarn_k4v2_g128", &c) != KVQ_OK) return 1;
  if (c.bits_k != 4 || c.bits_v != 2 || c.tile_tokens != 128) return 2;
  if (kvq_cache_layout(&c, sizes) != KVQ_OK) return 3;
  printf("%s %zu %zu %zu\n", kvq_version(), sizes[0], sizes[3], sizeof(kvq_config));
  return strcmp(kvq_status_string(KVQ_ERR_PARTIAL_TILE), "KVQ_ERR_PARTIAL_TILE") != 0;
}
""")
    lib = os.path.join(ROOT, "kv_cache_quantization_03_b200", "libkvq.so")
    exe = tmp_path / "abi"
    r = subprocess.run([gcc, "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"), str(src), lib,
                        "-Wl,-rpath," + os.path.dirname(lib), "-o", str(exe)], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([str(exe)], capture_output=True, text=True)
    assert r.returncode == 0, (r.returncode, r.stdout, r.stderr)
    n = 2 * 10 * 8
    assert r.stdout.split()[1:] == [str(n * 128 * 128 * 4 // 8), str(n * 128 * 128 * 2 // 8),
                                     str(ctypes.sizeof(kvq.kvq_config))]     # the binding's struct is the header's
