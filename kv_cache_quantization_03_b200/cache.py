"""Device memory for a quantised cache, allocated with torch (plumbing only).

Every array is a flat uint8/float32/bf16 torch tensor sized by
kvq_cache_layout; ``view`` is the kvq_cache_view the C ABI takes.
"""
from __future__ import annotations

import torch

from . import kvq

NAMES = ("k_codes", "k_tok_scale", "k_chan_scale", "v_codes", "v_tok_scale", "v_chan_scale", "rope")


class QuantizedCache:
    def __init__(self, cfg: "kvq.kvq_config", device="cuda"):
        self.cfg = cfg
        sizes = kvq.kvq_cache_layout(cfg)
        self.arrays = {}
        for name, nbytes in zip(NAMES, sizes):
            if nbytes == 0:
                self.arrays[name] = None
            elif name.endswith("codes"):
                self.arrays[name] = torch.zeros(nbytes, dtype=torch.uint8, device=device)
            elif name == "rope":
                self.arrays[name] = torch.zeros(nbytes // 2, dtype=torch.bfloat16, device=device)
            elif cfg.meta_f16:     # a, z, c as IEEE half
                self.arrays[name] = torch.zeros(nbytes // 2, dtype=torch.float16, device=device)
            else:
                self.arrays[name] = torch.zeros(nbytes // 4, dtype=torch.float32, device=device)
        self.view = kvq.make_view([self.arrays[n] for n in NAMES])

    def __getitem__(self, name):
        return self.arrays[name]

    def slot_shape(self):
        c = self.cfg
        return (c.num_layers, c.num_pages, c.num_kv_heads)

    def codes(self, which="k"):
        """Codes as [layers][pages][heads][bytes per tile] (a view, no copy)."""
        c = self.cfg
        bits = c.bits_k if which == "k" else c.bits_v
        return self.arrays[which + "_codes"].view(*self.slot_shape(), c.tile_tokens * c.head_dim * bits // 8)

    def tok_scale(self, which="k"):
        """Group scales: (a, z) per token [..][T][2], or, for per-channel keys, (s, m) per channel [..][d][2]."""
        c = self.cfg
        groups = c.head_dim if (which == "k" and c.k_per_channel) else c.tile_tokens
        return self.arrays[which + "_tok_scale"].view(*self.slot_shape(), groups, 2)

    def chan_scale(self, which="k"):
        c = self.cfg
        return self.arrays[which + "_chan_scale"].view(*self.slot_shape(), c.head_dim)
