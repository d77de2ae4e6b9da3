"""Throughput of the KVarN-style hot path on B200: quantize-append + decode attention.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload long] [--impl kvq|reference]
                    [--no-extra] [--no-cpu-baseline]

One step = the whole hot path over one batch of the workload: every new K/V
row of the batch is rotated, normalised, quantised and packed into the paged
cache (kvq_quantize_append), then one decode step of attention runs over the
quantised cache (kvq_decode_attention, split-KV + combine).  The default
workload is the largest single-GPU one, long-context decode: 4 sequences x
131072 tokens, 8 kv / 64 query heads, head_dim 128, bf16 inputs (Student-t
keys), 3-bit K, 4-bit V, 6 normalisation rounds, 16-token pages.  The other
workloads (gqa, prefill, mla, the kvarn_k4v2_g128 preset, the saw4 ablation
and the rt1k round trip) are timed after it with fewer steps and reported
under "workloads" in the same line (--no-extra skips them).

value  = KV tokens quantized per second (all ranks; one token = all kv-heads'
         K and V rows of one position), inputs resident in HBM;
e2e    = the same through the C ABI with the step's inputs copied from pinned
         host memory and the attention output read back, inside the timing;
roofline = the quantize kernel (the larger share of the step's bytes) against
         the measured HBM copy bandwidth; decode_attn gives the decode kernel's
         algorithmic GB/s and fraction the same way.
Multi-GPU (torchrun): every rank runs its own shard (own batch, own seed), no
data-path collective; time = max over ranks.  --impl reference times the
float64 CPU oracle on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import dataclasses
import hashlib
import json
import math
import os
import re
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "KV tokens quantized/s; quantized decode-attn HBM GB/s and % of B200 peak"
UNIT = "tokens/s"


def load_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


def load_tensor_peak():
    """Dense f16/bf16 tensor peak for a kernel timed inside a long step (sustained)."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["bf16_tflops_sustained"]), "measured sustained"
    except Exception:
        return 1400.0, "fallback sustained"


def algorithmic_bytes(w):
    """(quantize bytes, decode bytes) one step must move, from the cache format."""
    T, d, H = w.tile_tokens, w.head_dim, w.num_kv_heads
    mb = 2 if w.meta_f16 else 4                           # bytes of one a, z or c
    if w.mla:
        lat_row = d * w.bits_k / 8 + 2 * mb + d * mb / T    # codes + (a, z) + channel-scale share
        rope_row = w.rope_dim * 2
        tokens = w.num_layers * w.n_tok
        q_bytes = tokens * (d * 2 + rope_row) + tokens * (lat_row + rope_row)
        dec_bytes = w.batch * w.seq_len * (lat_row + rope_row) + w.batch * w.num_q_heads * ((d + w.rope_dim) * 2 + d * 4)
        return q_bytes, dec_bytes
    rows = w.num_layers * w.n_tok * H
    per_row_in = d * 2
    def cache_row(bits):                       # codes + (a, z) + c share of one row
        return d * bits / 8 + 2 * mb + d * mb / T
    k_row = (d * w.bits_k / 8 + d * 2 * mb / T) if w.k_per_channel else cache_row(w.bits_k)  # (s, m) per channel
    q_bytes = rows * 2 * per_row_in + rows * (k_row + cache_row(w.bits_v))
    dec_bytes = w.batch * w.seq_len * H * (k_row + cache_row(w.bits_v)) \
        + w.batch * w.num_q_heads * d * (2 + 4)
    return q_bytes, dec_bytes


def fill_bytes(w, fill_tiles, tail_tokens):
    """Bytes a decode step with quantise-on-fill moves beyond the plain
    decode: the filled tails (input rows in, cache rows out) and the
    remaining tails' rows read by the attention."""
    mb = 2 if w.meta_f16 else 4
    d, T, H = w.head_dim, w.tile_tokens, w.num_kv_heads
    if w.mla:
        lat_row = d * w.bits_k / 8 + 2 * mb + d * mb / T
        rope = w.rope_dim * 2
        return fill_tiles * T * (d * 2 + rope + lat_row + rope) + tail_tokens * (d * 2 + rope)
    def cache_row(bits):
        return d * bits / 8 + 2 * mb + d * mb / T
    k_row = (d * w.bits_k / 8 + d * 2 * mb / T) if w.k_per_channel else cache_row(w.bits_k)
    return fill_tiles * T * H * (2 * d * 2 + k_row + cache_row(w.bits_v)) + tail_tokens * H * 2 * d * 2


def traffic_from_profile(kernel_file: str, profile_name: str):
    """DRAM bytes of one quantize-append call (the K and the V launch, or the latent launch) from a
    committed ncu summary, if the kernel source is unchanged since the counters were taken."""
    path = os.path.join(ROOT, "profiles", profile_name)
    src = os.path.join(ROOT, "kv_cache_quantization_03_b200", "csrc", kernel_file)
    try:
        txt = open(path).read()
        sha = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
        m = re.search(r"traffic_bytes_per_call:\s*([0-9.eE+]+)\s+source_sha256_16:\s*([0-9a-f]+)", txt)
        if m and m.group(2) == sha:
            return float(m.group(1))
    except OSError:
        pass
    return None


class ClockSampler:
    """Polls SM clock and throttle reasons through NVML while the timed region runs."""

    REASONS = {0x8: "hw_slowdown", 0x40: "hw_thermal_slowdown", 0x20: "sw_thermal_slowdown",
               0x4: "sw_power_cap", 0x80: "hw_power_brake_slowdown"}

    def __init__(self, index: int):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self._stop = threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self.nv = None

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                r = self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for bit, name in self.REASONS.items():
                    if r & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(0.002)

    def __enter__(self):
        if self.nv:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        if self.nv:
            self._stop.set()
            self.t.join()

    def summary(self):
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons), "samples": len(self.samples)}


# --------------------------------------------------------------------------- oracle leg
def oracle_sample_step(w, sample):
    """Float64 oracle over one (sequence, kv-head) of the workload: quantise its K
    and V rows, then decode its query group over the sequence.  Returns the token
    equivalents processed (positions x kv-heads / H_kv)."""
    import numpy as np
    from oracle import kvarn_oracle as O
    from kv_cache_quantization_03_b200 import workloads as W
    xk, xv, q = sample
    meta = "f16" if w.meta_f16 else "f32"
    kt = O.quantize_tiles_per_channel(xk, w.bits_k, w.block) if w.k_per_channel else \
        O.quantize_tiles(xk, w.bits_k, w.sinkhorn_iters, w.block, meta=meta)
    if w.mla:   # xv holds the rope keys
        O.mla_decode_attention(q, kt, xv, w.softmax_scale)
        return xk.shape[0] * xk.shape[1]
    vt = O.quantize_tiles(xv, w.bits_v, w.sinkhorn_iters, w.block, meta=meta)
    O.decode_attention(q, kt, vt, w.softmax_scale, block=w.block)
    return xk.shape[0] * xk.shape[1] / w.num_kv_heads


def oracle_sample_inputs(w, tokens):
    import numpy as np
    from kv_cache_quantization_03_b200 import workloads as W
    sub = slice(0, max(tokens, W.CHUNK_TOKENS))
    xk = W.half_bits_to_f64(W.kv_inputs(w, "k", sub)[0, :tokens, 0], w.in_dtype)
    xk = xk.reshape(-1, w.tile_tokens, w.head_dim)
    if w.mla:
        small = w.scaled(batch=1, seq_len=tokens)
        rope = W.half_bits_to_f64(W.rope_inputs(small)[0], "bf16")
        q = W.half_bits_to_f64(W.queries(w)[0], "bf16")
        return xk, rope, q
    xv = W.half_bits_to_f64(W.kv_inputs(w, "v", sub)[0, :tokens, 0], w.in_dtype)
    xv = xv.reshape(-1, w.tile_tokens, w.head_dim)
    q = W.half_bits_to_f64(W.queries(w)[0, :w.group], "bf16")
    return xk, xv, q


def blas_threads():
    """Threads the oracle's dense products run on (numpy's BLAS pool)."""
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return 1


def host_cpu():
    """(logical CPUs this process may use, CPU model name)."""
    try:
        n = len(os.sched_getaffinity(0))
    except AttributeError:
        n = os.cpu_count() or 1
    model = "unknown"
    try:
        with open("/proc/cpuinfo") as f:
            for ln in f:
                if ln.startswith("model name"):
                    model = ln.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return n, model


def cpu_baseline(w, budget_s=12.0, tokens=4096):
    sample = oracle_sample_inputs(w, tokens)
    t0 = time.perf_counter()
    done = 0.0
    n = 0
    while True:
        done += oracle_sample_step(w, sample)
        n += 1
        if time.perf_counter() - t0 >= budget_s:
            break
    dt = time.perf_counter() - t0
    nproc, model = host_cpu()
    return {"value": done / dt, "unit": UNIT, "cores": blas_threads(), "nproc": nproc, "cpu_model": model,
            "kind": "oracle",
            "sample": "%d x {quantize K and V of one kv-head over %d tokens of sequence 0 (float64, dense "
                      "Hadamard) + decode of its %d query heads over them}; %.1f s" % (n, tokens, w.group, dt)}


def run_reference(args, w):
    if rank_env()[1] != 0:       # under torchrun only rank 0 times the CPU oracle
        return
    tokens = 1024
    sample = oracle_sample_inputs(w, tokens)
    for _ in range(args.warmup):
        oracle_sample_step(w, sample)
    t0 = time.perf_counter()
    done = 0.0
    for _ in range(args.steps):
        done += oracle_sample_step(w, sample)
    dt = time.perf_counter() - t0
    v = done / dt
    line = {"metric": METRIC, "value": v, "unit": UNIT, "impl": "reference", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * dt / max(args.steps, 1),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": config_dict(w, args),
            "cpu_baseline": {"value": v, "unit": UNIT, "cores": blas_threads(), "nproc": host_cpu()[0],
                             "cpu_model": host_cpu()[1], "kind": "oracle",
                             "sample": "each step: one kv-head of sequence 0, %d tokens: quantize K and V + "
                                       "decode of its %d query heads (float64 oracle)" % (tokens, w.group)},
            "e2e": {"value": v, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line))


def config_dict(w, args):
    return {"workload": w.name, "description": w.description, "batch": w.batch, "seq_len": w.seq_len,
            "num_kv_heads": w.num_kv_heads, "num_q_heads": w.num_q_heads, "head_dim": w.head_dim,
            "bits_k": w.bits_k, "bits_v": w.bits_v, "tile_tokens": w.tile_tokens,
            "sinkhorn_iters": w.sinkhorn_iters, "hadamard_block": w.hadamard_block or w.head_dim,
            "metadata": "f16" if w.meta_f16 else "f32", "key_groups": "channel" if w.k_per_channel else "token",
            "layers": w.num_layers,
            "parallelism": "dp%d (independent shards)" % args.gpus,
            "l2": ("inputs larger than L2 (latent + rope bf16 %.2f GB per rank)" % (
                w.num_layers * w.n_tok * (w.head_dim + w.rope_dim) * 2 / 1e9)) if w.mla else
                  ("inputs larger than L2 (K+V bf16 %.2f GB per rank)" % (
                      2 * w.num_layers * w.n_tok * w.num_kv_heads * w.head_dim * 2 / 1e9))}


# --------------------------------------------------------------------------- ranks
def rank_env():
    """(world, rank, local_rank) from the torchrun environment (1, 0, 0 alone)."""
    return (int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")),
            int(os.environ.get("LOCAL_RANK", "0")))


def shard(w, rank: int):
    """This rank's shard of a weak-scaling run: the same shape with its own
    batch of sequences (a seed of its own); ranks share nothing."""
    return dataclasses.replace(w, seed=w.seed + 7919 * rank)


def max_over_ranks(values, world: int, device=None):
    """Element-wise max of a list of floats over all ranks (the slowest rank
    sets the time); a no-op for one rank."""
    if world <= 1:
        return list(values)
    import torch
    import torch.distributed as dist
    t = torch.tensor(values, dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


# --------------------------------------------------------------------------- GPU leg
QUANTIZE_ONLY = ("prefill",)       # workloads whose step is quantise-append alone
EXTRA_WORKLOADS = ("gqa", "gqa16", "prefill", "mla", "g128", "saw4", "hadonly", "kivi", "rt1k")


def kernel_names(w):
    """(quantize kernel, decode kernels) as launched for the workload."""
    if w.mla:
        return "quantize_kernel<D=512>", "mla_prep_q + decode_mla (tcgen05) + combine_mla"
    return "quantize_kernel<D=128, T=%d>" % w.tile_tokens, "decode_d128 + combine_d128"


def graph_time(fns, steps):
    """Mean device time (s) of one replay of the calls fns(sp=stream), captured
    once into a CUDA graph.  A sleep kernel queued first lets the host enqueue
    every replay before the first one runs, so the time is the graph's own:
    its kernels and the gaps between them, without host launch costs."""
    import torch

    g = torch.cuda.CUDAGraph()
    cap = torch.cuda.Stream()
    cap.wait_stream(torch.cuda.current_stream())
    with torch.cuda.graph(g, stream=cap, capture_error_mode="relaxed"):
        for f in fns:
            f(sp=cap.cuda_stream)
    stream = torch.cuda.current_stream()
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    torch.cuda._sleep(2_000_000)
    for a, b in ev:
        a.record(stream)
        g.replay()
        b.record(stream)
    torch.cuda.synchronize()
    t = sum(a.elapsed_time(b) for a, b in ev) / steps / 1e3
    del g
    return t


def measure(w, steps, warmup, rank=0, world=1, local=0, e2e=True, clocks=False, graph=False):
    """Times `steps` steps of workload w on this rank's GPU (CUDA events on the
    launching stream).  Returns a dict of seconds and byte counts.  With
    graph, the step (and the decode alone) is also timed as a replayed CUDA
    graph."""
    import numpy as np
    import torch

    from kv_cache_quantization_03_b200 import kvq, workloads as W
    from kv_cache_quantization_03_b200.cache import QuantizedCache

    ws = shard(w, rank)
    q_only = any(w.name == n or w.name.startswith(n + "-") for n in QUANTIZE_ONLY)
    cfg = kvq.make_config(head_dim=w.head_dim, num_kv_heads=w.num_kv_heads, tile_tokens=w.tile_tokens,
                          bits_k=w.bits_k, bits_v=w.bits_v, sinkhorn_iters=w.sinkhorn_iters, mla=w.mla,
                          rope_dim=w.rope_dim, num_layers=w.num_layers, num_pages=w.num_pages, in_dtype=w.in_dtype,
                          hadamard_block=w.hadamard_block or None, meta_f16=w.meta_f16,
                          k_per_channel=w.k_per_channel)
    cache = QuantizedCache(cfg)
    host = {"k": torch.from_numpy(W.kv_inputs(ws, "k").view(np.int16))}
    if w.mla:
        host["rope"] = torch.from_numpy(W.rope_inputs(ws).view(np.int16))
    else:
        host["v"] = torch.from_numpy(W.kv_inputs(ws, "v").view(np.int16))
    host["dst"] = torch.from_numpy(W.page_assignment(ws))
    if not q_only:
        host.update({"q": torch.from_numpy(W.queries(ws).view(np.int16)),
                     "bt": torch.from_numpy(np.ascontiguousarray(W.block_table(ws))),
                     "sl": torch.from_numpy(W.seq_lens(ws))})
    if e2e:
        host = {k: v.pin_memory() for k, v in host.items()}
    dev = {k: v.cuda() for k, v in host.items()}
    out = torch.empty(w.batch, w.num_q_heads, w.head_dim, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    ws_bytes = kvq.kvq_decode_workspace_bytes(cfg, w.batch, w.num_q_heads, w.seq_len)
    work = torch.empty(max(ws_bytes, 256), dtype=torch.uint8, device="cuda")
    stream = torch.cuda.current_stream()
    s_ptr = stream.cuda_stream

    def quantize(d=dev, sp=None):
        kvq.kvq_quantize_append(cfg, cache.view, d["k"], d.get("v"), d.get("rope"), w.n_tok, d["dst"], err,
                                s_ptr if sp is None else sp)

    def decode(d=dev, sp=None):
        if not q_only:
            kvq.kvq_decode_attention(cfg, cache.view, 0, d["q"], d["bt"], w.tiles_per_seq, d["sl"], w.batch,
                                     w.num_q_heads, w.softmax_scale, out, work, ws_bytes, err,
                                     s_ptr if sp is None else sp)

    for _ in range(max(warmup, 3)):
        quantize()
        decode()
    torch.cuda.synchronize()
    st, bits = kvq.kvq_read_error(err, s_ptr)
    if st != kvq.KVQ_OK or bits:
        raise RuntimeError("device error word %#x after warm-up" % bits)

    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(steps)]
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    torch.cuda.synchronize()
    clk = ClockSampler(local) if clocks else None
    if clk:
        clk.__enter__()
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    start.record(stream)
    for i in range(steps):
        ev[i][0].record(stream)
        quantize()
        ev[i][1].record(stream)
        decode()
        ev[i][2].record(stream)
    end.record(stream)
    torch.cuda.synchronize()
    if clk:
        clk.__exit__()
    if world > 1:
        dist.barrier()
    r = {"elapsed": start.elapsed_time(end) / 1e3,
         "t_q": sum(e[0].elapsed_time(e[1]) for e in ev) / steps / 1e3,
         "t_d": sum(e[1].elapsed_time(e[2]) for e in ev) / steps / 1e3,
         "q_only": q_only, "clocks": clk.summary() if clk else None}
    if graph:
        r["graph_step_s"] = graph_time([quantize, decode], steps)
        if not q_only:
            r["graph_decode_s"] = graph_time([decode], steps)

    if e2e:  # inputs from pinned host memory, output back to the host, each step
        # Two input buffers, as a serving loop would keep them: the copy of
        # step i + 1's inputs (on a copy stream) overlaps step i's kernels;
        # every step's copy lies inside the timed region.
        out_host = torch.empty_like(out, device="cpu").pin_memory()
        Ke = max(1, min(steps, 10))
        bufs = [dev, {k: torch.empty_like(v) for k, v in dev.items()}]
        cstream = torch.cuda.Stream()
        copied = [torch.cuda.Event() for _ in range(Ke)]
        done = [torch.cuda.Event() for _ in range(Ke)]

        def load(i):
            with torch.cuda.stream(cstream):
                if i >= 2:
                    cstream.wait_event(done[i - 2])  # step i - 2 has read this buffer
                for k in host:
                    bufs[i % 2][k].copy_(host[k], non_blocking=True)
                copied[i].record(cstream)

        torch.cuda.synchronize()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        cstream.wait_event(e0)  # the first copy starts inside the timed region
        load(0)
        for i in range(Ke):
            if i + 1 < Ke:
                load(i + 1)
            stream.wait_event(copied[i])
            quantize(bufs[i % 2])
            decode(bufs[i % 2])
            out_host.copy_(out, non_blocking=True)
            done[i].record(stream)
        e1.record(stream)
        torch.cuda.synchronize()
        r["e2e_s"] = e0.elapsed_time(e1) / 1e3 / Ke
        r["h2d"] = sum(host[k].numel() * host[k].element_size() for k in host)
        r["d2h"] = out.numel() * out.element_size()
    if not q_only:
        r.update(measure_fill(w, ws, cfg, cache, dev, out, work, ws_bytes, err, stream, steps))
    st, bits = kvq.kvq_read_error(err, s_ptr)
    if st != kvq.KVQ_OK or bits:
        raise RuntimeError("device error word %#x" % bits)
    del cache, dev, host, work, out
    torch.cuda.empty_cache()
    return r


def fill_state(ws):
    """A decode step of the serving reading with unquantised tails: every
    sequence b with b % 16 == 0 has just filled its tail (quantised into the
    last page of its block table row, which the step's decode then reads);
    the others keep a tail of tail_lens[b] < T tokens.  Returns (tail_lens,
    fill_page) as int32 arrays."""
    import numpy as np

    from kv_cache_quantization_03_b200 import workloads as W

    tl = W.tail_lens(ws).copy()
    bt = W.block_table(ws)
    fill = np.full(ws.batch, -1, dtype=np.int32)
    for b in range(0, ws.batch, 16):
        tl[b] = 0
        fill[b] = bt[b, ws.tiles_per_seq - 1]
    return tl, fill


def measure_fill(w, ws, cfg, cache, dev, out, work, ws_bytes, err, stream, steps):
    """Times kvq_decode_attention_fill (decode-time append): the filled tails
    are quantised into their pages and attention runs over the cached pages
    plus the remaining tails, in one call."""
    import numpy as np
    import torch

    from kv_cache_quantization_03_b200 import kvq, workloads as W

    tl, fill = fill_state(ws)
    kt = torch.from_numpy(W.tail_inputs(ws, "k").view(np.int16)).cuda()
    vt = torch.from_numpy((W.tail_rope_inputs(ws) if w.mla else W.tail_inputs(ws, "v")).view(np.int16)).cuda()
    tl_d, fill_d = torch.from_numpy(tl).cuda(), torch.from_numpy(fill).cuda()
    s_ptr = stream.cuda_stream

    def step():
        kvq.kvq_decode_attention_fill(cfg, cache.view, 0, dev["q"], dev["bt"], w.tiles_per_seq, dev["sl"], kt, vt,
                                      tl_d, fill_d, w.batch, w.num_q_heads, w.softmax_scale, out, work, ws_bytes,
                                      err, s_ptr)

    for _ in range(3):
        step()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    e0.record(stream)
    for _ in range(steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    return {"t_f": e0.elapsed_time(e1) / 1e3 / steps, "fill_tiles": int((fill >= 0).sum()),
            "tail_tokens": int(tl.sum())}


def summarize(w, r, peak, world=1):
    """Per-kernel throughput of one measured workload."""
    qb_bytes, db_bytes = algorithmic_bytes(w)
    t_q, t_d = r["t_q"], r["t_d"]
    qk, dk = kernel_names(w)
    q_gbs = qb_bytes / t_q / 1e9
    res = {"ms_per_step": 1e3 * r["elapsed"] / max(r.get("steps", 1), 1),
           "quantize": {"kernel": qk, "us": 1e6 * t_q, "gbs": q_gbs, "frac_of_measured": q_gbs / peak,
                        "frac_of_8tbs": q_gbs / 8000.0, "algorithmic_bytes": qb_bytes,
                        "rows_per_s": w.num_layers * w.n_tok * w.num_kv_heads * (1 if w.mla else 2) / t_q}}
    if not r["q_only"]:
        d_gbs = db_bytes / t_d / 1e9
        res["decode_attn"] = {"kernel": dk, "us": 1e6 * t_d, "gbs": d_gbs, "frac_of_measured": d_gbs / peak,
                              "frac_of_8tbs": d_gbs / 8000.0, "algorithmic_bytes": db_bytes}
        if "t_f" in r:  # decode-time append: filled tails quantised, then decode over cache + tails
            fb = fill_bytes(w, r["fill_tiles"], r["tail_tokens"])
            res["decode_fill"] = {"us": 1e6 * r["t_f"], "filled_pages": r["fill_tiles"],
                                  "tail_tokens": r["tail_tokens"], "algorithmic_bytes": db_bytes + fb,
                                  "gbs": (db_bytes + fb) / r["t_f"] / 1e9,
                                  "frac_of_measured": (db_bytes + fb) / r["t_f"] / 1e9 / peak}
        if w.mla:   # 128 heads share every latent: a dense contraction, tensor-bound
            flops = 2.0 * w.batch * w.seq_len * w.num_q_heads * (w.head_dim + w.rope_dim + w.head_dim)
            tf = flops / t_d / 1e12
            tpeak, tsrc = load_tensor_peak()
            res["decode_attn"].update({"tflops": tf, "frac_of_tensor_peak": tf / tpeak, "tensor_peak": tpeak,
                                       "tensor_peak_source": tsrc, "flops": flops})
    return res


def run_gpu(args, w):
    import torch
    import torch.distributed as dist

    world, rank, local = rank_env()
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    K = args.steps
    r = measure(w, K, args.warmup, rank, world, local, e2e=True, clocks=True)
    elapsed, e2e_s, t_q, t_d, t_f = max_over_ranks([r["elapsed"], r["e2e_s"], r["t_q"], r["t_d"], r.get("t_f", 0.0)],
                                                   world, device="cuda")
    r.update({"elapsed": elapsed, "e2e_s": e2e_s, "t_q": t_q, "t_d": t_d, "steps": K})
    if "t_f" in r:
        r["t_f"] = t_f
    if world > 1:
        dist.destroy_process_group()
    if rank != 0:
        return

    tokens = w.batch * w.seq_len * world
    peak, peak_kind = load_peaks()
    summ = summarize(w, r, peak, world)
    qb_bytes, _ = algorithmic_bytes(w)
    qk, dk = kernel_names(w)
    profile = "quantize_d512_mla.md" if w.mla else "quantize_d128_%s.md" % w.name
    traffic = traffic_from_profile("quantize.cu", profile)
    line = {
        "metric": METRIC, "value": tokens * K / elapsed, "unit": UNIT, "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": 1e3 * elapsed / K, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32", "data": "synthetic (seeded; see workloads.py)",
        "config": config_dict(w, args),
        "roofline": {"kernel": qk, "bound": "hbm", "achieved": summ["quantize"]["gbs"], "peak": peak,
                     "unit": "GB/s", "frac": summ["quantize"]["gbs"] / peak, "peak_source": peak_kind,
                     "traffic": traffic, "algorithmic_bytes": qb_bytes,
                     "per": "one quantize-append call (the K and the V launch; MLA: the latent launch)"},
        "quantize": summ["quantize"],
        "e2e": {"value": tokens / e2e_s, "unit": UNIT, "h2d_bytes_per_step": r["h2d"], "d2h_bytes_per_step": r["d2h"]},
        # quantize: one launch per quantised stream (latent, or K and V); decode:
        # decode + combine (MLA: query prep + decode + combine)
        "gpu_launches": (1 if w.mla else 2) * K + (0 if r["q_only"] else (3 if w.mla else 2) * K),
        "clocks": r["clocks"],
    }
    if "decode_attn" in summ:
        line["decode_attn"] = summ["decode_attn"]
        line["decode_fill"] = summ["decode_fill"]
        if w.mla and t_d >= t_q:
            d = summ["decode_attn"]
            line["roofline"] = {"kernel": dk, "bound": "tensor", "achieved": d["tflops"], "peak": d["tensor_peak"],
                                "unit": "TFLOP/s", "frac": d["frac_of_tensor_peak"],
                                "peak_source": d["tensor_peak_source"] + " bf16 dense (f16 same rate)",
                                "traffic": None, "algorithmic_flops": d["flops"]}
    if world == 1 and not args.no_extra:
        extra = {}
        for name in EXTRA_WORKLOADS:
            if name == w.name:
                continue
            wx = W_WORKLOADS()[name]
            rx = measure(wx, min(K, 10), 3, e2e=False, graph=(name == "rt1k"))
            rx["steps"] = min(K, 10)
            sx = summarize(wx, rx, peak)
            sx["tokens_per_s"] = wx.batch * wx.seq_len / (rx["elapsed"] / rx["steps"])
            if name == "rt1k":
                sx["note"] = "L2-resident: latency, not a roofline figure"
            if "graph_step_s" in rx:  # the same step replayed as one CUDA graph (no host cost per launch)
                n_launch = (1 if wx.mla else 2) + (0 if rx["q_only"] else (3 if wx.mla else 2))
                sx["graph"] = {"step_us": 1e6 * rx["graph_step_s"], "launches_per_step": n_launch,
                               "note": "device time per replay of the step captured as one CUDA graph"}
                if "graph_decode_s" in rx:
                    sx["graph"]["decode_us"] = 1e6 * rx["graph_decode_s"]
            extra[name] = sx
        line["workloads"] = extra
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w)
    print(json.dumps(line))


def W_WORKLOADS():
    from kv_cache_quantization_03_b200 import workloads as W
    return W.WORKLOADS


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="long")
    ap.add_argument("--impl", default="kvq", choices=["kvq", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extra", action="store_true", help="time the chosen workload only")
    ap.add_argument("--batch", type=int, default=None, help="override the batch (profiling small cases)")
    ap.add_argument("--seq-len", type=int, default=None, help="override the context length")
    args = ap.parse_args()
    from kv_cache_quantization_03_b200 import workloads as W
    w = W.WORKLOADS[args.workload]
    if args.batch or args.seq_len:
        w = w.scaled(batch=args.batch, seq_len=args.seq_len, name="%s-b%d-l%d" % (
            w.name, args.batch or w.batch, args.seq_len or w.seq_len))
    if not w.mla and w.num_q_heads // w.num_kv_heads > 8:
        raise SystemExit("GQA decode covers query groups of up to 8 heads")
    if args.impl == "reference":
        run_reference(args, w)
    else:
        run_gpu(args, w)


if __name__ == "__main__":
    main()
