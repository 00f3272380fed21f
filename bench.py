"""Benchmark of attention over a cross-layer shared KV cache on B200.

Default workload (one step = one decode step over all 22 layers of the
1.1B-shaped CLA2 model: 32 q / 4 kv heads, d 64, bf16, batch 32, context
2048). Secondary lines time the DepthGraft pair-mix decode (24 layers, 16/4
heads, d 128, batch 16, context 8192).

Timing: W untimed warm-up steps, then K timed steps between a barrier +
synchronize on both sides. One step is one replay of a CUDA graph holding every
layer's decode launch (consecutive launches overlap through programmatic
dependent launch), bracketed by CUDA events on the launching stream. L2 (126
MB) is flushed before every step, outside the events; inside the step the
layers run in "cold order" (every first reader of a source before any second
reader), so a layer's source was last read hundreds of MB earlier and comes
from HBM, as in a full model whose weights stream through L2 between the two
layers of a pair. Secondary figures: the same step in model order, and
`cold_layer_*` (every layer alone between its own events, L2 flushed before
each). Step time is the mean over the K steps, max over ranks. `e2e` times the
host-buffer entry point (q H2D, decode, out and lse D2H) in the same cold order.

--impl reference times the fp64 CPU oracle (the reference arm) on a bounded
sample of the same workload on the host cores.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from synth.configs import BY_NAME, LOWRANK, MIX  # noqa: E402

METRIC = "decode tok/s and KV GB/s (% of HBM peak); prefill TFLOP/s, 1×B200"

# ncu dram__bytes_read.sum + dram__bytes_write.sum per launch of the dominant kernel,
# for the kernel as currently built (None until captured for this build): mean over the
# 22 launches of one replayed step, captured without cache control
# (ncu --metrics dram__bytes_read.sum,dram__bytes_write.sum,gpu__time_duration.sum
#  --cache-control none --clock-control none -k regex:decode_bf16 -s 88 -c 22
#  python bench.py --steps 1 --warmup 3 --no-secondary --no-cpu-baseline):
# 67,244,079 B read + 953,519 B written
NCU_TRAFFIC_BYTES = {"cla2_1p1b": 68197597}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), float(d.get("bf16_tflops_sustained", d["bf16_tflops"])), "measured"
    return 6650.0, 1590.0, 1400.0, "fallback"


def decode_read_bytes(cfg, l):
    """Algorithmic bytes one decode layer reads: its source(s)' K and V."""
    kind = cfg.layer_map[l][0]
    nsrc = 2 if kind == 1 else 1
    es = 4 if cfg.dtype == "f32" else 2
    return nsrc * 2 * cfg.batch * cfg.kv_heads * cfg.context * cfg.head_dim * es


class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        self.dev = device_index
        self.rows = []
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.dev), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.rows.append([x.strip() for x in line.split(",")])

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        if not self.rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"]}
        sm = [float(r[1]) for r in self.rows if len(r) > 8 and r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in self.rows if len(r) > 8 and r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = set()
        for r in self.rows:
            for n, v in zip(names, r[5:9]):
                if v.strip().lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted(reasons), "samples": len(self.rows)}


# ----------------------------------------------------------------------------- GPU arm
class DecodeRunner:
    def __init__(self, cfg, K, torch, sgpu):
        self.cfg, self.K, self.torch = cfg, K, torch
        self.dev = {n: sgpu.make_device(cfg, n) for n in cfg.recipe()}
        _, self.h = K.kvshare_create(cfg.layers, cfg.q_heads, cfg.kv_heads, cfg.head_dim,
                                     K.KVS_F32 if cfg.dtype == "f32" else K.KVS_BF16, cfg.batch, cfg.context,
                                     basis_rank=cfg.basis_rank)
        self.w = None if cfg.lowrank else cfg.make("w")
        K.kvshare_set_map(self.h, cfg.layer_map, self.w)
        # nothing writes the cache while the timed steps run, so consecutive decode
        # launches may request their first K/V tiles before the previous one finishes
        K.kvshare_set_kv_overlap(self.h, True)
        self.out = torch.empty(cfg.layers, cfg.batch, cfg.q_heads, cfg.head_dim, device="cuda")
        self.lse = torch.empty(cfg.layers, cfg.batch, cfg.q_heads, device="cuda")
        self.stream = torch.cuda.current_stream()
        l2 = torch.cuda.get_device_properties(0).L2_cache_size
        self.flush_buf = torch.empty(2 * l2, dtype=torch.int8, device="cuda")
        self.flush_read = torch.ones(2 * l2 // 4, dtype=torch.float32, device="cuda")
        self.pack_ms = None
        if cfg.lowrank:
            d = self.dev
            L, B, T, Hkv = cfg.layers, cfg.batch, cfg.context, cfg.kv_heads
            self.rank = torch.empty((L, B, T), dtype=torch.uint8, device="cuda")
            self.ck = torch.empty((L, B, Hkv, T, 16), dtype=torch.int8, device="cuda")
            self.cv = torch.empty_like(self.ck)
            self.sk = torch.empty((L, B, Hkv, T), dtype=torch.int16, device="cuda")
            self.sv = torch.empty_like(self.sk)
            times = []
            for i in range(4):
                self.flush()
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record(self.stream)
                K.kvshare_pack_residual(self.h, d["score"], d["u_k"], d["u_v"], self.rank, self.ck, self.cv,
                                        self.sk, self.sv, B, T, self.stream)
                e1.record(self.stream)
                times.append((e0, e1))
            torch.cuda.synchronize()
            self.pack_ms = statistics.median([a.elapsed_time(b) for a, b in times[1:]])
            self.pack_bytes = (d["u_k"].numel() * 4 * 2 + d["score"].numel() * 4 + self.rank.numel()
                               + self.ck.numel() * 2 + self.sk.numel() * 2 * 2)
            del d["u_k"], d["u_v"]
            self.cache = K.Cache(batch=B, context=T, coef_k=d["coef_k"], coef_v=d["coef_v"], basis_k=d["basis_k"],
                                 basis_v=d["basis_v"], u_k=self.ck, u_v=self.cv, s_k=self.sk, s_v=self.sv,
                                 r_k=d["r_k"], r_v=d["r_v"], rank=self.rank, pairs=cfg.pairs)
            # algorithmic bytes per layer: coefficients, codes at each token's rank, scales of
            # tokens with rank > 0, the rank byte, bases and residual factors
            r = self.rank.to(torch.int64)
            per_layer_codes = (2 * Hkv * r.sum(dim=(1, 2))).cpu().numpy()
            per_layer_scales = (2 * 2 * Hkv * (r > 0).sum(dim=(1, 2))).cpu().numpy()
            fixed = (2 * B * Hkv * T * cfg.basis_rank * 2 + B * T + 2 * Hkv * cfg.basis_rank * cfg.head_dim * 2
                     + 2 * Hkv * 16 * cfg.head_dim * 2)
            self.layer_bytes = [int(fixed + per_layer_codes[l] + per_layer_scales[l]) for l in range(L)]
        else:
            self.cache = K.Cache(batch=cfg.batch, context=cfg.context, k=self.dev["k"], v=self.dev["v"],
                                 slots=cfg.slots)
            self.layer_bytes = [decode_read_bytes(cfg, l) for l in range(cfg.layers)]

    def flush(self):
        # evict the cache by writing 2x L2, then read another 2x L2 so the lines left are
        # clean: the timed kernel neither hits L2 nor pays for the flush's write-backs
        self.flush_buf.fill_(1)
        self._sink = self.flush_read.sum()

    def layer(self, l):
        self.K.kvshare_decode(self.h, self.cache, self.dev["q"], self.out, self.lse, l, l + 1, self.stream)

    def all_layers(self):
        self.K.kvshare_decode(self.h, self.cache, self.dev["q"], self.out, self.lse, 0, self.cfg.layers,
                              self.stream)

    def capture_step(self):
        """One decode step (every layer once, in cold_order) captured as a CUDA graph."""
        torch, K = self.torch, self.K
        self.order = cold_order(self.cfg)
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            for l in self.order:      # one eager pass first: attributes and tensor maps are set up
                K.kvshare_decode(self.h, self.cache, self.dev["q"], self.out, self.lse, l, l + 1, side)
        torch.cuda.current_stream().wait_stream(side)
        torch.cuda.synchronize()
        self.graph = torch.cuda.CUDAGraph()
        n0 = K.kvshare_launch_count(self.h)
        with torch.cuda.graph(self.graph, capture_error_mode="thread_local"):
            cap = torch.cuda.current_stream()
            for l in self.order:
                K.kvshare_decode(self.h, self.cache, self.dev["q"], self.out, self.lse, l, l + 1, cap)
        self.graph_launches = K.kvshare_launch_count(self.h) - n0
        torch.cuda.synchronize()

    def step_graph(self):
        self.graph.replay()

    def step_flushed(self, events=None):
        torch = self.torch
        for l in range(self.cfg.layers):
            self.flush()
            if events is not None:
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record(self.stream)
                self.layer(l)
                e1.record(self.stream)
                events.append((l, e0, e1))
            else:
                self.layer(l)

    def close(self):
        self.K.kvshare_destroy(self.h)


def cold_order(cfg):
    """Order of the layers inside a timed step: by how many earlier layers read one of the
    layer's sources (store slot, or basis pair for the low-rank form), then by index. For
    adjacent sharing this issues every first reader of a source before any second reader,
    so the source a layer reads was last read several hundred MB of other reads ago and
    comes from HBM, not L2, as in a full model where each layer's weights stream through
    L2 between two layers sharing a source. Each layer's attention depends only on its own
    q and sources, so the order changes no result."""
    seen = {}
    rank = []
    for kind, s0, s1 in cfg.layer_map:
        keys = [("pair", s0)] if kind == LOWRANK else [("slot", s0)] + ([("slot", s1)] if kind == MIX else [])
        rank.append(max(seen.get(k, 0) for k in keys))
        for k in keys:
            seen[k] = seen.get(k, 0) + 1
    return sorted(range(len(cfg.layer_map)), key=lambda l: (rank[l], l))


def gpu_arm(args, cfg_name, secondary=False):
    import torch
    import synth.gpu as sgpu
    from cross_layer_kv_shared_b200 import kvshare as K

    cfg = BY_NAME[cfg_name]
    r = DecodeRunner(cfg, K, torch, sgpu)

    # one decode step = every layer once, back to back (consecutive launches overlap
    # through programmatic dependent launch), replayed from a CUDA graph; L2 is flushed
    # before the step outside its events, and the layer order keeps shared sources cold
    r.capture_step()

    def step(events=None):
        r.flush()
        if events is None:
            r.step_graph()
            return
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(r.stream)
        r.step_graph()
        e1.record(r.stream)
        events.append((e0, e1))

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if dist_on():
        import torch.distributed as dist
        dist.barrier()
    torch.cuda.synchronize()
    n0 = K.kvshare_launch_count(r.h)
    events = []
    with ClockSampler(torch.cuda.current_device()) as clk:
        t_wall = time.perf_counter()
        for _ in range(args.steps):
            step(events)
        torch.cuda.synchronize()
        t_wall = time.perf_counter() - t_wall
    if dist_on():
        import torch.distributed as dist
        dist.barrier()
    torch.cuda.synchronize()
    launches = r.graph_launches * args.steps + (K.kvshare_launch_count(r.h) - n0)
    st = K.kvshare_sync_status(r.h)
    assert st == K.KVS_OK, K.kvshare_status_string(st)
    step_ms = sum(a.elapsed_time(b) for a, b in events) / len(events)
    step_ms = max_over_ranks(step_ms)

    # secondary: the step in model order, one call for all layers; a layer that shares a
    # source with the layer before it may find that source in L2
    K.kvshare_set_layer_order(r.h, None)
    io = []
    for i in range(3 + max(3, args.steps // 2)):
        r.flush()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(r.stream)
        r.all_layers()
        e1.record(r.stream)
        if i >= 3:
            io.append((e0, e1))
    torch.cuda.synchronize()
    in_order_ms = statistics.median([a.elapsed_time(b) for a, b in io])

    # secondary: every layer alone on a cold L2 (flushed before each layer, one launch
    # between its own events), so no layer can find a shared source in L2
    for _ in range(2):
        r.step_flushed()
    torch.cuda.synchronize()
    cold = []
    for _ in range(max(3, args.steps // 2)):
        r.step_flushed(cold)
    torch.cuda.synchronize()
    per_layer = np.zeros(cfg.layers)
    for l, e0, e1 in cold:
        per_layer[l] += e0.elapsed_time(e1)
    per_layer /= max(3, args.steps // 2)
    cold_ms = float(per_layer.sum())

    # e2e through the host-buffer entry point: q H2D + decode + out/lse D2H, the layers
    # in the same cold order as the device-timed step
    K.kvshare_set_layer_order(r.h, r.order)
    q_host = r.dev["q"].cpu().pin_memory()
    out_host = torch.empty(r.out.shape, dtype=torch.float32).pin_memory()
    lse_host = torch.empty(r.lse.shape, dtype=torch.float32).pin_memory()
    e2e = []
    for i in range(args.warmup + args.steps):
        r.flush()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(r.stream)
        K.kvshare_decode_host(r.h, r.cache, q_host, out_host, lse_host, 0, cfg.layers, r.stream)
        e1.record(r.stream)
        if i >= args.warmup:
            e2e.append((e0, e1))
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(statistics.median([a.elapsed_time(b) for a, b in e2e]))

    extra = lowrank_extras(args, r, cfg, K, torch) if cfg.lowrank else {}

    read_bytes = sum(r.layer_bytes)
    res = {
        "cfg": cfg, "step_ms": step_ms, "per_layer_ms": per_layer, "launches": launches,
        "kv_gbs": read_bytes / (step_ms * 1e-3) / 1e9, "tok_s": cfg.batch / (step_ms * 1e-3),
        "cold_layer_ms": cold_ms, "in_order_ms": in_order_ms, "e2e_ms": e2e_ms, "wall_s": t_wall, "clocks": clk.summary(),
        "h2d": q_host.numel() * q_host.element_size(),
        "d2h": out_host.numel() * 4 + lse_host.numel() * 4,
        "read_bytes": read_bytes, "pack_ms": r.pack_ms,
        "pack_bytes": getattr(r, "pack_bytes", None), "extra": extra,
    }
    r.close()
    del r
    torch.cuda.empty_cache()
    return res


def lowrank_extras(args, r, cfg, K, torch):
    """The low-rank workload's other per-step paths: the decode step with the router's
    attention statistics (one statistics kernel after every layer), and the append of one
    new token to every layer's cache (coefficients, residual codes, scales, ranks)."""
    L, B, Hq, Hkv, T, d = cfg.layers, cfg.batch, cfg.q_heads, cfg.kv_heads, cfg.context, cfg.head_dim
    mass = torch.empty((L, B, Hkv, T), device="cuda")
    score = torch.empty((L, B, T), device="cuda")
    ent = torch.empty((L, B, Hq), device="cuda")
    peak = torch.empty((L, B, Hq), device="cuda")
    order = cold_order(cfg)
    for l in order:   # eager pass first: the score buffer is allocated and the kernels set up
        K.kvshare_decode_stats(r.h, r.cache, r.dev["q"], r.out, r.lse, mass, score, ent, peak, l, l + 1, r.stream)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, capture_error_mode="thread_local"):
        cap = torch.cuda.current_stream()
        for l in order:
            K.kvshare_decode_stats(r.h, r.cache, r.dev["q"], r.out, r.lse, mass, score, ent, peak, l, l + 1, cap)
    ev = []
    for i in range(3 + max(5, args.steps // 2)):
        r.flush()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(r.stream)
        graph.replay()
        e1.record(r.stream)
        if i >= 3:
            ev.append((e0, e1))
    torch.cuda.synchronize()
    stats_ms = statistics.median([a.elapsed_time(b) for a, b in ev])
    del graph
    # append: the new token of every layer written at the last position of the store
    gen = torch.Generator(device="cuda").manual_seed(7)
    k_new = torch.randn((L, B, Hkv, d), device="cuda", generator=gen).to(torch.bfloat16)
    v_new = torch.randn((L, B, Hkv, d), device="cuda", generator=gen).to(torch.bfloat16)
    sc_new = torch.rand((L, B), device="cuda", generator=gen)
    pos = torch.full((B,), T - 1, dtype=torch.int32, device="cuda")
    app = []
    for i in range(13):
        r.flush()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(r.stream)
        K.kvshare_append_lowrank(r.h, r.cache, k_new, v_new, sc_new, pos, r.stream)
        e1.record(r.stream)
        if i >= 3:
            app.append((e0, e1))
    torch.cuda.synchronize()
    st = K.kvshare_sync_status(r.h)
    assert st == K.KVS_OK, K.kvshare_status_string(st)
    append_us = statistics.median([a.elapsed_time(b) for a, b in app]) * 1e3
    return {"stats_ms_per_step": stats_ms, "append_us_per_token": append_us}


def ragged_arm(args, cfg_name="cla2_1p1b"):
    """The 1.1B CLA2 decode step with per-sequence lengths drawn uniformly from 1..T (seeded):
    bytes read = each layer's source K and V over every sequence's own tokens."""
    import torch
    import synth.gpu as sgpu
    from cross_layer_kv_shared_b200 import kvshare as K
    cfg = BY_NAME[cfg_name]
    r = DecodeRunner(cfg, K, torch, sgpu)
    rng = np.random.default_rng(cfg.seed)
    lens = rng.integers(1, cfg.context + 1, size=cfg.batch).astype(np.int32)
    r.cache.lengths = torch.from_numpy(lens).cuda()
    r.capture_step()
    ev = []
    for i in range(3 + max(5, args.steps)):
        r.flush()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(r.stream)
        r.step_graph()
        e1.record(r.stream)
        if i >= 3:
            ev.append((e0, e1))
    torch.cuda.synchronize()
    st = K.kvshare_sync_status(r.h)
    assert st == K.KVS_OK, K.kvshare_status_string(st)
    ms = statistics.mean([a.elapsed_time(b) for a, b in ev])
    es = 4 if cfg.dtype == "f32" else 2
    read = sum((2 if cfg.layer_map[l][0] == MIX else 1) * 2 * cfg.kv_heads * cfg.head_dim * es * int(lens.sum())
               for l in range(cfg.layers))
    r.close()
    del r
    torch.cuda.empty_cache()
    return {"ms_per_step": ms, "tok_s": cfg.batch / (ms * 1e-3), "kv_gbs": read / (ms * 1e-3) / 1e9,
            "algorithmic_bytes_per_step": read, "mean_length": float(lens.mean()),
            "lengths": "uniform on 1..%d, seeded" % cfg.context}


def prefill_flops(cfg):
    """Causal prefill FLOPs credited per step: 2 * B * Hq * w * S^2 per layer (QK^T + PV,
    causal half), with w = d, or for a low-rank layer the absorbed operand width
    Rb + 16 = 48 (the MMAs run padded to 64; the padding is not credited)."""
    w = cfg.basis_rank + cfg.max_resid_rank if cfg.lowrank else cfg.head_dim
    return 2.0 * cfg.batch * cfg.q_heads * w * cfg.context ** 2 * cfg.layers


def prefill_arm(args, cfg_name="depthgraft_prefill"):
    """Times kvshare_prefill over all layers; per-layer CUDA events, no L2 flush (tensor-bound)."""
    import torch
    import synth.gpu as sgpu
    from cross_layer_kv_shared_b200 import kvshare as K

    cfg = BY_NAME[cfg_name]
    dev = {n: sgpu.make_device(cfg, n) for n in cfg.recipe()}
    _, h = K.kvshare_create(cfg.layers, cfg.q_heads, cfg.kv_heads, cfg.head_dim, K.KVS_BF16, cfg.batch, cfg.context)
    K.kvshare_set_map(h, cfg.layer_map, None if cfg.lowrank else cfg.make("w"))
    S = cfg.context
    out = torch.empty((cfg.layers, cfg.batch, cfg.q_heads, S, cfg.head_dim), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((cfg.layers, cfg.batch, cfg.q_heads, S), device="cuda")
    if cfg.lowrank:
        L, B, Hkv = cfg.layers, cfg.batch, cfg.kv_heads
        rank = torch.empty((L, B, S), dtype=torch.uint8, device="cuda")
        ck = torch.empty((L, B, Hkv, S, 16), dtype=torch.int8, device="cuda")
        cv = torch.empty_like(ck)
        sk = torch.empty((L, B, Hkv, S), dtype=torch.int16, device="cuda")
        sv = torch.empty_like(sk)
        K.kvshare_pack_residual(h, dev["score"], dev["u_k"], dev["u_v"], rank, ck, cv, sk, sv, B, S)
        cache = K.Cache(batch=B, context=S, coef_k=dev["coef_k"], coef_v=dev["coef_v"], basis_k=dev["basis_k"],
                        basis_v=dev["basis_v"], u_k=ck, u_v=cv, s_k=sk, s_v=sv, r_k=dev["r_k"], r_v=dev["r_v"],
                        rank=rank, pairs=cfg.pairs)
    else:
        cache = K.Cache(batch=cfg.batch, context=S, k=dev["k"], v=dev["v"], slots=cfg.slots)
    stream = torch.cuda.current_stream()
    for _ in range(args.warmup):
        K.kvshare_prefill(h, cache, dev["q"], out, lse, stream=stream)
    torch.cuda.synchronize()
    n0 = K.kvshare_launch_count(h)
    ev = []
    with ClockSampler(torch.cuda.current_device()) as clk:
        for _ in range(args.steps):
            for l in range(cfg.layers):
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record(stream)
                K.kvshare_prefill(h, cache, dev["q"], out, lse, l, l + 1, stream=stream)
                e1.record(stream)
                ev.append((l, e0, e1))
        torch.cuda.synchronize()
    st = K.kvshare_sync_status(h)
    assert st == K.KVS_OK, K.kvshare_status_string(st)
    launches = K.kvshare_launch_count(h) - n0
    per_layer = np.zeros(cfg.layers)
    for l, e0, e1 in ev:
        per_layer[l] += e0.elapsed_time(e1)
    per_layer /= args.steps
    step_ms = max_over_ranks(float(per_layer.sum()))
    single = [l for l in range(cfg.layers) if cfg.layer_map[l][0] != MIX]
    mixed = [l for l in range(cfg.layers) if cfg.layer_map[l][0] == MIX]
    K.kvshare_destroy(h)
    del dev, out, lse
    torch.cuda.empty_cache()
    fl = prefill_flops(cfg)
    per_layer_fl = fl / cfg.layers
    return {"cfg": cfg, "step_ms": step_ms, "tflops": fl / (step_ms * 1e-3) / 1e12,
            "single_layer_tflops": per_layer_fl / (float(np.mean(per_layer[single])) * 1e-3) / 1e12,
            "mix_layer_tflops": (per_layer_fl / (float(np.mean(per_layer[mixed])) * 1e-3) / 1e12) if mixed else None,
            "launches": launches, "clocks": clk.summary(), "tokens": cfg.batch * S}


def dist_on():
    return int(os.environ.get("WORLD_SIZE", "1")) > 1


def max_over_ranks(x: float) -> float:
    """Max of a per-rank time over all ranks (the job is as slow as its slowest rank)."""
    import torch.distributed as dist
    if not dist_on() or not dist.is_initialized():
        return x
    import torch
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def arm_config(cfg, world: int) -> dict:
    """The `config` object of the JSON line, shared by both arms."""
    return {"workload": cfg.name, "layers": cfg.layers, "batch_per_gpu": cfg.batch, "context": cfg.context,
            "q_heads": cfg.q_heads, "kv_heads": cfg.kv_heads, "head_dim": cfg.head_dim,
            "layer_map": "CLA2: layer l reads slot l//2" if cfg.name == "cla2_1p1b" else cfg.name,
            "parallelism": f"replicas x{world}",
            "l2": ("flushed before every timed step outside its events (2x L2 write, then 2x L2 read, so the "
                   "lines left are clean); one step reads several times the 126 MB L2. cold_layer_*: flushed "
                   "before every layer, each layer timed alone")}


# ----------------------------------------------------------------------------- oracle (CPU) arm
def oracle_sample(cfg, seconds: float, rng_seed: int = 0, distinct: int = 4):
    """Time the fp64 oracle on (layer, batch) units of the workload for about ``seconds``.

    ``distinct`` units are drawn outside the timed region and evaluated in turn
    until the budget is spent. Returns (seconds per unit, units, threads).
    """
    from oracle import kvshare_ref as ref
    w = cfg.make("w")
    rng = np.random.default_rng(rng_seed)
    pool = []
    for _ in range(distinct):
        l = int(rng.integers(cfg.layers))
        b = int(rng.integers(cfg.batch))
        kind, s0, s1 = cfg.layer_map[l]
        store = {}
        for s in [s0] + ([s1] if kind == 1 else []):
            store[("k", s)] = cfg.make("k", (s, b))
            store[("v", s)] = cfg.make("v", (s, b))
        pool.append((l, b, store, cfg.make("q", (l, b))))
    timed = 0.0
    units = 0
    g = cfg.group
    while timed < seconds and units < 100000:
        l, b, store, qlb = pool[units % distinct]

        def get(name, index, store=store):
            return ref.to_f64(store[(name, index[0])][index[2]], cfg.dtype)
        t0 = time.perf_counter()
        for j in range(cfg.kv_heads):
            ref.decode_head_group(cfg.layer_map, l, b, j, ref.to_f64(qlb[j * g:(j + 1) * g], cfg.dtype), get, w=w)
        timed += time.perf_counter() - t0
        units += 1
    return timed / units, units, blas_threads()


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info()]
        return max(n) if n else 1
    except Exception:  # noqa: BLE001
        return os.cpu_count() or 1


def cpu_baseline(cfg, seconds=12.0, seconds_1core=4.0):
    per_unit, units, threads = oracle_sample(cfg, seconds)
    step_s = per_unit * cfg.layers * cfg.batch
    out = {"value": cfg.batch / step_s, "unit": "tok/s", "cores": threads, "kind": "oracle",
           "sample": f"{units} (layer, batch) units of {cfg.name}, fp64 numpy, extrapolated to "
                     f"{cfg.layers} layers x {cfg.batch} batch"}
    # the same oracle on one host core (BLAS threads limited to 1)
    try:
        from threadpoolctl import threadpool_limits
        with threadpool_limits(limits=1):
            per1, units1, _ = oracle_sample(cfg, seconds_1core, rng_seed=1)
        out["value_1core"] = cfg.batch / (per1 * cfg.layers * cfg.batch)
        out["sample_1core"] = f"{units1} units, BLAS limited to 1 thread"
    except ImportError:
        out["value_1core"] = None
    return out


def data_desc(cfg):
    """The synthetic input recipe of a workload, for the JSON line's "data" key."""
    s = cfg.qkv_scale
    if s == 1.0:
        dist = "N(0,1)"
    elif (1.0 / s).is_integer():
        dist = f"N(0,1)/{1.0 / s:g}"
    else:
        dist = f"{s:g} x N(0,1)"
    return f"synthetic (seeded Philox, q/k/v {dist})"


def reference_arm(args):
    cfg = BY_NAME[args.config]
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    for _ in range(args.warmup):
        oracle_sample(cfg, 0.2, rng_seed=1, distinct=1)
    times = []
    units_total = 0
    threads = 1
    for s in range(args.steps):
        per_unit, units, threads = oracle_sample(cfg, 2.0, rng_seed=100 + s, distinct=2)
        times.append(per_unit * cfg.layers * cfg.batch)
        units_total += units
    step_s = statistics.median(times)
    val = cfg.batch / step_s
    line = {
        "impl": "reference", "metric": METRIC, "value": val, "unit": "tok/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": step_s * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": data_desc(cfg),
        "config": arm_config(cfg, int(os.environ.get("WORLD_SIZE", "1"))),
        "cpu_baseline": {"value": val, "unit": "tok/s", "cores": threads, "kind": "oracle",
                         "sample": f"{units_total} (layer, batch) units over {args.steps} steps, extrapolated"},
        "e2e": {"value": val, "unit": "tok/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line))


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="kvshare", choices=["kvshare", "reference"])
    ap.add_argument("--config", default="cla2_1p1b")
    ap.add_argument("--no-secondary", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-prefill", action="store_true")
    ap.add_argument("--only", choices=["prefill"], default=None,
                    help="profiling aid: run only a causal prefill workload (the two-source one, or the "
                         "prefill workload --config names) and print its numbers")
    ap.add_argument("--layers", type=int, default=0,
                    help="profiling aid: keep only the first N layers of the --config decode workload "
                         "(its layer pattern, fewer layers: a smaller case of the same kernels)")
    ap.add_argument("--batch", type=int, default=0,
                    help="profiling aid: batch of the prefill workload (with --only prefill) or of the "
                         "--config decode workload (a smaller case of the same kernels)")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)

    if args.only == "prefill":
        import torch
        torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", "0")))
        # the two-source prefill unless --config names another prefill workload
        base = args.config if BY_NAME[args.config].mode == "prefill" else "depthgraft_prefill"
        name = base
        if args.batch > 0:
            name = f"{base}_b{args.batch}"
            BY_NAME[name] = BY_NAME[base].replace(name=name, batch=args.batch)
        pr = prefill_arm(args, name)
        print(json.dumps({"workload": name, "tflops": pr["tflops"], "ms_per_step": pr["step_ms"],
                          "single_source_layer_tflops": pr["single_layer_tflops"],
                          "mix_layer_tflops": pr["mix_layer_tflops"], "gpu_launches": pr["launches"]}))
        return

    if args.impl == "reference":
        reference_arm(args)
        return

    import torch
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))

    hbm_peak, bf16_peak, bf16_sust, peak_src = load_peaks()
    if args.batch > 0:
        name = f"{args.config}_b{args.batch}"
        BY_NAME[name] = BY_NAME[args.config].replace(name=name, batch=args.batch)
        args.config = name
    if args.layers > 0:
        c = BY_NAME[args.config]
        n_l = min(args.layers, c.layers)
        name = f"{args.config}_l{n_l}"
        kw = dict(name=name, layers=n_l, layer_map=c.layer_map[:n_l])
        if c.lowrank:
            kw["pairs"] = (n_l + 1) // 2
        BY_NAME[name] = c.replace(**kw)
        args.config = name
    main_res = gpu_arm(args, args.config)
    cfg = main_res["cfg"]
    sec = {}
    if not args.no_secondary:
        for name in ("depthgraft_decode", "depthweave_decode"):
            if name == args.config:
                continue
            r2 = gpu_arm(argparse.Namespace(steps=max(5, args.steps // 2), warmup=3), name)
            sec[name] = {"tok_s": r2["tok_s"] * world, "kv_gbs": r2["kv_gbs"],
                         "hbm_frac": r2["kv_gbs"] / hbm_peak, "ms_per_step": r2["step_ms"],
                         "algorithmic_bytes_per_step": r2["read_bytes"],
                         "cold_layer_ms_per_step": r2["cold_layer_ms"],
                         "in_model_order_ms_per_step": r2["in_order_ms"], "gpu_launches": r2["launches"],
                         "e2e_tok_s": r2["cfg"].batch * world / (r2["e2e_ms"] * 1e-3)}
            if r2["pack_ms"] is not None:
                sec[name]["pack_residual_ms"] = r2["pack_ms"]
                sec[name]["pack_residual_gbs"] = r2["pack_bytes"] / (r2["pack_ms"] * 1e-3) / 1e9
            if r2["extra"]:
                sec[name]["with_router_stats_ms_per_step"] = r2["extra"]["stats_ms_per_step"]
                sec[name]["append_us_per_token"] = r2["extra"]["append_us_per_token"]
        rg = ragged_arm(argparse.Namespace(steps=max(5, args.steps // 2), warmup=3))
        sec["cla2_1p1b_ragged_lengths"] = dict(rg, hbm_frac=rg["kv_gbs"] / hbm_peak)
    if not args.no_secondary and not args.no_prefill:
        pl = prefill_arm(argparse.Namespace(steps=max(3, args.steps // 3), warmup=3), "depthweave_prefill")
        sec["depthweave_prefill"] = {
            "tflops_absorbed": pl["tflops"], "ms_per_step": pl["step_ms"],
            "tok_s": pl["tokens"] * world / (pl["step_ms"] * 1e-3),
            "tensor_frac_of_burst_padded": pl["tflops"] * 64 / 48 / bf16_peak,
            "equivalent_d128_tflops": pl["tflops"] * 128 / 48,
            "flops_per_step": prefill_flops(pl["cfg"]), "gpu_launches": pl["launches"], "clocks": pl["clocks"]}
        pr = prefill_arm(argparse.Namespace(steps=max(3, args.steps // 3), warmup=3))
        sec["depthgraft_prefill"] = {
            "tflops": pr["tflops"], "ms_per_step": pr["step_ms"], "tok_s": pr["tokens"] * world / (pr["step_ms"] * 1e-3),
            "tensor_frac_of_burst": pr["tflops"] / bf16_peak, "tensor_frac_of_sustained": pr["tflops"] / bf16_sust,
            "single_source_layer_tflops": pr["single_layer_tflops"], "mix_layer_tflops": pr["mix_layer_tflops"],
            "flops_per_step": prefill_flops(pr["cfg"]), "gpu_launches": pr["launches"], "clocks": pr["clocks"]}
    # average launch duration over the timed region: the step's time over its launches
    # (gaps between launches included)
    avg_launch_ms = main_res["step_ms"] / cfg.layers
    per_launch_bytes = main_res["read_bytes"] / cfg.layers
    achieved = per_launch_bytes / (avg_launch_ms * 1e-3) / 1e9
    kname = ("decode_lowrank_kernel<%d,%d>" % (cfg.head_dim, cfg.basis_rank) if cfg.lowrank else
             "decode_%s_kernel<%d,%s>" % (cfg.dtype, cfg.head_dim, "mix" if cfg.has_mix else "single"))
    traffic = NCU_TRAFFIC_BYTES.get(cfg.name)
    line = {
        "metric": METRIC,
        "value": main_res["tok_s"] * world,
        "unit": "tok/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": main_res["step_ms"],
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": cfg.dtype,
        "data": data_desc(cfg),
        "config": arm_config(cfg, world),
        "kv_gbs": main_res["kv_gbs"],
        "hbm_frac": main_res["kv_gbs"] / hbm_peak,
        "layer_order": "cold order (first readers of each source, then second readers)",
        "cold_layer_ms_per_step": main_res["cold_layer_ms"],
        "cold_layer_tok_s": cfg.batch * world / (main_res["cold_layer_ms"] * 1e-3),
        "in_model_order_ms_per_step": main_res["in_order_ms"],
        "gpu_launches": main_res["launches"],
        "clocks": main_res["clocks"],
        "e2e": {"value": cfg.batch * world / (main_res["e2e_ms"] * 1e-3), "unit": "tok/s",
                "h2d_bytes_per_step": main_res["h2d"], "d2h_bytes_per_step": main_res["d2h"],
                "ms_per_step": main_res["e2e_ms"], "layer_order": "cold order, as the device-timed step"},
        "roofline": {"kernel": kname, "bound": "hbm", "achieved": achieved,
                     "peak": hbm_peak, "unit": "GB/s", "frac": achieved / hbm_peak,
                     "traffic": traffic, "algorithmic_bytes_per_launch": per_launch_bytes,
                     "peak_source": f"{peak_src} hbm_gbs (MEASURED_PEAKS.json)"},
        "secondary": sec,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(cfg)
    if rank == 0:
        print(json.dumps(line))
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
