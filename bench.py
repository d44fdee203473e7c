"""Benchmark of the compressed-KV decode step on B200 (one JSON line on rank 0).

A step is one decode step of every unit of every layer of the workload:
kvpack_select (rank mask from the previous step's attention mass) followed by
kvpack_decode_attn (rank-space scores, split-T online softmax, V-coefficient
sum, projection through B_V, uncompressed text tail, attention mass).  The
text tail grows by one token per step.  The compressed cache is synthetic
(seeded; shapes of the LLaVA-1.5-7B-style workload by default) and resident
in HBM; every step reads far more than the 126 MB L2, so no flush is needed.

    python bench.py [--gpus N --steps K --warmup W] [--config C1] [--hi-frac 0.25]
    python bench.py --impl reference ...      # the fp64 CPU oracle on a bounded sample

Multi-GPU (torchrun, one process per GPU): every rank decodes its own batch of
the workload (independent units, no collective on the data path); the step
time is the max over ranks and value counts the units of all ranks.
"""
import argparse
import dataclasses
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import synth  # noqa: E402
from synth import cases  # noqa: E402

FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
POOL = 8   # distinct host-generated units tiled over the cache
# kernels of ours launched per step: kvpack_select (1) + kvpack_decode_attn (q~/text, text statistics,
# visual, finish, mass)
LAUNCHES_PER_STEP = 6


# ------------------------------------------------------------------ accounting

def step_bytes(w: synth.Workload, L_text: int, k_hi: int) -> int:
    """Algorithmic HBM bytes of one step (select + decode), all units:
    coefficients at each token's rank (K and V), both bases, the text tail,
    q and out, the mask, the mass written by decode and read by select, the
    new mask written by select."""
    T, Hg = w.T, w.Hg
    per_unit = ((k_hi * 64 + (T - k_hi) * 16) * 2 * 2
                + 2 * 64 * 512 * 2
                + L_text * 512 * 2 * 2
                + 2 * Hg * 128 * 2
                + ((T + 31) // 32) * 4 * 2
                + T * 4 * 2)
    return per_unit * w.units


def decode_bytes(w: synth.Workload, L_text: int, k_hi: int) -> int:
    """Algorithmic bytes of kvpack_decode_attn alone (everything above but select's mass read and mask write)."""
    T = w.T
    return step_bytes(w, L_text, k_hi) - w.units * (T * 4 + ((T + 31) // 32) * 4)


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            mp = json.load(f)
        return float(mp["hbm_gbs"]), float(mp["bf16_tflops"]), "measured (MEASURED_PEAKS.json)"
    except Exception:
        return FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS, "fallback (profiling recipe)"


class Ranks:
    """The bench's steps across ranks: barriers and max-over-ranks reductions of device
    times.  Every rank takes the same steps in the same order; without a process group
    (one GPU) they are no-ops.  The backend is NCCL on the GPUs and gloo for the CPU tests."""

    def __init__(self, dist=None, device="cpu"):
        self.dist, self.device = dist, device

    def barrier(self):
        if self.dist is not None:
            self.dist.barrier()

    def max(self, *values):
        if self.dist is None:
            return tuple(float(v) for v in values)
        import torch
        t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=self.device)
        self.dist.all_reduce(t, op=self.dist.ReduceOp.MAX)
        return tuple(float(x) for x in t.cpu())


def whole_job_value(world: int, batch: int, ms_per_step: float) -> float:
    """Query tokens per second of the whole job: every rank decodes its own batch (weak
    scaling), and the step time is the slowest rank's."""
    return world * batch / (ms_per_step / 1e3)


DECODE_SOURCES = ("decode.cuh", "rstream.cuh", "quant.cuh", "common.cuh", "kvpack.cu")


def sources_digest(names=DECODE_SOURCES) -> str:
    h = hashlib.sha256()
    for n in names:
        with open(os.path.join(ROOT, "rank_compressed_kv_b200", "csrc", n), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel: str, config: str):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on the current kernel sources."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f)
        ent = rec[f"{kernel}:{config}"]
        return ent["bytes_per_launch"] if ent["sources_sha256_16"] == sources_digest() else None
    except (OSError, KeyError, ValueError):
        return None


# ------------------------------------------------------------------ clocks

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.dev = device_index
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(prefix="kvpack_clocks_", suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "50",
                 "-i", str(self.dev)], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    rows.append(dict(sm=float(parts[1]), smax=float(parts[2]), reasons=parts[4:9]))
                except ValueError:
                    continue
        os.unlink(self.path)
        if not rows:
            return None
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        active = set()
        for r in rows:
            for n, v in zip(names, r["reasons"][1:]):
                if v.lower().startswith("active"):
                    active.add(n)
        return {"sm_mhz": statistics.median(r["sm"] for r in rows), "sm_max_mhz": max(r["smax"] for r in rows),
                "reasons": sorted(active), "samples": len(rows)}


# ------------------------------------------------------------------ our arm

def build_cache(kv, torch, w: synth.Workload, Lcap: int, dev):
    """Device-resident compressed cache of the whole workload: POOL host-generated
    units (seeded, per the workload's recipe) tiled over all units."""
    U, T = w.units, w.T
    pool = [cases.unit_inputs(w, 0, i % w.batch, i % w.groups, T, Lcap, mask="ones") for i in range(POOL)]

    def tile(key, shape, sl=None):
        arr = np.stack([p[key] if sl is None else p[key][..., sl] for p in pool])
        src = torch.from_numpy(np.ascontiguousarray(arr).view(np.int16)).to(dev)
        full = torch.empty((U,) + shape, dtype=torch.int16, device=dev)
        reps = U // POOL
        full[:reps * POOL].view(reps, POOL, *shape).copy_(src.unsqueeze(0).expand(reps, *src.shape))
        if U % POOL:
            full[reps * POOL:].copy_(src[:U % POOL])
        return full.view(torch.bfloat16)

    c = {}
    c["CK_lo"] = tile("CK", (T, 16), slice(0, 16))
    c["CK_hi"] = tile("CK", (T, 48), slice(16, 64))
    c["CV_lo"] = tile("CV", (T, 16), slice(0, 16))
    c["CV_hi"] = tile("CV", (T, 48), slice(16, 64))
    c["BK"] = tile("BK", (64, 512))
    c["BV"] = tile("BV", (64, 512))
    c["K_text"] = tile("K_text", (Lcap, 4, 128))
    c["V_text"] = tile("V_text", (Lcap, 4, 128))
    return c


def measure_workload(kv, torch, w: synth.Workload, K: int, W: int, dev, ranks, world: int, headline: bool,
                     baselines: bool = False):
    """Device-timed decode steps of one workload (select + decode over all layers), the same
    steps as per-layer calls in one CUDA graph, and, for the headline workload, the end-to-end
    leg with host buffers.  Returns the measurements as a dict."""
    T, L0 = w.T, w.text0
    Lcap = L0 + W + 2 * K + 2
    k_hi = w.k_hi
    dims = kv.Dims(batch=w.batch, n_q_heads=w.n_q, n_kv_heads=w.n_kv, T_vis=T, L_text_cap=Lcap)
    n_layers = w.layers
    c = build_cache(kv, torch, w, Lcap, dev)
    NQ = 4
    q_host = [torch.from_numpy(np.stack([synth.query(w, l, b, s) for l in range(n_layers) for b in range(w.batch)])
                               .view(np.int16)).view(torch.bfloat16).pin_memory() for s in range(NQ)]
    q_dev = [qh.to(dev) for qh in q_host]
    out = torch.empty(n_layers * w.batch, w.n_q, 128, dtype=torch.bfloat16, device=dev)
    mass = torch.zeros(w.units, T, dtype=torch.float32, device=dev)
    nwords = (T + 31) // 32
    mask = torch.empty(w.units, nwords, dtype=torch.int32, device=dev)
    mask.copy_(torch.from_numpy(synth.all_ones_mask(T).view(np.int32)).to(dev).unsqueeze(0).expand(w.units, nwords))
    ws = torch.empty(kv.decode_workspace(dims, n_layers), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def decode(step, q):
        kv.decode_attn(dims, n_layers, q, c["CK_lo"], c["CK_hi"], c["BK"], c["CV_lo"], c["CV_hi"], c["BV"],
                       c["K_text"], c["V_text"], L0 + step, mask, 1.0, out, mass, ws)

    # step 0: all tokens at full rank (no previous mass), then warm-up steps
    decode(0, q_dev[0])
    for s in range(1, W + 1):
        kv.select(dims, n_layers, mass, None, 0.0, k_hi, mask)
        decode(s, q_dev[s % NQ])
    torch.cuda.synchronize()

    # device-resident timed region: events per decode launch and around the whole run
    ev_dec = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    local = dev.index if dev.index is not None else 0
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    ranks.barrier()
    torch.cuda.synchronize()
    wall0 = time.perf_counter()
    ev0.record(stream)
    for i in range(K):
        s = W + 1 + i
        kv.select(dims, n_layers, mass, None, 0.0, k_hi, mask)
        ev_dec[i][0].record(stream)
        decode(s, q_dev[s % NQ])
        ev_dec[i][1].record(stream)
    ev1.record(stream)
    torch.cuda.synchronize()
    wall = time.perf_counter() - wall0
    clk = clocks.stop()
    st = kv.last_device_status()
    if st != 0:
        raise RuntimeError(f"device status {kv.STATUS_NAMES[st]} during the timed region ({w.name})")
    ms_total = ev0.elapsed_time(ev1)
    dec_ms = [a.elapsed_time(b) for a, b in ev_dec]
    ms_total, dec_sum = ranks.max(ms_total, sum(dec_ms))
    ms_step = ms_total / K
    res = {"w": w, "ms_step": ms_step, "dec_avg_ms": dec_sum / K, "clocks": clk, "wall": wall,
           "L_mean": L0 + W + 1 + (K - 1) / 2.0}

    if headline:
        # end-to-end through the public API with host buffers: every step's q comes from pinned host
        # memory and its output goes back to pinned host memory.  The copies run on a second stream,
        # double-buffered, so step i + 1's upload and step i's download overlap the computation, as a
        # serving loop would run them; each step still moves its own bytes.  The text lengths are those
        # of the device-timed steps, so the two numbers time the same work.
        out_host = torch.empty_like(out, device="cpu").pin_memory()
        torch.cuda.synchronize()
        ranks.barrier()
        hs, ds = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)   # uploads, downloads
        qd = [torch.empty_like(q_dev[0]) for _ in range(2)]
        outd = [torch.empty_like(out) for _ in range(2)]
        outh = [out_host, torch.empty_like(out, device="cpu").pin_memory()]
        ev_q = [torch.cuda.Event() for _ in range(2)]
        ev_done = [torch.cuda.Event() for _ in range(2)]
        ev_d2h = [torch.cuda.Event() for _ in range(2)]
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s_base = W + 1 + K
        e0.record(stream)
        hs.wait_event(e0)
        with torch.cuda.stream(hs):
            qd[0].copy_(q_host[s_base % NQ], non_blocking=True)
            ev_q[0].record(hs)
        for i in range(K):
            s, b = s_base + i, i % 2
            stream.wait_event(ev_q[b])
            if i >= 2:
                stream.wait_event(ev_d2h[b])        # outd[b] has been read back
            kv.select(dims, n_layers, mass, None, 0.0, k_hi, mask)
            kv.decode_attn(dims, n_layers, qd[b], c["CK_lo"], c["CK_hi"], c["BK"], c["CV_lo"], c["CV_hi"],
                           c["BV"], c["K_text"], c["V_text"], L0 + W + 1 + i, mask, 1.0, outd[b], mass, ws)
            ev_done[b].record(stream)
            if i + 1 < K:                            # next step's q, once step i - 1 has finished reading qd[1 - b]
                with torch.cuda.stream(hs):
                    if i >= 1:
                        hs.wait_event(ev_done[1 - b])
                    qd[1 - b].copy_(q_host[(s + 1) % NQ], non_blocking=True)
                    ev_q[1 - b].record(hs)
            with torch.cuda.stream(ds):              # this step's output
                ds.wait_event(ev_done[b])
                outh[b].copy_(outd[b], non_blocking=True)
                ev_d2h[b].record(ds)
        stream.wait_event(ev_d2h[(K - 1) % 2])
        e1.record(stream)
        torch.cuda.synchronize()
        e2e_ms, = ranks.max(e0.elapsed_time(e1) / K)
        res["e2e_ms"] = e2e_ms
        res["h2d"] = q_host[0].numel() * 2
        res["d2h"] = out.numel() * 2

    # per-layer launches, as a framework that runs attention layer by layer would call the
    # library: one kvpack_select and one kvpack_decode_attn per layer (layer slices of the same
    # buffers), captured once into a CUDA graph and replayed K times; the text length stays at the
    # captured value
    upl = w.units_per_layer
    ws1 = torch.empty(kv.decode_workspace(dims, 1), dtype=torch.uint8, device=dev)
    L_g = L0 + W + 1 + 2 * K
    qg = q_dev[0]

    def per_layer_step():
        for l in range(n_layers):
            u0, u1, r0, r1 = l * upl, (l + 1) * upl, l * w.batch, (l + 1) * w.batch
            kv.select(dims, 1, mass[u0:u1], None, 0.0, k_hi, mask[u0:u1])
            kv.decode_attn(dims, 1, qg[r0:r1], c["CK_lo"][u0:u1], c["CK_hi"][u0:u1], c["BK"][u0:u1],
                           c["CV_lo"][u0:u1], c["CV_hi"][u0:u1], c["BV"][u0:u1], c["K_text"][u0:u1],
                           c["V_text"][u0:u1], L_g, mask[u0:u1], 1.0, out[r0:r1], mass[u0:u1], ws1)

    per_layer_step()                      # library set-up outside the capture
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        per_layer_step()
    for _ in range(3):
        graph.replay()
    torch.cuda.synchronize()
    ranks.barrier()
    g0, g1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    g0.record(stream)
    for _ in range(K):
        graph.replay()
    g1.record(stream)
    torch.cuda.synchronize()
    st = kv.last_device_status()
    if st != 0:
        raise RuntimeError(f"device status {kv.STATUS_NAMES[st]} in the per-layer graph ({w.name})")
    g_ms, = ranks.max(g0.elapsed_time(g1) / K)
    del graph
    res["graph_ms"] = g_ms
    res["L_graph"] = L_g
    del ws1
    if baselines:
        res["baselines"] = measure_baselines(kv, torch, w, dims, c, mask, q_dev[0], out, ws, L0 + W + 1, dev, ranks,
                                             max(3, min(K, 10)))
        res["q4"] = measure_q4(kv, torch, w, dims, c, mask, q_dev[0], out, ws, L0 + W + 1, dev, ranks,
                               max(3, min(K, 20)))
    del c, ws
    torch.cuda.empty_cache()
    return res


def measure_baselines(kv, torch, w, dims, c, mask, q, out, ws, L_text, dev, ranks, K):
    """The rank-space decode call against the two routes it replaces, on the same cache, mask and
    query: standard attention over the uncompressed bf16 cache (T + L tokens, built here by
    decompressing every token at full rank), and decompress-then-attend (materialise K^ and V^ at
    each token's rank, then the same dense attention).  CUDA events around K calls of each."""
    n_layers, T = w.layers, w.T
    U = w.units
    Lc = T + L_text
    dims_full = kv.Dims(batch=w.batch, n_q_heads=w.n_q, n_kv_heads=w.n_kv, T_vis=T, L_text_cap=dims.L_text_cap)
    Kd = torch.empty((U, Lc, 4, 128), dtype=torch.bfloat16, device=dev)
    Vd = torch.empty((U, Lc, 4, 128), dtype=torch.bfloat16, device=dev)
    Kd[:, T:].copy_(c["K_text"][:, :L_text])
    Vd[:, T:].copy_(c["V_text"][:, :L_text])
    ones = torch.full_like(mask, -1)
    kv.decompress(dims_full, n_layers, c["CK_lo"], c["CK_hi"], c["BK"], c["CV_lo"], c["CV_hi"], c["BV"], ones,
                  Kd, Vd, Lc)
    wsd = torch.empty(kv.dense_decode_workspace(dims, n_layers, Lc), dtype=torch.uint8, device=dev)
    mass = torch.empty(U, T, dtype=torch.float32, device=dev)

    def rank_space():
        kv.decode_attn(dims, n_layers, q, c["CK_lo"], c["CK_hi"], c["BK"], c["CV_lo"], c["CV_hi"], c["BV"],
                       c["K_text"], c["V_text"], L_text, mask, 1.0, out, mass, ws)

    def dense():
        kv.dense_decode_attn(dims, n_layers, q, Kd, Vd, Lc, Lc, 1.0, out, wsd)

    def decompress_then_attend():
        kv.decompress(dims, n_layers, c["CK_lo"], c["CK_hi"], c["BK"], c["CV_lo"], c["CV_hi"], c["BV"], mask,
                      Kd, Vd, Lc)
        kv.dense_decode_attn(dims, n_layers, q, Kd, Vd, Lc, Lc, 1.0, out, wsd)

    def timed(fn):
        for _ in range(2):
            fn()
        torch.cuda.synchronize()
        ranks.barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(K):
            fn()
        e1.record()
        torch.cuda.synchronize()
        ms, = ranks.max(e0.elapsed_time(e1) / K)
        return ms

    r_ms = timed(rank_space)
    d_ms = timed(dense)
    dta_ms = timed(decompress_then_attend)
    st = kv.last_device_status()
    if st != 0:
        raise RuntimeError(f"device status {kv.STATUS_NAMES[st]} in the baselines ({w.name})")
    hbm, _, _ = measured_peaks()
    dense_bytes = U * Lc * 512 * 2 * 2 + 2 * U * w.Hg * 128 * 2
    del Kd, Vd, wsd
    torch.cuda.empty_cache()
    return {"text_len": L_text, "calls_timed": K,
            "rank_space_ms": round(r_ms, 4), "dense_ms": round(d_ms, 4), "decompress_then_attend_ms": round(dta_ms, 4),
            "speedup_vs_dense": round(d_ms / r_ms, 2), "speedup_vs_decompress_then_attend": round(dta_ms / r_ms, 2),
            "dense_GBps": round(dense_bytes / (d_ms / 1e3) / 1e9, 1), "dense_frac": round(dense_bytes / (d_ms / 1e3) / 1e9 / hbm, 4),
            "note": "rank-space call also writes the attention mass; the baselines write the output only"}


def measure_text_basis(kv, torch, w: synth.Workload, dev, ranks, K: int):
    """The decode call with the text tokens compressed too (kvpack_decode_attn_tb: the workload's
    text0 prompt tokens factored with a basis of their own, attended at the full rank, plus one
    uncompressed generated token) against the same attention with all text0 + 1 text tokens
    uncompressed (kvpack_decode_attn), on the same visual cache, mask and query.  CUDA events
    around K calls of each; algorithmic bytes per call for both."""
    n_layers, T, U, L_c = w.layers, w.T, w.units, w.text0
    Lcap = L_c + 1
    dims = kv.Dims(batch=w.batch, n_q_heads=w.n_q, n_kv_heads=w.n_kv, T_vis=T, L_text_cap=Lcap)
    c = build_cache(kv, torch, w, Lcap, dev)
    pool = []
    for i in range(POOL):
        ck, bk = synth.text_compressed_unit(w, 0, i % w.batch, i % w.groups, synth.K_TEXT, L_c)
        cv, bv = synth.text_compressed_unit(w, 0, i % w.batch, i % w.groups, synth.V_TEXT, L_c)
        pool.append((ck, bk, cv, bv))

    def tile(j, sl, shape):
        arr = np.stack([p[j] if sl is None else p[j][..., sl] for p in pool])
        src = torch.from_numpy(np.ascontiguousarray(arr).view(np.int16)).to(dev)
        idx = torch.arange(U, device=dev) % POOL
        return src[idx].reshape((U,) + shape).contiguous().view(torch.bfloat16)

    tb = (tile(0, slice(0, 16), (L_c, 16)), tile(0, slice(16, 64), (L_c, 48)), tile(1, None, (64, 512)),
          tile(2, slice(0, 16), (L_c, 16)), tile(2, slice(16, 64), (L_c, 48)), tile(3, None, (64, 512)), L_c)
    q = torch.from_numpy(np.stack([synth.query(w, l, b, 1) for l in range(n_layers) for b in range(w.batch)])
                         .view(np.int16)).view(torch.bfloat16).to(dev)
    gen = torch.Generator(device=dev)
    gen.manual_seed(77 + w.seed)
    mask = torch.empty(U, (T + 31) // 32, dtype=torch.int32, device=dev)
    kv.select(dims, n_layers, torch.rand(U, T, generator=gen, device=dev), None, 0.0, w.k_hi, mask)
    out = torch.empty(n_layers * w.batch, w.n_q, 128, dtype=torch.bfloat16, device=dev)
    mass = torch.empty(U, T, dtype=torch.float32, device=dev)
    ws_plain = torch.empty(kv.decode_workspace(dims, n_layers), dtype=torch.uint8, device=dev)
    ws_tb = torch.empty(kv.decode_tb_workspace(dims, n_layers, L_c), dtype=torch.uint8, device=dev)

    def plain():
        kv.decode_attn(dims, n_layers, q, c["CK_lo"], c["CK_hi"], c["BK"], c["CV_lo"], c["CV_hi"], c["BV"],
                       c["K_text"], c["V_text"], L_c + 1, mask, 1.0, out, mass, ws_plain)

    def compressed_text():
        kv.decode_attn_tb(dims, n_layers, q, c["CK_lo"], c["CK_hi"], c["BK"], c["CV_lo"], c["CV_hi"], c["BV"], tb,
                          c["K_text"], c["V_text"], 1, mask, 1.0, out, mass, ws_tb)

    def timed(fn):
        for _ in range(3):
            fn()
        torch.cuda.synchronize()
        ranks.barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(K):
            fn()
        e1.record()
        torch.cuda.synchronize()
        ms, = ranks.max(e0.elapsed_time(e1) / K)
        return ms

    p_ms = timed(plain)
    t_ms = timed(compressed_text)
    st = kv.last_device_status()
    if st != 0:
        raise RuntimeError(f"device status {kv.STATUS_NAMES[st]} in the text-basis leg ({w.name})")
    plain_bytes = decode_bytes(w, L_c + 1, w.k_hi)
    tb_bytes = plain_bytes - U * L_c * 512 * 2 * 2 + U * (L_c * 64 * 2 * 2 + 2 * 64 * 512 * 2 + ((L_c + 31) // 32) * 4)
    del c, tb, ws_plain, ws_tb
    torch.cuda.empty_cache()
    return {"workload": f"{w.name}: {L_c} prompt text tokens compressed (rank 64, own basis) + 1 generated token",
            "calls_timed": K, "text_uncompressed_ms": round(p_ms, 4), "text_compressed_ms": round(t_ms, 4),
            "speedup": round(p_ms / t_ms, 2), "bytes_text_uncompressed": int(plain_bytes),
            "bytes_text_compressed": int(tb_bytes),
            "GBps_text_compressed": round(tb_bytes / (t_ms / 1e3) / 1e9, 1)}


def measure_q4(kv, torch, w: synth.Workload, dims, c, mask, q, out, ws, L_text, dev, ranks, K: int):
    """The decode call over 4-bit visual coefficients (kvpack_quantize4 once, then
    kvpack_decode_attn_q4) against the 16-bit call, on the same cache, mask and query.  CUDA events
    around K calls of each; algorithmic bytes per call for the 4-bit one (codes and exponents at
    each token's rank, K and V, instead of the 16-bit rows)."""
    n_layers, T, U = w.layers, w.T, w.units
    planes = []
    for side in ("K", "V"):
        Q_lo = torch.empty((U, T, 8), dtype=torch.uint8, device=dev)
        Q_hi = torch.empty((U, T, 24), dtype=torch.uint8, device=dev)
        E = torch.empty((U, T, 2), dtype=torch.int8, device=dev)
        kv.quantize4(dims, n_layers, T, c[f"C{side}_lo"], c[f"C{side}_hi"], Q_lo, Q_hi, E)
        planes.append((Q_lo, Q_hi, E))
    mass = torch.empty(U, T, dtype=torch.float32, device=dev)

    def sixteen():
        kv.decode_attn(dims, n_layers, q, c["CK_lo"], c["CK_hi"], c["BK"], c["CV_lo"], c["CV_hi"], c["BV"],
                       c["K_text"], c["V_text"], L_text, mask, 1.0, out, mass, ws)

    def four():
        (a, b, e), (f, g, h) = planes
        kv.decode_attn_q4(dims, n_layers, q, a, b, e, c["BK"], f, g, h, c["BV"], c["K_text"], c["V_text"], L_text,
                          mask, 1.0, out, mass, ws)

    def timed(fn):
        for _ in range(3):
            fn()
        torch.cuda.synchronize()
        ranks.barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(K):
            fn()
        e1.record()
        torch.cuda.synchronize()
        ms, = ranks.max(e0.elapsed_time(e1) / K)
        return ms

    s_ms = timed(sixteen)
    f_ms = timed(four)
    st = kv.last_device_status()
    if st != 0:
        raise RuntimeError(f"device status {kv.STATUS_NAMES[st]} in the 4-bit leg ({w.name})")
    k = w.k_hi
    sixteen_bytes = decode_bytes(w, L_text, k)
    four_bytes = sixteen_bytes - U * ((k * 64 + (T - k) * 16) * 2 * 2) + U * ((k * 34 + (T - k) * 9) * 2)
    hbm, _, _ = measured_peaks()
    del planes
    torch.cuda.empty_cache()
    return {"calls_timed": K, "sixteen_bit_ms": round(s_ms, 4), "four_bit_ms": round(f_ms, 4),
            "speedup": round(s_ms / f_ms, 2), "bytes_four_bit": int(four_bytes),
            "GBps_four_bit": round(four_bytes / (f_ms / 1e3) / 1e9, 1),
            "frac_four_bit": round(four_bytes / (f_ms / 1e3) / 1e9 / hbm, 4),
            "format": "int4 codes, a power-of-two scale per token and plane (ranks 0-15, 16-63)"}


def roofline_block(w: synth.Workload, L_mean: float, dec_avg_ms: float):
    """Roofline of the dominant call (kvpack_decode_attn): algorithmic bytes per launch over its
    CUDA-event duration, against the measured copy bandwidth."""
    hbm, _, peak_kind = measured_peaks()
    dbytes = decode_bytes(w, L_mean, w.k_hi)
    achieved = dbytes / (dec_avg_ms / 1e3) / 1e9
    return {"bound": "hbm",
            "kernel": "kvpack_decode_attn (all of its kernels on one stream)",
            "achieved": round(achieved, 1), "peak": hbm, "unit": "GB/s",
            "frac": round(achieved / hbm, 4), "frac_of_8TBps": round(achieved / 8000.0, 4),
            "peak_kind": peak_kind,
            "bytes_per_launch": int(dbytes), "avg_launch_ms": round(dec_avg_ms, 4),
            "traffic": recorded_traffic("decode", w.name)}


def config_block(res, world: int):
    """The per-workload summary that goes under "configs" in the bench line."""
    w = res["w"]
    return {"workload": f"{w.name}: batch {w.batch} x {w.layers} layers, {w.n_q} q / {w.n_kv} kv heads, "
                        f"T={w.T} visual + {w.text0}+step text, top {round(w.hi_frac * 100)}% full rank",
            "value": round(whole_job_value(world, w.batch, res["ms_step"]), 1), "unit": "query-tokens/s",
            "ms_per_step": round(res["ms_step"], 4),
            "us_per_decode_call": round(res["dec_avg_ms"] * 1e3, 1),
            "roofline": roofline_block(w, res["L_mean"], res["dec_avg_ms"]),
            "per_layer_graph": {"value": round(whole_job_value(world, w.batch, res["graph_ms"]), 1),
                                "ms_per_step": round(res["graph_ms"], 4), "text_len": res["L_graph"]},
            "clocks": res["clocks"],
            "baselines": res.get("baselines"), "q4": res.get("q4")}


EXTRA_CONFIGS = (("C2", 0.25), ("C3", 0.25), ("C4", 0.25), ("C4", 0.10))


def run_ours(args, w: synth.Workload, rank: int, world: int):
    import torch
    import rank_compressed_kv_b200 as kv

    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist = None
    if world > 1:
        import torch.distributed as dist
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    ranks = Ranks(dist, dev)

    K, W = args.steps, args.warmup
    res = measure_workload(kv, torch, w, K, W, dev, ranks, world, headline=True, baselines=not args.no_baselines)
    ms_step = res["ms_step"]
    value = whole_job_value(world, w.batch, ms_step)
    L_mean = res["L_mean"]
    sbytes = step_bytes(w, L_mean, w.k_hi)
    line = {
        "metric": "compressed-KV decode attn query-tokens/s and achieved HBM GB/s vs 8 TB/s peak",
        "value": round(value, 1),
        "unit": "query-tokens/s",
        "n_gpus": world,
        "steps": K,
        "warmup": W,
        "ms_per_step": round(ms_step, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (seeded low-rank-plus-noise compressed cache, 8 generated units tiled)",
        "config": {"workload": f"{w.name}: batch {w.batch} x {w.layers} layers, {w.n_q} q / {w.n_kv} kv heads, "
                               f"T={w.T} visual + {w.text0}+step text, r=64/16, top {round(w.hi_frac * 100)}% full rank",
                   "global_batch": world * w.batch, "units": w.units, "hi_frac": w.hi_frac,
                   "parallelism": f"dp{world}" if world > 1 else "single-gpu",
                   "l2": "inputs larger than L2 (no flush needed)",
                   "step": "kvpack_select + kvpack_decode_attn over all layers"},
        "step_bytes": int(sbytes),
        "step_GBps": round(sbytes / (ms_step / 1e3) / 1e9, 1),
        "roofline": roofline_block(w, L_mean, res["dec_avg_ms"]),
        "e2e": {"value": round(whole_job_value(world, w.batch, res["e2e_ms"]), 1), "unit": "query-tokens/s",
                "h2d_bytes_per_step": res["h2d"], "d2h_bytes_per_step": res["d2h"],
                "ms_per_step": round(res["e2e_ms"], 4)},
        "gpu_launches": LAUNCHES_PER_STEP * K,
        "per_layer_graph": {"value": round(whole_job_value(world, w.batch, res["graph_ms"]), 1),
                            "unit": "query-tokens/s", "ms_per_step": round(res["graph_ms"], 4),
                            "launches_per_step": LAUNCHES_PER_STEP * w.layers, "text_len": res["L_graph"],
                            "mode": "per layer: kvpack_select + kvpack_decode_attn, captured in one CUDA graph"},
        "clocks": res["clocks"],
        "wall_s_timed": round(res["wall"], 3),
        "baselines": res.get("baselines"),
        "q4": res.get("q4"),
    }
    if not args.no_baselines:
        line["text_basis"] = measure_text_basis(kv, torch, w, dev, ranks, max(10, min(K, args.config_steps)))
    if not args.headline_only:
        # the workloads the HBM-roofline target is set on, measured the same way (device-resident,
        # CUDA events, max over ranks); the headline value above stays the first workload's
        K2 = max(10, min(K, args.config_steps))
        blocks = {}
        for name, f in EXTRA_CONFIGS:
            wx = synth.WORKLOADS[name].with_hi_frac(f)
            blocks[f"{name}@{round(f * 100)}%"] = config_block(
                measure_workload(kv, torch, wx, K2, W, dev, ranks, world, headline=False,
                                 baselines=not args.no_baselines), world)
        line["configs"] = blocks
    if rank == 0 and not args.no_cpu_baseline and world == 1:
        line["cpu_baseline"] = cpu_baseline(w, budget_s=args.cpu_seconds)
    if not args.no_compress and rank == 0:
        line["compress"] = {n: bench_compress(kv, torch, synth.WORKLOADS[n], dev) for n in ("C2", "C4")}
    ranks.barrier()
    if dist:
        dist.destroy_process_group()
    return line


def bench_compress(kv, torch, w, dev):
    """kvpack_compress on one layer of the workload (K side: batch x groups units), timed with CUDA
    events; per-kernel device times from the CUDA profiler give the Gram's rate against the measured
    bf16 peak.  The Gram's algorithmic count is the symmetric rank-k update T n (n + 1) per matrix
    (the kernel computes the upper 128-row bands and mirrors them)."""
    from torch.profiler import profile, ProfilerActivity
    units = w.batch * (w.n_kv // 4)
    dims = kv.Dims(batch=units, n_q_heads=4, n_kv_heads=4, T_vis=w.T, L_text_cap=1)
    pool = [synth.visual_kv(w, 0, b, 0, synth.K_VIS) for b in range(min(POOL, units))]
    X = torch.empty(units, w.T, 512, dtype=torch.bfloat16, device=dev)
    for u in range(units):
        X[u].copy_(torch.from_numpy(pool[u % len(pool)].view(np.int16)).view(torch.bfloat16))
    C_lo = torch.empty(units, w.T, 16, dtype=torch.bfloat16, device=dev)
    C_hi = torch.empty(units, w.T, 48, dtype=torch.bfloat16, device=dev)
    B = torch.empty(units, 64, 512, dtype=torch.bfloat16, device=dev)
    sig = torch.empty(units, 64, dtype=torch.float32, device=dev)
    ws = torch.empty(kv.compress_workspace(dims, 1), dtype=torch.uint8, device=dev)

    def run():
        kv.compress(dims, 1, X, C_lo, C_hi, B, sig, ws)

    run()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    run()
    e1.record()
    torch.cuda.synchronize()
    st = kv.last_device_status()
    with profile(activities=[ProfilerActivity.CUDA]) as prof:
        run()
        torch.cuda.synchronize()
    kern = {}
    for e in prof.events():
        if e.device_type.name == "CUDA":
            name = e.name.split("(")[0].split("::")[-1].split("<")[0]
            kern[name] = kern.get(name, 0.0) + e.device_time_total / 1e3
    _, bf16, peak_kind = measured_peaks()
    gram_ms = kern.get("gram_tc_kernel", float("nan"))
    n = 512
    syrk = float(units) * w.T * n * (n + 1)                 # symmetric rank-k update: the algorithmic count
    full = 2.0 * units * w.T * n * n                         # the full product X^T X, for reference
    tf = syrk / (gram_ms / 1e3) / 1e12
    del X, C_lo, C_hi, B, sig, ws
    torch.cuda.empty_cache()
    return {"workload": f"{w.name}: one layer, K side, {units} units of T={w.T}", "units": units, "T": w.T,
            "ms_per_layer_matrix": round(e0.elapsed_time(e1), 3), "status": kv.STATUS_NAMES.get(st, st),
            "kernel_ms": {k: round(v, 3) for k, v in kern.items()},
            "gram": {"bound": "tensor", "count": "SYRK T*n*(n+1) per matrix", "flops": syrk,
                     "achieved": round(tf, 1), "unit": "TFLOP/s", "peak": bf16, "peak_kind": peak_kind,
                     "frac": round(tf / bf16, 4),
                     "full_product_tflops": round(full / (gram_ms / 1e3) / 1e12, 1),
                     "kernel_ms": round(gram_ms, 4)}}


# ------------------------------------------------------------------ oracle (CPU) arm

def _oracle_inputs(w: synth.Workload, n_units: int, L_text: int):
    import oracle
    f = oracle.bf16_to_f64
    pool = [cases.unit_inputs(w, 0, i % w.batch, i % w.groups, w.T, L_text, mask="random") for i in range(POOL)]
    idx = [i % POOL for i in range(n_units)]
    q = np.stack([synth.query(w, 0, i % w.batch, 0)[: w.Hg] for i in range(POOL)])
    return dict(
        CK=f(np.stack([pool[i]["CK"] for i in idx])), BK=f(np.stack([pool[i]["BK"] for i in idx])),
        CV=f(np.stack([pool[i]["CV"] for i in idx])), BV=f(np.stack([pool[i]["BV"] for i in idx])),
        Kt=f(np.stack([pool[i]["K_text"] for i in idx])), Vt=f(np.stack([pool[i]["V_text"] for i in idx])),
        mask=np.stack([pool[i]["mask"] for i in idx]), q=f(np.stack([q[i] for i in idx])),
    )


def _oracle_step(inp, k_hi, mass_prev):
    import oracle
    mask, _ = oracle.select(mass_prev, k_hi)
    out, mass = oracle.decode(inp["CK"], inp["BK"], inp["CV"], inp["BV"], inp["Kt"], inp["Vt"], mask, inp["q"])
    return mass.astype(np.float32)


def cpu_baseline(w: synth.Workload, budget_s: float = 15.0):
    """The oracle as it stands (fp64 decompress-then-attend + fp32 top-k), OpenMP over
    units on the host cores, on a bounded sample of the workload's units; the metric
    is extrapolated to a full step of all units."""
    import oracle
    L = w.text0
    probe = _oracle_inputs(w, 2 * oracle.num_threads(), L)
    m0 = np.random.default_rng(0).random((probe["CK"].shape[0], w.T)).astype(np.float32)
    t0 = time.perf_counter()
    _oracle_step(probe, w.k_hi, m0)
    per_unit = (time.perf_counter() - t0) / probe["CK"].shape[0]
    n = int(max(oracle.num_threads(), min(w.units, 2048, budget_s / max(per_unit, 1e-6))))
    n = max(oracle.num_threads(), (n // oracle.num_threads()) * oracle.num_threads())
    inp = _oracle_inputs(w, n, L)
    m0 = np.random.default_rng(1).random((n, w.T)).astype(np.float32)
    t0 = time.perf_counter()
    _oracle_step(inp, w.k_hi, m0)
    el = time.perf_counter() - t0
    step_s = el * w.units / n
    return {"value": round(w.batch / step_s, 3), "unit": "query-tokens/s", "cores": oracle.num_threads(),
            "kind": "oracle",
            "sample": f"{n} of {w.units} units of one step (select + decode, fp64), {el:.1f} s, extrapolated"}


def run_reference(args, w: synth.Workload):
    """--impl reference: the fp64 CPU oracle timed on the host cores, each step a bounded
    sample of the workload's units, extrapolated to the full step."""
    import oracle
    K, W = args.steps, args.warmup
    threads = oracle.num_threads()
    # size the per-step sample so that W + K steps take about args.cpu_seconds in total
    probe = _oracle_inputs(w, 2 * threads, w.text0)
    m0 = np.random.default_rng(0).random((probe["CK"].shape[0], w.T)).astype(np.float32)
    t0 = time.perf_counter()
    _oracle_step(probe, w.k_hi, m0)
    per_unit = (time.perf_counter() - t0) / probe["CK"].shape[0]
    n = int(args.cpu_seconds / max(per_unit, 1e-6) / (K + W))
    n = max(threads, min(w.units, 2048, (n // threads) * threads))
    inp = _oracle_inputs(w, n, w.text0)
    mass = np.random.default_rng(1).random((n, w.T)).astype(np.float32)
    for _ in range(W):
        mass = _oracle_step(inp, w.k_hi, mass)
    t0 = time.perf_counter()
    for _ in range(K):
        mass = _oracle_step(inp, w.k_hi, mass)
    el = time.perf_counter() - t0
    step_s = el / K * w.units / n
    value = w.batch / step_s
    sample = f"{n} of {w.units} units per step (select + decode, fp64), extrapolated to the full step"
    return {
        "impl": "reference",
        "metric": "compressed-KV decode attn query-tokens/s and achieved HBM GB/s vs 8 TB/s peak",
        "value": round(value, 4), "unit": "query-tokens/s", "n_gpus": 1, "steps": K, "warmup": W,
        "ms_per_step": round(step_s * 1e3, 3), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.name, "global_batch": w.batch, "units": w.units},
        "cpu_baseline": {"value": round(value, 4), "unit": "query-tokens/s", "cores": threads, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": round(value, 4), "unit": "query-tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--config", default="C1", choices=sorted(synth.WORKLOADS))
    ap.add_argument("--hi-frac", type=float, default=None)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--no-compress", action="store_true", help="skip the kvpack_compress block")
    ap.add_argument("--headline-only", action="store_true", help="measure the --config workload only")
    ap.add_argument("--no-baselines", action="store_true", help="skip the dense and decompress-then-attend baselines")
    ap.add_argument("--config-steps", type=int, default=50, help="timed steps of each extra workload")
    ap.add_argument("--only-compress", action="store_true",
                    help="time kvpack_compress on one layer of --config only (a small case for profiler captures)")
    ap.add_argument("--layers", type=int, default=None,
                    help="run the config with fewer layers (a small case for profiler captures; named in the line)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    w = synth.WORKLOADS[args.config]
    if args.hi_frac is not None:
        w = w.with_hi_frac(args.hi_frac)
    if args.layers is not None:
        if not 1 <= args.layers <= w.layers:
            ap.error(f"--layers must be in 1..{w.layers}")
        w = dataclasses.replace(w, name=f"{w.name}[{args.layers} of {w.layers} layers]", layers=args.layers)
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if args.gpus != world and args.impl == "ours":
        ap.error(f"--gpus {args.gpus} needs one process per GPU: launch with torchrun --nproc-per-node {args.gpus}")
    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args, w)), flush=True)
        return
    if args.only_compress:
        import torch
        import rank_compressed_kv_b200 as kv
        torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", "0")))
        print(json.dumps(bench_compress(kv, torch, w, torch.device("cuda", torch.cuda.current_device()))),
              flush=True)
        return
    line = run_ours(args, w, rank, world)
    if rank == 0:
        print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
