#!/usr/bin/env python
"""One decode step of absorbed MLA over a compressed latent cache, timed on the GPU.

A step is the whole hot path over one batch: cache append of the new token (a1), query absorption
(a2), absorbed split-KV decode with its log-sum-exp merge (a3 + a4) and the per-head output
projection through W_UV (a5). The default workload is the DeepSeek-V2/V3-shaped batch: 64 sequences
of 4096 cached positions, H=128, d_c=512, d_r=64, bf16 storage, fp32 accumulation.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--workload NAME]

N > 1 runs under torch.distributed.run, one process per GPU: every rank runs the full batch on its
own GPU (independent sequences, weak scaling, no collective in the data path); timing is the max
over ranks. `--impl reference` times the fp64 CPU oracle on a bounded sample of the same workload
(rank 0 only).
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "MLA decode cache-positions/s and tokens/s; % of B200 roofline (HBM or TC)"
UNIT = "positions/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# nominal B200 figures (context for the measured fractions): HBM3e ~8 TB/s, dense bf16 2.25 PFLOP/s
NOMINAL_PEAKS = {"hbm_gbs": 8000.0, "bf16_tflops": 2250.0}


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=400)
    p.add_argument("--warmup", type=int, default=20)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--workload", default="dsv3_b64_l4096")
    p.add_argument("--cpu-seconds", type=float, default=12.0, help="bound on the CPU-baseline sample")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-secondary", action="store_true", help="skip the other configurations' decode timings")
    p.add_argument("--decode-only", action="store_true",
                   help="time the workload's decode call alone (inputs drawn on the GPU) and print its line; "
                        "a per-configuration diagnostic, not the whole step")
    return p.parse_args()


def dist_env():
    return int(os.environ.get("RANK", 0)), int(os.environ.get("WORLD_SIZE", 1)), int(os.environ.get("LOCAL_RANK", 0))


def max_over_ranks(x, world, device=None):
    """The largest x over all ranks, returned on every rank (a time is the slowest rank's; a flag
    raised on any rank is raised on all). Every rank must call it at the same point."""
    if world <= 1:
        return float(x)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in FALLBACK_PEAKS if k in d}, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# ------------------------------------------------------------------------------------------------
# algorithmic counts of the decode kernel (bytes that must move, FLOPs that must be done)
# ------------------------------------------------------------------------------------------------
# DRAM traffic of one decode_kernel launch (dram__bytes_read.sum + dram__bytes_write.sum) from an
# ncu capture at dsv3_b64_l4096; reported only while the kernel's sources are the ones it was taken
# on (their hash), otherwise the roofline's traffic is null.
DECODE_TRAFFIC = {"workload": "dsv3_b64_l4096", "bytes": 311_842_816 + 3_818_752, "sources_sha256_16": "4c5ed38ef3a23a6b"}
DECODE_SOURCES = ("decode_sm100.cuh", "ptx_sm100.cuh", "common.cuh")
# the same for one gqla_kernel launch at gqla_g8_b32_l8192
GQLA_TRAFFIC = {"workload": "gqla_g8_b32_l8192", "bytes": 1_115_248_640 + 10_563_072, "sources_sha256_16": "c67edddacfb49765"}
GQLA_SOURCES = ("gqla_sm100.cuh", "ptx_sm100.cuh", "common.cuh")


def captured_traffic(workload, record=DECODE_TRAFFIC, sources=DECODE_SOURCES):
    import hashlib
    csrc = os.path.join(os.path.dirname(os.path.abspath(__file__)), "mla_compressed_latent_b200", "csrc")
    h = hashlib.sha256()
    for name in sources:
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(f.read())
    if workload == record["workload"] and h.hexdigest()[:16] == record["sources_sha256_16"]:
        return record["bytes"]
    return None


def decode_counts(w, lens):
    total = int(sum(int(L) for L in lens))
    e = 2 if w.dtype == "bf16" else 4
    n_tok = w.B * w.s_q
    # a cached row: the latent in e bytes per value (or one E4M3 byte plus a 4-byte scale per row),
    # the RoPE key in e bytes per value
    row = (w.d_c * e if getattr(w, "latent_bits", 16) == 16 else w.d_c + 4) + w.d_r * e
    bytes_ = total * row + n_tok * w.H * ((w.d_c + w.d_r) + w.d_c) * e + n_tok * w.H * 4
    visible = sum(int(L) * w.s_q - w.s_q * (w.s_q - 1) // 2 for L in lens)
    flops = 2 * w.H * (2 * w.d_c + w.d_r) * visible
    return bytes_, flops, total


# ------------------------------------------------------------------------------------------------
# clocks during the timed region (NVML reads only; no setting is touched)
# ------------------------------------------------------------------------------------------------
class ClockSampler:
    REASONS = {
        0x0000000000000001: "gpu_idle", 0x0000000000000002: "applications_clocks_setting",
        0x0000000000000004: "sw_power_cap", 0x0000000000000008: "hw_slowdown",
        0x0000000000000010: "sync_boost", 0x0000000000000020: "sw_thermal_slowdown",
        0x0000000000000040: "hw_thermal_slowdown", 0x0000000000000080: "hw_power_brake_slowdown",
        0x0000000000000100: "display_clock_setting",
    }

    def __init__(self, index):
        self.samples = []
        self.reasons = set()
        self.ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as ex:  # noqa: BLE001
            self.err = repr(ex)
        self._stop = threading.Event()

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                r = self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for bit, name in self.REASONS.items():
                    if r & bit:
                        self.reasons.add(name)
            except Exception:  # noqa: BLE001
                pass
            time.sleep(0.002)

    def __enter__(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self._stop.set()
            self.t.join()

    def summary(self):
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "error": getattr(self, "err", "nvml")}
        med = statistics.median(self.samples) if self.samples else None
        return {"sm_mhz": med, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons - {"gpu_idle"}),
                "samples": len(self.samples)}

    def rejected(self):
        bad = {"hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown"}
        return bool(self.reasons & bad)


# ------------------------------------------------------------------------------------------------
# CPU side: the oracle on a bounded sample (baseline and reference arm)
# ------------------------------------------------------------------------------------------------
def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [d.get("num_threads", 1) for d in threadpool_info() if d.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:  # noqa: BLE001
        return os.cpu_count() or 1


_ORACLE_SETUP = {}
_ORACLE_ROWS = {}


def _oracle_setup(w):
    """The oracle's weights (fp64) and this step's inputs, drawn once per workload."""
    if w not in _ORACLE_SETUP:
        import numpy as np
        import synth
        W = synth.weights(w)
        _ORACLE_SETUP[w] = (W["W_UK"].astype(np.float64), W["W_UV"].astype(np.float64),
                            synth.decode_step_inputs(w))
    return _ORACLE_SETUP[w]


def _oracle_rows(w, n):
    """(b, c, k_r) in fp64 for the first n sequences, in order; the rows of a one- or two-sequence
    sample are kept for the next call (the reference arm times the same sequence every step)."""
    import numpy as np
    import synth
    if (w, n) in _ORACLE_ROWS:
        yield from _ORACLE_ROWS[(w, n)]
        return
    lens = synth.seq_lengths(w)[:n]
    chunks = synth.cache_row_chunks(w, int(lens.sum()))
    pend_c = np.zeros((0, w.d_c), np.float32)
    pend_k = np.zeros((0, w.d_r), np.float32)
    keep = [] if n <= 2 else None
    for b, L in enumerate(lens):
        L = int(L)
        while len(pend_c) < L:
            _, c, kr = next(chunks)
            pend_c = np.concatenate([pend_c, c])
            pend_k = np.concatenate([pend_k, kr])
        item = (b, pend_c[:L].astype(np.float64), pend_k[:L].astype(np.float64))
        pend_c, pend_k = pend_c[L:], pend_k[L:]
        if keep is not None:
            keep.append(item)
            if len(keep) == n:
                _ORACLE_ROWS[(w, n)] = keep
        yield item


def oracle_sample(w, seconds, max_seqs=None):
    """Run the fp64 oracle's decode step (absorb, absorbed decode, W_UV projection) sequence by
    sequence until `seconds` of oracle time pass; drawing the inputs is not timed. Returns
    (positions, tokens, oracle seconds, sequences)."""
    from oracle import mla_oracle as O
    W_UK, W_UV, step = _oracle_setup(w)
    n = w.B if max_seqs is None else min(w.B, max_seqs)
    pos_done = tok_done = seqs = 0
    el = 0.0
    for b, c, kr in _oracle_rows(w, n):
        L = len(c)
        t0 = time.perf_counter()
        pos = O.token_positions(L, w.s_q)
        q_abs = O.absorb_query(step["q_nope"][b], step["q_rope_raw"][b], W_UK, pos, w.rope_base)
        o_lat, _ = O.absorbed_decode(q_abs, c, kr, L, w.sm_scale)
        O.out_projection(o_lat, W_UV)
        el += time.perf_counter() - t0
        pos_done += L
        tok_done += w.s_q
        seqs += 1
        if el >= seconds:
            break
    return pos_done, tok_done, el, seqs


def run_reference(args, rank, world):
    import synth
    if rank != 0:
        return
    w = synth.workload(args.workload)
    per_step_seconds = max(0.5, min(10.0, 120.0 / max(1, args.steps + args.warmup)))
    for _ in range(args.warmup):
        oracle_sample(w, per_step_seconds, max_seqs=1)
    pos = tok = 0
    el = 0.0
    for _ in range(args.steps):
        p, t, e, s = oracle_sample(w, per_step_seconds, max_seqs=1)
        pos += p
        tok += t
        el += e
    value = pos / el
    cores = blas_threads()
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * el / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.name, "B": w.B, "seq_len": w.lengths[1] if w.lengths[0] == "fixed" else list(w.lengths),
                   "H": w.H, "d_c": w.d_c, "d_r": w.d_r, "s_q": w.s_q},
        "tokens_per_s": tok / el,
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": f"each step: sequence 0 of {w.name} ({int(synth.seq_lengths(w)[0])} positions, "
                                   f"all {w.H} heads), fp64 absorb + absorbed decode + W_UV projection"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------------------------------------
# GPU arm
# ------------------------------------------------------------------------------------------------
def build_inputs(w, device):
    import numpy as np
    import torch
    import synth
    tdt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    lens = synth.seq_lengths(w)
    table, num_pages = synth.block_table(w, lens)
    total = int(lens.sum())
    pool = torch.zeros(num_pages * 64, w.d_c + w.d_r, dtype=tdt, device=device)
    # logical row r of sequence b -> pool row through the page table
    idx = np.empty(total, dtype=np.int64)
    off = 0
    for b, L in enumerate(lens):
        p = np.arange(L)
        idx[off:off + L] = table[b, p // 64].astype(np.int64) * 64 + p % 64
        off += L
    W = synth.weights(w)
    step = synth.decode_step_inputs(w)
    from_hidden = w.dtype == "bf16" and w.lengths[0] == "fixed" and w.lengths[1] % 64 == 0
    if from_hidden:
        # the configured recipe: every cached row is c = RMSNorm(x·W_DKV), k_r = RoPE(x·W_KR) of hidden
        # states x ~ N(0, 1), written by the library's own cache append, 64 positions of every
        # sequence per call (x drawn on the GPU by torch's CUDA generator)
        fill_cache_from_hidden_states(w, pool, num_pages, table, lens, W, device)
    else:
        for start, c, kr in synth.cache_row_chunks(w, total):
            n = len(c)
            rows = torch.from_numpy(np.concatenate([c, kr], axis=1)).to(device=device, dtype=tdt)
            pool[torch.from_numpy(idx[start:start + n]).to(device)] = rows
    dev = {
        "pool": pool, "num_pages": num_pages, "lens": lens,
        "cache_recipe": ("rows written by mla_append_cache from hidden states x ~ N(0,1): c = RMSNorm(x W_DKV), "
                         "k_r = RoPE(x W_KR)") if from_hidden else
                        "latent rows uniform on the sphere of radius sqrt(d_c), RoPE keys N(0,1)",
        "seqlens": torch.from_numpy(lens).to(device), "table": torch.from_numpy(table).to(device),
        "w_dkv_kr": torch.from_numpy(np.concatenate([W["W_DKV"], W["W_KR"]], 1)).to(device=device, dtype=tdt),
        "W_UK": torch.from_numpy(W["W_UK"]).to(device=device, dtype=tdt),
        "W_UV": torch.from_numpy(W["W_UV"]).to(device=device, dtype=tdt),
        "x_host": torch.from_numpy(step["x"]).to(tdt).pin_memory(),
        "q_nope_host": torch.from_numpy(step["q_nope"]).to(tdt).pin_memory(),
        "q_rope_host": torch.from_numpy(step["q_rope_raw"]).to(tdt).pin_memory(),
    }
    if w.d_q:   # the query chain's weights
        for k in ("W_DQ", "gamma_q", "W_UQ", "W_QR"):
            dev[k] = torch.from_numpy(W[k]).to(device=device, dtype=tdt)
    dev["x"] = dev["x_host"].to(device)
    dev["q_nope"] = dev["q_nope_host"].to(device)
    dev["q_rope_raw"] = dev["q_rope_host"].to(device)
    return dev


# configurations whose decode call the default run also times on its own: long-context split-KV,
# the GQLA grouped path, multi-token steps with 2 and 4 new tokens
SECONDARY = ("longctx_b8", "gqla_g8_b32_l8192", "mtp_sq2_b128", "mtp_sq4_b128", "dsv3_fp8_b64_l4096")


def run_e2e(args, w, dev, step, out, stream, device, world, from_x, e_steps):
    """End-to-end steps through the public API with host buffers: returns ({ms, h2d, d2h}, graph_ok)."""
    import torch
    import torch.distributed as dist
    x_host, qn_host, qr_host = dev["x_host"], dev["q_nope_host"], dev["q_rope_host"]
    ins = [(torch.empty_like(x_host, device=device), torch.empty_like(qn_host, device=device),
            torch.empty_like(qr_host, device=device)) for _ in range(2)]
    outs = [torch.empty_like(out) for _ in range(2)]
    out_host = [torch.empty(out.shape, dtype=out.dtype).pin_memory() for _ in range(2)]
    for k in range(2):
        ins[k][0].copy_(x_host)
        ins[k][1].copy_(qn_host)
        ins[k][2].copy_(qr_host)

    def body(k):
        xi, qn, qr = ins[k]
        step(xi, None if from_x else qn, None if from_x else qr, out_t=outs[k])

    graphs, graph_ok = [], True
    try:
        side = torch.cuda.Stream(device)
        side.wait_stream(stream)
        with torch.cuda.stream(side):
            for k in range(2):
                body(k)
        stream.wait_stream(side)
        torch.cuda.synchronize()
        for k in range(2):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                body(k)
            graphs.append(g)
        torch.cuda.synchronize()
    except Exception:  # noqa: BLE001  (capture unavailable: the same calls, launched directly)
        graphs, graph_ok = [], False
        torch.cuda.synchronize()

    def device_step(k):
        if graph_ok:
            graphs[k].replay()
        else:
            body(k)

    h2d_s, d2h_s = torch.cuda.Stream(device), torch.cuda.Stream(device)
    ev = {n: [torch.cuda.Event() for _ in range(2)] for n in ("in_ready", "done", "out_free")}
    for k in range(2):   # every event recorded once, so the first waits return at once
        for n in ev:
            ev[n][k].record(stream)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(e_steps):
        k = i % 2
        h2d_s.wait_event(ev["done"][k])            # step i-2 has finished reading these inputs
        with torch.cuda.stream(h2d_s):
            ins[k][0].copy_(x_host, non_blocking=True)
            if not from_x:
                ins[k][1].copy_(qn_host, non_blocking=True)
                ins[k][2].copy_(qr_host, non_blocking=True)
        ev["in_ready"][k].record(h2d_s)
        stream.wait_event(ev["in_ready"][k])
        stream.wait_event(ev["out_free"][k])       # step i-2's result has left this buffer
        device_step(k)
        ev["done"][k].record(stream)
        d2h_s.wait_event(ev["done"][k])
        with torch.cuda.stream(d2h_s):
            out_host[k].copy_(outs[k], non_blocking=True)
        ev["out_free"][k].record(d2h_s)
    for k in range(2):
        stream.wait_event(ev["out_free"][k])
    e1.record(stream)
    torch.cuda.synchronize()
    ms = max_over_ranks(e0.elapsed_time(e1), world, device)
    h2d = x_host.numel() * x_host.element_size()
    if not from_x:
        h2d += qn_host.numel() * qn_host.element_size() + qr_host.numel() * qr_host.element_size()
    d2h = out_host[0].numel() * out_host[0].element_size()
    del graphs
    return {"ms": ms, "h2d": h2d, "d2h": d2h}, graph_ok


def gpu_latent_pool(w, num_pages, device, seed=2):
    """A paged latent pool drawn on the GPU with the recipe of synth.cache_row_chunks: latent rows
    uniform on the sphere of radius sqrt(d_c), RoPE keys N(0, 1) (drawn by torch's CUDA generator,
    in chunks, so that large pools need no host work)."""
    import torch
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    rows = num_pages * 64
    pool = torch.empty(rows, w.d_c + w.d_r, dtype=torch.bfloat16, device=device)
    step = 1 << 20
    for r0 in range(0, rows, step):
        n = min(step, rows - r0)
        g = torch.randn(n, w.d_c, generator=gen, device=device)
        pool[r0:r0 + n, :w.d_c] = g * (math.sqrt(w.d_c) / g.norm(dim=1, keepdim=True))
        pool[r0:r0 + n, w.d_c:] = torch.randn(n, w.d_r, generator=gen, device=device)
    return pool


def time_decode_alone(name, device, steps, warmup, peaks):
    """The decode call of one workload on its own (absorbed, or grouped for a GQLA workload), timed
    with CUDA events around each call on the launching stream; returns its line fragment."""
    import numpy as np
    import torch
    import synth
    from mla_compressed_latent_b200 import ops
    from mla_compressed_latent_b200.ops import Dims, LatentCache, GqaCache
    w = synth.workload(name)
    dims = Dims.of(w)
    lens = synth.seq_lengths(w)
    table, num_pages = synth.block_table(w, lens)
    tbl = torch.from_numpy(table).to(device)
    seqlens = torch.from_numpy(lens).to(device)
    gen = torch.Generator(device=device)
    gen.manual_seed(1)
    stream = torch.cuda.current_stream()
    total = int(lens.sum())
    n_tok = w.B * w.s_q
    if w.g:
        rows = num_pages * 64
        K = torch.randn(rows, w.g, w.D, generator=gen, device=device).to(torch.bfloat16)
        V = torch.randn(rows, w.g, w.d_v, generator=gen, device=device).to(torch.bfloat16)
        R = torch.randn(rows, w.d_r, generator=gen, device=device).to(torch.bfloat16)
        qn = torch.randn(w.B, w.s_q, w.H, w.D, generator=gen, device=device).to(torch.bfloat16)
        qr = torch.randn(w.B, w.s_q, w.H, w.d_r, generator=gen, device=device).to(torch.bfloat16)
        cache = GqaCache(K, V, R, num_pages)
        out = torch.empty(w.B, w.s_q, w.H, w.d_v, dtype=torch.bfloat16, device=device)
        lse = torch.empty(w.B, w.s_q, w.H, dtype=torch.float32, device=device)
        import ctypes
        from mla_compressed_latent_b200 import _lib as L
        dc = dims.c()
        ws = torch.empty(max(16, int(L.load().mla_gqla_workspace_size(ctypes.byref(dc), L.MLA_BF16, w.B, w.s_q,
                                                                      table.shape[1]))),
                         dtype=torch.uint8, device=device)

        def call():
            ops.mla_decode_gqla_grouped(dims, qn, qr, cache, tbl, seqlens, out=out, lse=lse, workspace=ws)
        bytes_ = total * (w.g * (w.D + w.d_v) + w.d_r) * 2 + n_tok * w.H * (w.D + w.d_r + w.d_v) * 2 + n_tok * w.H * 4
        flops = total * w.H * 2 * ((w.D + w.d_r) + w.d_v)
        kernel = "mla_decode_gqla_grouped (decode + split merge)"
    else:
        pool = gpu_latent_pool(w, num_pages, device)
        cache = LatentCache(pool[:, :w.d_c], pool[:, w.d_c:], num_pages)
        q_abs = torch.randn(w.B, w.s_q, w.H, w.d_c + w.d_r, generator=gen, device=device)
        q_abs[..., :w.d_c] *= math.sqrt(w.D / w.d_c)
        q_abs = q_abs.to(torch.bfloat16)
        o_lat = torch.empty(w.B, w.s_q, w.H, w.d_c, dtype=torch.bfloat16, device=device)
        lse = torch.empty(w.B, w.s_q, w.H, dtype=torch.float32, device=device)
        bytes_, flops, _ = decode_counts(w, lens)
        if w.latent_bits == 8:
            # the 16-bit pool converted once by the library's quantiser; the RoPE keys stay 16-bit
            from mla_compressed_latent_b200.ops import LatentCacheFp8
            cache8 = LatentCacheFp8.empty_like(cache)
            ops.mla_quantize_latent_fp8(dims, cache.latent, cache8.codes, cache8.scales)
            del pool, cache
            import ctypes
            from mla_compressed_latent_b200 import _lib as L
            dc = dims.c()
            ws = torch.empty(max(16, int(L.load().mla_decode_fp8_workspace_size(ctypes.byref(dc), w.B, w.s_q,
                                                                                 table.shape[1]))),
                             dtype=torch.uint8, device=device)

            def call():
                ops.mla_decode_absorbed_fp8(dims, q_abs, cache8, tbl, seqlens, o_lat=o_lat, lse=lse, workspace=ws)
            kernel = "mla_decode_absorbed_fp8 (pages dequantised to a bf16 scratch, then the tensor-core decode)"
        else:
            ws = torch.empty(max(16, ops.mla_decode_workspace_size(dims, torch.bfloat16, w.B, w.s_q, table.shape[1])),
                             dtype=torch.uint8, device=device)

            def call():
                ops.mla_decode_absorbed(dims, q_abs, cache, tbl, seqlens, o_lat=o_lat, lse=lse, workspace=ws)
            kernel = "mla_decode_absorbed (decode + split merge)"
    for _ in range(warmup):
        call()
    torch.cuda.synchronize()
    rc = ops.mla_check_status()
    if rc != 0:
        raise RuntimeError(f"{name}: device status {ops.mla_status_string(rc)}")
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    for a, b in evs:
        a.record(stream)
        call()
        b.record(stream)
    torch.cuda.synchronize()
    sec = statistics.mean(a.elapsed_time(b) for a, b in evs) / 1e3
    gbs, tfs = bytes_ / sec / 1e9, flops / sec / 1e12
    t_hbm, t_tc = bytes_ / (peaks["hbm_gbs"] * 1e9), flops / (peaks["bf16_tflops"] * 1e12)
    if t_tc > t_hbm:
        roof = {"bound": "tensor", "achieved": tfs, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                "frac": tfs / peaks["bf16_tflops"],
                "frac_sustained": tfs / peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"]),
                "frac_nominal": tfs / NOMINAL_PEAKS["bf16_tflops"], "hbm_gbs": gbs}
    else:
        roof = {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": gbs / peaks["hbm_gbs"], "frac_nominal": gbs / NOMINAL_PEAKS["hbm_gbs"], "tensor_tflops": tfs}
    roof.update({"traffic": None, "kernel": kernel, "bytes_per_launch": bytes_, "flops_per_launch": flops})
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    return {"decode_us": sec * 1e6, "positions_per_s": total / sec, "tokens_per_s": n_tok / sec,
            "config": {"B": w.B, "s_q": w.s_q, "lengths": list(w.lengths), "pages": w.pages, "g": w.g,
                       "positions": total},
            "roofline": roof, "steps": steps, "inputs": "drawn on the GPU (torch CUDA generator), synth recipe"}


def fill_cache_from_hidden_states(w, pool, num_pages, table, lens, W, device, seed=2):
    """Fill every sequence's cached rows through mla_append_cache from x ~ N(0, 1) (all sequences
    the same length, a multiple of 64): call k appends positions 64k .. 64k+63 of every sequence."""
    import numpy as np
    import torch
    from mla_compressed_latent_b200 import ops
    from mla_compressed_latent_b200.ops import Dims, LatentCache
    dims = Dims.of(w)
    cache = LatentCache(pool[:, :w.d_c], pool[:, w.d_c:], num_pages)
    wcat = torch.from_numpy(np.concatenate([W["W_DKV"], W["W_KR"]], 1)).to(device=device, dtype=torch.bfloat16)
    tbl = torch.from_numpy(table).to(device)
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    L = int(lens[0])
    for k in range(L // 64):
        x = torch.randn(w.B, 64, w.C, generator=gen, device=device).to(torch.bfloat16)
        sl = torch.full((w.B,), 64 * (k + 1), dtype=torch.int32, device=device)
        ops.mla_append_cache(dims, x, wcat, None, sl, tbl, cache)
    torch.cuda.synchronize()
    rc = ops.mla_check_status()
    if rc != 0:
        raise RuntimeError(f"cache fill: device status {ops.mla_status_string(rc)}")


def run_grouped(args, w, dims, device, world, rank, local):
    """The GQLA grouped decode (g key/value groups, shared RoPE key) on its own: each step is one
    mla_decode_gqla_grouped call over the whole batch (RoPE of the query included)."""
    import numpy as np
    import torch
    import torch.distributed as dist
    import synth
    from mla_compressed_latent_b200 import ops
    from mla_compressed_latent_b200.ops import GqaCache
    lens = synth.seq_lengths(w)
    table, num_pages = synth.block_table(w, lens)
    n = num_pages * 64
    K = torch.empty(n, w.g, w.D, dtype=torch.bfloat16, device=device)
    V = torch.empty(n, w.g, w.d_v, dtype=torch.bfloat16, device=device)
    R = torch.empty(n, w.d_r, dtype=torch.bfloat16, device=device)
    gcache = GqaCache(K, V, R, num_pages)
    seqlens = torch.from_numpy(lens).to(device)
    tbl = torch.from_numpy(table).to(device)
    L0 = int(lens[0])
    if (lens == L0).all() and L0 % 64 == 0:
        # the expanded cache written by mla_append_gqa_cache from hidden states x ~ N(0, 1): call k
        # appends positions 64k .. 64k+63 of every sequence (K_g = W_UK[g] c, V_g = c W_UV[g], k_r)
        W = synth.weights(w)
        wcat = torch.from_numpy(np.concatenate([W["W_DKV"], W["W_KR"]], 1)).to(device=device, dtype=torch.bfloat16)
        wuk = torch.from_numpy(W["W_UK_g"]).to(device=device, dtype=torch.bfloat16)
        wuv = torch.from_numpy(W["W_UV_g"]).to(device=device, dtype=torch.bfloat16)
        gen = torch.Generator(device=device)
        gen.manual_seed(2)
        for k in range(L0 // 64):
            x = torch.randn(w.B, 64, w.C, generator=gen, device=device).to(torch.bfloat16)
            sl = torch.full((w.B,), 64 * (k + 1), dtype=torch.int32, device=device)
            ops.mla_append_gqa_cache(dims, x, wcat, None, wuk, wuv, sl, tbl, gcache)
        cache_note = "rows written by mla_append_gqa_cache from hidden states x ~ N(0,1)"
    else:
        for start, k, v, r in synth.gqla_cache_chunks(w, n):
            K[start:start + len(k)] = torch.from_numpy(k).to(device=device, dtype=torch.bfloat16)
            V[start:start + len(k)] = torch.from_numpy(v).to(device=device, dtype=torch.bfloat16)
            R[start:start + len(k)] = torch.from_numpy(r).to(device=device, dtype=torch.bfloat16)
        cache_note = "rows drawn with the synth recipe"
    torch.cuda.synchronize()
    rc = ops.mla_check_status()
    if rc != 0:
        raise RuntimeError(f"GQA cache fill: device status {ops.mla_status_string(rc)}")
    step_in = synth.decode_step_inputs(w)
    qn = torch.from_numpy(step_in["q_nope"]).to(device=device, dtype=torch.bfloat16)
    qr = torch.from_numpy(step_in["q_rope_raw"]).to(device=device, dtype=torch.bfloat16)
    out = torch.empty(w.B, w.s_q, w.H, w.d_v, dtype=torch.bfloat16, device=device)
    lse = torch.empty(w.B, w.s_q, w.H, dtype=torch.float32, device=device)
    stream = torch.cuda.current_stream()

    def step():
        ops.mla_decode_gqla_grouped(dims, qn, qr, gcache, tbl, seqlens, out=out, lse=lse)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    assert ops.mla_check_status() == 0
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    n0 = ops.mla_launch_count()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:
        t0.record(stream)
        for _ in range(args.steps):
            step()
        t1.record(stream)
        torch.cuda.synchronize()
    launches = ops.mla_launch_count() - n0
    ms = max_over_ranks(t0.elapsed_time(t1), world, device)
    total = int(lens.sum())
    n_tok = w.B * w.s_q
    # per cached position: K and V of every group plus the shared RoPE key; per token: the query
    # parts, the head outputs and the lse
    bytes_ = total * (w.g * (w.D + w.d_v) + w.d_r) * 2 + n_tok * w.H * (w.D + w.d_r + w.d_v) * 2 + n_tok * w.H * 4
    flops = total * w.H * 2 * ((w.D + w.d_r) + w.d_v)
    peaks, peak_kind = load_peaks()
    sec = ms / 1e3 / args.steps
    gbs = bytes_ / sec / 1e9
    line = {
        "metric": METRIC, "value": world * total / sec, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": w.dtype, "data": "synthetic",
        "config": {"workload": w.name, "B": w.B, "seq_len": w.lengths[1] if w.lengths[0] == "fixed" else list(w.lengths),
                   "H": w.H, "g": w.g, "D": w.D, "d_r": w.d_r, "d_v": w.d_v, "s_q": w.s_q,
                   "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                   "l2": f"inputs larger than L2: {total * (w.g * (w.D + w.d_v) + w.d_r) * 2 / 1e6:.0f} MB cache read per step",
                   "cache": cache_note},
        "tokens_per_s": world * n_tok / sec,
        "roofline": {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                     "frac": gbs / peaks["hbm_gbs"],
                     "traffic": captured_traffic(w.name, GQLA_TRAFFIC, GQLA_SOURCES), "peak_source": peak_kind,
                     "kernel": "mla_decode_gqla_grouped (decode + split merge)",
                     "tensor_tflops": flops / sec / 1e12},
        "gpu_launches": int(launches),
        "clocks": clk.summary(),
    }
    if world > 1:
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


def main():
    args = parse()
    rank, world, local = dist_env()
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    import numpy as np
    import torch
    import torch.distributed as dist
    import synth
    from mla_compressed_latent_b200 import ops
    from mla_compressed_latent_b200.ops import Dims, LatentCache

    assert args.warmup >= 3, "at least 3 warm-up steps"
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=180), device_id=device)

    w = synth.workload(args.workload)
    dims = Dims.of(w)
    if args.decode_only:
        peaks, peak_kind = load_peaks()
        with ClockSampler(local) as clk:
            r = time_decode_alone(w.name, device, args.steps, args.warmup, peaks)
        ms = max_over_ranks(r["decode_us"] / 1e3, world, device)
        r["roofline"]["peak_source"] = peak_kind
        line = {"metric": METRIC, "value": world * r["positions_per_s"] * (r["decode_us"] / 1e3) / ms, "unit": UNIT,
                "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": w.dtype, "data": "synthetic",
                "config": {"workload": w.name, **r["config"], "step": "the decode call alone"},
                "tokens_per_s": world * r["tokens_per_s"] * (r["decode_us"] / 1e3) / ms, "decode_us": r["decode_us"],
                "roofline": r["roofline"], "clocks": clk.summary()}
        if world > 1:
            dist.destroy_process_group()
        if rank == 0:
            print(json.dumps(line), flush=True)
        return
    if w.g:
        return run_grouped(args, w, dims, device, world, rank, local)
    dev = build_inputs(w, device)
    cache = LatentCache(dev["pool"][:, :w.d_c], dev["pool"][:, w.d_c:], dev["num_pages"])
    n_tok = w.B * w.s_q
    tdt = dev["pool"].dtype
    q_abs = torch.empty(w.B, w.s_q, w.H, w.d_c + w.d_r, dtype=tdt, device=device)
    o_lat = torch.empty(w.B, w.s_q, w.H, w.d_c, dtype=tdt, device=device)
    lse = torch.empty(w.B, w.s_q, w.H, dtype=torch.float32, device=device)
    out = torch.empty(w.B, w.s_q, w.H, w.d_v, dtype=tdt, device=device)
    max_pages = dev["table"].shape[1]
    ws_dec = torch.empty(max(16, ops.mla_decode_workspace_size(dims, tdt, w.B, w.s_q, max_pages)), dtype=torch.uint8,
                         device=device)
    from mla_compressed_latent_b200 import _lib as L
    import ctypes
    dc = dims.c()
    ws_app = torch.empty(max(16, L.load().mla_append_workspace_size(ctypes.byref(dc), w.B, w.s_q, w.C)),
                         dtype=torch.uint8, device=device)
    stream = torch.cuda.current_stream()
    dec_ev = []
    # a workload with a query latent starts from hidden states: its queries come from x through the
    # query chain inside the step
    from_x = w.d_q > 0
    if from_x:
        qn_buf = torch.empty(w.B, w.s_q, w.H, w.D, dtype=tdt, device=device)
        qr_buf = torch.empty(w.B, w.s_q, w.H, w.d_r, dtype=tdt, device=device)
        ws_q = torch.empty(max(16, L.load().mla_query_workspace_size(ctypes.byref(dc), w.B, w.s_q, w.C, w.d_q)),
                           dtype=torch.uint8, device=device)

    lens_host = np.ascontiguousarray(dev["lens"], dtype=np.int32)

    def step(x, q_nope, q_rope, events=None, out_t=None):
        """One decode step. events: None; "decode" (two events around the decode call, which is all
        the timed region carries, so the other kernels keep overlapping their launches); or "all"
        (an event after every call, for the per-call breakdown outside the timed region)."""
        every = events == "all"
        marks = []

        def mark(name):
            e = torch.cuda.Event(enable_timing=True)
            e.record(stream)
            marks.append((name, e))

        if every:
            mark("start")
        if from_x:
            q_nope, q_rope = ops.mla_project_query(dims, x, dev["W_DQ"], dev["gamma_q"], dev["W_UQ"], dev["W_QR"],
                                                   q_nope=qn_buf, q_rope_raw=qr_buf, workspace=ws_q)
            if every:
                mark("project_q")
        # a1 + a2 in one call: the cache append, then the query absorption (whose CTAs stream W_UK
        # while the append's finish runs)
        ops.mla_append_cache_absorb_q(dims, x, dev["w_dkv_kr"], None, q_nope, q_rope, dev["W_UK"], dev["seqlens"],
                                      dev["table"], cache, q_abs=q_abs, workspace=ws_app)
        if events:
            mark("append_absorb")
        # a3 + a4, with the host's copy of the lengths (a serving host has it): no split machinery
        # when nothing is cut
        ops.mla_decode_absorbed(dims, q_abs, cache, dev["table"], dev["seqlens"], o_lat=o_lat, lse=lse, workspace=ws_dec,
                                seqlens_host=lens_host)
        if events:
            mark("decode")
        ops.mla_out_proj(dims, o_lat, dev["W_UV"], out=out if out_t is None else out_t)
        if every:
            mark("out_proj")
        if events:
            dec_ev.append(dict(marks))

    def between(m, a, b):
        return m[a].elapsed_time(m[b])

    for _ in range(args.warmup):
        step(dev["x"], dev["q_nope"], dev["q_rope_raw"])
    torch.cuda.synchronize()
    rc = ops.mla_check_status()
    if rc != 0:
        raise RuntimeError(f"device status after warm-up: {ops.mla_status_string(rc)}")

    def timed_region():
        dec_ev.clear()
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        n0 = ops.mla_launch_count()
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with ClockSampler(local) as clk:
            t0.record(stream)
            for _ in range(args.steps):
                step(dev["x"], dev["q_nope"], dev["q_rope_raw"], events="decode")
            t1.record(stream)
            torch.cuda.synchronize()
        launches = ops.mla_launch_count() - n0
        ms = max_over_ranks(t0.elapsed_time(t1), world, device)
        if world > 1:
            dist.barrier()
        return ms, launches, clk

    ms, launches, clk = timed_region()
    remeasured = False
    # measured again on every rank if any rank's clocks were rejected (the ranks' collectives stay in step)
    if max_over_ranks(1.0 if clk.rejected() else 0.0, world, device) > 0:
        ms, launches, clk = timed_region()
        remeasured = True
    dec_ms = statistics.mean(between(m, "append_absorb", "decode") for m in dec_ev)
    # per-call breakdown, outside the timed region (its events stop the calls' launches overlapping)
    dec_ev.clear()
    for _ in range(min(args.steps, 50)):
        step(dev["x"], dev["q_nope"], dev["q_rope_raw"], events="all")
    torch.cuda.synchronize()
    calls = (("project_q",) if from_x else ()) + ("append_absorb", "decode", "out_proj")
    order = ("start",) + calls
    breakdown = {c: statistics.mean(between(m, order[i], c) for m in dec_ev) * 1e3 for i, c in enumerate(calls)}
    assert ops.mla_check_status() == 0

    # end to end through the public API: pinned host inputs in, host result out, every step. The
    # device part of a step is one CUDA graph replay (its library calls captured once per buffer
    # set); step i's inputs are copied in on one stream and step i-1's result copied out on another
    # while step i runs on the compute stream (double-buffered device inputs and outputs).
    e_steps = max(3, min(args.steps, 200))
    e2e, graph_ok = run_e2e(args, w, dev, step, out, stream, device, world, from_x, e_steps)
    bytes_, flops, positions = decode_counts(w, dev["lens"])
    peaks, peak_kind = load_peaks()
    step_s = ms / 1e3 / args.steps
    value = world * positions / step_s
    achieved_gbs = bytes_ / (dec_ms / 1e3) / 1e9
    achieved_tf = flops / (dec_ms / 1e3) / 1e12
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": w.dtype, "data": "synthetic",
        "config": {"workload": w.name, "B": w.B, "seq_len": w.lengths[1] if w.lengths[0] == "fixed" else list(w.lengths),
                   "H": w.H, "D": w.D, "d_c": w.d_c, "d_r": w.d_r, "d_v": w.d_v, "s_q": w.s_q,
                   "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                   "l2": f"inputs larger than L2: {positions * (w.d_c + w.d_r) * (2 if w.dtype == 'bf16' else 4) / 1e6:.0f} MB cache read per step",
                   "cache": dev["cache_recipe"]},
        "tokens_per_s": world * n_tok / step_s,
        "decode_us": dec_ms * 1e3,
        "step_breakdown_us": breakdown,
        "roofline": {"bound": "hbm", "achieved": achieved_gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                     "frac": achieved_gbs / peaks["hbm_gbs"], "frac_nominal": achieved_gbs / NOMINAL_PEAKS["hbm_gbs"],
                     "peak_nominal": NOMINAL_PEAKS["hbm_gbs"], "traffic": captured_traffic(w.name), "peak_source": peak_kind,
                     "kernel": "mla_decode_absorbed (decode + split merge)",
                     "tensor_tflops": achieved_tf, "tensor_frac": achieved_tf / peaks["bf16_tflops"],
                     "bound_frac": max(bytes_ / (peaks["hbm_gbs"] * 1e9), flops / (peaks["bf16_tflops"] * 1e12)) / (dec_ms / 1e3),
                     # the decode runs back to back inside the step, under the power cap: against the
                     # sustained tensor peak its FLOPs take longer than its bytes (tensor-bound there)
                     "tensor_frac_sustained": achieved_tf / peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"]),
                     "bound_frac_sustained": max(bytes_ / (peaks["hbm_gbs"] * 1e9),
                                                 flops / (peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"]) * 1e12))
                                             / (dec_ms / 1e3)},
        "gpu_launches": int(launches),
        "clocks": {**clk.summary(), "remeasured": remeasured},
        "e2e": {"value": world * positions / (e2e["ms"] / 1e3 / e_steps), "unit": UNIT,
                "h2d_bytes_per_step": e2e["h2d"], "d2h_bytes_per_step": e2e["d2h"], "steps": e_steps,
                "ms_per_step": e2e["ms"] / e_steps, "cuda_graph": graph_ok,
                "overlap": "inputs copied in and outputs copied out on their own streams, double-buffered"},
    }
    if from_x:
        # the query chain is bound by its weights: W_DQ, W_UQ, W_QR read once per step
        e = 2 if w.dtype == "bf16" else 4
        q_bytes = (w.C * w.d_q + w.d_q * w.H * (w.D + w.d_r)) * e + n_tok * (w.C + w.H * (w.D + w.d_r)) * e
        q_us = breakdown["project_q"]
        line["query_chain"] = {"us": q_us, "bytes": q_bytes, "achieved_gbs": q_bytes / (q_us / 1e6) / 1e9,
                               "frac": q_bytes / (q_us / 1e6) / 1e9 / peaks["hbm_gbs"],
                               "note": "timed with an event after every call (no launch overlap)"}
    if world == 1 and not args.no_secondary:
        # the other configurations' decode calls, each timed on its own (a few seconds in all)
        line["secondary"] = {}
        for name in SECONDARY:
            if name != w.name:
                line["secondary"][name] = time_decode_alone(name, device, max(5, min(args.steps, 20)), 3, peaks)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        pos, tok, el, seqs = oracle_sample(w, args.cpu_seconds)
        line["cpu_baseline"] = {"value": pos / el, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
                                "sample": f"{seqs} of {w.B} sequences ({pos} positions, all {w.H} heads): fp64 absorb + "
                                          f"absorbed decode + W_UV projection, {el:.1f} s"}
    if world > 1:
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
