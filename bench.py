"""Benchmark: prefill attention TFLOP/s and paged-decode KV GB/s on B200.

One step is one pass of the whole hot path over one batch of synthetic input:
  * prefill half: ragged THD causal prefill, 64 sequences with lengths
    U[128, 8192], Hq/Hkv 32/8, D 128, per-batch padded LSE seeded -inf
    (device work list, padded-LSE fill, tcgen05 prefill kernel);
  * decode half: paged-KV decode, batch 128, KV lengths U[1024, 32768], page
    64 with a random page permutation, Hq/Hkv 64/8, D 128, split-KV + LSE merge.
`value` is the prefill half's TFLOP/s (the headline); the decode half is
reported beside it under "decode".  Every input is larger than L2 (126 MB), so
no flush is needed between timed steps.  Also measured per run: the dense
causal prefill (B 8, S 4096) and the absorbed-MLA decode (B 64, 576/512).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Under torchrun (N > 1) every rank runs its own independently seeded batch of
the same shape (weak scaling, no data-path collective); rank 0 prints the
JSON line with the device time maxed over ranks.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "prefill attention TFLOPS and paged-decode KV GB/s, % of B200 roofline"
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}

# DRAM bytes (read + write) from the latest ncu capture of each kernel on its
# small case, as a ratio to the bytes that scale with the launch, applied to
# the full launch.  None when the kernel changed after the counters were taken
# or has no capture.
#   ragged_prefill: per Q+K+V+O byte, 16 sequences (1.0432 / 1.0611 GB)
#   paged_decode: per K/V byte, batch 16, 2 splits (1.3665 / 1.3589 GB)
#   mla_decode: per K/V byte, batch 8 (0.3439 / 0.3355 GB; the partials grow with the
#     batch like the K/V bytes)
#   paged_prefill: per Q+O+K+V byte, 4 chunks of 1024 queries (0.6825 / 0.6345 GB)
#   dense_prefill: per Q+K+V+O byte, the bench's own size, batch 8 (0.7054 / 0.6711 GB)
TRAFFIC_RATIO = {"ragged_prefill": 0.9831, "paged_decode": 1.0056, "mla_decode": 1.0262, "paged_prefill": 1.0756,
                 "dense_prefill": 1.0511}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return dict(PEAKS_FALLBACK), "fallback"


# --------------------------------------------------------------------------- #
# workload sizes (algorithmic units)
# --------------------------------------------------------------------------- #
def prefill_flops(lq, lkv, Hq, D, causal=True):
    """4 * D flops per visible (query, key) pair per query head (QK^T and PV)."""
    tot = 0
    for a, b in zip(lq, lkv):
        a, b = int(a), int(b)
        if causal:
            # rows i see min(b, i + b - a + 1) keys (bottom-right)
            i = np.arange(a, dtype=np.int64)
            tot += int(np.clip(i + b - a + 1, 0, b).sum())
        else:
            tot += a * b
    return 4.0 * D * Hq * tot


def decode_kv_bytes(kv_lens, Hkv, Dqk, Dv, alias):
    per_tok = Hkv * (Dqk if alias else Dqk + Dv) * 2
    return float(np.sum(np.asarray(kv_lens, dtype=np.int64)) * per_tok)


# --------------------------------------------------------------------------- #
# clocks sampler
# --------------------------------------------------------------------------- #
class ClockSampler:
    """SM clock, its maximum and the clock-event reasons, sampled while the
    parts are timed: read-only NVML queries every 20 ms from a thread (the GPU
    matched by PCI bus id, which holds under CUDA_VISIBLE_DEVICES), else
    `nvidia-smi -lms 100`.  Lines are kept in nvidia-smi's CSV field order."""
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    # NVML clock-event reason bits (nvml.h): hw_slowdown, hw_thermal_slowdown,
    # sw_thermal_slowdown, sw_power_cap, in FIELDS order
    REASON_BITS = (0x8, 0x40, 0x20, 0x4)

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.nvml = None
        self.lines = []
        # samples are kept only while a part is being timed (not in the idle gaps
        # between parts, whose clocks say nothing about the measurement)
        self.active = False

    def __enter__(self):
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            p = torch.cuda.get_device_properties(self.index)
            bus = f"{p.pci_domain_id:08X}:{p.pci_bus_id:02X}:{p.pci_device_id:02X}.0"
            self.handle = pynvml.nvmlDeviceGetHandleByPciBusId(bus)
            self.nvml = pynvml
            self._stop = threading.Event()
            self._sample_nvml(force=True)  # one sample before the timing starts
            self._t = threading.Thread(target=self._loop_nvml, daemon=True)
            self._t.start()
            return self
        except Exception:
            self.nvml = None
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self._t = threading.Thread(target=self._read, daemon=True)
            self._t.start()
        except (OSError, ValueError):
            self.proc = None
        return self

    def _sample_nvml(self, force=False):
        if not (self.active or force):
            return
        n, h = self.nvml, self.handle
        sm = n.nvmlDeviceGetClockInfo(h, n.NVML_CLOCK_SM)
        mx = n.nvmlDeviceGetMaxClockInfo(h, n.NVML_CLOCK_SM)
        watts = n.nvmlDeviceGetPowerUsage(h) / 1000.0
        r = n.nvmlDeviceGetCurrentClocksEventReasons(h)
        flags = ["Active" if r & bit else "Not Active" for bit in self.REASON_BITS]
        self.lines.append(", ".join([str(sm), str(mx), f"{watts:.1f}", hex(r)] + flags))

    def _loop_nvml(self):
        while not self._stop.wait(0.02):
            try:
                self._sample_nvml()
            except Exception:
                return

    def _read(self):
        for ln in self.proc.stdout:
            if self.active:
                self.lines.append(ln.strip())

    def __exit__(self, *a):
        if self.nvml is not None:
            self._stop.set()
            self._t.join(timeout=5)
            try:
                self.nvml.nvmlShutdown()
            except Exception:
                pass
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                mx = float(parts[1])
            except ValueError:
                continue
            for n, val in zip(names, parts[4:8]):
                if val.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# --------------------------------------------------------------------------- #
# our implementation
# --------------------------------------------------------------------------- #
class Part:
    """One half of the hot path: inputs resident on the device plus a step()."""

    def __init__(self, name, unit, units_per_step, launches_per_step, step, e2e=None, info=None):
        self.name, self.unit, self.units = name, unit, units_per_step
        self.launches = launches_per_step
        self.step = step
        self.e2e = e2e
        self.info = info or {}


def _with_batch(synth, w, B):
    return w if not B else synth.Workload(**{**w.__dict__, "B": B})


def make_ragged_prefill(torch, rsd, synth, dev, seed_offset, B=0):
    w = _with_batch(synth, synth.WORKLOADS["ragged_prefill"], B)
    L = synth.uniform_lengths(w.B, *w.len_range, w.seed + seed_offset)
    q, k, v, cu = synth.make_ragged(w, dev, lengths=L)
    T = q.shape[0]
    smax = int(L.max())
    o = torch.empty_like(q)
    lse = torch.empty((w.B, smax, w.Hq), dtype=torch.float32, device=dev)
    ws = torch.empty(rsd.attn_fwd_ragged_workspace_size(w.B, smax, T, w.Hq, w.Hkv), dtype=torch.uint8,
                     device=dev)
    cud = torch.as_tensor(cu, device=dev)

    def step(qq=q, kk=k, vv=v, oo=o, ll=lse, cc=cud):
        rsd.attn_fwd_ragged(qq, kk, vv, oo, ll, cc, cc, max_seqlen_q=smax, max_seqlen_kv=smax,
                            scale=w.scale, causal=True, workspace=ws)

    def e2e_setup():
        hq, hk, hv = (t.cpu().pin_memory() for t in (q, k, v))
        hcu = torch.as_tensor(cu).pin_memory()
        ho = [torch.empty(o.shape, dtype=o.dtype).pin_memory() for _ in range(2)]
        hl = [torch.empty(lse.shape, dtype=lse.dtype).pin_memory() for _ in range(2)]
        # two sets of device buffers, so one step's copies overlap the other's compute
        dev_in = [(torch.empty_like(q), torch.empty_like(k), torch.empty_like(v), torch.empty_like(cud))
                  for _ in range(2)]
        dev_out = [(torch.empty_like(o), torch.empty_like(lse)) for _ in range(2)]

        def h2d(b):
            for dst, src in zip(dev_in[b], (hq, hk, hv, hcu)):
                dst.copy_(src, non_blocking=True)

        def compute(b):
            dq, dk, dv, dcu = dev_in[b]
            step(dq, dk, dv, dev_out[b][0], dev_out[b][1], dcu)

        def d2h(b):
            ho[b].copy_(dev_out[b][0], non_blocking=True)
            hl[b].copy_(dev_out[b][1], non_blocking=True)

        def read(b):
            return float(hl[b][0, 0, 0])
        h2d_bytes = sum(t.numel() * t.element_size() for t in (hq, hk, hv, hcu))
        d2h_bytes = ho[0].numel() * ho[0].element_size() + hl[0].numel() * hl[0].element_size()
        return (h2d, compute, d2h, read), h2d_bytes, d2h_bytes

    flops = prefill_flops(L, L, w.Hq, w.Dqk)
    io_gb = T * (2 * w.Hq * w.Dqk + w.Hkv * (w.Dqk + w.Dv)) * 2 / 1e9
    info = {"workload": w.notes, "B": w.B, "total_tokens": int(T), "max_seqlen": smax,
            "Hq": w.Hq, "Hkv": w.Hkv, "D": w.Dqk, "flop_per_step": flops,
            "flop_per_unit": "4*D per visible (query, key) pair per query head",
            "traffic_basis_gb": io_gb}
    data = dict(q=q, k=k, v=v, cu=cu, L=L, w=w)
    return Part("ragged_prefill", "TFLOP/s", flops / 1e12, 2, step, e2e_setup, info), data


def make_dense_prefill(torch, rsd, synth, dev, seed_offset, B=0):
    w = _with_batch(synth, synth.WORKLOADS["dense_prefill"], B)
    g = synth.Workload(**{**w.__dict__, "seed": w.seed + seed_offset})
    q, k, v = synth.make_dense(g, dev)
    o = torch.empty_like(q)
    lse = torch.empty((w.B, w.Hq, w.S), dtype=torch.float32, device=dev)
    ws = torch.empty(rsd.attn_fwd_dense_workspace_size(w.B, w.S, w.Hq, w.Hkv), dtype=torch.uint8, device=dev)

    def step():
        rsd.attn_fwd_dense(q, k, v, o, lse, scale=w.scale, causal=True, workspace=ws)
    flops = prefill_flops([w.S] * w.B, [w.S] * w.B, w.Hq, w.Dqk)
    # bytes that scale with the launch: Q, K, V and O
    io_gb = w.B * w.S * (2 * w.Hq * w.Dqk + w.Hkv * (w.Dqk + w.Dv)) * 2 / 1e9
    info = {"workload": w.notes, "flop_per_step": flops, "traffic_basis_gb": io_gb}
    # the device work list and the prefill kernel
    return Part("dense_prefill", "TFLOP/s", flops / 1e12, 2, step, None, info), None


def make_paged_prefill(torch, rsd, synth, dev, seed_offset, B=0):
    w = _with_batch(synth, synth.WORKLOADS["paged_prefill"], B)
    L = synth.uniform_lengths(w.B, *w.len_range, w.seed + seed_offset)
    q, kp, vp, table, kl, cu_q, lq = synth.make_paged_prefill(w, dev, kv_lens=L)
    T = q.shape[0]
    smax = int(lq.max())
    o = torch.empty_like(q)
    lse = torch.empty((w.B, smax, w.Hq), dtype=torch.float32, device=dev)
    ws = torch.empty(rsd.attn_fwd_paged_prefill_workspace_size(w.B, smax, T, w.Hq, w.Hkv, w.Dqk, 1), dtype=torch.uint8,
                     device=dev)
    cud = torch.as_tensor(cu_q, device=dev)
    pt = torch.as_tensor(table, device=dev)
    kld = torch.as_tensor(kl, device=dev)
    maxL = int(L.max())

    def step():
        rsd.attn_fwd_paged_prefill(q, kp, vp, o, lse, cud, pt, kld, max_seqlen_q=smax, page_size=w.page_size,
                                   max_kv_len=maxL, scale=w.scale, causal=True, workspace=ws)
    flops = prefill_flops(lq, L, w.Hq, w.Dqk)
    # bytes that scale with the launch: Q and O of every query, K and V of every cached key
    io_gb = (T * 2 * w.Hq * w.Dqk * 2 + int(L.sum()) * 2 * w.Hkv * w.Dqk * 2) / 1e9
    info = {"workload": w.notes, "flop_per_step": flops, "query_tokens": int(T),
            "kv_tokens": int(L.sum()), "total_pages": int(kp.shape[0]), "traffic_basis_gb": io_gb}
    # padded-LSE fill, the short-row decode kernel (its blocks leave at once: every
    # sequence here has 1024 queries), the work list and the prefill kernel
    return Part("paged_prefill", "TFLOP/s", flops / 1e12, 3, step, None, info), None


def make_mixed(torch, rsd, synth, dev, seed_offset, num_sms, subset="all"):
    """The mixed decode / chunked-prefill batch over a paged cache through
    attn_fwd_paged_prefill: subset "all" (one call for every row), "short"
    (only the 1-4-query rows: K/V GB/s of the split-KV decode kernel) or
    "chunks" (only the 1024-query chunks: TFLOP/s of the prefill kernel)."""
    w0 = synth.WORKLOADS["mixed_batch"]
    w = synth.Workload(**{**w0.__dict__, "seed": w0.seed + seed_offset})
    q, kp, vp, table, kl, cu_q, lq = synth.make_mixed_batch(w, dev, subset)
    L = kl.astype(np.int64)
    T = int(cu_q[-1])
    smax = int(lq.max())
    o = torch.empty_like(q)
    lse = torch.empty((T, w.Hq), dtype=torch.float32, device=dev)
    maxL = int(L.max())
    n_short = int(np.sum((lq >= 1) & (lq <= 4)))
    # the split count of the short rows (none to split without them)
    S = rsd.attn_paged_suggest_splits(n_short, w.Hq, w.Hkv, w.Dqk, w.Dv, maxL, w.page_size, num_sms) if n_short else 1
    ws = torch.empty(rsd.attn_fwd_paged_prefill_workspace_size(w.B, smax, T, w.Hq, w.Hkv, w.Dqk, S),
                     dtype=torch.uint8, device=dev)
    cud = torch.as_tensor(cu_q, device=dev)
    pt = torch.as_tensor(table, device=dev)
    kld = torch.as_tensor(kl, device=dev)

    def step():
        rsd.attn_fwd_paged_prefill(q, kp, vp, o, lse, cud, pt, kld, max_seqlen_q=smax, page_size=w.page_size,
                                   max_kv_len=maxL, scale=w.scale, causal=True, workspace=ws, num_splits=S,
                                   lse_layout=rsd.ATTN_LSE_PACKED_TH)
    flops = prefill_flops(lq, L, w.Hq, w.Dqk)
    short = (lq >= 1) & (lq <= 4)
    kv_short = float(np.sum(L[short])) * w.Hkv * (w.Dqk + w.Dv) * 2
    qmax = min(4, 64 // (w.Hq // w.Hkv), smax)
    # the work list; the short rows' decode (after its split schedule); the prefill kernel
    launches = 1 + (1 + (1 if S > 1 else 0) if qmax > 0 else 0) + (1 if smax > qmax else 0)
    info = {"workload": w.notes, "subset": subset, "num_splits_short_rows": S, "query_tokens": T,
            "short_sequences": n_short, "chunk_sequences": int(np.sum(lq > 4)), "flop_per_step": flops,
            "kv_bytes_short_rows": kv_short, "traffic_basis_gb": kv_short / 1e9}
    if subset == "short":
        info["bytes_per_unit"] = f"{w.Hkv * (w.Dqk + w.Dv) * 2} B of K/V per cached token of a short sequence"
        return Part("mixed_short_rows", "GB/s", kv_short / 1e9, launches, step, None, info)
    name = "mixed_chunks" if subset == "chunks" else "mixed_batch"
    return Part(name, "TFLOP/s", flops / 1e12, launches, step, None, info)


def make_paged(torch, rsd, synth, dev, seed_offset, name, num_sms, B=0):
    w = _with_batch(synth, synth.WORKLOADS[name], B)
    L = synth.uniform_lengths(w.B, *w.len_range, w.seed + seed_offset)
    q, kp, vp, table, kl = synth.make_paged(w, dev, kv_lens=L)
    Dv = w.Dv
    o = torch.empty((w.B, w.Hq, Dv), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((w.B, w.Hq), dtype=torch.float32, device=dev)
    maxL = int(L.max())
    S = rsd.attn_paged_suggest_splits(w.B, w.Hq, w.Hkv, w.Dqk, Dv, maxL, w.page_size, num_sms)
    ws_n = rsd.attn_fwd_paged_workspace_size(w.B, w.Hq, Dv, S)
    ws = torch.empty(max(ws_n, 1), dtype=torch.uint8, device=dev)
    pt = torch.as_tensor(table, device=dev)
    kld = torch.as_tensor(kl, device=dev)

    def step(qq=q, kk=kp, vv=vp, ptt=pt, kll=kld, oo=o, ll=lse):
        rsd.attn_fwd_paged(qq, kk, vv, oo, ll, ptt, kll, page_size=w.page_size, max_kv_len=maxL,
                           scale=w.scale, num_splits=S, workspace=ws)

    def e2e_setup():
        hq = q.cpu().pin_memory()
        hk = kp.cpu().pin_memory()
        hv = hk if w.v_aliases_k else vp.cpu().pin_memory()
        hpt = pt.cpu().pin_memory()
        hkl = kld.cpu().pin_memory()
        ho = [torch.empty(o.shape, dtype=o.dtype).pin_memory() for _ in range(2)]
        hl = [torch.empty(lse.shape, dtype=lse.dtype).pin_memory() for _ in range(2)]
        # two sets of device buffers, so one step's copies overlap the other's compute
        dev_in = []
        for _ in range(2):
            dk = torch.empty_like(kp)
            dv = dk if w.v_aliases_k else torch.empty_like(vp)
            dev_in.append((torch.empty_like(q), dk, dv, torch.empty_like(pt), torch.empty_like(kld)))
        dev_out = [(torch.empty_like(o), torch.empty_like(lse)) for _ in range(2)]

        def h2d(b):
            dq, dk, dv, dpt, dkl = dev_in[b]
            dq.copy_(hq, non_blocking=True)
            dk.copy_(hk, non_blocking=True)
            if not w.v_aliases_k:
                dv.copy_(hv, non_blocking=True)
            dpt.copy_(hpt, non_blocking=True)
            dkl.copy_(hkl, non_blocking=True)

        def compute(b):
            step(*dev_in[b], dev_out[b][0], dev_out[b][1])

        def d2h(b):
            ho[b].copy_(dev_out[b][0], non_blocking=True)
            hl[b].copy_(dev_out[b][1], non_blocking=True)

        def read(b):
            return float(hl[b][0, 0])
        srcs = [hq, hk, hpt, hkl] + ([] if w.v_aliases_k else [hv])
        h2d_bytes = sum(t.numel() * t.element_size() for t in srcs)
        d2h_bytes = ho[0].numel() * ho[0].element_size() + hl[0].numel() * hl[0].element_size()
        return (h2d, compute, d2h, read), h2d_bytes, d2h_bytes

    nbytes = decode_kv_bytes(L, w.Hkv, w.Dqk, Dv, w.v_aliases_k)
    flops = float(np.sum(L)) * w.Hq * 2.0 * (w.Dqk + Dv)
    info = {"workload": w.notes, "num_splits": S, "kv_bytes_per_step": nbytes, "traffic_basis_gb": nbytes / 1e9,
            "flop_per_step": flops, "total_pages": int(kp.shape[0]),
            "bytes_per_unit": f"{w.Hkv * (w.Dqk if w.v_aliases_k else w.Dqk + Dv) * 2} B of K/V per cached token"}
    data = dict(q=q, kp=kp, vp=vp, table=table, L=L, w=w, S=S)
    # with splits: GQA the split schedule and the decode (which merges), MLA the launch-order
    # sort, the decode and the merge
    launches = (3 if w.Dqk == 576 else 2) if S > 1 else 1
    return Part(name, "GB/s", nbytes / 1e9, launches, step, e2e_setup, info), data


def rank_seed_offset(rank):
    """Each rank draws its own synthetic batch of the same shape (weak scaling)."""
    return 1000 * rank


def reduce_over_ranks(value, dist, op, device):
    """One number reduced over all ranks (MAX for times, SUM for units of work);
    the value itself on a single process.  Every rank must call it in the same order."""
    if dist is None:
        return float(value)
    import torch
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=op)
    return float(t.item())


def time_part(torch, part, steps, warmup, dist, world):
    """Device time of `steps` back-to-back steps (barrier + sync on both sides),
    max over ranks; also per-step event durations on the launching stream."""
    stream = torch.cuda.current_stream()
    for _ in range(warmup):
        part.step()
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(steps + 1)]
    ev[0].record(stream)
    for i in range(steps):
        part.step()
        ev[i + 1].record(stream)
    torch.cuda.synchronize()
    total_ms = ev[0].elapsed_time(ev[-1])
    per = [ev[i].elapsed_time(ev[i + 1]) for i in range(steps)]
    if dist is not None:
        total_ms = reduce_over_ranks(total_ms, dist, dist.ReduceOp.MAX, "cuda")
        dist.barrier()
    return total_ms, per


def time_e2e(torch, part, steps, dist):
    """End to end through the public API with host buffers: every step copies
    its inputs from pinned host memory, runs the call and copies the result
    back, and the host reads it.  Steps are pipelined the way a serving loop
    runs them: step i's input copy (one stream) and step i-1's result copy
    (another) overlap step i-1's / step i's compute, on two sets of device
    buffers; the host reads step i-1's result while step i is in flight.
    Device time from the first input copy to the last result copy, max over
    ranks."""
    (h2d, compute, d2h, read), h2d_bytes, d2h_bytes = part.e2e()
    s_in, s_run, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_run = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]

    def run(n, t0=None, t1=None):
        for i in range(n):
            b = i % 2
            with torch.cuda.stream(s_in):
                if i >= 2:
                    s_in.wait_event(ev_run[b])   # step i-2's compute has read buffer set b
                if i == 0 and t0 is not None:
                    t0.record(s_in)
                h2d(b)
                ev_in[b].record(s_in)
            with torch.cuda.stream(s_run):
                s_run.wait_event(ev_in[b])
                if i >= 2:
                    s_run.wait_event(ev_out[b])  # step i-2's result has left output set b
                compute(b)
                ev_run[b].record(s_run)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_run[b])
                d2h(b)
                ev_out[b].record(s_out)
                if i == n - 1 and t1 is not None:
                    t1.record(s_out)
            if i >= 1:
                ev_out[(i - 1) % 2].synchronize()
                read((i - 1) % 2)
        ev_out[(n - 1) % 2].synchronize()
        read((n - 1) % 2)

    run(2)  # warm-up
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    run(steps, t0, t1)
    torch.cuda.synchronize()
    ms = t0.elapsed_time(t1)
    if dist is not None:
        ms = reduce_over_ranks(ms, dist, dist.ReduceOp.MAX, "cuda")
    return ms, h2d_bytes, d2h_bytes


def oracle_prefill_sample(data, seconds):
    """The fp64 oracle on a random sample of rows of the prefill batch.
    Returns (TFLOP/s, threads, description)."""
    import oracle
    import synth
    w, L, cu = data["w"], data["L"], data["cu"]
    orc = oracle.default()
    qb, kb, vb = (synth.bf16_bits(data[n]) for n in ("q", "k", "v"))
    rng = np.random.default_rng(12345)

    def draw(n):
        b = rng.integers(0, len(L), n)
        i = (rng.random(n) * L[b]).astype(np.int64)
        h = rng.integers(0, w.Hq, n)
        return np.stack([b, h, i], 1).astype(np.int32)

    def run(rows):
        t0 = time.perf_counter()
        orc.attn_ragged_rows(qb, kb, vb, cu, cu, w.Hq, w.Hkv, w.scale, True, rows)
        dt = time.perf_counter() - t0
        fl = 4.0 * w.Dqk * float(np.sum(rows[:, 2].astype(np.int64) + 1))
        return fl, dt

    fl, dt = run(draw(256))
    n = int(max(256, min(2_000_000, 256 * seconds / max(dt, 1e-3))))
    rows = draw(n)
    fl, dt = run(rows)
    return fl / dt / 1e12, orc.num_threads(), (
        f"{n} random (sequence, head, query) rows of the ragged prefill batch, "
        f"{fl / 1e9:.1f} GFLOP in {dt:.1f} s")


def oracle_decode_sample(data, seconds):
    """The fp64 oracle on a random sample of (sequence, kv head) groups of the
    decode batch (all G query heads of each group).  Returns (GB/s, threads, desc)."""
    import oracle
    import synth
    w, L, table = data["w"], data["L"], data["table"]
    orc = oracle.default()
    qb = synth.bf16_bits(data["q"])
    kb = synth.bf16_bits(data["kp"])
    vb = kb if w.v_aliases_k else synth.bf16_bits(data["vp"])
    kp = data["kp"]
    ks = (kp.stride(0), kp.stride(2), kp.stride(1))
    vs = ks if w.v_aliases_k else (data["vp"].stride(0), data["vp"].stride(2), data["vp"].stride(1))
    G = w.Hq // w.Hkv
    rng = np.random.default_rng(54321)

    def run(ngroups):
        b = rng.integers(0, w.B, ngroups)
        g = rng.integers(0, w.Hkv, ngroups)
        rows = np.array([(bb, gg * G + j) for bb, gg in zip(b, g) for j in range(G)], dtype=np.int32)
        t0 = time.perf_counter()
        orc.attn_paged_rows(qb, kb, vb, table, L.astype(np.int32), w.page_size, w.Hq, w.Hkv, w.Dqk,
                            w.Dv, ks, vs, w.scale, rows)
        dt = time.perf_counter() - t0
        nb = float(np.sum(L[b])) * (w.Dqk if w.v_aliases_k else w.Dqk + w.Dv) * 2
        return nb, dt, len(rows)

    nb, dt, _ = run(4)
    n = int(max(4, min(100_000, 4 * seconds / max(dt, 1e-3))))
    nb, dt, nrows = run(n)
    return nb / dt / 1e9, orc.num_threads(), (
        f"{n} random (sequence, kv head) groups ({nrows} query rows) of the decode batch, "
        f"{nb / 1e9:.2f} GB of K/V in {dt:.1f} s")


def run_ours(args):
    import torch
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    dist = None
    if world > 1:
        import datetime

        import torch.distributed as tdist
        torch.cuda.set_device(local)
        tdist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
        dist = tdist
    else:
        torch.cuda.set_device(0)
    dev = "cuda"
    import ragged_scaled_dot_b200 as rsd
    import synth
    rsd.lib()  # fails loudly if the CUDA library is missing
    peaks, peak_src = load_peaks()
    num_sms = torch.cuda.get_device_properties(local).multi_processor_count

    off = rank_seed_offset(rank)
    prefill, pdata = make_ragged_prefill(torch, rsd, synth, dev, off)
    decode, ddata = make_paged(torch, rsd, synth, dev, off, "paged_decode", num_sms)
    extras = []
    if not args.no_extras:
        extras.append(make_dense_prefill(torch, rsd, synth, dev, off)[0])
        extras.append(make_paged_prefill(torch, rsd, synth, dev, off)[0])
        mla, _ = make_paged(torch, rsd, synth, dev, off, "mla_decode", num_sms)
        extras.append(mla)
        small, _ = make_paged(torch, rsd, synth, dev, off, "decode_small_batch", num_sms)
        extras.append(small)
        for subset in ("all", "short", "chunks"):
            extras.append(make_mixed(torch, rsd, synth, dev, off, num_sms, subset))
    torch.cuda.synchronize()

    results = {}
    with ClockSampler(local) as clocks:
        for i, part in enumerate([prefill, decode] + extras):
            if i > 0 and args.part_gap > 0:
                # every part starts from an idle GPU: the power state one part leaves
                # behind would otherwise carry into the next (the dense prefill measured
                # ~12 % slower right after the ragged prefill than after 2 s idle)
                torch.cuda.synchronize()
                time.sleep(args.part_gap)
            clocks.active = True
            total_ms, per = time_part(torch, part, args.steps, args.warmup, dist, world)
            clocks.active = False
            results[part.name] = (total_ms, per)
    assert rsd.attn_get_device_error() == rsd.ATTN_OK, "device-side error during the bench"

    sum_op = dist.ReduceOp.SUM if dist is not None else None
    # units of work of all ranks (their seeded batches differ in length)
    all_units = {p.name: reduce_over_ranks(p.units, dist, sum_op, "cuda") for p in [prefill, decode] + extras}

    def part_summary(part, bound):
        total_ms, per = results[part.name]
        ms = total_ms / args.steps
        value = all_units[part.name] / (total_ms / 1e3 / args.steps)
        # dominant kernel: the part's launch sequence, timed per step on its stream
        kern_ms = statistics.mean(per)
        if bound == "tensor":
            achieved = part.units / (kern_ms / 1e3)
            peak = peaks["bf16_tflops"]
            tpu = TRAFFIC_RATIO.get(part.name)
            roof = {"bound": "tensor", "achieved": round(achieved, 2), "peak": peak, "unit": "TFLOP/s",
                    "frac": round(achieved / peak, 4),
                    "traffic": None if tpu is None else round(part.info["traffic_basis_gb"] * tpu, 3),
                    "traffic_unit": "GB per launch (dram read + write)",
                    "frac_of_sustained": round(achieved / peaks.get("bf16_tflops_sustained", peak), 4),
                    "peak_source": f"{peak_src} bf16_tflops (burst)"}
        else:
            achieved = part.units / (kern_ms / 1e3)
            peak = peaks["hbm_gbs"]
            tpu = TRAFFIC_RATIO.get(part.name)
            roof = {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                    "frac": round(achieved / peak, 4),
                    "traffic": None if tpu is None else round(part.info["traffic_basis_gb"] * tpu, 3),
                    "traffic_unit": "GB per launch (dram read + write)",
                    "peak_source": f"{peak_src} hbm_gbs"}
        return value, ms, roof

    p_val, p_ms, p_roof = part_summary(prefill, "tensor")
    d_val, d_ms, d_roof = part_summary(decode, "hbm")

    e2e = {}
    for part in ((prefill, decode) if not args.no_e2e else ()):
        n_e2e = max(1, min(6, args.steps))
        ms, h2d, d2h = time_e2e(torch, part, n_e2e, dist)
        e2e[part.name] = {"value": round(all_units[part.name] / (ms / 1e3 / n_e2e), 3),
                          "unit": part.unit, "h2d_bytes_per_step": int(h2d),
                          "d2h_bytes_per_step": int(d2h), "ms_per_step": round(ms / n_e2e, 3),
                          "steps": n_e2e, "pipelined": "copies of one step overlap the compute of the next"}

    cpu = {}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import oracle
        orc = oracle.default()
        all_cores = orc.num_threads()
        v, c, desc = oracle_prefill_sample(pdata, args.cpu_seconds)
        cpu["prefill"] = {"value": round(v, 6), "unit": "TFLOP/s", "cores": c, "kind": "oracle", "sample": desc}
        v, c, desc = oracle_decode_sample(ddata, args.cpu_seconds)
        cpu["decode"] = {"value": round(v, 4), "unit": "GB/s", "cores": c, "kind": "oracle", "sample": desc}
        # the same oracle on one core, on a smaller bounded sample
        orc.set_num_threads(1)
        try:
            v, c, desc = oracle_prefill_sample(pdata, args.cpu_seconds / 3)
            cpu["prefill_single_core"] = {"value": round(v, 7), "unit": "TFLOP/s", "cores": c, "kind": "oracle",
                                          "sample": desc}
            v, c, desc = oracle_decode_sample(ddata, args.cpu_seconds / 3)
            cpu["decode_single_core"] = {"value": round(v, 5), "unit": "GB/s", "cores": c, "kind": "oracle",
                                         "sample": desc}
        finally:
            orc.set_num_threads(all_cores)

    extra_out = {}
    for part in extras:
        bound = "tensor" if part.unit == "TFLOP/s" else "hbm"
        v, ms, roof = part_summary(part, bound)
        extra_out[part.name] = {"value": round(v, 2), "unit": part.unit, "ms_per_step": round(ms, 4),
                                "roofline": roof, **part.info}
        if part.name == "decode_small_batch":
            # the pages print a latency for this shape: 44 us for cuDNN's decode engine (GPU not
            # named), context rather than a target
            extra_out[part.name]["us_per_call"] = round(ms * 1e3, 1)
            extra_out[part.name]["pages_decode_engine_us"] = 44.0
        if part.name == "mla_decode":
            tflops = part.info["flop_per_step"] / 1e12 / (ms / 1e3)
            extra_out[part.name]["tflops"] = round(tflops, 2)
            extra_out[part.name]["tensor_frac"] = round(tflops / peaks["bf16_tflops"], 4)
            ridge_ms = max(part.units / peaks["hbm_gbs"], part.info["flop_per_step"] / 1e12 / peaks["bf16_tflops"]) * 1e3
            extra_out[part.name]["roofline_frac_max_bound"] = round(ridge_ms / ms, 4)

    if rank == 0:
        ck = clocks.summary()
        line = {
            "metric": METRIC,
            "value": round(p_val, 2),
            "unit": "TFLOP/s",
            "n_gpus": world,
            "steps": args.steps,
            "warmup": args.warmup,
            "ms_per_step": round(p_ms, 4),
            "higher_is_better": True,
            "scaling": "weak",
            "vs_baseline": None,
            "dtype": "bf16",
            "data": "synthetic: N(0,1) bf16 Q/K/V, seeded lengths and page permutation",
            "config": {"workload": "ragged THD causal prefill, 64 seqs U[128,8192], Hq/Hkv 32/8, "
                                   "D 128, padded LSE (headline) + paged decode B 128 kv U[1024,32768] "
                                   "page 64, Hq/Hkv 64/8, D 128, split-KV",
                       "global_batch": prefill.info["B"] * world, "seq_len": prefill.info["max_seqlen"],
                       "parallelism": f"replicas x{world} (independent batches)",
                       "l2": "inputs larger than L2 (126 MB); no flush needed",
                       "prefill": prefill.info, "decode": decode.info},
            "roofline": p_roof,
            "e2e": e2e.get("ragged_prefill"),
            "decode": {"metric": "paged-decode KV GB/s", "value": round(d_val, 1), "unit": "GB/s",
                       "ms_per_step": round(d_ms, 4), "roofline": d_roof, "e2e": e2e.get("paged_decode")},
            "extras": extra_out,
            "gpu_launches": args.steps * (prefill.launches + decode.launches)
                            + sum(args.steps * p.launches for p in extras),
            "clocks": {"sm_mhz": ck["sm_mhz"], "sm_max_mhz": ck["sm_max_mhz"], "reasons": ck["reasons"],
                       "samples": ck["samples"]},
        }
        if cpu:
            line["cpu_baseline"] = dict(cpu["prefill"], decode=cpu["decode"],
                                        single_core={"prefill": cpu.get("prefill_single_core"),
                                                     "decode": cpu.get("decode_single_core")})
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()


def run_one(args):
    """Profiling helper: build one part (optionally with a smaller batch), run
    warm-up + timed steps, print a short JSON line.  Not the benchmark line."""
    import torch
    import ragged_scaled_dot_b200 as rsd
    import synth
    torch.cuda.set_device(0)
    rsd.lib()
    num_sms = torch.cuda.get_device_properties(0).multi_processor_count
    if args.only == "ragged_prefill":
        part = make_ragged_prefill(torch, rsd, synth, "cuda", 0, args.batch)[0]
    elif args.only == "dense_prefill":
        part = make_dense_prefill(torch, rsd, synth, "cuda", 0, args.batch)[0]
    elif args.only == "paged_prefill":
        part = make_paged_prefill(torch, rsd, synth, "cuda", 0, args.batch)[0]
    elif args.only.startswith("mixed"):
        part = make_mixed(torch, rsd, synth, "cuda", 0, num_sms,
                          {"mixed_batch": "all", "mixed_short_rows": "short", "mixed_chunks": "chunks"}[args.only])
    else:
        part = make_paged(torch, rsd, synth, "cuda", 0, args.only, num_sms, args.batch)[0]
    total_ms, per = time_part(torch, part, args.steps, args.warmup, None, 1)
    assert rsd.attn_get_device_error() == rsd.ATTN_OK
    print(json.dumps({"part": part.name, "unit": part.unit, "units_per_step": part.units,
                      "ms_per_step": total_ms / args.steps,
                      "value": part.units / (total_ms / 1e3 / args.steps), "info": part.info}), flush=True)


# --------------------------------------------------------------------------- #
# reference arm: the fp64 oracle as it stands, on the host cores
# --------------------------------------------------------------------------- #
def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import torch

    import synth
    w = synth.WORKLOADS["ragged_prefill"]
    L = synth.uniform_lengths(w.B, *w.len_range, w.seed)
    q, k, v, cu = synth.make_ragged(w, "cpu", lengths=L)
    data = dict(q=q, k=k, v=v, cu=cu, L=L, w=w)
    per_step = max(2.0, args.cpu_seconds / 4)
    for _ in range(args.warmup if args.warmup < 2 else 1):
        oracle_prefill_sample(data, 1.0)
    vals, desc, cores = [], "", 1
    t0 = time.perf_counter()
    for _ in range(args.steps):
        v_, cores, desc = oracle_prefill_sample(data, per_step)
        vals.append(v_)
    wall = time.perf_counter() - t0
    value = statistics.mean(vals)
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": "TFLOP/s",
        "n_gpus": int(os.environ.get("WORLD_SIZE", "1")), "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(wall / args.steps * 1e3, 1), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic (same seeds as our arm)",
        "config": {"workload": "ragged THD causal prefill, 64 seqs U[128,8192], Hq/Hkv 32/8, D 128 "
                               "(each step a bounded random row sample)"},
        "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                         "sample": desc},
        "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    del torch
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extras", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--part-gap", type=float, default=2.0,
                    help="seconds of idle GPU before each part after the first")
    ap.add_argument("--only", choices=["ragged_prefill", "paged_decode", "dense_prefill", "paged_prefill",
                                       "mla_decode", "decode_small_batch", "mixed_batch", "mixed_short_rows",
                                       "mixed_chunks"],
                    help="profiling: time one part only and print its own line")
    ap.add_argument("--batch", type=int, default=0, help="profiling: override the part's batch size")
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "ours":
        args.warmup = 3
    if args.impl == "reference":
        run_reference(args)
    elif args.only:
        run_one(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
