#!/usr/bin/env python
"""NVFP4 KV-cache decode benchmark on B200: KV-tokens/s and achieved HBM GB/s.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl native|reference]
                    [--workload NAME] [--no-aux] [--no-cpu-baseline]

One step is one pass of the whole decode hot path over one batch: quantize
every sequence's new token (K and V: E2M1 codes + E4M3 block scales under the
calibrated fp32 tensor scale) and append it to the NVFP4 cache, then run
decode attention over the cache with the NVFP4 -> FP8 dequantization fused in
(plus the merge of split units).

Default workload ("ragged", the large-batch case): B=128 sequences, 32 query
heads, 8 KV heads, head_dim 128, cached lengths uniform in [1024, 8192]
(seeded) plus the appended token, contiguous per-sequence cache slabs, bf16
inputs N(0,1) x per-channel LogNormal(0, 0.5).  Tensor-scale calibration and
the prefill quantization run once during set-up; their throughput is reported
under "aux", next to the other workloads' attention lines (64K context,
128K context with GQA group 12 and 2048-token chunked appends, the 4K GQA
decode step, a paged cache, a hot-L2 run).

Timing: CUDA graphs of consecutive steps replayed on one stream, CUDA events
around exactly K steps after W warm-up steps, barrier + synchronize on both
sides, max over ranks.  Inputs are larger than L2: R replica caches (each with
its own new-token and query buffers) are rotated so that the cache bytes
touched between two visits of a replica exceed twice the L2 size.  N > 1 runs
N independent replicas (one per GPU, no collective in the data path).
"""
import argparse
import datetime
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

import synthetic  # noqa: E402

METRIC = "NVFP4 decode-attention KV-tokens/s and achieved HBM GB/s (% of peak) at 1 B200"
UNIT = "KV-tokens/s"
DTYPE = ("nvfp4 storage (e2m1 codes + e4m3 block scales + f32 tensor scale); e4m3 tcgen05 MMA "
         "operands (K, V exact FP8; q as 2 e4m3 terms, P as 3 e4m3 terms); f32 accumulate")
DEFAULT_WORKLOAD = "ragged"
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
ATTN_SOURCES = ["bit_decode_attention_b200/csrc/nvfp4kv_decode_attention_tc.cu",
                "bit_decode_attention_b200/csrc/nvfp4kv_attention_common.cuh",
                "bit_decode_attention_b200/csrc/nvfp4kv_tcgen05.cuh",
                "bit_decode_attention_b200/csrc/nvfp4kv_device.cuh",
                "bit_decode_attention_b200/csrc/nvfp4kv_pipeline.cuh"]
GEN_SEQS = 16          # sequences drawn per host block when generating prefill inputs


# ---------------------------------------------------------------------------
# helpers
# ---------------------------------------------------------------------------
def env_rank():
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def source_digest(paths):
    h = hashlib.sha256()
    for p in paths:
        with open(os.path.join(ROOT, p), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def profiled_traffic(name):
    """(DRAM bytes per launch from a committed ncu summary, why it is None):
    the bytes only while the kernel source still matches the one that was
    profiled."""
    path = os.path.join(ROOT, "profiles", name)
    try:
        with open(path) as f:
            d = json.load(f)
    except Exception:
        return None, "no ncu capture of this workload under profiles/"
    if d.get("source_digest") != source_digest(ATTN_SOURCES):
        return None, ("kernel sources changed since the capture in profiles/%s (digest %s, %s DRAM "
                      "bytes per launch then); not re-captured"
                      % (name, d.get("source_digest"), d.get("dram_bytes_per_launch")))
    return d.get("dram_bytes_per_launch"), None


def kv_bytes_per_token(Hkv, D):
    """Algorithmic HBM bytes to read one cached token (all KV heads, K and V)."""
    return Hkv * 2 * (D // 2 + D // 16)


def gen_block(w, L, which, c):
    """Host block c of the prefill inputs: sequences GEN_SEQS*c .. +GEN_SEQS-1,
    fp32 values exact in the workload dtype, [nb][L][H_kv][D] (stream 1000 + c
    of the workload's generator)."""
    b0 = c * GEN_SEQS
    nb = min(GEN_SEQS, w.B - b0)
    return synthetic.kv_tokens(w, L, which, stream=1000 + c, batch=nb)


def gen_inputs(w, L, which, device="cuda"):
    """K or V prefill inputs [B][L][H_kv][D] in the workload dtype on `device`,
    drawn on the host one block of GEN_SEQS sequences at a time (gen_block), so
    host memory stays bounded."""
    out = torch.empty(w.B, L, w.Hkv, w.D, dtype=w.torch_dtype(), device=device)
    for c in range((w.B + GEN_SEQS - 1) // GEN_SEQS):
        x = gen_block(w, L, which, c)
        out[c * GEN_SEQS:c * GEN_SEQS + x.shape[0]].copy_(x.to(w.torch_dtype()))
        del x
    return out


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples while the GPU works."""
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        self.samples = []
        self.proc = None
        try:
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            self.id = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
        except Exception:
            self.id = str(device_index)

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "--query-gpu=" + self.QUERY, "--format=csv,noheader,nounits",
                 "-lms", "100", "-i", self.id],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.samples.append((time.time(), line.strip()))

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self, t0, t1):
        rows = []
        for t, line in self.samples:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append((t, float(parts[1]), float(parts[2]), parts))
            except ValueError:
                continue
        inside = [r for r in rows if t0 <= r[0] <= t1]
        window = "timed"
        if not inside:
            inside = [r for r in rows if t0 - 0.5 <= r[0] <= t1 + 0.5]
            window = "timed +-0.5 s"
        if not inside:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0,
                    "note": "no nvidia-smi sample in the timed window"}
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = set()
        for r in inside:
            for i, n in enumerate(names):
                if r[3][5 + i].lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(r[1] for r in inside),
                "sm_max_mhz": max(r[2] for r in inside), "reasons": sorted(reasons),
                "samples": len(inside), "window": window}


def time_events(fn, reps=5, warm=2):
    """Average CUDA-event time (ms) of fn() over `reps` calls after `warm` calls."""
    for _ in range(warm):
        fn()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    a.record()
    for _ in range(reps):
        fn()
    b.record()
    torch.cuda.synchronize()
    return a.elapsed_time(b) / reps


# ---------------------------------------------------------------------------
# the decode workload
# ---------------------------------------------------------------------------
class DecodeWorkload:
    """R replica NVFP4 caches of one workload.  Sequence b holds lens0[b]
    cached tokens; a step appends one token at slot lens0[b] (the same slot
    every visit, so every step attends exactly lens0[b] + 1 tokens) and runs
    decode attention.  `prefill_chunk` prefills through appends of that many
    tokens (timed); `measure_setup` times calibration, prefill, the MXFP4
    codec and the standalone dequant on this workload."""

    def __init__(self, w, replicas, with_append=True, paged=False, prefill_chunk=None,
                 measure_setup=False):
        import bit_decode_attention_b200 as nv
        self.nv = nv
        assert not (paged and with_append), "the timed append writes contiguous planes"
        self.w, self.R, self.with_append, self.paged = w, replicas, with_append, paged
        B, Hq, Hkv, D = w.B, w.Hq, w.Hkv, w.D
        self.lens0 = [int(x) for x in synthetic.seq_lens(w)]
        L_max = max(self.lens0)
        self.S_max = synthetic.capacity(L_max + 1)
        dev = "cuda"
        dt = w.torch_dtype()
        xk = gen_inputs(w, L_max, "k")
        xv = gen_inputs(w, L_max, "v")
        nk = synthetic.kv_tokens(w, replicas, "k", stream=1)   # one new token per replica
        nv_ = synthetic.kv_tokens(w, replicas, "v", stream=1)
        self.new_k = [nk[:, j:j + 1].contiguous().to(dt).to(dev) for j in range(replicas)]
        self.new_v = [nv_[:, j:j + 1].contiguous().to(dt).to(dev) for j in range(replicas)]
        self.q = [synthetic.queries(w, stream=j).to(dt).to(dev) for j in range(replicas)]
        self.status = torch.zeros(1, dtype=torch.int32, device=dev)
        self.aux = {}
        # calibration: one fp32 scale per tensor over every token the cache will hold
        allk = torch.cat([xk.reshape(-1), nk.to(dt).to(dev).reshape(-1)])
        allv = torch.cat([xv.reshape(-1), nv_.to(dt).to(dev).reshape(-1)])
        self.sk = nv.nvfp4_calib_tensor_scale(allk, status=self.status)
        self.sv = nv.nvfp4_calib_tensor_scale(allv, status=self.status)
        if measure_setup:
            ms = time_events(lambda: (nv.nvfp4_calib_tensor_scale(allk, self.sk, status=self.status),
                                      nv.nvfp4_calib_tensor_scale(allv, self.sv, status=self.status)))
            nbytes = (allk.numel() + allv.numel()) * allk.element_size()
            self.aux["calib_gbs"] = nbytes / (ms / 1e3) / 1e9
            self.aux["calib_note"] = ("warm, mean of 5 calls; K and V calibrated over %.0f MB of %s"
                                      % (nbytes / 1e6, w.dtype))
        del allk, allv
        # replica 0 prefilled through the quantizer, the others copied from it
        zeros = torch.zeros(B, dtype=torch.int32, device=dev)
        k0 = nv.KVPlane.allocate(B, Hkv, self.S_max, D)
        v0 = nv.KVPlane.allocate(B, Hkv, self.S_max, D)
        elems = 2 * B * L_max * Hkv * D
        if prefill_chunk:
            starts = [torch.full((B,), lo, dtype=torch.int32, device=dev)
                      for lo in range(0, L_max, prefill_chunk)]
            chunks = [(xk[:, lo:lo + prefill_chunk].contiguous(), xv[:, lo:lo + prefill_chunk].contiguous())
                      for lo in range(0, L_max, prefill_chunk)]

            def prefill():
                for s, (a, b) in zip(starts, chunks):
                    nv.nvfp4_kv_quantize_append_kv(a, b, s, self.sk, self.sv, k0, v0, status=self.status)
            ms = time_events(prefill, reps=3, warm=1)
            self.aux["chunked_append_gbs"] = (elems * xk.element_size() + elems * 9 // 16) / (ms / 1e3) / 1e9
            self.aux["chunked_append_note"] = ("%d appends of %d tokens x B%d x %d KV heads, K and V per launch, "
                                               "mean of 3 passes" % (len(starts), prefill_chunk, B, Hkv))
            del chunks
        else:
            def prefill():
                nv.nvfp4_kv_quantize_append_kv(xk, xv, zeros, self.sk, self.sv, k0, v0, status=self.status)
            if measure_setup:
                ms = time_events(prefill, reps=3, warm=1)
                self.aux["prefill_quantize_gbs"] = (elems * xk.element_size() + elems * 9 // 16) / (ms / 1e3) / 1e9
            else:
                prefill()
        if measure_setup:
            # the MXFP4 comparison codec on the same prefill (32-element blocks,
            # E8M0 scales): 0.53125 B written per element
            mk = nv.KVPlane.allocate_mxfp4(B, Hkv, self.S_max, D)
            mv = nv.KVPlane.allocate_mxfp4(B, Hkv, self.S_max, D)
            ms = time_events(lambda: (nv.mxfp4_kv_quantize_append(xk, zeros, mk, status=self.status),
                                      nv.mxfp4_kv_quantize_append(xv, zeros, mv, status=self.status)),
                             reps=3, warm=1)
            self.aux["mxfp4_prefill_quantize_gbs"] = (elems * xk.element_size() + elems * 17 // 32) / (ms / 1e3) / 1e9
            del mk, mv
            # the standalone dequant to FP8 (0.5625 B read + 1 B written per element)
            lens_t = torch.tensor(self.lens0, dtype=torch.int32, device=dev)
            fp8 = torch.empty(B, Hkv, self.S_max, D, dtype=torch.uint8, device=dev)
            ms = time_events(lambda: nv.nvfp4_kv_dequant_fp8(k0, self.sk, lens_t, out=fp8, status=self.status))
            self.aux["dequant_fp8_gbs"] = sum(self.lens0) * Hkv * D * (1 + 9 / 16) / (ms / 1e3) / 1e9
            del fp8
        del xk, xv
        self.k, self.v, self.out = [k0], [v0], []
        for r in range(1, replicas):
            k = nv.KVPlane(k0.codes.clone(), k0.scales.clone())
            v = nv.KVPlane(v0.codes.clone(), v0.scales.clone())
            self.k.append(k)
            self.v.append(v)
        for r in range(replicas):
            self.out.append(torch.empty(B, Hq, D, dtype=torch.float32, device=dev))
        self.start = torch.tensor(self.lens0, dtype=torch.int32, device=dev)
        self.lens_att = [L + 1 for L in self.lens0] if with_append else list(self.lens0)
        self.lens = torch.tensor(self.lens_att, dtype=torch.int32, device=dev)
        self.ws = nv.new_workspace(B, Hq, Hkv, D)
        if paged:
            self._page_replicas(nv)
        torch.cuda.synchronize()
        assert self.status.item() == 0, "device status %d during set-up" % self.status.item()

    def _page_replicas(self, nv, P=128):
        """Move every replica cache into a pool of 128-token pages handed out in a
        shuffled order (a seeded block table per replica, shared by K and V)."""
        B, H = self.w.B, self.w.Hkv
        M = (self.S_max + P - 1) // P
        g = torch.Generator().manual_seed(7)
        for r in range(self.R):
            table = torch.randperm(B * M, generator=g).to(torch.int32).view(B, M).cuda()
            planes = []
            for pl in (self.k[r], self.v[r]):
                pools = []
                for t in (pl.codes, pl.scales):
                    x = torch.nn.functional.pad(t, (0, 0, 0, M * P - self.S_max))
                    x = x.view(B, H, M, P, -1).permute(0, 2, 1, 3, 4).reshape(B * M, H, P, -1)
                    pool = torch.empty_like(x)
                    pool[table.view(-1).long()] = x
                    pools.append(pool)
                planes.append(nv.PagedKVPlane(pools[0], pools[1], table))
            self.k[r], self.v[r] = planes

    # kernels per step (ours): the attention kernel (which appends the new
    # tokens itself on the tensor-core path) + the split-K merge
    @property
    def launches_per_step(self):
        return 2

    def tokens_per_step(self):
        return sum(self.lens_att)

    def attention_bytes(self):
        """Algorithmic bytes of one attention launch: cache reads + q + out."""
        w = self.w
        kv = self.tokens_per_step() * kv_bytes_per_token(w.Hkv, w.D)
        qb = w.B * w.Hq * w.D * self.q[0].element_size()
        ob = w.B * w.Hq * w.D * 4
        return kv + qb + ob

    def step(self, j, events=None):
        """One decode step on replica j % R: append + attention in one call
        (nvfp4_decode_attention_append), or attention alone."""
        nv, r = self.nv, j % self.R
        if events is not None:
            events[0].record()
        if self.with_append:
            nv.nvfp4_decode_attention_append(self.q[r], self.new_k[r], self.new_v[r], self.start, self.k[r],
                                             self.v[r], self.sk, self.sv, out=self.out[r], workspace=self.ws,
                                             status=self.status)
        else:
            attend = nv.nvfp4_decode_attention_paged if self.paged else nv.nvfp4_decode_attention
            attend(self.q[r], self.k[r], self.v[r], self.sk, self.sv, self.lens,
                   out=self.out[r], workspace=self.ws, status=self.status)
        if events is not None:
            events[1].record()

    def capture(self, first, count, with_events):
        """One CUDA graph holding steps first .. first+count-1; optional
        external timing events around each attention launch."""
        evs = [(torch.cuda.Event(enable_timing=True, external=True),
                torch.cuda.Event(enable_timing=True, external=True)) for _ in range(count)] \
            if with_events else [None] * count
        g = torch.cuda.CUDAGraph()
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            for j in range(count):          # warm the launch path outside capture
                self.step(first + j)
        torch.cuda.current_stream().wait_stream(s)
        torch.cuda.synchronize()
        with torch.cuda.graph(g):
            for j in range(count):
                self.step(first + j, evs[j])
        torch.cuda.synchronize()
        return g, evs


def run_steps(graph_full, graph_tail, per_graph, n_steps):
    for _ in range(n_steps // per_graph):
        graph_full.replay()
    if n_steps % per_graph:
        graph_tail[n_steps % per_graph].replay()


def time_decode(wl, steps, warmup, world, sampler=None, graph_steps=None, nvtx_name="timed"):
    """Returns (elapsed_ms max over ranks, attention ms per launch, launches sampled, clocks)."""
    G = graph_steps or wl.R * max(1, 16 // wl.R)
    G = max(G, wl.R)
    G -= G % wl.R
    full, evs = wl.capture(0, G, with_events=True)
    tails = {n: wl.capture(0, n, with_events=False)[0] for n in range(1, G)} \
        if steps % G or warmup % G else {}
    run_steps(full, tails, G, warmup)
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t_wall0 = time.time()
    torch.cuda.nvtx.range_push(nvtx_name)
    start.record()
    run_steps(full, tails, G, steps)
    end.record()
    torch.cuda.nvtx.range_pop()
    torch.cuda.synchronize()
    t_wall1 = time.time()
    if world > 1:
        torch.distributed.barrier()
    ms = max_over_ranks(start.elapsed_time(end), world, "cuda")
    # the attention launches of the last full replay inside the timed region
    att = [a.elapsed_time(b) for a, b in evs] if steps >= G else []
    clocks = sampler.summary(t_wall0, t_wall1) if sampler is not None else None
    del full, tails
    return ms, (statistics.mean(att) if att else None), len(att), clocks


def time_e2e(wl, steps):
    """The same step through the public API from pinned host buffers: per step
    H2D of the new K/V token (when the step appends) and the query, the step's
    launches, D2H of the attention output.  Returns (ms, h2d bytes/step, d2h
    bytes/step)."""
    nv = wl.nv
    R = wl.R
    h_k = [t.cpu().pin_memory() for t in wl.new_k]
    h_v = [t.cpu().pin_memory() for t in wl.new_v]
    h_q = [t.cpu().pin_memory() for t in wl.q]
    h_out = [torch.empty_like(wl.out[0], device="cpu").pin_memory() for _ in range(R)]
    d_k = [torch.empty_like(t) for t in wl.new_k]
    d_v = [torch.empty_like(t) for t in wl.new_v]
    d_q = [torch.empty_like(t) for t in wl.q]
    attend = nv.nvfp4_decode_attention_paged if wl.paged else nv.nvfp4_decode_attention

    def one(j):
        r = j % R
        if wl.with_append:
            d_k[r].copy_(h_k[r], non_blocking=True)
            d_v[r].copy_(h_v[r], non_blocking=True)
        d_q[r].copy_(h_q[r], non_blocking=True)
        if wl.with_append:
            nv.nvfp4_decode_attention_append(d_q[r], d_k[r], d_v[r], wl.start, wl.k[r], wl.v[r], wl.sk, wl.sv,
                                             out=wl.out[r], workspace=wl.ws, status=wl.status)
        else:
            attend(d_q[r], wl.k[r], wl.v[r], wl.sk, wl.sv, wl.lens, out=wl.out[r], workspace=wl.ws,
                   status=wl.status)
        h_out[r].copy_(wl.out[r], non_blocking=True)

    for j in range(min(steps, 3 * R)):
        one(j)
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for j in range(steps):
        one(j)
    b.record()
    torch.cuda.synchronize()
    h2d = d_q[0].numel() * d_q[0].element_size()
    if wl.with_append:
        h2d += d_k[0].numel() * d_k[0].element_size() + d_v[0].numel() * d_v[0].element_size()
    d2h = wl.out[0].numel() * 4
    return a.elapsed_time(b), h2d, d2h


def roofline_block(wl, att_ms, att_n, peak, peak_kind, traffic_name=None):
    """HBM roofline of the step's attention call (append + attention when the
    step appends): algorithmic cache bytes / event-timed call duration."""
    if not att_ms:
        return None
    achieved = wl.attention_bytes() / (att_ms / 1e3) / 1e9
    g = wl.w.Hq // wl.w.Hkv
    traffic, why = profiled_traffic(traffic_name) if traffic_name else (None, "no capture named")
    block = {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
             "frac": achieved / peak,
             "peak_kind": peak_kind + " (MEASURED_PEAKS.json hbm_gbs)" if peak_kind == "measured"
             else "fallback",
             "traffic": traffic,
             "kernel": "decode_attention_tc_kernel<%d> + merge_split_units_kernel (tcgen05, head_dim "
                       "128, bf16 queries, GQA group %d)" % (1 if g <= 8 else 2, g),
             "algorithmic_bytes_per_launch": wl.attention_bytes(),
             "launch_ms": att_ms, "launches_sampled": att_n,
             "frac_of_nominal_8tbs": achieved / 8000.0}
    if why:
        block["traffic_note"] = why
    return block


def workload_label(w, wl):
    lens = "L %d" % w.L if w.L is not None else "L~U[%d,%d] (sum %d)" % (
        w.L_range[0], w.L_range[1], sum(wl.lens0))
    what = ("append 1 token per sequence (K and V) + decode attention" if wl.with_append
            else "decode attention")
    return "%s: B%d Hq%d Hkv%d D%d, %s cached tokens, %s%s" % (
        w.name, w.B, w.Hq, w.Hkv, w.D, lens, what, " over 128-token pages" if wl.paged else "")


# ---------------------------------------------------------------------------
# CPU oracle timings (cpu_baseline leg and the reference arm)
# ---------------------------------------------------------------------------
class OracleSample:
    """The oracle's decode step for ONE sequence of the workload (with sequence
    0's length): quantize and append its new K/V token, then fp64 decode
    attention over its cached tokens + 1.  Inputs come from the same seeded
    distributions as the GPU run's."""

    def __init__(self, w, L0=None):
        import oracle
        self.oracle = oracle
        self.w = w
        L0 = L0 if L0 is not None else int(synthetic.seq_lens(w)[0])
        self.L0 = L0
        S_max = synthetic.capacity(L0 + 1)
        one = synthetic.shrink(w, B=1)
        xk = synthetic.kv_tokens(one, L0, "k", stream=1000)
        xv = synthetic.kv_tokens(one, L0, "v", stream=1000)
        self.nk = synthetic.kv_tokens(one, 1, "k", stream=1).numpy()
        self.nv = synthetic.kv_tokens(one, 1, "v", stream=1).numpy()
        self.q = synthetic.queries(one).numpy()
        _, self.sk = oracle.tensor_scale(np.concatenate([xk.numpy().ravel(), self.nk.ravel()]))
        _, self.sv = oracle.tensor_scale(np.concatenate([xv.numpy().ravel(), self.nv.ravel()]))
        self.kc, self.ks = oracle.new_planes(1, w.Hkv, S_max, w.D)
        self.vc, self.vs = oracle.new_planes(1, w.Hkv, S_max, w.D)
        z = np.zeros(1, np.int32)
        oracle.quantize_append(xk.numpy(), z, self.sk, self.kc, self.ks)
        oracle.quantize_append(xv.numpy(), z, self.sv, self.vc, self.vs)
        self.start = np.array([L0], np.int32)
        self.lens = np.array([L0 + 1], np.int32)

    def step(self):
        o = self.oracle
        o.quantize_append(self.nk, self.start, self.sk, self.kc, self.ks)
        o.quantize_append(self.nv, self.start, self.sv, self.vc, self.vs)
        return o.decode_attention_nvfp4(self.q, self.kc, self.ks, self.vc, self.vs, self.sk, self.sv,
                                        self.lens)

    @property
    def tokens(self):
        return self.L0 + 1


def cpu_baseline(w, budget_s=15.0, single_budget_s=5.0):
    """The oracle, untuned, on every host core (OpenMP over KV heads), and
    single-threaded on a shorter budget."""
    import oracle

    def timed(threads, budget):
        oracle.set_threads(threads)
        s = OracleSample(w)
        s.step()
        n, t0 = 0, time.perf_counter()
        while True:
            s.step()
            n += 1
            if time.perf_counter() - t0 >= budget:
                break
        dt = time.perf_counter() - t0
        return n, s.tokens, dt, oracle.get_threads()

    n1, tok1, dt1, _ = timed(1, single_budget_s)
    n, tok, dt, cores = timed(os.cpu_count() or 1, budget_s)
    return {"value": n * tok / dt, "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": "%d oracle decode steps of one sequence of the workload (append 1 token + fp64 "
                      "attention over %d tokens, %d KV heads, group %d) in %.1f s" % (n, tok, w.Hkv, w.g, dt),
            "single_thread": {"value": n1 * tok1 / dt1, "unit": UNIT, "cores": 1,
                              "sample": "%d steps in %.1f s" % (n1, dt1)}}


def run_reference(args, rank, world, w):
    if rank != 0:
        return
    import oracle
    threads = os.cpu_count() or 1
    oracle.set_threads(threads)
    s = OracleSample(w)
    # size the per-step sample so warm-up + steps end in about two minutes:
    # every KV head of one sequence, over a prefix of L_s cached tokens
    t0 = time.perf_counter()
    s.step()
    full = time.perf_counter() - t0
    total = args.steps + args.warmup
    per_step_budget = 120.0 / max(total, 1)
    L0 = s.L0
    L_s = L0 if full <= per_step_budget else max(16, int(L0 * per_step_budget / full))
    sub = s if L_s == L0 else OracleSample(w, L_s)
    for _ in range(args.warmup):
        sub.step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        sub.step()
    dt = time.perf_counter() - t0
    tokens = args.steps * sub.tokens
    value = tokens / dt
    desc = ("per step: oracle append + fp64 decode attention for 1 sequence of the workload, all %d KV "
            "heads, %d tokens (of %d)" % (w.Hkv, sub.tokens, L0 + 1))
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * dt / max(args.steps, 1),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64 (oracle)",
        "data": "synthetic (seeded)", "config": config_block(w, None),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": oracle.get_threads(), "kind": "oracle",
                         "sample": desc},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def config_block(w, wl):
    lens = [int(x) for x in synthetic.seq_lens(w)]
    cfg = {"workload": "%s: B%d Hq%d Hkv%d D%d, %s cached tokens + 1 appended per sequence per step, "
                       "append K/V + decode attention" % (
                           w.name, w.B, w.Hq, w.Hkv, w.D,
                           ("L %d" % w.L) if w.L is not None else
                           ("L~U[%d,%d] seeded, sum %d" % (w.L_range[0], w.L_range[1], sum(lens)))),
           "B": w.B, "H_q": w.Hq, "H_kv": w.Hkv, "head_dim": w.D,
           "seq_len": (w.L + 1) if w.L is not None else [min(lens) + 1, max(lens) + 1],
           "input_dtype": w.dtype, "parallelism": "replicas"}
    if wl is not None:
        touched = wl.R * wl.attention_bytes()
        cfg["l2"] = ("inputs larger than L2: %d replica caches rotated, %.0f MB touched per "
                     "rotation" % (wl.R, touched / 1e6))
    return cfg


# ---------------------------------------------------------------------------
def max_over_ranks(value, world, device):
    """The largest per-rank value (elapsed time) across the process group."""
    if world <= 1:
        return value
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return t.item()


def job_throughput(world, tokens_per_step, steps, max_ms):
    """Whole-job KV-tokens/s: the tokens all ranks processed over the slowest rank's time."""
    return world * tokens_per_step * steps / (max_ms / 1e3)


def replicas_for(bytes_per_replica, l2_bytes):
    return max(2, math.ceil(2 * l2_bytes / bytes_per_replica))


def aux_attention(name, w, l2, steps, world, peak, peak_kind, with_append=False, paged=False,
                  replicas=None, prefill_chunk=None, e2e_steps=200, label_extra=""):
    """Timed aux line for one workload: attention (or the append + attention
    step), its roofline, and the same through the public API from host buffers."""
    lens = synthetic.seq_lens(w)
    per = (sum(lens) + len(lens)) * kv_bytes_per_token(w.Hkv, w.D)
    R = replicas or replicas_for(per, l2)
    wl = DecodeWorkload(w, R, with_append=with_append, paged=paged, prefill_chunk=prefill_chunk)
    ms, att, att_n, _ = time_decode(wl, steps, 20, world, nvtx_name="timed_aux_" + name)
    e2e_ms, h2d, d2h = time_e2e(wl, e2e_steps)
    tok = wl.tokens_per_step()
    roof = roofline_block(wl, att, att_n, peak, peak_kind, "decode_attention_%s_traffic.json" % name)
    line = {"workload": workload_label(w, wl) + label_extra,
            "kv_tokens_per_s": world * tok * steps / (ms / 1e3), "ms_per_step": ms / steps,
            "steps": steps, "replicas": R, "roofline": roof,
            "launch_ms": att, "achieved_gbs": roof["achieved"] if roof else None,
            "frac_of_measured": roof["frac"] if roof else None,
            "e2e": {"value": world * tok * e2e_steps / (e2e_ms / 1e3), "unit": UNIT,
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": e2e_steps}}
    line.update(wl.aux)
    status = wl.status.item()
    if status:
        line["device_status"] = status
    del wl
    torch.cuda.empty_cache()
    return line


def aux_prefill(w, C=2048, reps=5):
    """Chunked-prefill attention on the tensor cores: the last C-token chunk of
    the workload's context (queries at positions L - C .. L - 1 over the whole
    cache), timed with CUDA events; tensor roofline in algorithmic FLOPs (the
    visible query-token pairs, 2 matmuls x 2 FLOP x head_dim)."""
    import bit_decode_attention_b200 as nv
    wl = DecodeWorkload(w, 1, with_append=False)
    L = wl.lens0[0]
    start = L - C
    g = torch.Generator().manual_seed(31)
    q = torch.randn(w.B, C, w.Hq, w.D, generator=g).to(torch.bfloat16).cuda()
    start_d = torch.full((w.B,), start, dtype=torch.int32, device="cuda")
    out = torch.empty(w.B, C, w.Hq, w.D, dtype=torch.float32, device="cuda")
    run = lambda: nv.nvfp4_prefill_attention(q, wl.k[0], wl.v[0], wl.sk, wl.sv, start_d, out=out,
                                             status=wl.status)
    ms = time_events(run, reps=reps, warm=2)
    pairs = w.B * w.Hq * (C * start + C * (C + 1) // 2)
    flops = 4.0 * w.D * pairs
    tflops = flops / (ms / 1e3) / 1e12
    peaks = {}
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            peaks = json.load(f)
    except Exception:
        pass
    peak, kind = (float(peaks["bf16_tflops"]), "measured bf16 dense (burst)") if "bf16_tflops" in peaks \
        else (FALLBACK_BF16_TFLOPS, "fallback")
    line = {"workload": "%s: prefill chunk C=%d at positions %d..%d, B%d Hq%d Hkv%d D%d" %
                        (w.name, C, start, L - 1, w.B, w.Hq, w.Hkv, w.D),
            "launch_ms": ms, "achieved_tflops": tflops,
            "roofline": {"bound": "tensor", "achieved": tflops, "peak": peak, "unit": "TFLOP/s",
                         "frac": tflops / peak, "peak_kind": kind, "traffic": None,
                         "note": "kind::f16 MMAs (the bf16 rate); P.V runs twice (two-term P), so the "
                                 "tensor pipe executes 1.5x the algorithmic FLOPs"},
            "gpu_launches": reps, "device_status": wl.status.item()}
    del wl, q, out
    torch.cuda.empty_cache()
    return line


def profile_launches(name):
    """A few launches of one kernel for an ncu capture (nothing timed)."""
    import bit_decode_attention_b200 as nv
    if name == "prefill":
        w = synthetic.shrink(synthetic.get("moe128k"), L=16384)
        wl = DecodeWorkload(w, 1, with_append=False)
        C, start = 2048, wl.lens0[0] - 2048
        q = torch.randn(w.B, C, w.Hq, w.D, generator=torch.Generator().manual_seed(31)).to(torch.bfloat16).cuda()
        start_d = torch.full((w.B,), start, dtype=torch.int32, device="cuda")
        for _ in range(3):
            nv.nvfp4_prefill_attention(q, wl.k[0], wl.v[0], wl.sk, wl.sv, start_d, status=wl.status)
    else:
        wl = DecodeWorkload(synthetic.get(name), 2, with_append=False)
        for j in range(4):
            wl.step(j)
    torch.cuda.synchronize()
    print("profile launches done, device status", wl.status.item())


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=4000)
    ap.add_argument("--warmup", type=int, default=200)
    ap.add_argument("--impl", choices=["native", "reference"], default="native")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=[w.name for w in synthetic.WORKLOADS])
    ap.add_argument("--no-aux", action="store_true", help="skip the other workloads' lines")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=500)
    ap.add_argument("--profile", metavar="WORKLOAD",
                    help="for ncu captures: build WORKLOAD's cache (2 replicas), run 4 attention "
                         "launches (plus the split-K merges) and exit; 'prefill' runs 3 prefill "
                         "launches (B1 Hq96 Hkv8, a 2048-token chunk after 14336 cached tokens)")
    args = ap.parse_args()
    if args.profile:
        profile_launches(args.profile)
        return
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    rank, world, local_rank = env_rank()
    w = synthetic.get(args.workload)

    if args.impl == "reference":
        run_reference(args, rank, world, w)
        return

    torch.cuda.set_device(local_rank)
    if world > 1:
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=180),
                                             device_id=torch.device("cuda", local_rank))
    props = torch.cuda.get_device_properties(local_rank)
    l2 = getattr(props, "L2_cache_size", 126 * 1024 * 1024)
    lens = synthetic.seq_lens(w)
    per_replica = (sum(lens) + len(lens)) * kv_bytes_per_token(w.Hkv, w.D)
    R = replicas_for(per_replica, l2)
    wl = DecodeWorkload(w, R, measure_setup=True)
    sampler = ClockSampler(local_rank)
    sampler.start()
    time.sleep(0.3)
    ms, att_ms, att_n, clocks = time_decode(wl, args.steps, args.warmup, world, sampler)
    sampler.stop()
    e2e_steps = min(args.e2e_steps, args.steps)
    e2e_ms, h2d, d2h = time_e2e(wl, e2e_steps)
    status = wl.status.item()

    tokens = wl.tokens_per_step()
    value = job_throughput(world, tokens, args.steps, ms)
    peak, peak_kind = measured_peaks()
    roof = roofline_block(wl, att_ms, att_n, peak, peak_kind, "decode_attention_%s_traffic.json" % w.name)
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": DTYPE,
        "data": "synthetic (seeded; bf16 K/V ~ N(0,1) x per-channel LogNormal, no weights needed)",
        "config": config_block(w, wl),
        "hbm_gbs_step": world * tokens * kv_bytes_per_token(w.Hkv, w.D) * args.steps / (ms / 1e3) / 1e9,
        "roofline": roof,
        "e2e": {"value": world * tokens * e2e_steps / (e2e_ms / 1e3), "unit": UNIT,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": e2e_steps,
                "path": "Python binding -> C ABI, pinned host buffers, eager launches"},
        "gpu_launches": wl.launches_per_step * args.steps,
        "clocks": clocks,
        "device_status": status,
    }
    aux = dict(wl.aux)
    del wl
    torch.cuda.empty_cache()
    if not args.no_aux:
        n_aux = max(64, min(2000, args.steps))
        aux["long64k_attention"] = aux_attention("long64k", synthetic.get("long64k"), l2, n_aux, world,
                                                 peak, peak_kind)
        aux["moe128k_attention"] = aux_attention("moe128k", synthetic.get("moe128k"), l2, n_aux, world,
                                                 peak, peak_kind, prefill_chunk=2048)
        aux["gqa_step"] = aux_attention("gqa", synthetic.get("gqa"), l2, n_aux, world, peak, peak_kind,
                                        with_append=True)
        aux["gqa_paged_attention"] = aux_attention("gqa_paged", synthetic.get("gqa"), l2, n_aux, world,
                                                   peak, peak_kind, paged=True)
        aux["moe128k_prefill_attention"] = aux_prefill(synthetic.get("moe128k"))
        aux["gqa_attention_hot_l2"] = aux_attention(
            "gqa_hot", synthetic.get("gqa"), l2, n_aux, world, peak, peak_kind, replicas=1,
            label_extra=" -- HOT L2: one cache (38 MB < L2) re-read every step, not a DRAM number")
    line["aux"] = aux
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w)
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
