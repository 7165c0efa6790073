#!/usr/bin/env python
"""NVFP4 KV-cache decode benchmark on B200: KV-tokens/s and achieved HBM GB/s.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl native|reference]

One step is one pass of the whole decode hot path over one batch: quantize the
new token's K and V (E2M1 codes + E4M3 block scales under the calibrated fp32
tensor scale) and append them to the NVFP4 cache, then run decode attention
over the cache with NVFP4 -> FP8 dequantization fused in.  Default workload:
B=8 sequences, 32 query heads, 8 KV heads, head_dim 128, 4096 cached tokens +
the appended one (4097 attended), bf16 inputs with per-channel log-normal
scales.  Tensor-scale calibration and the 4096-token prefill quantization run
once during set-up; their throughput is reported under "aux".

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
DTYPE = "nvfp4 (e2m1 + e4m3 block scale) storage, fp8 e4m3 values, f16 MMA inputs, f32 accumulate"
FALLBACK_HBM_GBS = 6650.0
ATTN_SOURCES = ["bit_decode_attention_b200/csrc/nvfp4kv_decode_attention_tc.cu",
                "bit_decode_attention_b200/csrc/nvfp4kv_attention_common.cuh",
                "bit_decode_attention_b200/csrc/nvfp4kv_tcgen05.cuh",
                "bit_decode_attention_b200/csrc/nvfp4kv_device.cuh"]


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
    """DRAM bytes per launch from a committed ncu summary, only while the
    kernel source still matches the one that was profiled."""
    path = os.path.join(ROOT, "profiles", name)
    try:
        with open(path) as f:
            d = json.load(f)
    except Exception:
        return None
    if d.get("source_digest") != source_digest(ATTN_SOURCES):
        return None
    return d.get("dram_bytes_per_launch")


def kv_bytes_per_token(Hkv, D):
    """Algorithmic HBM bytes to read one cached token (all KV heads, K and V)."""
    return Hkv * 2 * (D // 2 + D // 16)


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


# ---------------------------------------------------------------------------
# the decode workload
# ---------------------------------------------------------------------------
class DecodeWorkload:
    """R replica NVFP4 caches of one workload, each prefilled with L0 tokens;
    a step appends one token at slot L0 (the same slot every visit, so every
    step attends exactly L0 + 1 tokens) and runs decode attention."""

    def __init__(self, w, L0, replicas, with_append=True, paged=False):
        import bit_decode_attention_b200 as nv
        self.nv = nv
        assert not (paged and with_append), "the timed append writes contiguous planes"
        self.w, self.L0, self.R, self.with_append, self.paged = w, L0, replicas, with_append, paged
        B, Hq, Hkv, D = w.B, w.Hq, w.Hkv, w.D
        self.S_max = synthetic.capacity(L0 + 1)
        dev = "cuda"
        bf = torch.bfloat16 if w.dtype == "bf16" else torch.float32
        xk = synthetic.kv_tokens(w, L0, "k")
        xv = synthetic.kv_tokens(w, L0, "v")
        nk = synthetic.kv_tokens(w, replicas, "k", stream=1)   # one new token per replica
        nv_ = synthetic.kv_tokens(w, replicas, "v", stream=1)
        self.xk_d = xk.to(bf).to(dev)
        self.xv_d = xv.to(bf).to(dev)
        del xk, xv
        self.new_k = [nk[:, j:j + 1].contiguous().to(bf).to(dev) for j in range(replicas)]
        self.new_v = [nv_[:, j:j + 1].contiguous().to(bf).to(dev) for j in range(replicas)]
        self.q = [synthetic.queries(w, stream=j).to(bf).to(dev) for j in range(replicas)]
        self.status = torch.zeros(1, dtype=torch.int32, device=dev)
        # calibration: one fp32 scale per tensor over every token the cache will hold
        t0 = time.perf_counter()
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
        allk = torch.cat([self.xk_d, nk.to(bf).to(dev)], dim=1)
        allv = torch.cat([self.xv_d, nv_.to(bf).to(dev)], dim=1)
        ev[0].record()
        self.sk = nv.nvfp4_calib_tensor_scale(allk, status=self.status)
        self.sv = nv.nvfp4_calib_tensor_scale(allv, status=self.status)
        ev[1].record()
        torch.cuda.synchronize()
        self.calib_ms = ev[0].elapsed_time(ev[1])
        self.calib_bytes = (allk.numel() + allv.numel()) * allk.element_size()
        del allk, allv
        # replica caches, prefilled
        self.k, self.v, self.out = [], [], []
        zeros = torch.zeros(B, dtype=torch.int32, device=dev)
        self.prefill_ms = 0.0
        for r in range(replicas):
            k = nv.KVPlane.allocate(B, Hkv, self.S_max, D)
            v = nv.KVPlane.allocate(B, Hkv, self.S_max, D)
            ev[0].record()
            nv.nvfp4_kv_quantize_append(self.xk_d, zeros, self.sk, k, status=self.status)
            nv.nvfp4_kv_quantize_append(self.xv_d, zeros, self.sv, v, status=self.status)
            ev[1].record()
            torch.cuda.synchronize()
            self.prefill_ms += ev[0].elapsed_time(ev[1])
            self.k.append(k)
            self.v.append(v)
            self.out.append(torch.empty(B, Hq, D, dtype=torch.float32, device=dev))
        elems = 2 * B * L0 * Hkv * D
        self.prefill_bytes = replicas * (elems * self.xk_d.element_size() + elems * 9 // 16)
        # the MXFP4 comparison codec on the same prefill (32-element blocks, E8M0
        # scales): 0.53125 B written per element; timed, then freed
        mk = nv.KVPlane.allocate_mxfp4(B, Hkv, self.S_max, D)
        mv = nv.KVPlane.allocate_mxfp4(B, Hkv, self.S_max, D)
        reps = 3
        ev[0].record()
        for _ in range(reps):
            nv.mxfp4_kv_quantize_append(self.xk_d, zeros, mk, status=self.status)
            nv.mxfp4_kv_quantize_append(self.xv_d, zeros, mv, status=self.status)
        ev[1].record()
        torch.cuda.synchronize()
        self.mx_prefill_ms = ev[0].elapsed_time(ev[1]) / reps
        self.mx_prefill_bytes = elems * self.xk_d.element_size() + elems * 17 // 32
        del mk, mv
        self.start = torch.full((B,), L0, dtype=torch.int32, device=dev)
        self.lens = torch.full((B,), L0 + 1 if with_append else L0, dtype=torch.int32, device=dev)
        self.ws = nv.new_workspace(B, Hq, Hkv, D)
        self.L_att = L0 + 1 if with_append else L0
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

    # kernels per step (ours): 1 append of K and V + 1 attention
    @property
    def launches_per_step(self):
        return 2 if self.with_append else 1

    def tokens_per_step(self):
        return self.w.B * self.L_att

    def attention_bytes(self):
        """Algorithmic bytes of one attention launch: cache reads + q + out."""
        w = self.w
        kv = self.w.B * self.L_att * kv_bytes_per_token(w.Hkv, w.D)
        qb = w.B * w.Hq * w.D * self.q[0].element_size()
        ob = w.B * w.Hq * w.D * 4
        return kv + qb + ob

    def step(self, j, events=None):
        nv, r = self.nv, j % self.R
        if self.with_append:
            nv.nvfp4_kv_quantize_append_kv(self.new_k[r], self.new_v[r], self.start, self.sk, self.sv,
                                           self.k[r], self.v[r], status=self.status)
        if events is not None:
            events[0].record()
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
    """Returns (elapsed_ms max over ranks, attention ms per launch, clocks)."""
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
    """Same step through the public API from pinned host buffers: per step
    H2D of the new K/V token and the query, the step's launches, D2H of the
    attention output.  Returns (ms, h2d bytes/step, d2h bytes/step)."""
    nv = wl.nv
    R = wl.R
    h_k = [t.cpu().pin_memory() for t in wl.new_k]
    h_v = [t.cpu().pin_memory() for t in wl.new_v]
    h_q = [t.cpu().pin_memory() for t in wl.q]
    h_out = [torch.empty_like(wl.out[0], device="cpu").pin_memory() for _ in range(R)]
    d_k = [torch.empty_like(t) for t in wl.new_k]
    d_v = [torch.empty_like(t) for t in wl.new_v]
    d_q = [torch.empty_like(t) for t in wl.q]

    def one(j):
        r = j % R
        d_k[r].copy_(h_k[r], non_blocking=True)
        d_v[r].copy_(h_v[r], non_blocking=True)
        d_q[r].copy_(h_q[r], non_blocking=True)
        nv.nvfp4_kv_quantize_append_kv(d_k[r], d_v[r], wl.start, wl.sk, wl.sv, wl.k[r], wl.v[r],
                                       status=wl.status)
        nv.nvfp4_decode_attention(d_q[r], wl.k[r], wl.v[r], wl.sk, wl.sv, wl.lens, out=wl.out[r],
                                  workspace=wl.ws, status=wl.status)
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
    h2d = (d_k[0].numel() * d_k[0].element_size() + d_v[0].numel() * d_v[0].element_size()
           + d_q[0].numel() * d_q[0].element_size())
    d2h = wl.out[0].numel() * 4
    return a.elapsed_time(b), h2d, d2h


# ---------------------------------------------------------------------------
# CPU oracle timings (cpu_baseline leg and the reference arm)
# ---------------------------------------------------------------------------
class OracleSample:
    """The oracle's decode step for ONE sequence of the workload: quantize and
    append its new K/V token, then fp64 decode attention over L0 + 1 tokens.
    Inputs are the same seeded tensors the GPU run uses."""

    def __init__(self, w, L0, seconds_hint=None):
        import oracle
        self.oracle = oracle
        self.w, self.L0 = w, L0
        S_max = synthetic.capacity(L0 + 1)
        one = synthetic.shrink(w, B=1)
        xk = synthetic.kv_tokens(one, L0, "k")
        xv = synthetic.kv_tokens(one, L0, "v")
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


def cpu_baseline(w, L0, budget_s=15.0, single_budget_s=5.0):
    """The oracle, untuned, on every host core (OpenMP over KV heads), and
    single-threaded on a shorter budget."""
    import oracle

    def timed(threads, budget):
        oracle.set_threads(threads)
        s = OracleSample(w, L0)
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
            "sample": "%d oracle decode steps of one sequence (append 1 token + fp64 attention over "
                      "%d tokens, %d KV heads, group %d) in %.1f s" % (n, tok, w.Hkv, w.g, dt),
            "single_thread": {"value": n1 * tok1 / dt1, "unit": UNIT, "cores": 1,
                              "sample": "%d steps in %.1f s" % (n1, dt1)}}


def run_reference(args, rank, world, w, L0):
    if rank != 0:
        return
    import oracle
    threads = os.cpu_count() or 1
    oracle.set_threads(threads)
    s = OracleSample(w, L0)
    # size the per-step sample so warm-up + steps end in about two minutes:
    # every KV head of one sequence, over a prefix of L_s cached tokens
    t0 = time.perf_counter()
    s.step()
    full = time.perf_counter() - t0
    total = args.steps + args.warmup
    per_step_budget = 120.0 / max(total, 1)
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
    desc = ("per step: oracle append + fp64 decode attention for 1 sequence, all %d KV heads, "
            "%d tokens (of %d)" % (w.Hkv, sub.tokens, L0 + 1))
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * dt / max(args.steps, 1),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64 (oracle)",
        "data": "synthetic (seeded)", "config": config_block(w, L0, None),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": oracle.get_threads(), "kind": "oracle",
                         "sample": desc},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def config_block(w, L0, wl):
    cfg = {"workload": "%s: B%d Hq%d Hkv%d D%d, %d cached + 1 appended token per step, append K/V "
                       "+ decode attention" % (w.name, w.B, w.Hq, w.Hkv, w.D, L0),
           "B": w.B, "H_q": w.Hq, "H_kv": w.Hkv, "head_dim": w.D, "seq_len": L0 + 1,
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


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20000)
    ap.add_argument("--warmup", type=int, default=2000)
    ap.add_argument("--impl", choices=["native", "reference"], default="native")
    ap.add_argument("--workload", default="gqa", choices=[w.name for w in synthetic.WORKLOADS])
    ap.add_argument("--no-aux", action="store_true", help="skip the 64K attention-only line")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=2000)
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    rank, world, local_rank = env_rank()
    w = synthetic.get(args.workload)
    L0 = w.L if w.L is not None else w.L_range[1]

    if args.impl == "reference":
        run_reference(args, rank, world, w, L0)
        return

    torch.cuda.set_device(local_rank)
    if world > 1:
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=180),
                                             device_id=torch.device("cuda", local_rank))
    props = torch.cuda.get_device_properties(local_rank)
    l2 = getattr(props, "L2_cache_size", 126 * 1024 * 1024)
    per_replica = w.B * (L0 + 1) * kv_bytes_per_token(w.Hkv, w.D)
    R = replicas_for(per_replica, l2)
    wl = DecodeWorkload(w, L0, R)
    sampler = ClockSampler(local_rank)
    sampler.start()
    time.sleep(0.3)
    ms, att_ms, att_n, clocks = time_decode(wl, args.steps, args.warmup, world, sampler)
    sampler.stop()
    e2e_ms, h2d, d2h = time_e2e(wl, min(args.e2e_steps, args.steps))
    e2e_steps = min(args.e2e_steps, args.steps)
    status = wl.status.item()

    tokens = wl.tokens_per_step()
    value = job_throughput(world, tokens, args.steps, ms)
    peak, peak_kind = measured_peaks()
    roof = None
    if att_ms:
        achieved = wl.attention_bytes() / (att_ms / 1e3) / 1e9
        roof = {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                "frac": achieved / peak, "peak_kind": peak_kind + " (MEASURED_PEAKS.json hbm_gbs)"
                if peak_kind == "measured" else "fallback",
                "traffic": profiled_traffic("decode_attention_%s_traffic.json" % w.name),
                "kernel": "decode_attention_tc_kernel<%d> (tcgen05, head_dim 128, bf16 queries)"
                          % (1 if w.Hq // w.Hkv <= 8 else 2),
                "algorithmic_bytes_per_launch": wl.attention_bytes(),
                "launch_ms": att_ms, "launches_sampled": att_n,
                "frac_of_nominal_8tbs": achieved / 8000.0}
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": DTYPE,
        "data": "synthetic (seeded; bf16 K/V ~ N(0,1) x per-channel LogNormal, no weights needed)",
        "config": config_block(w, L0, wl),
        "hbm_gbs_step": world * tokens * kv_bytes_per_token(w.Hkv, w.D) * args.steps / (ms / 1e3) / 1e9,
        "roofline": roof,
        "e2e": {"value": world * tokens * e2e_steps / (e2e_ms / 1e3), "unit": UNIT,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": e2e_steps,
                "path": "Python binding -> C ABI, pinned host buffers, eager launches"},
        "gpu_launches": wl.launches_per_step * args.steps,
        "clocks": clocks,
        "device_status": status,
    }
    aux = {"calib_gbs": wl.calib_bytes / (wl.calib_ms / 1e3) / 1e9,
           "prefill_quantize_gbs": wl.prefill_bytes / (wl.prefill_ms / 1e3) / 1e9,
           "mxfp4_prefill_quantize_gbs": wl.mx_prefill_bytes / (wl.mx_prefill_ms / 1e3) / 1e9}
    del wl
    torch.cuda.empty_cache()
    if not args.no_aux:
        lw = synthetic.get("long64k")
        per = lw.B * lw.L * kv_bytes_per_token(lw.Hkv, lw.D)
        lwl = DecodeWorkload(lw, lw.L, replicas_for(per, l2), with_append=False)
        n_aux = max(64, min(2000, args.steps))
        lms, latt, lat_n, _ = time_decode(lwl, n_aux, 20, world, nvtx_name="timed_aux")
        ach = lwl.attention_bytes() / (latt / 1e3) / 1e9 if latt else None
        aux["long64k_attention"] = {
            "workload": "long64k: B1 Hq64 Hkv8 D128 L65536, decode attention only (split-K)",
            "kv_tokens_per_s": world * lwl.tokens_per_step() * n_aux / (lms / 1e3),
            "launch_ms": latt, "achieved_gbs": ach, "frac_of_measured": ach / peak if ach else None,
            "frac_of_nominal_8tbs": ach / 8000.0 if ach else None, "steps": n_aux,
            "replicas": lwl.R}
        del lwl
        torch.cuda.empty_cache()
        # the gqa attention over a paged cache (128-token pages, shuffled block table)
        gw = synthetic.get("gqa")
        per = gw.B * gw.L * kv_bytes_per_token(gw.Hkv, gw.D)
        pwl = DecodeWorkload(gw, gw.L, replicas_for(per, l2), with_append=False, paged=True)
        pms, patt, pat_n, _ = time_decode(pwl, n_aux, 20, world, nvtx_name="timed_aux_paged")
        pach = pwl.attention_bytes() / (patt / 1e3) / 1e9 if patt else None
        aux["gqa_paged_attention"] = {
            "workload": "gqa paged: B8 Hq32 Hkv8 D128 L4096, 128-token pages in shuffled order",
            "kv_tokens_per_s": world * pwl.tokens_per_step() * n_aux / (pms / 1e3),
            "launch_ms": patt, "achieved_gbs": pach, "frac_of_measured": pach / peak if pach else None,
            "steps": n_aux, "replicas": pwl.R}
        del pwl
        torch.cuda.empty_cache()
    line["aux"] = aux
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w, L0)
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
