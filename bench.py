#!/usr/bin/env python3
"""Decode-step benchmark for the FSQ decode-attention library on B200.

One step = the hot path over one batch: append this step's token of every
batch row to the packed code cache (encoder GEMM -> FSQ -> pack, written at
row T-1) and run single-token GQA decode attention over the T cached tokens.
Metric: context tokens/s (B*T per step) and code GB/s (B*T*G/2 per step).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl fsq|reference]
                    [--workload qwen3_8b_32x] [--B 16] [--T 131072] [--variant absorbed]

With N > 1 it runs under torch.distributed.run, one rank per GPU; batch rows
are sharded across ranks (each rank owns B rows of its own; weak scaling) and
no collective touches the data path.  `--impl reference` times the fp64 CPU
oracle on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

DEFAULT_WORKLOAD = ("qwen3_8b_32x", 16, 131072)
SECOND_WORKLOAD = ("qwen3_8b_97x", 16, 131072)
HEAD_START_CYCLES = 1_000_000  # about 0.5 ms at B200 clocks: the host's head start before a timed loop
L2_BYTES = 126 * 1024 * 1024


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained"), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


# Source files that make up each split kernel (its digest voids a stored
# traffic figure once any of them changes).  Names as fsq_decode_attn_kernel
# reports them.
KERNEL_SOURCES = {
    "absorbed_split_tc": ("decode_tc.cu", "tc_decode.cuh", "tc_ptx.cuh", "common.cuh"),
    "absorbed_split_gen": ("absorbed_gen.cu", "tc_decode.cuh", "tc_ptx.cuh", "common.cuh"),
    "hybrid_split_tc": ("expand_tc.cu", "tc_decode.cuh", "tc_ptx.cuh", "common.cuh"),
    "expand_split_tc": ("expand_tc.cu", "tc_decode.cuh", "tc_ptx.cuh", "common.cuh"),
    "absorbed_split_simt": ("decode_v0.cu", "common.cuh"),
    "expand_split_simt": ("decode_v0.cu", "common.cuh"),
}


def src_digest(kernel):
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "fsq_latent_decode_b200", "csrc")
    for f in KERNEL_SOURCES[kernel]:
        h.update(open(os.path.join(csrc, f), "rb").read())
    return h.hexdigest()[:16]


def traffic_record(kernel, workload_key):
    """Per-launch DRAM traffic from the committed ncu summary, or None when the
    kernel's sources changed since the counters were taken."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    d = json.load(open(p))
    rec = d.get(kernel, {}).get(workload_key)
    if not rec or rec.get("src_digest") != src_digest(kernel):
        return None
    return rec.get("bytes_per_launch")


class ClockSampler:
    """nvidia-smi clocks/throttle reasons sampled during the timed region."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.f = None

    def start(self):
        try:
            self.f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.Q}",
                                          "--format=csv,noheader,nounits", "-lms", "50"],
                                         stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        time.sleep(0.3)

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.15)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.f.flush()
        rows = [r.split(",") for r in open(self.f.name).read().strip().splitlines() if r.count(",") >= 8]
        os.unlink(self.f.name)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        sm = [float(r[1]) for r in rows if r[1].strip().replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].strip().replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if "Active" in r[5 + i] and "Not" not in r[5 + i]})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}


class RawEvents:
    """cudaEvent_t pairs created through the CUDA runtime directly, so that the
    library can record them inside its C-ABI call; timed with
    cudaEventElapsedTime."""

    def __init__(self, n):
        import ctypes
        self.rt = None
        for name in ("libcudart.so.12", "libcudart.so"):
            try:
                self.rt = ctypes.CDLL(name)
                break
            except OSError:
                continue
        if self.rt is None:
            raise RuntimeError("libcudart not found")
        self.ct = ctypes
        self.ev = []
        for _ in range(n):
            a, b = ctypes.c_void_p(), ctypes.c_void_p()
            assert self.rt.cudaEventCreate(ctypes.byref(a)) == 0 and self.rt.cudaEventCreate(ctypes.byref(b)) == 0
            self.ev.append((a.value, b.value))

    def pair(self, i):
        class _E:  # the binding reads .cuda_event
            def __init__(self, h):
                self.cuda_event = h
        a, b = self.ev[i]
        return (_E(a), _E(b))

    def elapsed_ms(self, i):
        ms = self.ct.c_float()
        a, b = self.ev[i]
        rc = self.rt.cudaEventElapsedTime(self.ct.byref(ms), self.ct.c_void_p(a), self.ct.c_void_p(b))
        if rc != 0:
            raise RuntimeError(f"cudaEventElapsedTime failed ({rc})")
        return ms.value

    def close(self):
        for a, b in self.ev:
            self.rt.cudaEventDestroy(self.ct.c_void_p(a))
            self.rt.cudaEventDestroy(self.ct.c_void_p(b))


def max_over_ranks(torch, dist, values, device):
    """Element-wise maximum of per-rank timings (ms) over all ranks; the
    values unchanged when there is no process group."""
    if dist is None:
        return [float(v) for v in values]
    t = torch.tensor([float(v) for v in values], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.tolist()]


def job_throughput(world, B, T, ms):
    """Whole-job context tokens/s: every rank owns B rows of T tokens and a
    step takes ms (the slowest rank's time)."""
    return world * B * T / (ms * 1e-3)


def rank_seed(synth, rank, B, T, G):
    """Seed of a rank's inputs: each rank draws its own batch rows."""
    return synth.workload_seed(0, rank, B, T, G)


def dist_env():
    return int(os.environ.get("RANK", 0)), int(os.environ.get("WORLD_SIZE", 1)), int(os.environ.get("LOCAL_RANK", 0))


# --------------------------------------------------------------------------- GPU arm
def build_state(torch, F, synth, wl, B, T, rank, device, n_copies):
    """Device-resident cache(s) plus the step's new-token rows, weights and
    queries.  Cached rows are the library's FSQ codes of seeded pre-activations
    u ~ N(0, 4), the law of E x for the seeded E and x (so the full cache does
    not need x materialised); each step's new token goes through the whole
    append path (encoder GEMM, FSQ, pack)."""
    G, C = wl.G, wl.C
    half = F.row_bytes(G, wl.levels)  # bytes per cached token
    T_max = T
    while (T_max * half) % 16:
        T_max += 1
    seed = rank_seed(synth, rank, B, T, G)
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    E = synth.normal((G, C), (4.0 / C) ** 0.5, gen, device=device)
    W_kv, q = synth.decoder_inputs(B, wl.n_q, wl.n_kv, wl.d_h, G, gen, device=device, levels=wl.levels)
    caches = []
    chunk = 1 << 16
    for c in range(n_copies):
        cache = torch.empty((B, T_max, half), dtype=torch.uint8, device=device)
        flat = cache.view(B * T_max, half)
        for b in range(B):
            for t0 in range(0, T, chunk):
                n = min(chunk, T - t0)
                u = synth.preactivations(n, G, gen, device=device)
                F.quantize_pack_f32(u, out=flat[b * T_max + t0: b * T_max + t0 + n], levels=wl.levels)
        caches.append(cache)
    x_new = synth.normal((B, C), 1.0, gen, device=device)
    torch.cuda.synchronize()
    return dict(E=E, W_kv=W_kv, q=q, caches=caches, x_new=x_new, T_max=T_max)


def run_gpu(args, wl_name, B, T, torch, F, synth, dist, rank, world, device, timed=True):
    wl = synth.WORKLOADS[wl_name]
    G = wl.G
    half = F.row_bytes(G, wl.levels)
    code_bytes = B * T * half
    n_copies = max(1, math.ceil(2 * L2_BYTES / code_bytes)) if code_bytes < 2 * L2_BYTES else 1
    n_copies = min(n_copies, 8)
    st = build_state(torch, F, synth, wl, B, T, rank, device, n_copies)
    q, W_kv, E, x_new = st["q"], st["W_kv"], st["E"], st["x_new"]
    T_max = st["T_max"]
    bstride = T_max * half
    ws = F.Workspace(device)
    out = torch.empty((B, wl.n_q, wl.d_h), dtype=torch.bfloat16, device=device)
    stream = torch.cuda.current_stream()
    qp = F.quant_params(levels=wl.levels)
    nbytes_ws = F.workspace_size(B, T, wl.n_q, wl.n_kv, wl.d_h, G,
                                 F.attn_opts(variant=args.variant, rope_knorm=args.rope, levels=wl.levels))
    wbuf = ws.get(nbytes_ws)
    sptr = stream.cuda_stream
    gain = None
    if args.rope:  # key RMS-norm gain ~ 1 + N(0, 0.1^2), seeded
        g_gen = torch.Generator(device=device)
        g_gen.manual_seed(rank_seed(synth, rank, B, T, G) + 17)
        gain = (1.0 + 0.1 * torch.randn(wl.d_h, generator=g_gen, device=device)).to(torch.bfloat16)

    def make_opts(prof=None):
        return F.attn_opts(variant=args.variant, prof_events=prof, rope_knorm=args.rope, rope_base=1.0e6,
                           knorm_gain=gain, knorm_eps=1e-6, levels=wl.levels)

    def step(i, prof=None):
        cache = st["caches"][i % n_copies]
        # append this step's token of every batch row at position T-1 (rows strided by the batch stride)
        rc = F.encode_pack_raw(x_new.data_ptr(), B, wl.C, wl.C, E.data_ptr(), G, qp,
                               cache.data_ptr() + (T - 1) * half, bstride, sptr)
        if rc:
            raise F.FsqError(rc, "fsq_encode_pack")
        opts = make_opts(prof)
        rc = F.decode_attn_raw(q.data_ptr(), B, wl.n_q, wl.d_h, cache.data_ptr(), bstride, T, G,
                               W_kv.data_ptr(), wl.n_kv, opts, wbuf.data_ptr(), wbuf.numel(), out.data_ptr(), sptr)
        if rc:
            raise F.FsqError(rc, "fsq_decode_attn")

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    K = args.steps
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(torch.cuda.current_device()) if (timed and rank == 0) else None
    if clocks:
        clocks.start()
    # throughput: K steps exactly as a user issues them (no profiling events).
    # A short device-side sleep before the start event lets the host queue the
    # first steps, so the timed region holds K steps of device work rather
    # than the host's start-up latency (it matters only for small K).
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        torch.cuda._sleep(HEAD_START_CYCLES)
    t0.record(stream)
    for i in range(K):
        step(i)
    t1.record(stream)
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    ms = t0.elapsed_time(t1) / K
    # main-kernel duration: K more steps with events recorded by the library
    # around the split kernel on its own stream
    evs = RawEvents(K)
    for i in range(K):
        step(i, evs.pair(i))
    torch.cuda.synchronize()
    clk = clocks.stop() if clocks else None
    kern_ms = sum(evs.elapsed_ms(i) for i in range(K)) / K
    evs.close()
    ms, kern_ms = max_over_ranks(torch, dist, [ms, kern_ms], device)

    # end to end through the public API with host buffers: every step copies
    # its inputs (the new tokens x and the queries q) from pinned host memory
    # and reads its output o back.  As a serving loop would, the copies run on
    # a second stream, double-buffered: step i+1's inputs go up and step i's
    # output comes back while step i computes; events order the buffers.
    e2e = None
    if timed:
        q_h = q.cpu().pin_memory()
        x_h = x_new.cpu().pin_memory()
        o_h = [torch.empty((B, wl.n_q, wl.d_h), dtype=torch.bfloat16).pin_memory() for _ in range(2)]
        q_d = [torch.empty_like(q) for _ in range(2)]
        x_d = [torch.empty_like(x_new) for _ in range(2)]
        o_d = [torch.empty_like(out) for _ in range(2)]
        cs = torch.cuda.Stream()
        ev = lambda: torch.cuda.Event()
        in_ready, done, d2h = [ev(), ev()], [ev(), ev()], [ev(), ev()]

        def h2d(i):
            s_ = i % 2
            if i >= 2:
                cs.wait_event(done[s_])  # step i-2 has finished reading these buffers
            with torch.cuda.stream(cs):
                q_d[s_].copy_(q_h, non_blocking=True)
                x_d[s_].copy_(x_h, non_blocking=True)
            in_ready[s_].record(cs)

        def e2e_run(n):
            h2d(0)
            for i in range(n):
                s_ = i % 2
                if i + 1 < n:
                    h2d(i + 1)
                stream.wait_event(in_ready[s_])
                if i >= 2:
                    stream.wait_event(d2h[s_])  # o_d[s_] of step i-2 has been read back
                cache = st["caches"][i % n_copies]
                rc = F.encode_pack_raw(x_d[s_].data_ptr(), B, wl.C, wl.C, E.data_ptr(), G, qp,
                                       cache.data_ptr() + (T - 1) * half, bstride, sptr)
                if rc:
                    raise F.FsqError(rc, "fsq_encode_pack")
                rc = F.decode_attn_raw(q_d[s_].data_ptr(), B, wl.n_q, wl.d_h, cache.data_ptr(), bstride, T, G,
                                       W_kv.data_ptr(), wl.n_kv, make_opts(), wbuf.data_ptr(),
                                       wbuf.numel(), o_d[s_].data_ptr(), sptr)
                if rc:
                    raise F.FsqError(rc, "fsq_decode_attn")
                done[s_].record(stream)
                cs.wait_event(done[s_])
                with torch.cuda.stream(cs):
                    o_h[s_].copy_(o_d[s_], non_blocking=True)
                d2h[s_].record(cs)
            stream.wait_event(d2h[(n - 1) % 2])  # the last output is on the host
            if n >= 2:
                stream.wait_event(d2h[(n - 2) % 2])

        e2e_run(max(args.warmup, 2))
        torch.cuda.synchronize()
        if dist is not None:
            dist.barrier()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        cs.wait_event(a)  # the first input copy starts inside the timed region
        e2e_run(K)
        b.record(stream)
        torch.cuda.synchronize()
        e_ms = a.elapsed_time(b) / K
        (e_ms,) = max_over_ranks(torch, dist, [e_ms], device)
        e2e = {"value": job_throughput(world, B, T, e_ms), "unit": "context tokens/s",
               "h2d_bytes_per_step": q_h.numel() * 2 + x_h.numel() * 2, "d2h_bytes_per_step": o_h[0].numel() * 2,
               "ms_per_step": e_ms,
               "copies": "pinned host buffers; a second stream carries step i+1's inputs up and step i's output "
                         "back while step i computes (double-buffered, event-ordered)"}
    return dict(ms=ms, kern_ms=kern_ms, clocks=clk, e2e=e2e, n_copies=n_copies, wl=wl, B=B, T=T,
                code_bytes=code_bytes, variant=args.variant, rope=args.rope)


def roofline(res, peaks, kernel_name):
    """Roofline of the split (attention) kernel, timed alone by the library's
    events: `frac` and `frac_of_roofline` are that kernel's.  The whole decode
    step (append, query prologue, split kernel, merge) is reported beside it as
    `frac_of_roofline_step` when its device time is known."""
    wl, B, T = res["wl"], res["B"], res["T"]
    G, n_q, n_kv, d_h = wl.G, wl.n_q, wl.n_kv, wl.d_h
    variant, rope = res.get("variant", "absorbed"), res.get("rope", False)
    bytes_alg = B * T * (G * {4: 2, 16: 4, 256: 8}[wl.levels] // 8)
    if rope:
        # keys must be rebuilt per position (RoPE): key expansion + scores + latent pooling
        flops_alg = B * T * (2 * n_kv * d_h * G + 2 * n_q * d_h + 2 * n_q * G)
    else:
        flops_alg = B * T * 4 * n_q * G  # scores + latent pooling; per-query W_k^T q and W_v run outside this kernel
    # tensor-core work the variant actually issues per token (its own utilisation)
    if variant == "expand":
        flops_variant = B * T * (2 * 2 * n_kv * d_h * G + 2 * n_q * d_h * 2)
    elif variant == "hybrid":
        flops_variant = B * T * (2 * n_kv * d_h * G + 2 * n_q * d_h + 2 * n_q * G)
    else:
        flops_variant = flops_alg
    t = res["kern_ms"] * 1e-3
    t_b = bytes_alg / (peaks["hbm_gbs"] * 1e9)
    t_f = flops_alg / (peaks["bf16_tflops"] * 1e12)
    key = f"{wl.name}_B{B}_T{T}"
    traffic = traffic_record(kernel_name, key)
    if t_f >= t_b:
        ach = flops_alg / t / 1e12
        r = {"bound": "tensor", "achieved": ach, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
             "frac": ach / peaks["bf16_tflops"]}
    else:
        ach = bytes_alg / t / 1e9
        r = {"bound": "hbm", "achieved": ach, "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": ach / peaks["hbm_gbs"]}
    r["variant_flops"] = flops_variant
    r["variant_tflops"] = flops_variant / t / 1e12
    r["variant_frac_of_tensor_peak"] = flops_variant / t / 1e12 / peaks["bf16_tflops"]
    r.update({"traffic": traffic, "kernel": kernel_name, "kernel_ms": res["kern_ms"],
              "scope": "split (attention) kernel only; the step adds the append, the query prologue and the merge",
              "code_gbs": bytes_alg / t / 1e9, "frac_of_roofline": max(t_b, t_f) / t,
              "algorithmic_bytes": bytes_alg, "algorithmic_flops": flops_alg,
              "peak_source": peaks["source"] + " (burst)"})
    if res.get("ms"):
        r["step_ms"] = res["ms"]
        r["frac_of_roofline_step"] = max(t_b, t_f) / (res["ms"] * 1e-3)
    return r


POINT_WORKLOADS = ("tiny_0p6b", "qwen3_1p7b_32x", "qwen3_8b_32x", "qwen3_8b_97x", "long_8b_97x")


def points(args, torch, F, synth, peaks):
    """Every (workload, batch, length) point of the five configurations: one
    JSON line each with the decode step's time (append + decode call), the
    split kernel's time and its roofline fraction.  Each step is timed alone
    with CUDA events, after a write of twice L2 that evicts the codes, so
    small caches are read from HBM as large ones are."""
    device = torch.device("cuda", 0)
    flush = torch.empty(2 * L2_BYTES, dtype=torch.uint8, device=device)
    stream = torch.cuda.current_stream()
    sptr = stream.cuda_stream
    qp = F.quant_params()
    rows = []
    for wl_name in POINT_WORKLOADS:
        wl = synth.WORKLOADS[wl_name]
        G, half = wl.G, wl.G // 2
        for B in wl.batches:
            for T in wl.lengths:
                st = build_state(torch, F, synth, wl, B, T, 0, device, 1)
                bstride = st["T_max"] * half
                out = torch.empty((B, wl.n_q, wl.d_h), dtype=torch.bfloat16, device=device)
                ws = F.Workspace(device)
                wbuf = ws.get(F.workspace_size(B, T, wl.n_q, wl.n_kv, wl.d_h, G, F.attn_opts(variant="absorbed")))
                cache = st["caches"][0]

                def step(prof=None):
                    rc = F.encode_pack_raw(st["x_new"].data_ptr(), B, wl.C, wl.C, st["E"].data_ptr(), G, qp,
                                           cache.data_ptr() + (T - 1) * half, bstride, sptr)
                    if rc:
                        raise F.FsqError(rc, "fsq_encode_pack")
                    rc = F.decode_attn_raw(st["q"].data_ptr(), B, wl.n_q, wl.d_h, cache.data_ptr(), bstride, T, G,
                                           st["W_kv"].data_ptr(), wl.n_kv,
                                           F.attn_opts(variant="absorbed", prof_events=prof), wbuf.data_ptr(),
                                           wbuf.numel(), out.data_ptr(), sptr)
                    if rc:
                        raise F.FsqError(rc, "fsq_decode_attn")

                for _ in range(max(3, args.warmup)):
                    step()
                K = max(5, args.steps)
                evs = RawEvents(K)
                ab = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
                for i in range(K):
                    flush.zero_()
                    ab[i][0].record(stream)
                    step(evs.pair(i))
                    ab[i][1].record(stream)
                torch.cuda.synchronize()
                step_ms = sorted(a.elapsed_time(b) for a, b in ab)[K // 2]
                kern_ms = sorted(evs.elapsed_ms(i) for i in range(K))[K // 2]
                evs.close()
                rf = roofline(dict(wl=wl, B=B, T=T, kern_ms=kern_ms), peaks,
                              F.split_kernel(B, T, wl.n_q, wl.n_kv, wl.d_h, G, F.attn_opts(variant="absorbed")))
                row = {"point": wl_name, "G": G, "n_q": wl.n_q, "C": wl.C, "B": B, "T": T,
                       "step_us": step_ms * 1e3, "kernel_us": kern_ms * 1e3,
                       "ctx_tok_s": B * T / (step_ms * 1e-3), "code_gbs": rf["code_gbs"],
                       "roofline_bound": rf["bound"], "roofline_frac": rf["frac_of_roofline"]}
                print(json.dumps(row), flush=True)
                rows.append(row)
                del st, out, ws, wbuf, cache
                torch.cuda.empty_cache()
    return rows


# Multi-query points: speculative verification of n_new draft tokens per row,
# and one chunked-prefill chunk attending to a long cache.
MULTI_POINTS = (("qwen3_8b_32x", 16, 4, 32768), ("qwen3_8b_32x", 16, 8, 32768), ("qwen3_8b_97x", 16, 8, 32768),
                ("qwen3_8b_32x", 1, 256, 32768))


def multi_points(args, torch, F, synth, peaks):
    """fsq_decode_attn_multi: n_new queries per row, each attending causally to
    the code cache.  A step appends each row's n_new new tokens (one append
    call for all rows: groups of n_new tokens, one group per cache row) and
    runs the multi-query attention.  One JSON line per point with the step time, the
    split kernel's time and its roofline (codes read once; FLOPs of n_new
    queries per cached token)."""
    device = torch.device("cuda", 0)
    stream = torch.cuda.current_stream()
    sptr = stream.cuda_stream
    out_rows = []
    for wl_name, B, n_new, T in MULTI_POINTS:
        wl = synth.WORKLOADS[wl_name]
        G, rb = wl.G, F.row_bytes(wl.G, wl.levels)
        qp = F.quant_params(levels=wl.levels)
        code_bytes = B * T * rb
        n_copies = min(8, max(1, math.ceil(2 * L2_BYTES / code_bytes)))
        st = build_state(torch, F, synth, wl, B, T, 0, device, n_copies)
        bstride = st["T_max"] * rb
        gen = torch.Generator(device=device)
        gen.manual_seed(synth.workload_seed(5, B, n_new, T))
        q = synth.normal((B, n_new, wl.n_q, wl.d_h), 1.0, gen, device=device)
        x_new = synth.normal((B * n_new, wl.C), 1.0, gen, device=device)
        out = torch.empty((B, n_new, wl.n_q, wl.d_h), dtype=torch.bfloat16, device=device)
        opts = F.attn_opts(levels=wl.levels)
        wbuf = F.Workspace(device).get(F.multi_workspace_size(B, n_new, T, wl.n_q, wl.n_kv, wl.d_h, G, opts))

        grouped = F.encode_opts(tokens_per_row=n_new, row_stride_bytes=bstride)

        def step(i, prof=None):
            cache = st["caches"][i % n_copies]
            # row b's n_new new tokens (x_new rows b*n_new ..) at positions T - n_new .. T - 1
            rc = F.encode_pack_raw(x_new.data_ptr(), B * n_new, wl.C, wl.C, st["E"].data_ptr(), G, qp,
                                   cache.data_ptr() + (T - n_new) * rb, rb, sptr, grouped)
            if rc:
                raise F.FsqError(rc, "fsq_encode_pack")
            rc = F.decode_attn_multi_raw(q.data_ptr(), B, n_new, wl.n_q, wl.d_h, cache.data_ptr(), bstride, T, G,
                                         st["W_kv"].data_ptr(), wl.n_kv,
                                         F.attn_opts(levels=wl.levels, prof_events=prof), wbuf.data_ptr(),
                                         wbuf.numel(), out.data_ptr(), sptr)
            if rc:
                raise F.FsqError(rc, "fsq_decode_attn_multi")

        for i in range(max(3, args.warmup)):
            step(i)
        torch.cuda.synchronize()
        K = max(5, args.steps)
        a_, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a_.record(stream)
        for i in range(K):
            step(i)
        b_.record(stream)
        torch.cuda.synchronize()
        step_ms = a_.elapsed_time(b_) / K
        evs = RawEvents(K)
        for i in range(K):
            step(i, evs.pair(i))
        torch.cuda.synchronize()
        kern_ms = sum(evs.elapsed_ms(i) for i in range(K)) / K
        evs.close()
        t = kern_ms * 1e-3
        flops = B * n_new * (T - (n_new - 1) / 2) * 4 * wl.n_q * G  # scores + pooling over each query's prefix
        t_b = code_bytes / (peaks["hbm_gbs"] * 1e9)
        t_f = flops / (peaks["bf16_tflops"] * 1e12)
        row = {"multi_query": wl_name, "what": "speculative verification" if n_new <= 16 else "chunked prefill chunk",
               "B": B, "n_new": n_new, "T": T, "G": G, "n_q": wl.n_q, "step_us": step_ms * 1e3,
               "kernel_us": kern_ms * 1e3, "query_context_tok_s": B * n_new * T / (step_ms * 1e-3),
               "roofline_bound": "tensor" if t_f >= t_b else "hbm", "roofline_frac": max(t_b, t_f) / t,
               "tflops": flops / t / 1e12, "code_gbs": code_bytes / t / 1e9,
               "l2": f"{n_copies} rotating caches" if n_copies > 1 else "codes larger than L2",
               "launches_per_step": 4, "peak_source": peaks["source"] + " (burst)"}
        print(json.dumps(row), flush=True)
        out_rows.append(row)
        del st, q, x_new, out, wbuf
        torch.cuda.empty_cache()
    return out_rows


def _oracle_setup(wl_name, Ts):
    from fsq_latent_decode_b200 import synth
    from oracle import fsq_oracle as O
    wl = synth.WORKLOADS[wl_name]
    gen = synth._gen(123)
    W, q = synth.decoder_inputs(1, wl.n_q, wl.n_kv, wl.d_h, wl.G, gen, levels=wl.levels)
    u = synth.preactivations(Ts, wl.G, gen).numpy()
    codes = O.quantize_pack(u, O.default_h(wl.levels), 0.5, wl.levels)[None]
    qn, Wn = q.float().numpy(), W.float().numpy()
    return lambda: O.decode_attn(qn, codes, Wn, wl.n_kv, wl.G, levels=wl.levels), wl


def _blas_threads():
    try:
        from threadpoolctl import threadpool_info
        return int(max([i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"] or [1]))
    except Exception:
        return os.cpu_count() or 1


PAPER_SDPA_RATIOS = {  # decode tokens/s of the full model vs native SDPA, Qwen3-8B-Base, NVIDIA L40S
    256: {"ratio": 1.01, "ci95": [0.98, 1.05], "compression": "32x"},
    84: {"ratio": 1.54, "ci95": [1.16, 1.88], "compression": "97.5x"},
}


def sdpa_context(torch, B, T, n_q, n_kv, d_h, device, steps=20, warmup=3):
    """torch scaled_dot_product_attention (default dispatch, bf16, enable_gqa)
    for one decode query per row over an uncompressed [B, n_kv, T, d_h] K/V
    cache of the same shape: context tokens/s, for comparison only."""
    F_ = torch.nn.functional
    g = torch.Generator(device=device)
    g.manual_seed(0)
    k = torch.randn((B, n_kv, T, d_h), generator=g, device=device, dtype=torch.bfloat16)
    v = torch.randn((B, n_kv, T, d_h), generator=g, device=device, dtype=torch.bfloat16)
    q = torch.randn((B, n_q, 1, d_h), generator=g, device=device, dtype=torch.bfloat16)
    for _ in range(warmup):
        F_.scaled_dot_product_attention(q, k, v, enable_gqa=True)
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(steps):
        F_.scaled_dot_product_attention(q, k, v, enable_gqa=True)
    b.record()
    torch.cuda.synchronize()
    ms = a.elapsed_time(b) / steps
    kv_bytes = 2 * B * n_kv * T * d_h * 2
    del k, v, q
    torch.cuda.empty_cache()
    return {"value": B * T / (ms * 1e-3), "unit": "context tokens/s", "ms_per_call": ms,
            "kv_cache_bytes": kv_bytes, "kv_gbs": kv_bytes / (ms * 1e-3) / 1e9,
            "what": f"torch.nn.functional.scaled_dot_product_attention (default dispatch, torch {torch.__version__}), "
                    f"bf16 K,V [{B}, {n_kv}, {T}, {d_h}] ({kv_bytes // (B * T)} B/token), q [{B}, {n_q}, 1, {d_h}], "
                    "enable_gqa=True; inputs larger than L2"}


def append_prefill(torch, F, synth, wl, device, peaks, n_new=4096, reps=20):
    """The append leg of a chunked prefill: fsq_encode_pack of n_new tokens
    (encoder GEMM -> FSQ -> pack) into a cache slice; x rotates over copies
    larger than L2 in total."""
    C, G = wl.C, wl.G
    gen = torch.Generator(device=device)
    gen.manual_seed(synth.workload_seed(0, n_new, C, G))
    E = synth.normal((G, C), (4.0 / C) ** 0.5, gen, device=device)
    xb = n_new * C * 2
    ncop = max(2, min(8, math.ceil(2 * L2_BYTES / xb)))
    xs = [synth.normal((n_new, C), 1.0, gen, device=device) for _ in range(ncop)]
    rb = F.row_bytes(G, wl.levels)
    out = torch.empty((n_new, rb), dtype=torch.uint8, device=device)
    for i in range(3):
        F.encode_pack(xs[i % ncop], E, out=out, levels=wl.levels)
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for i in range(reps):
        F.encode_pack(xs[i % ncop], E, out=out, levels=wl.levels)
    b.record()
    torch.cuda.synchronize()
    t = a.elapsed_time(b) / reps * 1e-3
    flops = 2.0 * n_new * C * G
    nbytes = xb + G * C * 2 + n_new * rb
    t_roof = max(flops / (peaks["bf16_tflops"] * 1e12), nbytes / (peaks["hbm_gbs"] * 1e9))
    return {"what": f"fsq_encode_pack of {n_new} tokens, C={C}, G={G}, {wl.levels} levels "
                    "(bf16 x bf16 -> fp32 on tcgen05, FSQ, pack)",
            "us_per_call": t * 1e6, "tokens_per_s": n_new / t, "tflops": flops / t / 1e12, "gbs": nbytes / t / 1e9,
            "frac_of_roofline": t_roof / t, "l2": f"{ncop} rotating x copies"}


def cpu_baseline_oracle(wl_name, T, budget_s=20.0):
    """The fp64 oracle as it stands, timed on one batch row of the workload."""
    Ts = min(T, 8192)
    fn, wl = _oracle_setup(wl_name, Ts)
    reps, el = 0, 0.0
    while True:
        t0 = time.perf_counter()
        fn()
        el += time.perf_counter() - t0
        reps += 1
        if reps >= 50 or el * (reps + 1) / reps > budget_s:
            break
    return {"value": reps * Ts / el, "unit": "context tokens/s", "cores": _blas_threads(), "kind": "oracle",
            "sample": f"fp64 oracle decode of 1 batch row x {Ts} cached tokens (all {wl.n_q} heads, K and V expanded "
                      f"through W_kv), {reps} repetitions in {el:.1f} s"}


def reference_arm(wl_name, T, K, W, total_budget_s=150.0):
    """--impl reference: the oracle as the reference arm, K timed steps of a
    bounded sample (one batch row, Ts cached tokens) sized to end in minutes."""
    cal_fn, _ = _oracle_setup(wl_name, 1024)
    t0 = time.perf_counter()
    cal_fn()
    per_tok = (time.perf_counter() - t0) / 1024
    Ts = int(total_budget_s / max(1, K + W) / max(per_tok, 1e-9))
    Ts = max(256, min(T, 8192, Ts))
    fn, wl = _oracle_setup(wl_name, Ts)
    for _ in range(W):
        fn()
    t0 = time.perf_counter()
    for _ in range(K):
        fn()
    el = time.perf_counter() - t0
    val = K * Ts / el
    cb = {"value": val, "unit": "context tokens/s", "cores": _blas_threads(), "kind": "oracle",
          "sample": f"per step: fp64 oracle decode of 1 batch row x {Ts} cached tokens (all {wl.n_q} heads)"}
    return val, el / K * 1e3, cb


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="fsq", choices=["fsq", "reference"])
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD[0])
    ap.add_argument("--B", type=int, default=None)
    ap.add_argument("--T", type=int, default=None)
    ap.add_argument("--variant", default="absorbed", choices=["absorbed", "expand", "hybrid"])
    ap.add_argument("--rope", action="store_true", help="key RMS-norm + RoPE on (the pages' full key path)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-second", action="store_true", help="skip the G=84 companion measurement")
    ap.add_argument("--no-sdpa", action="store_true", help="skip the uncompressed-cache SDPA context measurement")
    ap.add_argument("--no-append", action="store_true", help="skip the 4096-token prefill append measurement")
    ap.add_argument("--points", action="store_true",
                    help="time every (workload, batch, length) point of the five configurations, one JSON line each")
    ap.add_argument("--multi", action="store_true",
                    help="time the multi-query points (speculative verification, chunked prefill), one line each")
    args = ap.parse_args()
    if args.points or args.multi:
        import torch
        import fsq_latent_decode_b200 as F
        from fsq_latent_decode_b200 import synth
        (points if args.points else multi_points)(args, torch, F, synth, load_peaks())
        return
    rank, world, local = dist_env()
    wl_name = args.workload
    from fsq_latent_decode_b200 import synth
    wl = synth.WORKLOADS[wl_name]
    B = args.B if args.B is not None else (DEFAULT_WORKLOAD[1] if wl_name == DEFAULT_WORKLOAD[0] else wl.batches[-1])
    T = args.T if args.T is not None else (DEFAULT_WORKLOAD[2] if wl_name == DEFAULT_WORKLOAD[0] else wl.lengths[-1])
    rbytes = wl.G * {4: 2, 16: 4, 256: 8}[wl.levels] // 8
    config = {"workload": f"{wl_name}: Qwen3-8B-shaped layer, n_q={wl.n_q} n_kv={wl.n_kv} d_h={wl.d_h} G={wl.G} "
                          f"L={wl.levels} ({rbytes} B/token), C={wl.C}, batch {B} per GPU, T={T}",
              "B_per_gpu": B, "T": T, "G": wl.G, "levels": wl.levels, "n_q": wl.n_q, "n_kv": wl.n_kv,
              "d_h": wl.d_h, "C": wl.C,
              "variant": args.variant, "rope_knorm": args.rope,
              "parallelism": f"replicas x{world} (batch rows sharded, no collective)"}

    if args.impl == "reference":
        if rank != 0:
            return 0
        val, ms, cb = reference_arm(wl_name, T, max(1, args.steps), max(0, args.warmup))
        line = {"impl": "reference", "metric": "FSQ decode-attn context tok/s & code GB/s, Qwen3-8B G=256/84; % roofline",
                "value": val, "unit": "context tokens/s", "n_gpus": 0, "steps": args.steps, "warmup": args.warmup,
                "ms_per_step": ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
                "dtype": "f64", "data": "synthetic (seeded; codes = oracle FSQ of u ~ N(0,4))", "config": config,
                "cpu_baseline": cb,
                "e2e": {"value": val, "unit": "context tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
        print(json.dumps(line))
        return 0

    import torch
    import fsq_latent_decode_b200 as F
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist_mod
        torch.cuda.set_device(local)
        dist_mod.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                    device_id=torch.device("cuda", local))
        dist = dist_mod
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    peaks = load_peaks()
    kernel_name = F.split_kernel(B, T, wl.n_q, wl.n_kv, wl.d_h, wl.G,
                                 F.attn_opts(variant=args.variant, rope_knorm=args.rope, levels=wl.levels))
    res = run_gpu(args, wl_name, B, T, torch, F, synth, dist, rank, world, device)
    also = None
    if not args.no_second and wl_name == DEFAULT_WORKLOAD[0] and args.B is None and args.T is None:
        r2 = run_gpu(args, SECOND_WORKLOAD[0], SECOND_WORKLOAD[1], SECOND_WORKLOAD[2], torch, F, synth, dist, rank,
                     world, device, timed=False)
        rf2 = roofline(r2, peaks, kernel_name)
        also = {"workload": f"{SECOND_WORKLOAD[0]} B={SECOND_WORKLOAD[1]} T={SECOND_WORKLOAD[2]} G=84",
                "value": job_throughput(world, r2["B"], r2["T"], r2["ms"]), "unit": "context tokens/s",
                "ms_per_step": r2["ms"], "code_gbs": rf2["code_gbs"], "roofline": rf2,
                "l2": f"{r2['n_copies']} rotating caches"}
    cb = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cb = cpu_baseline_oracle(wl_name, T)
    appf = None
    if rank == 0 and not args.no_append:
        appf = append_prefill(torch, F, synth, wl, device, peaks)
    sdpa = None
    if rank == 0 and not args.no_sdpa:
        sdpa = sdpa_context(torch, B, T, wl.n_q, wl.n_kv, wl.d_h, device)
        fsq_ctx = B * T / (res["ms"] * 1e-3)
        sdpa["fsq_step_over_sdpa"] = fsq_ctx / sdpa["value"]
        pr = PAPER_SDPA_RATIOS.get(wl.G)
        if pr:
            sdpa["paper"] = dict(pr, what="full-model decode tokens/s vs native SDPA, Qwen3-8B-Base, NVIDIA L40S "
                                          "(context only: another scope and GPU)")
        if also is not None:
            also["fsq_step_over_sdpa"] = also["value"] / world / sdpa["value"]
            also["paper"] = dict(PAPER_SDPA_RATIOS[84], what=sdpa["paper"]["what"]) if "paper" in sdpa else None
    if rank == 0:
        rf = roofline(res, peaks, kernel_name)
        value = job_throughput(world, B, T, res["ms"])
        l2 = ("codes larger than L2 (%.0f MB per cache)" % (res["code_bytes"] / 1e6) if res["n_copies"] == 1
              else f"{res['n_copies']} rotating caches > 2x L2")
        if sdpa is not None:
            # the copy peak counts read + write; SDPA's K/V read rate in the same run is a read-stream reference
            rf["code_gbs_over_sdpa_read_gbs"] = rf["code_gbs"] / sdpa["kv_gbs"]
            if also is not None:
                also["roofline"]["code_gbs_over_sdpa_read_gbs"] = also["roofline"]["code_gbs"] / sdpa["kv_gbs"]
        line = {"metric": "FSQ decode-attn context tok/s & code GB/s, Qwen3-8B G=256/84; % roofline",
                "value": value, "unit": "context tokens/s", "n_gpus": world, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": res["ms"], "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None,
                "dtype": ({"absorbed_split_tc": "u4 codes; s8 x u8 score MMA (s32), f16 pooling MMA (f32), f32 "
                                                "softmax/merge, bf16 in/out",
                           "absorbed_split_gen": f"u{rbytes * 8 // wl.G} codes as f16 levels; f16 score MMA (two-term "
                                                 "query, f32), f16 pooling MMA (f32), f32 softmax/merge, bf16 in/out",
                           "hybrid_split_tc": "u4 codes; f16 key, score and pooling MMAs (f32), f32 key norm/RoPE/"
                                              "softmax/merge, bf16 in/out",
                           "expand_split_tc": "u4 codes; f16 key, value, score and output MMAs (f32), f32 softmax/"
                                              "merge, bf16 in/out"}.get(kernel_name,
                                                                        f"u{rbytes * 8 // wl.G} codes; f32 CUDA-core "
                                                                        "scores, pooling, softmax and merge, bf16 in/out")
                          if wl.levels == 16 or kernel_name != "absorbed_split_tc" else
                          "u8 codes read as u4 nibble pairs; s8 x u8 score MMA (s32), f16 pooling MMA (f32), f32 "
                          "softmax/merge, bf16 in/out"),
                "data": "synthetic (seeded; cache = FSQ codes of u ~ N(0,4), the law of E x; new token x ~ N(0,1) appended each step)",
                "config": config, "l2": l2, "code_gbs": world * res["code_bytes"] / (res["ms"] * 1e-3) / 1e9,
                "roofline": rf, "cpu_baseline": cb, "e2e": res["e2e"], "clocks": res["clocks"],
                "gpu_launches": args.steps * 4, "also": also, "sdpa_context": sdpa, "append_prefill": appf}
        print(json.dumps(line))
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
