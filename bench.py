#!/usr/bin/env python
"""Benchmark of one MLA decode step on B200: append -> absorb -> decode -> out_up.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME] [--impl reference]

A step is one pass of the whole decode path over one batch of synthetic input already
resident in HBM: mla_cache_append of the q new tokens, mla_absorb_q, mla_decode_attn
(paged, split-KV, combine) and mla_out_up. ``value`` is decode tokens per second (B*q per
step) over all ranks; ``roofline`` describes mla_decode_attn (the dominant kernel),
timed with CUDA events around its launches inside the timed region; ``e2e`` repeats the
step through the same public API from pinned HOST buffers, with the host->device copy of
the step's inputs and the device->host read of its output inside the timed region.
Under torchrun every rank runs an independent replica on its own GPU (the path has no
exchange step); time is the max over ranks.

``--impl reference`` times the fp64 CPU oracle (the unabsorbed form) on the host cores on
a bounded sample of the same workload.
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

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "MLA decode attn: tokens/s, latent-cache HBM GB/s, TFLOP/s, % of roofline"
DEFAULT_CONFIG = "deepseek_v2"
L2_BYTES = 126 * 1024 * 1024


def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        d = json.load(open(path))
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


def algorithmic_work(cfg, seq_lens):
    """Latent-cache bytes read and FLOPs of one mla_decode_attn launch.

    Bytes: every cached row (D bf16) of every sequence, read once for all heads and query
    rows. FLOPs: 2*H*(r + d_r) for the scores and 2*H*r for o_ per query row and visible
    cached token (padding of the rotary slots and of the UMMA tiles not counted); for the
    single-latent K = V form the value is the whole row, 2*H*D + 2*H*D."""
    D = cfg.row_width
    tokens = int(np.sum(seq_lens, dtype=np.int64))
    nbytes = tokens * D * 2
    q, H, r, dr = cfg.q_len, cfg.num_heads, cfg.kv_lora_rank, cfg.rope_dim
    vis = 0
    for L in seq_lens:
        L = int(L)
        vis += q * L - (q * (q - 1)) // 2 if cfg.causal else q * L
    per = 4 * H * D if cfg.name.startswith("nanowhale") else 2 * H * (r + dr) + 2 * H * r
    return nbytes, vis * per


# Child process of ClockSampler: polls NVML in a tight loop (no GIL shared with the timed
# loop) and appends "time, sm_mhz, max_mhz, power_w, reasons" rows to a file until killed.
_NVML_SAMPLER = r"""
import sys, time
import pynvml
pynvml.nvmlInit()
gpu, path = sys.argv[1], sys.argv[2]
h = (pynvml.nvmlDeviceGetHandleByUUID(gpu) if gpu.startswith("GPU-")
     else pynvml.nvmlDeviceGetHandleByIndex(int(gpu)))
reasons = getattr(pynvml, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
    pynvml.nvmlDeviceGetCurrentClocksThrottleReasons
mx = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
with open(path, "w", buffering=1) as fh:
    while True:
        t = time.time()
        sm = pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM)
        rs = int(reasons(h))
        pw = pynvml.nvmlDeviceGetPowerUsage(h) / 1000.0
        fh.write(f"{t:.6f},{sm},{mx},{pw:.2f},{rs}\n")
"""


class ClockSampler:
    """SM clock, power and clock-event (throttle) reasons of this GPU during the timed region:
    a child process polls NVML as fast as it answers (a timed region of a few milliseconds
    still gets samples); nvidia-smi every 200 ms when NVML is not importable. Only samples
    between mark_start() and mark_end() count. Rows go to the file MLA_BENCH_CLOCKS_CSV names
    (with the rank appended before .csv), else to a temporary file."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    # NVML clock-event reason bits, in the order of the last four nvidia-smi columns above
    BITS = (0x8, 0x40, 0x20, 0x4)
    NAMES = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")

    def __init__(self, gpu_id: str):
        self.gpu = gpu_id  # a UUID ("GPU-...") or an index
        self.proc = None
        self.kind = None   # "nvml" or "nvidia-smi"
        self.path = None
        self.rows = None   # (time, sm_mhz, max_mhz, power_w, reasons bitmask) for "nvml"
        self.tmp = False   # the sample file is a temporary file of ours (removed after use)
        self.t0 = self.t1 = None

    def __enter__(self):
        try:
            rank = os.environ.get("RANK", "0")
            want = os.environ.get("MLA_BENCH_CLOCKS_CSV")
            if want:
                root, ext = os.path.splitext(want)
                self.path = f"{root}_rank{rank}{ext or '.csv'}"
                os.makedirs(os.path.dirname(os.path.abspath(self.path)), exist_ok=True)
                if os.path.exists(self.path):
                    os.remove(self.path)
            else:
                fd, self.path = tempfile.mkstemp(prefix=f"mla_clocks_rank{rank}_", suffix=".csv")
                os.close(fd)
                self.tmp = True
                os.remove(self.path)   # the sampler creates it; its size tells it has started
        except Exception:
            self.path = None
            return self
        try:
            import pynvml  # noqa: F401  (the child needs it)
            self.proc = subprocess.Popen([sys.executable, "-c", _NVML_SAMPLER, str(self.gpu), self.path],
                                         stdout=subprocess.DEVNULL, stderr=subprocess.DEVNULL)
            self.kind = "nvml"
            t_end = time.time() + 10.0
            while time.time() < t_end and self.proc.poll() is None:
                if os.path.exists(self.path) and os.path.getsize(self.path) > 0:
                    break
                time.sleep(0.01)
            if self.proc.poll() is not None:
                raise RuntimeError("NVML sampler exited")
        except Exception:
            self._stop()
            self.kind = None
            try:
                self.fh = open(self.path, "w")
                self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.Q}",
                                              "--format=csv,noheader,nounits", "-lms", "200"],
                                             stdout=self.fh, stderr=subprocess.DEVNULL)
                self.kind = "nvidia-smi"
                time.sleep(0.3)
            except Exception:
                self.proc = None
        return self

    def mark_start(self):
        self.t0 = time.time()

    def mark_end(self):
        self.t1 = time.time()

    def _stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
        self.proc = None

    def __exit__(self, *a):
        if self.kind == "nvidia-smi":
            time.sleep(0.25)
            self._stop()
            self.fh.close()
        else:
            time.sleep(0.02)
            self._stop()
            self.rows = []
            try:
                for line in open(self.path):
                    f = line.strip().split(",")
                    if len(f) == 5:
                        self.rows.append((float(f[0]), float(f[1]), float(f[2]), float(f[3]), int(f[4])))
            except Exception:
                pass

    def summary(self):
        out = self._summary()
        if self.tmp and self.path is not None:
            try:
                os.remove(self.path)
            except OSError:
                pass
        return out

    def _summary(self):
        if self.kind == "nvml":
            rows = [r for r in (self.rows or [])
                    if self.t0 is None or self.t1 is None or self.t0 <= r[0] <= self.t1]
            if not rows:
                return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
            reasons = sorted({n for r in rows for n, b in zip(self.NAMES, self.BITS) if r[4] & b})
            return {"sm_mhz": statistics.median(r[1] for r in rows), "sm_max_mhz": rows[0][2],
                    "power_w": round(statistics.median(r[3] for r in rows), 1),
                    "samples": len(rows), "source": "nvml", "reasons": reasons}
        if self.kind != "nvidia-smi" or self.path is None or not os.path.exists(self.path):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        sms, mx, reasons = [], None, set()
        for line in open(self.path):
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm, mx = float(f[1]), float(f[2])
            except ValueError:
                continue
            sms.append(sm)
            for n, v in zip(self.NAMES, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sms:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        loaded = [s for s in sms if s > 0.5 * (mx or max(sms))] or sms
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": mx, "samples": len(sms),
                "source": "nvidia-smi", "reasons": sorted(reasons)}


def uses_pair_kernel(cfg):
    """True when mla_decode_attn runs this shape on the two-CTA latent-split kernel (more than
    64 query rows, rank a multiple of 128, rotary columns of 32, 64 or 128)."""
    rope = cfg.num_kv_groups * cfg.rope_dim
    return (cfg.q_len * cfg.num_heads > 64 and cfg.kv_lora_rank % 128 == 0
            and rope in (32, 64, 128))


def decode_kernel_name(cfg):
    return "mla_decode_pair_kernel" if uses_pair_kernel(cfg) else "mla_decode_kernel"


def _source_hash(cfg):
    """Hash of the sources of the decode kernel that runs this shape: its .cu file, the
    schedule and PTX helpers, and its parameter struct (the rest of kernels.h belongs to the
    other kernels)."""
    csrc = os.path.join(ROOT, "head_latent_attention_attn_b200", "csrc")
    files = ("decode_pair.cu" if uses_pair_kernel(cfg) else "decode.cu", "decode_sched.cuh",
             "ptx.cuh")
    h = hashlib.sha256()
    for f in files:
        h.update(open(os.path.join(csrc, f), "rb").read())
    hdr = open(os.path.join(csrc, "kernels.h")).read()
    i = hdr.index("struct DecodeParams {")
    h.update(hdr[i:hdr.index("};", i)].encode())
    return h.hexdigest()[:16]


def _traffic(cfg):
    """Per-launch DRAM bytes of the decode kernel from a committed ncu summary, if it was
    taken on the current kernel source; else None."""
    path = os.path.join(ROOT, "profiles", "decode_traffic.json")
    if not os.path.exists(path):
        return None
    d = json.load(open(path))
    e = d.get(cfg.name)
    if not e or e.get("source_hash") != _source_hash(cfg):
        return None
    return e.get("dram_bytes_per_launch")


def max_over_ranks(values, dist, device):
    """Element-wise maximum of `values` over all ranks (each rank's own list when `dist` is
    None). Every rank must call it with the same length, in the same order."""
    import torch
    vec = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    if dist is not None:
        dist.all_reduce(vec, op=dist.ReduceOp.MAX)
    return [float(x) for x in vec.tolist()]


def cpu_oracle_sample(cfg, wl, budget_s=12.0, max_seqs=None, absorbed=False):
    """Time the fp64 oracle on whole sequences of the workload until ``budget_s`` is spent
    (None: every sequence). ``absorbed``: the oracle's absorbed form (einsums 3-5 of the
    DeepSeek-V2 page's matrix absorption) instead of the unabsorbed one."""
    import oracle.mla_oracle as O
    fn = O.mla_decode_absorbed if absorbed else O.mla_decode_reference
    try:
        from threadpoolctl import threadpool_info
        cores = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    except Exception:
        cores = os.cpu_count()
    order = list(np.argsort(-wl.seq_lens)) if cfg.lens_range else list(range(cfg.batch))
    done, tok_ctx, t0 = [], 0, time.perf_counter()
    for b in order:
        c_kv, k_r = wl.context(int(b))
        fn(wl.q_nope[b], wl.q_pe[b], c_kv, k_r, wl.w_uk, wl.w_uv, wl.bias, wl.theta,
           wl.query_positions()[b], cfg.softmax_scale, causal=cfg.causal)
        done.append(int(b))
        tok_ctx += int(wl.seq_lens[b])
        if ((budget_s is not None and time.perf_counter() - t0 >= budget_s) or
                (max_seqs and len(done) >= max_seqs)):
            break
    el = time.perf_counter() - t0
    form = "absorbed" if absorbed else "unabsorbed"
    return {"value": len(done) * cfg.q_len / el, "unit": "tokens/s", "cores": int(cores),
            "kind": "oracle_absorbed" if absorbed else "oracle",
            "sample": f"{len(done)} of {cfg.batch} sequences ({tok_ctx} cached tokens, all "
                      f"{cfg.num_heads} heads), fp64 {form} form, {el:.1f} s"}


def run_reference(args, cfg, rank, world):
    from mla_inputs import make_workload
    if rank != 0:
        return
    wl = make_workload(cfg)
    per_step = []
    for it in range(args.warmup + args.steps):
        s = cpu_oracle_sample(cfg, wl, budget_s=0.0, max_seqs=1)
        if it >= args.warmup:
            per_step.append(s)
    v = statistics.mean(x["value"] for x in per_step)
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1000.0 * cfg.q_len / v,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": _config_json(cfg),
            "cpu_baseline": {"value": v, "unit": "tokens/s", "cores": per_step[0]["cores"],
                             "kind": "oracle", "sample": "each step: " + per_step[0]["sample"]},
            "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def _config_json(cfg):
    return {"workload": cfg.name, "batch": cfg.batch, "q_len": cfg.q_len, "heads": cfg.num_heads,
            "kv_groups": cfg.num_kv_groups, "kv_lora_rank": cfg.kv_lora_rank,
            "rope_dim_per_group": cfg.rope_dim, "qk_nope_dim": cfg.qk_nope_dim,
            "v_head_dim": cfg.v_head_dim, "page_size": cfg.page_size,
            "context": cfg.context if cfg.lens_range is None else f"U{list(cfg.lens_range)}",
            "parallelism": "replicas"}


def roofline_of(cfg, seq_lens, t_ms, peaks):
    """Roofline object of one mla_decode_attn launch of `t_ms` milliseconds."""
    nbytes, flops = algorithmic_work(cfg, seq_lens)
    gbs = nbytes / (t_ms * 1e-3) / 1e9
    tfl = flops / (t_ms * 1e-3) / 1e12
    t_hbm = nbytes / (peaks["hbm_gbs"] * 1e9)
    t_tc = flops / (peaks["bf16_tflops"] * 1e12)
    if t_hbm >= t_tc:
        roof = {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": gbs / peaks["hbm_gbs"]}
    else:
        roof = {"bound": "tensor", "achieved": tfl, "peak": peaks["bf16_tflops"],
                "unit": "TFLOP/s", "frac": tfl / peaks["bf16_tflops"]}
    roof.update({"traffic": _traffic(cfg), "peak_source": peaks["source"],
                 "kernel": decode_kernel_name(cfg) + " (+ merge of cut units when the work is split)",
                 "algorithmic_bytes_per_launch": nbytes, "algorithmic_flops_per_launch": flops,
                 "achieved_gbs": gbs, "achieved_tflops": tfl,
                 "roofline_time_us": 1e6 * max(t_hbm, t_tc),
                 "pct_of_roofline": 100.0 * max(t_hbm, t_tc) / (t_ms * 1e-3)})
    return roof


def time_calls(fn, n, stream, flush=None):
    """Per-call times (ms) of `n` back-to-back calls of fn(stream), CUDA events on the
    launching stream; an L2 flush between calls when `flush` is given."""
    import torch
    evs = []
    for _ in range(n):
        if flush is not None:
            flush.zero_()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        fn(stream)
        b.record(stream)
        evs.append((a, b))
    torch.cuda.synchronize()
    return [a.elapsed_time(b) for a, b in evs]


def time_decode(prob, cfg, n, stream, flush=None, kv_shared=False):
    """Per-launch times (ms) of `n` back-to-back mla_decode_attn calls (for the K = V form,
    the decode over whole rows that kv_shared_step set up)."""
    import head_latent_attention_attn_b200 as mla
    if kv_shared:
        args = (prob.kv_dims, prob.q_ext_kv, prob.o_lat_kv, prob.lse_kv, prob.ws_kv)
    else:
        args = (prob.dims, prob.q_ext, prob.o_latent, prob.lse, prob.workspace)
    dims, q_ext, o_lat, lse, ws = args

    def call(stream):
        mla.mla_decode_attn(dims, q_ext, prob.cache, prob.block_table, prob.seq_lens,
                            prob.max_seq_len, ws, o_lat, lse, causal=cfg.causal,
                            num_splits=prob.num_splits, stream=stream)
    return time_calls(call, n, stream, flush)


# Workloads timed after the headline in the default run: every other decode shape, the
# single-latent K = V layer, the prefill chunks and the fused down-projection + append.
PER_CONFIG = ("tiny", "qwen25_7b", "qwen3_30b_a3b", "hybrid_1m_q1", "hybrid_1m_q4",
              "hybrid_256k_q1", "hybrid_256k_q4", "nanowhale_kv_shared",
              "prefill_deepseek_v2_q64", "prefill_deepseek_v2_q256", "prefill_deepseek_v2_q1024",
              "prefill_hybrid_q64", "prefill_hybrid_q256", "prefill_hybrid_q1024")
DOWN_KV = ("deepseek_v2", "qwen3_30b_a3b")   # mla_down_kv_append at these decode batches
OUT_PROJ = ("deepseek_v2",)                  # mla_out_proj at this decode batch
CPU_FULL = ("tiny", "qwen25_7b")             # both fp64 CPU forms timed over every sequence
DECODE_BLOCK = 60   # decode launches timed back to back for the roofline figure


def run_gpu(args, cfg, rank, world, dist):
    import torch

    import head_latent_attention_attn_b200 as mla
    from mla_inputs import CONFIGS, make_workload
    from mla_inputs.device import DeviceProblem

    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    mla.lib()
    wl = make_workload(cfg)
    prob = DeviceProblem(wl, num_splits=args.splits, device=str(dev))
    stream = torch.cuda.current_stream()
    cache_bytes, _ = algorithmic_work(cfg, wl.seq_lens)
    flush = None
    if cache_bytes < 2 * L2_BYTES:
        flush = torch.empty(4 * L2_BYTES // 4, dtype=torch.float32, device=dev)
    plan_splits_ws = prob.workspace.numel()

    def barrier():
        if dist is not None:
            dist.barrier()
        torch.cuda.synchronize()

    def one_step():
        # One library call: the append folded into the absorption kernel, the decode (and
        # the merge of cut sequences), the up-projection. Each kernel is launched so that it
        # may start while the previous one drains (programmatic dependent launch), so no
        # event is recorded between them (a stream event between two kernels would
        # serialise them).
        prob.step(stream)

    for _ in range(args.warmup):
        if flush is not None:
            flush.zero_()
        one_step()
    time_decode(prob, cfg, 3, stream, flush)
    barrier()
    with ClockSampler(_gpu_id(local)) as clk:
        barrier()
        clk.mark_start()
        if flush is None:
            # inputs larger than L2: the K steps run back to back between two events
            t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            t0.record(stream)
            for _ in range(args.steps):
                one_step()
            t1.record(stream)
            torch.cuda.synchronize()
            step_ms = [t0.elapsed_time(t1) / args.steps]
        else:
            # small caches: an L2 flush between steps, each step between its own events
            step_ms = time_calls(lambda st: one_step(), args.steps, stream, flush)
        # the decode alone, back to back: the roofline figure (median of DECODE_BLOCK launches)
        dec_block = time_decode(prob, cfg, DECODE_BLOCK, stream, flush)
        # the same step as four library calls (append, absorb, decode + merge, out_up)
        if flush is None:
            t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            t0.record(stream)
            for _ in range(args.steps):
                prob.step_four_calls(stream)
            t1.record(stream)
            torch.cuda.synchronize()
            step4_ms = [t0.elapsed_time(t1) / args.steps]
        else:
            step4_ms = time_calls(lambda st: prob.step_four_calls(stream), args.steps, stream,
                                  flush)
        barrier()
        clk.mark_end()
    t_step = statistics.mean(step_ms)
    t_dec = statistics.median(dec_block)
    t_dec_mean = statistics.mean(dec_block)
    status = mla.mla_get_device_status(prob.workspace.view(torch.int32)[:1])
    if status != mla.MLA_OK:
        raise RuntimeError(f"device error word set: {mla.STATUS_NAMES[status]}")

    # ---- end to end through the public API with pinned host buffers ------------------------
    # Every step copies its inputs from pinned host memory and reads its outputs back. The
    # inputs of a step sit in one pinned buffer (each at a 256-byte aligned offset) and go to
    # the device in one copy; o and lse come back in one copy. Two buffer sets and three
    # streams let step k's host->device copy, step k-1's compute and step k-2's device->host
    # copy run at once, as a serving loop would.
    in_names = ("c_new", "k_new", "cos_q", "sin_q", "start_pos", "q_nope", "q_pe")

    def packed(like, device):
        """One uint8 buffer (pinned on the host) holding tensors shaped like `like`."""
        offs, off = {}, 0
        for k, t in like.items():
            offs[k] = off
            off += (t.numel() * t.element_size() + 255) // 256 * 256
        buf = torch.empty(off, dtype=torch.uint8, device=device)
        if device == "cpu":
            buf = buf.pin_memory()
        views = {k: buf[o:o + t.numel() * t.element_size()].view(t.dtype).view(t.shape)
                 for (k, t), o in zip(like.items(), offs.values())}
        return buf, views

    like_in = {k: getattr(prob, k) for k in in_names}
    like_out = {"o": prob.o, "lse": prob.lse}
    host_in, dev_in, host_out, dev_out = [], [], [], []
    for _ in range(2):
        hb, hv = packed(like_in, "cpu")
        for k in in_names:
            hv[k].copy_(like_in[k].cpu())
        host_in.append((hb, hv))
        dev_in.append(packed(like_in, dev))
        host_out.append(packed(like_out, "cpu"))
        dev_out.append(packed(like_out, dev))
    h2d = host_in[0][0].numel()
    d2h = host_out[0][0].numel()
    s_h2d, s_d2h = torch.cuda.Stream(), torch.cuda.Stream()
    ev_in = [torch.cuda.Event() for _ in range(2)]      # inputs of a set copied in
    ev_comp = [torch.cuda.Event() for _ in range(2)]    # a set's step computed
    ev_out = [torch.cuda.Event() for _ in range(2)]     # a set's outputs copied out

    def e2e_steps(n):
        for k in range(n):
            s = k % 2
            with torch.cuda.stream(s_h2d):
                s_h2d.wait_event(ev_comp[s])            # step k-2 finished reading the set
                dev_in[s][0].copy_(host_in[s][0], non_blocking=True)
                ev_in[s].record(s_h2d)
            stream.wait_event(ev_in[s])
            stream.wait_event(ev_out[s])                # step k-2's outputs already read back
            d, o = dev_in[s][1], dev_out[s][1]
            mla.mla_decode_step(prob.dims, c_kv_new=d["c_new"], k_r_new=d["k_new"],
                                cos_new=d["cos_q"], sin_new=d["sin_q"], start_pos=d["start_pos"],
                                q_nope=d["q_nope"], q_pe=d["q_pe"], cos_q=d["cos_q"],
                                sin_q=d["sin_q"], w_uk=prob.w_uk, w_uv=prob.w_uv, bias=prob.bias,
                                cache=prob.cache, block_table=prob.block_table,
                                seq_lens=prob.seq_lens, max_seq_len=prob.max_seq_len,
                                q_ext=prob.q_ext, workspace=prob.workspace,
                                o_latent=prob.o_latent, lse=o["lse"], o=o["o"],
                                causal=cfg.causal, num_splits=args.splits, stream=stream)
            ev_comp[s].record(stream)
            with torch.cuda.stream(s_d2h):
                s_d2h.wait_event(ev_comp[s])
                host_out[s][0].copy_(dev_out[s][0], non_blocking=True)
                ev_out[s].record(s_d2h)

    for e in ev_comp + ev_out:
        e.record(stream)
    e2e_steps(max(args.warmup, 2))
    barrier()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(s_h2d)
    e2e_steps(args.steps)
    t1.record(s_d2h)       # after the last read-back in stream order
    barrier()
    t_e2e = t0.elapsed_time(t1) / args.steps
    # the outputs read back match the device-resident step's
    if not all(torch.equal(host_out[i][1]["o"], prob.o.cpu()) and
               torch.equal(host_out[i][1]["lse"], prob.lse.cpu()) for i in range(2)):
        raise RuntimeError("end-to-end outputs differ from the device-resident step")

    # ---- max over ranks -------------------------------------------------------------------
    t_step, t_dec, t_dec_mean, t_e2e, t_step4 = max_over_ranks(
        [t_step, t_dec, t_dec_mean, t_e2e, statistics.mean(step4_ms)], dist, dev)
    peaks = _peaks()
    tokens = cfg.batch * cfg.q_len
    value = world * tokens / (t_step * 1e-3)
    roof = roofline_of(cfg, wl.seq_lens, t_dec, peaks)
    # absorb with the append folded in, decode, out_up (+ the split combine when the plan has
    # > 1 split; a one-split plan needs only the 256-byte error-word workspace)
    merge = 1 if plan_splits_ws > 256 else 0
    # the one-call steps, the decode block and the four-call steps
    launches = (3 + merge) * args.steps + (1 + merge) * DECODE_BLOCK + (4 + merge) * args.steps
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": t_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": dict(_config_json(cfg), l2=("cache > L2, no flush" if flush is None
                                              else "L2 flushed between launches (504 MB write)")),
        "step_four_calls_ms": t_step4,
        "decode_us": 1e3 * t_dec, "decode_us_mean": 1e3 * t_dec_mean,
        "decode_launches_timed": DECODE_BLOCK,
        "step_timing": ("K steps back to back between two events" if flush is None
                        else "each step between its own events, L2 flushed before each"),
        "decode_gbs": roof["achieved_gbs"], "decode_tflops": roof["achieved_tflops"],
        "roofline": roof,
        "e2e": {"value": world * tokens / (t_e2e * 1e-3), "unit": "tokens/s",
                "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
                "ms_per_step": t_e2e,
                "method": "every step: its inputs copied in from one pinned host buffer and "
                          "o + lse read back into another (one copy each way); copies of "
                          "neighbouring steps overlap the compute on separate streams"},
        "gpu_launches": launches,
        "clocks": clk.summary(),
    }
    del prob, flush
    torch.cuda.empty_cache()
    if not args.no_per_config:
        line["per_config"] = per_config_block(args, cfg, dev, stream, dist, peaks)
    if rank != 0:
        return
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_oracle_sample(cfg, wl, budget_s=args.cpu_budget)
        # the absorbed fp64 form beside it: a second CPU baseline
        line["cpu_baseline_absorbed"] = cpu_oracle_sample(cfg, wl, budget_s=args.cpu_budget / 2,
                                                          absorbed=True)
    print(json.dumps(line), flush=True)


def per_config_block(args, head_cfg, dev, stream, dist, peaks):
    """mla_decode_attn on every other workload, in the same process: the median of
    DECODE_BLOCK launches, its roofline and the clocks seen while it ran; then the fused
    down-projection + append. Every rank runs the same workloads (timings maxed over ranks)."""
    import torch

    import head_latent_attention_attn_b200 as mla
    from mla_inputs import CONFIGS, make_down_kv_inputs, make_o_proj_inputs, make_workload
    from mla_inputs.device import DeviceProblem
    out = {}
    only = {x.strip() for x in args.per_config.split(",") if x.strip()}
    want = (lambda key: not only or key in only)
    for name in PER_CONFIG:
        if name == head_cfg.name or not want(name):
            continue
        cfg = CONFIGS[name]
        kv = name.startswith("nanowhale")
        wl = make_workload(cfg)
        prob = DeviceProblem(wl, device=str(dev))
        if kv:
            prob.kv_shared_step()
        else:
            prob.step()
        nbytes, _ = algorithmic_work(cfg, wl.seq_lens)
        flush = (torch.empty(4 * L2_BYTES // 4, dtype=torch.float32, device=dev)
                 if nbytes < 2 * L2_BYTES else None)
        time_decode(prob, cfg, 3, stream, flush, kv)
        with ClockSampler(_gpu_id(dev.index or 0)) as clk:
            clk.mark_start()
            ms = time_decode(prob, cfg, DECODE_BLOCK, stream, flush, kv)
            clk.mark_end()
        t_med, t_mean = max_over_ranks([statistics.median(ms), statistics.mean(ms)], dist, dev)
        out[name] = {"decode_us": 1e3 * t_med, "decode_us_mean": 1e3 * t_mean,
                     "launches": DECODE_BLOCK,
                     "tokens_per_s": cfg.batch * cfg.q_len / (t_med * 1e-3),
                     "roofline": roofline_of(cfg, wl.seq_lens, t_med, peaks),
                     "l2": "cache > L2, no flush" if flush is None else "L2 flushed between launches",
                     "clocks": clk.summary()}
        # the two smallest workloads: both fp64 CPU forms over every sequence (rank 0, N = 1)
        if name in CPU_FULL and not args.no_cpu_baseline and dist is None:
            out[name]["cpu_baseline"] = cpu_oracle_sample(cfg, wl, budget_s=None)
            out[name]["cpu_baseline_absorbed"] = cpu_oracle_sample(cfg, wl, budget_s=None,
                                                                   absorbed=True)
        del prob, flush, wl
        torch.cuda.empty_cache()
    # einsums (5) and (6) fused (mla_out_proj) at the DeepSeek-V2 decode batch
    for name in (OUT_PROJ if want("out_proj") else ()):
        cfg = CONFIGS[name]
        rows = cfg.batch * cfg.q_len
        dims = mla.make_dims(cfg.num_heads, cfg.num_kv_groups, cfg.kv_lora_rank, cfg.qk_nope_dim,
                             cfg.rope_dim, cfg.v_head_dim, cfg.page_size, cfg.softmax_scale)
        g = torch.Generator(device=dev)
        g.manual_seed(cfg.seed)
        o_lat = (torch.randn(rows, cfg.num_heads, cfg.kv_lora_rank, device=dev, generator=g) /
                 math.sqrt(cfg.kv_lora_rank)).to(torch.bfloat16)
        w_uv = make_workload(cfg.with_(context=64, lens_range=None, batch=1)).w_uv.to(dev)
        w_o, _ = make_o_proj_inputs(cfg)
        w_o = w_o.to(dev)
        o = torch.empty(rows, cfg.num_heads, cfg.v_head_dim, dtype=torch.bfloat16, device=dev)
        u = torch.empty(rows, cfg.hidden_size, dtype=torch.bfloat16, device=dev)
        ws = torch.zeros(mla.mla_out_proj_workspace_size(dims, cfg.hidden_size, rows),
                         dtype=torch.uint8, device=dev)
        flush = torch.empty(4 * L2_BYTES // 4, dtype=torch.float32, device=dev)

        def call(stream, dims=dims, o_lat=o_lat, w_uv=w_uv, w_o=w_o, ws=ws, o=o, u=u):
            mla.mla_out_proj(dims, o_lat, w_uv, w_o, ws, o, u, stream=stream)
        time_calls(call, 3, stream, flush)
        with ClockSampler(_gpu_id(dev.index or 0)) as clk:
            clk.mark_start()
            ms = time_calls(call, DECODE_BLOCK, stream, flush)
            clk.mark_end()
        t_med, t_mean = max_over_ranks([statistics.median(ms), statistics.mean(ms)], dist, dev)
        nbytes = (w_uv.numel() + w_o.numel() + o_lat.numel() + o.numel() + u.numel()) * 2
        flops = 2 * rows * cfg.num_heads * cfg.v_head_dim * (cfg.kv_lora_rank + cfg.hidden_size)
        gbs = nbytes / (t_med * 1e-3) / 1e9
        out[f"out_proj[{name}]"] = {
            "us": 1e3 * t_med, "us_mean": 1e3 * t_mean, "launches": DECODE_BLOCK, "rows": rows,
            "hidden_size": cfg.hidden_size,
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": gbs / peaks["hbm_gbs"], "algorithmic_bytes_per_launch": nbytes,
                         "algorithmic_flops_per_launch": flops, "peak_source": peaks["source"],
                         "kernel": "oproj_kernel (einsum 5 then einsum 6, one cooperative launch)"},
            "l2": "L2 flushed between launches", "clocks": clk.summary()}
        del o_lat, w_uv, w_o, o, u, ws, flush
        torch.cuda.empty_cache()
    for name in (DOWN_KV if want("down_kv") else ()):
        cfg = CONFIGS[name]
        wl = make_workload(cfg.with_(context=128, lens_range=None))
        prob = DeviceProblem(wl, device=str(dev))
        hidden, w_dkv = make_down_kv_inputs(cfg, cfg.q_len)
        hidden, w_dkv = hidden.to(dev), w_dkv.to(dev)
        flush = torch.empty(4 * L2_BYTES // 4, dtype=torch.float32, device=dev)

        def call(stream, prob=prob, hidden=hidden, w_dkv=w_dkv):
            mla.mla_down_kv_append(prob.dims, hidden, w_dkv, prob.cos_q, prob.sin_q,
                                   prob.block_table, prob.start_pos, prob.cache,
                                   dev_error=prob.err, stream=stream)
        time_calls(call, 3, stream, flush)
        with ClockSampler(_gpu_id(dev.index or 0)) as clk:
            clk.mark_start()
            ms = time_calls(call, DECODE_BLOCK, stream, flush)
            clk.mark_end()
        t_med, t_mean = max_over_ranks([statistics.median(ms), statistics.mean(ms)], dist, dev)
        rows = cfg.batch * cfg.q_len
        nbytes = (w_dkv.numel() + hidden.numel() + rows * cfg.row_width) * 2
        flops = 2 * rows * cfg.row_width * cfg.hidden_size
        gbs = nbytes / (t_med * 1e-3) / 1e9
        out[f"down_kv_append[{name}]"] = {
            "us": 1e3 * t_med, "us_mean": 1e3 * t_mean, "launches": DECODE_BLOCK,
            "rows": rows, "hidden_size": cfg.hidden_size,
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": gbs / peaks["hbm_gbs"], "algorithmic_bytes_per_launch": nbytes,
                         "algorithmic_flops_per_launch": flops, "peak_source": peaks["source"],
                         "kernel": "down_kv_kernel (split-K on clusters, cache-append epilogue)"},
            "l2": "L2 flushed between launches", "clocks": clk.summary()}
        del prob, flush, hidden, w_dkv, wl
        torch.cuda.empty_cache()
    return out


def _gpu_id(local: int) -> str:
    import torch
    try:
        u = str(torch.cuda.get_device_properties(local).uuid)
        return u if u.startswith("GPU-") else "GPU-" + u
    except Exception:
        return str(local)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--config", default=DEFAULT_CONFIG)
    ap.add_argument("--impl", default="b200", choices=["b200", "reference"])
    ap.add_argument("--splits", type=int, default=0, help="KV splits per sequence (0 = auto)")
    ap.add_argument("--cpu-budget", type=float, default=12.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-per-config", action="store_true",
                    help="time only the headline workload")
    ap.add_argument("--per-config", default="",
                    help="comma-separated subset of the per-config entries to time (workload "
                         "names, 'out_proj', 'down_kv'); default all")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)

    from mla_inputs import CONFIGS
    cfg = CONFIGS[args.config]
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    dist = None
    if world > 1:
        import datetime

        import torch
        import torch.distributed as tdist
        if args.impl == "reference":
            if rank == 0:
                run_reference(args, cfg, rank, world)
            return
        torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", "0")))
        tdist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
        dist = tdist
    try:
        if args.impl == "reference":
            run_reference(args, cfg, rank, world)
        else:
            run_gpu(args, cfg, rank, world, dist)
    finally:
        if dist is not None:
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
