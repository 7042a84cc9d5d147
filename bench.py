"""Throughput of the per-frame AR decode of the 36-layer 8B Global LLM on B200.

Workload (default): the full 36-layer Qwen3-8B-shaped body (hidden 4096,
32/8 heads of 128, SwiGLU 12288) + final RMSNorm + lm_head sliced to 16384
of 200000 vocab rows + CFG 1.5 + Gumbel-argmax at T = 1, bf16 weights drawn
N(0, 0.02^2) from a seed, bf16 KV cache of a 1500-frame (60 s) song grown
in 256-frame buckets, 2 rows (one cond/uncond pair).

A step is one frame.  The K timed frames sit at evenly spaced positions of
the song, (i + 1/2) * 1500 / K, so their mean is the song's mean frame time
whatever K is; the cache holds seeded N(0, 1) keys/values for earlier
positions.  Weights (14 GB) are far larger than L2 (126 MB), so no flush is
needed between frames.

Prints one JSON line (rank 0).  Under torchrun each rank decodes its own
independent 2-row replica on its GPU (no collective on the data path) and
the timing is the max over ranks.  `--impl reference` times the CPU oracle
on a bounded sample of the same frame.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

SONG_FRAMES = 1500
ROWS = 2
CFG_SCALE = 1.5
METRIC = "AR frames/s per row (8B, bf16, 2 rows)"
WORKLOAD = "qwen3-8b-36L-bf16-2rows-song1500-cfg1.5"


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=60)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", default="ours", choices=["ours", "reference"])
    p.add_argument("--wdtype", default="bf16", choices=["bf16", "int8"])
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--layers", type=int, default=36,
                   help="body layers (36 = the workload; fewer only for profiling small cases)")
    p.add_argument("--kv", default="bf16", choices=["bf16", "f16"])
    p.add_argument("--top-k", type=int, default=0,
                   help="top-k filter of the frame draw (0 keeps every logit, as the timed "
                        "configs do)")
    p.add_argument("--depth", action="store_true",
                   help="run the RVQ depth decoder (7 codes) after every frame")
    p.add_argument("--generate", type=int, default=0, metavar="F",
                   help="time the GPU generation loop (m3_generate) over F frames of a song "
                        "after a 300-position prompt, against host-driven m3_decode_frame")
    p.add_argument("--prefill", type=int, default=0, metavar="P",
                   help="time the prompt prefill (m3_prefill) of P tokens into one row")
    p.add_argument("--rows", type=int, default=ROWS,
                   help="batch rows (even: CFG pairs); 2 = the workload")
    p.add_argument("--ctx", type=int, default=0,
                   help="every timed frame at this context (prefilled) instead of the "
                        "1500-frame song's spread of positions; for profiling cases")
    p.add_argument("--depth-only", action="store_true",
                   help="time the RVQ depth decoder (m3_depth_decode) alone, int8 group-128, "
                        "on a frame's hidden state")
    p.add_argument("--dit", action="store_true",
                   help="the DiT chunk-denoise workload: full-size DiT (36 blocks, width 2048, "
                        "FFN 8192), one 200-frame chunk = 689 latent frames, cond + uncond as "
                        "one batch-2 forward; a step is one denoising step")
    p.add_argument("--sweep", action="store_true",
                   help="batched-variations sweep: rows 1..16 x context 1500/4500/9000, "
                        "bf16 and int8; one JSON line per point")
    return p.parse_args()


# ----------------------------------------------------------- distributed ----

def dist_env():
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def replica_seed(rank: int) -> int:
    """Each rank decodes an independent replica (its own seeds): weights are
    shared in distribution, inputs and noise differ."""
    return 1000 + rank


def max_over_ranks(value: float, world: int, device=None) -> float:
    if world <= 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def song_positions(k: int, song: int = SONG_FRAMES):
    return [min(song - 1, int((i + 0.5) * song / k)) for i in range(k)]


# ---------------------------------------------------------------- clocks ----

class ClockSampler:
    """SM clock and clock-event reasons sampled DURING the timed region.

    An NVML polling thread (every 5 ms, read-only queries) finds this
    process's GPU by PCI bus id; where NVML is missing it falls back to an
    `nvidia-smi -lms 200` child process."""
    REASONS = (("hw_slowdown", 0x8), ("hw_thermal_slowdown", 0x40),
               ("sw_thermal_slowdown", 0x20), ("sw_power_cap", 0x4))
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, local: int, path: str):
        self.local = local
        self.path = path
        self.samples = []
        self.stop_flag = False
        self.thread = None
        self.proc = None
        self.nvml = None
        self.handle = None
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            p = torch.cuda.get_device_properties(local)
            want = (int(p.pci_domain_id), int(p.pci_bus_id), int(p.pci_device_id))
            for i in range(pynvml.nvmlDeviceGetCount()):
                h = pynvml.nvmlDeviceGetHandleByIndex(i)
                info = pynvml.nvmlDeviceGetPciInfo(h)
                if (int(info.domain), int(info.bus), int(info.device)) == want:
                    self.handle = h
                    break
            if self.handle is not None:
                self.nvml = pynvml
        except Exception:
            self.nvml = None

    def _poll(self):
        nv = self.nvml
        while not self.stop_flag:
            try:
                sm = nv.nvmlDeviceGetClockInfo(self.handle, nv.NVML_CLOCK_SM)
                smax = nv.nvmlDeviceGetMaxClockInfo(self.handle, nv.NVML_CLOCK_SM)
                rs = nv.nvmlDeviceGetCurrentClocksEventReasons(self.handle)
                self.samples.append((float(sm), float(smax), int(rs)))
            except Exception:
                pass
            time.sleep(0.005)

    def start(self):
        if self.nvml is not None:
            import threading
            self.thread = threading.Thread(target=self._poll, daemon=True)
            self.thread.start()
            return
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", f"-i={self.local}",
                                          f"--query-gpu={self.QUERY}", "--format=csv,noheader",
                                          "-lms", "200"], stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self) -> dict:
        if self.thread is not None:
            self.stop_flag = True
            self.thread.join()
            sm = [s for s, _, _ in self.samples]
            smax = [m for _, m, _ in self.samples]
            reasons = {n for _, _, r in self.samples for n, bit in self.REASONS if r & bit}
            return {"sm_mhz": statistics.median(sm) if sm else None,
                    "sm_max_mhz": max(smax) if smax else None, "reasons": sorted(reasons),
                    "samples": len(sm), "source": "nvml, 5 ms"}
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["clock sampling unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.f.close()
        sm, smax, reasons = [], [], set()
        for line in open(self.path):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1].split()[0]))
                smax.append(float(parts[2].split()[0]))
            except ValueError:
                continue
            for (n, _), v in zip(self.REASONS, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None, "reasons": sorted(reasons),
                "samples": len(sm), "source": "nvidia-smi, 200 ms"}


# ------------------------------------------------------------ our arm ------

def build_model(torch, m3, synth, seed: int, wdtype: int, layers: int = 36, depth: bool = False,
                max_rows: int = ROWS, end_token: bool = False):
    import dataclasses
    s = dataclasses.replace(synth.FULL8B_END if end_token else synth.FULL8B, n_layers=layers)
    cfg = m3.config_from_shapes(s, synth.DEPTH if depth else None, max_rows=max_rows)
    ctx = m3.m3_create(cfg)
    for l in range(s.n_layers):  # generate on the GPU, load layer by layer
        Lw = synth.layer_weights(s, 0, l, device="cuda")
        m3.m3_load_weights(ctx, [Lw], first_layer=l, wdtype=wdtype)
        del Lw
    m3.m3_load_weights(ctx, [], final_norm=synth.final_norm(s, 0, device="cuda"),
                       lm_head=synth.lm_head_slice(s, 0, device="cuda"), wdtype=wdtype,
                       lm_end_row=synth.lm_head_end_row(s, 0, device="cuda") if end_token
                       else None)
    if depth:
        m3.m3_load_depth_weights(ctx, synth.depth_weights(synth.DEPTH, 0, device="cuda"))
    torch.cuda.synchronize()
    return s, ctx


def prefill_kv(torch, m3, synth, s, ctx, rows: int, n_pos: int, seed: int, kv_f16: bool):
    m3.m3_kv_alloc(ctx, rows, n_pos, m3.M3_KV_F16 if kv_f16 else m3.M3_KV_BF16, 256)
    for r in range(rows):  # one row at a time bounds the staging memory
        K, V = synth.kv_prefill(s, 1, n_pos, seed + 17 * r, device="cuda")
        m3.m3_kv_set(ctx, r, K[0], V[0])
        del K, V
    torch.cuda.synchronize()


def run_ours(args, rank, world, local):
    import torch
    from autoregressive_audio_token_b200 import m3
    import synth

    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    seed = replica_seed(rank)
    rows = args.rows
    song = args.ctx if args.ctx > 0 else SONG_FRAMES
    wdtype = m3.M3_W_INT8 if args.wdtype == "int8" else m3.M3_W_BF16
    s, ctx = build_model(torch, m3, synth, seed, wdtype, args.layers, depth=args.depth,
                         max_rows=rows)
    m3.m3_set_top_k(ctx, args.top_k)
    prefill_kv(torch, m3, synth, s, ctx, rows, song, seed, args.kv == "f16")
    xs = synth.normal((64, rows, s.hidden), seed, "bench/x_in", std=0.02, device="cuda")
    codes = torch.empty(rows, dtype=torch.int32, device="cuda")
    h_dev = torch.empty((rows, s.hidden), dtype=torch.bfloat16, device="cuda")
    dcodes = torch.empty((rows, synth.DEPTH.codebooks), dtype=torch.int32, device="cuda")
    stream = torch.cuda.current_stream()
    cfg = CFG_SCALE if rows % 2 == 0 else 0.0

    def frame_positions(k):
        # the song's evenly spaced positions, or every frame at the given context
        return [song - 1] * k if args.ctx > 0 else song_positions(k)

    def frame(i, pos):
        if args.depth:
            m3.m3_decode_frame(ctx, [pos] * rows, seed, i, xs[i % 64], cfg, 1.0, codes, h_dev)
            m3.m3_depth_decode(ctx, h_dev, codes, seed, i, cfg, 1.0, dcodes)
        else:
            m3.m3_decode_frame(ctx, [pos] * rows, seed, i, xs[i % 64], cfg, 1.0, codes)

    # capture every bucket's graph before timing, then warm up
    for b in range(0, song, 256):
        frame(0, b)
    warm = frame_positions(max(args.warmup, 3))
    for i, p in enumerate(warm):
        frame(i, p)
    torch.cuda.synchronize()
    m3.m3_sync_status(ctx)

    # ---- device-timed region: inputs resident in HBM -----------------------
    positions = frame_positions(args.steps)
    clocks = ClockSampler(local, f"/tmp/m3_clocks_rank{rank}.csv")
    barrier(world)
    torch.cuda.synchronize()
    clocks.start()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i, p in enumerate(positions):
        frame(i, p)
    e1.record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    barrier(world)
    ms = e0.elapsed_time(e1)
    m3.m3_sync_status(ctx)
    ms_max = max_over_ranks(ms, world, torch.device("cuda", local))
    ms_per_step = ms_max / args.steps

    # ---- end to end through the C ABI with host buffers ---------------------
    x_host = xs[:64].cpu().pin_memory()
    codes_host = torch.empty((args.steps, rows), dtype=torch.int32).pin_memory()
    nc = synth.DEPTH.codebooks if args.depth else 0
    dcodes_host = torch.empty((args.steps, rows, max(nc, 1)), dtype=torch.int32).pin_memory()
    x_dev = torch.empty((rows, s.hidden), dtype=torch.bfloat16, device="cuda")
    barrier(world)
    torch.cuda.synchronize()
    e2, e3 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e2.record(stream)
    for i, p in enumerate(positions):
        x_dev.copy_(x_host[i % 64], non_blocking=True)
        if args.depth:  # the frame and its residual codes, both read back
            m3.m3_decode_frame(ctx, [p] * rows, seed, i, x_dev, cfg, 1.0, codes, h_dev)
            m3.m3_depth_decode(ctx, h_dev, codes, seed, i, cfg, 1.0, dcodes)
            dcodes_host[i].copy_(dcodes, non_blocking=True)
        else:
            m3.m3_decode_frame(ctx, [p] * rows, seed, i, x_dev, cfg, 1.0, codes)
        codes_host[i].copy_(codes, non_blocking=True)
    e3.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    e2e_ms = max_over_ranks(e2.elapsed_time(e3), world, torch.device("cuda", local)) / args.steps

    # ---- the dominant kernel in isolation (gate/up + SwiGLU GEMV) ----------
    kernels = {}
    for which, name in [(2, "gate_up_swiglu"), (3, "down"), (0, "qkv"), (1, "o_proj"),
                        (4, "lm_head_sample")]:
        kms, kbytes = m3.m3_time_gemv(ctx, which, rows, 72 if which != 4 else 20)
        kernels[name] = {"ms": kms, "bytes": kbytes, "gbs": kbytes / kms / 1e6}

    mean_ctx = sum(positions) / len(positions)
    frame_bytes = m3.m3_frame_bytes(ctx, rows, int(round(mean_ctx)))
    peaks = {}
    try:
        peaks = json.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json")))
    except Exception:
        pass
    hbm_peak = peaks.get("hbm_gbs", 6650.0)
    peak_src = "measured" if "hbm_gbs" in peaks else "fallback"
    dom = kernels["gate_up_swiglu"]
    traffic = None
    try:
        prof = json.load(open(os.path.join(ROOT, "profiles", "gemv_traffic.json")))
        src_hash = prof.get("source_sha256")
        if src_hash == kernel_source_hash() and args.wdtype == "bf16":
            traffic = prof.get("gate_up_swiglu_bytes_per_launch")
    except Exception:
        pass

    fps = 1000.0 / ms_per_step * world
    variant = workload_name(args)
    out = {
        "metric": METRIC if args.wdtype == "bf16" else METRIC.replace("bf16", "int8"),
        "value": fps,
        "unit": "frames/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms_per_step,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": args.wdtype,
        "data": "synthetic (seeded N(0,0.02^2) weights, N(0,1) KV prefill, random-init 8B shape)",
        "config": {"workload": variant,
                   "rows": rows, "song_frames": song, "mean_ctx": mean_ctx,
                   "cfg_scale": cfg, "temperature": 1.0, "kv": f"{args.kv} pages of 256",
                   "depth_decoder": bool(args.depth), "top_k": args.top_k,
                   "l2": "no flush: 14 GB of weights per frame >> 126 MB L2",
                   "parallelism": f"replicas x{world}" if world > 1 else "single GPU"},
        "gpu_launches": None,
        "frame": {"algorithmic_bytes": frame_bytes, "achieved_gbs": frame_bytes / ms_per_step / 1e6,
                  "frac_of_measured_hbm": frame_bytes / ms_per_step / 1e6 / hbm_peak,
                  "frac_of_8tbs": frame_bytes / ms_per_step / 1e6 / 8000.0},
        "roofline": {"bound": "hbm",
                     "kernel": f"gemv_dyn_kernel gate/up + SwiGLU ({args.wdtype}, {rows} rows)",
                     "achieved": dom["gbs"], "peak": hbm_peak, "unit": "GB/s",
                     "frac": dom["gbs"] / hbm_peak, "peak_source": peak_src,
                     "traffic": traffic, "algorithmic_bytes_per_launch": dom["bytes"]},
        "kernels": kernels,
        "e2e": {"value": 1000.0 / e2e_ms * world, "unit": "frames/s",
                "h2d_bytes_per_step": rows * s.hidden * 2 + 4 * rows,
                "d2h_bytes_per_step": 4 * rows * (1 + nc)},
        "clocks": clk,
    }
    # per frame: parameter block + RoPE table + 5 kernels per layer (qkv,
    # attention, o, gate/up, down) + lm_head sampler, as the library counts
    # them; the depth decoder adds
    # its parameter block, projection, 7 embeddings, 8 positions x layers x 5
    # kernels and 7 heads
    depth_launches = m3.m3_depth_kernels(ctx, rows) if args.depth else 0
    out["gpu_launches"] = (m3.m3_frame_kernels(ctx, rows) + depth_launches) * args.steps
    m3.m3_destroy(ctx)
    del xs
    torch.cuda.empty_cache()
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline()
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return out


def kernel_source_hash() -> str:
    import hashlib
    h = hashlib.sha256()
    d = os.path.join(ROOT, "autoregressive_audio_token_b200", "csrc")
    for f in sorted(os.listdir(d)):
        if f.startswith("gemv") or f in ("common.cuh",):
            h.update(open(os.path.join(d, f), "rb").read())
    return h.hexdigest()


# -------------------------------------------------------- the oracle arm ----

SAMPLE_LAYERS = 2


class OracleSample:
    """A bounded sample of the frame on the CPU oracle (as it stands): the
    first SAMPLE_LAYERS of the 36 body layers for the 2 rows at the song's
    mean context, then the final norm + sliced lm_head + CFG + Gumbel-argmax.
    One step = one such sample, scaled to a full frame as
    36 / SAMPLE_LAYERS x body time + head time."""

    def __init__(self):
        import dataclasses
        import synth
        from oracle import oracle as O
        self.O = O
        s = synth.FULL8B
        sub = dataclasses.replace(s, n_layers=SAMPLE_LAYERS)
        layers = [synth.layer_weights(s, 0, l) for l in range(SAMPLE_LAYERS)]
        self.body = O.Body(sub, layers, synth.final_norm(s, 0), synth.lm_head_slice(s, 0))
        self.ctx = SONG_FRAMES // 2
        self.kc, self.vc = self.body.new_cache(ROWS, self.ctx + 1)
        K, V = synth.kv_prefill(sub, ROWS, self.ctx, 7)
        self.kc[:, :, :self.ctx] = O.bits(K)
        self.vc[:, :, :self.ctx] = O.bits(V)
        self.x = O.bits(synth.frame_input(s, ROWS, 7, 0))
        self.n_layers = s.n_layers

    def frame_seconds(self, i: int) -> float:
        t0 = time.perf_counter()
        hx = self.body.body(self.kc, self.vc, [self.ctx] * ROWS, self.x)
        t1 = time.perf_counter()
        self.body.sample(hx, 7, i, cfg_scale=CFG_SCALE)
        t2 = time.perf_counter()
        return (t1 - t0) * self.n_layers / SAMPLE_LAYERS + (t2 - t1)

    def describe(self, frames: int) -> str:
        return (f"{frames} frame(s), each {SAMPLE_LAYERS} of 36 layers at ctx {self.ctx} for "
                f"{ROWS} rows + lm_head/CFG/draw, scaled to a full frame as "
                f"36/{SAMPLE_LAYERS} x body + head")


def tiny_oracle_frames() -> dict:
    """The oracle on the tiny 1-layer model: 16 consecutive frames, each
    frame's code fed back through the token embedding (the tiny workload the
    GPU parity tests run), all host cores."""
    import synth
    from oracle import oracle as O
    s = synth.TINY
    body = O.Body(s, [synth.layer_weights(s, 0, 0)], synth.final_norm(s, 0),
                  synth.lm_head_slice(s, 0))
    kc, vc = body.new_cache(1, 128)
    K, V = synth.kv_prefill(s, 1, 64, 0)
    kc[:, :, :64] = O.bits(K)
    vc[:, :, :64] = O.bits(V)
    E = O.bits(synth.embedding(s, 0))
    x = O.bits(synth.frame_input(s, 1, 0, 0))
    t0 = time.perf_counter()
    for f in range(16):
        codes, _, _ = body.decode_frame(kc, vc, [64 + f], 0, f, x)
        x = E[s.slice_start + codes].copy()
    return {"ms_per_frame": (time.perf_counter() - t0) * 1000.0 / 16, "frames": 16}


def cpu_baseline(frames: int = 2) -> dict:
    """The CPU oracle as it stands on this host's cores (OracleSample), plus
    the same sample on one core and the tiny model's 16-frame run."""
    O = __import__("oracle.oracle", fromlist=["oracle"])
    smp = OracleSample()
    cores = O.num_threads()
    t = [smp.frame_seconds(i) for i in range(frames)]
    O.set_threads(1)
    try:
        t1 = smp.frame_seconds(0)
    finally:
        O.set_threads(cores)
    frame_s = statistics.mean(t)
    return {"value": 1.0 / frame_s, "unit": "frames/s", "cores": cores,
            "kind": "oracle", "ms_per_frame": frame_s * 1000.0,
            "sample": smp.describe(frames),
            "one_core": {"ms_per_frame": t1 * 1000.0, "frames_per_s": 1.0 / t1, "cores": 1},
            "tiny_1layer_16frames": tiny_oracle_frames()}


def run_reference(args, rank, world):
    """The oracle arm: W untimed warm-up samples, then exactly K timed steps,
    each one OracleSample frame; rank 0 only."""
    if rank != 0:
        return None
    O = __import__("oracle.oracle", fromlist=["oracle"])
    smp = OracleSample()
    for i in range(args.warmup):
        smp.frame_seconds(i)
    t = [smp.frame_seconds(args.warmup + i) for i in range(args.steps)]
    frame_s = statistics.mean(t)
    value = 1.0 / frame_s
    cb = {"value": value, "unit": "frames/s", "cores": O.num_threads(), "kind": "oracle",
          "ms_per_frame": frame_s * 1000.0, "sample": smp.describe(args.steps)}
    return {"metric": METRIC, "value": value, "unit": "frames/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": frame_s * 1000.0,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic", "impl": "reference",
            "config": {"workload": WORKLOAD, "rows": ROWS, "song_frames": SONG_FRAMES,
                       "sample": smp.describe(args.steps)},
            "cpu_baseline": cb,
            "e2e": {"value": value, "unit": "frames/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


def workload_name(args) -> str:
    name = WORKLOAD.replace("bf16", args.wdtype)
    if args.rows != ROWS:
        name = name.replace("2rows", f"{args.rows}rows")
    if args.ctx > 0:
        name = name.replace("song1500", f"ctx{args.ctx}")
    if args.rows % 2:
        name = name.replace("-cfg1.5", "")
    if args.layers != 36:
        name = name.replace("36L", f"{args.layers}L")
    if args.kv != "bf16":
        name += f"-{args.kv}kv"
    if args.depth:
        name += "-depth7"
    if args.top_k:
        name += f"-top{args.top_k}"
    return name


def run_sweep(args):
    """Batched-variations sweep: one unguided row (CFG off), then K = 1, 2, 4, 8
    same-prompt variations decoded in lockstep (rows = 2K, CFG on), contexts
    1500 / 4500 / 9000, bf16 and int8 weights, bf16 KV; per point one JSON line
    with frames/s per row, ms/frame, the frame's algorithmic bytes and GB/s,
    T_rows / T_1, and the cost of each extra row (pair) relative to the 1-row
    (2-row) frame at the same context."""
    import torch
    from autoregressive_audio_token_b200 import m3
    import synth
    torch.cuda.set_device(0)
    for wname in ("bf16", "int8"):
        wd = m3.M3_W_INT8 if wname == "int8" else m3.M3_W_BF16
        s, ctx = build_model(torch, m3, synth, 7, wd, max_rows=16)
        for n_ctx in (1500, 4500, 9000):
            base = None
            t1 = None
            for rows in (1, 2, 4, 8, 16):
                prefill_kv(torch, m3, synth, s, ctx, rows, n_ctx, 7, False)
                xs = synth.normal((rows, s.hidden), 7, "sweep/x", std=0.02, device="cuda")
                codes = torch.empty(rows, dtype=torch.int32, device="cuda")
                pos = [n_ctx - 1] * rows
                cfg = CFG_SCALE if rows % 2 == 0 else 0.0
                for i in range(3):
                    m3.m3_decode_frame(ctx, pos, 7, i, xs, cfg, 1.0, codes)
                torch.cuda.synchronize()
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                steps = 10
                e0.record()
                for i in range(steps):
                    m3.m3_decode_frame(ctx, pos, 7, i, xs, cfg, 1.0, codes)
                e1.record()
                torch.cuda.synchronize()
                m3.m3_sync_status(ctx)
                ms = e0.elapsed_time(e1) / steps
                fb = m3.m3_frame_bytes(ctx, rows, n_ctx - 1)
                if rows == 1:
                    t1 = ms
                if rows == 2:
                    base = ms
                print(json.dumps({"sweep": "batched variations", "weights": wname, "kv": "bf16",
                                  "rows": rows, "variations": rows // 2, "ctx": n_ctx,
                                  "ms_per_frame": ms, "frames_per_s_per_row": 1000.0 / ms,
                                  "row_frames_per_s": rows * 1000.0 / ms,
                                  "algorithmic_bytes": fb, "achieved_gbs": fb / ms / 1e6,
                                  "cfg_scale": cfg,
                                  "t_rows_over_t1": ms / t1,
                                  "extra_row_cost_vs_1row": (ms / t1 - 1.0) / max(1, rows - 1),
                                  "extra_pair_cost_vs_2rows": (ms / base - 1.0) / max(1, rows // 2 - 1)
                                  if rows > 2 else 0.0}), flush=True)
                del xs
        m3.m3_destroy(ctx)
        torch.cuda.empty_cache()


def run_generate(args):
    """The GPU generation loop over a whole song on the full 8B: F frames from
    position 300 (a prompt's worth of N(0,1) KV), 2 rows (one CFG pair), the
    end token sampleable, feedback through the token and audio embeddings.
    Timed with CUDA events around one m3_generate call (graphs captured by
    an untimed run first), and against the same frames driven from the host
    one m3_decode_frame (+ m3_depth_decode) call at a time."""
    import torch
    from autoregressive_audio_token_b200 import m3
    import synth
    torch.cuda.set_device(0)
    F, P = args.generate, 300
    wdtype = m3.M3_W_INT8 if args.wdtype == "int8" else m3.M3_W_BF16
    s, ctx = build_model(torch, m3, synth, 0, wdtype, args.layers, depth=args.depth,
                         end_token=True)
    m3.m3_set_top_k(ctx, args.top_k)
    nc = synth.DEPTH.codebooks if args.depth else 0
    m3.m3_load_feedback(ctx, synth.embedding_slice(s, 0, device="cuda"),
                        synth.audio_embeddings(synth.DEPTH, s.hidden, 0, device="cuda")
                        if args.depth else None)
    prefill_kv(torch, m3, synth, s, ctx, ROWS, P + F + 1, 0, args.kv == "f16")
    x0 = synth.normal((ROWS, s.hidden), 0, "bench/x0", std=0.02, device="cuda")
    codes = torch.empty((F, ROWS, 1 + nc), dtype=torch.int32, device="cuda")
    stream = torch.cuda.current_stream()
    m3.m3_generate(ctx, [P] * ROWS, 1, 0, x0, CFG_SCALE, 1.0, F, codes)  # capture, warm
    torch.cuda.synchronize()
    clocks = ClockSampler(0, "/tmp/m3_clocks_gen.csv")
    clocks.start()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    rc, nf = m3.m3_generate(ctx, [P] * ROWS, 1, 0, x0, CFG_SCALE, 1.0, F, codes)
    e1.record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    m3.m3_sync_status(ctx)
    ms = e0.elapsed_time(e1)
    # frames the loop ran: all F, or up to the 16-frame read after the end
    ran = F if nf[0] >= F else min(F, 16 * ((nf[0] + 1 + 15) // 16))
    # the same frames driven from the host, one call per frame
    xs = torch.empty((ROWS, s.hidden), dtype=torch.bfloat16, device="cuda")
    c1 = torch.empty(ROWS, dtype=torch.int32, device="cuda")
    h1 = torch.empty((ROWS, s.hidden), dtype=torch.bfloat16, device="cuda")
    d1 = torch.empty((ROWS, max(nc, 1)), dtype=torch.int32, device="cuda")
    xs.copy_(x0)

    def host_frame(i):
        m3.m3_decode_frame(ctx, [P + i] * ROWS, 1, i, xs, CFG_SCALE, 1.0, c1, h1)
        if nc:
            m3.m3_depth_decode(ctx, h1, c1, 1, i, CFG_SCALE, 1.0, d1)

    for i in range(3):
        host_frame(i)
    torch.cuda.synchronize()
    e2, e3 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e2.record(stream)
    for i in range(ran):
        host_frame(i)
    e3.record(stream)
    torch.cuda.synchronize()
    m3.m3_sync_status(ctx)
    ms_host = e2.elapsed_time(e3)
    mean_ctx = P + (ran - 1) / 2.0
    fb = m3.m3_frame_bytes(ctx, ROWS, int(round(mean_ctx)))
    name = workload_name(args).replace("song1500", f"generate{F}-prompt{P}") + "-end"
    print(json.dumps({
        "metric": "AR frames/s per row, GPU generation loop (8B, 2 rows)",
        "value": 1000.0 * ran / ms, "unit": "frames/s", "n_gpus": 1, "higher_is_better": True,
        "ms_per_frame": ms / ran, "dtype": args.wdtype, "data": "synthetic",
        "config": {"workload": name, "frames": F, "prompt_positions": P, "rows": ROWS,
                   "cfg_scale": CFG_SCALE, "top_k": args.top_k, "depth_decoder": bool(nc),
                   "status": rc, "n_frames": nf, "frames_run": ran},
        "frame_bytes_mean_ctx": fb, "achieved_gbs": fb / (ms / ran) / 1e6,
        "host_driven": {"ms_per_frame": ms_host / ran, "frames_per_s": 1000.0 * ran / ms_host},
        "clocks": clk}))
    m3.m3_destroy(ctx)


DIT_CFG = 1.7


def dit_step_flops(s, T: int) -> float:
    """FLOPs of one denoising step (batch 2 x T tokens): every projection as
    2 M N K plus attention's Q K^T and P V (4 B T^2 W per block)."""
    M = 2 * T
    W, F, Cin = s.width, s.ffn, 2 * s.latent + s.cond
    per_block = 3 * W * W + W * W + 2 * F * W + F * W
    gemm = 2.0 * M * (Cin * W + s.n_layers * per_block + W * s.latent)
    attn = 4.0 * 2 * T * T * W * s.n_layers
    return gemm + attn


def run_dit(args):
    """The DiT chunk-denoise step on one GPU: the full-size DiT, one 200-frame
    chunk (689 latent frames), cond + uncond as one batch-2 forward, CFG 1.7.
    W untimed steps, then K steps in one m3_dit_denoise call between CUDA
    events; every step streams 4.8 GB of fp16 weights and 1378 tokens'
    activations (far beyond L2), so no flush is needed."""
    import torch
    from autoregressive_audio_token_b200 import dit as D
    import synth
    torch.cuda.set_device(0)
    import dataclasses
    s, T = synth.DIT, synth.DIT_CHUNK_T
    if args.layers != 36:  # fewer blocks only for profiling small cases
        s = dataclasses.replace(s, n_layers=args.layers)
    h = D.m3_dit_create(D.config_from_shape(s, T))
    for l in range(s.n_layers):  # generate on the GPU, load block by block
        D.m3_dit_load(h, {"layers": [synth.dit_layer_weights(s, 0, l, device="cuda")]},
                      first_layer=l, outer=False)
    w = synth.dit_weights(s, 0, device="cuda", layers=[])
    D.m3_dit_load(h, w)
    x, ctx, cond = synth.dit_inputs(s, T, 1, device="cuda")
    K, Wm = args.steps, max(args.warmup, 3)
    sig = [1.0 - i / K for i in range(K + 1)]
    xw = x.clone()
    D.m3_dit_denoise(h, xw, ctx, cond, [1.0 - i / Wm for i in range(Wm + 1)], DIT_CFG)
    torch.cuda.synchronize()
    D.m3_dit_sync_status(h)
    clocks = ClockSampler(0, "/tmp/m3_clocks_dit.csv")
    xt = x.clone()
    torch.cuda.synchronize()
    clocks.start()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    D.m3_dit_denoise(h, xt, ctx, cond, sig, DIT_CFG)
    e1.record()
    torch.cuda.synchronize()
    clk = clocks.stop()
    D.m3_dit_sync_status(h)
    ms = e0.elapsed_time(e1) / K
    # end to end: inputs from pinned host memory and the latent back, per step
    xh, ch, dh = x.cpu().pin_memory(), ctx.cpu().pin_memory(), cond.cpu().pin_memory()
    xo = torch.empty_like(xh).pin_memory()
    xd, cd, dd = torch.empty_like(x), torch.empty_like(ctx), torch.empty_like(cond)
    e2, e3 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e2.record()
    for i in range(K):
        xd.copy_(xh, non_blocking=True)
        cd.copy_(ch, non_blocking=True)
        dd.copy_(dh, non_blocking=True)
        D.m3_dit_step(h, xd, cd, dd, sig[i], sig[i + 1], DIT_CFG)
        xo.copy_(xd, non_blocking=True)
    e3.record()
    torch.cuda.synchronize()
    D.m3_dit_sync_status(h)
    e2e_ms = e2.elapsed_time(e3) / K
    kernels = {}
    for which, name in [(2, "gate_up_glu"), (3, "down"), (0, "qkv_rope"), (1, "o_proj")]:
        kms, kfl = D.m3_dit_time_gemm(h, which, T, max(36, s.n_layers))
        kernels[name] = {"ms": kms, "flops": kfl, "tflops": kfl / kms / 1e9}
    D.m3_dit_destroy(h)
    peaks = {}
    try:
        peaks = json.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json")))
    except Exception:
        pass
    # a kernel timed alone takes the burst peak; fp16 and bf16 share the rate
    peak = peaks.get("bf16_tflops", 1590.0)
    flops = dit_step_flops(s, T)
    dom = kernels["gate_up_glu"]
    out = {
        "metric": "DiT chunk-denoise steps/s (36 blocks, 2 x 689 tokens, fp16)",
        "value": 1000.0 / ms, "unit": "steps/s", "n_gpus": 1, "steps": K, "warmup": Wm,
        "ms_per_step": ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f16", "data": "synthetic (seeded N(0,0.02^2) fp16 weights, N(0,1) latents and "
                                "condition)",
        "config": {"workload": f"dit-{s.n_layers}L-2048-ffn8192-chunk200-T689-batch2-cfg1.7",
                   "tokens": 2 * T, "cfg_scale": DIT_CFG,
                   "l2": "no flush: 4.8 GB of weights per step >> 126 MB L2"},
        "achieved_tflops": flops / ms / 1e9, "flops_per_step": flops,
        "roofline": {"bound": "tensor", "kernel": "dit_gemm_kernel gate/up + GLU (f16)",
                     "achieved": dom["tflops"], "peak": peak, "unit": "TFLOP/s",
                     "frac": dom["tflops"] / peak,
                     "peak_source": "measured" if "bf16_tflops" in peaks else "fallback",
                     "traffic": None, "flops_per_launch": dom["flops"]},
        "kernels": kernels,
        "e2e": {"value": 1000.0 / e2e_ms, "unit": "steps/s",
                "h2d_bytes_per_step": x.numel() * 4 + ctx.numel() * 2 + cond.numel() * 2,
                "d2h_bytes_per_step": x.numel() * 4},
        "gpu_launches": (1 + 3 + 1 + 7 * s.n_layers + 2 + 1) * K,
        "clocks": clk,
    }
    print(json.dumps(out))


def run_depth_only(args):
    """The RVQ depth decoder alone (int8 weights, one scale per group of 128):
    m3_depth_decode on a fixed final hidden state and semantic code, --rows
    rows (2 = one CFG pair, the workload), timed with CUDA events over
    --steps calls after --warmup. The body is a single layer, loaded only
    because the context needs one."""
    import torch
    from autoregressive_audio_token_b200 import m3
    import synth
    torch.cuda.set_device(0)
    rows = args.rows
    s, ctx = build_model(torch, m3, synth, 0, m3.M3_W_INT8, 1, depth=True, max_rows=max(2, rows))
    h = synth.normal((rows, s.hidden), 0, "bench/depth_h", std=1.0, device="cuda")
    code0 = torch.tensor([5 + 7 * (r // 2) for r in range(rows)], dtype=torch.int32, device="cuda")
    dcodes = torch.empty((rows, synth.DEPTH.codebooks), dtype=torch.int32, device="cuda")
    for i in range(max(args.warmup, 3)):
        m3.m3_depth_decode(ctx, h, code0, 1, i, CFG_SCALE, 1.0, dcodes)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for i in range(args.steps):
        m3.m3_depth_decode(ctx, h, code0, 1, i, CFG_SCALE, 1.0, dcodes)
    e1.record()
    torch.cuda.synchronize()
    m3.m3_sync_status(ctx)
    ms = e0.elapsed_time(e1) / args.steps
    D = synth.DEPTH
    wbytes = (D.n_layers * (4 * D.hidden * D.n_heads * D.head_dim + 3 * D.hidden * D.ffn) *
              (D.codebooks + 1) + D.hidden * D.in_hidden + D.codebooks * D.vocab * D.hidden)
    print(json.dumps({"metric": f"depth decoder calls/s (7 residual codes, {rows} rows)",
                      "value": 1000.0 / ms, "unit": "calls/s", "ms_per_call": ms,
                      "steps": args.steps, "dtype": "int8 g128",
                      "kernels_per_call": m3.m3_depth_kernels(ctx, rows),
                      "weight_bytes_per_call": wbytes, "achieved_gbs": wbytes / ms / 1e6,
                      "config": {"workload": f"depth-decoder-4L-1024-int8g128-{rows}rows-cfg1.5"}}))
    m3.m3_destroy(ctx)


def run_prefill(args):
    """Prompt prefill of P tokens (a prompt's worth, N(0, 0.02^2) embeddings)
    into one cache row of the full 8B: chunks of M3_PREFILL_CHUNK tokens
    (2048 for bf16, 256 for int8) through the tcgen05 GEMMs (the default for
    bf16 weights, M3_PREFILL_TC=1 for int8), or chunks of 16 through the
    decode GEMVs (the default for int8, M3_PREFILL_TC=0 for bf16); timed with
    CUDA events over 3 runs after one untimed run."""
    import torch
    from autoregressive_audio_token_b200 import m3
    import synth
    torch.cuda.set_device(0)
    P = args.prefill
    wdtype = m3.M3_W_INT8 if args.wdtype == "int8" else m3.M3_W_BF16
    s, ctx = build_model(torch, m3, synth, 0, wdtype, args.layers, max_rows=16)
    m3.m3_kv_alloc(ctx, 2, P + 1, m3.M3_KV_F16 if args.kv == "f16" else m3.M3_KV_BF16, 256)
    x = synth.normal((P, s.hidden), 0, "bench/prompt", std=0.02, device="cuda")
    h = torch.empty(s.hidden, dtype=torch.bfloat16, device="cuda")
    m3.m3_prefill(ctx, 0, 0, x, h)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(3):
        m3.m3_prefill(ctx, 1, 0, x, h)
    e1.record()
    torch.cuda.synchronize()
    m3.m3_sync_status(ctx)
    ms = e0.elapsed_time(e1) / 3
    tc = os.environ.get("M3_PREFILL_TC", "1" if args.wdtype == "bf16" else "0") == "1"
    chunk = (int(os.environ.get("M3_PREFILL_CHUNK", "2048" if args.wdtype == "bf16" else "256"))
             if tc else 16)
    path = "tcgen05 GEMM" if tc else "decode GEMV"
    layer_w = m3.m3_frame_bytes(ctx, 0, -1)  # weights only (no KV)
    flops = 2.0 * P * (layer_w / (1 if wdtype == m3.M3_W_INT8 else 2))
    print(json.dumps({"metric": "prompt prefill tokens/s (8B, one row)", "value": 1000.0 * P / ms,
                      "unit": "tokens/s", "ms": ms, "tokens": P, "chunk": chunk, "path": path,
                      "dtype": args.wdtype, "approx_tflops": flops / ms / 1e9,
                      "config": {"workload": f"qwen3-8b-{args.layers}L-{args.wdtype}-prefill{P}"}}))
    m3.m3_destroy(ctx)


def main():
    args = parse()
    rank, world, local = dist_env()
    if args.prefill:
        if rank == 0:
            run_prefill(args)
        return
    if args.depth_only:
        if rank == 0:
            run_depth_only(args)
        return
    if args.dit:
        if rank == 0:
            run_dit(args)
        return
    if args.generate:
        if rank == 0:
            run_generate(args)
        return
    if args.sweep:
        if rank == 0:
            run_sweep(args)
        return
    if args.impl == "reference":
        out = run_reference(args, rank, world)
    else:
        out = run_ours(args, rank, world, local)
    if rank == 0 and out is not None:
        print(json.dumps(out))


if __name__ == "__main__":
    main()
