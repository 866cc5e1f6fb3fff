"""Benchmark of the frame-wise GDN frame scan on B200.

python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                [--config NAME] [--plan auto|chunked|sequential|separate]
                [--e2e-steps K2] [--no-cpu-baseline]

One step = one full pass of the scan (contraction, the chains of the
recurrence, readout) over one batch of the workload, inputs resident in HBM.
The default workload is the 60 s 720p rollout, one GDN layer: B=1, H=16,
D=128, S=80x45=3600 tokens per latent frame, T=121 latent frames, bf16 q/k/v,
fp32 state. The default plan is the library's own choice (for this workload:
the sequential chains running alongside the contraction in one launch);
--plan chunked times the span-composed scan (8-frame spans), --plan separate
the sequential chains as their own launch.

Metric: frame·head·tokens/s = B*H*T*S / step time, and the fraction of the
HBM roofline. Under torchrun (N>1) every rank runs its own copy of the
workload on its own GPU (the heads shard with no data-path collective: weak
scaling); NCCL carries only the barrier and the max-over-ranks timing.

--impl reference times the float64 CPU oracle (the reference implementation
of this build) on a bounded sample of the same workload, on rank 0 only.
"""

from __future__ import annotations

import argparse
import dataclasses
import hashlib
import glob
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from frame_wise_gated_b200 import synth  # noqa: E402

METRIC = "GDN frame-scan frame·head·tokens/s (% of HBM roofline), 1xB200"
UNIT = "frame·head·tokens/s"
METRIC_BWD = "GDN frame-scan BACKWARD frame·head·tokens/s (% of HBM roofline), 1xB200"
METRIC_TRAIN = ("GDN frame-scan TRAINING STEP (forward + backward from saved forward) "
                "frame·head·tokens/s (% of HBM roofline), 1xB200")
FALLBACK_HBM_GBS = 6650.0
# nominal HBM3e peak of a B200 (about 8 TB/s); its fraction is reported beside
# the fraction of the measured copy bandwidth
NOMINAL_HBM_GBS = 8000.0
L2_BYTES = 126 << 20
FALLBACK_BF16_TFLOPS = 1590.0


def env_int(name, default):
    try:
        return int(os.environ.get(name, default))
    except ValueError:
        return default


def algorithmic_bytes(cfg, step=True):
    """Bytes the method must move per step: q, k, v in and o out (raw q, k
    plus two outputs for the bidirectional prologue workload), beta and gamma,
    and the per-head state in/out."""
    e = 2 if cfg.bf16 else 4
    n_t = 5 if cfg.prologue else 4
    per_fh = cfg.S * (n_t * cfg.D * e + 4) + 4
    state = 2 * cfg.D * cfg.D * 4
    camera = 2 * cfg.B * cfg.T * cfg.S * 64 if cfg.ucpe else 0  # 4x4 fp32 for q and k per token
    return cfg.frame_heads * per_fh + cfg.B * cfg.H * state + camera


def backward_bytes(cfg):
    """Bytes the backward must move per step: q, k, v and dL/dO in, dq, dk, dv
    out, beta in and dbeta out, gamma in and dgamma out, the state and its
    gradients (state_in, dL/d(state_out) in; dL/d(state_in) out)."""
    e = 2 if cfg.bf16 else 4
    per_fh = cfg.S * (7 * cfg.D * e + 8) + 8
    return cfg.frame_heads * per_fh + cfg.B * cfg.H * 3 * cfg.D * cfg.D * 4


def phase_bytes(cfg):
    """Algorithmic bytes per launch of each kernel phase (per frame-head
    figure x frame-heads)."""
    e = 2 if cfg.bf16 else 4
    fh = cfg.frame_heads
    nro = 2 if cfg.bidir_block else 1
    return {
        "contract": fh * cfg.S * (2 * cfg.D * e + 4),          # K, V, beta
        "contract_scan": fh * cfg.S * (2 * cfg.D * e + 4),     # same, chains alongside
        "readout": fh * cfg.S * (2 + (1 if cfg.bidir_block else 0)) * cfg.D * e,  # Q in, O (and O_rev) out
        "scan_readout": fh * cfg.S * 2 * cfg.D * e,             # Q in, O out (replay fused)
        "prologue": fh * cfg.S * 4 * cfg.D * e,                 # raw q, k in; q^, k^ out
        "_readout_launches_per_step": nro,
    }


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d.get("hbm_gbs", FALLBACK_HBM_GBS), d.get("bf16_tflops", FALLBACK_BF16_TFLOPS), "measured"
    return FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS, "fallback"


def csrc_digest():
    h = hashlib.sha256()
    for f in sorted(glob.glob(os.path.join(ROOT, "frame_wise_gated_b200", "csrc", "*"))):
        h.update(open(f, "rb").read())
    return h.hexdigest()[:16]


def ncu_traffic(kernel_phase, cfg_name):
    """DRAM bytes per launch from the committed ncu summary, if it was taken
    on the current kernel sources and this workload; else None."""
    p = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    if not os.path.exists(p):
        return None
    try:
        d = json.load(open(p))
    except ValueError:
        return None
    ent = d.get(kernel_phase)
    if not ent or ent.get("csrc_sha") != csrc_digest() or ent.get("workload") != cfg_name:
        return None
    return ent.get("dram_bytes_per_launch")


class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 7:
                continue
            try:
                sm.append(float(parts[0]))
                smax.append(float(parts[1]))
            except ValueError:
                continue
            for n, v in zip(names, parts[3:7]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax),
                "reasons": sorted(reasons), "samples": len(sm)}


def cpu_oracle_budget(cfg, seconds=10.0):
    """Times the oracle on whole (b, h) slabs of the workload until about
    `seconds` of CPU work (at least one slab, at most all of them)."""
    tot_t, tot_tok, n = 0.0, 0, 0
    for bh in range(cfg.B * cfg.H):
        _, dt, toks, _ = cpu_oracle_sample(cfg, slab=divmod(bh, cfg.H))
        tot_t += dt
        tot_tok += toks
        n += 1
        if tot_t >= seconds:
            break
    return tot_tok / tot_t, tot_t, f"{n} of {cfg.B * cfg.H} (b,h) slabs x {cfg.T} frames x {cfg.S} tokens"


def cpu_oracle_sample(cfg, frames=None, slab=(0, 0)):
    """Times the float64 oracle on one (b, h) slab (first `frames` frames).
    Returns (tokens per second, seconds, tokens, description)."""
    from oracle import gdn_oracle as O
    b, h = slab
    sl = synth.make_slab(cfg, b, h)
    T = cfg.T if frames is None else min(frames, cfg.T)
    wid = (lambda x: synth.bf16_bits_to_f32(x[:T]).astype(np.float64)) if cfg.bf16 else \
        (lambda x: x[:T].astype(np.float64))
    q, k, v = wid(sl["q"]), wid(sl["k"]), wid(sl["v"])
    beta = sl["beta"][:T].astype(np.float64)
    gamma = sl["gamma"][:T].astype(np.float64)
    st = synth.make_state(cfg)
    s0 = None if st is None else st[b, h]
    cam = None
    if cfg.ucpe:
        mq, mk = synth.make_camera(cfg.B, cfg.T, cfg.grid_h, cfg.grid_w, cfg.seed)
        cam = (mq[b, :T], mk[b, :T])
    t0 = time.perf_counter()
    if cfg.prologue:
        wq, wk = synth.make_weights(cfg)
        qh, kh = O.qk_prologue(q, k, wq, wk, cfg.grid_w, ucpe=cam)
        O.frame_scan(qh, kh, v, beta, gamma, s0, keys_scaled=True)
        O.frame_scan(qh, kh, v, beta, gamma, s0, reverse=True, block=cfg.bidir_block,
                     keys_scaled=True)
    else:
        O.frame_scan(q, k, v, beta, gamma, s0)
    dt = time.perf_counter() - t0
    toks = T * cfg.S
    return toks / dt, dt, toks, f"one (b,h) slab, {T} of {cfg.T} frames x {cfg.S} tokens"


def host_cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def run_reference(args, cfg):
    rank = env_int("RANK", 0)
    if rank != 0:
        return 0
    frames = max(1, min(cfg.T, args.ref_frames))
    times = []
    for i in range(args.warmup + args.steps):
        _, dt, toks, desc = cpu_oracle_sample(cfg, frames=frames, slab=(0, i % cfg.H))
        if i >= args.warmup:
            times.append(dt)
    tot = sum(times)
    value = toks * len(times) / tot
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * tot / len(times), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": cfg.name, "B": cfg.B, "H": cfg.H, "T": cfg.T, "S": cfg.S,
                   "D": cfg.D, "sample_per_step": desc},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": host_cores(), "kind": "oracle",
                         "sample": f"{desc} per step; float64 NumPy oracle as it stands"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def reduce_step_time(ms, dist=None, device=None):
    """Max over ranks of a per-rank elapsed time (ms); identity on one rank."""
    if dist is None or not dist.is_initialized() or dist.get_world_size() == 1:
        return float(ms)
    import torch
    t = torch.tensor([float(ms)], dtype=torch.float64,
                     device=device if device is not None else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_value(tokens_per_rank, world, ms_per_step):
    """Whole-job throughput: the units all ranks processed / the slowest rank's time."""
    return tokens_per_rank * world / (ms_per_step * 1e-3)


PLANS = {
    "auto": {},
    "chunked": {"chunked": True},
    "sequential": {"sequential": True},
    "separate": {"sequential": True, "overlap": False},
}


def plan_kw(plan):
    return dict(PLANS[plan])


def plan_desc(plan, phases):
    """What ran: read from the phases the library recorded."""
    ran = {p for p in phases if phases[p][1] > 0}
    if "contract_scan" in ran:
        how = "sequential chains alongside the contraction (one cooperative launch)"
    elif "compose" in ran:
        how = "chunked (8-frame spans, composed)"
    elif "scan_readout" in ran:
        how = "spans replayed inside the readout"
    else:
        how = "sequential chains (own launch)"
    return f"{how}; plan {plan}"


def run_ours(args, cfg):
    import torch
    from frame_wise_gated_b200 import api, build

    world = env_int("WORLD_SIZE", 1)
    rank = env_int("RANK", 0)
    local = env_int("LOCAL_RANK", 0)
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)
    build.build()
    api.lib()

    # ---- inputs (seeded, synthetic), resident in HBM ----
    arr = synth.make_inputs(cfg)
    et = torch.bfloat16 if cfg.bf16 else torch.float32

    def dev_t(x):
        t = torch.from_numpy(x)
        if cfg.bf16 and x.dtype == np.uint16:
            t = t.view(torch.bfloat16)
        return t.to(dev)

    q, k, v = dev_t(arr["q"]), dev_t(arr["k"]), dev_t(arr["v"])
    beta = torch.from_numpy(arr["beta"]).to(dev)
    gamma = torch.from_numpy(arr["gamma"]).to(dev)
    s0 = None if arr["state"] is None else torch.from_numpy(arr["state"]).to(dev)
    pro = None
    if cfg.prologue:
        pro = dict(w_q=torch.from_numpy(arr["w_q"]).to(dev), w_k=torch.from_numpy(arr["w_k"]).to(dev),
                   grid_h=cfg.grid_h, grid_w=cfg.grid_w)
        if cfg.ucpe:
            mq, mk = synth.make_camera(cfg.B, cfg.T, cfg.grid_h, cfg.grid_w, cfg.seed)
            pro["ucpe_q"], pro["ucpe_k"] = torch.from_numpy(mq).to(dev), torch.from_numpy(mk).to(dev)
    kw = dict(prologue=pro, bidir=bool(cfg.bidir_block), block_reset=bool(cfg.bidir_block),
              block=cfg.bidir_block or 3, fused_replay=args.fused_replay, **plan_kw(args.plan))
    if cfg.bidir_block and cfg.T == cfg.bidir_block:
        kw["state_in_rev"] = None  # streaming step: the reverse scan stays inside the block
    out = torch.empty_like(q)
    out_rev = torch.empty_like(q) if cfg.bidir_block else None
    st_out = torch.empty((cfg.B, cfg.H, cfg.D, cfg.D), device=dev, dtype=torch.float32)
    st_rev = torch.empty_like(st_out) if cfg.bidir_block else None
    flags = (api.UCPE if cfg.ucpe else 0) | api.scan_flags(
        bf16=cfg.bf16, prologue=pro is not None, bidir=bool(cfg.bidir_block),
                           block_reset=bool(cfg.bidir_block), block=cfg.bidir_block or 3,
                           fused_replay=args.fused_replay, **plan_kw(args.plan))
    ws = torch.empty(api.workspace_bytes(cfg.B, cfg.H, cfg.T, cfg.S, cfg.D, flags),
                     device=dev, dtype=torch.uint8)
    stream = torch.cuda.current_stream(dev)

    def step():
        api.frame_scan_fwd_ex(q, k, v, beta, gamma, s0, out=out, state_out=st_out,
                              out_rev=out_rev, state_out_rev=st_rev, workspace=ws, **kw)

    if args.bwd:
        # the backward pass: upstream gradients dL/dO and dL/d(state_out), seeded
        if cfg.prologue:
            raise SystemExit("--bwd: the backward covers the scan without the prologue")
        g = torch.Generator(device="cpu").manual_seed(7)
        d_out = torch.randn(q.shape, generator=g).to(dtype=q.dtype, device=dev)
        d_st = torch.randn((cfg.B, cfg.H, cfg.D, cfg.D), generator=g).to(dev)
        flags_b = api.scan_flags(bf16=cfg.bf16)
        ws_b = torch.empty(int(api.lib().gdn_bwd_workspace_bytes(cfg.B, cfg.H, cfg.T, cfg.S, cfg.D,
                                                                 flags_b)),
                           device=dev, dtype=torch.uint8)

        if args.train:
            def step():  # noqa: F811
                # forward, then the backward from the forward's saved workspace
                api.frame_scan_fwd_ex(q, k, v, beta, gamma, s0, out=out, state_out=st_out,
                                      workspace=ws, save_for_backward=True, **kw)
                api.frame_scan_bwd(q, k, v, beta, gamma, s0, d_out, d_st, workspace=ws_b,
                                   saved_workspace=ws)
        else:
            def step():  # noqa: F811
                api.frame_scan_bwd(q, k, v, beta, gamma, s0, d_out, d_st, workspace=ws_b)

    def barrier():
        if dist is not None:
            dist.barrier()

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    api.check_device_status()

    # ---- timed region: K steps, CUDA events on the launch stream ----
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    api.launch_count(reset=True)
    api.profile_enable(True)
    barrier()
    torch.cuda.synchronize(dev)
    step_bytes0 = algorithmic_bytes(cfg) if not args.bwd else backward_bytes(cfg)
    flush = None
    if step_bytes0 < 2 * L2_BYTES:
        # a step this small would find its inputs in L2: flush it before every
        # step and time the steps alone (one event pair each)
        flush = torch.empty(2 * L2_BYTES, dtype=torch.uint8, device=dev)
    if flush is None:
        ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ev0.record(stream)
        for _ in range(args.steps):
            step()
        ev1.record(stream)
        torch.cuda.synchronize(dev)
        elapsed = ev0.elapsed_time(ev1)
    else:
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(args.steps)]
        for e0, e1 in evs:
            flush.zero_()
            e0.record(stream)
            step()
            e1.record(stream)
        torch.cuda.synchronize(dev)
        elapsed = sum(e0.elapsed_time(e1) for e0, e1 in evs)
    barrier()
    launches = api.launch_count(reset=True)
    phases = api.profile_read()
    api.profile_enable(False)
    clk = clocks.stop()
    api.check_device_status()
    ms = reduce_step_time(elapsed, dist, dev)
    ms_step = ms / args.steps
    value = whole_job_value(cfg.tokens, world, ms_step)

    # ---- dominant kernel roofline (live per-kernel events over the timed region) ----
    hbm, bf16_tf, peak_kind = peaks()
    pb = phase_bytes(cfg)
    roof = None
    timed = [p for p in phases if phases[p][1] > 0]
    dom_all = max(timed, key=lambda p: phases[p][0]) if timed else None
    cand = [p for p in timed if p in pb]
    alg = None
    if cand:
        dom = max(cand, key=lambda p: phases[p][0])
        dom_ms = phases[dom][0] / phases[dom][1]
        alg = pb.get(dom)
    if alg is not None and not args.bwd:
        ach = alg / (dom_ms * 1e-3) / 1e9
        traffic = ncu_traffic(dom, cfg.name)
        roof = {"kernel": dom, "bound": "hbm", "achieved": ach, "peak": hbm, "unit": "GB/s",
                "frac": ach / hbm, "traffic": traffic, "peak_source": peak_kind,
                "frac_of_nominal_8tbs": ach / NOMINAL_HBM_GBS,
                "alg_bytes_per_launch": alg, "ms_per_launch": dom_ms,
                "dominant_kernel_overall": dom_all}
    step_bytes = algorithmic_bytes(cfg) if not args.bwd else backward_bytes(cfg)
    if args.bwd and args.train:
        step_bytes += algorithmic_bytes(cfg)
    if args.bwd:
        ach = step_bytes / (ms_step * 1e-3) / 1e9
        roof = {"kernel": "backward step (all kernels)", "bound": "hbm", "achieved": ach,
                "peak": hbm, "unit": "GB/s", "frac": ach / hbm, "traffic": None,
                "peak_source": peak_kind, "alg_bytes_per_launch": step_bytes,
                "ms_per_launch": ms_step}
    step_gbs = step_bytes / (ms_step * 1e-3) / 1e9
    step_roof = {"alg_bytes_per_step": step_bytes, "achieved_gbs": step_gbs,
                 "frac": step_gbs / hbm, "frac_of_nominal_8tbs": step_gbs / NOMINAL_HBM_GBS}

    # ---- end to end through the C ABI with host buffers ----
    e2e = None
    if args.e2e_steps > 0 and not args.bwd:
        e2e = run_e2e(args, cfg, arr, dev, api, barrier, dist, world)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline and not args.bwd:
        val, dt, desc = cpu_oracle_budget(cfg, seconds=args.cpu_seconds)
        cpu = {"value": val, "unit": UNIT, "cores": host_cores(), "kind": "oracle",
               "sample": f"{desc}; {dt:.1f} s of float64 NumPy oracle (BLAS threads = all cores)"}

    if rank == 0:
        line = {
            "metric": METRIC if not args.bwd else (METRIC_TRAIN if args.train else METRIC_BWD),
            "value": value, "unit": UNIT,
            "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16" if cfg.bf16 else "f32", "data": "synthetic",
            "config": {"workload": cfg.name, "B": cfg.B, "H": cfg.H, "T": cfg.T, "S": cfg.S,
                       "D": cfg.D, "grid": f"{cfg.grid_w}x{cfg.grid_h}",
                       "scan": plan_desc(args.plan, phases) if not args.bwd else
                       ("forward, then backward from its saved workspace" if args.train else
                        "backward: recompute, adjoint chain, per-frame and per-token gradients"),
                       "prologue": cfg.prologue, "bidir_block": cfg.bidir_block,
                       "camera_encoding": cfg.ucpe,
                       "l2": (f"inputs larger than L2 ({step_bytes / 1e9:.2f} GB algorithmic per step)"
                              if flush is None else
                              f"L2 flushed before every step ({2 * L2_BYTES >> 20} MiB written); "
                              f"{step_bytes / 1e6:.0f} MB algorithmic per step"),
                       "parallelism": f"replica x{world} (heads shard, no collective)"},
            "roofline": roof, "step_roofline": step_roof,
            "phases_ms_per_step": {p: phases[p][0] / args.steps for p in phases if phases[p][1]},
            "gpu_launches": launches, "clocks": clk, "e2e": e2e, "cpu_baseline": cpu,
        }
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def run_e2e(args, cfg, arr, dev, api, barrier, dist, world):
    """Same metric through the C-ABI host-buffer call gdn_frame_scan_fwd_host
    (heads in chunks, copies in and out overlapping the scans on three
    streams inside the library) with inputs and outputs in pinned host
    memory: every step copies all inputs to the device and all outputs back,
    inside the timed region."""
    import torch
    if cfg.prologue:
        return None  # the host-streaming call takes prepared q, k (no fused prologue)

    def pinned(x):
        t = torch.from_numpy(x)
        if cfg.bf16 and x.dtype == np.uint16:
            t = t.view(torch.bfloat16)
        return t.pin_memory()

    hq, hk, hv = pinned(arr["q"]), pinned(arr["k"]), pinned(arr["v"])
    hb, hg = pinned(arr["beta"]), pinned(arr["gamma"])
    hs0 = None if arr["state"] is None else pinned(arr["state"])
    hout = torch.empty(hq.shape, dtype=hq.dtype).pin_memory()
    hst = torch.empty((cfg.B, cfg.H, cfg.D, cfg.D), dtype=torch.float32).pin_memory()
    h2d = sum(x.numel() * x.element_size() for x in (hq, hk, hv, hb, hg) + ((hs0,) if hs0 is not None else ()))
    d2h = hout.numel() * hout.element_size() + hst.numel() * 4
    hpc = max(1, (cfg.B * cfg.H) // max(1, args.e2e_chunks))

    def step():
        api.frame_scan_fwd_host(hq, hk, hv, hb, hg, hs0, out=hout, state_out=hst,
                                heads_per_chunk=hpc, device=dev, **plan_kw(args.plan))

    step()
    torch.cuda.synchronize(dev)
    stream = torch.cuda.current_stream(dev)
    barrier()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev0.record(stream)
    for _ in range(args.e2e_steps):
        step()
    ev1.record(stream)
    torch.cuda.synchronize(dev)
    barrier()
    ms = reduce_step_time(ev0.elapsed_time(ev1), dist, dev)
    ms_step = ms / args.e2e_steps
    return {"value": whole_job_value(cfg.tokens, world, ms_step), "unit": UNIT,
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": ms_step,
            "steps": args.e2e_steps,
            "entry": f"gdn_frame_scan_fwd_host (pinned host buffers, {hpc} heads per chunk, "
                     "copies overlapping the scans inside the library)"}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--config", default="rollout60s_720p", choices=sorted(synth.CONFIGS))
    ap.add_argument("--plan", choices=sorted(PLANS), default="auto",
                    help="scan plan: the library's choice, spans, or sequential chains "
                         "(alongside the contraction, or as their own launch)")
    ap.add_argument("--fused-replay", action="store_true",
                    help="replay spans inside the readout kernel")
    ap.add_argument("--bwd", action="store_true",
                    help="time the backward pass (gdn_frame_scan_bwd) instead of the forward")
    ap.add_argument("--train", action="store_true",
                    help="with --bwd: time forward + backward from the forward's saved workspace")
    ap.add_argument("--e2e-steps", type=int, default=5)
    ap.add_argument("--e2e-chunks", type=int, default=8,
                    help="head chunks of the end-to-end host-streaming call (copies of one "
                         "chunk overlap the scan of the next)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--ref-frames", type=int, default=6,
                    help="frames of one slab per reference step")
    ap.add_argument("--cpu-seconds", type=float, default=10.0,
                    help="CPU work budget of the cpu_baseline sample")
    ap.add_argument("--frames", type=int, default=0,
                    help="override the workload's number of latent frames T (a smaller "
                         "case of the same shape, e.g. for profiler captures)")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    cfg = synth.CONFIGS[args.config]
    if args.frames > 0:
        cfg = dataclasses.replace(cfg, name=f"{cfg.name}_T{args.frames}", T=args.frames)
    if args.impl == "reference":
        return run_reference(args, cfg)
    return run_ours(args, cfg)


if __name__ == "__main__":
    sys.exit(main())
