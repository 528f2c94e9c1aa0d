#!/usr/bin/env python
"""Benchmark: video tokens/s of one VDN hybrid attention forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--config 768p_bf16]

A step is one whole forward (VDA state path, window+anchor Softmax, linear
readout, gated dual projection) over the 768p-shaped workload (B=1, H=24,
T=75 latent frames, N=1536 tokens/frame, d=128, 512 text tokens, bf16 inputs,
FP32 state and output), with every input resident in HBM.  The inputs (q, k,
v and the gates: 3.5 GB) are larger than L2 (126 MB), so no flush is needed
between steps.  Timing: W untimed steps, then K steps between a barrier +
synchronize on both sides, CUDA events on the launching stream, max over
ranks.  Under torchrun each rank runs its own replica of the workload
(independent problems, no collective on the data path: weak scaling).

``--impl reference`` times the CPU oracle (float64 NumPy, the correctness
reference of this repo) on the host cores, each step a fixed sample of query
rows of the same workload.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "video tokens/s per VDN hybrid-attn fwd on 1×B200; % of roofline"
UNIT = "video tokens/s"


# ----------------------------------------------------------------------------
# work model (FLOPs and minimum bytes of one forward)
# ----------------------------------------------------------------------------

def visible_frames(t, T, C, R):
    if t in (0, T - 1):
        return T
    c = t // C
    lo, hi = max(0, (c - R) * C), min(T, (c + R + 1) * C)
    return len(set(range(lo, hi)) | {0, T - 1})


def work_model(cfg, out_bytes=4, text_keys=False):
    B, H, T, N, d, C, R = cfg.B, cfg.H, cfg.T, cfg.N, cfg.d, cfg.chunk, cfg.window_radius
    L, D = T * N, H * d
    frame_pairs = sum(visible_frames(t, T, C, R) for t in range(T))
    pairs = B * H * N * N * frame_pairs              # masked (query, key) pairs
    if text_keys:
        pairs += B * H * L * cfg.n_text              # every video query x every text key
    f_soft = 4.0 * d * pairs                          # QK^T and PV
    f_proj = 2.0 * B * L * (2 * D) * D                # [g_s o_s | g_l RMS(o_l)] [W_s; W_l]
    n_fh = B * H * (T + 1)                            # frame-heads incl. the text frame
    f_vda = n_fh * (4.0 * N * d * d + (1.0 / 3 + 4.0) * d ** 3) + B * H * L * 4.0 * d * d
    bytes_min = (5 * B * L * D * 2                    # q, k, v, g_s, g_l (bf16)
                 + B * L * D * out_bytes              # out
                 + 2 * D * D * 2                      # W_soft, W_lin
                 + 2 * B * cfg.n_text * D * 2 + B * H * (T + 1) * 4)
    return dict(pairs=pairs, frame_pairs=frame_pairs, f_soft=f_soft, f_proj=f_proj,
                f_vda=f_vda, f_total=f_soft + f_proj + f_vda, bytes_min=bytes_min)


# DRAM bytes (read + write) of one attn_tc_kernel launch, from an ncu capture
# (dram__bytes_read.sum + dram__bytes_write.sum) of the 4-head copy of the
# 768p workload: 987.6 MB + 113.5 MB, scaled by the head count (the launch is
# one independent problem per head).  None for any other workload.
ATTN_TRAFFIC_PER_HEAD = (987.616256e6 + 113.466368e6) / 4
ATTN_TRAFFIC_SHAPES = {(75, 1536, 128)}


# B200 datasheet figures (dense bf16 tensor throughput, HBM3e bandwidth):
# context for the fractions, which are also given against the measured peaks.
DATASHEET_BF16_TFLOPS = 2250.0
DATASHEET_HBM_GBS = 7700.0


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        pk = json.load(open(path))
        return dict(hbm=pk["hbm_gbs"], tc=pk["bf16_tflops"],
                    tc_sust=pk.get("bf16_tflops_sustained", pk["bf16_tflops"]), src="measured")
    return dict(hbm=6650.0, tc=1590.0, tc_sust=1400.0, src="fallback")


# ----------------------------------------------------------------------------
# clocks during the timed region
# ----------------------------------------------------------------------------

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.file = None

    def start(self):
        try:
            self.file = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=self.file, stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.file.flush()
        rows = []
        with open(self.file.name) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.file.name)
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons,
                "samples": len(rows)}


# ----------------------------------------------------------------------------
# CPU oracle timing (the reported baseline / the reference arm)
# ----------------------------------------------------------------------------

def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return max(n)
    except Exception:
        pass
    return os.cpu_count()


def oracle_sample(cfg, inp):
    """A fixed, bounded sample of the workload for the CPU oracle (about 10 s
    on 16 host cores at 768p): 4 query tokens of the anchor frame 0 and 4 of
    each of seven frames in different chunks (7, 12, 27, 37, 52, 62, 72), with
    all heads, including the frame-by-frame VDA recurrence each chunk needs."""
    import numpy as np
    frames = sorted({0} | {min(cfg.T - 2, f) for f in (7, 12, 27, 37, 52, 62, 72)})
    pick = (0, cfg.N // 3, 2 * cfg.N // 3, cfg.N - 1)
    return np.array([t * cfg.N + n for t in frames for n in pick])


def sample_frames(cfg, rows):
    return sorted({int(r) // cfg.N for r in rows})


def time_oracle(cfg, inp, rows):
    from oracle import vdn_oracle as O
    t0 = time.perf_counter()
    O.hybrid_forward(inp, cfg.T, cfg.N, cfg.chunk, cfg.window_radius, rows=rows)
    return time.perf_counter() - t0


# ----------------------------------------------------------------------------
# arms
# ----------------------------------------------------------------------------

def base_line(args, cfg, value, ms_per_step, n_gpus):
    return {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": n_gpus, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": cfg.name, "B": cfg.B, "H": cfg.H, "T": cfg.T, "N": cfg.N,
                   "d": cfg.d, "n_text": cfg.n_text, "chunk": cfg.chunk,
                   "window_radius": cfg.window_radius, "video_tokens_per_step": cfg.B * cfg.L,
                   "inputs": "seeded synthetic (q,k L2-normalised, v N(0,1), beta sigmoid(N(0,1)), "
                             "gates 0.5, W N(0,1/d)); inputs > L2, no flush",
                   "out_dtype": "f32", "parallelism": f"replicas x{n_gpus}",
                   "decay_gate": "U[0.9,1]" if getattr(args, "alpha", False) else "none",
                   "text_keys_in_softmax": bool(getattr(args, "text_softmax", False)),
                   "write_gate": "per token" if getattr(args, "beta_per_token", False)
                                 else "per frame",
                   "projection": "MXFP8 (E4M3, 32-element UE8M0 blocks, FP32 accumulation)"
                                 if getattr(args, "proj_mxfp8", False) else "fp16 operands",
                   "frame_rule": "frozen-state (comparison)"
                                 if getattr(args, "frozen_state", False) else "VDA",
                   "linear_feature_map": "VDA-Prep in the step (3x3 spatial + 5-tap temporal "
                                         "conv, SiLU, L2; random filters)"
                                         if getattr(args, "prep", False) else "inputs prepared"},
    }


def run_reference(args, cfg):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    from synth import make_inputs
    inp = make_inputs(cfg)
    rows = oracle_sample(cfg, inp)
    for _ in range(args.warmup):
        time_oracle(cfg, inp, rows)
    times = [time_oracle(cfg, inp, rows) for _ in range(args.steps)]
    tot = sum(times)
    value = len(rows) * args.steps / tot
    line = base_line(args, cfg, value, 1e3 * tot / args.steps, int(os.environ.get("WORLD_SIZE", "1")))
    line["dtype"] = "f64"
    line["impl"] = "reference"
    sample = (f"{len(rows)} query tokens (frames {sample_frames(cfg, rows)}) with all {cfg.H} "
              "heads, plus the VDA recurrence of their chunks, per step")
    line["cpu_baseline"] = {"value": value, "unit": UNIT, "cores": blas_threads(),
                            "kind": "oracle", "sample": sample}
    line["e2e"] = {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
    print(json.dumps(line), flush=True)
    return 0


def ranks_max(x: float, dist, device) -> float:
    """Max of x over all ranks (x itself when no process group is up): every
    multi-GPU time is the slowest rank's."""
    if dist is None:
        return x
    import torch
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(world: int, units_per_rank_step: int, steps: int, elapsed_ms: float) -> float:
    """Units per second over all ranks: each of the `world` replicas processed
    `units_per_rank_step` units in each of `steps` steps within elapsed_ms."""
    return world * units_per_rank_step * steps / (elapsed_ms / 1e3)


def run_ours(args, cfg):
    import torch
    import softmax_attention_video_chunk_b200 as vdn
    from synth import make_inputs

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))

    def barrier():
        if dist is not None:
            dist.barrier()

    inp = make_inputs(cfg, alpha_range=(0.9, 1.0) if args.alpha else None,
                      beta_per_token=args.beta_per_token)
    d = {k: (v.cuda() if v is not None else None) for k, v in inp.items()}
    if args.frozen_state:  # keys scaled by 1/sqrt(N) (a reading of SANA-WM's frame-size scaling)
        d["k"] = (d["k"].float() / float(cfg.N) ** 0.5).to(d["k"].dtype)
    p = vdn.params_for(d["q"], d["v"], d["text_k"], cfg.T, d["W_soft"], chunk=cfg.chunk,
                       window_radius=cfg.window_radius, text_softmax=args.text_softmax,
                       beta_per_token=args.beta_per_token, frozen_state=args.frozen_state,
                       proj_mxfp8=args.proj_mxfp8)
    ws = vdn.alloc_workspace(p)
    out = torch.empty(cfg.B, cfg.L, p.D_out, dtype=torch.float32, device="cuda")
    stream = torch.cuda.current_stream()
    lin = None
    if args.prep:  # raw projections -> VDA-Prep -> the linear branch's q, k, v
        from synth import make_prep_inputs
        pin = make_prep_inputs(cfg)
        dp = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in pin.items()}
        lin = tuple(torch.empty_like(dp[n]) for n in ("q_raw", "k_raw", "v_raw"))
        pp = vdn.make_prep_params(cfg.B, cfg.H, cfg.T, pin["grid_h"], pin["grid_w"], cfg.d,
                                  cfg.dtype)
        prep_ws = torch.zeros(vdn.PREP_WORKSPACE_BYTES, dtype=torch.uint8, device="cuda")
    prep_ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
    tq = None
    if args.text_softmax:  # text queries too: the text rows of the joint Softmax
        from synth import make_text_queries
        tq = make_text_queries(cfg).cuda()
    tq_ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]

    def step(events=None, i=None):
        if lin is not None:
            if i is not None:
                prep_ev[i][0].record(stream)
            vdn.vda_prep(dp["q_raw"], dp["k_raw"], dp["v_raw"], dp["wk_s"], dp["wk_t"],
                         dp["wv_s"], dp["wv_t"], cfg.T, pin["grid_h"], pin["grid_w"], out=lin,
                         workspace=prep_ws, params=pp)
            if i is not None:
                prep_ev[i][1].record(stream)
        vdn.hybrid_attn_fwd(d["q"], d["k"], d["v"], d["beta"], d["text_k"], d["text_v"],
                            d["W_soft"], d["W_lin"], d["gates"], cfg.T, alpha=d["alpha"],
                            out=out, workspace=ws, params=p, events=events, lin=lin)
        if tq is not None:  # the text rows of the joint Softmax (dense over every key)
            if i is not None:
                tq_ev[i][0].record(stream)
            vdn.text_query_attn(tq, d["k"], d["v"], d["text_k"], d["text_v"], cfg.T,
                                workspace=ws, params=p)
            if i is not None:
                tq_ev[i][1].record(stream)

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize()
    st = vdn.device_status(p, ws)
    if st != 0:
        raise RuntimeError(f"device status after warm-up: {vdn.STATUS[st]}")

    nS = vdn.N_STAGES
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(nS + 1)] for _ in range(args.steps)]
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(local)
    barrier()
    torch.cuda.synchronize()
    sampler.start()
    time.sleep(0.3)
    t_start.record(stream)
    for i in range(args.steps):
        step(evs[i], i)
    t_end.record(stream)
    torch.cuda.synchronize()
    barrier()
    clocks = sampler.stop()
    elapsed_ms = t_start.elapsed_time(t_end)
    stage_ms = [sum(evs[i][s].elapsed_time(evs[i][s + 1]) for i in range(args.steps)) / args.steps
                for s in range(nS)]
    elapsed_ms = ranks_max(elapsed_ms, dist, "cuda")
    st = vdn.device_status(p, ws)
    if st != 0:
        raise RuntimeError(f"device status after timing: {vdn.STATUS[st]}")
    tq_ms = None
    if tq is not None:
        tq_ms = sum(e[0].elapsed_time(e[1]) for e in tq_ev) / args.steps
    prep_ms = None
    if lin is not None:
        prep_ms = sum(e[0].elapsed_time(e[1]) for e in prep_ev) / args.steps
        st = vdn.device_status(None, prep_ws)
        if st != 0:
            raise RuntimeError(f"device status of VDA-Prep: {vdn.STATUS[st]}")
        del dp, lin

    ms_per_step = elapsed_ms / args.steps
    tokens = cfg.B * cfg.L
    value = whole_job_rate(world, tokens, args.steps, elapsed_ms)

    # ---- end to end: pinned host inputs -> device, forward, result -> host,
    # through the C ABI's host-buffer entry (vdn_hybrid_attn_fwd_host): uploads,
    # compute and download of consecutive steps overlap on three streams
    host = {k: (v.pin_memory() if v is not None else None) for k, v in inp.items()}
    outs_host = [torch.empty(out.shape, dtype=out.dtype, pin_memory=True) for _ in range(2)]
    del d, ws, out
    torch.cuda.empty_cache()
    pipe = vdn.HostPipeline(host, cfg.T, params=p)
    for i in range(2):
        h2d, d2h = pipe.submit(host, outs_host[i % 2])
    pipe.synchronize()
    e2e_steps = max(3, args.steps)  # as many pipelined steps as the device-timed leg
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(pipe.s_h2d)
    pipe.s_cmp.wait_event(e0)
    pipe.s_d2h.wait_event(e0)
    for i in range(e2e_steps):
        pipe.submit(host, outs_host[i % 2])
    e1.record(pipe.s_d2h)  # after the last download, which follows every earlier step
    pipe.synchronize()
    e2e_ms = e0.elapsed_time(e1)
    e2e_ms = ranks_max(e2e_ms, dist, "cuda")
    pipe.close()
    e2e_value = whole_job_rate(world, tokens, e2e_steps, e2e_ms)

    if rank == 0:
        wm = work_model(cfg, text_keys=args.text_softmax)
        pk = measured_peaks()
        soft_ms = stage_ms[2]
        achieved = wm["f_soft"] / (soft_ms / 1e3) / 1e12
        t_roof = max(wm["f_total"] / (pk["tc"] * 1e12), wm["bytes_min"] / (pk["hbm"] * 1e9))
        line = base_line(args, cfg, value, ms_per_step, world)
        line["tflops"] = wm["f_total"] / (ms_per_step / 1e3) / 1e12
        line["roofline"] = {
            "bound": "tensor", "kernel": "attn_tc_kernel (window+anchor Softmax)",
            "achieved": achieved, "peak": pk["tc_sust"], "unit": "TFLOP/s",
            "frac": achieved / pk["tc_sust"],
            "frac_of_burst_peak": achieved / pk["tc"],
            "frac_of_datasheet_peak": achieved / DATASHEET_BF16_TFLOPS,
            "traffic": (ATTN_TRAFFIC_PER_HEAD * cfg.B * cfg.H
                        if (cfg.T, cfg.N, cfg.d) in ATTN_TRAFFIC_SHAPES else None),
            "traffic_note": "ncu capture of the 4-head 768p shape, scaled by heads",
            "peak_kind": f"{pk['src']} bf16 dense, sustained (kernel timed inside the step loop)",
            "algorithmic_flops_per_launch": wm["f_soft"], "ms_per_launch": soft_ms,
        }
        # the whole forward against the larger of FLOPs / tensor peak and bytes
        # / HBM bandwidth: the headline fraction, given against the measured
        # burst and sustained peaks and the datasheet ones
        def path_frac(tc, hbm):
            return 1e3 * max(wm["f_total"] / (tc * 1e12), wm["bytes_min"] / (hbm * 1e9)) / ms_per_step
        line["path_roofline"] = {
            "flops": wm["f_total"], "bytes_min": wm["bytes_min"],
            "t_roofline_ms": 1e3 * t_roof, "frac": 1e3 * t_roof / ms_per_step,
            "peak_tflops": pk["tc"], "peak_hbm_gbs": pk["hbm"], "peaks": pk["src"] + " (burst)",
            "frac_of_sustained_peak": path_frac(pk["tc_sust"], pk["hbm"]),
            "frac_of_datasheet_peak": path_frac(DATASHEET_BF16_TFLOPS, DATASHEET_HBM_GBS),
            "datasheet_peaks": {"bf16_tflops": DATASHEET_BF16_TFLOPS, "hbm_gbs": DATASHEET_HBM_GBS},
        }
        line["stages_ms"] = dict(zip(vdn.STAGE_NAMES, [round(x, 4) for x in stage_ms]))
        line["gpu_launches"] = args.steps * (vdn.forward_launches(p) +
                                             (2 if prep_ms is not None else 0))
        if tq_ms is not None:
            line["stages_ms"]["text_rows"] = round(tq_ms, 4)
            # V^T conversion, text-row Softmax split over key shares, combine
            line["gpu_launches"] += args.steps * 3
        if prep_ms is not None:
            es = 2 if cfg.dtype == "bf16" else 4
            prep_bytes = 6 * cfg.B * cfg.L * cfg.H * cfg.d * es  # read q, k, v; write 3
            line["stages_ms"]["prep"] = round(prep_ms, 4)
            line["prep_roofline"] = {
                "bound": "hbm", "kernel": "prep_conv_kernel + prep_l2_kernel (VDA-Prep)",
                "achieved": prep_bytes / (prep_ms / 1e3) / 1e9, "peak": pk["hbm"], "unit": "GB/s",
                "frac": prep_bytes / (prep_ms / 1e3) / 1e9 / pk["hbm"], "traffic": None,
                "algorithmic_bytes_per_launch": prep_bytes, "ms_per_launch": prep_ms,
                "peak_kind": f"{pk['src']} HBM copy"}
        line["clocks"] = clocks
        line["e2e"] = {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d,
                       "d2h_bytes_per_step": d2h, "steps": e2e_steps,
                       "api": "vdn_hybrid_attn_fwd_host (C ABI; pinned host buffers, "
                              "3 streams, 2 device slots alternating)"}
        if args.prep:
            line["e2e"]["note"] = "the forward on prepared inputs; VDA-Prep is not in this leg"
        if world == 1 and not args.no_cpu_baseline:
            rows = oracle_sample(cfg, inp)
            secs = time_oracle(cfg, inp, rows)
            line["cpu_baseline"] = {
                "value": len(rows) / secs, "unit": UNIT, "cores": blas_threads(),
                "kind": "oracle",
                "sample": f"{len(rows)} query tokens (frames {sample_frames(cfg, rows)}), all "
                          f"heads, float64 NumPy oracle, {secs:.1f} s"}
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def main():
    from synth import CONFIGS
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1,
                    help="GPUs of the job (one replica per rank under torchrun)")
    ap.add_argument("--steps", type=int, default=10, help="timed forwards")
    ap.add_argument("--warmup", type=int, default=3, help="untimed forwards before them")
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours",
                    help="ours: the library; reference: the float64 oracle on a sample")
    ap.add_argument("--config", default="768p_bf16",
                    help="workload: " + ", ".join(sorted(CONFIGS)))
    ap.add_argument("--no-cpu-baseline", action="store_true",
                    help="skip the timed oracle sample on the host cores")
    ap.add_argument("--text-softmax", action="store_true",
                    help="video queries also attend all text tokens in the Softmax branch")
    ap.add_argument("--beta-per-token", action="store_true",
                    help="one write gate per token instead of per frame")
    ap.add_argument("--frozen-state", action="store_true",
                    help="frame updates by the frozen-state comparison rule instead of VDA")
    ap.add_argument("--prep", action="store_true",
                    help="time VDA-Prep (linear-branch feature map of raw q, k, v) in every step")
    ap.add_argument("--proj-mxfp8", action="store_true",
                    help="output projections in MXFP8 (block-scaled E4M3, FP32 accumulation)")
    ap.add_argument("--alpha", action="store_true",
                    help="channel-wise decay gate alpha ~ U[0.9, 1] instead of none")
    args = ap.parse_args()
    cfg = CONFIGS[args.config]
    if args.impl == "reference":
        return run_reference(args, cfg)
    return run_ours(args, cfg)


if __name__ == "__main__":
    sys.exit(main())
