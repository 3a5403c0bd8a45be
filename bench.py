#!/usr/bin/env python
"""Throughput of the Jamba Mamba mixer on B200: one JSON line on rank 0.

A step is one prefill of a 131072-token sequence (batch 1) through the whole
mixer at Jamba width (d_model 4096, d_inner 8192, d_state 16, dt_rank 256,
inner RMSNorm): in_proj, conv+SiLU, x_proj, inner norms, dt_proj+softplus,
selective scan + gate, out_proj.  Beside it the same line carries the decode
step (batch 64, CUDA graph), the selective scan alone at 128K context, the
RMSNorm -> Mamba -> RMSNorm -> top-2-of-16 MoE layer pair, the roofline of the
dominant kernel and the fp64 oracle timed on this host as the CPU baseline.

  python bench.py [--gpus N --steps K --warmup W] [--impl reference] [--quick]

With N > 1 (launched by torchrun) every rank runs its own sequence: no
collective on the data path, weak scaling, max time over ranks.
"""
import argparse
import json
import os
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

PREFILL_L = 131072
DECODE_B, DECODE_PREFILL, DECODE_STEPS = 64, 2048, 1024
SCAN_L, SCAN_DI = 131072, 8192
PAIR_B, PAIR_L = 4, 8192
ATTN_L = 32768
METRIC = "Mamba-layer tokens/s (prefill 128K, decode) at d_model=4096; scan HBM GB/s vs peak"
# DRAM bytes (read + write) of one in_proj + conv launch pair at 131072 tokens: ncu at 16384 tokens
# (GEMM 0.715 GB read + 0.542 GB written, slab-row kernel 0.050 + 0.0004 GB) scaled by 8, since
# operand re-reads and the outputs all grow with the token count
IN_PROJ_TRAFFIC_128K = 8 * (0.714592512e9 + 0.542140928e9 + 0.050384896e9 + 0.000403968e9)


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="product", choices=["product", "reference"])
    ap.add_argument("--quick", action="store_true", help="skip the side measurements")
    ap.add_argument("--only", default="all",
                    help="comma list of parts to run (prefill,gemm,scan,decode,pair,moe8,moe8dec,moe,attn,e2e,cpu); "
                         "for profiling")
    ap.add_argument("--seqlen", type=int, default=PREFILL_L, help="prefill tokens")
    ap.add_argument("--scan-seqlen", type=int, default=SCAN_L)
    ap.add_argument("--decode-steps", type=int, default=DECODE_STEPS)
    ap.add_argument("--decode-layers", type=int, default=4,
                    help="distinct Mamba layers the decode steps cycle through (their weights do not fit L2 together)")
    ap.add_argument("--pair-seqlen", type=int, default=PAIR_L)
    ap.add_argument("--attn-seqlen", type=int, default=ATTN_L)
    ap.add_argument("--moe8-tokens", type=int, default=64, help="tokens of the moe8dec part")
    ap.add_argument("--moe-tokens", type=int, default=4096, help="tokens of the moe part (bf16 experts alone)")
    ap.add_argument("--decode-prefill", type=int, default=DECODE_PREFILL,
                    help="prefill tokens that fill the decode caches (profiling: a short one keeps the "
                         "device footprint small; the caches have their full size either way)")
    ap.add_argument("--cpu-table", action="store_true",
                    help="time the fp64 oracle of every workload on this host (single thread and all cores)")
    return ap.parse_args()


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            d = json.load(f)
        return dict(hbm=d["hbm_gbs"], bf16=d["bf16_tflops"], bf16_sus=d["bf16_tflops_sustained"], src="measured")
    except Exception:
        return dict(hbm=6650.0, bf16=1590.0, bf16_sus=1400.0, src="fallback")


# ------------------------------------------------------------------ clocks
class Clocks:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, dev):
        self.proc = None
        self.path = None
        try:
            uuid = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
        except Exception:
            uuid = None
        self.sel = ["-i", uuid] if uuid else []

    def start(self):
        """Start sampling and return once the sampler writes (at most ~5 s), so that
        the samples taken from here on cover the timed region that follows: the
        lines already written are skipped by stop()."""
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        self.skip = 0
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "--query-gpu=" + self.FIELDS, "--format=csv,noheader,nounits",
                                          "-lms", "20"] + self.sel, stdout=open(self.path, "w"),
                                         stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
            return
        t_end = time.time() + 5.0
        while time.time() < t_end and self.proc.poll() is None:
            with open(self.path) as f:
                n = f.read().count("\n")
            if n > 0:
                self.skip = n
                break
            time.sleep(0.01)

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        sm, mx, reasons = [], 0.0, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        lines = open(self.path).read().splitlines()
        # samples from the timed region (the last one before it as well when it was shorter than a sample period)
        lines = lines[self.skip:] or lines[-1:]
        for line in lines:
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = max(mx, float(f[2]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        os.unlink(self.path)
        if not sm:
            return None
        busy = [v for v in sm if v > 0.5 * mx] or sm
        busy.sort()
        return {"sm_mhz": busy[len(busy) // 2], "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ------------------------------------------------------------------ helpers
def event_time_ms(fn, reps, stream, flush=None):
    """mean device time of fn() over reps launches on `stream`, L2 flushed before each"""
    times = []
    for _ in range(reps):
        if flush is not None:
            flush()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        fn()
        b.record(stream)
        b.synchronize()
        times.append(a.elapsed_time(b))
    return sum(times) / len(times), times


def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(local)
    return world, rank, local


def max_over_ranks(v, world):
    """the slowest rank's time (the job takes as long as its slowest replica)"""
    if world == 1:
        return v
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([v], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def rank_seed(rank):
    """each replica prefills its own sequence: the input seed is the rank"""
    return rank


def aggregate_tokens_per_s(world, tokens_per_rank, max_ms):
    """whole-job throughput: all ranks' tokens over the slowest rank's time"""
    return world * tokens_per_rank / (max_ms / 1e3)


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# ------------------------------------------------------------------ CPU baseline
def cpu_baseline(sample_tokens=1024):
    """fp64 oracle prefill of `sample_tokens` tokens at Jamba width on this host's cores."""
    import numpy as np
    from oracle import mamba as om
    from synthetic import mamba_input, mamba_params, workload
    sh = workload("prefill_4k")["mamba"]
    p64 = om.params64(mamba_params(sh, seed=0))
    u = om.to64(mamba_input(sh, 1, sample_tokens, seed=0))
    t0 = time.perf_counter()
    om.mamba_prefill(p64, u, sh, scan="c")
    dt = time.perf_counter() - t0
    try:
        cores = len(os.sched_getaffinity(0))
    except Exception:
        cores = os.cpu_count()
    try:
        from threadpoolctl import threadpool_info
        threads = max([i.get("num_threads", 1) for i in threadpool_info()] or [cores])
    except Exception:
        threads = cores
    _ = np
    return {"value": sample_tokens / dt, "unit": "tokens/s", "cores": int(threads), "kind": "oracle",
            "sample": "fp64 oracle prefill of %d tokens (batch 1) at d_model 4096 / d_inner 8192, numpy "
                      "matmul + C scan; %.1f s" % (sample_tokens, dt)}


# ------------------------------------------------------------------ product arm
def run_product(args):
    import mamba_selective_scan_mixer_b200 as J
    from synthetic import AttnShape, MoEShape, attn_input, attn_params, block_norm_params, decode_inputs, \
        mamba_input, mamba_params, moe_input, moe_params, scan_inputs, workload

    world, rank, local = dist_setup(args)
    dev = torch.device("cuda", local)
    pk = peaks()
    sh = workload("prefill_4k")["mamba"]
    L = args.seqlen
    stream = torch.cuda.current_stream(dev)

    parts = {"prefill", "gemm", "scan", "decode", "pair", "moe8", "attn", "e2e", "cpu"} if args.only == "all" else \
        set(args.only.split(","))
    if args.quick:
        parts &= {"prefill"}
    params = {k: v.to(dev) for k, v in mamba_params(sh, seed=0).items()}
    mixer = J.MambaMixer(params, sh)
    u = mamba_input(sh, 1, L, seed=rank_seed(rank), device=dev) if ({"prefill", "gemm", "e2e"} & parts) else None
    out = torch.empty_like(u) if u is not None else None
    cs, ss = mixer.new_states(1)
    flush_buf = torch.empty(512 << 20, dtype=torch.uint8, device=dev)
    flush = lambda: flush_buf.zero_()
    step = lambda: mixer.prefill(u, out=out, conv_state_out=cs, ssm_state_out=ss)

    ms, clk, value = None, None, None
    if "prefill" in parts:
        for _ in range(args.warmup):
            step()
        torch.cuda.synchronize()
        J.device_status()
        clocks = Clocks(dev)
        clocks.start()   # returns once sampling runs; the barrier then lines the ranks up for the timed steps
        barrier(world)
        torch.cuda.synchronize()
        ms, per = event_time_ms(step, args.steps, stream, flush)
        torch.cuda.synchronize()
        barrier(world)
        clk = clocks.stop()
        J.device_status()
        ms = max_over_ranks(ms, world)
        value = aggregate_tokens_per_s(world, L, ms)

    res = {"metric": METRIC, "value": None if value is None else round(value, 1), "unit": "tokens/s",
           "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
           "ms_per_step": None if ms is None else round(ms, 4), "higher_is_better": True, "scaling": "weak",
           "vs_baseline": None, "dtype": "bf16",
           "data": "synthetic: seeded N(0,1) input, N(0,0.02) weights, A=-(n+1), D=1, dt_bias log-uniform",
           "config": {"workload": "prefill_128k: Mamba mixer prefill, batch 1, L=%d, d_model 4096, d_inner 8192, "
                                  "d_state 16, dt_rank 256, inner RMSNorm, bf16 weights/activations, fp32 state" % L,
                      "global_batch": world, "seq_len": L, "parallelism": "replicas" if world > 1 else "single",
                      "l2": "512 MB buffer written before every timed step (outside the events)"},
           # per prefill step: in_proj + conv, conv slab rows, x_proj, x_proj sum + norms, dt_proj, scan, out_proj
           "gpu_launches": None if ms is None else 7 * args.steps, "clocks": clk}

    if rank == 0 and "gemm" in parts:
        # dominant kernel: in_proj on the tensor cores with the conv in its
        # epilogue (+ the slab-row kernel after it), the same launches as inside the step
        xz = torch.empty(1, L, 2 * sh.d_inner, dtype=torch.bfloat16, device=dev)
        xc = torch.empty(1, L, sh.d_inner, dtype=torch.bfloat16, device=dev)
        g = lambda: J.in_proj_conv1d(u, params["in_proj"], params["conv_w"], params["conv_b"], xz=xz, xc=xc)
        for _ in range(2):
            g()
        gms, _ = event_time_ms(g, 5, stream, flush)
        flops = 2.0 * L * 2 * sh.d_inner * sh.d_model
        ach = flops / (gms / 1e3) / 1e12
        res["roofline"] = {"kernel": "in_proj + conv1d: gemm_bf16_tc_kernel<256,4,EPI_CONVP> + conv_fixup_kernel "
                                     "(%dx%dx%d)" % (L, 2 * sh.d_inner, sh.d_model),
                           "bound": "tensor", "achieved": round(ach, 1), "peak": pk["bf16"], "unit": "TFLOP/s",
                           "frac": round(ach / pk["bf16"], 4),
                           "traffic": IN_PROJ_TRAFFIC_128K if L == PREFILL_L else None,
                           "peak_source": "%s bf16 burst (kernel timed alone)" % pk["src"],
                           "ms": round(gms, 3)}
        del xz, xc
    if rank == 0 and "scan" in parts:
        # selective scan alone at 128K context
        SL = args.scan_seqlen
        s = {k: v.to(dev) for k, v in scan_inputs(1, SL, SCAN_DI, 16, seed=0, device=dev).items()}
        y = torch.empty_like(s["x"])
        sc = lambda: J.selective_scan(s["x"], s["z"], s["dt"], s["B"], s["C"], s["A"], s["D"], y=y, ws=scan_ws,
                                      want_state=True)
        import ctypes
        nbytes = ctypes.c_size_t()
        J.lib().jamba_selective_scan_workspace_size(1, SL, SCAN_DI, 16, 0, ctypes.byref(nbytes))
        scan_ws = torch.empty(nbytes.value, dtype=torch.uint8, device=dev)
        for _ in range(2):
            sc()
        torch.cuda.synchronize()
        sclocks = Clocks(dev)
        sclocks.start()
        sms, _ = event_time_ms(sc, 20, stream, flush)
        torch.cuda.synchronize()
        sclk = sclocks.stop()
        sbytes = SL * (SCAN_DI * (2 + 2 + 4 + 2) + 16 * 2 * 2)
        gbs = sbytes / (sms / 1e3) / 1e9
        # the arithmetic bound: 64 fp32 lane-ops per (token, channel) in the power
        # form (16 decay powers, 16 dt*x*B, 16 state FMAs, 16 C.h FMAs) against
        # 128 fp32 lanes per SM per clock, at the clock seen while the scan ran
        mhz = (sclk or clk or {}).get("sm_mhz") or 1965.0
        alu_ms = 1e3 * SL * SCAN_DI * 64 / (128 * torch.cuda.get_device_properties(dev).multi_processor_count
                                            * mhz * 1e6)
        res["scan"] = {"workload": "scan_128k: selective scan + D + SiLU(z) gate alone, batch 1, L=%d, "
                                   "d_inner 8192, bf16 x/z/B/C/y, fp32 dt" % SL,
                       "ms": round(sms, 4), "GB/s": round(gbs, 1), "frac_of_measured_hbm": round(gbs / pk["hbm"], 4),
                       "frac_of_8TBs": round(gbs / 8000.0, 4), "algorithmic_bytes": sbytes,
                       "alu_floor_ms": round(alu_ms, 4), "frac_of_fp32_pipe": round(alu_ms / sms, 4),
                       "alu_clock_mhz": mhz, "clocks": sclk, "tokens/s": round(SL / (sms / 1e3), 1)}
        del s, y, scan_ws
    if rank == 0 and "decode" in parts:
        # decode: batch 64, caches from a 2048-token prefill, steps in one CUDA graph
        B = DECODE_B
        NST = args.decode_steps
        NLAY = args.decode_layers
        # NLAY distinct layers (weights and caches), stepped in turn as in a
        # multi-layer model, so that no layer finds its own weights still in L2
        layers = [mixer] + [J.MambaMixer({k: v.to(dev) for k, v in mamba_params(sh, seed=10 + l).items()}, sh)
                            for l in range(1, NLAY)]
        u0 = mamba_input(sh, B, args.decode_prefill, seed=1, device=dev)
        caches = []
        for lm in layers:
            dcs, dss = lm.new_states(B)
            lm.prefill(u0, conv_state_out=dcs, ssm_state_out=dss)
            torch.cuda.synchronize()
            lm.release_workspace()   # the prefill's ~21 GB; the decode steps need a few MB
            caches.append((dcs, dss))
        steps_u = decode_inputs(sh, B, NST, seed=1, device=dev)
        dout = torch.empty(B, sh.d_model, dtype=torch.bfloat16, device=dev)
        for lm, (dcs, dss) in zip(layers, caches):
            lm.step(steps_u[0], dcs, dss, out=dout)       # sizes the workspaces before capture
        torch.cuda.synchronize()
        gs = torch.cuda.Stream(dev)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=gs):
            for t in range(NST):
                lm = layers[t % NLAY]
                lm.step(steps_u[t], caches[t % NLAY][0], caches[t % NLAY][1], out=dout)
        graph.replay()
        torch.cuda.synchronize()
        dms, _ = event_time_ms(graph.replay, 3, stream, flush)
        per_step_us = dms * 1e3 / NST
        wbytes = sum(v.numel() * v.element_size() for v in params.values())
        step_bytes = wbytes + 2 * (B * sh.d_inner * 16 * 4 + B * sh.d_inner * 3 * 4) + 2 * B * sh.d_model * 2
        res["decode"] = {"workload": "decode_b64: batch 64, one token per step, %d steps in one CUDA graph "
                                     "over %d layer(s) in turn, caches from a %d-token prefill"
                                     % (NST, NLAY, args.decode_prefill),
                         "tokens/s": round(B * NST / (dms / 1e3), 1), "us_per_step": round(per_step_us, 2),
                         "GB/s": round(step_bytes / (per_step_us / 1e6) / 1e9, 1),
                         "frac_of_measured_hbm": round(step_bytes / (per_step_us / 1e6) / 1e9 / pk["hbm"], 4),
                         # in_proj (conv in its epilogue), x_proj, x_proj sum + norms, dt_proj, state update,
                         # out_proj, split-K sum
                         "algorithmic_bytes_per_step": step_bytes, "launches_per_step": 7}
        del graph, u0, steps_u, layers, caches
    if rank == 0 and "pair" in parts:
        # layer pair: RMSNorm -> Mamba -> residual -> RMSNorm -> top-2-of-16 MoE -> residual
        PL = args.pair_seqlen
        es = MoEShape()
        mp = moe_params(es, seed=0, device=dev)
        moe = J.MoE(mp, es)
        g1, g2 = block_norm_params(sh.d_model, device=dev)
        xp = mamba_input(sh, PAIR_B, PL, seed=2, device=dev)
        pair = lambda: J.layer_pair(mixer, moe, xp, g1, g2)
        pair()
        torch.cuda.synchronize()
        pms, _ = event_time_ms(pair, 3, stream, flush)
        T = PAIR_B * PL
        pflops = T * (2.0 * (2 * sh.d_inner * sh.d_model + (sh.dt_rank + 32) * sh.d_inner +
                             sh.dt_rank * sh.d_inner + sh.d_model * sh.d_inner)
                      + 2 * 2.0 * (3 * es.d_model * es.d_ff) + 2.0 * 16 * es.d_model)
        res["layer_pair"] = {"workload": "layer_pair: batch 4 x %d tokens, Mamba (as prefill) + 16-expert "
                                         "top-2 SwiGLU MoE (d_ff 14336)" % PL,
                             "tokens/s": round(T / (pms / 1e3), 1), "ms": round(pms, 3),
                             "TFLOP/s": round(pflops / (pms / 1e3) / 1e12, 1),
                             "frac_of_bf16_sustained": round(pflops / (pms / 1e3) / 1e12 / pk["bf16_sus"], 4)}
        if "moe8" in parts:
            # ExpertsInt8: the same MoE with int8 expert codes, at the layer pair's token count
            # (tensor-bound) and at a decode batch of 64 tokens (bound by the expert weight bytes)
            pq = J.quantize_experts_int8(mp)
            moe8 = J.MoE(pq, es)
            pair8 = lambda: J.layer_pair(mixer, moe8, xp, g1, g2)
            pair8()
            torch.cuda.synchronize()
            p8ms, _ = event_time_ms(pair8, 3, stream, flush)
            wb16 = sum(mp[k].numel() * mp[k].element_size() for k in ("w_gate", "w_up", "w_down"))
            wb8 = sum(pq[k].numel() * pq[k].element_size() for k in ("w_gate", "w_up", "w_down",
                                                                      "s_gate", "s_up", "s_down"))
            moe_t = {}
            for name, m in (("bf16", moe), ("int8", moe8)):
                for tok in (T, 64):
                    v = moe_input(es, tok, seed=3, device=dev)
                    f = (lambda m=m, v=v: m.forward(v))
                    # the decode batch runs ~0.1 s before its timing, so that the SM clock is that of
                    # this bandwidth-bound call and not the one the preceding tensor-bound calls left
                    for _ in range(1 if tok == T else 128):
                        f()
                    torch.cuda.synchronize()
                    moe_t[(name, tok)] = event_time_ms(f, 5 if tok == T else 20, stream, flush)[0]
            eflops = T * 2 * 2.0 * (3 * es.d_model * es.d_ff)
            res["moe_int8"] = {
                "workload": "ExpertsInt8: 16-expert top-2 SwiGLU MoE (d_model 4096, d_ff 14336) with int8 "
                            "expert codes and per-row fp32 scales, bf16 activations",
                "expert_weight_bytes": {"bf16": wb16, "int8": wb8},
                "layer_pair_ms": round(p8ms, 3), "layer_pair_tokens/s": round(T / (p8ms / 1e3), 1),
                "moe_%d_tokens_ms" % T: {"bf16": round(moe_t[("bf16", T)], 3), "int8": round(moe_t[("int8", T)], 3)},
                "moe_%d_tokens_TFLOP/s_int8" % T: round(eflops / (moe_t[("int8", T)] / 1e3) / 1e12, 1),
                "moe_64_tokens_us": {"bf16": round(1e3 * moe_t[("bf16", 64)], 1),
                                     "int8": round(1e3 * moe_t[("int8", 64)], 1)},
                "moe_64_tokens_weight_GB/s": {"bf16": round(wb16 / (moe_t[("bf16", 64)] / 1e3) / 1e9, 1),
                                              "int8": round(wb8 / (moe_t[("int8", 64)] / 1e3) / 1e9, 1)},
                "moe_64_tokens_int8_frac_of_measured_hbm": round(wb8 / (moe_t[("int8", 64)] / 1e3) / 1e9 / pk["hbm"], 4)}
            del pq, moe8
        del mp, moe, xp
        J.device_status()

    if rank == 0 and "attn" in parts:
        # the block's GQA attention layer: prefill of 32768 tokens, and a batch-64 decode step
        # over 2048-token caches
        ash = AttnShape()
        AL = args.attn_seqlen
        att = J.Attention(attn_params(ash, seed=0, device=dev), ash)
        xa = attn_input(ash, 1, AL, seed=5, device=dev)
        outa = torch.empty_like(xa)
        fa = lambda: att.prefill(xa, out=outa)
        fa()
        torch.cuda.synchronize()
        ams, _ = event_time_ms(fa, 3, stream, flush)
        H, G, D, dm = ash.n_heads, ash.n_kv_heads, ash.head_dim, ash.d_model
        core = 2.0 * AL * AL * H * D                   # causal: QK^T and PV over the lower triangle
        proj = 2.0 * AL * dm * (H + 2 * G) * D + 2.0 * AL * H * D * dm
        del xa, outa
        DB, DL, DS = 64, 2048, 32
        kc, vc, lens = att.new_cache(DB, DL + DS)
        kc.normal_()
        vc.normal_()
        xd = attn_input(ash, DB, 1, seed=6, device=dev)[:, 0].contiguous()
        od = torch.empty_like(xd)

        def dec():
            for _ in range(DS):
                att.step(xd, kc, vc, lens, out=od)

        lens.fill_(DL)
        dec()
        torch.cuda.synchronize()
        dts = []
        for _ in range(3):
            lens.fill_(DL)
            dts.append(event_time_ms(dec, 1, stream, flush)[0])
        dus = 1e3 * min(dts) / DS
        kv_bytes = 2.0 * DB * G * (DL + DS / 2 + 1) * D * 2
        w_bytes = 2.0 * ((H + 2 * G) * D * dm + dm * H * D)
        res["attention"] = {
            "workload": "attn_32k: GQA attention layer (32 query heads over 8 KV heads of 128, d_model 4096, no "
                        "positional encoding), causal prefill of %d tokens; decode: batch 64 over %d-token caches" %
                        (AL, DL),
            "prefill_ms": round(ams, 3), "prefill_tokens/s": round(AL / (ams / 1e3), 1),
            "prefill_TFLOP/s": round((core + proj) / (ams / 1e3) / 1e12, 1),
            "prefill_frac_of_bf16_sustained": round((core + proj) / (ams / 1e3) / 1e12 / pk["bf16_sus"], 4),
            "prefill_flops": {"attention_core": core, "projections": proj},
            "decode_us_per_step": round(dus, 2),
            "decode_GB/s": round((kv_bytes + w_bytes) / (dus / 1e6) / 1e9, 1),
            "decode_frac_of_measured_hbm": round((kv_bytes + w_bytes) / (dus / 1e6) / 1e9 / pk["hbm"], 4)}
        del att, kc, vc
        J.device_status()
    if rank == 0 and "moe" in parts:
        # bf16 experts alone (16 experts, d_ff 14336, a few GB resident): the small case the
        # grouped expert GEMM profiles are taken on
        es = MoEShape()
        moe = J.MoE(moe_params(es, seed=0, device=dev), es)
        v = moe_input(es, args.moe_tokens, seed=3, device=dev)
        f = lambda: moe.forward(v)
        for _ in range(args.warmup):
            f()
        torch.cuda.synchronize()
        mms, _ = event_time_ms(f, args.steps, stream, flush)
        eflops = args.moe_tokens * 2 * 2.0 * (3 * es.d_model * es.d_ff)
        res["moe_bf16"] = {"workload": "top-2-of-16 SwiGLU MoE, bf16 experts, %d tokens, d_model 4096, d_ff 14336"
                                       % args.moe_tokens,
                           "ms": round(mms, 3), "TFLOP/s": round(eflops / (mms / 1e3) / 1e12, 1)}
        del moe, v
        J.device_status()
    if rank == 0 and "moe8dec" in parts:
        # ExpertsInt8 decode batch alone, with only the int8 experts resident (a few GB): the
        # small case the expert-kernel profiles are taken on
        es = MoEShape()
        mp = moe_params(es, seed=0, device=dev)
        pq = J.quantize_experts_int8(mp)
        del mp
        torch.cuda.synchronize()
        torch.cuda.empty_cache()
        moe8 = J.MoE(pq, es)
        v = moe_input(es, args.moe8_tokens, seed=3, device=dev)
        f = lambda: moe8.forward(v)
        for _ in range(args.warmup):
            f()
        torch.cuda.synchronize()
        dms, _ = event_time_ms(f, args.steps, stream, flush)
        wb8 = sum(pq[k].numel() * pq[k].element_size() for k in ("w_gate", "w_up", "w_down", "s_gate", "s_up", "s_down"))
        res["moe_int8_decode"] = {"workload": "ExpertsInt8 MoE, %d tokens, 16 experts top-2, d_model 4096, d_ff 14336"
                                              % args.moe8_tokens,
                                  "us": round(1e3 * dms, 1),
                                  "weight_GB/s": round(wb8 / (dms / 1e3) / 1e9, 1),
                                  "frac_of_measured_hbm": round(wb8 / (dms / 1e3) / 1e9 / pk["hbm"], 4)}
        del pq, moe8
        J.device_status()

    # end to end through the public API with host buffers (pinned), copies inside the timed region
    if "e2e" in parts:
        hu = u.cpu().pin_memory()
        hout = torch.empty_like(hu).pin_memory()

        def e2e():
            # pinned host in and out; the library overlaps the transfers with the compute
            mixer.prefill_host(hu, out_host=hout, conv_state_out=cs, ssm_state_out=ss)

        e2e()
        torch.cuda.synchronize()
        ems, _ = event_time_ms(e2e, max(2, args.steps // 2), stream, flush)
        ems = max_over_ranks(ems, world)
        res["e2e"] = {"value": round(aggregate_tokens_per_s(world, L, ems), 1), "unit": "tokens/s",
                      "h2d_bytes_per_step": hu.numel() * hu.element_size(),
                      "d2h_bytes_per_step": hout.numel() * hout.element_size()}
    if rank == 0 and "cpu" in parts:
        res["cpu_baseline"] = cpu_baseline()
    if rank == 0:
        print(json.dumps(res), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def _host_cores():
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count()


def cpu_table(args):
    """The fp64 oracle timed on this host for every workload, single-threaded and
    on all cores, each on a bounded sample of the workload (batch rows, tokens
    and channels are independent, so per-unit rates carry over; time
    recurrences are never cut).  One JSON line."""
    import numpy as np
    from threadpoolctl import threadpool_limits
    from oracle import mamba as om
    from oracle import moe as omoe
    from synthetic import MoEShape, block_norm_params, mamba_input, mamba_params, moe_params, scan_inputs, \
        workload

    class _Lazy:   # expert weights widened to fp64 one expert at a time
        def __init__(self, t):
            self.t = t

        def __getitem__(self, e):
            return om.to64(self.t[e])

    def timed(fn):
        t0 = time.perf_counter()
        fn()
        return time.perf_counter() - t0

    tiny = workload("tiny_fp32")
    jam = workload("prefill_4k")["mamba"]
    pt = om.params64(mamba_params(tiny["mamba"], seed=0))
    ut = om.to64(mamba_input(tiny["mamba"], 1, tiny["seqlen"] + tiny["steps"], seed=0))

    def run_tiny():
        r = om.mamba_prefill(pt, ut[:, :tiny["seqlen"]], tiny["mamba"])
        cs, ss = r["conv_state"], r["ssm_state"]
        for t in range(tiny["steps"]):
            _, cs, ss = om.mamba_step(pt, ut[:, tiny["seqlen"] + t], tiny["mamba"], cs, ss)

    pj = om.params64(mamba_params(jam, seed=0))
    up = om.to64(mamba_input(jam, 1, 512, seed=0))
    sc = {k: om.to64(v) for k, v in scan_inputs(1, SCAN_L, 256, 16, seed=0).items()}
    ud = om.to64(mamba_input(jam, DECODE_B, 4, seed=1))
    cs0 = np.zeros((DECODE_B, jam.d_inner, 3))
    ss0 = np.zeros((DECODE_B, jam.d_inner, 16))
    es = MoEShape()
    mp = moe_params(es, seed=0)
    ep = {"router": om.to64(mp["router"]), **{k: _Lazy(mp[k]) for k in ("w_gate", "w_up", "w_down")}}
    g1, g2 = (om.to64(g) for g in block_norm_params(jam.d_model))
    xp = om.to64(mamba_input(jam, 1, 256, seed=2))

    def run_decode():
        cs, ss = cs0, ss0
        for t in range(4):
            _, cs, ss = om.mamba_step(pj, ud[:, t], jam, cs, ss)

    cases = [
        ("tiny_fp32", "prefill of 256 tokens + 16 decode steps (whole workload)", tiny["seqlen"] + tiny["steps"],
         run_tiny),
        ("prefill_4k / prefill_128k", "prefill of 512 tokens at Jamba width (the per-token cost of both)", 512,
         lambda: om.mamba_prefill(pj, up, jam, scan="c")),
        ("scan_128k", "C scan of 256 of the 8192 channels over all 131072 steps, counted at 8192 channels",
         SCAN_L * 256 / SCAN_DI,
         lambda: om.selective_scan_c(sc["x"], sc["dt"], sc["A"], sc["B"], sc["C"], sc["D"], sc["z"])),
        ("decode_b64", "4 decode steps of all 64 rows at Jamba width", 4 * DECODE_B, run_decode),
        ("layer_pair", "layer pair on 256 tokens (Mamba + 16-expert top-2 MoE, d_ff 14336)", 256,
         lambda: omoe.layer_pair(pj, ep, xp, jam, es.top_k, g1, g2, scan="c")),
    ]
    rows = {}
    for name, sample, units, fn in cases:
        with threadpool_limits(1):
            t1 = timed(fn)
        tn = timed(fn)
        rows[name] = {"sample": sample, "unit": "tokens/s", "single_thread": round(units / t1, 3),
                      "all_cores": round(units / tn, 3), "seconds": [round(t1, 2), round(tn, 2)]}
    print(json.dumps({"cpu_table": rows, "cores": _host_cores(), "kind": "oracle",
                      "note": "the C scan loop is single-threaded; numpy's BLAS uses the cores"}), flush=True)


def run_reference(args):
    """The oracle as it stands, on this host's cores, same metric and workload (bounded sample)."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    times = []
    base = None
    for _ in range(args.warmup):
        cpu_baseline(256)
    for _ in range(args.steps):
        base = cpu_baseline(256)
        times.append(256 / base["value"])
    ms = 1e3 * sum(times) / len(times)
    v = 256 / (ms / 1e3)
    base["value"] = round(v, 2)
    print(json.dumps({"impl": "reference", "metric": METRIC, "value": round(v, 2), "unit": "tokens/s",
                      "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 2),
                      "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
                      "data": "synthetic", "config": {"workload": "prefill_128k (oracle sample: 256 tokens per "
                                                                  "step at the same widths)"},
                      "cpu_baseline": base,
                      "e2e": {"value": round(v, 2), "unit": "tokens/s", "h2d_bytes_per_step": 0,
                              "d2h_bytes_per_step": 0}}), flush=True)


if __name__ == "__main__":
    a = parse()
    if a.cpu_table:
        cpu_table(a)
    elif a.impl == "reference":
        run_reference(a)
    else:
        run_product(a)
