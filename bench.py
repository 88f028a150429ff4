"""Benchmark of the SpinQuant W4A4 + online-Hadamard hot path on B200.

One step = the down_proj path at Qwen3-8B shape ("SpinQuant, Reproduced",
section Q5): online R4 rotation H12 (x) H1024 + per-token INT4 quantization of
x [4096, 12288] (sq_rotate_quant), then the W4A4 GEMM against INT4 weights
[4096, 12288] with the dequant epilogue to bf16 (sq_w4a4_linear).

Usage:  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
For N > 1 launch one process per GPU with torch.distributed.run; every rank
runs the full step on its own GPU (the path shards by tokens with no data
exchange), and rank 0 prints one JSON line with the max-over-ranks time.

metric  : W4A4 linear TOPS (2*M*N*K per step / step time), step inputs resident
          in HBM; rotate+quant GB/s and the GEMM's own TOPS ride along.
e2e     : the same metric through the public API with the step's input x in
          pinned host memory and the bf16 result copied back each step.
roofline: the GEMM against the int8 tensor peak (measured bf16 peak x 2, the
          nominal int8/bf16 ratio); the rotate+quant kernel against HBM.
cpu_baseline / --impl reference: the CPU oracle on a bounded sample of the
          same workload, extrapolated to one full step.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

M, K, N = 4096, 12288, 4096
N_SMALL, N_POW2 = 12, 1024
OPS = 2.0 * M * N * K
# algorithmic bytes of sq_rotate_quant per row: bf16 in, packed INT4 out, f32 scale
RQ_BYTES = M * (2 * K + K // 2 + 4)
# ... of sq_rotate_quant8: bf16 in, one byte per code out, f32 scale
RQ8_BYTES = M * (2 * K + K + 4)
# ... of sq_swiglu_rotate_quant: bf16 gate and up in, packed INT4 out, f32 scale
SWIGLU_BYTES = M * (2 * 2 * K + K // 2 + 4)
KV_T, KV_HQ, KV_HKV = 16 * 4096, 32, 8
# ... of one decode step of sq_kv4_decode_attention (B 16 x S 4096): both
# caches with their scales and zeros, bf16 queries in and outputs out
DECODE_BYTES = 2 * KV_T * KV_HKV * (64 + 4 + 1) + 2 * (16 * KV_HQ * 128 * 2)
# ... of sq_kv8_decode_attention: one byte per code
DECODE8_BYTES = 2 * KV_T * KV_HKV * (128 + 4 + 1) + 2 * (16 * KV_HQ * 128 * 2)
# Cayley R2 learner on the o_proj layer (2048 tokens, 32 heads of 128, 4096
# outputs).  Algorithmic work of one loss-and-gradient evaluation: the INT4
# product Q(xR) Q(wR)^T, the two straight-through gradient products E Q(wR)
# and E^T Q(xR) (tensor cores, float operand as two bf16 halves, so executed
# twice), and the float32 rotations and G
R2_T, R2_H, R2_D, R2_N = 2048, 32, 128, 4096
R2_K = R2_H * R2_D
R2_INT_OPS = 2 * R2_T * R2_N * R2_K
R2_GRAD_FLOPS = 2 * 2 * R2_T * R2_N * R2_K
R2_F32_FLOPS = 2 * (R2_T + R2_N) * R2_K * R2_D + 2 * (R2_T + R2_N) * R2_H * R2_D * R2_D
R2_ALPHA = 3.0      # step size: of 0.3, 1, 3 and 10 on this layer, 3 and 10 end lowest
METRIC = "W4A4 linear TOPS & rotate+quant GB/s at 1 B200; % of int8/HBM roofline"
# DRAM bytes (read + write) per launch from one ncu capture of the current
# kernels (profiles/w4a4_gemm_pair_ts_*.md, profiles/rotate_quant_h12x1024_tc_*.md);
# set to None whenever the kernel changes until it is captured again.
GEMM_TRAFFIC = 50544896 + 12481280
RQ_TRAFFIC = 100713984 + 5578496
WORKLOAD = "down_proj_M4096_K12288_N4096_R4_H12xH1024"


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            pk = json.load(f)
        return pk["hbm_gbs"], pk["bf16_tflops"], pk.get("bf16_tflops_sustained"), "measured"
    except Exception:
        return 6650.0, 1590.0, 1400.0, "fallback"


# ----------------------------------------------------------------- clocks

class ClockSampler:
    """Samples SM clock and throttle reasons while the timed region runs.

    NVML is polled from a background thread every 2 ms (nvidia-smi's own
    loop is too coarse for a region of a few tens of milliseconds).
    """
    REASONS = {"hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
               "sw_power_cap": 0x4}

    def __init__(self, index: int):
        self.index = index
        self.samples = []
        self.result = {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}

    def _run(self):
        import pynvml
        h = pynvml.nvmlDeviceGetHandleByIndex(self.index)
        while not self._stop.is_set():
            try:
                sm = pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM)
                rs = pynvml.nvmlDeviceGetCurrentClocksEventReasons(h)
                self.samples.append((sm, rs))
            except Exception:
                pass
            self._stop.wait(0.002)

    def __enter__(self):
        import threading
        self._stop = threading.Event()
        self._thread = None
        try:
            import pynvml
            pynvml.nvmlInit()
            h = pynvml.nvmlDeviceGetHandleByIndex(self.index)
            self.sm_max = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()
        except Exception:
            self._thread = None
        return self

    def __exit__(self, *a):
        if self._thread is None:
            return
        self._stop.set()
        self._thread.join(timeout=2)
        if not self.samples:
            return
        sm = [s for s, _ in self.samples]
        reasons = sorted({n for _, r in self.samples for n, bit in self.REASONS.items() if r & bit})
        self.result = {"sm_mhz": statistics.median(sm), "sm_max_mhz": self.sm_max,
                       "reasons": reasons, "samples": len(sm)}


# --------------------------------------------------------------- our arm

def run_ours(args, rank, world, local_rank):
    import numpy as np
    import torch
    import torch.distributed as dist

    import rotation_ptq_b200 as sq
    from rotation_ptq_b200 import shard
    from workloads import synthetic as W

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    # one model (the canonical weights) on every rank; each rank serves its
    # own M-token shard of the global batch (rank 0's is the 1-GPU workload)
    wl = W.down_proj(M=M, K=K, N=N)
    hs = sq.paley_h12()
    if rank == 0:
        x = wl.x.to(dev)
    else:
        x = W.down_proj(M=M, K=K, N=N, seed=shard.shard_seed(W.SEED_BASE + 1, rank),
                        with_weights=False).x.to(dev)
    w_q, w_s = sq.quantize_weights(wl.w.to(dev), hs, N_POW2)
    del wl
    a_q = torch.empty((M, K // 2), dtype=torch.uint8, device=dev)
    a_s = torch.empty((M,), dtype=torch.float32, device=dev)
    out = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)   # 2x the 126 MB L2
    stream = torch.cuda.current_stream(dev)

    def step():
        sq.rotate_quant(x, hs, N_POW2, 1.0, a_q=a_q, a_scale=a_s)
        sq.w4a4_linear(a_q, a_s, w_q, w_s, out=out)

    ev = lambda: torch.cuda.Event(enable_timing=True)  # noqa: E731
    for _ in range(args.warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    if sq.device_status() != 0:
        raise RuntimeError("device status set during warm-up")

    # timed region: K steps, L2 flushed between steps (outside the events)
    t_step, t_rq, t_gemm = [], [], []
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local_rank) as clk:
        for _ in range(args.steps):
            flush.zero_()
            e0, e1, e2 = ev(), ev(), ev()
            e0.record(stream)
            sq.rotate_quant(x, hs, N_POW2, 1.0, a_q=a_q, a_scale=a_s)
            e1.record(stream)
            sq.w4a4_linear(a_q, a_s, w_q, w_s, out=out)
            e2.record(stream)
            t_step.append((e0, e2))
            t_rq.append((e0, e1))
            t_gemm.append((e1, e2))
        torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    ms = lambda pairs: sum(a.elapsed_time(b) for a, b in pairs) / len(pairs)  # noqa: E731
    ms_step, ms_rq, ms_gemm = ms(t_step), ms(t_rq), ms(t_gemm)
    status = sq.device_status()

    # the R4 rotate+quant back to back over three copies of x (302 MB)
    xs = [x] + [x.clone() for _ in range(2)]
    us_rq_b2b = back_to_back_us([lambda xx=xx: sq.rotate_quant(xx, hs, N_POW2, 1.0, a_q=a_q,
                                                               a_scale=a_s) for xx in xs])
    del xs

    # e2e: pinned host input, H2D + path + D2H every step, device-timed
    x_host = x.cpu().pin_memory()
    out_host = torch.empty((M, N), dtype=torch.bfloat16).pin_memory()
    x_dev = torch.empty_like(x)
    for _ in range(2):
        x_dev.copy_(x_host, non_blocking=True)
        sq.rotate_quant(x_dev, hs, N_POW2, 1.0, a_q=a_q, a_scale=a_s)
        sq.w4a4_linear(a_q, a_s, w_q, w_s, out=out)
        out_host.copy_(out, non_blocking=True)
    torch.cuda.synchronize()
    e2e = []
    for _ in range(args.steps):
        e0, e1 = ev(), ev()
        e0.record(stream)
        x_dev.copy_(x_host, non_blocking=True)
        sq.rotate_quant(x_dev, hs, N_POW2, 1.0, a_q=a_q, a_scale=a_s)
        sq.w4a4_linear(a_q, a_s, w_q, w_s, out=out)
        out_host.copy_(out, non_blocking=True)
        e1.record(stream)
        e2e.append((e0, e1))
    torch.cuda.synchronize()
    ms_e2e = ms(e2e)

    # KV path (config of the R3 rows), timed alone for the record
    kv_info = None
    if not args.no_kv:
        kvw = W.kv_path()
        q, k, v, pos = kvw.q.to(dev), kvw.k.to(dev), kvw.v.to(dev), kvw.pos.to(dev)
        cos, sin = sq.rope_tables(kvw.theta, kvw.max_pos, 128, device=dev)
        kvo = sq.kv_rotate_quant(q, k, v, pos, cos, sin)
        kdq = sq.kv_dequant(kvo["k_cache"], kvo["k_scale"], kvo["k_zero"])
        vdq = sq.kv_dequant(kvo["v_cache"], kvo["v_scale"], kvo["v_zero"])
        torch.cuda.synchronize()
        tq, td = [], []
        for _ in range(max(3, args.steps)):
            flush.zero_()
            e0, e1, e2 = ev(), ev(), ev()
            e0.record(stream)
            sq.kv_rotate_quant(q, k, v, pos, cos, sin, out=kvo)
            e1.record(stream)
            sq.kv_dequant(kvo["k_cache"], kvo["k_scale"], kvo["k_zero"], out=kdq)
            sq.kv_dequant(kvo["v_cache"], kvo["v_scale"], kvo["v_zero"], out=vdq)
            e2.record(stream)
            tq.append((e0, e1))
            td.append((e1, e2))
        torch.cuda.synchronize()
        d = 128
        kv_fwd_bytes = KV_T * (2 * (KV_HQ * d * 2) + 2 * (KV_HKV * d * 2) + 2 * KV_HKV * (d // 2 + 5))
        kv_rb_bytes = 2 * KV_T * KV_HKV * ((d // 2 + 5) + d * 2)
        mq, md = ms(tq), ms(td)
        kv_info = {"workload": "kv_T65536_hq32_hkv8_d128", "rotate_quant_us": mq * 1e3,
                   "rotate_quant_gbs": kv_fwd_bytes / (mq * 1e-3) / 1e9,
                   "dequant_us": md * 1e3, "dequant_gbs": kv_rb_bytes / (md * 1e-3) / 1e9}
        # the same tokens into 8-bit caches (W4A8KV8) and their read-back
        kvo8 = sq.kv_rotate_quant8(q, k, v, pos, cos, sin)
        sq.kv8_dequant(kvo8["k_cache"], kvo8["k_scale"], kvo8["k_zero"], out=kdq)
        torch.cuda.synchronize()
        tq, td = [], []
        for _ in range(max(3, args.steps)):
            flush.zero_()
            e0, e1, e2 = ev(), ev(), ev()
            e0.record(stream)
            sq.kv_rotate_quant8(q, k, v, pos, cos, sin, out=kvo8)
            e1.record(stream)
            sq.kv8_dequant(kvo8["k_cache"], kvo8["k_scale"], kvo8["k_zero"], out=kdq)
            sq.kv8_dequant(kvo8["v_cache"], kvo8["v_scale"], kvo8["v_zero"], out=vdq)
            e2.record(stream)
            tq.append((e0, e1))
            td.append((e1, e2))
        torch.cuda.synchronize()
        kv8_fwd_bytes = KV_T * (2 * (KV_HQ * d * 2) + 2 * (KV_HKV * d * 2) + 2 * KV_HKV * (d + 5))
        kv8_rb_bytes = 2 * KV_T * KV_HKV * ((d + 5) + d * 2)
        mq, md = ms(tq), ms(td)
        kv_info["kv8"] = {"rotate_quant8_us": mq * 1e3,
                          "rotate_quant8_gbs": kv8_fwd_bytes / (mq * 1e-3) / 1e9,
                          "dequant8_us": md * 1e3,
                          "dequant8_gbs": kv8_rb_bytes / (md * 1e-3) / 1e9}
        del q, k, v, kvo, kdq, vdq, kvo8

    # fused SwiGLU + R4 rotate + quant on the gate_up output of the same
    # tokens (the step before down_proj), timed alone for the record
    sw_info = None
    if not args.no_kv:
        gu = W.gate_up_out(M=M, K=K).to(dev)
        sq.swiglu_rotate_quant(gu, hs, N_POW2, 1.0, a_q=a_q, a_scale=a_s)
        torch.cuda.synchronize()
        tsw = []
        for _ in range(max(3, args.steps)):
            flush.zero_()
            e0, e1 = ev(), ev()
            e0.record(stream)
            sq.swiglu_rotate_quant(gu, hs, N_POW2, 1.0, a_q=a_q, a_scale=a_s)
            e1.record(stream)
            tsw.append((e0, e1))
        torch.cuda.synchronize()
        msw = ms(tsw)
        sw_info = {"workload": "gate_up_out_M%d_K%d_swiglu_R4" % (M, K), "us": msw * 1e3,
                   "GB/s": SWIGLU_BYTES / (msw * 1e-3) / 1e9, "bytes": SWIGLU_BYTES}
        del gu

    # W4A8 on the same down_proj step: 8-bit rotate+quant, INT8 x INT4 GEMM
    a8_info = None
    if not args.no_kv:
        a8 = torch.empty((M, K), dtype=torch.int8, device=dev)
        out8 = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
        sq.rotate_quant8(x_dev, hs, N_POW2, 1.0, a_q=a8, a_scale=a_s)
        sq.w4a8_linear(a8, a_s, w_q, w_s, out=out8)
        torch.cuda.synchronize()
        tq8, tg8 = [], []
        for _ in range(max(3, args.steps)):
            flush.zero_()
            e0, e1, e2 = ev(), ev(), ev()
            e0.record(stream)
            sq.rotate_quant8(x_dev, hs, N_POW2, 1.0, a_q=a8, a_scale=a_s)
            e1.record(stream)
            sq.w4a8_linear(a8, a_s, w_q, w_s, out=out8)
            e2.record(stream)
            tq8.append((e0, e1))
            tg8.append((e1, e2))
        torch.cuda.synchronize()
        mq8, mg8 = ms(tq8), ms(tg8)
        a8_info = {"workload": WORKLOAD.replace("down_proj", "down_proj_W4A8"),
                   "rotate_quant8_us": mq8 * 1e3,
                   "rotate_quant8_GB/s": RQ8_BYTES / (mq8 * 1e-3) / 1e9,
                   "gemm_us": mg8 * 1e3, "gemm_TOPS": OPS / (mg8 * 1e-3) / 1e12,
                   "step_us": (mq8 + mg8) * 1e3}
        del a8, out8

    # one decode step of attention over 4-bit caches of the KV configuration
    dec_info = None
    if not args.no_kv:
        dw = W.kv4_decode()
        dq, dkc, dks, dkz = dw.q.to(dev), dw.k_cache.to(dev), dw.k_scale.to(dev), dw.k_zero.to(dev)
        dvc, dvs, dvz, dln = dw.v_cache.to(dev), dw.v_scale.to(dev), dw.v_zero.to(dev), dw.lengths.to(dev)
        dout = sq.kv4_decode_attention(dq, dkc, dks, dkz, dvc, dvs, dvz, dln, dw.S_max)
        torch.cuda.synchronize()
        tde = []
        for _ in range(max(3, args.steps)):
            flush.zero_()
            e0, e1 = ev(), ev()
            e0.record(stream)
            sq.kv4_decode_attention(dq, dkc, dks, dkz, dvc, dvs, dvz, dln, dw.S_max, out=dout)
            e1.record(stream)
            tde.append((e0, e1))
        torch.cuda.synchronize()
        mde = ms(tde)
        dec_bytes = DECODE_BYTES
        # back to back over four copies of the caches (290 MB)
        copies = [(dq, dkc, dks, dkz, dvc, dvs, dvz)] + \
            [tuple(t.clone() for t in (dq, dkc, dks, dkz, dvc, dvs, dvz)) for _ in range(3)]
        us_dec_b2b = back_to_back_us([
            lambda c=c: sq.kv4_decode_attention(*c, dln, dw.S_max, out=dout) for c in copies])
        del copies
        dec_info = {"workload": dw.name, "us": mde * 1e3,
                    "GB/s": dec_bytes / (mde * 1e-3) / 1e9, "bytes": dec_bytes,
                    "back_to_back": {"us": us_dec_b2b,
                                     "GB/s": dec_bytes / (us_dec_b2b * 1e-6) / 1e9,
                                     "how": "8 launches over 4 copies of the caches (290 MB) "
                                            "between one event pair"}}
        del dq, dkc, dks, dkz, dvc, dvs, dvz, dln, dout
        # the same step over 8-bit caches
        dw = W.kv8_decode()
        t8 = [x.to(dev) for x in (dw.q, dw.k_cache, dw.k_scale, dw.k_zero, dw.v_cache,
                                  dw.v_scale, dw.v_zero, dw.lengths)]
        dout = sq.kv8_decode_attention(*t8, dw.S_max)
        torch.cuda.synchronize()
        tde = []
        for _ in range(max(3, args.steps)):
            flush.zero_()
            e0, e1 = ev(), ev()
            e0.record(stream)
            sq.kv8_decode_attention(*t8, dw.S_max, out=dout)
            e1.record(stream)
            tde.append((e0, e1))
        torch.cuda.synchronize()
        mde = ms(tde)
        dec_info["kv8"] = {"workload": dw.name, "us": mde * 1e3,
                           "GB/s": DECODE8_BYTES / (mde * 1e-3) / 1e9, "bytes": DECODE8_BYTES,
                           "frac_of_hbm": DECODE8_BYTES / (mde * 1e-3) / 1e9 / load_peaks()[0]}
        del t8, dout

    # Cayley SGD for R2 on one o_proj layer: loss-and-gradient evaluations and
    # whole learner steps (loss, gradient and the float64 Cayley update)
    r2_info = None
    if not args.no_kv:
        ow = W.o_proj_layer()
        prob = sq.R2Problem(torch.from_numpy(ow.x).to(dev), torch.from_numpy(ow.w).to(dev), R2_H)
        starts = sq.r2_random_hadamard(torch.from_numpy(ow.signs).to(dev))   # [32, d, d]
        R0 = starts[0].contiguous()
        R32 = R0.float()
        prob.loss_grad(R32)
        torch.cuda.synchronize()
        tlg, tlearn = [], []
        iters = 10
        for _ in range(max(3, args.steps)):
            e0, e1, e2 = ev(), ev(), ev()
            e0.record(stream)
            prob.loss_grad(R32)
            e1.record(stream)
            prob.learn(R0, R2_ALPHA, iters)
            e2.record(stream)
            tlg.append((e0, e1))
            tlearn.append((e1, e2))
        torch.cuda.synchronize()
        mlg, mlearn = ms(tlg), ms(tlearn)
        # the learner as the page runs it: 120 steps from the first draw,
        # against all 32 draws
        draws = torch.cat([prob.loss_grad(starts[i].float(), grad=False)[0]
                           for i in range(starts.shape[0])]).cpu()
        R, losses = prob.learn(R0, R2_ALPHA, 120)
        L = losses.cpu()
        orth = float(sq.orth_error(R)[0])
        r2_info = {"workload": ow.name, "alpha": R2_ALPHA,
                   "loss_grad_us": mlg * 1e3,
                   "loss_grad_work": {"int4_gop": R2_INT_OPS / 1e9,
                                      "grad_products_gflop": R2_GRAD_FLOPS / 1e9,
                                      "f32_gflop": R2_F32_FLOPS / 1e9},
                   "learner_step_us": mlearn * 1e3 / iters,
                   "loss_first_draw": float(L[0]), "loss_after_120": float(L[-1]),
                   "best_of_32_draws": float(draws.min()), "worst_of_32_draws": float(draws.max()),
                   "learned_vs_best_draw": float(L[-1]) / float(draws.min()) - 1.0,
                   "orth_error_after_120": orth}
        del prob, starts
    # the R1-folded projections (M 8192, K 4096, N 4096 / 1024 / 12288) and
    # the decode-to-prefill M sweep, timed alone for the record
    r1_info = sweep_info = None
    if not args.no_kv:
        r1_info = r1_folded_record(dev, flush, args.steps)
        recs, peaks = sweep_records(min(args.steps, 10), 3)
        sweep_info = {"peaks": peaks, "points": recs}
    # max over ranks
    ms_step, ms_rq, ms_gemm, ms_e2e = shard.max_over_ranks([ms_step, ms_rq, ms_gemm, ms_e2e])
    return dict(ms_step=ms_step, ms_rq=ms_rq, ms_gemm=ms_gemm, ms_e2e=ms_e2e, status=status,
                clocks=clk.result, kv=kv_info, swiglu=sw_info, decode=dec_info, a8=a8_info,
                r2=r2_info, r1=r1_info, sweep=sweep_info, us_rq_b2b=us_rq_b2b)


# ------------------------------------------------------------ oracle arm

def oracle_sample(rows=64, cols=512, min_seconds=10.0, max_steps=None, prepared=None):
    """Time the CPU oracle on rows x cols of the workload; extrapolate one full step.

    The oracle's step is rotate+quant of x (cost per row) then the integer GEMM
    and dequant (cost per row x column).  Weight codes are prepared offline and
    not timed, as on the GPU side; `prepared` (the result's "prepared" entry)
    reuses them.
    """
    from oracle import oracle as O
    from workloads import synthetic as W

    if prepared is None:
        wl = W.down_proj(M=rows, K=K, N=cols, seed=1001)
        x = wl.x.double().numpy()
        wp, ws, _ = O.quantize_weights(wl.w.double().numpy(), N_SMALL, N_POW2)
        O.rotate_quant(x[:2], N_SMALL, N_POW2)      # builds and caches the dense H
        prepared = (x, wp, ws)
    x, wp, ws = prepared
    t_rot, t_gemm, n = 0.0, 0.0, 0
    t_start = time.perf_counter()
    while True:
        t0 = time.perf_counter()
        ap, sa, _, _ = O.rotate_quant(x, N_SMALL, N_POW2)
        t1 = time.perf_counter()
        O.w4a4_linear(ap, sa, wp, ws)
        t2 = time.perf_counter()
        t_rot += t1 - t0
        t_gemm += t2 - t1
        n += 1
        if time.perf_counter() - t_start >= min_seconds or (max_steps and n >= max_steps):
            break
    per_row = t_rot / n / rows
    per_cell = t_gemm / n / (rows * cols)
    full_s = per_row * M + per_cell * M * N
    try:
        from threadpoolctl import threadpool_info
        cores = max(i.get("num_threads", 1) for i in threadpool_info()) if threadpool_info() else 1
    except Exception:
        cores = os.cpu_count()
    return {"value": OPS / full_s / 1e12, "unit": "TOPS", "cores": int(cores), "kind": "oracle",
            "sample": "%d rows x %d cols of the workload, %d repetitions (%.1f s), extrapolated "
                      "to one full step (rotation cost per row, GEMM cost per row x col)"
                      % (rows, cols, n, t_rot + t_gemm), "full_step_s": full_s,
            "repetitions": n, "timed_s": t_rot + t_gemm, "prepared": prepared}


PROFILE_CASES = ("down_proj_gemm", "down_proj_gemm_1cta", "down_proj_gemm_pair",
                 "decode_gemm_m1", "decode_gemm_m16", "decode_gemm_m64", "rotate_quant_r4",
                 "kv_rotate_quant",
                 "swiglu_rotate_quant_r4", "kv4_decode", "kv8_decode", "kv_rotate_quant8",
                 "r2_loss_grad", "quant_only_r1", "kv_rotate_quant_t16k", "kv_rotate_quant8_t16k")


def run_profile_case(case, steps, warmup):
    """Launch one kernel of the path `warmup + steps` times (for ncu captures)."""
    import torch
    import rotation_ptq_b200 as sq
    from workloads import synthetic as W
    torch.cuda.set_device(0)
    if case.startswith("down_proj_gemm") or case.startswith("decode_gemm"):
        m = {"decode_gemm_m1": 1, "decode_gemm_m16": 16, "decode_gemm_m64": 64}.get(case, M)
        a = torch.from_numpy(W.random_packed(11, m, K)).cuda()
        w = torch.from_numpy(W.random_packed(12, N, K)).cuda()
        sa = torch.from_numpy(W.random_scales(13, m)).cuda()
        sw = torch.from_numpy(W.random_scales(14, N)).cuda()
        out = torch.empty((m, N), dtype=torch.bfloat16, device="cuda")
        sq.debug_set_gemm_path({"down_proj_gemm_1cta": 1, "down_proj_gemm_pair": 2}.get(case, 0))
        fn = lambda: sq.w4a4_linear(a, sa, w, sw, out=out)  # noqa: E731
    elif case == "rotate_quant_r4":
        x = W.down_proj(M=M, K=K, N=N, with_weights=False).x.cuda()
        hs = sq.paley_h12()
        a_q = torch.empty((M, K // 2), dtype=torch.uint8, device="cuda")
        a_s = torch.empty((M,), dtype=torch.float32, device="cuda")
        fn = lambda: sq.rotate_quant(x, hs, N_POW2, 1.0, a_q=a_q, a_scale=a_s)  # noqa: E731
    elif case == "quant_only_r1":
        # the R1-folded projections' input: M 8192, K 4096, no online rotation
        x = W.r1_folded(Ns=(16,))[0].x.cuda()
        a_q = torch.empty((x.shape[0], x.shape[1] // 2), dtype=torch.uint8, device="cuda")
        a_s = torch.empty((x.shape[0],), dtype=torch.float32, device="cuda")
        fn = lambda: sq.rotate_quant(x, None, 1, 1.0, a_q=a_q, a_scale=a_s)  # noqa: E731
    elif case == "swiglu_rotate_quant_r4":
        gu = W.gate_up_out(M=M, K=K).cuda()
        hs = sq.paley_h12()
        a_q = torch.empty((M, K // 2), dtype=torch.uint8, device="cuda")
        a_s = torch.empty((M,), dtype=torch.float32, device="cuda")
        fn = lambda: sq.swiglu_rotate_quant(gu, hs, N_POW2, 1.0, a_q=a_q, a_scale=a_s)  # noqa: E731
    elif case == "kv4_decode":
        dw = W.kv4_decode()
        t = [x.cuda() for x in (dw.q, dw.k_cache, dw.k_scale, dw.k_zero, dw.v_cache, dw.v_scale,
                                dw.v_zero, dw.lengths)]
        o = sq.kv4_decode_attention(*t, dw.S_max)
        fn = lambda: sq.kv4_decode_attention(*t, dw.S_max, out=o)  # noqa: E731
    elif case == "r2_loss_grad":
        ow = W.o_proj_layer()
        prob = sq.R2Problem(torch.from_numpy(ow.x).cuda(), torch.from_numpy(ow.w).cuda(), R2_H)
        R32 = sq.r2_random_hadamard(torch.from_numpy(ow.signs[:1]).cuda())[0].float()
        fn = lambda: prob.loss_grad(R32)  # noqa: E731
    elif case == "kv8_decode":
        dw = W.kv8_decode()
        t = [x.cuda() for x in (dw.q, dw.k_cache, dw.k_scale, dw.k_zero, dw.v_cache, dw.v_scale,
                                dw.v_zero, dw.lengths)]
        o = sq.kv8_decode_attention(*t, dw.S_max)
        fn = lambda: sq.kv8_decode_attention(*t, dw.S_max, out=o)  # noqa: E731
    elif case in ("kv_rotate_quant8", "kv_rotate_quant8_t16k"):
        kw = W.kv_path(batch=16 if case == "kv_rotate_quant8" else 4)
        q, k, v, pos = kw.q.cuda(), kw.k.cuda(), kw.v.cuda(), kw.pos.cuda()
        cos, sin = sq.rope_tables(kw.theta, kw.max_pos, 128)
        o = sq.kv_rotate_quant8(q, k, v, pos, cos, sin)
        fn = lambda: sq.kv_rotate_quant8(q, k, v, pos, cos, sin, out=o)  # noqa: E731
    elif case in ("kv_rotate_quant", "kv_rotate_quant_t16k"):
        kvw = W.kv_path(batch=16 if case == "kv_rotate_quant" else 4)
        q, k, v, pos = kvw.q.cuda(), kvw.k.cuda(), kvw.v.cuda(), kvw.pos.cuda()
        cos, sin = sq.rope_tables(kvw.theta, kvw.max_pos, 128)
        o = sq.kv_rotate_quant(q, k, v, pos, cos, sin)
        fn = lambda: sq.kv_rotate_quant(q, k, v, pos, cos, sin, out=o)  # noqa: E731
    else:
        raise SystemExit("unknown case %s" % case)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    for _ in range(warmup + steps):
        flush.zero_()
        fn()
    torch.cuda.synchronize()
    if sq.device_status() != 0:
        raise SystemExit("device status set")
    print("profile case %s: %d launches" % (case, warmup + steps))


SWEEP_M = (1, 4, 16, 64, 256, 1024, 4096, 16384)
SWEEP_SHAPES = (("down_proj", 12288, 4096), ("gate_up", 4096, 24576))


def back_to_back_us(calls, rounds=5):
    """Average launch duration with the launches back to back: `calls` (one
    per input copy, the copies together larger than the L2, so each launch
    finds its input evicted by the others) run twice over between one pair
    of CUDA events, after a 256 MB write; the median of `rounds` rounds.
    Unlike the single-launch events it excludes the launch latency of an
    idle stream, as in a model's forward, where kernels follow each other."""
    import statistics
    import torch
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    for c in calls:
        c()
    torch.cuda.synchronize()
    per = []
    for _ in range(rounds):
        flush.zero_()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _rep in range(2):
            for c in calls:
                c()
        e1.record()
        torch.cuda.synchronize()
        per.append(e0.elapsed_time(e1) * 1e3 / (2 * len(calls)))
    del flush
    return statistics.median(per)


def sweep_records(steps, warmup):
    """The decode-to-prefill M sweep of the W4A4 GEMM: one record per point.

    Operands are seeded random packed codes of the configuration's shapes;
    each point is timed with CUDA events over `steps` launches after `warmup`,
    the L2 flushed (256 MB write) before each and the device kept busy (a
    ~0.1 ms device sleep) while the host prepares the launch, so that the
    events bracket the kernel alone.  Bytes are the algorithmic
    operand + output bytes (packed weights N*K/2, packed activations M*K/2,
    scales 4(M+N), bf16 output 2MN); the roofline is the slower of the
    measured-HBM and int8-tensor times.  For M <= 64 the point is also timed
    as eight launches back to back in a CUDA graph, each on its own copy of
    the weights (8 copies exceed the L2), so that neither launch overhead nor
    a warm L2 enters the per-launch time.
    """
    import torch
    import rotation_ptq_b200 as sq
    from workloads import synthetic as W
    hbm, bf16, _, peak_src = load_peaks()
    int8_peak = 2.0 * bf16
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    recs = []
    for name, K, N in SWEEP_SHAPES:
        w = torch.from_numpy(W.random_packed(21, N, K)).cuda()
        sw = torch.from_numpy(W.random_scales(22, N)).cuda()
        for m in SWEEP_M:
            a = torch.from_numpy(W.random_packed(23 + m, m, K)).cuda()
            sa = torch.from_numpy(W.random_scales(24 + m, m)).cuda()
            out = torch.empty((m, N), dtype=torch.bfloat16, device="cuda")
            for _ in range(warmup):
                sq.w4a4_linear(a, sa, w, sw, out=out)
            torch.cuda.synchronize()
            times = []
            for _ in range(steps):
                flush.zero_()
                torch.cuda._sleep(200000)
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record()
                sq.w4a4_linear(a, sa, w, sw, out=out)
                e1.record()
                torch.cuda.synchronize()
                times.append(e0.elapsed_time(e1) * 1e-3)
            if sq.device_status() != 0:
                raise SystemExit("device status set")
            t = statistics.median(times)
            t_graph = None
            if m <= 64:
                copies = [w.clone() for _ in range(8)]
                for c in copies:
                    sq.w4a4_linear(a, sa, c, sw, out=out)
                torch.cuda.synchronize()
                g = torch.cuda.CUDAGraph()
                s_cap = torch.cuda.Stream()
                with torch.cuda.stream(s_cap):
                    with torch.cuda.graph(g, stream=s_cap):
                        for c in copies:
                            sq.w4a4_linear(a, sa, c, sw, out=out)
                g.replay()
                torch.cuda.synchronize()
                gt = []
                for _ in range(max(3, steps // 2)):
                    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                    e0.record()
                    g.replay()
                    e1.record()
                    torch.cuda.synchronize()
                    gt.append(e0.elapsed_time(e1) * 1e-3 / len(copies))
                t_graph = statistics.median(gt)
                del g, copies
            ops = 2.0 * m * N * K
            nbytes = N * K // 2 + m * K // 2 + 4 * (m + N) + 2 * m * N
            t_roof = max(nbytes / (hbm * 1e9), ops / (int8_peak * 1e12))
            recs.append({
                "sweep": name, "M": m, "K": K, "N": N, "us": t * 1e6,
                "TOPS": ops / t / 1e12, "GB/s": nbytes / t / 1e9,
                "bound": "hbm" if nbytes / (hbm * 1e9) >= ops / (int8_peak * 1e12) else "tensor",
                "roofline_us": t_roof * 1e6, "frac": t_roof / t,
                "graph_us": t_graph * 1e6 if t_graph else None,
                "graph_frac": t_roof / t_graph if t_graph else None})
            del a, sa, out
        del w, sw
    del flush
    return recs, "%s HBM %.1f GB/s, int8 %.0f TOPS" % (peak_src, hbm, int8_peak)


def run_sweep(steps, warmup):
    """--sweep: the M sweep alone, one JSON line per point."""
    import torch
    torch.cuda.set_device(0)
    recs, peaks = sweep_records(steps, warmup)
    for r in recs:
        print(json.dumps(dict(r, peaks=peaks)), flush=True)


def r1_folded_record(dev, flush, steps):
    """The R1-folded projections at hidden 4096 (M 8192 tokens, K 4096): the
    quant-only sq_rotate_quant of the activations (no online rotation: R1 is
    folded into the weights), then the W4A4 GEMM for N = 4096 (q, o), 1024
    (k, v) and 12288 (gate, up), weights folded and quantized offline."""
    import torch
    import rotation_ptq_b200 as sq
    from workloads import synthetic as W
    hbm, bf16, _, _ = load_peaks()
    int8_peak = 2.0 * bf16
    wls = W.r1_folded()
    x = wls[0].x.to(dev)
    Mr, Kr = x.shape
    a_q = torch.empty((Mr, Kr // 2), dtype=torch.uint8, device=dev)
    a_s = torch.empty((Mr,), dtype=torch.float32, device=dev)
    ev = lambda: torch.cuda.Event(enable_timing=True)  # noqa: E731
    sq.rotate_quant(x, None, 1, 1.0, a_q=a_q, a_scale=a_s)
    torch.cuda.synchronize()
    tq = []
    for _ in range(max(3, steps)):
        flush.zero_()
        e0, e1 = ev(), ev()
        e0.record()
        sq.rotate_quant(x, None, 1, 1.0, a_q=a_q, a_scale=a_s)
        e1.record()
        tq.append((e0, e1))
    torch.cuda.synchronize()
    mq = sum(a.elapsed_time(b) for a, b in tq) / len(tq)
    q_bytes = Mr * (2 * Kr + Kr // 2 + 4)
    xs = [x] + [x.clone() for _ in range(3)]
    us_b2b = back_to_back_us([lambda xx=xx: sq.rotate_quant(xx, None, 1, 1.0, a_q=a_q, a_scale=a_s)
                              for xx in xs])
    del xs
    rec = {"workload": "r1_folded_M%d_K%d" % (Mr, Kr),
           "rotate_quant": {"us": mq * 1e3, "GB/s": q_bytes / (mq * 1e-3) / 1e9,
                            "frac_of_hbm": q_bytes / (mq * 1e-3) / 1e9 / hbm, "bytes": q_bytes,
                            "back_to_back": {"us": us_b2b,
                                             "frac_of_hbm": q_bytes / (us_b2b * 1e-6) / 1e9 / hbm,
                                             "how": "8 launches over 4 copies of x (268 MB) "
                                                    "between one event pair"}},
           "gemm": []}
    for wl in wls:
        wq, ws = sq.quantize_weights(wl.w.to(dev), None, 1)
        out = torch.empty((Mr, wl.N), dtype=torch.bfloat16, device=dev)
        for _ in range(3):
            sq.w4a4_linear(a_q, a_s, wq, ws, out=out)
        torch.cuda.synchronize()
        tg = []
        for _ in range(max(3, steps)):
            flush.zero_()
            e0, e1 = ev(), ev()
            e0.record()
            sq.w4a4_linear(a_q, a_s, wq, ws, out=out)
            e1.record()
            tg.append((e0, e1))
        torch.cuda.synchronize()
        mg = sum(a.elapsed_time(b) for a, b in tg) / len(tg)
        ops = 2.0 * Mr * wl.N * Kr
        tops = ops / (mg * 1e-3) / 1e12
        rec["gemm"].append({"N": wl.N, "us": mg * 1e3, "TOPS": tops,
                            "frac_of_int8_peak": tops / int8_peak})
        del wq, ws, out
    if sq.device_status() != 0:
        raise RuntimeError("device status set in the R1-folded record")
    del x, a_q, a_s, wls
    return rec


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-kv", action="store_true")
    ap.add_argument("--sweep", action="store_true",
                    help="time the GEMM over the decode-to-prefill M sweep and exit")
    ap.add_argument("--profile-case", choices=PROFILE_CASES, default=None,
                    help="launch one kernel of the path warmup+steps times and exit (for ncu)")
    args = ap.parse_args()
    if args.profile_case:
        run_profile_case(args.profile_case, args.steps, args.warmup)
        return
    if args.sweep:
        run_sweep(min(args.steps, 20), max(args.warmup, 3))
        return
    args.warmup = max(args.warmup, 3)

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    hbm, bf16, bf16_sus, peak_src = load_peaks()
    int8_peak = 2.0 * bf16            # nominal dense int8 : bf16 ratio is 2 (4.5 : 2.25 PFLOP/s)

    if args.impl == "reference":
        if rank != 0:
            return
        cb = oracle_sample(min_seconds=max(10.0, 2.0 * args.steps), max_steps=None)
        line = {"impl": "reference", "metric": METRIC, "value": cb["value"], "unit": "TOPS",
                "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
                "ms_per_step": cb["full_step_s"] * 1e3, "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "f64",
                "data": "synthetic (seeded numpy; Qwen3-8B down_proj shape)",
                "config": {"workload": WORKLOAD, "M": M, "K": K, "N": N},
                "cpu_baseline": {k: cb[k] for k in ("value", "unit", "cores", "kind", "sample")},
                "e2e": {"value": cb["value"], "unit": "TOPS", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0},
                # no full step is timed: ms_per_step is the sample's cost scaled
                # to one step, not a measured region
                "extrapolated": True,
                "timed": {"repetitions": cb["repetitions"], "seconds": cb["timed_s"],
                          "rows": 64, "cols": 512}}
        print(json.dumps(line), flush=True)
        return

    import torch
    import torch.distributed as dist
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    try:
        r = run_ours(args, rank, world, local_rank)
    finally:
        if world > 1:
            dist.destroy_process_group()
    if rank != 0:
        return
    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        cb = oracle_sample()
        cpu = {k: cb[k] for k in ("value", "unit", "cores", "kind", "sample")}
        # the same sample on one host thread (the BLAS pool limited to 1)
        try:
            from threadpoolctl import threadpool_limits
            with threadpool_limits(limits=1):
                one = oracle_sample(min_seconds=5.0, prepared=cb["prepared"])
            cpu["one_thread"] = {"value": one["value"], "unit": "TOPS", "cores": 1,
                                 "sample": one["sample"]}
        except ImportError:
            pass
    from rotation_ptq_b200.shard import job_rate
    # whole job: every rank's M tokens over the slowest rank's step time
    tops_job = job_rate(world * OPS, r["ms_step"] * 1e-3) / 1e12
    tops_gemm = OPS / (r["ms_gemm"] * 1e-3) / 1e12
    gbs_rq = RQ_BYTES / (r["ms_rq"] * 1e-3) / 1e9
    tops_e2e_job = job_rate(world * OPS, r["ms_e2e"] * 1e-3) / 1e12
    line = {
        "metric": METRIC, "value": tops_job, "unit": "TOPS", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": r["ms_step"],
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "int4",
        "data": "synthetic (seeded numpy; SwiGLU of Student-t(3) + 8 outlier channels, "
                "W ~ N(0, 0.02); Qwen3-8B down_proj shape)",
        "config": {"workload": WORKLOAD, "M": M, "K": K, "N": N, "tokens_per_gpu": M,
                   "parallelism": "replicas (token-sharded, no collective)" if world > 1 else "1 GPU",
                   "l2": "flushed (256 MB write) between timed steps"},
        "kernels": {
            "rotate_quant": {"us": r["ms_rq"] * 1e3, "GB/s": gbs_rq,
                             "frac_of_hbm": gbs_rq / hbm, "bytes": RQ_BYTES,
                             "back_to_back": {"us": r["us_rq_b2b"],
                                              "frac_of_hbm": RQ_BYTES / (r["us_rq_b2b"] * 1e-6) / 1e9 / hbm,
                                              "how": "6 launches over 3 copies of x (302 MB) "
                                                     "between one event pair"}},
            "w4a4_gemm": {"us": r["ms_gemm"] * 1e3, "TOPS": tops_gemm,
                          "frac_of_int8_peak": tops_gemm * 1e12 / (int8_peak * 1e12)},
            "kv_path": r["kv"],
            "swiglu_rotate_quant": (dict(r["swiglu"], frac_of_hbm=r["swiglu"]["GB/s"] / hbm)
                                    if r["swiglu"] else None),
            "kv4_decode_attention": (dict(r["decode"], frac_of_hbm=r["decode"]["GB/s"] / hbm)
                                     if r["decode"] else None),
            "w4a8": (dict(r["a8"], rotate_quant8_frac_of_hbm=r["a8"]["rotate_quant8_GB/s"] / hbm,
                          gemm_frac_of_int8_peak=r["a8"]["gemm_TOPS"] / int8_peak)
                     if r["a8"] else None),
            "r2_cayley_learner": r["r2"],
            "r1_folded": r["r1"],
            "m_sweep": r["sweep"],
        },
        "roofline": {"bound": "tensor", "achieved": tops_gemm, "peak": int8_peak,
                     "unit": "TOPS", "frac": tops_gemm / int8_peak, "traffic": GEMM_TRAFFIC,
                     "kernel": "w4a4_gemm_pair_ts_kernel",
                     "peak_source": "%s bf16 %.1f TFLOP/s x 2 (nominal int8/bf16)" % (peak_src, bf16)},
        "roofline_rotate_quant": {"bound": "hbm", "achieved": gbs_rq, "peak": hbm, "unit": "GB/s",
                                  "frac": gbs_rq / hbm, "traffic": RQ_TRAFFIC,
                                  "peak_source": peak_src + " copy bandwidth"},
        "cpu_baseline": cpu,
        "e2e": {"value": tops_e2e_job, "unit": "TOPS", "h2d_bytes_per_step": M * K * 2,
                "d2h_bytes_per_step": M * N * 2},
        "gpu_launches": 2 * args.steps,
        "clocks": r["clocks"],
        "device_status": r["status"],
    }
    print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
