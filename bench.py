#!/usr/bin/env python3
"""Benchmark of one MLA decode step (rope_append -> absorb_q -> decode -> up_v)
on the DeepSeek-V2 decode workload, printed as one JSON line.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload v2_decode|varlen|long|multi_token|tiny|prefill_chunk|prefill]

N > 1 runs under torch.distributed.run, one process per GPU.  Sequences are
independent, so every rank runs its own full copy of the workload (weak scaling)
with no data-path collective; the process group is only used for the barrier
around the timed region and the max-over-ranks of the device time.

--impl reference times the fp64 CPU oracle on rank 0 on a bounded sample of the
same workload (a few heads of one sequence per step).
"""

from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "MLA decode tokens/s + achieved HBM TB/s & TFLOP/s vs roofline (1×B200)"
L2_FLUSH_BYTES = 256 << 20
ALU_CLOCK_GHZ = 1.965   # B200 clocks.max.sm
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="v2_decode")
    ap.add_argument("--kernel-impl", type=int, default=0, help="mla_config_t.impl (0 auto)")
    ap.add_argument("--max-splits", type=int, default=0)
    ap.add_argument("--fold", action="store_true",
                    help="the step with the folded projections: c^Q -> q_abs with W^UK folded into W^UQ, and "
                         "latent -> u with W^UV folded into W^O (the model width)")
    ap.add_argument("--cache", choices=["bf16", "e4m3"], default="bf16",
                    help="latent cache format: bf16 rows, or the low-bit e4m3 rows (portable decode kernel)")
    ap.add_argument("--yarn", action="store_true",
                    help="YaRN-scaled RoPE on k^R (s = 40, alpha = 1, beta = 32, 4K training length) "
                         "and its attention temperature in the score scale")
    return ap.parse_args()


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


class Ranks:
    """Barrier and max-over-ranks on the process group (pg None: one process).

    Every rank calls the same methods in the same order; the reduction runs
    on `device` (the rank's GPU under NCCL, the CPU under gloo)."""

    def __init__(self, pg, device):
        self.pg, self.device = pg, device

    def barrier(self):
        if self.pg is not None:
            self.pg.barrier()

    def max(self, x: float) -> float:
        if self.pg is None:
            return float(x)
        import torch
        t = torch.tensor([float(x)], dtype=torch.float64, device=self.device)
        self.pg.all_reduce(t, op=self.pg.ReduceOp.MAX)
        return float(t.item())


def aggregate_rate(world: int, units_per_step_per_rank: int, steps: int, max_ms: float) -> float:
    """Whole-job units per second: every rank processes its own copy of the
    workload, and the job takes as long as its slowest rank."""
    return world * units_per_step_per_rank * steps / (max_ms / 1e3)


# ---------------------------------------------------------------------------
# clocks during the timed region (NVML polling thread)
# ---------------------------------------------------------------------------

class ClockSampler:
    REASONS = {
        "gpu_idle": 0x1, "applications_clocks_setting": 0x2, "sw_power_cap": 0x4,
        "hw_slowdown": 0x8, "sync_boost": 0x10, "sw_thermal_slowdown": 0x20,
        "hw_thermal_slowdown": 0x40, "hw_power_brake_slowdown": 0x80,
        "display_clock_setting": 0x100,
    }

    def __init__(self, index):
        self.samples, self.reasons, self.ok = [], 0, False
        self.max_mhz = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.ok = False
        self._stop = threading.Event()

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                self.reasons |= int(self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h))
            except Exception:
                pass
            time.sleep(0.001)

    def __enter__(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
            time.sleep(0.002)   # the first samples precede the timed work
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self.ok:
            self.t.join()

    def summary(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0}
        names = [k for k, v in self.REASONS.items() if self.reasons & v and k != "gpu_idle"]
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": names, "samples": len(self.samples)}


# ---------------------------------------------------------------------------
# the oracle arm
# ---------------------------------------------------------------------------

# YaRN parameters of the long-context extension (4K -> 128K on k^R)
YARN = dict(s=40.0, alpha=1.0, beta=32.0, orig_len=4096, coeff=0.0707)


def oracle_sample_rate(spec, steps, warmup, heads_per_step=8, budget_s=None, yarn=False, cache="bf16"):
    """Time the fp64 oracle on `heads_per_step` heads of one sequence per step.

    Returns (tokens/s, seconds, description).  A token's output needs all n_h
    heads, so a step credits heads_per_step / n_h of each of its T_q tokens."""
    from oracle.evaluate import reference
    kw = {"cache": cache}
    if yarn:
        from oracle import mla_oracle as O
        kw.update(inv_freq=O.yarn_inv_freq(spec.d_r, s=YARN["s"], alpha=YARN["alpha"], beta=YARN["beta"],
                                           orig_len=YARN["orig_len"]),
                  scale=O.yarn_score_scale(spec.d_h, spec.d_r, s=YARN["s"], coeff=YARN["coeff"]))
    b = 0
    heads_all = list(range(spec.n_h))
    heads_per_step = min(heads_per_step, spec.n_h)
    done_heads, t_total, k = 0, 0.0, 0
    for i in range(warmup + steps):
        hs = [heads_all[(i * heads_per_step + j) % spec.n_h] for j in range(heads_per_step)]
        t0 = time.perf_counter()
        reference(spec, b, heads=hs, **kw)
        dt = time.perf_counter() - t0
        if i >= warmup:
            t_total += dt
            done_heads += len(hs)
            k += 1
            if budget_s is not None and t_total > budget_s:
                break
    tokens = done_heads / spec.n_h * spec.T_q
    desc = (f"{k} steps x {heads_per_step} of {spec.n_h} heads of sequence {b} "
            f"(context {int(spec.seq_lens[b])}, T_q={spec.T_q}), explicit K/V reconstruction in fp64")
    return tokens / t_total, t_total, desc


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else os.cpu_count()
    except Exception:
        return os.cpu_count()


def bench_config(spec, args, world):
    """The workload description both arms print (the same keys and values)."""
    return {"workload": spec.name, "B": spec.B, "T_q": spec.T_q, "n_h": spec.n_h,
            "d_c": spec.d_c, "d_r": spec.d_r, "block_size": spec.block_size,
            "context": [int(spec.seq_lens.min()), int(spec.seq_lens.max())],
            "l2": f"flushed between steps ({L2_FLUSH_BYTES >> 20} MiB write)",
            "parallelism": f"replicas x{world}", "rope": "yarn" if args.yarn else "plain",
            "projections": "folded" if args.fold else "per head", "cache": args.cache}


def run_reference(args):
    world, rank, _ = dist_env()
    if rank != 0:
        return 0
    from mla_latent_kv_38_b200.workloads import workload_specs
    spec = workload_specs()[args.workload]
    rate, secs, desc = oracle_sample_rate(spec, args.steps, args.warmup, yarn=args.yarn, cache=args.cache)
    line = {
        "metric": METRIC, "impl": "reference", "value": rate, "unit": "tokens/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * secs / max(args.steps, 1), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": bench_config(spec, args, world),
        "cpu_baseline": {"value": rate, "unit": "tokens/s", "cores": blas_threads(),
                         "kind": "oracle", "sample": desc},
        "e2e": {"value": rate, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line))
    return 0


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------

DECODE_SOURCES = ("common.cuh", "sm100_decode.cu", "sm100_decode.h", "sm100_ptx.cuh", "tensor_map.h")


def decode_source_hash():
    """Hash of the sources the tcgen05 decode kernels are built from."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "mla_latent_kv_38_b200", "csrc")
    for f in DECODE_SOURCES:
        with open(os.path.join(csrc, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def profiled_traffic(workload, kernel_hash):
    """DRAM bytes per decode launch from the committed ncu summary, if it was
    taken on the current decode kernel sources; else None."""
    p = os.path.join(ROOT, "profiles", "decode_traffic.txt")
    if not os.path.exists(p):
        return None
    for line in open(p):
        parts = line.split("#")[0].split()
        if len(parts) == 3 and parts[0] == workload and parts[1] == kernel_hash:
            return int(parts[2])
    return None


def run_ours(args):
    import torch
    world, rank, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    pg = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)
        pg = dist
    from mla_latent_kv_38_b200 import binding as M
    from mla_latent_kv_38_b200.runner import DeviceCase
    from mla_latent_kv_38_b200.workloads import workload_specs

    spec = workload_specs()[args.workload]
    dc = DeviceCase(spec, impl=args.kernel_impl, max_splits=args.max_splits, device=f"cuda:{local}",
                    yarn=YARN if args.yarn else None, cache=args.cache)
    stream = torch.cuda.current_stream(dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    if args.cache == "bf16":
        launches_decode = M.mla_decode_launches(dc.cfg, spec.B, spec.T_q, args.max_splits)
    else:   # the portable kernel (and its merge when the rows are split)
        portable = M.MlaConfig(spec.n_h, spec.d_c, spec.d_h, spec.d_r, spec.block_size, dc.cfg.scale, M.IMPL_SIMT)
        launches_decode = M.mla_decode_launches(portable, spec.B, spec.T_q, args.max_splits)
    launches_per_step = 3 + launches_decode       # absorb_q, rope_append, up_v + decode
    fold = None
    if args.fold:
        # the folded weights, once (not timed), and the step's other ends: the
        # query latent in, the model-width output out
        def bits(a):
            return torch.from_numpy(np.ascontiguousarray(a)).view(torch.bfloat16).to(dev)
        fold = {"F": torch.empty((spec.n_h, spec.d_c, spec.d_cq), dtype=torch.bfloat16, device=dev),
                "G": torch.empty((spec.d_model, spec.n_h, spec.d_c), dtype=torch.bfloat16, device=dev),
                "h_c_q": spec.c_q()}
        fold["c_q"] = bits(fold["h_c_q"])
        fold["u"] = torch.empty((spec.n_tok, spec.d_model), dtype=torch.bfloat16, device=dev)
        fold["ws"] = torch.zeros(M.mla_up_o_folded_workspace_bytes(dc.cfg, spec.d_model, spec.n_tok),
                                 dtype=torch.uint8, device=dev)
        M.mla_fold_weights(dc.cfg, spec.d_cq, spec.d_model, bits(spec.w_uq()), dc.w_uk, dc.w_uv, bits(spec.w_o()),
                           fold["F"], fold["G"])
        launches_per_step += 1                    # the output side adds its partials in a second kernel

    def first_call(q_in, st=None):
        if fold is None:
            M.mla_absorb_q(dc.cfg, q_in, dc.w_uk, dc.q_abs, spec.n_tok, dc.status, st)
        else:
            M.mla_absorb_q_folded(dc.cfg, spec.d_cq, q_in, fold["F"], dc.q_abs, spec.n_tok, dc.status, st)

    def last_call(out, st=None):
        if fold is None:
            M.mla_up_v(dc.cfg, dc.latent, dc.w_uv, out, spec.n_tok, dc.status, st)
        else:
            M.mla_up_o_folded(dc.cfg, spec.d_model, dc.latent, fold["G"], out, spec.n_tok, fold["ws"], dc.status,
                              st)

    q_in = dc.q_c if fold is None else fold["c_q"]
    step_out = dc.out if fold is None else fold["u"]

    ranks = Ranks(pg, dev)
    barrier, max_over_ranks = ranks.barrier, ranks.max

    # warm-up
    for _ in range(max(args.warmup, 3)):
        dc.reset_step_inputs()
        dc.rope_append()
        first_call(q_in)
        dc.decode_only()
        last_call(step_out)
    torch.cuda.synchronize(dev)
    st = dc.decode_status() | dc.append_status()
    if st:
        raise RuntimeError(f"device status {st} after warm-up")

    K = args.steps
    s = dc.spec

    def step_inputs():
        flush.zero_()                             # L2 flush, outside the timed events
        dc.q_r.copy_(dc.q_r_pre)

    def absorb():
        first_call(q_in)

    def rope_append():
        dc.rope_append()

    def up_v():
        last_call(step_out)

    # The device-timed passes replay the library calls from CUDA graphs
    # (captured from the same C-ABI calls), so that the host's enqueueing
    # (ctypes, argument checks, tensor-map encoding) never leaves the GPU
    # idle inside the timed region; the end-to-end pass below calls the API
    # directly.
    def capture(*fns):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for fn in fns:
                fn()
        return g

    def dec():
        dc.decode_only()

    # RoPE + append goes first: it and absorb_q read disjoint inputs, and
    # absorb_q's CTAs fetch their weight tiles while the append runs.
    step_inputs()
    g_step = capture(rope_append, absorb, dec, up_v)
    g_calls = [capture(fn) for fn in (rope_append, absorb, dec, up_v)]
    torch.cuda.synchronize(dev)

    sampler = ClockSampler(local)
    sampler.__enter__()
    # Pass 1, the headline: whole steps, the four calls back to back (each
    # kernel's launch overlaps the end of the one before it).
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(K)]
    barrier()
    torch.cuda.synchronize(dev)
    for k in range(K):
        step_inputs()
        ev[k][0].record(stream)
        g_step.replay()
        ev[k][1].record(stream)
    torch.cuda.synchronize(dev)
    barrier()
    step_each = [e[0].elapsed_time(e[1]) for e in ev]
    step_ms = sum(step_each)

    # Pass 2: the same steps with an event after every call, for the time of
    # each call (the decode call's time is the roofline's denominator).  The
    # events stop the launch overlap between the calls.
    evp = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(K)]
    barrier()
    torch.cuda.synchronize(dev)
    for k in range(K):
        step_inputs()
        evp[k][0].record(stream)
        for j, g in enumerate(g_calls):
            g.replay()
            evp[k][j + 1].record(stream)
    torch.cuda.synchronize(dev)
    barrier()
    names = (["rope_append", "absorb_q", "decode", "up_v"] if fold is None else
             ["rope_append", "absorb_q_folded", "decode", "up_o_folded"])
    phases = {n: [1e3 * e[j].elapsed_time(e[j + 1]) for e in evp] for j, n in enumerate(names)}
    phases_us = {n: sum(v) / K for n, v in phases.items()}
    phases_med_us = {n: statistics.median(v) for n, v in phases.items()}
    decode_ms = phases_us["decode"] / 1e3
    step_ms = max_over_ranks(step_ms)
    del g_step, g_calls
    tokens_per_step = spec.n_tok
    value = aggregate_rate(world, tokens_per_step, K, step_ms)

    # End to end through the public API with host buffers: every step copies its
    # inputs (query parts, new cache rows, positions) from one pinned host
    # staging buffer into a device buffer, runs the four calls on views of it,
    # and copies the head output back.  Steps are pipelined the way a serving
    # loop would run them: step k + 1's inputs go up on an upload stream while
    # step k computes, and step k's output comes back on a read-back stream;
    # inputs and outputs are double-buffered and ordered by events.  No L2 flush runs
    # here (it would sit inside the timed region); the cache alone is larger
    # than L2.
    h_q_in = dc.h_q_c if fold is None else fold["h_c_q"]
    parts = [a.view(np.uint8).reshape(-1) for a in
             (h_q_in, dc.h_q_r, dc.h_k_r_new, dc.h_c_kv_new, dc.h_positions)]
    offs, tot = [], 0
    for a in parts:
        offs.append(tot)
        tot += (a.size + 255) // 256 * 256
    h_stage = torch.zeros(tot, dtype=torch.uint8).pin_memory()
    for a, o in zip(parts, offs):
        h_stage[o:o + a.size].copy_(torch.from_numpy(a))
    d_stage = [torch.empty(tot, dtype=torch.uint8, device=dev) for _ in range(2)]
    d_out = [torch.empty_like(step_out) for _ in range(2)]
    h_out = [torch.empty(step_out.shape, dtype=torch.bfloat16).pin_memory() for _ in range(2)]

    def view(i, j, like):
        n = like.numel() * like.element_size()
        return d_stage[i][offs[j]:offs[j] + n].view(like.dtype).view(like.shape)

    views = [tuple(view(i, j, t) for j, t in enumerate((q_in, dc.q_r, dc.k_r_new, dc.c_kv_new, dc.positions)))
             for i in range(2)]
    h2d = sum(a.size for a in parts)
    d2h = h_out[0].numel() * 2
    # Copies go through cudaMemcpyAsync on raw stream handles (no Python
    # stream contexts on the host's path); uploads and read-backs have a
    # stream each, so step k + 1's upload is not queued behind step k's
    # read-back.
    import ctypes
    cudart = ctypes.CDLL("libcudart.so.12")
    cudart.cudaMemcpyAsync.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int,
                                       ctypes.c_void_p]
    s_up, s_down = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    h_up, h_down, h_st = s_up.cuda_stream, s_down.cuda_stream, stream.cuda_stream
    h_stage_p = h_stage.data_ptr()
    d_stage_p = [t.data_ptr() for t in d_stage]
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_done = [torch.cuda.Event() for _ in range(2)]
    ev_read = [torch.cuda.Event() for _ in range(2)]
    append_fn = M.mla_rope_append if args.cache == "bf16" else M.mla_rope_append_e4m3
    decode_fn = M.mla_decode if args.cache == "bf16" else M.mla_decode_e4m3
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize(dev)
    barrier()
    e0.record(stream)
    s_up.wait_event(e0)
    h0 = time.perf_counter()
    for k in range(K):
        i = k % 2
        v_q_c, v_q_r, v_k_r, v_c_kv, v_pos = views[i]
        if k >= 2:
            s_up.wait_event(ev_done[i])       # step k - 2 is done with this staging buffer
        cudart.cudaMemcpyAsync(d_stage_p[i], h_stage_p, tot, 1, h_up)            # host -> device
        ev_in[i].record(s_up)
        stream.wait_event(ev_in[i])
        if k >= 2:
            stream.wait_event(ev_read[i])     # step k - 2's output has been read back
        append_fn(dc.cfg, v_q_r, v_k_r, v_c_kv, v_pos, dc.rope_table, dc.max_pos, dc.block_table,
                  s.max_blocks, dc.pool, s.num_blocks, s.B, s.T_q, dc.status, h_st)
        first_call(v_q_c, h_st)
        decode_fn(dc.cfg, dc.q_abs, v_q_r, dc.pool, s.num_blocks, dc.block_table, s.max_blocks, dc.seq_lens,
                  s.B, s.T_q, dc.max_splits, dc.ws, dc.ws_bytes, dc.latent, dc.lse, h_st)
        last_call(d_out[i], h_st)
        ev_done[i].record(stream)
        s_down.wait_event(ev_done[i])
        cudart.cudaMemcpyAsync(h_out[i].data_ptr(), d_out[i].data_ptr(), d2h, 2, h_down)   # device -> host
        ev_read[i].record(s_down)
    host_s = time.perf_counter() - h0
    e1.record(s_down)
    torch.cuda.synchronize(dev)
    e2e_ms = e0.elapsed_time(e1)
    e2e_ms = max_over_ranks(e2e_ms)
    e2e_value = aggregate_rate(world, tokens_per_step, K, e2e_ms)

    peaks, peak_src = load_peaks()
    row_bytes = None if args.cache == "bf16" else M.mla_e4m3_row_bytes(spec.d_c, spec.d_r)
    bytes_alg = spec.algorithmic_bytes(row_bytes=row_bytes)
    flops_alg = spec.algorithmic_flops()
    dec_s = decode_ms / 1e3
    hbm_gbs = bytes_alg / dec_s / 1e9
    tflops = flops_alg / dec_s / 1e12
    t_hbm = bytes_alg / (peaks["hbm_gbs"] * 1e9)
    t_tc = flops_alg / (peaks["bf16_tflops"] * 1e12)
    bound = "hbm" if t_hbm >= t_tc else "tensor"
    if args.cache == "e4m3":
        # the portable kernel: float32 FMAs on the CUDA cores, 148 SMs x 128
        # lanes x 2 FLOP per cycle at the highest SM clock
        alu_tflops = 148 * 128 * 2 * ALU_CLOCK_GHZ / 1e3
        t_alu = flops_alg / (alu_tflops * 1e12)
        roof = {"bound": "alu", "achieved": tflops, "peak": alu_tflops, "unit": "TFLOP/s",
                "frac": tflops / alu_tflops, "hbm_frac": hbm_gbs / peaks["hbm_gbs"]}
        t_tc = max(t_tc, t_alu)
    elif bound == "hbm":
        roof = {"bound": "hbm", "achieved": hbm_gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": hbm_gbs / peaks["hbm_gbs"]}
    else:
        roof = {"bound": "tensor", "achieved": tflops, "peak": peaks["bf16_tflops"],
                "unit": "TFLOP/s", "frac": tflops / peaks["bf16_tflops"]}
    khash = decode_source_hash()
    roof["traffic"] = profiled_traffic(args.workload, khash) if args.cache == "bf16" else None
    roof["peak_source"] = f"MEASURED_PEAKS.json ({peak_src})"
    roof["kernel"] = ("mla_decode (decode + split merge)" if args.cache == "bf16" else
                      "mla_decode_e4m3 (portable decode + split merge)")
    roof["roofline_time_us"] = 1e6 * max(t_hbm, t_tc)
    roof["decode_us"] = decode_ms * 1e3
    fold_line = None
    if fold is not None:
        # the folded products against the HBM peak: the weights once plus activations and outputs
        n_tok = spec.n_tok
        q_bytes = spec.n_h * spec.d_c * spec.d_cq * 2 + n_tok * spec.d_cq * 2 + n_tok * spec.n_h * spec.d_c * 2
        o_bytes = spec.d_model * spec.n_h * spec.d_c * 2 + n_tok * spec.n_h * spec.d_c * 2 + n_tok * spec.d_model * 2
        fold_line = {}
        for key, nbytes, name in (("q", q_bytes, "absorb_q_folded"), ("o", o_bytes, "up_o_folded")):
            t = phases_us[name] * 1e-6
            fold_line[key] = {"us": phases_us[name], "bytes": nbytes, "achieved_gbs": nbytes / t / 1e9,
                              "frac": nbytes / t / 1e9 / peaks["hbm_gbs"]}

    if rank != 0:
        if pg is not None:
            pg.destroy_process_group()
        return 0

    cpu = None
    if world == 1:
        rate, secs, desc = oracle_sample_rate(spec, steps=4, warmup=1, budget_s=20.0, yarn=args.yarn,
                                              cache=args.cache)
        cpu = {"value": rate, "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle",
               "sample": desc}

    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": step_ms / K,
        "ms_per_step_median": statistics.median(step_each), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16" if args.cache == "bf16" else "f32",
        "data": "synthetic",
        "config": bench_config(spec, args, world),
        "phases_us": phases_us, "phases_median_us": phases_med_us,
        **({"fold": fold_line} if fold_line is not None else {}),
        "timing": "device passes replay CUDA graphs of the C-ABI calls; e2e calls the API directly",
        "host_enqueue_us_per_step": 1e6 * host_s / K,
        "decode_hbm_tbs": hbm_gbs / 1e3, "decode_tflops": tflops,
        "decode_tflops_frac_sustained": tflops / peaks.get("bf16_tflops_sustained", 1e9),
        "roofline": roof,
        "cpu_baseline": cpu,
        "e2e": {"value": e2e_value, "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h,
                "how": "C-ABI calls from Python with pinned host buffers; steps pipelined (uploads and "
                       "read-backs on two more streams, double-buffered); no L2 flush (cache larger than L2)"},
        "gpu_launches": launches_per_step * K,
        "clocks": sampler.summary(),
        "decode_kernel_hash": khash,
    }
    print(json.dumps(line))
    if pg is not None:
        pg.destroy_process_group()
    return 0


def main():
    args = parse()
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
