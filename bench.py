"""Benchmark: one NABLA attention layer per step on B200, through the C ABI.

A step is the whole hot path on one batch of synthetic input already
resident in HBM, Q, K, V in grid order, in three timed stages:
  1. pooling of Q and K straight from grid order: each block's 64 tokens
     gathered in the fractal (flattened) order (nabla_flatten_pool_qk
     without flattened copies);
  2. the adaptive block mask on the pooled workspace: reduced attention, CDF
     threshold, STA union, compaction (nabla_build_mask_pooled);
  3. block-sparse attention on the kept tiles reading Q, K, V in grid order
     through 5-D TMA boxes (the flattening done by the copy) and storing O
     and the LSE in grid order (nabla_sparse_attn_fwd_grid).
L2 is flushed (a 256 MB write) between timed steps, outside the timed events.
With --config hunyuan-sta the mask is the static sliding-tile window alone
(nabla_build_mask_sta replaces stages 1 and 2; Q and K are not read for it).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config long]
    python bench.py --impl reference ...   # the CPU oracle, same metric

Prints one JSON line (rank 0).  `value` is kept-tile attention TFLOP/s over
the whole step (4*64*64*D FLOP per kept 64x64 tile); per-stage times,
attention TFLOP/s with its roofline, the mask's score-phase roofline and the
flatten stage's GB/s are extra keys.  With --gpus N > 1 each rank runs an
independent replica of the layer (the method runs on one GPU; there is no
exchange between ranks).
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from block_sparse_attention_flatten_b200 import inputs  # noqa: E402

METRIC = "sparse-attn TFLOP/s on kept tiles & ms/layer; mask-build GB/s (1×B200)"
CONFIGS = {
    "tiny": inputs.TINY,
    "wan13b": inputs.WAN13B,
    "hunyuan": inputs.HUNYUAN,
    "long": inputs.LONG,
    "long-4h": inputs.LONG_4H,
    "hunyuan-sta": inputs.HUNYUAN_STA,
    "hunyuan-radial": inputs.HUNYUAN_RADIAL,
    "long-radial": inputs.LONG_RADIAL,
}
CONFIGS.update({f"sweep-a{w.alpha}-t{w.thr}": w for w in inputs.sweep_points()})
# AB-Attention (second workload): sampling plan + attention on the samples
AB_CONFIGS = {"ab-wan13b": inputs.AB_WAN13B, "ab-tiny": inputs.AB_TINY}
L2_FLUSH_BYTES = 256 << 20


def max_over_ranks(x: float, device) -> float:
    """The largest x over all ranks (x itself on one rank): a step is timed
    on every rank's device and the slowest rank sets the job's time."""
    t = torch.tensor([x], dtype=torch.float64, device=device)
    if torch.distributed.is_available() and torch.distributed.is_initialized() and \
            torch.distributed.get_world_size() > 1:
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def whole_job_tflops(world: int, flop_per_step_per_rank: float, steps: int, max_ms: float) -> float:
    """Units all ranks processed over the slowest rank's time: each of the
    `world` replicas runs `steps` steps of flop_per_step_per_rank FLOP."""
    return world * flop_per_step_per_rank * steps / (max_ms * 1e-3) / 1e12


def load_peaks():
    """(bf16 burst TFLOP/s, bf16 sustained TFLOP/s, HBM GB/s, kind): the
    measured figures, else this pool's earlier measurements."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as fh:
            d = json.load(fh)
        burst = float(d["bf16_tflops"])
        return burst, float(d.get("bf16_tflops_sustained", burst)), float(d["hbm_gbs"]), "measured"
    return 1590.0, 1400.0, 6650.0, "fallback"


# A kernel timed inside a timed region at least this long runs under the
# power cap (the long-video layer's 20 steps take ~1.4 s at ~1.4 GHz), so its
# roofline takes the sustained bf16 figure; shorter regions take the burst one.
SUSTAINED_REGION_MS = 500.0


def tensor_peak(timed_ms: float):
    burst, sustained, _, kind = load_peaks()
    if timed_ms >= SUSTAINED_REGION_MS:
        return sustained, burst, f"{kind} bf16 sustained (timed region {timed_ms / 1e3:.2f} s, under the power cap)"
    return burst, burst, f"{kind} bf16 burst"


def config_dict(w: inputs.Workload):
    return {
        "workload": w.name,
        "B": w.B,
        "heads": w.Hh,
        "head_dim": w.D,
        "grid_THW": [w.T, w.H, w.W],
        "tokens": w.S,
        "blocks": w.Nb,
        "mask": ("adaptive (CDF)" + (" OR static STA window" if any(w.sta) else "") +
                 (f" OR radial window r0={w.radial}" if w.radial else "")) if w.mask == "nabla"
                else ("static STA window only" if w.mask == "sta" else f"static radial window r0={w.radial} only"),
        "thr": w.thr if w.mask == "nabla" else None,
        "sta": list(w.sta) if any(w.sta) else None,
        "locality_amplitude": w.alpha,
        "seed": w.seed,
        "l2": "flushed between timed steps (256 MB write)",
    }


def kept_flops(w, total_kept):
    return 4.0 * 64 * 64 * w.D * total_kept


def mask_bytes(w, total_kept):
    """Compulsory bytes of the whole mask build: Q and K read once, the
    block counts and the kept list entries written."""
    return 2.0 * w.B * w.S * w.Hh * w.D * 2 + 4.0 * w.B * w.Hh * w.Nb + 4.0 * total_kept


def pool_bytes(w):
    """Compulsory bytes of the pooling stage: Q and K read once, the pooled
    Q and K (fp32) written."""
    return 2.0 * w.B * w.S * w.Hh * w.D * 2 + 2.0 * 4 * w.B * w.Hh * w.Nb * w.D


def score_flops(w):
    """fp32 FLOPs of the mask's block scores (2 per multiply-add)."""
    return 2.0 * w.B * w.Hh * w.Nb * w.Nb * w.D


# fp32 FMA peak of one B200: 148 SMs x 128 lanes x 2 FLOP per clock at the
# 1965 MHz maximum SM clock
FP32_PEAK_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12


# ----------------------------------------------------------------------------- clocks
class ClockSampler:
    """Samples the SM clock and the clock-event reasons every 10 ms (NVML,
    read-only) while the timed region runs."""

    REASONS = (("hw_slowdown", "nvmlClocksEventReasonHwSlowdown"),
               ("hw_thermal_slowdown", "nvmlClocksEventReasonHwThermalSlowdown"),
               ("sw_thermal_slowdown", "nvmlClocksEventReasonSwThermalSlowdown"),
               ("sw_power_cap", "nvmlClocksEventReasonSwPowerCap"),
               ("hw_power_brake_slowdown", "nvmlClocksEventReasonHwPowerBrakeSlowdown"))

    def __init__(self, device_index: int):
        self.dev = device_index
        self.samples = []
        self.thread = None
        self.stop_flag = False

    def _run(self, nvml, handle):
        while not self.stop_flag:
            try:
                sm = nvml.nvmlDeviceGetClockInfo(handle, nvml.NVML_CLOCK_SM)
                reasons = nvml.nvmlDeviceGetCurrentClocksEventReasons(handle)
                self.samples.append((sm, reasons))
            except Exception:  # noqa: BLE001 - sampling is best effort
                pass
            time.sleep(0.01)

    def start(self):
        try:
            import threading

            import pynvml as nvml
            nvml.nvmlInit()
            handle = nvml.nvmlDeviceGetHandleByIndex(self.dev)
            self.max_mhz = nvml.nvmlDeviceGetMaxClockInfo(handle, nvml.NVML_CLOCK_SM)
            self.nvml = nvml
            self.thread = threading.Thread(target=self._run, args=(nvml, handle), daemon=True)
            self.thread.start()
        except Exception:  # noqa: BLE001
            self.thread = None

    def stop(self):
        if self.thread is None:
            return None
        self.stop_flag = True
        self.thread.join()
        if not self.samples:
            return None
        reasons = sorted({name for _, bits in self.samples for name, const in self.REASONS
                          if bits & getattr(self.nvml, const, 0)})
        return {"sm_mhz": statistics.median(s for s, _ in self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": reasons, "samples": len(self.samples), "source": "NVML, 10 ms"}


# ----------------------------------------------------------------------------- GPU arm
def run_gpu(args, rank, world, local_rank):
    from block_sparse_attention_flatten_b200 import nabla
    from block_sparse_attention_flatten_b200 import build as nbuild

    nbuild.build()
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    w = CONFIGS[args.config]
    q, k, v = inputs.make_qkv(w)
    stream = torch.cuda.current_stream()

    # device-resident inputs and outputs (allocated once; the library allocates nothing)
    qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
    og = torch.empty_like(qd)  # attention output, grid order
    kv_count = torch.empty((w.B, w.Hh, w.Nb), dtype=torch.int32, device=dev)
    kv_idx = torch.empty((w.B, w.Hh, w.Nb, w.Nb), dtype=torch.int32, device=dev)
    static = w.mask in ("sta", "radial")  # a static window alone: no pooling, no scores
    prm = nabla.params(w.thr, w.sta, radial=w.radial)
    ws = None if static else torch.empty(nabla.mask_workspace_bytes(w.B, w.Hh, w.D, w.T, w.H, w.W, prm),
                                         dtype=torch.uint8, device=dev)
    lse = torch.empty((w.B, w.Hh, w.S), dtype=torch.float32, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    split = args.attn_split if args.attn_split > 0 else auto_split(w)
    split_ws = (torch.empty(nabla.attn_split_workspace_bytes(w.B, w.Hh, w.D, w.T, w.H, w.W, split),
                            dtype=torch.uint8, device=dev) if split > 1 else None)

    def static_lists():
        if w.mask == "sta":
            nabla.build_mask_sta(w.B, w.Hh, w.T, w.H, w.W, w.sta, kv_count=kv_count, kv_idx=kv_idx)
        else:
            nabla.build_mask_radial(w.B, w.Hh, w.T, w.H, w.W, w.radial, kv_count=kv_count, kv_idx=kv_idx)

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        if static:
            # 1-2. the window's block lists (nothing read)
            static_lists()
            if ev is not None:
                ev[1].record(stream)
                ev[2].record(stream)
        else:
            # 1. pooling of Q and K straight from grid order (each block's 64
            #    tokens gathered in flattened order; no flattened copies)
            nabla.flatten_pool_qk(qd, kd, w.T, w.H, w.W, workspace=ws, thr=w.thr, sta=w.sta, write_flat=False)
            if ev is not None:
                ev[1].record(stream)
            # 2. mask rows on the pooled workspace
            nabla.build_mask_pooled(ws, w.B, w.Hh, w.D, w.T, w.H, w.W, w.thr, w.sta, kv_count=kv_count,
                                    kv_idx=kv_idx, radial=w.radial)
            if ev is not None:
                ev[2].record(stream)
        # 3. attention reading Q, K, V in grid order through 5-D TMA boxes
        #    and storing O in grid order
        nabla.sparse_attn_fwd(qd, kd, vd, kv_count, kv_idx, out=og, lse=lse, grid=(w.T, w.H, w.W), split=split,
                              workspace=split_ws)
        if ev is not None:
            ev[3].record(stream)

    # (window lists | pooling, scores, selection), attention (+ the merge of a split walk)
    launches_per_step = (2 if static else 4) + (1 if split > 1 else 0)
    for _ in range(args.warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    status = nabla.get_status()
    if status != 0:
        raise RuntimeError(f"device status after warm-up: {nabla.strerror(status)}")
    total_kept = float(kv_count.double().sum().item())

    events = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    sampler = ClockSampler(local_rank)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    sampler.start()
    for s in range(args.steps):
        flush.zero_()
        step(events[s])
    torch.cuda.synchronize()
    clocks = sampler.stop()
    if world > 1:
        torch.distributed.barrier()
    status = nabla.get_status()
    if status != 0:
        raise RuntimeError(f"device status after timing: {nabla.strerror(status)}")

    def stage(a, b):
        return [events[s][a].elapsed_time(events[s][b]) for s in range(args.steps)]

    step_ms = stage(0, 3)
    pool_ms, mask_ms, attn_ms = stage(0, 1), stage(1, 2), stage(2, 3)
    total_ms_max = max_over_ranks(sum(step_ms), dev)

    # end to end through the public API: pinned host inputs in, result out.
    # Every step copies its Q, K, V from pinned host memory and reads its O
    # back, all inside the timed region; the copies run on their own streams
    # so they overlap the computation: V's upload overlaps the mask (which
    # needs only Q and K), and step s+1's uploads and step s's download
    # overlap step s's computation (device inputs and outputs are double
    # buffered).  The last downloaded O is checked against the device-only
    # result.
    e2e = None
    if args.e2e_steps > 0:
        qh, kh, vh = q.pin_memory(), k.pin_memory(), v.pin_memory()
        oh = torch.empty(og.shape, dtype=og.dtype, pin_memory=True)
        o_ref = og.clone()  # output of the device-only steps
        sets = [(qd, kd, vd, og), tuple(torch.empty_like(x) for x in (qd, kd, vd, og))]
        up, down = torch.cuda.Stream(), torch.cuda.Stream()
        ev = lambda: torch.cuda.Event()  # noqa: E731
        qk_in, v_in, done, out = [ev(), ev()], [ev(), ev()], [ev(), ev()], [ev(), ev()]
        n_e2e = args.e2e_steps + 1  # the first step warms the copy engines and is not timed

        def e2e_step(s_, qd_, kd_, vd_, og_):
            b_ = s_ & 1
            with torch.cuda.stream(up):
                if s_ >= 2:
                    up.wait_event(done[b_])  # step s-2 has finished reading this input set
                qd_.copy_(qh, non_blocking=True)
                kd_.copy_(kh, non_blocking=True)
                qk_in[b_].record(up)
                vd_.copy_(vh, non_blocking=True)
                v_in[b_].record(up)
            stream.wait_event(qk_in[b_])
            if static:
                static_lists()
            else:
                nabla.flatten_pool_qk(qd_, kd_, w.T, w.H, w.W, workspace=ws, thr=w.thr, sta=w.sta,
                                      write_flat=False)
                nabla.build_mask_pooled(ws, w.B, w.Hh, w.D, w.T, w.H, w.W, w.thr, w.sta, kv_count=kv_count,
                                        kv_idx=kv_idx, radial=w.radial)
            stream.wait_event(v_in[b_])
            if s_ >= 2:
                stream.wait_event(out[b_])  # step s-2's output has been downloaded
            nabla.sparse_attn_fwd(qd_, kd_, vd_, kv_count, kv_idx, out=og_, lse=lse, grid=(w.T, w.H, w.W),
                                  split=split, workspace=split_ws)
            done[b_].record(stream)
            with torch.cuda.stream(down):
                down.wait_event(done[b_])
                oh.copy_(og_, non_blocking=True)
                out[b_].record(down)

        torch.cuda.synchronize()
        e2e_step(0, *sets[0])  # untimed
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(up)
        stream.wait_event(e0)
        down.wait_event(e0)
        for s in range(1, n_e2e):
            e2e_step(s, *sets[s & 1])
        e1.record(down)  # after the last download, which follows everything else
        torch.cuda.synchronize()
        if not torch.equal(oh, o_ref.cpu()):
            raise RuntimeError("end-to-end output differs from the device-only steps")
        te = max_over_ranks(e0.elapsed_time(e1), dev)
        e2e_ms = [te / (n_e2e - 1)] * (n_e2e - 1)
        bi = 3 * qd.numel() * qd.element_size()
        bo = og.numel() * og.element_size()
        e2e = {"value": whole_job_tflops(world, kept_flops(w, total_kept), len(e2e_ms), te),
               "unit": "TFLOP/s", "h2d_bytes_per_step": bi, "d2h_bytes_per_step": bo,
               "ms_per_step": te / len(e2e_ms)}

    # the materialised fractal flattening (not on the hot path: the pooling
    # and the attention's loads flatten on the fly), timed over back-to-back
    # launches so the writes still draining from L2 at a launch's end are
    # charged to the next one; not part of `value`
    flatten = None
    if not static and args.flatten_launches > 0:
        qflat = torch.empty_like(qd)
        nabla.flatten(qd, w.T, w.H, w.W, out=qflat)
        torch.cuda.synchronize()
        fe = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
        fe[0].record(stream)
        for _ in range(args.flatten_launches):
            nabla.flatten(qd, w.T, w.H, w.W, out=qflat)
        fe[1].record(stream)
        torch.cuda.synchronize()
        t_fl = fe[0].elapsed_time(fe[1]) / args.flatten_launches
        nbytes = 2.0 * qd.numel() * qd.element_size()
        flatten = {"ms_per_tensor": t_fl, "gbs": nbytes / (t_fl * 1e-3) / 1e9, "bytes_per_launch": nbytes,
                   "launches": args.flatten_launches, "timing": "back-to-back launches, CUDA events"}
        del qflat

    # backward pass over the same lists (training), timed on its own: the
    # column lists, then Delta, dQ and dK/dV; not part of `value`
    backward = None
    if args.backward_steps > 0:
        do = inputs.randn_bf16(tuple(qd.shape), seed=w.seed + 1000).to(dev)  # output gradient
        q_count, q_idx = torch.empty_like(kv_count), torch.empty_like(kv_idx)
        dq_, dk_, dv_ = torch.empty_like(qd), torch.empty_like(kd), torch.empty_like(vd)
        delta = torch.empty_like(lse)
        nabla.sparse_attn_fwd(qd, kd, vd, kv_count, kv_idx, out=og, lse=lse, grid=(w.T, w.H, w.W))

        def bstep(ev=None):
            if ev is not None:
                ev[0].record(stream)
            nabla.transpose_lists(kv_count, kv_idx, q_count=q_count, q_idx=q_idx)
            if ev is not None:
                ev[1].record(stream)
            nabla.sparse_attn_bwd(qd, kd, vd, og, do, lse, kv_count, kv_idx, q_lists=(q_count, q_idx), dq=dq_,
                                  dk=dk_, dv=dv_, delta=delta, grid=(w.T, w.H, w.W))
            if ev is not None:
                ev[2].record(stream)

        for _ in range(3):
            flush.zero_()
            bstep()
        bev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.backward_steps)]
        for s in range(args.backward_steps):
            flush.zero_()
            bstep(bev[s])
        torch.cuda.synchronize()
        status = nabla.get_status()
        if status != 0:
            raise RuntimeError(f"device status after the backward: {nabla.strerror(status)}")
        t_tr = statistics.mean(e[0].elapsed_time(e[1]) for e in bev)
        t_bw = statistics.mean(e[1].elapsed_time(e[2]) for e in bev)
        bwd_flops = 2.5 * kept_flops(w, total_kept)  # S, dP, dV, dK, dQ: five 64x64xD products per tile
        backward = {"ms": t_tr + t_bw, "transpose_lists_ms": t_tr, "attn_bwd_ms": t_bw,
                    "tflops_kept": bwd_flops / ((t_tr + t_bw) * 1e-3) / 1e12,
                    "flop_count": "10*64*64*D per kept tile (five products; the kernels recompute S and dP "
                                  "in both passes, 14*64*64*D executed)",
                    "steps": args.backward_steps, "launches_per_step": 4}
        del do, q_count, q_idx, dq_, dk_, dv_, delta

    # the same step captured once in a CUDA graph and replayed: the calls
    # allocate nothing and never synchronise, so one graph holds the whole
    # layer and its replay pays one launch instead of one per kernel.  Each
    # replay is timed with events on the launching stream, the L2 flushed
    # before it; not part of `value`
    graph = None
    if args.graph_steps > 0:
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            step()
        for _ in range(3):
            flush.zero_()
            g.replay()
        gev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.graph_steps)]
        for s in range(args.graph_steps):
            flush.zero_()
            gev[s][0].record(stream)
            g.replay()
            gev[s][1].record(stream)
        torch.cuda.synchronize()
        status = nabla.get_status()
        if status != 0:
            raise RuntimeError(f"device status after the graph replays: {nabla.strerror(status)}")
        t_g = statistics.mean(e[0].elapsed_time(e[1]) for e in gev)
        graph = {"ms_per_step": t_g, "value": kept_flops(w, total_kept) / (t_g * 1e-3) / 1e12, "unit": "TFLOP/s",
                 "eager_ms_per_step": total_ms_max / args.steps, "replays": args.graph_steps,
                 "kernels_per_replay": launches_per_step}
        del g

    _, _, peak_gbs, peak_kind = load_peaks()
    peak_tf, burst_tf, tf_kind = tensor_peak(total_ms_max)
    attn_avg = statistics.mean(attn_ms)
    mask_avg = statistics.mean(mask_ms)
    mask_gbs = (mask_bytes(w, total_kept) - (0 if not static else 4.0 * w.B * w.S * w.Hh * w.D)) / \
        ((statistics.mean(pool_ms) + mask_avg) * 1e-3) / 1e9
    achieved = kept_flops(w, total_kept) / (attn_avg * 1e-3) / 1e12
    traffic = load_traffic(args.config)
    result = {
        "metric": METRIC,
        "value": whole_job_tflops(world, kept_flops(w, total_kept), args.steps, total_ms_max),
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": total_ms_max / args.steps,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic",
        "config": dict(config_dict(w), attn_key_ranges=split),
        # per layer: the whole step, since Q, K, V, O stay in grid order (the
        # flattening and its inverse happen inside the pooling and attention)
        "ms_per_layer": statistics.mean(pool_ms) + mask_avg + attn_avg,
        "stages_ms": ({"window_lists": statistics.mean(pool_ms), "sparse_attn": attn_avg} if static else
                      {"pool_qk": statistics.mean(pool_ms), "mask_rows": mask_avg, "sparse_attn": attn_avg}),
        # mask build = pooling + rows: Q and K read once, kv_count and the kept
        # kv_idx entries written, over its time (the static window reads
        # nothing: only the lists are written)
        "mask_build_gbs": mask_gbs,
        "attn_tflops_kept": achieved,
        "pool_gbs": None if static else pool_bytes(w) / (statistics.mean(pool_ms) * 1e-3) / 1e9,
        "kept_tile_fraction": total_kept / (w.B * w.Hh * w.Nb * w.Nb),
        "roofline": {"bound": "tensor", "kernel": "attn_fwd_kernel<128>", "achieved": achieved, "peak": peak_tf,
                     "unit": "TFLOP/s", "frac": achieved / peak_tf, "peak_kind": tf_kind,
                     "frac_of_burst": achieved / burst_tf, "traffic": traffic},
        # the mask build (pooling + rows) against HBM: Q and K read once, the
        # lists written, over the two stages' time
        "mask_roofline": None if static else {
            "bound": "hbm", "kernels": "pool_kernel<true> + score_tile_kernel + select_rows_kernel",
            "achieved": mask_gbs, "peak": peak_gbs, "unit": "GB/s", "frac": mask_gbs / peak_gbs,
            "peak_kind": f"{peak_kind} HBM copy", "target_frac": 0.6},
        # the rows stage alone against the fp32 FMA peak (its scores are an
        # fp32 GEMM of 2*B*Hh*Nb^2*D FLOP)
        "mask_score_roofline": None if static else {
            "bound": "alu", "kernels": "score_tile_kernel + select_rows_kernel",
            "achieved": score_flops(w) / (mask_avg * 1e-3) / 1e12, "peak": FP32_PEAK_TFLOPS, "unit": "TFLOP/s",
            "frac": score_flops(w) / (mask_avg * 1e-3) / 1e12 / FP32_PEAK_TFLOPS,
            "peak_kind": "derived: 148 SMs x 128 fp32 lanes x 2 FLOP x 1965 MHz"},
        "e2e": e2e,
        "backward": backward,
        "flatten": flatten,
        "graph": graph,
        "clocks": clocks,
        "gpu_launches": launches_per_step * args.steps,
    }
    return result, (q, k, v, w, total_kept)


def run_gpu_ab(args, rank, world, local_rank):
    """AB-Attention layer: a step is the sampling plan (key means, clusters,
    centroid logits, scores, inclusion probabilities, the sample) and the
    attention on the sampled 4-token blocks, Q, K, V in grid order.  value =
    attention FLOPs on the sampled blocks (4 * 128 * 4 * D per (query block,
    sampled key block)) over the whole step."""
    from block_sparse_attention_flatten_b200 import nabla
    from block_sparse_attention_flatten_b200 import build as nbuild

    nbuild.build()
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    w = AB_CONFIGS[args.config]
    base = w.base
    q, k, v = inputs.make_qkv(base)
    u = inputs.ab_uniforms(w)
    stream = torch.cuda.current_stream()
    qd, kd, vd, ud = q.to(dev), k.to(dev), v.to(dev), u.to(dev)
    kcount = torch.empty((base.B, base.Hh, w.nqb), dtype=torch.int32, device=dev)
    kidx = torch.empty((base.B, base.Hh, w.nqb, w.nkb), dtype=torch.int32, device=dev)
    kshift = torch.empty((base.B, base.Hh, w.nqb, w.nkb), dtype=torch.float32, device=dev)
    ws = torch.empty(nabla.ab_workspace_bytes(base.B, base.S, base.Hh, base.D), dtype=torch.uint8, device=dev)
    og = torch.empty_like(qd)
    lse = torch.empty((base.B, base.Hh, base.S), dtype=torch.float32, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        nabla.ab_plan(qd, kd, ud, w.budget, w.kmeans_iters, kcount=kcount, kidx=kidx, kshift=kshift, workspace=ws)
        if ev is not None:
            ev[1].record(stream)
        nabla.ab_attn_fwd(qd, kd, vd, kcount, kidx, kshift, out=og, lse=lse)
        if ev is not None:
            ev[2].record(stream)

    for _ in range(args.warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    status = nabla.get_status()
    if status != 0:
        raise RuntimeError(f"device status after warm-up: {nabla.strerror(status)}")
    sampled = float(kcount.double().sum().item())
    flop = 4.0 * 128 * 4 * base.D * sampled
    events = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    sampler = ClockSampler(local_rank)
    torch.cuda.synchronize()
    sampler.start()
    for s_ in range(args.steps):
        flush.zero_()
        step(events[s_])
    torch.cuda.synchronize()
    clocks = sampler.stop()
    plan_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in events)
    attn_ms = statistics.mean(e[1].elapsed_time(e[2]) for e in events)
    total = max_over_ranks(sum(e[0].elapsed_time(e[2]) for e in events), dev)
    peak_tf, burst_tf, tf_kind = tensor_peak(total)
    achieved = flop / (attn_ms * 1e-3) / 1e12
    cfg = config_dict(base)
    cfg.update({"workload": w.name, "mask": "AB-Attention sample (IBCS clusters + SIP, 4-token key blocks)",
                "thr": None, "budget_blocks_per_query_block": w.budget, "kmeans_iters": w.kmeans_iters,
                "query_block": 128, "key_block": 4})
    return {
        "metric": METRIC,
        "value": whole_job_tflops(world, flop, args.steps, total),
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": total / args.steps,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic",
        "config": cfg,
        "stages_ms": {"ab_plan": plan_ms, "ab_attn": attn_ms},
        "sampled_block_fraction": sampled / (base.B * base.Hh * w.nqb * w.nkb),
        "attn_tflops_sampled": achieved,
        "roofline": {"bound": "tensor", "kernel": "ab_attn_fwd_kernel<128>", "achieved": achieved, "peak": peak_tf,
                     "unit": "TFLOP/s", "frac": achieved / peak_tf, "peak_kind": tf_kind, "frac_of_burst": achieved / burst_tf,
                     "traffic": None},
        "clocks": clocks,
        "gpu_launches": 5 * args.steps,
        "cpu_baseline": None,
        "e2e": None,
    }, (q, k, v, u)


# Key ranges of the attention walk when --attn-split is 0: a head's K and V
# larger than half of the 126 MB L2 (the long-video layer's are 123 MB) do
# not stay in it while one wave of CTAs walks lists spread over the whole
# sequence; two ranges halve that working set.  Measured on the long-video
# layer (20 steps, power-capped): 1 range 59.5 ms at 1.44 GHz, 2 ranges 57.9
# ms at 1.58 GHz, 4 ranges 59.5 ms, 8 ranges 65.8 ms; on the Wan-like layer
# (30 MB per head) 4 ranges double the attention time.
def auto_split(w) -> int:
    head_kv_bytes = w.Nb * 64 * w.D * 2 * 2
    return 2 if head_kv_bytes > (63 << 20) else 1


def load_traffic(config):
    """DRAM bytes (read + write) per attention launch from the committed ncu
    capture of this workload, or None when there is none or the kernel source
    changed since it was taken."""
    import hashlib
    path = os.path.join(ROOT, "profiles", f"attn_fwd_{config}.json")
    if not os.path.exists(path):
        return None
    with open(path) as fh:
        d = json.load(fh)
    h = hashlib.sha256()
    for name in ("attn_fwd.cuh", "common.cuh"):
        with open(os.path.join(ROOT, "block_sparse_attention_flatten_b200", "csrc", name), "rb") as fh:
            h.update(fh.read())
    if h.hexdigest() != d.get("source_sha256"):
        return None
    return d.get("dram_bytes_per_launch")


# ----------------------------------------------------------------------------- oracle
def oracle_sample(w, q, k, v, n_blocks, heads=1):
    """Time the CPU oracle on a bounded sample of the layer: `heads` seeded
    heads (all their tokens: flattening, pooling and the full mask of every
    query block), plus attention on n_blocks seeded query blocks of those
    heads; the stage times are extrapolated to all heads (flattening,
    pooling, mask) and to all kept tiles (attention).  Returns the dict for
    `cpu_baseline`."""
    import oracle
    oracle.build()
    heads = min(heads, w.Hh)
    hsel = np.sort(np.random.default_rng(4321).choice(w.Hh, size=heads, replace=False))
    sub = [np.ascontiguousarray(x.view(torch.int16).numpy().view(np.uint16)[:, :, hsel]) for x in (q, k, v)]
    t0 = time.perf_counter()
    qf, kf, vf = (oracle.flatten(x, w.T, w.H, w.W).reshape(x.shape) for x in sub)
    t1 = time.perf_counter()
    if w.mask in ("sta", "radial"):
        c1, i1 = (oracle.sta_lists(w.T, w.nbh, w.nbw, w.sta) if w.mask == "sta" else
                  oracle.radial_lists(w.T, w.nbh, w.nbw, w.radial))
        cnt = np.broadcast_to(c1, (w.B, heads, w.Nb))
        idx = np.broadcast_to(i1, (w.B, heads, w.Nb, w.Nb))
    else:
        qbar, kbar = oracle.pool(qf), oracle.pool(kf)
        cnt, idx, _, _ = oracle.build_mask(qbar, kbar, w.thr, w.scale, w.nbh, w.nbw, sta_window=w.sta,
                                           want_status=False, radial_r0=w.radial)
    t2 = time.perf_counter()
    qblocks = inputs.sample_query_blocks(w.Nb, n_blocks, seed=1234)
    oracle.attention(qf, kf, vf, cnt, idx, w.scale, qblocks=qblocks)
    t3 = time.perf_counter()
    head_kept = float(cnt.astype(np.float64).sum())
    sample_kept = float(cnt[:, :, qblocks].astype(np.float64).sum())
    all_kept = head_kept * w.Hh / heads  # kept tiles of the whole layer, from the sampled heads
    mask_full_s = (t2 - t0) * w.Hh / heads
    attn_full_s = (t3 - t2) * all_kept / max(sample_kept, 1.0)
    step_s = mask_full_s + attn_full_s
    return {
        "value": kept_flops(w, all_kept) / step_s / 1e12,
        "unit": "TFLOP/s",
        "cores": oracle.num_threads(),
        "kind": "oracle",
        "sample": (f"{heads} of {w.Hh} heads: flatten+{'pool+full mask' if w.mask == 'nabla' else 'window lists'} "
                   f"({t2 - t0:.2f} s, x{w.Hh / heads:g} for all heads) and attention on {len(qblocks)} seeded "
                   f"query blocks ({t3 - t2:.2f} s, extrapolated to all {w.Nb} blocks by kept-tile count)"),
        "ms_per_step_extrapolated": step_s * 1e3,
        "sample_s": t3 - t0,
    }


def oracle_sample_ab(w, q, k, v, u, n_blocks, heads=1):
    """The CPU oracle on a bounded sample of an AB-Attention layer: `heads`
    seeded heads (key means, clustering, scores, inclusion and the sample of
    every query block) plus attention on n_blocks query blocks of them,
    extrapolated to all heads and all sampled blocks."""
    import oracle
    oracle.build()
    base = w.base
    heads = min(heads, base.Hh)
    hsel = np.sort(np.random.default_rng(4321).choice(base.Hh, size=heads, replace=False))
    qs, ks, vs = (np.ascontiguousarray(x.view(torch.int16).numpy().view(np.uint16)[:, :, hsel]) for x in (q, k, v))
    us = u.numpy()[:, hsel]
    t0 = time.perf_counter()
    kbar = oracle.ab_key_means(ks)
    cent, counts, _ = oracle.ab_kmeans(qs, iters=w.kmeans_iters)
    score = oracle.ab_scores(cent, counts, kbar, base.scale)
    pi = oracle.ab_inclusion(score, w.budget)
    cnt, idx, shift = oracle.ab_sample(pi, us)
    t1 = time.perf_counter()
    qblocks = inputs.sample_query_blocks(w.nqb, n_blocks, seed=1234)
    oracle.ab_attention(qs, ks, vs, cnt, idx, shift, base.scale, qblocks=qblocks)
    t2 = time.perf_counter()
    all_sampled = float(cnt.sum()) * base.Hh / heads
    frac = float(cnt.sum()) / max(float(cnt[:, :, qblocks].sum()), 1.0)
    step_s = (t1 - t0) * base.Hh / heads + (t2 - t1) * frac * base.Hh / heads
    return {
        "value": 4.0 * 128 * 4 * base.D * all_sampled / step_s / 1e12,
        "unit": "TFLOP/s",
        "cores": oracle.num_threads(),
        "kind": "oracle",
        "sample": (f"{heads} of {base.Hh} heads: sampling plan ({t1 - t0:.2f} s, x{base.Hh / heads:g}) and attention "
                   f"on {len(qblocks)} query blocks ({t2 - t1:.2f} s, extrapolated by sampled-block count)"),
        "ms_per_step_extrapolated": step_s * 1e3,
    }


def run_reference(args):
    if args.config in AB_CONFIGS:
        w = AB_CONFIGS[args.config]
        q, k, v = inputs.make_qkv(w.base)
        u = inputs.ab_uniforms(w)
        times, vals, last = [], [], None
        for s_ in range(args.warmup + args.steps):
            t0 = time.perf_counter()
            last = oracle_sample_ab(w, q, k, v, u, args.ref_blocks, heads=args.ref_heads)
            if s_ >= args.warmup:
                times.append(time.perf_counter() - t0)
                vals.append(last["value"])
        value = statistics.mean(vals)
        cfg = config_dict(w.base)
        cfg["workload"] = w.name
        return {"impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": 1,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": last["ms_per_step_extrapolated"],
                "sample_s_per_step": statistics.mean(times), "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": "f64", "data": "synthetic", "config": cfg,
                "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": last["cores"], "kind": "oracle",
                                 "sample": last["sample"]},
                "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    w = CONFIGS[args.config]
    q, k, v = inputs.make_qkv(w)
    times, vals = [], []
    last = None
    for s in range(args.warmup + args.steps):
        t0 = time.perf_counter()
        last = oracle_sample(w, q, k, v, args.ref_blocks, heads=args.ref_heads)
        dt = time.perf_counter() - t0
        if s >= args.warmup:
            times.append(dt)
            vals.append(last["value"])
    value = statistics.mean(vals)
    return {
        "impl": "reference",
        "metric": METRIC,
        "value": value,
        "unit": "TFLOP/s",
        "n_gpus": 1,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": last["ms_per_step_extrapolated"],
        "sample_s_per_step": statistics.mean(times),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f64",
        "data": "synthetic",
        "config": config_dict(w),
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": last["cores"], "kind": "oracle",
                         "sample": last["sample"]},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--config", default="long", choices=sorted(CONFIGS) + sorted(AB_CONFIGS))
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--e2e-steps", type=int, default=5)
    ap.add_argument("--backward-steps", type=int, default=20, help="timed steps of the backward pass (0: skip)")
    ap.add_argument("--graph-steps", type=int, default=0,
                    help="timed replays of the step captured in a CUDA graph (0: skip)")
    ap.add_argument("--attn-split", type=int, default=0,
                    help="split each head's attention walk into this many key ranges (1: no split; 0: two ranges "
                         "when a head's K and V exceed half the L2, else one)")
    ap.add_argument("--flatten-launches", type=int, default=10,
                    help="back-to-back launches of the materialised flattening to time (0: skip)")
    ap.add_argument("--cpu-blocks", type=int, default=8, help="query blocks in the CPU-baseline sample")
    ap.add_argument("--ref-blocks", type=int, default=2, help="query blocks per reference-arm step")
    ap.add_argument("--ref-heads", type=int, default=1, help="heads per reference-arm step")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        if rank != 0:
            return
        print(json.dumps(run_reference(args)), flush=True)
        return

    if world > 1:
        import datetime
        torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                             device_id=torch.device("cuda", local_rank))
    if args.config in AB_CONFIGS:
        result, (q, k, v, u) = run_gpu_ab(args, rank, world, local_rank)
        if rank == 0:
            if world == 1 and not args.no_cpu_baseline:
                result["cpu_baseline"] = oracle_sample_ab(AB_CONFIGS[args.config], q, k, v, u, args.cpu_blocks,
                                                          heads=args.ref_heads)
            print(json.dumps(result), flush=True)
        if world > 1:
            torch.distributed.destroy_process_group()
        return
    try:
        result, (q, k, v, w, total_kept) = run_gpu(args, rank, world, local_rank)
        if rank == 0:
            if world == 1 and not args.no_cpu_baseline:
                result["cpu_baseline"] = oracle_sample(w, q, k, v, args.cpu_blocks, heads=args.ref_heads)
                if w is inputs.TINY:
                    # the tiny layer's oracle also on one core (its loops are
                    # over independent rows, so the results are the same)
                    import oracle
                    cores = oracle.num_threads()
                    oracle.set_num_threads(1)
                    one = oracle_sample(w, q, k, v, args.cpu_blocks, heads=args.ref_heads)
                    oracle.set_num_threads(cores)
                    result["cpu_baseline"]["single_core"] = {"value": one["value"], "unit": one["unit"], "cores": 1,
                                                             "sample_s": one["sample_s"]}
            else:
                result["cpu_baseline"] = None
            print(json.dumps(result), flush=True)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
