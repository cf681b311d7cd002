"""Throughput of the W4 decode step on B200.

One step = one pass of the whole hot path over one batch of synthetic input:
the 48 W4 body weights of a GPT-2-small-shaped decoder in ONE grouped launch
(each weight with its own fresh fp32 input row, M = 1), then the int8 tied
LM head on the last position (M = 1, V = 50257). The metric is effective
weight GB/s (4-bit nibbles + scales + zero points + int8 table + head scales
read per step) and decode tokens/s = 1 / step time; the body kernel's GB/s is
also given as a fraction of the measured HBM copy bandwidth.

    python bench.py [--gpus N --steps K --warmup W] [--impl ours|reference]

With N > 1 (torchrun, one process per GPU) every rank runs an independent
replica (the decode step has no cross-GPU exchange); value = all ranks' bytes
/ the slowest rank's time.
"""

from __future__ import annotations

import argparse
import ctypes as C
import json
import os
import statistics
import subprocess
import sys
import tempfile
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from int8_weight_quantized_w4_b200 import synth  # noqa: E402

METRIC = "weight GB/s and decode tokens/s (GPT-2-small W4 stack, M=1) as % of HBM roofline"
WORKLOAD = "gpt2-small W4 decode step: 48 body weights (12 x [768x2304, 768x768, 768x3072, 3072x768]) " \
           "+ int8 tied head [768x50257] on the last position, M=1, fp32"
HEAD_K, HEAD_V = synth.GPT2_HIDDEN, synth.GPT2_VOCAB


def body_bytes() -> int:
    return sum(synth.w4_bytes(K, N) for _, K, N in synth.gpt2_stack_shapes())


def head_bytes() -> int:
    return synth.i8_head_bytes(HEAD_K, HEAD_V)


def profiled_traffic(summary: str):
    """DRAM bytes per launch (dram__bytes_read.sum + dram__bytes_write.sum)
    recorded in an ncu summary under profiles/, or None when the kernel's
    source has changed since that capture (its hash no longer matches)."""
    import hashlib
    path = os.path.join(ROOT, "profiles", summary)
    try:
        fields = {}
        for line in open(path):
            if ":" in line and line.startswith("    "):
                k, v = line.strip().split(":", 1)
                fields[k.strip()] = v.strip()
        src = os.path.join(ROOT, fields["source"])
        digest = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
        if digest != fields["source_sha256_16"]:
            return None
        return int(fields["dram_bytes_per_launch"])
    except (OSError, KeyError, ValueError):
        return None


def measured_peaks() -> dict:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        d["_source"] = "measured"
        return d
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "_source": "fallback"}


# ---------------------------------------------------------------- clocks

def gpu_id(local: int) -> str:
    """nvidia-smi id of a torch device (its UUID, whatever CUDA_VISIBLE_DEVICES says)."""
    import torch
    try:
        return "GPU-" + str(torch.cuda.get_device_properties(local).uuid)
    except Exception:
        return str(local)


class ClockSampler:
    """nvidia-smi samples during the timed region (read-only queries)."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append((float(parts[1]), float(parts[2]), parts))
            except ValueError:
                continue
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        reasons = set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for _, _, parts in rows:
            for n, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(r[0] for r in rows), "sm_max_mhz": max(r[1] for r in rows),
                "reasons": sorted(reasons), "samples": len(rows)}


# ---------------------------------------------------------------- distributed

def dist_init(n_gpus: int):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(v: float, world: int) -> float:
    """The slowest rank's time (every rank gets it). A control-plane
    reduction of one number: NCCL on the GPU, or gloo on the CPU."""
    if world == 1:
        return v
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([v], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_gbs(bytes_per_step: int, n_ranks: int, ms_per_step: float) -> float:
    """Aggregate weight GB/s of n independent replicas, each stepping in
    ms_per_step (the slowest rank's time)."""
    return bytes_per_step * n_ranks / (ms_per_step * 1e-3) / 1e9


# ---------------------------------------------------------------- workload

class Workload:
    """Device-resident weights (R rotating copies), inputs and outputs."""

    def __init__(self, copies: int, seed: int = synth.BASE_SEED):
        import torch
        import int8_weight_quantized_w4_b200 as w4
        self.w4 = w4
        self.shapes = synth.gpt2_stack_shapes()
        dev = torch.device("cuda")
        host_w = [synth.w4_weight(K, N, i, seed=seed) for i, (_, K, N) in enumerate(self.shapes)]
        H = synth.i8_head(HEAD_K, HEAD_V, seed=seed)
        self.x_host = [synth.activations(1, K, i, seed=seed) for i, (_, K, _) in enumerate(self.shapes)]
        self.h_host = synth.activations(1, HEAD_K, 999, seed=seed)
        # every input row (the 48 x and the head's h) in one device buffer, every
        # output (the 48 y and the logits) in another, so that a step's inputs
        # and outputs each cross PCIe in one copy; every row starts 16-byte aligned
        self.in_host = np.concatenate([x.reshape(-1) for x in self.x_host] + [self.h_host.reshape(-1)])
        self.in_dev = torch.from_numpy(self.in_host).to(dev)
        self.xs, off = [], 0
        for _, K, _ in self.shapes:
            self.xs.append(self.in_dev[off:off + K].view(1, K))
            off += K
        self.h = self.in_dev[off:off + HEAD_K].view(1, HEAD_K)
        n_out = sum(N for _, _, N in self.shapes) + HEAD_V
        self.out_dev = torch.empty(n_out, dtype=torch.float32, device=dev)
        self.ys, off = [], 0
        for _, _, N in self.shapes:
            self.ys.append(self.out_dev[off:off + N].view(1, N))
            off += N
        self.logits = self.out_dev[off:off + HEAD_V].view(1, HEAD_V)
        assert all(t.data_ptr() % 16 == 0 for t in self.xs + self.ys + [self.h, self.logits])
        base = [{k: torch.from_numpy(W[k]).to(dev) for k in ("qw", "scales", "zp")} for W in host_w]
        table = torch.from_numpy(H["table"]).to(dev)
        hsc = torch.from_numpy(H["scales"]).to(dev)
        self.copies = []
        for r in range(copies):
            ws = base if r == 0 else [{k: v.clone() for k, v in d.items()} for d in base]
            items = [{"x": self.xs[i], "y": self.ys[i], "K": K, "N": N, **ws[i]}
                     for i, (_, K, N) in enumerate(self.shapes)]
            descs = w4.make_descs(items)
            # the same weights in the streaming layout (repacked once, at load)
            wrs = [w4.w4_repack(d["qw"], d["scales"], d["zp"], K, N) for d, (_, K, N) in zip(ws, self.shapes)]
            rdescs = w4.make_rdescs([{"x": self.xs[i], "y": self.ys[i], "K": K, "N": N, "wr": wrs[i]}
                                     for i, (_, K, N) in enumerate(self.shapes)])
            t = table if r == 0 else table.clone()
            s = hsc if r == 0 else hsc.clone()
            tr = w4.i8_head_repack(t, s, HEAD_K, HEAD_V)  # the head in its streaming layout (once, at load)
            tt = w4.i8t_head_repack(t, s, HEAD_K, HEAD_V)  # and in the tensor cores' tile layout
            # the descriptors hold raw pointers: keep every tensor they name alive
            self.copies.append((descs, t, s, ws, rdescs, wrs, tr, tt))
        need = max(w4.w4_matmul_grouped_workspace_size(self.copies[0][0]),
                   w4.i8_head_workspace_size(1, HEAD_K, HEAD_V))
        self.ws = torch.zeros(max(need, 16), dtype=torch.uint8, device=dev)
        self.ws_bytes = self.ws.numel()
        self.lib = w4.lib()
        torch.cuda.synchronize()

    def body(self, r: int, stream_handle: int):
        """The 48 weights, repacked, in grouped decode launches (the product path)."""
        rdescs = self.copies[r][4]
        st = self.lib.w4r_matmul_grouped(rdescs, len(rdescs), stream_handle)
        if st != 0:
            raise RuntimeError(f"w4r_matmul_grouped failed: {st} {self.lib.w4_last_error()}")

    def body_page_format(self, r: int, stream_handle: int):
        """The same 48 weights in the page format through the split-K GEMV."""
        descs = self.copies[r][0]
        st = self.lib.w4_matmul_grouped(descs, len(descs), self.ws.data_ptr(), self.ws_bytes, stream_handle)
        if st != 0:
            raise RuntimeError(f"w4_matmul_grouped failed: {st} {self.lib.w4_last_error()}")

    def head(self, r: int, stream_handle: int):
        """The int8 head on the last position, repacked (the product path)."""
        tr = self.copies[r][6]
        st = self.lib.i8r_head_logits(self.h.data_ptr(), tr.data_ptr(), HEAD_K, HEAD_V, self.logits.data_ptr(),
                                      stream_handle)
        if st != 0:
            raise RuntimeError(f"i8r_head_logits failed: {st} {self.lib.w4_last_error()}")

    def step_fused(self, r: int, stream_handle: int):
        """The whole decode step in one launch: the 48 repacked weights and
        the head in its streaming layout, streamed by the same CTAs."""
        rdescs, tr = self.copies[r][4], self.copies[r][6]
        st = self.lib.w4r_decode_step(rdescs, len(rdescs), self.h.data_ptr(), tr.data_ptr(), HEAD_K, HEAD_V,
                                      self.logits.data_ptr(), stream_handle)
        if st != 0:
            raise RuntimeError(f"w4r_decode_step failed: {st} {self.lib.w4_last_error()}")

    def head_tile(self, r: int, stream_handle: int):
        """The int8 head on the tensor cores (tile layout, integer MMAs)."""
        tt = self.copies[r][7]
        st = self.lib.i8t_head_logits(self.h.data_ptr(), HEAD_K, tt.data_ptr(), HEAD_K, HEAD_V, 1,
                                      self.logits.data_ptr(), HEAD_V, stream_handle)
        if st != 0:
            raise RuntimeError(f"i8t_head_logits failed: {st} {self.lib.w4_last_error()}")

    def head_page_format(self, r: int, stream_handle: int):
        _, t, s = self.copies[r][:3]
        st = self.lib.i8_head_logits(self.h.data_ptr(), HEAD_K, t.data_ptr(), HEAD_V, s.data_ptr(),
                                     self.logits.data_ptr(), HEAD_V, 1, HEAD_K, HEAD_V, self.ws.data_ptr(),
                                     self.ws_bytes, stream_handle)
        if st != 0:
            raise RuntimeError(f"i8_head_logits failed: {st} {self.lib.w4_last_error()}")


def rotation_copies(step_bytes: int) -> int:
    import torch
    l2 = torch.cuda.get_device_properties(0).L2_cache_size
    return max(2, -(-3 * l2 // step_bytes) + 1)


def run_ours(args, world, rank, local):
    import torch
    step_bytes = body_bytes() + head_bytes()
    R = rotation_copies(step_bytes)
    wl = Workload(R)
    stream = torch.cuda.current_stream()
    sh = int(stream.cuda_stream)
    warm = max(3, args.warmup)
    for i in range(warm):
        wl.step_fused(i % R, sh)
        wl.body(i % R, sh)
        wl.head(i % R, sh)
    torch.cuda.synchronize()

    # ---- device-resident timing (value, roofline). Launch-bound work (a step
    # is one launch of about twenty microseconds), so the K timed steps are
    # captured in one CUDA graph and replayed on the stream the timing events
    # are recorded on; an untimed replay uploads each graph first. The step
    # is one launch (w4r_decode_step), so its average launch duration is the
    # step time; the same step as two launches (body, then head) and the body
    # and head kernels alone are timed the same way for comparison.
    K = args.steps
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())

    def capture(fns):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.stream(side):
            hs = int(side.cuda_stream)
            with torch.cuda.graph(g, stream=side):
                for i in range(K):
                    for fn in fns:
                        fn((warm + i) % R, hs)
        with torch.cuda.stream(side):
            g.replay()
        torch.cuda.synchronize()
        return g

    def timed(g, reps=1):
        """ms of `reps` back-to-back replays of g (K steps each)."""
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        barrier(world)
        torch.cuda.synchronize()
        with torch.cuda.stream(side):
            t0.record(side)
            for _ in range(reps):
                g.replay()
            t1.record(side)
        torch.cuda.synchronize()
        barrier(world)
        return t0.elapsed_time(t1)

    def reps_for(g, seconds):
        """Replays of g that fill about `seconds` (from one untimed replay);
        the same on every rank."""
        one = max_over_ranks(timed(g), world)
        return max(1, int(round(seconds * 1e3 / max(one, 1e-3))))

    g_step = capture([wl.step_fused])
    g_two = capture([wl.body, wl.head])
    g_body = capture([wl.body])
    g_head = capture([wl.head])
    g_page = capture([wl.body_page_format])
    g_hpage = capture([wl.head_page_format])
    g_htile = capture([wl.head_tile])
    g_step_t = capture([wl.body, wl.head_tile])
    n_step = reps_for(g_step, args.seconds)
    n_two = reps_for(g_two, args.seconds / 2)
    n_body = reps_for(g_body, args.seconds / 2)
    n_head = reps_for(g_head, args.seconds / 2)
    n_page = reps_for(g_page, args.seconds / 4)
    n_hpage = reps_for(g_hpage, args.seconds / 4)
    n_htile = reps_for(g_htile, args.seconds / 4)
    n_step_t = reps_for(g_step_t, args.seconds / 4)
    sampler = ClockSampler(gpu_id(local if world > 1 else 0))
    sampler.start()
    time.sleep(0.2)
    total_ms = max_over_ranks(timed(g_step, n_step), world)
    two_avg = timed(g_two, n_two) / (K * n_two)
    body_avg = timed(g_body, n_body) / (K * n_body)
    head_avg = timed(g_head, n_head) / (K * n_head)
    page_avg = timed(g_page, n_page) / (K * n_page)
    hpage_avg = timed(g_hpage, n_hpage) / (K * n_hpage)
    htile_avg = timed(g_htile, n_htile) / (K * n_htile)
    step_t_avg = timed(g_step_t, n_step_t) / (K * n_step_t)
    clocks = sampler.stop()
    steps_timed = K * n_step
    ms_step = total_ms / steps_timed
    del g_step, g_two, g_body, g_head, g_page, g_hpage, g_htile, g_step_t

    # ---- end to end through the public API with host buffers
    e2e = run_e2e(wl, args, world, R)

    peaks = measured_peaks()
    achieved = step_bytes / (ms_step * 1e-3) / 1e9  # the step's one launch
    body_achieved = body_bytes() / (body_avg * 1e-3) / 1e9
    n = world
    value = whole_job_gbs(step_bytes, n, ms_step)
    line = {
        "metric": METRIC,
        "value": round(value, 2),
        "unit": "GB/s",
        "n_gpus": n,
        "steps": steps_timed,
        "steps_per_graph": K,
        "graph_replays": n_step,
        "warmup": warm,
        "ms_per_step": round(ms_step, 5),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f32",
        "data": "synthetic (seeded uniform nibbles / int8, fp32 N(0,1) activations)",
        "config": {
            "workload": WORKLOAD,
            "weight_bytes_per_step": step_bytes,
            "body_bytes": body_bytes(),
            "head_bytes": head_bytes(),
            "M": 1,
            "parallelism": f"replicas x{n}" if n > 1 else "1 GPU",
            "l2": f"rotating {R} weight copies ({R * step_bytes / 1e6:.0f} MB, > 3x L2): every step L2-cold",
            "seed": synth.BASE_SEED,
            "body_path": "one launch per step (w4r_decode_step): the 48 weights in the streaming layout "
                         "(repacked once at load, same bytes) and the head in its streaming layout, streamed by "
                         "the same persistent CTAs",
            "timing": "a CUDA graph of K steps replayed back to back for about --seconds, CUDA events on the "
                      "replay stream; step_two_launches, body_only, head_only: K steps (launches) of that "
                      "form per graph, replayed the same way",
        },
        "tokens_per_s": round(n * 1e3 / ms_step, 1),
        "step_two_launches": {"ms": round(two_avg, 5),
                              "GB_per_s": round(step_bytes / (two_avg * 1e-3) / 1e9, 1),
                              "kernels": "w4r_gemv_m1_kernel<false> (48 weights), then i8r_head_kernel"},
        "body_only": {"ms": round(body_avg, 5), "GB_per_s": round(body_achieved, 1),
                      "frac_of_hbm": round(body_achieved / peaks["hbm_gbs"], 4),
                      "tokens_per_s": round(1e3 / body_avg, 1), "launches_timed": K * n_body,
                      "traffic": profiled_traffic("w4r_gemv_gpt2_m1.md")},
        "body_page_format": {"ms": round(page_avg, 5),
                             "GB_per_s": round(body_bytes() / (page_avg * 1e-3) / 1e9, 1),
                             "kernel": "w4_gemv_kernel<1> (split-K GEMV on the page-format buffers)"},
        "head_only": {"ms": round(head_avg, 5), "kernel": "i8r_head_kernel (streaming layout)",
                      "GB_per_s": round(head_bytes() / (head_avg * 1e-3) / 1e9, 1),
                      "frac_of_hbm": round(head_bytes() / (head_avg * 1e-3) / 1e9 / peaks["hbm_gbs"], 4),
                      "traffic": profiled_traffic("i8r_head_gpt2_m1.md")},
        "head_tile": {"ms": round(htile_avg, 5), "kernel": "i8t_head_kernel<16> (tile layout, tcgen05 kind::i8)",
                      "GB_per_s": round(head_bytes() / (htile_avg * 1e-3) / 1e9, 1),
                      "frac_of_hbm": round(head_bytes() / (htile_avg * 1e-3) / 1e9 / peaks["hbm_gbs"], 4),
                      "traffic": profiled_traffic("i8t_head_gpt2_m1.md"),
                      "step_ms_with_it": round(step_t_avg, 5)},
        "head_page_format": {"ms": round(hpage_avg, 5),
                             "GB_per_s": round(head_bytes() / (hpage_avg * 1e-3) / 1e9, 1),
                             "kernel": "i8_rows_kernel<1> (page-format table)"},
        "frac_of_hbm_step": round(value / n / peaks["hbm_gbs"], 4),
        "roofline": {
            "kernel": "w4r_gemv_m1_kernel<true> (the decode step: 48 repacked weights and the head, one launch)",
            "bound": "hbm",
            "achieved": round(achieved, 1),
            "algorithmic_bytes_per_launch": step_bytes,
            "peak": peaks["hbm_gbs"],
            "peak_source": f"{peaks['_source']} hbm_gbs (copy, burst)",
            "unit": "GB/s",
            "frac": round(achieved / peaks["hbm_gbs"], 4),
            "traffic": profiled_traffic("w4r_step_gpt2_m1.md"),
            "traffic_source": "profiles/w4r_step_gpt2_m1.md (ncu dram__bytes_read.sum + dram__bytes_write.sum, "
                              "one launch; null when the kernel source changed since)",
        },
        "e2e": e2e,
        "gpu_launches": steps_timed,  # one launch per step in the timed replays
        "clocks": clocks,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(args.cpu_seconds)
    if world == 1 and not args.no_configs:
        line["configs"] = run_configs(args, wl, peaks, clocks)
    return line


def run_e2e(wl, args, world, R):
    """Same step through the public binding with host buffers: per step, copy
    the step's inputs (the 48 x and h) from pinned host memory, run the step
    (one launch), read the step's result, the logits, back to pinned host
    memory. The body's outputs stay on the device, as a decoder's hidden
    states do."""
    import torch
    stream = torch.cuda.current_stream()
    sh = int(stream.cuda_stream)
    inh = torch.from_numpy(wl.in_host).pin_memory()  # the 48 x and h, contiguous
    outh = torch.empty(wl.logits.shape, dtype=torch.float32).pin_memory()  # the logits
    h2d = inh.numel() * 4
    d2h = outh.numel() * 4

    def step(r):
        wl.in_dev.copy_(inh, non_blocking=True)
        wl.step_fused(r, sh)
        outh.copy_(wl.logits, non_blocking=True)

    for i in range(3):
        step(i % R)
    torch.cuda.synchronize()
    K = args.steps
    barrier(world)
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    for i in range(K):
        step(i % R)
        stream.synchronize()  # the step's result is on the host before the next step
    el = time.perf_counter() - t0
    barrier(world)
    el = max_over_ranks(el, world)
    step_bytes = body_bytes() + head_bytes()
    return {"value": round(step_bytes * world / (el / K) / 1e9, 2), "unit": "GB/s",
            "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
            "ms_per_step": round(el / K * 1e3, 5), "tokens_per_s": round(world * K / el, 1)}


# ---------------------------------------------------------------- every config

FP32_FMA_PER_SM_CLK = 128  # fp32 FMA lanes per SM per clock (B200)


def fp32_alu_peak_tflops(sm_mhz: float | None) -> float:
    """Dense fp32 FMA peak of the part: SMs x 128 FMA lanes x 2 flops x clock."""
    import torch
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    mhz = sm_mhz or 1965.0
    return sms * FP32_FMA_PER_SM_CLK * 2 * mhz * 1e6 / 1e12


def tf32_peak(peaks: dict) -> float:
    return peaks["bf16_tflops"] * (1.1 / 2.25)  # the nominal dense tf32 : bf16 ratio of the part


def graph_ms(calls, reps: int) -> float:
    """ms per call of `calls` (a list of zero-argument launches, each taking
    the current stream handle) captured once into a CUDA graph and replayed
    `reps` times back to back; CUDA events on the replay stream."""
    import torch
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(side):
        hs = int(side.cuda_stream)
        with torch.cuda.graph(g, stream=side):
            for c in calls:
                c(hs)
        g.replay()
    torch.cuda.synchronize()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(side):
        t0.record(side)
        for _ in range(reps):
            g.replay()
        t1.record(side)
    torch.cuda.synchronize()
    ms = t0.elapsed_time(t1) / (reps * len(calls))
    del g
    return ms


def _ok(st, lib, what):
    if st != 0:
        raise RuntimeError(f"{what} failed: {st} {lib.w4_last_error()}")


def _oracle_rate(fn, units: float, budget_s: float) -> tuple[float, int, float]:
    """(units per second, calls, seconds) of the oracle call fn, repeated for about budget_s."""
    n, t0 = 0, time.perf_counter()
    while True:
        fn()
        n += 1
        el = time.perf_counter() - t0
        if el >= budget_s:
            break
    return units * n / el, n, el


def _cpu(value, unit, sample, n, el):
    return {"value": value, "unit": unit, "cores": _blas_threads(), "kind": "oracle",
            "sample": f"{sample}: {n} call(s) in {el:.1f} s"}


def config0(peaks, budget):
    """Single W4 768x768, M = 1, repacked, L2-cold (1000 rotating copies)."""
    import torch
    import int8_weight_quantized_w4_b200 as w4
    import oracle
    K = N = 768
    W = synth.w4_weight(K, N)
    dev = torch.device("cuda")
    qw, sc, zp = (torch.from_numpy(W[k]).to(dev) for k in ("qw", "scales", "zp"))
    wr0 = w4.w4_repack(qw, sc, zp, K, N)
    R = max(64, -(-3 * torch.cuda.get_device_properties(0).L2_cache_size // wr0.numel()))
    wrs = [wr0] + [wr0.clone() for _ in range(R - 1)]
    x = torch.from_numpy(synth.activations(1, K)).to(dev)
    y = torch.empty((1, N), device=dev)
    lib = w4.lib()
    descs = [w4.make_rdescs([{"x": x, "wr": t, "y": y, "K": K, "N": N}]) for t in wrs]
    calls = [lambda hs, d=d: _ok(lib.w4r_matmul_grouped(d, 1, hs), lib, "w4r") for d in descs]
    ms = graph_ms(calls, 10)
    nbytes = synth.w4_bytes(K, N)
    xh = synth.activations(1, K)
    rate, n, el = _oracle_rate(lambda: oracle.w4_matmul_ref(xh, W["qw"], W["scales"], W["zp"], K, N),
                               nbytes / 1e9, budget)
    gbs = nbytes / (ms * 1e-3) / 1e9
    return {"workload": "single W4 matmul 768x768, M=1 (streaming layout)", "metric": "weight GB/s",
            "value": round(gbs, 1), "unit": "GB/s", "us_per_call": round(ms * 1e3, 3),
            "l2": f"{R} rotating copies ({R * wr0.numel() / 1e6:.0f} MB)",
            "roofline": {"kernel": "w4r_gemv_m1_kernel", "bound": "hbm", "achieved": round(gbs, 1),
                         "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": round(gbs / peaks["hbm_gbs"], 4),
                         "note": "0.38 MB per call: launch- and latency-bound, reported not targeted"},
            "cpu_baseline": _cpu(round(rate, 4), "GB/s", "oracle w4_matmul_ref on this weight", n, el)}


def config2(peaks, budget):
    """int8 tied head [768, 50257], last position: M = 1 (streaming layout and
    tile layout) and M = 8 (tile layout, tensor cores; the page-format
    stream-K kernel beside it)."""
    import torch
    import int8_weight_quantized_w4_b200 as w4
    import oracle
    K, V = HEAD_K, HEAD_V
    H = synth.i8_head(K, V)
    dev = torch.device("cuda")
    t0_, s0_ = torch.from_numpy(H["table"]).to(dev), torch.from_numpy(H["scales"]).to(dev)
    tr0 = w4.i8_head_repack(t0_, s0_, K, V)
    tt0 = w4.i8t_head_repack(t0_, s0_, K, V)
    R = max(2, -(-3 * torch.cuda.get_device_properties(0).L2_cache_size // tr0.numel()) + 1)
    trs = [tr0] + [tr0.clone() for _ in range(R - 1)]
    tts = [tt0] + [tt0.clone() for _ in range(R - 1)]
    tabs = [(t0_, s0_)] + [(t0_.clone(), s0_.clone()) for _ in range(R - 1)]
    lib = w4.lib()
    nbytes = synth.i8_head_bytes(K, V)
    out = {"workload": "int8 tied LM head [768x50257], last position", "l2": f"{R} rotating copies"}
    h1 = torch.from_numpy(synth.activations(1, K, 999)).to(dev)
    lg1 = torch.empty((1, V), device=dev)
    calls = [lambda hs, t=t: _ok(lib.i8r_head_logits(h1.data_ptr(), t.data_ptr(), K, V, lg1.data_ptr(), hs), lib,
                                 "i8r_head_logits") for t in trs]
    ms1 = graph_ms(calls, 20)
    g1 = nbytes / (ms1 * 1e-3) / 1e9

    def tile_calls(h, lg, M):
        return [lambda hs, t=t: _ok(lib.i8t_head_logits(h.data_ptr(), K, t.data_ptr(), K, V, M, lg.data_ptr(), V,
                                                        hs), lib, "i8t_head_logits") for t in tts]

    ms1t = graph_ms(tile_calls(h1, lg1, 1), 20)
    g1t = nbytes / (ms1t * 1e-3) / 1e9
    M8 = 8
    h8 = torch.from_numpy(synth.activations(M8, K, 998)).to(dev)
    lg8 = torch.empty((M8, V), device=dev)
    ms8 = graph_ms(tile_calls(h8, lg8, M8), 20)
    g8 = nbytes / (ms8 * 1e-3) / 1e9
    wsb = w4.i8_head_workspace_size(M8, K, V)
    ws = torch.zeros(max(wsb, 16), dtype=torch.uint8, device=dev)
    calls8 = [lambda hs, t=t, s=s_: _ok(lib.i8_head_logits(h8.data_ptr(), K, t.data_ptr(), V, s.data_ptr(),
                                                             lg8.data_ptr(), V, M8, K, V, ws.data_ptr(), ws.numel(),
                                                             hs), lib, "i8_head_logits")
              for t, s_ in tabs]
    ms8p = graph_ms(calls8, 5)
    hh1, hh8 = synth.activations(1, K, 999), synth.activations(M8, K, 998)
    r1, n1, e1 = _oracle_rate(lambda: oracle.i8_head_ref(hh1, H["table"], H["scales"], K, V), nbytes / 1e9, budget / 2)
    r8, n8, e8 = _oracle_rate(lambda: oracle.i8_head_ref(hh8, H["table"], H["scales"], K, V), nbytes / 1e9, budget / 2)
    out["M1"] = {"metric": "weight GB/s", "value": round(g1, 1), "unit": "GB/s", "us_per_call": round(ms1 * 1e3, 3),
                 "roofline": {"kernel": "i8r_head_kernel (streaming layout)", "bound": "hbm",
                              "achieved": round(g1, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
                              "frac": round(g1 / peaks["hbm_gbs"], 4)},
                 "tile_layout": {"us_per_call": round(ms1t * 1e3, 3), "GB_per_s": round(g1t, 1),
                                 "frac": round(g1t / peaks["hbm_gbs"], 4),
                                 "kernel": "i8t_head_kernel<16> (tcgen05 kind::i8)"},
                 "cpu_baseline": _cpu(round(r1, 4), "GB/s", "oracle i8_head_ref, M=1", n1, e1)}
    out["M8"] = {"metric": "weight GB/s", "value": round(g8, 1), "unit": "GB/s", "us_per_call": round(ms8 * 1e3, 3),
                 "roofline": {"kernel": "i8t_head_kernel<64> (tile layout, tcgen05 kind::i8, N 64)", "bound": "hbm",
                              "achieved": round(g8, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
                              "frac": round(g8 / peaks["hbm_gbs"], 4),
                              "traffic": profiled_traffic("i8t_head_gpt2_m8.md")},
                 "page_format": {"us_per_call": round(ms8p * 1e3, 3),
                                 "GB_per_s": round(nbytes / (ms8p * 1e-3) / 1e9, 1),
                                 "kernel": "i8_head_kernel<8> (page format, stream-K, fp32 FMA)"},
                 "cpu_baseline": _cpu(round(r8, 4), "GB/s", "oracle i8_head_ref, M=8", n8, e8)}
    return out


def tile_roofline(tf: float, peaks: dict, kernel: str) -> dict:
    """Roofline of the tile GEMM: algorithmic 2MKN flops against the tf32
    peak, and the bf16 MMA flops it issues (three per product) against the
    bf16 peak."""
    pk = tf32_peak(peaks)
    return {"kernel": kernel, "bound": "tensor", "achieved": round(tf, 2), "unit": "TFLOP/s",
            "achieved_note": "algorithmic 2MKN flops", "peak": round(pk, 1),
            "peak_note": "tf32 dense = bf16 peak x 1.1 / 2.25", "frac": round(tf / pk, 4),
            "issued_bf16": round(3 * tf, 2), "peak_bf16": peaks["bf16_tflops"],
            "frac_issued_bf16": round(3 * tf / peaks["bf16_tflops"], 4)}


def config3(peaks, budget, wl):
    """GPT-2 prefill: M = 58 rows through the 48 weights (tile layout, tensor
    cores, grouped), then the head on row 57 of the last layer's output
    (streaming head)."""
    import torch
    import int8_weight_quantized_w4_b200 as w4
    import oracle
    M = synth.GPT2_PROMPT
    dev = torch.device("cuda")
    lib = w4.lib()
    xs = [torch.from_numpy(synth.activations(M, K, i)).to(dev) for i, (_, K, _) in enumerate(wl.shapes)]
    ys = [torch.empty((M, N), device=dev) for (_, _, N) in wl.shapes]
    K, V = HEAD_K, HEAD_V
    steps = []
    for r, cp in enumerate(wl.copies):
        ws = cp[3]
        wts = [w4.w4t_repack(ws[i]["qw"], ws[i]["scales"], ws[i]["zp"], K_, N_)
               for i, (_, K_, N_) in enumerate(wl.shapes)]
        descs = w4.make_rdescs([{"x": xs[i], "y": ys[i], "wr": wts[i], "K": K_, "N": N_}
                                for i, (_, K_, N_) in enumerate(wl.shapes)])
        tr = w4.i8_head_repack(cp[1], cp[2], K, V)
        steps.append((descs, tr, wts))
    scratch = torch.empty(max(w4.w4t_workspace_size(steps[0][0]), 16), dtype=torch.uint8, device=dev)
    h = ys[-1][M - 1:M]
    lg = torch.empty((1, V), device=dev)

    def body(hs, d):
        _ok(lib.w4t_matmul_grouped(d, len(d), scratch.data_ptr(), scratch.numel(), hs), lib, "w4t_matmul_grouped")

    def step(hs, d, tr):
        body(hs, d)
        _ok(lib.i8r_head_logits(h.data_ptr(), tr.data_ptr(), K, V, lg.data_ptr(), hs), lib, "i8r_head_logits")

    ms = graph_ms([lambda hs, d=d, tr=tr: step(hs, d, tr) for d, tr, _ in steps], 20)
    msb = graph_ms([lambda hs, d=d: body(hs, d) for d, _, _ in steps], 20)
    flops = 2.0 * M * sum(K_ * N_ for _, K_, N_ in wl.shapes)
    tf = flops / (msb * 1e-3) / 1e12
    W = synth.w4_weight(3072, 768, 3)
    xh = synth.activations(M, 3072, 3)
    rate, n, el = _oracle_rate(lambda: oracle.w4_matmul_ref(xh, W["qw"], W["scales"], W["zp"], 3072, 768),
                               2.0 * M * 3072 * 768 / 1e12, budget)
    return {"workload": "GPT-2 prefill: M=58 through the 48 W4 weights (tile layout, tcgen05 bf16 with an exact "
                        "three-piece split of x, grouped) + int8 head on row 57 of the last output (streaming head)",
            "metric": "prefill TFLOP/s (algorithmic 2MKN, body)", "value": round(tf, 2), "unit": "TFLOP/s",
            "us_per_step": round(ms * 1e3, 2), "us_body": round(msb * 1e3, 2),
            "roofline": tile_roofline(tf, peaks, "w4t_gemm_kernel<64> (tcgen05.mma kind::f16, 3 MMAs per product)"),
            "cpu_baseline": _cpu(round(rate, 6), "TFLOP/s", "oracle w4_matmul_ref, one 3072x768 weight at M=58",
                                 n, el)}


def _scaled(v, k):
    return None if v is None else int(v) * k


def config4(peaks, budget, clocks):
    """3.8B-dense-shaped stack, 32 layers x [3072x9216, 3072x3072, 3072x16384,
    8192x3072]: decode at M = 1 (streaming layout), 8 (split-K GEMV) and 32
    (tile layout, tensor cores), prefill at M = 2048 (tile layout, tensor
    cores). 128 distinct weights
    (2.32 GB: L2-cold by size), generated on the GPU with a seeded generator
    in the synthetic distributions (uniform nibbles, scales U[0.005, 0.02])."""
    import torch
    import int8_weight_quantized_w4_b200 as w4
    import oracle
    dev = torch.device("cuda")
    lib = w4.lib()
    shapes = [(K, N) for _, K, N in synth.dense38_stack_shapes()]
    gen = torch.Generator(device=dev)
    gen.manual_seed(synth.BASE_SEED + 38)
    weights = []
    for K, N in shapes:
        nb = K // 32
        qw = torch.randint(0, 256, (K * N // 2,), dtype=torch.uint8, device=dev, generator=gen)
        sc = torch.empty((nb, N), device=dev).uniform_(0.005, 0.02, generator=gen)
        zp = torch.randint(0, 256, (nb * N // 2,), dtype=torch.uint8, device=dev, generator=gen)
        weights.append({"qw": qw, "scales": sc, "zp": zp})
    nbytes = sum(synth.w4_bytes(K, N) for K, N in shapes)
    wsum = sum(K * N for K, N in shapes)
    out = {"workload": "3.8B-dense-shaped W4 stack: 32 layers x [3072x9216, 3072x3072, 3072x16384, 8192x3072], "
                       "128 distinct weights", "weight_bytes": nbytes}
    # decode M = 1 on the streaming layout
    wrs = [w4.w4_repack(Wd["qw"], Wd["scales"], Wd["zp"], K, N) for Wd, (K, N) in zip(weights, shapes)]
    x1 = {K: torch.randn((1, K), device=dev, generator=gen) for K in (3072, 8192)}
    y1 = [torch.empty((1, N), device=dev) for _, N in shapes]
    rd = w4.make_rdescs([{"x": x1[K], "wr": wrs[i], "y": y1[i], "K": K, "N": N} for i, (K, N) in enumerate(shapes)])
    ms1 = graph_ms([lambda hs: _ok(lib.w4r_matmul_grouped(rd, len(rd), hs), lib, "w4r")], 20)
    del wrs
    g1 = nbytes / (ms1 * 1e-3) / 1e9
    out["decode_M1"] = {"metric": "weight GB/s", "value": round(g1, 1), "unit": "GB/s",
                        "ms_per_step": round(ms1, 4), "tokens_per_s": round(1e3 / ms1, 1),
                        "roofline": {"kernel": "w4r_gemv_m1_kernel", "bound": "hbm", "achieved": round(g1, 1),
                                     "peak": peaks["hbm_gbs"], "unit": "GB/s",
                                     "frac": round(g1 / peaks["hbm_gbs"], 4),
                                     "traffic": _scaled(profiled_traffic("w4r_gemv_3p8b_4layers_m1.md"), 8),
                                     "traffic_note": "ncu DRAM bytes of 4 of the 32 layers (one launch of 16 weights) "
                                                     "x 8: the traffic grows with the layers streamed"}}
    # the tile layout of the 128 weights, for M = 32 and the prefill
    wts = [w4.w4t_repack(Wd["qw"], Wd["scales"], Wd["zp"], K, N) for Wd, (K, N) in zip(weights, shapes)]

    def tile_ms(M, reps):
        xm = {K: torch.randn((M, K), device=dev, generator=gen) for K in (3072, 8192)}
        ym = [torch.empty((M, N), device=dev) for _, N in shapes]
        td = w4.make_rdescs([{"x": xm[K], "wr": wts[i], "y": ym[i], "K": K, "N": N} for i, (K, N) in enumerate(shapes)])
        scratch = torch.empty(max(w4.w4t_workspace_size(td), 16), dtype=torch.uint8, device=dev)
        return graph_ms([lambda hs: _ok(lib.w4t_matmul_grouped(td, len(td), scratch.data_ptr(), scratch.numel(), hs),
                                        lib, "w4t_matmul_grouped")], reps)

    # decode M = 8 (split-K GEMV, page format)
    for M in (8,):
        xm = {K: torch.randn((M, K), device=dev, generator=gen) for K in (3072, 8192)}
        ym = [torch.empty((M, N), device=dev) for _, N in shapes]
        items = [{"x": xm[K], "y": ym[i], "K": K, "N": N, **weights[i]} for i, (K, N) in enumerate(shapes)]
        descs = w4.make_descs(items)
        wsb = w4.w4_matmul_grouped_workspace_size(descs)
        ws = torch.zeros(max(wsb, 16), dtype=torch.uint8, device=dev)
        msm = graph_ms([lambda hs: _ok(lib.w4_matmul_grouped(descs, len(descs), ws.data_ptr(), ws.numel(), hs), lib,
                                       "w4_matmul_grouped")], 5)
        tfl = 2.0 * M * wsum / (msm * 1e-3) / 1e12
        gb = nbytes / (msm * 1e-3) / 1e9
        pk = fp32_alu_peak_tflops(clocks.get("sm_mhz"))
        roof = {"kernel": "w4_gemv_kernel<8> (split-K GEMV)", "bound": "alu", "achieved": round(tfl, 2),
                "peak": round(pk, 1), "unit": "TFLOP/s", "frac": round(tfl / pk, 4),
                "peak_source": "148 SMs x 128 fp32 FMA lanes x 2 x the sampled SM clock",
                "traffic": _scaled(profiled_traffic("w4_gemv_pageformat_3p8b_4layers_m8.md"), 8),
                "traffic_note": "ncu DRAM bytes of 4 of the 32 layers x 8"}
        out[f"decode_M{M}"] = {"metric": "TFLOP/s (algorithmic 2MKN)", "value": round(tfl, 2), "unit": "TFLOP/s",
                               "weight_GB_per_s": round(gb, 1), "ms_per_step": round(msm, 4), "roofline": roof}
        del xm, ym, items, descs, ws
    # decode M = 32 on the tile layout (tensor cores, 32-row tiles)
    M = 32
    msm = tile_ms(M, 5)
    tfl = 2.0 * M * wsum / (msm * 1e-3) / 1e12
    out["decode_M32"] = {"metric": "TFLOP/s (algorithmic 2MKN)", "value": round(tfl, 2), "unit": "TFLOP/s",
                         "weight_GB_per_s": round(nbytes / (msm * 1e-3) / 1e9, 1), "ms_per_step": round(msm, 4),
                         "roofline": tile_roofline(tfl, peaks, "w4t_gemm_kernel<32> (tcgen05.mma kind::f16)")}
    # prefill M = 2048 on the tile layout: x shared by the weights of one K
    # (its pieces made once per call), y distinct per weight
    M = 2048
    msp = tile_ms(M, 2)
    tfp = 2.0 * M * wsum / (msp * 1e-3) / 1e12
    out["prefill_M2048"] = {"metric": "prefill TFLOP/s (algorithmic 2MKN)", "value": round(tfp, 2), "unit": "TFLOP/s",
                            "ms_per_step": round(msp, 3),
                            "roofline": tile_roofline(tfp, peaks, "w4t_gemm_kernel<128> (tcgen05.mma kind::f16)")}
    del wts, weights
    torch.cuda.empty_cache()
    # the oracle on one o_proj weight (3072x3072) at each M, scaled to the metric
    W = synth.w4_weight(3072, 3072, 38)
    per = {}
    for M, key, unit in ((1, "decode_M1", "GB/s"), (8, "decode_M8", "TFLOP/s"), (32, "decode_M32", "TFLOP/s"),
                         (2048, "prefill_M2048", "TFLOP/s")):
        xh = synth.activations(M, 3072, 38)
        units = synth.w4_bytes(3072, 3072) / 1e9 if unit == "GB/s" else 2.0 * M * 3072 * 3072 / 1e12
        r, n, el = _oracle_rate(lambda: oracle.w4_matmul_ref(xh, W["qw"], W["scales"], W["zp"], 3072, 3072), units,
                                budget / 4)
        out[key]["cpu_baseline"] = _cpu(round(r, 6), unit, f"oracle w4_matmul_ref, one 3072x3072 weight at M={M}",
                                        n, el)
    return out


def run_configs(args, wl, peaks, clocks) -> dict:
    """Every workload the decode step does not cover, each with its roofline
    and a bounded oracle sample (N = 1 only)."""
    res = {}
    budget = args.cpu_seconds / 4
    for name, fn in (("config0", lambda: config0(peaks, budget)), ("config2", lambda: config2(peaks, budget)),
                     ("config3", lambda: config3(peaks, budget, wl)), ("config4", lambda: config4(peaks, budget, clocks))):
        t0 = time.perf_counter()
        try:
            res[name] = fn()
        except Exception as e:  # one config failing must not lose the headline line
            res[name] = {"error": f"{type(e).__name__}: {e}"}
        res[name]["wall_s"] = round(time.perf_counter() - t0, 1)
    return res


# ---------------------------------------------------------------- oracle on the host

def _blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [p.get("num_threads", 1) for p in threadpool_info() if p.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return 1


_ORACLE_INPUTS = None


def _oracle_inputs():
    """The decode step's seeded inputs for the oracle (built once, not timed):
    a list of (bytes, call) for the 48 weights and the head."""
    global _ORACLE_INPUTS
    if _ORACLE_INPUTS is None:
        import oracle
        ops = []
        for i, (_, K, N) in enumerate(synth.gpt2_stack_shapes()):
            W = synth.w4_weight(K, N, i)
            x = synth.activations(1, K, i)
            ops.append((synth.w4_bytes(K, N),
                        lambda W=W, x=x: oracle.w4_matmul_ref(x, W["qw"], W["scales"], W["zp"], W["K"], W["N"])))
        H = synth.i8_head(HEAD_K, HEAD_V)
        h = synth.activations(1, HEAD_K, 999)
        ops.append((head_bytes(), lambda: oracle.i8_head_ref(h, H["table"], H["scales"], HEAD_K, HEAD_V)))
        _ORACLE_INPUTS = ops
    return _ORACLE_INPUTS


def _oracle_step(ops, sel=None) -> int:
    """One oracle decode step (or the ops `sel` of it); returns the weight bytes done."""
    done = 0
    for j, (nbytes, call) in enumerate(ops):
        if sel is None or j in sel:
            call()
            done += nbytes
    return done


def _cpu_model() -> str:
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def cpu_baseline(budget_s: float) -> dict:
    """The oracle, as it stands, on this host's cores: whole decode steps of
    the same workload (48 weights + head), repeated until ~budget_s (inputs
    generated once, outside the timing)."""
    ops = _oracle_inputs()
    steps = 0
    t0 = time.perf_counter()
    while True:
        _oracle_step(ops)
        steps += 1
        el = time.perf_counter() - t0
        if el >= budget_s or steps >= 50:
            break
    per_step = el / steps
    return {"value": round((body_bytes() + head_bytes()) / per_step / 1e9, 4), "unit": "GB/s",
            "tokens_per_s": round(1 / per_step, 3), "cores": _blas_threads(), "nproc": os.cpu_count(),
            "cpu_model": _cpu_model(), "kind": "oracle",
            "sample": f"{steps} full decode steps (48 weights + head), {el:.1f} s; numpy unpack/dequantize "
                      f"single-threaded, fp64 matmul on BLAS threads"}


REFERENCE_BUDGET_S = 150.0  # timed seconds of the reference arm, at most (about)


def run_reference(args, world, rank):
    """The oracle as the reference arm, on this host's cores: K timed steps of
    the decode workload. A step is the whole step while K of them fit the
    budget; otherwise a bounded sample of it (a round-robin subset of the 49
    ops, the same for every K-th window), and the metric counts the bytes
    actually processed."""
    if rank != 0:
        return None
    K = max(1, args.steps)
    warm = max(0, min(args.warmup, 1))
    ops = _oracle_inputs()
    t1 = time.perf_counter()
    _oracle_step(ops)  # untimed: warm-up and the per-step estimate
    t1 = time.perf_counter() - t1
    for _ in range(warm - 1):
        _oracle_step(ops)
    nops = len(ops)
    per_step = max(1, min(nops, int(nops * REFERENCE_BUDGET_S / (K * t1))))
    done = 0
    t0 = time.perf_counter()
    for i in range(K):
        sel = None if per_step == nops else {(i * per_step + j) % nops for j in range(per_step)}
        done += _oracle_step(ops, sel)
    el = time.perf_counter() - t0
    ms = el / K * 1e3
    val = done / el / 1e9
    sample = (f"{K} full decode steps (48 weights + head) on the host" if per_step == nops else
              f"{K} steps of {per_step} of the 49 ops each (48 weights + head, round-robin), "
              f"{done / 1e9:.2f} GB of weights in {el:.1f} s on the host")
    cb = {"value": round(val, 4), "unit": "GB/s", "cores": _blas_threads(), "nproc": os.cpu_count(),
          "cpu_model": _cpu_model(), "kind": "oracle", "sample": sample}
    step_ms = (body_bytes() + head_bytes()) / (val * 1e9) * 1e3  # a whole step at the measured rate
    return {"impl": "reference", "metric": METRIC, "value": round(val, 4), "unit": "GB/s", "n_gpus": world,
            "steps": K, "warmup": warm, "ms_per_step": round(step_ms, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": WORKLOAD, "M": 1, "weight_bytes_per_step": body_bytes() + head_bytes()},
            "tokens_per_s": round(1e3 / step_ms, 3), "cpu_baseline": cb,
            "e2e": {"value": round(val, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def profile_case(name: str, calls: int) -> None:
    """Run one workload's kernels `calls` times (no timing, no output but one
    line) so that a profiler can capture them: "step" (the decode step in one
    launch: the 48 GPT-2 weights and the head, streaming layouts, M = 1),
    "body" (the 48 GPT-2 weights in the streaming layout, M = 1),
    "decode-3p8b" / "decode-3p8b-m8" (four layers of the 3.8B-shaped stack, 16
    weights, 290 MB: the streaming GEMV at M = 1, the page-format split-K
    GEMV at M = 8), "head" (the int8 head, streaming
    layout, M = 1), "head-tile" / "head-tile-m8" (the int8 head in the tile
    layout, tensor cores, M = 1 / 8), "prefill-gpt2" (the 48 weights in the tile layout at
    M = 58), "prefill-3p8b" (one 3.8B-shaped layer, 4 weights in the tile
    layout, at M = 2048)."""
    import torch
    import int8_weight_quantized_w4_b200 as w4
    dev = torch.device("cuda", 0)
    lib = w4.lib()
    hs = int(torch.cuda.current_stream().cuda_stream)
    if name in ("body", "step", "prefill-gpt2", "prefill-3p8b"):
        shapes = synth.gpt2_stack_shapes() if name != "prefill-3p8b" else synth.dense38_stack_shapes()[:4]
        M = {"body": 1, "step": 1, "prefill-gpt2": synth.GPT2_PROMPT, "prefill-3p8b": 2048}[name]
        items = []
        for i, (_, K, N) in enumerate(shapes):
            W = synth.w4_weight(K, N, i)
            qw, sc, zp = (torch.from_numpy(W[k]).to(dev) for k in ("qw", "scales", "zp"))
            rep = w4.w4_repack if name in ("body", "step") else w4.w4t_repack
            items.append({"x": torch.from_numpy(synth.activations(M, K, i)).to(dev), "wr": rep(qw, sc, zp, K, N),
                          "y": torch.empty((M, N), device=dev), "K": K, "N": N})
        descs = w4.make_rdescs(items)
        if name == "body":
            run = lambda: _ok(lib.w4r_matmul_grouped(descs, len(descs), hs), lib, "w4r")
        elif name == "step":
            H = synth.i8_head(HEAD_K, HEAD_V)
            tr = w4.i8_head_repack(torch.from_numpy(H["table"]).to(dev), torch.from_numpy(H["scales"]).to(dev),
                                   HEAD_K, HEAD_V)
            h = torch.from_numpy(synth.activations(1, HEAD_K, 999)).to(dev)
            lg = torch.empty((1, HEAD_V), device=dev)
            run = lambda: _ok(lib.w4r_decode_step(descs, len(descs), h.data_ptr(), tr.data_ptr(), HEAD_K, HEAD_V,
                                                  lg.data_ptr(), hs), lib, "w4r_decode_step")
        else:
            scratch = torch.empty(max(w4.w4t_workspace_size(descs), 16), dtype=torch.uint8, device=dev)
            run = lambda: _ok(lib.w4t_matmul_grouped(descs, len(descs), scratch.data_ptr(), scratch.numel(), hs), lib,
                              "w4t")
    elif name in ("decode-3p8b", "decode-3p8b-m8"):
        gen = torch.Generator(device=dev)
        gen.manual_seed(synth.BASE_SEED + 38)
        M = 8 if name.endswith("m8") else 1
        items = []
        for _, K, N in synth.dense38_stack_shapes()[:16]:
            qw = torch.randint(0, 256, (K * N // 2,), dtype=torch.uint8, device=dev, generator=gen)
            sc = torch.empty((K // 32, N), device=dev).uniform_(0.005, 0.02, generator=gen)
            zp = torch.randint(0, 256, (K // 32 * N // 2,), dtype=torch.uint8, device=dev, generator=gen)
            it = {"x": torch.randn((M, K), device=dev, generator=gen), "y": torch.empty((M, N), device=dev), "K": K,
                  "N": N}
            if M == 1:
                it["wr"] = w4.w4_repack(qw, sc, zp, K, N)
            else:
                it.update({"qw": qw, "scales": sc, "zp": zp})
            items.append(it)
        if M == 1:
            descs = w4.make_rdescs(items)
            run = lambda: _ok(lib.w4r_matmul_grouped(descs, len(descs), hs), lib, "w4r")
        else:
            descs = w4.make_descs(items)
            ws = torch.zeros(max(w4.w4_matmul_grouped_workspace_size(descs), 16), dtype=torch.uint8, device=dev)
            run = lambda: _ok(lib.w4_matmul_grouped(descs, len(descs), ws.data_ptr(), ws.numel(), hs), lib,
                              "w4_matmul_grouped")
    elif name in ("head-tile", "head-tile-m8"):
        H = synth.i8_head(HEAD_K, HEAD_V)
        tt = w4.i8t_head_repack(torch.from_numpy(H["table"]).to(dev), torch.from_numpy(H["scales"]).to(dev),
                                HEAD_K, HEAD_V)
        M = 8 if name == "head-tile-m8" else 1
        h = torch.from_numpy(synth.activations(M, HEAD_K, 998)).to(dev)
        lg = torch.empty((M, HEAD_V), device=dev)
        run = lambda: _ok(lib.i8t_head_logits(h.data_ptr(), HEAD_K, tt.data_ptr(), HEAD_K, HEAD_V, M, lg.data_ptr(),
                                              HEAD_V, hs), lib, "i8t")
    elif name == "head":
        H = synth.i8_head(HEAD_K, HEAD_V)
        tr = w4.i8_head_repack(torch.from_numpy(H["table"]).to(dev), torch.from_numpy(H["scales"]).to(dev),
                               HEAD_K, HEAD_V)
        h = torch.from_numpy(synth.activations(1, HEAD_K, 999)).to(dev)
        lg = torch.empty((1, HEAD_V), device=dev)
        run = lambda: _ok(lib.i8r_head_logits(h.data_ptr(), tr.data_ptr(), HEAD_K, HEAD_V, lg.data_ptr(), hs), lib,
                          "i8r")
    else:
        raise SystemExit(f"unknown profile case {name}")
    torch.cuda.synchronize()
    for _ in range(calls):
        run()
    torch.cuda.synchronize()
    print(json.dumps({"profile_case": name, "calls": calls}), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--seconds", type=float, default=1.0,
                    help="device seconds of the timed step replays (the body and head alone get half each)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-configs", action="store_true", help="skip the per-config measurements (configs 0, 2, 3, 4)")
    ap.add_argument("--profile-case", choices=["step", "body", "decode-3p8b", "decode-3p8b-m8", "head", "head-tile", "head-tile-m8", "prefill-gpt2", "prefill-3p8b"],
                    default=None,
                    help="only run one workload's kernels a few times, for a profiler (see profiles/)")
    ap.add_argument("--calls", type=int, default=4, help="calls of --profile-case")
    args = ap.parse_args()
    if args.profile_case:
        profile_case(args.profile_case, args.calls)
        return
    if args.impl == "reference":
        world = int(os.environ.get("WORLD_SIZE", "1"))
        rank = int(os.environ.get("RANK", "0"))
        line = run_reference(args, world, rank)
        if line is not None:
            print(json.dumps(line), flush=True)
        return
    world, rank, local = dist_init(args.gpus)
    try:
        line = run_ours(args, world, rank, local)
        if rank == 0:
            print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
