"""Throughput of the hot path on B200: block self-attention + windowed
cross-attention over one packed batch per step.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl nle|reference]
                    [--config 1..5] [--seed S]

A step is one pass of the whole path over one packed batch: the 200-frame
block self-attention of the encoder and the projector's 15-frame / 3-query
windowed cross-attention over the same utterances.  The default workload is
config 4, the batch-128 one (128 utterances of 100-800 frames, 16 heads x
64, the model card's batch-128 throughput setting); --config selects another
of the five synthetic workloads.  Inputs are seeded N(0,1) bf16, resident in
HBM before timing; each kernel is also timed alone (median over the K
steps).  One JSON line is printed by rank 0.

The `configs` field of the line times the kernels on all five workloads
(median of >= 50 launches each, L2 flushed by a write of twice the L2 size before every
launch, and back to back for the two small workloads that fit in L2).

Multi-GPU (torchrun, one process per GPU): data-parallel replicas, each
rank runs its own batch of the same shape (weak scaling); there is no
collective on the data path.  Time is the max over ranks.

--impl reference times the fp64 CPU oracle (the test oracle, untuned) on the
host cores for the same metric: each step is a bounded sample of whole
utterances of the same workload.
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
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from chunked_block_self_b200 import workloads as wl  # noqa: E402

METRIC = "block-attn TFLOP/s & encoder frames/s on 1 B200; % of dense BF16 peak"
CFG = 4          # the headline workload; --config changes it
SEED = None      # --seed; None: the config's default seed
B, W, QW, D = 200, 15, 3, 64

# ncu DRAM traffic (dram__bytes_read.sum + dram__bytes_write.sum) of each
# kernel on the batch-128 workload, per unit of algorithmic bytes so that it
# scales to any launch; valid only for the kernel source whose hash is given
# (reported as null once the source changes).  Read below 1.0: part of the
# output is still dirty in the 126 MB L2 when the launch ends.
NCU_TRAFFIC = {
    "block_attn": {"files": ('block_attn_sm100a.cu', 'attn_softmax.cuh', 'nle_device.cuh'),
                   "source_sha256": "2a512fbb082b30453f6b625a669dad782a2366369105c5f0acea1ed58d417a24",
                   "traffic_over_algorithmic": (378595072 + 67184128) / 482533376,
                   "tensor_pipe_pct": 19.1},
    "window_xattn": {"files": ('window_xattn_sm100a.cu', 'nle_device.cuh'),
                    "source_sha256": "44c247f038150ebc19ef8299c838232d7615b43f47cd5c35f050e4399dac1c65",
                    "traffic_over_algorithmic": (265965568 + 7668992) / 290320384},
    # full-utterance attention: the long-clip workload, the same launch as the bench's
    "varlen_attn": {"files": ('varlen_attn_sm100a.cu', 'attn_softmax.cuh', 'nle_device.cuh'),
                   "source_sha256": "f687eb567c9643601dca019254550645b968652fd7c4f8d2a9e54cf02edc976e",
                   "traffic_over_algorithmic": (345912064 + 88160512) / 439304192,
                   "tensor_pipe_pct": 27.2},
    # fused projection + block attention on the batch-128 workload (d_model 1024,
    # 16 heads); X is read from DRAM about four times (the CTAs of the 16 heads
    # reach a row at different times and X is about the size of L2), and DRAM
    # writes sit below the output's bytes because part of it is still in L2
    # when the kernel ends
    "qkv_attn": {"files": ('qkv_attn_sm100a.cu', 'attn_softmax.cuh', 'nle_device.cuh'),
                 "source_sha256": "6cf4f4b5b448092c88c5f08d7fdf1ac3700dc546ffb1959819c0fe2b3f61e9ee",
                 "traffic_over_algorithmic": (511541248 + 110533632) / 247564288,
                 "tensor_pipe_pct": 38.5},
    # posterior pooling over the whole batch-128 workload (58,903 frames)
    "posterior_pool": {"files": ('pool_sm100a.cu', 'nle_device.cuh'),
                      "source_sha256": "9c30451e84816fe70b5bf4476faf488635d46f14fb73b2cdcfebbd7b1724dfca",
                      "traffic_over_algorithmic": (150827776 + 28794368) / 211398236},
    # CTC argmax: captured on 16 utterances (3,300 rows, 662.4 MB); traffic grows
    # with rows, so the ratio is applied to the full batch
    "ctc_argmax": {"files": ('ctc_sm100a.cu', 'nle_device.cuh'),
                   "source_sha256": "af3b98a165bb857fe898335cb7332fb1bcf9b440f0dcdd33ddc3ec7de87ee833",
                   "traffic_over_algorithmic": (662674944 + 3137536) / 662369464},
}


def kernel_source_sha(kernel: str = "block_attn") -> str:
    h = hashlib.sha256()
    for f in NCU_TRAFFIC[kernel]["files"]:
        with open(os.path.join(ROOT, "chunked_block_self_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()


def ncu_traffic(kernel: str, algorithmic_bytes: int):
    e = NCU_TRAFFIC[kernel]
    if e["source_sha256"] != kernel_source_sha(kernel):
        return None
    return e["traffic_over_algorithmic"] * algorithmic_bytes


def ncu_tensor_pipe_pct(kernel: str):
    """sm__pipe_tensor_cycles_active (% of active cycles) from the ncu capture
    of `kernel`, or None when the source changed since (or none was taken).
    It counts the padded MMA work (keys up to ceil16(L), 128-row tiles)."""
    e = NCU_TRAFFIC.get(kernel)
    if not e or "tensor_pipe_pct" not in e or e["source_sha256"] != kernel_source_sha(kernel):
        return None
    return e["tensor_pipe_pct"]


def measured_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), float(p["bf16_tflops"]), float(p["bf16_tflops_sustained"]), "measured"
    except Exception:
        return 6650.0, 1590.0, 1400.0, "fallback"


# ------------------------------------------------------------------ work counts
def block_work(lengths, heads):
    """Algorithmic FLOPs and bytes of block attention (padding excluded)."""
    s1 = s2 = 0
    for t in lengths:
        full, rem = divmod(int(t), B)
        s1 += full * B + rem
        s2 += full * B * B + rem * rem
    flops = 4 * D * heads * s2            # QK^T and PV, 2 flops per MAC
    bytes_ = 4 * 2 * D * heads * s1       # Q, K, V read + O written, bf16
    return flops, bytes_


def window_work(lengths, heads):
    n_win = s1 = 0
    for t in lengths:
        nw = -(-int(t) // W)
        n_win += nw
        s1 += int(t)
    flops = 4 * QW * D * heads * s1
    bytes_ = 2 * D * heads * (2 * QW * n_win + 2 * s1)   # Q + O rows, K + V rows
    return flops, bytes_, n_win


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """Polls NVML (SM clock, clock-event reasons) while the timed region runs."""

    NAMES = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
             0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown", 0x2: "applications_clocks_setting",
             0x1: "gpu_idle", 0x10: "sync_boost"}

    def __init__(self, device_index: int):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self._stop = threading.Event()
        self._h = None
        try:
            import pynvml
            pynvml.nvmlInit()
            p = torch.cuda.get_device_properties(device_index)
            bus = f"{p.pci_domain_id:08X}:{p.pci_bus_id:02X}:{p.pci_device_id:02X}.0"
            self._h = pynvml.nvmlDeviceGetHandleByPciBusId(bus)
            self._nv = pynvml
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception as e:  # no NVML: report that, no clocks
            self.error = repr(e)

    def _run(self):
        nv = self._nv
        get_reasons = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            nv.nvmlDeviceGetCurrentClocksThrottleReasons
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
                r = get_reasons(self._h)
                for bit, name in self.NAMES.items():
                    if r & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(0.002)

    def __enter__(self):
        if self._h is not None:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *a):
        if self._h is not None:
            self._stop.set()
            self._t.join()

    def summary(self):
        if self._h is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "note": getattr(self, "error", "")}
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons - {"gpu_idle"}),
                "samples": len(self.samples)}


# ------------------------------------------------------------------ distributed
def dist_setup(n_gpus):
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    return rank, world, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int) -> float:
    """The largest of every rank's x, on every rank (one all-reduce; NCCL
    reduces CUDA tensors, gloo CPU ones)."""
    if world == 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ------------------------------------------------------------------ CPU oracle timing
def oracle_sample(lengths, q, k, v, cu, qw, kw, vw, heads, budget_s: float):
    """Time the fp64 oracle on whole utterances of the workload, in order
    (wrapping around to the first utterance after the last), until `budget_s`
    seconds have passed.  Returns (flops, frames, seconds, utterances,
    threads)."""
    import oracle
    starts = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int64)
    qstarts = np.concatenate([[0], np.cumsum([QW * -(-int(t) // W) for t in lengths])]).astype(np.int64)
    flops = frames = 0
    n_utt = 0
    t0 = time.perf_counter()
    while n_utt == 0 or time.perf_counter() - t0 < budget_s:
        i = n_utt % len(lengths)
        t, a, qrow = int(lengths[i]), int(starts[i]), int(qstarts[i])
        local = np.array([0, t], np.int32)
        oracle.block_attn(q[a:a + t], k[a:a + t], v[a:a + t], local, block_frames=B, n_threads=0)
        nw = -(-t // W)
        oracle.window_xattn(qw[qrow:qrow + QW * nw], kw[a:a + t], vw[a:a + t], local, W, QW, n_threads=0)
        f1, _ = block_work([t], heads)
        f2, _, _ = window_work([t], heads)
        flops += f1 + f2
        frames += t
        n_utt += 1
    return flops, frames, time.perf_counter() - t0, n_utt, oracle.threads_used(0)


def cpu_info():
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


# ------------------------------------------------------------------ arms
WORKLOAD_NAMES = {
    1: "single utterance: 400 frames (8 s at 50 Hz), 8 heads x 64",
    2: "800-frame bucket: one utterance of 800 frames (16 s), 16 heads x 64, values x0.5",
    3: "long clips: 16 utterances of 1950-4700 frames (39-94 s), partial last blocks, 16 heads x 64",
    4: "batch-128: 128 utterances of 100-800 frames (2-16 s at 50 Hz), 16 heads x 64",
    5: "projector batch: 64 utterances of 4700 frames (94 s), 16 heads x 64",
}


def base_seed(rank):
    return (wl.default_seed(CFG) if SEED is None else SEED) + rank


def build_inputs(rank):
    """Block inputs (host) of the headline workload and window inputs over the
    same utterances; the projector workload's window inputs are those of
    config 5."""
    seed = base_seed(rank)
    x = wl.block_inputs(CFG, seed=seed)
    lengths, heads = x["lengths"], x["heads"]
    n_win = sum(-(-int(t) // W) for t in lengths)
    if CFG == 5:
        y = wl.window_inputs(QW * n_win, cfg=5, seed=seed)
    else:
        y = wl.window_inputs(QW * n_win, cfg=None, lengths=lengths, heads=heads, seed=seed + 100)
    return x, y


def config_dict(x, n_win):
    gb = (4 * x["q"].numel() * 2 + (2 * QW * n_win + 2 * int(x["total"])) * int(x["heads"]) * D * 2) / 1e9
    l2 = (f"inputs ~{gb:.2f} GB per rank > 126 MB L2; not flushed between steps" if gb > 0.126 else
          f"inputs ~{gb * 1e3:.0f} MB per rank fit in the 126 MB L2; back to back, hot (the `configs` "
          "field also times them L2-flushed)")
    return {"workload": f"config {CFG}, {WORKLOAD_NAMES[CFG]}; 200-frame block self-attention + "
                        "15-frame/3-query windowed cross-attention over the same utterances",
            "config": CFG, "n_seq": int(len(x["lengths"])), "total_frames": int(x["total"]),
            "heads": int(x["heads"]), "d_head": D, "block_frames": B, "window_frames": W,
            "queries_per_window": QW, "windows": int(n_win), "seed": base_seed(0), "l2": l2,
            "parallelism": "data-parallel replicas by utterance (no collective)"}


def run_reference(args, rank, world):
    if rank != 0:
        return 0
    x, y = build_inputs(0)
    lengths, heads = x["lengths"], x["heads"]
    n_win = sum(-(-int(t) // W) for t in lengths)
    steps, warm = args.steps, args.warmup
    budget = max(0.05, min(2.0, 90.0 / (steps + warm)))   # whole run stays within a few minutes
    q, k, v, cu = x["q"], x["k"], x["v"], x["cu"]
    for _ in range(warm):
        oracle_sample(lengths, q, k, v, cu, y["q"], y["k"], y["v"], heads, budget)
    tot_f = tot_fr = tot_t = 0.0
    utts = 0
    for _ in range(steps):
        f, fr, t, nu, threads = oracle_sample(lengths, q, k, v, cu, y["q"], y["k"], y["v"], heads, budget)
        tot_f += f
        tot_fr += fr
        tot_t += t
        utts += nu
    value = tot_f / tot_t / 1e12
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus,
            "steps": steps, "warmup": warm, "ms_per_step": 1e3 * tot_t / steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": config_dict(x, n_win),
            "frames_per_s": tot_fr / tot_t,
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
                             "sample": f"{utts} whole utterances over {steps} steps (block + window oracle, "
                                       f"~{budget:.2f} s per step), {cpu_info()}"},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def l2_flush_buffer(dev):
    """A buffer twice the device's L2 (its size read at run time): writing it
    before a launch evicts everything the previous launch left in L2."""
    l2 = int(getattr(torch.cuda.get_device_properties(dev), "L2_cache_size", 0) or (126 << 20))
    return torch.empty(2 * l2, dtype=torch.uint8, device=dev)


def time_launches(fn, stream, reps, flush=None, clean=False):
    """Median and mean (ms) of `reps` launches of fn, each bracketed by CUDA
    events on `stream` (torch's current stream); with `flush`, a write of
    that buffer (larger than L2) precedes every launch (and keeps the GPU
    busy while the launch is queued, so the first event is taken right
    before the kernel starts).  The write leaves L2 full of dirty lines,
    which the timed launch then writes back as it evicts them; with
    `clean`, the buffer is also read back before the launch, so L2 holds
    only clean lines of it (still none of the kernel's inputs)."""
    ts = []
    for _ in range(reps):
        if flush is not None:
            flush.fill_(1)
            if clean:
                flush.view(torch.int64).sum()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        fn()
        b.record(stream)
        b.synchronize()
        ts.append(a.elapsed_time(b))
    return statistics.median(ts), float(np.mean(ts))


def time_back_to_back(fn, stream, reps):
    """Mean time (ms) of one launch of fn in a run of `reps` launches queued
    back to back between two CUDA events (hot L2, no host gaps), taken as the
    median over 5 such runs."""
    runs = []
    for _ in range(5):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(reps):
            fn()
        b.record(stream)
        b.synchronize()
        runs.append(a.elapsed_time(b) / reps)
    return statistics.median(runs)


def measure_configs(nle, dev, stream, reps, rank, hbm_peak, tf_peak):
    """Each kernel of the path on each of the five workloads, alone: the
    block kernel on configs 1-4, the window kernel on configs 4 and 5 (the
    projector batch: 64 x 4700 frames, 20,096 windows).  Inputs are drawn on
    the device (seeded torch generator, same distributions as the host
    recipe).  Median of `reps` launches with L2 flushed before each; the
    two small workloads (which fit in L2) are also timed hot: `reps`
    launches queued back to back, mean per launch (median of 5 runs)."""
    sp = stream.cuda_stream
    flush = l2_flush_buffer(dev)
    res = {}
    for c in (1, 2, 3, 4, 5):
        seed = wl.default_seed(c) + rank
        lengths = wl.draw_lengths(c, seed)
        heads = wl.CONFIGS[c].heads
        total = int(sum(int(t) for t in lengths))
        cu = torch.from_numpy(wl.cu_seqlens(lengths)).to(dev)
        e = {"workload": WORKLOAD_NAMES[c], "n_seq": int(len(lengths)), "total_frames": total, "heads": heads,
             "seed": seed, "reps": reps, "timing": "median of CUDA-event times of single launches"}
        if c <= 4:
            x = wl.block_inputs(c, seed=seed, device=dev)
            out = torch.empty_like(x["q"])

            def blk():
                nle.nle_block_attn_fwd(x["q"], x["k"], x["v"], out, cu, len(lengths), total, heads, D, B,
                                       stream=sp)

            for _ in range(3):
                blk()
            f, by = block_work(lengths, heads)
            med, mean = time_launches(blk, stream, reps, flush)
            blk_e = {"us_flushed": 1e3 * med, "us_flushed_mean": 1e3 * mean,
                     "tflops": f / (med * 1e-3) / 1e12, "gbs": by / (med * 1e-3) / 1e9,
                     "pct_of_hbm_peak": 100.0 * by / (med * 1e-3) / 1e9 / hbm_peak,
                     "pct_of_dense_bf16_peak": 100.0 * f / (med * 1e-3) / 1e12 / tf_peak,
                     "frames_per_s": total / (med * 1e-3), "algorithmic_flops": f, "algorithmic_bytes": by,
                     "hbm_floor_us": 1e6 * by / (hbm_peak * 1e9)}
            if by < (96 << 20):   # fits in L2: the layer-after-layer case
                hot = time_back_to_back(blk, stream, reps)
                blk_e.update({"us_hot": 1e3 * hot, "tflops_hot": f / (hot * 1e-3) / 1e12,
                              "frames_per_s_hot": total / (hot * 1e-3)})
            if c == 2:   # the same call in each of the encoder's 16 layers
                blk_e["frames_per_s_16_layer_stack_flushed"] = total / (16 * med * 1e-3)
                blk_e["frames_per_s_16_layer_stack_hot"] = total / (16 * hot * 1e-3)
            e["block_attn"] = blk_e
            del x, out
        if c >= 4:
            n_win = sum(-(-int(t) // W) for t in lengths)
            y = wl.window_inputs(QW * n_win, cfg=c, seed=seed, device=dev)
            ow = torch.empty_like(y["q"])

            def win():
                nle.nle_window_xattn_fwd(y["q"], y["k"], y["v"], ow, cu, len(lengths), total, QW * n_win, heads,
                                         D, W, QW, stream=sp)

            for _ in range(3):
                win()
            f, by, _ = window_work(lengths, heads)
            med, mean = time_launches(win, stream, reps, flush)
            e["window_xattn"] = {"windows": int(n_win), "us_flushed": 1e3 * med, "us_flushed_mean": 1e3 * mean,
                                 "gbs": by / (med * 1e-3) / 1e9,
                                 "pct_of_hbm_peak": 100.0 * by / (med * 1e-3) / 1e9 / hbm_peak,
                                 "tflops": f / (med * 1e-3) / 1e12, "algorithmic_bytes": by,
                                 "hbm_floor_us": 1e6 * by / (hbm_peak * 1e9)}
            del y, ow
        res[str(c)] = e
        torch.cuda.empty_cache()
    del flush
    torch.cuda.empty_cache()
    return res


def measure_qkv_attn(nle, dev, stream, reps, rank, lengths, tf_peak):
    """The QKV projection fused with block attention on the step's
    utterances at the encoder's width (d_model 1024 = 16 heads x 64): X
    N(0, 1), W N(0, 1/1024), bias N(0, 0.25), all bf16, drawn on the device.
    Median of `reps` launches, L2 flushed before each.  The same work done
    unfused -- the projection as one cuBLAS GEMM (torch) writing Q|K|V to
    memory, then the block kernel reading them -- is timed beside it."""
    sp = stream.cuda_stream
    heads, dm = 16, 1024
    cu_h = wl.cu_seqlens(lengths)
    T = int(cu_h[-1])
    cu = torch.from_numpy(cu_h).to(dev)
    seed = wl.default_seed(CFG) + 5000 + rank
    x = wl.device_normal((T, dm), 1.0, seed, dev)
    w = wl.device_normal((3 * heads * 64, dm), 1.0 / 32.0, seed + 1, dev)
    b = wl.device_normal((3 * heads * 64,), 0.5, seed + 2, dev)
    out = torch.empty((T, heads, 64), dtype=torch.bfloat16, device=dev)
    flush = l2_flush_buffer(dev)

    def fused():
        nle.nle_block_attn_qkv_fwd(x, w, b, out, cu, block_frames=B, stream=sp)

    qkv = torch.empty((T, 3 * heads * 64), dtype=torch.bfloat16, device=dev)
    out2 = torch.empty_like(out)

    def unfused():
        torch.addmm(b, x, w.t(), out=qkv)
        q3 = qkv.view(T, 3, heads, 64)
        nle.nle_block_attn_fwd_ex(q3[:, 0], q3[:, 1], q3[:, 2], out2, cu, len(lengths), T, heads, D, B,
                                  row_stride_qkv=3 * heads * 64, stream=sp)

    for _ in range(3):
        fused()
        unfused()
    med, mean = time_launches(fused, stream, reps, flush)
    umed, _ = time_launches(unfused, stream, reps, flush)
    f_att, _ = block_work(lengths, heads)
    f_proj = 2 * T * dm * 3 * heads * 64
    flops = f_proj + f_att
    tflops = flops / (med * 1e-3) / 1e12
    byt = 2 * (T * dm + 3 * heads * 64 * dm + 3 * heads * 64 + T * heads * 64)   # X, W, b read; O written
    res = {"workload": f"config {CFG} utterances ({len(lengths)}, {T} frames), d_model {dm}, {heads} heads x 64, "
                       "synthetic X ~ N(0,1), W ~ N(0,1/1024), bias ~ N(0,0.25), bf16",
           "ms": med, "ms_mean": mean,
           "timing": f"median of {reps} launches, L2 flushed (a write of twice the L2 size) before each",
           "algorithmic_flops": flops, "projection_flops": f_proj, "attention_flops": f_att,
           "tflops": tflops, "pct_of_dense_bf16_peak": 100.0 * tflops / tf_peak,
           "roofline": {"bound": "tensor", "achieved": tflops, "peak": tf_peak, "unit": "TFLOP/s",
                        "frac": tflops / tf_peak, "ai_flop_per_byte": flops / byt},
           "tensor_pipe_pct": ncu_tensor_pipe_pct("qkv_attn"), "traffic": ncu_traffic("qkv_attn", byt),
           "unfused_ms": umed, "unfused_tflops": flops / (umed * 1e-3) / 1e12,
           "unfused": "torch.addmm (cuBLAS) X W^T + b -> Q|K|V in memory, then the block kernel",
           "speedup_vs_unfused": umed / med, "kernels": 1}
    del x, w, b, out, qkv, out2, flush
    torch.cuda.empty_cache()
    return res


def run_nle(args, rank, world, local):
    from chunked_block_self_b200 import nle

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    x, y = build_inputs(rank)
    lengths, heads = x["lengths"], x["heads"]
    n_win = sum(-(-int(t) // W) for t in lengths)
    assert nle.window_query_rows(x["cu"], W, QW) == QW * n_win
    f_blk, by_blk = block_work(lengths, heads)
    f_win, by_win, _ = window_work(lengths, heads)
    flops_step = f_blk + f_win
    frames_step = int(x["total"])

    # device-resident inputs
    q, k, v = (x[n].to(dev) for n in ("q", "k", "v"))
    cu = torch.from_numpy(x["cu"]).to(dev)
    qw, kw, vw = (y[n].to(dev) for n in ("q", "k", "v"))
    out = torch.empty_like(q)
    ow = torch.empty_like(qw)
    total = int(x["total"])
    n_seq = len(lengths)
    stream = torch.cuda.current_stream()
    sp = stream.cuda_stream

    def step():
        nle.nle_block_attn_fwd(q, k, v, out, cu, n_seq, total, heads, D, B, stream=sp)
        nle.nle_window_xattn_fwd(qw, kw, vw, ow, cu, n_seq, total, QW * n_win, heads, D, W, QW, stream=sp)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    barrier(world)

    K = args.steps
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(2 * K + 1)]
    clocks = ClockSampler(local)
    with clocks:
        torch.cuda.synchronize()
        barrier(world)
        torch.cuda.synchronize()
        start = torch.cuda.Event(enable_timing=True)
        end = torch.cuda.Event(enable_timing=True)
        start.record(stream)
        ev[0].record(stream)
        for i in range(K):
            nle.nle_block_attn_fwd(q, k, v, out, cu, n_seq, total, heads, D, B, stream=sp)
            ev[2 * i + 1].record(stream)
            nle.nle_window_xattn_fwd(qw, kw, vw, ow, cu, n_seq, total, QW * n_win, heads, D, W, QW, stream=sp)
            ev[2 * i + 2].record(stream)
        end.record(stream)
        torch.cuda.synchronize()
        barrier(world)
        torch.cuda.synchronize()
    elapsed_ms = start.elapsed_time(end)
    blk_ts = [ev[2 * i].elapsed_time(ev[2 * i + 1]) for i in range(K)]
    win_ts = [ev[2 * i + 1].elapsed_time(ev[2 * i + 2]) for i in range(K)]
    t_blk, t_win = statistics.median(blk_ts), statistics.median(win_ts)
    elapsed_ms = max_over_ranks(elapsed_ms, world)
    ms_step = elapsed_ms / K

    # ---- end to end through the public API with HOST buffers: one
    # nle_path_fwd_host call per step copies the step's inputs from pinned
    # host memory, runs both kernels and copies both outputs back (chunks of
    # utterances pipelined over two streams inside the library)
    host = {"q": x["q"].pin_memory(), "k": x["k"].pin_memory(), "v": x["v"].pin_memory(),
            "qw": y["q"].pin_memory(), "kw": y["k"].pin_memory(), "vw": y["v"].pin_memory(),
            "cu": torch.from_numpy(np.ascontiguousarray(x["cu"])).pin_memory()}
    host["out"] = torch.empty(out.shape, dtype=out.dtype, pin_memory=True)
    host["out_w"] = torch.empty(ow.shape, dtype=ow.dtype, pin_memory=True)
    devb = {"q": q, "k": k, "v": v, "qw": qw, "kw": kw, "vw": vw, "out": out, "out_w": ow, "cu": cu}
    h2d = sum(host[n].numel() * host[n].element_size() for n in ("q", "k", "v", "qw", "kw", "vw", "cu"))
    d2h = sum(host[n].numel() * host[n].element_size() for n in ("out", "out_w"))

    def e2e_step():
        nle.nle_path_fwd_host(host, devb, block_frames=B, window_frames=W, queries_per_window=QW, stream=sp)

    ke = max(3, min(K, 20))
    for _ in range(3):
        e2e_step()
    torch.cuda.synchronize()
    barrier(world)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(ke):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world) / ke
    barrier(world)

    # ---- CPU baseline: the oracle on the host cores, rank 0 at N=1 only
    cpu_base = None
    if world == 1 and not args.no_cpu_baseline:
        f, fr, t, nu, threads = oracle_sample(lengths, x["q"], x["k"], x["v"], x["cu"], y["q"], y["k"], y["v"],
                                              heads, args.cpu_seconds)
        cpu_base = {"value": f / t / 1e12, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
                    "frames_per_s": fr / t,
                    "sample": f"{nu} whole utterances of the {n_seq}-utterance batch, in order, wrapping "
                              f"({fr} frames; block + window oracle, {t:.1f} s, fp64, {threads} threads), "
                              f"{cpu_info()}"}

    # ---- downstream of the encoder, on the same utterances: the BPE head's
    # posterior-weighted pooling (windows of 2 frames, weights from a
    # 256-class mid-layer head) and CTC greedy decoding of the BPE head's
    # logits (100,353 classes, one row per pooled window); inputs generated
    # on the device, L2 flushed before every timed launch
    pool = ctc = None
    if not args.no_ctc:
        del host, devb
        torch.cuda.empty_cache()
        clen = lengths if args.ctc_utts <= 0 else lengths[:args.ctc_utts]
        cu_f = torch.from_numpy(wl.cu_seqlens(clen)).to(dev)
        rows_u = [-(-int(t) // wl.POOL_FRAMES) for t in clen]
        cu_r = torch.from_numpy(wl.cu_seqlens(rows_u)).to(dev)
        n_rows, n_fr = int(sum(rows_u)), int(sum(int(t) for t in clen))
        flush = l2_flush_buffer(dev)

        def timed(fn, reps):
            return time_launches(fn, stream, reps, flush)[0]   # median

        px = wl.pool_inputs(clen, seed=wl.default_seed(CFG) + 4000 + rank, device=dev)
        pooled = torch.empty((n_rows, wl.HIDDEN_DIM), dtype=torch.bfloat16, device=dev)
        pw = torch.empty(n_fr, dtype=torch.float32, device=dev)

        def pool_step():
            nle.nle_posterior_pool_fwd(px["hidden"], px["logits"], cu_f, pooled, pw, wl.POOL_FRAMES, stream=sp)

        for _ in range(3):
            pool_step()
        pool_ms = timed(pool_step, 50)
        pool_clean_ms = time_launches(pool_step, stream, 50, flush, clean=True)[0]
        # hidden and logits once, pooled rows and weights written
        pool_bytes = n_fr * (wl.HIDDEN_DIM + wl.CHAR_CLASSES) * 2 + n_rows * wl.HIDDEN_DIM * 2 + n_fr * 4
        pool = {"frames": n_fr, "rows": n_rows, "pool_frames": wl.POOL_FRAMES, "dim": wl.HIDDEN_DIM,
                "char_classes": wl.CHAR_CLASSES, "ms": pool_ms, "gbs": pool_bytes / (pool_ms * 1e-3) / 1e9,
                "algorithmic_bytes": pool_bytes, "traffic": ncu_traffic("posterior_pool", pool_bytes),
                "l2": "flushed (a write of twice the L2 size) before each launch", "kernels": 1,
                "timing": "median of 50 launches",
                # the same launches after the flush is also read back: the
                # flush's dirty lines are written out before the launch
                # instead of during it
                "ms_clean_l2": pool_clean_ms, "gbs_clean_l2": pool_bytes / (pool_clean_ms * 1e-3) / 1e9}
        del px, pooled, pw

        logits = wl.ctc_logits(rows_u, seed=wl.default_seed(CFG) + 3000 + rank, device=dev)
        fcl = torch.empty(n_rows, dtype=torch.int32, device=dev)
        tok = torch.empty_like(fcl)
        ntk = torch.empty(len(clen), dtype=torch.int32, device=dev)

        def ctc_step():
            nle.nle_ctc_greedy_fwd(logits, cu_r, fcl, tok, ntk, stream=sp)

        for _ in range(3):
            ctc_step()
        ctc_ms = timed(ctc_step, 20)
        # logits once; frame classes written, read twice by the collapse;
        # tokens written; one count per utterance
        ctc_bytes = logits.numel() * 2 + n_rows * 12 + len(clen) * 4
        ctc = {"rows": n_rows, "utterances": len(clen), "classes": int(logits.shape[1]), "ms": ctc_ms,
               "rows_per_s": n_rows / (ctc_ms * 1e-3), "gbs": ctc_bytes / (ctc_ms * 1e-3) / 1e9,
               "algorithmic_bytes": ctc_bytes, "l2": "flushed (a write of twice the L2 size) before each launch", "kernels": 2,
               "timing": "median of 20 launches",
               # the argmax kernel's DRAM bytes (logits once, classes written)
               "traffic_argmax": ncu_traffic("ctc_argmax", logits.numel() * 2 + n_rows * 4)}
        del logits, flush
        torch.cuda.empty_cache()

    # ---- full bidirectional attention over whole utterances (the encoder
    # without blocks; the editor's attention) on the long-clip workload:
    # 16 utterances of 1950-4700 frames, 16 heads x 64
    va = None
    if not args.no_varlen:
        xv = wl.block_inputs(3, seed=wl.default_seed(3) + rank)
        qv, kv, vv = (xv[n].to(dev) for n in ("q", "k", "v"))
        cuv = torch.from_numpy(xv["cu"]).to(dev)
        outv = torch.empty_like(qv)

        def va_step():
            nle.nle_varlen_attn_fwd(qv, kv, vv, outv, cuv, stream=sp)

        for _ in range(3):
            va_step()
        torch.cuda.synchronize()
        va_ms, _ = time_launches(va_step, stream, 50)   # median; inputs > L2
        lens_v = [int(t) for t in xv["lengths"]]
        hv_ = int(xv["heads"])
        va_flops = 4 * D * hv_ * sum(t * t for t in lens_v)
        va_bytes = 8 * D * hv_ * sum(lens_v)
        va = {"workload": "long clips: 16 utterances of 1950-4700 frames (39-94 s at 50 Hz), 16 heads x 64, "
                          "full attention inside each utterance",
              "frames": int(sum(lens_v)), "ms": va_ms, "tflops": va_flops / (va_ms * 1e-3) / 1e12,
              "algorithmic_flops": va_flops, "algorithmic_bytes": va_bytes,
              "l2": "inputs ~0.32 GB > 126 MB L2; not flushed", "kernels": 1,
              "timing": "median of 50 launches", "tensor_pipe_pct": ncu_tensor_pipe_pct("varlen_attn"),
              "traffic": ncu_traffic("varlen_attn", va_bytes)}
        del qv, kv, vv, outv

    hbm_peak, tf_peak, tf_sust, peak_src = measured_peaks()
    per_cfg = None
    if not args.no_configs:
        per_cfg = measure_configs(nle, dev, stream, args.config_reps, rank, hbm_peak, tf_peak)
    qkv_att = None
    if not args.no_qkv:
        qkv_att = measure_qkv_attn(nle, dev, stream, args.config_reps, rank, lengths, tf_peak)
    if va is not None:
        # the exp unit's ceiling: one exp per (query row, key, head) at 16
        # ex2 results per clock per SM (4 per SM sub-partition), at the SM
        # clock seen during the timed steps
        mhz = clocks.summary().get("sm_mhz") or 1965.0
        sms = torch.cuda.get_device_properties(dev).multi_processor_count
        exps = va["algorithmic_flops"] / (4 * D)
        va["exp_ceiling_ms"] = 1e3 * exps / (16 * sms * mhz * 1e6)
        va["frac_of_exp_ceiling"] = va["exp_ceiling_ms"] / va["ms"]
        va["pct_of_dense_bf16_peak"] = 100.0 * va["tflops"] / tf_peak
        va["roofline"] = {"bound": "tensor", "achieved": va["tflops"], "peak": tf_peak, "unit": "TFLOP/s",
                          "frac": va["tflops"] / tf_peak,
                          "peak_source": f"{peak_src} (MEASURED_PEAKS.json bf16_tflops)"}
    for extra in (pool, ctc):
        if extra is not None:
            extra["pct_of_hbm_peak"] = 100.0 * extra["gbs"] / hbm_peak
    if pool is not None:
        pool["pct_of_hbm_peak_clean_l2"] = 100.0 * pool["gbs_clean_l2"] / hbm_peak
    achieved_gbs = by_blk / (t_blk * 1e-3) / 1e9
    traffic = ncu_traffic("block_attn", by_blk)
    blk_tflops = f_blk / (t_blk * 1e-3) / 1e12
    value = world * flops_step / (ms_step * 1e-3) / 1e12
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": K, "warmup": args.warmup,
        "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16", "data": "synthetic", "config": config_dict(x, n_win),
        "frames_per_s": world * frames_step / (ms_step * 1e-3),
        "pct_of_dense_bf16_peak": 100.0 * value / (world * tf_peak),
        "block_attn": {"tflops": blk_tflops, "pct_of_dense_bf16_peak": 100.0 * blk_tflops / tf_peak,
                       "achieved_gbs": achieved_gbs, "ms": t_blk, "ms_mean": float(np.mean(blk_ts)),
                       "timing": f"median of {K} launches (CUDA events around each)",
                       "frames_per_s": frames_step / (t_blk * 1e-3),
                       "frames_per_s_16_layer_stack": frames_step / (16 * t_blk * 1e-3),
                       "attainable_tflops": min(tf_peak, f_blk / by_blk * hbm_peak / 1e3),
                       "ai_flop_per_byte": f_blk / by_blk,
                       "tensor_pipe_pct": ncu_tensor_pipe_pct("block_attn")},
        "tensor_pipe_pct": ncu_tensor_pipe_pct("block_attn"),
        "qkv_attn": qkv_att,
        "configs": per_cfg,
        "window_xattn": {"gbs": by_win / (t_win * 1e-3) / 1e9, "ms": t_win, "ms_mean": float(np.mean(win_ts)),
                         "tflops": f_win / (t_win * 1e-3) / 1e12,
                         "pct_of_hbm_peak": 100.0 * by_win / (t_win * 1e-3) / 1e9 / hbm_peak,
                         "algorithmic_bytes": by_win, "traffic": ncu_traffic("window_xattn", by_win)},
        "roofline": {"kernel": "block_attn_kernel", "bound": "hbm", "achieved": achieved_gbs, "peak": hbm_peak,
                     "unit": "GB/s", "frac": achieved_gbs / hbm_peak, "traffic": traffic,
                     "algorithmic_bytes": by_blk, "peak_source": f"{peak_src} (MEASURED_PEAKS.json hbm_gbs)"},
        "clocks": clocks.summary(),
        "e2e": {"value": world * flops_step / (e2e_ms * 1e-3) / 1e12, "unit": "TFLOP/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms, "steps": ke},
        "varlen_attn": va,
        "posterior_pool": pool,
        "ctc_decode": ctc,
        "gpu_launches": 2 * K * world,   # block + window kernel per step, all ranks
        "cpu_baseline": cpu_base,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["nle", "reference"], default="nle")
    ap.add_argument("--cpu-seconds", type=float, default=15.0, help="oracle sample budget (N=1 only)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-ctc", action="store_true",
                    help="skip the pooling and CTC decoding measurements")
    ap.add_argument("--no-varlen", action="store_true", help="skip the full-utterance attention measurement")
    ap.add_argument("--ctc-utts", type=int, default=0,
                    help="pool and decode only the first N utterances (0: the whole batch)")
    ap.add_argument("--config", type=int, choices=[1, 2, 3, 4, 5], default=4,
                    help="the step's workload (default 4, the batch-128 one)")
    ap.add_argument("--seed", type=int, default=None, help="input seed (default: 1000 + config)")
    ap.add_argument("--no-configs", action="store_true", help="skip the per-config kernel timings")
    ap.add_argument("--no-qkv", action="store_true", help="skip the fused QKV projection + attention timing")
    ap.add_argument("--config-reps", type=int, default=50, help="launches per kernel and config (>= 50)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    global CFG, SEED
    CFG, SEED = args.config, args.seed
    if args.impl == "reference":
        rank = int(os.environ.get("RANK", "0"))
        world = int(os.environ.get("WORLD_SIZE", "1"))
        return run_reference(args, rank, world)
    rank, world, local = dist_setup(args.gpus)
    try:
        return run_nle(args, rank, world, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    sys.exit(main())
