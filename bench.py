"""Benchmark: one step = the whole hot path on one batch of synthetic input.

Workload: the spatial/temporal head-mask case on the HunyuanVideo 720p latent
grid (30 x 48 x 80 = 115,200 tokens, 24 heads, head_dim 128, bf16; 12 spatial
heads keeping their frame +-1, 12 temporal heads in the frame-major layout,
226 sink tokens). A step is sparse_attn_build_mask + sparse_attn_forward
(frame-major permutation + block-sparse attention), inputs resident in HBM.

Metric: attended TFLOP/s, counted at tile granularity as executed
(4 * d * kept key-block pairs * 128 * 128 per call), over the whole step; the
attention kernel's own rate against the measured bf16 tensor peak is in
``roofline``.

    python bench.py [--gpus N --steps K --warmup W] [--impl reference]
    torchrun --nproc-per-node N bench.py --gpus N ...   (independent replicas)
"""
import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "sparse attn ms/call & attended TFLOP/s (% BF16 TC peak) at 115k-token grid"
WORKLOAD = "spatiotemporal_hunyuan_720p"
ATTN_SRC = os.path.join(ROOT, "sparse_attention_video_b200", "csrc", "sa_attn.cu")
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "attn_fwd_traffic.txt")


def _args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--e2e-steps", type=int, default=6)
    ap.add_argument("--no-dense", action="store_true", help="skip the dense-mask comparison")
    ap.add_argument("--no-cpu", action="store_true", help="skip the CPU oracle baseline")
    ap.add_argument("--no-fp8", action="store_true", help="skip the FP8 attention timing")
    ap.add_argument("--no-mask-roofline", action="store_true",
                    help="skip the per-kernel timing of the memory-bound mask kernels")
    ap.add_argument("--no-profile", action="store_true",
                    help="skip the head-profiler timing (spatial/temporal workload only)")
    ap.add_argument("--workload", default=WORKLOAD,
                    help="workload name (synthetic.CONFIGS); the bench line uses the default")
    ap.add_argument("--mask-once", default="",
                    help="comma-separated workload names: build each one's mask twice through "
                         "the public API and exit (a short program for ncu launch lists of the "
                         "mask kernels); prints no bench line")
    ap.add_argument("--heads", type=int, default=0,
                    help="run only this many heads (half of them temporal); for small "
                         "profiler captures, not for bench lines")
    return ap.parse_args()


_T0 = time.perf_counter()


def log(msg):
    print(f"[bench {time.perf_counter() - _T0:7.1f}s] {msg}", file=sys.stderr, flush=True)


def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d["bf16_tflops"], d["bf16_tflops_sustained"], d["hbm_gbs"], "measured"
    return 1590.0, 1400.0, 6650.0, "fallback"


# ---------------------------------------------------------------- CPU oracle sample
def _threads():
    try:
        from threadpoolctl import threadpool_info
        return max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    except Exception:
        return os.cpu_count() or 1


def cpu_model():
    """The host CPU's model name (lscpu, else /proc/cpuinfo)."""
    try:
        out = subprocess.run(["lscpu"], capture_output=True, text=True, timeout=10).stdout
        for line in out.splitlines():
            if line.startswith("Model name:"):
                return line.split(":", 1)[1].strip()
    except Exception:
        pass
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                return line.split(":", 1)[1].strip()
    except Exception:
        pass
    return "unknown"


def cpu_oracle_sample(wl, x, budget_s=20.0, single_thread=False):
    """Time the oracle on a bounded sample of the workload: the full mask of
    one spatial and one temporal head (FG: of head 0), then masked attention
    for sampled query blocks (groups) of those heads. Returns a dict with the
    attended TFLOP/s over the whole sample, the per-query-block attention
    time and a labelled extrapolation to one full call."""
    from oracle import attention, pipeline
    from synthetic import bf16_bits_to_f32
    limit = None
    if single_thread:
        try:
            from threadpoolctl import threadpool_limits
            limit = threadpool_limits(limits=1)
        except Exception:
            limit = None
    try:
        threads = 1 if single_thread else _threads()
        rng = np.random.default_rng(0)
        flops = 0.0
        n_rows = 0
        mask_s = attn_s = 0.0
        t0 = time.perf_counter()
        if wl.kind == "fg":
            heads = [0]
            q, k, v = (bf16_bits_to_f32(x[n][0, 0]) for n in "qkv")
            keep = pipeline.head_mask(wl, q, k, 0)["keep_groups"]
            mask_s = time.perf_counter() - t0
            a0 = time.perf_counter()
            for g in rng.permutation(keep.shape[0]):
                attention.slice_attention(q, k, v, keep, wl.fg_group, [int(g)])
                flops += 4.0 * wl.head_dim * float(keep[g].sum()) * wl.fg_group
                n_rows += 1
                if time.perf_counter() - t0 > budget_s:
                    break
            attn_s = time.perf_counter() - a0
            unit_rows = wl.fg_group
            units_per_head = keep.shape[0]
            what = f"query groups of {wl.fg_group}"
        else:
            heads = [0, wl.temporal_heads[0]] if wl.temporal_heads else [0]
            units_per_head = 0
            for h in heads:
                q, k, v = (bf16_bits_to_f32(x[n][0, h]) for n in "qkv")
                m0 = time.perf_counter()
                ref = pipeline.head_mask(wl, q, k, h)
                mask_s += time.perf_counter() - m0
                blk, bm = ref["order_blocks"], ref["bmask"]
                units_per_head = max(units_per_head, blk.shape[0])
                a0 = time.perf_counter()
                for qb in rng.permutation(blk.shape[0]):
                    attention.block_sparse_attention(q, k, v, blk, bm, [int(qb)])
                    flops += 4.0 * wl.head_dim * float(bm[qb].sum()) * wl.block * wl.block
                    n_rows += 1
                    if time.perf_counter() - t0 > budget_s * (heads.index(h) + 1) / len(heads):
                        break
                attn_s += time.perf_counter() - a0
            unit_rows = wl.block
            what = f"query blocks of {wl.block} tokens"
        dt = time.perf_counter() - t0
    finally:
        if limit is not None:
            limit.restore_original_limits()
    per_unit = attn_s / max(n_rows, 1)
    full_s = mask_s / len(heads) * wl.heads + per_unit * units_per_head * wl.heads
    desc = (f"oracle on heads {heads}: full mask per head + masked attention (float64) for "
            f"{n_rows} sampled {what}")
    return {"value": flops / dt / 1e12, "desc": desc, "threads": threads,
            "mask_s_per_head": mask_s / len(heads),
            "attn_s_per_query_block": per_unit, "rows_per_query_block": unit_rows,
            "extrapolated_full_call_s": full_s}


# ---------------------------------------------------------------- clocks
class ClockSampler:
    """SM clock and clock-event reasons of one GPU, sampled during the timed
    region: NVML every 10 ms from a thread (enough samples even for a
    fraction of a second), else nvidia-smi every 200 ms."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    REASONS = (("hw_slowdown", 0x8), ("hw_thermal_slowdown", 0x40),
               ("sw_thermal_slowdown", 0x20), ("sw_power_cap", 0x4))

    def __init__(self, device):
        self.device = device
        self.proc = None
        self.thread = None
        self.samples = []
        self.reasons = set()
        self.max_mhz = None
        self.source = None
        self.path = tempfile.mktemp(suffix=".csv")

    def _nvml_handle(self):
        import pynvml
        import torch
        pynvml.nvmlInit()
        props = torch.cuda.get_device_properties(self.device)
        bus = getattr(props, "pci_bus_id", None)
        if bus is not None:
            busid = "%08x:%02x:%02x.0" % (getattr(props, "pci_domain_id", 0), bus,
                                          getattr(props, "pci_device_id", 0))
            try:
                return pynvml, pynvml.nvmlDeviceGetHandleByPciBusId(busid)
            except Exception:
                pass
        return pynvml, pynvml.nvmlDeviceGetHandleByIndex(self.device.index or 0)

    def start(self):
        import threading
        try:
            nv, h = self._nvml_handle()
            self.max_mhz = float(nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM))
            get_reasons = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons",
                                  getattr(nv, "nvmlDeviceGetCurrentClocksThrottleReasons", None))
            self._stop = threading.Event()

            def loop():
                while not self._stop.is_set():
                    try:
                        self.samples.append(float(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)))
                        bits = int(get_reasons(h))
                        for name, bit in self.REASONS:
                            if bits & bit:
                                self.reasons.add(name)
                    except Exception:
                        pass
                    self._stop.wait(0.01)

            self.thread = threading.Thread(target=loop, daemon=True)
            self.thread.start()
            self.source = "nvml, 10 ms"
            return
        except Exception:
            self.thread = None
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.device.index or 0), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=self.f, stderr=subprocess.DEVNULL)
            self.source = "nvidia-smi, 200 ms"
        except Exception:
            self.proc = None

    def stop(self):
        if self.thread is not None:
            self._stop.set()
            self.thread.join(timeout=5)
            if not self.samples:
                return None
            return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                    "reasons": sorted(self.reasons), "samples": len(self.samples),
                    "source": self.source}
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.f.close()
        sm, mx, reasons = [], None, set()
        names = [n for n, _ in self.REASONS]
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for n, val in zip(names, parts[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(n)
        os.unlink(self.path)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm), "source": self.source}


def kernel_times(fn, device):
    """Device time of every kernel ``fn`` launches, from one run under the
    CUDA activity profiler (CUPTI timestamps, not ncu): {name: (launches,
    total ms)}. Returns {} if the profiler is unavailable."""
    import torch
    try:
        from torch.profiler import ProfilerActivity, profile
        torch.cuda.synchronize(device)
        with profile(activities=[ProfilerActivity.CUDA]) as prof:
            fn()
            torch.cuda.synchronize(device)
        out = {}
        for e in prof.events():
            dt = getattr(e, "device_time", None)
            if dt is None:
                dt = getattr(e, "cuda_time", 0.0)
            if getattr(e, "device_type", None) is not None and "CUDA" not in str(e.device_type):
                continue
            if not dt:
                continue
            n, t = out.get(e.name, (0, 0.0))
            out[e.name] = (n + 1, t + dt / 1e3)
        return out
    except Exception as exc:                          # profiler missing or CUPTI refused
        log(f"kernel timing unavailable: {exc}")
        return {}


def _kernel_ms(times, fragment):
    """(launches, ms) of the kernels whose name contains ``fragment``."""
    n, t = 0, 0.0
    for name, (k, ms) in times.items():
        if fragment in name:
            n += k
            t += ms
    return n, t


def attn_kernel_name(wl):
    """The attention kernel a workload's attend() launches: policies that bound
    a row's kept blocks run the one-warpgroup kernel (two CTAs per SM)."""
    if wl.kind == "fg":
        return "attn_fwd_kernel<%d,%d,gather>" % (wl.head_dim, wl.block)
    if wl.kind in ("topk", "sta", "spatiotemporal"):
        return "attn_solo_kernel<%d,%d>" % (wl.head_dim, wl.block)
    return "attn_fwd_kernel<%d,%d,block>" % (wl.head_dim, wl.block)


def _traffic_per_launch(kernel):
    """DRAM bytes per attention launch from the committed ncu summary, if it was
    taken on the current attention source and of this kernel; else None."""
    if not os.path.exists(TRAFFIC_FILE):
        return None
    kv = {}
    for line in open(TRAFFIC_FILE):
        if "=" in line and not line.startswith("#"):
            a, b = line.split("=", 1)
            kv[a.strip()] = b.strip()
    src_hash = hashlib.sha256(open(ATTN_SRC, "rb").read()).hexdigest()[:16]
    if kv.get("source_sha256_16") != src_hash or kv.get("kernel") != kernel:
        return None
    try:
        return float(kv["dram_bytes_per_launch"])
    except (KeyError, ValueError):
        return None


def policy_kwargs(wl):
    """The workload's mask policy as make_policy() arguments."""
    if wl.kind == "topk":
        return dict(kind="topk", block=wl.block, tile=wl.tile, topk=wl.topk,
                    keep_diagonal=wl.keep_diagonal, summarizer=wl.summarizer)
    if wl.kind == "sta":
        return dict(kind="sta", block=wl.block, tile=wl.tile, window=wl.window,
                    head_windows=wl.head_windows or None)
    if wl.kind == "spatiotemporal":
        return dict(kind="spatiotemporal", block=wl.block, temporal_heads=wl.temporal_heads,
                    heads=wl.heads, sink_tokens=wl.sink_tokens, frame_radius=1)
    if wl.kind == "spade":
        return dict(kind="spade", block=wl.block, candidates=wl.candidates, top_p=wl.top_p,
                    window=wl.window, summarizer=wl.summarizer)
    return dict(kind="fg", block=wl.block, fg_group=wl.fg_group,
                fg_keep_fraction=wl.fg_keep_fraction)


# kernels of ours launched by one step (build_mask + permute + attend)
# (the bench line counts them from one step under the CUDA activity profiler;
# this table is the fallback when the profiler is unavailable)
LAUNCHES_PER_STEP = {"topk": 5, "sta": 3, "spatiotemporal": 4, "spade": 5, "fg": 25}


def launches_in(times):
    """Kernel launches in a kernel_times() result (copies and memsets excluded)."""
    return sum(n for name, (n, _) in times.items() if "kernel" in name)


def _block_valid(info, T, H, W, block):
    """Valid tokens of each block of a head's working layout (int64 [nb])."""
    nb = info.nb
    if info.layout == 2:                      # 3D tile layout, raster tiles
        b = np.arange(nb)
        tw, th, tt = b % info.nw, (b // info.nw) % info.nh, b // (info.nw * info.nh)
        vt = np.minimum(info.bt, T - tt * info.bt)
        vh = np.minimum(info.bh, H - th * info.bh)
        vw = np.minimum(info.bw, W - tw * info.bw)
        return (vt * vh * vw).astype(np.int64)
    n = T * H * W
    return np.minimum(block, n - block * np.arange(nb)).astype(np.int64)


def useful_flops(wl, sa):
    """4 * d * (valid query, valid key) pairs of the kept blocks: the work
    without the pad slots that the tile-granularity count includes."""
    from sparse_attention_video_b200 import SA_EXPORT_BLOCK_BITS
    infos = sa.export(2)
    words = sa.export(SA_EXPORT_BLOCK_BITS)
    # rows are sized for the largest block count of the policy's layouts,
    # which may exceed every head's own (SPADE: the candidates not chosen)
    nbmax = max(i.nb for i in infos)
    while len(infos) * nbmax * ((nbmax + 31) // 32) < words.size:
        nbmax += 1
    w32 = (nbmax + 31) // 32
    words = words.reshape(len(infos), nbmax, w32)
    pairs = 0
    for h, info in enumerate(infos):
        valid = _block_valid(info, wl.T, wl.H, wl.W, wl.block)
        bits = np.unpackbits(words[h, :info.nb].view(np.uint8), axis=1,
                             bitorder="little")[:, :info.nb].astype(np.int64)
        pairs += int(valid @ bits @ valid)
    return 4.0 * wl.head_dim * pairs


def fg_method_flops(wl, sa):
    """4 * d * M * kept (group, key) slices: the FG method's own work (each
    kept slice is one key against the M queries of its group)."""
    from sparse_attention_video_b200 import SA_EXPORT_FG_BITS
    bits = sa.export(SA_EXPORT_FG_BITS)
    kept = int(np.bitwise_count(bits).sum(dtype=np.int64))
    return 4.0 * wl.head_dim * wl.fg_group * kept, kept


# Algorithmic bytes per launch of the memory-bound mask kernels (read + write
# of what the step must touch once), per workload: name fragment -> bytes.
def mask_kernel_bytes(wl, n_frame_major_heads=0):
    tok = wl.N * wl.head_dim * 2                      # one head's tensor, bf16
    out = {}
    if n_frame_major_heads:
        out["permute_fm"] = 3 * 2 * tok * n_frame_major_heads
    if wl.kind in ("spade", "topk"):
        out["pool_atoms"] = 2 * tok * wl.heads        # Q and K read once
    if wl.kind == "fg":
        out["fg_qbar"] = tok * wl.heads               # Q read once
    return out


def mask_kernel_bytes_entry(wl, times, hbm, extra=None):
    fm = len(wl.temporal_heads) if wl.kind == "spatiotemporal" else 0
    nbytes = mask_kernel_bytes(wl, fm)
    nbytes.update(extra or {})
    return mask_roofline_entry(wl, times, nbytes, hbm)


def fg_mask_extras(wl, sa):
    """FG mask kernels beyond fg_qbar: fg_pair_count's bytes (the slice
    bitmask read once, one count per 128-query tile written), fg_compact's
    (the bitmask read once, the union lists written once: 4 bytes per entry)
    and fg_score's FLOPs (three bf16 terms of each (group, key) score per
    pass)."""
    from sparse_attention_video_b200 import SA_EXPORT_FG_TILE_KEYS
    G = (wl.N + wl.fg_group - 1) // wl.fg_group
    words = (wl.N + 31) // 32
    tiles = (wl.N + 127) // 128
    entries = float(sa.export(SA_EXPORT_FG_TILE_KEYS).astype(np.float64).sum())
    bitmask = 4 * G * words * wl.heads
    score_pass = 3 * 2.0 * G * wl.N * wl.head_dim * wl.heads
    return {"fg_pair_count": bitmask + 4 * tiles * wl.heads,
            "fg_compact": bitmask + 4 * entries}, score_pass


def fg_score_entry(wl, times, flops_per_pass, peak_tflops, passes=2.0625):
    n, ms = _kernel_ms(times, "fg_score")
    if n == 0:
        return {}
    tf = passes * flops_per_pass / (ms * 1e-3) / 1e12
    return {"fg_score": {"workload": wl.name, "ms_all_passes": ms, "launches": n,
                         "bound": "tensor", "tflop_per_pass": flops_per_pass / 1e12,
                         "passes": passes,
                         "achieved_tflops": tf, "peak_tflops": peak_tflops,
                         "frac": tf / peak_tflops,
                         "note": "level 0 on a sixteenth of the key tiles, the windowed exact "
                                 "histogram, the bitmask; launches for heads outside the window "
                                 "or with an overflowing list return at once"}}


def mask_roofline_entry(wl, times, nbytes, hbm):
    res = {}
    for frag, b in nbytes.items():
        n, ms = _kernel_ms(times, frag)
        if n == 0:
            continue
        per = ms / n
        gbs = b / (per * 1e-3) / 1e9
        res[frag] = {"workload": wl.name, "ms": per, "algorithmic_bytes": b,
                     "achieved_gbs": gbs, "peak_gbs": hbm, "frac": gbs / hbm}
    return res


# ---------------------------------------------------------------- multi-rank helpers
def rank_workload(wl, rank):
    """Rank r runs its own problem of the same shape (weak scaling, no data
    exchange): the seeds differ by rank."""
    return wl.with_(config_id=wl.config_id + 1000 * rank)


def max_over_ranks(values, dist=None, device="cpu"):
    """Element-wise maximum of a list of floats over all ranks (the step time of
    a multi-GPU run is its slowest rank)."""
    if dist is None or not dist.is_initialized() or dist.get_world_size() == 1:
        return list(values)
    import torch
    t = torch.tensor(list(values), dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def aggregate_tflops(world, flops_per_rank_step, ms_per_step):
    """Whole-job throughput: every rank's work over the slowest rank's time."""
    return world * flops_per_rank_step / (ms_per_step * 1e-3) / 1e12


# ---------------------------------------------------------------- reference arm
def run_reference(args, rank, world):
    if rank != 0:
        return
    from synthetic import CONFIGS, make_qkv
    wl = CONFIGS[WORKLOAD]
    x = make_qkv(wl, heads=[0, wl.temporal_heads[0]])
    xx = {n: np.zeros((1, wl.heads) + x[n].shape[2:], np.uint16) for n in "qkv"}
    for n in "qkv":
        xx[n][0, 0] = x[n][0, 0]
        xx[n][0, wl.temporal_heads[0]] = x[n][0, 1]
    vals = []
    for i in range(args.warmup + args.steps):
        c = cpu_oracle_sample(wl, xx, budget_s=max(2.0, 60.0 / (args.steps + args.warmup)))
        desc, threads = c["desc"], c["threads"]
        if i >= args.warmup:
            vals.append(c["value"])
    value = statistics.mean(vals)
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic",
            "config": {"workload": WORKLOAD, "grid": "30x48x80", "tokens": wl.N,
                       "heads": wl.heads, "head_dim": wl.head_dim, "batch": 1},
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": threads,
                             "kind": "oracle", "sample": desc, "cpu_model": cpu_model()},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------- mask kernels only
def mask_once(names, local, heads=0):
    """Each named workload's mask built twice (the second build runs with its
    kernels warm) on the seeded inputs, through SparseAttention.build_mask;
    ``heads`` > 0 keeps only that many heads (a smaller case for profiling)."""
    import torch

    from sparse_attention_video_b200 import SparseAttention, make_policy
    from synthetic import CONFIGS, make_qkv

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    for name in names:
        wl = CONFIGS[name]
        if heads:
            th = tuple(h for h in wl.temporal_heads if h < heads)
            wl = wl.with_(heads=heads, temporal_heads=th)
        x = make_qkv(wl)
        q, k = (torch.from_numpy(x[n].view(np.int16)).view(torch.bfloat16).to(dev) for n in "qk")
        sa = SparseAttention(1, wl.heads, wl.T, wl.H, wl.W, wl.head_dim,
                             make_policy(**policy_kwargs(wl)), device=dev)
        stream = torch.cuda.current_stream(dev)
        for _ in range(2):
            sa.build_mask(q, k, stream)
        torch.cuda.synchronize(dev)
        status = sa.status()
        log(f"{name}: mask built twice, status {status}")
        if status != 0:
            raise SystemExit(f"{name}: device status {status}")
        del q, k, sa


# ---------------------------------------------------------------- our arm
def main():
    args = _args()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    if args.mask_once:
        mask_once(args.mask_once.split(","), local, args.heads)
        return

    import torch
    import torch.distributed as dist
    from datetime import timedelta

    from sparse_attention_video_b200 import SparseAttention, make_policy
    from synthetic import CONFIGS, make_qkv

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", timeout=timedelta(seconds=600),
                                device_id=dev)

    wl = CONFIGS[args.workload]
    if args.heads:
        th = tuple(range(args.heads // 2, args.heads)) if wl.temporal_heads else ()
        wl = wl.with_(heads=args.heads, temporal_heads=th)
    wl_r = rank_workload(wl, rank)
    log("generating inputs")
    x = make_qkv(wl_r)
    log("inputs ready")
    host = {n: torch.from_numpy(x[n].view(np.int16)).view(torch.bfloat16).pin_memory() for n in "qkv"}
    q, k, v = (host[n].to(dev) for n in "qkv")
    pol = make_policy(**policy_kwargs(wl))
    sa = SparseAttention(1, wl.heads, wl.T, wl.H, wl.W, wl.head_dim, pol, device=dev)
    o = torch.empty_like(q)
    lse = torch.empty(q.shape[:3], dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step(ev=None):
        if ev:
            ev[0].record(stream)
        sa.build_mask(q, k, stream)
        if ev:
            ev[1].record(stream)
        sa.permute(q, k, v, stream)
        if ev:
            ev[2].record(stream)
        sa.attend(q, k, v, o, lse, stream)
        if ev:
            ev[3].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    log("warm-up done")
    per_step = launches_in(kernel_times(step, dev)) or LAUNCHES_PER_STEP[wl.kind]
    assert sa.status() == 0, "device status word set during warm-up"
    method = {}
    if wl.kind == "fg":
        # executed work: every 128-query tile against the union of its groups' kept keys
        from sparse_attention_video_b200 import SA_EXPORT_FG_TILE_KEYS
        keys = float(sa.export(SA_EXPORT_FG_TILE_KEYS).astype(np.float64).sum())
        flops_call = 4.0 * wl.head_dim * keys * 128
        mflops, kept_slices = fg_method_flops(wl, sa)
        method = {"method_tflop_per_call": mflops / 1e12, "kept_slices": kept_slices,
                  "method_note": "4 * d * M * kept slices; the roofline counts the executed "
                                 "union work of each 128-query tile"}
        useful = mflops
    else:
        kept = sum(h.kept for h in sa.export(2))
        flops_call = 4.0 * wl.head_dim * kept * wl.block * wl.block
        useful = useful_flops(wl, sa)

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(dev)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    clocks.start()
    t_start.record(stream)
    for i in range(args.steps):
        step(evs[i])
    t_end.record(stream)
    torch.cuda.synchronize(dev)
    clk = clocks.stop()
    if world > 1:
        dist.barrier()
    log("timed steps done")
    ms_total = t_start.elapsed_time(t_end)
    mask_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in evs)
    perm_ms = statistics.mean(e[1].elapsed_time(e[2]) for e in evs)
    attn_ms = statistics.mean(e[2].elapsed_time(e[3]) for e in evs)
    ms_total, attn_ms, mask_ms, perm_ms = max_over_ranks([ms_total, attn_ms, mask_ms, perm_ms],
                                                          dist, dev)
    assert sa.status() == 0, "device status word set during the timed steps"
    ms_step = ms_total / args.steps
    value = aggregate_tflops(world, flops_call, ms_step)

    # ---- memory-bound mask kernels: device time of each kernel of one
    # build_mask (+ permute) from CUPTI, against its algorithmic bytes
    mask_roof = {}
    if not args.no_mask_roofline:
        times = kernel_times(lambda: (sa.build_mask(q, k, stream), sa.permute(q, k, v, stream)), dev)
        hbm_peak = _peaks()[2]
        extra, score_pass = fg_mask_extras(wl, sa) if wl.kind == "fg" else ({}, 0.0)
        mask_roof.update(mask_kernel_bytes_entry(wl, times, hbm_peak, extra))
        if wl.kind == "fg":
            mask_roof.update(fg_score_entry(wl, times, score_pass, _peaks()[0]))
        if wl.name == WORKLOAD and not args.heads:
            for other in ("spade_wan21_14b_720p", "fg_slices_hunyuan_720p"):
                owl = rank_workload(CONFIGS[other], rank)
                ox = make_qkv(owl)
                oq, ok_ = (torch.from_numpy(ox[n].view(np.int16)).view(torch.bfloat16).to(dev)
                           for n in "qk")
                del ox
                osa = SparseAttention(1, owl.heads, owl.T, owl.H, owl.W, owl.head_dim,
                                      make_policy(**policy_kwargs(owl)), device=dev)
                osa.build_mask(oq, ok_, stream)
                otimes = kernel_times(lambda: osa.build_mask(oq, ok_, stream), dev)
                assert osa.status() == 0, f"device status word set in the {other} mask build"
                extra, score_pass = fg_mask_extras(owl, osa) if owl.kind == "fg" else ({}, 0.0)
                mask_roof.update(mask_kernel_bytes_entry(owl, otimes, hbm_peak, extra))
                if owl.kind == "fg":
                    mask_roof.update(fg_score_entry(owl, otimes, score_pass, _peaks()[0]))
                del oq, ok_, osa
                torch.cuda.empty_cache()
        log("mask kernel rooflines done")

    # ---- end to end through the public API with host buffers: each step is
    # one sparse_attn_forward_host call (Q, K, V copied in, mask, forward, O
    # and LSE copied out); steps alternate between two streams, each with its
    # own workspaces and device buffers, so one step's copies overlap the
    # other's kernels and the other direction's copies
    sa2 = SparseAttention(1, wl.heads, wl.T, wl.H, wl.W, wl.head_dim,
                          make_policy(**policy_kwargs(wl)), device=dev)
    lanes = [(sa, stream), (sa2, torch.cuda.Stream(dev))]
    outs = [(torch.empty(o.shape, dtype=torch.bfloat16).pin_memory(),
             torch.empty(lse.shape, dtype=torch.float32).pin_memory()) for _ in lanes]
    for (obj, st_), (oh, lh) in zip(lanes, outs):        # staging buffers allocated here
        obj.forward_host(host["q"], host["k"], host["v"], oh, lh, st_)
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    lanes[1][1].wait_event(e0)
    for i in range(args.e2e_steps):
        (obj, st_), (oh, lh) = lanes[i % 2], outs[i % 2]
        obj.forward_host(host["q"], host["k"], host["v"], oh, lh, st_)
    done2 = torch.cuda.Event()
    done2.record(lanes[1][1])
    stream.wait_event(done2)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    assert sa2.status() == 0, "device status word set in the end-to-end steps"
    log("end-to-end steps done")
    e2e_ms = e0.elapsed_time(e1) / args.e2e_steps
    o_host, lse_host = outs[0]
    e2e_ms = max_over_ranks([e2e_ms], dist, dev)[0]
    h2d = sum(host[n].numel() * 2 for n in "qkv")
    d2h = o_host.numel() * 2 + lse_host.numel() * 4

    # ---- the same kernel with every block kept
    dense = {}
    if not args.no_dense and wl.head_dim == 128 and wl.block == 128:
        nb = (wl.N + wl.block - 1) // wl.block
        w32 = (nb + 31) // 32
        words = torch.full((wl.heads, nb, w32), -1, dtype=torch.int32, device=dev)
        dpol = make_policy("explicit", block=wl.block, explicit_layout=0, explicit_bits=words)
        dsa = SparseAttention(1, wl.heads, wl.T, wl.H, wl.W, wl.head_dim, dpol, device=dev)
        dsa.build_mask(q, k, stream)
        dsa.attend(q, k, v, o, lse, stream)
        d0, d1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize(dev)
        d0.record(stream)
        for _ in range(2):
            dsa.attend(q, k, v, o, lse, stream)
        d1.record(stream)
        torch.cuda.synchronize(dev)
        log("dense-mask run done")
        dense_ms = d0.elapsed_time(d1) / 2
        dense_flops = 4.0 * wl.head_dim * wl.heads * nb * nb * wl.block * wl.block
        dense = {"dense_mask_attn_ms": dense_ms,
                 "dense_mask_attn_tflops": dense_flops / (dense_ms * 1e-3) / 1e12,
                 "speedup_vs_dense_mask": dense_ms / attn_ms}
        del dsa, words

    # ---- FP8 attention (Sparse VideoGen review: optional FP8 quantization):
    # the same mask and kernel structure on E4M3 operands, kind::f8f6f4
    fp8 = {}
    if not args.no_fp8 and wl.head_dim == 128 and wl.block == 128 and wl.kind != "fg":
        from sparse_attention_video_b200 import quantize_e4m3
        o8 = torch.empty_like(q)
        l8 = torch.empty_like(lse)
        _, _, quantized = sa.forward_fp8(q, k, v, o8, l8, stream)
        (q8, qi), (k8, ki), (v8, vi) = quantized
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
        reps = 5
        torch.cuda.synchronize(dev)
        ev[0].record(stream)
        for _ in range(reps):
            for t in (q, k, v):
                quantize_e4m3(t, stream)
        ev[1].record(stream)
        for _ in range(reps):
            sa.permute_fp8(q8, k8, v8, stream)
        ev[2].record(stream)
        for _ in range(reps):
            sa.attend_fp8(q8, k8, v8, qi, ki, vi, o8, l8, stream)
        ev[3].record(stream)
        torch.cuda.synchronize(dev)
        assert sa.status() == 0, "device status word set in the FP8 attention"
        qz_ms, pm_ms, at_ms = (ev[i].elapsed_time(ev[i + 1]) / reps for i in range(3))
        at_ms = max_over_ranks([at_ms], dist, dev)[0]
        pb = _peaks()[0]
        fp8 = {"fp8_attention": {
            "kernel": attn_kernel_name(wl).replace(">", ",fp8>") + " (tcgen05.mma kind::f8f6f4)",
            "attend_ms": at_ms, "quantize_ms": qz_ms, "permute_ms": pm_ms,
            "tflops": flops_call / (at_ms * 1e-3) / 1e12,
            "peak": 2.0 * pb, "frac": flops_call / (at_ms * 1e-3) / 1e12 / (2.0 * pb),
            "peak_note": "2 x the measured bf16 burst peak (the nominal fp8 : bf16 ratio), "
                         "not a measured fp8 figure",
            "speedup_vs_bf16_attention": attn_ms / at_ms}}
        del o8, l8, quantized, q8, k8, v8, qi, ki, vi
        log("fp8 attention timed")

    # ---- the head profiler (Sparse VideoGen review, key machinery) on 1 % of
    # each head's query rows; reported beside the step, not part of it
    prof = {}
    if not args.no_profile and wl.kind == "spatiotemporal":
        from sparse_attention_video_b200 import profile_heads
        from synthetic import sample_rows
        rows = torch.from_numpy(sample_rows(wl.N, wl.heads, 0.01, seed=2024)).to(dev)
        for _ in range(2):
            profile_heads(q, k, v, rows, wl.T, wl.H, wl.W, block=wl.block,
                          sink_tokens=wl.sink_tokens, stream=stream)
        p0, p1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize(dev)
        p0.record(stream)
        for _ in range(5):
            is_t, _, _ = profile_heads(q, k, v, rows, wl.T, wl.H, wl.W, block=wl.block,
                                       sink_tokens=wl.sink_tokens, stream=stream)
        p1.record(stream)
        torch.cuda.synchronize(dev)
        prof_ms = p0.elapsed_time(p1) / 5
        # the full pass alone: every sampled row against every key, on the
        # attention kernel (its device time from the activity profiler)
        full_flops = 4.0 * wl.head_dim * rows.numel() * wl.N
        kt = kernel_times(lambda: profile_heads(q, k, v, rows, wl.T, wl.H, wl.W, block=wl.block,
                                                sink_tokens=wl.sink_tokens, stream=stream), dev)
        n_a, attn_full_ms = _kernel_ms(kt, "attn_fwd")
        n_p, masked_ms = _kernel_ms(kt, "profile_kernel")
        prof = {"profile_heads": {
            "ms": prof_ms, "rows_per_head": int(rows.shape[1]),
            "full_pass_tflops_over_call": full_flops / (prof_ms * 1e-3) / 1e12,
            "full_pass_kernel_ms": attn_full_ms if n_a else None,
            "full_pass_kernel_tflops": (full_flops / (attn_full_ms * 1e-3) / 1e12) if n_a else None,
            "full_pass_kernel_frac": (full_flops / (attn_full_ms * 1e-3) / 1e12 / _peaks()[0])
                                     if n_a else None,
            "masked_passes_ms": masked_ms if n_p else None,
            "temporal_heads_found": int(is_t.sum().item()),
            "kernel": "full pass: attn_fwd_kernel (tcgen05, dense key list over gathered rows); "
                      "masked passes: profile_kernel (mma.sync m16n8k16)"}}
        log("head profiler timed")
    if not args.no_profile and wl.kind == "sta":
        # the STA per-head window search (Sliding Tile Attention review, key
        # machinery) on 1 % of each head's rows, four candidate windows
        from sparse_attention_video_b200 import sta_window_search
        from synthetic import sample_rows
        rows = torch.from_numpy(sample_rows(wl.N, wl.heads, 0.01, seed=2024)).to(dev)
        cands = [(3, 3, 3), (1, 3, 5), (5, 3, 1), (3, 5, 3)]
        for _ in range(2):
            sta_window_search(q, k, v, rows, wl.T, wl.H, wl.W, wl.tile, cands, block=wl.block,
                              stream=stream)
        p0, p1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize(dev)
        p0.record(stream)
        for _ in range(5):
            choice, _, _ = sta_window_search(q, k, v, rows, wl.T, wl.H, wl.W, wl.tile, cands,
                                             block=wl.block, stream=stream)
        p1.record(stream)
        torch.cuda.synchronize(dev)
        ms = p0.elapsed_time(p1) / 5
        full_flops = 4.0 * wl.head_dim * rows.numel() * wl.N
        kt = kernel_times(lambda: sta_window_search(q, k, v, rows, wl.T, wl.H, wl.W, wl.tile, cands,
                                                    block=wl.block, stream=stream), dev)
        n_a, attn_full_ms = _kernel_ms(kt, "attn_fwd")
        n_p, masked_ms = _kernel_ms(kt, "profile_kernel")
        prof = {"window_search": {
            "ms": ms, "rows_per_head": int(rows.shape[1]), "candidates": cands,
            "full_pass_tflops_over_call": full_flops / (ms * 1e-3) / 1e12,
            "full_pass_kernel_ms": attn_full_ms if n_a else None,
            "full_pass_kernel_tflops": (full_flops / (attn_full_ms * 1e-3) / 1e12) if n_a else None,
            "masked_passes_ms": masked_ms if n_p else None,
            "choices": torch.bincount(choice.long().cpu(), minlength=len(cands)).tolist(),
            "kernel": "full pass: attn_fwd_kernel (tcgen05); window passes: profile_kernel, "
                      "tile-window mode (mma.sync m16n8k16)"}}
        log("window search timed")

    if wl.kind == "fg" and not args.no_profile and dense:
        # FG cached mask from the LSE of full attention (an explicit policy
        # keeping every block); the union lists are sized for every slice
        nb = (wl.N + wl.block - 1) // wl.block
        words = torch.full((wl.heads, nb, (nb + 31) // 32), -1, dtype=torch.int32, device=dev)
        fpol = make_policy("explicit", block=wl.block, explicit_layout=0, explicit_bits=words)
        fsa = SparseAttention(1, wl.heads, wl.T, wl.H, wl.W, wl.head_dim, fpol, device=dev)
        fsa.build_mask(q, k, stream)
        fsa.attend(q, k, v, o, lse, stream)
        del fsa, words
        cpol = make_policy("fg", block=wl.block, fg_group=wl.fg_group, fg_keep_fraction=1.0)
        csa = SparseAttention(1, wl.heads, wl.T, wl.H, wl.W, wl.head_dim, cpol, device=dev)
        csa.build_mask_fg_cached(q, k, lse, stream=stream)
        c0, c1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize(dev)
        c0.record(stream)
        for _ in range(2):
            csa.build_mask_fg_cached(q, k, lse, stream=stream)
        c1.record(stream)
        torch.cuda.synchronize(dev)
        ms = c0.elapsed_time(c1) / 2
        from sparse_attention_video_b200 import SA_EXPORT_FG_BITS
        bits = csa.export(SA_EXPORT_FG_BITS)
        kept = int(np.bitwise_count(bits).sum(dtype=np.int64))
        G = (wl.N + wl.fg_group - 1) // wl.fg_group
        prof["fg_cached"] = {
            "ms": ms, "status": csa.status(),
            "score_tflops": 2.0 * wl.head_dim * wl.N * wl.N * wl.heads / (ms * 1e-3) / 1e12,
            "kept_fraction": kept / (G * wl.N * wl.heads),
            "kernel": "fg_score_kernel, cached mode (tcgen05), then the union lists"}
        del csa
        log("cached mask timed")

    if not args.no_profile:
        from sparse_attention_video_b200 import quantize_e4m3
        quantize_e4m3(q, stream)
        z0, z1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize(dev)
        z0.record(stream)
        for _ in range(5):
            quantize_e4m3(q, stream)
        z1.record(stream)
        torch.cuda.synchronize(dev)
        ms = z0.elapsed_time(z1) / 5
        algo = q.numel() * 3                      # 2 bytes read and 1 byte written per element
        prof["quantize_e4m3"] = {
            "ms": ms, "algorithmic_gbs": algo / (ms * 1e-3) / 1e9,
            "frac_of_hbm": algo / (ms * 1e-3) / 1e9 / _peaks()[2],
            "note": "Q of every head; each element is read twice (amax, then encode)"}
        log("quantizer timed")

    if rank != 0:
        if world > 1:
            dist.barrier()
            dist.destroy_process_group()
        return

    peak_burst, peak_sust, hbm, peak_src = _peaks()
    achieved = flops_call / (attn_ms * 1e-3) / 1e12
    traffic = _traffic_per_launch(attn_kernel_name(wl))
    cpu = None
    if not args.no_cpu:
        c = cpu_oracle_sample(wl_r, x)
        c1 = cpu_oracle_sample(wl_r, x, budget_s=6.0, single_thread=True)
        log("cpu oracle samples done")
        cpu = {"value": c["value"], "unit": "TFLOP/s", "cores": c["threads"], "kind": "oracle",
               "sample": c["desc"], "cpu_model": cpu_model(),
               "single_thread": {"value": c1["value"], "unit": "TFLOP/s", "cores": 1,
                                 "sample": c1["desc"]},
               "mask_s_per_head": c["mask_s_per_head"],
               "attn_s_per_query_block": c["attn_s_per_query_block"],
               "rows_per_query_block": c["rows_per_query_block"],
               "extrapolated_full_call_s": c["extrapolated_full_call_s"],
               "extrapolation_note": ("extrapolated, not measured: the mean mask time per "
                                      "sampled head x heads + the mean attention time per "
                                      "sampled query block x query blocks x heads")}
    sm_mhz = clk["sm_mhz"] if clk else None
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": wl.name, "grid": f"{wl.T}x{wl.H}x{wl.W}", "tokens": wl.N,
                   "heads": wl.heads, "head_dim": wl.head_dim, "batch": 1, "block": wl.block,
                   "parallelism": f"replicas x{world}",
                   "l2": (f"inputs larger than L2 (Q, K, V = {h2d / 1e9:.2f} GB per step)"
                          if h2d > 126e6 else "inputs smaller than L2: not flushed")},
        "step_breakdown_ms": {"build_mask": mask_ms, "permute": perm_ms, "attention": attn_ms},
        "attended_tflop_per_call": flops_call / 1e12,
        "attention_ms_per_call": attn_ms,
        "useful_tflop_per_call": useful / 1e12,
        "useful_tflops_attention": useful / (attn_ms * 1e-3) / 1e12,
        **method,
        "roofline": {"kernel": attn_kernel_name(wl),
                     "bound": "tensor",
                     "achieved": achieved, "peak": peak_burst, "unit": "TFLOP/s",
                     "frac": achieved / peak_burst,
                     "peak_note": (f"{peak_src} burst cuBLAS bf16 (the kernel is timed per call "
                                   f"inside short steps); the sustained figure is a second number"),
                     "peak_sustained": peak_sust, "frac_of_sustained": achieved / peak_sust,
                     "attn_kcycles_per_call": (attn_ms * sm_mhz) if sm_mhz else None,
                     "traffic": traffic if wl.name == WORKLOAD and not args.heads else None},
        "mask_roofline": mask_roof,
        **({"method_tflops_attention": method["method_tflop_per_call"] * 1e12 / (attn_ms * 1e-3) / 1e12,
            "method_frac": method["method_tflop_per_call"] * 1e12 / (attn_ms * 1e-3) / 1e12 / peak_burst}
           if method else {}),
        "cpu_baseline": cpu,
        "e2e": {"value": aggregate_tflops(world, flops_call, e2e_ms), "unit": "TFLOP/s",
                "ms_per_step": e2e_ms, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "call": "sparse_attn_forward_host, steps alternating between two streams"},
        "gpu_launches": per_step * args.steps,
        "clocks": clk,
        **dense,
        **fp8,
        **prof,
    }
    print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
