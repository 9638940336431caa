"""Benchmark of the BSA forward pass (pool -> compress/select -> fine attention).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload nside128] [--impl ours|reference]

One step = one pass of the whole hot path over one batch of the workload's
synthetic inputs, resident in HBM. Prints ONE JSON line on rank 0.

tokens/s counts batch x N tokens per step (a token's heads are not counted
separately); `head_rows_per_s` gives batch x heads x N per second beside it.

Multi-GPU (torchrun, one rank per GPU): the (batch, head) slabs of BSA are
independent problems, so every rank runs its own full batch with no
collective on the data path ("scaling": "weak"); the step time is the max
over ranks of the device-timed region and `value` counts all ranks' tokens.

--impl reference times the fp64 CPU oracle on the host cores (rank 0 only),
each step a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from block_sparse_spherical_b200.configs import CONFIGS, HEADLINE  # noqa: E402

METRIC = "BSA fwd tokens/s & TFLOP/s at Nside=128 (1 B200); % of BF16 tensor/HBM peak"
UNIT = "tokens/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                  "sm_max_mhz": 1965.0}
NOMINAL_HBM_GBS = 8000.0       # nominal HBM3e bandwidth of a B200 (DGX figure)
SM_COUNT_B200 = 148
TF32_PER_BF16 = 1.1 / 2.25     # nominal dense tf32 : bf16 tensor rate (B200)


def measured_m64_rate() -> float:
    """Multiply-adds per clock per SM of back-to-back M=64 bf16 tcgen05.mma from four issuing warps
    (the library's microbenchmark hook; best over N = 64, 128, 256 and three repeats)."""
    import torch
    from block_sparse_spherical_b200 import abi
    best = 0.0
    cyc = torch.zeros(4, dtype=torch.int64, device="cuda")
    for _ in range(3):
        for n in (64, 128, 256):
            abi.bsa_testing_mma_rate(64, n, 4, cyc)
            c = max(cyc.cpu().tolist())
            if c > 0:
                best = max(best, 64 * n * 16 * 256 * 4 / c)
    if best <= 0:
        raise RuntimeError("the tcgen05.mma rate microbenchmark did not complete")
    return best


def compress_on_tensor_cores(cfg) -> bool:
    """The library runs the compressed branch on the tensor cores (three-pass tf32) for these shapes."""
    return cfg.head_dim == 64 and cfg.top_n in (16, 32)


def kernels_per_step(cfg) -> int:
    """Kernels one step launches: pool, compressed branch (+ the tf32 split of its operands into the
    workspace on the tensor-core path), fine attention."""
    return 4 if compress_on_tensor_cores(cfg) else 3


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def workload_config(cfg):
    return {"workload": cfg.name, "nside": cfg.nside, "n_tokens": cfg.n_tokens, "batch": cfg.batch,
            "heads": cfg.heads, "head_dim": cfg.head_dim, "block_size": cfg.block_size,
            "n_blocks": cfg.n_blocks, "top_n": cfg.top_n, "window_blocks": cfg.window_blocks,
            "seed": cfg.seed,
            "l2": l2_note(cfg)}


def l2_note(cfg):
    mb = cfg.slabs * cfg.n_tokens * cfg.head_dim * cfg.elt_bytes / 1e6
    if mb > 126:
        return f"inputs larger than L2: q, k, v {mb:.0f} MB each"
    return f"inputs fit in L2 (q, k, v {mb:.1f} MB each): a test-size workload, not a bench line"


# ------------------------------------------------------------------ clocks

class ClockSampler:
    """nvidia-smi samples (200 ms) of SM clock and throttle reasons during the timed region."""
    FIELDS = ["clocks.sm", "clocks.max.sm", "power.draw", "utilization.gpu",
              "clocks_event_reasons.hw_slowdown", "clocks_event_reasons.hw_thermal_slowdown",
              "clocks_event_reasons.sw_thermal_slowdown", "clocks_event_reasons.sw_power_cap"]

    def __init__(self, gpu_id: str | None):
        self.gpu_id = gpu_id
        self.proc = None
        self.lines: list[str] = []
        self.thread = None

    def start(self):
        cmd = ["nvidia-smi", "--query-gpu=" + ",".join(self.FIELDS), "--format=csv,noheader,nounits",
               "-lms", "200"]
        if self.gpu_id:
            cmd += ["--id=" + self.gpu_id]
        try:
            self.proc = subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, FileNotFoundError):
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        if self.thread:
            self.thread.join(timeout=2)
        rows = []
        for l in self.lines:
            parts = [p.strip() for p in l.split(",")]
            if len(parts) != len(self.FIELDS):
                continue
            try:
                rows.append((float(parts[0]), float(parts[1]), float(parts[3]), parts[4:]))
            except ValueError:
                continue
        if not rows:
            return None
        loaded = [r for r in rows if r[2] >= 50.0] or rows
        reasons = set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in loaded:
            for n, v in zip(names, r[3]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(r[0] for r in loaded), "sm_max_mhz": max(r[1] for r in rows),
                "reasons": sorted(reasons), "samples": len(rows), "samples_under_load": len(loaded)}


# ----------------------------------------------------------------- oracle leg

_SLAB_CACHE = {}


def _slab64(cfg, slab):
    from block_sparse_spherical_b200.synthetic import make_slab
    key = (cfg.name, slab)
    if key not in _SLAB_CACHE:
        if len(_SLAB_CACHE) > 2:
            _SLAB_CACHE.clear()
        s = make_slab(cfg, slab)
        _SLAB_CACHE[key] = tuple(x.astype(np.float64) for x in (s.q, s.k, s.v, s.gates))
    return _SLAB_CACHE[key]


def oracle_sample(cfg, target_s: float, lib=None):
    """Time the oracle on a bounded sample of the workload; return (tokens/s, description, seconds).

    The oracle works slab by slab (one batch element, one head); tokens/s counts
    batch x N tokens like the GPU leg, i.e. the head rows done per second / heads.

    Whole slabs (pool, compressed rows, selection+local+combine) are timed one
    after another until about target_s seconds of oracle time are spent; the
    last slab may be cut to its first query blocks (pooling pro-rated).
    """
    import oracle
    lib = lib or oracle.load_native()
    bk, n, w, m = cfg.block_size, cfg.top_n, cfg.window_blocks, cfg.n_blocks
    spent, tokens, slabs_done, part = 0.0, 0, 0, None
    for slab in range(cfg.slabs):
        q, k, v, g = _slab64(cfg, slab)
        t0 = time.perf_counter()
        qb, kb, vb = (oracle.pool(x, bk, lib=lib) for x in (q, k, v))
        t_pool = time.perf_counter() - t0
        left = target_s - spent
        # estimate the per-block cost on a short probe, then size this slab's share
        probe = min(m, 8)
        t0 = time.perf_counter()
        c = oracle.compressed_rows(qb, kb, vb, n, rows=(0, probe), lib=lib)
        ocg = np.zeros((m, cfg.head_dim)); ocg[:probe] = c["o_cg"]
        idx = np.zeros((m, n), np.int32); idx[:probe] = c["idx"]
        oracle.fine_rows(q, k, v, g, ocg, idx, bk, n, w, qblocks=(0, probe), lib=lib)
        t_probe = time.perf_counter() - t0
        nblk = int(min(m, max(probe, probe * left / max(t_probe, 1e-6))))
        t0 = time.perf_counter()
        c = oracle.compressed_rows(qb, kb, vb, n, rows=(0, nblk), lib=lib)
        ocg = np.zeros((m, cfg.head_dim)); ocg[:nblk] = c["o_cg"]
        idx = np.zeros((m, n), np.int32); idx[:nblk] = c["idx"]
        oracle.fine_rows(q, k, v, g, ocg, idx, bk, n, w, qblocks=(0, nblk), lib=lib)
        spent += time.perf_counter() - t0 + t_pool * nblk / m
        tokens += nblk * bk
        if nblk < m:
            part = nblk
            break
        slabs_done += 1
        if spent >= target_s:
            break
    desc = f"{slabs_done} whole slab(s) of {cfg.name}"
    if part is not None:
        desc += f" + query blocks 0..{part - 1} of the next ({tokens} head rows in all; its pooling pro-rated)"
    else:
        desc += f" ({tokens} head rows)"
    desc += ("; each slab: pooling, compressed rows over all key blocks with top-n, selection+local+combine; "
             "oracle built -O3 -march=native -ffp-contract=off on this host")
    return tokens / spent / cfg.heads, desc, spent


def omp_threads():
    return int(os.environ.get("OMP_NUM_THREADS") or os.cpu_count() or 1)


def run_reference(args, cfg, rank):
    if rank != 0:
        return
    os.environ.setdefault("OMP_NUM_THREADS", str(os.cpu_count() or 1))
    import oracle
    lib = oracle.load_native()
    per_step = float(os.environ.get("BSA_ORACLE_STEP_S", "3.0"))
    for _ in range(args.warmup):
        oracle_sample(cfg, min(per_step, 0.5), lib=lib)
    rates, descs, secs = [], [], 0.0
    for _ in range(args.steps):
        r, d, e = oracle_sample(cfg, per_step, lib=lib)
        rates.append(r)
        descs.append(d)
        secs += e
    value = statistics.median(rates)
    tokens_step = cfg.batch * cfg.n_tokens
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * tokens_step / value, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic", "config": workload_config(cfg),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": omp_threads(), "kind": "oracle",
                             "sample": descs[-1] + "; value = median over steps, ms_per_step extrapolated "
                                                   "to the whole workload"},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------- GPU leg

def traffic_for(kernel_file: str, key: str):
    """DRAM bytes per launch from a committed ncu summary, if the kernel source is unchanged."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        d = json.load(f).get(key)
    if not d:
        return None
    src = os.path.join(ROOT, "block_sparse_spherical_b200", "csrc", kernel_file)
    sha = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
    if d.get("source_sha") != sha:
        return None
    return d.get("bytes_per_launch_full_workload")


def run_ours(args, cfg, rank, world, local_rank):
    import torch
    import torch.distributed as dist
    from block_sparse_spherical_b200 import abi, api
    from block_sparse_spherical_b200.replicas import (barrier, job_head_rows_per_step, job_tokens_per_step,
                                                      max_over_ranks, replica_config)
    from block_sparse_spherical_b200.synthetic import make_inputs

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=300), device_id=dev)

    # independent problem per rank: same workload, rank-offset seed
    qh, kh, vh, gh = make_inputs(replica_config(cfg, rank))
    tdt = torch.bfloat16 if cfg.dtype == "bf16" else torch.float32

    def host(a):
        t = torch.from_numpy(a)
        return t.view(torch.bfloat16) if a.dtype == np.uint16 else t

    q, k, v, g = (host(a).to(dev) for a in (qh, kh, vh, gh))
    stream = torch.cuda.current_stream(dev)
    bsa = api.BSA.from_config(cfg, device=dev)
    c = bsa.cfg
    m, d, n = cfg.n_blocks, cfg.head_dim, cfg.top_n
    qb, kb, vb, ocg = (torch.empty((cfg.batch, cfg.heads, m, d), dtype=torch.float32, device=dev) for _ in range(4))
    idx = torch.empty((cfg.batch, cfg.heads, m, n), dtype=torch.int32, device=dev)
    out = torch.empty_like(q)
    status = torch.zeros(1, dtype=torch.int32, device=dev)

    def step(evs=None):
        if evs:
            evs[0].record(stream)
        abi.bsa_pool(c, q, k, v, qb, kb, vb, stream)
        if evs:
            evs[1].record(stream)
        abi.bsa_compress_select_ws(c, qb, kb, vb, ocg, idx, bsa.workspace, bsa.workspace_bytes, stream)
        if evs:
            evs[2].record(stream)
        abi.bsa_fine_attention(c, q, k, v, g, ocg, idx, out, status, stream)
        if evs:
            evs[3].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    if abi.bsa_check_status(status, stream) != 0:
        raise RuntimeError("kernel status word reports an error")

    gpu_id = None
    try:
        gpu_id = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid) if rank == 0 else None
    except Exception:
        gpu_id = None
    sampler = ClockSampler(gpu_id) if rank == 0 else None
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    barrier(dev)
    torch.cuda.synchronize(dev)
    if sampler:
        sampler.start()
        time.sleep(0.5)
    for s in range(args.steps):
        step(evs[s])
    torch.cuda.synchronize(dev)
    clocks = sampler.stop() if sampler else None
    barrier(dev)
    total_ms = evs[0][0].elapsed_time(evs[-1][3])
    k_ms = {"pool": [e[0].elapsed_time(e[1]) for e in evs],
            "compress_select": [e[1].elapsed_time(e[2]) for e in evs],
            "fine_attention": [e[2].elapsed_time(e[3]) for e in evs]}
    total_ms = max_over_ranks(total_ms, dev)
    if abi.bsa_check_status(status, stream) != 0:
        raise RuntimeError("kernel status word reports an error")

    # ---- the fused kernel with a cold L2: a buffer twice the L2 size is written before each launch
    #      (outside the timed span), so no key/value tile of the previous launch is still cached
    flush = torch.empty(2 * 126 * 2**20, dtype=torch.uint8, device=dev)
    cold = []
    for _ in range(max(3, args.steps // 2)):
        flush.fill_(1)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        abi.bsa_fine_attention(c, q, k, v, g, ocg, idx, out, status, stream)
        e1.record(stream)
        cold.append((e0, e1))
    torch.cuda.synchronize(dev)
    cold_ms = statistics.median(a0.elapsed_time(a1) for a0, a1 in cold)
    del flush

    # ---- end to end through the public API with host buffers (pinned), rank-local: every step
    #      copies its inputs in and its output back (api.BSAStream overlaps those copies with the
    #      computation of the neighbouring steps, as a serving loop over batches would)
    e2e = None
    if not args.no_e2e:
        qp, kp, vp, gp = (host(a).pin_memory() for a in (qh, kh, vh, gh))
        outs = [torch.empty(out.shape, dtype=tdt).pin_memory() for _ in range(2)]
        pipe = api.BSAStream(bsa)
        e2e_steps = max(4, args.steps // 2)
        pipe.run([(qp, kp, vp, gp)] * 2, outs)        # warm-up
        pipe.synchronize()
        torch.cuda.synchronize(dev)
        barrier(dev)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(pipe.streams[0])
        pipe.run([(qp, kp, vp, gp)] * e2e_steps, [outs[i % 2] for i in range(e2e_steps)])
        b.record(pipe.streams[2])
        pipe.synchronize()
        torch.cuda.synchronize(dev)
        te_ms = max_over_ranks(a.elapsed_time(b), dev)
        h2d = sum(x.numel() * x.element_size() for x in (qp, kp, vp, gp))
        e2e = {"value": e2e_steps * job_tokens_per_step(cfg, world) / (te_ms / 1e3), "unit": UNIT,
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": outs[0].numel() * outs[0].element_size(),
               "steps": e2e_steps,
               "api": "api.BSAStream.run -> bsa_forward (C ABI); host copies overlapped with the neighbouring steps"}
        if bsa.check_status() != 0:
            raise RuntimeError("kernel status word reports an error")

    if world > 1:
        dist.destroy_process_group()
    if rank != 0:
        return

    peaks, peak_src = load_peaks()
    ms_step = total_ms / args.steps
    value = job_tokens_per_step(cfg, world) / (ms_step / 1e3)
    head_rows = job_head_rows_per_step(cfg, world) / (ms_step / 1e3)
    fine_flops, comp_flops = cfg.fine_flops(), cfg.compressed_flops()
    mean = {kname: statistics.mean(v) for kname, v in k_ms.items()}
    median = {kname: statistics.median(v) for kname, v in k_ms.items()}
    fine_tflops = fine_flops / (mean["fine_attention"] / 1e3) / 1e12
    pool_gbs = cfg.pool_bytes() / (mean["pool"] / 1e3) / 1e9
    comp_tflops = comp_flops / (mean["compress_select"] / 1e3) / 1e12
    comp_gbs = cfg.compress_min_bytes() / (mean["compress_select"] / 1e3) / 1e9
    fine_gbs = cfg.fused_min_bytes() / (mean["fine_attention"] / 1e3) / 1e9
    sm_mhz = (clocks or {}).get("sm_mhz") or peaks.get("sm_max_mhz", 1965.0)
    m64_rate = measured_m64_rate()
    m64_ceiling = m64_rate * 2 * SM_COUNT_B200 * sm_mhz * 1e6 / 1e12
    fp32_peak = SM_COUNT_B200 * 128 * 2 * peaks.get("sm_max_mhz", 1965.0) * 1e6 / 1e12
    # Each kernel runs for a few milliseconds inside a step loop well under the power cap, so the
    # burst GEMM figure is its denominator; the sustained (power-capped) one is reported beside it.
    tensor_peak = peaks["bf16_tflops"]
    tensor_sustained = peaks["bf16_tflops_sustained"]
    if compress_on_tensor_cores(cfg):
        # fp32-accurate products as three tf32 MMAs each: the ceiling for the algorithmic
        # (fp32) flops is a third of the tf32 tensor rate
        tf32_peak = tensor_peak * TF32_PER_BF16
        comp = {"ms": mean["compress_select"], "ms_median": median["compress_select"], "bound": "tensor",
                "kernel": "split_images_kernel + compress_tc_kernel (three-pass tf32)",
                "achieved_tflops_fp32": comp_tflops, "peak_tflops_fp32": tf32_peak / 3,
                "frac": comp_tflops / (tf32_peak / 3), "tf32_issued_tflops": 3 * comp_tflops,
                "peak_tflops_tf32": tf32_peak,
                "peak_source": f"{peak_src} bf16_tflops (burst) x {TF32_PER_BF16:.3f} (nominal tf32:bf16) / 3 passes",
                "frac_of_sustained": comp_tflops / (tensor_sustained * TF32_PER_BF16 / 3),
                "achieved_gbs": comp_gbs, "frac_hbm": comp_gbs / peaks["hbm_gbs"], "algorithmic_flops": comp_flops}
    else:
        comp = {"ms": mean["compress_select"], "bound": "alu", "kernel": "compress_select_kernel (fp32 CUDA cores)",
                "achieved_tflops_fp32": comp_tflops, "peak_tflops_fp32": fp32_peak, "frac": comp_tflops / fp32_peak,
                "peak_source": "148 SMs x 128 FP32 lanes x 2 flop x max SM clock",
                "achieved_gbs": comp_gbs, "frac_hbm": comp_gbs / peaks["hbm_gbs"], "algorithmic_flops": comp_flops}
    kernels = {
        # a read-mostly stream can beat the measured copy bandwidth (a read+write copy): the ratio
        # to it is labelled as such, and the fraction of the nominal HBM3e bandwidth stays below 1
        "pool": {"ms": mean["pool"], "ms_median": median["pool"], "bound": "hbm", "achieved_gbs": pool_gbs,
                 "frac": pool_gbs / peaks["hbm_gbs"], "frac_is": f"of the {peak_src} copy bandwidth (hbm_gbs)",
                 "frac_nominal_hbm": pool_gbs / NOMINAL_HBM_GBS, "nominal_hbm_gbs": NOMINAL_HBM_GBS,
                 "algorithmic_bytes": cfg.pool_bytes()},
        "compress_select": comp,
        "fine_attention": {"ms": mean["fine_attention"], "ms_median": median["fine_attention"],
                           "ms_cold_l2": cold_ms, "tflops_cold_l2": fine_flops / (cold_ms / 1e3) / 1e12,
                           "bound": "tensor", "achieved_tflops": fine_tflops,
                           "frac": fine_tflops / tensor_peak, "frac_is": f"of the {peak_src} burst bf16_tflops",
                           "frac_of_sustained": fine_tflops / tensor_sustained,
                           # M=64 tiles drive half of the tensor datapath: the library's tcgen05.mma
                           # microbenchmark measures the M=64 multiply-add rate per clock per SM here, and
                           # the ceiling takes it at the SM clock sampled during the timed region
                           "m64_rate_mac_per_clk_sm": m64_rate,
                           "m64_ceiling_tflops": m64_ceiling,
                           "frac_of_m64_ceiling": fine_tflops / m64_ceiling,
                           "achieved_gbs": fine_gbs, "algorithmic_flops": fine_flops},
    }
    dom = max(kernels, key=lambda kk: kernels[kk]["ms"])
    kd = kernels[dom]
    if dom == "compress_select" and kd["bound"] == "tensor":
        roof = {"kernel": dom, "bound": "tensor", "achieved": kd["achieved_tflops_fp32"],
                "peak": kd["peak_tflops_fp32"], "unit": "TFLOP/s", "frac": kd["frac"], "peak_source": kd["peak_source"]}
    elif kd["bound"] == "tensor":
        roof = {"kernel": dom, "bound": "tensor", "achieved": kd["achieved_tflops"], "peak": tensor_peak,
                "unit": "TFLOP/s", "frac": kd["frac"],
                "peak_source": f"{peak_src} bf16_tflops (burst: a few-ms kernel below the power cap)",
                "frac_of_sustained": kd["frac_of_sustained"], "sustained_peak": tensor_sustained}
    elif kd["bound"] == "hbm":
        roof = {"kernel": dom, "bound": "hbm", "achieved": kd["achieved_gbs"], "peak": peaks["hbm_gbs"],
                "unit": "GB/s", "frac": kd["frac"], "peak_source": f"{peak_src} hbm_gbs (copy bandwidth)"}
    else:
        roof = {"kernel": dom, "bound": "alu", "achieved": kd["achieved_tflops_fp32"], "peak": fp32_peak,
                "unit": "TFLOP/s", "frac": kd["frac"],
                "peak_source": "148 SMs x 128 FP32 lanes x 2 flop x max SM clock"}
    kfile = {"fine_attention": "attend_tc.cu", "pool": "pool.cu",
             "compress_select": "compress_tc.cu" if compress_on_tensor_cores(cfg) else "compress_select.cu"}[dom]
    roof["traffic"] = traffic_for(kfile, f"{dom}:{cfg.name}")

    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        os.environ.setdefault("OMP_NUM_THREADS", str(os.cpu_count() or 1))
        rate, desc, secs = oracle_sample(cfg, float(os.environ.get("BSA_ORACLE_SAMPLE_S", "12")))
        cpu = {"value": rate, "unit": UNIT, "cores": omp_threads(), "kind": "oracle",
               "sample": desc, "seconds": secs}

    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": cfg.dtype, "data": "synthetic",
            "config": dict(workload_config(cfg), parallelism=f"{world} independent replica(s), no collective"),
            "tflops": world * (fine_flops + comp_flops) / (ms_step / 1e3) / 1e12,
            "head_rows_per_s": head_rows,
            "tokens_definition": "batch x N tokens per step (x world); head_rows_per_s = batch x heads x N",
            "kernels": kernels, "roofline": roof, "cpu_baseline": cpu, "e2e": e2e,
            "gpu_launches": kernels_per_step(cfg) * args.steps, "clocks": clocks,
            "gpu": torch.cuda.get_device_name(dev)}
    print(json.dumps(line), flush=True)


def run_sharded(args, cfg, rank, world, local_rank):
    """One problem split by (batch, head) slab over the ranks (sharding.ShardedBSA): each rank runs
    bsa_forward on its contiguous slab range, then one NCCL all-gather reassembles the output on
    every rank. A step = shard forward + all-gather; "scaling": "strong" (the job's work is fixed)."""
    import torch
    import torch.distributed as dist
    from block_sparse_spherical_b200.replicas import barrier, max_over_ranks
    from block_sparse_spherical_b200.sharding import ShardedBSA
    from block_sparse_spherical_b200.synthetic import make_inputs

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=300), device_id=dev)
    qh, kh, vh, gh = make_inputs(cfg)
    host = lambda a: torch.from_numpy(a).view(torch.bfloat16) if a.dtype == np.uint16 else torch.from_numpy(a)
    q, k, v, g = (host(a).to(dev) for a in (qh, kh, vh, gh))
    layer = ShardedBSA(cfg.batch, cfg.heads, cfg.n_tokens, cfg.head_dim, cfg.block_size, cfg.top_n,
                       cfg.window_blocks, torch.bfloat16 if cfg.dtype == "bf16" else torch.float32, device=dev,
                       gather="fused" if args.fused_gather else "nccl")
    for _ in range(args.warmup):
        layer(q, k, v, g)
    torch.cuda.synchronize(dev)
    stream = torch.cuda.current_stream(dev)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(dev)
    torch.cuda.synchronize(dev)
    a.record(stream)
    for _ in range(args.steps):
        layer(q, k, v, g)
    b.record(stream)
    torch.cuda.synchronize(dev)
    total_ms = max_over_ranks(a.elapsed_time(b), dev)
    if world > 1:
        dist.destroy_process_group()
    if rank != 0:
        return
    ms = total_ms / args.steps
    line = {"metric": METRIC, "mode": "sharded", "value": cfg.batch * cfg.n_tokens / (ms / 1e3), "unit": UNIT,
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "strong", "vs_baseline": None, "dtype": cfg.dtype,
            "data": "synthetic",
            "config": dict(workload_config(cfg), parallelism=f"(batch, head) slabs split over {world} rank(s) + "
                                                             + ("output rows stored to every rank by the kernel"
                                                                if args.fused_gather else "NCCL all-gather of the output")),
            "tflops": (cfg.fine_flops() + cfg.compressed_flops()) / (ms / 1e3) / 1e12,
            "gpu_launches": 4 * args.steps, "gpu": torch.cuda.get_device_name(dev)}
    print(json.dumps(line), flush=True)


def _event_ms(fn, steps, warmup, dev):
    import torch
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize(dev)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(steps):
        fn()
    b.record()
    torch.cuda.synchronize(dev)
    return a.elapsed_time(b) / steps


def run_interp(args, rank, local_rank):
    """Lat-lon -> HEALPix cross-attention interpolation: a 0.25 degree grid (721 x 1440) onto the
    786,432 pixels of Nside 256, d = 64, bf16 features, batch 8 (the Nside 256 workload's heads).
    One step = bsa_latlon_to_healpix over the plan (built once, outside the timed region)."""
    import torch
    from block_sparse_spherical_b200 import abi, api
    if rank != 0:
        return
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    nside, nlat, nlon, d, batch = 256, 721, 1440, 64, 8
    g = torch.Generator(device=dev).manual_seed(9)
    k = torch.randn((batch, nlat * nlon, d), generator=g, device=dev).to(torch.bfloat16)
    v = torch.randn((batch, nlat * nlon, d), generator=g, device=dev).to(torch.bfloat16)
    wq = (torch.randn((d, 3), generator=g, device=dev) / 3 ** 0.5).float()
    layer = api.LatLonToHealpix(nside, nlat, nlon, device=dev)
    out = torch.empty((batch, layer.npix, d), dtype=torch.bfloat16, device=dev)
    plan_ms = _event_ms(lambda: abi.bsa_latlon_healpix_plan(nside, nlat, nlon, layer.nbr, layer.rel), 3, 1, dev)
    ms = _event_ms(lambda: layer(k, v, wq, out=out), args.steps, args.warmup, dev)
    npix = layer.npix
    # bytes the kernel must move at least: the plan (16 indices + 48 floats per pixel), the output,
    # and the gathered rows (16 neighbours' k and v per pixel), which come from L2 (source 2 x 133 MB)
    plan_b = npix * (16 * 4 + 48 * 4)
    out_b = batch * npix * d * 2
    gather_b = batch * npix * 16 * 2 * d * 2
    peaks, src = load_peaks()
    line = {"metric": "lat-lon -> HEALPix interpolation pixels/s (0.25 deg grid onto Nside 256, d 64, bf16)",
            "pass": "interp", "value": batch * npix / (ms / 1e3), "unit": "pixels/s", "n_gpus": 1,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
            "dtype": "bf16", "data": "synthetic",
            "config": {"workload": "interp_0.25deg_to_nside256", "nlat": nlat, "nlon": nlon, "nside": nside,
                       "head_dim": d, "batch": batch, "neighbours": 16},
            "plan_ms": plan_ms,
            "roofline": {"kernel": "interp_kernel", "bound": "hbm", "achieved": (plan_b + out_b) / (ms / 1e3) / 1e9,
                         "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": (plan_b + out_b) / (ms / 1e3) / 1e9 / peaks["hbm_gbs"],
                         "l2_gather_gbs": gather_b / (ms / 1e3) / 1e9, "peak_source": f"{src} hbm_gbs",
                         "traffic": None},
            "gpu_launches": args.steps, "gpu": torch.cuda.get_device_name(dev)}
    print(json.dumps(line), flush=True)


def run_latlon(args, cfg, rank, local_rank):
    """BSA over lat-lon blocks (the note's "BSA but not HEALPix" ablation) at the workload's size:
    N points of a 384 x 512 (Nside 128: 196,608) lat-lon grid in 8 x 8 patches. One step = permute q,
    k, v, gates to block-contiguous order, bsa_forward, permute the output back."""
    import torch
    from block_sparse_spherical_b200 import abi, api, layouts
    from block_sparse_spherical_b200.synthetic import make_inputs
    if rank != 0:
        return
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    grids = {12288: (96, 128), 49152: (192, 256), 196608: (384, 512), 786432: (768, 1024)}
    nlat, nlon = grids[cfg.n_tokens]
    perm = torch.from_numpy(layouts.latlon_patches(nlat, nlon, 8, 8)).to(dev)
    inv = torch.from_numpy(layouts.inverse(layouts.latlon_patches(nlat, nlon, 8, 8))).to(dev)
    host = lambda a: torch.from_numpy(a).view(torch.bfloat16) if a.dtype == np.uint16 else torch.from_numpy(a)
    q, k, v, g = (host(a).to(dev) for a in make_inputs(cfg))
    qp, kp, vp, gp = (torch.empty_like(x) for x in (q, k, v, g))
    bsa = api.BSA.from_config(cfg, device=dev)
    out, outr = torch.empty_like(q), torch.empty_like(q)
    S, n = cfg.slabs, cfg.n_tokens

    def step():
        for src, dst in ((q, qp), (k, kp), (v, vp), (g, gp)):
            abi.bsa_permute_tokens(S, n, src.shape[-1] * src.element_size(), perm, src, dst)
        bsa(qp, kp, vp, gp, out=out)
        abi.bsa_permute_tokens(S, n, out.shape[-1] * out.element_size(), inv, out, outr)

    ms = _event_ms(step, args.steps, args.warmup, dev)
    perm_b = 2 * (3 * q.numel() * q.element_size() + g.numel() * 4 + out.numel() * out.element_size())
    fwd_ms = _event_ms(lambda: bsa(q, k, v, g, out=out), args.steps, args.warmup, dev)
    line = {"metric": "BSA fwd tokens/s over lat-lon 8x8-patch blocks (permute, forward, permute back)",
            "pass": "latlon", "value": cfg.batch * n / (ms / 1e3), "unit": "tokens/s", "n_gpus": 1,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
            "dtype": cfg.dtype, "data": "synthetic",
            "config": dict(workload_config(cfg), grid=f"{nlat} x {nlon} lat-lon, 8 x 8 patches"),
            "forward_alone_ms": fwd_ms, "permute_ms": ms - fwd_ms,
            "permute_gbs": perm_b / ((ms - fwd_ms) / 1e3) / 1e9 if ms > fwd_ms else None,
            "gpu_launches": 6 * args.steps, "gpu": torch.cuda.get_device_name(dev)}
    print(json.dumps(line), flush=True)


def run_backward(args, cfg, rank, world, local_rank):
    """Training pass: one step = bsa_backward (every backward kernel) on the saved tensors of one
    bsa_forward_train of the workload, with a seeded dout; the forward itself is not timed."""
    import torch
    import torch.distributed as dist
    from block_sparse_spherical_b200 import abi, api
    from block_sparse_spherical_b200.replicas import barrier, job_tokens_per_step, max_over_ranks, replica_config
    from block_sparse_spherical_b200.synthetic import f32_to_bf16_bits, make_inputs

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=300), device_id=dev)
    rcfg = replica_config(cfg, rank)
    qh, kh, vh, gh = make_inputs(rcfg)
    host = lambda a: torch.from_numpy(a).view(torch.bfloat16) if a.dtype == np.uint16 else torch.from_numpy(a)
    q, k, v, g = (host(a).to(dev) for a in (qh, kh, vh, gh))
    rng = np.random.default_rng(rcfg.seed + 77)
    dout = host(f32_to_bf16_bits(rng.standard_normal(qh.shape, dtype=np.float32))).to(dev)
    layer = api.BSATrain.from_config(cfg, device=dev)
    layer(q, k, v, g)
    grads = (torch.empty_like(q), torch.empty_like(k), torch.empty_like(v), torch.empty_like(g))
    for _ in range(args.warmup):
        layer.backward(dout, grads)
    torch.cuda.synchronize(dev)
    if layer.check_status() != 0 or layer.check_backward_status() != 0:
        raise RuntimeError("kernel status word reports an error")
    stream = torch.cuda.current_stream(dev)
    sampler = ClockSampler(None) if rank == 0 else None
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(dev)
    torch.cuda.synchronize(dev)
    if sampler:
        sampler.start()
        time.sleep(0.5)
    a.record(stream)
    for _ in range(args.steps):
        layer.backward(dout, grads)
    b.record(stream)
    torch.cuda.synchronize(dev)
    clocks = sampler.stop() if sampler else None
    total_ms = max_over_ranks(a.elapsed_time(b), dev)
    if layer.check_backward_status() != 0:
        raise RuntimeError("kernel status word reports an error")
    if world > 1:
        dist.destroy_process_group()
    if rank != 0:
        return
    peaks, peak_src = load_peaks()
    ms = total_ms / args.steps
    # algorithmic work: per (query, key) pair the backward recomputes S and forms dP, dV, dK and dQ,
    # 10*d flops against the forward's 4*d, in both the fine branches and the compressed branch
    flops = 2.5 * (cfg.fine_flops() + cfg.compressed_flops())
    tf = world * flops / (ms / 1e3) / 1e12
    line = {"metric": "BSA bwd tokens/s & TFLOP/s (training gradient of the forward; selection held fixed)",
            "pass": "backward", "value": job_tokens_per_step(cfg, world) / (ms / 1e3), "unit": UNIT,
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": cfg.dtype,
            "data": "synthetic", "config": dict(workload_config(cfg), parallelism=f"{world} independent replica(s)"),
            "tflops": tf, "algorithmic_flops": flops,
            "roofline": {"kernel": "whole backward (10 kernels; attend_bwd_tc dominant, see profiles/)",
                         "bound": "tensor", "achieved": tf / world, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                         "frac": tf / world / peaks["bf16_tflops"], "peak_source": f"{peak_src} bf16_tflops (burst)",
                         "traffic": None},
            "gpu_launches": 10 * args.steps, "clocks": clocks, "gpu": torch.cuda.get_device_name(dev)}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=HEADLINE, choices=sorted(CONFIGS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--pass", dest="which", default="forward", choices=["forward", "backward", "interp", "latlon"],
                    help="backward: the training gradient (bsa_backward); interp: the lat-lon -> HEALPix "
                         "interpolation; latlon: BSA over lat-lon patch blocks (with the permutations)")
    ap.add_argument("--shard", action="store_true",
                    help="split one problem's (batch, head) slabs over the ranks (strong scaling) instead of "
                         "running an independent replica per rank")
    ap.add_argument("--block-size", type=int, default=None,
                    help="override the workload's block size (tokens per block: 64, 256 or 1024 for bf16)")
    ap.add_argument("--top-n", type=int, default=None, help="override the workload's top-n")
    ap.add_argument("--fused-gather", action="store_true",
                    help="with --shard: the kernel's epilogue stores output rows into every rank's buffer "
                         "(symmetric memory) instead of an NCCL all-gather after the forward")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    cfg = CONFIGS[args.workload]
    if args.block_size or args.top_n:
        bk = args.block_size or cfg.block_size
        cfg = cfg.with_(name=f"{cfg.name}_block{bk}_n{args.top_n or cfg.top_n}", block_size=bk,
                        top_n=args.top_n or cfg.top_n)
    if args.impl == "reference":
        run_reference(args, cfg, rank)
    elif args.which == "backward":
        run_backward(args, cfg, rank, world, local_rank)
    elif args.which == "interp":
        run_interp(args, rank, local_rank)
    elif args.which == "latlon":
        run_latlon(args, cfg, rank, local_rank)
    elif args.shard:
        run_sharded(args, cfg, rank, world, local_rank)
    else:
        run_ours(args, cfg, rank, world, local_rank)


if __name__ == "__main__":
    main()
