#!/usr/bin/env python
"""Throughput of the image half of the Mistral 3 / Pixtral forward on B200.

One step = the whole path on one batch of synthetic input: the 24-layer
vision tower (vlm_encode), the 2x2 merge + projector (vlm_merge_project) and
the masked scatter of the image embeddings into a text-embedding sequence
(vlm_scatter). Metric: vision patches per second (whole job, all ranks).

    python bench.py [--gpus N --steps K --warmup W] [--workload NAME] [--impl reference]

N > 1 runs one independent replica per GPU (launched by torch.distributed.run;
no collective on the data path; a NCCL all-reduce only takes the max of the
ranks' timings).
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "vision patches/sec through 24-layer tower+merger+projector; % BF16 TC peak"

# Workloads: image sizes (H, W) of one step and the text sequences the
# embeddings are scattered into.
WORKLOADS = {
    "mistral3_1540": dict(preset="mistral3", sizes=[(1540, 1540)], n_seq=1, seq_len=4096,
                          desc="one 1540x1540 image (110x110 = 12,100 patches -> 3,025 merged tokens), "
                               "24-layer tower + 2x2 merge + projector 1024->5120->5120 + scatter into "
                               "4,096 text tokens"),
    "packed8": dict(preset="mistral3", sizes="packed", n_seq=1, seq_len=16384,
                    desc="8 images, sides 28*U{10..55} (seed 0), packed into one sequence"),
    "pixtral_4096": dict(preset="pixtral12b", sizes=[(1024, 1024)] * 16, n_seq=16, seq_len=4352,
                         desc="Pixtral-12B-style: one 4096x4096 image as 16 tiles of 1024x1024 = 65,536 patches, "
                              "no merge, projector 1024->5120->5120"),
    "mistral3_1540_fp8": dict(preset="mistral3", sizes=[(1540, 1540)], n_seq=1, seq_len=4096, fp8=True,
                              desc="one 1540x1540 image (12,100 patches -> 3,025 merged tokens), 24-layer tower with "
                                   "E4M3 QKV/O/gate-up/down GEMMs (per-row weight scales, static activation scales; "
                                   "bf16 attention, norms, patch embed) + 2x2 merge + bf16 projector + scatter"),
    "mistral3_1540_nvfp4": dict(preset="mistral3", sizes=[(1540, 1540)], n_seq=1, seq_len=4096, nvfp4=True,
                                desc="one 1540x1540 image (12,100 patches -> 3,025 merged tokens), 24-layer tower "
                                     "with NVFP4 QKV/O/gate-up/down GEMMs (E2M1 with E4M3 block scales per 16 "
                                     "values; weight global scales from the data, static activation global scales; "
                                     "every GEMM input quantised in the kernel that produces it; bf16 attention, "
                                     "norms, patch embed) + 2x2 merge + bf16 projector + scatter"),
    "photo_4032x3024": dict(preset="mistral3", photo=(3024, 4032), sizes=[(1176, 1540)], n_seq=1, seq_len=4096,
                            desc="one decoded 4032x3024 u8 RGB photo: GPU resize to 1176x1540 (longest edge 1540, "
                                 "28-px grid; 84x110 = 9,240 patches -> 2,310 merged tokens), 24-layer tower + "
                                 "merge + projector, device placeholder expansion of one marker, scatter into "
                                 "4,096 ids"),
    "e2e4": dict(preset="mistral3", sizes=[(896, 1344)] * 4, n_seq=4, seq_len=4096,
                 desc="4 x 896x1344 images (6,144 patches -> 1,536 placeholders each) scattered into 4 x 4,096 ids"),
}


# (patch, merge, layers) of the two presets, for describing a workload without the library
PRESET_SHAPES = {"mistral3": (14, 2, 24), "pixtral12b": (16, 1, 24)}


def workload_config(wl: dict, sizes, world: int) -> dict:
    """The JSON line's `config`: the same object for both arms of the bench."""
    p, m, layers = PRESET_SHAPES[wl["preset"]]
    patches = sum((h // p) * (w // p) for h, w in sizes)
    merged = sum((h // p) * (w // p) // (m * m) for h, w in sizes)
    return {"workload": wl["desc"], "patches": patches, "merged_tokens": merged, "layers": layers,
            "images": len(sizes), "text_tokens": wl["n_seq"] * wl["seq_len"] if not wl.get("photo") else wl["seq_len"],
            "parallelism": f"replicas{world}",
            "l2": "inputs larger than L2 (weights 0.88 GB + activations per step)"}


def parse_args():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=20)
    p.add_argument("--warmup", type=int, default=3)
    p.add_argument("--impl", default="ours", choices=["ours", "reference"])
    p.add_argument("--workload", default="mistral3_1540", choices=sorted(WORKLOADS))
    p.add_argument("--seed", type=int, default=0)
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--graph", action="store_true",
                   help="replay each step as one captured CUDA graph (headline and e2e loops)")
    p.add_argument("--side-stream", action="store_true",
                   help="also measure the encoder on a side stream overlapped with a decode-like GEMV loop")
    p.add_argument("--sm-budget", type=int, default=0,
                   help="vlm_config.sm_budget: SMs the encoder's persistent kernels may hold and twice the CTAs of "
                        "each attention grid (0 = every SM); with --side-stream the rest of the GPU is left to the "
                        "other stream")
    p.add_argument("--gemm-shapes", action="store_true",
                   help="instead of a step: time the tower's GEMM shapes (12,100 rows), bf16, E4M3 and NVFP4, each "
                        "with its fused epilogue and with a plain store, beside torch's cuBLAS / cuBLASLt GEMM; one "
                        "JSON line per shape and dtype")
    p.add_argument("--scatter", default="fused", choices=["fused", "separate"],
                   help="fused (default): vlm_merge_project_scatter, the masked scatter in the projector's last "
                        "linear, no embedding buffer; separate: vlm_merge_project then vlm_scatter")
    p.add_argument("--profile-steps", type=int, default=0,
                   help="for ncu: run this many plain steps after warmup and exit (no JSON)")
    return p.parse_args()


def sizes_of(wl: dict, seed: int):
    from vision_language_model_b200 import synth
    return synth.packed_sizes(seed, 8) if wl["sizes"] == "packed" else list(wl["sizes"])


def measured_peaks() -> dict:
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as fh:
            d = json.load(fh)
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d["bf16_tflops_sustained"], "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


# ---------------------------------------------------------------------------
# FLOP accounting (2 FLOPs per multiply-add; attention over each block's own L_b^2 pairs)
# ---------------------------------------------------------------------------

def flops_breakdown(cfg, sizes) -> dict:
    D, F, E, m, p, L = cfg.width, cfg.mlp, cfg.proj_out, cfg.merge, cfg.patch, cfg.layers
    lens = [(h // p) * (w // p) for h, w in sizes]
    T = sum(lens)
    Tm = sum(n // (m * m) for n in lens)
    gemm = 2.0 * T * 3 * p * p * D
    gemm += L * 2.0 * T * (3 * D * D + D * D + 2 * F * D + F * D)
    gemm += (2.0 * Tm * m * m * D * D if m > 1 else 0.0) + 2.0 * Tm * (D * E + E * E)
    attn_per_launch = sum(4.0 * n * n * D for n in lens)
    return {"T": T, "Tm": Tm, "gemm": gemm, "attn_per_launch": attn_per_launch, "attn": L * attn_per_launch,
            "total": gemm + L * attn_per_launch}


# ---------------------------------------------------------------------------
# Clocks sampled during the timed region
# ---------------------------------------------------------------------------

class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.proc = None
        self.lines = []
        try:
            uuid = "GPU-" + str(torch.cuda.get_device_properties(device_index).uuid)
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", uuid, f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.lines:
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 7:
                continue
            try:
                sm.append(float(parts[0]))
                smax.append(float(parts[1]))
            except ValueError:
                continue
            for n, v in zip(names, parts[3:7]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": float(np.median(sm)) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------------------
# Distributed plumbing (replicas; the all-reduce only takes max over ranks)
# ---------------------------------------------------------------------------

def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=180),
                                device_id=torch.device("cuda", local))
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(world, value: float) -> float:
    """The largest of the ranks' values (every rank gets it)."""
    if world == 1:
        return value
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([value], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(units_per_rank: int, world: int, steps: int, ms_max: float) -> float:
    """Whole-job units per second: every rank's units over the slowest rank's time."""
    return units_per_rank * world * steps / (ms_max / 1000.0)


# ---------------------------------------------------------------------------
# CPU baseline: the oracle, on a bounded sample of the same workload
# ---------------------------------------------------------------------------

def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return int(max(n)) if n else 1
    except Exception:
        return os.cpu_count() or 1


class OracleSample:
    """Times the oracle on the workload: patch embed + ln_pre on all patches,
    one tower block (keys/values of all patches once, then every per-row step
    on a strided slice of 1/`frac` of the patches), and the projector on all
    merged tokens; the tower time is extrapolated to all rows and all layers."""

    def __init__(self, wl: dict, seed: int, frac: int):
        from oracle import vlm_oracle as O
        from vision_language_model_b200 import synth
        self.O = O
        self.sizes = sizes_of(wl, seed)
        base = O.MISTRAL3 if wl["preset"] == "mistral3" else O.PIXTRAL12B
        self.cfg = dict(base)
        self.frac = frac
        tw = synth.tower_weights(seed, 1, base["width"], base["mlp"], base["patch"])
        self.tw = {k: v.double().numpy() for k, v in tw.items()}
        self.lw = O.layer_weights(self.tw, 0)
        pw = synth.projector_weights(seed, base["width"], base["merge"], base["proj_out"])
        self.pw = {k: v.double().numpy() for k, v in pw.items()}
        self.imgs = [im.double().numpy() for im in synth.images(seed, self.sizes)]
        self.quantised = bool(wl.get("fp8") or wl.get("nvfp4"))
        self.grids = [O.patch_grid(h, w, base["patch"]) for h, w in self.sizes]
        self.T = sum(h * w for h, w in self.grids)
        self.step_i = 0

    def prepare(self):
        O = self.O
        t0 = time.perf_counter()
        x = np.concatenate([O.patch_embed(O.normalize_pixels(im), self.tw["w_pe"]) for im in self.imgs])
        self.x = O.rms_norm(x, self.tw["g_pre"], self.cfg["eps"])
        t1 = time.perf_counter()
        rows, cols, self.cu = O.positions(self.grids)
        self.ang = O.rope_angles(rows, cols, self.cfg["rope_theta"], self.cfg["head_dim"])
        self.kv = O.block_keys_values(self.x, self.lw, self.ang, self.cfg)
        t2 = time.perf_counter()
        O.projector(self.x, self.grids, self.pw, self.cfg)
        t3 = time.perf_counter()
        self.t_embed, self.t_kv, self.t_proj = t1 - t0, t2 - t1, t3 - t2

    def step(self) -> float:
        rows = np.arange(self.step_i % self.frac, self.T, self.frac)
        self.step_i += 1
        t0 = time.perf_counter()
        self.O.tower_block_rows(self.x, self.lw, self.ang, self.cu, self.cfg, rows, kv=self.kv)
        return (time.perf_counter() - t0) * self.T / len(rows)

    def patches_per_s(self, t_rows_full: float, layers: int) -> float:
        return self.T / (self.t_embed + layers * (self.t_kv + t_rows_full) + self.t_proj)

    def describe(self) -> str:
        quant = (" (the unquantised block: the oracle's quantised block runs the same products plus its "
                 "quantisation passes)" if self.quantised else "")
        return (f"oracle (numpy fp64): patch embed of all {self.T} patches, keys/values of one tower block for all "
                f"patches, the rest of that block on every {self.frac}th patch{quant}, projector on all merged "
                f"tokens; tower time extrapolated to all patches and 24 layers")


def cpu_baseline(wl, seed) -> dict:
    s = OracleSample(wl, seed, frac=4)
    s.prepare()
    t_rows = s.step()
    return {"value": s.patches_per_s(t_rows, 24), "unit": "patches/s", "cores": blas_threads(), "kind": "oracle",
            "sample": s.describe()}


def run_reference(args, wl):
    world, rank, _ = int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")), 0
    if rank != 0:
        return
    s = OracleSample(wl, args.seed, frac=16)
    s.prepare()
    for _ in range(args.warmup):
        s.step()
    t0 = time.perf_counter()
    per = [s.step() for _ in range(args.steps)]
    wall = time.perf_counter() - t0
    value = s.patches_per_s(float(np.mean(per)), 24)
    cfg_out = workload_config(wl, s.sizes, world)
    line = {"metric": METRIC, "value": value, "unit": "patches/s", "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": 1000.0 * wall / max(1, args.steps), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
            "config": cfg_out,
            "cpu_baseline": {"value": value, "unit": "patches/s", "cores": blas_threads(), "kind": "oracle",
                             "sample": s.describe() + "; each step = one 1/16 row slice of the block"},
            "e2e": {"value": value, "unit": "patches/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------
# Our arm
# ---------------------------------------------------------------------------

def source_hash(*names) -> str:
    h = hashlib.sha1()
    for n in names:
        with open(os.path.join(ROOT, "vision_language_model_b200", "csrc", n), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:12]


def ncu_traffic(kernel: str) -> float | None:
    """DRAM bytes per launch from the committed ncu summary, if it was taken
    on the current source of that kernel."""
    path = os.path.join(ROOT, "profiles", "traffic_per_launch.json")
    if not os.path.exists(path):
        return None
    with open(path) as fh:
        table = json.load(fh)
    ent = table.get(kernel)
    if not ent or ent.get("bytes_per_launch") is None:
        return None
    if ent.get("source_hash") != source_hash(*ent.get("sources", [])):
        return None  # the kernel changed since the counters were taken
    return float(ent["bytes_per_launch"])


KERNEL_SOURCES = {"attention": ["attention_tc.cu", "exp2_poly.cuh", "common.cuh", "kernels.cuh"],
                  "gemm": ["gemm_tcgen05.cu", "common.cuh", "kernels.cuh"],
                  "resize": ["frontend.cu", "common.cuh", "kernels.cuh"]}


def exp_unit_line(attn_flops_per_launch: float, ms_per_launch: float, clk, sms: int) -> dict:
    """Attention's other bound: one exponential per score (4 * 64 FLOPs per score at
    head_dim 64), 7 of every 8 on the MUFU pipe (the kernel computes one score pair
    in eight with an FMA-pipe polynomial), against 16 MUFU ex2 per SM per clock (the
    pipe's issue rate on sm_100, 15.9 measured) x the SM count x the median SM clock
    sampled during the timed region."""
    scores = attn_flops_per_launch / (4 * 64)
    per_s = scores / (ms_per_launch / 1000.0)
    mhz = (clk or {}).get("sm_mhz")
    peak = 16 * sms * mhz * 1e6 if mhz else None
    mufu = per_s * 7 / 8
    return {"scores_per_s": per_s, "mufu_ex2_per_s": mufu, "peak_mufu_ex2_per_s": peak,
            "frac": mufu / peak if peak else None, "clock_mhz": mhz}


def gemm_shapes(args) -> None:
    """Per-shape GEMM throughput of the tower's four GEMMs at M = 12,100 rows,
    CUDA events around 20 back-to-back launches after 3 warm-ups."""
    from vision_language_model_b200 import vlm

    def timeit(fn, n=20):
        for _ in range(3):
            fn()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        for _ in range(n):
            fn()
        b.record()
        torch.cuda.synchronize()
        return a.elapsed_time(b) / n

    M = 12100
    g = torch.Generator(device="cuda")
    g.manual_seed(args.seed)
    pos = torch.zeros(M, dtype=torch.int32, device="cuda")
    rope = vlm.rope_table(1e4, 64, 128)
    st = vlm.new_status()
    shapes = [("gate/up", 8192, 1024, vlm.EPI_SWIGLU), ("qkv", 3072, 1024, vlm.EPI_ROPE),
              ("o", 1024, 1024, vlm.EPI_RESID), ("down", 1024, 4096, vlm.EPI_RESID)]
    for name, N, K, epi in shapes:
        fl = 2.0 * M * N * K
        kw = dict(pos=pos, rope=rope, rope_cols=2048) if epi == vlm.EPI_ROPE else {}
        for dt in ("bf16", "e4m3"):
            if dt == "bf16":
                a = (torch.randn((M, K), device="cuda", generator=g)).to(torch.bfloat16)
                b = (torch.randn((N, K), device="cuda", generator=g) * 0.02).to(torch.bfloat16)
            else:
                a = (torch.randn((M, K), device="cuda", generator=g) * 20).to(torch.float8_e4m3fn)
                b = (torch.randn((N, K), device="cuda", generator=g) * 20).to(torch.float8_e4m3fn)
                cs = torch.full((N,), 1e-3, device="cuda")
            if epi == vlm.EPI_RESID:
                c = torch.zeros((M, N), dtype=torch.float32, device="cuda")
            elif epi == vlm.EPI_SWIGLU:
                c = torch.empty((M, N // 2), dtype=torch.bfloat16 if dt == "bf16" else torch.uint8, device="cuda")
            else:
                c = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
            plain = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
            if dt == "bf16":
                kw16 = dict(pos=pos, rope_table=rope, rope_cols=2048) if epi == vlm.EPI_ROPE else {}
                fused = timeit(lambda: vlm.gemm(epi, a, b, c, status=st, **kw16))
                store = timeit(lambda: vlm.gemm(vlm.EPI_BF16, a, b, plain, status=st))
                lib_ms = timeit(lambda: torch.matmul(a, b.t()))
                lib = "torch.matmul (cuBLAS)"
            else:
                au, bu = a.view(torch.uint8), b.view(torch.uint8)
                fused = timeit(lambda: vlm.gemm_fp8(epi, au, bu, cs, c, out_scale=28.0, status=st, **kw))
                store = timeit(lambda: vlm.gemm_fp8(vlm.EPI_BF16, au, bu, cs, plain, status=st))
                one = torch.ones((), device="cuda")
                lib_ms = timeit(lambda: torch._scaled_mm(a, b.t(), scale_a=one, scale_b=one, out_dtype=torch.bfloat16))
                lib = "torch._scaled_mm (cuBLASLt)"
            print(json.dumps({"gemm": name, "dtype": dt, "M": M, "N": N, "K": K, "epilogue": epi,
                              "fused_ms": fused, "fused_tflops": fl / fused / 1e9,
                              "plain_store_ms": store, "plain_store_tflops": fl / store / 1e9,
                              "library": lib, "library_ms": lib_ms, "library_tflops": fl / lib_ms / 1e9}), flush=True)
        # NVFP4: bf16 activations quantised with a static global scale, weights with their own
        x = torch.randn((M, K), device="cuda", generator=g).to(torch.bfloat16)
        w = (torch.randn((N, K), device="cuda", generator=g) * 0.02).to(torch.bfloat16)
        ga = torch.full((1,), 12.0 / 2688.0, device="cuda")
        gw = vlm.amax_scale(w)
        qa, sfa = vlm.quant_nvfp4(x, ga)
        qw, sfw = vlm.quant_nvfp4(w, gw)
        quant = timeit(lambda: vlm.quant_nvfp4(x, ga, q=qa, sf=sfa))
        plain = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
        store = timeit(lambda: vlm.gemm_nvfp4(vlm.EPI_BF16, (qa, sfa, ga), (qw, sfw, gw), plain, status=st))
        if epi == vlm.EPI_RESID:
            c = torch.zeros((M, N), dtype=torch.float32, device="cuda")
            fused = timeit(lambda: vlm.gemm_nvfp4(vlm.EPI_RESID, (qa, sfa, ga), (qw, sfw, gw), c, status=st))
        elif epi == vlm.EPI_SWIGLU:
            hq = torch.empty((M, N // 4), dtype=torch.uint8, device="cuda")
            hsf = torch.zeros(vlm.nvfp4_sf_bytes(M, N // 2), dtype=torch.uint8, device="cuda")
            fused = timeit(lambda: vlm.gemm_nvfp4_swiglu((qa, sfa, ga), (qw, sfw, gw), 16.0 / 2688.0, q=hq, sf=hsf,
                                                         status=st))
        else:
            fused = timeit(lambda: vlm.gemm_nvfp4_rope((qa, sfa, ga), (qw, sfw, gw), plain, pos, rope, 2048, status=st))
        lib, lib_ms = "torch._scaled_mm (cuBLASLt, NVFP4)", None
        try:
            fa, fw = qa.view(torch.float4_e2m1fn_x2), qw.view(torch.float4_e2m1fn_x2)
            sa8, sw8 = sfa.view(torch.float8_e4m3fn), sfw.view(torch.float8_e4m3fn)
            lib_ms = timeit(lambda: torch._scaled_mm(fa, fw.t(), scale_a=sa8, scale_b=sw8, out_dtype=torch.bfloat16))
        except Exception as e:  # the library call is a comparison only
            lib = f"torch._scaled_mm NVFP4 unavailable: {type(e).__name__}: {str(e)[:120]}"
        print(json.dumps({"gemm": name, "dtype": "nvfp4", "M": M, "N": N, "K": K, "epilogue": epi,
                          "fused_ms": fused, "fused_tflops": fl / fused / 1e9 if fused else None,
                          "plain_store_ms": store, "plain_store_tflops": fl / store / 1e9,
                          "quantise_activations_ms": quant, "library": lib, "library_ms": lib_ms,
                          "library_tflops": fl / lib_ms / 1e9 if lib_ms else None}), flush=True)


def side_stream_overlap(pipe, pix, ids, text, cfg, scatter_ws, dev, steps: int) -> dict:
    """The image path on a side stream while another stream runs a decode-like
    loop (bf16 GEMVs [8, 5120] x [5120, 5120]^T over 48 distinct weight
    matrices, 2.5 GB read per pass: memory-bound, like a decoder step). Times
    each alone, then both together with the decode loop on a default-priority
    and on a high-priority stream; CUDA events on the launching streams."""
    from vision_language_model_b200 import vlm

    main = torch.cuda.current_stream(dev)
    w = torch.empty((48, 5120, 5120), dtype=torch.bfloat16, device=dev).normal_(0, 0.02)
    x = torch.empty((8, 5120), dtype=torch.bfloat16, device=dev).normal_()
    y = torch.empty((8, 5120), dtype=torch.bfloat16, device=dev)

    def decode_pass():
        for i in range(48):
            torch.matmul(x, w[i].t(), out=y)

    side = vlm.EncoderSideStream(pipe)

    def encode_request():
        side.submit(pix)
        side.scatter(ids, text, workspace=scatter_ws)

    def time_it(fn, reps):
        for _ in range(2):
            fn()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(main)
        for _ in range(reps):
            fn()
        b.record(main)
        torch.cuda.synchronize()
        return a.elapsed_time(b) / reps

    enc_ms = time_it(encode_request, steps)
    enc_full_ms = enc_ms
    if cfg.sm_budget:  # the same request with every SM, for the comparison against serial full-GPU runs
        budget, cfg.sm_budget = cfg.sm_budget, 0
        enc_full_ms = time_it(encode_request, steps)
        cfg.sm_budget = budget
    dec_ms = time_it(decode_pass, 20)
    n_dec = max(1, round(enc_ms / dec_ms))

    def concurrent(priority):
        dstream = torch.cuda.Stream(device=dev, priority=priority)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        d0, d1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        totals, decs = [], []
        for rep in range(steps + 2):
            torch.cuda.synchronize()
            a.record(main)
            side.submit(pix)
            dstream.wait_stream(main)
            with torch.cuda.stream(dstream):
                d0.record(dstream)
                for _ in range(n_dec):
                    decode_pass()
                d1.record(dstream)
            main.wait_stream(dstream)
            side.scatter(ids, text, workspace=scatter_ws)
            b.record(main)
            torch.cuda.synchronize()
            if rep >= 2:
                totals.append(a.elapsed_time(b))
                decs.append(d0.elapsed_time(d1) / n_dec)
        return sum(totals) / len(totals), sum(decs) / len(decs)

    both_ms, dec_conc = concurrent(0)
    both_hi_ms, dec_conc_hi = concurrent(-1)
    serial = enc_ms + n_dec * dec_ms
    del w
    return {"encode_ms": enc_ms, "decode_pass_ms": dec_ms, "decode_passes": n_dec, "serial_ms": serial,
            "overlapped_ms": both_ms, "decode_pass_ms_during_encode": dec_conc,
            "overlapped_ms_decode_high_priority": both_hi_ms, "decode_pass_ms_during_encode_high_priority": dec_conc_hi,
            "hidden_frac": (serial - both_ms) / min(enc_ms, n_dec * dec_ms),
            "encoder_sm_budget": cfg.sm_budget or None, "encode_ms_every_sm": enc_full_ms,
            "gain_vs_serial_every_sm": 1.0 - min(both_ms, both_hi_ms) / (enc_full_ms + n_dec * dec_ms),
            "note": "encoder + scatter of one request on a side stream, decode-like GEMV passes on another stream; "
                    "hidden_frac = time saved against running them one after the other / the shorter of the two; "
                    "gain_vs_serial_every_sm = time saved against running them one after the other with the "
                    "encoder on every SM"}


def run_ours(args, wl):
    from vision_language_model_b200 import synth, vlm

    world, rank, local = dist_setup()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    sizes = sizes_of(wl, args.seed)
    cfg = vlm.preset(wl["preset"], sm_budget=args.sm_budget)
    fl = flops_breakdown(cfg, sizes)
    T, Tm = fl["T"], fl["Tm"]

    tw = {k: v.to(dev) for k, v in synth.tower_weights(args.seed, cfg.layers, cfg.width, cfg.mlp, cfg.patch).items()}
    pw = {k: v.to(dev) for k, v in synth.projector_weights(args.seed, cfg.width, cfg.merge, cfg.proj_out).items()}
    pipe = vlm.ImagePipeline(cfg, tw, pw, sizes, device=dev,
                             fp8_act_scales=synth.fp8_act_scales(cfg.layers) if wl.get("fp8") else None,
                             nvfp4_act_scales=synth.nvfp4_act_scales(cfg.layers) if wl.get("nvfp4") else None)
    del tw, pw
    photo = wl.get("photo")
    if photo:
        assert sizes == [vlm.resize_target(*photo, 1540, cfg.patch * cfg.merge)]
        pix_host = synth.photo_u8(args.seed + rank, "photo", *photo).reshape(-1).pin_memory()
        photo_dev = pix_host.to(dev)
        pix = torch.empty(sum(3 * h * w for h, w in sizes), dtype=torch.float32, device=dev)
    else:
        imgs = synth.images(args.seed + rank, sizes)
        pix_host = torch.cat([im.reshape(-1) for im in imgs]).pin_memory()
        pix = pix_host.to(dev)
    per_seq = [[] for _ in range(wl["n_seq"])]
    lens_m = [(h // cfg.patch) * (w // cfg.patch) // (cfg.merge * cfg.merge) for h, w in sizes]
    for i, n in enumerate(lens_m):
        per_seq[i % wl["n_seq"]].append(n)
    if photo:
        marker = 7
        ids_host = synth.prompt_with_markers(args.seed, wl["seq_len"] - sum(lens_m), len(lens_m), marker).pin_memory()
        marker_ids = ids_host.to(dev)
        ids = torch.empty(wl["seq_len"], dtype=torch.int64, device=dev)
        expand_ws = torch.empty(max(256, vlm.expand_placeholders_workspace_size(marker_ids.numel(), len(lens_m))),
                                dtype=torch.uint8, device=dev)
    else:
        ids_host = synth.text_sequences(args.seed, wl["n_seq"], wl["seq_len"], per_seq).reshape(-1).pin_memory()
        ids = ids_host.to(dev)
    text = synth.text_embeddings(args.seed, ids.numel(), cfg.proj_out).to(dev)
    scatter_ws = torch.empty(max(256, vlm.scatter_workspace_size(ids.numel())), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    fused = args.scatter == "fused"

    def step():
        if photo:
            vlm.preprocess(photo_dev, [photo], sizes, out=pix)
        if fused:
            if photo:
                vlm.expand_placeholders(marker_ids, marker, lens_m, cfg.image_token_id, out=ids, workspace=expand_ws,
                                        status=pipe.status)
            pipe.embed_into(pix, ids, text)
            return
        emb = pipe(pix)
        if photo:
            vlm.expand_placeholders(marker_ids, marker, lens_m, cfg.image_token_id, out=ids, workspace=expand_ws,
                                    status=pipe.status)
        vlm.scatter(ids, emb, text, cfg.image_token_id, workspace=scatter_ws, status=pipe.status)

    for _ in range(args.warmup):
        step()
    rc = vlm.status_sync(pipe.status)
    if rc != vlm.OK:
        raise RuntimeError(f"device status after warm-up: {vlm.status_string(rc)}")

    if args.profile_steps:
        for _ in range(args.profile_steps):
            step()
        torch.cuda.synchronize()
        return

    graph = vlm.GraphStep(step, warmup=0) if args.graph else None
    run_step = graph if graph is not None else step

    def timed(profile: bool) -> float:
        """Device milliseconds of args.steps steps, bracketed by barrier + synchronize."""
        vlm.profile_enable(profile)
        start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier(world)
        torch.cuda.synchronize()
        start.record(stream)
        for _ in range(args.steps):
            (step if profile else run_step)()
        stop.record(stream)
        torch.cuda.synchronize()
        barrier(world)
        return start.elapsed_time(stop)

    # ---- timed region: inputs resident in HBM, no instrumentation between launches ----
    clocks = ClockSampler(local)
    time.sleep(0.3)
    launches0 = vlm.launch_count()
    ms = timed(False)
    launches = vlm.launch_count() - launches0
    if graph is not None:  # replays launch the captured kernels without calling the library
        launches = graph.launches_per_replay * args.steps
    clk = clocks.stop()
    ms_max = max_over_ranks(world, ms)
    # ---- the same steps again with a CUDA event pair around every launch: per-kernel times ----
    ms_profiled = timed(True)
    n_gemm, ms_gemm = vlm.profile_query("gemm")
    n_attn, ms_attn = vlm.profile_query("attention")
    n_norm, ms_norm = vlm.profile_query("rmsnorm")
    n_resize, ms_resize = vlm.profile_query("resize")
    n_expand, ms_expand = vlm.profile_query("expand")
    n_im2col, ms_im2col = vlm.profile_query("im2col")
    n_merge, ms_merge = vlm.profile_query("merge")
    n_scatter, ms_scatter = vlm.profile_query("scatter")
    vlm.profile_enable(False)
    rc = vlm.status_sync(pipe.status)
    if rc != vlm.OK:
        raise RuntimeError(f"device status after timed steps: {vlm.status_string(rc)}")

    # ---- e2e: every step's inputs from pinned host memory, its result back to it; the copies of
    # step i+1's inputs and step i's result overlap step i+1's and i's compute (vlm.HostFedSteps) ----
    out_host = torch.empty(text.shape, dtype=text.dtype, pin_memory=True)

    def host_fed_step(inputs, result):
        pix_in, ids_in = inputs
        if photo:
            vlm.preprocess(pix_in, [photo], sizes, out=pix)
            if fused:
                vlm.expand_placeholders(ids_in, marker, lens_m, cfg.image_token_id, out=ids, workspace=expand_ws,
                                        status=pipe.status)
                pipe.embed_into(pix, ids, result)
                return
            emb = pipe(pix)
            vlm.expand_placeholders(ids_in, marker, lens_m, cfg.image_token_id, out=ids, workspace=expand_ws,
                                    status=pipe.status)
            vlm.scatter(ids, emb, result, cfg.image_token_id, workspace=scatter_ws, status=pipe.status)
        elif fused:
            pipe.embed_into(pix_in, ids_in, result)
        else:
            emb = pipe(pix_in)
            vlm.scatter(ids_in, emb, result, cfg.image_token_id, workspace=scatter_ws, status=pipe.status)

    fed = vlm.HostFedSteps(host_fed_step, [photo_dev if photo else pix, marker_ids if photo else ids], text)
    fed.run([pix_host, ids_host], out_host, 2)  # warm-up of the copy path
    barrier(world)
    torch.cuda.synchronize()
    e_start, e_stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e_start.record(stream)
    fed.run([pix_host, ids_host], out_host, args.steps)
    e_stop.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    e_ms = max_over_ranks(world, e_start.elapsed_time(e_stop))
    rc = vlm.status_sync(pipe.status)
    if rc != vlm.OK:
        raise RuntimeError(f"device status after the end-to-end steps: {vlm.status_string(rc)}")

    peaks = measured_peaks()
    value = job_throughput(T, world, args.steps, ms_max)
    # dominant kernel of the step
    if ms_attn >= ms_gemm:
        kern, achieved = "attention", fl["attn_per_launch"] / (ms_attn / n_attn / 1000.0) / 1e12
    else:
        kern, achieved = "gemm", fl["gemm"] * args.steps / (ms_gemm / 1000.0) / 1e12
    # the kernel is timed inside a loop of well under a second: the burst figure is its peak
    peak = peaks["bf16_tflops"]
    step_tflops = fl["total"] / (ms / args.steps / 1000.0) / 1e12
    wcfg = workload_config(wl, sizes, world)
    if args.sm_budget:
        wcfg["sm_budget"] = args.sm_budget
    assert (wcfg["patches"], wcfg["merged_tokens"], wcfg["text_tokens"]) == (T, Tm, int(ids.numel()))
    line = {
        "metric": METRIC, "value": value, "unit": "patches/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_max / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "e4m3+bf16" if wl.get("fp8") else "e2m1+bf16" if wl.get("nvfp4") else "bf16", "data": "synthetic",
        "config": wcfg,
        "roofline": {"kernel": kern, "bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                     "frac": achieved / peak, "peak_source": f"bf16_tflops, burst ({peaks['source']})",
                     "traffic": ncu_traffic(kern)},
        "step_tflops": step_tflops,
        "attention_exp_unit": exp_unit_line(fl["attn_per_launch"], ms_attn / n_attn, clk,
                                            torch.cuda.get_device_properties(dev).multi_processor_count),
        "step_frac_of_bf16_peak": {"measured_sustained": step_tflops / peak,
                                   "measured_burst": step_tflops / peaks["bf16_tflops"],
                                   "nominal_2250": step_tflops / 2250.0},
        "kernels_ms_per_step": {"gemm": ms_gemm / args.steps, "attention": ms_attn / args.steps,
                                "rmsnorm": ms_norm / args.steps, "patch_gather": ms_im2col / args.steps,
                                "merge_gather": ms_merge / args.steps, "scatter": ms_scatter / args.steps,
                                "step_with_events": ms_profiled / args.steps,
                                "note": "per-kernel CUDA events on the launch stream, in a second pass of the "
                                        "same steps"},
        "e2e": {"value": job_throughput(T, world, args.steps, e_ms), "unit": "patches/s",
                "h2d_bytes_per_step": int(pix_host.numel() * pix_host.element_size() + ids_host.numel() * 8),
                "d2h_bytes_per_step": int(out_host.numel() * out_host.element_size()),
                "note": "pinned host inputs in and the merged embedding sequence out every step; the copies run on "
                        "a copy stream, double-buffered, overlapping the neighbouring steps' compute"},
        "gpu_launches": int(launches),
        "clocks": clk,
    }
    if photo:
        # distinct source rows the vertical taps touch (half-pixel centres, clamped)
        (sh, sw), (oh, _) = photo, sizes[0]
        ys = np.clip((np.arange(oh) + 0.5) * (sh / oh) - 0.5, 0, sh - 1)
        rows_read = len(set(np.floor(ys).astype(int)) | set(np.minimum(np.floor(ys).astype(int) + 1, sh - 1)))
        src_bytes = rows_read * 3 * sw
        out_bytes = sum(12 * h * w for h, w in sizes)
        # the resize alone: 3 photo/output buffer pairs (174 MB, more than L2) in rotation,
        # 30 launches back to back between two events on the launch stream
        srcs = [photo_dev] + [synth.photo_u8(args.seed + 100 + k, "photo", *photo).reshape(-1).to(dev)
                              for k in range(2)]
        outs = [pix] + [torch.empty_like(pix) for _ in range(2)]
        for k in range(3):
            vlm.preprocess(srcs[k], [photo], sizes, out=outs[k])
        r_start, r_stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        r_start.record(stream)
        for k in range(30):
            vlm.preprocess(srcs[k % 3], [photo], sizes, out=outs[k % 3])
        r_stop.record(stream)
        torch.cuda.synchronize()
        r_ms = r_start.elapsed_time(r_stop) / 30
        resize_gbs = (src_bytes + out_bytes) / (r_ms / 1000.0) / 1e9
        line["front_end"] = {
            "resize": {"ms_per_launch": r_ms, "in_step_ms_per_launch": ms_resize / max(n_resize, 1),
                       "algorithmic_bytes": src_bytes + out_bytes, "achieved_gbs": resize_gbs,
                       "peak_gbs": peaks["hbm_gbs"], "frac": resize_gbs / peaks["hbm_gbs"],
                       "bytes_note": f"u8 source rows the taps touch ({rows_read} of {sh}) read once + fp32 CHW "
                                     "output written once; timed alone, 30 launches over 3 rotating buffer pairs "
                                     "larger than L2 together",
                       "traffic": ncu_traffic("resize")},
            "expand_ms_per_step": ms_expand / args.steps,
        }
    # memory-bound kernels: algorithmic bytes per step / their event-timed device time
    D_, p_ = cfg.width, cfg.patch
    kp_ = -(-3 * p_ * p_ // 64) * 64
    row_bytes = cfg.proj_out * 2
    # the norm's output per value: bf16, E4M3, or E2M1 codes plus one E4M3 scale per 16 values
    out_b, out_name = (1.0, "E4M3") if wl.get("fp8") else (0.5 + 1.0 / 16, "NVFP4") if wl.get("nvfp4") else (2.0, "bf16")
    mb = {
        "rmsnorm": (2 * cfg.layers * T * D_ * (4 + out_b) + T * D_ * 4, ms_norm,
                    f"per launch: fp32 row read + the {out_name} row written (+ the fp32 write-back of ln_pre once)"),
        "patch_gather": (T * (3 * p_ * p_ * 4 + kp_ * 2), ms_im2col, "fp32 pixels read + bf16 patch rows written"),
        "merge_gather": (2 * T * D_ * 2, ms_merge, "bf16 tower rows read + bf16 merged rows written"),
    }
    if not fused:
        mb["scatter"] = (2 * Tm * row_bytes + ids.numel() * 8, ms_scatter,
                         "image rows read + written into the text rows + ids read")
    line["memory_bound_kernels"] = {
        k: {"bytes_per_step": int(b), "ms_per_step": t / args.steps,
            "achieved_gbs": b / (t / args.steps / 1e3) / 1e9 if t > 0 else None,
            "frac_of_hbm": b / (t / args.steps / 1e3) / 1e9 / peaks["hbm_gbs"] if t > 0 else None, "bytes": note}
        for k, (b, t, note) in mb.items()}
    if fused:  # (config stays the workload's own keys, the same as the reference arm's)
        line["scatter_fused"] = {
            "positions_ms_per_step": ms_scatter / args.steps,
            "entry": "vlm_merge_project_scatter (the masked scatter fused into the projector's last linear)",
            "note": "the image rows go from the last projector GEMM's epilogue straight to their text rows (counted "
                    "with the GEMMs); what is left of the scatter is the kernel that finds the placeholders' rows "
                    "(one launch up to 4,096 ids; count, scan and positions kernels above that)"}
    if args.graph:
        line["config"]["launch"] = f"one CUDA graph per step ({graph.launches_per_replay} kernels)"
    if args.side_stream:
        line["side_stream"] = side_stream_overlap(pipe, pix, ids, text, cfg, scatter_ws, dev, args.steps)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(wl, args.seed)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def main():
    args = parse_args()
    wl = WORKLOADS[args.workload]
    if args.gemm_shapes:
        gemm_shapes(args)
        return
    if args.impl == "reference":
        run_reference(args, wl)
    else:
        run_ours(args, wl)


if __name__ == "__main__":
    main()
