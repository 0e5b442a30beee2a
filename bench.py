"""Benchmark of the π0.5 action-expert 10-step denoise loop (2-view: 512-token prefix KV
cache, chunk 63, batch 1, 18 layers) through the rtvla C ABI.

One step = one full 10-step denoise loop (one rtvla_sample_actions call) on inputs already
resident in HBM.  Prints one JSON line (rank 0).  Multi-GPU runs are independent replicas
(the method does not shard); the timed region is bracketed by a barrier and a device
synchronize, and the time is the max over ranks.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--batch B]
                  [--workload 2-view|1-view|3-view|e2e|stream|pi0|vision|pipeline] [--views V]

Other workloads print their own line: the e2e prefill + denoise, the pi0 variant, the image
encoder alone (vision) and full pi0 inference from camera views (pipeline).

--impl reference times the fp64 CPU oracle (plain numpy) on the host cores: each step is
one full 10-step loop of the same workload, after --warmup untimed loops.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "10-step denoise latency ms (2-view, chunk 63); achieved HBM GB/s vs roofline"
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=20)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", default="ours", choices=["ours", "reference"])
    p.add_argument("--batch", type=int, default=1)
    p.add_argument("--engine", type=int, default=0)
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--workload", default="2-view",
                   choices=["2-view", "1-view", "3-view", "e2e", "stream", "pi0", "vision", "pipeline"],
                   help="2-view (the headline line), 1-view, 3-view (with --batch), e2e: prefill of the "
                        "544-token prefix, then the denoise loop; stream: frames of e2e back to back, the "
                        "prefill of frame n+1 overlapping the denoise of frame n (layered engine); pi0: the "
                        "2-view workload on the pi0 suffix variant (state token, action-time MLP); vision: "
                        "the image encoder (27-layer SigLIP tower + projector) on --views views; pipeline: "
                        "full pi0 inference on --views views (image encoder, prefix pass over the image "
                        "tokens with an empty prompt, 10-step pi0 loop, chunk 63)")
    p.add_argument("--views", type=int, default=2, choices=[1, 2, 3])
    return p.parse_args()


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        d = json.load(open(path))
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), float(d.get("bf16_tflops_sustained", d["bf16_tflops"])), "measured"
    return FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS, 1400.0, "fallback"


def workload(batch, name="2-view"):
    from synth import workloads as WL
    if name == "1-view":
        return WL.workload(2)
    if name == "3-view":
        return WL.workload(4, batch=batch)
    if name in ("e2e", "stream"):
        return WL.workload(5)
    return WL.workload(3) if batch == 1 else WL.workload(4, batch=batch)


def workload_config(wl, world):
    """The `config` object of the JSON line: the workload only, the same on both arms."""
    c = {"workload": wl.name, "batch": wl.batch, "chunk": wl.chunk, "prefix": wl.prefix_cap,
         "valid_prefix": list(wl.valid_lens)[:4], "layers": wl.expert.n_layers,
         "steps_per_loop": wl.expert.n_steps, "parallelism": f"replicas{world}"}
    if wl.prefill is not None:
        c["prefill_layers"] = wl.prefill.n_layers
    return c


def prefill_algorithmic(wl):
    """Bytes and FLOPs of one prefill pass: every layer's weights read once; 2 * T * params plus
    the bidirectional attention over the valid prefix; the last layer computes K and V only."""
    s = wl.prefill
    D, F, H, hd = s.width, s.mlp_dim, s.n_q_heads, s.head_dim
    kvd = s.n_kv_heads * hd
    full = H * hd * D + 2 * kvd * D + D * H * hd + 2 * F * D + D * F
    kv_only = 2 * kvd * D
    T = sum(wl.valid_lens)
    flops = (s.n_layers - 1) * (2 * T * full + sum(4 * H * l * l * hd for l in wl.valid_lens)) + 2 * T * kv_only
    bytes_ = ((s.n_layers - 1) * full + kv_only) * 2 + s.n_layers * wl.batch * wl.prefix_cap * kvd * 2 * 2
    return bytes_, flops


def prefill_kernels(n_layers):
    """Kernels of one rtvla_prefill graph at the sizes benched here (the attention split into
    several key ranges, the gate/up GEMM with the GELU epilogue): the mask and embedding
    kernels; per layer RMSNorm, QKV GEMM and QKV post; per full layer (all but the last)
    attention, its split combine, O GEMM, RMSNorm, gate/up GEMM and down GEMM.  158 at 18
    layers, as the ncu launch list of the 544-token prefill counts."""
    return 2 + 3 * n_layers + 6 * (n_layers - 1)


def pi0_algorithmic(wl):
    """Bytes and FLOPs of one 10-step pi0 loop: the 18 layers' weights, the folded action-time
    MLP (fp32 W_fold [1024][32] and its output linear), state and action projections, the
    valid prefix KV, the norm tables and the suffix K/V of C + 1 tokens."""
    s = wl.expert
    L, D, F, H, hd, A, S = s.n_layers, s.width, s.mlp_dim, s.n_q_heads, s.head_dim, s.action_dim, s.n_steps
    per_layer_params = (H * hd + 2 * hd) * D + D * H * hd + 2 * F * D + D * F
    T = wl.chunk + 1
    M = wl.batch * T
    bf16_params = L * per_layer_params + D * D + 2 * D * A      # layers, action-time out, state + action out
    lv = sum(wl.valid_lens)
    bytes_step = (bf16_params * 2 + D * A * 4 + D * 4 + L * lv * hd * 2 * 2 + L * 2 * D * 4
                  + L * M * hd * 2 * 2 * 2)
    attn = sum(4 * H * T * (l + T) * hd for l in wl.valid_lens) * L
    flops_step = 2 * M * (L * per_layer_params + D * D) + 2 * wl.batch * wl.chunk * (D * A * 2) + attn
    return bytes_step * S, flops_step * S


def algorithmic(wl):
    """Bytes and FLOPs one 10-step loop must move / execute (weights streamed every step,
    valid prefix KV read, per-step tables, suffix K/V written and read)."""
    s = wl.expert
    L, D, F, H, hd, A, S = s.n_layers, s.width, s.mlp_dim, s.n_q_heads, s.head_dim, s.action_dim, s.n_steps
    per_layer_params = (H * hd + 2 * hd) * D + D * H * hd + 2 * F * D + D * F
    params = L * per_layer_params + 2 * D * A
    M = wl.batch * wl.chunk
    lv = sum(wl.valid_lens)
    w_bytes = params * 2
    kv_bytes = L * lv * hd * 2 * 2
    table_bytes = L * (4 * D + (H * hd + 2 * hd) + 2 * F) * 4
    suffix_bytes = L * M * hd * 2 * 2 * 2
    bytes_step = w_bytes + kv_bytes + table_bytes + suffix_bytes
    attn_flops = sum(4 * H * wl.chunk * (l + wl.chunk) * hd for l in wl.valid_lens) * L
    flops_step = 2 * M * params + attn_flops
    return bytes_step * S, flops_step * S, w_bytes * S


def vision_algorithmic(vcfg, n_img):
    """Bytes and FLOPs of one encode of n_img images: every weight matrix read once (bf16), the
    images read (f32) and the embeddings written (bf16); 2 * tokens * MACs of the patch
    convolution, the 27 layers' linears and the projector, plus 4 * heads * 256^2 * 72 of
    attention per image and layer."""
    W, Fv, L, T = vcfg.width, vcfg.mlp_dim, vcfg.n_layers, vcfg.tokens
    patch = W * vcfg.channels * vcfg.patch ** 2
    layer = 4 * W * W + 2 * W * Fv
    proj = vcfg.out_width * W
    tok = n_img * T
    flops = 2 * tok * (patch + L * layer + proj) + L * n_img * 4 * vcfg.n_heads * T * T * vcfg.head_dim
    bytes_ = (patch + L * layer + proj) * 2 + n_img * vcfg.channels * vcfg.image ** 2 * 4 + tok * vcfg.out_width * 2
    return bytes_, flops


def vision_config(vcfg, views, world):
    """The `config` object of the image-encoder line, the same on both arms."""
    return {"workload": f"SigLIP-So400m/14 shape, {views} x 224x224 views -> {views * vcfg.tokens} prefix embeddings",
            "layers": vcfg.n_layers, "width": vcfg.width, "mlp": vcfg.mlp_dim, "heads": vcfg.n_heads,
            "images": views, "tokens": views * vcfg.tokens, "parallelism": f"replicas{world}"}


def vision_metric(views):
    return f"image encoder latency ms ({views}-view, 27-layer SigLIP tower + projector)"


def reduce_max(vals, device):
    """Each value's maximum over the ranks of the current process group (a replica job takes
    as long as its slowest rank); the values themselves without a group or with one rank."""
    import torch
    import torch.distributed as dist
    if not dist.is_available() or not dist.is_initialized() or dist.get_world_size() == 1:
        return [float(v) for v in vals]
    t = torch.tensor([float(v) for v in vals], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.tolist()]


class Clocks:
    """nvidia-smi sampling of SM clocks and throttle reasons during the timed region."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.Q}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *a):
        self.rows = []
        if self.proc is None:
            return
        time.sleep(0.25)
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        for line in out.strip().splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) >= 9:
                self.rows.append(f)

    def summary(self):
        if not getattr(self, "rows", None):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        sm = [float(r[1]) for r in self.rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in self.rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in self.rows for i in range(4) if r[5 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(self.rows)}


KERNEL_SOURCES = ("csrc/persistent.cu", "csrc/persistent.h", "csrc/common.cuh", "csrc/rtvla_api.cu")


def strip_comments(src):
    """C/C++ source without comments and with whitespace collapsed: what the compiler sees."""
    import re
    out, i, n = [], 0, len(src)
    while i < n:
        if src.startswith("//", i):
            j = src.find("\n", i)
            i = n if j < 0 else j
        elif src.startswith("/*", i):
            j = src.find("*/", i + 2)
            i = n if j < 0 else j + 2
        elif src[i] == '"':  # string literal (the asm templates), copied as is
            j = i + 1
            while j < n and src[j] != '"':
                j += 2 if src[j] == "\\" else 1
            out.append(src[i:j + 1])
            i = j + 1
        else:
            out.append(src[i])
            i += 1
    return re.sub(r"\s+", " ", "".join(out)).strip()


def kernel_source_hash():
    """sha256 of the persistent kernel's sources with comments and whitespace removed, so a
    recorded capture stays valid across comment edits and is invalidated by any code change."""
    import hashlib
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES:
        with open(os.path.join(ROOT, "flow_matching_action_expert_b200", rel), encoding="utf-8") as f:
            h.update(strip_comments(f.read()).encode())
        h.update(b"\0")
    return h.hexdigest()


def measured_traffic(workload_name, engine):
    """DRAM bytes (read + write) per launch of the persistent kernel, from the committed ncu
    summary of this workload.  None unless the summary's source hash equals the hash of the
    sources now, i.e. the kernel has not changed since the counters were taken."""
    if engine != "persistent":
        return None
    import re
    slug = re.sub(r"[^0-9A-Za-z]+", "_", workload_name)
    path = os.path.join(ROOT, "profiles", f"k_persistent_{slug}.md")
    if not os.path.exists(path):
        return None
    fields = {}
    for line in open(path):
        if line.startswith("- ") and ": " in line:
            k, v = line[2:].split(": ", 1)
            fields[k.strip().strip("`")] = v.strip().strip("`")
    if fields.get("source_sha256") != kernel_source_hash():
        return None
    try:
        return int(fields["dram_bytes_per_launch"])
    except (KeyError, ValueError):
        return None


def cpu_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads") for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count()


class OracleLoop:
    """The fp64 oracle's full S-step denoise loop on the workload (weights widened once, not
    timed)."""

    def __init__(self, wl):
        from oracle import model as O
        from synth import gen
        from synth import workloads as WL
        self.O, self.wl = O, wl
        self.W = O.Weights(WL.as_f32(WL.expert_weights(wl.expert)))
        kb, vb, self.valid = WL.kv_cache(wl)
        self.kf, self.vf = gen.bf16_to_f32(kb), gen.bf16_to_f32(vb)
        self.noise = WL.noise(wl)
        for name in list(self.W._d):
            self.W[name]

    def run(self):
        self.O.sample_actions(self.W, self.wl.expert, self.noise, self.kf, self.vf, self.valid)

    def time_ms(self, n):
        times = []
        for _ in range(n):
            t0 = time.perf_counter()
            self.run()
            times.append((time.perf_counter() - t0) * 1e3)
        return times


def run_reference(args, rank):
    if rank != 0:
        return
    if args.workload == "vision":
        return run_reference_vision(args)
    if args.workload == "pipeline":
        print(json.dumps({"impl": "reference", "unavailable": "one step of the oracle chain (tower, 18-layer prefix "
                          "pass, 10-step loop) takes minutes on the host cores; the vision and denoise workloads "
                          "time its parts"}), flush=True)
        return
    wl = workload(args.batch, args.workload if args.workload not in ("e2e", "stream") else "2-view")
    loop = OracleLoop(wl)
    for _ in range(args.warmup):
        loop.run()
    times = loop.time_ms(max(1, args.steps))
    per_loop = statistics.mean(times)
    line = {
        "impl": "reference", "metric": METRIC, "value": round(per_loop, 3), "unit": "ms",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(per_loop, 3),
        "higher_is_better": False, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded N(0,0.02) bf16 weights, N(0,1) KV and noise)",
        "config": workload_config(wl, args.gpus),
        "engine": "oracle (fp64 numpy, host cores)",
        "cpu_baseline": {"value": round(per_loop, 3), "unit": "ms", "cores": cpu_threads(), "kind": "oracle",
                         "sample": f"{len(times)} full {wl.expert.n_steps}-step loops of the workload "
                                   f"(fp64 oracle), after {args.warmup} untimed"},
        "e2e": {"value": round(per_loop, 3), "unit": "ms", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def run_reference_vision(args):
    """The fp64 image-encoder oracle on the host cores: each step encodes one of the --views
    images (a bounded sample of the workload) and counts as views x its time."""
    from oracle import vision as OV
    from synth import workloads as WL
    vcfg = WL.VisionShape()
    V = args.views
    W = WL.as_f32(WL.vision_weights(vcfg, tag="vision"))
    imgs = WL.images(vcfg, V)
    for i in range(args.warmup):
        OV.encode_image(imgs[i % V], W, vcfg)
    times = []
    for i in range(max(1, args.steps)):
        t0 = time.perf_counter()
        OV.encode_image(imgs[i % V], W, vcfg)
        times.append((time.perf_counter() - t0) * 1e3 * V)
    per = statistics.mean(times)
    line = {
        "impl": "reference", "metric": vision_metric(V), "value": round(per, 1), "unit": "ms",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(per, 1),
        "higher_is_better": False, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded N(0,0.02) bf16 weights, uniform [-1,1) f32 pixels)",
        "config": vision_config(vcfg, V, args.gpus),
        "engine": "oracle (fp64 numpy, host cores)",
        "cpu_baseline": {"value": round(per, 1), "unit": "ms", "cores": cpu_threads(), "kind": "oracle",
                         "sample": f"each step one of the {V} images through the fp64 tower, times {V}, after "
                                   f"{args.warmup} untimed"},
        "e2e": {"value": round(per, 1), "unit": "ms", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def run_ours(args, rank, world, local_rank):
    import torch

    import flow_matching_action_expert_b200 as R
    from synth import workloads as WL

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    if args.workload == "vision":
        return run_vision(args, rank, world, local_rank)
    if args.workload == "pipeline":
        return run_pipeline(args, rank, world, local_rank)
    wl = workload(args.batch, args.workload)
    if args.workload == "e2e":
        return run_e2e(args, rank, world, local_rank, wl)
    if args.workload == "stream":
        return run_stream(args, rank, world, local_rank, wl)
    if args.workload == "pi0":
        return run_pi0(args, rank, world, local_rank, wl)
    bits = WL.expert_weights(wl.expert)
    dw = {k: torch.from_numpy(v.view(np.int16)).view(torch.bfloat16).to(dev) for k, v in bits.items()}
    cfg = R.make_config(n_layers=wl.expert.n_layers, chunk=wl.chunk, max_prefix=wl.prefix_cap,
                        max_batch=wl.batch, engine=args.engine)
    ctx = R.rtvla_create(dw, cfg)
    del dw
    kb, vb, valid = WL.kv_cache(wl)
    noise_np = WL.noise(wl)
    k = torch.from_numpy(kb.view(np.int16)).view(torch.bfloat16).to(dev)
    v = torch.from_numpy(vb.view(np.int16)).view(torch.bfloat16).to(dev)
    vl = torch.from_numpy(valid).to(dev)
    noise = torch.from_numpy(noise_np).to(dev)
    out = torch.empty_like(noise)
    kv = R.make_kv(k, v, vl, wl.batch, wl.prefix_cap)
    stream = torch.cuda.current_stream(dev)
    flush = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)

    def call():
        R.rtvla_sample_actions(ctx, noise, kv, out, stream)

    for _ in range(max(3, args.warmup)):
        call()
    torch.cuda.synchronize()
    st = R.rtvla_sync_status(ctx, stream)
    if st != 0:
        raise RuntimeError(f"device status {R.STATUS[st]}")

    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    with Clocks(local_rank) as clk:
        for i in range(args.steps):
            flush.fill_(float(i))              # L2 flush (256 MiB write) outside the timed events
            starts[i].record(stream)
            call()
            ends[i].record(stream)
        torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    per = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    ms = reduce_max([statistics.mean(per)], dev)[0]
    st = R.rtvla_sync_status(ctx, stream)
    if st != 0:
        raise RuntimeError(f"device status {R.STATUS[st]}")
    kernels = R.rtvla_kernels_per_call(ctx, wl.batch)

    # end to end through the host-buffer entry point (pinned noise + KV in, actions out)
    hk = torch.from_numpy(kb.view(np.int16)).pin_memory()
    hv = torch.from_numpy(vb.view(np.int16)).pin_memory()
    hl = torch.from_numpy(valid).pin_memory()
    hn = torch.from_numpy(noise_np).pin_memory()
    ho = torch.empty_like(hn).pin_memory()
    for _ in range(2):
        R.rtvla_sample_actions_host(ctx, hn, hk, hv, hl, wl.batch, wl.prefix_cap, ho, stream)
    e2e = []
    for i in range(args.steps):
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        R.rtvla_sample_actions_host(ctx, hn, hk, hv, hl, wl.batch, wl.prefix_cap, ho, stream)
        e1.record(stream)
        e1.synchronize()
        e2e.append(e0.elapsed_time(e1))
    e2e_ms = reduce_max([statistics.mean(e2e)], dev)[0]
    h2d = hn.numel() * 4 + hk.numel() * 2 + hv.numel() * 2 + hl.numel() * 4
    d2h = ho.numel() * 4
    R.rtvla_destroy(ctx)

    if rank != 0:
        return
    hbm, bf16_pk, bf16_sus, src = peaks()
    bytes_loop, flops_loop, w_bytes = algorithmic(wl)
    achieved_gbs = bytes_loop / (ms * 1e-3) / 1e9
    achieved_tf = flops_loop / (ms * 1e-3) / 1e12
    t_mem = bytes_loop / (hbm * 1e9)
    t_tc = flops_loop / (bf16_sus * 1e12)
    bound = "hbm" if t_mem >= t_tc else "tensor"
    engine = "persistent" if kernels == 1 else "layered"   # the engine the call actually ran
    line = {
        "metric": METRIC, "value": round(ms, 4), "unit": "ms", "n_gpus": world, "steps": args.steps,
        "warmup": max(3, args.warmup), "ms_per_step": round(ms, 4), "higher_is_better": False,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded N(0,0.02) bf16 weights, N(0,1) KV and noise)",
        "config": workload_config(wl, world),
        "engine": engine,
        "l2": "flushed by a 256 MiB write between timed loops; weights (623 MB) exceed L2",
        "hbm_gbs_achieved": round(achieved_gbs, 1),
        "chunks_per_s": round(world * wl.batch / (ms * 1e-3), 2),
        "latency_ms": {"p10": round(float(np.percentile(per, 10)), 4), "p50": round(float(np.median(per)), 4),
                       "p90": round(float(np.percentile(per, 90)), 4)},
        "roofline": {"bound": bound,
                     "kernel": ("k_persistent (one launch = one call)" if engine == "persistent"
                                else "rtvla_sample_actions (layered engine, one graph replay)"),
                     "achieved": round(achieved_gbs if bound == "hbm" else achieved_tf, 1),
                     "peak": hbm if bound == "hbm" else bf16_sus,
                     "unit": "GB/s" if bound == "hbm" else "TFLOP/s",
                     "frac": round((achieved_gbs / hbm) if bound == "hbm" else (achieved_tf / bf16_sus), 4),
                     "traffic": measured_traffic(wl.name, engine), "peak_source": src,
                     "algorithmic_bytes_per_launch": int(bytes_loop), "algorithmic_flops_per_launch": int(flops_loop),
                     "roofline_ms": round(max(t_mem, t_tc) * 1e3, 4)},
        "e2e": {"value": round(e2e_ms, 4), "unit": "ms", "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h)},
        "gpu_launches": int(kernels * args.steps) if kernels > 0 else None,
        "kernels_per_step": kernels,
        "clocks": clk.summary(),
    }
    if world == 1 and not args.no_cpu_baseline:
        times = OracleLoop(wl).time_ms(3)
        line["cpu_baseline"] = {"value": round(statistics.mean(times), 1), "unit": "ms", "cores": cpu_threads(),
                                "kind": "oracle",
                                "sample": f"3 full {wl.expert.n_steps}-step loops of the same workload (fp64 oracle)"}
    print(json.dumps(line), flush=True)


def run_pi0(args, rank, world, local_rank, wl):
    """The 2-view workload on the pi0 suffix variant: the suffix is [state token ; 63 action
    tokens], the action tokens come from the folded action-time MLP, plain RMSNorm, ungated
    residuals (the persistent kernel at batch 1 unless --engine 1).  e2e: pinned host noise,
    state and cache copied in, the call, the actions copied out, all inside the timed region."""
    import torch

    import flow_matching_action_expert_b200 as R
    from synth import workloads as WL

    dev = torch.device("cuda", local_rank)
    bits = WL.pi0_expert_weights(wl.expert, bias_std=0.02)
    dw = {k: torch.from_numpy(v.view(np.int16)).view(torch.bfloat16).to(dev) for k, v in bits.items()}
    cfg = R.make_config(n_layers=wl.expert.n_layers, chunk=wl.chunk, max_prefix=wl.prefix_cap,
                        max_batch=wl.batch, engine=args.engine, variant=R.VARIANT_PI0)
    ctx = R.rtvla_create(dw, cfg)
    del dw
    kb, vb, valid = WL.kv_cache(wl)
    noise_np, state_np = WL.noise(wl), WL.state(wl)
    k = torch.from_numpy(kb.view(np.int16)).view(torch.bfloat16).to(dev)
    v = torch.from_numpy(vb.view(np.int16)).view(torch.bfloat16).to(dev)
    vl = torch.from_numpy(valid).to(dev)
    noise = torch.from_numpy(noise_np).to(dev)
    state = torch.from_numpy(state_np).to(dev)
    out = torch.empty_like(noise)
    kv = R.make_kv(k, v, vl, wl.batch, wl.prefix_cap)
    stream = torch.cuda.current_stream(dev)
    flush = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)

    def call():
        R.rtvla_sample_actions_pi0(ctx, noise, state, kv, out, stream)

    for _ in range(max(3, args.warmup)):
        call()
    torch.cuda.synchronize()
    st = R.rtvla_sync_status(ctx, stream)
    if st != 0:
        raise RuntimeError(f"device status {R.STATUS[st]}")
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    with Clocks(local_rank) as clk:
        for i in range(args.steps):
            flush.fill_(float(i))
            ev[i][0].record(stream)
            call()
            ev[i][1].record(stream)
        torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    per = [a.elapsed_time(b) for a, b in ev]
    ms = reduce_max([statistics.mean(per)], dev)[0]
    kernels = R.rtvla_kernels_per_call(ctx, wl.batch)
    # end to end: pinned host inputs in, the call, the actions out
    hk = torch.from_numpy(kb.view(np.int16)).view(torch.bfloat16).pin_memory()
    hv = torch.from_numpy(vb.view(np.int16)).view(torch.bfloat16).pin_memory()
    hl, hn = torch.from_numpy(valid).pin_memory(), torch.from_numpy(noise_np).pin_memory()
    hs, ho = torch.from_numpy(state_np).pin_memory(), torch.empty_like(hn).pin_memory()
    e2e = []
    for i in range(args.steps + 2):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for d, h in ((noise, hn), (state, hs), (k, hk), (v, hv), (vl, hl)):
            d.copy_(h, non_blocking=True)
        call()
        ho.copy_(out, non_blocking=True)
        e1.record(stream)
        e1.synchronize()
        if i >= 2:
            e2e.append(e0.elapsed_time(e1))
    e2e_ms = reduce_max([statistics.mean(e2e)], dev)[0]
    st = R.rtvla_sync_status(ctx, stream)
    R.rtvla_destroy(ctx)
    if st != 0:
        raise RuntimeError(f"device status {R.STATUS[st]}")
    if rank != 0:
        return
    hbm, bf16_pk, bf16_sus, src = peaks()
    b_loop, f_loop = pi0_algorithmic(wl)
    t_mem, t_tc = b_loop / (hbm * 1e9), f_loop / (bf16_sus * 1e12)
    gbs = b_loop / (ms * 1e-3) / 1e9
    line = {
        "metric": "pi0 10-step denoise latency ms (2-view, chunk 63 + state token)", "value": round(ms, 4),
        "unit": "ms", "n_gpus": world, "steps": args.steps, "warmup": max(3, args.warmup),
        "ms_per_step": round(ms, 4), "higher_is_better": False, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16", "data": "synthetic (seeded N(0,0.02) bf16 weights and biases, N(0,1) KV, noise, state)",
        "config": dict(workload_config(wl, world), workload="pi0 " + wl.name, suffix_tokens=wl.chunk + 1),
        "engine": "persistent" if kernels == 1 else "layered",
        "l2": "flushed by a 256 MiB write between timed loops",
        "roofline": {"bound": "hbm" if t_mem >= t_tc else "tensor",
                     "kernel": ("k_persistent (one launch = one call)" if kernels == 1
                                else "rtvla_sample_actions_pi0 (one graph replay)"),
                     "achieved": round(gbs, 1), "peak": hbm, "unit": "GB/s", "frac": round(gbs / hbm, 4),
                     "traffic": None, "peak_source": src, "algorithmic_bytes_per_launch": int(b_loop),
                     "algorithmic_flops_per_launch": int(f_loop), "roofline_ms": round(max(t_mem, t_tc) * 1e3, 4)},
        "e2e": {"value": round(e2e_ms, 4), "unit": "ms",
                "h2d_bytes_per_step": int(hn.numel() * 4 + hs.numel() * 4 + hk.numel() * 2 * 2 + hl.numel() * 4),
                "d2h_bytes_per_step": int(ho.numel() * 4)},
        "gpu_launches": int(kernels * args.steps) if kernels > 0 else None, "kernels_per_step": kernels,
        "clocks": clk.summary(),
    }
    print(json.dumps(line), flush=True)


def run_e2e(args, rank, world, local_rank, wl):
    """Prefill of the prefix (Gemma-2B shaped, 18 layers, the last K/V only) into a device KV
    cache, then the 10-step denoise loop on it; both on the device, timed per step."""
    import torch

    import flow_matching_action_expert_b200 as R
    from synth import workloads as WL

    dev = torch.device("cuda", local_rank)
    bits = WL.expert_weights(wl.expert)
    bits.update(WL.prefill_weights(wl.prefill))
    dw = {k: torch.from_numpy(v.view(np.int16)).view(torch.bfloat16).to(dev) for k, v in bits.items()}
    del bits
    cfg = R.make_config(n_layers=wl.expert.n_layers, chunk=wl.chunk, max_prefix=wl.prefix_cap,
                        max_batch=wl.batch, has_prefill=True, engine=args.engine)
    ctx = R.rtvla_create(dw, cfg)
    del dw
    torch.cuda.empty_cache()
    emb_bits, mask_np = WL.prefill_inputs(wl)
    emb = torch.from_numpy(emb_bits.view(np.int16)).view(torch.bfloat16).to(dev)
    mask = torch.from_numpy(mask_np).to(dev)
    L, B, P = wl.expert.n_layers, wl.batch, wl.prefix_cap
    k = torch.zeros((L, B, P, 256), dtype=torch.bfloat16, device=dev)
    v = torch.zeros_like(k)
    valid = torch.zeros(B, dtype=torch.int32, device=dev)
    kv = R.make_kv(k, v, valid, B, P)
    noise = torch.from_numpy(WL.noise(wl)).to(dev)
    out = torch.empty_like(noise)
    stream = torch.cuda.current_stream(dev)
    flush = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)

    def step(e0=None, e1=None, e2=None):
        if e0 is not None:
            e0.record(stream)
        R.rtvla_prefill(ctx, emb, mask, B, P, kv, stream)
        if e1 is not None:
            e1.record(stream)
        R.rtvla_sample_actions(ctx, noise, kv, out, stream)
        if e2 is not None:
            e2.record(stream)

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize()
    st = R.rtvla_sync_status(ctx, stream)
    if st != 0:
        raise RuntimeError(f"device status {R.STATUS[st]}")
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    with Clocks(local_rank) as clk:
        for i in range(args.steps):
            flush.fill_(float(i))
            step(*ev[i])
        torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    pre = [a.elapsed_time(b) for a, b, _ in ev]
    den = [b.elapsed_time(c) for _, b, c in ev]
    tot = [a.elapsed_time(c) for a, _, c in ev]
    ms, pre_ms, den_ms = reduce_max([statistics.mean(tot), statistics.mean(pre), statistics.mean(den)], dev)
    st = R.rtvla_sync_status(ctx, stream)
    if st != 0:
        raise RuntimeError(f"device status {R.STATUS[st]}")
    kernels = R.rtvla_kernels_per_call(ctx, wl.batch) + prefill_kernels(wl.prefill.n_layers)
    R.rtvla_destroy(ctx)
    if rank != 0:
        return
    hbm, bf16_pk, bf16_sus, src = peaks()
    pb, pf = prefill_algorithmic(wl)
    db, df, _ = algorithmic(wl)
    t_pre = max(pb / (hbm * 1e9), pf / (bf16_sus * 1e12))
    t_den = max(db / (hbm * 1e9), df / (bf16_sus * 1e12))
    line = {
        "metric": "prefill + 10-step denoise latency ms (2-view e2e, 544-token prefix, chunk 63)",
        "value": round(ms, 4), "unit": "ms", "n_gpus": world, "steps": args.steps,
        "warmup": max(3, args.warmup), "ms_per_step": round(ms, 4), "higher_is_better": False,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded N(0,0.02) bf16 weights, N(0,1)*sqrt(2048) prefix embeddings, N(0,1) noise)",
        "config": workload_config(wl, world),
        "l2": "flushed by a 256 MiB write between timed steps; weights (4.4 GB) exceed L2",
        "prefill_ms": round(pre_ms, 4), "denoise_ms": round(den_ms, 4),
        "roofline": {"bound": "tensor", "kernel": "rtvla_prefill (layered tcgen05 GEMMs + attention)",
                     "achieved": round(pf / (pre_ms * 1e-3) / 1e12, 1), "peak": bf16_sus, "unit": "TFLOP/s",
                     "frac": round(pf / (pre_ms * 1e-3) / 1e12 / bf16_sus, 4), "traffic": None,
                     "peak_source": src, "algorithmic_flops_per_launch": int(pf),
                     "algorithmic_bytes_per_launch": int(pb), "roofline_ms": round(t_pre * 1e3, 4),
                     "denoise_roofline_ms": round(t_den * 1e3, 4),
                     "denoise_frac": round(t_den * 1e3 / den_ms, 4)},
        "gpu_launches": kernels * args.steps,
        "kernels_per_step": kernels,
        "clocks": clk.summary(),
    }
    print(json.dumps(line), flush=True)


def run_stream(args, rank, world, local_rank, wl):
    """Full streaming inference: every frame is a prefill of the 544-token prefix into one of
    two caller-owned KV caches, then the denoise loop on that cache.  Sequential: frame n+1
    starts when frame n has finished.  Pipelined: prefill and denoise run on two streams, the
    prefill of frame n+1 overlapping the denoise of frame n; a prefill waits only for the
    denoise that last read its cache.  The denoise runs on the layered engine (the persistent
    kernel's cooperative launch needs every SM and would not overlap).  The last frame's
    actions of the two schedules must agree."""
    import torch

    import flow_matching_action_expert_b200 as R
    from synth import workloads as WL

    dev = torch.device("cuda", local_rank)
    bits = WL.expert_weights(wl.expert)
    bits.update(WL.prefill_weights(wl.prefill))
    dw = {k: torch.from_numpy(v.view(np.int16)).view(torch.bfloat16).to(dev) for k, v in bits.items()}
    del bits
    cfg = R.make_config(n_layers=wl.expert.n_layers, chunk=wl.chunk, max_prefix=wl.prefix_cap,
                        max_batch=wl.batch, has_prefill=True, engine=R.ENGINE_LAYERED)
    ctx = R.rtvla_create(dw, cfg)
    del dw
    torch.cuda.empty_cache()
    emb_bits, mask_np = WL.prefill_inputs(wl)
    emb = torch.from_numpy(emb_bits.view(np.int16)).view(torch.bfloat16).to(dev)
    mask = torch.from_numpy(mask_np).to(dev)
    L, B, P = wl.expert.n_layers, wl.batch, wl.prefix_cap
    kvs = []
    for _ in range(2):
        k = torch.zeros((L, B, P, 256), dtype=torch.bfloat16, device=dev)
        v = torch.zeros_like(k)
        valid = torch.zeros(B, dtype=torch.int32, device=dev)
        kvs.append((k, v, valid, R.make_kv(k, v, valid, B, P)))
    noise = torch.from_numpy(WL.noise(wl)).to(dev)
    outs = [torch.empty_like(noise) for _ in range(2)]
    s_pre, s_den = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    n = max(4, args.steps)

    def frames(pipelined):
        ev_p = [torch.cuda.Event() for _ in range(n)]
        ev_d = [torch.cuda.Event() for _ in range(n)]
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0.record(s_pre)
        s_den.wait_event(t0)
        for i in range(n):
            kv = kvs[i % 2][3]
            if pipelined:
                if i >= 2:
                    s_pre.wait_event(ev_d[i - 2])  # the denoise that last read this cache
            elif i >= 1:
                s_pre.wait_event(ev_d[i - 1])      # strictly one frame after the other
            R.rtvla_prefill(ctx, emb, mask, B, P, kv, s_pre)
            ev_p[i].record(s_pre)
            s_den.wait_event(ev_p[i])
            R.rtvla_sample_actions(ctx, noise, kv, outs[i % 2], s_den)
            ev_d[i].record(s_den)
        t1.record(s_den)
        t1.synchronize()
        return t0.elapsed_time(t1) / n, outs[(n - 1) % 2].clone()

    for _ in range(max(1, args.warmup)):
        frames(False)
    torch.cuda.synchronize()
    seq_ms, seq_out = frames(False)
    pip_ms, pip_out = frames(True)
    torch.cuda.synchronize()
    st = R.rtvla_sync_status(ctx)
    if st != 0:
        raise RuntimeError(f"device status {R.STATUS[st]}")
    diff = float((seq_out - pip_out).abs().max())
    if not diff <= 1e-2:
        raise RuntimeError(f"pipelined frames differ from sequential ones: max-abs {diff}")
    seq_ms, pip_ms = reduce_max([seq_ms, pip_ms], dev)
    R.rtvla_destroy(ctx)
    if rank != 0:
        return
    line = {
        "metric": "sustained frames/s, prefill (544 tokens) + 10-step denoise per frame, pipelined on two streams",
        "value": round(world * 1e3 / pip_ms, 2), "unit": "frames/s", "n_gpus": world, "steps": n,
        "warmup": max(1, args.warmup), "ms_per_step": round(pip_ms, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded N(0,0.02) bf16 weights, N(0,1)*sqrt(2048) prefix embeddings, N(0,1) noise)",
        "config": workload_config(wl, world), "engine": "layered (prefill and denoise graphs on two streams)",
        "sequential_ms_per_frame": round(seq_ms, 4), "pipelined_ms_per_frame": round(pip_ms, 4),
        "overlap_gain": round(seq_ms / pip_ms, 3), "pipelined_vs_sequential_max_abs": diff,
    }
    print(json.dumps(line), flush=True)


def _vision_ctx(vcfg, n_img, dev, tag="vision"):
    import torch

    import flow_matching_action_expert_b200 as R
    from synth import workloads as WL
    bits = WL.vision_weights(vcfg, tag=tag)
    dw = {k: torch.from_numpy(v.view(np.int16)).view(torch.bfloat16).to(dev) for k, v in bits.items()}
    ctx = R.rtvla_vision_create(dw, R.make_vision_config(n_layers=vcfg.n_layers, max_images=n_img))
    del dw
    return ctx, bits


def run_vision(args, rank, world, local_rank):
    """The image encoder alone: --views camera views (one sample) through the 27-layer SigLIP
    tower and the projector into a prefix buffer, one rtvla_encode_images call (one graph
    replay) per step, inputs resident.  e2e: the images copied from pinned host memory and the
    embeddings read back, every step."""
    import torch

    import flow_matching_action_expert_b200 as R
    from synth import workloads as WL

    dev = torch.device("cuda", local_rank)
    vcfg = WL.VisionShape()
    V = args.views
    ctx, bits = _vision_ctx(vcfg, V, dev)
    imgs_np = WL.images(vcfg, V)
    imgs = torch.from_numpy(imgs_np).to(dev)
    P = V * vcfg.tokens
    emb = torch.zeros((1, P, vcfg.out_width), dtype=torch.bfloat16, device=dev)
    stream = torch.cuda.current_stream(dev)
    flush = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)

    def call():
        R.rtvla_encode_images(ctx, imgs, 1, V, emb, P, stream)

    for _ in range(max(3, args.warmup)):
        call()
    torch.cuda.synchronize()
    st = R.rtvla_vision_sync_status(ctx, stream)
    if st != 0:
        raise RuntimeError(f"device status {R.STATUS[st]}")
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    with Clocks(local_rank) as clk:
        for i in range(args.steps):
            flush.fill_(float(i))
            ev[i][0].record(stream)
            call()
            ev[i][1].record(stream)
        torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    times = [a.elapsed_time(b) for a, b in ev]
    # end to end: pinned host images in, embeddings out, every step
    h_imgs = torch.from_numpy(imgs_np).pin_memory()
    h_emb = torch.empty(emb.shape, dtype=emb.dtype).pin_memory()
    e2e_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    for i in range(args.steps):
        flush.fill_(float(i))
        e2e_ev[i][0].record(stream)
        imgs.copy_(h_imgs, non_blocking=True)
        call()
        h_emb.copy_(emb, non_blocking=True)
        e2e_ev[i][1].record(stream)
    torch.cuda.synchronize()
    e2e_times = [a.elapsed_time(b) for a, b in e2e_ev]
    ms, e2e_ms = reduce_max([statistics.mean(times), statistics.mean(e2e_times)], dev)
    st = R.rtvla_vision_sync_status(ctx, stream)
    if st != 0:
        raise RuntimeError(f"device status {R.STATUS[st]}")
    kernels = R.rtvla_vision_kernels_per_call(ctx, V)
    R.rtvla_vision_destroy(ctx)
    if rank != 0:
        return
    hbm, bf16_pk, bf16_sus, src = peaks()
    vb, vf = vision_algorithmic(vcfg, V)
    t_roof = max(vb / (hbm * 1e9), vf / (bf16_pk * 1e12))
    achieved = vf / (ms * 1e-3) / 1e12
    line = {
        "metric": vision_metric(V),
        "value": round(ms, 4), "unit": "ms", "n_gpus": world, "steps": args.steps,
        "warmup": max(3, args.warmup), "ms_per_step": round(ms, 4), "higher_is_better": False,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded N(0,0.02) bf16 weights, uniform [-1,1) f32 pixels)",
        "config": vision_config(vcfg, V, world),
        "l2": "flushed by a 256 MiB write between timed steps",
        "roofline": {"bound": "tensor", "kernel": "rtvla_encode_images (tcgen05 GEMMs + attention, one graph)",
                     "achieved": round(achieved, 1), "peak": bf16_pk, "unit": "TFLOP/s",
                     "frac": round(achieved / bf16_pk, 4), "traffic": None, "peak_source": src,
                     "algorithmic_flops_per_launch": int(vf), "algorithmic_bytes_per_launch": int(vb),
                     "roofline_ms": round(t_roof * 1e3, 4)},
        "e2e": {"value": round(e2e_ms, 4), "unit": "ms", "h2d_bytes_per_step": int(imgs.numel() * 4),
                "d2h_bytes_per_step": int(emb.numel() * 2)},
        "gpu_launches": kernels * args.steps,
        "kernels_per_step": kernels,
        "clocks": clk.summary(),
    }
    if not args.no_cpu_baseline:
        from oracle import vision as OV
        W = WL.as_f32(bits)
        t0 = time.perf_counter()
        OV.encode_image(imgs_np[0], W, vcfg)
        one = (time.perf_counter() - t0) * 1e3
        line["cpu_baseline"] = {"value": round(one * V, 1), "unit": "ms", "cores": cpu_threads(), "kind": "oracle",
                                "sample": f"1 of the {V} images through the fp64 oracle tower, scaled by {V}"}
    print(json.dumps(line), flush=True)


PAGES_PI0_MS = {1: 20.0, 2: 27.3, 3: 36.8}   # Realtime-VLA, full π0 inference on one RTX 4090


def run_pipeline(args, rank, world, local_rank):
    """Full π0 inference as the pages time it (empty prompt, chunk 63, 10 steps, batch 1):
    --views camera views -> image encoder -> prefix pass over the views * 256 image tokens
    (Gemma-2B shape, 18 layers) -> the π0 10-step loop (the persistent kernel).  value: device
    time per inference with inputs resident; e2e: the same with images, robot state and noise
    copied from pinned host memory and the actions copied back, every step."""
    import torch

    import flow_matching_action_expert_b200 as R
    from synth import workloads as WL

    dev = torch.device("cuda", local_rank)
    V = args.views
    vcfg = WL.VisionShape()
    P = V * vcfg.tokens
    wl = WL.Workload(f"pi0 pipeline {V}-view: SigLIP L27 + prefill P{P} + L18 C63 B1", WL.ExpertShape(), 63, 1, P,
                     (P,), prefill=WL.PrefillShape(), description="empty prompt")
    vctx, _ = _vision_ctx(vcfg, V, dev)
    bits = WL.pi0_expert_weights(wl.expert, bias_std=0.02)
    bits.update(WL.prefill_weights(wl.prefill))
    dw = {k: torch.from_numpy(v.view(np.int16)).view(torch.bfloat16).to(dev) for k, v in bits.items()}
    del bits
    cfg = R.make_config(n_layers=wl.expert.n_layers, chunk=wl.chunk, max_prefix=P, max_batch=1, has_prefill=True,
                        engine=args.engine, variant=R.VARIANT_PI0)
    ctx = R.rtvla_create(dw, cfg)
    del dw
    torch.cuda.empty_cache()
    imgs_np, noise_np, state_np = WL.images(vcfg, V), WL.noise(wl), WL.state(wl)
    imgs = torch.from_numpy(imgs_np).to(dev)
    noise = torch.from_numpy(noise_np).to(dev)
    state = torch.from_numpy(state_np).to(dev)
    out = torch.empty_like(noise)
    emb = torch.zeros((1, P, 2048), dtype=torch.bfloat16, device=dev)
    mask = torch.ones((1, P), dtype=torch.uint8, device=dev)
    L = wl.expert.n_layers
    k = torch.zeros((L, 1, P, 256), dtype=torch.bfloat16, device=dev)
    v = torch.zeros_like(k)
    valid = torch.zeros(1, dtype=torch.int32, device=dev)
    kv = R.make_kv(k, v, valid, 1, P)
    stream = torch.cuda.current_stream(dev)
    flush = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)

    def step(ev=None):
        if ev:
            ev[0].record(stream)
        R.rtvla_encode_images(vctx, imgs, 1, V, emb, P, stream)
        if ev:
            ev[1].record(stream)
        R.rtvla_prefill(ctx, emb, mask, 1, P, kv, stream)
        if ev:
            ev[2].record(stream)
        R.rtvla_sample_actions_pi0(ctx, noise, state, kv, out, stream)
        if ev:
            ev[3].record(stream)

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize()
    for c, f in ((vctx, R.rtvla_vision_sync_status), (ctx, R.rtvla_sync_status)):
        st = f(c, stream)
        if st != 0:
            raise RuntimeError(f"device status {R.STATUS[st]}")
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    with Clocks(local_rank) as clk:
        for i in range(args.steps):
            flush.fill_(float(i))
            step(evs[i])
        torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    vis = statistics.mean(e[0].elapsed_time(e[1]) for e in evs)
    pre = statistics.mean(e[1].elapsed_time(e[2]) for e in evs)
    den = statistics.mean(e[2].elapsed_time(e[3]) for e in evs)
    tot = statistics.mean(e[0].elapsed_time(e[3]) for e in evs)
    # end to end: pinned host images, state and noise in, actions out, every step
    h_imgs = torch.from_numpy(imgs_np).pin_memory()
    h_state = torch.from_numpy(state_np).pin_memory()
    h_noise = torch.from_numpy(noise_np).pin_memory()
    h_out = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    e2e_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    for i in range(args.steps):
        flush.fill_(float(i))
        e2e_ev[i][0].record(stream)
        imgs.copy_(h_imgs, non_blocking=True)
        state.copy_(h_state, non_blocking=True)
        noise.copy_(h_noise, non_blocking=True)
        step()
        h_out.copy_(out, non_blocking=True)
        e2e_ev[i][1].record(stream)
    torch.cuda.synchronize()
    e2e = statistics.mean(a.elapsed_time(b) for a, b in e2e_ev)
    tot, vis, pre, den, e2e = reduce_max([tot, vis, pre, den, e2e], dev)
    for c, f in ((vctx, R.rtvla_vision_sync_status), (ctx, R.rtvla_sync_status)):
        st = f(c, stream)
        if st != 0:
            raise RuntimeError(f"device status {R.STATUS[st]}")
    kernels = (R.rtvla_vision_kernels_per_call(vctx, V) + prefill_kernels(wl.prefill.n_layers)
               + R.rtvla_kernels_per_call(ctx, 1))
    R.rtvla_vision_destroy(vctx)
    R.rtvla_destroy(ctx)
    if rank != 0:
        return
    hbm, bf16_pk, bf16_sus, src = peaks()
    vb, vf = vision_algorithmic(vcfg, V)
    pb, pf = prefill_algorithmic(wl)
    db, df = pi0_algorithmic(wl)
    t_vis = max(vb / (hbm * 1e9), vf / (bf16_sus * 1e12)) * 1e3
    t_pre = max(pb / (hbm * 1e9), pf / (bf16_sus * 1e12)) * 1e3
    t_den = max(db / (hbm * 1e9), df / (bf16_sus * 1e12)) * 1e3
    h2d = int(imgs.numel() * 4 + state.numel() * 4 + noise.numel() * 4)
    line = {
        "metric": f"full pi0 inference latency ms ({V}-view, empty prompt, chunk 63: image encoder + prefix pass "
                  f"+ 10-step loop)",
        "value": round(tot, 4), "unit": "ms", "n_gpus": world, "steps": args.steps,
        "warmup": max(3, args.warmup), "ms_per_step": round(tot, 4), "higher_is_better": False,
        "scaling": "weak", "vs_baseline": round(tot / PAGES_PI0_MS[V], 4),
        "baseline_context": f"{PAGES_PI0_MS[V]} ms: Realtime-VLA, full pi0 inference on one RTX 4090 (the pages' "
                            f"Table 1); another machine's number",
        "dtype": "bf16",
        "data": "synthetic (seeded bf16 weights, uniform [-1,1) pixels, N(0,1) state and noise)",
        "config": workload_config(wl, world) | {"views": V, "vision_layers": vcfg.n_layers},
        "l2": "flushed by a 256 MiB write between timed steps; weights (5.9 GB) exceed L2",
        "vision_ms": round(vis, 4), "prefill_ms": round(pre, 4), "denoise_ms": round(den, 4),
        "roofline": {"bound": "tensor", "kernel": "rtvla_encode_images (the stage this line adds)",
                     "achieved": round(vf / (vis * 1e-3) / 1e12, 1), "peak": bf16_sus, "unit": "TFLOP/s",
                     "frac": round(vf / (vis * 1e-3) / 1e12 / bf16_sus, 4), "traffic": None, "peak_source": src,
                     "stage_roofline_ms": {"vision": round(t_vis, 4), "prefill": round(t_pre, 4),
                                           "denoise": round(t_den, 4)},
                     "pipeline_frac": round((t_vis + t_pre + t_den) / tot, 4)},
        "e2e": {"value": round(e2e, 4), "unit": "ms", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": int(out.numel() * 4)},
        "gpu_launches": kernels * args.steps,
        "kernels_per_step": kernels,
        "clocks": clk.summary(),
    }
    print(json.dumps(line), flush=True)


def main():
    args = parse()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank)
        return
    if world > 1:
        import datetime

        import torch
        torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    try:
        run_ours(args, rank, world, local_rank)
    finally:
        if world > 1:
            import torch
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
