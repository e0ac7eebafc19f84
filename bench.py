#!/usr/bin/env python
"""Benchmark: one streamed QLoRA SFT step through a 32-layer Llama-3.1-8B-shaped
NF4 stack (batch 1, seq 512, LoRA r16 on all seven projections, cross-entropy,
AdamW on the LoRA masters), the stack in page-locked host memory and fed to the
GPU through two VRAM layer buffers.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Prints one JSON line (rank 0).  N > 1 runs data-parallel replicas (one rank per
GPU, torch.distributed over NCCL): every rank streams its own stack copy on its
own micro-batch, the LoRA gradients are averaged with an NCCL all-reduce, then
every rank applies the same AdamW update ("scaling": "weak").

--impl reference times the CPU oracle (the slow fp64 restatement of the method)
on the host cores instead, on a bounded sample of the same workload.
"""
import argparse
import csv
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, HERE)

METRIC = "streamed QLoRA train tokens/sec (8B shapes, seq 512) and % of step roofline"
WORKLOAD = ("Llama-3.1-8B-shaped 32-layer NF4 stack (block 64, fp32 absmax) streamed from "
            "pinned host memory through two VRAM layer buffers; bf16 untied embedding and "
            "lm_head (vocab 128256) resident; batch 1 x seq 512 per GPU; one SFT step "
            "(cross-entropy + AdamW on LoRA r16 alpha32, all 7 projections)")
BATCH, SEQ = 1, 512
# DRAM bytes per launch of the fused NF4 GEMM classes at the 8B shapes with T = 512
# (one ncu capture of every GEMM launch of one layer's forward + recomputing
# backward; each launch reads its algorithmic bytes once).  The per-step mix of
# launches is the same as in that layer, so the averages hold for the step.
DRAM_BYTES_PER_LAUNCH_8B_T512 = {"gemm_nf4_fwd": 37.11e6, "gemm_nf4_dx": 42.15e6}
# Profiler classes whose one timed region spans several kernels: the rank-r
# products lora_rank_r_{u,v,dA,dB} (the product and the fixed-order sum of its
# reduction slices).  The roofline object describes
# one kernel, so these are reported in step_roofline.kernels (each, and summed
# as "lora_rank_r") but never chosen as its subject.
MULTI_KERNEL_PREFIXES = ("lora_rank_r",)
METRIC_QWEN = ("streamed LoRA train tokens/sec (Qwen2.5-3B shapes, bf16 base, seq 2048) and % of "
               "step roofline")
WORKLOAD_QWEN = ("Qwen2.5-3B-shaped 36-layer stack, unquantised bf16 weights (154.1 MB per "
                 "layer), streamed from pinned host memory through two VRAM layer buffers; bf16 "
                 "tied embedding / lm_head (vocab 151936) resident; batch 8 x seq 2048 per GPU; "
                 "one SFT step (cross-entropy + AdamW on LoRA r64 alpha128, all 7 projections)")
FALLBACK_PEAKS = dict(hbm_gbs=6650.0, bf16_tflops=1590.0, bf16_tflops_sustained=1400.0)


def dominant_kernel(prof):
    """The single-kernel class with the most device time in the profiled steps."""
    single = {k: v for k, v in prof.items() if not k.startswith(MULTI_KERNEL_PREFIXES)}
    return max((single or prof).items(), key=lambda kv: kv[1]["total_ms"])


def kernel_table(prof, steps):
    """Per-step launches, time, TF/s and algorithmic GB/s of every profiled class,
    plus the rank-r products summed over their kinds as "lora_rank_r"."""
    rows = dict(prof)
    kinds = [v for k, v in prof.items() if k.startswith("lora_rank_r_")]
    if kinds:
        rows["lora_rank_r"] = {f: sum(v[f] for v in kinds)
                               for f in ("launches", "total_ms", "flops", "bytes")}
    return {k: dict(launches_per_step=e["launches"] / steps, ms_per_step=e["total_ms"] / steps,
                    tflops=(e["flops"] / e["total_ms"] * 1e-9) if e["total_ms"] > 0 else None,
                    gbs=(e["bytes"] / e["total_ms"] * 1e-6) if e["total_ms"] > 0 else None)
            for k, e in rows.items()}


def workload_name(absmax_bits, dpo=False, pairs=2, batch=1, micro_batches=1):
    w = WORKLOAD
    if absmax_bits == 8:
        w = w.replace("fp32 absmax", "8-bit double-quantised absmax, one fp32 scale per 256 "
                      "blocks")
    if dpo:
        w = w.replace("batch 1 x seq 512 per GPU; one SFT step (cross-entropy + AdamW",
                      "%d chosen/rejected pairs x seq 512 per GPU; one DPO step (beta 0.1, the "
                      "same streamed base with its adapter off as reference, run from the same "
                      "layer buffer; AdamW" % pairs)
    elif batch != 1 or micro_batches != 1:
        w = w.replace("batch 1 x seq 512 per GPU; one SFT step",
                      "batch %d x seq 512 x %d gradient-accumulation micro-batches per GPU; one "
                      "SFT step" % (batch, micro_batches))
    return w


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true",
                    help="skip the oracle timing (for quick runs)")
    ap.add_argument("--absmax-bits", type=int, choices=(32, 8), default=32,
                    help="32: fp32 absmax per NF4 block (the default workload); 8: the absmax "
                         "double-quantised to 8 bits with one fp32 scale per 256 blocks, the "
                         "pages' 113 MB layers / 3.60 GB store")
    ap.add_argument("--model", choices=("llama8b", "qwen3b"), default="llama8b",
                    help="llama8b: the 32-layer Llama-3.1-8B-shaped NF4 stack, seq 512 (default); "
                         "qwen3b: the 36-layer Qwen2.5-3B-shaped stack streamed unquantised "
                         "(bf16), tied embedding, LoRA r64, batch 8 x seq 2048")
    ap.add_argument("--batch", type=int, default=None,
                    help="sequences per micro-batch (SFT step; default 1, or 8 for qwen3b)")
    ap.add_argument("--micro-batches", type=int, default=1,
                    help="gradient-accumulation micro-batches per optimiser step (SFT step)")
    ap.add_argument("--pairs", type=int, default=2, help="chosen/rejected pairs (DPO step)")
    ap.add_argument("--case", choices=("step", "dpo", "layer", "gemm"), default="step",
                    help="step: the streamed 32-layer SFT step (default); dpo: the streamed DPO "
                         "step (beta 0.1, adapter-off reference); layer: one resident "
                         "8B-shaped layer forward + recomputing backward; gemm: one fused NF4 "
                         "GEMM at the q|k|v shape (a small case for profiling)")
    ap.add_argument("--shard-layers", action="store_true",
                    help="data-parallel layer sharding: each of the N ranks copies 1/N of every "
                         "layer from host memory and an NCCL all-gather on the GPUs assembles it "
                         "(stream_stack_shard); off by default")
    return ap.parse_args()


def peaks():
    p = os.path.join(HERE, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return dict(hbm_gbs=d["hbm_gbs"], bf16_tflops=d["bf16_tflops"],
                    bf16_tflops_sustained=d["bf16_tflops_sustained"], source="measured")
    return dict(FALLBACK_PEAKS, source="fallback")


# ---------------------------------------------------------------- CPU oracle leg
def oracle_sample(seed=1):
    """Bounded sample of one step, run by the CPU oracle: one 8B-shaped layer's
    forward and its recomputing backward (T = 512), and the lm_head forward and
    input-gradient products on a 8192-row slice of the vocabulary.  Returns
    (seconds for a whole step, description, threads)."""
    import numpy as np
    from layer_streamed_qlora_nf4_b200 import synth
    from oracle import model as om
    from oracle import nf4 as onf4
    cfg = synth.LLAMA8B
    lw = synth.layer_weights(seed, cfg)
    W = {}
    for p in synth.PROJ:
        N, K = lw["W"][p].shape
        W[p] = onf4.dequantize(*onf4.quantize(lw["W"][p]), N, K)
    params = dict(W=W, A=lw["A"], B=lw["B"], g1=synth.bf16_bits_to_f32(lw["g1"]),
                  g2=synth.bf16_bits_to_f32(lw["g2"]))
    T = BATCH * SEQ
    x = synth.bf16_bits_to_f32(synth.activations(seed + 1, T, cfg["hidden"]))
    dout = synth.normal_f32(synth.rng(seed + 2), (T, cfg["hidden"]), 1.0)
    t0 = time.perf_counter()
    om.decoder_layer_fwd(params, x, cfg, SEQ)
    t1 = time.perf_counter()
    om.decoder_layer_bwd(params, x, dout, cfg, SEQ)
    t2 = time.perf_counter()
    vs = 8192
    g = synth.rng(seed + 3)
    head = synth.bf16_bits_to_f32(synth.normal_bf16(g, (vs, cfg["hidden"]), 0.02)).astype(np.float64)
    hf = x.astype(np.float64)
    t3 = time.perf_counter()
    logits = hf @ head.T
    _ = logits @ head
    t4 = time.perf_counter()
    L = cfg["n_layers"]
    step_s = L * ((t1 - t0) + (t2 - t1)) + (t4 - t3) * cfg["vocab"] / vs
    desc = ("fp64 oracle: one 8B-shaped layer forward (%.2fs) + recomputing backward (%.2fs) at "
            "T=512, x%d layers; lm_head fwd+dX on %d of %d vocab rows (%.2fs), scaled"
            % (t1 - t0, t2 - t1, L, vs, cfg["vocab"], t4 - t3))
    return step_s, desc


def cpu_threads():
    """Threads the oracle runs on: the size of numpy's BLAS pool (its only multi-threaded
    part), else the host's CPU count."""
    try:
        import numpy as np
        from threadpoolctl import threadpool_info
        np.ones((2, 2)) @ np.ones((2, 2))   # the BLAS library is loaded by its first use
        n = [i["num_threads"] for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return max(n)
    except Exception:
        pass
    return os.cpu_count()


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import numpy as np  # noqa: F401
    times, samples = [], []
    desc = ""
    for i in range(args.warmup + args.steps):
        t0 = time.perf_counter()
        s, desc = oracle_sample(seed=1)
        if i >= args.warmup:
            times.append(s)
            samples.append(time.perf_counter() - t0)
    step_s = statistics.median(times)
    tok = BATCH * SEQ / step_s
    # Each step here is a bounded sample of the workload (one layer's forward and
    # backward and an lm_head slice), not a whole step: ms_per_step is the time
    # of that sample as run; the whole-step time it scales to is in cpu_baseline.
    line = dict(impl="reference", metric=METRIC, value=tok, unit="tokens/s", n_gpus=args.gpus,
                steps=args.steps, warmup=args.warmup,
                ms_per_step=statistics.median(samples) * 1e3,
                ms_per_step_kind="bounded sample per step (see cpu_baseline.sample); the full "
                                 "step it scales to takes %.0f ms" % (step_s * 1e3),
                higher_is_better=True, scaling="weak", vs_baseline=None, dtype="f64",
                data="synthetic",
                config=dict(workload=WORKLOAD, global_batch=BATCH, seq_len=SEQ,
                            parallelism="cpu oracle, rank 0 only"),
                cpu_baseline=dict(value=tok, unit="tokens/s", cores=cpu_threads(), kind="oracle",
                                  sample=desc),
                e2e=dict(value=tok, unit="tokens/s", h2d_bytes_per_step=0, d2h_bytes_per_step=0))
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("uuid,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, uuid):
        self.uuid = uuid
        self.f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        self.p = None

    def start(self):
        try:
            self.p = subprocess.Popen(["nvidia-smi", "--query-gpu=" + self.FIELDS,
                                       "--format=csv,noheader,nounits", "-lms", "200"],
                                      stdout=self.f, stderr=subprocess.DEVNULL)
        except OSError:
            self.p = None

    def stop(self):
        if self.p is None:
            return None
        self.p.terminate()
        try:
            self.p.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.p.kill()
        self.f.flush()
        self.f.seek(0)
        rows = [r for r in csv.reader(self.f) if len(r) >= 8]
        os.unlink(self.f.name)
        mine = [r for r in rows if self.uuid and r[0].strip() in self.uuid] or rows
        if not mine:
            return None
        sm = [float(r[1]) for r in mine if r[1].strip().replace(".", "").isdigit()]
        mx = [float(r[2]) for r in mine if r[2].strip().replace(".", "").isdigit()]
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        reasons = sorted({names[i] for r in mine for i in range(4) if "Active" == r[4 + i].strip()})
        return dict(sm_mhz=statistics.median(sm) if sm else None,
                    sm_max_mhz=max(mx) if mx else None, reasons=reasons, samples=len(mine))


# ---------------------------------------------------------------- our arm
def build_stack(L, cfg, rank, tok_shape=(1, SEQ), tied=False, buf_bytes=None):
    import torch
    from layer_streamed_qlora_nf4_b200 import pack, synth
    lay = L.lsq_layer_layout_get(cfg)
    g = torch.Generator(device="cuda").manual_seed(2)      # same frozen stack on every rank
    shapes = synth.proj_shapes(cfg)
    ones = torch.ones(cfg["hidden"], dtype=torch.bfloat16, device="cuda")
    host_blobs = []
    tmp = torch.empty(lay.bytes, dtype=torch.uint8, device="cuda")
    for _ in range(cfg["n_layers"]):
        W = {p: torch.randn(shapes[p], generator=g, device="cuda") * 0.02 for p in synth.PROJ}
        pack.pack_layer(cfg, W, ones, ones, tmp)
        hb = torch.empty(lay.bytes, dtype=torch.uint8).pin_memory()
        hb.copy_(tmp)
        host_blobs.append(hb)
        del W
    r = cfg["lora_r"]
    A = {p: torch.randn(r, shapes[p][1], generator=g, device="cuda") / r for p in synth.PROJ}
    B = {p: torch.randn(shapes[p][0], r, generator=g, device="cuda") * 0.01 for p in synth.PROJ}
    lora = torch.cat([pack.lora_block(cfg, A, B) for _ in range(cfg["n_layers"])])
    emb = (torch.randn(cfg["vocab"], cfg["hidden"], generator=g, device="cuda") * 0.02).bfloat16()
    head = emb if tied else \
        (torch.randn(cfg["vocab"], cfg["hidden"], generator=g, device="cuda") * 0.02).bfloat16()
    gt = torch.Generator(device="cuda").manual_seed(1000 + rank)
    tokens = torch.randint(0, cfg["vocab"], (8,) + tuple(tok_shape), generator=gt, device="cuda",
                           dtype=torch.int32)
    bufs = [torch.empty(buf_bytes or lay.bytes, dtype=torch.uint8, device="cuda") for _ in range(2)]
    return dict(lay=lay, host_blobs=host_blobs, lora=lora, emb=emb, head=head, gf=ones,
                tokens=tokens, bufs=bufs)


def h2d_bandwidth(host_blobs, dev_buf, reps=2):
    """Pinned host->device bandwidth (GB/s) of the stack's own layer blobs into a
    VRAM layer buffer, on a non-default stream: the best single copy over every
    layer, `reps` passes (the memory and the copy the streamer itself uses)."""
    import torch
    s = torch.cuda.Stream()
    best = 0.0
    with torch.cuda.stream(s):
        for _ in range(reps):
            for hb in host_blobs:
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record(s)
                dev_buf.copy_(hb, non_blocking=True)
                e1.record(s)
                e1.synchronize()
                best = max(best, hb.numel() / (e0.elapsed_time(e1) * 1e-3) / 1e9)
    return best


def run_ours(args):
    import torch
    from layer_streamed_qlora_nf4_b200 import dp
    _, _, local = dp.env()
    if int(os.environ.get("WORLD_SIZE", "1")) > 1:
        torch.cuda.set_device(local)
    rank, world = dp.init("nccl", device=torch.device("cuda", local))
    from layer_streamed_qlora_nf4_b200 import lib as L
    from layer_streamed_qlora_nf4_b200 import synth
    L.load()
    qwen = args.model == "qwen3b"
    cfg = synth.QWEN3B if qwen else dict(synth.LLAMA8B, absmax_bits=args.absmax_bits)
    SEQ = 2048 if qwen else globals()["SEQ"]
    dpo = args.case == "dpo"
    batch = args.batch if args.batch is not None else (8 if qwen else 1)
    batch, mbs = (2 * args.pairs, 1) if dpo else (batch, args.micro_batches)
    tok_shape = (args.pairs, 2, SEQ) if dpo else (mbs, batch, SEQ)
    tokens_per_step = mbs * batch * SEQ
    buf_bytes = None
    if args.shard_layers:
        buf_bytes = world * L.lsq_shard_bytes(L.lsq_layer_layout_get(cfg).bytes, world)
    st = build_stack(L, cfg, rank, tok_shape, tied=qwen, buf_bytes=buf_bytes)
    lay = st["lay"]
    handle = L.StreamStack(cfg, st["host_blobs"], st["bufs"][0], st["bufs"][1], False)
    if args.shard_layers:
        dp.shard_stack(L, handle, buf_bytes)
    if world > 1:   # the LoRA-gradient average, per layer inside the step (NCCL)
        dp.reduce_grads_stack(L, handle)
    ws_bytes = (L.stream_stack_dpo_workspace_bytes(cfg, args.pairs, SEQ) if dpo
                else L.stream_stack_workspace_bytes(cfg, batch, SEQ))
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device="cuda")
    lora, grad = st["lora"], torch.zeros_like(st["lora"])
    m, v = torch.zeros_like(lora), torch.zeros_like(lora)
    opt = dict(lr=2e-4, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=0.0, step=1, m=m, v=v)
    stream = torch.cuda.current_stream()
    pool = st["tokens"]           # a few distinct batches, cycled

    cur = dict(h=handle)              # the stack the steps run on

    def step(tokens):
        o = opt
        h = cur["h"]
        if dpo:
            loss, _ = L.stream_stack_dpo_step(h, tokens, args.pairs, SEQ, 0.1, st["emb"],
                                              st["head"], st["gf"], lora, grad, o, ws)
        else:
            loss = L.stream_stack_step(h, tokens, mbs, batch, SEQ, st["emb"], st["head"],
                                       st["gf"], lora, grad, o, ws)
        opt["step"] += 1
        return loss

    def timed(steps, tokens_of, profile=False, label="timed"):
        """Device time per step over `steps` steps (barrier + sync on both sides,
        CUDA events on the compute stream, max over ranks)."""
        dp.barrier()
        torch.cuda.synchronize()
        copies, wait_ms, h2d = 0, 0.0, 0
        if profile:
            L.lsq_profile_enable(True)
        n0 = L.lsq_launch_counter()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        torch.cuda.nvtx.range_push(label)     # lets a profiler select exactly these steps
        loss = None
        for i in range(steps):
            loss = step(tokens_of(i))
            s = L.stream_stack_last_stats(cur["h"])
            copies += s["layer_copies"]
            h2d += s["h2d_bytes"]
            wait_ms += s["copy_wait_ms"]
        torch.cuda.nvtx.range_pop()
        e1.record(stream)
        torch.cuda.synchronize()
        dp.barrier()
        launches = L.lsq_launch_counter() - n0
        prof = None
        if profile:
            L.lsq_profile_enable(False)
            prof = L.lsq_profile_read()
        ms = dp.max_over_ranks(e0.elapsed_time(e1) / steps, "cuda")
        return ms, loss, (copies, h2d), wait_ms, launches, prof

    # measured before the first step: the handle then holds no layer in its buffers,
    # so overwriting buffer 0 here cannot leave it a stale layer to reuse
    h2d_gbs = h2d_bandwidth(st["host_blobs"], st["bufs"][0])
    for i in range(args.warmup):
        loss = step(pool[i % len(pool)])
    torch.cuda.synchronize()

    # ------------------------------------------------------------ timed region (headline)
    uuid = str(getattr(torch.cuda.get_device_properties(torch.cuda.current_device()), "uuid", ""))
    sampler = ClockSampler(uuid)
    sampler.start()
    ms, loss, (copies, h2d), wait_ms, launches, _ = timed(args.steps,
                                                          lambda i: pool[i % len(pool)])
    clocks = sampler.stop()
    value = world * tokens_per_step / (ms * 1e-3)

    # ------------------------------------------------------------ same steps, kernels timed
    # Every kernel launch bracketed by CUDA events on its stream.  In the streamed
    # step each event record is itself delayed by the layer copy that saturates
    # PCIe (~25 us per region on B200), while the kernels are not: the unprofiled
    # streamed step computes for as long as the resident one.  So the kernel
    # table comes from the same steps run with the stack resident (device copies
    # of the same layer blobs); the streamed per-launch figure is kept beside it.
    ms_prof_s, _, _, _, _, prof_s = timed(args.steps, lambda i: pool[i % len(pool)],
                                          profile=True, label="timed_kernels_streamed")
    res_blobs = [hb.cuda() for hb in st["host_blobs"]]
    res_handle = L.StreamStack(cfg, res_blobs, None, None, True)
    if world > 1:
        dp.reduce_grads_stack(L, res_handle)
    cur["h"] = res_handle
    step(pool[0])                                  # captures the resident graphs
    torch.cuda.synchronize()
    ms_res, _, _, _, _, _ = timed(args.steps, lambda i: pool[i % len(pool)],
                                  label="timed_resident")
    ms_prof, _, _, _, _, prof = timed(args.steps, lambda i: pool[i % len(pool)], profile=True,
                                      label="timed_kernels")
    cur["h"] = handle
    res_handle.close()
    del res_blobs

    # ------------------------------------------------------------ end to end (host buffers)
    tok_host = pool.cpu().pin_memory()
    tok_dev = torch.empty_like(pool[0])

    def from_host(i):
        tok_dev.copy_(tok_host[i % len(tok_host)], non_blocking=True)
        return tok_dev                  # the step itself returns the loss on the host
    e2e_ms = timed(args.steps, from_host, label="timed_e2e")[0]
    e2e = dict(value=world * tokens_per_step / (e2e_ms * 1e-3), unit="tokens/s",
               h2d_bytes_per_step=tok_dev.numel() * 4, d2h_bytes_per_step=4,
               layer_stream_h2d_bytes_per_step=h2d // args.steps)

    pk = peaks()
    dom_name, dom = dominant_kernel(prof)
    per_launch_ms = dom["total_ms"] / dom["launches"]
    dom_s = prof_s.get(dom_name)
    per_launch_ms_streamed = dom_s["total_ms"] / dom_s["launches"] if dom_s else None
    achieved = (dom["flops"] / dom["launches"]) / (per_launch_ms * 1e-3) / 1e12
    peak = pk["bf16_tflops_sustained"]
    traffic = None
    if not qwen and args.absmax_bits == 32 and tokens_per_step // mbs == SEQ:
        traffic = DRAM_BYTES_PER_LAUNCH_8B_T512.get(dom_name)
    roofline = dict(bound="tensor", kernel=dom_name, achieved=achieved, peak=peak, unit="TFLOP/s",
                    frac=achieved / peak, traffic=traffic,
                    traffic_source=("dram__bytes_read.sum + dram__bytes_write.sum per launch, "
                                    "averaged over the class's launches of one 8B layer (ncu)")
                    if traffic else None,
                    peak_source="%s bf16 sustained (kernel timed inside a long step)" % pk["source"],
                    launches_per_step=dom["launches"] / args.steps, per_launch_ms=per_launch_ms,
                    per_launch_ms_streamed_events=per_launch_ms_streamed,
                    step_share=dom["total_ms"] / args.steps / ms_prof,
                    timing="CUDA events around every launch of the class on its stream, over a "
                           "timed region of the same %d steps with the stack resident (%.1f "
                           "ms/step with the events, %.1f without); in the streamed step the "
                           "same events, delayed by the PCIe-saturating layer copy, give %s ms "
                           "per launch" % (args.steps, ms_prof, ms_res,
                                            "%.4f" % per_launch_ms_streamed
                                            if per_launch_ms_streamed else "n/a"))
    # step roofline: slowest of tensor FLOPs at peak, algorithmic DRAM bytes at the
    # measured copy bandwidth, and the streamed layer bytes at the measured H2D bandwidth
    flops_step = sum(e["flops"] for e in prof.values()) / args.steps
    bytes_step = sum(e["bytes"] for e in prof.values()) / args.steps
    cps = copies / args.steps
    t_tc = flops_step / (pk["bf16_tflops_sustained"] * 1e12) * 1e3
    t_hbm = (bytes_step + cps * lay.bytes) / (pk["hbm_gbs"] * 1e9) * 1e3
    # this rank's host->device bytes (a 1/N slice of each layer when sharded)
    t_h2d = h2d / args.steps / (h2d_gbs * 1e9) * 1e3
    # sharded: each GPU receives the other ranks' slices over NVLink (measured peer
    # copy bandwidth, 770 GB/s per direction)
    t_nvl = (cps * lay.bytes * (world - 1) / world / 770e9 * 1e3) if args.shard_layers else 0.0
    t_roof = max(t_tc, t_hbm, t_h2d, t_nvl)
    step_roof = dict(t_tensor_ms=t_tc, t_hbm_ms=t_hbm, t_h2d_ms=t_h2d, t_nvlink_ms=t_nvl,
                     bound=["tensor", "hbm", "h2d", "nvlink"][
                         [t_tc, t_hbm, t_h2d, t_nvl].index(t_roof)],
                     frac=t_roof / ms, frac_e2e=t_roof / e2e_ms, h2d_gbs_measured=h2d_gbs,
                     layer_copies_per_step=cps, layer_bytes=lay.bytes,
                     h2d_bytes_per_step=h2d / args.steps,
                     copy_wait_ms_per_step=wait_ms / args.steps,
                     compute_ms_per_step=ms - wait_ms / args.steps,
                     resident_ms_per_step=ms_res,
                     tflop_per_step=flops_step / 1e12,
                     kernels=kernel_table(prof, args.steps))

    cpu = None
    if (rank == 0 and world == 1 and not args.no_cpu_baseline and not dpo and not qwen
            and tokens_per_step == SEQ):
        s, desc = oracle_sample(seed=1)
        cpu = dict(value=BATCH * SEQ / s, unit="tokens/s", cores=cpu_threads(), kind="oracle",
                   sample=desc)
    handle.close()
    if rank == 0:
        line = dict(metric=METRIC_QWEN if qwen else METRIC, value=value, unit="tokens/s", n_gpus=world, steps=args.steps,
                    warmup=args.warmup, ms_per_step=ms, higher_is_better=True, scaling="weak",
                    vs_baseline=None, dtype="bf16", data="synthetic (seeded random weights and "
                    "uniform token ids at the 8B shapes)",
                    config=dict(workload=WORKLOAD_QWEN if qwen else
                                workload_name(args.absmax_bits, dpo, args.pairs, batch, mbs),
                                global_batch=world * tokens_per_step // SEQ, seq_len=SEQ,
                                parallelism="dp%d" % world + (
                                    " + layer all-gather" if args.shard_layers else ""),
                                l2="inputs larger than L2: %.2f GB of layer bytes stream per step"
                                % (cps * lay.bytes / 1e9)),
                    loss=loss, roofline=roofline, step_roofline=step_roof, cpu_baseline=cpu,
                    e2e=e2e, gpu_launches=int(launches), clocks=clocks)
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


def run_layer(args):
    """One resident 8B-shaped decoder layer: forward + recomputing backward (batch 1, seq 512)."""
    import torch
    from layer_streamed_qlora_nf4_b200 import lib as L
    from layer_streamed_qlora_nf4_b200 import pack, synth
    L.load()
    cfg = dict(synth.LLAMA8B, absmax_bits=args.absmax_bits)
    lay = L.lsq_layer_layout_get(cfg)
    g = torch.Generator(device="cuda").manual_seed(3)
    shapes = synth.proj_shapes(cfg)
    ones = torch.ones(cfg["hidden"], dtype=torch.bfloat16, device="cuda")
    blob = torch.empty(lay.bytes, dtype=torch.uint8, device="cuda")
    W = {p: torch.randn(shapes[p], generator=g, device="cuda") * 0.02 for p in synth.PROJ}
    pack.pack_layer(cfg, W, ones, ones, blob)
    del W
    r = cfg["lora_r"]
    A = {p: torch.randn(r, shapes[p][1], generator=g, device="cuda") / r for p in synth.PROJ}
    B = {p: torch.randn(shapes[p][0], r, generator=g, device="cuda") * 0.01 for p in synth.PROJ}
    lora = pack.lora_block(cfg, A, B)
    grad = torch.zeros_like(lora)
    T = BATCH * SEQ
    x = (torch.randn(T, cfg["hidden"], generator=g, device="cuda")).bfloat16().float()
    y = torch.empty_like(x)
    dy = torch.randn(T, cfg["hidden"], generator=g, device="cuda")
    dx = torch.empty_like(dy)
    ws = torch.empty(L.decoder_layer_workspace_bytes(cfg, BATCH, SEQ), dtype=torch.uint8,
                     device="cuda")
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")   # > L2, between iterations

    def it():
        L.decoder_layer_fwd(cfg, blob, lora, x, BATCH, SEQ, y, ws)
        L.decoder_layer_bwd(cfg, blob, lora, x, dy, BATCH, SEQ, dx, grad, ws)

    for _ in range(args.warmup):
        it()
    torch.cuda.synchronize()
    L.lsq_profile_enable(True)
    n0 = L.lsq_launch_counter()
    tot = 0.0
    for _ in range(args.steps):
        flush.zero_()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        it()
        e1.record()
        torch.cuda.synchronize()
        tot += e0.elapsed_time(e1)
    launches = L.lsq_launch_counter() - n0
    L.lsq_profile_enable(False)
    prof = L.lsq_profile_read()
    ms = tot / args.steps
    pk = peaks()
    flops = sum(e["flops"] for e in prof.values()) / args.steps
    gemm = {k: e for k, e in prof.items() if k.startswith("gemm")}
    gms = sum(e["total_ms"] for e in gemm.values()) / args.steps
    gfl = sum(e["flops"] for e in gemm.values()) / args.steps
    line = dict(metric="decoder layer fwd + recomputing bwd tokens/s (one 8B-shaped NF4 layer, "
                "resident, seq 512)", value=T / (ms * 1e-3), unit="tokens/s", n_gpus=1,
                steps=args.steps, warmup=args.warmup, ms_per_step=ms, higher_is_better=True,
                scaling="weak", vs_baseline=None, dtype="bf16", data="synthetic",
                config=dict(workload="one Llama-3.1-8B-shaped NF4 decoder layer, batch 1, seq "
                            "512, forward + backward with recompute, resident", global_batch=1,
                            seq_len=SEQ, parallelism="dp1", l2="L2 flushed (256 MB write) "
                            "between iterations"),
                roofline=dict(bound="tensor", kernel="all tensor-core GEMMs of the layer",
                              achieved=gfl / (gms * 1e-3) / 1e12, peak=pk["bf16_tflops"],
                              unit="TFLOP/s", frac=gfl / (gms * 1e-3) / 1e12 / pk["bf16_tflops"],
                              traffic=None, peak_source="%s (bf16 burst)" % pk["source"]),
                layer_roofline=dict(t_tensor_ms=flops / (pk["bf16_tflops"] * 1e12) * 1e3,
                                    frac=flops / (pk["bf16_tflops"] * 1e12) * 1e3 / ms),
                kernels={k: dict(launches=e["launches"] / args.steps,
                                 ms=e["total_ms"] / args.steps,
                                 tflops=e["flops"] / e["total_ms"] * 1e-9)
                         for k, e in prof.items()},
                gpu_launches=int(launches))
    print(json.dumps(line), flush=True)
    return 0


def run_gemm(args):
    """One fused NF4 + LoRA GEMM at the stacked q|k|v shape (M 6144, K 4096, T 512)."""
    import torch
    from layer_streamed_qlora_nf4_b200 import lib as L
    L.load()
    N, K, T, r = 6144, 4096, BATCH * SEQ, 16
    g = torch.Generator(device="cuda").manual_seed(4)
    W = torch.randn(N, K, generator=g, device="cuda") * 0.02
    codes = torch.empty(N * K // 2, dtype=torch.uint8, device="cuda")
    absmax = torch.empty(N * K // 64, dtype=torch.float32, device="cuda")
    L.nf4_quantize(W, codes, absmax)
    del W
    # rotate over copies of the weight totalling > 2x L2, so each launch reads it from DRAM
    n_copies = 24
    wts = [(codes.clone(), absmax.clone()) for _ in range(n_copies)]
    A = torch.randn(r, K, generator=g, device="cuda") / r
    B = torch.randn(N, r, generator=g, device="cuda") * 0.01
    x = torch.randn(T, K, generator=g, device="cuda").bfloat16().half()
    y = torch.empty(T, N, dtype=torch.float16, device="cuda")
    dy = torch.randn(T, N, generator=g, device="cuda").bfloat16()
    dx = torch.empty(T, K, dtype=torch.bfloat16, device="cuda")
    dA, dB = torch.empty(r, K, device="cuda"), torch.empty(N, r, device="cuda")
    ws = torch.empty(L.nf4_lora_linear_workspace_bytes(T, K, N, r), dtype=torch.uint8,
                     device="cuda")

    def it(i):
        c, a = wts[i % n_copies]
        L.nf4_lora_linear_fwd(x, c, a, A, B, 2.0, y, ws=ws)
        L.nf4_lora_linear_bwd(dy, x, c, a, A, B, 2.0, dx, dA, dB, ws=ws)

    for i in range(args.warmup):
        it(i)
    torch.cuda.synchronize()
    L.lsq_profile_enable(True)
    for i in range(args.steps):
        it(args.warmup + i)
    torch.cuda.synchronize()
    L.lsq_profile_enable(False)
    out = dict(case="gemm_qkv", M=N, K=K, T=T)
    for k, e in L.lsq_profile_read().items():
        ms = e["total_ms"] / e["launches"]
        tf = e["flops"] / e["launches"] / (ms * 1e-3) / 1e12
        out[k] = dict(us=ms * 1e3, tflops=tf, frac_of_burst=tf / peaks()["bf16_tflops"])
    print(json.dumps(out), flush=True)
    return 0


def main():
    args = parse()
    if args.impl == "reference":
        return run_reference(args)
    if args.case == "layer":
        return run_layer(args)
    if args.case == "gemm":
        return run_gemm(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
