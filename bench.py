#!/usr/bin/env python
"""Benchmark of the LLA decode hot path on B200 — prints ONE JSON line (rank 0).

A step is one full decode step of a looped model over a batch of sequences:
for every loop t and layer d, one LLA decode-attention call over the cached
latents of every sequence, then one encode call that appends each sequence's
new token (its complete loop stack) to the latent store.  Workload default:
Ouro-1.4B shapes (D=24, T=4, H=16, d_head=128) at ratio 21.3 (r_k=16,
r_v=32), batch 768, context 4096: a 116 GB latent store resident in HBM.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

With N > 1 (launched by torchrun) each rank runs the same per-GPU workload
on its own sequences (weak scaling, no data-path collective); the timed
region is bracketed by a barrier and the max over ranks is reported.
`--impl reference` times the FP64 CPU oracle on the host cores instead.
"""

from __future__ import annotations

import argparse
import hashlib
import re
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import lla_synth as syn  # noqa: E402

METRIC = "LLA decode attn: ctx-tokens/s/GPU and achieved HBM GB/s vs peak at ρ=21.3"
UNIT = "ctx-tokens/s"
DEFAULT_WORKLOAD = "ouro_rho21_b768_n4096"
# kernels the library launches per call (our own kernels only; memsets excluded)
LAUNCHES_PER_DECODE = {"simt": 2, "tc": 3}
LAUNCHES_PER_ENCODE = 1
KERNEL_SOURCES = {"simt": ["decode_simt.cu", "sm100.cuh"], "tc": ["decode_tc.cu", "decode_tc2d.cuh", "sm100.cuh", "walk.cuh"],
                  "full": ["decode_full.cu", "sm100.cuh", "walk.cuh"], "recon": ["reconstruct.cu", "sm100.cuh"]}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(syn.CONFIGS))
    ap.add_argument("--kernel", choices=["auto", "simt", "tc"], default="auto")
    ap.add_argument("--e2e-steps", type=int, default=2)
    ap.add_argument("--kernel-sample", type=int, default=8,
                    help="time the decode kernel with CUDA events around every Nth call of the timed steps; "
                         "the other calls launch as without events (programmatic dependent launch)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--batch", type=int, default=0, help="override the workload's batch (profiling runs)")
    ap.add_argument("--layers", type=int, default=0, help="override the workload's layer count (profiling runs)")
    ap.add_argument("--mode", choices=["decode", "encode", "full", "fit"], default="decode",
                    help="encode: time prefill encoding of teacher stacks instead of the decode step")
    ap.add_argument("--encode-tokens", type=int, default=4096, help="tokens per encode call (encode mode)")
    ap.add_argument("--paged", action="store_true",
                    help="latent store as a pool of 128-token pages in shuffled order with a block table")
    ap.add_argument("--self-slot", action="store_true",
                    help="decode calls attend to the current token's exact K/V as well (lla_decode_attn_self)")
    ap.add_argument("--calib", type=int, default=1024, help="fit mode: calibration stacks per (layer, head, axis)")
    ap.add_argument("--q-std", type=float, default=1.0,
                    help="decode mode: queries drawn N(0, q_std^2); 8 spreads the logits by ~2.4 (peaked attention)")
    ap.add_argument("--final-loop", action="store_true",
                    help="full mode: cache only the final loop's K/V and use it for every loop (zero-parameter "
                         "matched-budget baseline: 1/T of the full cache)")
    return ap.parse_args()


def rank_tag(workload: str, rank: int) -> str:
    """Seed namespace of one rank: every rank decodes its own sequences (no shared data)."""
    return f"bench/{workload}/rank{rank}"


def max_over_ranks(ms: float, device) -> float:
    """Max of a per-rank duration over all ranks (identity without a process group)."""
    import torch
    import torch.distributed as dist

    t = torch.tensor([ms], dtype=torch.float64, device=device)
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_value(units_per_rank_step: float, steps: int, world: int, max_ms: float) -> float:
    """Whole-job throughput: the units all ranks processed over the slowest rank's time."""
    return world * units_per_rank_step * steps / (max_ms / 1e3)


def rho_of(cfg):
    if cfg["variant"] == 0:
        return 2 * cfg["T"] * cfg["d_head"] / (cfg["r_k"] + cfg["r_v"])
    return 2 * cfg["T"] * cfg["H"] * cfg["d_head"] / (cfg["r_k"] + cfg["r_v"])


def bytes_per_call(cfg):
    """Algorithmic bytes of one (layer, loop) decode call: the latents it must read."""
    per_tok = (cfg["r_k"] + cfg["r_v"]) * 2 * (cfg["H"] if cfg["variant"] == 0 else 1)
    return cfg["batch"] * cfg["context"] * per_tok


def config_json(cfg, name, n_gpus):
    return {"workload": name, "batch_per_gpu": cfg["batch"], "context": cfg["context"], "D": cfg["D"], "T": cfg["T"],
            "H": cfg["H"], "d_head": cfg["d_head"], "r_k": cfg["r_k"], "r_v": cfg["r_v"],
            "variant": "per-head" if cfg["variant"] == 0 else "2d", "rho": round(rho_of(cfg), 3),
            "step": f"{cfg['T']}x{cfg['D']} decode calls + 1 encode append",
            "l2": "inputs larger than L2 (latent store >> 126 MB), no flush",
            "parallelism": f"{n_gpus} replica(s), sequences sharded per GPU"}


# ---------------------------------------------------------------------------------------------
# CPU oracle timing (cpu_baseline leg and --impl reference)
# ---------------------------------------------------------------------------------------------

def oracle_sample_rate(cfg, seconds, n_seq=2):
    """ctx-tokens/s of the FP64 oracle on a bounded sample: one (layer, loop) call, n_seq sequences."""
    from oracle import lla_oracle as O

    T, H, d, rk, rv, N = cfg["T"], cfg["H"], cfg["d_head"], cfg["r_k"], cfg["r_v"], cfg["context"]
    codec1 = syn.seeded_codec(dict(cfg, D=1), "bench/cpu")
    if cfg["variant"] == 0:
        cK = syn.round_bf16(syn.gaussian("bench/cpu/cK", (n_seq, N, H, rk)))
        cV = syn.round_bf16(syn.gaussian("bench/cpu/cV", (n_seq, N, H, rv)))
        fn = O.lla_decode
        muK, muV = codec1["mu_k"][0].reshape(H, T, d), codec1["mu_v"][0].reshape(H, T, d)
    else:
        cK = syn.round_bf16(syn.gaussian("bench/cpu/cK", (n_seq, N, rk)))
        cV = syn.round_bf16(syn.gaussian("bench/cpu/cV", (n_seq, N, rv)))
        fn = O.lla_decode_2d
        muK, muV = codec1["mu_k"][0].reshape(T, H, d), codec1["mu_v"][0].reshape(T, H, d)
    q = syn.gaussian("bench/cpu/q", (n_seq, H, d))
    lens = np.full(n_seq, N)
    reps, t0 = 0, time.perf_counter()
    while True:
        fn(q, cK, cV, muK, codec1["w_up_k"][0], muV, codec1["w_up_v"][0], reps % T, lens, lens, 1 / math.sqrt(d),
           cfg["rope_base"])
        reps += 1
        el = time.perf_counter() - t0
        if el >= seconds:
            break
    cores = len(os.sched_getaffinity(0))
    return reps * n_seq * N / el, cores, (f"{reps} oracle calls x {n_seq} sequences x {N} tokens x {H} heads "
                                         f"(one layer, loop t = call mod T), {el:.1f} s")


def run_reference(a, cfg):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    rates = []
    sample = ""
    for i in range(a.warmup + a.steps):
        r, cores, sample = oracle_sample_rate(cfg, 0.0, n_seq=2)
        if i >= a.warmup:
            rates.append(r)
    value = statistics.median(rates)
    per_step_tokens = 2 * cfg["context"]
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": a.gpus,
            "steps": a.steps, "warmup": a.warmup, "ms_per_step": per_step_tokens / value * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": config_json(cfg, a.workload, 1),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                             "sample": "each step: " + sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------------------------------------
# clocks during the timed region
# ---------------------------------------------------------------------------------------------

class ClockSampler:
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
         "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
         "clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.idx = gpu_index
        self.p = None

    def __enter__(self):
        try:
            self.p = subprocess.Popen(["nvidia-smi", "-i", str(self.idx), f"--query-gpu={self.Q}",
                                       "--format=csv,noheader,nounits", "-lms", "200"],
                                      stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.p = None
        return self

    def __exit__(self, *exc):
        self.out = ""
        if self.p is not None:
            self.p.terminate()
            try:
                self.out, _ = self.p.communicate(timeout=5)
            except Exception:
                self.p.kill()
        return False

    def summary(self):
        rows = []
        for ln in (self.out or "").strip().splitlines():
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                rows.append((float(f[1]), float(f[2]), float(f[3]), f[5:9]))
            except ValueError:
                continue
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"]}
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i, v in enumerate(r[3]) if v.lower() == "active"})
        return {"sm_mhz": statistics.median(r[0] for r in rows), "sm_max_mhz": max(r[1] for r in rows),
                "power_w_max": max(r[2] for r in rows), "samples": len(rows), "reasons": reasons}


# ---------------------------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------------------------

def measured_peak(key="hbm_gbs"):
    """(peak, "measured"|"fallback"): HBM GB/s, or dense bf16 TFLOP/s ("bf16_tflops_sustained")."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            j = json.load(f)
        if key in j:
            return float(j[key]), "measured"
    return {"hbm_gbs": 6650.0, "bf16_tflops_sustained": 1400.0}[key], "fallback"


def flops_per_call(cfg):
    """Algorithmic tensor-core work of one decode call: reconstructing every head's keys from the
    latents, [tokens x r_k] . [r_k x H d] (the position-GEMM form does the same contraction)."""
    return 2.0 * cfg["batch"] * cfg["context"] * cfg["H"] * cfg["d_head"] * cfg["r_k"]


def roofline(cfg, kernel_name, kern_ms, workload):
    """The bound that binds the decode kernel: HBM for per-head latents, tensor cores for LLA-2D
    on the tensor-core kernel (683 flop per latent byte).  The kernel is timed inside a long
    step, so the tensor peak is the sustained figure."""
    kmean = statistics.mean(kern_ms)
    byt = bytes_per_call(cfg)
    hbm_peak, hbm_kind = measured_peak("hbm_gbs")
    hbm_achieved = byt / (kmean / 1e3) / 1e9
    r = {"kernel": f"lla decode ({kernel_name})", "kernel_ms_mean": kmean, "kernel_ms_min": min(kern_ms),
         "algorithmic_bytes_per_launch": byt}
    if cfg["variant"] == 1 and kernel_name == "tc":
        tf_peak, tf_kind = measured_peak("bf16_tflops_sustained")
        fl = flops_per_call(cfg)
        achieved = fl / (kmean / 1e3) / 1e12
        r.update({"bound": "tensor", "achieved": achieved, "peak": tf_peak, "unit": "TFLOP/s",
                  "frac": achieved / tf_peak, "traffic": traffic_record(kernel_name, workload),
                  "peak_source": f"{tf_kind} bf16_tflops_sustained (fp16 operands: same dense rate)",
                  "algorithmic_flops_per_launch": fl, "hbm_achieved_gbs": hbm_achieved,
                  "hbm_frac": hbm_achieved / hbm_peak})
    else:
        r.update({"bound": "hbm", "achieved": hbm_achieved, "peak": hbm_peak, "unit": "GB/s",
                  "frac": hbm_achieved / hbm_peak, "traffic": traffic_record(kernel_name, workload),
                  "peak_source": f"{hbm_kind} hbm_gbs"})
    return r


_COMMENT = re.compile(r'//[^\n]*|/\*.*?\*/|"(?:\\.|[^"\\])*"', re.S)


def _code_only(src):
    """The source with its comments removed (string literals kept) and blank runs collapsed:
    a traffic record stays valid across comment-only edits."""
    out = _COMMENT.sub(lambda m: m.group(0) if m.group(0).startswith('"') else " ", src)
    return "\n".join(ln.rstrip() for ln in out.splitlines() if ln.strip())


def upload_pieces(numel: int, ncalls: int) -> list:
    """[begin, end) element ranges of the step's new-token stacks that go up behind each of the
    step's ncalls queries: equal pieces (the last ones shorter or empty) that cover [0, numel)."""
    piece = -(-numel // ncalls) if ncalls > 0 else numel
    return [(min(k * piece, numel), min((k + 1) * piece, numel)) for k in range(ncalls)]


def kernel_sha(kernel):
    """SHA-256 of the kernel's sources without comments (the code the traffic was taken on)."""
    h = hashlib.sha256()
    for name in KERNEL_SOURCES[kernel]:
        with open(os.path.join(ROOT, "decode_attention_lla_b200", "csrc", name), encoding="utf-8") as f:
            h.update(_code_only(f.read()).encode())
    return h.hexdigest()


def traffic_record(kernel, workload):
    """DRAM bytes per launch from a committed ncu summary of this kernel on this workload, if it
    was taken on the current kernel sources (else None)."""
    rec = os.path.join(ROOT, "profiles", f"traffic_{kernel}_{workload}.json")
    if not os.path.exists(rec):
        return None
    with open(rec) as f:
        j = json.load(f)
    return j.get("dram_bytes_per_launch") if j.get("source_sha256") == kernel_sha(kernel) else None


def run_ours(a, cfg):
    import torch
    import torch.distributed as dist

    import decode_attention_lla_b200 as lla

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta

        dist.init_process_group("nccl", device_id=dev, timeout=timedelta(seconds=600))

    T, D, H, d, rk, rv = cfg["T"], cfg["D"], cfg["H"], cfg["d_head"], cfg["r_k"], cfg["r_v"]
    B, N = cfg["batch"], cfg["context"]
    cap = N + 1  # one free slot per sequence for the token appended by the step
    tag = rank_tag(a.workload, rank)
    codec_np = syn.seeded_codec(cfg, f"bench/{a.workload}/codec")
    desc = lla.Desc(D, T, H, d, rk, rv, cfg["variant"], cfg["rope_base"], cap + 1)
    codec = lla.Codec(desc, codec_np["w_down_k"], codec_np["w_down_v"], codec_np["w_up_k"], codec_np["w_up_v"],
                      codec_np["mu_k"], codec_np["mu_v"])
    del codec_np
    pages = (cap + lla.PAGE_TOKENS - 1) // lla.PAGE_TOKENS  # per sequence
    table = None
    if a.paged:  # every sequence's pages scattered over the pool in a seeded random order
        nbytes = lla.paged_store_bytes(desc, B * pages)
        perm = syn.rng(tag + "/pages").permutation(B * pages).astype(np.int32).reshape(B, pages)
        table = torch.from_numpy(perm).to(dev)
    else:
        nbytes = lla.store_bytes(desc, B, cap)
    store = torch.empty(nbytes // 2, dtype=torch.bfloat16, device=dev)
    syn.fill_gaussian_bf16_(store, tag + "/store")
    q_all = torch.empty(T, D, B, H, d, dtype=torch.float32, device=dev)
    q_all.normal_(0.0, a.q_std, generator=syn.torch_generator(tag + "/q", dev))
    S = T * d if cfg["variant"] == 0 else T * H * d
    x_shape = (B, D, H, 2, S) if cfg["variant"] == 0 else (B, D, 2, S)
    kv_self = None
    if a.self_slot:  # the current token's exact loop-t key and value per call: [T][D][2][B][H][d]
        kv_self = torch.empty(T, D, 2, B, H, d, dtype=torch.float32, device=dev)
        kv_self.normal_(generator=syn.torch_generator(tag + "/kv_self", dev))
    x_new = torch.empty(x_shape, dtype=torch.bfloat16, device=dev)
    x_new.normal_(generator=syn.torch_generator(tag + "/x", dev))
    seq_idx = torch.arange(B, dtype=torch.int32, device=dev)
    tok_idx = torch.full((B,), N, dtype=torch.int32, device=dev)
    lens = torch.full((B,), N, dtype=torch.int32, device=dev)
    qpos = torch.full((B,), N, dtype=torch.int32, device=dev)
    out = torch.empty(B, H, d, dtype=torch.float32, device=dev)
    ws = torch.empty(codec.workspace_bytes(B, pages * lla.PAGE_TOKENS if a.paged else cap), dtype=torch.uint8,
                     device=dev)
    impl = {"auto": lla.IMPL_AUTO, "simt": lla.IMPL_SIMT, "tc": lla.IMPL_TC}[a.kernel]
    scale = 1.0 / math.sqrt(d)
    kernel_name = a.kernel
    def decode_call(layer, t, q, ks, vs, impl, ev, o=None):
        o = out if o is None else o
        if table is not None:
            lla.decode_attn_paged(codec, store, B * pages, table, pages, B, layer, t, q, qpos, lens, scale, o, ws,
                                  k_self=ks, v_self=vs, impl=impl, events=ev)
        elif ks is not None:
            lla.decode_attn_self(codec, store, B, cap, layer, t, q, qpos, lens, ks, vs, scale, o, ws, impl=impl,
                                 events=ev)
        else:
            lla.decode_attn(codec, store, B, cap, layer, t, q, qpos, lens, scale, o, ws, impl=impl, events=ev)

    if a.kernel == "auto":  # find which kernel "auto" runs
        try:
            decode_call(0, 0, q_all[0, 0], None, None, lla.IMPL_TC, None)
            kernel_name = "tc"
        except lla.LLAError:
            kernel_name = "simt"
        impl = {"tc": lla.IMPL_TC, "simt": lla.IMPL_SIMT}[kernel_name]

    def step(events=None):
        k = 0
        for t in range(T):
            for layer in range(D):
                ev = events[k] if events is not None else None
                ks = vs = None
                if kv_self is not None:
                    ks, vs = kv_self[t, layer][0], kv_self[t, layer][1]
                decode_call(layer, t, q_all[t, layer], ks, vs, impl, ev)
                k += 1
        encode_step(x_new)

    def encode_step(x):
        if table is not None:
            lla.encode_paged(codec, x, B, 0, D, seq_idx, tok_idx, store, B * pages, table, pages, B)
        else:
            lla.encode(codec, x, B, 0, D, seq_idx, tok_idx, store, B, cap)

    def step_e2e(host):
        """One step through host buffers: every call's query (and self-slot K/V) goes up from pinned
        memory and its output comes back, and the step's new-token stacks go up.  The copies run on
        a copy-in and a copy-out stream beside the compute stream, into double-buffered device
        slots ordered by events, so the transfers of neighbouring calls overlap the decode.  The
        stacks (all layers of every sequence's new token, the largest copy of the step) go up in
        one piece per call behind that call's query, so no query waits behind all of them."""
        cs = torch.cuda.current_stream(dev)
        cin, cout = host["cin"], host["cout"]
        xs_host, xs_dev = host["x"].view(-1), x_new.view(-1)
        ncalls = T * D
        pieces = upload_pieces(xs_host.numel(), ncalls)
        with torch.cuda.stream(cin):  # the stacks' slots are free once the last encode read them
            cin.wait_event(host["x_free"])
        k = 0
        for t in range(T):
            for layer in range(D):
                sl = k % 2
                with torch.cuda.stream(cin):
                    cin.wait_event(host["done"][sl])  # the decode two calls back has read this slot
                    host["q_dev"][sl].copy_(host["q"][t, layer], non_blocking=True)
                    if kv_self is not None:
                        host["kv_dev"][sl].copy_(host["kv"][t, layer], non_blocking=True)
                    host["ready"][sl].record(cin)
                    a0, b0 = pieces[k]
                    if b0 > a0:
                        xs_dev[a0:b0].copy_(xs_host[a0:b0], non_blocking=True)
                    if k == ncalls - 1:
                        host["x_ready"].record(cin)
                cs.wait_event(host["ready"][sl])
                cs.wait_event(host["out_free"][sl])  # its output two calls back has been copied out
                ks = vs = None
                if kv_self is not None:
                    ks, vs = host["kv_dev"][sl][0], host["kv_dev"][sl][1]
                decode_call(layer, t, host["q_dev"][sl], ks, vs, impl, None, host["out_dev"][sl])
                host["done"][sl].record(cs)
                with torch.cuda.stream(cout):
                    cout.wait_event(host["done"][sl])
                    host["out"][t, layer].copy_(host["out_dev"][sl], non_blocking=True)
                    host["out_free"][sl].record(cout)
                k += 1
        cs.wait_event(host["x_ready"])
        encode_step(x_new)
        host["x_free"].record(cs)
        for sl in range(2):  # the step ends when its last outputs are in host memory
            cs.wait_event(host["out_free"][sl])

    for _ in range(a.warmup):
        step()
    torch.cuda.synchronize()

    # kernel events: a (begin, end) pair around every kernel_sample-th decode call of the timed
    # steps (an event between two kernels keeps the second from overlapping the first's tail,
    # so the other calls launch as they do without events)
    every = max(1, a.kernel_sample)
    ev_objs = [[(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) if k % every == 0
                else None for k in range(T * D)] for _ in range(a.steps)]
    for row in ev_objs:
        for pair in row:
            if pair is not None:
                pair[0].record()
                pair[1].record()
    torch.cuda.synchronize()
    raw = [[(p[0].cuda_event, p[1].cuda_event) if p is not None else None for p in row] for row in ev_objs]

    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    g0, g1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:
        g0.record()
        for s in range(a.steps):
            step(events=raw[s])
        g1.record()
        torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    ms = g0.elapsed_time(g1)
    kern_ms = [p[0].elapsed_time(p[1]) for row in ev_objs for p in row if p is not None]
    ms_max = max_over_ranks(ms, dev)
    ctx_tokens_step = B * N * T * D
    value = job_value(ctx_tokens_step, a.steps, world, ms_max)

    # end to end through the C ABI with host buffers: q in, out back, new-token stacks in
    e2e_value = None
    if a.e2e_steps > 0:
        host = {"q": torch.empty(T, D, B, H, d, dtype=torch.float32, pin_memory=True),
                "out": torch.empty(T, D, B, H, d, dtype=torch.float32, pin_memory=True),
                "x": torch.empty(x_shape, dtype=torch.bfloat16, pin_memory=True),
                "q_dev": [torch.empty(B, H, d, dtype=torch.float32, device=dev) for _ in range(2)],
                "out_dev": [torch.empty(B, H, d, dtype=torch.float32, device=dev) for _ in range(2)],
                "cin": torch.cuda.Stream(dev), "cout": torch.cuda.Stream(dev),
                "ready": [torch.cuda.Event() for _ in range(2)], "done": [torch.cuda.Event() for _ in range(2)],
                "out_free": [torch.cuda.Event() for _ in range(2)],
                "x_ready": torch.cuda.Event(), "x_free": torch.cuda.Event()}
        host["q"].copy_(q_all.cpu())
        if kv_self is not None:
            host["kv"] = torch.empty(kv_self.shape, dtype=torch.float32, pin_memory=True)
            host["kv"].copy_(kv_self.cpu())
            host["kv_dev"] = [torch.empty(kv_self.shape[2:], dtype=torch.float32, device=dev) for _ in range(2)]
        host["x"].copy_(x_new.cpu())
        step_e2e(host)
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(a.e2e_steps):
            step_e2e(host)
        e1.record()
        torch.cuda.synchronize()
        e2e_value = job_value(ctx_tokens_step, a.e2e_steps, world, max_over_ranks(e0.elapsed_time(e1), dev))
    h2d = T * D * B * H * d * 4 * (3 if kv_self is not None else 1) + int(np.prod(x_shape)) * 2
    d2h = T * D * B * H * d * 4

    if rank == 0:
        line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": a.steps,
                "warmup": a.warmup, "ms_per_step": ms_max / a.steps, "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
                "config": dict(config_json(cfg, a.workload, world),
                               **({"self_slot": "current token's exact K/V attended in every call"}
                                  if kv_self is not None else {}),
                               **({"store": f"paged: {pages} pages of {lla.PAGE_TOKENS} tokens per sequence, "
                                            "shuffled over the pool"} if table is not None else {}),
                               **({"query_std": a.q_std} if a.q_std != 1.0 else {})),
                "hbm_gbs_per_gpu_step": bytes_per_call(cfg) * T * D / (ms_max / a.steps / 1e3) / 1e9,
                "roofline": dict(roofline(cfg, kernel_name, kern_ms, a.workload),
                                 timed_launches=f"{len(kern_ms)} of {a.steps * T * D}: every {every}th decode call "
                                                "of the timed steps, bracketed by CUDA events on its stream"),
                "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
                "clocks": clk.summary(),
                "gpu_launches": a.steps * (T * D * LAUNCHES_PER_DECODE[kernel_name] + LAUNCHES_PER_ENCODE)}
        if world == 1 and not a.no_cpu_baseline:
            v, cores, sample = oracle_sample_rate(cfg, a.cpu_seconds)
            line["cpu_baseline"] = {"value": v, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample}
        print(json.dumps(line), flush=True)
    codec.close()
    if world > 1:
        dist.destroy_process_group()
    return 0


def main():
    a = parse()
    cfg = dict(syn.CONFIGS[a.workload])
    if a.batch or a.layers:
        cfg.update(batch=a.batch or cfg["batch"], D=a.layers or cfg["D"])
        a.workload = f"{a.workload}[batch={cfg['batch']},layers={cfg['D']}]"
    if getattr(a, "paged", False) or getattr(a, "self_slot", False):
        a.workload += "[" + ",".join(k for k, on in (("paged", a.paged), ("self-slot", a.self_slot)) if on) + "]"
    if a.impl == "reference":
        return run_reference(a, cfg)
    if a.mode == "full":
        return run_full(a, cfg)
    if a.mode == "encode":
        return run_encode(a, cfg)
    if a.mode == "fit":
        return run_fit(a, cfg)
    return run_ours(a, cfg)


# fp64 CUDA-core peak: 148 SMs x 64 fp64 FMA per clock x 2 flop at the 1965 MHz maximum SM clock
FP64_PEAK_TFLOPS = 148 * 64 * 2 * 1.965e9 / 1e12


def run_fit(a, cfg):
    """GPU codec fit (lla_fit_codec): the SVD initialisation of every (layer, head) codec of the
    workload, K and V axes, from `--calib` seeded calibration stacks each (S = T*d_head, or
    T*H*d_head for 2D).  A step fits all of them; reports codec fits per second.  The CPU
    baseline is the oracle's FP64 SVD fit on a bounded sample of the same problems."""
    import torch

    import decode_attention_lla_b200 as lla

    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", "0")))
    torch.cuda.set_device(dev)
    T, D, H, d = cfg["T"], cfg["D"], cfg["H"], cfg["d_head"]
    two_d = cfg.get("variant", 0) == 1
    S = T * d * (H if two_d else 1)
    P = D * (1 if two_d else H)  # problems per axis
    n = a.calib
    R = cfg.get("traj_rank", 24)
    noise = cfg.get("noise_var", 1e-2)
    tag = f"bench/{a.workload}/fit"
    # calibration stacks: a few distinct seeded slots repeated over the problems (the fit's cost
    # does not depend on the values)
    base = np.stack([syn.smooth_stacks(f"{tag}/{i}", n, T, d * (H if two_d else 1), R, noise,
                                       syn.gaussian(f"{tag}/mu/{i}", S, cfg.get("mu_var", 0.1)))
                     for i in range(4)]).astype(np.float32)
    Xh = np.concatenate([base] * ((P + 3) // 4))[:P]
    X = torch.from_numpy(Xh).to(dev)
    out = {}
    for axis, r in (("k", cfg["r_k"]), ("v", cfg["r_v"])):
        ws = torch.empty(lla.fit_codec_workspace_bytes(P, n, S, r), dtype=torch.uint8, device=dev)
        out[axis] = (r, ws, torch.empty(P, S, device=dev), torch.empty(P, S, r, device=dev),
                     torch.empty(P, r, device=dev))

    def step():
        for axis in ("k", "v"):
            r, ws, mu, W, sig = out[axis]
            lla.fit_codec(P, n, S, r, X, mu, W, sig, ws)

    for _ in range(a.warmup):
        step()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(int(os.environ.get("LOCAL_RANK", "0"))) as clk:
        e0.record()
        for _ in range(a.steps):
            step()
        e1.record()
        torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / a.steps
    flags = max(lla.workspace_flags(out[ax][1]) for ax in ("k", "v"))
    # fp64 GEMM work of the algorithm (Gram, 24 products with G, 13 shifted CholeskyQR3, Ritz)
    def gemm_flops(r):
        m = min(n, S)
        k = min(m, max(2 * r, r + 16))
        orths = 1 + 12
        back = 2.0 * S * n * r if n < S else 0.0  # left singular vectors -> right ones
        return P * (2.0 * n * S * m / 2 + 24 * 2.0 * m * m * k + orths * 3 * 2 * 2.0 * m * k * k
                    + 2.0 * m * m * k + 2.0 * m * k * k + 2.0 * m * k * r + back)
    fl = gemm_flops(cfg["r_k"]) + gemm_flops(cfg["r_v"])
    achieved = fl / (ms / 1e3) / 1e12
    # CPU baseline: the oracle's FP64 fit on a bounded sample of the same problems
    from oracle import lla_oracle as O
    t0, done, cores = time.perf_counter(), 0, os.cpu_count()
    while time.perf_counter() - t0 < a.cpu_seconds / 2 and done < 2 * P:
        axis_r = cfg["r_k"] if done % 2 == 0 else cfg["r_v"]
        O.fit_codec_svd(Xh[done % P].astype(np.float64), axis_r)
        done += 1
    cpu_rate = done / (time.perf_counter() - t0)
    line = {"metric": "GPU codec fit: (layer, head, axis) codecs fitted per second", "value": 2 * P / (ms / 1e3),
            "unit": "codec fits/s", "n_gpus": 1, "steps": a.steps, "warmup": a.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": a.workload, "problems_per_axis": P, "calib_stacks": n, "S": S,
                       "r_k": cfg["r_k"], "r_v": cfg["r_v"], "iterations": 24, "flags": flags},
            "roofline": {"bound": "alu", "achieved": achieved, "peak": FP64_PEAK_TFLOPS, "unit": "TFLOP/s",
                         "frac": achieved / FP64_PEAK_TFLOPS, "traffic": None,
                         "kernel": "whole fit (fp64 GEMM work / fit time; latency of the small factorisations bounds it)",
                         "peak_source": "derived: 148 SMs x 64 fp64 FMA/clk x 2 x 1.965 GHz"},
            "cpu_baseline": {"value": cpu_rate, "unit": "codec fits/s", "cores": cores, "kind": "oracle",
                             "sample": f"{done} FP64 SVD fits of {n} x {S} stacks"},
            "clocks": clk.summary()}
    print(json.dumps(line), flush=True)
    return 0


def run_encode(a, cfg):
    """Prefill throughput of lla_encode: stacks of n tokens for every layer -> latents.

    One step encodes `--encode-tokens` tokens (all layers, heads and both axes) into
    distinct store slots; the stacks are resident in HBM.  Reports tokens/s and the
    HBM rate on the stacks, the bytes the encode must read.
    """
    import torch

    import decode_attention_lla_b200 as lla

    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", "0")))
    torch.cuda.set_device(dev)
    T, D, H, d, rk, rv = cfg["T"], cfg["D"], cfg["H"], cfg["d_head"], cfg["r_k"], cfg["r_v"]
    n = a.encode_tokens
    codec_np = syn.seeded_codec(cfg, f"bench/{a.workload}/codec")
    desc = lla.Desc(D, T, H, d, rk, rv, cfg["variant"], cfg["rope_base"], 16)
    codec = lla.Codec(desc, codec_np["w_down_k"], codec_np["w_down_v"], codec_np["w_up_k"], codec_np["w_up_v"],
                      codec_np["mu_k"], codec_np["mu_v"])
    S = T * d if cfg["variant"] == 0 else T * H * d
    x_shape = (n, D, H, 2, S) if cfg["variant"] == 0 else (n, D, 2, S)
    x = torch.empty(x_shape, dtype=torch.bfloat16, device=dev)
    x.normal_(generator=syn.torch_generator(f"bench/{a.workload}/enc_x", dev))
    slots = 4
    store = torch.empty(lla.store_bytes(desc, slots, n) // 2, dtype=torch.bfloat16, device=dev)
    seq = torch.zeros(n, dtype=torch.int32, device=dev)
    tok = torch.arange(n, dtype=torch.int32, device=dev)
    for i in range(a.warmup):
        seq.fill_(i % slots)
        lla.encode(codec, x, n, 0, D, seq, tok, store, slots, n)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(dev.index) as clk:
        e0.record()
        for i in range(a.steps):
            seq.fill_(i % slots)
            lla.encode(codec, x, n, 0, D, seq, tok, store, slots, n)
        e1.record()
        torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / a.steps
    in_bytes = int(np.prod(x_shape)) * 2
    peak, kind = measured_peak()
    line = {"metric": "LLA encode: prefill tokens/s (all layers and heads)", "value": n / (ms / 1e3),
            "unit": "tokens/s", "n_gpus": 1, "steps": a.steps, "warmup": a.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": dict(config_json(cfg, a.workload, 1), step=f"encode {n} tokens x {D} layers"),
            "roofline": {"bound": "hbm", "achieved": in_bytes / (ms / 1e3) / 1e9, "peak": peak, "unit": "GB/s",
                         "frac": in_bytes / (ms / 1e3) / 1e9 / peak, "traffic": None, "kernel": "lla encode",
                         "peak_source": f"{kind} hbm_gbs", "algorithmic_bytes_per_launch": in_bytes,
                         "latent_bytes_written": n * D * (H if cfg["variant"] == 0 else 1) * (rk + rv) * 2},
            "clocks": clk.summary()}
    print(json.dumps(line), flush=True)
    codec.close()
    return 0


def run_full(a, cfg):
    """The full-cache comparator: the same decode step (T*D calls, loop-major) over an
    uncompressed bf16 K/V cache [B][D][T][H][N+1][d] with keys stored rotated, where it fits.
    With --final-loop the cache keeps one loop slot per layer ([B][D][1][H][N+1][d], the final
    loop's K/V) and every loop's call reads it.  Reports the same ctx-tokens/s and the HBM rate
    on the bytes the call must read (one loop's keys and values)."""
    import torch

    import decode_attention_lla_b200 as lla

    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", "0")))
    torch.cuda.set_device(dev)
    T, D, H, d = cfg["T"], cfg["D"], cfg["H"], cfg["d_head"]
    B, N = cfg["batch"], cfg["context"]
    cap = N + 1
    TS = 1 if a.final_loop else T  # loop slots kept per layer
    elems = B * D * TS * cap * H * d
    free = torch.cuda.mem_get_info(dev)[0]
    if d != 128 or 2 * elems * 2 > free - (4 << 30):
        print(json.dumps({"metric": "full-cache decode comparator", "unavailable":
                          f"full K/V cache of {2 * elems * 2 / 1e9:.0f} GB does not fit (or d_head != 128)"}))
        return 0
    tag = f"bench/{a.workload}/full"
    K = torch.empty(elems, dtype=torch.bfloat16, device=dev)
    V = torch.empty(elems, dtype=torch.bfloat16, device=dev)
    seq_stride = D * TS * cap * H * d
    lens = torch.full((B,), N, dtype=torch.int32, device=dev)
    # The fast path's cache: rebuilt once from a seeded latent store of the workload's codec
    # (lla_reconstruct_cache), one (layer, loop) slice per call, timed as its own roofline.
    # Where store and cache do not fit together the cache is filled with seeded Gaussians.
    recon = None
    desc = lla.Desc(D, T, H, d, cfg["r_k"], cfg["r_v"], cfg["variant"], cfg["rope_base"], cap + 1)
    store_b = lla.store_bytes(desc, B, cap)
    if store_b < torch.cuda.mem_get_info(dev)[0] - (4 << 30):
        codec_np = syn.seeded_codec(cfg, tag + "/codec")
        rnd = {k: (syn.round_bf16(v) if k.startswith("w_down") else syn.round_f32(v)) for k, v in codec_np.items()}
        codec = lla.Codec(desc, rnd["w_down_k"], rnd["w_down_v"], rnd["w_up_k"], rnd["w_up_v"], rnd["mu_k"], rnd["mu_v"])
        store = torch.empty(store_b // 2, dtype=torch.bfloat16, device=dev)
        syn.fill_gaussian_bf16_(store, tag + "/latents")
        loops = [T - 1] if a.final_loop else list(range(T))

        def rebuild():
            for si, t in enumerate(loops):
                for layer in range(D):
                    off = 2 * (layer * TS + si) * cap * H * d
                    lla.reconstruct_cache(codec, store, B, cap, layer, t, lens, K.data_ptr() + off, V.data_ptr() + off,
                                          seq_stride, cap)

        rebuild()  # warm-up
        torch.cuda.synchronize()
        r0, r1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        r0.record()
        rebuild()
        r1.record()
        torch.cuda.synchronize()
        rms = r0.elapsed_time(r1)
        slices = len(loops) * D
        per_slice = B * N * H * ((cfg["r_k"] + cfg["r_v"]) * 2 + 2 * d * 2)  # latents read + K, V rows written
        peak_r, kind_r = measured_peak()
        ach = per_slice * slices / (rms / 1e3) / 1e9
        recon = {"kernel": "lla_reconstruct_cache (one (layer, loop) slice per call)", "ms_total": rms,
                 "ms_per_slice": rms / slices, "slices": slices, "algorithmic_bytes_per_slice": per_slice,
                 "bound": "hbm", "achieved": ach, "peak": peak_r, "unit": "GB/s", "frac": ach / peak_r,
                 "traffic": traffic_record("recon", a.workload), "peak_source": f"{kind_r} hbm_gbs"}
        del store
        codec.close()
        torch.cuda.empty_cache()
    else:
        syn.fill_gaussian_bf16_(K, tag + "/K")
        syn.fill_gaussian_bf16_(V, tag + "/V")
    q_all = torch.empty(T, D, B, H, d, dtype=torch.float32, device=dev)
    q_all.normal_(generator=syn.torch_generator(tag + "/q", dev))
    out = torch.empty(B, H, d, dtype=torch.float32, device=dev)
    ws = torch.empty(lla.full_decode_workspace_bytes(H, d, B), dtype=torch.uint8, device=dev)
    scale = 1.0 / math.sqrt(d)

    def step():
        for t in range(T):
            for layer in range(D):
                off = 2 * (layer * TS + (0 if a.final_loop else t)) * cap * H * d
                lla.full_decode_attn(H, d, cfg["rope_base"], K.data_ptr() + off, V.data_ptr() + off, seq_stride, B,
                                     cap, q_all[t, layer], lens, lens, scale, out, ws)

    for _ in range(a.warmup):
        step()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(int(os.environ.get("LOCAL_RANK", "0"))) as clk:
        e0.record()
        for _ in range(a.steps):
            step()
        e1.record()
        torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / a.steps
    per_call = B * N * H * d * 2 * 2
    peak, kind = measured_peak()
    achieved = per_call * T * D / (ms / 1e3) / 1e9
    what = "final-loop reuse (one loop slot per layer)" if a.final_loop else "full-cache decode comparator"
    line = {"metric": f"{what}: ctx-tokens/s/GPU", "value": B * N * T * D / (ms / 1e3),
            "unit": "ctx-tokens/s", "n_gpus": 1, "steps": a.steps, "warmup": a.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": dict(config_json(cfg, a.workload, 1),
                           step=f"{T}x{D} decode calls over a full bf16 K/V cache (comparator, no LLA)",
                           cache_gb=2 * elems * 2 / 1e9, loop_slots=TS,
                           cache_source="rebuilt from a seeded latent store by lla_reconstruct_cache" if recon
                           else "seeded Gaussians (store and cache do not fit together)"),
            "reconstruct": recon,
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                         "traffic": traffic_record("full", a.workload),
                         "kernel": "full-cache decode (prologue + decode + combine, per step)",
                         "peak_source": f"{kind} hbm_gbs", "algorithmic_bytes_per_launch": per_call},
            "clocks": clk.summary()}
    print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
