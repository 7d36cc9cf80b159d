#!/usr/bin/env python
"""Benchmark of the DSA hot path (lightning indexer -> top-k -> sparse MLA) on B200.

One step = one DSA prefill forward over the L = 131072 workload (k = 2048, 64 FP8 indexer
heads, 128-head MLA-MQA): the fused indexer + top-k kernel, then the sparse MLA kernel, both
through the C ABI.  The decode chain (64 sequences, 8K-128K contexts, paged caches) is timed in
the same run and reported under "decode".  Inputs are seeded synthetic tensors generated on
the device (about 40 GB per prefill step, far larger than L2, so no flush is needed).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Under torchrun (N > 1) every rank runs an independent prefill problem of the same size
(no data-path collective; weak scaling) and the step time is the max over ranks.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "DSA prefill tokens/s at L=128K, k=2048; decode tokens/s; % of roofline"
PREFILL = "prefill_128k"
DECODE = "decode_64"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
KERNEL_SOURCES = {
    "indexer_topk": ["indexer.cuh", "select.cuh", "sm100.cuh", "common.cuh"],
    "sparse_mla": ["sparse_mla_pair.cuh", "mla_common.cuh", "sm100.cuh", "common.cuh"],
}


def log(*a):
    print(*a, file=sys.stderr, flush=True)


# fp32 lane operations per second (one op per lane and cycle): 148 SMs x 128 lanes x 1.965 GHz;
# an FMA counts 2 flops, so the fp32 FMA peak is twice this in FLOP/s
FP32_LANE_OPS_T = 148 * 128 * 1.965e9 / 1e12


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in FALLBACK_PEAKS}, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def source_hash(kernel):
    h = hashlib.sha256()
    for f in KERNEL_SOURCES[kernel]:
        with open(os.path.join(ROOT, "sparse_attention_09_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def profile_traffic(kernel):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on this source."""
    p = os.path.join(ROOT, "profiles", f"{kernel}_{PREFILL}.txt")
    if not os.path.exists(p):
        return None
    vals = {}
    with open(p) as f:
        for line in f:
            if ":" in line:
                k, v = line.split(":", 1)
                vals[k.strip()] = v.strip()
    if vals.get("source_sha") != source_hash(kernel):
        return None
    try:
        return float(vals["dram_bytes_per_launch"])
    except (KeyError, ValueError):
        return None


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples taken while the timed region runs."""

    def __init__(self, index):
        self.path = tempfile.mktemp(suffix=".csv")
        q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(index), f"--query-gpu={q}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm.append(float(parts[1]))
                    smax.append(float(parts[2]))
                except ValueError:
                    continue
                for n, v in zip(names, parts[5:9]):
                    if v.lower() == "active":
                        reasons.add(n)
        os.unlink(self.path)
        if not sm:
            return None
        return {"sm_mhz": float(np.median(sm)), "sm_max_mhz": float(max(smax)), "reasons": sorted(reasons),
                "samples": len(sm)}


def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(local)
    return world, rank, local


def max_over_ranks(x, world):
    """The slowest rank's value (device time of the timed region), identical on every rank."""
    if world == 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_value(world, tokens_per_rank, ms_per_step):
    """Whole-job throughput: the tokens all ranks processed in one step over the slowest rank's step."""
    return world * tokens_per_rank / (ms_per_step * 1e-3)


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# ------------------------------------------------------------------------------------------
# oracle timing (the CPU baseline and the reference arm)
# ------------------------------------------------------------------------------------------
def oracle_prefill_sample(inp, k, rows, sm):
    import oracle
    seq = synth.seq_slice_numpy(inp, 0, rows=rows)
    t0 = time.perf_counter()
    oracle.dsa_prefill_rows(seq, k, sm, rows)
    return time.perf_counter() - t0


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [d.get("num_threads") for d in threadpool_info() if d.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count() or 1


# ------------------------------------------------------------------------------------------
# our arm
# ------------------------------------------------------------------------------------------
def prefill_config(workload, world, cfg):
    """The JSON `config` of a prefill line (the same for both arms)."""
    return {"workload": (f"{PREFILL}: DSA prefill, batch 1 per GPU, L=131072, top-k 2048, 64 e4m3 "
                         "indexer heads d_I=128, 128-head MLA-MQA (576 qk / 512 v), bf16, 5% planted keys")
            if workload == PREFILL else f"{workload} (profiling case, not the headline)",
            "global_batch": world * len(cfg["seqlens"]), "seq_len": cfg["seqlens"][0], "k": cfg["k"],
            "parallelism": f"independent problems x{world}",
            "l2": "inputs (~40 GB/step) larger than L2; no flush"}


def prefill_work(cfg):
    L = cfg["seqlens"][0]
    pairs = sum(s * (s + 1) // 2 for s in cfg["seqlens"])
    sel_pairs = sum(sum(min(cfg["k"], t + 1) for t in range(s)) for s in cfg["seqlens"])
    idx_flops = pairs * 2 * cfg["H_I"] * cfg["d_I"]
    mla_flops = sel_pairs * 2 * cfg["H"] * (576 + 512)
    return L, idx_flops, mla_flops, sel_pairs


# ------------------------------------------------------------------------------------------
# strong scaling: one sequence sharded by query rows (NEXT row f4)
# ------------------------------------------------------------------------------------------
def run_strong(args, world, rank, local):
    """One L=131072 prefill sharded over the ranks by query-row blocks (the library's sharding
    helpers): the key (k_I, k_scale) and latent rows each rank holds are all-gathered once for
    the sequence, then every step runs the fused indexer top-k and sparse MLA on the rank's own
    rows.  The blocks are balanced with the two kernels' measured whole-sequence times
    (--idx-ms, --mla-ms).  value = L tokens per (slowest rank's) step."""
    import sparse_attention_09_b200 as dsa
    from sparse_attention_09_b200 import sharding
    cfg = dict(synth.WORKLOADS[args.workload])
    k, sm, H, H_I, d_I = cfg["k"], 1.0 / math.sqrt(576), cfg["H"], cfg["H_I"], cfg["d_I"]
    inp = synth.prefill_inputs(device="cuda", **cfg)  # same seed on every rank: rank r keeps its blocks
    L = inp["q"].shape[0]
    rb = sharding.row_blocks(L, k, world, args.idx_ms, args.mla_ms)
    q0, q1 = rb[rank], rb[rank + 1]
    kb = sharding.even_blocks(L, world)
    k0, k1 = kb[rank], kb[rank + 1]
    my_k8, my_ks, my_lat = inp["k8"][k0:k1].clone(), inp["k_scale"][k0:k1].clone(), inp["latent"][k0:k1].clone()
    for t in (inp["k8"], inp["k_scale"], inp["latent"]):  # only the gathered rows may reach the kernels
        t.zero_()
    sharding.gather_sequence(my_k8, inp["k8"], world, rank)
    sharding.gather_sequence(my_ks, inp["k_scale"], world, rank)
    sharding.gather_sequence(my_lat, inp["latent"], world, rank)
    keys = dsa.contiguous_desc(inp["k8"], inp["cu_seqlens"], L, scale=inp["k_scale"])
    lat = dsa.contiguous_desc(inp["latent"], inp["cu_seqlens"], L)
    R = q1 - q0
    idx = torch.empty((R, k), dtype=torch.int32, device="cuda")
    out = torch.empty((R, H, 512), dtype=torch.bfloat16, device="cuda")
    qb = (inp["q8"][q0:q1], inp["q_scale"][q0:q1], inp["w"][q0:q1], inp["q"][q0:q1])

    def step():
        dsa.dsa_indexer_topk_rows(qb[0], qb[1], qb[2], keys, H_I, d_I, k, q0, q1, idx)
        dsa.dsa_sparse_mla_prefill_rows(qb[3], lat, idx, H, k, sm, q0, q1, out)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    assert dsa.dsa_device_error() == 0, "device error during warm-up"
    clocks = ClockSampler(local)
    barrier(world)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.steps):
        step()
    e1.record()
    torch.cuda.synchronize()
    barrier(world)
    clk = clocks.stop()
    ms_per_step = max_over_ranks(e0.elapsed_time(e1), world) / args.steps
    assert dsa.dsa_device_error() == 0
    if rank == 0:
        line = {"metric": METRIC, "value": L / (ms_per_step * 1e-3), "unit": "tokens/s", "n_gpus": world,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
                "scaling": "strong", "vs_baseline": None, "dtype": "e4m3+bf16 (fp32 accumulate)", "data": "synthetic",
                "config": {"workload": f"{args.workload}: one sequence sharded by query-row blocks {rb}, "
                                       "keys and latent all-gathered once per sequence",
                           "global_batch": 1, "seq_len": L, "k": k, "parallelism": f"row-sharded x{world}",
                           "l2": "inputs larger than L2; no flush"},
                "clocks": clk, "gpu_launches": 2 * args.steps}
        print(json.dumps(line), flush=True)


def run_ours(args, world, rank, local):
    import sparse_attention_09_b200 as dsa

    peaks, peak_src = load_peaks()
    cfg = dict(synth.WORKLOADS[args.workload])
    cfg["seed"] = cfg["seed"] + rank
    k, sm = cfg["k"], 1.0 / math.sqrt(576)
    inp = synth.prefill_inputs(device="cuda", **cfg)
    T = inp["q"].shape[0]
    H = cfg["H"]
    keys = dsa.contiguous_desc(inp["k8"], inp["cu_seqlens"], max(inp["seqlens"]), scale=inp["k_scale"])
    lat = dsa.contiguous_desc(inp["latent"], inp["cu_seqlens"], max(inp["seqlens"]))
    out = torch.empty((T, H, 512), dtype=torch.bfloat16, device="cuda")
    idx = torch.empty((T, k), dtype=torch.int32, device="cuda")
    stream = torch.cuda.current_stream()
    nseq = len(cfg["seqlens"])

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        dsa.dsa_indexer_topk(inp["q8"], inp["q_scale"], inp["w"], keys, nseq, cfg["H_I"], cfg["d_I"], k, idx)
        if ev is not None:
            ev[1].record(stream)
        dsa.dsa_sparse_mla_prefill(inp["q"], lat, idx, nseq, H, k, sm, out)
        if ev is not None:
            ev[2].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    assert dsa.dsa_device_error() == 0, "device error during warm-up"
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    clocks = ClockSampler(local)
    barrier(world)
    torch.cuda.synchronize()
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    t_start.record(stream)
    for i in range(args.steps):
        step(evs[i])
    t_end.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    clk = clocks.stop()
    total_ms = t_start.elapsed_time(t_end)
    idx_ms = float(np.mean([e[0].elapsed_time(e[1]) for e in evs]))
    mla_ms = float(np.mean([e[1].elapsed_time(e[2]) for e in evs]))
    err = dsa.dsa_device_error()
    assert err == 0, f"device error {err}"
    total_ms = max_over_ranks(total_ms, world)
    ms_per_step = total_ms / args.steps
    L, idx_flops, mla_flops, sel_pairs = prefill_work(cfg)
    value = job_value(world, T, ms_per_step)

    fp8_peak = 2.0 * peaks["bf16_tflops_sustained"]     # nominal fp8/bf16 ratio 2 (4.5 / 2.25 PF)
    bf16_peak = peaks["bf16_tflops_sustained"]
    kernels = {
        "indexer_topk": {"ms": idx_ms, "tflops": idx_flops / (idx_ms * 1e-3) / 1e12, "peak_tflops": fp8_peak,
                         "dtype": "e4m3", "flops": idx_flops},
        "sparse_mla": {"ms": mla_ms, "tflops": mla_flops / (mla_ms * 1e-3) / 1e12, "peak_tflops": bf16_peak,
                       "dtype": "bf16", "flops": mla_flops,
                       "gather_gbs": sel_pairs * 1152 / (mla_ms * 1e-3) / 1e9},
    }
    for kk in kernels.values():
        kk["frac"] = kk["tflops"] / kk["peak_tflops"]
    # the indexer epilogue's own floor: ReLU and the weighted head sum, 2*H_I ops per causal pair,
    # against one fp32 op per lane and cycle (148 SMs x 128 lanes x 1.965 GHz = 37.2 T ops/s)
    alu_ops = idx_flops / cfg["d_I"]
    kernels["indexer_topk"]["epilogue_alu"] = {
        "ops": alu_ops, "tops": alu_ops / (idx_ms * 1e-3) / 1e12, "peak_tops": FP32_LANE_OPS_T,
        "frac": alu_ops / (idx_ms * 1e-3) / 1e12 / FP32_LANE_OPS_T}
    dom = max(kernels, key=lambda n: kernels[n]["ms"])
    dk = kernels[dom]
    traffic = profile_traffic(dom)
    roofline = {"bound": "tensor", "kernel": dom, "achieved": dk["tflops"], "peak": dk["peak_tflops"],
                "unit": "TFLOP/s", "frac": dk["frac"], "traffic": traffic,
                "peak_source": f"{peak_src} (bf16 sustained x{'2 for e4m3' if dom == 'indexer_topk' else '1'})"}

    # ---- decode chain, same process ----
    decode = run_decode(args, dsa, sm, peaks) if (rank == 0 and not args.no_decode) else None
    next_rows = ({"f1_quantize_fp8": run_quantizer(dsa, peaks), "f2_masked_mla": run_masked(dsa, sm),
                  "f3_indexer_kl": run_kl(dsa, inp, idx, cfg, sm)}
                 if (rank == 0 and not args.no_decode) else None)

    # ---- end to end through dsa_forward with host buffers ----
    e2e = run_e2e(args, dsa, inp, cfg, sm) if (rank == 0 and not args.no_e2e) else None
    if e2e is not None:  # the pipelined host-to-host result equals the device-resident step's output
        rows_chk, got = e2e.pop("_check_rows"), e2e.pop("_check")
        assert torch.equal(got, out[rows_chk]), "pipelined e2e output differs from the device-resident step"
        e2e["matches_device_path"] = True

    # ---- oracle on a bounded sample ----
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        rows = synth.sample_rows(L, k, args.cpu_rows, seed=3)
        secs = oracle_prefill_sample(inp, k, rows, sm)
        cpu = {"value": len(rows) / secs, "unit": "tokens/s", "cores": blas_threads(), "host_cores": os.cpu_count(),
               "kind": "oracle",
               "sample": f"{len(rows)} query rows of the L=131072 prefill (full causal prefix each: indexer, "
                         f"top-k, attention), {secs:.1f} s",
               "extrapolation": f"the whole L=131072 prefill at this rate: about {L * secs / len(rows) / 3600:.1f} h "
                                f"(the rows are drawn uniformly over the sequence, so their mean cost is that of "
                                f"an average row; estimate, not measured)"}
        cpu["c1_full"] = oracle_prefill_full(dict(synth.WORKLOADS["tiny_256"]), sm)   # a few seconds
        if args.cpu_c2_full:
            cpu["c2_full"] = oracle_prefill_full(dict(synth.WORKLOADS["prefill_8k"]), sm)

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "e4m3+bf16 (fp32 accumulate)", "data": "synthetic",
            "config": prefill_config(args.workload, world, cfg),
            "roofline": roofline, "kernels": kernels, "decode": decode, "next_rows": next_rows,
            "cpu_baseline": cpu, "e2e": e2e,
            "clocks": clk, "gpu_launches": 2 * args.steps,
        }
        print(json.dumps(line), flush=True)


def run_profile_case(args, dsa, sm):
    """Small cases of the bench's kernels for counter captures (the full-size step holds ~40 GB on
    the device and runs 0.1-s kernels, too much for a capture).  Every kernel is launched twice,
    a warm-up and the launch to capture (ncu -s 1 -c 1 with -k naming the kernel).
      rows_128k      the last 2048 query rows of the L=131072 prefill (keys, k_scale and latent of
                     the whole sequence, queries of the block only): dsa_indexer_topk_rows, then
                     dsa_sparse_mla_prefill_rows.  Both kernels' DRAM bytes per query row scale to
                     the full launch (per row: its queries, selection and output, and the latent
                     rows gathered for its 2048 selected entries, as for every row of the run).
      decode_8x128k  8 sequences at contexts drawn from [122880, 131072]: the fused decode
                     selection (paged indexer scan + selection kernel), sparse MLA decode and
                     the combine (8 splits per sequence).
      decode_64      the bench's decode workload (64 sequences, contexts U[8192, 131072]), the
                     same calls (one split per sequence: no combine).
      indexer_128k   the whole fused indexer + top-k launch of the L=131072 prefill (the bench's
                     own call and launch shape) with only the indexer's operands on the device
                     (~2.3 GB): its per-launch DRAM bytes need no scaling.
      mla_quarters_128k  dsa_sparse_mla_prefill_rows on four blocks of 2048 query rows of the
                     L=131072 sequence, centred on the midpoints of its quarters (the whole latent
                     on the device): midpoint-rule samples of the per-row DRAM bytes, whose
                     sum x 16 estimates the full launch.  Each block is launched twice in turn."""
    cfg = dict(synth.WORKLOADS[PREFILL])
    k = cfg["k"]
    out = {"profile_case": args.profile_case}
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(6)]
    if args.profile_case == "rows_128k":
        L, R = cfg["seqlens"][0], 2048
        blk = synth.prefill_block_inputs(L, L - R, L, cfg["H_I"], cfg["d_I"], cfg["H"], seed=cfg["seed"],
                                         device="cuda", w_dist=cfg.get("w_dist", "normal8"),
                                         planted=cfg.get("planted", 0.0))
        keys = dsa.contiguous_desc(blk["k8"], blk["cu_seqlens"], L, scale=blk["k_scale"])
        lat = dsa.contiguous_desc(blk["latent"], blk["cu_seqlens"], L)
        idx = torch.empty((R, k), dtype=torch.int32, device="cuda")
        o = torch.empty((R, cfg["H"], 512), dtype=torch.bfloat16, device="cuda")
        for i in range(2):
            evs[0].record()
            dsa.dsa_indexer_topk_rows(blk["q8"], blk["q_scale"], blk["w"], keys, cfg["H_I"], cfg["d_I"], k, L - R, L, idx)
            evs[1].record()
            dsa.dsa_sparse_mla_prefill_rows(blk["q"], lat, idx, cfg["H"], k, sm, L - R, L, o, None)
            evs[2].record()
        torch.cuda.synchronize()
        out.update(rows=R, L=L, indexer_topk_ms=evs[0].elapsed_time(evs[1]),
                   sparse_mla_ms=evs[1].elapsed_time(evs[2]))
    elif args.profile_case in ("decode_8x128k", "decode_64"):
        if args.profile_case == "decode_64":
            d = synth.decode_inputs(device="cuda", **dict(synth.WORKLOADS[DECODE]))
        else:
            d = synth.decode_inputs(B=8, ctx_lo=122880, ctx_hi=131072, H_I=64, d_I=128, H=128, seed=31, device="cuda")
        B = d["B"]
        keys = dsa.paged_desc(d["kcache8"], d["block_table"], d["ctx"], d["max_ctx"], scale=d["kscale_cache"])
        lat = dsa.paged_desc(d["latent_cache"], d["block_table"], d["ctx"], d["max_ctx"])
        idx = torch.empty((B, k), dtype=torch.int32, device="cuda")
        o = torch.empty((B, 128, 512), dtype=torch.bfloat16, device="cuda")
        ws = torch.empty(dsa.dsa_workspace_size(dsa.DSA_MODE_DECODE, B, 0, d["max_ctx"], 128, k), dtype=torch.uint8,
                         device="cuda")
        ws_sel = torch.empty(dsa.dsa_decode_select_workspace_size(B, d["max_ctx"]), dtype=torch.uint8, device="cuda")
        for i in range(2):
            evs[0].record()
            dsa.dsa_indexer_topk_decode(d["q8"], d["q_scale"], d["w"], keys, B, 64, 128, k, idx, ws_sel)
            evs[1].record()
            dsa.dsa_sparse_mla_decode(d["q"], lat, idx, B, 128, k, sm, o, None, ws)
            evs[2].record()
        torch.cuda.synchronize()
        out.update(B=B, ctx=[int(c) for c in d["ctx_host"]], indexer_topk_ms=evs[0].elapsed_time(evs[1]),
                   sparse_mla_decode_ms=evs[1].elapsed_time(evs[2]))
    elif args.profile_case == "indexer_128k":
        L = cfg["seqlens"][0]
        blk = synth.prefill_block_inputs(L, 0, L, cfg["H_I"], cfg["d_I"], cfg["H"], seed=cfg["seed"], device="cuda",
                                         w_dist=cfg.get("w_dist", "normal8"), planted=cfg.get("planted", 0.0),
                                         mla=False)
        keys = dsa.contiguous_desc(blk["k8"], blk["cu_seqlens"], L, scale=blk["k_scale"])
        idx = torch.empty((L, k), dtype=torch.int32, device="cuda")
        for i in range(2):
            evs[0].record()
            dsa.dsa_indexer_topk(blk["q8"], blk["q_scale"], blk["w"], keys, 1, cfg["H_I"], cfg["d_I"], k, idx)
            evs[1].record()
        torch.cuda.synchronize()
        out.update(L=L, indexer_topk_ms=evs[0].elapsed_time(evs[1]))
    elif args.profile_case == "mla_quarters_128k":
        L, R = cfg["seqlens"][0], 2048
        ms = []
        for j in range(4):
            mid = L // 8 + j * (L // 4)
            r0, r1 = mid - R // 2, mid + R // 2
            blk = synth.prefill_block_inputs(L, r0, r1, cfg["H_I"], cfg["d_I"], cfg["H"], seed=cfg["seed"] + j,
                                             device="cuda", w_dist=cfg.get("w_dist", "normal8"),
                                             planted=cfg.get("planted", 0.0))
            keys = dsa.contiguous_desc(blk["k8"], blk["cu_seqlens"], L, scale=blk["k_scale"])
            lat = dsa.contiguous_desc(blk["latent"], blk["cu_seqlens"], L)
            idx = torch.empty((R, k), dtype=torch.int32, device="cuda")
            o = torch.empty((R, cfg["H"], 512), dtype=torch.bfloat16, device="cuda")
            dsa.dsa_indexer_topk_rows(blk["q8"], blk["q_scale"], blk["w"], keys, cfg["H_I"], cfg["d_I"], k, r0, r1, idx)
            for i in range(2):
                evs[1].record()
                dsa.dsa_sparse_mla_prefill_rows(blk["q"], lat, idx, cfg["H"], k, sm, r0, r1, o, None)
                evs[2].record()
            torch.cuda.synchronize()
            ms.append(evs[1].elapsed_time(evs[2]))
            del blk, keys, lat, idx, o
        out.update(rows=R, L=L, blocks=[[L // 8 + j * (L // 4) - R // 2, L // 8 + j * (L // 4) + R // 2]
                                        for j in range(4)], sparse_mla_ms=ms)
    else:
        raise SystemExit(f"unknown profile case {args.profile_case}")
    assert dsa.dsa_device_error() == 0
    print(json.dumps(out), flush=True)


def run_quantizer(dsa, peaks):
    """NEXT row f1: the per-token FP8 quantiser on the q_I of the L=131072 prefill
    ([131072, 64 x 128] bf16 -> e4m3 + one scale per token) and on its k_I ([131072, 128]).
    HBM-bound; algorithmic bytes per row = 2*cols read + cols written + 4 (scale)."""
    out = {}
    for name, rows, cols in (("q_index", 131072, 64 * 128), ("k_index", 131072, 128)):
        x = torch.randn((rows, cols), dtype=torch.bfloat16, device="cuda")
        codes = torch.empty((rows, cols), dtype=torch.uint8, device="cuda")
        scale = torch.empty((rows,), dtype=torch.float32, device="cuda")
        for _ in range(3):
            dsa.dsa_quantize_fp8(x, codes, scale)
        torch.cuda.synchronize()
        n = 20
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(n):
            dsa.dsa_quantize_fp8(x, codes, scale)
        e1.record()
        torch.cuda.synchronize()
        ms = e0.elapsed_time(e1) / n
        nbytes = rows * (3 * cols + 4)
        gbs = nbytes / (ms * 1e-3) / 1e9
        out[name] = {"rows": rows, "cols": cols, "ms": ms, "gbs": gbs, "bytes": nbytes,
                     "frac_of_hbm": gbs / peaks["hbm_gbs"],
                     "l2": "input larger than L2" if rows * cols * 2 > 126e6 else "input fits in L2 (hot)"}
        del x, codes, scale
    torch.cuda.empty_cache()
    return out


def run_masked(dsa, sm):
    """NEXT row f2: the masked dense mode of sparse MLA against the sparse path on short
    prefills (selection from the fused indexer top-k, k = 2048), same outputs."""
    out = {}
    for L in (1024, 2048, 4096):
        cfg = dict(synth.WORKLOADS["prefill_8k"])
        cfg["seqlens"] = [L]
        inp = synth.prefill_inputs(device="cuda", **cfg)
        k, H = cfg["k"], cfg["H"]
        keys = dsa.contiguous_desc(inp["k8"], inp["cu_seqlens"], L, scale=inp["k_scale"])
        lat = dsa.contiguous_desc(inp["latent"], inp["cu_seqlens"], L)
        idx = torch.empty((L, k), dtype=torch.int32, device="cuda")
        dsa.dsa_indexer_topk(inp["q8"], inp["q_scale"], inp["w"], keys, 1, cfg["H_I"], cfg["d_I"], k, idx)
        o = torch.empty((L, H, 512), dtype=torch.bfloat16, device="cuda")
        row = {}
        for name, fn in (("masked", dsa.dsa_masked_mla_prefill), ("sparse", dsa.dsa_sparse_mla_prefill)):
            for _ in range(3):
                fn(inp["q"], lat, idx, 1, H, k, sm, o)
            torch.cuda.synchronize()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            for _ in range(10):
                fn(inp["q"], lat, idx, 1, H, k, sm, o)
            e1.record()
            torch.cuda.synchronize()
            row[name + "_ms"] = e0.elapsed_time(e1) / 10
        pairs = sum(min(k, t + 1) for t in range(L))
        row["sparse_tflops"] = pairs * 278528 / (row["sparse_ms"] * 1e-3) / 1e12
        row["masked_tflops_selected"] = pairs * 278528 / (row["masked_ms"] * 1e-3) / 1e12
        out[f"L{L}"] = row
    assert dsa.dsa_device_error() == 0
    return out


def run_kl(dsa, inp, idx, cfg, sm):
    """NEXT row f3: the indexer's KL alignment on the full prefill: the head-averaged attention
    distribution over each token's selection (from the forward's lse) and KL(p || softmax(I))
    with its gradient.  The indexer scores at the selected rows are a synthetic stand-in here
    (the loss kernel's cost does not depend on their values)."""
    T, H, k = inp["q"].shape[0], cfg["H"], cfg["k"]
    lat = dsa.contiguous_desc(inp["latent"], inp["cu_seqlens"], max(inp["seqlens"]))
    nseq = len(cfg["seqlens"])
    out = torch.empty((T, H, 512), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((T, H), device="cuda")
    dsa.dsa_sparse_mla_prefill(inp["q"], lat, idx, nseq, H, k, sm, out, lse)
    del out
    p = torch.empty((T, k), device="cuda")
    scores = torch.randn((T, k), device="cuda")
    loss = torch.empty((T,), device="cuda")
    grad = torch.empty((T, k), device="cuda")
    res = {}
    for name, fn in (("attn_distribution", lambda: dsa.dsa_attn_distribution(inp["q"], lat, idx, lse, nseq, H, k, sm, p)),
                     ("indexer_kl", lambda: dsa.dsa_indexer_kl(p, scores, idx, loss, grad))):
        for _ in range(2):
            fn()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(3):
            fn()
        e1.record()
        torch.cuda.synchronize()
        res[name + "_ms"] = e0.elapsed_time(e1) / 3
    pairs = sum(min(k, t + 1) for s in cfg["seqlens"] for t in range(s))
    res["attn_distribution_tflops"] = pairs * 2 * H * 576 / (res["attn_distribution_ms"] * 1e-3) / 1e12
    res["indexer_kl_gbs"] = T * k * 4 * 4 / (res["indexer_kl_ms"] * 1e-3) / 1e9  # p, scores, idx read; grad written
    res["mean_row_sum_p"] = float(p.sum(dim=1).mean().item())
    assert dsa.dsa_device_error() == 0
    del p, scores, loss
    torch.cuda.empty_cache()

    # dense warm-up target on the last 1024 query rows of the first sequence (their causal
    # prefixes are the longest); the sparse forward's lse stands in for the dense one (the
    # kernel's cost does not depend on its values)
    L0 = cfg["seqlens"][0]
    R = min(1024, L0)
    pd = torch.empty((R, L0), device="cuda")
    # the indexer backward over every token's selection; the KL gradient is a random stand-in
    H_I, d_I = cfg["H_I"], cfg["d_I"]
    keys = dsa.contiguous_desc(inp["k8"], inp["cu_seqlens"], max(inp["seqlens"]), scale=inp["k_scale"])
    dw = torch.empty((T, H_I), device="cuda")
    dq = torch.empty((T, H_I, d_I), device="cuda")
    dkey = torch.empty((T, d_I), device="cuda")
    grad.normal_()
    for name, fn, reps in (
            ("attn_distribution_dense", lambda: dsa.dsa_attn_distribution_dense(
                inp["q"], lat, lse, nseq, H, L0 - R, L0, sm, pd), 3),
            ("indexer_backward", lambda: dsa.dsa_indexer_backward(
                inp["q8"], inp["q_scale"], inp["w"], keys, nseq, H_I, d_I, idx, grad, dw, dq, dkey), 1)):
        fn()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(reps):
            fn()
        e1.record()
        torch.cuda.synchronize()
        res[name + "_ms"] = e0.elapsed_time(e1) / reps
    dense_pairs = sum(t + 1 for t in range(L0 - R, L0))
    res["attn_distribution_dense_rows"] = f"rows {L0 - R}..{L0 - 1} of a {L0}-token sequence"
    res["attn_distribution_dense_tflops"] = dense_pairs * 2 * H * 576 / (res["attn_distribution_dense_ms"] * 1e-3) / 1e12
    # three fp32 contractions of H_I x d_I per selected (token, key) pair: logits, dq, dk
    bwd_flops = pairs * H_I * d_I * 2 * 3
    res["indexer_backward_tflops_fp32"] = bwd_flops / (res["indexer_backward_ms"] * 1e-3) / 1e12
    # CUDA-core fp32 peak from the unit counts: 148 SMs x 128 FP32 lanes x 2 flops x 1.965 GHz
    res["indexer_backward_frac_of_fp32_alu"] = res["indexer_backward_tflops_fp32"] / (2 * FP32_LANE_OPS_T)
    assert dsa.dsa_device_error() == 0
    del pd, dw, dq, dkey, grad, lse
    torch.cuda.empty_cache()
    return res


def run_decode(args, dsa, sm, peaks):
    cfg = dict(synth.WORKLOADS[DECODE])
    d = synth.decode_inputs(device="cuda", **cfg)
    B, k = d["B"], cfg["k"]
    keys = dsa.paged_desc(d["kcache8"], d["block_table"], d["ctx"], d["max_ctx"], scale=d["kscale_cache"])
    lat = dsa.paged_desc(d["latent_cache"], d["block_table"], d["ctx"], d["max_ctx"])
    ws = torch.empty(dsa.dsa_workspace_size(dsa.DSA_MODE_DECODE, B, 0, d["max_ctx"], 128, k), dtype=torch.uint8,
                     device="cuda")
    out = torch.empty((B, 128, 512), dtype=torch.bfloat16, device="cuda")

    def step():
        dsa.dsa_forward(dsa.DSA_MODE_DECODE, d["q8"], d["q_scale"], d["w"], keys, d["q"], lat, B, 64, 128, 128, k, sm,
                        out, None, None, ws)

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize()
    n = max(10, args.steps)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(n):
        step()
    e1.record()
    torch.cuda.synchronize()
    assert dsa.dsa_device_error() == 0
    ms = e0.elapsed_time(e1) / n
    keys_scanned = int(sum(d["ctx_host"]))

    # the same chain call by call, each call bracketed by events on the launching stream; the
    # paged scan alone (dsa_indexer_scores) is timed beside the fused selection call, whose
    # selection kernel takes the difference
    ld = (d["max_ctx"] + 3) // 4 * 4
    S = torch.empty((B, ld), device="cuda")
    idx = torch.empty((B, k), dtype=torch.int32, device="cuda")
    ws_sel = torch.empty(dsa.dsa_decode_select_workspace_size(B, d["max_ctx"]), dtype=torch.uint8, device="cuda")
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(n)]
    for i in range(-3, n):
        e = ev[i] if i >= 0 else None
        if e:
            e[0].record()
        dsa.dsa_indexer_scores(d["q8"], d["q_scale"], d["w"], keys, B, 64, 128, 0, B, S)
        if e:
            e[1].record()
        dsa.dsa_indexer_topk_decode(d["q8"], d["q_scale"], d["w"], keys, B, 64, 128, k, idx, ws_sel)
        if e:
            e[2].record()
        dsa.dsa_sparse_mla_decode(d["q"], lat, idx, B, 128, k, sm, out, None, ws)
        if e:
            e[3].record()
    torch.cuda.synchronize()
    assert dsa.dsa_device_error() == 0
    t = [float(np.mean([e[j].elapsed_time(e[j + 1]) for e in ev])) for j in range(3)]
    hbm = peaks["hbm_gbs"]
    # algorithmic bytes: the paged scan reads 132 B per cached key (e4m3 key + fp32 scale) and
    # each query's q_I, w and scale, and writes a 4-byte score per key (and, in the fused call, a
    # 4-byte maximum per 16 keys); the selection reads the scores and maxima once and writes the
    # selection; sparse MLA gathers 1152 B per selected row and reads q, writes out
    q_bytes = B * (64 * 128 + 64 * 4 + 4)
    idx_bytes = keys_scanned * (132 + 4) + q_bytes
    sel_bytes = keys_scanned * (132 + 4 + 0.25 + 4 + 0.25) + q_bytes + B * k * 4
    mla_bytes = B * k * 1152 + B * 128 * 576 * 2 + B * 128 * 512 * 2 + B * k * 4
    mla_flops = B * k * 278528
    kernels = {
        "indexer_scores": {"ms": t[0], "bytes": idx_bytes, "gbs": idx_bytes / (t[0] * 1e-3) / 1e9},
        "indexer_topk_decode": {"ms": t[1], "bytes": sel_bytes, "gbs": sel_bytes / (t[1] * 1e-3) / 1e9,
                                "selection_ms": t[1] - t[0]},
        "sparse_mla_decode": {"ms": t[2], "bytes": mla_bytes, "gbs": mla_bytes / (t[2] * 1e-3) / 1e9,
                              "tflops": mla_flops / (t[2] * 1e-3) / 1e12,
                              "frac_of_bf16": mla_flops / (t[2] * 1e-3) / 1e12 / peaks["bf16_tflops"]},
    }
    for kk in kernels.values():
        kk["frac_of_hbm"] = kk["gbs"] / hbm
    res = {"workload": f"{DECODE}: 64 sequences, ctx ~ U[8192,131072] (sum {keys_scanned}), paged 64-token blocks",
           "value": B / (ms * 1e-3), "unit": "tokens/s", "ms_per_step": ms, "steps": n,
           "kernels": kernels, "peaks": {"hbm_gbs": hbm, "bf16_tflops": peaks["bf16_tflops"],
                                         "note": "measured; burst bf16 (kernels timed alone)"},
           "gpu_launches_per_step": 3 if B * 2 > 74 else 4}
    if not args.no_cpu_baseline:
        res["cpu_baseline"] = oracle_decode_sample(d, k, sm, args.cpu_decode_seqs)
    return res


def oracle_decode_sample(d, k, sm, nseq):
    """The oracle's decode step (paged indexer over the whole context, top-k, sparse MLA) on the
    first nseq sequences of the decode workload (all 64 by default: the step in full), timed on
    the host, one sequence at a time (its host copy is made outside the timed region);
    tokens/s = nseq / time."""
    import oracle
    secs = 0.0
    for b in range(nseq):
        seq = synth.decode_seq_numpy(d, b)
        t0 = time.perf_counter()
        oracle.dsa_decode(seq, k, sm)
        secs += time.perf_counter() - t0
        del seq
    full = nseq == d["B"]
    ctx = sum(int(d["ctx_host"][b]) for b in range(nseq))
    return {"value": nseq / secs, "unit": "tokens/s", "cores": blas_threads(), "host_cores": os.cpu_count(),
            "kind": "oracle",
            "sample": (f"the whole decode step: all {nseq} sequences" if full else f"{nseq} of the {d['B']} sequences")
                      + f" ({ctx} context keys), one decode token each, {secs:.1f} s"}


def oracle_prefill_full(cfg, sm, block=512):
    """The oracle on every query row of a prefill workload (tiny_256, prefill_8k), in row blocks of
    `block` rows to bound host memory; tokens/s = L / time (host copies outside the timed region)."""
    import oracle
    inp = synth.prefill_inputs(device="cuda", **cfg)
    L, k = cfg["seqlens"][0], cfg["k"]
    secs = 0.0
    for r0 in range(0, L, block):
        rows = list(range(r0, min(L, r0 + block)))
        seq = synth.seq_slice_numpy(inp, 0, rows=rows)
        t0 = time.perf_counter()
        oracle.dsa_prefill_rows(seq, k, sm, rows)
        secs += time.perf_counter() - t0
        del seq
    del inp
    torch.cuda.empty_cache()
    return {"value": L / secs, "unit": "tokens/s", "cores": blas_threads(), "host_cores": os.cpu_count(),
            "kind": "oracle", "sample": f"the whole L={L} prefill, every query row, {secs:.1f} s"}


def run_e2e(args, dsa, inp, cfg, sm, n_blocks=32):
    """The prefill end to end from pinned host memory: every step copies all of its inputs in
    and its output back.  A step is pipelined over query-row blocks of the sequence on three
    streams -- the key-side inputs (k_I, k_scale, latent) first, then per block the copy-in of
    its query-side rows, the fused indexer top-k and sparse MLA of those rows
    (dsa_indexer_topk_rows, dsa_sparse_mla_prefill_rows) and the copy-out of its output -- so
    that both copy directions overlap the kernels.  The device-side inputs and outputs are
    double-buffered, so step i+1 starts copying in while step i still computes and copies out;
    events keep each buffer's reuse behind the step that used it two steps before."""
    assert len(cfg["seqlens"]) == 1, "the pipelined step shards one sequence by rows"
    key_names = ["k8", "k_scale", "latent", "cu_seqlens"]
    row_names = ["q8", "q_scale", "w", "q"]
    host = {}
    for n in key_names + row_names:
        t = inp[n]
        try:
            h = torch.empty(t.shape, dtype=t.dtype, pin_memory=True)
        except RuntimeError:
            h = torch.empty(t.shape, dtype=t.dtype)
        h.copy_(t)
        host[n] = h
    T, H, k, H_I, d_I = inp["q"].shape[0], cfg["H"], cfg["k"], cfg["H_I"], cfg["d_I"]
    bufs = []
    for _ in range(2):
        dev = {n: torch.empty_like(inp[n]) for n in key_names + row_names}
        bufs.append({"dev": dev,
                     "out": torch.empty((T, H, 512), dtype=torch.bfloat16, device="cuda"),
                     "idx": torch.empty((T, k), dtype=torch.int32, device="cuda"),
                     "keys": dsa.contiguous_desc(dev["k8"], dev["cu_seqlens"], T, scale=dev["k_scale"]),
                     "lat": dsa.contiguous_desc(dev["latent"], dev["cu_seqlens"], T),
                     "inputs_free": None, "out_free": None})
    try:
        out_h = torch.empty((T, H, 512), dtype=torch.bfloat16, pin_memory=True)
    except RuntimeError:
        out_h = torch.empty((T, H, 512), dtype=torch.bfloat16)
    h2d = sum(host[n].numel() * host[n].element_size() for n in key_names + row_names)
    d2h = out_h.numel() * out_h.element_size()
    bounds = [T * b // n_blocks for b in range(n_blocks + 1)]
    s_in, s_run, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    main = torch.cuda.current_stream()
    for s in (s_in, s_run, s_out):
        s.wait_stream(main)

    def step(i):
        B = bufs[i & 1]
        dev, out, idx = B["dev"], B["out"], B["idx"]
        with torch.cuda.stream(s_in):
            if B["inputs_free"] is not None:
                s_in.wait_event(B["inputs_free"])      # the step two back has finished reading them
            for n in key_names:
                dev[n].copy_(host[n], non_blocking=True)
            keys_in = torch.cuda.Event()
            keys_in.record(s_in)
        s_run.wait_event(keys_in)
        if B["out_free"] is not None:
            s_run.wait_event(B["out_free"])            # the step two back has copied its output out
        for b in range(n_blocks):
            r0, r1 = bounds[b], bounds[b + 1]
            with torch.cuda.stream(s_in):
                for n in row_names:
                    dev[n][r0:r1].copy_(host[n][r0:r1], non_blocking=True)
                rows_in = torch.cuda.Event()
                rows_in.record(s_in)
            with torch.cuda.stream(s_run):
                s_run.wait_event(rows_in)
                dsa.dsa_indexer_topk_rows(dev["q8"][r0:r1], dev["q_scale"][r0:r1], dev["w"][r0:r1], B["keys"], H_I,
                                          d_I, k, r0, r1, idx[r0:r1])
                dsa.dsa_sparse_mla_prefill_rows(dev["q"][r0:r1], B["lat"], idx[r0:r1], H, k, sm, r0, r1, out[r0:r1])
                done = torch.cuda.Event()
                done.record(s_run)
            with torch.cuda.stream(s_out):
                s_out.wait_event(done)
                out_h[r0:r1].copy_(out[r0:r1], non_blocking=True)
        B["inputs_free"] = torch.cuda.Event()
        B["inputs_free"].record(s_run)
        B["out_free"] = torch.cuda.Event()
        B["out_free"].record(s_out)

    def drain():
        for s in (s_in, s_run, s_out):
            main.wait_stream(s)

    step(0)
    drain()
    torch.cuda.synchronize()
    # the pipelined result equals the device-resident path's on sampled rows
    rows = torch.linspace(0, T - 1, 8).long().tolist()
    check = torch.stack([out_h[r] for r in rows]).to("cuda")
    n = max(2, min(max(args.steps, 4), args.e2e_steps))
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for s in (s_in, s_run, s_out):
        s.wait_stream(main)
    for i in range(1, n + 1):
        step(i)
    drain()
    e1.record()
    torch.cuda.synchronize()
    assert dsa.dsa_device_error() == 0
    ms = e0.elapsed_time(e1) / n
    return {"value": T / (ms * 1e-3), "unit": "tokens/s", "ms_per_step": ms, "steps": n,
            "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
            "pinned": bool(host["q"].is_pinned()),
            "pipeline": f"{n_blocks} query-row blocks, 3 streams, double-buffered across steps",
            "_check_rows": rows, "_check": check}


# ------------------------------------------------------------------------------------------
# reference arm: the oracle, on the host cores
# ------------------------------------------------------------------------------------------
def run_reference(args, world, rank):
    if rank != 0:
        return
    cfg = dict(synth.WORKLOADS[PREFILL])
    k, sm = cfg["k"], 1.0 / math.sqrt(576)
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    inp = synth.prefill_inputs(device=dev, **cfg)
    L = cfg["seqlens"][0]
    per_step = args.ref_rows
    rs = np.random.default_rng(0)
    times = []
    for i in range(args.warmup + args.steps):
        rows = sorted(rs.choice(L, size=per_step, replace=False).tolist())
        secs = oracle_prefill_sample(inp, k, rows, sm)
        if i >= args.warmup:
            times.append(secs)
    ms = 1e3 * float(np.mean(times))
    value = per_step / (ms * 1e-3)
    cores = blas_threads()
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": prefill_config(PREFILL, world, cfg),
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "host_cores": os.cpu_count(), "kind": "oracle",
                             "sample": f"{per_step} random query rows per step of the L=131072 prefill (each row's "
                                       "whole causal prefix: indexer, top-k, attention); tokens/s = rows / time"},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=4)
    ap.add_argument("--cpu-rows", type=int, default=256)
    ap.add_argument("--cpu-decode-seqs", type=int, default=64,
                    help="decode sequences the oracle baseline runs (64 = the whole decode_64 step)")
    ap.add_argument("--cpu-c2-full", action="store_true",
                    help="also time the oracle on the whole prefill_8k workload (about two minutes of CPU)")
    ap.add_argument("--ref-rows", type=int, default=2)
    ap.add_argument("--workload", default=PREFILL, choices=[w for w, c in synth.WORKLOADS.items() if c["kind"] == "prefill"],
                    help="prefill workload of the timed step (the headline is prefill_128k; smaller ones are for profiling)")
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--profile-case", choices=["rows_128k", "decode_8x128k", "decode_64", "indexer_128k",
                                                  "mla_quarters_128k"], default=None,
                    help="run one small case of the kernels for a counter capture and exit")
    ap.add_argument("--idx-ms", type=float, default=142.0,
                    help="--strong: measured time of the fused indexer top-k over the whole sequence")
    ap.add_argument("--mla-ms", type=float, default=93.0,
                    help="--strong: measured time of sparse MLA over the whole sequence")
    ap.add_argument("--strong", action="store_true",
                    help="shard ONE sequence over the ranks by query rows (strong scaling) instead of one problem per rank")
    args = ap.parse_args()
    if args.warmup < 3:
        log("warm-up raised to the minimum of 3 steps")
        args.warmup = 3
    if args.impl == "reference":  # rank 0 runs the oracle; other ranks exit without work
        run_reference(args, int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")))
        return
    world, rank, local = dist_setup(args)
    if args.profile_case is not None:
        import sparse_attention_09_b200 as dsa
        run_profile_case(args, dsa, 1.0 / math.sqrt(576))
        return
    if args.strong:
        run_strong(args, world, rank, local)
    else:
        run_ours(args, world, rank, local)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
