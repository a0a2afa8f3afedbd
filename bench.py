"""Benchmark: CSA2 decode over an NVFP4 main-KV cache at 1M context, batch 8.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference] [--config 2|3|4|6]

One step = one FP4 quant-append of the new token of every sequence + the 20
decoder layers (Full + 3 Reuse, then 4 x (Reindex + 3 Reuse)), each layer
launched on its own through the C ABI, captured once in a CUDA graph.  The
cache (8 x 1,048,576 entries, random page permutation, 64-entry pages) is filled
before timing; L2 is flushed (a 256 MiB write, not timed) before every timed
step.  Prints one JSON line (rank 0).

Multi-GPU: one process per GPU (torchrun), each rank runs its own batch of 8
sequences (weak scaling, no collective on the data path); the step time is the
max over ranks.

--config 3 times a prefill chunk instead; --config 6 the encoder side of one
generated token: 18 ratio-2 layers (3 x (Full + 5 Reuse)) whose Full layers
select over every entry (8 x 524,288 entries = 1M tokens each).  --kv-host keeps
the main KV in pinned host memory (the decode driver stages each index set's
rows on the device once).

--impl reference times the CPU oracle (the plain C restatement of the method)
on the host cores on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "CSA2 decode attn tokens/s @1M ctx & achieved HBM GB/s (fraction of roofline)"
METRIC_ENC = "CSA2 encoder-side decode tokens/s @1M ctx (18 ratio-2 layers, flat indexer)"
UNIT = "tokens/s"
PAGE = 64
CH = 256


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=200)
    p.add_argument("--warmup", type=int, default=20)
    p.add_argument("--impl", default="cuda", choices=["cuda", "reference"])
    p.add_argument("--config", type=int, default=4, choices=[2, 3, 4, 6])
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-prefill", action="store_true", help="skip the prefill chunk timed beside the decode step")
    p.add_argument("--no-replay", action="store_true", help="skip the SWA replay timed beside the decode step")
    p.add_argument("--launch-floor", action="store_true",
                   help="time chains of empty dependent kernels in one CUDA graph (the launch floor)")
    p.add_argument("--kernel-reps", type=int, default=300)
    p.add_argument("--contiguous-pages", action="store_true")
    p.add_argument("--batch", type=int, default=0, help="override the batch (profiling runs)")
    p.add_argument("--seq-len", type=int, default=0, help="override the context (profiling runs)")
    p.add_argument("--breakdown", action="store_true", help="also time every call of the step on its own")
    p.add_argument("--kv-host", action="store_true",
                   help="main KV (codes, scales) in pinned host memory, read in place (decode configs)")
    return p.parse_args()


def workload(cfg_id: int) -> dict:
    import synth
    c = synth.CONFIGS[cfg_id]
    return dict(workload=c["name"], L=c["L"], B=c["B"], layers=c["layers"], seed=c["seed"],
                ratio=c.get("ratio", 1), decoder=c.get("decoder", True))


def unique_bytes_per_seq(L: int, layers: int = 20) -> dict:
    """Algorithmic bytes one decode step must move for one sequence (each byte
    counted once per step)."""
    nblk = (L + 7) // 8
    blk = nblk * 128 if nblk > 2048 else 0
    tok = min(L, 16384) * 128
    n_sets = 5  # Full + 4 Reindex layers
    kv = n_sets * min(512, L) * 144
    swa = layers * min(128, L) * 512
    append = 256 * 4 + 64 * 2 + 144 + 128
    q = layers * 16 * 128 * 2 + n_sets * (4 * 64 * 2 + 16)
    out = layers * (16 * 128 * 4 + 16 * 4)
    return dict(block=blk, token=tok, kv=kv, swa=swa, append=append, q=q, out=out,
                total=blk + tok + kv + swa + append + q + out)


def unique_bytes_per_seq_flat(L: int, layers: int, n_full: int, ratio: int = 2) -> dict:
    """Algorithmic bytes of one encoder-side decode step for one sequence:
    every Full layer reads the whole indexer K (it does not fit in L2, so each
    of the n_full passes counts), then gathers its 512 FP4 entries."""
    idx = n_full * L * 128
    kv = n_full * min(512, L) * 144
    swa = layers * min(128, L) * 512
    append = ratio * 256 * 4 + 64 * 2 + 144 + 128
    q = layers * 16 * 128 * 2 + n_full * (4 * 64 * 2 + 16)
    out = layers * (16 * 128 * 4 + 16 * 4)
    return dict(index=idx, kv=kv, swa=swa, append=append, q=q, out=out, total=idx + kv + swa + append + q + out)


def attn_bytes_per_row(L: int) -> int:
    """Algorithmic bytes of one decode row (sequence) of one attention launch:
    the selected FP4 entries, the SWA window, q, the index set, out and lse."""
    return min(512, L) * 144 + min(128, L) * 512 + 16 * 128 * 2 + 512 * 4 + 16 * 128 * 4 + 16 * 4


# dram__bytes_read.sum + dram__bytes_write.sum of one decode_attn_kernel launch
# (a Reuse layer) from an ncu capture of the current kernel source, keyed by
# (B, L): taken at B = 2 (518,144 B read, 0 B written) and scaled by the rows
ATTN_TRAFFIC = {(8, 1 << 20): 4 * 518144}
# dram__bytes_read.sum + dram__bytes_write.sum of one flat indexer launch
# (block_score_kernel + block_select_kernel<1>) keyed by (B, entries), taken at
# B = 2 (140,038,400 B) and scaled by the rows scored
FLAT_TRAFFIC = {(8, 1 << 19): 4 * 140038400}


class ClockSampler:
    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = os.path.join(tempfile.gettempdir(), f"csa2_clocks_{os.getpid()}.csv")

    def __enter__(self):
        os.makedirs(os.path.dirname(self.path), exist_ok=True)
        q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={q}", "--format=csv,noheader,nounits",
                                          "-lms", "100", "-i", str(self.index)], stdout=self.f,
                                         stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            self.f.close()

    def summary(self) -> dict:
        if self.proc is None or not os.path.exists(self.path):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        sm, smax, reasons, power = [], None, set(), []
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm.append(float(parts[1]))
                    smax = float(parts[2])
                    power.append(float(parts[3]))
                except ValueError:
                    continue
                for n, v in zip(names, parts[5:9]):
                    if v.lower().startswith("active"):
                        reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": smax, "reasons": ["no samples"]}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": smax, "reasons": sorted(reasons),
                "samples": len(sm), "power_w_max": max(power) if power else None}


# ---------------------------------------------------------------------------
# CUDA arm
# ---------------------------------------------------------------------------

def run_cuda(args, rank: int, world: int, local_rank: int):
    import torch
    import synth
    import fp4_kv_cache_nvfp4_b200 as csa2

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    csa2.lib()
    W = workload(args.config)
    if args.batch:
        W["B"] = args.batch
    if args.seq_len:
        W["L"] = args.seq_len
    if args.batch or args.seq_len:
        W["workload"] += f"-override-b{W['B']}-l{W['L']}"
    B, L, layers, seed = W["B"], W["L"], W["layers"], W["seed"] + 100 * rank
    ratio, flat = W["ratio"], not W["decoder"]  # flat: the encoder's layers (no block level)
    gen = torch.Generator(device=dev)
    gen.manual_seed(seed)

    # ---- cache: B sequences of L entries, pages permuted ----------------------
    lens = np.full(B, L, np.int64)
    table, n_phys = synth.page_table(seed, lens, PAGE, shuffle=not args.contiguous_pages)
    cache = csa2.KVCache(n_phys, PAGE, torch.from_numpy(table), device=dev, main_kv_on_host=args.kv_host)
    gain = torch.from_numpy(synth.gain(seed)).to(dev)
    tab_d = torch.from_numpy(table).to(dev).long()
    chunk = 1 << 16
    for b in range(B):
        for s0 in range(0, L, chunk):
            m = min(chunk, L - s0)
            pos = torch.arange(s0, s0 + m, device=dev)
            slots = (tab_d[b, pos // PAGE] * PAGE + pos % PAGE).contiguous()
            kv = torch.randn((m * ratio, CH), generator=gen, device=dev) * gain
            ik = torch.randn((m, 64), generator=gen, device=dev).to(torch.bfloat16).view(torch.int16)
            csa2.kv_quant_append(cache, kv, ik, slots, ratio=ratio)
    torch.cuda.synchronize()

    # ---- per-layer inputs -------------------------------------------------------
    modes = csa2.schedule(not flat)[:layers]
    descs = [csa2.default_desc(m, ratio, **({"keep_blocks": 0} if flat else {})) for m in modes]
    n_idx = sum(1 for m in modes if m != csa2.REUSE)
    # one packed device buffer holds every per-step input, so one H2D copy refreshes it
    # (swa_new: every layer's newest SWA row; the end-to-end run scatters it into the rings)
    sizes = dict(q=layers * B * 16 * 128 * 2, qi=layers * B * 4 * 64 * 2, w=layers * B * 4 * 4, kv=B * ratio * CH * 4,
                 ik=B * 64 * 2, swa_new=layers * B * CH * 2)
    offs, o = {}, 0
    for k, v in sizes.items():
        offs[k] = o
        o += (v + 255) // 256 * 256
    step_in = torch.empty(o, dtype=torch.uint8, device=dev)

    def view(k, shape, dtype):
        return step_in[offs[k]:offs[k] + sizes[k]].view(dtype).view(shape)

    q_all = view("q", (layers, B, 16, 128), torch.int16)
    qi_all = view("qi", (layers, B, 4, 64), torch.int16)
    w_all = view("w", (layers, B, 4), torch.float32)
    kv_new = view("kv", (B * ratio, CH), torch.float32)  # ratio source rows per appended entry
    ik_new = view("ik", (B, 64), torch.int16)
    q_all.copy_(torch.randn(q_all.shape, generator=gen, device=dev).to(torch.bfloat16).view(torch.int16))
    qi_all.copy_(torch.randn(qi_all.shape, generator=gen, device=dev).to(torch.bfloat16).view(torch.int16))
    w_all.copy_(torch.rand(w_all.shape, generator=gen, device=dev))
    kv_new.copy_(torch.randn(kv_new.shape, generator=gen, device=dev) * gain)
    ik_new.copy_(torch.randn(ik_new.shape, generator=gen, device=dev).to(torch.bfloat16).view(torch.int16))
    swa = torch.randn((layers, B, 128, CH), generator=gen, device=dev).mul_(gain).to(torch.bfloat16).view(
        torch.int16).contiguous()
    seq_lens = torch.full((B,), L, dtype=torch.int32, device=dev)
    pos_new = torch.full((B,), L - 1, dtype=torch.int64, device=dev)  # the step (re)writes the newest entry
    slot_new = (tab_d[torch.arange(B, device=dev), pos_new // PAGE] * PAGE + pos_new % PAGE).contiguous()
    outs = [torch.empty((B, 16, 128), dtype=torch.float32, device=dev) for _ in range(layers - 1)]
    lses = [torch.empty((B, 16), dtype=torch.float32, device=dev) for _ in range(layers - 1)]
    # the step's result (last layer's out and lse) in one buffer: one device-to-host copy
    result = torch.empty(B * 16 * 128 + B * 16, dtype=torch.float32, device=dev)
    outs.append(result[:B * 16 * 128].view(B, 16, 128))
    lses.append(result[B * 16 * 128:].view(B, 16))
    cand = None if flat else torch.empty((B, 2048), dtype=torch.int32, device=dev)
    sets = torch.empty((layers, B, 512), dtype=torch.int32, device=dev)
    ws = torch.zeros(csa2.workspace_bytes(descs[0], csa2.TOKEN if flat else csa2.BLOCK, B, L), dtype=torch.uint8,
                     device=dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)

    stream = torch.cuda.Stream(device=dev)

    def step():
        csa2.kv_quant_append(cache, kv_new, ik_new, slot_new, ratio=ratio, err=err, stream=stream)
        csa2.decode_layers(descs, cache, [qi_all[l] for l in range(layers)], [w_all[l] for l in range(layers)],
                           [q_all[l] for l in range(layers)], [swa[l] for l in range(layers)], seq_lens, cand, sets,
                           outs, lses, B, L, ws, err=err, stream=stream)

    # eager run, then capture
    with torch.cuda.stream(stream):
        step()
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        step()
    torch.cuda.synchronize()
    if flat:  # Full: block_score + block_select over entries (token score + select at <= 16,384), then attention
        launches_per_step = 1 + sum(3 if m != csa2.REUSE else 1 for m in modes)
    else:
        launches_per_step = 1 + sum({csa2.FULL: 5, csa2.REINDEX: 3, csa2.REUSE: 1}[m] for m in modes)
    if args.kv_host:  # each new index set's rows are staged on the device once
        launches_per_step += n_idx

    def barrier():
        if world > 1:
            torch.distributed.barrier()

    sampler = ClockSampler(local_rank)
    with sampler:
        with torch.cuda.stream(stream):
            for _ in range(max(args.warmup, 3)):
                graph.replay()
        torch.cuda.synchronize()
        # ---- timed: K steps, L2 flushed before each (flush not timed) ---------
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
        barrier()
        torch.cuda.synchronize()
        with torch.cuda.stream(stream):
            for k in range(args.steps):
                flush.fill_(k & 0xFF)
                ev[k][0].record(stream)
                graph.replay()
                ev[k][1].record(stream)
        torch.cuda.synchronize()
        barrier()
        step_ms = [a.elapsed_time(b) for a, b in ev]
        total_ms = max_over_ranks(sum(step_ms), world, dev)
        ms_per_step = total_ms / args.steps

        # ---- per-kernel rooflines: each launch timed alone between CUDA events,
        # after an untimed L2 flush, on the stream it is launched on ------------
        def time_launches(fn):
            ev_ = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                   for _ in range(args.kernel_reps)]
            with torch.cuda.stream(stream):
                for k in range(args.kernel_reps):
                    flush.fill_(k & 0xFF)
                    ev_[k][0].record(stream)
                    fn()
                    ev_[k][1].record(stream)
            torch.cuda.synchronize()
            return statistics.mean(a.elapsed_time(b) for a, b in ev_)

        # dominant kernel by share of the step: sparse attention (20 launches a
        # step); a Reuse layer's launch on the Full layer's index set
        reuse = next(l for l, m in enumerate(modes) if m == csa2.REUSE)
        a_ms = time_launches(lambda: csa2.sparse_attn_decode(descs[reuse], cache, q_all[reuse], sets[0], swa[reuse],
                                                             seq_lens, outs[reuse], lses[reuse], B, err=err,
                                                             stream=stream))
        # largest single HBM stream: the block-level indexer (scoring + select),
        # or the flat indexer over every entry of the encoder's Full layers
        if flat:
            k_ms = time_launches(lambda: csa2.indexer_topk(descs[0], cache, csa2.TOKEN, qi_all[0], w_all[0],
                                                           seq_lens, sets[0], B, L, ws, err=err, stream=stream))
        else:
            k_ms = time_launches(lambda: csa2.indexer_topk(descs[0], cache, csa2.BLOCK, qi_all[0], w_all[0],
                                                           seq_lens, cand, B, L, ws, err=err, stream=stream))

        # ---- end to end: pinned host inputs -> device, step, result -> host ----
        # one H2D copy of the packed inputs (q, q_idx, w, the appended entry and
        # every layer's newest SWA row), one strided device copy of those rows
        # into their ring slots, the step, one D2H copy of out and lse
        ring = (L - 1) % 128
        view("swa_new", (layers, B, CH), torch.int16).copy_(swa[:, :, ring, :])
        host_in = torch.empty(step_in.numel(), dtype=torch.uint8, pin_memory=True)
        host_in.copy_(step_in.cpu())
        host_res = torch.empty(result.numel(), dtype=torch.float32, pin_memory=True)
        swa_new = view("swa_new", (layers, B, CH), torch.int16)
        e2e_steps = max(10, min(args.steps, 100))
        eev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(e2e_steps)]
        with torch.cuda.stream(stream):
            for k in range(e2e_steps):
                flush.fill_(k & 0xFF)
                eev[k][0].record(stream)
                step_in.copy_(host_in, non_blocking=True)
                swa[:, :, ring, :].copy_(swa_new, non_blocking=True)
                graph.replay()
                host_res.copy_(result, non_blocking=True)
                eev[k][1].record(stream)
        torch.cuda.synchronize()
        e2e_ms = statistics.mean(a.elapsed_time(b) for a, b in eev)
    clocks = sampler.summary()
    assert int(err.item()) == 0, f"device error flags {int(err.item())}"
    breakdown = _breakdown(csa2, cache, descs, modes, qi_all, w_all, q_all, swa, seq_lens, cand, sets, outs, lses,
                           kv_new, ik_new, slot_new, ws, err, flush, stream, B, L, ratio,
                           flat) if args.breakdown else None

    h2d = step_in.numel()
    d2h = host_res.numel() * 4
    n_full = sum(1 for m in modes if m != csa2.REUSE)
    ub = unique_bytes_per_seq_flat(L, layers, n_full, ratio) if flat else unique_bytes_per_seq(L, layers)
    peaks = _peaks()
    hbm = peaks.get("hbm_gbs")
    k_bytes = B * (L if flat else (L + 7) // 8) * 128
    k_gbs = k_bytes / (k_ms * 1e-3) / 1e9
    a_bytes = B * attn_bytes_per_row(L)
    a_gbs = a_bytes / (a_ms * 1e-3) / 1e9
    peak_src = ("MEASURED_PEAKS.json hbm_gbs (measured, burst copy)" if peaks.get("source") == "measured"
                else "fallback 6650 GB/s (MEASURED_PEAKS.json absent)")
    attn_roof = dict(kernel="decode_attn_kernel (Reuse layer, B rows x 8 CTAs)", bound="hbm", achieved=a_gbs,
                     peak=hbm, unit="GB/s", frac=a_gbs / hbm if hbm else None, traffic=ATTN_TRAFFIC.get((B, L)),
                     bytes_per_launch=a_bytes, ms_per_launch=a_ms, peak_source=peak_src)
    idx_roof = dict(kernel="block_score_kernel + block_select_kernel" + (" over entries (flat indexer)" if flat else ""),
                    bound="hbm", achieved=k_gbs, peak=hbm, unit="GB/s", frac=k_gbs / hbm if hbm else None,
                    traffic=FLAT_TRAFFIC.get((B, L)) if flat else None, bytes_per_launch=k_bytes, ms_per_launch=k_ms,
                    peak_source=peak_src)
    schedule = "encoder: 3 x (F+5R), ratio 2, flat indexer" if flat else "decoder: F+3R, 4x(RI+3R)"
    res = dict(metric=METRIC_ENC if flat else METRIC, value=whole_job_tokens_per_s(B, world, ms_per_step), unit=UNIT,
               n_gpus=world, steps=args.steps,
               warmup=args.warmup, ms_per_step=ms_per_step, higher_is_better=True, scaling="weak",
               vs_baseline=None, dtype="fp4(e2m1)+e4m3 cache; bf16 q/idx; fp32 accumulate", data="synthetic",
               config=dict(workload=W["workload"], seq_len=L * ratio, entries=L, ratio=ratio, batch_per_gpu=B,
                           global_batch=world * B, layers=layers, schedule=schedule, page_size=PAGE,
                           pages="contiguous" if args.contiguous_pages else "random permutation",
                           l2="flushed before every timed step (256 MiB write, not timed)", parallelism=f"dp{world}",
                           kv_placement=("main KV (FP4 codes, E4M3 scales) in pinned host memory, read in "
                                         "place; indexer K and SWA rows in device memory"
                                         if args.kv_host else "device memory"),
                           graph="one CUDA graph per step, programmatic dependent launch between kernels"),
               step_bytes_unique=B * ub["total"], step_gbs=B * ub["total"] / (ms_per_step * 1e-3) / 1e9,
               step_frac_of_hbm=(B * ub["total"] / (ms_per_step * 1e-3) / 1e9) / hbm if hbm else None,
               e2e=dict(value=whole_job_tokens_per_s(B, world, max_over_ranks(e2e_ms, world, dev)), unit=UNIT,
                        h2d_bytes_per_step=h2d, d2h_bytes_per_step=d2h,
                        ms_per_step=e2e_ms),
               gpu_launches=launches_per_step * args.steps, launches_per_step=launches_per_step,
               clocks=clocks)
    if flat:  # the flat indexer's full scans dominate the encoder's step
        res["roofline"], res["roofline_attention"] = idx_roof, attn_roof
    else:
        res["roofline"], res["roofline_block_indexer"] = attn_roof, idx_roof
    if breakdown is not None:
        res["breakdown_us"] = breakdown
    return res


def _breakdown(csa2, cache, descs, modes, qi_all, w_all, q_all, swa, seq_lens, cand, sets, outs, lses, kv_new,
               ik_new, slot_new, ws, err, flush, stream, B, L, ratio=1, flat=False, reps=50):
    """Every call of the step timed on its own with CUDA events (mean over
    reps), once after an L2 flush (cold) and once right after the same call
    (warm)."""
    import torch
    full = descs[0]
    reuse = next(d for d, m in zip(descs, modes) if m == csa2.REUSE)
    calls = {"quant_append (B entries)": lambda: csa2.kv_quant_append(cache, kv_new, ik_new, slot_new, ratio=ratio,
                                                                       err=err, stream=stream)}
    if flat:
        calls["indexer, flat over every entry"] = lambda: csa2.indexer_topk(
            full, cache, csa2.TOKEN, qi_all[0], w_all[0], seq_lens, sets[0], B, L, ws, err=err, stream=stream)
    else:
        rei = next(d for d, m in zip(descs, modes) if m == csa2.REINDEX)
        calls["indexer block level (block_score + block_select)"] = lambda: csa2.indexer_topk(
            full, cache, csa2.BLOCK, qi_all[0], w_all[0], seq_lens, cand, B, L, ws, err=err, stream=stream)
        calls["indexer token level (token_topk)"] = lambda: csa2.indexer_topk(
            rei, cache, csa2.TOKEN, qi_all[4], w_all[4], seq_lens, sets[4], B, L, ws, cand_blocks=cand, err=err,
            stream=stream)
    calls["attention, Full/Reindex layer"] = lambda: csa2.sparse_attn_decode(
        full, cache, q_all[0], sets[0], swa[0], seq_lens, outs[0], lses[0], B, err=err, stream=stream)
    calls["attention, Reuse layer"] = lambda: csa2.sparse_attn_decode(
        reuse, cache, q_all[1], sets[0], swa[1], seq_lens, outs[1], lses[1], B, err=err, stream=stream)
    res = {}
    with torch.cuda.stream(stream):
        for name, fn in calls.items():
            fn()
            out = {}
            for mode in ("cold", "warm"):
                ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps)]
                for k in range(reps):
                    if mode == "cold":
                        flush.fill_(k & 0xFF)
                    else:
                        fn()
                    ev[k][0].record(stream)
                    fn()
                    ev[k][1].record(stream)
                torch.cuda.synchronize()
                out[mode] = round(statistics.mean(a.elapsed_time(b) for a, b in ev) * 1e3, 2)
            res[name] = out
    return res


def max_over_ranks(x: float, world: int, device=None) -> float:
    """The largest value of x over all ranks (the step time of a weak-scaling
    job is its slowest rank's)."""
    if world <= 1:
        return float(x)
    import torch
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def whole_job_tokens_per_s(batch_per_rank: int, world: int, ms_per_step: float) -> float:
    """Tokens decoded per second by all ranks together: each rank decodes its
    own batch of sequences per step."""
    return world * batch_per_rank / (ms_per_step * 1e-3)


def run_prefill(args, rank: int, world: int, local_rank: int):
    """Encoder prefill chunk (config 3): 32,768 tokens of context (16,384
    ratio-2 entries); the step appends the chunk's last 4096 tokens (2048
    entries), runs the Full layer's indexer for the 4096 query tokens and the
    attention of 6 layers (1 Full + 5 Reuse) over their Top-512 + window."""
    import torch
    import synth
    import fp4_kv_cache_nvfp4_b200 as csa2

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    csa2.lib()
    c = synth.CONFIGS[3]
    tokens, T, layers, seed = c["tokens"], c["T"], c["layers"], c["seed"] + 100 * rank
    n_ent, chunk_ent = tokens // 2, T // 2
    gen = torch.Generator(device=dev)
    gen.manual_seed(seed)
    table, n_phys = synth.page_table(seed, [n_ent], PAGE, shuffle=not args.contiguous_pages)
    cache = csa2.KVCache(n_phys, PAGE, torch.from_numpy(table), device=dev, pooled=False)
    gain = torch.from_numpy(synth.gain(seed)).to(dev)
    tab = torch.from_numpy(table).to(dev).long()
    pos = torch.arange(n_ent, device=dev)
    slots = (tab[0, pos // PAGE] * PAGE + pos % PAGE).contiguous()
    kv_all = (torch.randn((tokens, CH), generator=gen, device=dev) * gain).to(torch.bfloat16)
    ik_all = torch.randn((n_ent, 64), generator=gen, device=dev).to(torch.bfloat16).view(torch.int16)
    pre = n_ent - chunk_ent  # entries filled before the timed chunk
    csa2.kv_quant_append(cache, kv_all[:2 * pre], ik_all[:pre], slots[:pre], ratio=2)
    kv_chunk, ik_chunk, sl_chunk = kv_all[2 * pre:], ik_all[pre:], slots[pre:]
    q_pos = torch.arange(tokens - T, tokens, dtype=torch.int32, device=dev)
    bf = lambda shape: torch.randn(shape, generator=gen, device=dev).to(torch.bfloat16).view(torch.int16)  # noqa: E731
    q_idx, w = bf((T, 4, 64)), torch.rand((T, 4), generator=gen, device=dev)
    qs = [bf((T, 16, 128)) for _ in range(layers)]
    swa_start = tokens - T - 127
    swas = [(torch.randn((tokens - swa_start, CH), generator=gen, device=dev) * gain).to(torch.bfloat16)
            .view(torch.int16) for _ in range(layers)]
    d_full = csa2.default_desc(csa2.FULL, 2)
    d_reuse = csa2.default_desc(csa2.REUSE, 2)
    ws = torch.zeros(csa2.workspace_bytes(d_full, csa2.TOKEN, T, n_ent, prefill=True), dtype=torch.uint8,
                     device=dev)
    sets = torch.empty((T, 512), dtype=torch.int32, device=dev)
    outs = [torch.empty((T, 16, 128), device=dev) for _ in range(layers)]
    lses = [torch.empty((T, 16), device=dev) for _ in range(layers)]
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    nl = torch.tensor([n_ent], dtype=torch.int32, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.Stream(device=dev)

    def append():
        csa2.kv_quant_append(cache, kv_chunk, ik_chunk, sl_chunk, ratio=2, err=err, stream=stream)

    def indexer():
        csa2.indexer_topk(d_full, cache, csa2.TOKEN, q_idx, w, nl, sets, T, n_ent, ws, q_pos=q_pos, err=err,
                          stream=stream)

    def attn(l):
        csa2.sparse_attn_prefill(d_full if l == 0 else d_reuse, cache, qs[l], sets, q_pos, swas[l], swa_start, n_ent,
                                 outs[l], lses[l], T, err=err, stream=stream)

    def step():
        append()
        indexer()
        for l in range(layers):
            attn(l)

    with torch.cuda.stream(stream):
        step()
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        step()
    parts = {"append": append, "indexer": indexer, "attention layer (Full)": lambda: attn(0),
             "attention layer (Reuse)": lambda: attn(1)}
    pgraphs = {}
    for name, fn in parts.items():
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            fn()
        pgraphs[name] = g
    sampler = ClockSampler(local_rank)
    with sampler:
        with torch.cuda.stream(stream):
            for _ in range(max(args.warmup, 3)):
                graph.replay()
        torch.cuda.synchronize()
        steps = max(1, min(args.steps, 50))
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
        with torch.cuda.stream(stream):
            for k in range(steps):
                flush.fill_(k & 0xFF)
                ev[k][0].record(stream)
                graph.replay()
                ev[k][1].record(stream)
        torch.cuda.synchronize()
        ms = max_over_ranks(sum(a.elapsed_time(b) for a, b in ev), world, dev) / steps
        part_us = {}
        with torch.cuda.stream(stream):
            for name, g in pgraphs.items():
                pe = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(10)]
                for k in range(10):
                    flush.fill_(k & 0xFF)
                    pe[k][0].record(stream)
                    g.replay()
                    pe[k][1].record(stream)
                torch.cuda.synchronize()
                part_us[name] = round(statistics.mean(a.elapsed_time(b) for a, b in pe) * 1e3, 2)
    assert int(err.item()) == 0, f"device error flags {int(err.item())}"
    peaks = _peaks()
    # tensor work of the attention layers (QK and PV over 512 selected + 128 window keys, 16 heads x 128)
    att_flop = T * 16 * (512 + 128) * 128 * 2 * 2
    idx_flop = sum(min((p + 1) // 2, n_ent) for p in range(tokens - T, tokens)) * 4 * 64 * 2
    att_us = part_us["attention layer (Reuse)"]
    return dict(metric="CSA2 encoder prefill tokens/s (4096-token chunk, 32K context, 1F+5R layers)",
                value=world * T / (ms * 1e-3), unit="tokens/s", n_gpus=world, steps=steps, warmup=args.warmup,
                ms_per_step=ms, higher_is_better=True, scaling="weak", vs_baseline=None,
                dtype="fp4 cache; f16 mma, f32 accumulate; exact f32 indexer", data="synthetic",
                config=dict(workload=c["name"], context_tokens=tokens, chunk=T, entries=n_ent, ratio=2,
                            layers=layers, l2="flushed before every timed step"),
                breakdown_us=part_us,
                tensor=dict(attention_tflops=att_flop / (att_us * 1e-6) / 1e12, attention_flop_per_layer=att_flop,
                            chunk_flop=idx_flop + layers * att_flop,
                            indexer_gflop=idx_flop / 1e9,
                            indexer_tflops=idx_flop / (part_us["indexer"] * 1e-6) / 1e12,
                            peak_bf16_tflops=peaks.get("bf16_tflops")),
                clocks=sampler.summary())


def _peaks() -> dict:
    """Roofline denominators: the measured MEASURED_PEAKS.json when it is
    present (source "measured"), else the pool's earlier measurement (source
    "fallback": 6650 GB/s, 1590 TFLOP/s burst, 1400 sustained)."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        d["source"] = "measured"
        return d
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


# ---------------------------------------------------------------------------
# CPU oracle (reference arm and cpu_baseline)
# ---------------------------------------------------------------------------

def cpu_model() -> str:
    """The host CPU's model name (lscpu's "Model name")."""
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform
    return platform.processor() or "unknown"


def _oracle_cache(orc, seed: int, L: int, ratio: int):
    """One sequence's cache built by the oracle from the seeded generators."""
    import synth
    codes = np.empty((L, 128), np.uint8)
    scales = np.empty((L, 16), np.uint8)
    for e0 in range(0, L, 1 << 16):
        m = min(1 << 16, L - e0)
        codes[e0:e0 + m], scales[e0:e0 + m] = orc.quant_rows(synth.kv_rows(seed, 0, e0 * ratio, m * ratio),
                                                             ratio=ratio)
    return codes, scales, synth.idx_k_rows(seed, 0, 0, L)


def _layer_inputs(seed: int, layers: int, n_seq: int):
    import synth
    q_idx = np.stack([np.concatenate([synth.q_idx(seed, l, b) for l in range(layers)]) for b in range(n_seq)])
    w = np.stack([np.concatenate([synth.w_idx(seed, l, b) for l in range(layers)]) for b in range(n_seq)])
    q = np.stack([np.concatenate([synth.q_heads(seed, l, b) for l in range(layers)]) for b in range(n_seq)])
    swa = np.stack([np.stack([synth.swa_rows(seed, l, b, 128) for l in range(layers)]) for b in range(n_seq)])
    return q_idx, w, q, swa


def oracle_sample(cfg_id: int, budget_s: float = 15.0, max_steps: int = 1000, max_threads: int = 32):
    """Time the oracle's decode step on the host cores: the same step on
    sequences of the workload's length, one sequence per host thread (OpenMP),
    each with a cache of its own."""
    import oracle
    W = workload(cfg_id)
    L, layers, seed, ratio, flat = W["L"], W["layers"], W["seed"], W["ratio"], not W["decoder"]
    n_seq = max(1, min(os.cpu_count() or 1, max_threads))
    # Sequence 0's cache comes from the seeded generators; sequence b's is that
    # cache rotated by b * L / n_seq entries (a multiple of 8, so blocks stay
    # whole), so no two sampled sequences share an entry at any position.
    codes0, scales0, idx0 = _oracle_cache(oracle, seed, L, ratio)
    caches = []
    for b in range(n_seq):
        sh = (b * (L // max(n_seq, 1))) // 8 * 8
        c, s_, k = (np.roll(a, sh, axis=0) for a in (codes0, scales0, idx0))
        caches.append((c, s_, k, oracle.pool_blocks(k)))
    del codes0, scales0, idx0
    modes = oracle.schedule(not flat)[:layers]
    q_idx, w, q, swa = _layer_inputs(seed, layers, n_seq)
    steps, t0 = 0, time.perf_counter()
    while steps < max_steps:
        oracle.decode_batch(modes, [L] * n_seq, [c[0] for c in caches], [c[1] for c in caches],
                            [c[2] for c in caches], [c[3] for c in caches], q_idx, w, q, swa,
                            keep=0 if flat else 2048)
        steps += 1
        if time.perf_counter() - t0 > budget_s:
            break
    dt = time.perf_counter() - t0
    return dict(value=steps * n_seq / dt, unit=UNIT, cores=n_seq, kind="oracle", cpu_model=cpu_model(),
                host_threads=os.cpu_count(),
                sample=f"{steps} decode step(s) x {n_seq} sequences of the {W['workload']} workload "
                       f"({layers} layers, L={L}, a distinct cache per sequence); the quant-append of the step "
                       f"is not in the sample; {dt:.1f} s on {n_seq} of {os.cpu_count()} host threads "
                       f"(one OpenMP thread per sequence)")


def oracle_single_core(cfg_id: int, budget_s: float = 3.0) -> dict:
    """The oracle's decode step of one sequence on one core (no OpenMP)."""
    import oracle
    W = workload(cfg_id)
    L, layers, seed, ratio = W["L"], W["layers"], W["seed"], W["ratio"]
    codes, scales, idx = _oracle_cache(oracle, seed, L, ratio)
    pooled = oracle.pool_blocks(idx)
    modes = oracle.schedule(True)[:layers]
    q_idx, w, q, swa = (a[0] for a in _layer_inputs(seed, layers, 1))
    steps, t0 = 0, time.perf_counter()
    while True:
        oracle.decode_step(modes, L, codes, scales, idx, pooled, q_idx, w, q, swa)
        steps += 1
        if time.perf_counter() - t0 > budget_s:
            break
    dt = time.perf_counter() - t0
    return dict(value=steps / dt, unit=UNIT, cores=1, kind="oracle", ms_per_step=dt / steps * 1e3,
                sample=f"{steps} decode step(s) of one sequence of the {W['workload']} workload ({layers} "
                       f"layer(s), L={L}) on one core")


def oracle_prefill_sample(budget_s: float = 8.0) -> dict:
    """The oracle's prefill (indexer + 6 attention layers) on the host cores,
    timed on a sample of the chunk's queries spread over its positions."""
    import oracle
    import synth
    c = synth.CONFIGS[3]
    tokens, T, layers, seed = c["tokens"], c["T"], c["layers"], c["seed"]
    n_ent = tokens // 2
    codes, scales, idx = _oracle_cache(oracle, seed, n_ent, 2)
    swa_start = tokens - T - 127
    swas = [synth.swa_rows(seed, l, 0, tokens - swa_start) for l in range(layers)]
    done, t0, rounds = 0, time.perf_counter(), 0
    per = 64
    while True:
        lo = (rounds * 997) % (T - per)  # a different slice of the chunk each round
        q_pos = np.arange(tokens - T + lo, tokens - T + lo + per, dtype=np.int32)
        q_idx = synth.q_idx(seed, 0, rounds, per)
        w = synth.w_idx(seed, 0, rounds, per)
        sets = oracle.prefill_indexer(q_pos, 2, n_ent, idx, q_idx, w)
        for l in range(layers):
            oracle.prefill_attn(q_pos, synth.q_heads(seed, l, rounds, per), sets, codes, scales, swas[l], swa_start)
        done += per
        rounds += 1
        if time.perf_counter() - t0 > budget_s:
            break
    dt = time.perf_counter() - t0
    n_thr = min(os.cpu_count() or 1, per)
    return dict(value=done / dt, unit="tokens/s", cores=n_thr, kind="oracle", cpu_model=cpu_model(),
                sample=f"{done} query tokens of the {c['name']} chunk ({rounds} slices of {per}); indexer over "
                       f"the visible entries plus {layers} attention layers each; {dt:.1f} s on {n_thr} of "
                       f"{os.cpu_count()} host threads (OpenMP over the slice's queries)")


def W_DECODER(cfg_id: int) -> bool:
    return bool(workload(cfg_id)["decoder"])


def prefill_summary(p: dict) -> dict:
    """The prefill run's line, condensed into the decode line's "prefill" object."""
    peaks = _peaks()
    sus = peaks.get("bf16_tflops_sustained") or peaks.get("bf16_tflops")
    flop = p["tensor"]["chunk_flop"]
    ach = flop / (p["ms_per_step"] * 1e-3) / 1e12
    return dict(metric=p["metric"], value=p["value"], unit=p["unit"], ms_per_chunk=p["ms_per_step"],
                steps=p["steps"], config=p["config"], breakdown_us=p["breakdown_us"],
                tensor=dict(p["tensor"], chunk_tflops=ach, peak_tflops=sus,
                            peak_source=("MEASURED_PEAKS.json bf16_tflops_sustained (cuBLAS bf16, seconds-long loop)"
                                         if peaks.get("source") == "measured"
                                         else "fallback 1400 TFLOP/s sustained (MEASURED_PEAKS.json absent)"),
                            frac_of_peak=ach / sus if sus else None),
                clocks=p["clocks"])


def run_replay(args, local_rank: int, layers: int = 20, B: int = 8, reps: int = 20) -> dict:
    """SWA Bounded Replay after a miss: every layer's 128-token window of B
    sequences recomputed from synthetic hidden states (d_model 4096) with the
    tcgen05 projection, one launch per layer, all layers in one CUDA graph;
    the L2 is flushed before every timed replay."""
    import torch
    import synth
    import fp4_kv_cache_nvfp4_b200 as csa2
    dev = torch.device("cuda", local_rank)
    d = synth.D_MODEL
    gen = torch.Generator(device=dev)
    gen.manual_seed(1004)
    h = [torch.randn((B, 128, d), generator=gen, device=dev).to(torch.bfloat16).view(torch.int16)
         for _ in range(layers)]
    w = [(torch.randn((256, d), generator=gen, device=dev) / math.sqrt(d)).to(torch.bfloat16).view(torch.int16)
         for _ in range(layers)]
    swa = [torch.empty((B, 128, 256), dtype=torch.int16, device=dev) for _ in range(layers)]
    lens = torch.full((B,), 1 << 20, dtype=torch.int32, device=dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    st = torch.cuda.Stream(device=dev)

    def replay():
        for l in range(layers):
            csa2.swa_replay(h[l], w[l], lens, swa[l], B, err=err, stream=st)

    with torch.cuda.stream(st):
        replay()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=st):
        replay()
    with torch.cuda.stream(st):
        for _ in range(3):
            g.replay()
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps)]
    with torch.cuda.stream(st):
        for k in range(reps):
            flush.fill_(k & 0xFF)
            ev[k][0].record(st)
            g.replay()
            ev[k][1].record(st)
    torch.cuda.synchronize()
    assert int(err.item()) == 0, f"device error flags {int(err.item())}"
    us = statistics.mean(a.elapsed_time(b) for a, b in ev) * 1e3
    peaks = _peaks()
    flop = layers * B * 2 * 128 * 256 * d
    byt = layers * (B * 128 * d * 2 + 256 * d * 2 + B * 128 * 256 * 2)
    tf, gbs = flop / (us * 1e-6) / 1e12, byt / (us * 1e-6) / 1e9
    sus = peaks.get("bf16_tflops_sustained") or peaks.get("bf16_tflops")
    return dict(workload=f"{layers} layers x {B} sequences: 128-token windows from d_model {d} hidden states",
                us_per_replay=us, launches=layers, flop=flop, bytes=byt, tflops=tf, gbs=gbs,
                tensor_frac=tf / sus if sus else None, hbm_frac=gbs / peaks["hbm_gbs"],
                peak_source=peaks.get("source"))


def run_launch_floor(args, local_rank: int) -> dict:
    """Floor that kernel boundaries alone put under a step: chains of empty
    kernels with programmatic dependent launch, each chain captured in one CUDA
    graph and replayed, timed with CUDA events on the launching stream."""
    import torch
    import fp4_kv_cache_nvfp4_b200 as csa2
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    sink = torch.zeros(1, dtype=torch.int32, device=dev)
    stream = torch.cuda.Stream(device=dev)
    out = {}
    for n, ctas in ((33, 148), (28, 64), (28, 148), (28, 296), (20, 148), (1, 148)):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.stream(stream):
            csa2.test_empty_chain(n, ctas, 160, sink, stream=stream)
        torch.cuda.synchronize()
        with torch.cuda.graph(g, stream=stream):
            csa2.test_empty_chain(n, ctas, 160, sink, stream=stream)
        reps = max(args.steps, 50)
        with torch.cuda.stream(stream):
            for _ in range(max(args.warmup, 3)):
                g.replay()
        torch.cuda.synchronize()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps)]
        with torch.cuda.stream(stream):
            for k in range(reps):
                ev[k][0].record(stream)
                g.replay()
                ev[k][1].record(stream)
        torch.cuda.synchronize()
        us = [a.elapsed_time(b) * 1e3 for a, b in ev]
        out[f"{n}x{ctas}"] = dict(kernels=n, ctas=ctas, us_per_graph=statistics.median(us),
                                  us_per_kernel=statistics.median(us) / n, reps=reps)
        del g
    return dict(metric="launch-chain floor: empty dependent kernels (programmatic dependent launch) in one CUDA "
                       "graph", unit="us", chains=out)


def run_reference(args, rank: int, world: int):
    if rank != 0:
        return None
    W = workload(args.config)
    cb = oracle_sample(args.config, budget_s=max(10.0, min(60.0, 2.0 * args.steps)), max_steps=max(args.steps, 1))
    return dict(metric=METRIC if W["decoder"] else METRIC_ENC, value=cb["value"], unit=UNIT, n_gpus=world,
                steps=args.steps, warmup=args.warmup,
                ms_per_step=W["B"] / cb["value"] * 1e3 if cb["value"] else None, higher_is_better=True,
                scaling="weak", vs_baseline=None, dtype="f32 decisions / f64 attention (oracle)", data="synthetic",
                config=dict(workload=W["workload"], seq_len=W["L"] * W["ratio"], entries=W["L"], ratio=W["ratio"],
                            batch_per_gpu=W["B"], layers=W["layers"], parallelism="host cores"),
                impl="reference", cpu_baseline=cb,
                e2e=dict(value=cb["value"], unit=UNIT, h2d_bytes_per_step=0, d2h_bytes_per_step=0))


def main():
    args = parse()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        res = run_reference(args, rank, world)
        if res is not None:
            print(json.dumps(res), flush=True)
        return
    if world > 1:
        import datetime

        import torch
        torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    if args.config == 3:
        res = run_prefill(args, rank, world, local_rank)
        if world > 1:
            import torch
            torch.distributed.barrier()
            torch.distributed.destroy_process_group()
        if rank == 0:
            print(json.dumps(res), flush=True)
        return
    if args.launch_floor:
        res = run_launch_floor(args, local_rank)
        if rank == 0:
            print(json.dumps(res), flush=True)
        return
    res = run_cuda(args, rank, world, local_rank)
    if args.config == 4 and not args.no_replay:
        res["swa_replay"] = run_replay(args, local_rank)
    if args.config == 4 and not args.no_prefill:
        # the prefill chunk (configuration 3) timed in the same process: the
        # north star asks for decode and prefill tokens/s side by side
        res["prefill"] = prefill_summary(run_prefill(args, rank, world, local_rank))
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        res["cpu_baseline"] = oracle_sample(args.config, budget_s=15.0)
        if W_DECODER(args.config):
            res["cpu_baseline"]["single_core"] = {f"config{c}": oracle_single_core(c) for c in (1, 2)}
        if "prefill" in res:
            res["prefill"]["cpu_baseline"] = oracle_prefill_sample()
    if world > 1:
        import torch
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    if rank == 0:
        print(json.dumps(res), flush=True)


if __name__ == "__main__":
    main()
