"""Benchmark of one block-sparse causal prefill-attention layer (pool + mask + attention).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload llama128k]
    python bench.py --impl reference ...      # the fp64 CPU oracle on a bounded sample

One step = the whole path over one layer's synthetic inputs: fp_pool_qk -> fp_build_block_mask
-> fp_sparse_prefill_attn (or the paged entry), launched through the C ABI. Inputs (Q 1 GiB,
K and V 256 MiB each at 128K) are larger than the 126 MB L2, so steps run back to back
without an L2 flush. Timing: CUDA events on the launching stream, W warm-up steps, then K
timed steps bracketed by barrier + synchronize; multi-GPU runs report the max over ranks and
are either independent replicas (each rank its own layer; value = ms per step / N, weak
scaling) or, with --split heads, one layer split by KV-head group (each rank the whole path on
its heads, no exchange; value = ms per step, strong scaling). The only collectives are the
timing barrier and the max-reduction.

Prints one JSON line (rank 0).
"""
from __future__ import annotations

import argparse
import dataclasses
import json
import math
import os
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import block_sparse_long_qk_b200 as fp  # noqa: E402
from block_sparse_long_qk_b200 import synthetic as S  # noqa: E402

METRIC = "128K prefill-attn ms/layer incl. mask build; executed TFLOPS & % of B200 peak"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# B200 datasheet figures (dense bf16 tensor rate, HBM3e bandwidth), reported beside the
# measured denominators for context only.
NOMINAL_BF16_TFLOPS = 2250.0
NOMINAL_HBM_GBS = 7700.0


def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return FALLBACK_PEAKS, "fallback"


class Clocks:
    """Samples SM clocks and throttle reasons with one `nvidia-smi -lms 100` process that runs
    for the whole timed region."""
    Q = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
         "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
         "clocks_event_reasons.sw_power_cap")
    NAMES = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]

    def __init__(self, index):
        self.index = index
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self):
        rows = []
        if self.proc is not None:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=10)
            except Exception:
                self.proc.kill()
                out, _ = self.proc.communicate()
            rows = [[x.strip() for x in l.split(",")] for l in out.splitlines() if l.strip()]
        sm = [float(r[0]) for r in rows if r and r[0].replace(".", "").isdigit()]
        mx = [float(r[1]) for r in rows if len(r) > 1 and r[1].replace(".", "").isdigit()]
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        reasons = sorted({self.NAMES[i] for r in rows for i in range(4)
                          if len(r) > 3 + i and r[3 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(sm)}


class Layer:
    """Device-resident inputs and preallocated outputs of one layer, and the step."""

    def __init__(self, inp, dev):
        w = inp.workload
        self.w = w
        self.dev = dev
        self.q = inp.q.to(dev)
        self.k = inp.k.to(dev)
        self.v = inp.v.to(dev)
        self.scales = {n: (None if getattr(inp, n) is None else getattr(inp, n).to(dev))
                       for n in ("q_scale", "k_scale", "v_scale")}
        self.paged = None
        if w.page_size:
            self.paged = fp.PagedKV(inp.k_cache.to(dev), inp.v_cache.to(dev),
                                    inp.page_table.to(dev))
            self.k = self.v = None
        self.batch = self.cb = None
        if w.q_lens is not None:
            self.cb = fp.ChunkedBatch.make(w.q_lens, w.seqlens, w.block, dev)
            nkb = self.cb.total_kblocks
        else:
            self.batch = fp.Batch.make(w.seqlens, w.block, dev)
            nkb = self.batch.total_blocks
        self.k_split = torch.empty(fp.k_split_shape(w.Hkv, nkb, w.d), dtype=torch.bfloat16,
                                   device=dev)
        self.stream = torch.cuda.current_stream(dev)

    def step(self, events=None):
        w, b, cb = self.w, self.batch, self.cb
        sc = self.scales
        e = events
        if e is not None:
            e[0].record(self.stream)
        if cb is not None:
            qp, kp = fp.pool_qk_chunked(self.q, self.k, cb, q_scale=sc["q_scale"],
                                        k_scale=sc["k_scale"], paged=self.paged,
                                        k_split_out=self.k_split)
        else:
            qp, kp = fp.pool_qk(self.q, self.k, w.block, batch=b, q_scale=sc["q_scale"],
                                k_scale=sc["k_scale"], paged=self.paged,
                                k_split_out=self.k_split)
        if e is not None:
            e[1].record(self.stream)
        if cb is not None:
            _, cnt, idx = fp.build_block_mask_chunked(qp, kp, cb, w.alpha, mask_bits=False,
                                                      k_split=self.k_split)
        else:
            _, cnt, idx = fp.build_block_mask(qp, kp, w.alpha, block=w.block, batch=b,
                                              mask_bits=False, k_split=self.k_split)
        if e is not None:
            e[2].record(self.stream)
        kw = dict(q_scale=sc["q_scale"], k_scale=sc["k_scale"], v_scale=sc["v_scale"])
        if cb is not None:
            out, _ = fp.sparse_prefill_attn_chunked(self.q, self.k, self.v, cnt, idx, cb,
                                                    paged=self.paged, **kw)
        elif self.paged is not None:
            out, _ = fp.sparse_prefill_attn_paged(self.q, self.paged, cnt, idx, b, **kw)
        else:
            out, _ = fp.sparse_prefill_attn(self.q, self.k, self.v, cnt, idx, w.block, batch=b,
                                            **kw)
        if e is not None:
            e[3].record(self.stream)
        return out, cnt, idx


def _query_blocks(w):
    """Per query block (all requests in order): absolute block I and the query positions
    [lo, hi) it holds. Plain prefill is the case q_len = kv_len."""
    B = w.block
    q_lens = w.q_lens if w.q_lens is not None else w.seqlens
    Is, los, his = [], [], []
    for n, L in zip(q_lens, w.seqlens):
        if n == 0:
            continue
        P0 = L - n
        for I in range(P0 // B, (L + B - 1) // B):
            Is.append(I)
            los.append(max(P0, I * B))
            his.append(min(L, (I + 1) * B))
    return np.array(Is), np.array(los), np.array(his)


def work_counts(w, cnt, idx, batch=None):
    """Algorithmic and executed attention FLOPs and the kept-block density of one layer."""
    B, d = w.block, w.d
    c = cnt.long().cpu().numpy()                       # [Hq, query blocks]
    I, lo, hi = _query_blocks(w)
    n = hi - lo
    # a kept block below the diagonal is a full B-key block seen by the block's n queries;
    # in the diagonal block the query at position p sees keys I*B .. p
    a, b_ = lo - I * B, hi - I * B
    diag = (b_ * (b_ + 1) - a * (a + 1)) // 2
    pairs = (c - 1) * B * n[None, :] + diag[None, :]
    alg = 4.0 * d * float(pairs.sum())
    executed = 4.0 * 128 * B * d * float(c.sum())
    causal_blocks = float((I + 1).sum()) * w.Hq
    return alg, executed, float(c.sum()) / causal_blocks


def pool_mask_bytes(w):
    """(pool kernel bytes, pool + mask bytes): Q and K read once, the fp32 means and the bf16
    hi / lo split of the pooled keys written by the pool kernel and read by the mask kernel."""
    eb = 1 if w.dtype == "e4m3" else 2
    Tk = w.total_tokens
    Tq = sum(w.q_lens) if w.q_lens is not None else Tk
    nkb = sum((L + w.block - 1) // w.block for L in w.seqlens)
    nqb = len(_query_blocks(w)[0])
    inputs = (Tq * w.Hq + Tk * w.Hkv) * w.d * eb
    pooled = (nqb * w.Hq + nkb * w.Hkv) * w.d * 4 + nkb * w.Hkv * w.d * 4
    return inputs + pooled, inputs + 2 * pooled


def cpu_baseline(inp, rows_sample=32, seed=5):
    """The fp64 oracle as it stands, on a bounded sample of the same layer: pooling and the
    mask in full, attention on `rows_sample` seeded (head, query block) rows, extrapolated
    to the layer's rows."""
    import oracle as O
    try:
        from threadpoolctl import threadpool_info
        cores = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    except Exception:
        cores = os.cpu_count()
    w = inp.workload
    cu = inp.cu_seqlens.tolist()
    cu_q = inp.cu_q.tolist() if inp.cu_q is not None else cu
    cu_k = cu if inp.cu_q is not None else None
    q, k, v = inp.codes_f32("q"), inp.codes_f32("k"), inp.codes_f32("v")
    qs, ks, vs = inp.scale_f64("q"), inp.scale_f64("k"), inp.scale_f64("v")
    scale = 1.0 / math.sqrt(w.d)
    t0 = time.perf_counter()
    if cu_k is not None:
        qp = O.pool_query_blocks(q, w.block, cu_q, cu_k, scale=qs)
    else:
        qp = O.pool_blocks(q, w.block, cu, scale=qs)
    kp = O.pool_blocks(k, w.block, cu, scale=ks)
    sc = O.block_scores(qp, kp, cu_q, w.block, scale, cu_k=cu_k)
    info, off = O.query_blocks(cu_q, cu_k, w.block)
    keeps = [O.block_keep(s, w.alpha, row0=i[1]) for s, i in zip(sc, info)]
    t1 = time.perf_counter()
    rng = np.random.default_rng(seed)
    rows = [(int(rng.integers(w.Hq)), int(rng.integers(off[-1]))) for _ in range(rows_sample)]
    O.masked_causal_attention(q, k, v, keeps, cu_q, w.block, scale, rows=rows, q_scale=qs,
                              k_scale=ks, v_scale=vs, cu_k=cu_k)
    t2 = time.perf_counter()
    total_rows = w.Hq * off[-1]
    ms = 1e3 * ((t1 - t0) + (t2 - t1) * total_rows / rows_sample)
    sample = (f"pool+mask in full ({1e3 * (t1 - t0):.0f} ms) + attention on {rows_sample} of "
              f"{total_rows} (head, query-block) rows ({1e3 * (t2 - t1):.0f} ms), "
              f"extrapolated to the layer")
    sample += (f"; cores = the {cores} threads numpy's BLAS may use: the oracle's per-block and "
               "per-row Python loops run on one core, only its matrix products use more")
    return {"value": round(ms, 3), "unit": "ms/layer", "cores": cores, "kind": "oracle",
            "sample": sample}


def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        torch.distributed.init_process_group(
            "nccl" if args.impl == "native" else "gloo",
            timeout=datetime.timedelta(seconds=120))
    return world, rank, local


def barrier(world):
    if world > 1:
        torch.distributed.barrier()


def max_over_ranks(x, world, dev):
    if world == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def run_reference(args, world, rank):
    if rank != 0:
        return
    w = S.WORKLOADS[args.workload]
    inp = S.make_inputs(args.workload)
    times = []
    cb = None
    for i in range(args.warmup + args.steps):
        t = time.perf_counter()
        cb = cpu_baseline(inp, rows_sample=args.ref_rows, seed=5 + i)
        if i >= args.warmup:
            times.append(cb["value"])
    v = statistics.median(times)
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": "ms/layer",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": v, "higher_is_better": False, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": _config(w, args), "cpu_baseline": dict(cb, value=v),
            "e2e": {"value": v, "unit": "ms/layer", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def _config(w, args):
    return {"workload": f"{w.name}: L={'+'.join(map(str, w.seqlens)) if len(w.seqlens) < 9 else w.total_tokens} "
                        f"Hq={w.Hq} Hkv={w.Hkv} d={w.d} block={w.block} alpha={w.alpha} "
                        f"{w.dtype}" + (f" paged{w.page_size}" if w.page_size else "")
                        + (f" chunked: q={sum(w.q_lens)} new tokens after cached prefixes"
                           if w.q_lens is not None else ""),
            "tokens": w.total_tokens, "requests": w.batch,
            "parallelism": (f"heads{args.gpus}" if args.split == "heads"
                            else f"replicas{args.gpus}"),
            "l2": "inputs larger than L2 (no flush)"}


def shard_inputs(inp, rank, world):
    """The part of one layer that rank ``rank`` runs when the layer is split by KV-head group
    (``fp.head_shard``): contiguous copies of its query heads and KV heads, as the projections
    of a tensor-parallel model would produce them, with the head counts set to the slice's."""
    w = inp.workload
    qs, ks = fp.head_shard(w.Hq, w.Hkv, rank, world)

    def cut(t, sl, dim):
        if t is None:
            return None
        idx = [slice(None)] * t.dim()
        idx[dim] = sl
        return t[tuple(idx)].contiguous()
    ws = dataclasses.replace(w, name=f"{w.name}/heads{world}", Hq=qs.stop - qs.start,
                             Hkv=ks.stop - ks.start)
    return dataclasses.replace(inp, workload=ws, q=cut(inp.q, qs, 1), k=cut(inp.k, ks, 1),
                               v=cut(inp.v, ks, 1), q_scale=cut(inp.q_scale, qs, 0),
                               k_scale=cut(inp.k_scale, ks, 0), v_scale=cut(inp.v_scale, ks, 0),
                               k_cache=cut(inp.k_cache, ks, 2), v_cache=cut(inp.v_cache, ks, 2))


def measure_e4m3_peak(dev, n=8192, reps=10):
    """Dense e4m3 GEMM rate of this GPU in TFLOP/s: torch._scaled_mm on n^3 (fp32 accumulate,
    bf16 out), best of ``reps`` launches timed with CUDA events -- the same kind of burst figure
    as the bf16 peak of the measured-peaks file. None if the call is unavailable."""
    try:
        a = torch.randn(n, n, device=dev).to(torch.float8_e4m3fn)
        b = torch.randn(n, n, device=dev).to(torch.float8_e4m3fn).t()  # column-major operand
        one = torch.ones((), device=dev)

        def mm():
            return torch._scaled_mm(a, b, scale_a=one, scale_b=one, out_dtype=torch.bfloat16)
        for _ in range(3):
            mm()
        best = math.inf
        for _ in range(reps):
            s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            s.record()
            mm()
            e.record()
            torch.cuda.synchronize(dev)
            best = min(best, s.elapsed_time(e))
        del a, b
        return 2.0 * n ** 3 / (best * 1e-3) / 1e12
    except Exception:
        return None


def time_layer(layer, steps, warmup, world, dev, local):
    """W warm-up steps, then K steps timed with CUDA events between two barriers, with the SM
    clocks sampled over the timed region. Returns the max-over-ranks ms per step, the per-step
    stage times, the clock record and the last step's lists."""
    # The clock sampler starts before the warm-up, so that starting it does not land in the
    # timed region; its samples cover the warm-up and the timed steps.
    clocks = Clocks(local)
    clocks.start()
    for _ in range(warmup):
        layer.step()
    torch.cuda.synchronize(dev)
    fp.check_status(dev)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(steps)]
    barrier(world)
    torch.cuda.synchronize(dev)
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    # A device-side spin ahead of the start event (25 ms plus 1 ms per timed step, at 2 GHz;
    # longer at the lower clocks the power cap sets) lets the host enqueue every timed step
    # before the GPU reaches them, so a host-side stall while launching (a launch that waits
    # for the driver, e.g. while the clock sampler queries it) cannot leave the GPU idle inside
    # the timed region: the events would count that idle time.
    torch.cuda._sleep(2_000_000 * (25 + steps))
    t_start.record()
    for i in range(steps):
        out, cnt, idx = layer.step(evs[i])
    t_end.record()
    torch.cuda.synchronize(dev)
    barrier(world)
    clk = clocks.stop()
    fp.check_status(dev)
    ms_step = max_over_ranks(t_start.elapsed_time(t_end) / steps, world, dev)
    stages = {"pool": [e[0].elapsed_time(e[1]) for e in evs],
              "mask": [e[1].elapsed_time(e[2]) for e in evs],
              "attn": [e[2].elapsed_time(e[3]) for e in evs]}
    return ms_step, stages, clk, cnt, idx


def roofline(w, alg, executed, attn_ms, peaks, peak_src, clk, e4m3_peak):
    """The attention kernel's roofline entry. The denominator is the measured BURST dense rate
    of the kernel's own input type: the kernel is timed per launch (~10 ms), not in a
    seconds-long loop, so the sustained figure (taken at a lower clock under the power cap) is
    reported beside it, not used. e4m3 takes the live-measured e4m3 GEMM rate, else 2x the bf16
    burst (the datasheet ratio)."""
    burst = peaks["bf16_tflops"]
    sustained = peaks.get("bf16_tflops_sustained")
    e4m3 = w.dtype == "e4m3"
    if e4m3:
        if e4m3_peak:
            peak, src = e4m3_peak, "e4m3 dense GEMM (torch._scaled_mm 8192^3), measured in this run, burst"
        else:
            peak, src = 2.0 * burst, f"{peak_src} bf16 burst x2 (datasheet e4m3/bf16 ratio)"
    else:
        peak, src = burst, f"{peak_src} bf16 burst (cuBLAS 8192^3 best of 10)"
    ach = alg / (attn_ms * 1e-3) / 1e12
    exe = executed / (attn_ms * 1e-3) / 1e12
    traffic = None
    tf = os.path.join(ROOT, "profiles", "attn_traffic.json")
    if os.path.exists(tf):
        traffic = json.load(open(tf)).get(w.name) or None
    nominal = NOMINAL_BF16_TFLOPS * (2.0 if e4m3 else 1.0)
    r = {"bound": "tensor", "achieved": round(ach, 2), "peak": round(peak, 1), "unit": "TFLOP/s",
         "frac": round(ach / peak, 4), "traffic": traffic, "peak_source": src,
         "executed_tflops": round(exe, 2), "executed_frac": round(exe / peak, 4),
         # the datasheet's dense figure, for context (2.25 PFLOP/s bf16, 4.5 e4m3)
         "nominal_peak": nominal, "frac_of_nominal": round(ach / nominal, 4)}
    if sustained:
        sp = sustained * (e4m3_peak / burst if e4m3 and e4m3_peak else (2.0 if e4m3 else 1.0))
        r["frac_of_sustained"] = round(ach / sp, 4)
    sm, sm_max = clk.get("sm_mhz"), clk.get("sm_max_mhz")
    if sm and sm_max:
        # what the same cycles would deliver at the maximum SM clock (the kernel runs under the
        # 1 kW power cap at the sampled median clock)
        r["achieved_at_max_clock"] = round(ach * sm_max / sm, 2)
        r["frac_at_max_clock"] = round(ach * sm_max / sm / peak, 4)
    return r


def measure_extra(name, args, dev, local, peaks, peak_src, e4m3_peak):
    """Device-side figures of another workload in the same run (the e4m3 and the multi-head
    128K layers beside the bf16 one): stage times, work and roofline, timed as the main
    workload is."""
    w = S.WORKLOADS[name]
    inp = S.make_inputs(name)
    layer = Layer(inp, dev)
    del inp
    ms_step, st, clk, cnt, idx = time_layer(layer, args.steps, args.warmup, 1, dev, local)
    alg, executed, density = work_counts(w, cnt, idx)
    attn_ms = statistics.mean(st["attn"])
    pool_bytes, pm_bytes = pool_mask_bytes(w)
    pm_ms = statistics.mean(st["pool"]) + statistics.mean(st["mask"])
    out = {"workload": _config(w, args)["workload"], "ms_per_step": round(ms_step, 4),
           "stages_ms": {k: round(statistics.mean(v), 4) for k, v in st.items()},
           "block_density": round(density, 5),
           "attn_tflop": {"algorithmic": round(alg / 1e12, 3), "executed": round(executed / 1e12, 3)},
           "pool_mask_frac_hbm": round(pm_bytes / (pm_ms * 1e-3) / 1e9 / peaks["hbm_gbs"], 4),
           "roofline": roofline(w, alg, executed, attn_ms, peaks, peak_src, clk, e4m3_peak),
           "clocks": clk}
    del layer
    torch.cuda.empty_cache()
    return out


def run_native(args, world, rank, local):
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    w = S.WORKLOADS[args.workload]
    heads = args.split == "heads"
    # replicas: each rank its own layer; head split: every rank the same layer, its own heads
    inp = S.make_inputs(args.workload, seed=S.DEFAULT_SEEDS[w.name] + (0 if heads else 1000 * rank))
    if heads:
        inp = shard_inputs(inp, rank, world)
        w = inp.workload
    layer = Layer(inp, dev)
    peaks, peak_src = _peaks()
    per_layer = 1 if heads else world   # layers the job completes per step

    ms_step, st, clk, cnt, idx = time_layer(layer, args.steps, args.warmup, world, dev, local)
    pool_l, mask_l, attn_l = st["pool"], st["mask"], st["attn"]
    pool_ms, mask_ms, attn_ms = (statistics.mean(x) for x in (pool_l, mask_l, attn_l))

    alg, executed, density = work_counts(w, cnt, idx)
    pool_bytes, pm_bytes = pool_mask_bytes(w)
    extra_names = ([] if (args.no_extra or world > 1 or w.name != "llama128k")
                   else ["fp8_128k", "mha128k"])
    e4m3_peak = None
    if w.dtype == "e4m3" or extra_names:
        e4m3_peak = measure_e4m3_peak(dev)
    roof = roofline(w, alg, executed, attn_ms, peaks, peak_src, clk, e4m3_peak)

    # e2e: host (pinned) inputs -> device, the layer, output -> host, per step
    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(layer, inp, dev, args, world, per_layer)
    del layer
    torch.cuda.empty_cache()
    extra = {n: measure_extra(n, args, dev, local, peaks, peak_src, e4m3_peak)
             for n in extra_names}

    if rank == 0:
        cb = None
        if world == 1 and not args.no_cpu_baseline:
            cb = cpu_baseline(inp, rows_sample=args.ref_rows)
        line = {
            "metric": METRIC, "value": round(ms_step / per_layer, 4), "unit": "ms/layer",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(ms_step, 4), "higher_is_better": False,
            "scaling": "strong" if heads else "weak",
            "vs_baseline": None, "dtype": w.dtype, "data": "synthetic",
            "config": _config(w, args),
            "stages_ms": {"pool": round(pool_ms, 4), "mask": round(mask_ms, 4),
                          "attn": round(attn_ms, 4)},
            "stages_ms_median_max": {n: [round(statistics.median(x), 4), round(max(x), 4)]
                                     for n, x in (("pool", pool_l), ("mask", mask_l),
                                                  ("attn", attn_l))},
            "pool_mask": {"bytes": pm_bytes,
                          "gbs": round(pm_bytes / ((pool_ms + mask_ms) * 1e-3) / 1e9, 1),
                          "frac_hbm": round(pm_bytes / ((pool_ms + mask_ms) * 1e-3) / 1e9 /
                                            peaks["hbm_gbs"], 4),
                          "pool_bytes": pool_bytes,
                          "pool_frac_hbm": round(pool_bytes / (pool_ms * 1e-3) / 1e9 /
                                                 peaks["hbm_gbs"], 4),
                          "frac_hbm_nominal": round(pm_bytes / ((pool_ms + mask_ms) * 1e-3) /
                                                    1e9 / NOMINAL_HBM_GBS, 4)},
            "block_density": round(density, 5),
            "attn_tflop": {"algorithmic": round(alg / 1e12, 3),
                           "executed": round(executed / 1e12, 3)},
            "roofline": roof,
            "cpu_baseline": cb,
            "e2e": e2e,
            "gpu_launches": 3 * args.steps,
            "clocks": clk,
        }
        if e4m3_peak:
            line["e4m3_peak_tflops_measured"] = round(e4m3_peak, 1)
        if extra:
            line["extra"] = extra
        print(json.dumps(line), flush=True)


def run_e2e(layer, inp, dev, args, world, per_layer):
    """Same metric through the public API with host buffers: every step copies Q, K, V (or the
    paged K/V caches) from pinned host memory, runs the whole path and copies the output back.
    ``fp.HostPipeline`` overlaps one step's copies with the neighbouring steps' kernels; the
    time per step is the wall time of K pipelined steps on the device clock, fill and drain
    included."""
    w = layer.w
    hq = inp.q.pin_memory()
    houts = [torch.empty(layer.q.shape, dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    sc = layer.scales
    pt = layer.paged.page_table if layer.paged is not None else None
    append = layer.cb is not None and layer.paged is not None
    if append:
        # Chunked prefill on a paged cache: the cached prefix stays on the device; each step
        # copies in the chunk's Q, K and V rows and appends K/V to the cache before attention.
        cu = inp.cu_seqlens.tolist()
        rows = torch.cat([torch.arange(cu[b] + L - n, cu[b] + L)
                          for b, (n, L) in enumerate(zip(w.q_lens, w.seqlens))])
        hk, hv = inp.k[rows].pin_memory(), inp.v[rows].pin_memory()
    else:
        hk = (inp.k_cache if inp.k_cache is not None else inp.k).pin_memory()
        hv = (inp.v_cache if inp.v_cache is not None else inp.v).pin_memory()

    def run(q, k, v, out):
        kw = dict(q_scale=sc["q_scale"], k_scale=sc["k_scale"], v_scale=sc["v_scale"], out=out)
        if append:
            fp.append_paged_kv(k, v, layer.cb, layer.paged)
            fp.sparse_prefill_chunked(q, None, None, layer.cb, w.alpha, paged=layer.paged, **kw)
            return
        paged = fp.PagedKV(k, v, pt) if pt is not None else None
        if layer.cb is not None:
            fp.sparse_prefill_chunked(q, k, v, layer.cb, w.alpha, paged=paged, **kw)
        elif paged is not None:
            fp.sparse_prefill(q, alpha=w.alpha, block=w.block, batch=layer.batch, paged=paged,
                              **kw)
        else:
            fp.sparse_prefill(q, k, v, w.alpha, w.block, batch=layer.batch, **kw)

    pipe = fp.HostPipeline(run, (hq, hk, hv), houts[0], dev)
    steps = max(5, min(args.steps, 12))
    for i in range(2):
        pipe.submit((hq, hk, hv), houts[i % 2])
    pipe.synchronize()
    torch.cuda.synchronize(dev)
    barrier(world)
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record()
    for i in range(steps):
        pipe.submit((hq, hk, hv), houts[i % 2])
    pipe.synchronize()
    e.record()
    torch.cuda.synchronize(dev)
    ms = max_over_ranks(s.elapsed_time(e) / steps, world, dev)
    fp.check_status(dev)
    h2d = hq.numel() * hq.element_size() + hk.numel() * hk.element_size() + \
        hv.numel() * hv.element_size()
    return {"value": round(ms / per_layer, 4), "unit": "ms/layer", "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": houts[0].numel() * houts[0].element_size(), "steps": steps,
            "pipelined": "copy-in, kernels and copy-out of neighbouring steps overlap",
            "inputs": ("chunk Q, K, V rows (cached prefix resident in the paged cache; the "
                       "chunk's K/V appended each step)") if append else "Q, K, V"}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["native", "reference"], default="native")
    ap.add_argument("--workload", default="llama128k", choices=sorted(S.WORKLOADS))
    ap.add_argument("--ref-rows", type=int, default=32)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--split", choices=["replicas", "heads"], default="replicas",
                    help="N > 1: independent layers per rank (replicas, weak scaling) or one "
                         "layer split by KV-head group (heads, strong scaling; no exchange)")
    ap.add_argument("--no-extra", action="store_true",
                    help="skip the e4m3 and multi-head 128K layers that the default bf16 128K "
                         "run also times")
    args = ap.parse_args()
    world, rank, local = dist_setup(args)
    try:
        if args.impl == "reference":
            run_reference(args, world, rank)
        else:
            run_native(args, world, rank, local)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
