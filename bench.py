"""Benchmark of the CSA2 FP4 sparse-decode step on B200.

One step = one decode step of the workload's whole layer group: every Full
layer appends its new tokens (K1) and indexes (K2 + K3), every Reindex layer
indexes, every layer attends (K4 + K5). Default workload: batch 64, context
131,072, one Full layer, top-k 2,048 (the 128K-context batch-64 decode).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
  python bench.py --impl reference ...   # the CPU oracle, timed on host cores

Multi-GPU: one process per GPU (torchrun); every rank runs an independent
replica with its own seed (weak scaling, no collective on the data path);
time is the max over ranks. Rank 0 prints one JSON line.

Besides the step, the line carries two kernels outside the default step,
each timed with events around every launch:
  indexer_fp8_quant   csa2_quant_indexer_fp8 over B x T rows of 64 bf16
                      channels (more than L2 holds);
  indexer_pool_topk   csa2_indexer_pool_topk, a Reindex query selecting the
                      top-k inside the Full layer's top-4k, L2 flushed before
                      each launch (one GPU only).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import torch  # noqa: E402

from compressed_sparse_attention_quant_b200 import inputs, replicas  # noqa: E402

FALLBACK_HBM_GBS = 6650.0
NOMINAL_HBM_GBS = 8000.0            # the 8 TB/s the metric's roofline fraction is quoted against
L2_FLUSH_BYTES = 256 << 20
METRIC = "decode tokens/s and achieved HBM GB/s (% of 8 TB/s) for CSA2 FP4 sparse attn"
KERNEL_SOURCES = ("csrc/common.cuh", "csrc/indexer.cuh", "csrc/topk.cuh")


# Algorithmic bytes of one row of the indexer FP8 quantiser: 64 bf16 in,
# 64 E4M3 codes + one fp32 scale out.
Q8_BYTES_PER_ROW = 64 * 2 + 64 + 4


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def tensor_peak():
    """Burst bf16 dense TFLOP/s (measured cuBLAS), else the fallback 1590."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["bf16_tflops"]), "measured"
    except Exception:
        return 1590.0, "fallback"


def kernel_source_hash() -> str:
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES:
        with open(os.path.join(ROOT, "compressed_sparse_attention_quant_b200", rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic(workload: str):
    """DRAM bytes per indexer_topk call from a committed ncu summary, or None
    when missing or taken on different kernel sources."""
    path = os.path.join(ROOT, "profiles", f"indexer_topk_{workload}.json")
    try:
        with open(path) as f:
            d = json.load(f)
        if d.get("kernel_source_hash") != kernel_source_hash():
            return None
        return float(d["dram_bytes_per_call"])
    except Exception:
        return None


class ClockSampler:
    """SM clocks and clock-event reasons sampled by NVML from a thread while
    the timed region runs (a few ms between samples)."""

    # NVML clocks-event-reason bits
    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown"}

    def __init__(self, gpu_index: int, period_s: float = 0.002):
        self.gpu, self.period = gpu_index, period_s
        self.samples = []
        self.max_mhz = None
        self.ok = False

    def __enter__(self):
        import threading
        try:
            import pynvml
            pynvml.nvmlInit()
            vis = os.environ.get("CUDA_VISIBLE_DEVICES")
            idx = int(vis.split(",")[self.gpu]) if vis and vis.split(",")[0].isdigit() else self.gpu
            self.h = pynvml.nvmlDeviceGetHandleByIndex(idx)
            self.nv = pynvml
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            return self
        self.stop = threading.Event()

        def run():
            while not self.stop.is_set():
                try:
                    mhz = self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM)
                    rs = self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                    self.samples.append((mhz, rs))
                except Exception:
                    pass
                time.sleep(self.period)

        self.th = threading.Thread(target=run, daemon=True)
        self.th.start()
        return self

    def __exit__(self, *exc):
        if self.ok:
            self.stop.set()
            self.th.join(timeout=5)

    def summary(self):
        if not self.ok or not self.samples:
            return None
        sm = sorted(m for m, _ in self.samples)
        reasons = set()
        for _, rs in self.samples:
            for bit, name in self.REASONS.items():
                if rs & bit:
                    reasons.add(name)
        return {"sm_mhz": sm[len(sm) // 2], "sm_max_mhz": self.max_mhz, "samples": len(self.samples),
                "reasons": sorted(reasons)}


# ----------------------------------------------------------------- CPU oracle arm
class OracleArm:
    """The CPU oracle on sequences of the workload, generated on the CPU.

    prepare() quantizes the owners' caches of the first n_seqs sequences
    (set-up, untimed); step(b) times the oracle's per-step work for sequence
    b: append quantization of the new tokens, indexer scores, top-k and
    attention for every query token of every layer."""

    def __init__(self, wl: inputs.Workload, n_seqs: int):
        import oracle
        self.oracle = oracle
        self.wl = wl
        self.own, self.src = oracle.plan(wl.modes)
        self.seqs = list(range(min(n_seqs, wl.batch)))
        self.caches = {}
        self.layer_in = {}

    def prepare(self):
        o_, wl = self.oracle, self.wl
        for b in self.seqs:
            T = wl.lens()[b]
            for o in set(self.own):
                kv = torch.cat([r for _, r in inputs.kv_chunks(wl, o, b, "cpu")])
                codes, scales = o_.quant_fp4(o_.bf16_bits(kv[:T - wl.q_tokens]))
                self.caches[(o, b)] = (o_.bf16_bits(kv[T - wl.q_tokens:T]), codes, scales,
                                       inputs.kidx_rows(wl, o, b, 0, T, "cpu").numpy(),
                                       inputs.kidx_scale_rows(wl, o, b, 0, T, "cpu").numpy())
        for li in range(len(wl.modes)):
            self.layer_in[li] = (o_.bf16_bits(inputs.attn_query(wl, li, "cpu")),
                                 o_.bf16_bits(inputs.swa_rows(wl, li, "cpu")),
                                 inputs.idx_query(wl, li, "cpu").numpy(),
                                 inputs.idx_weights(wl, li, "cpu").numpy())

    def step(self, b: int) -> float:
        import numpy as np
        o_, wl = self.oracle, self.wl
        T, Sq, W = wl.lens()[b], wl.q_tokens, inputs.WINDOW
        scale = 1.0 / math.sqrt(576)
        t0 = time.perf_counter()
        cache = {}
        results = {}
        for li, mode in enumerate(wl.modes):
            new_bits, codes, scales, kid, ks = self.caches[(self.own[li], b)]
            if mode == "F":          # append: quantize the Sq new tokens into the cache
                nc, ns = o_.quant_fp4(new_bits)
                cache[li] = (np.concatenate([codes, nc]), np.concatenate([scales, ns]))
            codes, scales = cache[self.own[li]]
            q, swa, qi, w = (x[b] for x in self.layer_in[li])
            for j in range(Sq):
                pos = T - Sq + j
                if mode in ("F", "R"):
                    s = o_.indexer_scores(qi[j], w[j], kid[:pos + 1], ks[:pos + 1])
                    idx = o_.topk(s, pos + 1, wl.top_k)
                else:
                    idx = results[(self.src[li], j)]
                results[(li, j)] = idx
                rows = [r for r in range(j, j + W) if T - (W + Sq - 1) + r >= 0]
                o_.sparse_attn(q[j], codes, scales, idx, swa[rows], scale)
        return time.perf_counter() - t0

    def describe(self, n_timed: int, threads: int) -> str:
        wl = self.wl
        return (f"{n_timed} sequence-steps over sequences {self.seqs} of {wl.batch}: "
                f"{wl.q_tokens} query token(s) x {len(wl.modes)} layer(s), context {wl.lens()[0]}, "
                f"top-k {wl.top_k}; fp64 oracle on {threads} host thread(s); cache quantization untimed")


def cpu_baseline(wl: inputs.Workload, n_seqs: int, budget_s: float, threads: int) -> dict:
    """The oracle (its OpenMP build: bit-identical results, independent outer
    loops on `threads` host cores) on a bounded sample of the workload."""
    import oracle
    oracle.use_all_cores(True)
    oracle.set_threads(threads)
    arm = OracleArm(wl, n_seqs)
    arm.prepare()
    spent, n = 0.0, 0
    while spent < budget_s and n < 64:
        spent += arm.step(arm.seqs[n % len(arm.seqs)])
        n += 1
    tok = n * wl.q_tokens
    return {"value": tok / spent, "unit": "tokens/s", "cores": oracle.threads(), "kind": "oracle",
            "sample": arm.describe(n, oracle.threads())}


def run_reference(args, wl):
    rank = int(os.environ.get("RANK", "0"))
    if not replicas.reports(rank):
        return                      # the oracle arm runs on rank 0 only
    import oracle
    oracle.use_all_cores(True)      # the same oracle source, on every host core
    oracle.set_threads(oracle.host_cores())
    arm = OracleArm(wl, args.ref_seqs)
    arm.prepare()
    times = []
    for i in range(args.warmup + args.steps):
        t = arm.step(arm.seqs[i % len(arm.seqs)])
        if i >= args.warmup:
            times.append(t)
    per_seq = sum(times) / len(times)
    value = wl.q_tokens / per_seq
    desc = arm.describe(len(times), oracle.threads())
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": per_seq * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": wl.name, "batch": wl.batch, "q_tokens": wl.q_tokens,
                       "context": wl.context, "top_k": wl.top_k, "modes": "".join(wl.modes),
                       "step": "one sequence of the batch per step (bounded sample)"},
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": oracle.threads(), "kind": "oracle",
                             "sample": desc},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------- GPU arm
def pool_leg(args, wl, dw, lib, flush, stream, hbm) -> dict:
    """csa2_indexer_pool_topk (hierarchical sparse indexer): a Reindex query
    selecting the top-k inside the Full layer's top-C, C = 4k. The pool is
    built once (untimed) by csa2_indexer_topk with k = C; each timed launch
    follows an L2 flush. Errors are reported in the result, never raised."""
    try:
        g = dw.group
        k = g.k
        C = min(4 * k, 32768)
        cache = g.cache(0)
        pool = lib.indexer_topk(dw.q_idx[0], dw.w[0], cache, dw.page_table, dw.seq_lens, C, ws=g.ws_idx)
        q2 = dw.q_idx[0].roll(1, dims=-1).contiguous()        # another layer's query over the same pool
        out = torch.empty(wl.batch, wl.q_tokens, k, dtype=torch.int32, device=pool.device)
        for _ in range(2):
            lib.indexer_pool_topk(q2, dw.w[0], cache, dw.page_table, dw.seq_lens, pool, k, out=out)
        torch.cuda.synchronize()
        evs = []
        for _ in range(args.steps):
            flush.zero_()
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            lib.indexer_pool_topk(q2, dw.w[0], cache, dw.page_table, dw.seq_lens, pool, k, out=out)
            e1.record(stream)
            evs.append((e0, e1))
        torch.cuda.synchronize()
        ms = sum(a.elapsed_time(b) for a, b in evs) / args.steps
        rows = wl.batch * wl.q_tokens
        per_row = C * (64 + 4 + 4) + 4 * k + 272          # keys + sigma + pool indices, output, q + w
        achieved = rows * per_row / (ms * 1e-3) / 1e9
        return {"kernel": "csa2_indexer_pool_topk", "pool": C, "k": k, "rows": rows, "ms_per_launch": ms,
                "bytes_per_row": per_row, "achieved": achieved, "peak": hbm, "unit": "GB/s",
                "frac": achieved / hbm, "device_status": lib.status_string(lib.last_device_error()),
                "input": "pool = the Full layer's top-4k; query = the Full query rolled by one channel"}
    except Exception as e:                                  # the leg is optional: report, do not fail
        return {"kernel": "csa2_indexer_pool_topk", "error": f"{type(e).__name__}: {e}"[:300]}


def time_steps(dw, args, flush, stream):
    """Mean device time (ms) of one whole step of a DeviceWorkload: W untimed
    warm-up steps, then K steps, each preceded by an untimed L2 flush, CUDA
    events on the launching stream around each step. The step is the
    workload's CUDA graph (one replay launches every kernel of the step)
    unless --eager."""
    run = dw.step if args.eager else dw.capture().replay
    for _ in range(args.warmup):
        flush.zero_()
        run()
    torch.cuda.synchronize()
    evs = []
    for _ in range(args.steps):
        if not args.no_flush:
            flush.zero_()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        run()
        e1.record(stream)
        evs.append((e0, e1))
    torch.cuda.synchronize()
    return sum(a.elapsed_time(b) for a, b in evs) / args.steps


def other_workload(args, name, dev, flush, stream, hbm, with_cpu: bool) -> dict:
    """Step throughput and roofline fractions of another benchmark workload
    (its own inputs resident in HBM), with the oracle timed on a bounded
    sample on every host core. Errors are reported, never raised."""
    from compressed_sparse_attention_quant_b200 import lib, workload
    try:
        wl = inputs.WORKLOADS[name]
        dw = workload.DeviceWorkload(wl, dev)
        acct = dw.algorithmic_bytes()
        ms = time_steps(dw, args, flush, stream)
        gbs = acct["total"] / (ms * 1e-3) / 1e9
        out = {"value": wl.batch * wl.q_tokens / (ms * 1e-3), "unit": "tokens/s", "ms_per_step": ms,
               "config": {"batch": wl.batch, "q_tokens": wl.q_tokens, "context": wl.context, "top_k": wl.top_k,
                          "modes": "".join(wl.modes)},
               "algorithmic_bytes_per_step": acct["total"], "step_hbm_gbs": gbs,
               "step_frac_of_8tbs": gbs / NOMINAL_HBM_GBS, "step_frac_of_measured_copy": gbs / hbm,
               "attention_tflops_per_step": attention_flops(wl) / 1e12,
               "device_status": lib.status_string(lib.last_device_error())}
        del dw
        torch.cuda.empty_cache()
        if with_cpu:
            import oracle
            out["cpu_baseline"] = cpu_baseline(wl, 1, args.cpu_budget_other, oracle.host_cores())
        return out
    except Exception as e:                                  # optional leg: report, do not fail
        return {"error": f"{type(e).__name__}: {e}"[:300]}


def attention_flops(wl) -> float:
    """Algorithmic attention FLOPs of one step: QK and PV over k + 128 keys,
    16 heads x 576 channels, per query token and layer."""
    return 4.0 * 16 * 576 * (wl.top_k + 128) * wl.batch * wl.q_tokens * len(wl.modes)


def bulk_quant_leg(args, wl, dw, stream, hbm) -> dict:
    """csa2_quant_kv_fp4 as a bulk cache build: B x T tokens (the whole
    context of the workload, with their indexer keys), rewritten into the
    same slots. Events around each launch; inputs > L2."""
    from compressed_sparse_attention_quant_b200 import lib
    try:
        n = wl.batch * wl.context
        x = torch.randn(n, lib.DIM, device=stream.device, dtype=torch.bfloat16,
                        generator=torch.Generator(device=stream.device).manual_seed(7))
        kid = torch.randint(0, 120, (n, lib.IDX_DIM), device=stream.device, dtype=torch.uint8)
        ks = torch.ones(n, device=stream.device)
        pos = torch.arange(wl.context, device=stream.device)
        slots = torch.cat([lib.slot_mapping(dw.page_table, b, pos) for b in range(wl.batch)])
        cache = lib.PagedCache(dw.group.num_pages, stream.device)
        for _ in range(2):
            lib.quant_kv_fp4(x, slots, cache, kid, ks)
        torch.cuda.synchronize()
        evs = []
        for _ in range(args.steps):
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            lib.quant_kv_fp4(x, slots, cache, kid, ks)
            e1.record(stream)
            evs.append((e0, e1))
        torch.cuda.synchronize()
        ms = sum(a.elapsed_time(b) for a, b in evs) / args.steps
        per_tok = 576 * 2 + 4 + 64 + 4 + 288 + 36 + 64 + 4       # bf16 in, slot, key + sigma in; FP4 + scales + key + sigma out
        ach = n * per_tok / (ms * 1e-3) / 1e9
        del x, kid, ks, slots, cache
        torch.cuda.empty_cache()
        return {"kernel": "csa2_quant_kv_fp4", "tokens": n, "bytes_per_token": per_tok, "ms_per_launch": ms,
                "achieved": ach, "peak": hbm, "unit": "GB/s", "frac": ach / hbm, "frac_of_8tbs": ach / NOMINAL_HBM_GBS,
                "input": "B x T tokens of N(0,1) bf16 + indexer keys, rewritten into the workload's slots"}
    except Exception as e:
        return {"kernel": "csa2_quant_kv_fp4", "error": f"{type(e).__name__}: {e}"[:300]}


def replay_leg(args, wl, stream, hbm) -> dict:
    """csa2_swa_replay_attn (SWA bounded replay): every sequence of the
    workload recomputes its last 128 window positions, L = 128 queries over a
    255-row bf16 band. Reports queries/s and both rooflines: HBM (q in, o and
    lse out, band in) and tensor (QK + PV flops). Events around each launch;
    an L2 flush before each."""
    from compressed_sparse_attention_quant_b200 import lib
    try:
        B, L = wl.batch, lib.WINDOW
        g = torch.Generator(device=stream.device).manual_seed(11)
        q = torch.randn(B, L, lib.HEADS, lib.DIM, device=stream.device, dtype=torch.bfloat16, generator=g)
        swa = torch.randn(B, lib.WINDOW + L - 1, lib.DIM, device=stream.device, dtype=torch.bfloat16,
                          generator=g)
        lens = torch.full((B,), wl.context, dtype=torch.int32, device=stream.device)
        out = torch.empty(B, L, lib.HEADS, lib.DIM, dtype=torch.float32, device=stream.device)
        lse = torch.empty(B, L, lib.HEADS, dtype=torch.float32, device=stream.device)
        scale = 1.0 / lib.DIM ** 0.5
        flush = torch.empty(256 << 20, dtype=torch.uint8, device=stream.device)
        for _ in range(2):
            lib.swa_replay_attn(q, swa, lens, scale, out=out, lse=lse)
        torch.cuda.synchronize()
        evs = []
        for _ in range(args.steps):
            flush.zero_()
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            lib.swa_replay_attn(q, swa, lens, scale, out=out, lse=lse)
            e1.record(stream)
            evs.append((e0, e1))
        torch.cuda.synchronize()
        ms = sum(a.elapsed_time(b) for a, b in evs) / args.steps
        n_q = B * L
        nbytes = n_q * lib.HEADS * (lib.DIM * 2 + lib.DIM * 4 + 4) + B * (lib.WINDOW + L - 1) * lib.DIM * 2
        flops = 4.0 * lib.HEADS * lib.DIM * lib.WINDOW * n_q
        gbs = nbytes / (ms * 1e-3) / 1e9
        tfs = flops / (ms * 1e-3) / 1e12
        bf16_peak, bf16_kind = tensor_peak()
        del q, swa, out, lse, flush
        torch.cuda.empty_cache()
        return {"kernel": "csa2_swa_replay_attn", "sequences": B, "queries_per_sequence": L,
                "value": n_q / (ms * 1e-3), "unit": "queries/s", "ms_per_launch": ms,
                "bytes_per_launch": nbytes, "hbm_gbs": gbs, "hbm_frac": gbs / hbm,
                "flops_per_launch": flops, "tflops": tfs, "tensor_peak_tflops": bf16_peak,
                "tensor_frac": tfs / bf16_peak,
                "tensor_peak_kind": bf16_kind, "device_status": lib.status_string(lib.last_device_error()),
                "input": "N(0,1) bf16 queries and band, every row inside the sequence"}
    except Exception as e:
        return {"kernel": "csa2_swa_replay_attn", "error": f"{type(e).__name__}: {e}"[:300]}


def run_gpu(args, wl):
    from compressed_sparse_attention_quant_b200 import lib, workload
    from compressed_sparse_attention_quant_b200.group import StepGraph

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    # Each rank runs its own replica (different seed): weak scaling.
    wl_r = replicas.replica_workload(wl, rank)
    dw = workload.DeviceWorkload(wl_r, dev)
    g = dw.group
    stream = torch.cuda.current_stream(dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    acct = dw.algorithmic_bytes()
    n_idx_calls = sum(1 for m in wl.modes if m in ("F", "R"))

    # Timed step with events around the indexer_topk calls (the dominant op).
    def step_instrumented(ev_pairs):
        for li, mode in enumerate(g.modes):
            cache = g.cache(li)
            if mode == "F":
                x_new, slots, kid, ks = dw.append[li]
                lib.quant_kv_fp4(x_new, slots, cache, kid, ks)
            if mode in ("F", "R"):
                e0 = torch.cuda.Event(enable_timing=True)
                e1 = torch.cuda.Event(enable_timing=True)
                e0.record(stream)
                lib.indexer_topk(dw.q_idx[li], dw.w[li], cache, dw.page_table, dw.seq_lens, g.k,
                                 out=g._index[li], ws=g.ws_idx)
                e1.record(stream)
                ev_pairs.append((e0, e1))
            lib.sparse_attn_decode(dw.q[li], cache, dw.page_table, dw.seq_lens, g.index(li), dw.swa[li],
                                   g.scale, out=g.out[li], lse=g.lse[li], ws=g.ws_att)

    for _ in range(args.warmup):
        flush.zero_()
        step_instrumented([])
    # The timed step: the whole group step as one CUDA graph (the same
    # kernels, their programmatic overlap kept as graph edges), or the eager
    # library calls with --eager.
    if args.eager:
        run_step, per_step = dw.step, None
    else:
        sg = dw.capture()
        run_step, per_step = sg.replay, sg.launches
        for _ in range(args.warmup):
            flush.zero_()
            run_step()
    torch.cuda.synchronize(dev)
    if dist:
        dist.barrier()
    torch.cuda.synchronize(dev)

    # Timed region: K whole steps, events only around each step (events
    # between the step's kernels would break their programmatic overlap).
    # The roofline of the dominant call comes from a second region of K
    # steps with events around each csa2_indexer_topk call.
    step_events, idx_events = [], []
    with ClockSampler(local) as clk:
        time.sleep(0.01)                          # first clock sample before the region
        torch.cuda.nvtx.range_push("timed")
        launches0 = lib.launch_count()
        for _ in range(args.steps):
            if not args.no_flush:
                flush.zero_()                    # untimed: evict L2 between steps
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            run_step()
            e1.record(stream)
            step_events.append((e0, e1))
        # library kernels launched in the region: counted at each launch call
        # when eager, and per replay from the capture when graphed
        launches = lib.launch_count() - launches0 if per_step is None else per_step * args.steps
        torch.cuda.nvtx.range_pop()
        torch.cuda.synchronize(dev)
        for _ in range(args.steps):
            if not args.no_flush:
                flush.zero_()
            step_instrumented(idx_events)
        torch.cuda.synchronize(dev)
    if dist:
        dist.barrier()
    torch.cuda.synchronize(dev)
    step_ms = sum(a.elapsed_time(b) for a, b in step_events) / args.steps
    idx_ms = sum(a.elapsed_time(b) for a, b in idx_events) / max(len(idx_events), 1)
    status = lib.last_device_error()

    # End to end through the public API: every step uploads its inputs from
    # pinned host memory and downloads its outputs to pinned host memory. The
    # copies run on an upload and a download stream, double-buffered, so step
    # i+1's upload and step i's download overlap compute (a serving pipeline). The
    # per-step working set (627 MB at the 128K batch-64 workload) is larger
    # than L2, so no flush runs inside this region.
    def clone_inputs():
        return {"q": [t.clone() for t in dw.q],
                "q_idx": {li: t.clone() for li, t in dw.q_idx.items()},
                "w": {li: t.clone() for li, t in dw.w.items()},
                "append": {li: tuple(t.clone() for t in tup) for li, tup in dw.append.items()}}

    def flat_inputs(d):
        ts = list(d["q"]) + list(d["q_idx"].values()) + list(d["w"].values())
        for tup in d["append"].values():
            ts.extend(tup)
        return ts

    dev_in = [clone_inputs(), clone_inputs()]
    host_in = [t.cpu().pin_memory() for t in flat_inputs(dev_in[0])]
    dev_out = [([t.clone() for t in g.out], [t.clone() for t in g.lse]) for _ in range(2)]
    host_out = [[torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in g.out + g.lse] for _ in range(2)]
    h2d = sum(h.numel() * h.element_size() for h in host_in)
    d2h = sum(h.numel() * h.element_size() for h in host_out[0])
    ustream = torch.cuda.Stream(dev)                    # uploads (run ahead of compute)
    dstream = torch.cuda.Stream(dev)                    # downloads
    up_done = [torch.cuda.Event() for _ in range(2)]
    comp_done = [torch.cuda.Event() for _ in range(2)]
    down_done = [torch.cuda.Event() for _ in range(2)]
    used = [False, False]

    # One CUDA graph of the step per buffer set (graphs read and write the
    # tensors they were captured with); eager calls with --eager.
    if args.eager:
        e2e_graphs = None
    else:
        e2e_graphs = [StepGraph(g, dw.page_table, dw.seq_lens, dev_in[s]["q"], dw.swa, dev_in[s]["q_idx"],
                                dev_in[s]["w"], dev_in[s]["append"], out=dev_out[s][0], lse=dev_out[s][1])
                      for s in range(2)]

    def e2e_step(i):
        s = i % 2
        with torch.cuda.stream(ustream):
            if used[s]:
                ustream.wait_event(comp_done[s])        # step i-2 no longer reads this input set
            for d, h in zip(flat_inputs(dev_in[s]), host_in):
                d.copy_(h, non_blocking=True)
            up_done[s].record(ustream)
        stream.wait_event(up_done[s])
        if used[s]:
            stream.wait_event(down_done[s])             # step i-2's outputs have left this set
        if e2e_graphs is None:
            g.step(dw.page_table, dw.seq_lens, dev_in[s]["q"], dw.swa, dev_in[s]["q_idx"], dev_in[s]["w"],
                   dev_in[s]["append"], out=dev_out[s][0], lse=dev_out[s][1])
        else:
            e2e_graphs[s].replay()
        comp_done[s].record(stream)
        with torch.cuda.stream(dstream):
            dstream.wait_event(comp_done[s])
            for h, d in zip(host_out[s], dev_out[s][0] + dev_out[s][1]):
                h.copy_(d, non_blocking=True)
            down_done[s].record(dstream)
        used[s] = True

    for i in range(args.warmup):
        e2e_step(i)
    torch.cuda.synchronize(dev)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(ustream)
    for i in range(args.warmup, args.warmup + args.steps):
        e2e_step(i)
    e1.record(dstream)
    torch.cuda.synchronize(dev)
    e2e_ms = e0.elapsed_time(e1) / args.steps

    # The indexer FP8 quantiser (csa2_quant_indexer_fp8) over the keys of the
    # whole cache: B x T rows of 64 bf16 channels (seeded N(0, 1), generated
    # on the device), far larger than L2, so no flush. Events around each
    # launch on its stream.
    q8_rows = wl.batch * wl.context
    q8_gen = torch.Generator(device=dev).manual_seed(1000 + rank)
    q8_x = torch.randn(q8_rows, lib.IDX_DIM, generator=q8_gen, device=dev, dtype=torch.bfloat16)
    q8_codes = torch.empty(q8_rows, lib.IDX_DIM, dtype=torch.uint8, device=dev)
    q8_sigma = torch.empty(q8_rows, dtype=torch.float32, device=dev)
    for _ in range(2):
        lib.quant_indexer_fp8(q8_x, q8_codes, q8_sigma)
    torch.cuda.synchronize(dev)
    q8_events = []
    for _ in range(args.steps):
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        lib.quant_indexer_fp8(q8_x, q8_codes, q8_sigma)
        e1.record(stream)
        q8_events.append((e0, e1))
    torch.cuda.synchronize(dev)
    q8_ms = sum(a.elapsed_time(b) for a, b in q8_events) / args.steps
    del q8_x, q8_codes, q8_sigma

    step_ms, idx_ms, e2e_ms, q8_ms = replicas.max_over_ranks([step_ms, idx_ms, e2e_ms, q8_ms], dist, dev)

    tokens_per_rank = wl.batch * wl.q_tokens
    value = replicas.job_throughput(tokens_per_rank, world, step_ms)
    hbm, peak_kind = peaks()
    idx_bytes = (acct["indexer"] + acct["topk_io"]) / max(n_idx_calls, 1)
    achieved = idx_bytes / (idx_ms * 1e-3) / 1e9
    traffic = recorded_traffic(wl.name)
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": step_ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "fp4-e2m1/e4m3 cache, fp8 indexer, f16 mma, fp32 accum",
        "data": "synthetic",
        "config": {"workload": wl.name, "batch": wl.batch, "q_tokens": wl.q_tokens, "context": wl.context,
                   "top_k": wl.top_k, "modes": "".join(wl.modes), "parallelism": f"replicas x{world}",
                   "l2": "inputs > L2; plus 256 MB L2 flush between steps (untimed)"
                   if not args.no_flush else "inputs > L2, no flush",
                   "e2e": "pinned H2D inputs + D2H outputs every step, double-buffered on upload / "
                          "download streams overlapping compute; working set > L2, no flush",
                   "launch": "eager library calls" if args.eager else
                             "the step's library kernels replayed as one CUDA graph"},
        "step_hbm_gbs": acct["total"] / (step_ms * 1e-3) / 1e9,
        "step_frac_of_8tbs": acct["total"] / (step_ms * 1e-3) / 1e9 / NOMINAL_HBM_GBS,
        "step_frac_of_measured_copy": acct["total"] / (step_ms * 1e-3) / 1e9 / hbm,
        "roofline": {"bound": "hbm", "kernel": "csa2_indexer_topk (indexer score + exact top-k)",
                     "achieved": achieved, "peak": hbm, "peak_kind": peak_kind, "unit": "GB/s",
                     "frac": achieved / hbm, "frac_of_measured_copy": achieved / hbm,
                     "frac_of_8tbs": achieved / NOMINAL_HBM_GBS, "traffic": traffic, "ms_per_launch": idx_ms,
                     "algorithmic_bytes_per_launch": idx_bytes},
        "e2e": {"value": replicas.job_throughput(tokens_per_rank, world, e2e_ms), "unit": "tokens/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": launches,
        "device_status": lib.status_string(status),
        "indexer_fp8_quant": {"kernel": "csa2_quant_indexer_fp8", "rows": q8_rows,
                              "bytes_per_row": Q8_BYTES_PER_ROW, "ms_per_launch": q8_ms,
                              "achieved": q8_rows * Q8_BYTES_PER_ROW / (q8_ms * 1e-3) / 1e9, "peak": hbm,
                              "unit": "GB/s",
                              "frac": q8_rows * Q8_BYTES_PER_ROW / (q8_ms * 1e-3) / 1e9 / hbm,
                              "input": "B x T rows of 64 bf16 channels, N(0,1) seeded, > L2"},
    }
    clocks = clk.summary()
    if clocks:
        line["clocks"] = clocks
    line["attention_tflops_per_step"] = attention_flops(wl) / 1e12
    if world == 1:
        line["indexer_pool_topk"] = pool_leg(args, wl, dw, lib, flush, stream, hbm)
        line["kv_quant_bulk"] = bulk_quant_leg(args, wl, dw, stream, hbm)
        line["swa_replay"] = replay_leg(args, wl, stream, hbm)
    if world == 1 and not args.no_other_workloads:
        del dw, g
        torch.cuda.empty_cache()
        line["workloads"] = {name: other_workload(args, name, dev, flush, stream, hbm, not args.no_cpu_baseline)
                             for name in inputs.WORKLOADS if name != wl.name}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import oracle
        line["cpu_baseline"] = cpu_baseline(wl, args.ref_seqs, args.cpu_budget, oracle.host_cores())
        line["cpu_baseline_1core"] = cpu_baseline(wl, args.ref_seqs, args.cpu_budget / 2, 1)
    if dist:
        dist.barrier()
        dist.destroy_process_group()
    if replicas.reports(rank):
        print(json.dumps(line), flush=True)


def relaunch_under_torchrun(args) -> int:
    """`--gpus N` (N > 1) started as a plain process: run this same command as
    N ranks of one node under torch.distributed.run (127.0.0.1 rendezvous) and
    return its exit status. Rank 0's JSON line is the output."""
    import socket
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={args.gpus}",
           "--master-addr=127.0.0.1", f"--master-port={port}", os.path.abspath(__file__)] + sys.argv[1:]
    return subprocess.call(cmd)


def dry_run(args):
    """The launch path without the workload: every rank joins the process
    group (NCCL with GPUs, else gloo), the max-over-ranks reduction runs on a
    per-rank dummy time, and rank 0 prints one line with the world size."""
    import datetime
    import torch.distributed as dist
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    dev = None
    if world > 1:
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", "0")))
            torch.cuda.set_device(dev)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=60))
    (ms,) = replicas.max_over_ranks([1.0 + rank], dist if world > 1 else None, dev)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if replicas.reports(rank):
        print(json.dumps({"dry_run": True, "n_gpus": world, "ms_per_step": ms, "ranks_reporting": 1}),
              flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="csa2", choices=["csa2", "reference"])
    ap.add_argument("--workload", default="decode_b64_t128k",
                    choices=sorted(inputs.WORKLOADS) + sorted(inputs.PROFILE_WORKLOADS))
    ap.add_argument("--no-flush", action="store_true")
    ap.add_argument("--eager", action="store_true", help="time eager library calls instead of the step's CUDA graph")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-budget", type=float, default=10.0, help="seconds of oracle work (cpu_baseline)")
    ap.add_argument("--ref-seqs", type=int, default=2, help="sequences the oracle arm prepares")
    ap.add_argument("--dry-run", action="store_true", help="launch path only (process group, max over ranks)")
    ap.add_argument("--no-other-workloads", action="store_true", help="time only --workload")
    ap.add_argument("--cpu-budget-other", type=float, default=3.0,
                    help="seconds of oracle work per other workload")
    args = ap.parse_args()
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        sys.exit(relaunch_under_torchrun(args))
    if args.dry_run:
        dry_run(args)
        return
    wl = {**inputs.WORKLOADS, **inputs.PROFILE_WORKLOADS}[args.workload]
    if args.impl == "reference":
        run_reference(args, wl)
    else:
        run_gpu(args, wl)


if __name__ == "__main__":
    main()
