"""Benchmark of the KDA forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One JSON line on rank 0.  Headline: prefill tokens/s on the long-context
workload (1 x 131072 tokens, H=32, dk=dv=128, bf16), one kda_chunk_fwd call
per step, inputs resident in HBM and larger than L2 (6.4 GB read per step).
Alongside: the decode step (256 sequences x 32 heads, 512 MiB fp32 state,
1000 consecutive in-place steps) as achieved HBM GB/s, the roofline of both
against the measured peaks, an end-to-end figure through the same public
call with host buffers, and the fp64 CPU oracle timed on a bounded sample.

Multi-GPU (torchrun, one process per GPU): every rank runs its own replica of
the workload (sequences and heads are independent -- no data-path
collective); value = tokens over all ranks / max-over-ranks device time.
"""
from __future__ import annotations

import argparse
import dataclasses
import ctypes
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from kda_linear_attention_fwd_b200 import kda  # noqa: E402
from kda_linear_attention_fwd_b200 import workloads as W  # noqa: E402

METRIC = "KDA prefill tokens/s (H=32,d=128) & decode-step state GB/s vs B200 roofline"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# DRAM traffic of the dominant kernel, per launch: read from the committed
# ncu summary profiles/traffic.json, which records the figure together with a
# hash of the sources of the prefill call it was captured from (its entry
# point, the plan and scan, the chunk kernels and their headers).  When those
# differ from the hash (a kernel on the path changed since the capture) the
# figure is stale and `traffic` is reported as null.
PREFILL_SOURCES = ("kda_api.cu", "kda_args.h", "kda_chain.cu", "kda_plan.cu", "kda_prefill_c32.cu",
                   "kda_prefill_mma.cu", "kda_prefill_simt.cu", "kda_prefill_tc.cu", "kda_common.cuh",
                   "kda_prefill.cuh", "kda_sm100.cuh")


BACKWARD_SOURCES = ("kda_bwd.cu", "kda_common.cuh", "kda_sm100.cuh")


def source_hash(sources=PREFILL_SOURCES):
    import hashlib
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "kda_linear_attention_fwd_b200", "csrc")
    for name in sources:
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(name.encode() + b"\0" + f.read())
    return h.hexdigest()[:16]


def measured_traffic(workload, sources=PREFILL_SOURCES):
    """(bytes per launch of the dominant kernel, kernel name, source) or
    (None, None, reason); `workload` keys profiles/traffic.json, whose entry
    holds the hash of `sources` it was captured from."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None, None, "no committed capture"
    with open(path) as f:
        d = json.load(f).get(workload)
    if not d:
        return None, None, "no capture for this workload"
    if d.get("source_hash") != source_hash(sources):
        return None, d.get("kernel"), "stale: kernel sources changed since the capture"
    return float(d["bytes_per_launch"]), d.get("kernel"), d.get("source", "profiles/traffic.json")


def prefill_bytes(w, T, N):
    """Algorithmic HBM bytes of one prefill call: read q, k, g, v, gate, beta,
    write y (dtype), read the initial and write the final state (fp32)."""
    e = 2 if w.dtype == "bf16" else 4
    per_tok_head = (3 * w.dk + 3 * w.dv + 1) * e
    states = N * w.H * w.dk * w.dv * 4 * ((1 if w.init_state else 0) + 1)
    return T * w.H * per_tok_head + states


def prefill_flops(w, T):
    """Chunk-form FLOPs per token-head: the three state contractions
    (W S, Qd S, Kb^T U: 6 dk dv) and the intra-chunk products
    (Kd Ki^T, Qd Ki^T, W, U0, P U: 2 C (3 dk + 2 dv)), C = 16."""
    C = 16
    return T * w.H * (6 * w.dk * w.dv + 2 * C * (3 * w.dk + 2 * w.dv))


def decode_bytes(wd):
    nh = wd.num_seqs * wd.H
    e = 2
    return nh * (2 * wd.dk * wd.dv * 4 + (3 * wd.dk + 3 * wd.dv + 1) * e)


class Clocks:
    """nvidia-smi sampler for the timed region: samples every 20 ms, and
    only those whose timestamps fall between mark_start() and mark_end()
    count (the region can be shorter than one sample period; then the
    nearest samples stand in and `samples` says 0)."""

    def __init__(self, path):
        self.path = path
        self.proc = None
        self.t0 = self.t1 = None

    def start(self):
        try:
            uuid = "GPU-" + str(torch.cuda.get_device_properties(torch.cuda.current_device()).uuid)
            q = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
                 "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
                 "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", "-i", uuid, f"--query-gpu={q}",
                                          "--format=csv,noheader,nounits", "-lms", "20"],
                                         stdout=self.f, stderr=subprocess.DEVNULL)
            deadline = time.time() + 5.0  # until the sampler is live
            while time.time() < deadline and os.path.getsize(self.path) == 0:
                time.sleep(0.05)
        except Exception:
            self.proc = None

    def mark_start(self):
        self.t0 = time.time()

    def mark_end(self):
        self.t1 = time.time()

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.1)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.f.close()
        from datetime import datetime
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) < 10:
                    continue
                try:
                    t = datetime.strptime(parts[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
                    rows.append((t, float(parts[2]), float(parts[3]), parts[6:10]))
                except ValueError:
                    continue
        if not rows:
            return None
        t0 = self.t0 if self.t0 is not None else rows[0][0]
        t1 = self.t1 if self.t1 is not None else rows[-1][0]
        inside = [r for r in rows if t0 <= r[0] <= t1]
        used = inside or sorted(rows, key=lambda r: min(abs(r[0] - t0), abs(r[0] - t1)))[:2]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = {n for r in used for n, v in zip(names, r[3]) if v.lower() == "active"}
        mx = used[-1][2]
        load = [r[1] for r in used if r[1] > 0.5 * mx] or [r[1] for r in used]
        return {"sm_mhz": statistics.median(load), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(inside)}


def rank_env():
    return (int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")),
            int(os.environ.get("LOCAL_RANK", "0")))


def dist_setup(backend="nccl"):
    """One process per GPU: a process group for the barrier and the
    max-over-ranks timing only (the work itself needs no collective)."""
    ws, rank, local = rank_env()
    if ws > 1:
        import torch.distributed as dist
        from datetime import timedelta
        kw = {}
        if backend == "nccl":
            torch.cuda.set_device(local)
            kw["device_id"] = torch.device("cuda", local)
        dist.init_process_group(backend, timeout=timedelta(seconds=300), **kw)
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return ws, rank, local


def barrier(ws):
    if ws > 1:
        import torch.distributed as dist
        dist.barrier()


def reduce_max(x, ws, device="cuda"):
    """Max over ranks (device time of the slowest rank)."""
    if ws == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate(units_per_rank, ms_total, ws):
    """Whole-job throughput: units processed by all ranks / slowest time."""
    return ws * units_per_rank / (ms_total / 1e3)


def cpu_baseline(w, threads=None, tokens=None):
    """The fp64 oracle on a bounded sample of the workload: all heads of the
    first `tokens` tokens of one sequence.  Returns (tokens/s at H, cores,
    sample description)."""
    import numpy as np

    import oracle
    from concurrent.futures import ThreadPoolExecutor
    cores = threads or os.cpu_count() or 1
    if tokens is None:
        tokens = int(min(w.lengths[0], max(4096, 512 * cores)))
    with ThreadPoolExecutor(min(32, cores)) as ex:
        heads = list(ex.map(lambda h: W.head_inputs(w, 0, h, length=tokens), range(w.H)))
    st = lambda key: np.stack([x[key].numpy() for x in heads], axis=1)
    q, k, v, g, gate = st("q"), st("k"), st("v"), st("g"), st("gate")
    beta = np.stack([x["beta"].numpy() for x in heads], axis=1)
    t0 = time.perf_counter()
    _, _, used = oracle.varlen(q, k, v, g, beta, gate, [0, tokens], threads=cores)
    dt = time.perf_counter() - t0
    return tokens / dt, used, f"{tokens} tokens x {w.H} heads of {w.name} (fp64, per token)"


def workload_config(w, ws):
    """The `config` keys both arms share (the workload, named by its sizes)."""
    T, N = w.total_tokens, w.num_seqs
    return {"workload": f"{w.name}: {N} sequence(s), {T} tokens, H={w.H}, "
                        f"dk={w.dk}, dv={w.dv}, {w.dtype}, chunk=16",
            "global_batch": ws * N, "seq_len": T,
            "parallelism": f"replicas x{ws} (sequences/heads independent)",
            "l2": "inputs larger than L2 (%.1f GB per step)" % (prefill_bytes(w, T, N) / 1e9)}


def run_reference(args, ws, rank):
    """Reference arm: the fp64 CPU oracle, timed on the host cores, on a
    bounded sample of the same workload each step."""
    if rank != 0:
        return
    w = W.get(args.workload)
    cores = os.cpu_count() or 1
    tokens = args.ref_tokens or int(min(w.lengths[0], max(1024, 256 * cores)))
    for _ in range(args.warmup):
        cpu_baseline(w, cores, tokens)
    el = 0.0
    for _ in range(args.steps):  # oracle time only (input generation excluded)
        v, used, sample = cpu_baseline(w, cores, tokens)
        el += tokens / v
    value = args.steps * tokens / el
    line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": ws,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * el / args.steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": dict(workload_config(w, ws), sample_tokens_per_step=tokens),
            "impl": "reference",
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": used, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0},
            "gpu_launches": 0}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="long_bf16")
    ap.add_argument("--decode-steps", type=int, default=1000)
    ap.add_argument("--e2e-steps", type=int, default=4)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-kcp", action="store_true",
                    help="skip the per-rank context-parallel measurement")
    ap.add_argument("--no-ex", action="store_true",
                    help="skip the extended-path measurement (flags + state snapshots)")
    ap.add_argument("--no-bwd", action="store_true",
                    help="skip the backward measurement")
    ap.add_argument("--out-dir", default=os.path.join(tempfile.gettempdir(), "kda_bench"),
                    help="where the nvidia-smi clock samples of the timed region are written")
    ap.add_argument("--tokens", type=int, default=0,
                    help="profiling only: run a one-sequence workload at this length (a smaller case "
                         "of the same kernels); 0 = the workload's own length")
    ap.add_argument("--ref-tokens", type=int, default=0,
                    help="reference arm: tokens per step sample (0 = scale with cores)")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3) if args.impl == "ours" else args.warmup

    if args.impl == "reference":
        # CPU oracle on rank 0 only; other ranks exit without work and
        # without a process group (no collective can wait on them)
        ws, rank, _ = rank_env()
        run_reference(args, ws, rank)
        return
    ws, rank, local = dist_setup("nccl")

    from kda_linear_attention_fwd_b200 import build
    if rank == 0:
        build.build()
    barrier(ws)
    lib = kda.load()
    pk, pk_kind = peaks()
    dev = torch.device("cuda", torch.cuda.current_device())
    stream = torch.cuda.current_stream()

    # ---------------- prefill ----------------
    w = W.get(args.workload)
    if args.tokens:
        if len(w.lengths) != 1:
            raise SystemExit("--tokens applies to one-sequence workloads only")
        w = dataclasses.replace(w, lengths=(args.tokens,))
    T, N = w.total_tokens, w.num_seqs
    inp = W.fast_prefill(w, seed=w.seed + 1000 * rank, device=dev)
    out = torch.empty(T, w.H, w.dv, dtype=w.torch_dtype, device=dev)
    fin = torch.empty(N, w.H, w.dk, w.dv, dtype=torch.float32, device=dev)
    plan = kda.plan(T, N, w.H)
    ws_bytes = kda.workspace_size(T, N, w.H, w.dk, w.dv, w.torch_dtype)
    wsp = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    cu_host = inp["cu_seqlens"].tolist()

    def prefill():
        kda.chunk_fwd(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], inp["gate"],
                      inp["cu_seqlens"], initial_state=inp["initial_state"], final_state=fin,
                      out=out, workspace=wsp, cu_seqlens_host=cu_host, stream=stream)

    for _ in range(args.warmup):
        prefill()
    torch.cuda.synchronize()
    os.makedirs(args.out_dir, exist_ok=True)
    clocks = Clocks(os.path.join(args.out_dir, f"clocks_rank{rank}.csv"))
    clocks.start()
    barrier(ws)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks.mark_start()
    e0.record(stream)
    for _ in range(args.steps):
        prefill()
    e1.record(stream)
    torch.cuda.synchronize()
    clocks.mark_end()
    barrier(ws)
    ms_total = reduce_max(e0.elapsed_time(e1), ws)
    clk = clocks.stop()
    ms = ms_total / args.steps
    value = aggregate(T * args.steps, ms_total, ws)
    pbytes = prefill_bytes(w, T, N)
    pflops = prefill_flops(w, T)
    hbm = pk["hbm_gbs"]
    achieved = pbytes / (ms / 1e3) / 1e9
    traffic, _, traffic_src = (measured_traffic(args.workload) if not args.tokens
                               else (None, None, "shortened workload"))
    roofline = {"bound": "hbm", "achieved": achieved, "peak": hbm, "unit": "GB/s",
                "frac": achieved / hbm,
                "traffic": traffic,
                "traffic_source": traffic_src,
                "kernel": "kda_chunk_fwd call (%d launches)" % plan["launches"],
                "peak_source": f"{pk_kind} hbm_gbs",
                "tensor_tflops": pflops / (ms / 1e3) / 1e12,
                "tensor_frac_of_peak": pflops / (ms / 1e3) / 1e12 / pk["bf16_tflops"],
                "roofline_model_frac": max(pbytes / (hbm * 1e9),
                                           pflops / (pk["bf16_tflops"] * 1e12)) / (ms / 1e3)}

    # ------- extended path: in-kernel preprocessing + snapshots, same inputs -------
    exm = None
    if not args.no_ex:
        B = 8192  # a state snapshot every 8192 tokens of each sequence
        offs = kda.snapshot_offsets([cu_host[i + 1] - cu_host[i] for i in range(N)], B)
        offs_dev = torch.tensor(offs, dtype=torch.int32, device=dev)
        snaps = torch.empty(max(offs[-1], 1), w.H, w.dk, w.dv, dtype=torch.float32, device=dev)
        P = ctypes.c_void_p
        ptr = lambda t: P(t.data_ptr())
        cu_arr = (ctypes.c_int32 * len(cu_host))(*cu_host)
        ex_args = (ptr(inp["q"]), ptr(inp["k"]), ptr(inp["v"]), ptr(inp["g"]), ptr(inp["beta"]),
                   ptr(inp["gate"]), ptr(out), ptr(inp["cu_seqlens"]), ctypes.cast(cu_arr, P),
                   N, T, w.H, w.dk, w.dv, kda._dtype_code(inp["q"]), 1.0, 15,
                   None if inp["initial_state"] is None else ptr(inp["initial_state"]), ptr(fin),
                   B, ptr(snaps), ptr(offs_dev), ptr(wsp), ws_bytes, P(stream.cuda_stream))

        def ex_call():
            rc = lib.kda_chunk_fwd_ex(*ex_args)
            if rc != 0:
                raise RuntimeError(kda.status_string(rc))

        for _ in range(args.warmup):
            ex_call()
        torch.cuda.synchronize()
        barrier(ws)
        x0, x1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        x0.record(stream)
        for _ in range(args.steps):
            ex_call()
        x1.record(stream)
        torch.cuda.synchronize()
        barrier(ws)
        xms = reduce_max(x0.elapsed_time(x1), ws) / args.steps
        exm = {"value": ws * T / (xms / 1e3), "unit": "tokens/s", "ms_per_step": xms,
               "vs_plain_time": xms / ms, "flags": "qk_l2norm|beta_logits|gate_logits|clamp_decay",
               "snapshot_tokens": B, "snapshots_per_head": offs[-1],
               "snapshot_bytes": offs[-1] * w.H * w.dk * w.dv * 4,
               "gpu_launches": plan["launches"] * args.steps}
        del snaps, offs_dev

    # ------- context parallelism: what one rank of an 8-way split runs -------
    # (measured on this GPU: the map of its segment, the fold of the 7 maps
    # before it, the prefill of its segment; the all-gather is not timed here)
    kcpm = None
    if not args.no_kcp and N == 1:
        R = 8
        seg = T // R
        sl = slice((R - 1) * seg, R * seg)  # the last rank folds the most maps
        sk = {x: inp[x][sl].contiguous() for x in ("q", "k", "v", "g", "beta", "gate")}
        scu = torch.tensor([0, seg], dtype=torch.int32, device=dev)
        scu_h = [0, seg]
        Mz = torch.zeros(R - 1, 1, w.H, w.dk, w.dk, device=dev)
        Zz = torch.zeros(R - 1, 1, w.H, w.dk, w.dv, device=dev)
        sout = torch.empty(seg, w.H, w.dv, dtype=w.torch_dtype, device=dev)
        sfin = torch.empty(1, w.H, w.dk, w.dv, device=dev)

        def t_ms(fn, reps):
            for _ in range(2):
                fn()
            torch.cuda.synchronize()
            c0, c1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            c0.record(stream)
            for _ in range(reps):
                fn()
            c1.record(stream)
            torch.cuda.synchronize()
            return reduce_max(c0.elapsed_time(c1), ws) / reps

        ms_sum = t_ms(lambda: kda.chunk_summary(sk["k"], sk["v"], sk["g"], sk["beta"], scu,
                                                cu_seqlens_host=scu_h, workspace=wsp,
                                                stream=stream), args.steps)
        s_in = torch.zeros(1, w.H, w.dk, w.dv, device=dev)
        ms_cmp = t_ms(lambda: kda.state_compose(Mz, Zz, s_in, stream=stream), args.steps)
        ms_pre = t_ms(lambda: kda.chunk_fwd(sk["q"], sk["k"], sk["v"], sk["g"], sk["beta"],
                                            sk["gate"], scu, initial_state=s_in, final_state=sfin,
                                            out=sout, workspace=wsp, cu_seqlens_host=scu_h,
                                            stream=stream), args.steps)
        per_rank = ms_sum + ms_cmp + ms_pre
        kcpm = {"ranks_emulated": R, "segment_tokens": seg, "summary_ms": ms_sum,
                "fold_ms": ms_cmp, "segment_prefill_ms": ms_pre, "per_rank_ms": per_rank,
                "per_rank_tokens_per_s": seg / (per_rank / 1e3),
                "allgather_bytes_per_rank": w.H * w.dk * (w.dk + w.dv) * 4,
                "note": "one rank's kernels timed on one GPU; the all-gather is not measured"}
        del sk, Mz, Zz, sout

    # ------- backward (kda_bwd) on prefill_bf16: 2 x 4096 tokens, H = 16 -------
    bwdm = None
    if not args.no_bwd:
        wb = W.get("prefill_bf16")
        bi = W.fast_prefill(wb, seed=wb.seed + 1000 * rank, device=dev)
        Tb, Nb = wb.total_tokens, wb.num_seqs
        gb = torch.Generator(device=dev).manual_seed(wb.seed + 7)
        dyb = torch.randn(Tb, wb.H, wb.dv, generator=gb, device=dev).to(wb.torch_dtype)
        dsfb = torch.randn(Nb, wb.H, wb.dk, wb.dv, generator=gb, device=dev)
        f32b = dict(dtype=torch.float32, device=dev)
        gq, gk, gg = (torch.empty(Tb, wb.H, wb.dk, **f32b) for _ in range(3))
        gv, ggt = (torch.empty(Tb, wb.H, wb.dv, **f32b) for _ in range(2))
        gbt = torch.empty(Tb, wb.H, **f32b)
        gs0 = torch.empty(Nb, wb.H, wb.dk, wb.dv, **f32b)
        wsb_bytes = kda.bwd_workspace_size(Tb, Nb, wb.H, wb.dk, wb.dv)
        wsb = torch.empty(wsb_bytes, dtype=torch.uint8, device=dev)
        cub = bi["cu_seqlens"].tolist()
        cub_arr = (ctypes.c_int32 * len(cub))(*cub)
        Pb = ctypes.c_void_p
        pb = lambda t: Pb(t.data_ptr())
        bargs = (pb(bi["q"]), pb(bi["k"]), pb(bi["v"]), pb(bi["g"]), pb(bi["beta"]),
                 pb(bi["gate"]), pb(dyb), pb(bi["cu_seqlens"]), ctypes.cast(cub_arr, Pb), Nb, Tb,
                 wb.H, wb.dk, wb.dv, kda._dtype_code(bi["q"]), 1.0, None, pb(dsfb), pb(gq),
                 pb(gk), pb(gv), pb(gg), pb(gbt), pb(ggt), pb(gs0), pb(wsb), wsb_bytes,
                 Pb(stream.cuda_stream))

        def bwd_call():
            rc = lib.kda_bwd(*bargs)
            if rc != 0:
                raise RuntimeError(kda.status_string(rc))

        for _ in range(args.warmup):
            bwd_call()
        torch.cuda.synchronize()
        barrier(ws)
        b0, b1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        b0.record(stream)
        for _ in range(args.steps):
            bwd_call()
        b1.record(stream)
        torch.cuda.synchronize()
        barrier(ws)
        bms = reduce_max(b0.elapsed_time(b1), ws) / args.steps
        e = 2  # bf16 inputs
        bbytes = (Tb * wb.H * ((3 * wb.dk + 3 * wb.dv + 1) * e + 4 * (3 * wb.dk + 2 * wb.dv + 1))
                  + 2 * Nb * wb.H * wb.dk * wb.dv * 4)
        bgbs = bbytes / (bms / 1e3) / 1e9
        btraffic, _, btraffic_src = measured_traffic("backward_prefill_bf16", BACKWARD_SOURCES)
        bwdm = {"value": ws * Tb / (bms / 1e3), "unit": "tokens/s", "ms_per_call": bms,
                "workload": "prefill_bf16 backward: 2 x 4096 tokens, H=16, dk=dv=128, bf16 in, "
                            "fp32 gradients, final-state gradient given",
                "roofline": {"bound": "hbm", "achieved": bgbs, "peak": hbm, "unit": "GB/s",
                             "frac": bgbs / hbm, "traffic": btraffic,
                             "traffic_source": btraffic_src,
                             "kernel": "kda_bwd call (per-chunk operands, the forward and "
                                       "reverse chains in one launch, per-chunk gradients)",
                             "peak_source": f"{pk_kind} hbm_gbs"},
                "gpu_launches": 3 * args.steps}
        del bi, dyb, dsfb, gq, gk, gg, gv, ggt, gbt, gs0, wsb

    # ---------------- decode ----------------
    dec = None
    if not args.no_decode:
        wd = W.get("decode_bf16")
        S = args.decode_steps
        dd = W.fast_decode(wd, S, seed=wd.seed + 1000 * rank, device=dev)
        state = dd["state"]
        yout = torch.empty(wd.num_seqs, wd.H, wd.dv, dtype=torch.bfloat16, device=dev)
        P = ctypes.c_void_p
        ptr = lambda t: P(t.data_ptr())
        st_ptr = P(stream.cuda_stream)
        calls = [(ptr(dd["q"][s]), ptr(dd["k"][s]), ptr(dd["v"][s]), ptr(dd["g"][s]),
                  ptr(dd["beta"][s]), ptr(dd["gate"][s])) for s in range(S)]
        yp, sp = ptr(yout), ptr(state)

        def dstep(s):
            a = calls[s]
            rc = lib.kda_decode_step(a[0], a[1], a[2], a[3], a[4], a[5], yp, sp, wd.num_seqs,
                                     wd.H, wd.dk, wd.dv, kda.KDA_DTYPE_BF16, 1.0, 0, st_ptr)
            if rc != 0:
                raise RuntimeError(kda.status_string(rc))

        for s in range(3):
            dstep(s)
        torch.cuda.synchronize()
        barrier(ws)
        d0, d1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        d0.record(stream)
        for s in range(S):
            dstep(s)
        d1.record(stream)
        torch.cuda.synchronize()
        barrier(ws)
        dms = reduce_max(d0.elapsed_time(d1), ws)
        us = 1e3 * dms / S
        db = decode_bytes(wd)
        gbs = db / (us / 1e6) / 1e9
        dec = {"value": ws * gbs, "unit": "GB/s", "us_per_step": us, "steps": S,
               "tokens_per_s": ws * wd.num_seqs * S / (dms / 1e3),
               "workload": "decode_bf16: 256 seqs x H=32, dk=dv=128, 512 MiB fp32 state",
               "roofline": {"bound": "hbm", "achieved": gbs, "peak": hbm, "unit": "GB/s",
                            "frac": gbs / hbm, "traffic": None,
                            "kernel": "decode_step_kernel<128,128,bf16>",
                            "peak_source": f"{pk_kind} hbm_gbs"},
                "gpu_launches": S}
        del dd, state, calls

    # ---------------- end to end (host buffers) ----------------
    # Every step copies its inputs from pinned host memory, runs the call and
    # copies y and the final states back.  Two device buffer sets let step
    # i + 1's inputs cross the host link while step i computes and its result
    # goes back (the link is full duplex), as a serving loop would run it.
    e2e = None
    if not args.no_e2e:
        names = ("q", "k", "v", "g", "beta", "gate")
        host = {x: torch.empty(inp[x].shape, dtype=inp[x].dtype, pin_memory=True) for x in names}
        for x in names:
            host[x].copy_(inp[x])
        hout = torch.empty(out.shape, dtype=out.dtype, pin_memory=True)
        hfin = torch.empty(fin.shape, dtype=fin.dtype, pin_memory=True)
        h2d = sum(host[x].numel() * host[x].element_size() for x in names)
        d2h = hout.numel() * hout.element_size() + hfin.numel() * hfin.element_size()
        bufs = [{x: inp[x] for x in names}, {x: torch.empty_like(inp[x]) for x in names}]
        outs = [(out, fin), (torch.empty_like(out), torch.empty_like(fin))]
        s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
        ev_in = [torch.cuda.Event() for _ in range(2)]    # inputs of buffer b have landed
        ev_done = [torch.cuda.Event() for _ in range(2)]  # the call on buffer b is done
        ev_out = [torch.cuda.Event() for _ in range(2)]   # the result of buffer b is on the host

        def e2e_step(i):
            b = i % 2
            s_in.wait_event(ev_done[b])  # the previous call on these inputs is done
            with torch.cuda.stream(s_in):
                for x in names:
                    bufs[b][x].copy_(host[x], non_blocking=True)
            ev_in[b].record(s_in)
            stream.wait_event(ev_in[b])
            stream.wait_event(ev_out[b])  # the previous result in these outputs has left
            kda.chunk_fwd(bufs[b]["q"], bufs[b]["k"], bufs[b]["v"], bufs[b]["g"], bufs[b]["beta"],
                          bufs[b]["gate"], inp["cu_seqlens"], initial_state=inp["initial_state"],
                          final_state=outs[b][1], out=outs[b][0], workspace=wsp, cu_seqlens_host=cu_host,
                          stream=stream)
            ev_done[b].record(stream)
            s_out.wait_event(ev_done[b])
            with torch.cuda.stream(s_out):
                hout.copy_(outs[b][0], non_blocking=True)
                hfin.copy_(outs[b][1], non_blocking=True)
            ev_out[b].record(s_out)

        for i in range(2):
            e2e_step(i)
        torch.cuda.synchronize()
        barrier(ws)
        a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a0.record(s_in)
        for i in range(args.e2e_steps):
            e2e_step(i)
        s_in.wait_event(ev_out[(args.e2e_steps - 1) % 2])
        a1.record(s_in)
        torch.cuda.synchronize()
        barrier(ws)
        ems = reduce_max(a0.elapsed_time(a1), ws)
        e2e = {"value": ws * T * args.e2e_steps / (ems / 1e3), "unit": "tokens/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "ms_per_step": ems / args.e2e_steps, "steps": args.e2e_steps,
               "pipelined": "two device buffer sets: a step's host-to-device copy overlaps the "
                            "previous step's call and device-to-host copy"}
        del bufs, outs

    cpu = None
    if rank == 0 and ws == 1 and not args.no_cpu:
        v, used, sample = cpu_baseline(w)
        cpu = {"value": v, "unit": "tokens/s", "cores": used, "kind": "oracle", "sample": sample}

    if rank == 0:
        line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": ws,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
                "dtype": w.dtype, "data": "synthetic",
                "config": dict(workload_config(w, ws), piece_len=plan["piece_len"]),
                "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e,
                "gpu_launches": plan["launches"] * args.steps, "clocks": clk, "decode": dec,
                "extended": exm, "kcp": kcpm, "backward": bwdm}
        print(json.dumps(line), flush=True)
    if ws > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
