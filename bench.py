"""Benchmark of one QSA (c4) layer decode step on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Workload: decode, batch 64 per GPU, one query token per request, contexts
uniform in [120000, 131072], 16 query / 2 KV heads, d = 128, paged BF16 K/V
(64-token pages, seeded page permutation), 4 x 128 indexer heads; synthetic
inputs from qsa_gen.  One step = one qsa_decode call (ring append and
compression, query rotation, scoring of every complete block, top-512,
expansion, sparse GQA).  Every step streams ~650 MB (5x the L2), and the L2
is also flushed (512 MiB write) between timed steps, outside the timed
events.  Several GPUs run independent replicas (requests shard with no
exchange): weak scaling, time = max over ranks.

Prints one JSON line (rank 0).
"""
from __future__ import annotations

import argparse
import glob
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "QSA decode query-tok/s/layer at 128K ctx; achieved HBM GB/s vs ~8 TB/s"
UNIT = "query-tok/s"
FALLBACK_HBM_GBS = 6650.0


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--batch", type=int, default=64)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-prefill", action="store_true", help="skip the prefill-scorer measurement")
    ap.add_argument("--only-prefill", action="store_true",
                    help="run only the prefill-scorer measurement and print its JSON (for profiling it alone)")
    ap.add_argument("--no-extras", action="store_true",
                    help="skip the secondary measurements (FP8 K/V, index projection, varlen prefill, split decode)")
    ap.add_argument("--no-long-prefill", action="store_true",
                    help="with the prefill measurement, skip the 262144-token long-context prefill")
    ap.add_argument("--prefill-chunk", type=int, default=-1, metavar="POS0",
                    help="run only the 8192-query prefill chunk at POS0 of the 262144-token context, 3 times "
                         "(for profiling one chunk)")
    ap.add_argument("--cpu-seconds", type=float, default=12.0, help="target CPU work of the oracle baseline")
    return ap.parse_args()


def dist_env():
    return int(os.environ.get("RANK", 0)), int(os.environ.get("WORLD_SIZE", 1)), int(os.environ.get("LOCAL_RANK", 0))


def replica_seed(rank: int) -> int:
    """Seed of a rank's requests: every replica decodes its own batch (weak scaling, no exchange)."""
    return 2 + 1000 * rank


def max_over_ranks(times_ms, world: int, device=None):
    """Each timing's maximum over the ranks (all_reduce MAX when world > 1), so the whole job is
    as slow as its slowest replica; every rank gets the same values."""
    import torch
    import torch.distributed as dist

    t = torch.tensor([float(x) for x in times_ms], dtype=torch.float64, device=device)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        dist.barrier()
    return [float(x) for x in t.cpu()]


def job_throughput(batch_per_rank: int, world: int, step_ms_max: float) -> float:
    """Whole-job query-tokens/s: every rank's requests over the slowest rank's step time."""
    return batch_per_rank * world / (step_ms_max * 1e-3)


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return FALLBACK_HBM_GBS, "fallback"


def kernel_src_hash(files) -> str:
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


SCORER_SRC = ["block_sparse_attention_c4_b200/csrc/qsa_score.cu", "block_sparse_attention_c4_b200/csrc/qsa_common.cuh"]


def committed_traffic(src_hash: str):
    """DRAM bytes per launch of the scorer from a committed ncu summary, if it matches this source."""
    for path in glob.glob(os.path.join(ROOT, "profiles", "*.txt")):
        txt = open(path).read()
        m_h = re.search(r"^kernel_src_sha256_16:\s*(\w+)", txt, re.M)
        m_k = re.search(r"^kernel:\s*(\S+)", txt, re.M)
        m_b = re.search(r"^dram_bytes_per_full_launch:\s*([0-9.eE+]+)", txt, re.M)
        if m_h and m_k and m_b and m_k.group(1) == "k_score_topk" and m_h.group(1) == src_hash:
            return float(m_b.group(1)), os.path.relpath(path, ROOT)
    return None, None


class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled during the timed region."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
         "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
         "clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu, self.proc, self.lines = gpu_index, None, []

    def start(self):
        # NVML in a thread (10 ms period; read-only queries), else an nvidia-smi subprocess
        self.stop_flag = threading.Event()
        self.nv = self._nvml_handle()
        if self.nv is not None:
            self.t = threading.Thread(target=self._poll_nvml, daemon=True)
            self.t.start()
            return
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.Q}",
                                          "--format=csv,noheader,nounits", "-lms", "50"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except (OSError, FileNotFoundError):
            self.proc = None

    def _nvml_handle(self):
        try:
            import pynvml as nv
            import torch

            nv.nvmlInit()
            try:
                uuid = str(torch.cuda.get_device_properties(self.gpu).uuid)
                h = nv.nvmlDeviceGetHandleByUUID(uuid if uuid.startswith("GPU-") else "GPU-" + uuid)
            except Exception:
                h = nv.nvmlDeviceGetHandleByIndex(self.gpu)
            self.h = h
            return nv
        except Exception:
            return None

    def _poll_nvml(self):
        nv, h = self.nv, self.h
        bits = {"hw_slowdown": 0x8, "hw_thermal_slowdown": 0x40, "sw_thermal_slowdown": 0x20, "sw_power_cap": 0x4}
        get_reasons = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            nv.nvmlDeviceGetCurrentClocksThrottleReasons
        while not self.stop_flag.is_set():
            try:
                sm = nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)
                mx = nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM)
                r = int(get_reasons(h))
                act = ["Active" if r & b else "Not Active" for b in bits.values()]
                self.lines.append(", ".join([str(self.gpu), str(sm), str(mx), "0", hex(r)] + act))
            except Exception:
                pass
            time.sleep(0.01)

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.nv is not None:
            self.stop_flag.set()
            self.t.join(timeout=2)
            src = "nvml, 10 ms"
        elif self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        else:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.t.join(timeout=2)
            src = "nvidia-smi, 50 ms"
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm), "sampler": src}


def algorithmic_bytes(lens):
    """Bytes a decode step must move at minimum, per kernel (see the design notes):
    scorer: every complete block's compressed key (256 B) + query/weights + page-table entries + kept ids;
    gqa: K and V of both KV heads at every kept position (1 KiB) + query + output + kept ids."""
    score = gqa = 0
    for L in lens:
        nb = L // 4
        npos = 4 * min(nb, 512) + L % 4
        score += nb * 256 + 4 * 128 * 2 + 16 + 4 * ((nb + 15) // 16) + 4 * min(nb, 512)
        gqa += npos * 1024 + 16 * 128 * 2 * 2 + 4 * min(nb, 512)
    return score, gqa


def run_ours(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist

    import block_sparse_attention_c4_b200 as Q
    import block_sparse_attention_c4_b200.workload as W
    import qsa_gen as G
    from block_sparse_attention_c4_b200 import build

    build.build()
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    if world > 1:
        dist.init_process_group("nccl", device_id=dev, timeout=__import__("datetime").timedelta(seconds=300))

    wl = G.decode_128k(seed=replica_seed(rank), batch=args.batch)
    lens = [int(x) for x in wl.lens]
    t0 = time.time()
    cache = W.build_cache(wl, device=dev)
    inp = W.decode_inputs(wl, device=dev)
    torch.cuda.synchronize()
    setup_s = time.time() - t0
    B, max_len = wl.batch, max(lens)
    ws = Q.Workspace(Q.workspace_bytes(Q.OP_DECODE, B, max_len), device=dev)
    out = torch.empty(B, 16, 128, dtype=torch.bfloat16, device=dev)
    flush = torch.empty(512 << 20, dtype=torch.uint8, device=dev)
    nk = Q.decode_kernel_count(args.batch)
    knames = (["prologue"] if nk == 3 else []) + ["score_topk", "sparse_gqa"]

    def step():
        Q.decode(cache, inp["idx_k_new"], inp["idx_q"], inp["w"], inp["q"], inp["seq_len"], max_len, ws, out=out)

    for _ in range(max(args.warmup, 3)):
        step()
    torch.cuda.synchronize()
    if ws.device_error() != 0:
        raise RuntimeError("device error word set during warm-up")

    K = args.steps
    st = torch.cuda.current_stream()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    sampler = ClockSampler(local_rank)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    sampler.start()
    time.sleep(0.15)
    wall0 = time.perf_counter()
    for k in range(K):
        flush.zero_()
        ev[k][0].record(st)
        step()
        ev[k][1].record(st)
    torch.cuda.synchronize()
    wall = time.perf_counter() - wall0
    if world > 1:
        dist.barrier()
    clocks = sampler.stop()
    step_ms = [ev[k][0].elapsed_time(ev[k][1]) for k in range(K)]
    mean_ms = float(np.mean(step_ms))

    # Per-kernel breakdown, measured on separate steps: events recorded between the kernels cost a
    # few microseconds per step, so the timed steps above carry none.
    Kb = max(10, min(K, 200))
    evb = [[torch.cuda.Event(enable_timing=True) for _ in range(2 * nk)] for _ in range(Kb)]
    for e in evb:
        for x in e:
            x.record(st)  # materialise the events before handing them to the library
    torch.cuda.synchronize()
    for k in range(Kb):
        flush.zero_()
        Q.set_profile_events(evb[k])
        step()
    Q.set_profile_events(None)
    torch.cuda.synchronize()
    kern_ms = [[evb[k][2 * i].elapsed_time(evb[k][2 * i + 1]) for k in range(Kb)] for i in range(nk)]

    # ---- end to end through the host-buffer API ----
    sess = Q.DecodeSession(cache, max_len, device=dev)
    host_in = Q.DecodeSession.pinned_inputs(inp)
    for _ in range(3):
        sess.step(host_in)
    torch.cuda.synchronize()
    K2 = max(10, min(K, 500))
    e2 = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K2)]
    for k in range(K2):
        flush.zero_()
        e2[k][0].record(st)
        sess.step(host_in)
        e2[k][1].record(st)
    torch.cuda.synchronize()
    e2e_ms = float(np.mean([a.elapsed_time(b) for a, b in e2]))
    # the device-timed and host-fed results agree bit for bit
    if not torch.equal(sess.host_out.view(torch.int16), out.cpu().view(torch.int16)):
        raise RuntimeError("host-fed decode differs from the device-fed one")

    mean_ms_max, e2e_ms_max = max_over_ranks([mean_ms, e2e_ms], world, dev)

    score_b, gqa_b = algorithmic_bytes(lens)
    hbm_peak, peak_kind = measured_peaks()
    score_ms = float(np.mean(kern_ms[knames.index("score_topk")]))
    src_hash = kernel_src_hash(SCORER_SRC)
    traffic, traffic_src = committed_traffic(src_hash)
    res = None
    if rank == 0:
        achieved = score_b / (score_ms * 1e-3) / 1e9
        total_b = score_b + gqa_b
        res = {
            "metric": METRIC,
            "value": round(job_throughput(B, world, mean_ms_max), 1),
            "unit": UNIT,
            "n_gpus": world,
            "steps": K,
            "warmup": max(args.warmup, 3),
            "ms_per_step": round(mean_ms_max, 5),
            "higher_is_better": True,
            "scaling": "weak",
            "vs_baseline": None,
            "dtype": "bf16",
            "data": "synthetic (qsa_gen seeded generator; N(0,1) bf16 K/V, q, index keys with 5% planted blocks)",
            "config": {
                "workload": f"decode_b{B}_ctx120000-131072",
                "batch_per_gpu": B,
                "global_batch": B * world,
                "ctx_min": min(lens), "ctx_max": max(lens), "ctx_mean": round(float(np.mean(lens)), 1),
                "heads": "16q/2kv d128, indexer 4x128, top-512 of c4 blocks",
                "page_size": 64,
                "l2": "inputs 5x larger than L2 per step, plus a 512 MiB flush between timed steps (untimed)",
                "parallelism": f"replicas x{world} (requests sharded, no exchange)",
            },
            "gpu_launches": K * nk,
            "kernels_ms_mean": {n: round(float(np.mean(v)), 5) for n, v in zip(knames, kern_ms)},
            "kernels_note": f"CUDA events around each kernel, {Kb} separate steps (not the timed ones)",
            "step_bytes_algorithmic": int(total_b),
            "step_hbm_gbs": round(total_b / (mean_ms * 1e-3) / 1e9, 1),
            "step_frac_of_hbm": round(total_b / (mean_ms * 1e-3) / 1e9 / hbm_peak, 4),
            "roofline": {
                "kernel": "k_score_topk",
                "bound": "hbm",
                "achieved": round(achieved, 1),
                "peak": hbm_peak,
                "peak_source": f"{peak_kind} (MEASURED_PEAKS.json hbm_gbs)" if peak_kind == "measured" else
                "fallback 6.65 TB/s",
                "unit": "GB/s",
                "frac": round(achieved / hbm_peak, 4),
                "traffic": None if traffic is None else int(traffic),
                "traffic_source": traffic_src,
                "algorithmic_bytes_per_launch": int(score_b),
                "kernel_src_sha256_16": src_hash,
            },
            "e2e": {"value": round(job_throughput(B, world, e2e_ms_max), 1), "unit": UNIT,
                    "h2d_bytes_per_step": sess.h2d_bytes(), "d2h_bytes_per_step": sess.d2h_bytes()},
            "clocks": clocks,
            "wall_s_timed_region": round(wall, 3),
            "setup_s": round(setup_s, 1),
        }
    # free device memory before the secondary measurements and the CPU baseline
    del ws, sess
    if rank == 0 and not args.no_extras:
        res["extras"] = {}
        extra(res["extras"], "index_projection_two_stream", run_projection_decode, cache, inp, wl, dev, flush)
        extra(res["extras"], "fp8_kv_decode", run_fp8_decode, cache, inp, wl, dev, flush, score_b, gqa_b)
        extra(res["extras"], "varlen_prefill", run_varlen_prefill, cache, wl, dev, flush)
    del cache, flush
    torch.cuda.empty_cache()
    if rank == 0 and not args.no_prefill:
        res["prefill_scorer"] = run_prefill_scorer(dev)
        torch.cuda.empty_cache()
    if rank == 0 and not args.no_extras:
        extra(res["extras"], "split_context_decode_262k", run_split_decode, dev)
        torch.cuda.empty_cache()
    if world > 1:
        dist.destroy_process_group()
    return res, wl


def extra(out: dict, name: str, fn, *args):
    """A secondary measurement: its result under `name`, or the error it raised (the headline number
    above does not depend on it)."""
    import torch

    try:
        out[name] = fn(*args)
    except Exception as e:  # reported in the JSON line, not hidden
        out[name] = {"error": f"{type(e).__name__}: {e}"[:500]}
    torch.cuda.synchronize()


def time_calls(fn, reps: int, flush=None):
    """Mean CUDA-event time (ms) of `fn` on the current stream over `reps` calls (L2 flushed before each
    when `flush` is given, outside the events).  Without a flush the stream is first held by a device-side
    sleep long enough for the host to enqueue every call, so that the events time the GPU's work and not
    the host's launch cost of short calls."""
    import torch

    st = torch.cuda.current_stream()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps)]
    if flush is None:
        torch.cuda._sleep(min(200_000_000, 200_000 * reps))  # ~0.1 ms of host time per call at ~2 GHz
    for k in range(reps):
        if flush is not None:
            flush.zero_()
        ev[k][0].record(st)
        fn()
        ev[k][1].record(st)
    torch.cuda.synchronize()
    return float(np.mean([a.elapsed_time(b) for a, b in ev]))


def run_projection_decode(cache, inp, wl, dev, flush, hidden: int = 4096, reps: int = 200):
    """The decode step from hidden states: qsa_decode_indexer (index projection, append, scoring,
    top-512) and qsa_decode_attend, on one stream; and with the indexer on a second stream while the
    main stream runs a stand-in for the caller's Q/K/V projection (a bf16 GEMM [B, hidden] x
    [hidden, (16 + 2 + 2) x 128]), joined by an event before the attention."""
    import torch

    import block_sparse_attention_c4_b200 as Q
    import block_sparse_attention_c4_b200.workload as W
    import qsa_gen as G

    B, max_len = wl.batch, int(max(wl.lens))
    x = W.bits_to_bf16(np.stack([wl.hidden(r, hidden)[0] for r in range(B)]), dev)
    wp = W.bits_to_bf16(G.projection_weights(wl.seed, hidden), dev)
    w_qkv = torch.randn(hidden, 20 * 128, device=dev, dtype=torch.bfloat16) * hidden ** -0.5
    ws_i = Q.Workspace(Q.workspace_bytes(Q.OP_DECODE_INDEXER, B, max_len), device=dev)
    ws_a = Q.Workspace(Q.workspace_bytes(Q.OP_DECODE_ATTEND, B, max_len), device=dev)
    blocks = torch.empty(B, 512, dtype=torch.int32, device=dev)
    nblocks = torch.empty(B, dtype=torch.int32, device=dev)
    out = torch.empty(B, 16, 128, dtype=torch.bfloat16, device=dev)
    main, side = torch.cuda.current_stream(), torch.cuda.Stream(device=dev)
    done = torch.cuda.Event()

    def one_stream():
        Q.decode_indexer(cache, x, wp, inp["seq_len"], max_len, ws_i, blocks, nblocks)
        Q.decode_attend(cache, inp["q"], inp["seq_len"], max_len, blocks, nblocks, ws_a, out=out)

    def proj_only():
        Q.index_project(x, wp)

    def qkv():
        return x @ w_qkv

    def serial():
        qkv()
        one_stream()

    def overlapped():
        side.wait_stream(main)
        with torch.cuda.stream(side):
            Q.decode_indexer(cache, x, wp, inp["seq_len"], max_len, ws_i, blocks, nblocks, stream=side)
        done.record(side)
        qkv()
        main.wait_event(done)
        Q.decode_attend(cache, inp["q"], inp["seq_len"], max_len, blocks, nblocks, ws_a, out=out)

    for f in (one_stream, proj_only, qkv, serial, overlapped):
        for _ in range(3):
            f()
    torch.cuda.synchronize()
    if ws_i.device_error() != 0 or ws_a.device_error() != 0:
        raise RuntimeError("device error word set in the two-phase decode")
    t = {name: time_calls(f, reps, flush) for name, f in
         (("indexer_plus_attend_us", one_stream), ("projection_alone_us", proj_only), ("qkv_gemm_alone_us", qkv),
          ("qkv_then_decode_us", serial), ("decode_overlapping_qkv_us", overlapped))}
    wbytes = (4 * 128 + 128 + 4) * hidden * 2
    res = {k: round(v * 1e3, 2) for k, v in t.items()}
    res.update({"hidden": hidden, "batch": B, "projection_weight_bytes": wbytes,
                "projection_hbm_gbs": round((wbytes + B * hidden * 2) / (t["projection_alone_us"] * 1e-3) / 1e9, 1),
                "note": "indexer on a second stream while the main stream runs the caller's Q/K/V projection "
                        "stand-in (torch matmul, not part of this library); joined by an event"})
    return res


def run_fp8_decode(cache, inp, wl, dev, flush, score_b, gqa_b, reps: int = 400):
    """qsa_decode_fp8 on the headline workload: the same cache with its K/V as E4M3 codes (the bf16 pool
    divided by the scale and converted on the device), the same index cache."""
    import torch

    import block_sparse_attention_c4_b200 as Q

    B, max_len = wl.batch, int(max(wl.lens))
    scale = 0.25
    c8 = Q.LayerCache(cache.num_slots, B, cache.max_pages, rope_theta=cache.rope_theta, device=dev,
                      page_table=cache.page_table, kv_dtype="fp8")
    c8.cidx, c8.ring = cache.cidx, cache.ring
    step = 1 << 20
    for s0 in range(0, cache.num_slots, step):
        src = cache.kv[s0:s0 + step].float() / scale
        c8.kv[s0:s0 + step].copy_(src.to(torch.float8_e4m3fn).view(torch.uint8))
    ws = Q.Workspace(Q.workspace_bytes(Q.OP_DECODE, B, max_len), device=dev)
    out = torch.empty(B, 16, 128, dtype=torch.bfloat16, device=dev)

    def step_fn():
        Q.decode_fp8(c8, inp["idx_k_new"], inp["idx_q"], inp["w"], inp["q"], inp["seq_len"], max_len, ws, scale,
                     scale, out=out)

    for _ in range(5):
        step_fn()
    torch.cuda.synchronize()
    if ws.device_error() != 0:
        raise RuntimeError("device error word set in the FP8 decode")
    ms = time_calls(step_fn, reps, flush)
    total = score_b + gqa_b // 2  # K/V rows halve: 512 B per position
    hbm, _ = measured_peaks()
    del c8
    return {"ms_per_step": round(ms, 5), "query_tok_per_s": round(B / (ms * 1e-3), 1),
            "step_bytes_algorithmic": int(total), "step_hbm_gbs": round(total / (ms * 1e-3) / 1e9, 1),
            "step_frac_of_hbm": round(total / (ms * 1e-3) / 1e9 / hbm, 4),
            "note": "E4M3 K/V with one scale each for K and V; index path unchanged (bf16 compressed keys)"}


def run_varlen_prefill(cache, wl, dev, flush, reps: int = 20):
    """qsa_prefill_score_topk_varlen: one call over a ragged batch of causal chunks of four requests at
    different depths (8192 queries in all), against one qsa_prefill_score_topk call per chunk."""
    import torch

    import block_sparse_attention_c4_b200 as Q
    import block_sparse_attention_c4_b200.workload as W

    segs = [(0, 0, 4096), (1, 60000, 2048), (2, 110000, 1024), (3, 8000, 1024)]
    idx_q = W.bits_to_bf16(np.concatenate([wl.idx_q(r, q0=p0, n=T) for r, p0, T in segs]), dev)
    w = torch.from_numpy(np.concatenate([wl.w(r, q0=p0, n=T) for r, p0, T in segs])).to(dev)
    cu = np.concatenate([[0], np.cumsum([T for _, _, T in segs])]).astype(np.int32)
    Tall, max_len = int(cu[-1]), max(p0 + T for _, p0, T in segs)
    ws = Q.Workspace(Q.workspace_bytes(Q.OP_PREFILL_SCORE_TOPK, Tall, max_len), device=dev)
    blocks = torch.empty(Tall, 512, dtype=torch.int32, device=dev)
    nblocks = torch.empty(Tall, dtype=torch.int32, device=dev)
    ws1 = Q.Workspace(Q.workspace_bytes(Q.OP_PREFILL_SCORE_TOPK, 4096, max_len), device=dev)

    def varlen():
        Q.prefill_score_topk_varlen(cache, idx_q, w, [s[0] for s in segs], [s[1] for s in segs], cu, max_len, ws,
                                    blocks, nblocks)

    def separate():
        for i, (r, p0, T) in enumerate(segs):
            Q.prefill_score_topk(cache, idx_q[cu[i]:cu[i + 1]], w[cu[i]:cu[i + 1]], r, p0, ws1,
                                 blocks[cu[i]:cu[i + 1]], nblocks[cu[i]:cu[i + 1]])

    for f in (varlen, separate):
        for _ in range(3):
            f()
    torch.cuda.synchronize()
    if ws.device_error() != 0 or ws1.device_error() != 0:
        raise RuntimeError("device error word set in the varlen prefill")
    t_v, t_s = time_calls(varlen, reps, flush), time_calls(separate, reps, flush)
    flops = sum(prefill_flops(p0, T) for _, p0, T in segs)
    peak, _ = bf16_peak()
    return {"segments": [{"req": r, "pos0": p0, "queries": T} for r, p0, T in segs],
            "call_us": round(t_v * 1e3, 2), "one_call_per_chunk_us": round(t_s * 1e3, 2),
            "query_tok_per_s": round(Tall / (t_v * 1e-3), 1),
            "tflops": round(flops / (t_v * 1e-3) / 1e12, 1), "frac_of_bf16_peak": round(flops / (t_v * 1e-3) / 1e12 / peak, 4)}


def run_split_decode(dev, reps: int = 50):
    """Split-context decode of the 262,147-token request over 2 and 4 ranks, run as virtual ranks one after
    another on this GPU (exchanges by stacking): each rank's compute time (scoring its pages, the merge, its
    attention, the combine) and the bytes each exchange moves, next to qsa_decode of the whole context on one
    GPU.  No NVLink is involved here: the exchange time is not measured."""
    import torch

    import block_sparse_attention_c4_b200 as Q
    import block_sparse_attention_c4_b200.workload as W
    from block_sparse_attention_c4_b200 import split as SP
    import qsa_gen as G

    wl = G.long_262k()
    L = 262144
    t = L - 1
    raw = wl.idx_keys(0, 0, L)
    full = W.build_cache(wl, device=dev, prefix_tokens=[L - 1])
    knew = W.bits_to_bf16(raw[t:t + 1], dev)
    idx_q = W.bits_to_bf16(wl.idx_q(0, q0=t, n=1), dev)
    w = torch.from_numpy(wl.w(0, q0=t, n=1)).to(dev)
    q = W.bits_to_bf16(wl.q(0, q0=t, n=1), dev)
    seq_len = torch.tensor([L], dtype=torch.int32, device=dev)
    ws = Q.Workspace(Q.workspace_bytes(Q.OP_DECODE, 1, L), device=dev)
    single = time_calls(lambda: Q.decode(full, knew, idx_q, w, q, seq_len, L, ws), reps)
    res = {"context": L, "single_gpu_decode_us": round(single * 1e3, 2)}
    n_pages = (L + 63) // 64
    for world in (2, 4):
        lo, cnt = SP.partition_pages(n_pages, world)
        ranks = []
        for r in range(world):
            pt = torch.full((1, full.max_pages), -1, dtype=torch.int32, device=dev)
            pt[0, lo[r]:lo[r] + cnt[r]] = full.page_table[0, lo[r]:lo[r] + cnt[r]]
            # a view of the one pool whose page table maps only this rank's pages (no copy)
            view = Q.LayerCache(full.num_slots, 1, full.max_pages, rope_theta=full.rope_theta, device="meta",
                                page_table=pt)
            view.kv, view.k, view.v, view.cidx, view.ring = full.kv, full.k, full.v, full.cidx, full.ring
            view.kv_stride = full.kv_stride
            ranks.append(SP.SplitRank(view, [lo[r]], [cnt[r]], L, device=dev))
        cands = [rk.score(idx_q, w, seq_len) for rk in ranks]
        stack = [torch.stack([c[i] for c in cands]) for i in range(3)]
        blocks, nblocks = SP.merge(*stack)
        parts = [rk.attend(q, seq_len, blocks, nblocks) for rk in ranks]
        outs, lses = torch.stack([p[0] for p in parts]), torch.stack([p[1] for p in parts])
        torch.cuda.synchronize()
        per_rank, parts_us = [], []
        for rk in ranks:
            parts = [time_calls(lambda: rk.score(idx_q, w, seq_len), reps),
                     time_calls(lambda: SP.merge(*stack), reps),
                     time_calls(lambda: rk.attend(q, seq_len, blocks, nblocks), reps),
                     time_calls(lambda: SP.combine(outs, lses), reps)]
            per_rank.append(sum(parts))
            parts_us.append([round(x * 1e3, 2) for x in parts])
        res[f"world{world}"] = {"per_rank_compute_us_max": round(max(per_rank) * 1e3, 2),
                                "per_rank_compute_us": [round(x * 1e3, 2) for x in per_rank],
                                "rank0_score_merge_attend_combine_us": parts_us[0],
                                "exchange_bytes_per_rank": {"candidates": 512 * 8 + 4, "attention": 16 * 128 * 2 + 16 * 4}}
    res["note"] = ("virtual ranks on one GPU sharing one pool (each rank's page table maps only its pages); "
                   "per-rank time = its kernels timed separately; the two all-gathers are not timed")
    return res


def prefill_flops(pos0: int, T: int) -> int:
    """Algorithmic FLOPs of scoring a causal chunk: 4 heads x 128 dims x 2 per visible (query, block) pair."""
    t = np.arange(pos0, pos0 + T, dtype=np.int64)
    return int(((t + 1) // 4).sum()) * 4 * 128 * 2


def bf16_peak():
    pk = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(pk):
        return float(json.load(open(pk))["bf16_tflops"]), "measured burst bf16 (MEASURED_PEAKS.json bf16_tflops)"
    return 1590.0, "fallback 1.59 PFLOP/s"


def run_prefill_scorer(dev, reps: int = 20, long_context: bool = True):
    """Time qsa_prefill_score_topk (rotation, tensor-core scoring with candidate filtering, exact
    top-512) on the 32768-token causal chunk, every token a query, and on the 262144-token prefill
    of the long-context workload in its 32 causal chunks of 8192 queries."""
    import torch

    import block_sparse_attention_c4_b200 as Q
    import block_sparse_attention_c4_b200.workload as W
    import qsa_gen as G

    peak, src = bf16_peak()
    wl = G.prefill_32k()
    T = 32768
    cache = W.build_cache(wl, device=dev, prefix_tokens=[T])
    idx_q = W.bits_to_bf16(wl.idx_q(0, 0, T), dev)
    w = torch.from_numpy(wl.w(0, 0, T)).to(dev)
    ws = Q.Workspace(Q.workspace_bytes(Q.OP_PREFILL_SCORE_TOPK, T, T), device=dev)
    blocks = torch.empty(T, 512, dtype=torch.int32, device=dev)
    nblocks = torch.empty(T, dtype=torch.int32, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    for _ in range(3):
        Q.prefill_score_topk(cache, idx_q, w, 0, 0, ws, blocks, nblocks)
    torch.cuda.synchronize()
    if ws.device_error() != 0:
        raise RuntimeError("device error word set in the prefill scorer")
    rescored = Q.prefill_rescored_rows(ws, T, T)
    st = torch.cuda.current_stream()
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(6)] for _ in range(reps)]
    for e in ev:
        for x in e:
            x.record(st)
    torch.cuda.synchronize()
    for k in range(reps):
        flush.zero_()
        Q.set_profile_events(ev[k])
        Q.prefill_score_topk(cache, idx_q, w, 0, 0, ws, blocks, nblocks)
    Q.set_profile_events(None)
    torch.cuda.synchronize()
    ms = [[ev[k][2 * i].elapsed_time(ev[k][2 * i + 1]) for k in range(reps)] for i in range(3)]
    total = [ev[k][0].elapsed_time(ev[k][5]) for k in range(reps)]
    # the call without events between its kernels
    evc = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps)]
    for k in range(reps):
        flush.zero_()
        evc[k][0].record(st)
        Q.prefill_score_topk(cache, idx_q, w, 0, 0, ws, blocks, nblocks)
        evc[k][1].record(st)
    torch.cuda.synchronize()
    call_ms = float(np.mean([a.elapsed_time(b) for a, b in evc]))
    flops = prefill_flops(0, T)
    score_s = float(np.mean(ms[1])) * 1e-3
    call_ach = flops / (call_ms * 1e-3) / 1e12
    mma_ach = flops / score_s / 1e12
    res = {
        "workload": "prefill_L32768 (one causal chunk of 32768 queries)",
        "call_us": round(call_ms * 1e3, 2),
        "kernels_us": {"rotate": round(float(np.mean(ms[0])) * 1e3, 2), "score_tcgen05": round(score_s * 1e6, 2),
                       "select_and_rescore": round(float(np.mean(ms[2])) * 1e3, 2),
                       "sum_with_events": round(float(np.mean(total)) * 1e3, 2)},
        "rows_rescored_in_full": rescored,
        "query_tok_per_s": round(T / (call_ms * 1e-3), 1),
        "roofline": {"kernel": "qsa_prefill_score_topk (whole call)", "bound": "tensor", "achieved": round(call_ach, 1),
                     "peak": peak, "peak_source": src, "unit": "TFLOP/s", "frac": round(call_ach / peak, 4),
                     "algorithmic_flops_per_launch": flops},
        "roofline_mma_kernel": {"kernel": "k_prefill_score", "bound": "tensor", "achieved": round(mma_ach, 1),
                                "peak": peak, "unit": "TFLOP/s", "frac": round(mma_ach / peak, 4),
                                "note": "work tiles whose queries see more than 8192 blocks also score a 1/8 sample first (MMA not in "
                                        "the algorithmic FLOPs); at L = 32768 every tile writes all its keys"},
    }
    del cache, ws, blocks, nblocks, idx_q, w
    torch.cuda.empty_cache()
    if long_context:
        res["long_context_prefill"] = run_long_prefill(dev, flush)
    return res


def run_prefill_chunk(dev, pos0: int, chunk: int = 8192, L: int = 262144, reps: int = 3):
    """One causal chunk of the long-context prefill (the cache holds every index key), called `reps` times."""
    import torch

    import block_sparse_attention_c4_b200 as Q
    import block_sparse_attention_c4_b200.workload as W
    import qsa_gen as G

    wl = G.long_262k()
    cache = W.build_cache(wl, device=dev, prefix_tokens=[0])
    W.append_tokens(cache, wl, 0, 0, L)
    ws = Q.Workspace(Q.workspace_bytes(Q.OP_PREFILL_SCORE_TOPK, chunk, pos0 + chunk), device=dev)
    idx_q = W.bits_to_bf16(wl.idx_q(0, pos0, chunk), dev)
    w = torch.from_numpy(wl.w(0, pos0, chunk)).to(dev)
    torch.cuda.synchronize()
    ms = time_calls(lambda: Q.prefill_score_topk(cache, idx_q, w, 0, pos0, ws), reps)
    if ws.device_error() != 0:
        raise RuntimeError("device error word set in the prefill chunk")
    return {"pos0": pos0, "queries": chunk, "call_ms_mean": round(ms, 4),
            "rows_rescored_in_full": Q.prefill_rescored_rows(ws, chunk, pos0 + chunk)}


def run_long_prefill(dev, flush, chunk: int = 8192, L: int = 262144):
    """The 262144-token prefill in causal chunks of 8192 queries: every chunk's qsa_prefill_score_topk
    timed by CUDA events (the cache holds the index keys of all 262144 tokens; a chunk's queries only
    see the blocks before them)."""
    import torch

    import block_sparse_attention_c4_b200 as Q
    import block_sparse_attention_c4_b200.workload as W
    import qsa_gen as G

    peak, src = bf16_peak()
    wl = G.long_262k()
    cache = W.build_cache(wl, device=dev, prefix_tokens=[0])
    for t0 in range(0, L, chunk):
        W.append_tokens(cache, wl, 0, t0, chunk)
    ws = Q.Workspace(Q.workspace_bytes(Q.OP_PREFILL_SCORE_TOPK, chunk, L), device=dev)
    blocks = torch.empty(chunk, 512, dtype=torch.int32, device=dev)
    nblocks = torch.empty(chunk, dtype=torch.int32, device=dev)
    st = torch.cuda.current_stream()
    chunks = []
    for pos0 in range(0, L, chunk):
        idx_q = W.bits_to_bf16(wl.idx_q(0, pos0, chunk), dev)
        w = torch.from_numpy(wl.w(0, pos0, chunk)).to(dev)
        chunks.append((pos0, idx_q, w))
    for pos0, idx_q, w in chunks[-2:]:  # warm-up
        Q.prefill_score_topk(cache, idx_q, w, 0, pos0, ws, blocks, nblocks)
    torch.cuda.synchronize()
    if ws.device_error() != 0:
        raise RuntimeError("device error word set in the long-context prefill")
    times, rescored, split = [], 0, np.zeros(3)
    for pos0, idx_q, w in chunks:
        flush.zero_()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(st)
        Q.prefill_score_topk(cache, idx_q, w, 0, pos0, ws, blocks, nblocks)
        b.record(st)
        torch.cuda.synchronize()
        times.append(a.elapsed_time(b))
        rescored += Q.prefill_rescored_rows(ws, chunk, pos0 + chunk)
    for pos0, idx_q, w in chunks:  # the kernel split, on separate calls (events between the kernels)
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(6)]
        for x in ev:
            x.record(st)
        flush.zero_()
        Q.set_profile_events(ev)
        Q.prefill_score_topk(cache, idx_q, w, 0, pos0, ws, blocks, nblocks)
        Q.set_profile_events(None)
        torch.cuda.synchronize()
        split += [ev[2 * i].elapsed_time(ev[2 * i + 1]) for i in range(3)]
    if ws.device_error() != 0:
        raise RuntimeError("device error word set in the long-context prefill")
    flops = sum(prefill_flops(pos0, chunk) for pos0, _, _ in chunks)
    total_ms = float(np.sum(times))
    ach = flops / (total_ms * 1e-3) / 1e12
    return {
        "workload": f"prefill_L{L} in {len(chunks)} causal chunks of {chunk} queries",
        "total_ms": round(total_ms, 3),
        "chunk_ms_first_last": [round(times[0], 3), round(times[-1], 3)],
        "kernels_ms_total": {"rotate": round(float(split[0]), 3), "score_tcgen05": round(float(split[1]), 3),
                             "select_and_rescore": round(float(split[2]), 3)},
        "rows_rescored_in_full": rescored,
        "query_tok_per_s": round(L / (total_ms * 1e-3), 1),
        "roofline": {"kernel": "qsa_prefill_score_topk (whole calls)", "bound": "tensor", "achieved": round(ach, 1),
                     "peak": peak, "peak_source": src, "unit": "TFLOP/s", "frac": round(ach / peak, 4),
                     "algorithmic_flops": flops},
    }


def oracle_sample_step(wl, reqs, nthreads):
    """Prepare oracle state for requests `reqs` of a decode workload; return a callable running one
    decode step of those requests on the CPU oracle, plus its input size."""
    import oracle as O

    st = {"L": [], "ring": [], "comp": [], "knew": [], "iq": [], "w": [], "q": [], "K": [], "V": []}
    for r in reqs:
        L = int(wl.lens[r])
        raw = wl.idx_keys(r, 0, L)
        nb0 = (L - 1) // 4
        comp = np.zeros((max(L // 4, 1), 128), dtype=np.uint16)
        comp[:nb0] = O.compress(raw[:4 * nb0], nthreads=nthreads)
        ring = np.zeros((4, 128), dtype=np.uint16)
        for p in range(4 * nb0, L - 1):
            ring[p % 4] = raw[p]
        st["L"].append(L)
        st["ring"].append(ring)
        st["comp"].append(comp)
        st["knew"].append(np.ascontiguousarray(raw[L - 1]))
        st["iq"].append(wl.idx_q(r)[0])
        st["w"].append(wl.w(r)[0])
        st["q"].append(wl.q(r)[0])
        st["K"].append(wl.k(r, 0, L))
        st["V"].append(wl.v(r, 0, L))

    def run():
        O.decode_batch(st["L"], st["ring"], st["comp"], st["knew"], st["iq"], st["w"], st["q"], st["K"], st["V"],
                       theta=wl.rope_theta, nthreads=nthreads)

    return run


def cpu_threads():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def cpu_baseline(wl, seconds: float):
    nthreads = cpu_threads()
    n = min(wl.batch, max(nthreads, 8), 32)
    reqs = list(range(n))
    run = oracle_sample_step(wl, reqs, nthreads)
    t0 = time.perf_counter()
    run()
    one = time.perf_counter() - t0
    reps = max(1, int(seconds / max(one, 1e-3)))
    t0 = time.perf_counter()
    for _ in range(reps):
        run()
    dt = time.perf_counter() - t0
    return {"value": round(n * reps / dt, 2), "unit": UNIT, "cores": min(nthreads, n), "kind": "oracle",
            "sample": f"decode steps of {n} of the {wl.batch} requests (contexts {min(wl.lens[:n])}-"
                      f"{max(wl.lens[:n])}), {reps} repetitions after one warm-up, FP64 C++ oracle, "
                      f"one std::thread per request"}


def run_reference(args, rank, world):
    """The reference arm: the CPU oracle timed on the host cores (rank 0 only)."""
    if rank != 0:
        return None
    import qsa_gen as G

    wl = G.decode_128k(seed=2, batch=args.batch)
    nthreads = cpu_threads()
    n = min(wl.batch, nthreads, 32)
    run = oracle_sample_step(wl, list(range(n)), nthreads)
    for _ in range(max(args.warmup, 3)):
        run()
    # bound the run: at most ~120 s of timed work whatever --steps says
    t0 = time.perf_counter()
    run()
    one = time.perf_counter() - t0
    K = max(1, min(args.steps, int(120.0 / max(one, 1e-3))))
    t0 = time.perf_counter()
    for _ in range(K):
        run()
    dt = time.perf_counter() - t0
    value = round(n * K / dt, 2)
    return {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K, "warmup": max(args.warmup, 3),
        "ms_per_step": round(dt / K * 1e3, 3), "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f64", "data": "synthetic (qsa_gen)", "impl": "reference",
        "config": {"workload": f"decode_b{wl.batch}_ctx120000-131072", "sample_requests_per_step": n},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": min(nthreads, n), "kind": "oracle",
                         "sample": f"each step: decode of {n} of the {wl.batch} requests on the FP64 C++ oracle"
                                   f" ({K} steps; --steps {args.steps} bounded to ~120 s)"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main():
    args = parse()
    rank, world, local_rank = dist_env()
    if args.impl == "reference":
        res = run_reference(args, rank, world)
        if res is not None:
            print(json.dumps(res), flush=True)
        return
    if args.prefill_chunk >= 0:
        import torch

        from block_sparse_attention_c4_b200 import build

        build.build()
        torch.cuda.set_device(local_rank)
        if rank == 0:
            print(json.dumps({"prefill_chunk": run_prefill_chunk(torch.device("cuda", local_rank),
                                                                 args.prefill_chunk)}), flush=True)
        return
    if args.only_prefill:
        import torch

        from block_sparse_attention_c4_b200 import build

        build.build()
        torch.cuda.set_device(local_rank)
        if rank == 0:
            print(json.dumps({"prefill_scorer": run_prefill_scorer(torch.device("cuda", local_rank),
                                                                   long_context=not args.no_long_prefill)}),
                  flush=True)
        return
    res, wl = run_ours(args, rank, world, local_rank)
    if rank == 0:
        if world == 1 and not args.no_cpu_baseline:
            res["cpu_baseline"] = cpu_baseline(wl, args.cpu_seconds)
        print(json.dumps(res), flush=True)


if __name__ == "__main__":
    main()
