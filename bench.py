"""Benchmark of the TurboQuant hot path on B200 (one JSON line on rank 0).

Workload (default ``llama8b``): one Llama-3-8B-shaped layer, 8 KV / 32 query
heads, d = 128, 32768 cached tokens, batch 1, 3-bit K and V (no QJL).  The
prefill is quantized once into R cache replicas; a *step* is one decode step
of the whole hot path: quantize-on-append of one new token (8 KV heads, K and
V) followed by decode attention of the 32 query heads over the packed cache.
Step i uses replica i % R, so consecutive steps read disjoint memory and the
step-to-step working set (R x 26 MB) exceeds the 126 MB L2.

``value``  decode-attention effective GB/s: packed K/V bytes the step reads
           (codes + fp16 norms) / device time per step (CUDA graph of the K
           timed steps, CUDA events, max over ranks).
``e2e``    the same metric when every step goes through the C ABI eagerly
           with pinned host buffers: H2D of the token's K/V and of q, the two
           calls, D2H of the output.
``roofline`` the decode calls of the timed steps alone (same replicas and
           lengths) as one CUDA graph, events around its replay; algorithmic
           bytes = packed bytes per call.
``quantize_*`` prefill quantize of 32768 tokens (input 128 MB > L2): tokens/s,
           GB/s (bf16 read + packed write) and roofline fraction.
``cpu_baseline`` the CPU oracle on a bounded sample of the same decode step.

``--impl reference`` times the CPU oracle on the host instead (the reference
arm: the method has no other implementation to run).  Multi-GPU: one process
per GPU under torchrun; every rank runs its own replica of the workload
(the path has no cross-GPU exchange), ``value`` sums the ranks' bytes over
the slowest rank's time.
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

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "decode-attn over packed KV: effective GB/s (% HBM peak); quantize tokens/s"
WORKLOAD_DESCS = {
    "llama8b": ("llama8b: Llama-3-8B-shaped single layer, 8 KV / 32 query heads (GQA 4), d=128, "
                "32768 cached tokens, batch 1, bf16 K/V ~ N(0,I) x LogNormal(0,0.5) per (token, head), "
                "3-bit K and V (turbo3, no QJL); step = append-quantize 1 token + decode attention"),
    "llama70b": ("llama70b: 70B-shaped long context, 8 KV / 64 query heads (GQA 8), d=128, 131072 cached "
                 "tokens, batch 4, bf16 K/V ~ N(0,1) with 10 (head, channel) outliers x20, 3-bit K and V; "
                 "step = append-quantize 1 token per sequence + batched decode attention"),
    "tiny": ("tiny: 1 KV head, 1 query head, d=128, 1024 cached tokens, K, V, q iid N(0,1) (bf16 at the "
             "boundary), 3-bit K and V; step = append-quantize 1 token + decode attention"),
    "qwen": ("qwen: Qwen-like anisotropic norms, 4 KV / 28 query heads (GQA 7), d=128, 16384 cached tokens, "
             "K norms U[172,778], V norms U[2,4], directions uniform on the sphere, q on the unit sphere; "
             "step = append-quantize 1 token + decode attention"),
    "serving": ("serving: 32 sequences, lengths uniform on [1024, 65536] (seeded), 8 KV / 32 query heads, "
                "d=128, bf16 N(0,1); step = append-quantize 1 token per sequence + ragged batched decode"),
}
WORKLOAD_DESC = WORKLOAD_DESCS["llama8b"]


# DRAM bytes per attention-kernel launch (dram__bytes_read.sum +
# dram__bytes_write.sum) from one ncu capture of the default command, keyed by
# (workload, bits_k, bits_v, qjl); null elsewhere.  Re-captured whenever the
# kernel changes.
MEASURED_TRAFFIC = {("llama8b", 3, 3, False): 26352640.0}


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def max_over_ranks(values, device=None):
    """Each timing's maximum over the ranks (the slowest rank bounds the job)."""
    if not (torch.distributed.is_available() and torch.distributed.is_initialized()):
        return list(values)
    t = torch.tensor(values, dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return t.tolist()


def job_gbps(n_ranks: int, bytes_per_rank: float, ms: float) -> float:
    """Whole-job throughput: every rank's replica moves bytes_per_rank in the
    slowest rank's time ms (weak scaling, no exchange between ranks)."""
    return n_ranks * bytes_per_rank / (ms * 1e-3) / 1e9


class ClockSampler:
    """nvidia-smi clock/throttle samples taken while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.file = None

    def start(self):
        try:
            self.file = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=self.file, stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.file.flush()
        self.file.seek(0)
        rows = [r.split(",") for r in self.file.read().strip().splitlines() if r.strip()]
        os.unlink(self.file.name)
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            r = [x.strip() for x in r]
            if len(r) < 9:
                continue
            try:
                sm.append(float(r[1]))
                smax = float(r[2])
            except ValueError:
                continue
            for name, val in zip(names, r[5:9]):
                if val.lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": len(sm)}


class OracleDecodeSample:
    """The CPU oracle on a bounded sample of the llama8b decode step: the
    packed codes of `n_heads` KV heads (quantized once by the oracle, untimed),
    then per step: unpack them and run the oracle's decode attention for the
    heads' query heads."""

    def __init__(self, n_heads: int = 8, seq_len: int = 32768, seed: int = 1002):
        from oracle import turboquant_oracle as o
        from kv_cache_vector_12_b200 import workloads as wl
        self.o = o
        self.w = w = wl.WORKLOADS["llama8b"]
        self.p = p = o.Params(w.d, w.bits_k, w.bits_v, False, w.pi_seed)
        gen = wl.generator("cpu", seed)
        k, v = wl.kv_tokens(w, seq_len, gen, "cpu")
        self.q = wl.queries(w, 1, gen, "cpu").double().numpy()[0]
        k_new, v_new = wl.kv_tokens(w, 1, gen, "cpu")
        self.new_rows = [(k_new[:, h].double().numpy(), v_new[:, h].double().numpy()) for h in range(n_heads)]
        self.packed = []
        for h in range(n_heads):
            qk = o.quantize(k[:, h].double().numpy(), p.pi, p.ck, p.tk)
            qv = o.quantize(v[:, h].double().numpy(), p.pi, p.cv, p.tv)
            self.packed.append((o.pack_codes(qk.codes, w.bits_k), qk.norm,
                                o.pack_codes(qv.codes, w.bits_v), qv.norm))
        self.step_bytes = n_heads * seq_len * (w.d * (w.bits_k + w.bits_v) // 8 + 4)
        self.desc = (f"oracle append-quantize of 1 token + unpack + decode attention of {n_heads} KV heads x "
                     f"{seq_len} tokens (llama8b decode step, numpy fp64)")

    def step(self) -> float:
        o, w, p = self.o, self.w, self.p
        t0 = time.perf_counter()
        for h, (pk, nk, pv, nv) in enumerate(self.packed):
            kn, vn = self.new_rows[h]                      # append-quantize of the step's token
            o.pack_codes(o.quantize(kn, p.pi, p.ck, p.tk).codes, w.bits_k)
            o.pack_codes(o.quantize(vn, p.pi, p.cv, p.tv).codes, w.bits_v)
            ck = o.unpack_codes(pk, w.bits_k, w.d)
            cv = o.unpack_codes(pv, w.bits_v, w.d)
            o.decode_attention(self.q[h * w.group:(h + 1) * w.group], p.pi, p.ck, ck, nk, p.cv, cv, nv,
                               1 / math.sqrt(w.d))
        return time.perf_counter() - t0

    @staticmethod
    def threads() -> int:
        try:
            from threadpoolctl import threadpool_info
            return max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
        except Exception:
            return os.cpu_count() or 1


def cpu_baseline(min_seconds: float = 10.0) -> dict:
    smp = OracleDecodeSample(n_heads=8)
    total, reps = 0.0, 0
    while total < min_seconds:
        total += smp.step()
        reps += 1
    return {"value": reps * smp.step_bytes / total / 1e9, "unit": "GB/s", "cores": smp.threads(),
            "kind": "oracle", "sample": f"{smp.desc}, {reps} steps", "seconds": total}


def reference_arm(args):
    ws, rank, _ = dist_env()
    if rank != 0:
        return 0
    smp = OracleDecodeSample(n_heads=1)
    times = []
    for i in range(args.warmup + args.steps):
        dt = smp.step()
        if i >= args.warmup:
            times.append(dt)
    total_t = sum(times)
    value = len(times) * smp.step_bytes / total_t / 1e9
    desc = smp.desc + " per step"
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total_t / len(times),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": {"workload": WORKLOAD_DESC, "bits_k": 3, "bits_v": 3, "qjl": False,
                                            "codebook": "gaussian", "sample": desc},
            "cpu_baseline": {"value": value, "unit": "GB/s", "cores": smp.threads(), "kind": "oracle",
                             "sample": desc},
            "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def main(argv=None) -> int:
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=64)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="tq", choices=["tq", "reference"])
    ap.add_argument("--replicas", type=int, default=0, help="cache replicas (default: enough to exceed L2)")
    ap.add_argument("--workload", default="llama8b", choices=sorted(WORKLOAD_DESCS))
    ap.add_argument("--bits", type=int, nargs=2, metavar=("K", "V"), default=None,
                    help="code bits of K and V (default: the workload's)")
    ap.add_argument("--qjl", type=int, choices=[0, 1], default=None, help="1-bit QJL on K (default: the workload's)")
    ap.add_argument("--law", choices=["gaussian", "sphere"], default="gaussian",
                    help="coordinate law of the codebook (tq_law): N(0,1/d) or the exact unit-vector law")
    ap.add_argument("--paged", type=int, default=0, metavar="BLOCK",
                    help="paged cache with BLOCK tokens per block (a multiple of 64) and a shuffled block table")
    ap.add_argument("--breakdown", action="store_true",
                    help="also time each call kind alone (append quantize, decode) and add it to the line")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    if args.impl == "reference":
        return reference_arm(args)

    ws, rank, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if ws > 1:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=dev)

    from kv_cache_vector_12_b200 import tq
    from kv_cache_vector_12_b200 import workloads as wl
    w = wl.WORKLOADS[args.workload]
    bits_k, bits_v = args.bits if args.bits else (w.bits_k, w.bits_v)
    qjl = w.qjl if args.qjl is None else bool(args.qjl)
    H, HQ, D, B = w.n_kv_heads, w.n_q_heads, w.d, w.n_seqs
    lens0 = wl.serving_lengths(w, w.seed) if args.workload == "serving" else [w.seq_len] * B
    T = lens0[0]                       # the quantize measurement uses the first sequence's prefill
    bytes_per_token = H * (D * (bits_k + bits_v) // 8 + 4 + (D // 8 + 2 if qjl else 0))
    R = args.replicas or max(1, math.ceil(2 * 126e6 / (sum(lens0) * bytes_per_token)))
    n_steps_total = args.warmup + args.steps
    cap = int(math.ceil((max(lens0) + n_steps_total + 1) / 64) * 64)
    ctx = tq.Context(D, bits_k, bits_v, int(qjl), w.pi_seed, law=args.law)
    if args.paged:
        if args.paged % 64:
            raise SystemExit("--paged: the block size must be a multiple of 64")
        cap = int(math.ceil(cap / args.paged) * args.paged)
        per_seq = cap // args.paged
        tgen = torch.Generator().manual_seed(w.seed + 31)

        def paged_cache():
            table = torch.randperm(B * per_seq, generator=tgen).to(torch.int32).view(B, per_seq)
            return tq.PagedCache(ctx, B, H, cap, args.paged, n_blocks=B * per_seq, block_table=table, device=dev)
        caches = [paged_cache() for _ in range(R)]
    else:
        caches = [tq.Cache(ctx, B, H, cap, device=dev) for _ in range(R)]
    gen = wl.generator(dev, w.seed + 7919 * rank)
    outl = wl.outlier_scale(w, dev, w.seed) if args.workload == "llama70b" else None

    # ---- prefill quantize (also the quantize measurement: the first sequence) ----
    q_ms = None
    for b in range(B):
        n_b = lens0[b]
        pos0 = torch.arange(n_b, dtype=torch.int32, device=dev)
        k_pre, v_pre = wl.kv_tokens(w, n_b, gen, dev, outlier_mask=outl)
        seqb = torch.full((n_b,), b, dtype=torch.int32, device=dev)
        for c in caches:
            tq.quantize(ctx, c, k_pre, v_pre, seqb, pos0)
        if b == 0:
            torch.cuda.synchronize()
            qreps = 10
            qe = [torch.cuda.Event(enable_timing=True) for _ in range(2 * qreps)]
            for i in range(qreps):
                qe[2 * i].record()
                tq.quantize(ctx, caches[i % R], k_pre, v_pre, seqb, pos0)
                qe[2 * i + 1].record()
            torch.cuda.synchronize()
            q_ms = statistics.median(qe[2 * i].elapsed_time(qe[2 * i + 1]) for i in range(qreps))
        del k_pre, v_pre
    torch.cuda.synchronize()
    ctx.check_device_errors()

    # ---- per-step inputs, resident on the device ----
    k_new, v_new = wl.kv_tokens(w, n_steps_total * B, gen, dev, outlier_mask=outl)   # [steps*B, H, D]
    q_all = wl.queries(w, n_steps_total * B, gen, dev).view(n_steps_total, B, HQ, D)
    pos_steps = torch.empty(n_steps_total, B, dtype=torch.int32, device=dev)
    lens_steps = torch.empty(n_steps_total, B, dtype=torch.int32, device=dev)
    lens_t = torch.tensor(lens0, dtype=torch.int32, device=dev)
    for i in range(n_steps_total):
        pos_steps[i] = lens_t + i // R
        lens_steps[i] = lens_t + i // R + 1
    out = torch.empty(n_steps_total, B, HQ, D, device=dev)
    lse = torch.empty(n_steps_total, B, HQ, device=dev)
    max_len = cap
    wsb = tq.alloc_workspace(ctx, B, HQ, max_len, device=dev)
    seq_ids = torch.arange(B, dtype=torch.int32, device=dev)

    def step(i):
        c = caches[i % R]
        tq.quantize(ctx, c, k_new[i * B:(i + 1) * B], v_new[i * B:(i + 1) * B], seq_ids, pos_steps[i])
        tq.decode_attention(ctx, c, q_all[i], lens_steps[i], max_len, out[i], lse[i], wsb)

    step_bytes = [int(lens_steps[i].sum()) * bytes_per_token for i in range(n_steps_total)]

    # graphs of the warm-up and timed steps
    s = torch.cuda.Stream(device=dev)
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        for i in range(n_steps_total):       # eager pass before capture
            step(i)
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g_warm, g_timed, g_dec = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_warm):
        for i in range(args.warmup):
            step(i)
    with torch.cuda.graph(g_timed):
        for i in range(args.warmup, n_steps_total):
            step(i)
    g_warm.replay()
    torch.cuda.synchronize()
    ctx.check_device_errors()

    sampler = ClockSampler(local)
    if ws > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    sampler.start()
    # keep the GPU busy up to the timed region (clocks at their loaded level,
    # and the clock sampler sees load): about 50 ms of warm-up replays, then
    # the timed replay is queued behind them with no idle gap
    wb0, wb1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    wb0.record()
    g_warm.replay()
    wb1.record()
    torch.cuda.synchronize()
    n_burst = max(1, min(2000, int(50.0 / max(wb0.elapsed_time(wb1), 1e-3))))
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    for _ in range(n_burst):
        g_warm.replay()
    ev0.record()
    g_timed.replay()
    ev1.record()
    torch.cuda.synchronize()
    ms_total = ev0.elapsed_time(ev1)
    # decode calls alone: the timed steps' decode calls (same replicas, same
    # lengths, their tokens already appended) as one CUDA graph, events around
    # its replay on the launching stream
    with torch.cuda.graph(g_dec):
        for i in range(args.warmup, n_steps_total):
            tq.decode_attention(ctx, caches[i % R], q_all[i], lens_steps[i], max_len, out[i], lse[i], wsb)
    g_dec.replay()
    torch.cuda.synchronize()
    ed0, ed1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ed0.record()
    g_dec.replay()
    ed1.record()
    torch.cuda.synchronize()
    clocks = sampler.stop()
    dec_ms = [ed0.elapsed_time(ed1) / args.steps]
    ctx.check_device_errors()

    breakdown = None
    if args.breakdown:
        def timed(fn, reps=20):
            """Device time per call: a CUDA graph of `reps` calls, replayed 5 times."""
            gs = torch.cuda.Stream(device=dev)
            gs.wait_stream(torch.cuda.current_stream())
            with torch.cuda.stream(gs):
                fn()
            torch.cuda.current_stream().wait_stream(gs)
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                for _ in range(reps):
                    fn()
            g.replay()
            ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
            ev[0].record()
            for _ in range(5):
                g.replay()
            ev[1].record()
            torch.cuda.synchronize()
            del g
            return ev[0].elapsed_time(ev[1]) * 1e3 / (5 * reps)
        i_last = n_steps_total - 1
        c_last = caches[i_last % R]
        breakdown = {
            "append_quantize_us": timed(lambda: tq.quantize(ctx, c_last, k_new[i_last * B:(i_last + 1) * B],
                                                            v_new[i_last * B:(i_last + 1) * B], seq_ids,
                                                            pos_steps[i_last])),
            "decode_call_us": timed(lambda: tq.decode_attention(ctx, c_last, q_all[i_last], lens_steps[i_last],
                                                                max_len, out[i_last], lse[i_last], wsb)),
            "step_us": timed(lambda: (tq.quantize(ctx, c_last, k_new[i_last * B:(i_last + 1) * B],
                                                  v_new[i_last * B:(i_last + 1) * B], seq_ids, pos_steps[i_last]),
                                      tq.decode_attention(ctx, c_last, q_all[i_last], lens_steps[i_last], max_len,
                                                          out[i_last], lse[i_last], wsb))),
            "note": "CUDA graph of 20 calls (or steps) on one cache (warm L2), events around the replays",
        }
        torch.cuda.synchronize()

    # ---- end to end through the C ABI with pinned host buffers (eager) ----
    # each step's inputs (the new token's K and V, bf16, and q, bf16) sit in
    # one pinned host block and cross PCIe as one copy
    kb, qb = B * H * D * 2, B * HQ * D * 2
    step_in = 2 * kb + qb
    host_in = torch.empty(n_steps_total, step_in, dtype=torch.uint8).pin_memory()
    for i in range(n_steps_total):
        host_in[i, :kb] = k_new[i * B:(i + 1) * B].cpu().contiguous().view(torch.uint8).flatten()
        host_in[i, kb:2 * kb] = v_new[i * B:(i + 1) * B].cpu().contiguous().view(torch.uint8).flatten()
        host_in[i, 2 * kb:] = q_all[i].to(torch.bfloat16).cpu().contiguous().view(torch.uint8).flatten()
    dev_in = torch.empty(step_in, dtype=torch.uint8, device=dev)
    k_d = dev_in[:kb].view(torch.bfloat16).view(B, H, D)
    v_d = dev_in[kb:2 * kb].view(torch.bfloat16).view(B, H, D)
    q_d = dev_in[2 * kb:].view(torch.bfloat16).view(B, HQ, D)
    out_h = torch.empty(B, HQ, D).pin_memory()
    h2d = step_in
    d2h = out_h.numel() * 4

    # A host application's loop: the C ABI called directly with its
    # arguments prepared once, and the two copies as plain asynchronous
    # driver copies on the same stream (one host-to-device, one back).
    import ctypes
    cu = ctypes.CDLL("libcuda.so.1")
    cu.cuMemcpyHtoDAsync_v2.argtypes = [ctypes.c_uint64, ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p]
    cu.cuMemcpyDtoHAsync_v2.argtypes = [ctypes.c_void_p, ctypes.c_uint64, ctypes.c_size_t, ctypes.c_void_p]
    stream = torch.cuda.current_stream().cuda_stream
    cache_refs = [ctypes.byref(c.struct) for c in caches]
    in_ptrs = [host_in[i].data_ptr() for i in range(n_steps_total)]
    pos_ptrs = [pos_steps[i].data_ptr() for i in range(n_steps_total)]
    len_ptrs = [lens_steps[i].data_ptr() for i in range(n_steps_total)]
    out_ptrs = [out[i].data_ptr() for i in range(n_steps_total)]
    lse_ptrs = [lse[i].data_ptr() for i in range(n_steps_total)]
    dev_ptr, k_ptr, v_ptr, q_ptr = dev_in.data_ptr(), k_d.data_ptr(), v_d.data_ptr(), q_d.data_ptr()
    seq_ptr, out_h_ptr, ws_ptr, ws_len = seq_ids.data_ptr(), out_h.data_ptr(), wsb.data_ptr(), wsb.numel()
    handle, n_out = ctx.handle, out_h.numel() * 4

    def e2e_step(i):
        c = cache_refs[i % R]
        e = cu.cuMemcpyHtoDAsync_v2(dev_ptr, in_ptrs[i], step_in, stream)
        e |= tq.lib.tq_quantize(handle, c, k_ptr, v_ptr, seq_ptr, pos_ptrs[i], B, stream)
        e |= tq.lib.tq_decode_attention(handle, c, q_ptr, tq.TQ_BF16, HQ, len_ptrs[i], max_len, 0.0, out_ptrs[i],
                                        lse_ptrs[i], ws_ptr, ws_len, stream)
        e |= cu.cuMemcpyDtoHAsync_v2(out_h_ptr, out_ptrs[i], n_out, stream)
        if e:
            raise RuntimeError(f"e2e step {i} failed: {tq.lib.tq_last_error()}")

    for i in range(args.warmup):
        e2e_step(i)
    torch.cuda.synchronize()
    if ws > 1:
        torch.distributed.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for i in range(args.warmup, n_steps_total):
        e2e_step(i)
    e1.record()
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1)

    timed_bytes = sum(step_bytes[args.warmup:])
    ms_total, e2e_ms, dec_mean, q_ms = max_over_ranks([ms_total, e2e_ms, statistics.mean(dec_ms), q_ms], dev)
    peak, peak_kind = measured_peaks()
    value = job_gbps(ws, timed_bytes, ms_total)
    e2e_val = job_gbps(ws, timed_bytes, e2e_ms)
    dec_achieved = (timed_bytes / args.steps) / (dec_mean * 1e-3) / 1e9
    q_tokens = T / (q_ms * 1e-3)
    q_bytes = T * H * (2 * D * 2 + D * (bits_k + bits_v) // 8 + 4 + (D // 8 + 2 if qjl else 0))
    q_gbs = q_bytes / (q_ms * 1e-3) / 1e9

    if rank != 0:
        if ws > 1:
            torch.distributed.barrier()
            torch.distributed.destroy_process_group()
        return 0
    cpu = None if args.no_cpu_baseline else cpu_baseline()
    line = {
        "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": ws, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_total / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": {"workload": WORKLOAD_DESCS[args.workload], "bits_k": bits_k, "bits_v": bits_v, "qjl": qjl,
                   "codebook": args.law, "cache_layout": f"paged, {args.paged}-token blocks" if args.paged else "contiguous",
                   "replicas": R, "l2": f"inputs larger than L2: {R} rotating "
                   f"cache replicas of {caches[0].nbytes() / 1e6:.1f} MB", "graph": "CUDA graph of the timed steps",
                   "parallelism": f"replicas x{ws}"},
        "roofline": {"bound": "hbm", "achieved": dec_achieved, "peak": peak, "unit": "GB/s",
                     "frac": dec_achieved / peak,
                     "traffic": MEASURED_TRAFFIC.get((args.workload, bits_k, bits_v, qjl)),
                     "traffic_kernel": "decode_mma_kernel", "peak_source": peak_kind,
                     "kernel": "tq_decode_attention call (split-K attention with q rotation + merge)",
                     "algorithmic_bytes_per_call": timed_bytes / args.steps},
        "quantize": {"tokens_per_s": q_tokens, "GBps": q_gbs, "frac": q_gbs / peak, "ms": q_ms,
                     "tokens": T, "bytes": q_bytes},
        "cpu_baseline": cpu,
        "e2e": {"value": e2e_val, "unit": "GB/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": 3 * args.steps,
        "breakdown": breakdown,
        "clocks": clocks,
    }
    print(json.dumps(line), flush=True)
    if ws > 1:
        torch.distributed.barrier()
        del g_warm, g_timed, g_dec
        torch.distributed.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
