"""Benchmark of the TurboQuant hot path on B200 (one JSON line on rank 0).

Workload (default ``serving``, the largest single-GPU configuration): 32
decode sequences with seeded lengths uniform on [1024, 65536], 8 KV / 32
query heads, d = 128, bf16 K/V ~ N(0,1), 3-bit K and V (no QJL).  The
prefill is quantized once into R cache replicas; a *step* is one decode step
of the whole hot path: quantize-on-append of one new token per sequence (8 KV
heads, K and V) followed by the ragged batched decode attention of the 32
query heads over the packed cache.  Step i uses replica i % R; R is chosen so
the replicas exceed twice the 126 MB L2 (one replica of ~0.85 GB for
serving), so every step reads its cache cold.  ``--workload`` selects the
other configurations (llama8b, llama70b, qwen, tiny).

``value``  decode-attention effective GB/s: packed K/V bytes the step reads
           (codes + fp16 norms) / device time per step.  The K timed steps
           are one CUDA graph; it is replayed back to back for at least
           200 ms, each replay bracketed by CUDA events, and the median replay
           time is the time of K steps (max over ranks).
``e2e``    the same metric when every step goes through the C ABI eagerly
           with pinned host buffers: H2D of the tokens' K/V and of q, the two
           calls, D2H of the output.
``roofline`` the decode calls of the timed steps alone (same replicas and
           lengths) as one CUDA graph, replayed the same way; algorithmic
           bytes = packed bytes per call.
``quantize`` the whole prefill of the batch (every sequence's tokens, one
           call; inputs far larger than L2): tokens/s, GB/s (bf16 read +
           packed write) and roofline fraction.
``quality`` compressed vs exact (fp64, over the bf16 inputs) attention of a
           sampled (sequence, KV head): cosine similarity of the outputs,
           bias and RMS of the per-token score error relative to the RMS of
           the exact scores, and the cosine similarity of reconstructed V
           vectors, all read from the library's own kernels.
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
DEFAULT_WORKLOAD = "serving"


# DRAM bytes per attention-kernel launch (dram__bytes_read.sum +
# dram__bytes_write.sum) from one ncu capture of a full-size launch of the
# workload's default setting (d = 128, contiguous cache, Gaussian codebook,
# every sequence), keyed by (workload, bits_k, bits_v, qjl); null elsewhere.
# Re-captured whenever the kernel changes.
MEASURED_TRAFFIC = {("serving", 3, 3, False): 809885696.0 + 5876736.0}


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


def measured_tensor_peak():
    """Dense bf16 tensor peak (TFLOP/s) for a kernel timed alone: the measured
    burst figure, else the fallback measurement of this GPU type."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        if "bf16_tflops" in p:
            return float(p["bf16_tflops"]), "measured"
    return 1590.0, "fallback"


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
    """The CPU oracle on a bounded sample of one decode step of a workload:
    the first sequence's cache for `n_heads` KV heads (quantized once by the
    oracle, untimed), then per step: append-quantize of the step's token,
    unpack of the codes and the oracle's decode attention for the heads'
    query heads."""

    def __init__(self, workload: str, bits_k: int, bits_v: int, qjl: bool, n_heads: int = 8, head_dim: int = 128):
        import dataclasses
        from oracle import turboquant_oracle as o
        from kv_cache_vector_12_b200 import workloads as wl
        self.o = o
        self.w = w = dataclasses.replace(wl.WORKLOADS[workload], d=head_dim)
        self.bits_k, self.bits_v, self.qjl = bits_k, bits_v, qjl
        self.p = p = o.Params(w.d, bits_k, bits_v, qjl, w.pi_seed)
        n_heads = min(n_heads, w.n_kv_heads)
        seq_len = wl.serving_lengths(w, w.seed)[0] if workload == "serving" else w.seq_len
        gen = wl.generator("cpu", w.seed)
        outl = wl.outlier_scale(w, "cpu", w.seed) if workload == "llama70b" else None
        k, v = wl.kv_tokens(w, seq_len, gen, "cpu", outlier_mask=outl)
        self.q = wl.queries(w, 1, gen, "cpu").double().numpy()[0]
        k_new, v_new = wl.kv_tokens(w, 1, gen, "cpu", outlier_mask=outl)
        self.new_rows = [(k_new[:, h].double().numpy(), v_new[:, h].double().numpy()) for h in range(n_heads)]
        self.packed = []
        for h in range(n_heads):
            qk = o.quantize(k[:, h].double().numpy(), p.pi, p.ck, p.tk, s_matrix=p.s if qjl else None)
            qv = o.quantize(v[:, h].double().numpy(), p.pi, p.cv, p.tv)
            self.packed.append((o.pack_codes(qk.codes, bits_k), qk.norm, o.pack_codes(qv.codes, bits_v), qv.norm,
                                o.pack_signs(qk.qjl_signs) if qjl else None, qk.qjl_gamma if qjl else None))
        self.step_bytes = n_heads * seq_len * (w.d * (bits_k + bits_v) // 8 + 4 + (w.d // 8 + 2 if qjl else 0))
        self.desc = (f"oracle append-quantize of 1 token + unpack + decode attention of {n_heads} KV heads x "
                     f"{seq_len} tokens ({workload} decode step, first sequence, {bits_k}/{bits_v} bits"
                     f"{' + QJL' if qjl else ''}, numpy fp64)")

    def step(self) -> float:
        o, w, p = self.o, self.w, self.p
        s_mat = p.s if self.qjl else None
        t0 = time.perf_counter()
        for h, (pk, nk, pv, nv, pj, gj) in enumerate(self.packed):
            kn, vn = self.new_rows[h]                      # append-quantize of the step's token
            o.pack_codes(o.quantize(kn, p.pi, p.ck, p.tk, s_matrix=s_mat).codes, self.bits_k)
            o.pack_codes(o.quantize(vn, p.pi, p.cv, p.tv).codes, self.bits_v)
            ck = o.unpack_codes(pk, self.bits_k, w.d)
            cv = o.unpack_codes(pv, self.bits_v, w.d)
            signs = o.unpack_signs(pj, w.d) if self.qjl else None
            o.decode_attention(self.q[h * w.group:(h + 1) * w.group], p.pi, p.ck, ck, nk, p.cv, cv, nv,
                               1 / math.sqrt(w.d), s_matrix=s_mat, qjl_signs=signs, qjl_gamma=gj)
        return time.perf_counter() - t0

    @staticmethod
    def threads() -> int:
        try:
            from threadpoolctl import threadpool_info
            return max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
        except Exception:
            return os.cpu_count() or 1


def cpu_baseline(workload: str, bits_k: int, bits_v: int, qjl: bool, head_dim: int = 128,
                 min_seconds: float = 10.0) -> dict:
    smp = OracleDecodeSample(workload, bits_k, bits_v, qjl, n_heads=8, head_dim=head_dim)
    total, reps = 0.0, 0
    while total < min_seconds:
        total += smp.step()
        reps += 1
    return {"value": reps * smp.step_bytes / total / 1e9, "unit": "GB/s", "cores": smp.threads(),
            "kind": "oracle", "sample": f"{smp.desc}, {reps} steps", "seconds": total}


def resolve_setting(args):
    import dataclasses
    from kv_cache_vector_12_b200 import workloads as wl
    w = wl.WORKLOADS[args.workload]
    if args.head_dim != w.d:
        w = dataclasses.replace(w, d=args.head_dim)
    bits_k, bits_v = args.bits if args.bits else (w.bits_k, w.bits_v)
    qjl = w.qjl if args.qjl is None else bool(args.qjl)
    return w, bits_k, bits_v, qjl


def reference_arm(args):
    ws, rank, _ = dist_env()
    if rank != 0:
        return 0
    w, bits_k, bits_v, qjl = resolve_setting(args)
    smp = OracleDecodeSample(args.workload, bits_k, bits_v, qjl, n_heads=1, head_dim=w.d)
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
            "data": "synthetic", "config": {"workload": WORKLOAD_DESCS[args.workload], "bits_k": bits_k,
                                            "bits_v": bits_v, "qjl": qjl, "codebook": args.law, "sample": desc},
            "cpu_baseline": {"value": value, "unit": "GB/s", "cores": smp.threads(), "kind": "oracle",
                             "sample": desc},
            "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def quality_report(tq, ctx, cache, lens0, q_first, k_s0, v_s0, group, n_tokens=4096) -> dict:
    """Compressed vs exact attention on a sampled (sequence 0, KV head 0),
    every compressed figure read from the library's kernels.

    * attn_cos_sim: cosine similarity of the decode outputs of KV head 0's
      query heads over sequence 0 (its prefill length) with fp64 softmax
      attention over the bf16 K/V rows that were quantized (mean and min over
      the query heads).
    * score_bias_rel / score_rms_rel: the per-token score error (inner-product
      error times the softmax scale) of the first `n_tokens` tokens: a batch
      of one-token sequences, quantized by the library, whose decode returns
      each token's score as the log-sum-exp; bias and RMS of s_tq - s_exact,
      relative to the RMS of the exact scores.
    * v_cos_sim: the same one-token decodes return the reconstructed V
      vectors (o = Pi^T ||v|| c_V[codes]); mean cosine similarity with the
      original rows, the figure the pages quote per V bit width."""
    dev = q_first.device
    D = q_first.shape[-1]
    scale = 1.0 / math.sqrt(D)
    B, HQ = q_first.shape[0], q_first.shape[1]
    out = torch.empty(B, HQ, D, device=dev)
    ws = tq.alloc_workspace(ctx, B, HQ, max(lens0), device=dev)
    tq.decode_attention(ctx, cache, q_first, torch.tensor(lens0, dtype=torch.int32, device=dev), max(lens0), out,
                        None, ws)
    q0 = q_first[0, :group].double().cpu()                         # [G, d]
    k0, v0 = k_s0.double(), v_s0.double()                          # [T, d]
    s_ex = scale * (q0 @ k0.T)
    o_ex = torch.softmax(s_ex, dim=1) @ v0
    o_tq = out[0, :group].double().cpu()
    cos = torch.nn.functional.cosine_similarity(o_tq, o_ex, dim=1)

    n = min(n_tokens, k_s0.shape[0])
    one = tq.Cache(ctx, n, 1, 64, device=dev)
    idx = torch.arange(n, dtype=torch.int32, device=dev)
    tq.quantize(ctx, one, k_s0[:n, None].to(dev).contiguous(), v_s0[:n, None].to(dev).contiguous(), idx, idx * 0)
    q_rep = q_first[0, :group].float()[None].expand(n, group, D).contiguous()
    out1 = torch.empty(n, group, D, device=dev)
    lse1 = torch.empty(n, group, device=dev)
    ws1 = tq.alloc_workspace(ctx, n, group, 1, device=dev)
    tq.decode_attention(ctx, one, q_rep, torch.ones(n, dtype=torch.int32, device=dev), 1, out1, lse1, ws1)
    ctx.check_device_errors()
    s_tq = lse1.double().cpu().T                                   # [G, n]
    err = s_tq - s_ex[:, :n]
    rms_ex = float(s_ex[:, :n].pow(2).mean().sqrt())
    v_hat = out1[:, 0].double().cpu()
    v_cos = torch.nn.functional.cosine_similarity(v_hat, v0[:n], dim=1)
    return {"sample": f"sequence 0, KV head 0 ({k_s0.shape[0]} tokens, {group} query heads); scores and V "
                      f"vectors of its first {n} tokens",
            "attn_cos_sim": float(cos.mean()), "attn_cos_sim_min": float(cos.min()),
            "score_bias_rel": float(err.mean()) / rms_ex, "score_rms_rel": float(err.pow(2).mean().sqrt()) / rms_ex,
            "v_cos_sim": float(v_cos.mean()),
            "pages_v_cos_sim": {"2-bit V": 0.94, "4-bit V": 0.997},
            "reference": "exact softmax attention in fp64 over the bf16 K/V rows"}


def prefill_report(tq, ctx, cache, q_all, n_tok, n_q_heads, reps=3) -> dict:
    """Causal prefill attention of the first n_tok positions of sequence 0 of
    `cache` (every position a query; the cache holds the quantized prompt), as
    one tq_prefill_attention call: median device time of `reps` calls (CUDA
    events on the launching stream).  Logical flops per (query, key, query
    head) = 4 d (2 d for the score, 2 d for the value accumulation)."""
    dev = q_all.device
    D = q_all.shape[-1]
    B = cache.n_seqs
    cu = torch.tensor([0] + [n_tok] * B, dtype=torch.int32, device=dev)   # only sequence 0 has queries
    lens = torch.full((B,), n_tok, dtype=torch.int32, device=dev)
    out = torch.empty(n_tok, n_q_heads, D, device=dev)
    lse = torch.empty(n_tok, n_q_heads, device=dev)
    tq.prefill_attention(ctx, cache, q_all, cu, lens, n_tok, n_tok, out, lse)
    torch.cuda.synchronize()
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(2 * reps)]
    for i in range(reps):
        evs[2 * i].record()
        tq.prefill_attention(ctx, cache, q_all, cu, lens, n_tok, n_tok, out, lse)
        evs[2 * i + 1].record()
    torch.cuda.synchronize()
    ctx.check_device_errors()
    ms = statistics.median(evs[2 * i].elapsed_time(evs[2 * i + 1]) for i in range(reps))
    flops = n_tok * (n_tok + 1) / 2 * n_q_heads * 4 * D
    peak, kind = measured_tensor_peak()
    tflops = flops / (ms * 1e-3) / 1e12
    return {"tokens": n_tok, "ms": ms, "tokens_per_s": n_tok / (ms * 1e-3), "logical_TFLOPs": tflops,
            "roofline": {"bound": "tensor", "achieved": tflops, "peak": peak, "unit": "TFLOP/s",
                         "frac": tflops / peak, "peak_source": kind},
            "call": f"tq_prefill_attention over the first {n_tok} positions of sequence 0 (every position a "
                    f"query, causal), median of {reps}"}


def weight_report(tq, ctx, dev, n_out=14336, n_in=4096, token_counts=(1, 16), reps=20) -> dict:
    """Weight-quantization reuse on a Llama-3-8B-shaped MLP projection
    (W [14336][4096], seeded N(0,1) bf16): the rows quantized block by block
    (tq_weight_quantize) with the context's K bits, then y = x W~^T over the
    packed rows (tq_weight_gemm) for 1 and 16 tokens; median device time of
    `reps` calls each (a CUDA graph of the calls, so the host's launch time is
    not counted), beside torch's bf16 matmul of the same shape (the library
    product it replaces).  Effective GB/s = packed weight bytes per
    call / time."""
    gen = torch.Generator(device=dev).manual_seed(77)
    w = torch.randn(n_out, n_in, generator=gen, device=dev).to(torch.bfloat16)
    wc = tq.WeightCache(ctx, n_out, n_in, device=dev)
    tq.weight_quantize(ctx, wc, w)
    torch.cuda.synchronize()
    packed = wc.codes[:, :n_out].numel() + 2 * wc.norms[:, :n_out].numel()

    def med(fn):
        """Device time per call: `reps` calls captured as one CUDA graph (so
        host launch overhead is not timed), replayed 5 times; median replay."""
        gs = torch.cuda.Stream(device=dev)
        gs.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(gs):
            fn()
        torch.cuda.current_stream().wait_stream(gs)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for _ in range(reps):
                fn()
        g.replay()
        torch.cuda.synchronize()
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(10)]
        for i in range(5):
            ev[2 * i].record()
            g.replay()
            ev[2 * i + 1].record()
        torch.cuda.synchronize()
        del g
        return statistics.median(ev[2 * i].elapsed_time(ev[2 * i + 1]) for i in range(5)) / reps

    out = {"shape": [n_out, n_in], "bits": ctx.bits_k, "packed_bytes": packed, "bf16_bytes": 2 * n_out * n_in}
    for n_tok in token_counts:
        x = torch.randn(n_tok, n_in, generator=gen, device=dev).to(torch.bfloat16)
        y = torch.empty(n_tok, n_out, device=dev)
        ws = torch.empty(tq.weight_workspace_bytes(ctx, n_tok, n_in), dtype=torch.uint8, device=dev)
        ms = med(lambda: tq.weight_gemm(ctx, wc, x, y, ws))
        ms_ref = med(lambda: x @ w.T)
        ref = (x.float() @ w.float().T)
        out[f"tokens_{n_tok}"] = {"us": ms * 1e3, "GBps": packed / (ms * 1e-3) / 1e9, "bf16_matmul_us": ms_ref * 1e3,
                                  "speedup_vs_bf16": ms_ref / ms,
                                  "rel_error_vs_bf16": float((y - ref).norm() / ref.norm())}
    ctx.check_device_errors()
    return out


def prefill_only(args) -> int:
    """`--prefill-only N`: the prefill leg alone on one sequence of the
    workload's shapes and value law whose N tokens are quantized and then all
    attend causally (the command the prefill kernel's profile is taken on)."""
    from kv_cache_vector_12_b200 import tq
    from kv_cache_vector_12_b200 import workloads as wl
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    w, bits_k, bits_v, qjl = resolve_setting(args)
    n = args.prefill_only
    ctx = tq.Context(w.d, bits_k, bits_v, int(qjl), w.pi_seed, law=args.law)
    cache = tq.Cache(ctx, 1, w.n_kv_heads, (n + 63) // 64 * 64, device=dev)
    gen = wl.generator(dev, w.seed)
    outl = wl.outlier_scale(w, dev, w.seed) if args.workload == "llama70b" else None
    k, v = wl.kv_tokens(w, n, gen, dev, outlier_mask=outl)
    pos = torch.arange(n, dtype=torch.int32, device=dev)
    tq.quantize(ctx, cache, k, v, torch.zeros(n, dtype=torch.int32, device=dev), pos)
    rep = prefill_report(tq, ctx, cache, wl.queries(w, n, gen, dev), n, w.n_q_heads, reps=max(3, args.steps))
    print(json.dumps({"metric": "causal prefill attention over the packed cache", "value": rep["tokens_per_s"],
                      "unit": "tokens/s", "config": {"workload": WORKLOAD_DESCS[args.workload], "tokens": n,
                                                      "bits_k": bits_k, "bits_v": bits_v, "qjl": qjl},
                      "prefill": rep}), flush=True)
    return 0


def main(argv=None) -> int:
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=64)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="tq", choices=["tq", "reference"])
    ap.add_argument("--replicas", type=int, default=0, help="cache replicas (default: enough to exceed L2)")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(WORKLOAD_DESCS))
    ap.add_argument("--bits", type=int, nargs=2, metavar=("K", "V"), default=None,
                    help="code bits of K and V (default: the workload's)")
    ap.add_argument("--qjl", type=int, choices=[0, 1], default=None, help="1-bit QJL on K (default: the workload's)")
    ap.add_argument("--law", choices=["gaussian", "sphere"], default="gaussian",
                    help="coordinate law of the codebook (tq_law): N(0,1/d) or the exact unit-vector law")
    ap.add_argument("--head-dim", type=int, choices=[64, 128, 256], default=128,
                    help="head dimension d of the workload (its other shapes unchanged)")
    ap.add_argument("--paged", type=int, default=0, metavar="BLOCK",
                    help="paged cache with BLOCK tokens per block (a multiple of 64) and a shuffled block table")
    ap.add_argument("--breakdown", action="store_true",
                    help="also time each call kind alone (append quantize, decode) and add it to the line")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--max-seqs", type=int, default=0, metavar="N",
                    help="keep only the workload's first N sequences (a smaller case of the same kernels, for profiling)")
    ap.add_argument("--prefill-only", type=int, default=0, metavar="N",
                    help="only the prefill-attention leg, on one sequence of N tokens of the workload")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    if args.impl == "reference":
        return reference_arm(args)
    if args.prefill_only:
        return prefill_only(args)

    ws, rank, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if ws > 1:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=dev)

    from kv_cache_vector_12_b200 import tq
    from kv_cache_vector_12_b200 import workloads as wl
    w, bits_k, bits_v, qjl = resolve_setting(args)
    lens0 = wl.serving_lengths(w, w.seed) if args.workload == "serving" else [w.seq_len] * w.n_seqs
    if args.max_seqs:
        import dataclasses
        lens0 = lens0[:args.max_seqs]
        w = dataclasses.replace(w, n_seqs=len(lens0))
    H, HQ, D, B = w.n_kv_heads, w.n_q_heads, w.d, w.n_seqs
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

    # ---- prefill: every sequence's tokens in one quantize call per replica;
    # the same call, repeated, is the quantize measurement (inputs of
    # sum(lens) x H x d bf16 for K and V, far larger than L2) ----
    n_pre = sum(lens0)
    k_pre = torch.empty(n_pre, H, D, dtype=torch.bfloat16, device=dev)
    v_pre = torch.empty_like(k_pre)
    seq_pre = torch.empty(n_pre, dtype=torch.int32, device=dev)
    pos_pre = torch.empty(n_pre, dtype=torch.int32, device=dev)
    off = 0
    for b, n_b in enumerate(lens0):
        k_b, v_b = wl.kv_tokens(w, n_b, gen, dev, outlier_mask=outl)
        k_pre[off:off + n_b], v_pre[off:off + n_b] = k_b, v_b
        seq_pre[off:off + n_b] = b
        pos_pre[off:off + n_b] = torch.arange(n_b, dtype=torch.int32, device=dev)
        off += n_b
        del k_b, v_b
    # the sampled (sequence 0, KV head 0) of the quality report, kept on the host
    k_s0, v_s0 = k_pre[:lens0[0], 0].cpu(), v_pre[:lens0[0], 0].cpu()
    for c in caches:
        tq.quantize(ctx, c, k_pre, v_pre, seq_pre, pos_pre)
    torch.cuda.synchronize()
    qreps = 10
    qe = [torch.cuda.Event(enable_timing=True) for _ in range(2 * qreps)]
    for i in range(qreps):
        qe[2 * i].record()
        tq.quantize(ctx, caches[i % R], k_pre, v_pre, seq_pre, pos_pre)
        qe[2 * i + 1].record()
    torch.cuda.synchronize()
    q_ms = statistics.median(qe[2 * i].elapsed_time(qe[2 * i + 1]) for i in range(qreps))
    del k_pre, v_pre, seq_pre, pos_pre
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

    def replay_median(graph, min_ms=200.0):
        """Median device time (ms) of one replay of `graph`: replays queued
        back to back, each bracketed by CUDA events on the launching stream,
        for at least `min_ms` in total (three at least)."""
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        graph.replay()
        e1.record()
        torch.cuda.synchronize()
        n = max(3, min(1000, int(math.ceil(min_ms / max(e0.elapsed_time(e1), 1e-3)))))
        evs = [torch.cuda.Event(enable_timing=True) for _ in range(2 * n)]
        for j in range(n):
            evs[2 * j].record()
            graph.replay()
            evs[2 * j + 1].record()
        torch.cuda.synchronize()
        times = [evs[2 * j].elapsed_time(evs[2 * j + 1]) for j in range(n)]
        return statistics.median(times), n

    # decode calls alone: the timed steps' decode calls (same replicas, same
    # lengths, their tokens already appended) as one CUDA graph
    with torch.cuda.graph(g_dec):
        for i in range(args.warmup, n_steps_total):
            tq.decode_attention(ctx, caches[i % R], q_all[i], lens_steps[i], max_len, out[i], lse[i], wsb)
    g_dec.replay()
    torch.cuda.synchronize()

    sampler = ClockSampler(local)
    if ws > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    sampler.start()
    # keep the GPU busy up to the timed region (clocks at their loaded level,
    # and the clock sampler sees load): about 50 ms of warm-up replays, then
    # the timed replays are queued behind them with no idle gap
    wb0, wb1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    wb0.record()
    g_warm.replay()
    wb1.record()
    torch.cuda.synchronize()
    n_burst = max(1, min(2000, int(50.0 / max(wb0.elapsed_time(wb1), 1e-3))))
    for _ in range(n_burst):
        g_warm.replay()
    ms_total, n_replays = replay_median(g_timed)
    dec_total, _ = replay_median(g_dec)
    clocks = sampler.stop()
    dec_ms = [dec_total / args.steps]
    ctx.check_device_errors()
    quality = quality_report(tq, ctx, caches[0], lens0, q_all[args.warmup], k_s0, v_s0, w.group)
    prefill = None
    if D == 128:  # prefill attention is built for d = 128
        n_prefill = min(lens0[0], 32768)
        q_prefill = wl.queries(w, n_prefill, gen, dev)                 # [n_prefill, HQ, D]
        prefill = prefill_report(tq, ctx, caches[0], q_prefill, n_prefill, HQ)
        del q_prefill
    weights = weight_report(tq, ctx, dev) if D == 128 else None

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
    q_tokens = n_pre / (q_ms * 1e-3)
    q_bytes = n_pre * H * (2 * D * 2 + D * (bits_k + bits_v) // 8 + 4 + (D // 8 + 2 if qjl else 0))
    q_gbs = q_bytes / (q_ms * 1e-3) / 1e9

    if rank != 0:
        if ws > 1:
            torch.distributed.barrier()
            torch.distributed.destroy_process_group()
        return 0
    cpu = None if args.no_cpu_baseline else cpu_baseline(args.workload, bits_k, bits_v, qjl, D)
    line = {
        "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": ws, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_total / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": {"workload": WORKLOAD_DESCS[args.workload] + (f" (head dimension {D})" if D != 128 else "")
                   + (f" (first {B} sequences only)" if args.max_seqs else ""),
                   "bits_k": bits_k, "bits_v": bits_v, "qjl": qjl, "head_dim": D,
                   "codebook": args.law, "cache_layout": f"paged, {args.paged}-token blocks" if args.paged else "contiguous",
                   "replicas": R, "l2": f"inputs larger than L2: {R} rotating "
                   f"cache replicas of {caches[0].nbytes() / 1e6:.1f} MB", "graph": f"CUDA graph of the {args.steps} timed steps, replayed back to back "
                   f"{n_replays} times (>= 200 ms); median replay",
                   "parallelism": f"replicas x{ws}"},
        "roofline": {"bound": "hbm", "achieved": dec_achieved, "peak": peak, "unit": "GB/s",
                     "frac": dec_achieved / peak,
                     "traffic": (MEASURED_TRAFFIC.get((args.workload, bits_k, bits_v, qjl))
                                 if D == 128 and not args.paged and not args.max_seqs and args.law == "gaussian"
                                 else None),
                     "traffic_kernel": "decode_mma_kernel", "peak_source": peak_kind,
                     "kernel": "tq_decode_attention call (split-K attention with q rotation + merge)",
                     "algorithmic_bytes_per_call": timed_bytes / args.steps},
        "quantize": {"tokens_per_s": q_tokens, "GBps": q_gbs, "frac": q_gbs / peak, "ms": q_ms,
                     "tokens": n_pre, "bytes": q_bytes,
                     "call": f"one tq_quantize of the whole prefill ({B} sequences, {n_pre} tokens x {H} KV heads), "
                             "median of 10"},
        "quality": quality,
        "prefill": prefill,
        "weights": weights,
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
