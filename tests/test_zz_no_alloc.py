"""tq_decode_attention_noalloc against tq_decode_attention.

The allocation-free entry point serves callers that cannot allocate device
memory while they decode (inside CUDA graph stream capture, in engines
restricted to their own memory pool, in loops that cannot absorb
cudaMalloc's synchronisation).  It must give the same attention as the
entry point that takes a caller workspace, call after call, although every
call reuses one static scratch array.  This file is collected last so that a
run stopping at its first failure has run every other test; it also passes
on its own in a fresh process.
"""
import ctypes

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

D = 128
RTOL = 1e-3   # the parity tolerance of the attention tests


@pytest.fixture(scope="module")
def tq(cuda_device):
    from kv_cache_vector_12_b200 import tq as tqmod
    return tqmod


def _filled_cache(tq, ctx, lens, n_heads, seed):
    cap = int(np.ceil(max(lens) / 64) * 64)
    cache = tq.Cache(ctx, len(lens), n_heads, cap)
    g = torch.Generator().manual_seed(seed)
    for s, n in enumerate(lens):
        k = (torch.randn(n, n_heads, D, generator=g) * 2).to(torch.bfloat16).cuda()
        v = torch.randn(n, n_heads, D, generator=g).to(torch.bfloat16).cuda()
        tq.quantize(ctx, cache, k, v, torch.full((n,), s, dtype=torch.int32, device="cuda"),
                    torch.arange(n, dtype=torch.int32, device="cuda"))
    return cache, cap


def _noalloc(tq, ctx, cache, q, lens, max_len, out, lse):
    """Call the C entry point directly (no binding helper in between)."""
    return tq.lib.tq_decode_attention_noalloc(
        ctx.handle, ctypes.byref(cache.struct), q.data_ptr(), tq.TQ_F32, q.shape[1], lens.data_ptr(), max_len,
        ctypes.c_float(0.0), out.data_ptr(), lse.data_ptr(), torch.cuda.current_stream().cuda_stream)


def _agree(out_a, lse_a, out_b, lse_b):
    a, b = out_a.double().cpu().numpy(), out_b.double().cpu().numpy()
    den = np.maximum(np.abs(b).max(axis=-1), 1e-30)
    assert np.all(np.abs(a - b).max(axis=-1) / den <= RTOL)
    la, lb = lse_a.double().cpu().numpy(), lse_b.double().cpu().numpy()
    assert np.all(np.abs(la - lb) <= RTOL * np.maximum(1.0, np.abs(lb)))


def test_noalloc_matches_workspace_path_on_two_calls_in_a_row(tq):
    ctx = tq.Context(D, 3, 3, 0, 42)
    n_heads, group = 2, 4
    lens_all = [3000, 700]
    cache, cap = _filled_cache(tq, ctx, lens_all, n_heads, seed=21)
    g = torch.Generator().manual_seed(22)
    # two different calls: different queries, lengths and length bound
    for lens, max_len in (([3000, 700], cap), ([1500, 2999], 3008)):
        q = torch.randn(len(lens), n_heads * group, D, generator=g).cuda()
        seq_lens = torch.tensor(lens, dtype=torch.int32, device="cuda")
        out_ref = torch.empty(len(lens), n_heads * group, D, device="cuda")
        lse_ref = torch.empty(len(lens), n_heads * group, device="cuda")
        ws = tq.alloc_workspace(ctx, len(lens), n_heads * group, max_len)
        tq.decode_attention(ctx, cache, q, seq_lens, max_len, out_ref, lse_ref, ws)
        out = torch.full_like(out_ref, float("nan"))
        lse = torch.full_like(lse_ref, float("nan"))
        assert _noalloc(tq, ctx, cache, q, seq_lens, max_len, out, lse) == tq.TQ_OK, tq.lib.tq_last_error()
        ctx.check_device_errors()
        _agree(out, lse, out_ref, lse_ref)


def test_noalloc_rejects_workspace_beyond_static_scratch(tq):
    ctx = tq.Context(D, 3, 3, 0, 42)
    n_seqs, n_q = 128, 128          # 16384 query rows: one 528-byte partial each exceeds the scratch
    cache = tq.Cache(ctx, n_seqs, 8, 64)
    max_len = 64
    need = tq.workspace_bytes(ctx, n_seqs, n_q, max_len)
    assert need > 8 * 1024 * 1024
    q = torch.zeros(n_seqs, n_q, D, device="cuda")
    lens = torch.zeros(n_seqs, dtype=torch.int32, device="cuda")
    out = torch.full((n_seqs, n_q, D), 7.0, device="cuda")
    lse = torch.full((n_seqs, n_q), 7.0, device="cuda")
    assert _noalloc(tq, ctx, cache, q, lens, max_len, out, lse) == tq.TQ_ERR_INVALID
    assert b"static scratch" in tq.lib.tq_last_error()
    torch.cuda.synchronize()
    assert bool((out == 7.0).all()) and bool((lse == 7.0).all())   # nothing was launched


def test_noalloc_inside_cuda_graph_capture(tq):
    """The point of the entry point: captured in a CUDA graph (no allocation,
    no synchronisation inside the call), then replayed on new queries."""
    ctx = tq.Context(D, 3, 3, 0, 42)
    n_heads, group = 2, 4
    lens_all = [2500, 900]
    cache, cap = _filled_cache(tq, ctx, lens_all, n_heads, seed=31)
    seq_lens = torch.tensor(lens_all, dtype=torch.int32, device="cuda")
    q = torch.zeros(len(lens_all), n_heads * group, D, device="cuda")
    out = torch.empty(len(lens_all), n_heads * group, D, device="cuda")
    lse = torch.empty(len(lens_all), n_heads * group, device="cuda")
    assert _noalloc(tq, ctx, cache, q, seq_lens, cap, out, lse) == tq.TQ_OK   # first call outside capture
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        assert _noalloc(tq, ctx, cache, q, seq_lens, cap, out, lse) == tq.TQ_OK
    g = torch.Generator().manual_seed(32)
    ws = tq.alloc_workspace(ctx, len(lens_all), n_heads * group, cap)
    for _ in range(2):
        q.copy_(torch.randn(q.shape, generator=g))
        graph.replay()
        torch.cuda.synchronize()
        out_ref = torch.empty_like(out)
        lse_ref = torch.empty_like(lse)
        tq.decode_attention(ctx, cache, q, seq_lens, cap, out_ref, lse_ref, ws)
        ctx.check_device_errors()
        _agree(out, lse, out_ref, lse_ref)
