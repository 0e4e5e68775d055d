"""GPU parity of causal prefill attention over the packed cache
(tq_prefill_attention) against the oracle's prefill_attention, on the same
seeded inputs: prompts of 1, 127, 128, 129 and 4096 tokens, chunks of a
prompt whose earlier part is already cached, several sequences in one call
(one of them without queries), 1 to 16 query heads per KV head, every
(bits, QJL) setting, fp32 and bf16 queries, and a paged cache.  Outputs are
compared per (query, head) at ||o - o_ref||_inf <= 1e-3 ||o_ref||_inf and the
log-sum-exp at 1e-3 max(1, max_j |s_j|)."""
import math

import numpy as np
import pytest
import torch

from oracle import turboquant_oracle as o
from tests import parity_helpers as ph
from tests.test_gpu_parity import D, SETTINGS, _oracle_cache, _upload, make_rows, oracle_params

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def tq(cuda_device):
    from kv_cache_vector_12_b200 import tq as tqmod
    return tqmod


def _prefill_and_compare(tq, lens, n_q, n_heads, group, bits_k, bits_v, qjl, seed, q_dtype=torch.float32,
                         paged_block=0, sample=None):
    """lens[s]: cached tokens of sequence s; n_q[s]: its queries (its last
    n_q[s] positions).  sample: compare at most this many queries per
    sequence (seeded choice, the first and last always included)."""
    ctx = tq.Context(D, bits_k, bits_v, qjl, 42)
    ref = oracle_params(bits_k, bits_v, qjl)
    min_cap = max(lens)
    if paged_block:
        min_cap = int(math.ceil(max(min_cap, 1) / paged_block) * paged_block)
    per, planes, cap = _oracle_cache(ref, lens, n_heads, bits_k, bits_v, qjl, seed, min_cap=min_cap)
    cache = _upload(tq, ctx, planes, len(lens), n_heads, cap, paged=(paged_block, seed) if paged_block else None)
    n_qh = n_heads * group
    total = sum(n_q)
    g = torch.Generator().manual_seed(seed + 5)
    q = torch.randn(total, n_qh, D, generator=g).to(q_dtype)
    cu = torch.tensor([0] + list(np.cumsum(n_q)), dtype=torch.int32, device="cuda")
    out = torch.full((total, n_qh, D), float("nan"), device="cuda")
    lse = torch.full((total, n_qh), float("nan"), device="cuda")
    tq.prefill_attention(ctx, cache, q.cuda(), cu, torch.tensor(lens, dtype=torch.int32, device="cuda"),
                         max(max(n_q), 1), max(lens), out, lse)
    ctx.check_device_errors()
    out, lse = out.cpu().numpy(), lse.cpu().numpy()
    qd = q.double().numpy()
    rng = np.random.default_rng(seed)
    worst = 0.0
    for s, (n, nq) in enumerate(zip(lens, n_q)):
        if nq == 0:
            continue
        idx = np.arange(nq)
        if sample and nq > sample:
            idx = np.unique(np.concatenate([[0, nq - 1], rng.choice(nq, sample - 2, replace=False)]))
        rows = cu[s].item() + idx
        pos = n - nq + idx
        for h in range(n_heads):
            qk, qv = per[(s, h)]
            heads = slice(h * group, (h + 1) * group)
            o_ref, lse_ref, smax = o.prefill_attention(
                qd[rows, heads], pos, ref.pi, ref.ck, qk.codes, qk.norm, ref.cv, qv.codes, qv.norm, 1 / math.sqrt(D),
                s_matrix=ref.s if qjl else None, qjl_signs=qk.qjl_signs if qjl else None,
                qjl_gamma=qk.qjl_gamma if qjl else None)
            ok, w = ph.attention_ok(out[rows, heads], o_ref, lse[rows, heads], lse_ref, smax)
            worst = max(worst, w)
            assert ok, (s, h, w)
    return worst


@pytest.mark.parametrize("bits_k,bits_v,qjl", SETTINGS)
@pytest.mark.parametrize("n_tok", [1, 127, 128, 129])
def test_prefill_whole_prompt(tq, n_tok, bits_k, bits_v, qjl):
    _prefill_and_compare(tq, [n_tok], [n_tok], 2, 4, bits_k, bits_v, qjl, seed=n_tok + 3)


@pytest.mark.parametrize("bits_k,bits_v,qjl", [(3, 3, 0), (2, 4, 1)])
def test_prefill_4096_tokens(tq, bits_k, bits_v, qjl):
    _prefill_and_compare(tq, [4096], [4096], 2, 4, bits_k, bits_v, qjl, seed=41, sample=96)


@pytest.mark.parametrize("group", [1, 7, 8, 16])
def test_prefill_query_groups(tq, group):
    _prefill_and_compare(tq, [300, 65], [300, 65], 2, group, 3, 3, 0, seed=group)


@pytest.mark.parametrize("bits_k,bits_v,qjl", [(3, 3, 0), (4, 2, 1)])
def test_prefill_chunks_and_ragged_batch(tq, bits_k, bits_v, qjl):
    """Chunks whose earlier tokens are already cached, a sequence without
    queries, and a whole prompt, in one call."""
    _prefill_and_compare(tq, [1000, 513, 77, 200], [37, 0, 77, 200], 2, 4, bits_k, bits_v, qjl, seed=9)


def test_prefill_bf16_queries_and_paged_cache(tq):
    _prefill_and_compare(tq, [700, 250], [700, 130], 2, 8, 3, 3, 0, seed=12, q_dtype=torch.bfloat16,
                         paged_block=128)


def test_prefill_after_gpu_quantize_matches_decode_of_the_last_token(tq):
    """The whole path on the GPU: quantize a 900-token prompt, attend over it
    with tq_prefill_attention; the last query equals tq_decode_attention of
    that query over the full length (the same computation), and every query
    matches the oracle on the codes the GPU wrote."""
    n, n_heads, group = 900, 2, 4
    ctx = tq.Context(D, 3, 3, 1, 42)
    k = make_rows(n, n_heads, 71).cuda()
    v = make_rows(n, n_heads, 72).cuda()
    cache = tq.Cache(ctx, 1, n_heads, 960)
    pos = torch.arange(n, dtype=torch.int32, device="cuda")
    tq.quantize(ctx, cache, k, v, torch.zeros(n, dtype=torch.int32, device="cuda"), pos)
    q = torch.randn(n, n_heads * group, D, generator=torch.Generator().manual_seed(3)).cuda()
    out = torch.empty(n, n_heads * group, D, device="cuda")
    lse = torch.empty(n, n_heads * group, device="cuda")
    lens = torch.tensor([n], dtype=torch.int32, device="cuda")
    tq.prefill_attention(ctx, cache, q, torch.tensor([0, n], dtype=torch.int32, device="cuda"), lens, n, n, out, lse)
    dec = torch.empty(1, n_heads * group, D, device="cuda")
    dlse = torch.empty(1, n_heads * group, device="cuda")
    ws = tq.alloc_workspace(ctx, 1, n_heads * group, n)
    tq.decode_attention(ctx, cache, q[n - 1:].contiguous(), lens, n, dec, dlse, ws)
    ctx.check_device_errors()
    ok, w = ph.attention_ok(out[n - 1].cpu().numpy(), dec[0].cpu().numpy())
    assert ok, w
    ref = oracle_params(3, 3, 1)
    planes = {name: t.cpu().numpy() for name, t in cache.planes.items() if t is not None}
    fp16 = ph.f16_bits_to_f64
    sel = np.array([0, 1, 63, 64, 500, n - 1])
    for h in range(n_heads):
        heads = slice(h * group, (h + 1) * group)
        o_ref, lse_ref, smax = o.prefill_attention(
            q[sel, heads].double().cpu().numpy(), sel, ref.pi,
            ref.ck, o.unpack_codes(planes["codes_k"][0, h, :n], 3, D), fp16(planes["norm_k"][0, h, :n]),
            ref.cv, o.unpack_codes(planes["codes_v"][0, h, :n], 3, D), fp16(planes["norm_v"][0, h, :n]),
            1 / math.sqrt(D), s_matrix=ref.s, qjl_signs=o.unpack_signs(planes["qjl_bits"][0, h, :n], D),
            qjl_gamma=fp16(planes["qjl_norm"][0, h, :n]))
        ok, w = ph.attention_ok(out[sel, heads].cpu().numpy(), o_ref, lse[sel, heads].cpu().numpy(), lse_ref, smax)
        assert ok, (h, w)


def test_prefill_flags_more_queries_than_tokens(tq):
    ctx = tq.Context(D, 3, 3, 0, 42)
    cache = tq.Cache(ctx, 1, 1, 128)
    q = torch.randn(20, 1, D, device="cuda")
    out = torch.zeros(20, 1, D, device="cuda")
    tq.prefill_attention(ctx, cache, q, torch.tensor([0, 20], dtype=torch.int32, device="cuda"),
                         torch.tensor([10], dtype=torch.int32, device="cuda"), 20, 128, out)
    with pytest.raises(tq.TQError) as ei:
        ctx.check_device_errors()
    assert ei.value.status == tq.TQ_ERR_DEVICE
    with pytest.raises(tq.TQError) as ei:            # max_q above max_seq_len
        tq.prefill_attention(ctx, cache, q, torch.tensor([0, 20], dtype=torch.int32, device="cuda"),
                             torch.tensor([20], dtype=torch.int32, device="cuda"), 200, 128, out)
    assert ei.value.status == tq.TQ_ERR_INVALID
