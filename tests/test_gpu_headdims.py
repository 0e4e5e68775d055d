"""GPU parity at head dimensions 64 and 256 (the pages' coordinate law is
only close to Gaussian, and more so as d grows; the exact-law codebook is
the variant that matters at small d).  The same checks as at d = 128:
quantize (codes bit-exact outside the 1e-5 window, fp16 norms within one
ulp, QJL signs outside their window) and decode attention (outputs within
1e-3 ||o||_inf, lse within 1e-3 max(1, max |s|)) against the oracle, which is
generic in d, on ragged batches, several query heads per KV head, every
(bits, QJL) setting, both codebook laws and a paged cache."""
import math

import numpy as np
import pytest
import torch

from oracle import turboquant_oracle as o
from tests import parity_helpers as ph

pytestmark = pytest.mark.gpu

SETTINGS = [(3, 3, 0), (2, 2, 0), (4, 4, 0), (2, 4, 1), (4, 2, 1), (3, 3, 1)]
_PARAMS = {}


@pytest.fixture(scope="module")
def tq(cuda_device):
    from kv_cache_vector_12_b200 import tq as tqmod
    return tqmod


def params(d, bits_k, bits_v, qjl, law=o.LAW_GAUSSIAN):
    key = (d, bits_k, bits_v, qjl, law)
    if key not in _PARAMS:
        _PARAMS[key] = o.Params(d, bits_k, bits_v, bool(qjl), 42, law)
    return _PARAMS[key]


def rows(n, h, d, seed, lognormal=True):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(n, h, d, generator=g)
    if lognormal:
        x = x * torch.exp(0.5 * torch.randn(n, h, 1, generator=g))
    return x.to(torch.bfloat16)


@pytest.mark.parametrize("d", [64, 256])
@pytest.mark.parametrize("bits_k,bits_v,qjl", SETTINGS)
@pytest.mark.parametrize("n_tok", [300, 700])
def test_quantize_parity(tq, d, bits_k, bits_v, qjl, n_tok):
    """300 tokens x 2 heads: the per-row kernel; 700 x 2 (1400 rows, a ragged
    last tile of 120): the tcgen05 kernel (V, and K without QJL) and, for K
    with QJL, the batched QJL kernel (32 vectors per CTA, the last CTA 24)."""
    n_heads = 2
    k, v = rows(n_tok, n_heads, d, 5 + d), rows(n_tok, n_heads, d, 6 + d)
    _quantize_and_compare(tq, d, bits_k, bits_v, qjl, k, v)


@pytest.mark.parametrize("d", [64, 256])
@pytest.mark.parametrize("qjl", [0, 1])
def test_quantize_zero_and_tiny_vectors_in_batches(tq, d, qjl):
    """700 tokens x 2 heads (the batched kernels) with rows scaled by 2^-32
    (stored fp16 norm 0: the zero vector, whose residual is minus the centroid
    of code 2^(b-1) - 1) and by 2^-20 (a subnormal fp16 norm: ordinary
    codes), and exact zero rows."""
    n_tok, n_heads = 700, 2
    k, v = rows(n_tok, n_heads, d, 15 + d), rows(n_tok, n_heads, d, 16 + d)
    for x in (k, v):
        x[3:9] = (x[3:9].float() * 2.0 ** -32).to(torch.bfloat16)
        x[9:15] = (x[9:15].float() * 2.0 ** -20).to(torch.bfloat16)
        x[40:43] = 0
    _quantize_and_compare(tq, d, 3, 3, qjl, k, v)


def _quantize_and_compare(tq, d, bits_k, bits_v, qjl, k, v):
    n_tok, n_heads = k.shape[0], k.shape[1]
    ctx = tq.Context(d, bits_k, bits_v, qjl, 42)
    ref = params(d, bits_k, bits_v, qjl)
    cache = tq.Cache(ctx, 1, n_heads, (n_tok + 63) // 64 * 64)
    pos = torch.randperm(n_tok, generator=torch.Generator().manual_seed(d)).to(torch.int32)
    tq.quantize(ctx, cache, k.cuda(), v.cuda(), torch.zeros(n_tok, dtype=torch.int32, device="cuda"), pos.cuda())
    ctx.check_device_errors()
    pl = {n: (t.cpu().numpy() if t is not None else None) for n, t in cache.planes.items()}
    ps = pos.numpy()
    for which, x, c, t, bits in (("k", k, ref.ck, ref.tk, bits_k), ("v", v, ref.cv, ref.tv, bits_v)):
        for h in range(n_heads):
            qz = o.quantize(x[:, h].double().numpy(), ref.pi, c, t, s_matrix=ref.s if (qjl and which == "k") else None)
            cc = ph.compare_codes(pl["codes_" + which][0, h, ps], qz, bits, t, d=d)
            assert cc["outside_window"] == 0, cc
            assert ph.compare_fp16(pl["norm_" + which][0, h, ps], qz.norm)["worse"] == 0
            if qjl and which == "k":
                sc = ph.compare_signs(pl["qjl_bits"][0, h, ps], qz, skip_vectors=cc["vec_mismatch"])
                assert sc["outside_window"] == 0, sc
                assert ph.compare_fp16(pl["qjl_norm"][0, h, ps], qz.qjl_gamma)["worse"] == 0


@pytest.mark.parametrize("d", [64, 256])
@pytest.mark.parametrize("qjl", [0, 1])
def test_quantize_batches_flag_out_of_range_tokens(tq, d, qjl):
    """1200 rows per matrix (the batched kernels): tokens with a bad sequence
    or position are flagged and skipped, every other token lands."""
    ctx = tq.Context(d, 3, 3, qjl, 42)
    n_tok, n_heads = 600, 2
    cache = tq.Cache(ctx, 2, n_heads, 640)
    k = rows(n_tok, n_heads, d, 11).cuda()
    seq_idx = torch.zeros(n_tok, dtype=torch.int32)
    pos = torch.arange(n_tok, dtype=torch.int32)
    seq_idx[5], pos[17], pos[599] = 2, 640, -1                         # no sequence 2; pos outside [0, 640)
    tq.quantize(ctx, cache, k, k, seq_idx.cuda(), pos.cuda())
    with pytest.raises(tq.TQError) as ei:
        ctx.check_device_errors()
    assert ei.value.status == tq.TQ_ERR_DEVICE
    expect = torch.zeros(n_heads, 640, dtype=torch.bool)
    expect[:, torch.tensor([t for t in range(n_tok) if t not in (5, 17, 599)])] = True
    assert torch.equal(cache.planes["norm_k"][0].ne(0).cpu(), expect)
    assert torch.equal(cache.planes["norm_v"][0].ne(0).cpu(), expect)
    assert int(cache.planes["norm_k"][1].ne(0).sum()) == 0
    if qjl:
        assert torch.equal(cache.planes["qjl_norm"][0].ne(0).cpu(), expect)


@pytest.mark.parametrize("d", [64, 256])
@pytest.mark.parametrize("bits_k,bits_v,qjl", [(3, 3, 0), (2, 4, 1)])
def test_quantize_parity_many_tiles(tq, d, bits_k, bits_v, qjl):
    """20001 tokens x 4 heads (80004 rows per matrix): several tiles per
    persistent CTA, so the tile kernels' rings and barrier phases wrap, and
    the last tile is ragged (4 rows); every row is compared."""
    n_tok, n_heads = 20001, 4
    ctx = tq.Context(d, bits_k, bits_v, qjl, 42)
    ref = params(d, bits_k, bits_v, qjl)
    k, v = rows(n_tok, n_heads, d, 11 + d), rows(n_tok, n_heads, d, 12 + d)
    cache = tq.Cache(ctx, 1, n_heads, (n_tok + 63) // 64 * 64)
    pos = torch.arange(n_tok, dtype=torch.int32)
    tq.quantize(ctx, cache, k.cuda(), v.cuda(), torch.zeros(n_tok, dtype=torch.int32, device="cuda"), pos.cuda())
    ctx.check_device_errors()
    pl = {n: (t.cpu().numpy() if t is not None else None) for n, t in cache.planes.items()}
    for which, x, c, t, bits in (("k", k, ref.ck, ref.tk, bits_k), ("v", v, ref.cv, ref.tv, bits_v)):
        if qjl and which == "k":
            continue  # K with QJL runs the per-row kernel at these head dimensions (covered above)
        for h in range(n_heads):
            qz = o.quantize(x[:, h].double().numpy(), ref.pi, c, t)
            cc = ph.compare_codes(pl["codes_" + which][0, h, :n_tok], qz, bits, t, d=d)
            assert cc["outside_window"] == 0, cc
            assert ph.compare_fp16(pl["norm_" + which][0, h, :n_tok], qz.norm)["worse"] == 0


def _decode_and_compare(tq, d, lens, n_heads, group, bits_k, bits_v, qjl, seed, law=o.LAW_GAUSSIAN, paged=0,
                        q_dtype=torch.float32):
    ctx = tq.Context(d, bits_k, bits_v, qjl, 42, law=law)
    ref = params(d, bits_k, bits_v, qjl, law)
    cap = max(64, int(math.ceil(max(lens) / 64) * 64))
    if paged:
        cap = int(math.ceil(cap / paged) * paged)
    n_seqs = len(lens)
    per = {}
    planes = {"codes_k": np.zeros((n_seqs, n_heads, cap, d * bits_k // 8), np.uint8),
              "norm_k": np.zeros((n_seqs, n_heads, cap), np.uint16),
              "codes_v": np.zeros((n_seqs, n_heads, cap, d * bits_v // 8), np.uint8),
              "norm_v": np.zeros((n_seqs, n_heads, cap), np.uint16),
              "qjl_bits": np.zeros((n_seqs, n_heads, cap, d // 8), np.uint8) if qjl else None,
              "qjl_norm": np.zeros((n_seqs, n_heads, cap), np.uint16) if qjl else None}
    for s, n in enumerate(lens):
        if n == 0:
            continue
        k = rows(n, n_heads, d, seed + 10 * s).double().numpy()
        v = rows(n, n_heads, d, seed + 10 * s + 1, lognormal=False).double().numpy()
        for h in range(n_heads):
            qk = o.quantize(k[:, h], ref.pi, ref.ck, ref.tk, s_matrix=ref.s if qjl else None)
            qv = o.quantize(v[:, h], ref.pi, ref.cv, ref.tv)
            per[(s, h)] = (qk, qv)
            planes["codes_k"][s, h, :n] = o.pack_codes(qk.codes, bits_k)
            planes["codes_v"][s, h, :n] = o.pack_codes(qv.codes, bits_v)
            planes["norm_k"][s, h, :n] = qk.norm.astype(np.float16).view(np.uint16)
            planes["norm_v"][s, h, :n] = qv.norm.astype(np.float16).view(np.uint16)
            if qjl:
                planes["qjl_bits"][s, h, :n] = o.pack_signs(qk.qjl_signs)
                planes["qjl_norm"][s, h, :n] = qk.qjl_gamma.astype(np.float16).view(np.uint16)
    if paged:
        per_seq = cap // paged
        n_blocks = n_seqs * per_seq + 2
        table = torch.randperm(n_blocks, generator=torch.Generator().manual_seed(seed))[:n_seqs * per_seq]
        table = table.to(torch.int32).view(n_seqs, per_seq)
        cache = tq.PagedCache(ctx, n_seqs, n_heads, cap, paged, n_blocks=n_blocks, block_table=table)
        tab = table.numpy()
        for name, arr in planes.items():
            if arr is None:
                continue
            a = arr.view(np.int16) if arr.dtype == np.uint16 else arr
            phys = np.zeros((n_blocks, n_heads, paged) + a.shape[3:], dtype=a.dtype)
            for si in range(n_seqs):
                for j in range(per_seq):
                    phys[tab[si, j]] = a[si, :, j * paged:(j + 1) * paged]
            cache.planes[name].copy_(torch.from_numpy(phys))
    else:
        cache = tq.Cache(ctx, n_seqs, n_heads, cap)
        for name, arr in planes.items():
            if arr is not None:
                cache.planes[name].copy_(torch.from_numpy(arr.view(np.int16) if arr.dtype == np.uint16 else arr))
    n_q = n_heads * group
    q = torch.randn(n_seqs, n_q, d, generator=torch.Generator().manual_seed(seed + 99)).to(q_dtype)
    max_len = max(lens)
    out = torch.full((n_seqs, n_q, d), float("nan"), device="cuda")
    lse = torch.full((n_seqs, n_q), float("nan"), device="cuda")
    ws = tq.alloc_workspace(ctx, n_seqs, n_q, max_len)
    tq.decode_attention(ctx, cache, q.cuda(), torch.tensor(lens, dtype=torch.int32, device="cuda"), max_len, out,
                        lse, ws)
    ctx.check_device_errors()
    out, lse = out.cpu().numpy(), lse.cpu().numpy()
    qd = q.double().numpy()
    worst = 0.0
    for s, n in enumerate(lens):
        for h in range(n_heads):
            hs = slice(h * group, (h + 1) * group)
            if n == 0:
                assert np.all(out[s, hs] == 0) and np.all(np.isneginf(lse[s, hs]))
                continue
            qk, qv = per[(s, h)]
            o_ref, lse_ref, sc = o.decode_attention(
                qd[s, hs], ref.pi, ref.ck, qk.codes, qk.norm, ref.cv, qv.codes, qv.norm, 1 / math.sqrt(d),
                s_matrix=ref.s if qjl else None, qjl_signs=qk.qjl_signs if qjl else None,
                qjl_gamma=qk.qjl_gamma if qjl else None)
            ok, w = ph.attention_ok(out[s, hs], o_ref, lse[s, hs], lse_ref, np.abs(sc).max(axis=1))
            worst = max(worst, w)
            assert ok, (s, h, w)
    return worst


@pytest.mark.parametrize("d", [64, 256])
@pytest.mark.parametrize("bits_k,bits_v,qjl", SETTINGS)
@pytest.mark.parametrize("lens,n_heads,group", [([1], 1, 1), ([7, 129], 2, 4), ([1000, 0, 513], 2, 8),
                                                ([2500], 1, 16)])
def test_decode_parity(tq, d, lens, n_heads, group, bits_k, bits_v, qjl):
    _decode_and_compare(tq, d, lens, n_heads, group, bits_k, bits_v, qjl, seed=sum(lens) + group + d)


@pytest.mark.parametrize("d", [64, 256])
def test_decode_long_sequence_bf16_queries(tq, d):
    _decode_and_compare(tq, d, [20000], 1, 8, 3, 3, 0, seed=11, q_dtype=torch.bfloat16)


@pytest.mark.parametrize("d", [64, 256])
@pytest.mark.parametrize("bits_k,bits_v,qjl", [(3, 3, 0), (2, 4, 1)])
def test_decode_parity_sphere_codebook_and_paged(tq, d, bits_k, bits_v, qjl):
    _decode_and_compare(tq, d, [1000, 300], 2, 4, bits_k, bits_v, qjl, seed=3, law=o.LAW_SPHERE)
    _decode_and_compare(tq, d, [1000, 300], 2, 4, bits_k, bits_v, qjl, seed=4, paged=128)


@pytest.mark.parametrize("d", [64, 256])
def test_quantize_then_decode_end_to_end(tq, d):
    """The whole path at this head dimension on the GPU: quantize a prefill and
    an appended token, decode, compare with the oracle on the GPU's codes."""
    n, n_heads, group = 500, 2, 4
    ctx = tq.Context(d, 3, 3, 1, 42)
    ref = params(d, 3, 3, 1)
    k, v = rows(n, n_heads, d, 77).cuda(), rows(n, n_heads, d, 78).cuda()
    cache = tq.Cache(ctx, 1, n_heads, 512)
    zeros = torch.zeros(n, dtype=torch.int32, device="cuda")
    pos = torch.arange(n, dtype=torch.int32, device="cuda")
    tq.quantize(ctx, cache, k[:-1], v[:-1], zeros[:-1], pos[:-1])
    tq.quantize(ctx, cache, k[-1:], v[-1:], zeros[-1:], pos[-1:])
    q = torch.randn(1, n_heads * group, d, generator=torch.Generator().manual_seed(1)).cuda()
    out = torch.empty(1, n_heads * group, d, device="cuda")
    lse = torch.empty(1, n_heads * group, device="cuda")
    ws = tq.alloc_workspace(ctx, 1, n_heads * group, n)
    tq.decode_attention(ctx, cache, q, torch.tensor([n], dtype=torch.int32, device="cuda"), n, out, lse, ws)
    ctx.check_device_errors()
    pl = {name: t.cpu().numpy() for name, t in cache.planes.items() if t is not None}
    f16 = ph.f16_bits_to_f64
    for h in range(n_heads):
        hs = slice(h * group, (h + 1) * group)
        o_ref, lse_ref, sc = o.decode_attention(
            q[0, hs].double().cpu().numpy(), ref.pi,
            ref.ck, o.unpack_codes(pl["codes_k"][0, h, :n], 3, d), f16(pl["norm_k"][0, h, :n]),
            ref.cv, o.unpack_codes(pl["codes_v"][0, h, :n], 3, d), f16(pl["norm_v"][0, h, :n]), 1 / math.sqrt(d),
            s_matrix=ref.s, qjl_signs=o.unpack_signs(pl["qjl_bits"][0, h, :n], d),
            qjl_gamma=f16(pl["qjl_norm"][0, h, :n]))
        ok, w = ph.attention_ok(out[0, hs].cpu().numpy(), o_ref, lse[0, hs].cpu().numpy(), lse_ref,
                                np.abs(sc).max(axis=1))
        assert ok, (h, w)


def test_prefill_rejects_other_head_dims(tq):
    ctx = tq.Context(64, 3, 3, 0, 42)
    cache = tq.Cache(ctx, 1, 1, 64)
    one = torch.ones(1, dtype=torch.int32, device="cuda")
    with pytest.raises(tq.TQError) as ei:
        tq.prefill_attention(ctx, cache, torch.zeros(1, 1, 64, device="cuda"),
                             torch.tensor([0, 1], dtype=torch.int32, device="cuda"), one, 1, 1,
                             torch.zeros(1, 1, 64, device="cuda"))
    assert ei.value.status == tq.TQ_ERR_UNSUPPORTED
