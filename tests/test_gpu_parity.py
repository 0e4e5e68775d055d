"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle on the
same seeded inputs, at sizes that span several tiles and a ragged tail."""
import math

import numpy as np
import pytest
import torch

from oracle import turboquant_oracle as o
from tests import parity_helpers as ph

pytestmark = pytest.mark.gpu

D = 128
SETTINGS = [(3, 3, 0), (2, 2, 0), (4, 4, 0), (2, 4, 1), (4, 2, 1), (3, 3, 1)]


@pytest.fixture(scope="module")
def tq(cuda_device):
    from kv_cache_vector_12_b200 import tq as tqmod
    return tqmod


_PARAMS = {}


def oracle_params(bits_k, bits_v, qjl, seed=42, law=o.LAW_GAUSSIAN):
    key = (bits_k, bits_v, qjl, seed, law)
    if key not in _PARAMS:
        _PARAMS[key] = o.Params(D, bits_k, bits_v, bool(qjl), seed, law)
    return _PARAMS[key]


def make_rows(n, h, seed, lognormal=True):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(n, h, D, generator=g)
    if lognormal:
        x = x * torch.exp(0.5 * torch.randn(n, h, 1, generator=g))
    return x.to(torch.bfloat16)


@pytest.mark.parametrize("bits_k,bits_v,qjl", SETTINGS)
def test_device_params_match_oracle(tq, bits_k, bits_v, qjl):
    ctx = tq.Context(D, bits_k, bits_v, qjl, 42)
    p = ctx.params()
    ref = oracle_params(bits_k, bits_v, qjl)
    assert np.array_equal(p["pi"].double().numpy(), ref.pi)
    assert np.array_equal(p["centroids_k"].double().numpy(), ref.ck)
    assert np.array_equal(p["thresholds_v"].double().numpy(), ref.tv)
    if qjl:
        assert np.array_equal(p["s"].double().numpy(), ref.s)


def _quantize_and_compare(tq, n_tok, n_heads, bits_k, bits_v, qjl, seed, n_seqs=2, zero_rows=0, scaled_rows=(),
                          law=o.LAW_GAUSSIAN, paged_block=0):
    """scaled_rows: (first token, last token, exponent) ranges whose rows are
    multiplied by 2^exponent (exact in bf16)."""
    ctx = tq.Context(D, bits_k, bits_v, qjl, 42, law=law)
    ref = oracle_params(bits_k, bits_v, qjl, law=law)
    k = make_rows(n_tok, n_heads, seed)
    v = make_rows(n_tok, n_heads, seed + 1)
    if zero_rows:
        k[:zero_rows] = 0
        v[:zero_rows] = 0
    for t0, t1, e in scaled_rows:
        k[t0:t1] *= 2.0 ** e
        v[t0:t1] *= 2.0 ** e
    g = torch.Generator().manual_seed(seed + 2)
    seq_idx = torch.randint(0, n_seqs, (n_tok,), generator=g, dtype=torch.int32)
    pos = torch.empty(n_tok, dtype=torch.int32)
    for s in range(n_seqs):  # distinct positions per sequence, in shuffled order
        sel = (seq_idx == s).nonzero().flatten()
        pos[sel] = torch.randperm(len(sel), generator=g).to(torch.int32) + 3
    cap = int(math.ceil((n_tok + 3 + 1) / 64) * 64)
    if paged_block:
        cap = int(math.ceil(cap / paged_block) * paged_block)
        table, n_blocks = _block_table(n_seqs, cap // paged_block, seed)
        cache = tq.PagedCache(ctx, n_seqs, n_heads, cap, paged_block, n_blocks=n_blocks, block_table=table)
    else:
        cache = tq.Cache(ctx, n_seqs, n_heads, cap)
    dev = "cuda"
    tq.quantize(ctx, cache, k.to(dev), v.to(dev), seq_idx.to(dev), pos.to(dev))
    ctx.check_device_errors()
    planes = {n: (t.cpu().numpy() if t is not None else None) for n, t in cache.planes.items()}
    if paged_block:
        planes = _to_logical(planes, table, paged_block)
    si, ps = seq_idx.numpy(), pos.numpy()
    written = np.zeros((n_seqs, n_heads, cap), dtype=bool)
    for t in range(n_tok):
        written[si[t], :, ps[t]] = True
    for name, arr in planes.items():   # untouched slots stay zero
        if arr is not None:
            assert not np.any(arr[~written]), name

    def rows(name):
        return np.stack([planes[name][si[t], h, ps[t]] for t in range(n_tok) for h in range(n_heads)])

    stats = {}
    for which, x, c, t, bits in (("k", k, ref.ck, ref.tk, bits_k), ("v", v, ref.cv, ref.tv, bits_v)):
        xr = x.double().numpy().reshape(-1, D)
        qz = o.quantize(xr, ref.pi, c, t, s_matrix=ref.s if (qjl and which == "k") else None)
        cc = ph.compare_codes(rows("codes_" + which), qz, bits, t)
        assert cc["outside_window"] == 0, cc
        nn = ph.compare_fp16(rows("norm_" + which), qz.norm)
        assert nn["worse"] == 0, nn
        stats[which] = cc
        if qjl and which == "k":
            sc = ph.compare_signs(rows("qjl_bits"), qz, skip_vectors=cc["vec_mismatch"])
            assert sc["outside_window"] == 0, sc
            gg = ph.compare_fp16(rows("qjl_norm"), qz.qjl_gamma)
            assert gg["worse"] == 0, gg
    return stats


@pytest.mark.parametrize("bits_k,bits_v,qjl", SETTINGS)
@pytest.mark.parametrize("n_tok,n_heads", [(1, 1), (7, 3), (127, 1), (128, 2), (129, 1), (1000, 8), (1031, 3)])
def test_quantize_parity(tq, n_tok, n_heads, bits_k, bits_v, qjl):
    # up to 1024 rows per matrix: the one-CTA-per-row kernel; above: the
    # tcgen05 tile kernel, and the tiled QJL kernel for K with QJL (1031 x 3
    # rows leave a partial last tile in both)
    _quantize_and_compare(tq, n_tok, n_heads, bits_k, bits_v, qjl, seed=n_tok * 31 + n_heads)


@pytest.mark.parametrize("n_tok", [40, 700])   # row kernel; tile kernels
def test_quantize_zero_vectors(tq, n_tok):
    _quantize_and_compare(tq, n_tok, 2, 3, 3, 1, seed=5, zero_rows=9)


@pytest.mark.parametrize("n_tok,bits,qjl", [(40, 3, 1), (700, 3, 1), (700, 2, 0), (700, 4, 0)])
def test_quantize_tiny_and_small_norms(tq, n_tok, bits, qjl):
    """Rows scaled by 2^-32 (stored fp16 norm 0: the zero vector) and by 2^-20
    (fp16 subnormal norm: ordinary codes) through the row kernel (40 tokens)
    and the tile kernels (700 tokens x 2 heads)."""
    _quantize_and_compare(tq, n_tok, 2, bits, bits, qjl, seed=13, scaled_rows=((3, 9, -32), (9, 15, -20)))


def test_quantize_mismatch_rate_at_scale(tq):
    total = mism = 0
    for bits in (2, 3, 4):
        st = _quantize_and_compare(tq, 4096, 8, bits, bits, 0, seed=77 + bits, n_seqs=1)
        for s in st.values():
            total += s["n"]
            mism += s["mismatch"]
    assert mism / total <= ph.MAX_MISMATCH_RATE, (mism, total)


def test_quantize_out_of_range_tokens_are_flagged_not_written(tq):
    ctx = tq.Context(D, 3, 3, 0, 42)
    cache = tq.Cache(ctx, 1, 2, 64)
    k = make_rows(3, 2, 1).cuda()
    seq_idx = torch.tensor([0, 1, 0], dtype=torch.int32, device="cuda")   # seq 1 does not exist
    pos = torch.tensor([0, 0, 64], dtype=torch.int32, device="cuda")      # pos 64 >= capacity
    tq.quantize(ctx, cache, k, k, seq_idx, pos)
    with pytest.raises(tq.TQError) as ei:
        ctx.check_device_errors()
    assert ei.value.status == tq.TQ_ERR_DEVICE
    assert int(cache.planes["norm_k"][0, :, 0].ne(0).sum()) == 2      # the valid token landed
    assert int(cache.planes["norm_k"][0, :, 1:].ne(0).sum()) == 0
    ctx.check_device_errors()                                          # flags were cleared


@pytest.mark.parametrize("qjl", [0, 1])
def test_quantize_tile_kernels_flag_out_of_range_tokens(tq, qjl):
    """Batches above the row kernel's limit: tokens with a bad sequence or
    position are flagged and skipped, every other token lands."""
    ctx = tq.Context(D, 3, 3, qjl, 42)
    n_tok, n_heads = 600, 2                                            # 1200 rows per matrix
    cache = tq.Cache(ctx, 2, n_heads, 640)
    k = make_rows(n_tok, n_heads, 11).cuda()
    seq_idx = torch.zeros(n_tok, dtype=torch.int32)
    pos = torch.arange(n_tok, dtype=torch.int32)
    seq_idx[5], pos[17], pos[599] = 2, 640, -1                         # no sequence 2; pos outside [0, 640)
    tq.quantize(ctx, cache, k, k, seq_idx.cuda(), pos.cuda())
    with pytest.raises(tq.TQError) as ei:
        ctx.check_device_errors()
    assert ei.value.status == tq.TQ_ERR_DEVICE
    landed = cache.planes["norm_k"][0].ne(0).cpu()
    expect = torch.zeros(n_heads, 640, dtype=torch.bool)
    good = [t for t in range(n_tok) if t not in (5, 17, 599)]
    expect[:, torch.tensor(good)] = True
    assert torch.equal(landed, expect)
    assert int(cache.planes["norm_v"][1].ne(0).sum()) == 0
    if qjl:
        assert torch.equal(cache.planes["qjl_norm"][0].ne(0).cpu(), expect)


# ------------------------------------------------------------------ decode
def _oracle_cache(ref, lens, n_heads, bits_k, bits_v, qjl, seed, kind="lognormal", min_cap=0):
    """Quantize seeded K/V with the oracle; returns per-(seq, head) fields and
    the packed planes laid out like the device cache."""
    n_seqs = len(lens)
    cap = max(64, int(math.ceil(max(max(lens), min_cap) / 64) * 64))
    per = {}
    planes = {
        "codes_k": np.zeros((n_seqs, n_heads, cap, D * bits_k // 8), np.uint8),
        "norm_k": np.zeros((n_seqs, n_heads, cap), np.uint16),
        "codes_v": np.zeros((n_seqs, n_heads, cap, D * bits_v // 8), np.uint8),
        "norm_v": np.zeros((n_seqs, n_heads, cap), np.uint16),
        "qjl_bits": np.zeros((n_seqs, n_heads, cap, D // 8), np.uint8) if qjl else None,
        "qjl_norm": np.zeros((n_seqs, n_heads, cap), np.uint16) if qjl else None,
    }
    for s, n in enumerate(lens):
        if n == 0:
            continue
        k = make_rows(n, n_heads, seed + 10 * s, lognormal=(kind == "lognormal")).double().numpy()
        v = make_rows(n, n_heads, seed + 10 * s + 1, lognormal=False).double().numpy()
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
    return per, planes, cap


def _block_table(n_seqs, per_seq, seed, spare=3):
    """A shuffled block table: the sequences' logical blocks spread over
    n_seqs * per_seq + spare physical blocks in a seeded random order."""
    g = torch.Generator().manual_seed(seed)
    n_blocks = n_seqs * per_seq + spare
    return torch.randperm(n_blocks, generator=g)[:n_seqs * per_seq].to(torch.int32).view(n_seqs, per_seq), n_blocks


def _to_logical(planes, table, block_size):
    """Gather paged planes [n_blocks][H][block_size][...] into the logical
    layout [n_seqs][H][capacity][...] through the block table."""
    table = table.cpu().numpy()
    out = {}
    for name, arr in planes.items():
        if arr is None:
            out[name] = None
            continue
        blocks = arr[table]                                  # [n_seqs][per_seq][H][bs][...]
        blocks = np.moveaxis(blocks, 2, 1)                   # [n_seqs][H][per_seq][bs][...]
        out[name] = blocks.reshape(blocks.shape[0], blocks.shape[1], -1, *blocks.shape[4:])
    return out


def _upload(tq, ctx, planes, n_seqs, n_heads, cap, paged=None):
    """paged: (block_size, seed) stores the planes in a paged cache whose
    block table is shuffled."""
    if paged is None:
        cache = tq.Cache(ctx, n_seqs, n_heads, cap)
        for name, arr in planes.items():
            if arr is not None:
                t = torch.from_numpy(arr.view(np.int16) if arr.dtype == np.uint16 else arr)
                cache.planes[name].copy_(t)
        return cache
    bs, seed = paged
    table, n_blocks = _block_table(n_seqs, cap // bs, seed)
    cache = tq.PagedCache(ctx, n_seqs, n_heads, cap, bs, n_blocks=n_blocks, block_table=table)
    tab = table.numpy()
    for name, arr in planes.items():
        if arr is None:
            continue
        a = arr.view(np.int16) if arr.dtype == np.uint16 else arr
        phys = np.zeros((n_blocks,) + (n_heads, bs) + a.shape[3:], dtype=a.dtype)
        for si in range(n_seqs):
            for j in range(cap // bs):
                phys[tab[si, j]] = a[si, :, j * bs:(j + 1) * bs]
        cache.planes[name].copy_(torch.from_numpy(phys))
    return cache


def _decode_and_compare(tq, lens, n_heads, group, bits_k, bits_v, qjl, seed, q_dtype=torch.float32,
                        scale=0.0, max_seq_len=None, law=o.LAW_GAUSSIAN, paged_block=0):
    ctx = tq.Context(D, bits_k, bits_v, qjl, 42, law=law)
    ref = oracle_params(bits_k, bits_v, qjl, law=law)
    min_cap = max(max_seq_len or 0, max(lens))
    if paged_block:  # the logical capacity is a whole number of blocks
        min_cap = int(math.ceil(max(min_cap, 1) / paged_block) * paged_block)
    per, planes, cap = _oracle_cache(ref, lens, n_heads, bits_k, bits_v, qjl, seed, min_cap=min_cap)
    cache = _upload(tq, ctx, planes, len(lens), n_heads, cap, paged=(paged_block, seed) if paged_block else None)
    n_q = n_heads * group
    g = torch.Generator().manual_seed(seed + 99)
    q = torch.randn(len(lens), n_q, D, generator=g).to(q_dtype)
    max_len = max(lens) if max_seq_len is None else max_seq_len
    out = torch.full((len(lens), n_q, D), float("nan"), device="cuda")
    lse = torch.full((len(lens), n_q), float("nan"), device="cuda")
    ws = tq.alloc_workspace(ctx, len(lens), n_q, max_len)
    seq_lens = torch.tensor(lens, dtype=torch.int32, device="cuda")
    tq.decode_attention(ctx, cache, q.cuda(), seq_lens, max_len, out, lse, ws, scale=scale)
    ctx.check_device_errors()
    out, lse = out.cpu().numpy(), lse.cpu().numpy()
    sc = scale if scale > 0 else 1 / math.sqrt(D)
    worst = 0.0
    qd = q.double().numpy()
    for s, n in enumerate(lens):
        for h in range(n_heads):
            rows = slice(h * group, (h + 1) * group)
            if n == 0:
                assert np.all(out[s, rows] == 0) and np.all(np.isneginf(lse[s, rows]))
                continue
            qk, qv = per[(s, h)]
            o_ref, lse_ref, scores = o.decode_attention(
                qd[s, rows], ref.pi, ref.ck, qk.codes, qk.norm, ref.cv, qv.codes, qv.norm, sc,
                s_matrix=ref.s if qjl else None, qjl_signs=qk.qjl_signs if qjl else None,
                qjl_gamma=qk.qjl_gamma if qjl else None)
            ok, w = ph.attention_ok(out[s, rows], o_ref, lse[s, rows], lse_ref,
                                    np.abs(scores).max(axis=1))
            worst = max(worst, w)
            assert ok, (s, h, w)
    return worst


@pytest.mark.parametrize("bits_k,bits_v,qjl", SETTINGS)
@pytest.mark.parametrize("lens,n_heads,group", [([1], 1, 1), ([7, 129], 2, 4), ([128], 1, 7),
                                                ([1000, 0, 513], 2, 8), ([2500], 1, 16)])
def test_decode_parity_on_oracle_packed_cache(tq, lens, n_heads, group, bits_k, bits_v, qjl):
    _decode_and_compare(tq, lens, n_heads, group, bits_k, bits_v, qjl, seed=sum(lens) + group)


def test_decode_bf16_queries_explicit_scale_and_loose_bound(tq):
    _decode_and_compare(tq, [300, 77], 2, 4, 3, 3, 0, seed=3, q_dtype=torch.bfloat16, scale=0.05,
                        max_seq_len=640)


# The exact-law (sphere) codebook: same kernels, different tables.
@pytest.mark.parametrize("bits_k,bits_v,qjl", [(3, 3, 0), (2, 4, 1), (4, 2, 0)])
@pytest.mark.parametrize("n_tok,n_heads", [(129, 2), (1031, 3)])
def test_quantize_parity_sphere_codebook(tq, n_tok, n_heads, bits_k, bits_v, qjl):
    _quantize_and_compare(tq, n_tok, n_heads, bits_k, bits_v, qjl, seed=n_tok * 17 + n_heads, law=o.LAW_SPHERE)


@pytest.mark.parametrize("bits_k,bits_v,qjl", [(3, 3, 0), (2, 4, 1), (4, 4, 1)])
def test_decode_parity_sphere_codebook(tq, bits_k, bits_v, qjl):
    _decode_and_compare(tq, [1000, 0, 513], 2, 8, bits_k, bits_v, qjl, seed=21, law=o.LAW_SPHERE)


def test_sphere_device_params_match_oracle(tq):
    for bits in (2, 3, 4):
        ctx = tq.Context(D, bits, bits, 0, 42, law="sphere")
        p = ctx.params()
        ref = oracle_params(bits, bits, 0, law=o.LAW_SPHERE)
        assert np.array_equal(p["centroids_k"].double().numpy(), ref.ck)
        assert np.array_equal(p["thresholds_v"].double().numpy(), ref.tv)


# The paged layout: physical blocks in shuffled order behind a block table.
@pytest.mark.parametrize("bits_k,bits_v,qjl", [(3, 3, 0), (2, 4, 1)])
@pytest.mark.parametrize("n_tok,n_heads,block", [(129, 2, 64), (1031, 3, 128), (700, 2, 192)])
def test_quantize_parity_paged(tq, n_tok, n_heads, block, bits_k, bits_v, qjl):
    _quantize_and_compare(tq, n_tok, n_heads, bits_k, bits_v, qjl, seed=n_tok + block, paged_block=block)


@pytest.mark.parametrize("bits_k,bits_v,qjl", [(3, 3, 0), (4, 2, 1)])
@pytest.mark.parametrize("lens,n_heads,group,block", [([1000, 0, 513], 2, 8, 64), ([2500, 77], 1, 4, 128),
                                                      ([20000], 1, 8, 256)])
def test_decode_parity_paged(tq, lens, n_heads, group, block, bits_k, bits_v, qjl):
    _decode_and_compare(tq, lens, n_heads, group, bits_k, bits_v, qjl, seed=sum(lens) + block, paged_block=block)


def test_paged_block_table_out_of_range_is_flagged(tq):
    """A block-table entry outside [0, n_blocks): quantize skips the token and
    decode reads block 0 instead; both set the token-range flag."""
    ctx = tq.Context(D, 3, 3, 0, 42)
    table = torch.tensor([[1, -1], [0, 5]], dtype=torch.int32)
    cache = tq.PagedCache(ctx, 2, 1, 128, 64, n_blocks=2, block_table=table)
    k = make_rows(2, 1, 3).cuda()
    tq.quantize(ctx, cache, k, k, torch.tensor([0, 1], dtype=torch.int32, device="cuda"),
                torch.tensor([70, 70], dtype=torch.int32, device="cuda"))   # logical block 1 of both: invalid
    with pytest.raises(tq.TQError):
        ctx.check_device_errors()
    assert not torch.any(cache.planes["codes_k"]) and not torch.any(cache.planes["norm_k"])
    out = torch.empty(2, 1, D, device="cuda")
    ws = tq.alloc_workspace(ctx, 2, 1, 128)
    tq.decode_attention(ctx, cache, torch.randn(2, 1, D, device="cuda"),
                        torch.tensor([100, 100], dtype=torch.int32, device="cuda"), 128, out, None, ws)
    with pytest.raises(tq.TQError):
        ctx.check_device_errors()
    assert torch.all(torch.isfinite(out))


@pytest.mark.parametrize("lens,block", [([60, 130, 1], 64), ([250, 3], 128)])
def test_decode_paged_unassigned_blocks_past_length(tq, lens, block):
    """Table entries of blocks that hold no position below a sequence's length
    are never read: an engine may leave them -1, and decode neither flags them
    nor reads through them."""
    bits_k, bits_v, qjl, n_heads, group = 3, 3, 0, 2, 4
    ctx = tq.Context(D, bits_k, bits_v, qjl, 42)
    ref = oracle_params(bits_k, bits_v, qjl)
    cap = 4 * block
    per, planes, _ = _oracle_cache(ref, lens, n_heads, bits_k, bits_v, qjl, seed=17, min_cap=cap)
    per_seq = cap // block
    table = torch.full((len(lens), per_seq), -1, dtype=torch.int32)
    n_blocks, nxt = len(lens) * per_seq, 0
    for s, n in enumerate(lens):
        for j in range((n + block - 1) // block):   # blocks holding a position below the length
            table[s, j] = nxt
            nxt += 1
    cache = tq.PagedCache(ctx, len(lens), n_heads, cap, block, n_blocks=n_blocks, block_table=table)
    tab = table.numpy()
    for name, arr in planes.items():
        if arr is None:
            continue
        a = arr.view(np.int16) if arr.dtype == np.uint16 else arr
        phys = np.zeros((n_blocks, n_heads, block) + a.shape[3:], dtype=a.dtype)
        for s in range(len(lens)):
            for j in range(per_seq):
                if tab[s, j] >= 0:
                    phys[tab[s, j]] = a[s, :, j * block:(j + 1) * block]
        cache.planes[name].copy_(torch.from_numpy(phys))
    n_q = n_heads * group
    q = torch.randn(len(lens), n_q, D, generator=torch.Generator().manual_seed(5))
    out = torch.empty(len(lens), n_q, D, device="cuda")
    lse = torch.empty(len(lens), n_q, device="cuda")
    ws = tq.alloc_workspace(ctx, len(lens), n_q, cap)
    tq.decode_attention(ctx, cache, q.cuda(), torch.tensor(lens, dtype=torch.int32, device="cuda"), cap, out, lse,
                        ws)
    ctx.check_device_errors()                       # no range flag for the -1 entries past the lengths
    out, lse = out.cpu().numpy(), lse.cpu().numpy()
    for s in range(len(lens)):
        for h in range(n_heads):
            qk, qv = per[(s, h)]
            rows = slice(h * group, (h + 1) * group)
            o_ref, lse_ref, scores = o.decode_attention(q[s, rows].double().numpy(), ref.pi, ref.ck, qk.codes,
                                                        qk.norm, ref.cv, qv.codes, qv.norm, 1 / math.sqrt(D))
            ok, w = ph.attention_ok(out[s, rows], o_ref, lse[s, rows], lse_ref, np.abs(scores).max(axis=1))
            assert ok, (s, h, w)


def test_calls_on_another_device_are_rejected(tq):
    """A context belongs to the device it was created on; compute calls made
    while another device is current return TQ_ERR_INVALID and launch nothing."""
    if torch.cuda.device_count() < 2:
        pytest.skip("needs two CUDA devices")
    ctx = tq.Context(D, 3, 3, 0, 42)
    cache = tq.Cache(ctx, 1, 1, 64)
    k = torch.zeros(1, 1, D, dtype=torch.bfloat16, device="cuda:0")
    idx = torch.zeros(1, dtype=torch.int32, device="cuda:0")
    out = torch.empty(1, 1, D, device="cuda:0")
    ws = tq.alloc_workspace(ctx, 1, 1, 64)
    with torch.cuda.device(1):
        for call in (lambda: tq.quantize(ctx, cache, k, k, idx, idx),
                     lambda: tq.decode_attention(ctx, cache, torch.zeros(1, 1, D, device="cuda:0"), idx + 1, 64,
                                                 out, None, ws),
                     lambda: tq.decode_attention_noalloc(ctx, cache, torch.zeros(1, 1, D, device="cuda:0"),
                                                         idx + 1, 64, out, None)):
            with pytest.raises(tq.TQError) as ei:
                call()
            assert ei.value.status == tq.TQ_ERR_INVALID


def test_paged_cache_argument_checks(tq):
    ctx = tq.Context(D, 3, 3, 0, 42)
    k = torch.zeros(1, 1, D, dtype=torch.bfloat16, device="cuda")
    idx = torch.zeros(1, dtype=torch.int32, device="cuda")
    for bs, cap in ((96, 192), (128, 192)):   # block size not a multiple of 64; capacity not a multiple of it
        cache = tq.PagedCache(ctx, 1, 1, cap, bs, n_blocks=4,
                              block_table=torch.zeros(1, max(1, cap // bs), dtype=torch.int32))
        with pytest.raises(tq.TQError) as ei:
            tq.quantize(ctx, cache, k, k, idx, idx)
        assert ei.value.status == tq.TQ_ERR_INVALID


def test_decode_long_sequence_many_splits(tq):
    _decode_and_compare(tq, [20000], 1, 8, 3, 3, 0, seed=11)


def test_decode_seq_len_above_bound_is_flagged(tq):
    ctx = tq.Context(D, 3, 3, 0, 42)
    cache = tq.Cache(ctx, 1, 1, 128)
    q = torch.randn(1, 1, D, device="cuda")
    out = torch.empty(1, 1, D, device="cuda")
    ws = tq.alloc_workspace(ctx, 1, 1, 64)
    tq.decode_attention(ctx, cache, q, torch.tensor([100], dtype=torch.int32, device="cuda"), 64, out, None, ws)
    with pytest.raises(tq.TQError):
        ctx.check_device_errors()


def test_decode_rejects_bad_arguments(tq):
    ctx = tq.Context(D, 3, 3, 0, 42)
    cache = tq.Cache(ctx, 1, 2, 128)
    q = torch.randn(1, 3, D, device="cuda")        # 3 query heads over 2 KV heads
    out = torch.empty(1, 3, D, device="cuda")
    ws = tq.alloc_workspace(ctx, 1, 3, 64)
    lens = torch.tensor([10], dtype=torch.int32, device="cuda")
    with pytest.raises(tq.TQError) as ei:
        tq.decode_attention(ctx, cache, q, lens, 64, out, None, ws)
    assert ei.value.status == tq.TQ_ERR_INVALID
    q = torch.randn(1, 2, D, device="cuda")
    with pytest.raises(tq.TQError):                  # max_seq_len above capacity
        tq.decode_attention(ctx, cache, q, lens, 256, out, None, ws)
    small = torch.empty(16, dtype=torch.uint8, device="cuda")
    with pytest.raises(tq.TQError):                  # workspace too small
        tq.decode_attention(ctx, cache, q, lens, 64, out, None, small)


# -------------------------------------------------------------- end to end
def test_end_to_end_tiny_against_oracle_and_exact_attention(tq):
    """GPU quantize + GPU decode vs the oracle's quantize + decode on the tiny
    workload (fp32 inputs rounded to bf16), plus the quality figure."""
    from kv_cache_vector_12_b200 import workloads as wl
    w = wl.WORKLOADS["tiny"]
    gen = wl.generator("cpu", w.seed)
    k32, v32 = wl.kv_tokens(w, w.seq_len, gen, "cpu", dtype=torch.float32)
    q32 = wl.queries(w, 1, gen, "cpu", dtype=torch.float32)
    k, v = k32.to(torch.bfloat16), v32.to(torch.bfloat16)
    ctx = tq.Context(D, w.bits_k, w.bits_v, 0, w.pi_seed)
    cache = tq.Cache(ctx, 1, 1, 1024)
    idx = torch.zeros(w.seq_len, dtype=torch.int32, device="cuda")
    pos = torch.arange(w.seq_len, dtype=torch.int32, device="cuda")
    tq.quantize(ctx, cache, k.cuda(), v.cuda(), idx, pos)
    out = torch.empty(1, 1, D, device="cuda")
    lse = torch.empty(1, 1, device="cuda")
    ws = tq.alloc_workspace(ctx, 1, 1, w.seq_len)
    tq.decode_attention(ctx, cache, q32.cuda(), torch.tensor([w.seq_len], dtype=torch.int32, device="cuda"),
                        w.seq_len, out, lse, ws)
    ctx.check_device_errors()
    ref = oracle_params(3, 3, 0)
    qk = o.quantize(k[:, 0].double().numpy(), ref.pi, ref.ck, ref.tk)
    qv = o.quantize(v[:, 0].double().numpy(), ref.pi, ref.cv, ref.tv)
    o_ref, lse_ref, scores = o.decode_attention(q32[0].double().numpy(), ref.pi, ref.ck, qk.codes, qk.norm,
                                                ref.cv, qv.codes, qv.norm, 1 / math.sqrt(D))
    ok, worst = ph.attention_ok(out[0].cpu().numpy(), o_ref, lse[0].cpu().numpy(), lse_ref,
                                np.abs(scores).max(axis=1))
    assert ok, worst
    o_exact, _ = o.exact_attention(q32[0].double().numpy(), k32[:, 0].double().numpy(),
                                   v32[:, 0].double().numpy(), 1 / math.sqrt(D))
    assert o.cosine_similarity(out[0].cpu().numpy(), o_exact) > 0.9
