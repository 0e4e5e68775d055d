"""The seeded input recipes of the five workloads (CPU): shapes, sizes and
value distributions as the workload configurations state them, and
reproducibility from the seed."""
import math

import torch

from kv_cache_vector_12_b200 import workloads as wl

W = wl.WORKLOADS


def test_shapes_and_settings():
    assert (W["tiny"].n_kv_heads, W["tiny"].n_q_heads, W["tiny"].seq_len) == (1, 1, 1024)
    assert (W["llama8b"].n_kv_heads, W["llama8b"].n_q_heads, W["llama8b"].seq_len, W["llama8b"].n_seqs) == \
        (8, 32, 32768, 1)
    assert (W["qwen"].n_kv_heads, W["qwen"].n_q_heads, W["qwen"].seq_len) == (4, 28, 16384)
    assert set(W["qwen"].settings) == {(4, 2, False), (4, 4, False), (2, 2, True), (2, 4, True)}
    assert (W["llama70b"].n_kv_heads, W["llama70b"].n_q_heads, W["llama70b"].seq_len, W["llama70b"].n_seqs) == \
        (8, 64, 131072, 4)
    assert (W["serving"].n_kv_heads, W["serving"].n_q_heads, W["serving"].n_seqs) == (8, 32, 32)
    assert {(b, b, q) for b in (2, 3, 4) for q in (False, True)} == set(W["serving"].settings)
    for w in W.values():
        assert w.d == 128 and w.n_q_heads % w.n_kv_heads == 0


def test_llama8b_rows_have_lognormal_scales():
    """x ~ N(0, I) times LogNormal(0, 0.5) per (token, head): log ||x|| has
    standard deviation 0.5 (plus about 1/sqrt(2d) from the chi factor)."""
    w = W["llama8b"]
    k, v = wl.kv_tokens(w, 4096, wl.generator("cpu", 5), "cpu")
    assert k.shape == (4096, 8, 128) and k.dtype == torch.bfloat16
    for x in (k, v):
        ln = torch.log(torch.linalg.vector_norm(x.float(), dim=-1))
        sd = ln.std().item()
        assert abs(sd - math.sqrt(0.25 + 1 / 256)) < 0.02, sd
        assert abs(ln.mean().item() - math.log(math.sqrt(128))) < 0.03


def test_qwen_norms_and_directions():
    w = W["qwen"]
    k, v = wl.kv_tokens(w, 4096, wl.generator("cpu", 6), "cpu")
    kn = torch.linalg.vector_norm(k.float(), dim=-1)
    vn = torch.linalg.vector_norm(v.float(), dim=-1)
    # uniform on [172, 778] and [2, 4] (bf16 rounding moves a norm by < 0.4 %)
    assert kn.min() > 172 * 0.996 and kn.max() < 778 * 1.004 and abs(kn.mean().item() - 475) < 8
    assert vn.min() > 2 * 0.996 and vn.max() < 4 * 1.004 and abs(vn.mean().item() - 3) < 0.05
    q = wl.queries(w, 64, wl.generator("cpu", 7), "cpu")
    assert q.shape == (64, 28, 128)
    assert torch.allclose(torch.linalg.vector_norm(q.float(), dim=-1), torch.ones(64, 28), atol=0.01)


def test_llama70b_outlier_channels():
    w = W["llama70b"]
    m = wl.outlier_scale(w, "cpu", w.seed)
    assert m.shape == (8, 128)
    assert int((m == 20).sum()) == round(0.01 * 8 * 128) == 10 and int((m == 1).sum()) == 8 * 128 - 10
    assert torch.equal(m, wl.outlier_scale(w, "cpu", w.seed))        # seeded
    k, _ = wl.kv_tokens(w, 2048, wl.generator("cpu", 8), "cpu", outlier_mask=m)
    rms = k.float().pow(2).mean(dim=0).sqrt()                           # per (head, channel)
    assert torch.all(rms[m == 20] > 15) and torch.all(rms[m == 1] < 1.3)


def test_serving_lengths():
    w = W["serving"]
    lens = wl.serving_lengths(w, w.seed)
    assert len(lens) == 32 and all(1024 <= n <= 65536 for n in lens)
    assert lens == wl.serving_lengths(w, w.seed)                        # seeded
    assert len(set(lens)) > 28                                          # spread, not constant


def test_generators_are_reproducible():
    w = W["llama8b"]
    a = wl.kv_tokens(w, 64, wl.generator("cpu", 11), "cpu")[0]
    b = wl.kv_tokens(w, 64, wl.generator("cpu", 11), "cpu")[0]
    c = wl.kv_tokens(w, 64, wl.generator("cpu", 12), "cpu")[0]
    assert torch.equal(a, b) and not torch.equal(a, c)
