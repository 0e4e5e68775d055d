"""GPU parity of the attention scores themselves, token by token.

The decode call returns the output and the log-sum-exp of the scores, not
the scores.  A sequence of length 1 has exactly one score, and its
log-sum-exp is that score.  So a batch of T one-token sequences, the token of
sequence j being token j of one longer seeded sequence and every sequence
holding the same query, yields the T scores of that query against the T
tokens: lse[j][g] = s_gj.  These are compared with the oracle's scores of the
same query over the same T cached tokens, element by element, at the bar
max_j |s_gpu - s_ref| <= 1e-3 max_j |s_ref| per query head (the reading of
"scores within 1e-3 relative error").

The workloads' value laws are used: the llama8b lognormal norms, the
Qwen-like norms of 172 to 778 (sharp softmax, large scores), and the
llama70b outlier channels scaled by 20; every (bits, QJL) setting.
"""
import math

import numpy as np
import pytest
import torch

from oracle import turboquant_oracle as o
from tests import parity_helpers as ph

pytestmark = pytest.mark.gpu

D = 128
SETTINGS = [(3, 3, 0), (2, 2, 0), (4, 4, 0), (2, 4, 1), (4, 2, 1), (3, 3, 1)]
N_TOKENS = 320


@pytest.fixture(scope="module")
def env(cuda_device):
    from kv_cache_vector_12_b200 import tq
    from kv_cache_vector_12_b200 import workloads as wl
    return tq, wl


_PARAMS = {}


def params(bits_k, bits_v, qjl):
    key = (bits_k, bits_v, qjl)
    if key not in _PARAMS:
        _PARAMS[key] = o.Params(D, bits_k, bits_v, bool(qjl), 42)
    return _PARAMS[key]


def _inputs(wl, name, n_tok, seed):
    """K, V rows [n_tok, H, d] (bf16) and one query [H_q, d] of the workload."""
    w = wl.WORKLOADS[name]
    gen = wl.generator("cpu", seed)
    outl = wl.outlier_scale(w, "cpu", w.seed) if name == "llama70b" else None
    k, v = wl.kv_tokens(w, n_tok, gen, "cpu", outlier_mask=outl)
    q = wl.queries(w, 1, gen, "cpu", dtype=torch.float32)[0]
    return w, k, v, q


@pytest.mark.parametrize("bits_k,bits_v,qjl", SETTINGS)
@pytest.mark.parametrize("name", ["llama8b", "qwen", "llama70b"])
def test_scores_token_by_token(env, name, bits_k, bits_v, qjl):
    tq, wl = env
    w, k, v, q = _inputs(wl, name, N_TOKENS, seed=7000 + 10 * bits_k + bits_v + 100 * qjl)
    H, HQ, G = w.n_kv_heads, w.n_q_heads, w.group
    ref = params(bits_k, bits_v, qjl)
    ctx = tq.Context(D, bits_k, bits_v, qjl, 42)
    # one token per sequence: sequence j holds token j at position 0
    cache = tq.Cache(ctx, N_TOKENS, H, 64)
    per_head = []
    for h in range(H):
        kq = o.quantize(k[:, h].double().numpy(), ref.pi, ref.ck, ref.tk, s_matrix=ref.s if qjl else None)
        vq = o.quantize(v[:, h].double().numpy(), ref.pi, ref.cv, ref.tv)
        per_head.append((kq, vq))
        pl = cache.planes
        pl["codes_k"][:, h, 0] = torch.from_numpy(o.pack_codes(kq.codes, bits_k)).cuda()
        pl["codes_v"][:, h, 0] = torch.from_numpy(o.pack_codes(vq.codes, bits_v)).cuda()
        pl["norm_k"][:, h, 0] = torch.from_numpy(kq.norm.astype(np.float16).view(np.int16)).cuda()
        pl["norm_v"][:, h, 0] = torch.from_numpy(vq.norm.astype(np.float16).view(np.int16)).cuda()
        if qjl:
            pl["qjl_bits"][:, h, 0] = torch.from_numpy(o.pack_signs(kq.qjl_signs)).cuda()
            pl["qjl_norm"][:, h, 0] = torch.from_numpy(kq.qjl_gamma.astype(np.float16).view(np.int16)).cuda()
    q_all = q[None].expand(N_TOKENS, HQ, D).contiguous().cuda()
    lens = torch.ones(N_TOKENS, dtype=torch.int32, device="cuda")
    out = torch.empty(N_TOKENS, HQ, D, device="cuda")
    lse = torch.full((N_TOKENS, HQ), float("nan"), device="cuda")
    ws = tq.alloc_workspace(ctx, N_TOKENS, HQ, 1)
    tq.decode_attention(ctx, cache, q_all, lens, 1, out, lse, ws)
    ctx.check_device_errors()
    s_gpu = lse.cpu().double().numpy()                      # [token j][query head]
    scale = 1 / math.sqrt(D)
    worst = 0.0
    for h in range(H):
        kq, vq = per_head[h]
        rows = slice(h * G, (h + 1) * G)
        _, _, s_ref = o.decode_attention(
            q[rows].double().numpy(), ref.pi, ref.ck, kq.codes, kq.norm, ref.cv, vq.codes, vq.norm, scale,
            s_matrix=ref.s if qjl else None, qjl_signs=kq.qjl_signs if qjl else None,
            qjl_gamma=kq.qjl_gamma if qjl else None)         # [G][token j]
        err = np.abs(s_gpu[:, rows].T - s_ref).max(axis=1)
        bound = ph.ATTN_RTOL * np.abs(s_ref).max(axis=1)
        worst = max(worst, float((err / np.abs(s_ref).max(axis=1)).max()))
        assert np.all(err <= bound), f"head {h}: per-token score error {err} above {bound}"
        # a one-token sequence attends to its token alone: o = Pi^T (||v|| c_V[codes])
        o_ref = o.dequantize(ref.pi, ref.cv, vq.codes, vq.norm)
        o_gpu = out[:, rows].cpu().double().numpy()
        ok, w_o = ph.attention_ok(o_gpu, np.repeat(o_ref[:, None, :], G, axis=1))
        assert ok, (h, w_o)
    print(f"{name} {bits_k}/{bits_v} qjl={qjl}: worst per-token score error {worst:.2e} of max |s|")
