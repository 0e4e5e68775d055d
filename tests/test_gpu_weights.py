"""GPU parity of the weight-quantization reuse (tq_weight_quantize /
tq_weight_gemm) against the oracle's weight_quantize / weight_gemm: codes
bit-exact outside the 1e-5 window and fp16 norms within one ulp for every
block of every row, and y = x W~^T within 1e-3 of max |y_ref| per token
(the same relative bar as the attention outputs), at 2, 3 and 4 bits, bf16
and fp32 inputs, ragged row counts and token counts across the 16-token
groups, and the product also checked on the codes the GPU wrote."""
import numpy as np
import pytest
import torch

from oracle import turboquant_oracle as o
from tests import parity_helpers as ph

pytestmark = pytest.mark.gpu
D = 128


@pytest.fixture(scope="module")
def tq(cuda_device):
    from kv_cache_vector_12_b200 import tq as tqmod
    return tqmod


def _weights(n_out, n_in, seed):
    g = torch.Generator().manual_seed(seed)
    w = torch.randn(n_out, n_in, generator=g) * torch.exp(0.5 * torch.randn(n_out, 1, generator=g))
    return w.to(torch.bfloat16)


@pytest.mark.parametrize("bits", [2, 3, 4])
@pytest.mark.parametrize("n_out,n_in,n_tok", [(64, 128, 1), (200, 512, 5), (1100, 1024, 17), (4096, 2048, 3)])
def test_weight_quantize_and_gemm(tq, bits, n_out, n_in, n_tok):
    ctx = tq.Context(D, bits, bits, 0, 42)
    p = o.Params(D, bits, bits, False, 42)
    w = _weights(n_out, n_in, n_out + bits)
    wc = tq.WeightCache(ctx, n_out, n_in)
    tq.weight_quantize(ctx, wc, w.cuda())
    ctx.check_device_errors()
    ref = o.weight_quantize(w.double().numpy(), D, p.pi, p.ck, p.tk)
    nb = n_in // D
    codes = wc.codes[:, :n_out].cpu().numpy()                     # [nb, n_out, bytes]
    norms = wc.norms[:, :n_out].cpu().numpy()
    for b in range(nb):
        blk = o.Quantized(ref.codes[:, b], ref.norm[:, b], ref.y[:, b])
        cc = ph.compare_codes(codes[b], blk, bits, p.tk)
        assert cc["outside_window"] == 0, (b, cc)
        assert ph.compare_fp16(norms[b], blk.norm)["worse"] == 0
    g = torch.Generator().manual_seed(7)
    for x_dtype in (torch.float32, torch.bfloat16):
        x = torch.randn(n_tok, n_in, generator=g).to(x_dtype)
        y = torch.full((n_tok, n_out), float("nan"), device="cuda")
        ws = torch.empty(max(256, tq.weight_workspace_bytes(ctx, n_tok, n_in)), dtype=torch.uint8, device="cuda")
        tq.weight_gemm(ctx, wc, x.cuda(), y, ws)
        ctx.check_device_errors()
        # the oracle's product on the codes the GPU wrote
        gcodes = np.stack([o.unpack_codes(codes[b], bits, D) for b in range(nb)], axis=1)   # [n_out, nb, D]
        gnorm = ph.f16_bits_to_f64(norms.T)                                                # [n_out, nb]
        y_ref = o.weight_gemm(x.double().numpy(), p.pi, p.ck, gcodes, gnorm)
        err = np.abs(y.cpu().double().numpy() - y_ref).max(axis=1)
        assert np.all(err <= 1e-3 * np.abs(y_ref).max(axis=1)), (x_dtype, err.max())


def test_weight_gemm_repeated_calls_and_zero_rows(tq):
    """y is overwritten, not accumulated, by each call; zero rows give zero."""
    n_out, n_in = 300, 256
    ctx = tq.Context(D, 3, 3, 1, 42)                               # a QJL context: weights ignore QJL
    w = _weights(n_out, n_in, 1)
    w[17] = 0
    wc = tq.WeightCache(ctx, n_out, n_in)
    tq.weight_quantize(ctx, wc, w.cuda())
    x = torch.randn(4, n_in, device="cuda")
    y1 = torch.empty(4, n_out, device="cuda")
    y2 = torch.empty(4, n_out, device="cuda")
    ws = torch.empty(tq.weight_workspace_bytes(ctx, 4, n_in), dtype=torch.uint8, device="cuda")
    tq.weight_gemm(ctx, wc, x, y1, ws)
    tq.weight_gemm(ctx, wc, x, y2, ws)
    ctx.check_device_errors()
    assert torch.allclose(y1, y2, rtol=1e-6, atol=1e-6)
    assert torch.all(y1[:, 17] == 0)
    # the product approximates the bf16 product (3-bit rows: a few % error)
    rel = (y1 - x @ w.cuda().float().T).norm() / (x @ w.cuda().float().T).norm()
    assert rel < 0.25


def test_weight_arguments_are_checked(tq):
    ctx = tq.Context(D, 3, 3, 0, 42)
    wc = tq.WeightCache(ctx, 64, 256)
    wc.n_in = 200                                                # not a multiple of d: rejected before any launch
    with pytest.raises(tq.TQError) as ei:
        tq.weight_quantize(ctx, wc, torch.zeros(64, 200, dtype=torch.bfloat16, device="cuda"))
    assert ei.value.status == tq.TQ_ERR_INVALID
    wc.n_in = 256
    ws = torch.empty(16, dtype=torch.uint8, device="cuda")
    with pytest.raises(tq.TQError) as ei:
        tq.weight_gemm(ctx, wc, torch.zeros(2, 256, device="cuda"), torch.zeros(2, 64, device="cuda"), ws)
    assert ei.value.status == tq.TQ_ERR_INVALID
