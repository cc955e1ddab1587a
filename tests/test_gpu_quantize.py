"""GPU parity of tq_quantize against the oracle encoder: codes and sign bits
bit-exact except decisions within 1e-6 of a boundary (counted), norms exact
except fp16 rounding ties, tail of the last tile zero-filled."""
import numpy as np
import pytest
import torch

import vector_quantization_randomized_b200 as tq
import workloads as wl
from gpu_util import make_pair, gpu_quantize, compare_codes

pytestmark = pytest.mark.gpu


def _run(d, bits, mode, x, dtype, m=None, ld=None):
    p, op = make_pair(d, bits, mode, m)
    xt = torch.from_numpy(x).to(dtype)
    if ld is not None:
        big = torch.zeros((x.shape[0], ld), dtype=dtype)
        big[:, :d] = xt
        xt = big
    xt = xt.cuda()
    codes, norms, rn = gpu_quantize(p, xt)
    xin = xt[:, :d].float().cpu().numpy().astype(np.float64)   # the exact values the kernel read
    return compare_codes(op, xin, codes, norms, rn)


def test_single_head_fp32_keys_b4():
    # 4096 fp32 keys, d = 128, per-channel lognormal scales, 4 outliers x20, seed 0; b = 4, m = 128
    x = wl.head_vectors(4096, 128, seed=wl.SEED_KEYS, token_scale=False)
    r = _run(128, 4, tq.TQ_MODE_PROD, x, torch.float32)
    assert r["idx_mismatch"] <= r["idx_flagged"]


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_bf16_prod_ragged(bits):
    x = wl.to_bf16(wl.head_vectors(1000, 128, seed=3))
    _run(128, bits, tq.TQ_MODE_PROD, x, torch.bfloat16)


@pytest.mark.parametrize("bits", [1, 2, 3, 4])
def test_bf16_mse(bits):
    x = wl.to_bf16(wl.head_vectors(777, 128, seed=4))
    _run(128, bits, tq.TQ_MODE_MSE, x, torch.bfloat16)


@pytest.mark.parametrize("bits", [2, 4])
def test_padded_dim_200(bits):
    x = wl.to_bf16(wl.search_set(2000, 200, seed=5))
    _run(200, bits, tq.TQ_MODE_PROD, x, torch.bfloat16)


def test_fp16_small_m_and_stride():
    x = wl.head_vectors(70, 128, seed=6).astype(np.float16).astype(np.float32)
    _run(128, 3, tq.TQ_MODE_PROD, x, torch.float16, m=64, ld=136)


@pytest.mark.parametrize("n", [1, 31, 32, 33])
def test_edge_sizes_and_zero_vectors(n):
    x = wl.to_bf16(wl.head_vectors(n, 128, seed=7))
    x[0] = 0.0          # zero vector
    if n > 2:
        x[2] = 0.0
    _run(128, 4, tq.TQ_MODE_PROD, x, torch.bfloat16)


def test_short_dim_zero_padding():
    x = wl.to_bf16(wl.head_vectors(300, 64, seed=8))
    _run(64, 3, tq.TQ_MODE_PROD, x, torch.bfloat16)


def test_fp16_prod_full_m_and_stride():
    # fp16 input with a row stride of 136 elements (272 bytes) at m = 128
    x = wl.head_vectors(500, 128, seed=9).astype(np.float16).astype(np.float32)
    _run(128, 4, tq.TQ_MODE_PROD, x, torch.float16, ld=136)


@pytest.mark.parametrize("bits,mode", [(3, tq.TQ_MODE_PROD), (4, tq.TQ_MODE_MSE), (2, tq.TQ_MODE_PROD)])
def test_many_tiles_per_cta(bits, mode):
    # 148 * 128 * 5 + 77 vectors: every CTA of a one-per-SM grid takes five or six
    # tiles of 128, so the input ring and both accumulator buffers wrap several times
    n = 148 * 128 * 5 + 77
    x = wl.to_bf16(wl.head_vectors(n, 128, seed=10))
    _run(128, bits, mode, x, torch.bfloat16)


@pytest.mark.parametrize("bits", [1, 2, 3, 4])
def test_bf16_mse_token_sliced(bits):
    # value-cache layout: per tile and plane, one 32-bit word per coordinate over the tile's vectors
    from gpu_util import compare_codes_sliced
    x = wl.to_bf16(wl.head_vectors(1001, 128, seed=11))
    p, op = make_pair(128, bits, tq.TQ_MODE_MSE, layout=tq.TQ_LAYOUT_SLICED)
    xt = torch.from_numpy(x).to(torch.bfloat16).cuda()
    codes, norms, _ = gpu_quantize(p, xt)
    compare_codes_sliced(op, x.astype(np.float64), codes, norms)
    # the same indices as the canonical layout, and the same reconstruction
    p2, _ = make_pair(128, bits, tq.TQ_MODE_MSE)
    codes2, norms2, _ = gpu_quantize(p2, xt)
    from oracle import codec
    assert np.array_equal(codec.unpack_sliced(codes, 1001, 128, p.kb), codec.unpack(codes2, 1001, 128, p.kb, 0)[0])
    outs = []
    for pp, cc, nn in ((p, codes, norms), (p2, codes2, norms2)):
        out = torch.zeros((1001, 128), device="cuda")
        tq.tq_dequantize(pp, torch.from_numpy(cc).cuda(), torch.from_numpy(nn.view(np.int16)).cuda(), None, 1001, out)
        outs.append(out.cpu().numpy())
    assert np.array_equal(outs[0], outs[1])


def test_token_sliced_unsupported_shapes():
    p, _ = make_pair(128, 3, tq.TQ_MODE_MSE, layout=tq.TQ_LAYOUT_SLICED)
    x = torch.zeros((64, 128), dtype=torch.float32, device="cuda")     # fp32 input: not on the sliced path
    c = torch.zeros(p.code_bytes(64), dtype=torch.uint8, device="cuda")
    nn = torch.zeros(64, dtype=torch.int16, device="cuda")
    with pytest.raises(tq.TQError):
        tq.tq_quantize(p, x, c, nn)
    q = torch.zeros((4, 128), device="cuda")
    out = torch.zeros((4, 64), device="cuda")
    ws = torch.zeros(1 << 20, dtype=torch.uint8, device="cuda")
    with pytest.raises(tq.TQError):                                     # logits read canonical planes only
        tq.tq_logits(p, q, 4, c, nn, None, 64, 1, out, ws)
