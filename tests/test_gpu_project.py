"""GPU parity of tq_project_quantize (quantize-on-write): the projected vectors
against the oracle's bf16(x W_h^T) - equal except where the exact sum lies
within the fp32 accumulation error (2e-5 of the sum of |products|) of a bf16
rounding midpoint, and then a rounding of a value inside that band - and the codes against the oracle's encoding of those
vectors (bit-exact outside the 1e-6 decision band), plus bit identity with
tq_quantize run on the same vectors."""
import numpy as np
import pytest
import torch

import vector_quantization_randomized_b200 as tq
import workloads as wl
from oracle import project
from gpu_util import make_pair, compare_codes, gpu_quantize

pytestmark = pytest.mark.gpu


def _run(n_tok, hidden, n_heads, bits, mode, seed, with_k=True):
    p, op = make_pair(128, bits, mode)
    x, w = wl.projection_inputs(n_tok, hidden, n_heads, seed)
    xt = torch.from_numpy(x).to(torch.bfloat16).cuda()
    wt = torch.from_numpy(w).to(torch.bfloat16).cuda()
    n = n_heads * n_tok
    codes = torch.full((max(p.code_bytes(n), 16),), 0xAB, dtype=torch.uint8, device="cuda")
    norms = torch.zeros(n, dtype=torch.int16, device="cuda")
    rn = torch.zeros(n, dtype=torch.int16, device="cuda") if mode == tq.TQ_MODE_PROD else None
    k_out = torch.zeros((n_tok, n_heads * 128), dtype=torch.bfloat16, device="cuda") if with_k else None
    tq.tq_project_quantize(p, xt, wt, n_heads, codes, norms, rn, k_out)
    torch.cuda.synchronize()
    out = dict(p=p, op=op, x=x, w=w, codes=codes.cpu().numpy()[:p.code_bytes(n)],
               norms=norms.cpu().numpy().view(np.float16),
               rn=None if rn is None else rn.cpu().numpy().view(np.float16))
    if with_k:
        kk = k_out.float().cpu().numpy()  # [n_tok, n_heads*128] -> vector order h * n_tok + t
        out["k"] = np.concatenate([kk[:, h * 128:(h + 1) * 128] for h in range(n_heads)], axis=0)
    return out


def _check_projection(r, n_heads, rel=2e-5):
    want = project.project(r["x"], r["w"], n_heads)
    s, a = project.project_exact(r["x"], r["w"], n_heads)
    flags = project.bf16_tie_flags(s, a, rel)
    got = r["k"].astype(np.float64)
    dif = got != want
    assert not np.any(dif & ~flags), f"unflagged projection mismatches: {np.argwhere(dif & ~flags)[:10]}"
    # a flagged value must be the bf16 rounding of a sum within the fp32 accumulation band
    lo, hi = project.bf16_round(s - rel * a), project.bf16_round(s + rel * a)
    assert np.all((got[dif] >= lo[dif]) & (got[dif] <= hi[dif]))
    return int(dif.sum()), int(flags.sum())


@pytest.mark.parametrize("bits,mode", [(4, tq.TQ_MODE_PROD), (3, tq.TQ_MODE_PROD), (3, tq.TQ_MODE_MSE),
                                       (2, tq.TQ_MODE_PROD), (4, tq.TQ_MODE_MSE)])
def test_ragged_tokens_three_heads(bits, mode):
    # 300 tokens: three tiles per head, the last one 44 rows; vectors of a head follow the previous
    # head's without padding, so code tiles straddle heads
    n_tok, n_heads = 300, 3
    r = _run(n_tok, 256, n_heads, bits, mode, seed=31)
    _check_projection(r, n_heads)
    compare_codes(r["op"], r["k"], r["codes"], r["norms"], r["rn"])


def test_layer_width_hidden_4096():
    # the Llama-3.1-8B layer width: 64 K blocks of 64 per tile
    n_tok, n_heads = 256, 2
    r = _run(n_tok, 4096, n_heads, 3, tq.TQ_MODE_PROD, seed=32)
    _check_projection(r, n_heads)
    compare_codes(r["op"], r["k"], r["codes"], r["norms"], r["rn"])


@pytest.mark.parametrize("mode", [tq.TQ_MODE_PROD, tq.TQ_MODE_MSE])
def test_hidden_half_k_block(mode):
    # hidden 160 = two and a half K blocks of 64: the last block's box reads zeros past the row end
    n_tok, n_heads = 200, 2
    r = _run(n_tok, 160, n_heads, 3, mode, seed=36)
    _check_projection(r, n_heads)
    compare_codes(r["op"], r["k"], r["codes"], r["norms"], r["rn"])


@pytest.mark.parametrize("bits,mode", [(4, tq.TQ_MODE_PROD), (4, tq.TQ_MODE_MSE)])
def test_many_tiles_per_cta(bits, mode):
    # 8 heads x 47 token tiles = 376 tiles over <= 148 CTAs: the GEMM ring, both accumulators and the
    # slotted rotation / projection MMAs wrap several times.  Codes against the oracle's encoding of
    # the projected vectors; MSE codes also bit for bit against tq_quantize on those vectors (the same
    # rotation and coding kernel)
    n_tok, n_heads = 6000, 8
    r = _run(n_tok, 512, n_heads, bits, mode, seed=33)
    _check_projection(r, n_heads)
    compare_codes(r["op"], r["k"], r["codes"], r["norms"], r["rn"])
    if mode == tq.TQ_MODE_MSE:
        kt = torch.from_numpy(r["k"].astype(np.float32)).to(torch.bfloat16).cuda()
        codes_q, norms_q, _ = gpu_quantize(r["p"], kt)
        assert np.array_equal(codes_q, r["codes"])
        assert np.array_equal(norms_q.view(np.int16), r["norms"].view(np.int16))


def test_without_projected_copy():
    a = _run(200, 128, 2, 4, tq.TQ_MODE_PROD, seed=34, with_k=True)
    b = _run(200, 128, 2, 4, tq.TQ_MODE_PROD, seed=34, with_k=False)
    assert np.array_equal(a["codes"], b["codes"])
    assert np.array_equal(a["norms"].view(np.int16), b["norms"].view(np.int16))


def test_single_token_and_unsupported_shapes():
    r = _run(1, 64, 1, 4, tq.TQ_MODE_PROD, seed=35)
    _check_projection(r, 1)
    compare_codes(r["op"], r["k"], r["codes"], r["norms"], r["rn"])
    p, _ = make_pair(128, 4, tq.TQ_MODE_PROD)
    x = torch.zeros((4, 48), dtype=torch.bfloat16, device="cuda")   # hidden not a multiple of 32
    w = torch.zeros((128, 48), dtype=torch.bfloat16, device="cuda")
    c = torch.zeros(4096, dtype=torch.uint8, device="cuda")
    nn = torch.zeros(4, dtype=torch.int16, device="cuda")
    with pytest.raises(tq.TQError):
        tq.tq_project_quantize(p, x, w, 1, c, nn, nn)
    p2, _ = make_pair(100, 4, tq.TQ_MODE_PROD)                      # d < d_pad
    x2 = torch.zeros((4, 64), dtype=torch.bfloat16, device="cuda")
    w2 = torch.zeros((128, 64), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(tq.TQError):
        tq.tq_project_quantize(p2, x2, w2, 1, c, nn, nn)
