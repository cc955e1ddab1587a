"""GPU parity of tq_dequantize (the reconstruction Q^-1 of "TurboQuant
explainer" (m.163.com), "第二步：QJL") against the oracle's dequant_prod /
dequant_mse on oracle-made codes: ||delta x_hat|| <= 1e-5 ||x_hat|| per row
(fp32 sum of m signed S entries, relative error ~ m 2^-24 sqrt(m) in the
worst case, and seven fp32 rotation stages; the oracle is fp64).  Also:
<q, x_hat> from the GPU reconstruction agrees with tq_logits (linearity), and
re-encoding at a lower bit width (temporal decay, zhidx turboquant_plus
article) — quantize at b = 4, dequantize, quantize at b = 2 — gives the codes
the oracle gives for the same fp32 input."""
import numpy as np
import pytest
import torch

import vector_quantization_randomized_b200 as tq
import workloads as wl
from oracle import estimate
from gpu_util import make_pair, oracle_codes, compare_codes, logit_tolerance, gpu_quantize

pytestmark = pytest.mark.gpu
dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()


def _dequant(p, codes, norms, rnorms, n, d, ld):
    out = torch.full((n, ld), 7.0, dtype=torch.float32, device="cuda")
    tq.tq_dequantize(p, dev(codes), dev(norms.view(np.int16)),
                     dev(rnorms.view(np.int16)) if rnorms is not None else None, n, out, ld)
    o = out.cpu().numpy()
    assert np.all(o[:, d:] == 7.0)        # columns past d untouched
    return o[:, :d].astype(np.float64)


@pytest.mark.parametrize("d,bits,mode,m,n", [
    (128, 2, tq.TQ_MODE_PROD, 128, 1000),
    (128, 3, tq.TQ_MODE_PROD, 128, 333),
    (128, 4, tq.TQ_MODE_PROD, 64, 97),
    (200, 3, tq.TQ_MODE_PROD, 256, 257),
    (128, 1, tq.TQ_MODE_MSE, None, 64),
    (128, 3, tq.TQ_MODE_MSE, None, 1),
    (128, 4, tq.TQ_MODE_MSE, None, 500),
    (200, 2, tq.TQ_MODE_MSE, None, 40),
])
def test_reconstruction_matches_oracle(d, bits, mode, m, n):
    p, op = make_pair(d, bits, mode, m)
    x = wl.to_bf16(wl.head_vectors(n, d, seed=5, head=1))
    codes, norms, rnorms, enc = oracle_codes(op, x)
    if mode == tq.TQ_MODE_PROD:
        ref = estimate.dequant_prod(enc["idx"], enc["signs"], norms, rnorms, op.c, op.D, op.S, op.m, d)
    else:
        ref = estimate.dequant_mse(enc["idx"], norms, op.c, op.D, d)
    got = _dequant(p, codes, norms, rnorms, n, d, d + 8)
    err = np.linalg.norm(got - ref, axis=1)
    assert np.all(err <= 1e-5 * np.linalg.norm(ref, axis=1) + 1e-30), err.max()


def test_inner_product_with_reconstruction_is_the_logit():
    d, n, G = 128, 2048, 4
    p, op = make_pair(d, 4, tq.TQ_MODE_PROD)
    x = wl.to_bf16(wl.head_vectors(n, d, seed=6, head=0))
    codes, norms, rnorms, enc = oracle_codes(op, x)
    xh = _dequant(p, codes, norms, rnorms, n, d, d)
    q = wl.queries(G, d, seed=7)
    out = torch.empty((G, n), device="cuda")
    ws = torch.empty(tq.tq_logits_workspace(p, G), dtype=torch.uint8, device="cuda")
    tq.tq_logits(p, dev(q), G, dev(codes), dev(norms.view(np.int16)), dev(rnorms.view(np.int16)), n, 1, out, ws)
    lg = out.cpu().numpy().astype(np.float64)
    ip = q.astype(np.float64) @ xh.T
    tol = logit_tolerance(ip, norms, q) + 1e-5 * np.linalg.norm(q, axis=1)[:, None] * np.linalg.norm(xh, axis=1)[None, :]
    assert np.all(np.abs(lg - ip) <= tol)


@pytest.mark.parametrize("mode", [tq.TQ_MODE_PROD, tq.TQ_MODE_MSE])
def test_temporal_decay_reencode(mode):
    d, n = 128, 777
    hi, _ = make_pair(d, 4, mode)
    lo, olo = make_pair(d, 2, mode)
    x = torch.from_numpy(wl.to_bf16(wl.head_vectors(n, d, seed=8, head=2))).to(torch.bfloat16).cuda()
    c = torch.empty(hi.code_bytes(n), dtype=torch.uint8, device="cuda")
    nn = torch.empty(n, dtype=torch.int16, device="cuda")
    rn = torch.empty(n, dtype=torch.int16, device="cuda") if mode == tq.TQ_MODE_PROD else None
    tq.tq_quantize(hi, x, c, nn, rn)
    xh = torch.empty((n, d), dtype=torch.float32, device="cuda")
    tq.tq_dequantize(hi, c, nn, rn, n, xh)
    codes, norms, rnorms = gpu_quantize(lo, xh)
    compare_codes(olo, xh.cpu().numpy(), codes, norms, rnorms)


def test_rejects_bad_arguments():
    p, op = make_pair(128, 3, tq.TQ_MODE_PROD)
    c = torch.zeros(p.code_bytes(32), dtype=torch.uint8, device="cuda")
    nn = torch.zeros(32, dtype=torch.int16, device="cuda")
    out = torch.zeros((32, 128), device="cuda")
    with pytest.raises(tq.TQError):
        tq.tq_dequantize(p, c, nn, None, 32, out)          # product mode needs residual norms
    with pytest.raises(tq.TQError):
        tq.tq_dequantize(p, c, nn, nn, 32, out, ld=100)    # ld < d
