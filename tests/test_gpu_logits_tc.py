"""GPU parity of tq_logits on the shapes that take the tensor-memory scan
(d_pad 128, up to 4 query heads per KV head, key count a multiple of 32):
128-key items with ragged tails of 32/64/96 keys, every group size 1..4,
product codes at b = 2, 3, 4 and MSE codes at b = 1, 2, 3, several KV heads
(an item range that crosses heads reloads the query operand), and a launch
with about 55 items per CTA so the shared-memory ring of code tiles wraps
several times.  Oracle-made codes, |delta| <= 1e-4 |l| + 1e-5 n ||q||."""
import numpy as np
import pytest
import torch

import vector_quantization_randomized_b200 as tq
import workloads as wl
from oracle import estimate
from gpu_util import make_pair, oracle_codes, logit_tolerance

pytestmark = pytest.mark.gpu
dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()


def _check(bits, mode, n_heads, group, n_keys, seed=0):
    p, op = make_pair(128, bits, mode)
    keys = np.concatenate([wl.to_bf16(wl.head_vectors(n_keys, 128, seed=seed, head=h)) for h in range(n_heads)])
    q = wl.queries(n_heads * group, 128, seed=seed + 100)
    codes, norms, rnorms, enc = oracle_codes(op, keys)
    ref = estimate.logits_gqa(q, op.D, op.S, enc["idx"], enc.get("signs"), norms, rnorms, op.c, op.m,
                              n_heads, group, n_keys)
    out = torch.full((q.shape[0], n_keys), float("nan"), device="cuda")
    ws = torch.empty(tq.tq_logits_workspace(p, q.shape[0]), dtype=torch.uint8, device="cuda")
    tq.tq_logits(p, dev(q), group, dev(codes), dev(norms.view(np.int16)),
                 dev(rnorms.view(np.int16)) if rnorms is not None else None, n_keys, n_heads, out, ws)
    got = out.cpu().numpy().astype(np.float64)
    for h in range(q.shape[0]):
        g = h // group
        tol = logit_tolerance(ref[h:h + 1], norms[g * n_keys:(g + 1) * n_keys], q[h:h + 1])[0]
        bad = ~(np.abs(got[h] - ref[h]) <= tol)
        assert not np.any(bad), (h, np.argwhere(bad)[:5].ravel(), got[h][bad][:5], ref[h][bad][:5])


@pytest.mark.parametrize("bits,group,n_heads,n_keys", [
    (4, 4, 5, 4192),   # 33 items per head, tail of 96 keys
    (3, 4, 3, 160),    # one full item + 32-key tail
    (2, 3, 2, 32),     # a single 32-key item per head
    (3, 1, 2, 1088),   # tail of 64 keys, one query per head
    (4, 2, 1, 96),
    (3, 4, 8, 2048),
])
def test_prod_shapes(bits, group, n_heads, n_keys):
    _check(bits, tq.TQ_MODE_PROD, n_heads, group, n_keys)


@pytest.mark.parametrize("bits", [1, 2, 3])
def test_mse_shapes(bits):
    _check(bits, tq.TQ_MODE_MSE, 2, 4, 288)


def test_ring_wraps_many_items_per_cta():
    """512 KV heads x 16384 keys (8192 items): three heads carry oracle-made
    codes, the others zero codes (their logits are not compared)."""
    H, T, G = 512, 16384, 4
    p, op = make_pair(128, 3, tq.TQ_MODE_PROD)
    sample = [0, 257, 511]
    n = H * T
    codes = np.zeros(p.code_bytes(n), np.uint8)
    norms = np.zeros(n, np.float16)
    rnorms = np.zeros(n, np.float16)
    tb = p.code_bytes(32)
    encs = {}
    for h in sample:
        x = wl.to_bf16(wl.head_vectors(T, 128, seed=3, head=h))
        c, nn, rn, enc = oracle_codes(op, x)
        t0 = h * T // 32
        codes[t0 * tb:t0 * tb + c.size] = c
        norms[h * T:(h + 1) * T] = nn
        rnorms[h * T:(h + 1) * T] = rn
        encs[h] = enc
    q = wl.queries(H * G, 128, seed=9)
    out = torch.empty((H * G, T), dtype=torch.float32, device="cuda")
    ws = torch.empty(tq.tq_logits_workspace(p, H * G), dtype=torch.uint8, device="cuda")
    tq.tq_logits(p, dev(q), G, dev(codes), dev(norms.view(np.int16)), dev(rnorms.view(np.int16)), T, H, out, ws)
    torch.cuda.synchronize()
    for h in sample:
        enc = encs[h]
        qh = q[h * G:(h + 1) * G]
        ref = estimate.logits_gqa(qh, op.D, op.S, enc["idx"], enc["signs"], norms[h * T:(h + 1) * T],
                                  rnorms[h * T:(h + 1) * T], op.c, op.m, 1, G, T)
        got = out[h * G:(h + 1) * G].cpu().numpy().astype(np.float64)
        tol = logit_tolerance(ref, norms[h * T:(h + 1) * T], qh)
        assert np.all(np.abs(got - ref) <= tol), h


@pytest.mark.parametrize("bits,n_heads,n_keys", [(4, 700, 64), (3, 600, 128)])
def test_many_heads_per_cta(bits, n_heads, n_keys):
    """Short sequences over many KV heads: a CTA's item range crosses several heads,
    so the in-kernel query preparation refills its two B-image slots in turn."""
    _check(bits, tq.TQ_MODE_PROD, n_heads, 4, n_keys, seed=5)
