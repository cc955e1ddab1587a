"""GPU parity of tq_logits against the oracle estimator on oracle-made codes
(so the comparison never depends on boundary decisions):
|delta| <= 1e-4 |l| + 1e-5 n ||q||."""
import numpy as np
import pytest
import torch

import vector_quantization_randomized_b200 as tq
import workloads as wl
from oracle import estimate
from gpu_util import make_pair, oracle_codes, logit_tolerance

pytestmark = pytest.mark.gpu


def _check(d, bits, mode, n_heads, group, n_keys, seed=0, m=None):
    p, op = make_pair(d, bits, mode, m)
    keys = np.concatenate([wl.to_bf16(wl.head_vectors(n_keys, d, seed=seed, head=h)) for h in range(n_heads)])
    q = wl.queries(n_heads * group, d, seed=seed + 100)
    codes, norms, rnorms, enc = oracle_codes(op, keys)
    ref = estimate.logits_gqa(q, op.D, op.S, enc["idx"], enc.get("signs"), norms, rnorms, op.c, op.m,
                              n_heads, group, n_keys)
    dcodes = torch.from_numpy(codes).cuda()
    dn = torch.from_numpy(norms.view(np.int16)).cuda()
    drn = torch.from_numpy(rnorms.view(np.int16)).cuda() if rnorms is not None else None
    dq = torch.from_numpy(q).cuda()
    out = torch.full((q.shape[0], n_keys), float("nan"), device="cuda")
    ws = torch.empty(max(tq.tq_logits_workspace(p, q.shape[0]), 16), dtype=torch.uint8, device="cuda")
    tq.tq_logits(p, dq, group, dcodes, dn, drn, n_keys, n_heads, out, ws)
    got = out.cpu().numpy().astype(np.float64)
    for h in range(q.shape[0]):
        g = h // group
        tol = logit_tolerance(ref[h:h + 1], norms[g * n_keys:(g + 1) * n_keys], q[h:h + 1])[0]
        err = np.abs(got[h] - ref[h])
        bad = ~(err <= tol)
        assert not np.any(bad), (h, np.argwhere(bad)[:5].ravel(), got[h][bad][:5], ref[h][bad][:5])
    return got, ref


def test_single_head_16_queries_b4():
    # 4096 keys, 16 queries against all keys, b = 4 (3-bit Lloyd-Max + 128 QJL signs)
    _check(128, 4, tq.TQ_MODE_PROD, n_heads=1, group=16, n_keys=4096)


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_gqa4_ragged(bits):
    _check(128, bits, tq.TQ_MODE_PROD, n_heads=3, group=4, n_keys=1001)


@pytest.mark.parametrize("group", [1, 2, 5])
def test_group_sizes(group):
    _check(128, 3, tq.TQ_MODE_PROD, n_heads=2, group=group, n_keys=333)


@pytest.mark.parametrize("bits", [1, 2, 3])
def test_mse_codes(bits):
    _check(128, bits, tq.TQ_MODE_MSE, n_heads=2, group=4, n_keys=500)


@pytest.mark.parametrize("bits", [2, 3])
def test_padded_dim_256(bits):
    _check(200, bits, tq.TQ_MODE_PROD, n_heads=1, group=4, n_keys=700)


def test_small_m():
    _check(128, 4, tq.TQ_MODE_PROD, n_heads=2, group=4, n_keys=257, m=64)


def test_tiny():
    _check(128, 4, tq.TQ_MODE_PROD, n_heads=1, group=1, n_keys=1)
    _check(128, 4, tq.TQ_MODE_PROD, n_heads=1, group=4, n_keys=9)


# d_pad 256 with 3 index bits (b = 4 product codes at d = 200, config 4's codes; b = 3 MSE codes):
# the tensor-memory search scan writing every score
@pytest.mark.parametrize("bits,mode,n_heads,group,n_keys", [
    (4, tq.TQ_MODE_PROD, 1, 4, 700),      # one head, ragged key count
    (4, tq.TQ_MODE_PROD, 2, 5, 640),      # a 16-query chunk with 5 queries per head
    (4, tq.TQ_MODE_PROD, 2, 20, 320),     # two chunks per head
    (3, tq.TQ_MODE_MSE, 2, 4, 8992),      # three key splits per head
])
def test_padded_dim_256_three_index_bits(bits, mode, n_heads, group, n_keys):
    _check(200, bits, mode, n_heads=n_heads, group=group, n_keys=n_keys)


def test_padded_dim_256_three_index_bits_unsupported_shapes():
    p, _ = make_pair(200, 4, tq.TQ_MODE_PROD, m=128)   # the scan needs m = 256 (or MSE)
    q = torch.zeros((4, 200), device="cuda")
    c = torch.zeros(1 << 16, dtype=torch.uint8, device="cuda")
    nn = torch.zeros(64, dtype=torch.int16, device="cuda")
    out = torch.zeros((4, 64), device="cuda")
    ws = torch.zeros(1 << 20, dtype=torch.uint8, device="cuda")
    with pytest.raises(tq.TQError):
        tq.tq_logits(p, q, 4, c, nn, nn, 64, 1, out, ws)
    p2, _ = make_pair(200, 4, tq.TQ_MODE_PROD)         # several heads need n_keys % 32 == 0
    out2 = torch.zeros((8, 50), device="cuda")
    q2 = torch.zeros((8, 200), device="cuda")
    with pytest.raises(tq.TQError):
        tq.tq_logits(p2, q2, 4, c, nn, nn, 50, 2, out2, ws)
