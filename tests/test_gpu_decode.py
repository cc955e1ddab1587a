"""GPU parity of tq_decode_attn against the oracle's token-by-token fp64
decode attention on oracle-made K (product code) and V (MSE code):
||delta o|| <= 2e-3 ||o|| per output row."""
import numpy as np
import pytest
import torch

import vector_quantization_randomized_b200 as tq
import workloads as wl
from oracle import estimate
from gpu_util import make_pair, oracle_codes

pytestmark = pytest.mark.gpu


def _check(B, Hkv, Hq, T, seq_lens, kbits=3, vbits=3, d=128, scale=0.0):
    kp, kop = make_pair(d, kbits, tq.TQ_MODE_PROD, seed=42)
    vp, vop = make_pair(d, vbits, tq.TQ_MODE_MSE, seed=43)
    K = wl.kv_block(B, Hkv, T, d, seed=wl.SEED_KEYS).reshape(-1, d)
    V = wl.kv_block(B, Hkv, T, d, seed=wl.SEED_VALUES).reshape(-1, d)
    q = wl.queries(B * Hq, d, seed=wl.SEED_QUERIES).reshape(B, Hq, d)
    kc, kn, krn, ke = oracle_codes(kop, K)
    vc, vn, _, ve = oracle_codes(vop, V)
    ref = estimate.decode_attention(q, kop.D, kop.S, ke["idx"], ke["signs"], kn, krn, kop.c, kop.m,
                                    vop.D, ve["idx"], vn, vop.c, d, seq_lens, Hq, Hkv, T, scale=scale)
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    out = torch.full((B, Hq, d), float("nan"), device="cuda")
    ws = torch.empty(tq.tq_decode_attn_workspace(kp, B, Hq, Hkv, T), dtype=torch.uint8, device="cuda")
    sl = torch.tensor(seq_lens, dtype=torch.int32, device="cuda")
    tq.tq_decode_attn(kp, vp, dev(q), Hkv, dev(kc), dev(kn.view(np.int16)), dev(krn.view(np.int16)), dev(vc),
                      dev(vn.view(np.int16)), sl, T, out, ws, scale=scale)
    got = out.cpu().numpy().astype(np.float64)
    for b in range(B):
        for h in range(Hq):
            o, r = got[b, h], ref[b, h]
            if seq_lens[b] == 0:
                assert np.all(o == 0)
                continue
            assert np.linalg.norm(o - r) <= 2e-3 * np.linalg.norm(r), (b, h, np.linalg.norm(o - r) / np.linalg.norm(r))
    return got, ref


def test_decode_gqa4_chunks_and_ragged_lengths():
    _check(B=3, Hkv=2, Hq=8, T=1100, seq_lens=[1100, 517, 1])


def test_decode_empty_sequence_and_single_chunk():
    _check(B=2, Hkv=1, Hq=4, T=96, seq_lens=[0, 96])


@pytest.mark.parametrize("Hq", [2, 5])
def test_decode_group_sizes(Hq):
    _check(B=2, Hkv=1, Hq=Hq, T=600, seq_lens=[600, 333])


@pytest.mark.parametrize("kbits,vbits", [(2, 2), (4, 4), (4, 1)])
def test_decode_bit_widths(kbits, vbits):
    _check(B=1, Hkv=2, Hq=4, T=700, seq_lens=[650], kbits=kbits, vbits=vbits)


def test_decode_explicit_scale():
    _check(B=1, Hkv=1, Hq=4, T=256, seq_lens=[256], scale=0.02)
