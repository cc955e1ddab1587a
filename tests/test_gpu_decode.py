"""GPU parity of tq_decode_attn against the oracle's token-by-token fp64
decode attention on oracle-made K (product code) and V (MSE code):
||delta o|| <= 2e-3 ||o|| per output row."""
import numpy as np
import pytest
import torch

import vector_quantization_randomized_b200 as tq
import workloads as wl
from oracle import codec, estimate
from gpu_util import make_pair, oracle_codes

pytestmark = pytest.mark.gpu


def _check(B, Hkv, Hq, T, seq_lens, kbits=3, vbits=3, d=128, scale=0.0, layout=tq.TQ_LAYOUT_PLANES):
    kp, kop = make_pair(d, kbits, tq.TQ_MODE_PROD, seed=42)
    vp, vop = make_pair(d, vbits, tq.TQ_MODE_MSE, seed=43, layout=layout)
    K = wl.kv_block(B, Hkv, T, d, seed=wl.SEED_KEYS).reshape(-1, d)
    V = wl.kv_block(B, Hkv, T, d, seed=wl.SEED_VALUES).reshape(-1, d)
    q = wl.queries(B * Hq, d, seed=wl.SEED_QUERIES).reshape(B, Hq, d)
    kc, kn, krn, ke = oracle_codes(kop, K)
    vc, vn, _, ve = oracle_codes(vop, V)
    if layout == tq.TQ_LAYOUT_SLICED:
        vc = codec.pack_sliced(ve["idx"], vop.kb)  # the value cache in the token-sliced layout
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


# token-sliced values: the tensor-memory decode (keys with m = 128 and at most 3 index bits,
# values with at most 3, at most 4 query heads per KV head, max_tokens a multiple of 32)
SL = tq.TQ_LAYOUT_SLICED


def test_sliced_gqa4_segments_and_ragged_lengths():
    # 1120 tokens: two 1024-token segments, the second ragged; a 517-token and a 1-token sequence
    _check(B=3, Hkv=2, Hq=8, T=1120, seq_lens=[1120, 517, 1], layout=SL)


def test_sliced_empty_sequence_and_single_item():
    _check(B=2, Hkv=1, Hq=4, T=96, seq_lens=[0, 96], layout=SL)


@pytest.mark.parametrize("Hq", [1, 2])
def test_sliced_group_sizes(Hq):
    _check(B=2, Hkv=1, Hq=Hq, T=640, seq_lens=[640, 333], layout=SL)


@pytest.mark.parametrize("kbits,vbits", [(2, 1), (3, 2), (4, 3)])
def test_sliced_bit_widths(kbits, vbits):
    _check(B=1, Hkv=2, Hq=4, T=704, seq_lens=[650], kbits=kbits, vbits=vbits, layout=SL)


def test_sliced_many_units_per_cta():
    # 2 x 8 KV heads x 4096 tokens (64 segments over <= 148 CTAs, several per CTA, heads changing
    # inside a CTA's range), 32 query heads
    _check(B=2, Hkv=8, Hq=32, T=4096, seq_lens=[4096, 3000], layout=SL)


def test_sliced_explicit_scale_matches_planes():
    a, _ = _check(B=1, Hkv=1, Hq=4, T=256, seq_lens=[256], scale=0.02, layout=SL)
    b, _ = _check(B=1, Hkv=1, Hq=4, T=256, seq_lens=[256], scale=0.02)
    # both are within the oracle's tolerance; they agree row by row to the sum of the two
    for h in range(4):
        assert np.linalg.norm(a[0, h] - b[0, h]) <= 4e-3 * np.linalg.norm(b[0, h])


def test_sliced_unsupported_shapes():
    with pytest.raises(tq.TQError):   # five query heads per KV head
        _check(B=1, Hkv=1, Hq=5, T=128, seq_lens=[128], layout=SL)
    with pytest.raises(tq.TQError):   # max_tokens not a multiple of 32
        _check(B=1, Hkv=1, Hq=4, T=100, seq_lens=[100], layout=SL)
