"""Device-side wait timeouts reach the caller: a diagnostic kernel whose
barrier wait runs out (nothing arrives) sets its fault word, tq_device_status
reports TQ_ETIMEOUT naming it, clearing resets it, and the context keeps
working (a quantize + logits pass afterwards leaves the status clean)."""
import numpy as np
import pytest
import torch

import vector_quantization_randomized_b200 as tq
import workloads as wl

pytestmark = pytest.mark.gpu


def test_timeout_is_reported_and_cleared():
    torch.cuda.init()
    assert tq.tq_device_status(clear=True) in (tq.TQ_OK, tq.TQ_ETIMEOUT)  # start from a clean slate
    tq.tq_diag_bounded_wait(1000)
    assert tq.tq_device_status(clear=False) == tq.TQ_ETIMEOUT
    assert "diagnostic" in tq.tq_last_error()
    assert tq.tq_device_status(clear=True) == tq.TQ_ETIMEOUT
    assert tq.tq_device_status(clear=False) == tq.TQ_OK


def test_context_usable_after_timeout():
    tq.tq_diag_bounded_wait(100)
    tq.tq_device_status(clear=True)
    p = tq.Params(128, 3, tq.TQ_MODE_PROD, 128)
    n, G = 4096, 4
    x = torch.from_numpy(wl.to_bf16(wl.head_vectors(n, 128, seed=0, head=0))).to(torch.bfloat16).cuda()
    c = torch.empty(p.code_bytes(n), dtype=torch.uint8, device="cuda")
    nn = torch.empty(n, dtype=torch.int16, device="cuda")
    rn = torch.empty(n, dtype=torch.int16, device="cuda")
    tq.tq_quantize(p, x, c, nn, rn)
    q = torch.from_numpy(wl.queries(G, 128, seed=2)).cuda()
    out = torch.empty((G, n), device="cuda")
    ws = torch.empty(tq.tq_logits_workspace(p, G), dtype=torch.uint8, device="cuda")
    tq.tq_logits(p, q, G, c, nn, rn, n, 1, out, ws)
    assert tq.tq_device_status() == tq.TQ_OK
    assert torch.isfinite(out).all()


def test_diag_rejects_bad_polls():
    with pytest.raises(tq.TQError):
        tq.tq_diag_bounded_wait(0)
    with pytest.raises(tq.TQError):
        tq.tq_diag_bounded_wait((1 << 20) + 1)
