"""Independent CPU oracle for the TurboQuant hot path (TEST INFRASTRUCTURE ONLY).

This package is a plain, slow, obviously-correct fp64 restatement of what the
GPU library computes.  It exists to check the library; nothing in the library
imports it.  Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline
leg of ``bench.py`` may import or run it.

It shares no code with ``vector_quantization_randomized_b200`` (no kernels,
headers, helpers, tables or constant generators).  The seeded *input*
generators (the top-level ``workloads`` module) hold none of the
method's arithmetic and are the only thing both sides use.

Sources, by page and section (the pages are web articles about Google's
TurboQuant; they print no code and only one formula):

* "TurboQuant explainer" (m.163.com), section "TurboQuant 怎么做的":
  - "第一步：PolarQuant": random rotation makes every coordinate follow one
    known, concentrated (Beta) law, so one precomputed Max-Lloyd table serves
    all vectors; stage 1 uses b-1 bits.
  - "第二步：QJL": a Johnson-Lindenstrauss transform of the stage-1 residual,
    kept as one sign bit per row, with an estimator whose expectation is the
    true inner product (E[<y, Q^-1(Q(x))>] = <y, x>); a 1-bit MSE quantizer
    alone shrinks inner products by 2/pi.
  - "合起来": b-1 bits + 1 bit = b bits; distortion within about 2.7x of the
    information-theoretic bound.
  - "速度" / "向量搜索": attention logits straight from the codes; top-k
    inner-product search on quantized vectors.
* zhidx article on turboquant_plus, "01 turboquant_plus：介绍与详解": the
  rotation is a Walsh-Hadamard transform (WHT); turbo4 stores 4.25 bit/value;
  asymmetric K/V (keys with the product code, values MSE-only).

Modules
-------
philox    Philox4x32-10 counter-based generator (Salmon et al., SC'11).
params    the random sign flips D and the dense Gaussian QJL matrix S.
codebook  Lloyd-Max quantizer for the rotated-coordinate law.
codec     encode (norm, rotation, scalar codes, residual, QJL signs),
          canonical bit-packed layout, decision-boundary flags.
estimate  attention-logit estimator, MSE dequantisation, decode attention,
          top-k search.

Parity pins: see ``tests/test_oracle_*.py``.  Functions without an
independent pin say "parity unpinned" in their docstring.
"""
