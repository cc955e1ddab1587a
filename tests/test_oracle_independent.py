"""The oracle and the input generators run without the library.

A fresh interpreter draws inputs from `workloads`, encodes them with the
oracle, estimates logits and decode attention, and then checks its own memory
map: libtq.so (the CUDA library) must not be mapped, and the package that
loads it must not have been imported.  This is what lets the oracle check the
library rather than itself.
"""
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

SCRIPT = r"""
import sys
import numpy as np
import workloads as wl
from oracle import codec, estimate, polar
from oracle.codebook import stored_codebook
from oracle.params import sign_flips, qjl_matrix
K = wl.to_bf16(wl.head_vectors(64, 128, seed=wl.SEED_KEYS))
q = wl.queries(4, 128)
c, t = stored_codebook(128, 2)
D, S = sign_flips(wl.SEED_PARAMS, 128), qjl_matrix(wl.SEED_PARAMS, 128, 128)
e = codec.encode(K, D, c, t, S)
buf = codec.pack(e["idx"], e["signs"], 2, 128)
idx, sg = codec.unpack(buf, 64, 128, 2, 128)
lg = estimate.logits_gqa(q, D, S, idx, sg, e["norm_f16"], e["rnorm_f16"], c, 128, 1, 4, 64)
pe = polar.encode(K, D, 2)
assert np.all(np.isfinite(lg))
maps = open("/proc/self/maps").read()
assert "libtq" not in maps, "libtq.so is mapped in the oracle process"
assert "vector_quantization_randomized_b200" not in sys.modules, "the library package was imported"
print("independent")
"""


def test_oracle_process_does_not_load_the_library():
    env = dict(os.environ)
    env["PYTHONPATH"] = ROOT + os.pathsep + env.get("PYTHONPATH", "")
    r = subprocess.run([sys.executable, "-c", SCRIPT], cwd=ROOT, env=env, capture_output=True, text=True,
                       timeout=300)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "independent" in r.stdout
