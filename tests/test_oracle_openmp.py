"""The OpenMP build of the oracle (used only to time it on every host core)
gives bit-identical results to the single-threaded test build: the same
indexer scores, top-k, FP4 codes and attention on the same inputs."""
import hashlib
import os
import subprocess
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

SCRIPT = r'''
import sys, hashlib, numpy as np
sys.path.insert(0, sys.argv[1])
import oracle
if sys.argv[2] == "omp":
    oracle.use_all_cores(True)
rng = np.random.default_rng(5)
h = hashlib.sha256()
x = rng.standard_normal((300, 576)).astype(np.float32)
bits = (x.view(np.uint32) >> 16).astype(np.uint16)
codes, scales = oracle.quant_fp4(bits)
h.update(codes.tobytes()); h.update(scales.tobytes())
kid = rng.integers(0, 120, (3000, 64)).astype(np.uint8)
q = rng.integers(0, 120, (4, 64)).astype(np.uint8)
s = oracle.indexer_scores(q, np.array([0.25, 0.5, 1, 2], np.float32), kid, np.ones(3000, np.float32))
h.update(s.tobytes()); h.update(oracle.topk(s, 3000, 100).tobytes())
qb = (rng.standard_normal((16, 576)).astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)
o, l = oracle.sparse_attn(qb, codes, scales, np.arange(0, 300, 3, dtype=np.int32), bits[:128], 1 / 24.0)
h.update(o.tobytes()); h.update(l.tobytes())
c8, s8 = oracle.quant_index_fp8(bits[:, :64])
h.update(c8.tobytes()); h.update(s8.tobytes())
print(h.hexdigest(), oracle.threads())
'''


def run(variant: str):
    r = subprocess.run([sys.executable, "-c", SCRIPT, ROOT, variant], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    digest, threads = r.stdout.split()
    return digest, int(threads)


def test_openmp_build_is_bit_identical():
    d1, t1 = run("serial")
    d2, t2 = run("omp")
    assert t1 == 1 and t2 >= 1
    assert d1 == d2
