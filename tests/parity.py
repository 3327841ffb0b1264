"""Output comparison for the parity tests: max-abs and relative-L2 bounds.

Every comparison of an attention output with the oracle goes through
``check``; it records the observed errors (printed at the end of the session
by ``tests/conftest.py``, and appended as JSON lines to the file named by
``CA_PARITY_LOG`` when that variable is set) and asserts both bounds.

Bounds
------
max-abs: 1e-2 for bf16 inputs, 1e-5 for fp32 inputs (the method's stated
tolerance).

relative L2, ||got - want||_F / ||want||_F over the compared rows:

* bf16 (tensor-core kernel). Q, K, V are bf16 values, so the oracle sees the
  same inputs exactly; the products Q K^T and P V accumulate in fp32. Two
  roundings to bf16 dominate: P before the P V product and O at the store.
  A bf16 rounding has relative error at most 2^-8 and, over many elements,
  root-mean-square at most 2^-8 / sqrt(3) = 2.26e-3; the two are
  independent, so together about 3.2e-3. The remaining terms (fp32 logits,
  row sums over up to 2^18 terms, centroids carried as bf16 hi + lo, the
  FMA-pipe exponential's 7.5e-5) are each below 1e-4. Bound: 1e-2, three
  times the estimate.
* fp32 (SIMT kernel). A logit q.k / sqrt(d) computed in fp32 carries an
  absolute error of about u |q.k| / sqrt(d) (u = 2^-24), at most
  u |q||k| / sqrt(d) < 2e-6 at the test data's largest norms
  (|q||k| / sqrt(d) <= 30); a weight's relative error is its logit's
  absolute error, and the base-2 exponential's argument adds a relative u.
  O's relative error is a weighted mean of its weights' plus the fp32
  accumulation of the sums (about sqrt(n) u, n <= 1,024 keys: 2e-6). The
  estimate is ~5e-6; bound 2e-5.
"""
from __future__ import annotations

import json
import os

import numpy as np

MAX_ABS = {"bf16": 1e-2, "fp32": 1e-5}
REL_L2 = {"bf16": 1e-2, "fp32": 2e-5}

RECORDS: list = []


def errors(got, want):
    got = np.asarray(got, np.float64)
    want = np.asarray(want, np.float64)
    diff = got - want
    max_abs = float(np.abs(diff).max()) if diff.size else 0.0
    norm = float(np.linalg.norm(want))
    rel = float(np.linalg.norm(diff) / norm) if norm > 0 else float(np.linalg.norm(diff))
    return max_abs, rel


def check(label: str, got, want, dtype: str):
    """Assert max-abs <= MAX_ABS[dtype] and rel-L2 <= REL_L2[dtype]; record both."""
    max_abs, rel = errors(got, want)
    rec = dict(case=label, dtype=dtype, elements=int(np.asarray(want).size), max_abs=max_abs, rel_l2=rel,
               max_abs_bound=MAX_ABS[dtype], rel_l2_bound=REL_L2[dtype],
               want_rms=float(np.sqrt(np.mean(np.square(np.asarray(want, np.float64)))))
               if np.asarray(want).size else 0.0)
    RECORDS.append(rec)
    path = os.environ.get("CA_PARITY_LOG")
    if path:
        with open(path, "a") as f:
            f.write(json.dumps(rec) + "\n")
    assert max_abs <= MAX_ABS[dtype], f"{label}: max abs {max_abs:.3g} > {MAX_ABS[dtype]}"
    assert rel <= REL_L2[dtype], f"{label}: rel-L2 {rel:.3g} > {REL_L2[dtype]}"
    return max_abs, rel
