"""Float64 CPU oracle of the KVSculpt distillation solve (test infrastructure).

TEST INFRASTRUCTURE ONLY.  Nothing in the product path may import, call or
execute this package: only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` use it.  It shares no code with the CUDA
library (``kv_cache_compression_kvsculpt_b200``); the two meet only through the
seeded inputs of ``workload``.

Every function is a plain numpy float64 restatement of a step described on the
page "KVSculpt: KV Cache Compression as Distillation" (the structured summary,
section 2 "Methodology", and the abstract).  Matrix products, ``exp``/``log``,
a sort and a dense symmetric solve are taken from numpy/scipy as library
primitives; there is no blocking, fusion or reordering beyond what the
definitions state.

Readings of points the pages leave open (each one is also listed in the
design notes of the repository):

* Chunk-local attention: targets (Y, l) and the compressed outputs
  (Y_hat, l_hat) are attention over the compress zone only, so a chunk can be
  merged with the retain zone and later tokens by its log-sum-exp.
* Score scale s = 1/sqrt(d); log-sum-exp in natural log of the scaled scores.
* Loss = w_out/(n_q d) ||Y_hat - Y||_F^2 + w_lse/n_q ||l_hat - l||^2
  (means, weights 1).
* Ridge: V_c = (A^T A + lam I)^-1 A^T Y with absolute lam.
* Importance = column sums of the compress-zone attention probabilities over
  all training queries; top-k ties go to the lower position; indices are
  returned ascending.
* Initial V_c = ridge fit at the initial keys (iteration 0 = Select+Fit).
* L-BFGS: history h, H0 = gamma I with gamma = s^T y / y^T y of the newest pair,
  pair stored only if s^T y > 1e-10 y^T y, non-descent direction replaced by
  -g, first trial step 1 (min(1, 1/||g||) with empty history), Armijo
  sufficient decrease with halving and at most max_bt trials; a failed search
  leaves x unchanged, clears the history and flags LS_FAIL.  The history
  persists across value re-fits unless ``persist_history`` is 0.
* Allocation: k_b proportional to MSE_b^alpha (alpha = 0.5) under the total
  budget, clamped to [k_min, k_max_b] by water-filling, rounded by largest
  remainder with ties to the lower problem index.

Parity pins for every function live in ``tests/test_oracle_*.py``; the
end-to-end trajectory of ``compress`` is pinned only by those of its parts
(no page prints a worked example), i.e. "parity unpinned" for the trajectory
as a whole.
"""
from .kvsculpt import *  # noqa: F401,F403
from .kvsculpt import __all__  # noqa: F401
