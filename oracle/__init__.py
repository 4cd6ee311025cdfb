"""Plain float64 CPU oracle for KV-vector quantization (RotorQuant and TurboQuant).

TEST INFRASTRUCTURE ONLY. Nothing in the product imports this package: only the
tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` may
use it. It shares no code with the CUDA library (``kv_cache_vector_rq_b200``),
and never calls it.

Each step is written in the order and notation of the source pages, one
definition at a time, with numpy (float64) doing the arithmetic. The pages are:

* "TurboQuant + RotorQuant" -- the README of the RotorQuant repository
  (sections "How TurboQuant Works", "How RotorQuant Works", "FMA Count (d=128)",
  "Codebook Calibration Fix", "Non-Commutative Algebra Bug Fix",
  "MSE Quality (after codebook fix)").
* "TurboQuant 论文解读" -- a walkthrough blog of the TurboQuant paper
  (sections "随机旋转（Lemma 1）", "Beta 分布", "MSE 标量量化（Theorem 1）",
  "QJL 内积无偏估计（Theorem 2）", "与理论上界的比较", "简单复现 demo").
* The summary page of arXiv 2504.19874 (TurboQuant), section "方法"
  (Algorithm 1 and Algorithm 2 described in prose).
* "TurboQuant и PolarQuant: математика квантизации KV-кэша в LLM" -- the
  paragraph on building codebooks with Lloyd's algorithm, the attention
  formula in "Проблема KV-кэша в трансформерах", and PolarQuant
  ("Полярное преобразование", "Алгоритм PolarQuant на практике").

Modules:
  rng       counter-based splitmix64 + Box-Muller normals (parameter draws)
  clifford  generic Cl(3,0) geometric product, reverse, rotor sandwich
  codebook  Lloyd-Max centroids for the rotated-coordinate density
  params    random unit rotors, random orthogonal Pi, QJL Gaussian matrix
  codes     nearest-centroid scalar quantization and LSB-first bit packing
  rq        RotorQuant quantize / dequantize
  tq        TurboQuant-mse, TurboQuant-prod (QJL on the residual)
  score     inner products <q, k_hat> from packed codes, two ways
  attention decode attention softmax(q K_hat^T scale) V_hat over a packed cache
  polar     PolarQuant: preconditioning, recursive polar transform, angle codebooks
  rq4       RotorQuant in the pages' four-grade layout (172 indices per vector)

Parity status of every function: pinned (see tests/test_oracle_*.py). No
function here is "parity unpinned".
"""

from . import rng, clifford, codebook, params, codes, rq, tq, score, attention, polar, rq4  # noqa: F401
