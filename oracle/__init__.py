"""Plain fp64 CPU oracle for GPTQ layer-wise weight quantization and group min-max RTN.

TEST INFRASTRUCTURE ONLY. Nothing in the product path may import this package: only the
tests under ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` / reference leg
of ``bench.py`` use it. It shares no code, tables or constants with the CUDA library; the
two meet only in the seeded inputs they are both given.

Everything here is written for a reader to check by eye against the source pages:

* "大模型量化技术原理：GPTQ、AWQ、GGUF核心机制与部署选型指南" (0539edu.com/news/6111416),
  §2.1 (the affine quantizer and its INT8 worked example), §3.1 (layer objective ‖WX − W_qX‖²),
  §4.2 (group_size and its fp16 scale + zero storage cost).
* The GPTQ deep-dive page (hncyxsy.com/news/243429), §2.1 (Taylor/Hessian error model),
  §2.2 (OBS compensation with the inverse Hessian), §2.4 (fixed order, lazy batch updates,
  Cholesky), §3.1 (the four-step per-layer algorithm, H = 2XXᵀ + λI), §3.3 (group size,
  desc_act, damp_percent).
* "AWQ、MinMax、GPTQ 三大校准算法原理与选型指南" (gtnt.cn/news/115337), §4 (Hessian collection,
  column-wise quantization with compensation, block_size a multiple of group_size,
  perc_damp 0.01).
* The calibration-methods practitioner page (bhfrc.com/news/5741), §2.2 (group min-max),
  §2.3 (GPTQ in descending-Hessian-diagonal order, blocksize 128).

Arithmetic is fp64 throughout; inputs are the exact fp16/fp32 values. Library primitives
(numpy matmul, LAPACK Cholesky, a triangular solve, a stable sort) serve as single steps.

Modules:
  quantizer  the asymmetric min-max quantizer shared by RTN and GPTQ
  rtn        group min-max round-to-nearest, INT4 packing, storage accounting
  hessian    H = 2·XᵀX
  factor     damping and the upper Cholesky factor of H_d⁻¹
  gptq       act_order permutation, unblocked OBS reference, blocked (lazy) reference,
             output assembly
  loss       layer reconstruction loss tr(ΔHΔᵀ)/tr(WHWᵀ)
  w4a16      the W4A16 layer that consumes the output: fp16 reconstruction and X·Ŵᵀ
  awq        AWQ-lite: activation-aware channel scales, grid search over α
  sequential layer-by-layer GPTQ of a stack of MLP blocks, each layer's Hessian from the
             outputs of the already-quantized layers before it

Every function is pinned by a ``-m "not gpu"`` test in ``tests/test_oracle_*.py`` against
something other than itself (worked example, closed forms, brute force, invariants).
"""

from . import quantizer, rtn, hessian, factor, gptq, loss, w4a16, sequential, awq  # noqa: F401
