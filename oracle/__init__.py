"""CPU oracle for the Q-GaLore optimizer step and subspace refresh.

TEST INFRASTRUCTURE ONLY: imported by the tests, by the smoke check and by the
CPU-baseline / reference arm of the benchmark, never by the product path.  It
shares no code, header, table or helper with the CUDA implementation.

Pins (each checked by a CPU test against something other than the oracle):
  philox4x32_10         - cuRAND's host Philox4x32-10 generator; numpy's Philox4x64-10
                          for the shared round structure
  bf16_round            - torch's float32 -> bfloat16 conversion
  quant_int4_groups     - hand-worked golden groups, round-trip bound, idempotence
  quant_rowblock_int8   - same, plus ragged last block
  adam_moments          - torch.optim.Adam on the same gradients; closed form at t = 1
  project / backproject - brute-force loops on small non-square inputs
  stochastic_round_update - E[xi(y)] = y over 10^6 draws; the sum over all 2^16 draws is
                          rint of the update (ties included); odd in the update and no
                          drift over a dense grid; integers fixed; clamp
  cossim                - closed forms; scipy.linalg.subspace_angles
  randomized_topr       - exact SVD (LAPACK) when k = min(m, n) and on inputs with a gap
  schedule_after_refresh - scripted CosSim sequences; gamma > 1 gives a fixed interval
  step (composed)       - alpha = 0 leaves W unchanged; mean update over seeds equals
                          alpha * P N / s (unbiasedness at the step level)
  dequant_weight_bf16   - torch's float32 -> bfloat16 conversion of each float32
                          product, groups straddling rows; exact unit / power-of-two /
                          zero scales
  linear_forward / linear_backward_data / linear_backward_weight
                        - brute-force sums on small inputs; integer matrix products
  stochastic_round_rescale - equals stochastic_round_update inside the grid; the sum over
                          all 2^16 draws against the exact value; per-element unbiasedness
                          in groups carried off the grid; zero-scale, NaN and mixed groups
  refresh_moments       - reset and keep; rotation by the identity and by a permutation
  project_right / backproject_right / right-side refresh
                        - brute-force loops; the refresh finds the right singular vectors
  bf16_from_bits / dequant_P_bf16
                        - torch's bfloat16 decoding of every bit pattern; torch's
                          conversion of each INT4 product
  proj_dims / adam_constants / refresh_due
                        - closed forms and the scripted rule
"""
from .qgalore import *  # noqa: F401,F403
from . import qgalore  # noqa: F401
