"""CPU oracle for Joint Subspace Sparse Attention decode and calibration.

TEST INFRASTRUCTURE ONLY. Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU
baseline leg may import it. The CUDA library and its Python binding never use it and it uses
nothing of theirs; the two sides share only the seeded input generator in ``synth/``.

Precision: float64 throughout. Every function cites the page section or equation it follows.

Parity pins (tests marked ``not gpu``): E4M3 encoder exhaustively against torch's CPU cast and
the format's closed forms; the second moments and the calibration Grams against the pair sum of
squared score errors that eqs. (2)-(3) define (with planted per-head, centred and mis-indexed
moments caught); ``M M^T = I_r``; the Ky Fan closed form of the marginal objective at
the optimum; brute-force projector search for tiny ``d``; the bound of eq. (4) on random
projectors; LAPACK against an independent Jacobi solver; selection against brute-force sorting
with ties; ``r = d`` without FP8 reproducing the exact group-mean logits ranking; ``r = d`` with
``B = L`` reproducing dense attention; dense attention against torch's CPU scaled-dot-product
attention with grouped heads; paged against unpaged addressing; the printed 6.25% scoring-cache
size; the sign rule of the basis rows; bf16 scores through a coordinate basis against plain dot
products. Every function here has a pin. The pages print no worked example, so no end-to-end value
is compared with a printed number: the whole decode step is pinned through its special cases
(``r = d`` without FP8 gives the exact group-mean logits; ``r = d`` with ``B = L`` gives dense
attention, itself pinned to torch's CPU SDPA) and through the pins of each step it composes.
"""

from . import fp8, jssa, jacobi  # noqa: F401
