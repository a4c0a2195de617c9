"""fp64 CPU oracle for the KronQ per-layer quantization path.

TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check in
``__graft_entry__`` and the CPU-baseline leg of ``bench.py`` may import this
package.  The product (the CUDA library and its Python binding) never calls
it, and it shares no code with the CUDA path: both only read the seeded
inputs of the ``synth`` package.

Each function is the plain definition of its step (numpy, float64), written
from the KronQ pages:

* KronQ summary (hyper.ai), "Method": the empirical Fisher, the K-FAC
  factorisation H ~ H_X (x) H_G (Eq. 7), the Kronecker-factored objective,
  the column-wise OBS update (Prop. 1), bidirectional incoherence processing
  (Eqs. 11-12) and the sensitivity score s = tr(H_G) tr(H_X) (Eq. 14).
* KronQ review (pith.science), appendix fragments: Algorithm 2 (damping,
  inverse Cholesky, block loop), proofs of Proposition 1 and Theorem 1.
* KronQ README (GitHub), "Reproduce from scratch" and "Model zoo": the
  asymmetric per-channel / group-128 grid, packed int4/int2, --alpha 0.25,
  --incoh_mode, --inter_layer_mp.

Where the pages leave a step open, the reading taken is stated in the
function's docstring.  Every function here is pinned by a ``-m "not gpu"``
test against something other than itself (closed forms, invariants,
brute force on tiny inputs, textbook matrices) -- except where a docstring
says "parity unpinned".
"""

from . import covariance, transform, biip, sensitivity, cholesky, quantizer, pack, pipeline, diagnostics, deploy  # noqa: F401
