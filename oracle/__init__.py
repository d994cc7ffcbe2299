"""Oracle for video sparse attention (VSA).

TEST INFRASTRUCTURE ONLY.  This package is a plain, slow CPU restatement of
what the VSA hot path computes, used to check the CUDA path.  Only the test
suite, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` may
import it.  The CUDA library never calls it, and it shares no code with it.

Modules
-------
vsa_oracle : NumPy float64 restatement, stage by stage (tile permutation,
             cube pooling, coarse attention, top-k, block-sparse fine
             attention, gated combine, untile).
vsa_loops  : a second restatement with explicit Python loops and no BLAS, for
             tiny shapes only; it cross-checks ``vsa_oracle``.
vsa_backward : gradients of the forward with the selection held fixed.
vsa_linear : the low-rank linear compensation branch (sparse + linear).
vsa_dit    : the QKV and output projections of a DiT block around VSA.

Parity status per function is listed in each module's header.
"""
