"""fp64 CPU oracle for the shared-state GDN beam decode.

TEST INFRASTRUCTURE, not product code.  Only the test suite, the package's
smoke check and the CPU-baseline leg of the benchmark may import, call, link or
run anything in this folder.  It shares no code with the CUDA library and
imports nothing from it.

Modules
-------
gdn     numpy fp64 reference: prefill, full-state beam tree, replay
        formulation (for the replay == full-state identity), ancestry walk,
        and for the folding extension the shared-ancestor depth and the
        shared ancestor's full state.
cref    ctypes loader for ``c/gdn_fullstate.c``: the same full-state beam tree
        in plain C (fp64, OpenMP over beams), the timed CPU baseline.
beam    beam selection: the W best children (fp32 scores, ties to the smaller
        flat index), numpy sort.

Parity pins (what each function is checked against, tests/test_oracle_*.py):
closed form of one step in exact rational arithmetic; the textbook gated delta
rule written in its matrix form; the delta rule's exact-recall property;
replay == full state; W = 1 == sequential GDN; alpha = 1, beta = 0 leaves S0
unchanged; beta = 0 is a pure gate product; ancestry by brute-force tree
construction; linearity in (S0, v); permutation equivariance of beam labels;
a hand-worked scalar example (tests/golden/).  Beam selection: brute-force
ordering of Python tuples, fp32 rounding ties, signed zeros, NaN and -inf.
Folding: hand-built trees and a brute-force path walk for the shared depth;
the prefill recurrence for a single beam's folded state; decoding on from a
folded state equals the unfolded decode.
"""
from . import gdn  # noqa: F401
