"""Float64 CPU oracle for the forward Differential Attention V2 operator.

TEST INFRASTRUCTURE ONLY. Nothing on the product path imports, calls or links this
package: only the tests, the smoke check and the benchmark's CPU-baseline leg use it.
It shares no code with the CUDA library and imports nothing from it.

Two independent implementations live here:
  * `diffattn_f64` -- NumPy float64, the plain definition written out (scores, mask,
    two-pass softmax per branch, subtract, multiply by V), blocked only over query rows so
    that long sequences fit in memory.
  * `brute` -- stdlib-Python loops over lists, for tiny inputs, written from the lesson's
    list-of-lists toy; it is the second, independent check on the first.

Every function cites the passage of the pages it follows. All functions are pinned by
tests against what the pages and the mathematics fix (closed forms, reductions to a
library routine, invariants, a worked example); none says "parity unpinned".
"""
from . import brute, diffattn_f64  # noqa: F401
