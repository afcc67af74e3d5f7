"""CPU oracle for the DCKV per-token codec -- TEST INFRASTRUCTURE ONLY.

A plain, slow, step-by-step definition of what the codec computes, in fp64 numpy plus
a small scalar C rANS coder (``rans_oracle.c``).  It shares no code with the CUDA
library and does not import it.  Only the test-suite, ``__graft_entry__.smoke()`` and
the CPU-baseline leg of ``bench.py`` may import or call anything in this package; the
product path never does.

Every function cites the passage of "DCKV: Learned Transform Coding of the Prompt KV
Cache in Hybrid Language Models" (trove.briskstack.com summary, section "How it
works") that it follows.  Where the pages leave a step open, the reading taken is
stated in the function's docstring.
"""
from .codec import *  # noqa: F401,F403
from .fit import *  # noqa: F401,F403
from .codec import __all__ as _all_codec
from .fit import __all__ as _all_fit

__all__ = list(_all_codec) + list(_all_fit)
