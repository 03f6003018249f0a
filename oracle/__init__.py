"""Plain fp64 CPU oracle for Hessian-aware int4 weight quantization (GPTQ) and the
Bf16TrilDiagF32 Hessian codec.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path (``libhq.so`` and its Python
binding) imports, links or calls this package.  Only ``tests/``, ``__graft_entry__.smoke()``
and the CPU-baseline / reference legs of ``bench.py`` may use it.

Every function is a direct, unblocked restatement of what the source pages define; see
``oracle/hq_oracle.py`` for the citations and for the readings taken where the pages are
silent.  It shares no code, header, table or constant with the CUDA path.
"""

from .hq_oracle import *  # noqa: F401,F403
from .hq_oracle import __all__  # noqa: F401
