"""libpact: the NVFP4 data flow of PACT's LoRA frozen projections on B200 (sm_100a).

The C ABI is declared in include/pact.h; ``nvfp4_gemm_b200.pact`` is its thin Python
binding (same function names) and ``nvfp4_gemm_b200.layer`` composes the calls into
one decoder layer's forward and backward pass.
"""
from .pact import *  # noqa: F401,F403
from .pact import NVFP4Tensor, WeightCache, PactError, lora_struct  # noqa: F401
