"""CPU oracle for the Sparse-BitLinear operator (test infrastructure only).

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline
legs may import this package.  See ``oracle/sbl_oracle.py``.
"""
from .sbl_oracle import *  # noqa: F401,F403
from .sbl_oracle import (absmean_gamma, act_quant, backward_dw, backward_dx,  # noqa: F401
                         bf16_to_f32, effective_weight, forward, forward_acc,
                         forward_out, gemv_packed, nm_mask, pack, packed_layout,
                         ternary, unpack)
