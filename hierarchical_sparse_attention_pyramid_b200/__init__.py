"""B200-native Lighthouse attention layer (hierarchical sparse attention pyramid).

The compute path is the CUDA library ``liblh.so`` (C ABI, ``include/lh.h``);
this package only marshals torch tensors into its calls.  ``synth`` draws the
seeded synthetic inputs.
"""

from .api import (Buffers, Layer, LighthouseAttentionFn, attn_bwd, attn_bwd_rows, attn_fwd, attn_fwd_rows,  # noqa: F401
                  backward, check_error, forward, gather, lighthouse_attention, plan, pool_adjoint, pyramid_pool,
                  scatter_back, scatter_back_adjoint, score_topk)
from . import pisa  # noqa: F401
