"""Absorbed MLA decode over a paged latent cache on B200 (sm_100a).

The compute lives in ``libmla_b200.so`` (C ABI in ``include/mla.h``); this
package holds the ctypes binding (``_lib``), the in-tree build script
(``build``), a decode-step driver over the four calls (``layer``) and the seeded
input generator (``synth``).
"""

from ._lib import (MLA_BF16, MLA_FP32, MLA_ROPE_HALF, MLA_ROPE_INTERLEAVED, Dims, MlaError,  # noqa: F401
                   PagedCache, mla_absorb_q, mla_cache_append, mla_decode_attn,
                   mla_get_device_error, mla_unabsorb_out, mla_workspace_init,
                   mla_workspace_size, status_string)
