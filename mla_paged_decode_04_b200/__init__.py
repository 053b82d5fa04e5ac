"""B200 (sm_100a) MLA decode over a paged latent KV cache.

The compute path is the CUDA library ``libmla_decode.so`` (C ABI in
``include/mla_decode.h``); this package only binds it. ``inputs`` draws
seeded synthetic workloads.
"""
from ._lib import (MLA_DEV_BAD_PAGE, MLA_DEV_BAD_QLEN, MLA_DEV_BOUNDS, MLA_DEV_SEQ_TOO_LONG,  # noqa: F401
                   MLA_DEV_TIMEOUT, bounds_checked,
                   MlaDecoder, MlaPrefill, mla_prefill, mla_prefill_partial, mla_prefill_plan,
                   MlaError, MlaPlan, alloc_workspace, last_cuda_error, mla_decode, mla_decode_plan,
                   mla_decode_combine, mla_decode_partial, mla_decode_plan_custom, mla_decode_plan_window,
                   mla_decode_status, mla_version, status_string, kv_pack, kv_amax)
