"""Quantized gated delta-rule decode (GDN / KDA) on B200.

The CUDA library ``libstq.so`` (C ABI in ``include/stq.h``) holds the packed
state pool and the kernels; ``stq`` is its thin Python binding and ``synth``
the seeded input generator.
"""
from . import synth  # noqa: F401
from .stq import (  # noqa: F401
    STQ_GDN, STQ_KDA, Pool, StqError, load, stq_decode_readout, stq_decode_step, stq_decode_step_split,
    stq_decode_writeback, stq_dequantize_state, stq_desc_bytes, stq_pool_join,
    stq_allocate_bits, stq_lifetime_weight, stq_decode_step_static, stq_decode_step_host,
    stq_decode_step_host_block, stq_host_block_layout,
    stq_export_slot, stq_import_slot, stq_last_error, stq_launch_count, stq_page_layout,
    stq_pool_bytes, stq_pool_check, stq_pool_create, stq_pool_destroy, stq_quantize_state,
    stq_status_str,
)
