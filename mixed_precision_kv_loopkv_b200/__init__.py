"""LoopKV decode path on B200 (sm_100a).

LoopKV: Loop-Aware KV Cache Compression for Serving Looped Transformers
(Abstract): per-(loop, layer) KV cells stored 4-bit (split high/low 2-bit
planes), 2-bit, or as a reuse of the final loop's cell, executed by one fused
decode kernel.  The CUDA library (libloopkv.so, C ABI in include/loopkv.h)
does all the work; this package only marshals arguments and sequences the
per-cell calls of a looped decode step.
"""

from .loopkv import (  # noqa: F401
    KIND_CODES,
    LIB_PATH,
    LOOPKV_CELL_BF16,
    LOOPKV_CELL_Q2,
    LOOPKV_CELL_Q4,
    LOOPKV_CELL_REUSE,
    LOOPKV_DEVERR_BLOCK_ID,
    LOOPKV_DEVERR_RANGE,
    LOOPKV_DEVERR_SEQ_LEN,
    LOOPKV_DEVERR_TIMEOUT,
    LOOPKV_FLAG_PDL,
    LOOPKV_FLAG_SELECT_BLOCK,
    LOOPKV_FLAG_SELECT_GROUP,
    KVCells,
    LoopKVError,
    library,
    loopkv_append_decode_attention,
    loopkv_decode_attention,
    loopkv_decode_splits,
    loopkv_plan_cells,
    loopkv_quantize_append,
    loopkv_record_bytes,
    loopkv_selftest_wait_timeout,
    loopkv_status_string,
    mask_words,
)
from .step import LoopedDecodeStep, prefill  # noqa: F401
