"""B200-native paged KV-cache decode attention.

The compute path is the C-ABI CUDA library ``libpa.so`` (include/pa.h); this
package is its thin Python binding.  Importing fails if the library is not
built -- there is no CPU fallback.
"""

from ._lib import (  # noqa: F401
    BLOCK_SIZE,
    LIB_PATH,
    PA_ERR_CUDA,
    PA_ERR_INVALID_ARG,
    PA_ERR_NO_BLOCKS,
    PA_ERR_OUT_OF_RANGE,
    PA_ERR_TIMEOUT,
    PA_ERR_UNSUPPORTED,
    PA_OK,
    BlockManager,
    DecodeTuning,
    PagedAttentionError,
    check_copy_pairs,
    copy_blocks,
    decode,
    decode_launch_count,
    decode_plan,
    decode_workspace_size,
    error_string,
    make_workspace,
    prefill,
    prefill_workspace_size,
    reshape_and_cache,
    set_default_tuning,
    swap_blocks,
    tuning,
    version,
)
