"""Chunkwise-parallel (TFLA) mLSTM forward/backward for NVIDIA B200 (sm_100a).

The compute lives in the C-ABI CUDA library ``libmlstm.so`` (declared in
``include/mlstm.h``); ``binding`` is its thin Python binding.  The library is
loaded on first use, so importing this package never needs a GPU.
"""

from .binding import (  # noqa: F401
    BF16, EXP, FP32, SIG, MLSTMError, backward, forward, load, mlstm_bwd,
    mlstm_bwd_launch_count, mlstm_bwd_workspace_size, mlstm_fwd, mlstm_fwd_launch_count,
    mlstm_fwd_workspace_size, mlstm_saved_layout, mlstm_saved_size, mlstm_status_string,
    saved_views,
)
