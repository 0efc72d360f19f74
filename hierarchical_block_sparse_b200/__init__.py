"""B200 (sm_100a) PISA pyramid Top-K block-sparse attention.

The compute path is the C-ABI CUDA library ``libpisa.so`` (include/pisa.h);
``pisa`` is its thin Python binding. PyTorch provides device memory and
streams only.
"""
from . import pisa  # noqa: F401
from .pisa import (  # noqa: F401
    PisaCfg, PisaError, make_cfg, cfg_for, forward, alloc_outputs,
    pisa_num_levels, pisa_level_nodes, pisa_level_offset, pisa_pyramid_rows,
    pisa_build_pyramid, pisa_select, pisa_sparse_attn, pisa_forward, pisa_bsa_select,
    pisa_build_pyramid_prefix, pisa_pyramid_append, pisa_decode, pisa_status_string, pisa_version,
    pisa_workspace_bytes, pisa_select_ws, pisa_sparse_attn_ws, pisa_forward_ws, alloc_workspace,
    pisa_workspace_status,
)

__version__ = "0.1.0"
