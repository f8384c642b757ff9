"""Tensor-parallel sharded linears of a transformer block on one B200 (sm_100a).

The product is ``libtpl.so`` (C ABI, ``include/tpl.h``); this package is its
ctypes binding (``_tpl``), the block orchestration (``path``) and the build
script (``build``).
"""
from ._tpl import (EXPORTED, Partition, TplError, lib, lmhead_workspace,  # noqa: F401
                   tpl_column_linear, tpl_get_device_status, tpl_launch_count,
                   tpl_lmhead_argmax, tpl_lmhead_argmax_static, tpl_lmhead_workspace_size, tpl_partition_subparams,
                   tpl_rmsnorm, tpl_row_linear_reduce, tpl_status_string, LIB_PATH,
                   tpl_row_linear_reduce_scatter, tpl_column_linear_allgather,
                   tpl_swiglu_column_linear, tpl_embedding_lookup, tpl_selftest_wait_timeout)
from .path import TPMLP, TPStack, pack_row_weight, shard_views  # noqa: F401
