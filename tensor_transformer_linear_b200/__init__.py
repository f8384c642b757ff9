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
                   tpl_swiglu_column_linear, tpl_embedding_lookup, tpl_selftest_wait_timeout,
                   tpl_row_linear_scatter, tpl_reduce_slots, tpl_argmax_merge,
                   tpl_column_linear_gather, tpl_reduce_slots_allgather, tpl_reduce_slots_rmsnorm,
                   tpl_fold_norm_scale, Trace, tpl_tp_mlp_fp32,
                   tpl_column_linear_rmsnorm, tpl_column_linear_rmsnorm_workspace_size,
                   rmsnorm_linear_workspace)
from .path import (TPMLP, TPLMHeadRank, TPRankMLP, TPRowParallelAllReduceRank,  # noqa: F401
                   TPRowParallelRank, TPStack,
                   PeerBuffers,
                   exchange_peer_buffers, local_peer_buffers, pack_row_weight, recv_buffer_numel,
                   shard_views, sp_rows, sp_slice, sp_token_owner, stream_barrier)
