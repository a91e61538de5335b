"""csla: CSA/HCA hybrid compressed attention (compress -> lightning indexer ->
top-k -> MQA with window and sink, plus the state cache) for B200 (sm_100a).

The compute lives in libcsla.so (hand-written CUDA behind the C ABI of
include/csla.h); `csla` is the ctypes binding with the same entry-point
names, `layer` owns device buffers through torch.
"""
from . import csla
from .csla import (csla_compress_append, csla_csa_attend, csla_device_error, csla_hca_attend,
                   csla_indexer_scores, csla_strerror, csla_topk_select, csla_version,
                   csla_workspace_size)
from .layer import CompressParams, LayerBuffers, LayerShape, dtype_code

__all__ = ["csla", "csla_compress_append", "csla_indexer_scores", "csla_topk_select", "csla_csa_attend",
           "csla_hca_attend", "csla_workspace_size", "csla_device_error", "csla_strerror", "csla_version",
           "LayerBuffers", "LayerShape", "CompressParams", "dtype_code"]
