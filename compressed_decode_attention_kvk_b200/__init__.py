"""KV-Kaizen compressed MLA cache on B200: quantise-on-write and compressed decode attention.

The computation lives in ``libkvk.so`` (CUDA, sm_100a, C ABI in include/kvk.h);
``kvk`` is its Python binding.
"""
from .kvk import (KVK_BF16, KVK_F16, KVK_F32, KVK_FLAG_KEEP_INDEX, KVK_FLAG_NONFINITE,  # noqa: F401
                  KVK_FLAG_SEQ_LEN, KVK_FLAG_WRITE_RANGE, KVK_PATH_AUTO, KVK_PATH_CUDA_CORE,
                  KVK_PATH_TENSOR, KVK_PATH_TENSOR_GENERAL, KvkError, Layout, kvk_absorb, kvk_create_layout, kvk_decode_path_for,
                  kvk_decode_workspace_bytes, kvk_destroy, kvk_get_layer_info, kvk_mla_decode,
                  kvk_mla_decode_append, kvk_mla_decode_noalloc,
                  kvk_quant_write, kvk_read_status, kvk_set_decode_ctas, kvk_set_decode_path,
                  kvk_status_string)
