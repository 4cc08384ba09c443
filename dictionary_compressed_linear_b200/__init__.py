"""dictionary_compressed_linear_b200 — B200-native forward of a DictLLM projection.

Y = (X D_g) C_l with an NVFP4 dictionary D_g shared by a group of layers and a
sparse NVFP4 coefficient matrix C_l per layer (DictLLM technical review, Eq. (1)),
computed by hand-written sm_100a CUDA kernels behind the C ABI of
``libdictproj.so`` (include/dictproj.h). This package is the thin Python
binding of that ABI; it loads the in-tree library and fails loudly if it is
missing.
"""
from .binding import (  # noqa: F401
    PATH_AUTO, PATH_DECODE, PATH_PREFILL, DECODE_AUTO, DECODE_FUSED, DECODE_SPLIT, dictproj_set_decode_kernels,
    dictproj_get_decode_kernels, IFMT, dictproj_layer_upload_bitmap, dictproj_pack_layer_bitmap,
    dictproj_layer_upload_blocks, dictproj_pack_layer_blocks, dictproj_layer_index_format, dictproj_layer_export_bitmap,
    dictproj_layer_export_blocks, DeviceGroup, DeviceLayer, DictprojError, Group, Layer, LIB_PATH,
    SIGNATURES, dictproj_forward_noalloc, dictproj_forward_noalloc_status, lib,
    dictproj_check, dictproj_check_status, dictproj_diag_phase_times, dictproj_diag_gather_times, dictproj_launch_count, dictproj_selftest_wait_timeout, dictproj_coefficient_stage, dictproj_dictionary_stage, dictproj_dictionary_stage_prefill,
    dictproj_group_reserve_prefill, dictproj_forward, dictproj_rank_for_budget, dictproj_budget,
    dictproj_group_file_write, dictproj_group_file_read, dictproj_layer_file_write, dictproj_layer_file_read,
    dictproj_group_save, dictproj_group_load, dictproj_layer_save, dictproj_layer_load, dictproj_forward_batch, dictproj_forward_batch_stages, dictproj_decode_batch_plan, dictproj_forward_path, dictproj_forward_status,
    dictproj_group_export, dictproj_group_info, dictproj_group_packed_sizes, dictproj_group_upload,
    dictproj_last_error, dictproj_layer_export, dictproj_layer_info, dictproj_layer_packed_entries,
    dictproj_layer_upload, dictproj_pack, dictproj_pack_group, dictproj_pack_group_host,
    dictproj_pack_layer, dictproj_pack_layer_host, dictproj_pack_layer_bitmap_host, dictproj_pack_layer_blocks_host, dictproj_pack_layer_fmt_host, CFMT, dictproj_layer_upload_fmt,
    dictproj_pack_layer_fmt, dictproj_layer_format, dictproj_layer_export_fmt, dictproj_status_string, dictproj_version,
)
