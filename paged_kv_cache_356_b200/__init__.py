"""B200-native paged KV cache decode path.

The C ABI (include/pa.h, libpa_b200.so) holds the whole path: the host
ref-counted page allocator and the sm_100a kernels for writing tokens into
pages, copying pages (copy-on-write) and paged decode attention.  This
package is its thin Python binding (``binding``), the in-tree build
(``build``), a driver that runs a workload trace through the C ABI
(``runner``) and the seeded synthetic workloads (``workloads``).
"""
from .binding import (BlockAllocator, PagedAttentionError, PagedAttentionOOM, SequenceNotFound,  # noqa: F401
                      pa_block_alloc_allocate_sequence, pa_block_alloc_append_token, pa_block_alloc_append_tokens,
                      pa_block_alloc_block_table,
                      pa_block_alloc_block_tables, pa_block_alloc_create, pa_block_alloc_destroy,
                      pa_block_alloc_fork, pa_block_alloc_free_pool, pa_block_alloc_free_sequence,
                      pa_block_alloc_num_free, pa_block_alloc_num_sequences, pa_block_alloc_num_tokens,
                      pa_block_alloc_prefix_plan, pa_block_alloc_ref_count, pa_block_alloc_slot_mapping,
                      pa_block_alloc_stats, pa_copy_blocks, pa_decode, pa_decode_fixed_scratch,
                      pa_decode_partitions, pa_decode_reduce, pa_decode_shared_prefix, pa_decode_verify,
                      pa_decode_verify_workspace_size, pa_decode_workspace_size, pa_reshape_and_cache,
                      pa_set_decode_kernel, pa_set_decode_tiling, pa_set_shared_prefix_kernel,
                      pa_set_verify_path, pa_set_verify_tiling, pa_version, prefix_plan_to_device)
