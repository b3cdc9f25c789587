// pa_copy_blocks: copy whole physical pages (every kv head, every slot; K and
// V) -- the device half of a copy-on-write fork.
//
// What is PagedAttention?, "Copy-on-Write Memory Forking": pages are forked
// only when parallel outputs diverge.  PagedAttention Internals,
// "Copy-on-Write and Prefix Sharing".
//
// With the [page][kv_head][slot][dim] layout a page is one contiguous run of
// num_kv_heads * block_size * head_dim elements in each cache, so a pair is
// two plain memory copies.  CTA (x, pair) copies a contiguous slice of the K
// page and the same slice of the V page, kUnroll 16-byte chunks per thread,
// all loads issued before the stores.
#include "device.cuh"
#include "pa_internal.h"

namespace pa {
namespace {

constexpr int kThreads = 256;
constexpr int kUnroll = 4;

__global__ void __launch_bounds__(kThreads)
    copy_blocks_kernel(uint4* __restrict__ key_cache, uint4* __restrict__ value_cache,
                       const int64_t* __restrict__ block_mapping, int64_t num_pairs, int64_t page_chunks,
                       int num_blocks, int32_t* status) {
  const int64_t base = (int64_t)blockIdx.x * kThreads * kUnroll + threadIdx.x;
  for (int64_t pair = blockIdx.y; pair < num_pairs; pair += gridDim.y) {
    const int64_t src = __ldg(block_mapping + 2 * pair);
    const int64_t dst = __ldg(block_mapping + 2 * pair + 1);
    if (src < 0 || src >= num_blocks || dst < 0 || dst >= num_blocks) {
      if (blockIdx.x == 0 && threadIdx.x == 0) flag_status(status, PA_DEV_BAD_PAIR);
      continue;
    }
    uint4 k[kUnroll], v[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int64_t i = base + (int64_t)u * kThreads;
      if (i < page_chunks) {
        k[u] = key_cache[src * page_chunks + i];
        v[u] = value_cache[src * page_chunks + i];
      }
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int64_t i = base + (int64_t)u * kThreads;
      if (i < page_chunks) {
        key_cache[dst * page_chunks + i] = k[u];
        value_cache[dst * page_chunks + i] = v[u];
      }
    }
  }
}

}  // namespace
}  // namespace pa

using namespace pa;

extern "C" pa_status pa_copy_blocks(void* key_cache, void* value_cache, const int64_t* block_mapping,
                                    int32_t num_pairs, int32_t num_blocks, int32_t block_size,
                                    int32_t num_kv_heads, int32_t head_dim, pa_dtype dtype, int32_t* dev_status,
                                    void* stream) {
  const int eb = dtype_bytes(dtype);
  if (eb == 0) return fail(PA_ERR_INVALID, "copy_blocks: bad dtype %d", (int)dtype);
  if (num_pairs < 0 || num_blocks < 0 || block_size <= 0 || num_kv_heads <= 0 || head_dim <= 0)
    return fail(PA_ERR_INVALID, "copy_blocks: bad sizes");
  if (num_pairs == 0) return PA_OK;
  if (!key_cache || !value_cache || !block_mapping) return fail(PA_ERR_INVALID, "copy_blocks: NULL pointer");
  if (!aligned16(key_cache) || !aligned16(value_cache))
    return fail(PA_ERR_INVALID, "copy_blocks: caches must be 16-byte aligned");
  const int64_t page_bytes = (int64_t)num_kv_heads * block_size * head_dim * eb;
  if (page_bytes % 16 != 0) return fail(PA_ERR_INVALID, "copy_blocks: page bytes not a multiple of 16");
  const int64_t page_chunks = page_bytes / 16;
  const int64_t gx = (page_chunks + kThreads * kUnroll - 1) / (kThreads * kUnroll);
  if (gx > 0x7fffffffLL) return fail(PA_ERR_UNSUPPORTED, "copy_blocks: page too large");
  dim3 grid((unsigned)gx, (unsigned)(num_pairs < 65535 ? num_pairs : 65535));
  copy_blocks_kernel<<<grid, kThreads, 0, (cudaStream_t)stream>>>((uint4*)key_cache, (uint4*)value_cache,
                                                                   block_mapping, num_pairs, page_chunks, num_blocks,
                                                                   dev_status);
  cudaError_t err = cudaGetLastError();
  if (err != cudaSuccess) return fail(PA_ERR_CUDA, "copy_blocks launch: %s", cudaGetErrorString(err));
  return PA_OK;
}
