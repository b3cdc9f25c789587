// pa_reshape_and_cache: scatter new tokens' K and V rows into their physical
// slots of the paged cache.
//
// PagedAttention Internals, "2. The Dynamic Block Table": new tokens' K/V land
// in pages taken on demand from the free-page pool; the slot of a token is
// its page times the block size plus its offset in the block.
//
// Data movement only: one thread moves one 16-byte chunk of a (token, kv head)
// row of K and the matching chunk of V.  A CTA covers whole rows; rows of a
// token share its slot, read once per row from a broadcast load.
#include "device.cuh"
#include "pa_internal.h"

namespace pa {
namespace {

constexpr int kThreads = 256;

__global__ void __launch_bounds__(kThreads)
    reshape_and_cache_kernel(const uint4* __restrict__ key, const uint4* __restrict__ value,
                             int64_t key_stride_chunks, int64_t value_stride_chunks,
                             const int64_t* __restrict__ slot_mapping, int64_t num_rows, int num_kv_heads,
                             int chunks_per_row, int rows_per_cta, int64_t num_slots, int block_size,
                             uint4* __restrict__ key_cache, uint4* __restrict__ value_cache,
                             int32_t* status) {
  // A kernel launched after this one as a programmatic dependent (the decode
  // that reads these rows waits for this grid before it reads anything) may
  // start its own set-up now.
  if (threadIdx.x == 0) asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory");
  const int local_row = threadIdx.x / chunks_per_row;
  const int chunk = threadIdx.x - local_row * chunks_per_row;
  if (local_row >= rows_per_cta) return;
  const int64_t row = (int64_t)blockIdx.x * rows_per_cta + local_row;  // token * num_kv_heads + head
  if (row >= num_rows) return;
  const int64_t token = row / num_kv_heads;
  const int head = (int)(row - token * num_kv_heads);
  const int64_t slot = __ldg(slot_mapping + token);
  if (slot < 0) return;  // padding token
  if (slot >= num_slots) {
    if (chunk == 0) flag_status(status, PA_DEV_BAD_SLOT);
    return;
  }
  const int64_t page = slot / block_size;
  const int64_t offset = slot - page * block_size;
  const int64_t src_k = token * key_stride_chunks + (int64_t)head * chunks_per_row + chunk;
  const int64_t src_v = token * value_stride_chunks + (int64_t)head * chunks_per_row + chunk;
  const int64_t dst = ((page * num_kv_heads + head) * block_size + offset) * chunks_per_row + chunk;
  const uint4 k = __ldg(key + src_k);
  const uint4 v = __ldg(value + src_v);
  key_cache[dst] = k;
  value_cache[dst] = v;
}

}  // namespace
}  // namespace pa

using namespace pa;

extern "C" pa_status pa_reshape_and_cache(const void* key, const void* value, int64_t key_token_stride,
                                          int64_t value_token_stride, const int64_t* slot_mapping,
                                          int64_t num_tokens, void* key_cache, void* value_cache,
                                          int32_t num_blocks, int32_t block_size, int32_t num_kv_heads,
                                          int32_t head_dim, pa_dtype dtype, int32_t* dev_status, void* stream) {
  const int eb = dtype_bytes(dtype);
  if (eb == 0) return fail(PA_ERR_INVALID, "reshape_and_cache: bad dtype %d", (int)dtype);
  if (num_tokens < 0 || num_blocks < 0 || block_size <= 0 || num_kv_heads <= 0 || head_dim <= 0)
    return fail(PA_ERR_INVALID, "reshape_and_cache: bad sizes");
  if (num_tokens == 0) return PA_OK;
  if (!key || !value || !slot_mapping || !key_cache || !value_cache)
    return fail(PA_ERR_INVALID, "reshape_and_cache: NULL pointer");
  const int64_t row_bytes = (int64_t)head_dim * eb;
  if (row_bytes % 16 != 0) return fail(PA_ERR_INVALID, "reshape_and_cache: head_dim*elem not a multiple of 16 B");
  if (!aligned16(key) || !aligned16(value) || !aligned16(key_cache) || !aligned16(value_cache))
    return fail(PA_ERR_INVALID, "reshape_and_cache: pointers must be 16-byte aligned");
  const int64_t row_elems = (int64_t)num_kv_heads * head_dim;
  if (key_token_stride < row_elems || value_token_stride < row_elems ||
      (key_token_stride * eb) % 16 != 0 || (value_token_stride * eb) % 16 != 0)
    return fail(PA_ERR_INVALID, "reshape_and_cache: token strides must cover a token and be 16-byte multiples");
  const int chunks_per_row = (int)(row_bytes / 16);
  if (chunks_per_row > kThreads) return fail(PA_ERR_UNSUPPORTED, "reshape_and_cache: head_dim too large");
  const int rows_per_cta = kThreads / chunks_per_row;
  const int64_t num_rows = num_tokens * num_kv_heads;
  const int64_t grid = (num_rows + rows_per_cta - 1) / rows_per_cta;
  if (grid > 0x7fffffffLL) return fail(PA_ERR_UNSUPPORTED, "reshape_and_cache: too many tokens");
  reshape_and_cache_kernel<<<(unsigned)grid, kThreads, 0, (cudaStream_t)stream>>>(
      (const uint4*)key, (const uint4*)value, key_token_stride * eb / 16, value_token_stride * eb / 16,
      slot_mapping, num_rows, num_kv_heads, chunks_per_row, rows_per_cta, (int64_t)num_blocks * block_size,
      block_size, (uint4*)key_cache, (uint4*)value_cache, dev_status);
  cudaError_t err = cudaGetLastError();
  if (err != cudaSuccess) return fail(PA_ERR_CUDA, "reshape_and_cache launch: %s", cudaGetErrorString(err));
  return PA_OK;
}
