// pa_block_tables_apply: bring a device copy of the padded block tables up to
// date from the (row, column, page) updates of pa_block_alloc_table_updates.
//
// PagedAttention Internals, "2. The Dynamic Block Table": a sequence's table
// grows by one entry when a token starts a new block, and "Copy-on-Write and
// Prefix Sharing": an entry is replaced when a shared page is forked.  A decode
// step therefore changes a few entries of a table the kernels read in full;
// only those entries cross to the device.
//
// One thread per update.  The updates of one call name distinct entries, so
// they are written in any order.  Row -1 marks padding, so that a captured
// launch can take a buffer of fixed size whose tail holds no update.
#include "device.cuh"
#include "pa_internal.h"

namespace pa {
namespace {

constexpr int kThreads = 256;

__global__ void __launch_bounds__(kThreads)
    block_tables_apply_kernel(int32_t* __restrict__ tables, int32_t num_rows, int32_t max_blocks_per_seq,
                              const int32_t* __restrict__ updates, int32_t num_updates, int32_t* status) {
  const int32_t i = blockIdx.x * kThreads + threadIdx.x;
  if (i >= num_updates) return;
  const int32_t row = __ldg(updates + 3 * (int64_t)i);
  const int32_t col = __ldg(updates + 3 * (int64_t)i + 1);
  const int32_t page = __ldg(updates + 3 * (int64_t)i + 2);
  if (row == -1) return;  // padding of a fixed-size update buffer
  if ((unsigned)row >= (unsigned)num_rows || (unsigned)col >= (unsigned)max_blocks_per_seq) {
    flag_status(status, PA_DEV_BAD_UPDATE);
    return;
  }
  tables[(int64_t)row * max_blocks_per_seq + col] = page;
}

}  // namespace
}  // namespace pa

using namespace pa;

extern "C" pa_status pa_block_tables_apply(int32_t* block_tables, int32_t num_rows, int32_t max_blocks_per_seq,
                                           const int32_t* updates, int32_t num_updates, int32_t* dev_status,
                                           void* stream) {
  if (num_rows < 0 || max_blocks_per_seq < 0 || num_updates < 0)
    return fail(PA_ERR_INVALID, "block_tables_apply: bad sizes");
  if (num_updates == 0) return PA_OK;
  if (!block_tables || !updates) return fail(PA_ERR_INVALID, "block_tables_apply: NULL pointer");
  const int blocks = (int)((num_updates + kThreads - 1) / kThreads);
  block_tables_apply_kernel<<<blocks, kThreads, 0, (cudaStream_t)stream>>>(block_tables, num_rows,
                                                                           max_blocks_per_seq, updates,
                                                                           num_updates, dev_status);
  cudaError_t err = cudaGetLastError();
  if (err != cudaSuccess) return fail(PA_ERR_CUDA, "block_tables_apply launch: %s", cudaGetErrorString(err));
  return PA_OK;
}
