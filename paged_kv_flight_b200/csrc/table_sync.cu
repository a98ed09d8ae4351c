// table_sync.cu -- the device side of the host page allocator for a decode
// loop: applies the allocator's change log to a device copy of the block
// table and gathers the rows and lengths of the step's batch, so that a loop
// uploads a few triples and two short arrays per step instead of the table
// ("TensorRT-LLM Guide: High-Throughput GPU Inference Engine", section "2.
// Paged KV Cache & Memory Virtualization": the logical-to-physical table
// updated as pages are allocated on demand and released).
#include "pkv_internal.h"

namespace pkv {
namespace {

// table[slot][index] = value for every (slot, index, value) triple; the
// triples name distinct entries, so they are applied in parallel.
__global__ void apply_changes_kernel(const int32_t* __restrict__ chg, int n, int max_batch, int max_blocks,
                                     int32_t* __restrict__ table)
{
    for (int k = blockIdx.x * blockDim.x + threadIdx.x; k < n; k += gridDim.x * blockDim.x) {
        const int slot = chg[3 * k], i = chg[3 * k + 1];
        if (slot >= 0 && slot < max_batch && i >= 0 && i < max_blocks)
            table[(size_t)slot * max_blocks + i] = chg[3 * k + 2];
    }
}

// Row b of the batch: lens_out[b] = lens[b], bt_out[b][:] = table[slots[b]][:]
// (a slot outside the table gives a row of -1).
__global__ void gather_rows_kernel(const int32_t* __restrict__ slots, const int32_t* __restrict__ lens,
                                   int batch, int max_batch, int max_blocks, const int32_t* __restrict__ table,
                                   int32_t* __restrict__ bt_out, int32_t* __restrict__ lens_out)
{
    for (int b = blockIdx.x; b < batch; b += gridDim.x) {
        const int slot = slots[b];
        if (threadIdx.x == 0) lens_out[b] = lens[b];
        const bool ok = slot >= 0 && slot < max_batch;
        const int32_t* src = table + (size_t)(ok ? slot : 0) * max_blocks;
        int32_t* dst = bt_out + (size_t)b * max_blocks;
        for (int j = threadIdx.x; j < max_blocks; j += blockDim.x) dst[j] = ok ? src[j] : -1;
    }
}

}  // namespace
}  // namespace pkv

extern "C" pkv_status pkv_table_sync(const int32_t* upload, int n_changes, int batch, int max_batch,
                                     int max_blocks, int page_size, int32_t* table, int32_t* bt_out,
                                     int32_t* lens_out, cudaStream_t stream)
{
    if (n_changes < 0 || batch < 0 || batch > max_batch || max_blocks <= 0 || page_size <= 0)
        return PKV_ERR_INVALID_ARG;
    if (n_changes == 0 && batch == 0) return PKV_OK;
    if (!upload || !table || (batch > 0 && (!bt_out || !lens_out))) return PKV_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(upload) | reinterpret_cast<uintptr_t>(table) |
         reinterpret_cast<uintptr_t>(bt_out) | reinterpret_cast<uintptr_t>(lens_out)) & 3u)
        return PKV_ERR_INVALID_ARG;
    if (n_changes > 0) {
        const int blocks = (n_changes + 255) / 256;
        pkv::apply_changes_kernel<<<blocks < 148 ? blocks : 148, 256, 0, stream>>>(upload, n_changes, max_batch,
                                                                                   max_blocks, table);
        if (cudaGetLastError() != cudaSuccess) return PKV_ERR_CUDA;
    }
    if (batch > 0) {
        const int32_t* slots = upload + 3 * (size_t)n_changes;
        pkv::gather_rows_kernel<<<batch < 1184 ? batch : 1184, 128, 0, stream>>>(
            slots, slots + batch, batch, max_batch, max_blocks, table, bt_out, lens_out);
        if (cudaGetLastError() != cudaSuccess) return PKV_ERR_CUDA;
    }
    return PKV_OK;
}
