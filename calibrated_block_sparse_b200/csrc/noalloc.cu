// Allocation-free variant of calibatt_aggregate_masks.
//
// Some callers cannot allocate device memory at the point where they build a
// skip list: a plugin that only receives pointers from a host engine whose
// allocator owns all of the GPU's memory, or a serving loop that runs under a
// fixed memory budget where an extra allocation could fail or stall. This entry
// point takes only the inputs and outputs; the per-row kept counts that the
// aggregation needs between its passes live in the file-scope array below
// instead of a caller-supplied workspace.
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <mutex>

#include "calibatt.h"
#include "kernels.h"

namespace calibatt {

// The aggregation's span totals: at most one int32 per (head, block-row), at
// most CALIBATT_NOALLOC_MAX_ROWS rows: 1 MiB. Every GPU that loads the
// library holds this array until exit.
constexpr int64_t kNoallocScratchInts = CALIBATT_NOALLOC_MAX_ROWS;
static __device__ __align__(256) int32_t g_noalloc_row_cnt[kNoallocScratchInts];

namespace {

// Device address of the scratch array on the current device, looked up once
// per device. In host code the array's name is only a host-side stand-in, so
// the kernels are always given this address.
int32_t* noalloc_scratch() {
  static std::mutex mu;
  static int32_t* addr[64] = {nullptr};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (!addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_row_cnt) != cudaSuccess || p == nullptr) return nullptr;
    addr[dev] = static_cast<int32_t*>(p);
  }
  return addr[dev];
}

}  // namespace
}  // namespace calibatt

using namespace calibatt;

extern "C" int calibatt_aggregate_masks_noalloc(const uint16_t* counts, int n_inputs, int heads, int nb, double rho,
                                                uint8_t* mask, int32_t* row_ptr, int32_t* col_idx, int64_t nnz_cap,
                                                int64_t* nnz, calibatt_stream_t stream) {
  if (!counts || !mask || !row_ptr || !nnz || heads < 1 || nb < 1 || n_inputs < 1 || nnz_cap < 0 ||
      (nnz_cap > 0 && !col_idx) || !std::isfinite(rho))
    return CALIBATT_ERR_ARG;
  const int64_t rows = static_cast<int64_t>(heads) * nb;
  if (rows > CALIBATT_NOALLOC_MAX_ROWS) return CALIBATT_ERR_ARG;
  if (rows * nb > INT32_MAX) return CALIBATT_ERR_ARG;
  if ((reinterpret_cast<uintptr_t>(counts) & 1u) || (reinterpret_cast<uintptr_t>(row_ptr) & 3u) ||
      (col_idx && (reinterpret_cast<uintptr_t>(col_idx) & 3u)) || (reinterpret_cast<uintptr_t>(nnz) & 7u))
    return CALIBATT_ERR_ALIGN;
  if (aggregate_scratch_ints(rows) > kNoallocScratchInts) return CALIBATT_ERR_ARG;
  int32_t* scratch = noalloc_scratch();
  int* status = status_word();
  if (!scratch || !status) return CALIBATT_ERR_CUDA;
  int32_t thr = 0;
  calibatt_rho_threshold(n_inputs, rho, &thr);
  // The first pass writes every span total that the second reads, so the
  // array needs no clearing between calls.
  return launch_aggregate(counts, rows, nb, thr, mask, row_ptr, col_idx, nnz_cap, nnz, scratch, status,
                          reinterpret_cast<cudaStream_t>(stream));
}
