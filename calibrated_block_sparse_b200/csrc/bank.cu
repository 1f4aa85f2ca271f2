// Calibration bookkeeping around the hot path (explainer §三, "online
// inference: look up the table"): the keep-rate histogram of calibrated
// blocks (§二 observation 3) and the (t, l) mask bank that online inference
// reads its skip lists, work lists and repeated heads from.
#include <cuda_runtime.h>

#include <algorithm>
#include <climits>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <vector>

#include "calibatt.h"
#include "kernels.h"
#include "ptx.cuh"

namespace calibatt {
namespace {

constexpr int kHistThreads = 256;
constexpr int kHistMaxBins = 4097;  // n_inputs <= 4096

// One block-range of one head per CTA (grid.y = head): a shared-memory
// histogram of the counts, then one global atomic add per nonzero bin.
// Counts above n_inputs are reported and land in the last bin.
__global__ void __launch_bounds__(kHistThreads)
    keep_hist_kernel(const uint16_t* __restrict__ counts, int64_t cells, int n_inputs,
                     unsigned long long* __restrict__ hist, int* status) {
  __shared__ unsigned int bins[kHistMaxBins];
  const int nbins = n_inputs + 1;
  for (int i = threadIdx.x; i < nbins; i += blockDim.x) bins[i] = 0;
  __syncthreads();
  const uint16_t* c = counts + static_cast<int64_t>(blockIdx.y) * cells;
  bool over = false;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < cells;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    int v = __ldg(c + i);
    if (v > n_inputs) {
      over = true;
      v = n_inputs;
    }
    atomicAdd(&bins[v], 1u);
  }
  if (over) record_error(status, CALIBATT_ERR_ARG);
  __syncthreads();
  unsigned long long* h = hist + static_cast<int64_t>(blockIdx.y) * nbins;
  for (int i = threadIdx.x; i < nbins; i += blockDim.x)
    if (bins[i]) atomicAdd(h + i, static_cast<unsigned long long>(bins[i]));
}

}  // namespace
}  // namespace calibatt

// ------------------------------------------------------------------ mask bank
// A host-side index over caller-owned device memory. Each stored entry is one
// device buffer laid out as [row_ptr | col_idx | work_list | rep_heads], every
// part starting on a 256-byte boundary.
struct calibatt_bank {
  int T, L, heads, frames, H, W, k_anchor, nb;
  std::vector<calibatt_bank_entry> entries;
  std::vector<uint8_t> present;
};

namespace {

size_t round256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

struct EntryLayout {
  size_t row_ptr, col_idx, work, rep, total;
};

EntryLayout entry_layout(const calibatt_bank* b, int64_t nnz, int n_rep) {
  const int64_t nbq_b = (static_cast<int64_t>(b->frames) * b->k_anchor * b->W + 127) / 128;
  const size_t rows = static_cast<size_t>(b->heads) * b->nb;
  EntryLayout e;
  e.row_ptr = 0;
  e.col_idx = round256((rows + 1) * sizeof(int32_t));
  e.work = e.col_idx + round256(static_cast<size_t>(nnz) * sizeof(int32_t));
  e.rep = e.work + round256((rows + static_cast<size_t>(n_rep) * nbq_b) * sizeof(int32_t));
  e.total = e.rep + round256(static_cast<size_t>(n_rep) * sizeof(int32_t));
  return e;
}

}  // namespace

using namespace calibatt;

extern "C" {

int calibatt_keep_histogram(const uint16_t* counts, int heads, int64_t cells, int n_inputs, int64_t* hist,
                            calibatt_stream_t stream) {
  if (!counts || !hist || heads < 1 || heads > 65535 || cells < 1 || n_inputs < 1 || n_inputs >= kHistMaxBins)
    return CALIBATT_ERR_ARG;
  if ((reinterpret_cast<uintptr_t>(counts) & 1u) || (reinterpret_cast<uintptr_t>(hist) & 7u))
    return CALIBATT_ERR_ALIGN;
  int* status = status_word();
  if (!status) return CALIBATT_ERR_CUDA;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(hist, 0, static_cast<size_t>(heads) * (n_inputs + 1) * sizeof(int64_t), st) != cudaSuccess)
    return CALIBATT_ERR_CUDA;
  const int64_t per_cta = static_cast<int64_t>(kHistThreads) * 16;
  const int gx = static_cast<int>(std::min<int64_t>((cells + per_cta - 1) / per_cta, 1024));
  keep_hist_kernel<<<dim3(gx, heads), kHistThreads, 0, st>>>(counts, cells, n_inputs,
                                                              reinterpret_cast<unsigned long long*>(hist), status);
  return cudaGetLastError() == cudaSuccess ? CALIBATT_OK : CALIBATT_ERR_CUDA;
}

calibatt_bank* calibatt_bank_create(int timesteps, int layers, int heads, int frames, int H, int W, int k_anchor) {
  if (timesteps < 1 || layers < 1 || heads < 1 || frames < 1 || H < 1 || W < 1 || k_anchor < 1 || k_anchor > H)
    return nullptr;
  const int64_t n = static_cast<int64_t>(frames) * H * W;
  if (n > INT_MAX / 2 || static_cast<int64_t>(timesteps) * layers > (1 << 24)) return nullptr;
  calibatt_bank* b = new (std::nothrow) calibatt_bank;
  if (!b) return nullptr;
  b->T = timesteps;
  b->L = layers;
  b->heads = heads;
  b->frames = frames;
  b->H = H;
  b->W = W;
  b->k_anchor = k_anchor;
  b->nb = static_cast<int>((n + 127) / 128);
  b->entries.assign(static_cast<size_t>(timesteps) * layers, calibatt_bank_entry{});
  b->present.assign(static_cast<size_t>(timesteps) * layers, 0);
  return b;
}

void calibatt_bank_destroy(calibatt_bank* bank) { delete bank; }

size_t calibatt_bank_entry_bytes(const calibatt_bank* bank, int64_t nnz, int n_rep) {
  if (!bank || nnz < 0 || n_rep < 0 || n_rep > bank->heads) return 0;
  return entry_layout(bank, nnz, n_rep).total;
}

int calibatt_bank_put(calibatt_bank* bank, int t, int l, double eps, const int32_t* row_ptr_host,
                      const int32_t* col_idx, int64_t nnz, const int32_t* rep_heads_host, int n_rep, void* dst,
                      size_t dst_bytes, calibatt_stream_t stream) {
  if (!bank || t < 0 || t >= bank->T || l < 0 || l >= bank->L || !row_ptr_host || nnz < 0 ||
      (nnz > 0 && !col_idx) || n_rep < 0 || n_rep > bank->heads || (n_rep > 0 && !rep_heads_host) || !dst ||
      std::isnan(eps))
    return CALIBATT_ERR_ARG;
  const int64_t rows = static_cast<int64_t>(bank->heads) * bank->nb;
  if (row_ptr_host[0] != 0 || row_ptr_host[rows] != nnz) return CALIBATT_ERR_CSR;
  for (int i = 0; i < n_rep; ++i)
    if (rep_heads_host[i] < 0 || rep_heads_host[i] >= bank->heads) return CALIBATT_ERR_ARG;
  const EntryLayout lay = entry_layout(bank, nnz, n_rep);
  if (dst_bytes < lay.total) return CALIBATT_ERR_ARG;
  if (reinterpret_cast<uintptr_t>(dst) & 255u) return CALIBATT_ERR_ALIGN;
  const int64_t nbq_b = (static_cast<int64_t>(bank->frames) * bank->k_anchor * bank->W + 127) / 128;
  std::vector<int32_t> work(static_cast<size_t>(rows + n_rep * nbq_b));
  int32_t n_work = 0;
  int rc = calibatt_build_mixed_plan(row_ptr_host, bank->heads, bank->nb, nullptr, n_rep, rep_heads_host,
                                     bank->frames, bank->H, bank->W, bank->k_anchor, work.data(), &n_work);
  if (rc == CALIBATT_OK) rc = calibatt_balance_plan(work.data(), n_work, row_ptr_host, bank->heads, bank->nb, 0);
  if (rc != CALIBATT_OK) return rc;
  uint8_t* base = static_cast<uint8_t*>(dst);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  // pageable host sources: each copy has read its source when it returns
  if (cudaMemcpyAsync(base + lay.row_ptr, row_ptr_host, (rows + 1) * sizeof(int32_t), cudaMemcpyHostToDevice, st) !=
          cudaSuccess ||
      (nnz > 0 && cudaMemcpyAsync(base + lay.col_idx, col_idx, nnz * sizeof(int32_t), cudaMemcpyDeviceToDevice,
                                  st) != cudaSuccess) ||
      (n_work > 0 && cudaMemcpyAsync(base + lay.work, work.data(), n_work * sizeof(int32_t), cudaMemcpyHostToDevice,
                                     st) != cudaSuccess) ||
      (n_rep > 0 && cudaMemcpyAsync(base + lay.rep, rep_heads_host, n_rep * sizeof(int32_t), cudaMemcpyHostToDevice,
                                    st) != cudaSuccess))
    return CALIBATT_ERR_CUDA;
  calibatt_bank_entry& e = bank->entries[static_cast<size_t>(t) * bank->L + l];
  e.row_ptr = reinterpret_cast<const int32_t*>(base + lay.row_ptr);
  e.col_idx = reinterpret_cast<const int32_t*>(base + lay.col_idx);
  e.nnz = nnz;
  e.work_list = reinterpret_cast<const int32_t*>(base + lay.work);
  e.n_work = n_work;
  e.rep_heads = reinterpret_cast<const int32_t*>(base + lay.rep);
  e.n_rep = n_rep;
  e.eps = eps;
  bank->present[static_cast<size_t>(t) * bank->L + l] = 1;
  return CALIBATT_OK;
}

int calibatt_bank_get(const calibatt_bank* bank, int t, int l, calibatt_bank_entry* out) {
  if (!bank || !out || t < 0 || t >= bank->T || l < 0 || l >= bank->L) return CALIBATT_ERR_ARG;
  const size_t i = static_cast<size_t>(t) * bank->L + l;
  if (!bank->present[i]) return CALIBATT_ERR_ARG;
  *out = bank->entries[i];
  return CALIBATT_OK;
}

}  // extern "C"
