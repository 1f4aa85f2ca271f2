// Bandwidth-bound calibration and packing kernels: standalone greedy eps
// selection, mask accumulation over inputs, rho aggregation into a CSR skip
// list, and the anchor-row query gather of repeated heads.
#include <cooperative_groups.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "calibatt.h"
#include "kernels.h"
#include "ptx.cuh"
#include "sched.cuh"
#include "select.cuh"

namespace calibatt {


// ------------------------------------------------------------------ selection
// One warp per block-row of energies, four rows per CTA, each warp with 128
// bytes of shared scratch; no block barriers. PER (columns per lane, >= nb / 32)
// sizes the per-lane register arrays. Lanes read and write the row's columns
// interleaved (column lane + 32 i), so every access is coalesced.
template <int PER>
__global__ void __launch_bounds__(128) select_kernel(const float* __restrict__ energy, int64_t rows, int nb,
                                                     long long eps_fx, uint8_t* mask, int32_t* kept,
                                                     uint16_t* counts, uint8_t* tie, long long tie_fx) {
  __shared__ __align__(16) float scratch[4][kSelectScratchBytes / 4];
  const int w = threadIdx.x >> 5;
  const int64_t row = static_cast<int64_t>(blockIdx.x) * 4 + w;
  if (row >= rows) return;
  SelectOut out{mask ? mask + row * nb : nullptr, kept ? kept + row : nullptr, counts ? counts + row * nb : nullptr,
                tie ? tie + row : nullptr};
  warp_select<PER>(energy + row * nb, nb, eps_fx, tie_fx, scratch[w], out);
}

// ------------------------------------------------------------------ accumulation
__global__ void accumulate_kernel(const uint8_t* __restrict__ mask, int64_t cells, uint16_t* counts) {
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < cells; i += stride) {
    const uint16_t c = counts[i];
    if (mask[i] && c != 0xFFFFu) counts[i] = c + 1;
  }
}

// ------------------------------------------------------------------ aggregation
// Two launches over CTAs of kAggRows block-rows (one warp per row):
//  1. binarize: counts >= threshold -> mask row, the row's kept count, and
//     the CTA's total;
//  2. compact: each CTA adds up the totals of the CTAs before it (all final
//     once the first launch is done: no cross-CTA waiting), scans its own
//     rows' counts into row_ptr (global offsets), and writes each row's kept
//     columns in ascending order. The last CTA writes the grand total.
// Scratch: row_cnt[rows] then cta_sum[ceil(rows / kAggRows)].
constexpr int kAggRows = 32;  // = warps per CTA = lanes of a warp (partials are read one per lane)

__global__ void __launch_bounds__(kAggRows * 32) binarize_kernel(const uint16_t* __restrict__ counts, int64_t rows,
                                                                 int nb, int threshold, uint8_t* mask,
                                                                 int32_t* row_cnt, int32_t* cta_sum) {
  __shared__ int wsum[kAggRows];
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t row = static_cast<int64_t>(blockIdx.x) * kAggRows + w;
  int cnt = 0;
  if (row < rows) {
    const uint16_t* src = counts + row * nb;
    uint8_t* dst = mask + row * nb;
#pragma unroll 4
    for (int c = lane; c < nb; c += 32) {
      const uint8_t k = src[c] >= threshold ? 1 : 0;
      dst[c] = k;
      cnt += k;
    }
    cnt = static_cast<int>(__reduce_add_sync(0xffffffffu, static_cast<unsigned>(cnt)));
    if (lane == 0) row_cnt[row] = cnt;
  }
  if (lane == 0) wsum[w] = cnt;
  __syncthreads();
  if (w == 0) {
    const int t = static_cast<int>(__reduce_add_sync(0xffffffffu, static_cast<unsigned>(wsum[lane])));
    if (lane == 0) cta_sum[blockIdx.x] = t;
  }
}

__global__ void __launch_bounds__(kAggRows * 32) compact_kernel(const uint8_t* __restrict__ mask, int64_t rows,
                                                                int nb, const int32_t* __restrict__ row_cnt,
                                                                const int32_t* __restrict__ cta_sum,
                                                                int32_t* row_ptr, int32_t* col_idx, int64_t nnz_cap,
                                                                int64_t* nnz_out, int* status) {
  __shared__ long long wpart[kAggRows];
  __shared__ int wcnt[kAggRows];
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // the kept blocks of every earlier CTA
  long long before = 0;
  for (int64_t i = threadIdx.x; i < blockIdx.x; i += blockDim.x) before += cta_sum[i];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) before += __shfl_xor_sync(0xffffffffu, before, o);
  const int64_t row = static_cast<int64_t>(blockIdx.x) * kAggRows + w;
  const int cnt = row < rows ? row_cnt[row] : 0;
  if (lane == 0) {
    wpart[w] = before;
    wcnt[w] = cnt;
  }
  __syncthreads();
  // lane i of every warp takes warp i's partials
  long long base = wpart[lane];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) base += __shfl_xor_sync(0xffffffffu, base, o);
  const unsigned cw = static_cast<unsigned>(wcnt[lane]);
  const long long mine = __reduce_add_sync(0xffffffffu, lane < w ? cw : 0u);
  const long long total = __reduce_add_sync(0xffffffffu, cw);
  long long pos = base + mine;  // this row's first entry
  if (row < rows) {
    if (lane == 0) row_ptr[row] = static_cast<int32_t>(pos);
    const uint8_t* src = mask + row * nb;
    for (int c0 = 0; c0 < nb; c0 += 32) {
      const int c = c0 + lane;
      const bool k = c < nb && src[c];
      const uint32_t bal = __ballot_sync(0xffffffffu, k);
      if (k) {
        const int64_t at = pos + __popc(bal & ((1u << lane) - 1u));
        if (at < nnz_cap) col_idx[at] = c;
      }
      pos += __popc(bal);
    }
  }
  if (blockIdx.x == gridDim.x - 1 && threadIdx.x == 0) {
    const long long grand = base + total;
    row_ptr[rows] = static_cast<int32_t>(grand);
    *nnz_out = grand;
    if (grand > nnz_cap) record_error(status, CALIBATT_ERR_CAPACITY);
  }
}

// ------------------------------------------------------------------ anchor gather
// Packs the anchor-row queries of repeated heads: packed row q = f*(k*W) +
// j*W + c of head i is token f*H*W + anchors[j]*W + c of head rep_heads[i].
// 16 threads move one 256-byte row.
__global__ void gather_anchor_kernel(const uint4* __restrict__ q, int n, const int32_t* __restrict__ rep_heads,
                                     int n_rep, int H, int W, int k_anchor, AnchorTable tab, uint4* out,
                                     int heads, int* status) {
  const int64_t per_head = static_cast<int64_t>(n / (H * W)) * k_anchor * W;
  const int64_t total = per_head * n_rep * 16;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t t = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; t < total; t += stride) {
    const int part = static_cast<int>(t & 15);
    const int64_t prow = t >> 4;
    const int i = static_cast<int>(prow / per_head);
    const int64_t qi = prow % per_head;
    const int kw = k_anchor * W;
    const int64_t f = qi / kw;
    const int rem = static_cast<int>(qi % kw);
    const int j = rem / W, c = rem % W;
    int h = rep_heads[i];
    if (h < 0 || h >= heads) {
      record_error(status, CALIBATT_ERR_ARG);
      h = 0;
    }
    const int64_t tok = f * H * W + static_cast<int64_t>(tab.anchor[j]) * W + c;
    out[prow * 16 + part] = q[(static_cast<int64_t>(h) * n + tok) * 16 + part];
  }
}

}  // namespace calibatt

namespace calibatt {

int launch_select(const float* energy, int64_t rows, int nb, long long eps_fx, uint8_t* mask, int32_t* kept,
                  uint16_t* counts, uint8_t* tie, long long tie_fx, cudaStream_t stream) {
  if (rows <= 0) return CALIBATT_OK;
  const unsigned grid = static_cast<unsigned>((rows + 3) / 4);
  if (nb <= 256)
    select_kernel<8><<<grid, 128, 0, stream>>>(energy, rows, nb, eps_fx, mask, kept, counts, tie, tie_fx);
  else if (nb <= 512)
    select_kernel<16><<<grid, 128, 0, stream>>>(energy, rows, nb, eps_fx, mask, kept, counts, tie, tie_fx);
  else if (nb <= 768)
    select_kernel<24><<<grid, 128, 0, stream>>>(energy, rows, nb, eps_fx, mask, kept, counts, tie, tie_fx);
  else
    select_kernel<32><<<grid, 128, 0, stream>>>(energy, rows, nb, eps_fx, mask, kept, counts, tie, tie_fx);
  return cudaGetLastError() == cudaSuccess ? CALIBATT_OK : CALIBATT_ERR_CUDA;
}

int launch_accumulate(const uint8_t* mask, int64_t cells, uint16_t* counts, cudaStream_t stream) {
  if (cells <= 0) return CALIBATT_OK;
  int64_t blocks = (cells + 255) / 256;
  if (blocks > 148 * 16) blocks = 148 * 16;
  accumulate_kernel<<<static_cast<unsigned>(blocks), 256, 0, stream>>>(mask, cells, counts);
  return cudaGetLastError() == cudaSuccess ? CALIBATT_OK : CALIBATT_ERR_CUDA;
}

int launch_aggregate(const uint16_t* counts, int64_t rows, int nb, int threshold, uint8_t* mask, int32_t* row_ptr,
                     int32_t* col_idx, int64_t nnz_cap, int64_t* nnz, int32_t* scratch, int* status,
                     cudaStream_t stream) {
  const unsigned ctas = static_cast<unsigned>((rows + kAggRows - 1) / kAggRows);
  int32_t* row_cnt = scratch;
  int32_t* cta_sum = scratch + rows;
  binarize_kernel<<<ctas, kAggRows * 32, 0, stream>>>(counts, rows, nb, threshold, mask, row_cnt, cta_sum);
  compact_kernel<<<ctas, kAggRows * 32, 0, stream>>>(mask, rows, nb, row_cnt, cta_sum, row_ptr, col_idx, nnz_cap, nnz,
                                                     status);
  return cudaGetLastError() == cudaSuccess ? CALIBATT_OK : CALIBATT_ERR_CUDA;
}

int64_t aggregate_scratch_ints(int64_t rows) { return rows + (rows + kAggRows - 1) / kAggRows; }

int launch_gather(const void* q, int n, int heads, const int32_t* rep_heads, int n_rep, int H, int W, int k_anchor,
                  const AnchorTable& tab, void* out, int* status, cudaStream_t stream) {
  const int64_t total = static_cast<int64_t>(n / (H * W)) * k_anchor * W * n_rep * 16;
  if (total <= 0) return CALIBATT_OK;
  int64_t blocks = (total + 255) / 256;
  if (blocks > 148 * 8) blocks = 148 * 8;
  gather_anchor_kernel<<<static_cast<unsigned>(blocks), 256, 0, stream>>>(
      static_cast<const uint4*>(q), n, rep_heads, n_rep, H, W, k_anchor, tab, static_cast<uint4*>(out), heads, status);
  return cudaGetLastError() == cudaSuccess ? CALIBATT_OK : CALIBATT_ERR_CUDA;
}

}  // namespace calibatt

// ------------------------------------------------------------------ spatial score
// Per head, the mean over frames and non-anchor pixel rows r of the cosine
// similarity between the profile of r and that of its nearest anchor row
// (explainer §三, the spatial similarity score; §二 observation 4). A head is
// one thread-block cluster of kScoreCluster CTAs: CTA p of the cluster takes
// pixel rows p*8 + w, + 64, ... with warp w; each CTA sums its rows into
// per-warp partials in shared memory, and the cluster's first CTA adds all
// partials in a fixed order through distributed shared memory, so the score
// is reproducible for given profiles and needs no workspace.
namespace calibatt {
namespace {

namespace cg = cooperative_groups;

constexpr int kScoreWarps = 8;
constexpr int kScoreCluster = 8;

__global__ void __cluster_dims__(kScoreCluster, 1, 1) __launch_bounds__(kScoreWarps * 32)
    spatial_score_kernel(const float* __restrict__ pix, int frames, int H, int nb,
                         const __grid_constant__ RowAnchorTable tab, float gamma, float* score, uint8_t* flag) {
  cg::cluster_group cluster = cg::this_cluster();
  const int h = blockIdx.x / kScoreCluster;
  const int part = static_cast<int>(cluster.block_rank());
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t rows = static_cast<int64_t>(frames) * H;
  const float* base = pix + static_cast<int64_t>(h) * rows * nb;
  double sum = 0.0;
  int cnt = 0;
  for (int64_t R = part * kScoreWarps + warp; R < rows; R += kScoreCluster * kScoreWarps) {
    const int r = static_cast<int>(R % H);
    const int a = tab.row[r];
    if (a == r) continue;  // an anchor row is computed, not copied
    const float* x = base + R * nb;
    const float* y = base + (R - r + a) * nb;
    float xy = 0.f, xx = 0.f, yy = 0.f;
#pragma unroll 4
    for (int c = lane; c < nb; c += 32) {
      const float xv = __ldg(x + c), yv = __ldg(y + c);
      xy = fmaf(xv, yv, xy);
      xx = fmaf(xv, xv, xx);
      yy = fmaf(yv, yv, yy);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      xy += __shfl_xor_sync(0xffffffffu, xy, o);
      xx += __shfl_xor_sync(0xffffffffu, xx, o);
      yy += __shfl_xor_sync(0xffffffffu, yy, o);
    }
    sum += (xx > 0.f && yy > 0.f) ? static_cast<double>(xy) / (sqrt(static_cast<double>(xx)) * sqrt(static_cast<double>(yy)))
                                  : 0.0;
    ++cnt;
  }
  __shared__ double ssum[kScoreWarps];
  __shared__ int scnt[kScoreWarps];
  if (lane == 0) {
    ssum[warp] = sum;
    scnt[warp] = cnt;
  }
  cluster.sync();
  if (part == 0 && threadIdx.x == 0) {
    double t = 0.0;
    int c = 0;
    for (int q = 0; q < kScoreCluster; ++q) {
      const double* qs = cluster.map_shared_rank(ssum, q);
      const int* qc = cluster.map_shared_rank(scnt, q);
      for (int w = 0; w < kScoreWarps; ++w) {
        t += qs[w];
        c += qc[w];
      }
    }
    const float sc = c ? static_cast<float>(t / c) : 1.0f;
    score[h] = sc;
    if (flag) flag[h] = sc > gamma ? 1 : 0;
  }
  cluster.sync();  // every CTA's partials stay in place until they have been read
}

}  // namespace

int launch_spatial_score(const float* pix, int heads, int frames, int H, int nb, const RowAnchorTable& tab,
                         float gamma, float* score, uint8_t* flag, cudaStream_t stream) {
  spatial_score_kernel<<<heads * kScoreCluster, kScoreWarps * 32, 0, stream>>>(pix, frames, H, nb, tab, gamma, score,
                                                                                flag);
  return cudaGetLastError() == cudaSuccess ? CALIBATT_OK : CALIBATT_ERR_CUDA;
}

}  // namespace calibatt
