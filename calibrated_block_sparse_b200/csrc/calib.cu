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
// One warp per block-row of energies, four rows per CTA, each warp with its
// own 8 KB histogram; no block barriers. PER (columns per lane, >= nb / 32)
// sizes the per-lane register arrays. Lanes read and write the row's columns
// interleaved (column lane + 32 i), so every access is coalesced.
template <int PER>
__global__ void __launch_bounds__(128) select_kernel(const float* __restrict__ energy, int64_t rows, int nb,
                                                     long long eps_fx, uint8_t* mask, int32_t* kept,
                                                     uint16_t* counts, uint8_t* tie, long long tie_fx) {
  __shared__ __align__(16) unsigned long long hist[4][kSelectBuckets];
  const int w = threadIdx.x >> 5;
  const int64_t row = static_cast<int64_t>(blockIdx.x) * 4 + w;
  if (row >= rows) return;
  SelectOut out{mask ? mask + row * nb : nullptr, kept ? kept + row : nullptr, counts ? counts + row * nb : nullptr,
                tie ? tie + row : nullptr};
  warp_select<PER>(energy + row * nb, nb, eps_fx, tie_fx, hist[w], out);
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
// Pass 1: one warp per (head, block-row): binarise counts >= threshold, write
// the mask row and the row's kept count.
__global__ void binarize_kernel(const uint16_t* __restrict__ counts, int64_t rows, int nb, int threshold,
                                uint8_t* mask, int32_t* row_cnt) {
  const int64_t row = (blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  const uint16_t* src = counts + row * nb;
  uint8_t* dst = mask + row * nb;
  int cnt = 0;
  for (int c = lane; c < nb; c += 32) {
    const uint8_t k = src[c] >= threshold ? 1 : 0;
    dst[c] = k;
    cnt += k;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) cnt += __shfl_xor_sync(0xffffffffu, cnt, o);
  if (lane == 0) row_cnt[row] = cnt;
}

// Pass 2: a single CTA turns the row counts into the exclusive prefix row_ptr
// (global offsets) and the total. The counts are taken in tiles of
// kScanTile rows staged in shared memory (coalesced); each thread scans a
// contiguous run of its tile, one block-wide scan of the 1024 run totals
// joins them, and a carry crosses tiles. One padding word per 32 keeps the
// threads' runs on distinct banks.
constexpr int kScanThreads = 1024;
constexpr int kScanTile = 16384;  // rows per tile
constexpr int kScanSmem = (kScanTile + kScanTile / 32) * 4;

__device__ __forceinline__ int scan_pad(int i) { return i + (i >> 5); }

__global__ void __launch_bounds__(kScanThreads) scan_kernel(const int32_t* __restrict__ row_cnt, int64_t rows,
                                                            int32_t* row_ptr, int64_t nnz_cap, int64_t* nnz_out,
                                                            int* status) {
  extern __shared__ int32_t tile[];
  __shared__ long long warp_tot[32];
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  constexpr int kRun = kScanTile / kScanThreads;
  long long carry = 0;
  for (int64_t base = 0; base < rows; base += kScanTile) {
    const int n = static_cast<int>(rows - base < kScanTile ? rows - base : kScanTile);
    for (int i = tid; i < n; i += kScanThreads) tile[scan_pad(i)] = row_cnt[base + i];
    __syncthreads();
    long long run = 0;
#pragma unroll
    for (int k = 0; k < kRun; ++k) {
      const int i = tid * kRun + k;
      run += i < n ? tile[scan_pad(i)] : 0;
    }
    long long incl = run;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const long long t = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += t;
    }
    if (lane == 31) warp_tot[w] = incl;
    __syncthreads();
    long long wbefore = 0, all = 0;
    for (int ww = 0; ww < 32; ++ww) {
      const long long t = warp_tot[ww];
      wbefore += ww < w ? t : 0;
      all += t;
    }
    long long pos = carry + wbefore + incl - run;  // exclusive prefix of this thread's run
#pragma unroll
    for (int k = 0; k < kRun; ++k) {
      const int i = tid * kRun + k;
      if (i < n) {
        const int32_t v = tile[scan_pad(i)];
        tile[scan_pad(i)] = static_cast<int32_t>(pos);
        pos += v;
      }
    }
    __syncthreads();
    for (int i = tid; i < n; i += kScanThreads) row_ptr[base + i] = tile[scan_pad(i)];
    carry += all;
    __syncthreads();  // the tile and warp totals are reused
  }
  if (tid == 0) {
    row_ptr[rows] = static_cast<int32_t>(carry);
    *nnz_out = carry;
    if (carry > nnz_cap) record_error(status, CALIBATT_ERR_CAPACITY);
  }
}

// Pass 3: one warp per row writes the kept columns in ascending order.
__global__ void compact_kernel(const uint8_t* __restrict__ mask, int64_t rows, int nb,
                               const int32_t* __restrict__ row_ptr, int32_t* col_idx, int64_t nnz_cap) {
  const int64_t row = (blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  const uint8_t* src = mask + row * nb;
  int64_t pos = row_ptr[row];
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
                     int32_t* col_idx, int64_t nnz_cap, int64_t* nnz, int32_t* row_cnt, int* status,
                     cudaStream_t stream) {
  const unsigned warps_blocks = static_cast<unsigned>((rows * 32 + 255) / 256);
  static PerDeviceOnce scan_once;
  const int rc = set_max_smem_once(reinterpret_cast<const void*>(scan_kernel), kScanSmem, scan_once);
  if (rc != CALIBATT_OK) return rc;
  binarize_kernel<<<warps_blocks, 256, 0, stream>>>(counts, rows, nb, threshold, mask, row_cnt);
  scan_kernel<<<1, kScanThreads, kScanSmem, stream>>>(row_cnt, rows, row_ptr, nnz_cap, nnz, status);
  compact_kernel<<<warps_blocks, 256, 0, stream>>>(mask, rows, nb, row_ptr, col_idx, nnz_cap);
  return cudaGetLastError() == cudaSuccess ? CALIBATT_OK : CALIBATT_ERR_CUDA;
}

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
