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
// interleaved (column lane + 32 i), so every access is coalesced. The launch
// bounds hold the register count at 80 (96 for PER = 32) without spills, so
// that 6 (5) CTAs share an SM: the search's warp-sum chains need the warps.
template <int PER>
__global__ void __launch_bounds__(128, PER <= 24 ? 6 : 5)
    select_kernel(const float* __restrict__ energy, int64_t rows, int nb, long long eps_fx, uint8_t* mask,
                  int32_t* kept, uint16_t* counts, uint8_t* tie, long long tie_fx) {
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
// The CSR skip list of a mask holds its kept cells in flat (row-major) order:
// cell (row, col) goes to col_idx at its rank among the kept cells, and
// row_ptr[row] is the rank of cell (row, 0). Two launches over CTAs that each
// own one contiguous span of the flat arrays:
//  1. binarize: counts >= threshold -> mask, and the span's kept total;
//  2. compact: the totals of the spans before it (all final once the first
//     launch is done: no cross-CTA waiting) give the span's first rank; the
//     span is then walked in rounds of kAggRound cells, lane chunks of
//     kAggChunk cells ranked by a block scan per round; each warp stages its
//     kept columns in shared memory and stores them as one coalesced run.
//     The last CTA writes the grand total.
// Above kPrefixSpans spans a one-CTA scan turns the totals into exclusive
// prefixes between the two launches, so that a compaction CTA reads its
// first rank instead of adding up every earlier span.
// A span is a whole number of rounds, so with 16-byte aligned arrays every
// lane chunk is one 16-byte mask vector and two 16-byte count vectors.
// Scratch: one total per span.
constexpr int kAggThreads = 256;
constexpr int kAggWarps = kAggThreads / 32;
constexpr int kAggChunk = 16;
constexpr int kAggRound = kAggThreads * kAggChunk;
constexpr int64_t kAggFill = 148 * 8;  // CTAs that fill the SMs at 8 per SM

// 0/1 bytes for four counts (two per word) against the threshold pair t2.
__device__ __forceinline__ uint32_t keep4(uint32_t a, uint32_t b, uint32_t t2, bool none) {
  if (none) return 0u;
  const uint32_t fa = __vcmpgeu2(a, t2) & 0x00010001u, fb = __vcmpgeu2(b, t2) & 0x00010001u;
  return __byte_perm(fa, fb, 0x6420);
}

// One lane chunk's 0/1 mask bytes -> 16-bit kept bitmap (bit j = cell j).
// Within a word, bytes b0..b3 times 0x01020408 land b_i on bit 24 + i, every
// other partial product on a bit below 24 or past 31, with no carries.
__device__ __forceinline__ uint32_t chunk_bits(const uint32_t (&m)[4]) {
  uint32_t bits = 0;
#pragma unroll
  for (int q = 0; q < 4; ++q) bits |= (((m[q] & 0x01010101u) * 0x01020408u) >> 24) << (4 * q);
  return bits;
}

// Flat indices, ranks and spans fit in 32 bits (cells <= INT_MAX, a span at
// most cells + one round), which keeps the index arithmetic single-word.
template <bool kVec>
__device__ __forceinline__ int binarize_chunk(const uint16_t* __restrict__ counts, uint8_t* __restrict__ mask,
                                              uint32_t g, uint32_t s1, const uint4& a, const uint4& b, int threshold,
                                              uint32_t t2, bool none) {
  if (kVec && g + kAggChunk <= s1) {
    uint4 m;
    m.x = keep4(a.x, a.y, t2, none);
    m.y = keep4(a.z, a.w, t2, none);
    m.z = keep4(b.x, b.y, t2, none);
    m.w = keep4(b.z, b.w, t2, none);
    *reinterpret_cast<uint4*>(mask + g) = m;
    return __popc(m.x) + __popc(m.y) + __popc(m.z) + __popc(m.w);
  }
  int cnt = 0;
  for (uint32_t j = 0; j < kAggChunk && g + j < s1; ++j) {
    const int k = counts[g + j] >= threshold ? 1 : 0;
    mask[g + j] = static_cast<uint8_t>(k);
    cnt += k;
  }
  return cnt;
}

template <bool kVec>
__global__ void __launch_bounds__(kAggThreads) binarize_kernel(const uint16_t* __restrict__ counts, uint32_t cells,
                                                               uint32_t span, int threshold,
                                                               uint8_t* __restrict__ mask,
                                                               int32_t* __restrict__ span_sum) {
  __shared__ int wsum[kAggWarps];
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t s0 = blockIdx.x * span;
  const uint32_t s1 = cells - s0 > span ? s0 + span : cells;
  const bool none = threshold > 65535;  // counts are 16-bit
  const uint32_t t2 = static_cast<uint32_t>(threshold > 0 ? threshold : 0) * 0x10001u;
  int cnt = 0;
  // two rounds per step, both rounds' loads in flight before either is used
  for (uint32_t g = s0 + threadIdx.x * kAggChunk; g < s1; g += 2 * kAggRound) {
    const uint32_t h = g + kAggRound;
    uint4 a0 = {}, b0 = {}, a1 = {}, b1 = {};
    if (kVec && g + kAggChunk <= s1) {
      a0 = *reinterpret_cast<const uint4*>(counts + g);
      b0 = *reinterpret_cast<const uint4*>(counts + g + 8);
    }
    if (kVec && h + kAggChunk <= s1) {
      a1 = *reinterpret_cast<const uint4*>(counts + h);
      b1 = *reinterpret_cast<const uint4*>(counts + h + 8);
    }
    cnt += binarize_chunk<kVec>(counts, mask, g, s1, a0, b0, threshold, t2, none);
    if (h < s1) cnt += binarize_chunk<kVec>(counts, mask, h, s1, a1, b1, threshold, t2, none);
  }
  cnt = static_cast<int>(__reduce_add_sync(0xffffffffu, static_cast<unsigned>(cnt)));
  if (lane == 0) wsum[w] = cnt;
  __syncthreads();
  if (w == 0) {
    const int t = static_cast<int>(__reduce_add_sync(0xffffffffu, lane < kAggWarps ? wsum[lane] : 0u));
    if (lane == 0) span_sum[blockIdx.x] = t;
  }
}

// Large grids: the span totals become exclusive prefixes in place (one CTA,
// each thread a run of consecutive spans), so that a compaction CTA reads its
// first rank instead of adding up every earlier span (quadratic in spans).
constexpr int kScanThreads = 1024;
constexpr unsigned kPrefixSpans = 4096;  // above this many spans the totals are scanned first

__global__ void __launch_bounds__(kScanThreads) scan_spans_kernel(int32_t* span_sum, uint32_t spans) {
  __shared__ int wpart[kScanThreads / 32];
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t per = (spans + kScanThreads - 1) / kScanThreads;
  const uint32_t a = threadIdx.x * per;
  const uint32_t b = a + per < spans ? a + per : spans;
  int mine = 0;
  for (uint32_t i = a; i < b; ++i) mine += span_sum[i];
  int inc = mine;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int t = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += t;
  }
  if (lane == 31) wpart[w] = inc;
  __syncthreads();
  if (w == 0) {
    int v = wpart[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int t = __shfl_up_sync(0xffffffffu, v, o);
      if (lane >= o) v += t;
    }
    wpart[lane] = v;  // inclusive over warps
  }
  __syncthreads();
  int run = (w > 0 ? wpart[w - 1] : 0) + inc - mine;  // exclusive prefix of this thread's run
  for (uint32_t i = a; i < b; ++i) {
    const int t = span_sum[i];
    span_sum[i] = run;
    run += t;
  }
}

template <bool kVec>
__global__ void __launch_bounds__(kAggThreads) compact_kernel(const uint8_t* __restrict__ mask, uint32_t cells,
                                                              int nb, uint32_t rows, uint32_t span,
                                                              const int32_t* __restrict__ span_sum,
                                                              int32_t* __restrict__ row_ptr,
                                                              int32_t* __restrict__ col_idx, int64_t nnz_cap,
                                                              int64_t* nnz_out, int* status, bool prefixed) {
  __shared__ int wbefore[kAggWarps];
  __shared__ int wtot[2][kAggWarps];
  __shared__ int32_t stage[kAggWarps][32 * kAggChunk];  // a warp's columns of one round
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int cap = nnz_cap < cells ? static_cast<int>(nnz_cap) : static_cast<int>(cells);  // ranks < cells
  // the kept cells of every earlier span (already summed when prefixed)
  int before = 0;
  if (prefixed) {
    if (threadIdx.x == 0) before = span_sum[blockIdx.x];
  } else {
    for (uint32_t i = threadIdx.x; i < blockIdx.x; i += kAggThreads) before += span_sum[i];
  }
  before = static_cast<int>(__reduce_add_sync(0xffffffffu, static_cast<unsigned>(before)));
  if (lane == 0) wbefore[w] = before;
  __syncthreads();
  int rank0 = 0;  // rank of the current round's first kept cell
#pragma unroll
  for (int i = 0; i < kAggWarps; ++i) rank0 += wbefore[i];
  const uint32_t s0 = blockIdx.x * span;
  const uint32_t s1 = cells - s0 > span ? s0 + span : cells;
  // row and column of the lane's chunk start, advanced by one round per step
  const uint32_t unb = static_cast<uint32_t>(nb);
  const uint32_t g0 = s0 + threadIdx.x * kAggChunk;
  uint32_t row = g0 / unb;
  int col = static_cast<int>(g0 - row * unb);
  const uint32_t row_step = kAggRound / unb;
  const int col_step = static_cast<int>(kAggRound % unb);
  int32_t* const my_stage = stage[w];
  int buf = 0;
  for (uint32_t g = g0; g - threadIdx.x * kAggChunk < s1; g += kAggRound, buf ^= 1) {  // uniform over the CTA
    uint32_t m[4] = {0u, 0u, 0u, 0u};
    if (kVec && g + kAggChunk <= s1) {
      const uint4 v = *reinterpret_cast<const uint4*>(mask + g);
      m[0] = v.x;
      m[1] = v.y;
      m[2] = v.z;
      m[3] = v.w;
    } else {
      for (uint32_t j = 0; j < kAggChunk && g + j < s1; ++j)
        m[j >> 2] |= static_cast<uint32_t>(mask[g + j] != 0) << (8 * (j & 3));
    }
    const uint32_t bits = chunk_bits(m);
    const int c = __popc(bits);
    int inc = c;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int t = __shfl_up_sync(0xffffffffu, inc, o);
      if (lane >= o) inc += t;
    }
    if (lane == 31) wtot[buf][w] = inc;
    __syncthreads();  // wtot[buf] is rewritten two rounds later, after the next round's barrier
    int wbase = 0, rtot = 0;
#pragma unroll
    for (int i = 0; i < kAggWarps; ++i) {
      const int t = wtot[buf][i];
      wbase += i < w ? t : 0;
      rtot += t;
    }
    const int wpos = rank0 + wbase;  // the warp's first rank this round
    rank0 += rtot;
    int at = inc - c;  // the lane's first slot in the warp's stage
    if (g < s1) {
      const int len = s1 - g < kAggChunk ? static_cast<int>(s1 - g) : kAggChunk;
      if (col + len <= nb) {  // the chunk lies in one row
        if (col == 0) row_ptr[row] = wpos + at;
#pragma unroll
        for (int j = 0; j < kAggChunk; ++j)
          if ((bits >> j) & 1u) my_stage[at++] = col + j;
      } else {
        // rows that start in the chunk: their first cell's rank
        uint32_t rr = row + (col != 0 ? 1u : 0u);
        for (int j = col != 0 ? nb - col : 0; j < len; j += nb, ++rr)
          row_ptr[rr] = wpos + at + __popc(bits & ((1u << j) - 1u));
        for (uint32_t b = bits; b; b &= b - 1) {
          int cc = col + __ffs(b) - 1;
          while (cc >= nb) cc -= nb;
          my_stage[at++] = cc;
        }
      }
    }
    col += col_step;
    row += row_step;
    if (col >= nb) {
      col -= nb;
      ++row;
    }
    __syncwarp();
    // the warp's kept columns are one run of col_idx: coalesced stores
    const int wcount = __shfl_sync(0xffffffffu, inc, 31);
    const int lim = cap - wpos < wcount ? cap - wpos : wcount;
    for (int i = lane; i < lim; i += 32) col_idx[wpos + i] = my_stage[i];
    __syncwarp();
  }
  if (blockIdx.x == gridDim.x - 1 && threadIdx.x == 0) {
    row_ptr[rows] = rank0;
    *nnz_out = rank0;
    if (rank0 > nnz_cap) record_error(status, CALIBATT_ERR_CAPACITY);
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
  const int64_t cells = rows * nb;
  // rounds per span: at least one row's worth of cells (so spans <= rows),
  // else up to 4 while the grid still overfills the SMs
  const int64_t by_row = (nb + kAggRound - 1) / kAggRound;
  int64_t by_fill = (cells + kAggRound * kAggFill - 1) / (kAggRound * kAggFill);
  if (by_fill > 4) by_fill = 4;
  const int64_t span = (by_row > by_fill ? by_row : by_fill) * kAggRound;
  const unsigned ctas = static_cast<unsigned>((cells + span - 1) / span);
  const bool vec = ((reinterpret_cast<uintptr_t>(counts) | reinterpret_cast<uintptr_t>(mask)) & 15u) == 0;
  // cells <= INT_MAX (checked by every caller): 32-bit flat indices
  const uint32_t c32 = static_cast<uint32_t>(cells), s32 = static_cast<uint32_t>(span);
  const uint32_t r32 = static_cast<uint32_t>(rows);
  const bool prefixed = ctas > kPrefixSpans;
  if (vec) {
    binarize_kernel<true><<<ctas, kAggThreads, 0, stream>>>(counts, c32, s32, threshold, mask, scratch);
    if (prefixed) scan_spans_kernel<<<1, kScanThreads, 0, stream>>>(scratch, ctas);
    compact_kernel<true><<<ctas, kAggThreads, 0, stream>>>(mask, c32, nb, r32, s32, scratch, row_ptr, col_idx,
                                                           nnz_cap, nnz, status, prefixed);
  } else {
    binarize_kernel<false><<<ctas, kAggThreads, 0, stream>>>(counts, c32, s32, threshold, mask, scratch);
    if (prefixed) scan_spans_kernel<<<1, kScanThreads, 0, stream>>>(scratch, ctas);
    compact_kernel<false><<<ctas, kAggThreads, 0, stream>>>(mask, c32, nb, r32, s32, scratch, row_ptr, col_idx,
                                                            nnz_cap, nnz, status, prefixed);
  }
  return cudaGetLastError() == cudaSuccess ? CALIBATT_OK : CALIBATT_ERR_CUDA;
}

// spans <= rows: a span holds at least nb cells
int64_t aggregate_scratch_ints(int64_t rows) { return rows; }

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
