// Internal interface between the C-ABI entry points and the CUDA kernels.
#pragma once
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

namespace calibatt {

constexpr int kMaxAnchors = 64;

// Parameters of the persistent tensor-core attention kernel (all modes).
// Key blocks per chunk of the single-pass energy workspace.
constexpr int kEnergyChunk = 8;
// fp32 words of that workspace for `slots` query tiles of nb key blocks.
inline int64_t energy_ws_floats(int64_t slots, int64_t nb) {
  return slots * ((nb + kEnergyChunk - 1) / kEnergyChunk) * (kEnergyChunk + 1) * 128;
}

struct KernelParams {
  int n_q;        // query rows per head in the Q tensor
  int n_k;        // key rows per head
  int nbq, nbk;   // ceil(n_q / 128), ceil(n_k / 128)
  int heads_q;    // heads in the Q tensor
  int heads_kv;   // heads in K / V / O
  int n_units;    // work units
  float scale_log2;  // softmax scale * log2(e)
  const int32_t* work_list;  // unit -> hq * nbq + r (NULL: identity)
  const int32_t* row_ptr;    // skip list (NULL: every key block)
  const int32_t* col_idx;
  int64_t nnz;
  const int32_t* head_map;   // Q head -> K/V/O head (NULL: identity)
  __nv_bfloat16* o;          // output [heads_kv][n_out][128]
  float* lse;                // output [heads_kv][n_out] or NULL
  int64_t n_out;             // rows per head of o / lse
  // Second unit segment (attention only): anchor-query units of spatially
  // repeated heads, unit codes heads_q*nbq .. + heads_q_b*nbq_b - 1. Their Q
  // rows come from the packed anchor tensor (n_q_b rows per head), they take
  // every key block, and head_map_b gives their K/V/O head. nbq_b = 0: none.
  int n_q_b, nbq_b, heads_q_b;
  const int32_t* head_map_b;
  // optional skip list of the anchor-query units ([heads_q_b * nbq_b + 1]
  // global offsets into col_idx_b, columns ascending); NULL: every key block
  const int32_t* row_ptr_b;
  const int32_t* col_idx_b;
  int64_t nnz_b;
  // repeated heads: a packed anchor query q = f*(k*W) + j*W + c writes rows
  // band_lo[j] .. band_hi[j]-1 of frame f, column c
  int rep_H, rep_W, rep_k;
  int band_lo[kMaxAnchors], band_hi[kMaxAnchors];
  // energy passes
  float* lse_ws;       // [heads_q][nbq*128] row log2-sum-exp2 (log2 units)
  float* energy;       // [heads_q][nbq][nbk] or NULL
  int fuse_select;
  long long eps_fx;    // eps in fixed point (50 fraction bits), rounded up
  uint8_t* mask;
  int32_t* kept;
  uint16_t* counts;
  uint8_t* tie;        // [heads_q][nbq] tie-affected flags of the fused selection, or NULL
  long long tie_fx;    // tie window in fixed point (50 fraction bits)
  // pixel-row profiles (energy pass): pix_energy[hq][q / pix_W][c] += ... / pix_W
  float* pix_energy;   // [heads_q][pix_rows][nbk] or NULL
  int pix_W, pix_rows;
  float pix_inv_W;
  // single-pass energy: per slot, per chunk of kEnergyChunk key blocks, per
  // row: the chunk's tile sums relative to the row's running max at the
  // chunk's end, then that max
  float* energy_ws;    // [2 * grid][ceil(nbk / kEnergyChunk)][kEnergyChunk + 1][128]
  int* status;         // device status word
  uint64_t wait_limit_ns;  // limit of the pipeline's bounded waits
};

struct AnchorTable {
  int anchor[kMaxAnchors];
};

// For each row r of a frame, the row of its nearest anchor (spatial score).
constexpr int kMaxFrameRows = 512;
struct RowAnchorTable {
  int32_t row[kMaxFrameRows];
};

// qb: the packed anchor tensor of the second unit segment ([qb_heads][qb_rows][128])
// or NULL.
// Modes of launch_attention: 0 attention, 1 row LSE pass, 2 energy pass
// after it, 3 single-pass energy.
int launch_attention(int mode, const void* q, int q_rows, int q_heads, const void* k, const void* v, int kv_rows,
                     int kv_heads, const KernelParams& p, cudaStream_t stream, const void* qb = nullptr,
                     int qb_rows = 0, int qb_heads = 0);

long long eps_to_fixed(double eps);

int launch_select(const float* energy, int64_t rows, int nb, long long eps_fx, uint8_t* mask, int32_t* kept,
                  uint16_t* counts, uint8_t* tie, long long tie_fx, cudaStream_t stream);
int launch_accumulate(const uint8_t* mask, int64_t cells, uint16_t* counts, cudaStream_t stream);
// scratch: aggregate_scratch_ints(rows) int32 (one kept total per span of
// the flat mask, at most one span per row), rewritten by each call
int launch_aggregate(const uint16_t* counts, int64_t rows, int nb, int threshold, uint8_t* mask, int32_t* row_ptr,
                     int32_t* col_idx, int64_t nnz_cap, int64_t* nnz, int32_t* scratch, int* status,
                     cudaStream_t stream);
int64_t aggregate_scratch_ints(int64_t rows);
int launch_spatial_score(const float* pix, int heads, int frames, int H, int nb, const RowAnchorTable& tab,
                         float gamma, float* score, uint8_t* flag, cudaStream_t stream);
int launch_gather(const void* q, int n, int heads, const int32_t* rep_heads, int n_rep, int H, int W, int k_anchor,
                  const AnchorTable& tab, void* out, int* status, cudaStream_t stream);

// Device address of the status word on the current device (NULL on failure).
int* status_word();

// Limit of the bounded in-kernel waits of launches on the current device.
uint64_t wait_limit_ns();

// Tie window (in the greedy sum's units) in fixed point; 0 for none.
long long tie_window_fixed(double window);

}  // namespace calibatt
