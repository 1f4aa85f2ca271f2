// C-ABI entry points of libcalibatt: argument checks, host-side helpers
// (skip-list validation, tile-scheduler plan, anchor rows, thresholds) and
// kernel dispatch. Nothing here computes on the host what a kernel computes.
#include <cuda_runtime.h>

#include <algorithm>
#include <climits>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <numeric>
#include <vector>

#include "calibatt.h"
#include "kernels.h"
#include "sched.cuh"

namespace calibatt {

__device__ int g_status = 0;

int* status_word() {
  static std::mutex mu;
  static int* addr[64] = {nullptr};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (!addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_status) != cudaSuccess) return nullptr;
    addr[dev] = static_cast<int*>(p);
  }
  return addr[dev];
}

long long eps_to_fixed(double eps) {
  if (!(eps > 0.0)) return 0;
  if (eps >= 8192.0) return LLONG_MAX;
  return static_cast<long long>(std::ceil(std::ldexp(eps, 50)));
}

namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

int check_qkv(const void* q, const void* k, const void* v, const void* o, int heads, int n, int d) {
  if (!q || !k || (v == nullptr && o != nullptr)) return CALIBATT_ERR_ARG;
  if (heads < 1 || n < 1) return CALIBATT_ERR_ARG;
  if (d != CALIBATT_HEAD_DIM) return CALIBATT_ERR_UNSUPPORTED;
  const int64_t nb = (static_cast<int64_t>(n) + 127) / 128;
  if (nb * heads > INT_MAX / 2 || static_cast<int64_t>(n) * heads > (INT64_MAX >> 10)) return CALIBATT_ERR_ARG;
  if (!aligned16(q) || !aligned16(k) || (v && !aligned16(v)) || (o && !aligned16(o))) return CALIBATT_ERR_ALIGN;
  return CALIBATT_OK;
}

bool scale_ok(float s) { return std::isfinite(s) && s > 0.f; }

KernelParams base_params() {
  KernelParams p;
  std::memset(&p, 0, sizeof p);
  p.status = status_word();
  return p;
}


// Anchor-query segment of the attention kernel for n_rep repeated heads: the
// packed anchor queries (calibatt_repeat_workspace_size layout), the band of
// rows each anchor row is broadcast to (nearest anchor, ties to the lower
// one), and the anchor rows for the gather.
void set_repeat_segment(KernelParams& p, int frames, int H, int W, int k_anchor, int n_rep, const int32_t* rep_heads,
                        AnchorTable& tab) {
  int32_t anchors[kMaxAnchors];
  calibatt_anchor_rows(H, k_anchor, anchors);
  for (int j = 0; j < k_anchor; ++j) {
    p.band_lo[j] = INT_MAX;
    p.band_hi[j] = 0;
    tab.anchor[j] = anchors[j];
  }
  for (int r = 0; r < H; ++r) {
    int best = 0;
    for (int j = 1; j < k_anchor; ++j)
      if (std::abs(r - anchors[j]) < std::abs(r - anchors[best])) best = j;
    p.band_lo[best] = std::min(p.band_lo[best], r);
    p.band_hi[best] = std::max(p.band_hi[best], r + 1);
  }
  p.n_q_b = frames * k_anchor * W;
  p.nbq_b = (p.n_q_b + 127) / 128;
  p.heads_q_b = n_rep;
  p.head_map_b = rep_heads;
  p.rep_H = H;
  p.rep_W = W;
  p.rep_k = k_anchor;
}

}  // namespace
}  // namespace calibatt

using namespace calibatt;

extern "C" {

const char* calibatt_strerror(int code) {
  switch (code) {
    case CALIBATT_OK: return "ok";
    case CALIBATT_ERR_ARG: return "invalid argument";
    case CALIBATT_ERR_CSR: return "malformed skip list (row_ptr / col_idx)";
    case CALIBATT_ERR_ALIGN: return "device pointer not 16-byte aligned";
    case CALIBATT_ERR_UNSUPPORTED: return "unsupported shape (head dim must be 128; calibration needs nb <= 1024)";
    case CALIBATT_ERR_CUDA: return "CUDA call failed";
    case CALIBATT_ERR_TIMEOUT: return "bounded in-kernel wait ran out";
    case CALIBATT_ERR_CAPACITY: return "kept blocks exceed col_idx capacity";
    default: return "unknown status";
  }
}

int calibatt_version(void) { return 100; }

int calibatt_get_status(calibatt_stream_t stream) {
  if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) return CALIBATT_ERR_CUDA;
  int* w = status_word();
  if (!w) return CALIBATT_ERR_CUDA;
  int v = 0;
  if (cudaMemcpy(&v, w, sizeof v, cudaMemcpyDeviceToHost) != cudaSuccess) return CALIBATT_ERR_CUDA;
  if (v != 0) {
    const int zero = 0;
    if (cudaMemcpy(w, &zero, sizeof zero, cudaMemcpyHostToDevice) != cudaSuccess) return CALIBATT_ERR_CUDA;
  }
  return v;
}

double calibatt_eps_schedule(double A, double C, double k, double t, double T) {
  return A + (C - A) * std::exp(-k * t / T);
}

int calibatt_validate_csr(const int32_t* row_ptr, const int32_t* col_idx, int heads, int nb, int64_t nnz) {
  if (!row_ptr || heads < 1 || nb < 1 || nnz < 0 || (nnz > 0 && !col_idx)) return CALIBATT_ERR_ARG;
  const int64_t rows = static_cast<int64_t>(heads) * nb;
  if (row_ptr[0] != 0 || row_ptr[rows] != nnz) return CALIBATT_ERR_CSR;
  for (int64_t r = 0; r < rows; ++r) {
    const int64_t a = row_ptr[r], b = row_ptr[r + 1];
    if (b < a || b > nnz) return CALIBATT_ERR_CSR;
    for (int64_t i = a; i < b; ++i) {
      if (col_idx[i] < 0 || col_idx[i] >= nb) return CALIBATT_ERR_CSR;
      if (i > a && col_idx[i] <= col_idx[i - 1]) return CALIBATT_ERR_CSR;
    }
  }
  return CALIBATT_OK;
}

int calibatt_build_plan(const int32_t* row_ptr, int heads, int nb, const uint8_t* head_active, int32_t* work_list,
                        int32_t* n_work) {
  if (!row_ptr || !work_list || !n_work || heads < 1 || nb < 1) return CALIBATT_ERR_ARG;
  if (static_cast<int64_t>(heads) * nb > INT_MAX / 2) return CALIBATT_ERR_ARG;
  int32_t* out = work_list;
  std::vector<int32_t> units(static_cast<size_t>(nb));
  for (int h = 0; h < heads; ++h) {
    if (head_active && !head_active[h]) continue;
    for (int r = 0; r < nb; ++r) {
      units[r] = h * nb + r;
      if (row_ptr[units[r] + 1] < row_ptr[units[r]]) return CALIBATT_ERR_CSR;
    }
    // longest first within the head; equal counts keep block order
    std::stable_sort(units.begin(), units.end(), [&](int32_t a, int32_t b) {
      return (row_ptr[a + 1] - row_ptr[a]) > (row_ptr[b + 1] - row_ptr[b]);
    });
    out = std::copy(units.begin(), units.end(), out);
  }
  *n_work = static_cast<int32_t>(out - work_list);
  return CALIBATT_OK;
}

int calibatt_anchor_rows(int H, int k_anchor, int32_t* anchors) {
  if (!anchors || H < 1 || k_anchor < 1 || k_anchor > H) return CALIBATT_ERR_ARG;
  for (int j = 0; j < k_anchor; ++j)
    anchors[j] = static_cast<int32_t>((static_cast<int64_t>(2 * j + 1) * H) / (2 * static_cast<int64_t>(k_anchor)));
  return CALIBATT_OK;
}

int calibatt_rho_threshold(int n_inputs, double rho, int32_t* threshold) {
  if (!threshold || n_inputs < 1 || !std::isfinite(rho)) return CALIBATT_ERR_ARG;
  for (int c = 0; c <= n_inputs; ++c)
    if (static_cast<double>(c) / static_cast<double>(n_inputs) >= rho) {
      *threshold = c;
      return CALIBATT_OK;
    }
  *threshold = n_inputs + 1;
  return CALIBATT_OK;
}

int calibatt_sparse_attn_fwd(const calibatt_bf16* q, const calibatt_bf16* k, const calibatt_bf16* v, int heads,
                             int n, int d, float scale, const int32_t* row_ptr, const int32_t* col_idx, int64_t nnz,
                             const int32_t* work_list, int32_t n_work, calibatt_bf16* o, float* lse,
                             calibatt_stream_t stream) {
  if (!v || !o) return CALIBATT_ERR_ARG;
  int rc = check_qkv(q, k, v, o, heads, n, d);
  if (rc != CALIBATT_OK) return rc;
  const int nb = (n + 127) / 128;
  if (!scale_ok(scale) || !row_ptr || nnz < 0 || (nnz > 0 && !col_idx) || n_work < 0 ||
      static_cast<int64_t>(n_work) > static_cast<int64_t>(heads) * nb || (n_work > 0 && !work_list))
    return CALIBATT_ERR_ARG;
  if (lse && !aligned4(lse)) return CALIBATT_ERR_ALIGN;
  KernelParams p = base_params();
  if (!p.status) return CALIBATT_ERR_CUDA;
  p.n_q = p.n_k = n;
  p.nbq = p.nbk = nb;
  p.heads_q = p.heads_kv = heads;
  p.n_units = n_work;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.work_list = work_list;
  p.row_ptr = row_ptr;
  p.col_idx = col_idx;
  p.nnz = nnz;
  p.o = reinterpret_cast<__nv_bfloat16*>(o);
  p.lse = lse;
  p.n_out = n;
  return launch_attention(0, q, n, heads, k, v, n, heads, p, reinterpret_cast<cudaStream_t>(stream));
}

int calibatt_build_mixed_plan(const int32_t* row_ptr, int heads, int nb, const uint8_t* head_active, int n_rep,
                              const int32_t* rep_heads, int frames, int H, int W, int k_anchor, int32_t* work_list,
                              int32_t* n_work) {
  if (!row_ptr || !work_list || !n_work || heads < 1 || nb < 1 || n_rep < 0 || n_rep > heads ||
      (n_rep > 0 && !rep_heads) || frames < 1 || H < 1 || W < 1 || k_anchor < 1 || k_anchor > H)
    return CALIBATT_ERR_ARG;
  const int64_t nbq_b = (static_cast<int64_t>(frames) * k_anchor * W + 127) / 128;
  if (static_cast<int64_t>(heads) * nb + n_rep * nbq_b > INT_MAX / 2) return CALIBATT_ERR_ARG;
  for (int i = 0; i < n_rep; ++i)
    if (rep_heads[i] < 0 || rep_heads[i] >= heads) return CALIBATT_ERR_ARG;
  int32_t* out = work_list;
  // first the repeated heads' anchor-query units (each takes every key block)
  for (int i = 0; i < n_rep; ++i)
    for (int64_t b = 0; b < nbq_b; ++b) *out++ = static_cast<int32_t>(heads * nb + i * nbq_b + b);
  std::vector<int32_t> units(static_cast<size_t>(nb));
  for (int h = 0; h < heads; ++h) {
    bool repeated = false;
    for (int i = 0; i < n_rep; ++i) repeated = repeated || rep_heads[i] == h;
    if (repeated || (head_active && !head_active[h])) continue;
    for (int r = 0; r < nb; ++r) {
      units[r] = h * nb + r;
      if (row_ptr[units[r] + 1] < row_ptr[units[r]]) return CALIBATT_ERR_CSR;
    }
    std::stable_sort(units.begin(), units.end(), [&](int32_t a, int32_t b) {
      return (row_ptr[a + 1] - row_ptr[a]) > (row_ptr[b + 1] - row_ptr[b]);
    });
    out = std::copy(units.begin(), units.end(), out);
  }
  *n_work = static_cast<int32_t>(out - work_list);
  return CALIBATT_OK;
}

int calibatt_mixed_attn_fwd(const calibatt_bf16* q, const calibatt_bf16* k, const calibatt_bf16* v, int heads,
                            int frames, int H, int W, int d, int k_anchor, float scale, const int32_t* row_ptr,
                            const int32_t* col_idx, int64_t nnz, const int32_t* rep_heads, int32_t n_rep,
                            const int32_t* work_list, int32_t n_work, calibatt_bf16* o, float* lse, void* ws,
                            size_t ws_bytes, calibatt_stream_t stream) {
  if (!v || !o || frames < 1 || H < 1 || W < 1) return CALIBATT_ERR_ARG;
  const int64_t n64 = static_cast<int64_t>(frames) * H * W;
  if (n64 > INT_MAX / 2) return CALIBATT_ERR_ARG;
  const int n = static_cast<int>(n64);
  int rc = check_qkv(q, k, v, o, heads, n, d);
  if (rc != CALIBATT_OK) return rc;
  if (k_anchor < 1 || k_anchor > H) return CALIBATT_ERR_ARG;
  if (k_anchor > kMaxAnchors) return CALIBATT_ERR_UNSUPPORTED;
  const int nb = (n + 127) / 128;
  const int64_t nbq_b = (static_cast<int64_t>(frames) * k_anchor * W + 127) / 128;
  if (!scale_ok(scale) || !row_ptr || nnz < 0 || (nnz > 0 && !col_idx) || n_rep < 0 || n_rep > heads ||
      (n_rep > 0 && !rep_heads) || n_work < 0 ||
      static_cast<int64_t>(n_work) > static_cast<int64_t>(heads) * nb + n_rep * nbq_b ||
      (n_work > 0 && !work_list))
    return CALIBATT_ERR_ARG;
  if (n_rep > 0 && (!ws || ws_bytes < calibatt_repeat_workspace_size(n_rep, frames, H, W, k_anchor)))
    return CALIBATT_ERR_ARG;
  if ((n_rep > 0 && !aligned16(ws)) || (lse && !aligned4(lse))) return CALIBATT_ERR_ALIGN;
  KernelParams p = base_params();
  if (!p.status) return CALIBATT_ERR_CUDA;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (n_rep > 0) {
    AnchorTable tab;
    set_repeat_segment(p, frames, H, W, k_anchor, n_rep, rep_heads, tab);
    rc = launch_gather(q, n, heads, rep_heads, n_rep, H, W, k_anchor, tab, ws, p.status, st);
    if (rc != CALIBATT_OK) return rc;
  }
  p.n_q = p.n_k = n;
  p.nbq = p.nbk = nb;
  p.heads_q = p.heads_kv = heads;
  p.n_units = n_work;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.work_list = work_list;
  p.row_ptr = row_ptr;
  p.col_idx = col_idx;
  p.nnz = nnz;
  p.o = reinterpret_cast<__nv_bfloat16*>(o);
  p.lse = lse;
  p.n_out = n;
  return launch_attention(0, q, n, heads, k, v, n, heads, p, st, n_rep > 0 ? ws : nullptr, p.n_q_b, n_rep);
}

size_t calibatt_repeat_workspace_size(int n_rep, int frames, int H, int W, int k_anchor) {
  if (n_rep < 1 || frames < 1 || H < 1 || W < 1 || k_anchor < 1) return 0;
  const size_t bytes = static_cast<size_t>(n_rep) * frames * k_anchor * W * 128 * 2;
  return (bytes + 255) & ~static_cast<size_t>(255);
}

int calibatt_repeat_attn_fwd(const calibatt_bf16* q, const calibatt_bf16* k, const calibatt_bf16* v, int heads,
                             int frames, int H, int W, int d, int k_anchor, float scale, const int32_t* rep_heads,
                             int32_t n_rep, calibatt_bf16* o, float* lse, void* ws, size_t ws_bytes,
                             calibatt_stream_t stream) {
  if (!v || !o || frames < 1 || H < 1 || W < 1) return CALIBATT_ERR_ARG;
  const int64_t n64 = static_cast<int64_t>(frames) * H * W;
  if (n64 > INT_MAX / 2) return CALIBATT_ERR_ARG;
  const int n = static_cast<int>(n64);
  int rc = check_qkv(q, k, v, o, heads, n, d);
  if (rc != CALIBATT_OK) return rc;
  if (k_anchor < 1 || k_anchor > H) return CALIBATT_ERR_ARG;
  if (k_anchor > kMaxAnchors) return CALIBATT_ERR_UNSUPPORTED;
  if (!scale_ok(scale) || n_rep < 0 || n_rep > heads || (n_rep > 0 && !rep_heads)) return CALIBATT_ERR_ARG;
  if (n_rep == 0) return CALIBATT_OK;
  if (!ws || ws_bytes < calibatt_repeat_workspace_size(n_rep, frames, H, W, k_anchor)) return CALIBATT_ERR_ARG;
  if (!aligned16(ws) || (lse && !aligned4(lse))) return CALIBATT_ERR_ALIGN;

  KernelParams p = base_params();
  if (!p.status) return CALIBATT_ERR_CUDA;
  AnchorTable tab;
  set_repeat_segment(p, frames, H, W, k_anchor, n_rep, rep_heads, tab);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  rc = launch_gather(q, n, heads, rep_heads, n_rep, H, W, k_anchor, tab, ws, p.status, st);
  if (rc != CALIBATT_OK) return rc;
  p.n_k = n;
  p.nbk = (n + 127) / 128;
  p.heads_kv = heads;
  p.n_units = n_rep * p.nbq_b;  // every unit is an anchor-query unit (no first segment)
  p.scale_log2 = scale * 1.4426950408889634f;
  p.o = reinterpret_cast<__nv_bfloat16*>(o);
  p.lse = lse;
  p.n_out = n;
  return launch_attention(0, ws, p.n_q_b, n_rep, k, v, n, heads, p, st, ws, p.n_q_b, n_rep);
}

int calibatt_block_energy(const calibatt_bf16* q, const calibatt_bf16* k, int heads, int n, int d, float scale,
                          float* lse_ws, float* energy, int fuse_select, double eps, uint8_t* mask, int32_t* kept,
                          uint16_t* counts, calibatt_stream_t stream) {
  int rc = check_qkv(q, k, nullptr, nullptr, heads, n, d);
  if (rc != CALIBATT_OK) return rc;
  const int nb = (n + 127) / 128;
  if (nb > CALIBATT_MAX_CALIB_NB) return CALIBATT_ERR_UNSUPPORTED;
  if (!scale_ok(scale) || !lse_ws || std::isnan(eps)) return CALIBATT_ERR_ARG;
  if (fuse_select && !mask && !kept && !counts) return CALIBATT_ERR_ARG;
  if (!aligned4(lse_ws) || (energy && !aligned4(energy)) || (kept && !aligned4(kept)) ||
      (counts && (reinterpret_cast<uintptr_t>(counts) & 1u)))
    return CALIBATT_ERR_ALIGN;
  KernelParams p = base_params();
  if (!p.status) return CALIBATT_ERR_CUDA;
  p.n_q = p.n_k = n;
  p.nbq = p.nbk = nb;
  p.heads_q = p.heads_kv = heads;
  p.n_units = heads * nb;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.n_out = n;
  p.lse_ws = lse_ws;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  rc = launch_attention(1, q, n, heads, k, nullptr, n, heads, p, st);
  if (rc != CALIBATT_OK) return rc;
  p.energy = energy;
  p.fuse_select = fuse_select ? 1 : 0;
  p.eps_fx = eps_to_fixed(eps);
  p.mask = fuse_select ? mask : nullptr;
  p.kept = fuse_select ? kept : nullptr;
  p.counts = fuse_select ? counts : nullptr;
  return launch_attention(2, q, n, heads, k, nullptr, n, heads, p, st);
}

size_t calibatt_energy_workspace_size(int heads, int n) {
  if (heads < 1 || n < 1) return 0;
  const int64_t nb = (static_cast<int64_t>(n) + 127) / 128;
  const int64_t units = heads * nb;
  if (units > INT_MAX / 2 || nb > CALIBATT_MAX_CALIB_NB) return 0;
  const size_t bytes = static_cast<size_t>(2 * score_grid(static_cast<int>(units))) * nb * 128 * sizeof(float2);
  return (bytes + 255) & ~static_cast<size_t>(255);
}

int calibatt_block_energy_1pass(const calibatt_bf16* q, const calibatt_bf16* k, int heads, int n, int d,
                                float scale, void* ws, size_t ws_bytes, float* energy, int fuse_select, double eps,
                                uint8_t* mask, int32_t* kept, uint16_t* counts, float* pix_energy, int pix_W,
                                calibatt_stream_t stream) {
  int rc = check_qkv(q, k, nullptr, nullptr, heads, n, d);
  if (rc != CALIBATT_OK) return rc;
  const int nb = (n + 127) / 128;
  if (nb > CALIBATT_MAX_CALIB_NB) return CALIBATT_ERR_UNSUPPORTED;
  if (!scale_ok(scale) || !ws || std::isnan(eps)) return CALIBATT_ERR_ARG;
  if (ws_bytes < calibatt_energy_workspace_size(heads, n)) return CALIBATT_ERR_ARG;
  if (fuse_select && !mask && !kept && !counts) return CALIBATT_ERR_ARG;
  if (pix_energy && (pix_W < 1 || n % pix_W != 0)) return CALIBATT_ERR_ARG;
  if (!aligned16(ws) || (energy && !aligned4(energy)) || (kept && !aligned4(kept)) ||
      (counts && (reinterpret_cast<uintptr_t>(counts) & 1u)) || (pix_energy && !aligned4(pix_energy)))
    return CALIBATT_ERR_ALIGN;
  KernelParams p = base_params();
  if (!p.status) return CALIBATT_ERR_CUDA;
  p.n_q = p.n_k = n;
  p.nbq = p.nbk = nb;
  p.heads_q = p.heads_kv = heads;
  p.n_units = heads * nb;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.n_out = n;
  p.energy_ws = static_cast<float2*>(ws);
  p.energy = energy;
  p.fuse_select = fuse_select ? 1 : 0;
  p.eps_fx = eps_to_fixed(eps);
  p.mask = fuse_select ? mask : nullptr;
  p.kept = fuse_select ? kept : nullptr;
  p.counts = fuse_select ? counts : nullptr;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (pix_energy) {
    const size_t pix_bytes = static_cast<size_t>(heads) * (n / pix_W) * nb * sizeof(float);
    if (cudaMemsetAsync(pix_energy, 0, pix_bytes, st) != cudaSuccess) return CALIBATT_ERR_CUDA;
    p.pix_energy = pix_energy;
    p.pix_W = pix_W;
    p.pix_rows = n / pix_W;
    p.pix_inv_W = 1.0f / static_cast<float>(pix_W);
  }
  return launch_attention(3, q, n, heads, k, nullptr, n, heads, p, st);
}

int calibatt_select_mask(const float* energy, int heads, int nb, double eps, uint8_t* mask, int32_t* kept,
                         uint16_t* counts, calibatt_stream_t stream) {
  if (!energy || heads < 1 || nb < 1 || std::isnan(eps)) return CALIBATT_ERR_ARG;
  if (nb > CALIBATT_MAX_CALIB_NB) return CALIBATT_ERR_UNSUPPORTED;
  if (!mask && !kept && !counts) return CALIBATT_ERR_ARG;
  if (!aligned4(energy) || (kept && !aligned4(kept)) || (counts && (reinterpret_cast<uintptr_t>(counts) & 1u)))
    return CALIBATT_ERR_ALIGN;
  return launch_select(energy, static_cast<int64_t>(heads) * nb, nb, eps_to_fixed(eps), mask, kept, counts,
                       reinterpret_cast<cudaStream_t>(stream));
}

int calibatt_accumulate_masks(const uint8_t* mask, int64_t cells, uint16_t* counts, calibatt_stream_t stream) {
  if (cells < 0 || (cells > 0 && (!mask || !counts))) return CALIBATT_ERR_ARG;
  if (counts && (reinterpret_cast<uintptr_t>(counts) & 1u)) return CALIBATT_ERR_ALIGN;
  return launch_accumulate(mask, cells, counts, reinterpret_cast<cudaStream_t>(stream));
}

size_t calibatt_aggregate_workspace_size(int heads, int nb) {
  if (heads < 1 || nb < 1) return 0;
  const size_t bytes = static_cast<size_t>(heads) * nb * sizeof(int32_t);
  return (bytes + 255) & ~static_cast<size_t>(255);
}

int calibatt_pixel_row_energy(const calibatt_bf16* q, const calibatt_bf16* k, int heads, int frames, int H,
                              int W, int d, float scale, float* lse_ws, float* energy, float* pix_energy,
                              calibatt_stream_t stream) {
  if (frames < 1 || H < 1 || W < 1 || !pix_energy) return CALIBATT_ERR_ARG;
  const int64_t n64 = static_cast<int64_t>(frames) * H * W;
  if (n64 > INT_MAX / 2) return CALIBATT_ERR_ARG;
  const int n = static_cast<int>(n64);
  int rc = check_qkv(q, k, nullptr, nullptr, heads, n, d);
  if (rc != CALIBATT_OK) return rc;
  const int nb = (n + 127) / 128;
  if (nb > CALIBATT_MAX_CALIB_NB) return CALIBATT_ERR_UNSUPPORTED;
  if (!scale_ok(scale) || !lse_ws) return CALIBATT_ERR_ARG;
  if (!aligned4(lse_ws) || (energy && !aligned4(energy)) || !aligned4(pix_energy)) return CALIBATT_ERR_ALIGN;
  KernelParams p = base_params();
  if (!p.status) return CALIBATT_ERR_CUDA;
  p.n_q = p.n_k = n;
  p.nbq = p.nbk = nb;
  p.heads_q = p.heads_kv = heads;
  p.n_units = heads * nb;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.n_out = n;
  p.lse_ws = lse_ws;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const size_t pix_bytes = static_cast<size_t>(heads) * frames * H * nb * sizeof(float);
  if (cudaMemsetAsync(pix_energy, 0, pix_bytes, st) != cudaSuccess) return CALIBATT_ERR_CUDA;
  rc = launch_attention(1, q, n, heads, k, nullptr, n, heads, p, st);
  if (rc != CALIBATT_OK) return rc;
  p.energy = energy;
  p.pix_energy = pix_energy;
  p.pix_W = W;
  p.pix_rows = frames * H;
  p.pix_inv_W = 1.0f / static_cast<float>(W);
  return launch_attention(2, q, n, heads, k, nullptr, n, heads, p, st);
}

int calibatt_spatial_score(const float* pix_energy, int heads, int frames, int H, int nb, int k_anchor,
                           float gamma, float* score, uint8_t* flag, calibatt_stream_t stream) {
  static_assert(kMaxFrameRows == CALIBATT_MAX_FRAME_ROWS, "frame-row table size");
  if (!pix_energy || !score || heads < 1 || frames < 1 || H < 1 || nb < 1 || k_anchor < 1 || k_anchor > H ||
      std::isnan(gamma))
    return CALIBATT_ERR_ARG;
  if (H > CALIBATT_MAX_FRAME_ROWS) return CALIBATT_ERR_UNSUPPORTED;
  if (static_cast<int64_t>(heads) * frames * H * nb > (int64_t{1} << 40)) return CALIBATT_ERR_ARG;
  if (!aligned4(pix_energy) || !aligned4(score)) return CALIBATT_ERR_ALIGN;
  int32_t anchors[CALIBATT_MAX_FRAME_ROWS];
  calibatt_anchor_rows(H, k_anchor, anchors);
  RowAnchorTable tab;
  for (int r = 0; r < H; ++r) {
    int best = 0;  // nearest anchor, ties to the lower one
    for (int j = 1; j < k_anchor; ++j)
      if (std::abs(r - anchors[j]) < std::abs(r - anchors[best])) best = j;
    tab.row[r] = anchors[best];
  }
  return launch_spatial_score(pix_energy, heads, frames, H, nb, tab, gamma, score, flag,
                              reinterpret_cast<cudaStream_t>(stream));
}

int calibatt_aggregate_masks(const uint16_t* counts, int n_inputs, int heads, int nb, double rho, uint8_t* mask,
                             int32_t* row_ptr, int32_t* col_idx, int64_t nnz_cap, int64_t* nnz, void* ws,
                             size_t ws_bytes, calibatt_stream_t stream) {
  if (!counts || !mask || !row_ptr || !nnz || heads < 1 || nb < 1 || n_inputs < 1 || nnz_cap < 0 ||
      (nnz_cap > 0 && !col_idx) || !std::isfinite(rho))
    return CALIBATT_ERR_ARG;
  if (static_cast<int64_t>(heads) * nb * nb > INT_MAX) return CALIBATT_ERR_ARG;
  if (!ws || ws_bytes < calibatt_aggregate_workspace_size(heads, nb)) return CALIBATT_ERR_ARG;
  if ((reinterpret_cast<uintptr_t>(counts) & 1u) || !aligned4(row_ptr) || (col_idx && !aligned4(col_idx)) ||
      (reinterpret_cast<uintptr_t>(nnz) & 7u) || !aligned4(ws))
    return CALIBATT_ERR_ALIGN;
  int* status = status_word();
  if (!status) return CALIBATT_ERR_CUDA;
  int32_t thr = 0;
  calibatt_rho_threshold(n_inputs, rho, &thr);
  return launch_aggregate(counts, static_cast<int64_t>(heads) * nb, nb, thr, mask, row_ptr, col_idx, nnz_cap, nnz,
                          static_cast<int32_t*>(ws), status, reinterpret_cast<cudaStream_t>(stream));
}

}  // extern "C"
