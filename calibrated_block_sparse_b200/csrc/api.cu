// C-ABI entry points of libcalibatt: argument checks, host-side helpers
// (skip-list validation, tile-scheduler plan, anchor rows, thresholds) and
// kernel dispatch. Nothing here computes on the host what a kernel computes.
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
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

// Limit of the bounded in-kernel waits per device (0: the default).
std::atomic<uint64_t> g_wait_limit[64];

uint64_t wait_limit_ns() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return kWaitLimitNs;
  const uint64_t v = g_wait_limit[dev].load(std::memory_order_relaxed);
  return v ? v : kWaitLimitNs;
}

long long tie_window_fixed(double window) {
  if (!(window > 0.0)) return 0;
  if (window >= 8192.0) return LLONG_MAX;
  return static_cast<long long>(std::llround(std::ldexp(window, 50)));
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

// Query blocks of the packed anchor queries of one repeated head.
int64_t anchor_blocks(int frames, int W, int k_anchor) {
  return (static_cast<int64_t>(frames) * k_anchor * W + 127) / 128;
}

KernelParams base_params() {
  KernelParams p;
  std::memset(&p, 0, sizeof p);
  p.status = status_word();
  p.wait_limit_ns = wait_limit_ns();
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

int calibatt_version(void) { return 200; }

int calibatt_set_wait_limit(double seconds) {
  if (std::isnan(seconds) || seconds > 60.0) return CALIBATT_ERR_ARG;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return CALIBATT_ERR_CUDA;
  uint64_t ns = 0;  // default
  if (seconds > 0.0) {
    ns = static_cast<uint64_t>(std::llround(seconds * 1e9));
    if (ns == 0) ns = 1;
  }
  g_wait_limit[dev].store(ns, std::memory_order_relaxed);
  return CALIBATT_OK;
}

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

namespace {
// calibatt_balance_plan with the anchor-query units' costs taken from their
// own skip list (row_ptr_b [n_rep * nbq_b + 1]) when given.
int balance_plan(int32_t* work_list, int32_t n_work, const int32_t* row_ptr, int heads, int nb,
                 const int32_t* row_ptr_b, int64_t n_b_units, int n_slots) {
  if (!work_list || n_work < 0 || !row_ptr || heads < 1 || nb < 1) return CALIBATT_ERR_ARG;
  if (n_work == 0) return CALIBATT_OK;
  if (n_slots <= 0) {
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0)
      return CALIBATT_ERR_CUDA;
    n_slots = 2 * sms;
  }
  if (n_slots < 2) return CALIBATT_ERR_ARG;
  // the kernel's grid: one CTA of two slots per SM, no more CTAs than unit pairs
  const int64_t ctas = std::min<int64_t>(n_slots / 2, (static_cast<int64_t>(n_work) + 1) / 2);
  const int64_t G = 2 * ctas;
  const int64_t n_a = static_cast<int64_t>(heads) * nb;
  auto cost = [&](int32_t code) -> int64_t {
    if (code >= 0 && code < n_a) return static_cast<int64_t>(row_ptr[code + 1]) - row_ptr[code] + 2;
    if (code >= n_a && row_ptr_b && code - n_a < n_b_units)  // anchor-query unit with its own skip list
      return static_cast<int64_t>(row_ptr_b[code - n_a + 1]) - row_ptr_b[code - n_a] + 2;
    if (code >= n_a) return nb + 2;  // anchor-query unit: every key block
    return 2;
  };
  std::vector<int32_t> in(work_list, work_list + n_work);
  std::vector<int64_t> load(static_cast<size_t>(G), 0);
  std::vector<int64_t> units, slots;
  for (int64_t r = 0; r * G < n_work; ++r) {
    units.clear();
    slots.clear();
    for (int64_t i = r * G; i < std::min<int64_t>(n_work, (r + 1) * G); ++i) units.push_back(i);
    auto pos = [&](int64_t g) { return r * G + ((r & 1) ? (G - 1 - g) : g); };
    for (int64_t g = 0; g < G; ++g)
      if (pos(g) < n_work) slots.push_back(g);
    std::stable_sort(units.begin(), units.end(), [&](int64_t a, int64_t b) { return cost(in[a]) > cost(in[b]); });
    std::stable_sort(slots.begin(), slots.end(), [&](int64_t a, int64_t b) { return load[a] < load[b]; });
    for (size_t i = 0; i < units.size(); ++i) {
      work_list[pos(slots[i])] = in[units[i]];
      load[slots[i]] += cost(in[units[i]]);
    }
  }
  return CALIBATT_OK;
}
}  // namespace

int calibatt_balance_plan(int32_t* work_list, int32_t n_work, const int32_t* row_ptr, int heads, int nb,
                          int n_slots) {
  return balance_plan(work_list, n_work, row_ptr, heads, nb, nullptr, 0, n_slots);
}

int calibatt_balance_mixed_plan(int32_t* work_list, int32_t n_work, const int32_t* row_ptr, int heads, int nb,
                                const int32_t* row_ptr_b, int n_rep, int frames, int W, int k_anchor, int n_slots) {
  if (n_rep < 0 || frames < 1 || W < 1 || k_anchor < 1 || (n_rep > 0 && !row_ptr_b)) return CALIBATT_ERR_ARG;
  const int64_t units_b = static_cast<int64_t>(n_rep) * anchor_blocks(frames, W, k_anchor);
  if (row_ptr_b && (row_ptr_b[0] < 0 || row_ptr_b[units_b] < row_ptr_b[0])) return CALIBATT_ERR_CSR;
  return balance_plan(work_list, n_work, row_ptr, heads, nb, row_ptr_b, units_b, n_slots);
}

int calibatt_shard_heads(const int32_t* row_ptr_host, int heads, int nb, const int32_t* rep_heads_host, int n_rep,
                         int frames, int W, int k_anchor, int n_ranks, int32_t* owner, int64_t* load) {
  if (!row_ptr_host || !owner || heads < 1 || nb < 1 || n_rep < 0 || n_rep > heads || (n_rep > 0 && !rep_heads_host) ||
      frames < 1 || W < 1 || k_anchor < 1 || n_ranks < 1)
    return CALIBATT_ERR_ARG;
  std::vector<int64_t> cost(static_cast<size_t>(heads));
  for (int h = 0; h < heads; ++h) {
    const int64_t a = row_ptr_host[static_cast<int64_t>(h) * nb], b = row_ptr_host[static_cast<int64_t>(h + 1) * nb];
    if (b < a) return CALIBATT_ERR_CSR;
    cost[h] = b - a;
  }
  for (int i = 0; i < n_rep; ++i) {
    const int h = rep_heads_host[i];
    if (h < 0 || h >= heads) return CALIBATT_ERR_ARG;
    cost[h] = anchor_blocks(frames, W, k_anchor) * nb;  // anchor-query tiles over every key block
  }
  std::vector<int> order(static_cast<size_t>(heads));
  std::iota(order.begin(), order.end(), 0);
  std::stable_sort(order.begin(), order.end(), [&](int a, int b) { return cost[a] > cost[b]; });
  std::vector<int64_t> acc(static_cast<size_t>(n_ranks), 0);
  for (int h : order) {
    const int r = static_cast<int>(std::min_element(acc.begin(), acc.end()) - acc.begin());
    owner[h] = r;
    acc[r] += cost[h];
  }
  if (load) std::copy(acc.begin(), acc.end(), load);
  return CALIBATT_OK;
}

namespace {
int mixed_attn(const calibatt_bf16* q, const calibatt_bf16* k, const calibatt_bf16* v, int heads, int frames, int H,
               int W, int d, int k_anchor, float scale, const int32_t* row_ptr, const int32_t* col_idx, int64_t nnz,
               const int32_t* rep_heads, int32_t n_rep, const int32_t* row_ptr_b, const int32_t* col_idx_b,
               int64_t nnz_b, const int32_t* work_list, int32_t n_work, calibatt_bf16* o, float* lse, void* ws,
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
  p.row_ptr_b = n_rep > 0 ? row_ptr_b : nullptr;
  p.col_idx_b = n_rep > 0 ? col_idx_b : nullptr;
  p.nnz_b = nnz_b;
  return launch_attention(0, q, n, heads, k, v, n, heads, p, st, n_rep > 0 ? ws : nullptr, p.n_q_b, n_rep);
}
}  // namespace

int calibatt_mixed_attn_fwd(const calibatt_bf16* q, const calibatt_bf16* k, const calibatt_bf16* v, int heads,
                            int frames, int H, int W, int d, int k_anchor, float scale, const int32_t* row_ptr,
                            const int32_t* col_idx, int64_t nnz, const int32_t* rep_heads, int32_t n_rep,
                            const int32_t* work_list, int32_t n_work, calibatt_bf16* o, float* lse, void* ws,
                            size_t ws_bytes, calibatt_stream_t stream) {
  return mixed_attn(q, k, v, heads, frames, H, W, d, k_anchor, scale, row_ptr, col_idx, nnz, rep_heads, n_rep,
                    nullptr, nullptr, 0, work_list, n_work, o, lse, ws, ws_bytes, stream);
}

int calibatt_mixed_masked_attn_fwd(const calibatt_bf16* q, const calibatt_bf16* k, const calibatt_bf16* v,
                                   int heads, int frames, int H, int W, int d, int k_anchor, float scale,
                                   const int32_t* row_ptr, const int32_t* col_idx, int64_t nnz,
                                   const int32_t* rep_heads, int32_t n_rep, const int32_t* row_ptr_b,
                                   const int32_t* col_idx_b, int64_t nnz_b, const int32_t* work_list, int32_t n_work,
                                   calibatt_bf16* o, float* lse, void* ws, size_t ws_bytes,
                                   calibatt_stream_t stream) {
  if (n_rep > 0 && (!row_ptr_b || nnz_b < 0 || (nnz_b > 0 && !col_idx_b))) return CALIBATT_ERR_ARG;
  return mixed_attn(q, k, v, heads, frames, H, W, d, k_anchor, scale, row_ptr, col_idx, nnz, rep_heads, n_rep,
                    row_ptr_b, col_idx_b, nnz_b, work_list, n_work, o, lse, ws, ws_bytes, stream);
}

// ------------------------------------------------------------------ host buffers
// Streams and events of the host-buffer pipeline, created once per device
// (copies in and out overlap the attention; odd chunks' attention runs on a
// second compute stream, so that one chunk's launch fills the SMs that the
// previous chunk's last units leave idle).
namespace {
struct HostPipe {
  cudaStream_t in = nullptr, out = nullptr, cmp = nullptr;
  std::vector<cudaEvent_t> ev;  // [start, end, in_0, done_0, in_1, done_1, ...]
};

std::mutex g_pipe_mu[64];

// Caller holds g_pipe_mu[dev] for as long as it uses the pipe.
int host_pipe(int dev, int n_chunks, HostPipe** out) {
  static HostPipe pipes[64];
  HostPipe& hp = pipes[dev];
  // each stream on its own, so that a failed creation is retried on the next call
  for (cudaStream_t* st : {&hp.in, &hp.out, &hp.cmp})
    if (!*st && cudaStreamCreateWithFlags(st, cudaStreamNonBlocking) != cudaSuccess) {
      *st = nullptr;
      return CALIBATT_ERR_CUDA;
    }
  while (static_cast<int>(hp.ev.size()) < 2 + 2 * n_chunks) {
    cudaEvent_t e;
    if (cudaEventCreateWithFlags(&e, cudaEventDisableTiming) != cudaSuccess) return CALIBATT_ERR_CUDA;
    hp.ev.push_back(e);
  }
  *out = &hp;
  return CALIBATT_OK;
}
}  // namespace

size_t calibatt_mixed_host_workspace_size(int heads, int frames, int H, int W, int k_anchor, int n_rep,
                                          int heads_per_chunk) {
  if (heads < 1 || frames < 1 || H < 1 || W < 1 || k_anchor < 1 || k_anchor > H || n_rep < 0 || n_rep > heads)
    return 0;
  const int hpc = heads_per_chunk > 0 ? std::min(heads_per_chunk, heads) : std::min(2, heads);
  const int64_t n = static_cast<int64_t>(frames) * H * W;
  const int64_t nb = (n + 127) / 128;
  // two anchor buffers (consecutive chunks may run at once), then the lists
  const size_t anchors = n_rep > 0 ? calibatt_repeat_workspace_size(std::min(hpc, n_rep), frames, H, W, k_anchor) : 0;
  const size_t lists = static_cast<size_t>(heads * nb + n_rep * anchor_blocks(frames, W, k_anchor) + n_rep) * 4;
  return 2 * ((anchors + 255) & ~static_cast<size_t>(255)) + ((lists + 255) & ~static_cast<size_t>(255));
}

int calibatt_mixed_attn_fwd_host(const calibatt_bf16* q_host, const calibatt_bf16* k_host,
                                 const calibatt_bf16* v_host, calibatt_bf16* o_host, float* lse_host, int heads,
                                 int frames, int H, int W, int d, int k_anchor, float scale,
                                 const int32_t* row_ptr_host, const int32_t* row_ptr, const int32_t* col_idx,
                                 int64_t nnz, const int32_t* rep_heads_host, int32_t n_rep, int heads_per_chunk,
                                 calibatt_bf16* q_dev, calibatt_bf16* k_dev, calibatt_bf16* v_dev,
                                 calibatt_bf16* o_dev, float* lse_dev, void* ws, size_t ws_bytes,
                                 calibatt_stream_t stream) {
  if (!q_host || !k_host || !v_host || !o_host || !row_ptr_host || (lse_host && !lse_dev) || frames < 1 || H < 1 ||
      W < 1 || n_rep < 0 || n_rep > heads || (n_rep > 0 && !rep_heads_host) || !ws)
    return CALIBATT_ERR_ARG;
  const int64_t n64 = static_cast<int64_t>(frames) * H * W;
  if (n64 > INT_MAX / 2) return CALIBATT_ERR_ARG;
  const int n = static_cast<int>(n64);
  int rc = check_qkv(q_dev, k_dev, v_dev, o_dev, heads, n, d);
  if (rc != CALIBATT_OK) return rc;
  if (k_anchor < 1 || k_anchor > H) return CALIBATT_ERR_ARG;
  if (ws_bytes < calibatt_mixed_host_workspace_size(heads, frames, H, W, k_anchor, n_rep, heads_per_chunk))
    return CALIBATT_ERR_ARG;
  if (!aligned16(ws) || (lse_dev && !aligned4(lse_dev))) return CALIBATT_ERR_ALIGN;
  const int nb = (n + 127) / 128;
  const int hpc = heads_per_chunk > 0 ? std::min(heads_per_chunk, heads) : std::min(2, heads);
  // chunk boundaries: the first chunk holds half as many heads (rounded up),
  // so that the one copy-in that no attention overlaps is short; then chunks
  // of hpc heads, the last one what remains
  std::vector<int> bound{0};
  if (hpc < heads) bound.push_back((hpc + 1) / 2);
  while (bound.back() < heads) bound.push_back(std::min(heads, bound.back() + hpc));
  const int n_chunks = static_cast<int>(bound.size()) - 1;
  const int64_t nbq_b = anchor_blocks(frames, W, k_anchor);
  std::vector<uint8_t> is_rep(static_cast<size_t>(heads), 0);
  for (int i = 0; i < n_rep; ++i) {
    if (rep_heads_host[i] < 0 || rep_heads_host[i] >= heads) return CALIBATT_ERR_ARG;
    is_rep[rep_heads_host[i]] = 1;
  }
  std::vector<int32_t> anchors(static_cast<size_t>(k_anchor));
  calibatt_anchor_rows(H, k_anchor, anchors.data());
  // every chunk's work list and repeated heads, staged to the device in one
  // copy before any launch (a later pageable copy could wait for the stream)
  std::vector<int32_t> lists;
  std::vector<int> work_off(n_chunks), n_work(n_chunks), rep_off(n_chunks), n_rep_c(n_chunks);
  std::vector<int32_t> plan(static_cast<size_t>(heads * nb + n_rep * nbq_b));
  std::vector<uint8_t> active(static_cast<size_t>(heads));
  for (int c = 0; c < n_chunks; ++c) {
    const int h0 = bound[c], h1 = bound[c + 1];
    std::vector<int32_t> rep_c;
    for (int h = 0; h < heads; ++h) active[h] = (h >= h0 && h < h1) ? 1 : 0;
    for (int i = 0; i < n_rep; ++i)
      if (rep_heads_host[i] >= h0 && rep_heads_host[i] < h1) rep_c.push_back(rep_heads_host[i]);
    int32_t nw = 0;
    rc = calibatt_build_mixed_plan(row_ptr_host, heads, nb, active.data(), static_cast<int>(rep_c.size()),
                                   rep_c.empty() ? nullptr : rep_c.data(), frames, H, W, k_anchor, plan.data(), &nw);
    if (rc == CALIBATT_OK) rc = calibatt_balance_plan(plan.data(), nw, row_ptr_host, heads, nb, 0);
    if (rc != CALIBATT_OK) return rc;
    work_off[c] = static_cast<int>(lists.size());
    lists.insert(lists.end(), plan.begin(), plan.begin() + nw);
    n_work[c] = nw;
    rep_off[c] = static_cast<int>(lists.size());
    lists.insert(lists.end(), rep_c.begin(), rep_c.end());
    n_rep_c[c] = static_cast<int>(rep_c.size());
  }
  const size_t anchor_bytes =
      n_rep > 0 ? calibatt_repeat_workspace_size(std::min(hpc, n_rep), frames, H, W, k_anchor) : 0;
  uint8_t* ws8 = static_cast<uint8_t*>(ws);
  const size_t anchor_stride = (anchor_bytes + 255) & ~static_cast<size_t>(255);
  int32_t* lists_dev = reinterpret_cast<int32_t*>(ws8 + 2 * anchor_stride);
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return CALIBATT_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_pipe_mu[dev]);  // one caller of a device's pipe at a time
  HostPipe* hp = nullptr;
  rc = host_pipe(dev, n_chunks, &hp);
  if (rc != CALIBATT_OK) return rc;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const size_t head_elems = static_cast<size_t>(n) * 128;
  auto ok = [](cudaError_t e) { return e == cudaSuccess; };
  if (!lists.empty() &&
      !ok(cudaMemcpyAsync(lists_dev, lists.data(), lists.size() * 4, cudaMemcpyHostToDevice, st)))
    return CALIBATT_ERR_CUDA;
  // the device buffers may still be in use by earlier work on the stream
  if (!ok(cudaEventRecord(hp->ev[0], st)) || !ok(cudaStreamWaitEvent(hp->in, hp->ev[0], 0)) ||
      !ok(cudaStreamWaitEvent(hp->cmp, hp->ev[0], 0)))
    return CALIBATT_ERR_CUDA;
  for (int c = 0; c < n_chunks; ++c) {
    const int h0 = bound[c], h1 = bound[c + 1];
    const size_t off = static_cast<size_t>(h0) * head_elems, cnt = static_cast<size_t>(h1 - h0) * head_elems * 2;
    cudaEvent_t ev_in = hp->ev[2 + 2 * c], ev_done = hp->ev[3 + 2 * c];
    cudaStream_t cs = (c & 1) ? hp->cmp : st;
    // q: runs of whole heads; a repeated head reads only its anchor pixel rows,
    // so only those are copied (one strided copy per anchor row: one W-token
    // row of every frame)
    for (int h = h0; h < h1;) {
      if (is_rep[h]) {
        const size_t frame_bytes = static_cast<size_t>(H) * W * 128 * 2, row_bytes = static_cast<size_t>(W) * 128 * 2;
        for (int j = 0; j < k_anchor; ++j) {
          const size_t e0 = (static_cast<size_t>(h) * n + static_cast<size_t>(anchors[j]) * W) * 128;
          if (!ok(cudaMemcpy2DAsync(q_dev + e0, frame_bytes, q_host + e0, frame_bytes, row_bytes, frames,
                                    cudaMemcpyHostToDevice, hp->in)))
            return CALIBATT_ERR_CUDA;
        }
        ++h;
      } else {
        int e = h;
        while (e < h1 && !is_rep[e]) ++e;
        const size_t o0 = static_cast<size_t>(h) * head_elems;
        if (!ok(cudaMemcpyAsync(q_dev + o0, q_host + o0, static_cast<size_t>(e - h) * head_elems * 2,
                                cudaMemcpyHostToDevice, hp->in)))
          return CALIBATT_ERR_CUDA;
        h = e;
      }
    }
    if (!ok(cudaMemcpyAsync(k_dev + off, k_host + off, cnt, cudaMemcpyHostToDevice, hp->in)) ||
        !ok(cudaMemcpyAsync(v_dev + off, v_host + off, cnt, cudaMemcpyHostToDevice, hp->in)) ||
        !ok(cudaEventRecord(ev_in, hp->in)) || !ok(cudaStreamWaitEvent(cs, ev_in, 0)))
      return CALIBATT_ERR_CUDA;
    // chunks alternate between two compute streams and two anchor buffers
    rc = calibatt_mixed_attn_fwd(q_dev, k_dev, v_dev, heads, frames, H, W, d, k_anchor, scale, row_ptr, col_idx,
                                 nnz, n_rep_c[c] ? lists_dev + rep_off[c] : nullptr, n_rep_c[c],
                                 n_work[c] ? lists_dev + work_off[c] : nullptr, n_work[c], o_dev, lse_dev,
                                 ws8 + (c & 1) * anchor_stride, anchor_bytes, reinterpret_cast<calibatt_stream_t>(cs));
    if (rc != CALIBATT_OK) return rc;
    if (!ok(cudaEventRecord(ev_done, cs)) || !ok(cudaStreamWaitEvent(hp->out, ev_done, 0)) ||
        !ok(cudaMemcpyAsync(o_host + off, o_dev + off, cnt, cudaMemcpyDeviceToHost, hp->out)) ||
        (lse_host && !ok(cudaMemcpyAsync(lse_host + static_cast<size_t>(h0) * n, lse_dev + static_cast<size_t>(h0) * n,
                                         static_cast<size_t>(h1 - h0) * n * sizeof(float), cudaMemcpyDeviceToHost,
                                         hp->out))))
      return CALIBATT_ERR_CUDA;
  }
  // the call is complete when the caller's stream is
  if (!ok(cudaEventRecord(hp->ev[1], hp->out)) || !ok(cudaStreamWaitEvent(st, hp->ev[1], 0)))
    return CALIBATT_ERR_CUDA;
  return CALIBATT_OK;
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
                          uint16_t* counts, uint8_t* tie, double tie_window, calibatt_stream_t stream) {
  int rc = check_qkv(q, k, nullptr, nullptr, heads, n, d);
  if (rc != CALIBATT_OK) return rc;
  const int nb = (n + 127) / 128;
  if (nb > CALIBATT_MAX_CALIB_NB) return CALIBATT_ERR_UNSUPPORTED;
  if (!scale_ok(scale) || !lse_ws || std::isnan(eps) || std::isnan(tie_window)) return CALIBATT_ERR_ARG;
  if (fuse_select && !mask && !kept && !counts && !tie) return CALIBATT_ERR_ARG;
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
  p.tie = fuse_select ? tie : nullptr;
  p.tie_fx = tie_window_fixed(tie_window);
  return launch_attention(2, q, n, heads, k, nullptr, n, heads, p, st);
}

size_t calibatt_energy_workspace_size(int heads, int n) {
  if (heads < 1 || n < 1) return 0;
  const int64_t nb = (static_cast<int64_t>(n) + 127) / 128;
  const int64_t units = heads * nb;
  if (units > INT_MAX / 2 || nb > CALIBATT_MAX_CALIB_NB) return 0;
  const size_t bytes = static_cast<size_t>(energy_ws_floats(2 * score_grid(static_cast<int>(units)), nb)) * sizeof(float);
  return (bytes + 255) & ~static_cast<size_t>(255);
}

int calibatt_block_energy_1pass(const calibatt_bf16* q, const calibatt_bf16* k, int heads, int n, int d,
                                float scale, void* ws, size_t ws_bytes, float* energy, int fuse_select, double eps,
                                uint8_t* mask, int32_t* kept, uint16_t* counts, uint8_t* tie, double tie_window,
                                float* pix_energy, int pix_W, calibatt_stream_t stream) {
  int rc = check_qkv(q, k, nullptr, nullptr, heads, n, d);
  if (rc != CALIBATT_OK) return rc;
  const int nb = (n + 127) / 128;
  if (nb > CALIBATT_MAX_CALIB_NB) return CALIBATT_ERR_UNSUPPORTED;
  if (!scale_ok(scale) || !ws || std::isnan(eps) || std::isnan(tie_window)) return CALIBATT_ERR_ARG;
  if (ws_bytes < calibatt_energy_workspace_size(heads, n)) return CALIBATT_ERR_ARG;
  if (fuse_select && !mask && !kept && !counts && !tie) return CALIBATT_ERR_ARG;
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
  p.energy_ws = static_cast<float*>(ws);
  p.energy = energy;
  p.fuse_select = fuse_select ? 1 : 0;
  p.eps_fx = eps_to_fixed(eps);
  p.mask = fuse_select ? mask : nullptr;
  p.kept = fuse_select ? kept : nullptr;
  p.counts = fuse_select ? counts : nullptr;
  p.tie = fuse_select ? tie : nullptr;
  p.tie_fx = tie_window_fixed(tie_window);
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
                         uint16_t* counts, uint8_t* tie, double tie_window, calibatt_stream_t stream) {
  if (!energy || heads < 1 || nb < 1 || std::isnan(eps) || std::isnan(tie_window)) return CALIBATT_ERR_ARG;
  if (nb > CALIBATT_MAX_CALIB_NB) return CALIBATT_ERR_UNSUPPORTED;
  if (!mask && !kept && !counts && !tie) return CALIBATT_ERR_ARG;
  if (!aligned4(energy) || (kept && !aligned4(kept)) || (counts && (reinterpret_cast<uintptr_t>(counts) & 1u)))
    return CALIBATT_ERR_ALIGN;
  return launch_select(energy, static_cast<int64_t>(heads) * nb, nb, eps_to_fixed(eps), mask, kept, counts, tie,
                       tie_window_fixed(tie_window), reinterpret_cast<cudaStream_t>(stream));
}

int calibatt_accumulate_masks(const uint8_t* mask, int64_t cells, uint16_t* counts, calibatt_stream_t stream) {
  if (cells < 0 || (cells > 0 && (!mask || !counts))) return CALIBATT_ERR_ARG;
  if (counts && (reinterpret_cast<uintptr_t>(counts) & 1u)) return CALIBATT_ERR_ALIGN;
  return launch_accumulate(mask, cells, counts, reinterpret_cast<cudaStream_t>(stream));
}

size_t calibatt_aggregate_workspace_size(int heads, int nb) {
  if (heads < 1 || nb < 1) return 0;
  const size_t bytes = static_cast<size_t>(aggregate_scratch_ints(static_cast<int64_t>(heads) * nb)) * sizeof(int32_t);
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

size_t calibatt_anchor_energy_workspace_size(int heads, int n_rep, int frames, int H, int W, int k_anchor) {
  if (heads < 1 || n_rep < 1 || n_rep > heads || frames < 1 || H < 1 || W < 1 || k_anchor < 1 || k_anchor > H)
    return 0;
  const int64_t n = static_cast<int64_t>(frames) * H * W;
  const int64_t nb = (n + 127) / 128;
  const int64_t units = n_rep * anchor_blocks(frames, W, k_anchor);
  if (n > INT_MAX / 2 || units > INT_MAX / 2 || nb > CALIBATT_MAX_CALIB_NB) return 0;
  const size_t packed = calibatt_repeat_workspace_size(n_rep, frames, H, W, k_anchor);
  const size_t energy = static_cast<size_t>(energy_ws_floats(2 * score_grid(static_cast<int>(units)), nb)) * sizeof(float);
  return packed + ((energy + 255) & ~static_cast<size_t>(255));
}

int calibatt_anchor_block_energy(const calibatt_bf16* q, const calibatt_bf16* k, int heads, int frames, int H, int W,
                                 int d, int k_anchor, float scale, const int32_t* rep_heads, int32_t n_rep, void* ws,
                                 size_t ws_bytes, float* energy, int fuse_select, double eps, uint8_t* mask,
                                 int32_t* kept, uint16_t* counts, uint8_t* tie, double tie_window,
                                 calibatt_stream_t stream) {
  if (frames < 1 || H < 1 || W < 1 || !rep_heads || n_rep < 1 || n_rep > heads) return CALIBATT_ERR_ARG;
  const int64_t n64 = static_cast<int64_t>(frames) * H * W;
  if (n64 > INT_MAX / 2) return CALIBATT_ERR_ARG;
  const int n = static_cast<int>(n64);
  int rc = check_qkv(q, k, nullptr, nullptr, heads, n, d);
  if (rc != CALIBATT_OK) return rc;
  if (k_anchor < 1 || k_anchor > H) return CALIBATT_ERR_ARG;
  if (k_anchor > kMaxAnchors) return CALIBATT_ERR_UNSUPPORTED;
  const int nb = (n + 127) / 128;
  if (nb > CALIBATT_MAX_CALIB_NB) return CALIBATT_ERR_UNSUPPORTED;
  if (!scale_ok(scale) || !ws || std::isnan(eps) || std::isnan(tie_window)) return CALIBATT_ERR_ARG;
  if (ws_bytes < calibatt_anchor_energy_workspace_size(heads, n_rep, frames, H, W, k_anchor)) return CALIBATT_ERR_ARG;
  if (fuse_select && !mask && !kept && !counts && !tie) return CALIBATT_ERR_ARG;
  if (!aligned16(ws) || (energy && !aligned4(energy)) || (kept && !aligned4(kept)) ||
      (counts && (reinterpret_cast<uintptr_t>(counts) & 1u)))
    return CALIBATT_ERR_ALIGN;
  KernelParams p = base_params();
  if (!p.status) return CALIBATT_ERR_CUDA;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  // the anchor queries of the repeated heads, packed frame by frame
  AnchorTable tab;
  int32_t anchors[kMaxAnchors];
  calibatt_anchor_rows(H, k_anchor, anchors);
  for (int j = 0; j < k_anchor; ++j) tab.anchor[j] = anchors[j];
  const int n_q_b = frames * k_anchor * W;
  rc = launch_gather(q, n, heads, rep_heads, n_rep, H, W, k_anchor, tab, ws, p.status, st);
  if (rc != CALIBATT_OK) return rc;
  // their block energies over every key block, in one pass
  const size_t packed = calibatt_repeat_workspace_size(n_rep, frames, H, W, k_anchor);
  p.n_q = n_q_b;
  p.nbq = (n_q_b + 127) / 128;
  p.n_k = n;
  p.nbk = nb;
  p.heads_q = n_rep;
  p.heads_kv = heads;
  p.head_map = rep_heads;
  p.n_units = n_rep * p.nbq;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.n_out = n;
  p.energy_ws = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + packed);
  p.energy = energy;
  p.fuse_select = fuse_select ? 1 : 0;
  p.eps_fx = eps_to_fixed(eps);
  p.mask = fuse_select ? mask : nullptr;
  p.kept = fuse_select ? kept : nullptr;
  p.counts = fuse_select ? counts : nullptr;
  p.tie = fuse_select ? tie : nullptr;
  p.tie_fx = tie_window_fixed(tie_window);
  return launch_attention(3, ws, n_q_b, n_rep, k, nullptr, n, heads, p, st);
}

size_t calibatt_aggregate_rows_workspace_size(int64_t rows) {
  if (rows < 1 || rows > INT_MAX / 2) return 0;
  const size_t bytes = static_cast<size_t>(aggregate_scratch_ints(rows)) * sizeof(int32_t);
  return (bytes + 255) & ~static_cast<size_t>(255);
}

int calibatt_aggregate_mask_rows(const uint16_t* counts, int n_inputs, int64_t rows, int cols, double rho,
                                 uint8_t* mask, int32_t* row_ptr, int32_t* col_idx, int64_t nnz_cap, int64_t* nnz,
                                 void* ws, size_t ws_bytes, calibatt_stream_t stream) {
  if (!counts || !mask || !row_ptr || !nnz || rows < 1 || cols < 1 || n_inputs < 1 || nnz_cap < 0 ||
      (nnz_cap > 0 && !col_idx) || !std::isfinite(rho))
    return CALIBATT_ERR_ARG;
  if (rows > INT_MAX / 2 || rows * cols > INT_MAX) return CALIBATT_ERR_ARG;
  if (!ws || ws_bytes < calibatt_aggregate_rows_workspace_size(rows)) return CALIBATT_ERR_ARG;
  if ((reinterpret_cast<uintptr_t>(counts) & 1u) || !aligned4(row_ptr) || (col_idx && !aligned4(col_idx)) ||
      (reinterpret_cast<uintptr_t>(nnz) & 7u) || !aligned4(ws))
    return CALIBATT_ERR_ALIGN;
  int* status = status_word();
  if (!status) return CALIBATT_ERR_CUDA;
  int32_t thr = 0;
  calibatt_rho_threshold(n_inputs, rho, &thr);
  return launch_aggregate(counts, rows, cols, thr, mask, row_ptr, col_idx, nnz_cap, nnz, static_cast<int32_t*>(ws),
                          status, reinterpret_cast<cudaStream_t>(stream));
}

}  // extern "C"
