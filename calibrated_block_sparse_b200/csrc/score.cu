// The block-energy calibration (explainer §三, offline calibration steps
// 1-2) on the tensor core: S = Q K^T tile by tile over all key blocks, never
// storing P.
//   kLse:     per query row, log2 sum_j 2^(scale' S_ij)  -> lse_ws
//   kEnergy:  second pass: per tile, sum_ij 2^(scale' S_ij - lse_i) -> E[r][c],
//             then the greedy eps selection of the finished row (select.cuh)
//   kEnergy1: the same energies in one pass: each row keeps its exact
//             running max m and sum l, and stores every tile's sum t in a
//             workspace, chunks of 8 tiles relative to the m reached at the
//             chunk's end (when m grows, the chunk's stored sums are rescaled
//             with l), that m after them (36 bytes per 8 tiles); when the
//             row is done, t * 2^(m - lse) gives its share of E[r][c] as the
//             second pass would, and the row's tiles are reduced and selected
//             as above. S is computed once instead of twice.
//
// CTA (352 threads, one per SM): two query-tile slots; warps 0-3 and 4-7 are
// the slots' row warpgroups (thread = query row = TMEM lane), warp 8 loads Q
// and K tiles with TMA into one K ring per slot, warps 9 and 10 issue the
// tcgen05.mma of slot 0 and slot 1. Tensor memory holds two S buffers per
// slot (4 x 128 columns), so the MMA of the next tile overlaps the reduction
// of the current one. One issuer per slot: a stage's barrier checks and
// commits cost about as long as its eight MMAs, and with a single issuer the
// tensor pipe waited through them; with two, one slot's bookkeeping overlaps
// the other slot's MMAs.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>

#include "calibatt.h"
#include "kernels.h"
#include "ptx.cuh"
#include "sched.cuh"
#include "select.cuh"
#include "softmax.cuh"

#ifndef CALIBATT_SCORE_EMU
#define CALIBATT_SCORE_EMU 0x00u
#endif

namespace calibatt {
namespace {

constexpr int kScoreThreads = 352;
constexpr int kSlotRing = 2;                // K tiles in flight per slot
constexpr int kEnergyScratch = 16384;       // per slot: per-warp tile sums, then selection scratch
// Pairs of a row whose 2^x goes to the FMA-pipe polynomial (bit i%8 of the
// mask selects pair i) instead of MUFU; measured fastest with none.
constexpr unsigned kScoreEmu = CALIBATT_SCORE_EMU;

// Words the producer writes with each ring stage, read by the slot's issuer.
constexpr uint32_t kStageFirst = 1;  // starts a unit: wait for its Q
constexpr uint32_t kStageLast = 2;   // ends a unit: release its Q
constexpr uint32_t kStageEnd = 4;    // no more tiles for this slot

struct ScoreBarriers {
  uint64_t ring_full[2][kSlotRing];
  uint64_t ring_empty[2][kSlotRing];
  uint64_t q_full[2];
  uint64_t q_empty[2];
  uint64_t s_full[2][2];
  uint64_t s_empty[2][2];
  uint64_t mma_done[2];
  uint32_t flags[2][kSlotRing];
  uint32_t tmem_base;
  int abort;
};

template <int MODE>
struct ScoreLayout {
  static constexpr int kQOff = 0;
  static constexpr int kRingOff = 2 * kTile;
  static constexpr int kAuxOff = kRingOff + 2 * kSlotRing * kTile;
  static constexpr int kAuxBytes = (MODE == kEnergy || MODE == kEnergy1) ? 2 * kEnergyScratch : 0;
  static constexpr int kBarOff = kAuxOff + kAuxBytes;
  static constexpr int kBytes = kBarOff + static_cast<int>(sizeof(ScoreBarriers));
  static constexpr int kDynSmem = kBytes + 1024;  // + alignment slack
};

// The fused selection: one call per finished row, kept out of line so that
// its registers do not weigh on the kernel's main loop.
__device__ __noinline__ void warp_select_row1024(const float* E, int nb, long long eps_fx, long long tie_fx,
                                                 float* scratch, SelectOut out) {
  warp_select<32>(E, nb, eps_fx, tie_fx, scratch, out);
}

template <int MODE, bool SW>  // SW: the polling wait form of short (test) wait limits
__global__ void __launch_bounds__(kScoreThreads, 1)
    score_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                 const __grid_constant__ KernelParams p) {
  using L = ScoreLayout<MODE>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  const uint32_t sbase = smem_u32(smem);
  ScoreBarriers& bar = *reinterpret_cast<ScoreBarriers*>(smem + L::kBarOff);
  volatile int* abort_flag = &bar.abort;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int G = 2 * gridDim.x;

  if (threadIdx.x == 0) {
    for (int s = 0; s < 2; ++s)
      for (int i = 0; i < kSlotRing; ++i) {
        mbar_init(&bar.ring_full[s][i], 1);
        mbar_init(&bar.ring_empty[s][i], 1);
      }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bar.q_full[s], 1);
      mbar_init(&bar.q_empty[s], 1);
      for (int b = 0; b < 2; ++b) {
        mbar_init(&bar.s_full[s][b], 1);
        mbar_init(&bar.s_empty[s][b], 128);
      }
    }
    mbar_init(&bar.mma_done[0], 1);
    mbar_init(&bar.mma_done[1], 1);
    bar.abort = 0;
    fence_barrier_init();
  }
  if (warp == 9) tmem_alloc(&bar.tmem_base, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bar.tmem_base;

  if (warp == 8 && lane == 0) {
    // ---------------------------------------------------------- TMA producer
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    Cursor cur[2];
    for (int s = 0; s < 2; ++s) {
      cur[s].round = 0;
      cursor_seek(p, 2 * blockIdx.x + s, G, cur[s]);
    }
    uint32_t stage[2] = {0, 0}, phase[2] = {0, 0}, n_q[2] = {0, 0};
    bool ok = true;
    while (ok && (cur[0].valid || cur[1].valid)) {
      for (int s = 0; s < 2 && ok; ++s) {
        Cursor& c = cur[s];
        if (!c.valid) continue;
        if (c.j == 0) {
          if (!(ok = mbar_wait<SW>(&bar.q_empty[s], (n_q[s] & 1) ^ 1, abort_flag, p.status, p.wait_limit_ns))) break;
          uint8_t* dst = smem + L::kQOff + s * kTile;
          mbar_arrive_expect_tx(&bar.q_full[s], kTile);
          tma_load_3d(dst, &tm_q, &bar.q_full[s], 0, c.u.r * 128, c.u.hq);
          tma_load_3d(dst + kHalf, &tm_q, &bar.q_full[s], 64, c.u.r * 128, c.u.hq);
          ++n_q[s];
        }
        const uint32_t st = stage[s];
        if (!(ok = mbar_wait<SW>(&bar.ring_empty[s][st], phase[s] ^ 1, abort_flag, p.status, p.wait_limit_ns))) break;
        bar.flags[s][st] = (c.j == 0 ? kStageFirst : 0u) | (c.j == c.u.nnz - 1 ? kStageLast : 0u);
        uint8_t* dst = smem + L::kRingOff + (s * kSlotRing + st) * kTile;
        mbar_arrive_expect_tx(&bar.ring_full[s][st], kTile);
        tma_load_3d(dst, &tm_k, &bar.ring_full[s][st], 0, c.j * 128, c.u.hkv);
        tma_load_3d(dst + kHalf, &tm_k, &bar.ring_full[s][st], 64, c.j * 128, c.u.hkv);
        if (++stage[s] == kSlotRing) {
          stage[s] = 0;
          phase[s] ^= 1;
        }
        cursor_next(p, 2 * blockIdx.x + s, G, c);
      }
    }
    for (int s = 0; s < 2; ++s) {
      const uint32_t st0 = stage[s], ph0 = phase[s];
      bool marker = false;
      if (ok && mbar_wait<SW>(&bar.ring_empty[s][st0], ph0 ^ 1, abort_flag, p.status, p.wait_limit_ns)) {
        bar.flags[s][st0] = kStageEnd;
        mbar_arrive(&bar.ring_full[s][st0]);
        marker = true;
      } else {
        ok = false;
      }
      // no copy may still be landing when the CTA leaves: wait for the latest
      // phase of every stage of this slot's ring. With the end marker sent,
      // the latest phase of st0 is the marker's own (its earlier copy was
      // consumed before the producer could reuse the stage); without it (a
      // wait failed), st0 was not armed again and its latest phase is the
      // previous lap's.
      for (int i = 0; i < kSlotRing; ++i) {
        int st = static_cast<int>(st0) - (marker ? 0 : 1) - i;
        uint32_t ph = ph0;
        if (st < 0) {
          st += kSlotRing;
          ph ^= 1;
        }
        volatile int never = 0;
        mbar_wait(&bar.ring_full[s][st], ph, &never, p.status);
      }
    }
    for (int s = 0; s < 2; ++s)
      if (n_q[s] > 0) {
        volatile int never = 0;
        mbar_wait(&bar.q_full[s], (n_q[s] - 1) & 1, &never, p.status);
      }
  } else if ((warp == 9 || warp == 10) && lane == 0) {
    // ---------------------------------------------------------- MMA issuers, one per slot
    const int s = warp - 9;
    uint32_t stage = 0, phase = 0, n_q = 0, n_s = 0;
    const uint64_t qd = desc_k_base(sbase + L::kQOff) + s * (kTile >> 4);
    const uint64_t kdesc0 = desc_k_base(sbase + L::kRingOff) + s * kSlotRing * (kTile >> 4);
    while (true) {
      if (!mbar_wait<SW>(&bar.ring_full[s][stage], phase, abort_flag, p.status, p.wait_limit_ns)) break;
      // read the stage's word now: once ring_empty is committed below, the
      // producer may reuse the stage and rewrite it for its next tile
      const uint32_t f = *reinterpret_cast<volatile uint32_t*>(&bar.flags[s][stage]);
      if (f & kStageEnd) break;
      if (f & kStageFirst) {
        if (!mbar_wait<SW>(&bar.q_full[s], n_q & 1, abort_flag, p.status, p.wait_limit_ns)) break;
      }
      const int buf = n_s & 1;
      if (!mbar_wait<SW>(&bar.s_empty[s][buf], ((n_s >> 1) & 1) ^ 1, abort_flag, p.status, p.wait_limit_ns)) break;
      tc_fence_after();
      const uint32_t d_tmem = tmem + (2 * s + buf) * 128;
      const uint64_t kd = kdesc0 + stage * (kTile >> 4);
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) mma_ss(d_tmem, qd + desc_k_step(ks), kd + desc_k_step(ks), kIdescS, ks > 0);
      mma_commit(&bar.ring_empty[s][stage]);
      if (f & kStageLast) {
        mma_commit(&bar.q_empty[s]);
        ++n_q;
      }
      mma_commit(&bar.s_full[s][buf]);
      ++n_s;
      if (++stage == kSlotRing) {
        stage = 0;
        phase ^= 1;
      }
    }
    mma_commit(&bar.mma_done[s]);
    volatile int never = 0;
    mbar_wait(&bar.mma_done[s], 0, &never, p.status);
  } else if (warp < 8) {
    // ---------------------------------------------------------- row warpgroups
    // After a failed wait the warps keep walking their units with every wait
    // and tensor-memory access skipped, so that the warpgroup's named
    // barriers are still met by all four warps.
    const int s = warp >> 2;
    const int wl = warp & 3;
    const int row = wl * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(wl * 32) << 16;
    const int g = 2 * blockIdx.x + s;
    const bool ragged_k = (p.n_k & 127) != 0;
    const int valid_last = p.n_k - (p.nbk - 1) * 128;
    uint32_t n_sfull = 0;
    bool ok = true;  // warp-uniform
    float* part = reinterpret_cast<float*>(smem + L::kAuxOff + s * kEnergyScratch);
    // pixel-row profiles of key block j from each row's normalised tile sum v:
    // a segmented scan over the warp's rows (a pixel row is a run of
    // consecutive lanes), then one atomic add per pixel row from the run's
    // last lane. Warp-collective.
    int pix_key = -1;
    int pix_hq = 0;
    auto pix_add = [&](float v, int j) {
      const int key = pix_key;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const float vu = __shfl_up_sync(0xffffffffu, v, o);
        const int ku = __shfl_up_sync(0xffffffffu, key, o);
        if (lane >= o && ku == key) v += vu;
      }
      const int kn = __shfl_down_sync(0xffffffffu, key, 1);
      if (ok && key >= 0 && (lane == 31 || kn != key))
        atomicAdd(p.pix_energy + (static_cast<int64_t>(pix_hq) * p.pix_rows + key) * p.nbk + j, v * p.pix_inv_W);
    };

    for (int round = 0;; ++round) {
      Unit u;
      if (!load_unit(p, unit_index(g, G, round), u)) break;
      if (!u.write) continue;
      const int qrow = u.r * 128 + row;
      const bool row_valid = qrow < p.n_q;
      float lse2 = 0.f;
      if (MODE == kEnergy && row_valid) lse2 = p.lse_ws[static_cast<int64_t>(u.hq) * p.nbq * 128 + qrow];
      if (p.pix_energy) {
        pix_key = row_valid ? qrow / p.pix_W : -1;
        pix_hq = u.hq;
      }
      float m_run = -INFINITY, l_run = 0.f;
      // single pass: this row's words of the chunk holding key block j
      const int64_t n_chunks = (p.nbk + kEnergyChunk - 1) / kEnergyChunk;
      auto chunk_ws = [&](int j) {
        return p.energy_ws + ((static_cast<int64_t>(g) * n_chunks + j / kEnergyChunk) * (kEnergyChunk + 1)) * 128 + row;
      };
      for (int j = 0; j < u.nnz; ++j) {
        const int buf = n_sfull & 1;
        float acc = 0.f;
        if (ok) ok = __all_sync(0xffffffffu, mbar_wait<SW>(&bar.s_full[s][buf], (n_sfull >> 1) & 1, abort_flag,
                                                       p.status, p.wait_limit_ns));
        if (ok) {
          ++n_sfull;
          tc_fence_after();
          float sv[128];
          tmem_ld128_wait(tmem + lane_off + (2 * s + buf) * 128, sv);
          tc_fence_before();
          mbar_arrive(&bar.s_empty[s][buf]);
          const int nvalid = (ragged_k && j == p.nbk - 1) ? valid_last : 128;
          if (nvalid < 128) {
#pragma unroll
            for (int c = 0; c < 128; ++c)
              if (c >= nvalid) sv[c] = -INFINITY;
          }
          float ref;  // subtracted before the exponential
          if (MODE == kLse || MODE == kEnergy1) {
            const float mx = row_max128(sv) * p.scale_log2;
            const float m_new = fmaxf(m_run, mx);
            if (m_new > m_run && m_run != -INFINITY) {  // 2^0 = 1 exactly: no change to skip
              const float f = ex2_approx(m_run - m_new);
              l_run *= f;
              if (MODE == kEnergy1) {
                // the chunk's sums stored so far follow the new max (rare:
                // a row's max grows a few times, mostly in its first tiles)
                float* w = chunk_ws(j);
                for (int i = 0; i < j % kEnergyChunk; ++i) w[i * 128] *= f;
              }
            }
            m_run = m_new;
            ref = m_new;
          } else {
            ref = lse2;
          }
          if (MODE != kEnergy || row_valid) {
            const float2 c2 = make_float2(p.scale_log2, p.scale_log2);
            const float2 nr2 = make_float2(-ref, -ref);
            float2 a4[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                            make_float2(0.f, 0.f)};
#pragma unroll
            for (int i = 0; i < 64; ++i) {
              float2 e = exp2_pair<5, kScoreEmu>(i, ffma2(make_float2(sv[2 * i], sv[2 * i + 1]), c2, nr2));
              if (nvalid < 128) {
                e.x = 2 * i < nvalid ? e.x : 0.f;
                e.y = 2 * i + 1 < nvalid ? e.y : 0.f;
              }
              a4[i & 3] = fadd2(a4[i & 3], e);
            }
            const float2 s01 = fadd2(a4[0], a4[1]), s23 = fadd2(a4[2], a4[3]);
            acc = (s01.x + s01.y) + (s23.x + s23.y);
          }
          if (MODE != kEnergy) l_run += acc;
          // single pass: store the tile's sum relative to the running max,
          // and at the chunk's end that max
          if (MODE == kEnergy1) {
            const int slot = j % kEnergyChunk;
            float* w = chunk_ws(j);
            w[slot * 128] = acc;
            if (slot == kEnergyChunk - 1 || j == u.nnz - 1) w[kEnergyChunk * 128] = m_run;
          }
        }
        if (MODE == kEnergy && p.pix_energy) pix_add(acc, j);
        if (MODE == kEnergy) {
          // this warp's share of E[r][j]: sum over its 32 rows
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
          if (lane == 0) part[wl * 1024 + j] = acc;
        }
      }
      if (MODE == kLse) {
        if (ok) p.lse_ws[static_cast<int64_t>(u.hq) * p.nbq * 128 + qrow] = m_run + log2f(l_run);
      } else {
        if (MODE == kEnergy1) {
          // every chunk's tile sums rescaled to the row's final
          // log-sum-exp, then summed over the warp's 32 rows
          static_assert(kEnergyChunk == 8, "the reduction below takes eight key blocks at a time");
          const float lse_r = m_run + log2f(l_run);
          const float* wsr = p.energy_ws + static_cast<int64_t>(g) * n_chunks * (kEnergyChunk + 1) * 128 + row;
          for (int c0 = 0; c0 < p.nbk; c0 += 8) {
            const float* wc = wsr + static_cast<int64_t>(c0 / 8) * (kEnergyChunk + 1) * 128;
            const bool live = ok && row_valid;
            const float sc = live ? ex2_approx(wc[kEnergyChunk * 128] - lse_r) : 0.f;
            float v[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) v[i] = live && c0 + i < p.nbk ? wc[i * 128] * sc : 0.f;
            if (p.pix_energy) {
#pragma unroll
              for (int i = 0; i < 8; ++i)
                if (c0 + i < p.nbk) pix_add(v[i], c0 + i);
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
#pragma unroll
              for (int i = 0; i < 8; ++i) v[i] += __shfl_xor_sync(0xffffffffu, v[i], o);
            }
            if (lane == 0) {
#pragma unroll
              for (int i = 0; i < 8; ++i)
                if (c0 + i < p.nbk) part[wl * 1024 + c0 + i] = v[i];
            }
          }
        }
        named_bar_sync(1 + s, 128);
        const int rows = min(128, p.n_q - u.r * 128);
        const float inv_rows = 1.f / static_cast<float>(rows);
        const int64_t erow = (static_cast<int64_t>(u.hq) * p.nbq + u.r) * p.nbk;
        for (int c = row; c < p.nbk; c += 128) {
          // fixed summation order: the energy is reproducible run to run
          const float e = (((part[c] + part[1024 + c]) + part[2048 + c]) + part[3072 + c]) * inv_rows;
          part[c] = e;
          if (p.energy && ok) p.energy[erow + c] = e;
        }
        if (p.fuse_select) {
          // the finished row is selected by the warpgroup's first warp
          // (its candidate scratch behind the row in the slot's scratch)
          named_bar_sync(1 + s, 128);
          if (wl == 0) {
            const int64_t urow = erow / p.nbk;
            SelectOut out{p.mask ? p.mask + erow : nullptr, p.kept ? p.kept + urow : nullptr,
                          p.counts ? p.counts + erow : nullptr, p.tie ? p.tie + urow : nullptr};
            if (!ok) out = SelectOut{nullptr, nullptr, nullptr, nullptr};
            warp_select_row1024(part, p.nbk, p.eps_fx, p.tie_fx, part + 1024, out);
          }
        }
        named_bar_sync(1 + s, 128);
      }
    }
  }

  // ---------------------------------------------------------- teardown
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 9) {
    __syncwarp();
    tmem_dealloc(tmem, 512);
  }
}

template <int MODE>
int launch_mode(const CUtensorMap& mq, const CUtensorMap& mk, const KernelParams& p, cudaStream_t stream) {
  using L = ScoreLayout<MODE>;
  static_assert(L::kDynSmem <= 232448, "shared memory budget");
  static_assert(kEnergyScratch >= 4096 + kSelectScratchBytes, "selection scratch behind the energy row");
  const bool short_waits = p.wait_limit_ns < kShortWaitNs;
  const void* fn = short_waits ? reinterpret_cast<const void*>(score_kernel<MODE, true>)
                               : reinterpret_cast<const void*>(score_kernel<MODE, false>);
  static PerDeviceOnce smem_once[2];
  const int rc = set_max_smem_once(fn, L::kDynSmem, smem_once[short_waits ? 1 : 0]);
  if (rc != CALIBATT_OK) return rc;
  if (p.n_units <= 0) return CALIBATT_OK;
  if (short_waits)
    score_kernel<MODE, true><<<score_grid(p.n_units), kScoreThreads, L::kDynSmem, stream>>>(mq, mk, p);
  else
    score_kernel<MODE, false><<<score_grid(p.n_units), kScoreThreads, L::kDynSmem, stream>>>(mq, mk, p);
  return cudaGetLastError() == cudaSuccess ? CALIBATT_OK : CALIBATT_ERR_CUDA;
}

}  // namespace

int launch_score(int mode, const CUtensorMap& mq, const CUtensorMap& mk, const KernelParams& p,
                 cudaStream_t stream) {
  switch (mode) {
    case kLse: return launch_mode<kLse>(mq, mk, p, stream);
    case kEnergy: return launch_mode<kEnergy>(mq, mk, p, stream);
    case kEnergy1: return launch_mode<kEnergy1>(mq, mk, p, stream);
    default: return CALIBATT_ERR_ARG;
  }
}

}  // namespace calibatt
