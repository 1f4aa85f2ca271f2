// Block-sparse attention over a skip list, and the anchor-row pass of
// repeated heads, on the sm_100a tensor core (explainer §三, online
// inference): O = softmax(scale Q K^T) V over the kept 128 x 128 tiles.
//
// CTA (384 threads, one per SM, persistent: slot g of G takes work-list
// entries g, 2G-1-g, 2G+g, ..., which the host plan lays out head by head,
// longest first, each round matched to the least-loaded slots), two
// independent query-tile "slots" so that the tensor core works on one slot
// while the other slot's softmax runs:
//   warps 0-3  softmax warpgroup of slot 0 (thread = query row = TMEM lane)
//   warps 4-7  softmax warpgroup of slot 1
//   warp  8    TMA producer (one thread): Q tile per unit, K/V tiles per kept block
//   warp  9    MMA issuer (one thread): tcgen05.mma S = Q K^T and O += P V
//   warps 10-11 idle (they complete the third warpgroup)
// The third warpgroup hands registers to the softmax warpgroups (setmaxnreg):
// a softmax thread holds a whole 128-column row of S, and at the launch
// allotment of 168 registers it spilled.
// Tensor memory (512 columns): S (fp32, 128 columns) and O (fp32, 128
// columns) per slot; P (bf16) is written over the first 64 columns of S and
// read by the P V MMA from there. The MMA issue order merges the two slots'
// (S, P V) sequences; the producer walks the same order, so the K/V ring is
// consumed first in, first out.
//
// Measured on B200: the MMA forms used here run at the full 64 cycles per
// 128x128x16 instruction in isolation, and TMA streaming is not the limit; the
// kernel is bounded by each slot's chain S -> softmax -> P V, whose softmax
// leg (128 ex2 per row at 16 ex2/clk/SM) alone equals the tensor-core time
// of a tile. Two slots interleave those chains.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>

#include "calibatt.h"
#include "kernels.h"
#include "ptx.cuh"
#include "sched.cuh"
#include "softmax.cuh"

namespace calibatt {
namespace {

constexpr int kAttnThreads = 384;
constexpr int kSoftmaxRegs = 200;  // warps 0-7 after the split
constexpr int kControlRegs = 96;   // warps 8-11 after the split
// the split must fit in the launch allotment (checked against the compiled
// kernel's count before every launch): 168 registers x 384 threads
static_assert(256 * kSoftmaxRegs + 128 * kControlRegs <= 168 * kAttnThreads, "register split");
constexpr int kAttnRing = 5;               // K/V tiles in flight
constexpr float kRescaleThreshold = 8.0f;  // log2 units: move the running max only if it grows by more

struct AttnBarriers {
  uint64_t ring_full[kAttnRing];
  uint64_t ring_empty[kAttnRing];
  uint64_t q_full[2];  // per slot
  uint64_t q_empty[2];
  uint64_t s_full[2];
  uint64_t p_full[2];
  uint64_t o_full[2];
  uint64_t mma_done;
  uint32_t tmem_base;
  int abort;
};

struct AttnLayout {
  static constexpr int kQOff = 0;             // Q[2]
  static constexpr int kRingOff = 2 * kTile;  // K/V ring
  static constexpr int kBarOff = kRingOff + kAttnRing * kTile;
  static constexpr int kBytes = kBarOff + static_cast<int>(sizeof(AttnBarriers));
  static constexpr int kDynSmem = kBytes + 1024;  // + alignment slack
};

// Output rows of a query row of a unit: the row itself (block-sparse unit),
// or the band of rows its anchor row is broadcast to (anchor-query unit of a
// repeated head: same frame, same column); none for a padded row.
__device__ __forceinline__ void unit_dst(const KernelParams& p, const Unit& u, int qrow, bool row_valid,
                                         int64_t& dst0, int& n_dst, int& dst_stride) {
  dst0 = 0;
  n_dst = 0;
  dst_stride = 0;
  if (!row_valid) return;
  if (u.rep) {
    const int kw = p.rep_k * p.rep_W;
    const int f = qrow / kw, rem = qrow % kw;
    const int ja = rem / p.rep_W, c = rem % p.rep_W;
    const int lo = p.band_lo[ja], hi = p.band_hi[ja];
    dst0 = static_cast<int64_t>(f) * p.rep_H * p.rep_W + static_cast<int64_t>(lo) * p.rep_W + c;
    n_dst = hi - lo;
    dst_stride = p.rep_W;
  } else {
    dst0 = qrow;
    n_dst = 1;
  }
}

template <bool SW>  // SW: the polling wait form of short (test) wait limits
__global__ void __launch_bounds__(kAttnThreads, 1)
    attn_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_qb,
                const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                const __grid_constant__ KernelParams p) {
  using L = AttnLayout;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  const uint32_t sbase = smem_u32(smem);
  AttnBarriers& bar = *reinterpret_cast<AttnBarriers*>(smem + L::kBarOff);
  volatile int* abort_flag = &bar.abort;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int G = 2 * gridDim.x;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kAttnRing; ++i) {
      mbar_init(&bar.ring_full[i], 1);
      mbar_init(&bar.ring_empty[i], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bar.q_full[s], 1);
      mbar_init(&bar.q_empty[s], 1);
      mbar_init(&bar.s_full[s], 1);
      mbar_init(&bar.p_full[s], 128);
      mbar_init(&bar.o_full[s], 1);
    }
    mbar_init(&bar.mma_done, 1);
    bar.abort = 0;
    fence_barrier_init();
  }
  if (warp == 9) tmem_alloc(&bar.tmem_base, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bar.tmem_base;

  if (warp >= 8) {
    warpgroup_regs_dec<kControlRegs>();
    if (warp == 8 && lane == 0) {
      // ---------------------------------------------------------- TMA producer
      tma_prefetch_desc(&tm_q);
      if (p.nbq_b > 0) tma_prefetch_desc(&tm_qb);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      Cursor cur[2];
      for (int s = 0; s < 2; ++s) {
        cur[s].round = 0;
        cursor_seek(p, 2 * blockIdx.x + s, G, cur[s]);
      }
      uint32_t stage = 0, phase = 0, n_q[2] = {0, 0};
      bool ok = true;
      auto load_tile = [&](const CUtensorMap* map, int blk, int head) -> bool {
        if (!mbar_wait<SW>(&bar.ring_empty[stage], phase ^ 1, abort_flag, p.status, p.wait_limit_ns)) return false;
        uint8_t* dst = smem + L::kRingOff + stage * kTile;
        mbar_arrive_expect_tx(&bar.ring_full[stage], kTile);
        tma_load_3d(dst, map, &bar.ring_full[stage], 0, blk * 128, head);
        tma_load_3d(dst + kHalf, map, &bar.ring_full[stage], 64, blk * 128, head);
        if (++stage == kAttnRing) {
          stage = 0;
          phase ^= 1;
        }
        return true;
      };
      auto emit_s = [&](int s) -> bool {
        Cursor& c = cur[s];
        if (c.j == 0) {
          if (!mbar_wait<SW>(&bar.q_empty[s], (n_q[s] & 1) ^ 1, abort_flag, p.status, p.wait_limit_ns)) return false;
          uint8_t* dst = smem + L::kQOff + s * kTile;
          const CUtensorMap* qmap = c.u.rep ? &tm_qb : &tm_q;
          mbar_arrive_expect_tx(&bar.q_full[s], kTile);
          tma_load_3d(dst, qmap, &bar.q_full[s], 0, c.u.r * 128, c.u.hq);
          tma_load_3d(dst + kHalf, qmap, &bar.q_full[s], 64, c.u.r * 128, c.u.hq);
          ++n_q[s];
        }
        return load_tile(&tm_k, block_col(p, c.u, c.j), c.u.hkv);
      };
      for (int s = 0; s < 2 && ok; ++s)
        if (cur[s].valid) ok = emit_s(s);
      while (ok && (cur[0].valid || cur[1].valid)) {
        for (int s = 0; s < 2 && ok; ++s) {
          if (!cur[s].valid) continue;
          ok = load_tile(&tm_v, block_col(p, cur[s].u, cur[s].j), cur[s].u.hkv);
          if (!ok) break;
          cursor_next(p, 2 * blockIdx.x + s, G, cur[s]);
          if (cur[s].valid) ok = emit_s(s);
        }
      }
      // no copy may still be landing when the CTA leaves: the latest load of
      // every ring stage and Q buffer has completed
      for (int i = 0; i < kAttnRing; ++i) {
        int st = static_cast<int>(stage) - 1 - i;
        uint32_t ph = phase;
        if (st < 0) {
          st += kAttnRing;
          ph ^= 1;
        }
        volatile int never = 0;
        mbar_wait(&bar.ring_full[st], ph, &never, p.status);
      }
      for (int s = 0; s < 2; ++s)
        if (n_q[s] > 0) {
          volatile int never = 0;
          mbar_wait(&bar.q_full[s], (n_q[s] - 1) & 1, &never, p.status);
        }
    } else if (warp == 9 && lane == 0) {
      // ---------------------------------------------------------- MMA issuer
      Cursor cur[2];
      for (int s = 0; s < 2; ++s) {
        cur[s].round = 0;
        cursor_seek(p, 2 * blockIdx.x + s, G, cur[s]);
      }
      uint32_t stage = 0, phase = 0, n_q[2] = {0, 0}, n_pv[2] = {0, 0};
      const uint64_t qdesc0 = desc_k_base(sbase + L::kQOff);
      const uint64_t kdesc0 = desc_k_base(sbase + L::kRingOff);
      const uint64_t vdesc0 = desc_v_base(sbase + L::kRingOff);
      bool ok = true;
      auto next_stage = [&]() {
        if (++stage == kAttnRing) {
          stage = 0;
          phase ^= 1;
        }
      };
      auto issue_s = [&](int s) -> bool {
        Cursor& c = cur[s];
        if (c.j == 0) {
          if (!mbar_wait<SW>(&bar.q_full[s], n_q[s] & 1, abort_flag, p.status, p.wait_limit_ns)) return false;
        }
        if (!mbar_wait<SW>(&bar.ring_full[stage], phase, abort_flag, p.status, p.wait_limit_ns)) return false;
        tc_fence_after();
        const uint64_t qd = qdesc0 + s * (kTile >> 4), kd = kdesc0 + stage * (kTile >> 4);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)
          mma_ss(tmem + s * 128, qd + desc_k_step(ks), kd + desc_k_step(ks), kIdescS, ks > 0);
        mma_commit(&bar.ring_empty[stage]);
        if (c.j == c.u.nnz - 1) {
          mma_commit(&bar.q_empty[s]);
          ++n_q[s];
        }
        mma_commit(&bar.s_full[s]);
        next_stage();
        return true;
      };
      for (int s = 0; s < 2 && ok; ++s)
        if (cur[s].valid) ok = issue_s(s);
      while (ok && (cur[0].valid || cur[1].valid)) {
        for (int s = 0; s < 2 && ok; ++s) {
          if (!cur[s].valid) continue;
          // O += P V for the current block of slot s (P read from tensor memory)
          if (!(ok = mbar_wait<SW>(&bar.p_full[s], n_pv[s] & 1, abort_flag, p.status, p.wait_limit_ns))) break;
          if (!(ok = mbar_wait<SW>(&bar.ring_full[stage], phase, abort_flag, p.status, p.wait_limit_ns))) break;
          tc_fence_after();
          const uint64_t vd = vdesc0 + stage * (kTile >> 4);
#pragma unroll
          for (int ks = 0; ks < 8; ++ks)
            mma_ts(tmem + 256 + s * 128, tmem + s * 128 + ks * 8, vd + desc_v_step(ks), kIdescPV,
                   (cur[s].j > 0 || ks > 0) ? 1u : 0u);
          mma_commit(&bar.ring_empty[stage]);
          if (cur[s].j == cur[s].u.nnz - 1) mma_commit(&bar.o_full[s]);
          ++n_pv[s];
          next_stage();
          cursor_next(p, 2 * blockIdx.x + s, G, cur[s]);
          if (cur[s].valid) ok = issue_s(s);
        }
      }
      // every issued MMA has finished before tensor memory is released
      mma_commit(&bar.mma_done);
      volatile int never = 0;
      mbar_wait(&bar.mma_done, 0, &never, p.status);
    }
  } else {
    // ---------------------------------------------------------- softmax warpgroups
    warpgroup_regs_inc<kSoftmaxRegs>();
    // After a failed wait the warps keep walking their units with every wait
    // and tensor-memory access skipped, so that the CTA still reaches its
    // final barrier.
    const int s = warp >> 2;
    const int wl = warp & 3;
    const int row = wl * 32 + lane;  // query row inside the tile == TMEM lane
    const uint32_t lane_off = static_cast<uint32_t>(wl * 32) << 16;
    const int g = 2 * blockIdx.x + s;
    const bool ragged_k = (p.n_k & 127) != 0;
    const int valid_last = p.n_k - (p.nbk - 1) * 128;
    uint32_t n_sfull = 0, n_ofull = 0;
    bool ok = true;  // warp-uniform
    auto wait_warp = [&](uint64_t* b, uint32_t parity) -> bool {
      if (ok) ok = __all_sync(0xffffffffu, mbar_wait<SW>(b, parity, abort_flag, p.status, p.wait_limit_ns));
      return ok;
    };

    for (int round = 0;; ++round) {
      Unit u;
      if (!load_unit(p, unit_index(g, G, round), u)) break;
      if (!u.write) continue;
      const int qrow = u.r * 128 + row;
      const bool row_valid = qrow < (u.rep ? p.n_q_b : p.n_q);
      if (u.nnz == 0) {
        // no kept block: O = 0, lse = -inf (for every row a repeated head's
        // anchor row feeds)
        int64_t dst0;
        int n_dst, dst_stride;
        unit_dst(p, u, qrow, row_valid, dst0, n_dst, dst_stride);
        __nv_bfloat16* obase = p.o + static_cast<int64_t>(u.hkv) * p.n_out * 128;
        uint32_t z[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) z[i] = 0;
        for (int q = 0; q < n_dst; ++q) {
          const int64_t d = dst0 + static_cast<int64_t>(q) * dst_stride;
          for (int c = 0; c < 4; ++c) store_row_chunk(obase + d * 128 + c * 32, z);
          if (p.lse) p.lse[static_cast<int64_t>(u.hkv) * p.n_out + d] = -INFINITY;
        }
        continue;
      }
      float m_run = -INFINITY, l_run = 0.f;
      for (int j = 0; j < u.nnz; ++j) {
        const bool mask_tail = ragged_k && (block_col(p, u, j) == p.nbk - 1);
        if (!wait_warp(&bar.s_full[s], n_sfull & 1)) continue;
        ++n_sfull;
        tc_fence_after();
        float sv[128];
        tmem_ld128_wait(tmem + lane_off + s * 128, sv);
        if (mask_tail) {
#pragma unroll
          for (int c = 0; c < 128; ++c)
            if (c >= valid_last) sv[c] = -INFINITY;
        }
        const float mx = row_max128(sv) * p.scale_log2;  // eight independent 3-input max chains
        const float m_new = fmaxf(m_run, mx);
        // keep a stale running max unless it grew by more than the threshold
        // (P <= 2^8 stays exact enough in bf16/fp32 and O needs no rescale)
        const bool need = (m_run == -INFINITY) || (m_new > m_run + kRescaleThreshold);
        float m_use = need ? m_new : m_run;
        if (m_use == -INFINITY) m_use = 0.f;
        const float alpha = need ? ex2_approx(m_run - m_use) : 1.f;
        // two keys at a time: packed fp32x2 multiply-add for s * scale' - m and
        // packed adds into four partial row sums (half the issue slots of the
        // scalar forms; measured 3 % faster on the full Wan-720p step)
        float2 a4[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
        const float2 c2 = make_float2(p.scale_log2, p.scale_log2), nm2 = make_float2(-m_use, -m_use);
        uint32_t pk[32];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const float2 e = exp2_mufu2(ffma2(make_float2(sv[h * 64 + 2 * i], sv[h * 64 + 2 * i + 1]), c2, nm2));
            a4[i & 3] = fadd2(a4[i & 3], e);
            pk[i] = pack_bf16x2(e.x, e.y);
          }
          // P (bf16, two keys per column) over the first 64 columns of S
          tmem_st32(tmem + lane_off + s * 128 + h * 32, pk);
        }
        const float2 s01 = fadd2(a4[0], a4[1]), s23 = fadd2(a4[2], a4[3]);
        const float rs = (s01.x + s01.y) + (s23.x + s23.y);
        l_run = l_run * alpha + rs;
        m_run = m_use;
        // rescale the running O (its P V of block j-1 is complete: the
        // commit that signalled S(j) tracks every earlier MMA)
        if (j > 0 && __any_sync(0xffffffffu, need)) {
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            uint32_t r[32];
            tmem_ld32_wait(tmem + lane_off + 256 + s * 128 + c * 32, r);
#pragma unroll
            for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * alpha);
            tmem_st32(tmem + lane_off + 256 + s * 128 + c * 32, r);
          }
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&bar.p_full[s]);
      }
      if (!wait_warp(&bar.o_full[s], n_ofull & 1)) continue;
      ++n_ofull;
      tc_fence_after();
      const float inv_l = 1.f / l_run;
      const float lse_val = (m_run + log2f(l_run)) * kLn2;
      int64_t dst0;
      int n_dst, dst_stride;
      unit_dst(p, u, qrow, row_valid, dst0, n_dst, dst_stride);
      __nv_bfloat16* obase = p.o + static_cast<int64_t>(u.hkv) * p.n_out * 128;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t r[32];
        tmem_ld32_wait(tmem + lane_off + 256 + s * 128 + c * 32, r);
        uint32_t pkd[16];
#pragma unroll
        for (int i = 0; i < 16; ++i)
          pkd[i] = pack_bf16x2(__uint_as_float(r[2 * i]) * inv_l, __uint_as_float(r[2 * i + 1]) * inv_l);
        for (int q = 0; q < n_dst; ++q)
          store_row_chunk(obase + (dst0 + static_cast<int64_t>(q) * dst_stride) * 128 + c * 32, pkd);
      }
      if (p.lse)
        for (int q = 0; q < n_dst; ++q)
          p.lse[static_cast<int64_t>(u.hkv) * p.n_out + dst0 + static_cast<int64_t>(q) * dst_stride] = lse_val;
      // O has been read out; the next unit's first P V may now overwrite it
      tc_fence_before();
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

int launch_attn(const CUtensorMap& mq, const CUtensorMap& mqb, const CUtensorMap& mk, const CUtensorMap& mv,
                const KernelParams& p, cudaStream_t stream) {
  static_assert(AttnLayout::kDynSmem <= 232448, "shared memory budget");
  const bool short_waits = p.wait_limit_ns < kShortWaitNs;
  const void* fn = short_waits ? reinterpret_cast<const void*>(attn_kernel<true>)
                               : reinterpret_cast<const void*>(attn_kernel<false>);
  static PerDeviceOnce smem_once[2];
  int rc = set_max_smem_once(fn, AttnLayout::kDynSmem, smem_once[short_waits ? 1 : 0]);
  if (rc != CALIBATT_OK) return rc;
  // the register split needs the allotment it was sized for (a property of
  // the compiled kernels, the same on every device)
  static std::once_flag regs_once;
  static int launch_regs = 0;
  std::call_once(regs_once, [] {
    cudaFuncAttributes fa, fb;
    if (cudaFuncGetAttributes(&fa, attn_kernel<false>) == cudaSuccess &&
        cudaFuncGetAttributes(&fb, attn_kernel<true>) == cudaSuccess)
      launch_regs = fa.numRegs < fb.numRegs ? fa.numRegs : fb.numRegs;
  });
  if (launch_regs * kAttnThreads < 256 * kSoftmaxRegs + 128 * kControlRegs) return CALIBATT_ERR_CUDA;
  if (p.n_units <= 0) return CALIBATT_OK;
  int grid = (p.n_units + 1) / 2;
  const int sms = sm_count();
  if (grid > sms) grid = sms;
  if (short_waits)
    attn_kernel<true><<<grid, kAttnThreads, AttnLayout::kDynSmem, stream>>>(mq, mqb, mk, mv, p);
  else
    attn_kernel<false><<<grid, kAttnThreads, AttnLayout::kDynSmem, stream>>>(mq, mqb, mk, mv, p);
  return cudaGetLastError() == cudaSuccess ? CALIBATT_OK : CALIBATT_ERR_CUDA;
}

}  // namespace

int launch_attention(int mode, const void* q, int q_rows, int q_heads, const void* k, const void* v, int kv_rows,
                     int kv_heads, const KernelParams& p, cudaStream_t stream, const void* qb, int qb_rows,
                     int qb_heads) {
  CUtensorMap mq, mqb, mk, mv;
  int rc = make_map(&mq, q, q_rows, q_heads);
  if (rc == CALIBATT_OK) rc = qb ? make_map(&mqb, qb, qb_rows, qb_heads) : (mqb = mq, CALIBATT_OK);
  if (rc == CALIBATT_OK) rc = make_map(&mk, k, kv_rows, kv_heads);
  if (rc == CALIBATT_OK && mode == kAttn) rc = make_map(&mv, v, kv_rows, kv_heads);
  if (rc != CALIBATT_OK) return rc;
  switch (mode) {
    case kAttn: return launch_attn(mq, mqb, mk, mv, p, stream);
    case kLse:
    case kEnergy:
    case kEnergy1: return launch_score(mode, mq, mk, p, stream);
    default: return CALIBATT_ERR_ARG;
  }
}

}  // namespace calibatt
