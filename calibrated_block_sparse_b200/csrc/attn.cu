// Tensor-core attention kernels for sm_100a: block-sparse attention over a
// skip list, the anchor-row pass of repeated heads, and the two passes of the
// block-energy calibration (row log-sum-exp, then tile energy + greedy
// selection). One persistent kernel template serves all four; they differ in
// which tiles are visited and in the softmax-side epilogue.
//
// CTA layout (320 threads, one CTA per SM, two independent query tiles
// "slots" per CTA so that the tensor core works on one slot while the other
// slot's softmax runs):
//   warps 0-3  softmax warpgroup of slot 0 (thread = query row = TMEM lane)
//   warps 4-7  softmax warpgroup of slot 1
//   warp  8    TMA producer (one thread): Q tile per unit, K/V tiles per kept block
//   warp  9    MMA issuer (one thread): tcgen05.mma S = Q K^T and O += P V
// Shared memory: Q[2] (32 KB each) and a ring of 32 KB K/V tiles, all in the
// 128-byte-swizzled layout TMA writes and the MMA descriptors read.
// Tensor memory (512 columns): attention keeps S (fp32, 128 cols) and O
// (fp32, 128 cols) per slot, with P (bf16) written over S; the energy passes
// keep two S buffers per slot instead.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <cstdio>
#include <mutex>

#include "calibatt.h"
#include "kernels.h"
#include "ptx.cuh"
#include "select.cuh"

namespace calibatt {

constexpr int kThreads = 320;
constexpr int kTile = 32768;     // one 128 x 128 bf16 tile
constexpr int kHalf = 16384;     // one 64-column half (one TMA box)
constexpr int kRingAttn = 5;     // K/V tiles in flight, attention
constexpr int kRingScore = 4;    // K tiles in flight, energy passes
constexpr int kEnergyScratch = 16384;  // per slot: per-warp tile sums / sort keys
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRescaleThreshold = 8.0f;  // log2 units: rescale O only if the max grows by more

enum Mode : int { kAttn = 0, kLse = 1, kEnergy = 2 };

struct Barriers {
  uint64_t ring_full[8];
  uint64_t ring_empty[8];
  uint64_t q_full[2];
  uint64_t q_empty[2];
  uint64_t s_full[2][2];
  uint64_t s_empty[2][2];
  uint64_t p_full[2];
  uint64_t o_full[2];
  uint64_t mma_done;
  uint32_t tmem_base;
  int abort;
};

template <int MODE>
struct Layout {
  static constexpr int kRing = (MODE == kAttn) ? kRingAttn : kRingScore;
  static constexpr int kQOff = 0;
  static constexpr int kRingOff = 2 * kTile;
  static constexpr int kAuxOff = kRingOff + kRing * kTile;
  static constexpr int kAuxBytes = (MODE == kEnergy) ? 2 * kEnergyScratch : 0;
  static constexpr int kBarOff = kAuxOff + kAuxBytes;
  static constexpr int kBytes = kBarOff + static_cast<int>(sizeof(Barriers));
  static constexpr int kDynSmem = kBytes + 1024;  // + alignment slack
};

// ------------------------------------------------------------------ work units
struct Unit {
  int hq;    // head index in the Q tensor
  int hkv;   // head index in K / V / O
  int r;     // query block
  int nnz;   // kept key blocks
  int base;  // offset into col_idx
  bool write;  // false: malformed work-list entry, produce nothing
};

__device__ __forceinline__ int unit_index(int g, int G, int round) {
  // snake order over the longest-first list: slot g takes g in even rounds
  // and G-1-g in odd rounds
  return round * G + ((round & 1) ? (G - 1 - g) : g);
}

__device__ __forceinline__ bool load_unit(const KernelParams& p, int idx, Unit& u) {
  if (idx >= p.n_units) return false;
  int code = p.work_list ? __ldg(p.work_list + idx) : idx;
  u.write = true;
  if (code < 0 || code >= p.heads_q * p.nbq) {
    record_error(p.status, CALIBATT_ERR_CSR);
    u.write = false;
    code = 0;
  }
  u.hq = code / p.nbq;
  u.r = code % p.nbq;
  u.hkv = p.head_map ? __ldg(p.head_map + u.hq) : u.hq;
  if (u.hkv < 0 || u.hkv >= p.heads_kv) {
    record_error(p.status, CALIBATT_ERR_ARG);
    u.write = false;
    u.hkv = 0;
  }
  if (p.row_ptr) {
    const int a = __ldg(p.row_ptr + code), b = __ldg(p.row_ptr + code + 1);
    if (a < 0 || b < a || static_cast<int64_t>(b) > p.nnz) {
      record_error(p.status, CALIBATT_ERR_CSR);
      u.base = 0;
      u.nnz = 0;
    } else {
      u.base = a;
      u.nnz = b - a;
    }
  } else {
    u.base = 0;
    u.nnz = p.nbk;
  }
  if (!u.write) u.nnz = 0;
  return true;
}

__device__ __forceinline__ int block_col(const KernelParams& p, const Unit& u, int j) {
  if (!p.col_idx) return j;
  int c = __ldg(p.col_idx + u.base + j);
  if (c < 0 || c >= p.nbk) {
    record_error(p.status, CALIBATT_ERR_CSR);
    c = c < 0 ? 0 : p.nbk - 1;
  }
  return c;
}

// Per-slot cursor over the (unit, kept block) sequence, skipping units with
// no kept block. Used identically by the producer and the MMA issuer so that
// both walk the same tile order.
struct Cursor {
  int round;
  int j;
  bool valid;
  Unit u;
};

__device__ __forceinline__ void cursor_seek(const KernelParams& p, int g, int G, Cursor& c) {
  while (true) {
    if (!load_unit(p, unit_index(g, G, c.round), c.u)) {
      c.valid = false;
      return;
    }
    if (c.u.nnz > 0) {
      c.j = 0;
      c.valid = true;
      return;
    }
    ++c.round;
  }
}

__device__ __forceinline__ void cursor_next(const KernelParams& p, int g, int G, Cursor& c) {
  if (++c.j < c.u.nnz) return;
  ++c.round;
  cursor_seek(p, g, G, c);
}

// ------------------------------------------------------------------ MMA descriptors
// Q and K tiles: K-major (head dim contiguous), two 64-column halves, 128-byte
// swizzle; a K step of 16 elements advances 32 bytes inside a half.
__device__ __forceinline__ uint64_t desc_kmajor(uint32_t tile, int ks) {
  return smem_desc_sw128(tile + (ks >> 2) * kHalf + (ks & 3) * 32, 16, 1024);
}
// V tile as the B operand of P V: N (= head dim) contiguous, so MN-major; the
// two 64-column halves are the MN atoms (LBO), 8-key groups are 1 KB apart (SBO).
__device__ __forceinline__ uint64_t desc_v(uint32_t tile, int ks) {
  return smem_desc_sw128(tile + ks * 2048, kHalf, 1024);
}

constexpr uint32_t kIdescS = idesc_bf16_f32(128, 128, false);
constexpr uint32_t kIdescPV = idesc_bf16_f32(128, 128, true);

// ------------------------------------------------------------------ softmax-side helpers
__device__ __forceinline__ void store_out_row(__nv_bfloat16* dst, const uint32_t (&packed)[16]) {
  uint4* d = reinterpret_cast<uint4*>(dst);
#pragma unroll
  for (int i = 0; i < 4; ++i) d[i] = make_uint4(packed[4 * i], packed[4 * i + 1], packed[4 * i + 2], packed[4 * i + 3]);
}

// ------------------------------------------------------------------ the kernel
template <int MODE>
__global__ void __launch_bounds__(kThreads, 1)
    attn_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ KernelParams p) {
  using L = Layout<MODE>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  const uint32_t sbase = smem_u32(smem);
  Barriers& bar = *reinterpret_cast<Barriers*>(smem + L::kBarOff);
  volatile int* abort_flag = &bar.abort;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int G = 2 * gridDim.x;

  if (threadIdx.x == 0) {
    for (int i = 0; i < L::kRing; ++i) {
      mbar_init(&bar.ring_full[i], 1);
      mbar_init(&bar.ring_empty[i], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bar.q_full[s], 1);
      mbar_init(&bar.q_empty[s], 1);
      mbar_init(&bar.p_full[s], 128);
      mbar_init(&bar.o_full[s], 1);
      for (int b = 0; b < 2; ++b) {
        mbar_init(&bar.s_full[s][b], 1);
        mbar_init(&bar.s_empty[s][b], 128);
      }
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

  if (warp == 8) {
    // ---------------------------------------------------------- TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      if (MODE == kAttn) tma_prefetch_desc(&tm_v);
      Cursor cur[2];
      for (int s = 0; s < 2; ++s) {
        cur[s].round = 0;
        cursor_seek(p, 2 * blockIdx.x + s, G, cur[s]);
      }
      uint32_t n_tiles = 0, n_q[2] = {0, 0};
      bool ok = true;
      auto load_tile = [&](const CUtensorMap* map, int blk, int head) -> bool {
        const int st = n_tiles % L::kRing;
        const uint32_t ph = (n_tiles / L::kRing) & 1;
        if (!mbar_wait(&bar.ring_empty[st], ph ^ 1, abort_flag, p.status)) return false;
        uint8_t* dst = smem + L::kRingOff + st * kTile;
        mbar_arrive_expect_tx(&bar.ring_full[st], kTile);
        tma_load_3d(dst, map, &bar.ring_full[st], 0, blk * 128, head);
        tma_load_3d(dst + kHalf, map, &bar.ring_full[st], 64, blk * 128, head);
        ++n_tiles;
        return true;
      };
      auto emit_s = [&](int s) -> bool {
        Cursor& c = cur[s];
        if (c.j == 0) {
          if (!mbar_wait(&bar.q_empty[s], (n_q[s] & 1) ^ 1, abort_flag, p.status)) return false;
          uint8_t* dst = smem + L::kQOff + s * kTile;
          mbar_arrive_expect_tx(&bar.q_full[s], kTile);
          tma_load_3d(dst, &tm_q, &bar.q_full[s], 0, c.u.r * 128, c.u.hq);
          tma_load_3d(dst + kHalf, &tm_q, &bar.q_full[s], 64, c.u.r * 128, c.u.hq);
          ++n_q[s];
        }
        return load_tile(&tm_k, block_col(p, c.u, c.j), c.u.hkv);
      };
      if (MODE == kAttn) {
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
      } else {
        while (ok && (cur[0].valid || cur[1].valid)) {
          for (int s = 0; s < 2 && ok; ++s) {
            if (!cur[s].valid) continue;
            ok = emit_s(s);
            cursor_next(p, 2 * blockIdx.x + s, G, cur[s]);
          }
        }
      }
      // Do not leave while a copy may still be landing: the latest load of
      // every ring stage and Q buffer must have completed.
      for (uint32_t t = (n_tiles > static_cast<uint32_t>(L::kRing) ? n_tiles - L::kRing : 0); t < n_tiles; ++t) {
        volatile int never = 0;
        mbar_wait(&bar.ring_full[t % L::kRing], (t / L::kRing) & 1, &never, p.status);
      }
      for (int s = 0; s < 2; ++s)
        if (n_q[s] > 0) {
          volatile int never = 0;
          mbar_wait(&bar.q_full[s], (n_q[s] - 1) & 1, &never, p.status);
        }
    }
  } else if (warp == 9) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0) {
      Cursor cur[2];
      for (int s = 0; s < 2; ++s) {
        cur[s].round = 0;
        cursor_seek(p, 2 * blockIdx.x + s, G, cur[s]);
      }
      uint32_t n_tiles = 0, n_q[2] = {0, 0}, n_s[2] = {0, 0}, n_pv[2] = {0, 0};
      bool ok = true;
      auto issue_s = [&](int s) -> bool {
        Cursor& c = cur[s];
        if (c.j == 0) {
          if (!mbar_wait(&bar.q_full[s], n_q[s] & 1, abort_flag, p.status)) return false;
        }
        uint32_t d_tmem;
        int buf = 0;
        if (MODE == kAttn) {
          d_tmem = tmem + s * 128;
        } else {
          buf = n_s[s] & 1;
          if (!mbar_wait(&bar.s_empty[s][buf], ((n_s[s] >> 1) & 1) ^ 1, abort_flag, p.status)) return false;
          d_tmem = tmem + (2 * s + buf) * 128;
        }
        const int st = n_tiles % L::kRing;
        if (!mbar_wait(&bar.ring_full[st], (n_tiles / L::kRing) & 1, abort_flag, p.status)) return false;
        tc_fence_after();
        const uint32_t qa = sbase + L::kQOff + s * kTile;
        const uint32_t ka = sbase + L::kRingOff + st * kTile;
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) mma_ss(d_tmem, desc_kmajor(qa, ks), desc_kmajor(ka, ks), kIdescS, ks > 0);
        mma_commit(&bar.ring_empty[st]);
        if (c.j == c.u.nnz - 1) {
          mma_commit(&bar.q_empty[s]);
          ++n_q[s];
        }
        mma_commit(&bar.s_full[s][buf]);
        ++n_s[s];
        ++n_tiles;
        return true;
      };
      if (MODE == kAttn) {
        for (int s = 0; s < 2 && ok; ++s)
          if (cur[s].valid) ok = issue_s(s);
        while (ok && (cur[0].valid || cur[1].valid)) {
          for (int s = 0; s < 2 && ok; ++s) {
            if (!cur[s].valid) continue;
            // O += P V for the current block of slot s
            if (!(ok = mbar_wait(&bar.p_full[s], n_pv[s] & 1, abort_flag, p.status))) break;
            const int st = n_tiles % L::kRing;
            if (!(ok = mbar_wait(&bar.ring_full[st], (n_tiles / L::kRing) & 1, abort_flag, p.status))) break;
            tc_fence_after();
            const uint32_t va = sbase + L::kRingOff + st * kTile;
#pragma unroll
            for (int ks = 0; ks < 8; ++ks)
              mma_ts(tmem + 256 + s * 128, tmem + s * 128 + ks * 8, desc_v(va, ks), kIdescPV,
                     (cur[s].j > 0 || ks > 0) ? 1u : 0u);
            mma_commit(&bar.ring_empty[st]);
            if (cur[s].j == cur[s].u.nnz - 1) mma_commit(&bar.o_full[s]);
            ++n_pv[s];
            ++n_tiles;
            cursor_next(p, 2 * blockIdx.x + s, G, cur[s]);
            if (cur[s].valid) ok = issue_s(s);
          }
        }
      } else {
        while (ok && (cur[0].valid || cur[1].valid)) {
          for (int s = 0; s < 2 && ok; ++s) {
            if (!cur[s].valid) continue;
            ok = issue_s(s);
            cursor_next(p, 2 * blockIdx.x + s, G, cur[s]);
          }
        }
      }
      // all issued MMAs finished before TMEM is released
      mma_commit(&bar.mma_done);
      volatile int never = 0;
      mbar_wait(&bar.mma_done, 0, &never, p.status);
    }
  } else {
    // ---------------------------------------------------------- softmax warpgroups
    // After a failed (timed-out or aborted) wait the warps keep walking their
    // units with every wait and tensor-memory access skipped, so that the
    // named barriers of the warpgroup are still met by all four warps.
    const int s = warp >> 2;
    const int wl = warp & 3;
    const int row = wl * 32 + lane;  // query row inside the tile == TMEM lane
    const uint32_t lane_off = static_cast<uint32_t>(wl * 32) << 16;
    const int g = 2 * blockIdx.x + s;
    const bool ragged_k = (p.n_k & 127) != 0;
    const int valid_last = p.n_k - (p.nbk - 1) * 128;
    uint32_t n_sfull = 0, n_ofull = 0;
    bool ok = true;  // warp-uniform
    float* part = reinterpret_cast<float*>(smem + L::kAuxOff + s * kEnergyScratch);
    auto wait_warp = [&](uint64_t* b, uint32_t parity) -> bool {
      if (ok) ok = __all_sync(0xffffffffu, mbar_wait(b, parity, abort_flag, p.status));
      return ok;
    };

    for (int round = 0;; ++round) {
      Unit u;
      if (!load_unit(p, unit_index(g, G, round), u)) break;
      if (!u.write) continue;
      const int qrow = u.r * 128 + row;
      const bool row_valid = qrow < p.n_q;

      if (MODE == kAttn) {
        if (u.nnz == 0) {
          // no kept block: O = 0, lse = -inf
          if (row_valid) {
            uint32_t z[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) z[i] = 0;
            for (int c = 0; c < 4; ++c)
              store_out_row(p.o + (static_cast<int64_t>(u.hkv) * p.n_out + qrow) * 128 + c * 32, z);
            if (p.lse) p.lse[static_cast<int64_t>(u.hkv) * p.n_out + qrow] = -INFINITY;
          }
          continue;
        }
        float m_run = -INFINITY, l_run = 0.f;
        for (int j = 0; j < u.nnz; ++j) {
          const bool mask_tail = ragged_k && (block_col(p, u, j) == p.nbk - 1);
          if (!wait_warp(&bar.s_full[s][0], n_sfull & 1)) continue;
          ++n_sfull;
          tc_fence_after();
          float sv[128];
          tmem_ld128_wait(tmem + lane_off + s * 128, sv);
          if (mask_tail) {
#pragma unroll
            for (int c = 0; c < 128; ++c)
              if (c >= valid_last) sv[c] = -INFINITY;
          }
          float mx = sv[0];
#pragma unroll
          for (int c = 1; c < 128; ++c) mx = fmaxf(mx, sv[c]);
          mx *= p.scale_log2;
          const float m_new = fmaxf(m_run, mx);
          // keep a stale running max unless it grew by more than the threshold
          // (P <= 2^8 stays exact enough in bf16/fp32 and O needs no rescale)
          const bool need = (m_run == -INFINITY) || (m_new > m_run + kRescaleThreshold);
          float m_use = need ? m_new : m_run;
          if (m_use == -INFINITY) m_use = 0.f;
          const float alpha = need ? ex2_approx(m_run - m_use) : 1.f;
          float rs = 0.f;
          uint32_t pk[32];
#pragma unroll
          for (int h = 0; h < 2; ++h) {
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              const float p0 = ex2_approx(fmaf(sv[h * 64 + 2 * i], p.scale_log2, -m_use));
              const float p1 = ex2_approx(fmaf(sv[h * 64 + 2 * i + 1], p.scale_log2, -m_use));
              rs += p0 + p1;
              pk[i] = pack_bf16x2(p0, p1);
            }
            // P (bf16, two keys per column) over the first 64 columns of S
            tmem_st32(tmem + lane_off + s * 128 + h * 32, pk);
          }
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
        // destination rows: one per query (sparse), or a band of rows (repeat)
        int64_t dst0 = 0;
        int n_dst = 0, dst_stride = 0;
        if (row_valid) {
          if (p.rep_W > 0) {
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
        __nv_bfloat16* obase = p.o + static_cast<int64_t>(u.hkv) * p.n_out * 128;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t r[32];
          tmem_ld32_wait(tmem + lane_off + 256 + s * 128 + c * 32, r);
          uint32_t pkd[16];
#pragma unroll
          for (int i = 0; i < 16; ++i)
            pkd[i] = pack_bf16x2(__uint_as_float(r[2 * i]) * inv_l, __uint_as_float(r[2 * i + 1]) * inv_l);
          for (int t = 0; t < n_dst; ++t)
            store_out_row(obase + (dst0 + static_cast<int64_t>(t) * dst_stride) * 128 + c * 32, pkd);
        }
        if (p.lse)
          for (int t = 0; t < n_dst; ++t)
            p.lse[static_cast<int64_t>(u.hkv) * p.n_out + dst0 + static_cast<int64_t>(t) * dst_stride] = lse_val;
        // O has been read out; the next unit's first P V may now overwrite it
        tc_fence_before();
      } else {
        // ------------------------------------------------ energy passes (S only)
        float lse2 = 0.f;
        if (MODE == kEnergy && row_valid)
          lse2 = p.lse_ws[static_cast<int64_t>(u.hq) * p.nbq * 128 + qrow];
        float m_run = -INFINITY, l_run = 0.f;
        for (int j = 0; j < u.nnz; ++j) {
          const int buf = n_sfull & 1;
          float acc = 0.f;
          if (wait_warp(&bar.s_full[s][buf], (n_sfull >> 1) & 1)) {
            ++n_sfull;
            tc_fence_after();
            float sv[128];
            tmem_ld128_wait(tmem + lane_off + (2 * s + buf) * 128, sv);
            tc_fence_before();
            mbar_arrive(&bar.s_empty[s][buf]);
            const int nvalid = (ragged_k && j == p.nbk - 1) ? valid_last : 128;
            if (MODE == kLse) {
              float mx = -INFINITY;
#pragma unroll
              for (int c = 0; c < 128; ++c)
                if (c < nvalid) mx = fmaxf(mx, sv[c]);
              mx *= p.scale_log2;
              const float m_new = fmaxf(m_run, mx);
#pragma unroll
              for (int c = 0; c < 128; ++c)
                if (c < nvalid) acc += ex2_approx(fmaf(sv[c], p.scale_log2, -m_new));
              l_run = (m_run == -INFINITY ? 0.f : l_run * ex2_approx(m_run - m_new)) + acc;
              m_run = m_new;
            } else if (row_valid) {
              // this row's share of E[r][j]: sum_j exp(S_ij - lse_i)
#pragma unroll
              for (int c = 0; c < 128; ++c)
                if (c < nvalid) acc += ex2_approx(fmaf(sv[c], p.scale_log2, -lse2));
            }
          }
          if (MODE == kEnergy) {
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
            if (lane == 0) part[wl * 1024 + j] = acc;
          }
        }
        if (MODE == kLse) {
          if (ok) p.lse_ws[static_cast<int64_t>(u.hq) * p.nbq * 128 + qrow] = m_run + log2f(l_run);
        } else {
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
            named_bar_sync(1 + s, 128);
            SelectOut out{p.mask ? p.mask + erow : nullptr, p.kept ? p.kept + (erow / p.nbk) : nullptr,
                          p.counts ? p.counts + erow : nullptr};
            if (!ok) out = SelectOut{nullptr, nullptr, nullptr};
            select_row(part, p.nbk, p.eps_fx, reinterpret_cast<uint8_t*>(part + 1024),
                       reinterpret_cast<unsigned long long*>(part + 2048), row, 128, 1 + s, out);
          }
          named_bar_sync(1 + s, 128);
        }
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

// ------------------------------------------------------------------ host side
namespace {

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  });
  return fn;
}

// [heads][rows][128] bf16 viewed as a 3D tensor (128, rows, heads); boxes of
// 64 x 128 x 1 with 128-byte swizzle. Rows past `rows` read as zeros.
int make_map(CUtensorMap* map, const void* base, int rows, int heads) {
  EncodeTiledFn enc = get_encode();
  if (!enc) return CALIBATT_ERR_CUDA;
  cuuint64_t dims[3] = {128, static_cast<cuuint64_t>(rows), static_cast<cuuint64_t>(heads)};
  cuuint64_t strides[2] = {256, static_cast<cuuint64_t>(rows) * 256};
  cuuint32_t box[3] = {64, 128, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? CALIBATT_OK : CALIBATT_ERR_CUDA;
}

int sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) return 148;
  return n;
}

template <int MODE>
int launch_mode(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv, const KernelParams& p,
                cudaStream_t stream) {
  using L = Layout<MODE>;
  static_assert(L::kDynSmem <= 232448, "shared memory budget");
  static bool configured = false;  // per process; attribute is per function
  if (!configured) {
    if (cudaFuncSetAttribute(attn_kernel<MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kDynSmem) !=
        cudaSuccess)
      return CALIBATT_ERR_CUDA;
    configured = true;
  }
  if (p.n_units <= 0) return CALIBATT_OK;
  int grid = (p.n_units + 1) / 2;
  const int sms = sm_count();
  if (grid > sms) grid = sms;
  attn_kernel<MODE><<<grid, kThreads, L::kDynSmem, stream>>>(mq, mk, mv, p);
  return cudaGetLastError() == cudaSuccess ? CALIBATT_OK : CALIBATT_ERR_CUDA;
}

}  // namespace

int launch_attention(int mode, const void* q, int q_rows, int q_heads, const void* k, const void* v, int kv_rows,
                     int kv_heads, const KernelParams& p, cudaStream_t stream) {
  CUtensorMap mq, mk, mv;
  int rc = make_map(&mq, q, q_rows, q_heads);
  if (rc == CALIBATT_OK) rc = make_map(&mk, k, kv_rows, kv_heads);
  if (rc == CALIBATT_OK) rc = make_map(&mv, v ? v : k, kv_rows, kv_heads);
  if (rc != CALIBATT_OK) return rc;
  switch (mode) {
    case kAttn: return launch_mode<kAttn>(mq, mk, mv, p, stream);
    case kLse: return launch_mode<kLse>(mq, mk, mv, p, stream);
    case kEnergy: return launch_mode<kEnergy>(mq, mk, mv, p, stream);
    default: return CALIBATT_ERR_ARG;
  }
}

}  // namespace calibatt
