// Greedy eps selection of one block-row by one warp (explainer §三, step 3:
// keep the fewest key blocks whose cumulative energy reaches eps; greedy
// order: energy descending, equal energies by lower column first).
//
// No sort is needed. With every energy taken exactly in fixed point (50
// fraction bits, truncated), the greedy cut is fixed by the energy tau of the
// block at which the running sum first reaches eps:
//   tau = the largest energy v with  S(v) = sum_{E >= v} fx(E) >= eps_fx.
// S is non-increasing in v, and the float bit patterns of non-negative
// energies order like their values, so tau is found digit by digit over its
// bit pattern (a radix select weighted by energy): bits 30..21, 20..11 and
// 10..1 as three 10-bit digits, then bit 0. For each digit, the blocks that
// share the digits found so far are summed into a 1024-bucket shared-memory
// histogram of exact 64-bit fixed-point sums (integer atomics: order does
// not matter), and a two-stage warp suffix scan finds the largest digit whose
// suffix still reaches eps. Once 32 or fewer blocks share the prefix, the
// remaining search runs in registers (each lane one candidate). The kept set
// is every block with E > tau plus the first r blocks (in column order) with
// E == tau, r the fewest that reach eps. Because the sums are exact integers,
// the result equals a sequential greedy sum in sorted order, and it does not
// depend on how the row is split over lanes.
//
// Tie accounting (spec: decisions within a window delta of the
// threshold are counted): a row is tie-affected when the running sum with or
// without its last kept block lies within delta of eps, or when the last kept
// block's energy and the next one's in greedy order differ by less than delta.
#pragma once
#include <cstdint>

namespace calibatt {

constexpr int kFixBits = 50;
constexpr int kSelectBuckets = 1024;
constexpr int kSelectScratchBytes = kSelectBuckets * 8;  // per selecting warp

struct SelectOut {
  uint8_t* mask;     // [nb] or NULL
  int32_t* kept;     // [1] or NULL
  uint16_t* counts;  // [nb] or NULL (counts += mask, saturating)
  uint8_t* tie;      // [1] or NULL: 1 if the row's cut is tie-affected
};

__device__ __forceinline__ float clamp_energy(float e) {
  if (!(e > 0.f)) return 0.f;  // NaN, negative and zero
  return e > 4.f ? 4.f : e;
}

// floor(e * 2^50) for e in [0, 4], exact.
__device__ __forceinline__ long long energy_fixed(uint32_t b) {
  if (b == 0) return 0;
  int ex = static_cast<int>((b >> 23) & 0xFFu);
  uint32_t man = b & 0x7FFFFFu;
  if (ex == 0) ex = 1; else man |= 0x800000u;
  // e = man * 2^(ex - 150)  ->  e * 2^50 = man * 2^(ex - 100)
  const int sh = ex - 100;
  if (sh >= 0) return static_cast<long long>(man) << sh;
  if (-sh >= 24) return 0;
  return static_cast<long long>(man >> (-sh));
}

__device__ __forceinline__ long long warp_sum64(long long v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Inclusive suffix sum over lanes: lane l gets sum_{l' >= l} v.
__device__ __forceinline__ long long warp_suffix64(long long v, int lane) {
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const long long t = __shfl_down_sync(0xffffffffu, v, o);
    if (lane + o < 32) v += t;
  }
  return v;
}

// |a - b| < w for exact fixed-point values.
__device__ __forceinline__ bool fx_close(long long a, long long b, long long w) {
  const long long d = a > b ? a - b : b - a;
  return d < w;
}

// Adds v to a 64-bit bucket in shared memory (no return value needed).
__device__ __forceinline__ void shared_add64(unsigned long long* p, unsigned long long v) {
  asm volatile("red.shared.add.u64 [%0], %1;" ::"r"(static_cast<uint32_t>(__cvta_generic_to_shared(p))), "l"(v)
               : "memory");
}

// Column c = lane + 32 i of the row is element i of the lane's arrays.
// E: the row (shared or global memory, nb <= 32 * PER); hist: 8 KB of shared
// memory (never global) for this warp, 16-byte aligned; tie_fx: the tie
// window in fixed point (used only when out.tie is set). Every lane of the
// warp must call.
template <int PER>
__device__ __forceinline__ void warp_select(const float* E, int nb, long long eps_fx, long long tie_fx,
                                         unsigned long long* hist, SelectOut out) {
  const int lane = threadIdx.x & 31;
  const unsigned lt_mask = (1u << lane) - 1u;
  uint32_t bits[PER];
  long long tot = 0;
  int nz = 0;
  uint32_t my_top = 0;
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    const int c = lane + 32 * i;
    const float e = c < nb ? clamp_energy(E[c]) : 0.f;
    bits[i] = __float_as_uint(e);
    tot += energy_fixed(bits[i]);
    nz += e > 0.f;
    my_top = bits[i] > my_top ? bits[i] : my_top;
  }
  tot = warp_sum64(tot);
  nz = static_cast<int>(__reduce_add_sync(0xffffffffu, static_cast<unsigned>(nz)));
  const uint32_t top_bits = __reduce_max_sync(0xffffffffu, my_top);
  // greedy order's first block: the largest energy, lowest column
  int my_col = 0x7FFFFFFF;
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    const int c = lane + 32 * i;
    if (c < nb && bits[i] == top_bits && c < my_col) my_col = c;
  }
  const int top_col = static_cast<int>(__reduce_min_sync(0xffffffffu, static_cast<unsigned>(my_col)));

  // 0 = the single top block, 1 = every nonzero block, 2 = greedy cut at tau
  int mode = 2;
  if (eps_fx <= 0 || nz == 0) mode = 0;
  else if (tot < eps_fx) mode = 1;

  uint32_t tau = 0;
  long long above = 0;  // sum of fx over blocks with energy > tau
  if (mode == 2) {
    // prefix: tau's bits above `shift` found so far; base: sum of fx over the
    // blocks whose bits above the prefix's position are larger
    uint32_t prefix = 0;
    int shift = 31;
    long long base = 0;
    bool done = false;
    while (!done) {
      // candidates share the prefix; count them
      int m_mine = 0;
#pragma unroll
      for (int i = 0; i < PER; ++i)
        m_mine += (bits[i] != 0 && (shift >= 31 || (bits[i] >> shift) == prefix));
      const int m = static_cast<int>(__reduce_add_sync(0xffffffffu, static_cast<unsigned>(m_mine)));
      if (m <= 32 || shift == 0) {
        // compact the candidates (one per lane) and finish in registers
        int off = m_mine;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int t = __shfl_up_sync(0xffffffffu, off, o);
          if (lane >= o) off += t;
        }
        off -= m_mine;
        __syncwarp();
        uint32_t* cand = reinterpret_cast<uint32_t*>(hist);
#pragma unroll
        for (int i = 0; i < PER; ++i)
          if (bits[i] != 0 && (shift >= 31 || (bits[i] >> shift) == prefix)) cand[off++] = bits[i];
        __syncwarp();
        // m <= 32 here: shift == 0 leaves one value, so every candidate is equal
        const uint32_t cb = lane < m && lane < 32 ? cand[lane] : 0u;
        const long long cf = energy_fixed(cb);
        long long T = 0;  // sum of fx over candidates >= cb
        const int mm = m < 32 ? m : 32;
        for (int j = 0; j < mm; ++j) {
          const uint32_t bj = __shfl_sync(0xffffffffu, cb, j);
          const long long fj = __shfl_sync(0xffffffffu, cf, j);
          T += bj >= cb ? fj : 0;
        }
        if (m > 32) {
          // shift == 0 with more than 32 equal candidates: every one equals the first
          T = cf * m;
        }
        const bool ok = lane < mm && base + T >= eps_fx;
        tau = __reduce_max_sync(0xffffffffu, ok ? cb : 0u);
        above = base + warp_sum64(lane < mm && cb > tau ? cf : 0);
        if (m > 32) above = base;
        __syncwarp();
        done = true;
      } else {
        // one radix digit: histogram of the candidates' fx by digit
        const int dshift = shift >= 31 ? 21 : (shift == 21 ? 11 : (shift == 11 ? 1 : 0));
        const uint32_t dmask = dshift == 0 ? 1u : 1023u;
        uint4* h4 = reinterpret_cast<uint4*>(hist);
#pragma unroll
        for (int i = 0; i < kSelectScratchBytes / 16 / 32; ++i) h4[lane + 32 * i] = make_uint4(0u, 0u, 0u, 0u);
        __syncwarp();
#pragma unroll
        for (int i = 0; i < PER; ++i) {
          if (bits[i] != 0 && (shift >= 31 || (bits[i] >> shift) == prefix)) {
            const long long f = energy_fixed(bits[i]);
            if (f > 0) shared_add64(hist + ((bits[i] >> dshift) & dmask), static_cast<unsigned long long>(f));
          }
        }
        __syncwarp();
        // stage 1: lane l owns buckets 32 l .. 32 l + 31
        long long lsum = 0;
        const ulonglong2* h2 = reinterpret_cast<const ulonglong2*>(hist + 32 * lane);
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const ulonglong2 v = h2[i];
          lsum += static_cast<long long>(v.x) + static_cast<long long>(v.y);
        }
        const long long suf = warp_suffix64(lsum, lane);
        // the largest lane whose suffix reaches eps (lane 0's suffix always does)
        const unsigned reach = __ballot_sync(0xffffffffu, base + suf >= eps_fx);
        const int L = 31 - __clz(reach);
        const long long after_L = __shfl_sync(0xffffffffu, suf - lsum, L);  // buckets above lane L's
        // stage 2: lane j looks at bucket 32 L + j
        const long long bv = static_cast<long long>(hist[32 * L + lane]);
        const long long suf2 = warp_suffix64(bv, lane) + after_L;
        const unsigned reach2 = __ballot_sync(0xffffffffu, base + suf2 >= eps_fx);
        const int j = 31 - __clz(reach2);
        const int d = 32 * L + j;
        base += __shfl_sync(0xffffffffu, suf2 - bv, j);  // buckets above d
        __syncwarp();  // the histogram is reused by the next level
        prefix = shift >= 31 ? static_cast<uint32_t>(d) : ((prefix << (shift - dshift)) | static_cast<uint32_t>(d));
        shift = dshift;
      }
    }
  }

  // rank of each block among the blocks equal to tau, in column order, and
  // the keep decision
  const long long ft = mode == 2 ? energy_fixed(tau) : 0;
  const long long r_need = mode == 2 ? (ft > 0 ? (eps_fx - above + ft - 1) / ft : 1) : 0;
  int before = 0;  // equal blocks in earlier columns
  int kept_mine = 0;
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    const int c = lane + 32 * i;
    const bool in = c < nb;
    const bool eq = mode == 2 && in && bits[i] == tau;
    const unsigned bal = __ballot_sync(0xffffffffu, eq);
    bool k;
    if (mode == 0) k = in && c == top_col;
    else if (mode == 1) k = in && bits[i] > 0;
    else k = in && (bits[i] > tau || (eq && before + __popc(bal & lt_mask) < r_need));
    before += __popc(bal);
    kept_mine += k;
    if (in) {
      if (out.mask) out.mask[c] = k ? 1 : 0;
      if (out.counts && k) {
        const uint16_t old = out.counts[c];
        if (old != 0xFFFFu) out.counts[c] = old + 1;
      }
    }
  }
  if (out.kept) {
    const unsigned kept = __reduce_add_sync(0xffffffffu, static_cast<unsigned>(kept_mine));
    if (lane == 0) *out.kept = static_cast<int32_t>(kept);
  }
  if (out.tie) {
    // the cut in greedy order: running sums with and without the last kept
    // block, and the energies of the last kept block and of the next one
    long long cum_at = 0, cum_before = 0, e_last = 0, e_next = -1;
    if (mode == 2) {
      const int n_eq = before;  // every lane holds the total after the loop
      cum_at = above + r_need * ft;
      cum_before = cum_at - ft;
      e_last = ft;
      if (n_eq > r_need) {
        e_next = ft;
      } else {
        uint32_t nxt = 0;  // largest energy below tau, plus one (0: none)
#pragma unroll
        for (int i = 0; i < PER; ++i) {
          const int c = lane + 32 * i;
          if (c < nb && bits[i] < tau && bits[i] + 1 > nxt) nxt = bits[i] + 1;
        }
        nxt = __reduce_max_sync(0xffffffffu, nxt);
        if (nxt > 0) e_next = energy_fixed(nxt - 1);
      }
    } else if (mode == 1) {
      uint32_t mn = 0xFFFFFFFFu;  // smallest nonzero energy: the last kept block
#pragma unroll
      for (int i = 0; i < PER; ++i)
        if (bits[i] > 0 && bits[i] < mn) mn = bits[i];
      mn = __reduce_min_sync(0xffffffffu, mn);
      cum_at = tot;
      e_last = energy_fixed(mn);
      cum_before = tot - e_last;
      if (nz < nb) e_next = 0;  // a zero-energy block follows
    } else {
      // one block kept: the top one (every energy zero: the lowest column)
      e_last = nz > 0 ? energy_fixed(top_bits) : 0;
      cum_at = e_last;
      cum_before = 0;
      if (nb > 1) {
        uint32_t sec = 0;  // the next block in greedy order, plus one
#pragma unroll
        for (int i = 0; i < PER; ++i) {
          const int c = lane + 32 * i;
          if (c < nb && c != top_col && bits[i] + 1 > sec) sec = bits[i] + 1;
        }
        sec = __reduce_max_sync(0xffffffffu, sec);
        e_next = energy_fixed(sec - 1);
      }
    }
    const bool t = fx_close(cum_at, eps_fx, tie_fx) || fx_close(cum_before, eps_fx, tie_fx) ||
                   (e_next >= 0 && e_last - e_next < tie_fx);
    if (lane == 0) *out.tie = t ? 1 : 0;
  }
}

}  // namespace calibatt
