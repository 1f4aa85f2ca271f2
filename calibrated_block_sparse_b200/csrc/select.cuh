// Greedy eps selection of one block-row by one warp (explainer §三, step 3:
// keep the fewest key blocks whose cumulative energy reaches eps; greedy
// order: energy descending, equal energies by lower column first).
//
// No sort is needed. With every energy taken exactly in fixed point (50
// fraction bits, truncated), the greedy cut is fixed by the energy tau of the
// block at which the running sum first reaches eps:
//   tau = the largest energy v with  S(v) = sum_{E >= v} fx(E) >= eps_fx.
// S is non-increasing in v, and the float bit patterns of non-negative
// energies order like their values, so tau can be searched digit by digit
// over its bit pattern (a radix select weighted by energy). The digits (bits
// 30..20, then 19..10, then 9..0) are found by binary search with fp32 warp
// sums until 32 or fewer candidate blocks share the digits found so far.
// (Shared-memory histograms of the digits were measured slower on block
// energies: a row's tail crowds into few buckets and the atomics serialise.) Those
// are finished exactly in registers: each lane holds one candidate, and the
// exact fixed-point suffix sums over the candidates plus the exact sum of
// every larger block give tau. The fp32 digits only guide the search: the
// prefix range they lead to is accepted only if its exact bounds bracket eps
// (sum of the larger blocks < eps <= that plus the candidates); otherwise
// (a bucket boundary within fp32 rounding of eps) the row falls back to an
// exact binary search over bit patterns with 64-bit sums. The kept set is
// every block with E > tau plus the first r blocks (in column order) with
// E == tau, r the fewest that reach eps. Because all decisions use exact
// integer sums, the result equals a sequential greedy sum in sorted order
// and does not depend on how the row is split over lanes.
//
// Tie accounting (spec: decisions within a window delta of the
// threshold are counted): a row is tie-affected when the running sum with or
// without its last kept block lies within delta of eps, or when the last kept
// block's energy and the next one's in greedy order differ by less than delta.
#pragma once
#include <cstdint>

namespace calibatt {

constexpr int kFixBits = 50;
constexpr int kSelectScratchBytes = 128;  // per selecting warp: the compacted candidates

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

// floor(e * 2^50) for the bit pattern b of an energy e in [0, 4], exact:
// scaling by a power of two is exact in fp32 (no overflow below 2^52, no
// underflow), and truncating a non-negative float to an integer is its floor.
// (Opaque to the compiler, so that it recomputes the two instructions where
// needed instead of keeping 64-bit values of every block alive across passes.)
__device__ __forceinline__ long long energy_fixed(uint32_t b) {
  long long r;
  asm volatile("{\n\t.reg .f32 t;\n\tmul.f32 t, %1, 0f58800000;\n\tcvt.rzi.s64.f32 %0, t;\n\t}"
               : "=l"(r)
               : "f"(__uint_as_float(b)));
  return r;
}

__device__ __forceinline__ long long warp_sum64(long long v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ float warp_sumf(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Inclusive suffix sum over lanes: lane l gets sum_{l' >= l} v.
__device__ __forceinline__ float warp_suffixf(float v, int lane) {
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const float t = __shfl_down_sync(0xffffffffu, v, o);
    if (lane + o < 32) v += t;
  }
  return v;
}

// |a - b| < w for exact fixed-point values.
__device__ __forceinline__ bool fx_close(long long a, long long b, long long w) {
  const long long d = a > b ? a - b : b - a;
  return d < w;
}


// Exact cut by binary search over bit patterns (the fallback): the largest
// b in [0, hi] with S(b) >= eps_fx, and the sum of fx over blocks above it.
template <int PER>
__device__ __forceinline__ uint32_t exact_cut_search(const uint32_t (&bits)[PER], uint32_t hi, long long eps_fx,
                                                  long long& above) {
  uint32_t lo = 0;
  while (lo < hi) {
    const uint32_t mid = lo + (hi - lo + 1) / 2;
    long long sm = 0;
#pragma unroll
    for (int i = 0; i < PER; ++i) sm += bits[i] >= mid ? energy_fixed(bits[i]) : 0;
    sm = warp_sum64(sm);
    if (sm >= eps_fx)
      lo = mid;
    else
      hi = mid - 1;
  }
  long long a = 0;
#pragma unroll
  for (int i = 0; i < PER; ++i) a += bits[i] > lo ? energy_fixed(bits[i]) : 0;
  above = warp_sum64(a);
  return lo;
}

// Column c = lane + 32 i of the row is element i of the lane's arrays.
// E: the row (shared or global memory, nb <= 32 * PER); scratch: 128 bytes
// of shared memory for this warp, 16-byte aligned; tie_fx: the
// tie window in fixed point (used only when out.tie is set). Every lane of
// the warp must call.
template <int PER>
__device__ __forceinline__ void warp_select(const float* E, int nb, long long eps_fx, long long tie_fx,
                                            float* scratch, SelectOut out) {
  const int lane = threadIdx.x & 31;
  const unsigned lt_mask = (1u << lane) - 1u;
  const double eps_d = static_cast<double>(eps_fx) * 0x1p-50;
  const float eps32 = static_cast<float>(eps_d);
  // pass 1: load, clamp, totals
  uint32_t bits[PER];
  float tot32 = 0.f;
  int nz = 0;
  uint32_t my_top = 0;
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    const int c = lane + 32 * i;
    const float e = c < nb ? clamp_energy(E[c]) : 0.f;
    bits[i] = __float_as_uint(e);
    tot32 += e;
    nz += e > 0.f;
    my_top = bits[i] > my_top ? bits[i] : my_top;
  }
  tot32 = warp_sumf(tot32);
  nz = static_cast<int>(__reduce_add_sync(0xffffffffu, static_cast<unsigned>(nz)));
  const uint32_t top_bits = __reduce_max_sync(0xffffffffu, my_top);

  // the exact total, only when the fp32 one is near eps (its error is below
  // 24 roundings of 2^-24 relative, far inside this margin)
  long long tot = -1;
  auto exact_total = [&]() {
    long long t = 0;
#pragma unroll
    for (int i = 0; i < PER; ++i) t += energy_fixed(bits[i]);
    return warp_sum64(t);
  };
  if (fabs(static_cast<double>(tot32) - eps_d) <= 1e-5 * eps_d + nb * 0x1p-49) tot = exact_total();
  // 0 = the single top block, 1 = every nonzero block, 2 = greedy cut at tau
  int mode = 2;
  if (eps_fx <= 0 || nz == 0) mode = 0;
  else if (tot >= 0 ? tot < eps_fx : static_cast<double>(tot32) < eps_d) mode = 1;

  uint32_t tau = 0;
  long long above = 0;  // sum of fx over blocks with energy > tau
  int eq_count = -1;    // blocks with energy == tau, when the finish knows it
  if (mode == 2) {
    // prefix range [plo, phi] of tau's bit pattern, narrowed digit by digit
    // (bits 30..20, then 19..10, then 9..0) by binary search with fp32 sums,
    // until at most 32 blocks remain in it
    uint32_t plo = 0, phi = 0x7FFFFFFFu;
    int m = nz;  // blocks in the range (zero energies never matter)
    for (int shift = 20; m > 32 && shift >= 0; shift -= 10) {
      // the digit of tau at `shift`: the largest d with S32(start of d) >= eps
      const uint32_t d0 = plo >> shift;
      const uint32_t top = phi < top_bits ? phi : top_bits;
      uint32_t dlo = 0, dhi = (top >> shift) - d0;
      while (dlo < dhi) {
        const uint32_t mid = dlo + (dhi - dlo + 1) / 2;
        const uint32_t thr = (d0 + mid) << shift;
        float sm = 0.f;
#pragma unroll
        for (int i = 0; i < PER; ++i) sm += bits[i] >= thr ? __uint_as_float(bits[i]) : 0.f;
        sm = warp_sumf(sm);
        if (sm >= eps32)
          dlo = mid;
        else
          dhi = mid - 1;
      }
      const uint32_t nlo = (d0 + dlo) << shift;
      const uint32_t nhi = nlo | ((1u << shift) - 1u);
      plo = nlo > plo ? nlo : plo;
      phi = nhi < phi ? nhi : phi;
      int mm = 0;
#pragma unroll
      for (int i = 0; i < PER; ++i) mm += bits[i] != 0 && bits[i] >= plo && bits[i] <= phi;
      m = static_cast<int>(__reduce_add_sync(0xffffffffu, static_cast<unsigned>(mm)));
    }
    // exact finish over the final range: the blocks above it, and its
    // candidates (compacted, one per lane when at most 32)
    long long base = 0;
    int m_mine = 0;
#pragma unroll
    for (int i = 0; i < PER; ++i) {
      if (bits[i] > phi) base += energy_fixed(bits[i]);
      m_mine += bits[i] != 0 && bits[i] >= plo && bits[i] <= phi;
    }
    base = warp_sum64(base);
    int off = m_mine;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int t = __shfl_up_sync(0xffffffffu, off, o);
      if (lane >= o) off += t;
    }
    m = __shfl_sync(0xffffffffu, off, 31);
    off -= m_mine;
    bool exact = false;
    if (m <= 32) {
      uint32_t* cand = reinterpret_cast<uint32_t*>(scratch);
#pragma unroll
      for (int i = 0; i < PER; ++i)
        if (bits[i] != 0 && bits[i] >= plo && bits[i] <= phi) cand[off++] = bits[i];
      __syncwarp();
      const uint32_t cb = lane < m ? cand[lane] : 0u;
      const long long cf = energy_fixed(cb);
      long long T = 0;  // sum of fx over candidates >= cb
      for (int jj = 0; jj < m; ++jj) {
        const uint32_t bj = __shfl_sync(0xffffffffu, cb, jj);
        const long long fj = __shfl_sync(0xffffffffu, cf, jj);
        T += bj >= cb ? fj : 0;
      }
      const long long all_c = warp_sum64(cf);
      __syncwarp();
      // the range brackets the cut exactly: base < eps <= base + candidates
      if (base < eps_fx && base + all_c >= eps_fx) {
        exact = true;
        const bool ok = lane < m && base + T >= eps_fx;
        tau = __reduce_max_sync(0xffffffffu, ok ? cb : 0u);
        above = base + warp_sum64(lane < m && cb > tau ? cf : 0);
        eq_count = __popc(__ballot_sync(0xffffffffu, lane < m && cb == tau));  // tau's blocks are all candidates
      }
    } else if (plo == phi) {
      // more than 32 blocks with one energy: all candidates are equal
      const long long f = energy_fixed(plo);
      if (base < eps_fx && base + f * m >= eps_fx) {
        exact = true;
        tau = plo;
        above = base;
        eq_count = m;
      }
    }
    if (!exact) tau = exact_cut_search<PER>(bits, top_bits, eps_fx, above);
  }

  // greedy order's first block (modes 0): the largest energy, lowest column
  int top_col = 0;
  if (mode == 0) {
    int my_col = 0x7FFFFFFF;
#pragma unroll
    for (int i = 0; i < PER; ++i) {
      const int c = lane + 32 * i;
      if (c < nb && bits[i] == top_bits && c < my_col) my_col = c;
    }
    top_col = static_cast<int>(__reduce_min_sync(0xffffffffu, static_cast<unsigned>(my_col)));
  }

  // the keep decision, with each block's rank among the blocks equal to tau
  // in column order; the largest energy below tau on the way (tie report)
  const long long ft = mode == 2 ? energy_fixed(tau) : 0;
  long long r_need = 0;
  if (mode == 2) {
    const long long rem = eps_fx - above;  // > 0 and < 2^63, as is ft
    r_need = ft > 0 ? static_cast<long long>(ceil(static_cast<double>(rem) / static_cast<double>(ft))) : 1;
    // the double quotient may be off by one: settle it in integers
    while (r_need > 1 && (r_need - 1) * ft >= rem) --r_need;
    while (r_need * ft < rem) ++r_need;
  }
  // every block equal to tau is kept when the cut needs all of them (the
  // common case: one such block): no ranks among them are needed
  const bool all_eq = mode == 2 && eq_count >= 0 && eq_count <= r_need;
  int before = all_eq ? eq_count : 0;  // equal blocks in earlier columns (after the loop: all of them)
  int kept_mine = 0;
  uint32_t nxt = 0;  // largest energy below tau, plus one (0: none)
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    const int c = lane + 32 * i;
    const bool in = c < nb;
    bool k;
    if (all_eq) {
      k = in && bits[i] >= tau;
    } else {
      const bool eq = mode == 2 && in && bits[i] == tau;
      const unsigned bal = __ballot_sync(0xffffffffu, eq);
      if (mode == 0) k = in && c == top_col;
      else if (mode == 1) k = in && bits[i] > 0;
      else k = in && (bits[i] > tau || (eq && before + __popc(bal & lt_mask) < r_need));
      before += __popc(bal);
    }
    kept_mine += k;
    if (in && bits[i] < tau && bits[i] + 1 > nxt) nxt = bits[i] + 1;
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
        nxt = __reduce_max_sync(0xffffffffu, nxt);
        if (nxt > 0) e_next = energy_fixed(nxt - 1);
      }
    } else if (mode == 1) {
      if (tot < 0) tot = exact_total();
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
