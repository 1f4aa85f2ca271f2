// Greedy eps selection of one block-row, run cooperatively by T threads of a
// CTA (explainer §三, step 3: keep the fewest key blocks whose cumulative
// energy reaches eps; greedy order: energy descending, equal energies by lower
// column first).
//
// No sort is needed. With every energy taken exactly in fixed point (50
// fraction bits, truncated), the greedy cut is determined by the energy tau
// of the block at which the running sum first reaches eps:
//   tau = the largest energy v with  S(v) = sum_{E >= v} fx(E) >= eps_fx.
// S is non-increasing in v and the float bit patterns of non-negative
// energies order like their values, so tau is found by a binary search over
// bit patterns, each step one exact integer sum over the row. The kept set is
// every block with E > tau plus the first r blocks (in column order) with
// E == tau, r the fewest that reach eps. Because the sums are exact integers,
// the result equals a sequential greedy sum in sorted order.
#pragma once
#include <cstdint>

namespace calibatt {

constexpr int kFixBits = 50;

struct SelectOut {
  uint8_t* mask;     // [nb] or NULL
  int32_t* kept;     // [1] or NULL
  uint16_t* counts;  // [nb] or NULL (counts += mask, saturating)
};

__device__ __forceinline__ float clamp_energy(float e) {
  if (!(e > 0.f)) return 0.f;  // NaN, negative and zero
  return e > 4.f ? 4.f : e;
}

// floor(e * 2^50) for e in [0, 4], exact.
__device__ __forceinline__ long long energy_fixed(float e) {
  const uint32_t b = __float_as_uint(e);
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

__device__ __forceinline__ void group_sync(int bar_id, int T) {
  if (T == 32)
    __syncwarp();
  else
    asm volatile("bar.sync %0, %1;" ::"r"(bar_id), "r"(T) : "memory");
}

// Per-warp partials for reductions over T > 32 threads.
struct SelectScratch {
  long long wsum[32];
  int wcnt[32];
};

// Sum of a per-thread int64 and int over the T threads (T multiple of 32).
__device__ __forceinline__ void group_sum(long long& v, int& c, SelectScratch* sc, int tid, int T, int bar_id) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    v += __shfl_xor_sync(0xffffffffu, v, o);
    c += __shfl_xor_sync(0xffffffffu, c, o);
  }
  if (T == 32) return;
  if ((tid & 31) == 0) {
    sc->wsum[tid >> 5] = v;
    sc->wcnt[tid >> 5] = c;
  }
  group_sync(bar_id, T);
  v = 0;
  c = 0;
  for (int w = 0; w < (T >> 5); ++w) {
    v += sc->wsum[w];
    c += sc->wcnt[w];
  }
  group_sync(bar_id, T);
}

// Sum of a per-thread int64 over the T threads (T multiple of 32).
__device__ __forceinline__ long long group_sum64(long long v, SelectScratch* sc, int tid, int T, int bar_id) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  if (T == 32) return v;
  if ((tid & 31) == 0) sc->wsum[tid >> 5] = v;
  group_sync(bar_id, T);
  v = 0;
  for (int w = 0; w < (T >> 5); ++w) v += sc->wsum[w];
  group_sync(bar_id, T);
  return v;
}

// Max of a per-thread key over the T threads.
__device__ __forceinline__ unsigned long long group_max(unsigned long long v, SelectScratch* sc, int tid, int T,
                                                        int bar_id) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const unsigned long long u = __shfl_xor_sync(0xffffffffu, v, o);
    v = u > v ? u : v;
  }
  if (T == 32) return v;
  if ((tid & 31) == 0) sc->wsum[tid >> 5] = static_cast<long long>(v);
  group_sync(bar_id, T);
  v = 0;
  for (int w = 0; w < (T >> 5); ++w) {
    const unsigned long long u = static_cast<unsigned long long>(sc->wsum[w]);
    v = u > v ? u : v;
  }
  group_sync(bar_id, T);
  return v;
}

// E: [nb] energies (shared or global memory); aux: shared scratch of
// sizeof(SelectScratch) (unused when T == 32). Every one of the T threads (T a multiple of 32,
// nb <= PER * T) must call this. Thread tid owns columns tid*per .. +per-1.
template <int PER>
__device__ __forceinline__ void select_row(const float* E, int nb, long long eps_fx, uint8_t* aux, int tid, int T,
                                           int bar_id, SelectOut out) {
  SelectScratch* sc = reinterpret_cast<SelectScratch*>(aux);
  const int per = (nb + T - 1) / T;
  const int c0 = tid * per;
  uint32_t bits[PER];
  long long fx[PER];
  long long tot = 0;
  int nz = 0;
  // top block key (bits, inverted column): the largest energy, lowest column
  unsigned long long top = 0;
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    const int c = c0 + i;
    const bool in = i < per && c < nb;
    const float e = in ? clamp_energy(E[c]) : 0.f;
    bits[i] = __float_as_uint(e);
    fx[i] = energy_fixed(e);
    tot += fx[i];
    nz += e > 0.f;
    if (in) {
      const unsigned long long key = (static_cast<unsigned long long>(bits[i]) << 32) | (0xFFFFFFFFu - c);
      top = key > top ? key : top;
    }
  }
  top = group_max(top, sc, tid, T, bar_id);
  group_sum(tot, nz, sc, tid, T, bar_id);
  const int top_col = static_cast<int>(0xFFFFFFFFu - static_cast<uint32_t>(top));
  const uint32_t top_bits = static_cast<uint32_t>(top >> 32);

  // 0 = the single top block, 1 = every nonzero block, 2 = greedy cut at tau
  int mode = 2;
  if (eps_fx <= 0 || nz == 0) mode = 0;
  else if (tot < eps_fx) mode = 1;

  uint32_t tau = 0;
  long long above = 0;  // sum of fx over blocks with energy > tau
  if (mode == 2) {
    // largest b in [0, top_bits] with S(b) >= eps (S(0) = tot >= eps)
    uint32_t lo = 0, hi = top_bits;
    while (lo < hi) {
      const uint32_t mid = lo + (hi - lo + 1) / 2;
      long long s0 = 0, s1 = 0;  // two chains: half the add latency
#pragma unroll
      for (int i = 0; i < PER; i += 2) {
        s0 += bits[i] >= mid ? fx[i] : 0;
        if (i + 1 < PER) s1 += bits[i + 1] >= mid ? fx[i + 1] : 0;
      }
      const long long sm = group_sum64(s0 + s1, sc, tid, T, bar_id);
      if (sm >= eps_fx)
        lo = mid;
      else
        hi = mid - 1;
    }
    tau = lo;
#pragma unroll
    for (int i = 0; i < PER; ++i) above += bits[i] > tau ? fx[i] : 0;
    above = group_sum64(above, sc, tid, T, bar_id);
  }

  // rank of each block among the blocks equal to tau, in column order
  int n_eq = 0;
  if (mode == 2) {
#pragma unroll
    for (int i = 0; i < PER; ++i) n_eq += (i < per && c0 + i < nb && bits[i] == tau);
  }
  const int lane = tid & 31, w = tid >> 5;
  int incl = n_eq;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  int rank = incl - n_eq;
  if (T > 32) {
    if (lane == 31) sc->wcnt[w] = incl;
    group_sync(bar_id, T);
    for (int ww = 0; ww < w; ++ww) rank += sc->wcnt[ww];
    group_sync(bar_id, T);  // every rank read before the partials are reused
  }
  long long r_need = 0;
  if (mode == 2) {
    const long long ft = energy_fixed(__uint_as_float(tau));
    r_need = ft > 0 ? (eps_fx - above + ft - 1) / ft : 1;
  }
  int kept_mine = 0;
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    const int c = c0 + i;
    if (i >= per || c >= nb) continue;
    bool k;
    if (mode == 0) {
      k = (c == top_col);
    } else if (mode == 1) {
      k = bits[i] > 0;
    } else if (bits[i] > tau) {
      k = true;
    } else if (bits[i] == tau) {
      k = rank < r_need;
      ++rank;
    } else {
      k = false;
    }
    kept_mine += k;
    if (out.mask) out.mask[c] = k ? 1 : 0;
    if (out.counts && k) {
      const uint16_t old = out.counts[c];
      if (old != 0xFFFFu) out.counts[c] = old + 1;
    }
  }
  if (out.kept) {
    long long dummy = 0;
    group_sum(dummy, kept_mine, sc, tid, T, bar_id);
    if (tid == 0) *out.kept = kept_mine;
  }
  (void)top_bits;
}

}  // namespace calibatt
