// Greedy eps selection of one block-row, run cooperatively by T threads of a
// CTA (explainer §三, step 3: keep the fewest key blocks whose cumulative
// energy reaches eps).
//
// Order: energy descending, equal energies by lower column (a 64-bit key
// (~bits(E), col) sorted ascending by a bitonic network in shared memory).
// Running sums are exact: every energy is converted to an integer with 50
// fraction bits (truncated), so the parallel prefix scan gives the same cut as
// a sequential sum in the same order.
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

__device__ __forceinline__ unsigned long long energy_key(float e, int col) {
  return (static_cast<unsigned long long>(0xFFFFFFFFu - __float_as_uint(e)) << 32) | static_cast<uint32_t>(col);
}

__device__ __forceinline__ void group_sync(int bar_id, int T) {
  asm volatile("bar.sync %0, %1;" ::"r"(bar_id), "r"(T) : "memory");
}

// E: shared [nb] energies; aux: shared scratch >= 4 KB; keys: shared [1024].
// Every one of the T threads (T a multiple of 32, <= 1024) must call this.
static __device__ __noinline__ void select_row(const float* E, int nb, long long eps_fx, uint8_t* aux,
                                        unsigned long long* keys, int tid, int T, int bar_id, SelectOut out) {
  uint8_t* keep = aux;                                              // [1024]
  long long* warp_tot = reinterpret_cast<long long*>(aux + 1024);  // [32]
  int* first_hit = reinterpret_cast<int*>(aux + 1024 + 256);
  int* nonzero = first_hit + 1;

  int npow = 2;
  while (npow < nb) npow <<= 1;
  for (int i = tid; i < npow; i += T) keys[i] = (i < nb) ? energy_key(clamp_energy(E[i]), i) : ~0ull;
  for (int i = tid; i < nb; i += T) keep[i] = 0;
  if (tid == 0) {
    *first_hit = 0x7FFFFFFF;
    *nonzero = 0;
  }
  group_sync(bar_id, T);

  // bitonic sort, ascending keys
  for (int k = 2; k <= npow; k <<= 1) {
    for (int j = k >> 1; j > 0; j >>= 1) {
      for (int i = tid; i < npow; i += T) {
        const int ixj = i ^ j;
        if (ixj > i) {
          const unsigned long long a = keys[i], b = keys[ixj];
          const bool up = (i & k) == 0;
          if ((a > b) == up) {
            keys[i] = b;
            keys[ixj] = a;
          }
        }
      }
      group_sync(bar_id, T);
    }
  }

  // exact prefix sums of the sorted energies: contiguous chunk per thread
  const int per = (nb + T - 1) / T;
  const int i0 = tid * per;
  const int i1 = min(nb, i0 + per);
  long long local = 0;
  int nz = 0;
  for (int i = i0; i < i1; ++i) {
    const float e = __uint_as_float(0xFFFFFFFFu - static_cast<uint32_t>(keys[i] >> 32));
    local += energy_fixed(e);
    nz += e > 0.f;
  }
  // exclusive scan of the per-thread totals: shuffles inside a warp, then warps
  const int lane = tid & 31, w = tid >> 5;
  long long incl = local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const long long v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  if (lane == 31) warp_tot[w] = incl;
  if (nz) atomicAdd(nonzero, nz);
  group_sync(bar_id, T);
  long long run = incl - local;
  for (int ww = 0; ww < w; ++ww) run += warp_tot[ww];
  for (int i = i0; i < i1; ++i) {
    const float e = __uint_as_float(0xFFFFFFFFu - static_cast<uint32_t>(keys[i] >> 32));
    run += energy_fixed(e);
    if (run >= eps_fx) {
      atomicMin(first_hit, i + 1);
      break;
    }
  }
  group_sync(bar_id, T);
  int m = *first_hit;
  if (m == 0x7FFFFFFF) m = *nonzero;  // eps not reached: every nonzero-energy block
  if (m < 1) m = 1;
  if (m > nb) m = nb;
  for (int i = tid; i < m; i += T) keep[static_cast<uint32_t>(keys[i])] = 1;
  group_sync(bar_id, T);
  for (int c = tid; c < nb; c += T) {
    const uint8_t kbit = keep[c];
    if (out.mask) out.mask[c] = kbit;
    if (out.counts && kbit) {
      const uint16_t old = out.counts[c];
      if (old != 0xFFFFu) out.counts[c] = old + 1;
    }
  }
  if (tid == 0 && out.kept) *out.kept = m;
  group_sync(bar_id, T);
}

}  // namespace calibatt
