// Pieces shared by the tensor-core kernels: work units of the skip-list tile
// scheduler, tile-sequence cursors, shared-memory MMA descriptors, tensor-map
// construction and launch helpers.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "calibatt.h"
#include "kernels.h"
#include "ptx.cuh"

namespace calibatt {

constexpr int kTile = 32768;  // one 128 x 128 bf16 tile
constexpr int kHalf = 16384;  // one 64-column half (one TMA box)
constexpr float kLn2 = 0.6931471805599453f;

enum Mode : int { kAttn = 0, kLse = 1, kEnergy = 2, kEnergy1 = 3 };

// ------------------------------------------------------------------ work units
struct Unit {
  int hq;      // head index in the Q tensor (second segment: in the anchor tensor)
  int hkv;     // head index in K / V / O
  int r;       // query block
  int nnz;     // kept key blocks
  int base;    // offset into col_idx
  bool write;  // false: malformed work-list entry, produce nothing
  bool rep;    // second segment: anchor queries of a repeated head
};

// Static longest-first schedule: the work list is sorted by kept blocks,
// descending; worker g of G takes entries g, 2G-1-g, 2G+g, ... (snake order).
__device__ __forceinline__ int unit_index(int g, int G, int round) {
  return round * G + ((round & 1) ? (G - 1 - g) : g);
}

__device__ __forceinline__ bool load_unit(const KernelParams& p, int idx, Unit& u) {
  if (idx >= p.n_units) return false;
  int code = p.work_list ? __ldg(p.work_list + idx) : idx;
  const int n_a = p.heads_q * p.nbq;
  u.write = true;
  u.rep = false;
  if (code >= n_a && p.nbq_b > 0 && code - n_a < p.heads_q_b * p.nbq_b) {
    // anchor-query unit: K/V/O head from head_map_b; every key block, or the
    // blocks of its own skip list
    const int c = code - n_a;
    u.rep = true;
    u.hq = c / p.nbq_b;
    u.r = c % p.nbq_b;
    u.hkv = __ldg(p.head_map_b + u.hq);
    if (u.hkv < 0 || u.hkv >= p.heads_kv) {
      record_error(p.status, CALIBATT_ERR_ARG);
      u.write = false;
      u.hkv = 0;
    }
    u.base = 0;
    u.nnz = u.write ? p.nbk : 0;
    if (u.write && p.row_ptr_b) {
      const int a = __ldg(p.row_ptr_b + c), b = __ldg(p.row_ptr_b + c + 1);
      if (a < 0 || b < a || static_cast<int64_t>(b) > p.nnz_b) {
        record_error(p.status, CALIBATT_ERR_CSR);
        u.nnz = 0;
      } else {
        u.base = a;
        u.nnz = b - a;
      }
    }
    return true;
  }
  if (code < 0 || code >= n_a) {
    record_error(p.status, CALIBATT_ERR_CSR);
    u.write = false;
    code = 0;
  }
  const int nbq = p.nbq > 0 ? p.nbq : 1;
  u.hq = code / nbq;
  u.r = code % nbq;
  u.hkv = p.head_map ? __ldg(p.head_map + u.hq) : u.hq;
  if (u.hkv < 0 || u.hkv >= p.heads_kv) {
    record_error(p.status, CALIBATT_ERR_ARG);
    u.write = false;
    u.hkv = 0;
  }
  if (!u.write) {
    u.base = 0;
    u.nnz = 0;
  } else if (p.row_ptr) {
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
  return true;
}

// Key block of the j-th kept tile; out-of-range entries are clamped and reported.
__device__ __forceinline__ int block_col(const KernelParams& p, const Unit& u, int j) {
  const int32_t* ci = u.rep ? p.col_idx_b : p.col_idx;
  if (!ci) return j;
  int c = __ldg(ci + u.base + j);
  if (c < 0 || c >= p.nbk) {
    record_error(p.status, CALIBATT_ERR_CSR);
    c = c < 0 ? 0 : p.nbk - 1;
  }
  return c;
}

// Cursor over one worker's (unit, kept block) sequence, skipping units with
// no kept block. The producer and the MMA issuer walk identical sequences.
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
// Q and K tiles are K-major (head dim contiguous) in two 64-column halves with
// the 128-byte swizzle TMA writes: 8-row groups 1 KB apart (SBO); a K step of
// 16 elements moves 32 bytes inside a half, the second half is 16 KB on.
// V as the B operand of P V is MN-major (head dim = N contiguous): the two
// 64-column halves are the MN atoms (LBO = 16 KB), 8-key groups are 1 KB apart.
// Descriptor arithmetic: the start address sits in the low 14 bits (>> 4), so
// a byte offset d inside shared memory is added as d >> 4.
__device__ __forceinline__ uint64_t desc_k_base(uint32_t saddr) { return smem_desc_sw128(saddr, 16, 1024); }
__device__ __forceinline__ uint64_t desc_v_base(uint32_t saddr) { return smem_desc_sw128(saddr, kHalf, 1024); }
__device__ __forceinline__ uint32_t desc_k_step(int ks) { return (ks >> 2) * (kHalf >> 4) + (ks & 3) * 2; }
__device__ __forceinline__ uint32_t desc_v_step(int ks) { return ks * (2048 >> 4); }

constexpr uint32_t kIdescS = idesc_bf16_f32(128, 128, false);
constexpr uint32_t kIdescPV = idesc_bf16_f32(128, 128, true);

__device__ __forceinline__ void store_row_chunk(__nv_bfloat16* dst, const uint32_t (&packed)[16]) {
  uint4* d = reinterpret_cast<uint4*>(dst);
#pragma unroll
  for (int i = 0; i < 4; ++i) d[i] = make_uint4(packed[4 * i], packed[4 * i + 1], packed[4 * i + 2], packed[4 * i + 3]);
}

// ------------------------------------------------------------------ host helpers
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

inline EncodeTiledFn get_encode() {
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
inline int make_map(CUtensorMap* map, const void* base, int rows, int heads) {
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

inline int sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) return 148;
  return n;
}

// One-time setup of a kernel per device. cudaFuncSetAttribute acts on the
// current device, so a process that launches on several GPUs, or from several
// host threads, needs it once for each device; the flags are per device and
// read under a lock.
struct PerDeviceOnce {
  std::mutex mu;
  bool done[64] = {};
};

inline int set_max_smem_once(const void* fn, int bytes, PerDeviceOnce& once) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return CALIBATT_ERR_CUDA;
  std::lock_guard<std::mutex> lock(once.mu);
  if (!once.done[dev]) {
    if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) != cudaSuccess)
      return CALIBATT_ERR_CUDA;
    once.done[dev] = true;
  }
  return CALIBATT_OK;
}

// Energy-pass launcher (score.cu) and the grid it uses for n_units work units
// (one CTA of two slots per SM at most).
int launch_score(int mode, const CUtensorMap& mq, const CUtensorMap& mk, const KernelParams& p, cudaStream_t stream);
inline int score_grid(int n_units) {
  const int sms = sm_count();
  const int grid = (n_units + 1) / 2;
  return grid > sms ? sms : grid;
}

}  // namespace calibatt
