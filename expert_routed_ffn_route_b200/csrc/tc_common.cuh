// Building blocks shared by the tensor-core grouped GEMMs (tcgen05 + TMEM, TMA-fed): PTX
// wrappers for tensor memory, tiled TMA loads, MMA commits and shared-memory descriptors;
// the unit schedule over (expert slot, weight tile, token tile); the host-side tensor-map
// encoder.
#pragma once

#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "pipeline.cuh"

namespace moe {

constexpr int kTcM = 128;      // weight rows per tile (the MMA's M)
constexpr int kTcNMax = 64;    // token rows per tile
constexpr int kBoxes = 3;      // activation boxes of 16, 32, 64 rows

// ------------------------------------------------------------------ PTX wrappers

__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int c0, int c1,
                                            uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_u32(dst_smem)),
               "r"(ncols)
               : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// Commit of the warp's issued tensor-core operations to an mbarrier (one elected lane).
__device__ __forceinline__ void umma_commit_warp(uint64_t* bar) {
  asm volatile(
      "{\n\t.reg .pred e;\n\telect.sync _|e, 0xffffffff;\n\t"
      "@e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n\t}" ::"r"(
          smem_u32(bar))
      : "memory");
}

// 16 consecutive fp32 columns of this thread's TMEM lane.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16]) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,"
      "%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

// UMMA shared-memory descriptor, K-major, 128-byte swizzle: rows of 128 bytes, groups of
// 8 rows 1024 bytes apart (SBO), version 1 (sm_100), layout type 2 (128B swizzle).
__device__ __forceinline__ uint64_t umma_desc_sw128(uint32_t saddr) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFF);
  d |= (uint64_t)1 << 16;                 // LBO (unused for swizzled K-major)
  d |= (uint64_t)(1024 >> 4) << 32;       // SBO
  d |= (uint64_t)1 << 46;                 // version
  d |= (uint64_t)2 << 61;                 // SWIZZLE_128B
  return d;
}

// ------------------------------------------------------------------ schedule

struct TcUnit {
  int slot, e, shared, row0, nrows, ntile, mtile;
};

// S points at the CTA's shared-memory copy of the schedule.
__device__ __forceinline__ TcUnit tc_unit(const TcSched& S, int n_slots, int n_tiles, int u) {
  int lo = 0, hi = n_slots;  // largest s with mt_prefix[s] * n_tiles <= u
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (S.mt_prefix[mid] * n_tiles <= u) lo = mid;
    else hi = mid;
  }
  TcUnit t;
  t.slot = lo;
  const int local = u - S.mt_prefix[lo] * n_tiles;
  const int mts = (S.slot_rows[lo] + kTcNMax - 1) / kTcNMax;
  t.ntile = local / mts;
  t.mtile = local % mts;
  t.e = S.slot_expert[lo];
  t.shared = (t.e < 0);
  if (t.shared) t.e = 0;
  t.row0 = S.slot_row0[lo] + t.mtile * kTcNMax;
  t.nrows = min(kTcNMax, S.slot_rows[lo] - t.mtile * kTcNMax);
  return t;
}

__device__ __forceinline__ int box_index(int nrows) {
  return nrows <= 16 ? 0 : (nrows <= 32 ? 1 : (nrows <= 64 ? 2 : 3));
}

// ------------------------------------------------------------------ host side

inline PFN_cuTensorMapEncodeTiled_v12000 get_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    cudaDriverEntryPointQueryResult q;
    void* ptr = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  });
  return fn;
}

// 2-D map over a row-major [rows][cols] array.
inline bool make_map(CUtensorMap* m, CUtensorMapDataType dt, int esize, const void* base,
                     uint64_t cols, uint64_t rows, uint32_t box_cols, uint32_t box_rows, CUtensorMapSwizzle sw) {
  auto enc = get_encoder();
  if (!enc || !base) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * esize};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return enc(m, dt, 2, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace moe
