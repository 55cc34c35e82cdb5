// Shared device helpers and internal launch interfaces of the MoE FFN library.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include <algorithm>

#include "../../include/moe_b200.h"

namespace moe {

// Status word kept at the start of the workspace (device side).
enum : int32_t { DEV_OK = 0, DEV_TIMEOUT = 1, DEV_BOUNDS = 2 };

constexpr int kGroup = 128;      // quantisation group along K
constexpr int kMaxE = 1024;      // experts a layer
constexpr int kMaxK = 32;        // routed experts a token

__device__ __forceinline__ float bf16_to_f32(uint16_t b) {
  return __uint_as_float(static_cast<uint32_t>(b) << 16);
}

__device__ __forceinline__ uint16_t f32_to_bf16_rn(float f) {
  __nv_bfloat16 h = __float2bfloat16_rn(f);
  return *reinterpret_cast<uint16_t*>(&h);
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

__device__ __forceinline__ uint4 ld_nc_v4(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

__device__ __forceinline__ void set_status(int32_t* status, int32_t code) {
  if (status) atomicCAS(status, DEV_OK, code);
}

// ------------------------------------------------------------------ launch plumbing

// Everything a kernel needs about one call, resolved on the host.
struct Bank {
  int fmt;            // 16, 8, 4
  const void* w[3];   // gate, up, down
  const uint16_t* s[3];
};

struct Plan {
  // sizes
  int T, d, f, E, k, has_shared;
  // inputs
  const uint16_t* x;
  const uint16_t* router_w;
  const float* router_bias;
  Bank routed, shared;
  // routing results
  int32_t* topk_idx;   // [T*k]
  float* topk_w;       // [T*k]
  float* logits;       // [T*E]
  // plan
  int32_t* offsets;    // [E+1]
  int32_t* perm;       // [T*k]
  int32_t* inv;        // [T*k]
  int32_t* active;     // [E+2]: active[0] = number of active routed experts, then ids
  int32_t* cta_hist;   // [n_chunks * E]
  // intermediates
  uint16_t* h;         // bf16 [(T*k + T) * f]: routed rows, then shared rows
  float* y_assign;     // [T*k*d]
  float* y_shared;     // [T*d]
  int32_t* status;
};

// Permutation chunking (assignments per scatter CTA).
constexpr int kPermChunk = 256;
inline int perm_chunks(int T, int k) { return (T * k + kPermChunk - 1) / kPermChunk; }

// Launchers (each enqueues on `st`, returns cudaGetLastError()).
cudaError_t launch_router(const Plan& p, cudaStream_t st);
cudaError_t launch_topk(const Plan& p, cudaStream_t st);
cudaError_t launch_permute(const Plan& p, cudaStream_t st);
cudaError_t launch_schedule_from_offsets(const Plan& p, cudaStream_t st);
cudaError_t launch_gemv_gate_up(const Plan& p, cudaStream_t st);
cudaError_t launch_gemv_down(const Plan& p, cudaStream_t st);
cudaError_t launch_combine(const Plan& p, void* out, cudaStream_t st);

}  // namespace moe
