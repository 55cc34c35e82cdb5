// Shared device helpers and internal launch interfaces of the MoE FFN library.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include <algorithm>

#include "../../include/moe_b200.h"

namespace moe {

// Status word kept at the start of the workspace (device side).
enum : int32_t { DEV_OK = 0, DEV_TIMEOUT = 1, DEV_BOUNDS = 2, DEV_RANGE = 3 };

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

// Word 2 of the status block (byte 8 of the synchronisation block) keeps the site of the
// first bounded wait that gave up (kernel and wait, numbered in include/moe_b200.h).
constexpr int kSiteWord = 2;

// A bounded wait at `site` gave up: DEV_TIMEOUT in the status word, the site beside it (the
// first failure of a call wins both words).
__device__ __forceinline__ void set_timeout(int32_t* status, int32_t site) {
  if (!status) return;
  atomicCAS(status, DEV_OK, DEV_TIMEOUT);
  atomicCAS(status + kSiteWord, 0, site);
}

// ------------------------------------------------------------------ stable top-k

// Order-preserving map of a finite float to uint32 (larger float -> larger key); -0 and
// +0 map to the same key, so they tie like equal values do. key_value inverts it.
__device__ __forceinline__ uint32_t order_key(float v) {
  const uint32_t b = __float_as_uint(v + 0.0f);  // -0 + 0 = +0
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}
__device__ __forceinline__ float key_value(uint32_t key) {
  return __uint_as_float((key & 0x80000000u) ? (key & 0x7fffffffu) : ~key);
}

// Warp-cooperative stable top-k of one row of E <= 32 * PER keys (order_key values): the k
// largest, ties to the lower index, in rank order. Lane j < k ends with the j-th pick's index
// in *idx and its key in *key. Lane l holds keys l, l + 32, ... in registers. Each round is
// two warp reductions (the best key, then the lowest index holding it); only the lane that
// owned the pick rescans its PER registers (no memory traffic inside the rounds).
template <int PER>
__device__ __forceinline__ void warp_topk_regs(const float* row, int E, int k, int lane, int* idx,
                                               uint32_t* key) {
  uint32_t kv[PER];
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    const int e = lane + 32 * i;
    kv[i] = (e < E) ? order_key(__ldcg(row + e)) : 0u;  // 0: absent or taken
  }
  uint32_t bk = 0;
  int bi = 0;
#pragma unroll
  for (int i = 0; i < PER; ++i)
    if (kv[i] > bk) {  // strict: the lowest index wins among this lane's equal keys
      bk = kv[i];
      bi = i;
    }
  *idx = 0;
  *key = 0;
  for (int j = 0; j < k; ++j) {
    const uint32_t m = __reduce_max_sync(0xffffffffu, bk);
    const uint32_t mine = (bk == m && m != 0) ? (uint32_t)(lane + 32 * bi) : 0xffffffffu;
    const uint32_t win = __reduce_min_sync(0xffffffffu, mine);
    if (lane == j) {
      *idx = (int)win;
      *key = m;
    }
    if (mine == win) {  // the owner retires its pick and finds its next best
#pragma unroll
      for (int i = 0; i < PER; ++i)
        if (i == bi) kv[i] = 0;
      bk = 0;
      bi = 0;
#pragma unroll
      for (int i = 0; i < PER; ++i)
        if (kv[i] > bk) {
          bk = kv[i];
          bi = i;
        }
    }
  }
}

// Dispatch on the keys a lane holds (E <= 1024).
__device__ __forceinline__ void warp_topk(const float* row, int E, int k, int lane, int* idx,
                                          uint32_t* key) {
  if (E <= 256) warp_topk_regs<8>(row, E, k, lane, idx, key);
  else if (E <= 512) warp_topk_regs<16>(row, E, k, lane, idx, key);
  else warp_topk_regs<32>(row, E, k, lane, idx, key);
}

// Gates of the k picks held by lanes 0..k-1: softmax of their logits, summed in rank order.
__device__ __forceinline__ float warp_topk_gate(uint32_t my_key, uint32_t top_key, int k,
                                                int lane) {
  const float z = (lane < k) ? expf(key_value(my_key) - key_value(top_key)) : 0.f;
  float total = 0.f;
#pragma unroll 1
  for (int j = 0; j < k; ++j) total += __shfl_sync(0xffffffffu, z, j);
  return z / total;
}

// ------------------------------------------------------------------ launch plumbing

// Everything a kernel needs about one call, resolved on the host.
struct Bank {
  int fmt;            // 16, 8, 4, MOE_W_NVFP4
  const void* w[3];   // gate, up, down
  const uint16_t* s[3];  // group scales (NVFP4: the packed E4M3 block scales, as bytes)
  const float* g[3];     // NVFP4 tensor scales [n_exp] per matrix
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
  int32_t* ticket;     // [2]: the fused routing kernel's grid-barrier word and its ranking
                       // counter (zero between calls)
  int32_t* tile_cnt;   // [d / 16] per-output-tile arrival counters, zero between calls
  const int32_t* test_ctl;  // failure injection: [0] hold word, [1] wait budget (cycles)
  uint32_t* gbar;      // grid-barrier word of the single-kernel 1-token layer
  uint16_t* xg;        // tensor-core path: fp16 x rows in grouped order, then the shared
                       // expert's rows [(T*k + T)][d]
  int32_t* tc_sched;   // tensor-core path: per-slot schedule (TcSched view)
  // NVFP4 routed experts: the activations quantised per grouped row (E2M1 codes, packed
  // block scales by token tile, fp32 row scales), and h in fp32 before its quantisation
  uint8_t* xq;         // [T*k][d/2]
  uint8_t* xsf;        // [token tiles][d/64][512]
  float* gx;           // [T*k]
  float* h32;          // [T*k][f]
  uint8_t* hq;         // [T*k][f/2]
  uint8_t* hsf;        // [token tiles][f/64][512]
  float* gh;           // [T*k]
  int path;            // moe_path
};

// Per slot (active routed experts in ascending order, then the shared expert): rows, first
// row, expert id (-1: shared) and the running count of token tiles (m-tiles of kTcNMax
// rows), written by tc_prep_kernel. A GEMM with n_tiles weight tiles per expert has units
// [mt_prefix[s] * n_tiles, mt_prefix[s + 1] * n_tiles) in slot s. expert_mt[e] is the
// mt_prefix of routed expert e's slot (defined for experts with rows).
struct TcSched {
  int32_t* slot_rows;    // [E + 2]
  int32_t* slot_row0;    // [E + 2]
  int32_t* slot_expert;  // [E + 2]
  int32_t* mt_prefix;    // [E + 2]; mt_prefix[n_slots] = total m-tiles
  int32_t* expert_mt;    // [E + 2]
};

// The synchronisation block at the start of the workspace: status word (offset 0), the site
// of the first expired wait (8), routing tickets (16, 20), the single-kernel layer's grid-barrier word (32), the failure-injection
// words (64: hold, 68: wait budget; zero in normal use), then one arrival counter per 16-row
// output tile (256).
constexpr size_t kSyncStatus = 0, kSyncTicket = 16, kSyncGbar = 32, kSyncTest = 64,
                 kSyncTiles = 256;
inline size_t sync_bytes(int d) { return 256 + (size_t)4 * (d / 16); }

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
cudaError_t launch_combine(const Plan& p, void* out, cudaStream_t st, bool pdl);
// TMA-pipelined grouped GEMV (int4 weights, scales 16-byte aligned)
bool tma_gemv_supported(const Plan& p);
cudaError_t launch_tma_gate_up(const Plan& p, cudaStream_t st, bool pdl);
cudaError_t launch_tma_down(const Plan& p, cudaStream_t st, bool pdl);
// tcgen05 grouped GEMMs (tc_grouped.cu)
bool tc_supported(const Plan& p);
size_t tc_sched_bytes(int E);
TcSched tc_sched_view(void* base, int E);
cudaError_t launch_tc_prep(const Plan& p, const TcSched& S, uint16_t* xg, cudaStream_t st,
                           bool shared_rows_only = false);
cudaError_t launch_tc_gate_up(const Plan& p, const TcSched& S, const uint16_t* xg,
                              cudaStream_t st);
cudaError_t launch_tc_down(const Plan& p, const TcSched& S, cudaStream_t st);
// the shared expert alone (its bank's format), beside routed experts of another kind
cudaError_t launch_tc_shared_gate_up(const Plan& p, const TcSched& S, const uint16_t* xg,
                                     cudaStream_t st);
cudaError_t launch_tc_shared_down(const Plan& p, const TcSched& S, cudaStream_t st);
// NVFP4 routed experts on the FP4 tensor cores (nvfp4_grouped.cu)
constexpr int kNvfp4 = MOE_W_NVFP4;
size_t nv_tile_cap(int T, int k, int E);  // token tiles a call can have
bool nv_supported(const Plan& p);
cudaError_t launch_nv_quant_x(const Plan& p, const TcSched& S, cudaStream_t st);
cudaError_t launch_nv_gate_up(const Plan& p, const TcSched& S, cudaStream_t st);
cudaError_t launch_nv_quant_h(const Plan& p, const TcSched& S, cudaStream_t st);
cudaError_t launch_nv_down(const Plan& p, const TcSched& S, cudaStream_t st);
cudaError_t launch_nv_quant_rows(const float* v, int rows, int K, uint8_t* codes, uint8_t* scales,
                                 float* g, cudaStream_t st);
cudaError_t launch_nv_pack_scales(const uint8_t* src, uint8_t* dst, int n_mats, int rows, int K,
                                  cudaStream_t st);
// the whole layer of a 1-token call in one persistent kernel (decode_fused.cu)
bool decode_fused_supported(const Plan& p);
cudaError_t launch_decode_fused(const Plan& p, void* out, cudaStream_t st);
// router + top-k + plan in one launch (T <= 32)
bool route_fused_supported(const Plan& p);
cudaError_t launch_route_fused(const Plan& p, int32_t* ticket, cudaStream_t st);

}  // namespace moe
