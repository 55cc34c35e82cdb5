// Router: fp32 logits X Wr^T (+ b), then a deterministic stable top-k and the gates.
//
// Routing rule (Qwen3.8-Flash-Next-Dual-GPU README, "Independent decode lane": the
// 512-expert router uses a deterministic stable top-k): experts ordered by logit, largest
// first, ties to the lower expert index. Gates are the softmax over the k selected logits
// (equal to the softmax over all experts renormalised over the selected k). The router
// is kept in BF16 weights with F32 logits ("Model artifact and memory placement").
#include "common.cuh"

namespace moe {

// ------------------------------------------------------------------ logits, few tokens
// One warp per (expert, chunk of up to 8 tokens). Lanes stride over K in 16-byte pieces,
// so a warp reads its router row once per chunk with 512-byte coalesced requests.
constexpr int kRouterTok = 8;

__global__ void __launch_bounds__(256) router_small_kernel(
    const uint16_t* __restrict__ x, const uint16_t* __restrict__ wr,
    const float* __restrict__ bias, float* __restrict__ logits, int T, int d, int E) {
  const int lane = threadIdx.x & 31;
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int n_chunks = (T + kRouterTok - 1) / kRouterTok;
  if (warp >= E * n_chunks) return;
  const int e = warp % E;
  const int t0 = (warp / E) * kRouterTok;
  const int nt = min(kRouterTok, T - t0);
  float acc[kRouterTok];
#pragma unroll
  for (int i = 0; i < kRouterTok; ++i) acc[i] = 0.f;
  const uint4* wrow = reinterpret_cast<const uint4*>(wr + (size_t)e * d);
  const int n16 = d / 8;
  for (int c = lane; c < n16; c += 32) {
    uint4 wv = __ldg(wrow + c);
    float w[8];
    const uint32_t ww[4] = {wv.x, wv.y, wv.z, wv.w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      w[2 * q] = __uint_as_float(ww[q] << 16);
      w[2 * q + 1] = __uint_as_float(ww[q] & 0xffff0000u);
    }
#pragma unroll
    for (int i = 0; i < kRouterTok; ++i) {
      if (i < nt) {
        uint4 xv = __ldg(reinterpret_cast<const uint4*>(x + (size_t)(t0 + i) * d) + c);
        const uint32_t xx[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          acc[i] = fmaf(__uint_as_float(xx[q] << 16), w[2 * q], acc[i]);
          acc[i] = fmaf(__uint_as_float(xx[q] & 0xffff0000u), w[2 * q + 1], acc[i]);
        }
      }
    }
  }
#pragma unroll
  for (int i = 0; i < kRouterTok; ++i) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc[i] += __shfl_xor_sync(0xffffffffu, acc[i], o);
  }
  if (lane == 0) {
    const float b = bias ? bias[e] : 0.f;
#pragma unroll
    for (int i = 0; i < kRouterTok; ++i)
      if (i < nt) logits[(size_t)(t0 + i) * E + e] = acc[i] + b;
  }
}

// ------------------------------------------------------------------ logits, many tokens
// Classic shared-memory tiled SIMT product: 64 tokens x 64 experts per CTA, K step 32,
// 256 threads with a 4x4 register tile each.
constexpr int kRT = 64, kRE = 64, kRK = 32;

__global__ void __launch_bounds__(256) router_tiled_kernel(
    const uint16_t* __restrict__ x, const uint16_t* __restrict__ wr,
    const float* __restrict__ bias, float* __restrict__ logits, int T, int d, int E) {
  __shared__ float xs[kRK][kRT + 4];
  __shared__ float ws[kRK][kRE + 4];
  const int t0 = blockIdx.y * kRT, e0 = blockIdx.x * kRE;
  const int tid = threadIdx.x;
  const int tx = tid % 16, ty = tid / 16;  // 16 x 16 threads, 4 x 4 each
  float acc[4][4] = {};
  for (int k0 = 0; k0 < d; k0 += kRK) {
    // load 64 x 32 of X and of Wr: 2048 elements each, 8 per thread
    for (int i = tid; i < kRT * kRK / 8; i += 256) {
      const int row = i / (kRK / 8), c8 = i % (kRK / 8);
      uint4 v = make_uint4(0, 0, 0, 0);
      if (t0 + row < T) v = __ldg(reinterpret_cast<const uint4*>(x + (size_t)(t0 + row) * d + k0) + c8);
      const uint32_t vv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        xs[c8 * 8 + 2 * q][row] = __uint_as_float(vv[q] << 16);
        xs[c8 * 8 + 2 * q + 1][row] = __uint_as_float(vv[q] & 0xffff0000u);
      }
      uint4 w = make_uint4(0, 0, 0, 0);
      if (e0 + row < E) w = __ldg(reinterpret_cast<const uint4*>(wr + (size_t)(e0 + row) * d + k0) + c8);
      const uint32_t wv[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        ws[c8 * 8 + 2 * q][row] = __uint_as_float(wv[q] << 16);
        ws[c8 * 8 + 2 * q + 1][row] = __uint_as_float(wv[q] & 0xffff0000u);
      }
    }
    __syncthreads();
#pragma unroll 8
    for (int kk = 0; kk < kRK; ++kk) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = xs[kk][ty * 4 + i];
#pragma unroll
      for (int j = 0; j < 4; ++j) b[j] = ws[kk][tx * 4 + j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int t = t0 + ty * 4 + i;
    if (t >= T) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int e = e0 + tx * 4 + j;
      if (e < E) logits[(size_t)t * E + e] = acc[i][j] + (bias ? bias[e] : 0.f);
    }
  }
}

cudaError_t launch_router(const Plan& p, cudaStream_t st) {
  if (p.T <= 32) {
    const int warps = p.E * ((p.T + kRouterTok - 1) / kRouterTok);
    const int blocks = (warps * 32 + 255) / 256;
    router_small_kernel<<<blocks, 256, 0, st>>>(p.x, p.router_w, p.router_bias, p.logits, p.T,
                                                p.d, p.E);
  } else {
    dim3 grid((p.E + kRE - 1) / kRE, (p.T + kRT - 1) / kRT);
    router_tiled_kernel<<<grid, 256, 0, st>>>(p.x, p.router_w, p.router_bias, p.logits, p.T,
                                              p.d, p.E);
  }
  return cudaGetLastError();
}

// ------------------------------------------------------------------ top-k and gates
// One warp per token; the token's keys are staged in shared memory (warp_topk_smem).
constexpr int kTopkWarps = 4;

__global__ void __launch_bounds__(32 * kTopkWarps) topk_kernel(const float* __restrict__ logits,
                                                               int32_t* __restrict__ idx_out,
                                                               float* __restrict__ w_out, int T,
                                                               int E, int k) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const int t = blockIdx.x * kTopkWarps + w;
  if (t >= T) return;
  int e;
  uint32_t key;
  warp_topk(logits + (size_t)t * E, E, k, lane, &e, &key);
  const uint32_t top = __shfl_sync(0xffffffffu, key, 0);
  const float g = warp_topk_gate(key, top, k, lane);
  if (lane < k) {
    idx_out[(size_t)t * k + lane] = e;
    w_out[(size_t)t * k + lane] = g;
  }
}

cudaError_t launch_topk(const Plan& p, cudaStream_t st) {
  const int blocks = (p.T + kTopkWarps - 1) / kTopkWarps;
  topk_kernel<<<blocks, 32 * kTopkWarps, 0, st>>>(p.logits, p.topk_idx, p.topk_w, p.T, p.E, p.k);
  return cudaGetLastError();
}

}  // namespace moe
