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
// Tensor-core product (mma.sync m16n8k16, bf16 inputs, fp32 accumulation; the products of
// two bf16 values are exact in fp32): 64 tokens x 64 experts per CTA, 4 warps of 32 x 32,
// K in tiles of 64 staged by 16-byte cp.async copies (double buffered, rows padded to 72
// elements so the 8 rows an ldmatrix reads fall in distinct banks). Each logit is summed
// in one fixed order, so the result is reproducible.
constexpr int kRT = 64, kRE = 64, kRK = 64, kRPad = 72;

__device__ __forceinline__ void cp_async16(void* dst, const void* src, int src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(
                   static_cast<uint32_t>(__cvta_generic_to_shared(dst))),
               "l"(src), "r"(src_bytes)
               : "memory");
}

__device__ __forceinline__ void ldmatrix_x4(uint32_t (&r)[4], const void* p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(static_cast<uint32_t>(__cvta_generic_to_shared(p))));
}

__global__ void __launch_bounds__(128) router_mma_kernel(
    const uint16_t* __restrict__ x, const uint16_t* __restrict__ wr,
    const float* __restrict__ bias, float* __restrict__ logits, int T, int d, int E) {
  __shared__ __align__(16) uint16_t xs[2][kRT][kRPad];
  __shared__ __align__(16) uint16_t ws[2][kRE][kRPad];
  const int t0 = blockIdx.y * kRT, e0 = blockIdx.x * kRE;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int wt = (warp >> 1) * 32, we = (warp & 1) * 32;  // this warp's 32 x 32 block

  // tile k0 -> stage s: 64 rows x 8 pieces of 16 bytes for X and for Wr (1024 copies, 8 a
  // thread); rows past T or E read nothing and fill zeros
  auto load = [&](int s, int k0) {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int c = tid + 128 * i;  // 0 .. 1023
      const int which = c >> 9, row = (c >> 3) & 63, piece = c & 7;
      if (which == 0) {
        const int t = t0 + row;
        const uint16_t* src = x + (size_t)min(t, T - 1) * d + k0 + 8 * piece;
        cp_async16(&xs[s][row][8 * piece], src, t < T ? 16 : 0);
      } else {
        const int e = e0 + row;
        const uint16_t* src = wr + (size_t)min(e, E - 1) * d + k0 + 8 * piece;
        cp_async16(&ws[s][row][8 * piece], src, e < E ? 16 : 0);
      }
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
  };

  float acc[2][4][4];
#pragma unroll
  for (int i = 0; i < 2; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j)
#pragma unroll
      for (int q = 0; q < 4; ++q) acc[i][j][q] = 0.f;

  const int n_k = d / kRK;
  load(0, 0);
  for (int kt = 0; kt < n_k; ++kt) {
    const int s = kt & 1;
    if (kt + 1 < n_k) {
      load(s ^ 1, (kt + 1) * kRK);
      asm volatile("cp.async.wait_group 1;" ::: "memory");
    } else {
      asm volatile("cp.async.wait_group 0;" ::: "memory");
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < kRK; kk += 16) {
      // A (tokens x K, row-major): two 16 x 16 fragments; B (experts x K = the K-major "col"
      // operand): four 8-expert x 16 fragments, two per ldmatrix.x4
      uint32_t a[2][4], b[2][4];
#pragma unroll
      for (int i = 0; i < 2; ++i)
        ldmatrix_x4(a[i], &xs[s][wt + 16 * i + (lane & 15)][kk + 8 * (lane >> 4)]);
#pragma unroll
      for (int j = 0; j < 2; ++j)
        ldmatrix_x4(b[j], &ws[s][we + 16 * j + (lane & 7) + 8 * (lane >> 4)][kk + 8 * ((lane >> 3) & 1)]);
#pragma unroll
      for (int i = 0; i < 2; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const uint32_t b0 = b[j >> 1][2 * (j & 1)], b1 = b[j >> 1][2 * (j & 1) + 1];
          asm volatile(
              "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, "
              "{%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
              : "+f"(acc[i][j][0]), "+f"(acc[i][j][1]), "+f"(acc[i][j][2]), "+f"(acc[i][j][3])
              : "r"(a[i][0]), "r"(a[i][1]), "r"(a[i][2]), "r"(a[i][3]), "r"(b0), "r"(b1));
        }
    }
    __syncthreads();
  }
  // C fragment: rows grp and grp + 8 of the 16-token block, columns 2q, 2q + 1 of the 8
  const int grp = lane >> 2, q = lane & 3;
#pragma unroll
  for (int i = 0; i < 2; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j)
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int t = t0 + wt + 16 * i + grp + 8 * h;
        if (t >= T) continue;
#pragma unroll
        for (int c2 = 0; c2 < 2; ++c2) {
          const int e = e0 + we + 8 * j + 2 * q + c2;
          if (e < E) logits[(size_t)t * E + e] = acc[i][j][2 * h + c2] + (bias ? bias[e] : 0.f);
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
    router_mma_kernel<<<grid, 128, 0, st>>>(p.x, p.router_w, p.router_bias, p.logits, p.T, p.d,
                                            p.E);
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
