// Weighted combine: out_t = sum_{j<k} gate[t,j] * y[inv[t*k+j]] + y_shared[t], accumulated
// in fp32 in the order j = 0..k-1 and then the shared term, rounded once to bf16, with no
// atomics (Qwen3.8-Flash-Next-Dual-GPU README, "Dedicated prefill lane", step 5: each
// token's ten routes reduced in a fixed order without atomics; TandemLLM docs,
// "17 Qwen3.8-Flash-Next", Table 17.1: one shared expert runs on every token).
//
// The k row indices and gates of a token are read first; the k row loads that follow are
// independent of each other, so they are in flight together.
#include "pipeline.cuh"

namespace moe {

constexpr int kCombThreads = 128;

__global__ void __launch_bounds__(kCombThreads) combine_kernel(const float* __restrict__ y_assign,
                                                               const float* __restrict__ y_shared,
                                                               const int32_t* __restrict__ inv,
                                                               const float* __restrict__ gates,
                                                               uint16_t* __restrict__ out, int T,
                                                               int d, int k) {
  __shared__ int s_row[kMaxK];
  __shared__ float s_w[kMaxK];
  pdl_wait();
  const int t = blockIdx.y;
  if (threadIdx.x < k) {
    s_row[threadIdx.x] = inv[(size_t)t * k + threadIdx.x];
    s_w[threadIdx.x] = gates[(size_t)t * k + threadIdx.x];
  }
  __syncthreads();
  const int n = 4 * (blockIdx.x * blockDim.x + threadIdx.x);
  if (n >= d) return;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int j0 = 0; j0 < k; j0 += 8) {
    float4 y[8];
#pragma unroll
    for (int j = 0; j < 8; ++j)
      if (j0 + j < k) y[j] = __ldcg(reinterpret_cast<const float4*>(y_assign + (size_t)s_row[j0 + j] * d + n));
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      if (j0 + j < k) {
        const float w = s_w[j0 + j];
        acc.x = fmaf(w, y[j].x, acc.x);
        acc.y = fmaf(w, y[j].y, acc.y);
        acc.z = fmaf(w, y[j].z, acc.z);
        acc.w = fmaf(w, y[j].w, acc.w);
      }
    }
  }
  if (y_shared) {
    const float4 y = __ldcg(reinterpret_cast<const float4*>(y_shared + (size_t)t * d + n));
    acc.x += y.x;
    acc.y += y.y;
    acc.z += y.z;
    acc.w += y.w;
  }
  uint2 o;
  o.x = pack_bf16x2(acc.x, acc.y);
  o.y = pack_bf16x2(acc.z, acc.w);
  *reinterpret_cast<uint2*>(out + (size_t)t * d + n) = o;
}

cudaError_t launch_combine(const Plan& p, void* out, cudaStream_t st, bool pdl) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((p.d / 4 + kCombThreads - 1) / kCombThreads, p.T);
  cfg.blockDim = dim3(kCombThreads);
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = pdl ? 1 : 0;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const float* ys = p.has_shared ? p.y_shared : nullptr;
  return cudaLaunchKernelEx(&cfg, combine_kernel, (const float*)p.y_assign, ys,
                            (const int32_t*)p.inv, (const float*)p.topk_w,
                            static_cast<uint16_t*>(out), p.T, p.d, p.k);
}

}  // namespace moe
