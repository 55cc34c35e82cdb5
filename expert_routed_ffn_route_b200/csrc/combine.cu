// Weighted combine: out_t = sum_{j<k} gate[t,j] * y[inv[t*k+j]] + y_shared[t], accumulated
// in fp32 in the order j = 0..k-1 and then the shared term, rounded once to bf16, with no
// atomics (Qwen3.8-Flash-Next-Dual-GPU README, "Dedicated prefill lane", step 5: each
// token's ten routes reduced in a fixed order without atomics; TandemLLM docs,
// "17 Qwen3.8-Flash-Next", Table 17.1: one shared expert runs on every token).
#include "common.cuh"

namespace moe {

__global__ void __launch_bounds__(256) combine_kernel(const float* __restrict__ y_assign,
                                                      const float* __restrict__ y_shared,
                                                      const int32_t* __restrict__ inv,
                                                      const float* __restrict__ gates,
                                                      uint16_t* __restrict__ out, int T,
                                                      int d, int k) {
  const int t = blockIdx.y;
  const int n = 4 * (blockIdx.x * blockDim.x + threadIdx.x);
  if (n >= d) return;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int j = 0; j < k; ++j) {
    const float w = gates[(size_t)t * k + j];
    const int r = inv[(size_t)t * k + j];
    const float4 y = *reinterpret_cast<const float4*>(y_assign + (size_t)r * d + n);
    acc.x = fmaf(w, y.x, acc.x);
    acc.y = fmaf(w, y.y, acc.y);
    acc.z = fmaf(w, y.z, acc.z);
    acc.w = fmaf(w, y.w, acc.w);
  }
  if (y_shared) {
    const float4 y = *reinterpret_cast<const float4*>(y_shared + (size_t)t * d + n);
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

cudaError_t launch_combine(const Plan& p, void* out, cudaStream_t st) {
  dim3 grid((p.d / 4 + 255) / 256, p.T);
  combine_kernel<<<grid, 256, 0, st>>>(p.y_assign, p.has_shared ? p.y_shared : nullptr, p.inv,
                                       p.topk_w, static_cast<uint16_t*>(out), p.T, p.d, p.k);
  return cudaGetLastError();
}

}  // namespace moe
