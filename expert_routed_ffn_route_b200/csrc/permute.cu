// The route plan: per-expert counts, their exclusive scan, and a stable scatter of the
// T*k assignments into expert-major order (Qwen3.8-Flash-Next-Dual-GPU README,
// "Dedicated prefill lane", step 1: a deterministic expert-major route plan built on the
// GPU; TandemLLM docs, "17 Qwen3.8-Flash-Next", §17.4: rows sorted by expert).
//
// Determinism: counts come from integer atomics (order-free); the position of an
// assignment inside its expert's segment is its rank among the same expert's
// assignments with a smaller index a = t*k + j, computed exactly (no ordering races).
// Also writes the active-expert list used to schedule the grouped FFN.
#include <mutex>

#include "common.cuh"

namespace moe {

// Pass 1: one 32-thread CTA per chunk of kPermChunk assignments; its histogram goes to
// cta_hist[chunk][E].
__global__ void __launch_bounds__(32) perm_hist_kernel(const int32_t* __restrict__ idx,
                                                       int32_t* __restrict__ cta_hist, int n,
                                                       int E, int32_t* status) {
  extern __shared__ int32_t hist[];
  for (int e = threadIdx.x; e < E; e += 32) hist[e] = 0;
  __syncwarp();
  const int a0 = blockIdx.x * kPermChunk;
  for (int i = threadIdx.x; i < kPermChunk; i += 32) {
    const int a = a0 + i;
    if (a < n) {
      const int e = idx[a];
      if (e >= 0 && e < E) atomicAdd(&hist[e], 1);
      else set_status(status, DEV_BOUNDS);
    }
  }
  __syncwarp();
  for (int e = threadIdx.x; e < E; e += 32) cta_hist[(size_t)blockIdx.x * E + e] = hist[e];
}

// Block-wide exclusive scan of one value per thread (blockDim.x == 1024).
__device__ int block_exclusive_scan(int v, int* total) {
  __shared__ int warp_sums[32];
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  int incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int u = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += u;
  }
  if (lane == 31) warp_sums[w] = incl;
  __syncthreads();
  if (w == 0) {
    int s = warp_sums[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int u = __shfl_up_sync(0xffffffffu, s, o);
      if (lane >= o) s += u;
    }
    warp_sums[lane] = s;  // inclusive over warps
  }
  __syncthreads();
  const int base = (w > 0) ? warp_sums[w - 1] : 0;
  *total = warp_sums[31];
  __syncthreads();
  return base + incl - v;
}

// Pass 2: one 1024-thread CTA. Per expert: counts over chunks -> per-chunk bases within the
// expert (the scatter adds the expert's offset); then the exclusive scan over experts; then
// the active-expert list. The chunk counts are loaded 16 at a time (independent loads; only
// the running sum is serial), which keeps the pass from running at one L2 round trip a chunk.
__global__ void __launch_bounds__(1024) perm_scan_kernel(int32_t* __restrict__ cta_hist,
                                                         int32_t* __restrict__ offsets,
                                                         int32_t* __restrict__ active,
                                                         int n_chunks, int E) {
  constexpr int kBatch = 16;
  const int e = threadIdx.x;
  int cnt = 0;
  if (e < E) {
    int c = 0;
    for (; c + kBatch <= n_chunks; c += kBatch) {
      int h[kBatch];
#pragma unroll
      for (int j = 0; j < kBatch; ++j) h[j] = cta_hist[(size_t)(c + j) * E + e];
#pragma unroll
      for (int j = 0; j < kBatch; ++j) {
        cta_hist[(size_t)(c + j) * E + e] = cnt;  // exclusive base within the expert
        cnt += h[j];
      }
    }
    for (; c < n_chunks; ++c) {
      const int h = cta_hist[(size_t)c * E + e];
      cta_hist[(size_t)c * E + e] = cnt;
      cnt += h;
    }
  }
  int total;
  const int off = block_exclusive_scan(e < E ? cnt : 0, &total);
  const int flag = (e < E && cnt > 0) ? 1 : 0;
  int n_active;
  const int apos = block_exclusive_scan(flag, &n_active);
  if (e < E) {
    offsets[e] = off;
    if (flag) active[1 + apos] = e;
  }
  if (e == 0) {
    offsets[E] = total;
    active[0] = n_active;
  }
}

// Pass 3: each 32-thread CTA walks its chunk in order, 32 assignments at a time; inside a
// step, lanes with the same expert are ranked by lane (match_any), and a per-expert running
// position in shared memory (the expert's offset + the chunk's base within the expert)
// carries the order across steps.
__global__ void __launch_bounds__(32) perm_scatter_kernel(const int32_t* __restrict__ idx,
                                                          const int32_t* __restrict__ cta_base,
                                                          const int32_t* __restrict__ offsets,
                                                          int32_t* __restrict__ perm,
                                                          int32_t* __restrict__ inv, int n,
                                                          int E) {
  extern __shared__ int32_t run[];
  const int lane = threadIdx.x;
  for (int e = lane; e < E; e += 32) run[e] = offsets[e] + cta_base[(size_t)blockIdx.x * E + e];
  __syncwarp();
  const int a0 = blockIdx.x * kPermChunk;
  for (int s = 0; s < kPermChunk; s += 32) {
    const int a = a0 + s + lane;
    const bool valid = a < n;
    int e = valid ? idx[a] : -1;
    if (e < 0 || e >= E) e = -1;  // out-of-range ids were flagged by pass 1
    const unsigned mask = __match_any_sync(0xffffffffu, e);
    const int rank = __popc(mask & ((1u << lane) - 1u));
    int pos = 0;
    if (e >= 0) pos = run[e] + rank;
    __syncwarp();
    if (e >= 0 && (mask >> lane) == 1u) run[e] += __popc(mask);  // highest lane of the group
    __syncwarp();
    if (e >= 0) {
      perm[pos] = a;
      inv[a] = pos;
    } else if (valid) {
      inv[a] = 0;  // keep later gathers in bounds; the status word records the bad id
    }
  }
}

// Small calls (n <= 1024, one CTA of 1024 threads): all three passes in one launch.
// Warp w owns assignments [32w, 32w+32); cross-warp order comes from per-warp counts.
__global__ void __launch_bounds__(1024) perm_small_kernel(const int32_t* __restrict__ idx,
                                                          int32_t* __restrict__ offsets,
                                                          int32_t* __restrict__ perm,
                                                          int32_t* __restrict__ inv,
                                                          int32_t* __restrict__ active, int n,
                                                          int E, int32_t* status) {
  extern __shared__ uint16_t wcnt[];  // [32][E] counts per warp and expert
  __shared__ int soff[kMaxE];
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  for (int i = tid; i < 32 * E; i += 1024) wcnt[i] = 0;
  __syncthreads();
  int e = -1;
  if (tid < n) {
    e = idx[tid];
    if (e < 0 || e >= E) { set_status(status, DEV_BOUNDS); e = -1; }
  }
  const unsigned mask = __match_any_sync(0xffffffffu, e);
  const int rank = __popc(mask & ((1u << lane) - 1u));
  if (e >= 0 && (mask >> lane) == 1u) wcnt[w * E + e] = (uint16_t)__popc(mask);
  __syncthreads();
  // per expert: counts and the exclusive base of each warp (in place)
  int cnt = 0;
  if (tid < E) {
    for (int ww = 0; ww < 32; ++ww) {
      const int c = wcnt[ww * E + tid];
      wcnt[ww * E + tid] = (uint16_t)cnt;
      cnt += c;
    }
  }
  int total;
  const int off = block_exclusive_scan(tid < E ? cnt : 0, &total);
  const int flag = (tid < E && cnt > 0) ? 1 : 0;
  int n_active;
  const int apos = block_exclusive_scan(flag, &n_active);
  if (tid < E) {
    soff[tid] = off;
    offsets[tid] = off;
    if (flag) active[1 + apos] = tid;
  }
  if (tid == 0) {
    offsets[E] = total;
    active[0] = n_active;
  }
  __syncthreads();
  if (e >= 0) {
    const int pos = soff[e] + wcnt[w * E + e] + rank;
    perm[pos] = tid;
    inv[tid] = pos;
  } else if (tid < n) {
    inv[tid] = 0;  // keep later gathers in bounds; the status word records the bad id
  }
}

cudaError_t launch_permute(const Plan& p, cudaStream_t st) {
  const int n = p.T * p.k;
  if (n <= 1024) {
    const size_t smem = sizeof(uint16_t) * 32 * p.E;
    static std::once_flag once;  // opt in to the largest size (E = 1024) on the first call
    static cudaError_t once_err = cudaSuccess;
    std::call_once(once, [] {
      once_err = cudaFuncSetAttribute(perm_small_kernel,
                                      cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      (int)(sizeof(uint16_t) * 32 * kMaxE));
    });
    if (once_err != cudaSuccess) return once_err;
    perm_small_kernel<<<1, 1024, smem, st>>>(p.topk_idx, p.offsets, p.perm, p.inv, p.active, n,
                                             p.E, p.status);
    return cudaGetLastError();
  }
  const int chunks = perm_chunks(p.T, p.k);
  const size_t smem = sizeof(int32_t) * p.E;
  perm_hist_kernel<<<chunks, 32, smem, st>>>(p.topk_idx, p.cta_hist, n, p.E, p.status);
  perm_scan_kernel<<<1, 1024, 0, st>>>(p.cta_hist, p.offsets, p.active, chunks, p.E);
  perm_scatter_kernel<<<chunks, 32, smem, st>>>(p.topk_idx, p.cta_hist, p.offsets, p.perm, p.inv,
                                                 n, p.E);
  return cudaGetLastError();
}

// Active-expert list from caller-provided offsets (used by moe_grouped_ffn alone).
__global__ void __launch_bounds__(1024) schedule_kernel(const int32_t* __restrict__ offsets,
                                                        int32_t* __restrict__ active, int E) {
  const int e = threadIdx.x;
  const int flag = (e < E && offsets[e + 1] > offsets[e]) ? 1 : 0;
  int n_active;
  const int apos = block_exclusive_scan(flag, &n_active);
  if (flag) active[1 + apos] = e;
  if (e == 0) active[0] = n_active;
}

cudaError_t launch_schedule_from_offsets(const Plan& p, cudaStream_t st) {
  schedule_kernel<<<1, 1024, 0, st>>>(p.offsets, p.active, p.E);
  return cudaGetLastError();
}

}  // namespace moe
