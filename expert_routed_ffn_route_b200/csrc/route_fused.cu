// Routing and the route plan in one launch, for calls of up to 32 tokens (decode and
// verify rows), where three separate launches would cost more than the work.
//
// Phase 1 (all CTAs): router logits l[t][e] = x_t . Wr_e (+ b_e) in fp32, one warp per
// expert row, 128-bit loads, every token of the call against the row while it is in
// registers. Phase 2 (CTAs 0 .. T-1, once every CTA has counted itself in a ticket after a
// memory fence): CTA t ranks token t (stable top-k and gates). Phase 3 (the last of those to
// finish, found with a second ticket): the expert-major plan and the active-expert list,
// then the second ticket is cleared for the next call (the first is a grid barrier word
// that returns to its start value by itself).
//
// Rules followed: deterministic stable top-k, ties to the lower expert index
// (Qwen3.8-Flash-Next-Dual-GPU README, "Independent decode lane"); gates = softmax over the
// selected logits; plan = counts, exclusive scan, stable scatter (README, "Dedicated
// prefill lane", step 1).
#include <algorithm>

#include "pipeline.cuh"

namespace moe {


constexpr int kRFWarps = 4;
constexpr int kRFThreads = 32 * kRFWarps;
constexpr int kRFMaxT = 32;
static_assert(kRFMaxT % 2 == 0, "the logits take tokens two at a time");

__global__ void __launch_bounds__(kRFThreads) route_fused_kernel(Plan p, int32_t* ticket) {
  __shared__ int s_last;  // this CTA ranked the last token: it builds the plan
  __shared__ int s_idx[kRFMaxT * kMaxK];
  __shared__ int s_cnt[kMaxE];
  __shared__ int s_off[kMaxE + 1];
  __shared__ int s_wsum[kRFWarps];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int T = p.T, E = p.E, d = p.d, k = p.k;
  pdl_wait();

  // ---------------------------------------------------------------- logits
  // A lane owns 16-byte pieces c = lane + 32 i of the router row (d <= 8192: i < 32); the
  // row is loaded in batches of 8 pieces, all in flight together, then the tokens are applied
  // to the batch two at a time while it sits in registers: both tokens' 16 loads are issued
  // before their products (the second row index is clamped, so the loads need no guard; a
  // product past the last token is never written).
  const int n16 = d / 8;
  for (int e = blockIdx.x * kRFWarps + warp; e < E; e += gridDim.x * kRFWarps) {
    const uint4* wrow = reinterpret_cast<const uint4*>(p.router_w + (size_t)e * d);
    const float b = p.router_bias ? p.router_bias[e] : 0.f;
    float acc[kRFMaxT];
#pragma unroll
    for (int t = 0; t < kRFMaxT; ++t) acc[t] = 0.f;
    for (int c0 = 0; c0 < n16; c0 += 8 * 32) {
      uint4 wv[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int c = c0 + lane + 32 * i;
        wv[i] = (c < n16) ? __ldg(wrow + c) : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int t0 = 0; t0 < kRFMaxT; t0 += 2) {
        if (t0 >= T) break;
        const int t1 = min(t0 + 1, T - 1);
        const uint4* xa_row = reinterpret_cast<const uint4*>(p.x + (size_t)t0 * d);
        const uint4* xb_row = reinterpret_cast<const uint4*>(p.x + (size_t)t1 * d);
        uint4 xa[8], xb[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int c = c0 + lane + 32 * i;
          xa[i] = (c < n16) ? __ldg(xa_row + c) : make_uint4(0, 0, 0, 0);
          xb[i] = (c < n16) ? __ldg(xb_row + c) : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const uint32_t ww[4] = {wv[i].x, wv[i].y, wv[i].z, wv[i].w};
          const uint32_t aa[4] = {xa[i].x, xa[i].y, xa[i].z, xa[i].w};
          const uint32_t bb[4] = {xb[i].x, xb[i].y, xb[i].z, xb[i].w};
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const float w0 = __uint_as_float(ww[q] << 16), w1 = __uint_as_float(ww[q] & 0xffff0000u);
            acc[t0] = fmaf(__uint_as_float(aa[q] << 16), w0, acc[t0]);
            acc[t0] = fmaf(__uint_as_float(aa[q] & 0xffff0000u), w1, acc[t0]);
            acc[t0 + 1] = fmaf(__uint_as_float(bb[q] << 16), w0, acc[t0 + 1]);
            acc[t0 + 1] = fmaf(__uint_as_float(bb[q] & 0xffff0000u), w1, acc[t0 + 1]);
          }
        }
      }
    }
#pragma unroll
    for (int t = 0; t < kRFMaxT; ++t) {
      if (t >= T) break;
      float v = acc[t];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
      if (lane == 0) p.logits[(size_t)t * E + e] = v + b;
    }
  }

  // ---------------------------------------------------------------- tickets
  // Every CTA publishes its logits and arrives at a grid barrier on ticket[0] (the flip-bit
  // barrier of pipeline.cuh); CTAs T.. leave. CTA t < T waits, boundedly, for the barrier
  // (all CTAs of this grid are resident together: gridDim = max(E / 4, T) <= 256 small
  // CTAs), ranks token t, and counts itself in ticket[1]; the last one builds the plan and
  // clears ticket[1]. After a timeout the status word is set and the CTA goes on (its picks
  // are then unreliable); every CTA has arrived all the same, so the barrier word is
  // consistent for the next call.
  __shared__ uint32_t s_arrived;
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) s_arrived = gbar_arrive(reinterpret_cast<uint32_t*>(&ticket[0]));
  if ((int)blockIdx.x >= T) {
    return;  // an exited CTA counts as having released its dependents
  }
  if (threadIdx.x == 0) {
    if (!gbar_wait(reinterpret_cast<const uint32_t*>(&ticket[0]), s_arrived))
      set_timeout(p.status, 1);
    else if (!test_hold_wait(p.test_ctl))
      set_timeout(p.status, 2);
  }
  __syncthreads();
  __threadfence();

  // ---------------------------------------------------------------- top-k and gates
  if (warp == 0) {
    const int t = blockIdx.x;
    int e;
    uint32_t key;
    warp_topk(p.logits + (size_t)t * E, E, k, lane, &e, &key);
    const uint32_t top = __shfl_sync(0xffffffffu, key, 0);
    const float g = warp_topk_gate(key, top, k, lane);
    if (lane < k) {
      p.topk_idx[(size_t)t * k + lane] = e;
      p.topk_w[(size_t)t * k + lane] = g;
    }
  }
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) s_last = (atomicAdd(&ticket[1], 1) == T - 1);
  __syncthreads();
  if (!s_last) {
    return;
  }
  __threadfence();
  for (int a = threadIdx.x; a < T * k; a += kRFThreads) s_idx[a] = __ldcg(p.topk_idx + a);
  __syncthreads();

  // ---------------------------------------------------------------- plan
  const int n = T * k;
  if (n <= 32) {
    // Few assignments: warp 0 ranks them by (expert, index) directly; every thread fills
    // the offsets of its experts by counting smaller expert ids.
    __shared__ int s_sorted[32];
    if (warp == 0) {
      const int e_me = (lane < n) ? s_idx[lane] : 0x7fffffff;
      int rank = 0;
      for (int b = 0; b < n; ++b) {
        const int eb = __shfl_sync(0xffffffffu, e_me, b);
        rank += (eb < e_me) || (eb == e_me && b < lane);
      }
      if (lane < n) {
        p.perm[rank] = lane;
        p.inv[lane] = rank;
        s_sorted[rank] = e_me;
      }
      __syncwarp();
      const bool first = lane < n && (lane == 0 || s_sorted[lane - 1] != s_sorted[lane]);
      const unsigned m = __ballot_sync(0xffffffffu, first);
      if (first) p.active[1 + __popc(m & ((1u << lane) - 1u))] = s_sorted[lane];
      if (lane == 0) p.active[0] = __popc(m);
    }
    for (int e = threadIdx.x; e <= E; e += kRFThreads) {
      int c = 0;
      for (int a = 0; a < n; ++a) c += (s_idx[a] < e);
      p.offsets[e] = c;
    }
  } else {
    for (int e = threadIdx.x; e < E; e += kRFThreads) s_cnt[e] = 0;
    __syncthreads();
    for (int a = threadIdx.x; a < n; a += kRFThreads) atomicAdd(&s_cnt[s_idx[a]], 1);
    __syncthreads();
    // exclusive scan of s_cnt (each thread owns a contiguous run of experts)
    const int per = (E + kRFThreads - 1) / kRFThreads;
    const int e0 = threadIdx.x * per;
    int local = 0;
    for (int e = e0; e < min(E, e0 + per); ++e) local += s_cnt[e];
    int incl = local;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int u = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += u;
    }
    if (lane == 31) s_wsum[warp] = incl;
    __syncthreads();
    int base = 0;
    for (int w = 0; w < warp; ++w) base += s_wsum[w];
    int run = base + incl - local;
    for (int e = e0; e < min(E, e0 + per); ++e) {
      s_off[e] = run;
      p.offsets[e] = run;
      run += s_cnt[e];
    }
    if (threadIdx.x == kRFThreads - 1) {
      s_off[E] = run;
      p.offsets[E] = run;
    }
    __syncthreads();
    // active experts in ascending order (warp 0, 32 experts a step)
    if (warp == 0) {
      int nact = 0;
      for (int e0b = 0; e0b < E; e0b += 32) {
        const int e = e0b + lane;
        const bool on = (e < E) && s_cnt[e] > 0;
        const unsigned m = __ballot_sync(0xffffffffu, on);
        if (on) p.active[1 + nact + __popc(m & ((1u << lane) - 1u))] = e;
        nact += __popc(m);
      }
      if (lane == 0) p.active[0] = nact;
    }
    // stable scatter (warp 1; assignments in order, 32 a step)
    if (warp == 1) {
      for (int a0 = 0; a0 < n; a0 += 32) {
        const int a = a0 + lane;
        const int e = (a < n) ? s_idx[a] : -1;
        const unsigned m = __match_any_sync(0xffffffffu, e);
        const int rank = __popc(m & ((1u << lane) - 1u));
        int pos = 0;
        if (e >= 0) pos = s_off[e] + rank;
        __syncwarp();
        if (e >= 0 && (m >> lane) == 1u) s_off[e] += __popc(m);
        __syncwarp();
        if (e >= 0) {
          p.perm[pos] = a;
          p.inv[a] = pos;
        }
      }
    }
  }
  __syncthreads();
  __syncthreads();
  if (threadIdx.x == 0) ticket[1] = 0;
  // The next kernel is released only now: kernels whose CTAs wait early for this one share
  // the SMs and slow the last CTA down.
  pdl_trigger();
}

bool route_fused_supported(const Plan& p) { return p.T <= kRFMaxT && p.E <= kMaxE; }

// One CTA per 4 expert rows and at least one per token (CTA t ranks token t).
cudaError_t launch_route_fused(const Plan& p, int32_t* ticket, cudaStream_t st) {
  const int blocks = std::max((p.E + kRFWarps - 1) / kRFWarps, p.T);
  route_fused_kernel<<<blocks, kRFThreads, 0, st>>>(p, ticket);
  return cudaGetLastError();
}

}  // namespace moe
