// Grouped expert FFN for few rows per expert (decode and verify calls, 1..32 tokens):
// split-K, bandwidth-bound GEMV kernels over the touched experts only.
//
// Work unit = (active expert, 32 weight rows). A 256-thread CTA owns one unit at a time:
// warps 0-3 take rows 0-15, warps 4-7 rows 16-31, and within each half the four warps
// split the K groups round-robin; partial sums are added in a fixed order (no atomics),
// so results do not depend on scheduling. Weights stream straight from HBM into registers
// with 128-bit non-allocating loads (each expert row is read once per 8-token chunk), and
// the products run on the tensor cores with mma.sync m16n8k16 (bf16 in, fp32 out): the
// weights are the 16-row A operand, up to 8 tokens are the N = 8 B operand.
//
// The group scale multiplies the fp32 partial of its 128-wide K group, so quantised codes
// enter the tensor core exactly (integers |q| <= 127 are exact in bf16).
//
// int4 codes are widened with a bf16 bit trick: the nibble n (after flipping its sign bit,
// u = n ^ 8 = q + 8) is placed in the low mantissa bits of 128.0 (0x4300), giving the exact
// bf16 value 128 + u = q + 136; the constant 136 * sum(x over the group) is subtracted from
// each group's partial afterwards.
//
// What each part computes: gate/up kernel h = silu(Wg x) * (Wu x) for every grouped row
// (Qwen3.8-Flash-Next-Dual-GPU README, "Dedicated prefill lane", step 2: grouped W4/W8-A16
// products on the tensor cores); down kernel y = Wd h into one fp32 row per assignment
// (same section, step 4). Unselected experts are never read (TandemLLM docs,
// "17 Qwen3.8-Flash-Next", §17.4).
#include <mutex>

#include "gemv_frag.cuh"

namespace moe {

constexpr int kRowsCTA = 32;  // weight rows per CTA
constexpr int kKSplit = 4;    // warps sharing one 16-row tile along K
constexpr int kThreads = 256;

// Per-CTA view of one unit.
struct Unit {
  int e;          // expert index within its bank
  bool shared;
  int row_begin;  // first grouped row (routed) / first token (shared)
  int nrows;
  int tile;       // 32-row tile of the weight matrix
};

// part: 0 both banks, 1 the routed bank only, 2 the shared expert only (one launch per bank
// when the two banks have different formats).
__device__ __forceinline__ bool get_unit(const Plan& p, int u, int n_tiles, int part, Unit& out) {
  const int n_active = p.active[0];
  if (part == 2) u += n_active * n_tiles;  // skip the routed slots
  const int slot = u / n_tiles;
  out.tile = u % n_tiles;
  if (slot < n_active) {
    if (part == 2) return false;
    out.e = p.active[1 + slot];
    out.shared = false;
    out.row_begin = p.offsets[out.e];
    out.nrows = p.offsets[out.e + 1] - out.row_begin;
    return true;
  }
  if (slot == n_active && p.has_shared && part != 1) {
    out.e = 0;
    out.shared = true;
    out.row_begin = 0;
    out.nrows = p.T;
    return true;
  }
  return false;
}

// GATE_UP: weights gate+up [f][d], activations x (gathered by perm), output h (bf16).
// !GATE_UP: weights down [d][f], activations h, output y (fp32).
template <int FMT, bool GATE_UP>
__global__ void __launch_bounds__(kThreads) gemv_ffn_kernel(Plan p, int part) {
  constexpr int NM = GATE_UP ? 2 : 1;
  constexpr int U = FmtInfo<FMT>::U;
  constexpr int PF = (FMT == 4) ? 5 : (FMT == 8 ? (GATE_UP ? 3 : 4) : 2);
  const int K = GATE_UP ? p.d : p.f;
  const int N = GATE_UP ? p.f : p.d;
  const int G = K / kGroup;
  const int S = 2 * K + 8;
  const int n_tiles = N / kRowsCTA;
  const size_t row_bytes = (size_t)K * FmtInfo<FMT>::bits / 8;
  const size_t mat_bytes = row_bytes * N;

  extern __shared__ __align__(16) uint8_t smem[];
  uint8_t* xs = smem;
  float* xsum = reinterpret_cast<float*>(smem + kTok * S);
  float* red = xsum + kTok * G;  // [8 warps][32 lanes][NM*4]

  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int rt = warp / kKSplit, ks = warp % kKSplit;
  const int grp = lane >> 2, q4 = lane & 3;

  for (int u = blockIdx.x;; u += gridDim.x) {
    Unit un;
    if (!get_unit(p, u, n_tiles, part, un)) break;
    const Bank& bank = un.shared ? p.shared : p.routed;
    const int ra_row = un.tile * kRowsCTA + rt * 16 + grp;
    const int rb_row = ra_row + 8;
    const uint8_t* wbase[NM];
    const uint16_t* sbase[NM];
#pragma unroll
    for (int mi = 0; mi < NM; ++mi) {
      const int which = GATE_UP ? mi : 2;
      wbase[mi] = static_cast<const uint8_t*>(bank.w[which]) + (size_t)un.e * mat_bytes;
      sbase[mi] = bank.s[which] ? bank.s[which] + ((size_t)un.e * N) * G : nullptr;
    }
    for (int c0 = 0; c0 < un.nrows; c0 += kTok) {
      const int nr = min(kTok, un.nrows - c0);
      StageArgs sa;
      if (GATE_UP) {
        sa.src = p.x;
        sa.src_stride = p.d;
        sa.perm = un.shared ? nullptr : p.perm;
        sa.k = p.k;
        sa.row0 = un.row_begin + c0;
      } else {
        sa.src = p.h;
        sa.src_stride = p.f;
        sa.perm = nullptr;
        sa.k = 1;
        sa.row0 = (un.shared ? p.T * p.k : 0) + un.row_begin + c0;
      }
      sa.nrows = nr;
      __syncthreads();  // previous chunk's readers are done with xs / red
      stage_rows<FMT, kThreads>(sa, K, xs, S, xsum, threadIdx.x);
      __syncthreads();

      float acc[NM][4];
#pragma unroll
      for (int mi = 0; mi < NM; ++mi)
#pragma unroll
        for (int i = 0; i < 4; ++i) acc[mi][i] = 0.f;
      const uint8_t* xrow = xs + (size_t)grp * S;

      for (int gb = ks; gb < G; gb += kKSplit * PF) {
        uint4 wa[PF][NM][U], wb[PF][NM][U];
        float fsa[PF][NM], fsb[PF][NM];
#pragma unroll
        for (int pf = 0; pf < PF; ++pf) {
          const int g = gb + kKSplit * pf;
          if (g < G) {
#pragma unroll
            for (int mi = 0; mi < NM; ++mi) {
              const uint8_t* pa = wbase[mi] + (size_t)ra_row * row_bytes +
                                  (size_t)g * (kGroup * FmtInfo<FMT>::bits / 8) + q4 * (16 * U);
              const uint8_t* pb = pa + 8 * row_bytes;
#pragma unroll
              for (int uu = 0; uu < U; ++uu) {
                wa[pf][mi][uu] = ld_nc_v4(pa + 16 * uu);
                wb[pf][mi][uu] = ld_nc_v4(pb + 16 * uu);
              }
              if (sbase[mi]) {
                fsa[pf][mi] = bf16_to_f32(__ldg(sbase[mi] + (size_t)ra_row * G + g));
                fsb[pf][mi] = bf16_to_f32(__ldg(sbase[mi] + (size_t)rb_row * G + g));
              } else {
                fsa[pf][mi] = 1.f;
                fsb[pf][mi] = 1.f;
              }
            }
          }
        }
#pragma unroll
        for (int pf = 0; pf < PF; ++pf) {
          const int g = gb + kKSplit * pf;
          if (g < G)
            group_mma<FMT, NM>(wa[pf], wb[pf], fsa[pf], fsb[pf], xrow, xsum, G, g, q4, acc);
        }
      }
      // fixed-order reduction over the K split
      float* myred = red + ((size_t)warp * 32 + lane) * (NM * 4);
#pragma unroll
      for (int mi = 0; mi < NM; ++mi)
#pragma unroll
        for (int i = 0; i < 4; ++i) myred[mi * 4 + i] = acc[mi][i];
      __syncthreads();
      if (ks == 0) {
        float tot[NM][4];
#pragma unroll
        for (int mi = 0; mi < NM; ++mi)
#pragma unroll
          for (int i = 0; i < 4; ++i) tot[mi][i] = 0.f;
        for (int s = 0; s < kKSplit; ++s) {
          const float* r = red + ((size_t)(rt * kKSplit + s) * 32 + lane) * (NM * 4);
#pragma unroll
          for (int mi = 0; mi < NM; ++mi)
#pragma unroll
            for (int i = 0; i < 4; ++i) tot[mi][i] += r[mi * 4 + i];
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int tok = 2 * q4 + (i & 1);
          const int row = (i < 2) ? ra_row : rb_row;
          if (tok >= nr) continue;
          if constexpr (GATE_UP) {
            const float g = tot[0][i], up = tot[1][i];
            const float hval = g / (1.f + expf(-g)) * up;
            const size_t hrow = (un.shared ? (size_t)p.T * p.k : 0) + un.row_begin + c0 + tok;
            p.h[hrow * p.f + row] = f32_to_bf16_rn(hval);
          } else {
            float* dst = un.shared ? p.y_shared + (size_t)(un.row_begin + c0 + tok) * p.d
                                   : p.y_assign + (size_t)(un.row_begin + c0 + tok) * p.d;
            dst[row] = tot[0][i];
          }
        }
      }
    }
  }
}

// Per-instantiation launch facts (dynamic shared memory opt-in, resident CTAs per SM),
// settled on the first call so that later calls (and stream captures) make no attribute
// or occupancy queries.
struct LaunchCache {
  std::mutex mu;
  size_t smem = 0;
  int per_sm = 0, sms = 0;
};

template <int FMT, bool GATE_UP>
static cudaError_t launch_one(const Plan& p, int part, cudaStream_t st) {
  const int K = GATE_UP ? p.d : p.f;
  const int N = GATE_UP ? p.f : p.d;
  const int NM = GATE_UP ? 2 : 1;
  const size_t smem = (size_t)kTok * (2 * K + 8) + sizeof(float) * kTok * (K / kGroup) +
                      sizeof(float) * 8 * 32 * NM * 4;
  auto kern = gemv_ffn_kernel<FMT, GATE_UP>;
  static LaunchCache cache;
  int per_sm, sms;
  {
    std::lock_guard<std::mutex> lock(cache.mu);
    if (smem > cache.smem) {
      cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)smem);
      if (err != cudaSuccess) return err;
      int dev = 0;
      if ((err = cudaGetDevice(&dev)) != cudaSuccess) return err;
      if ((err = cudaDeviceGetAttribute(&cache.sms, cudaDevAttrMultiProcessorCount, dev)) !=
          cudaSuccess)
        return err;
      if ((err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&cache.per_sm, kern, kThreads,
                                                               smem)) != cudaSuccess)
        return err;
      cache.smem = smem;
    }
    per_sm = std::max(1, cache.per_sm);
    sms = cache.sms;
  }
  const int routed_slots = std::min(p.E, p.T * p.k), shared_slots = p.has_shared ? 1 : 0;
  const int max_slots = part == 1 ? routed_slots
                                  : (part == 2 ? shared_slots : routed_slots + shared_slots);
  const long long units = (long long)max_slots * (N / kRowsCTA);
  const int grid = (int)std::max(1LL, std::min<long long>(units, (long long)per_sm * sms));
  kern<<<grid, kThreads, smem, st>>>(p, part);
  return cudaGetLastError();
}

template <bool GATE_UP>
static cudaError_t launch_part(const Plan& p, int fmt, int part, cudaStream_t st) {
  switch (fmt) {
    case 4: return launch_one<4, GATE_UP>(p, part, st);
    case 8: return launch_one<8, GATE_UP>(p, part, st);
    default: return launch_one<16, GATE_UP>(p, part, st);
  }
}

// One launch for both banks when they share a format; otherwise the routed experts and the
// shared expert in two launches, each with its own format.
template <bool GATE_UP>
static cudaError_t launch_fmt(const Plan& p, cudaStream_t st) {
  if (!p.has_shared || p.shared.fmt == p.routed.fmt) return launch_part<GATE_UP>(p, p.routed.fmt, 0, st);
  const cudaError_t err = launch_part<GATE_UP>(p, p.routed.fmt, 1, st);
  if (err != cudaSuccess) return err;
  return launch_part<GATE_UP>(p, p.shared.fmt, 2, st);
}

cudaError_t launch_gemv_gate_up(const Plan& p, cudaStream_t st) { return launch_fmt<true>(p, st); }
cudaError_t launch_gemv_down(const Plan& p, cudaStream_t st) { return launch_fmt<false>(p, st); }

}  // namespace moe
