// The NVFP4 (W4A4) variant of the routed experts on the FP4 tensor cores: ModelOpt NVFP4 on
// the routed experts, weights and the activations entering them in 4-bit floating point, the
// shared expert kept BF16 (Anvil serving benchmarks, "Qwen3.8 Flash Next", section
// "Quantization boundary"). Routing, the plan, the shared expert and the combine are those of
// the integer layer; what changes is the grouped FFN of the routed experts:
//
//   nv_quant_x   x (bf16) -> NVFP4 per grouped row (the token's row of x): E2M1 codes
//                [T*k][d/2], E4M3 block scales by token tile, fp32 row scales
//   nv_grouped<gate/up>   D_g = Wg x, D_u = Wu x with tcgen05.mma kind::mxf4nvf4 (E2M1
//                operands, an E4M3 scale per 16 K values on both sides, applied by the tensor
//                core, fp32 accumulate); epilogue h = silu(g_w g_x D_g) * (g_w g_x D_u), fp32
//   nv_quant_h   h (fp32) -> NVFP4 per grouped row, as for x
//   nv_grouped<down>      y = g_w g_h (Wd h) -> fp32 y_assign rows, combined as usual
//
// Activation quantisation (per row v of K values): g = amax(v) / (6 * 448); per block of 16,
// s = E4M3(amax_block / (6 g)) rounded to nearest even and saturated at 448; the elements
// E2M1(v / (s * g)) rounded to nearest even and saturated at 6. Every step is one IEEE fp32
// operation, so the codes are a function of the row alone, whatever the call's other rows.
// Products of E2M1 values and E4M3 scales are exact in fp32; the tensor core sums them in
// fp32.
//
// GEMM kernel (one persistent CTA per SM, 6 warps; units as on the integer tensor-core path:
// (expert slot, 128-row weight tile, token tile of up to 64 rows), weight tile fastest):
//   warp 0      TMA producer: per stage of 256 K values, the weight tile(s) [128 rows x 128
//               bytes, 128-byte swizzle], the token tile [rows x 128 bytes], and the block
//               scales of both (bulk copies of 2 KB: four K steps of 512 bytes each)
//   warp 1      TMEM owner and MMA issuer (one elected lane): per stage, the block scales
//               into tensor memory (tcgen05.cp 32x128b.warpx4, one per K step and operand),
//               then the MMAs, then a commit that releases the stage
//   warps 2-5   epilogue: tcgen05.ld of 32 TMEM lanes each
// TMEM: accumulator buffers (gate/up: two of 128 columns, gate then up; down: two of 64),
// then the scale columns (4 per K step and operand). Scale columns are reused stage after
// stage: the copies and MMAs of one thread execute in issue order.
// Every wait is bounded; a timeout sets the status word, and every role stops.
#include <cuda_fp4.h>
#include <cuda_fp8.h>
#include <cuda_fp16.h>

#include <cstring>

#include "tc_common.cuh"

namespace moe {

namespace {

constexpr int kNvThreads = 192;
constexpr int kNvKS = 256;              // K values per stage: 128 bytes of a row
constexpr int kNvSteps = kNvKS / 64;    // MMA K steps per stage
constexpr int kSfChunk = 512;           // scales of 128 rows x one K step of 64
constexpr float kAmaxE2M1 = 6.f, kAmaxE4M3 = 448.f;

template <bool GATE_UP> struct NvCfg {
  static constexpr int NM = GATE_UP ? 2 : 1;               // weight matrices a unit
  static constexpr int W_BYTES = kTcM * 128;                // one weight tile stage
  static constexpr int X_BYTES = kTcNMax * 128;             // one token tile stage
  static constexpr int SF_BYTES = kNvSteps * kSfChunk;      // one operand's scales a stage
  static constexpr int STAGE = NM * W_BYTES + X_BYTES + (NM + 1) * SF_BYTES;
  static constexpr int NS = GATE_UP ? 4 : 6;                // stages
  static constexpr int ACC_COLS = NM * kTcNMax;             // one accumulator buffer
  static constexpr int SF_COL0 = 2 * ACC_COLS;              // after two accumulator buffers
  static_assert(STAGE % 1024 == 0, "stages keep the 1024-byte alignment of swizzled tiles");
  static_assert(SF_COL0 + (NM + 1) * 4 * kNvSteps <= 512, "TMEM budget");
};

struct NvMaps {
  CUtensorMap w[2];         // weight matrices of the launch (gate, up | down)
  CUtensorMap act[kBoxes];  // token rows (quantised x | quantised h), boxes of 16/32/64 rows
  int box_rows[kBoxes];
};

// ---------------------------------------------------------------- conversions

// Non-negative v -> E4M3 code, nearest even, saturating at 448.
__device__ __forceinline__ uint32_t e4m3_code(float v) {
  return (uint32_t)__nv_cvt_float_to_fp8(v, __NV_SATFINITE, __NV_E4M3);
}
__device__ __forceinline__ float e4m3_value(uint32_t code) {
  const __half_raw h = __nv_cvt_fp8_to_halfraw((__nv_fp8_storage_t)code, __NV_E4M3);
  return __half2float(__half(h));
}
// Two values -> one byte of E2M1 codes (lo in bits 0..3), nearest even, saturating at 6.
__device__ __forceinline__ uint32_t e2m1x2_code(float lo, float hi) {
  return (uint32_t)__nv_cvt_float2_to_fp4x2(make_float2(lo, hi), __NV_E2M1, cudaRoundNearest);
}

// Byte offset of the scale of row n (< 128) of a token or weight tile, block j (< 4) of a K
// step, inside that step's 512-byte chunk (the order tcgen05.cp 32x128b takes: 32 rows of 16
// bytes, row i holding rows i, i+32, i+64, i+96 of the tile, four blocks each).
__device__ __forceinline__ int sf_pos(int n, int j) { return 16 * (n & 31) + 4 * (n >> 5) + j; }

// One block of 16 values quantised with the row scale g: the E4M3 code of the block scale and
// the 8 bytes of E2M1 codes (element 2i in the low nibble of byte i).
__device__ __forceinline__ uint32_t quant_block(const float (&v)[16], float g, float denom,
                                                uint2* codes) {
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(v[i]));
  const float ratio = denom > 0.f ? __fdiv_rn(amax, denom) : 0.f;
  const uint32_t sc = e4m3_code(ratio);
  const float scale = __fmul_rn(e4m3_value(sc), g);
  uint32_t b[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float q0 = scale > 0.f ? __fdiv_rn(v[2 * i], scale) : 0.f;
    const float q1 = scale > 0.f ? __fdiv_rn(v[2 * i + 1], scale) : 0.f;
    b[i] = scale > 0.f ? e2m1x2_code(q0, q1) : 0u;
  }
  codes->x = b[0] | (b[1] << 8) | (b[2] << 16) | (b[3] << 24);
  codes->y = b[4] | (b[5] << 8) | (b[6] << 16) | (b[7] << 24);
  return sc;
}

// Where grouped row r's scales go: token tile (schedule numbering) and row within it. The
// row's expert is the e with offsets[e] <= r < offsets[e + 1] (a binary search).
__device__ __forceinline__ void row_tile(const Plan& p, const TcSched& S, int r, int* mt, int* n) {
  int lo = 0, hi = p.E;  // offsets[lo] <= r < offsets[hi]
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (__ldg(p.offsets + mid) <= r) lo = mid;
    else hi = mid;
  }
  const int i = r - __ldg(p.offsets + lo);
  *mt = S.expert_mt[lo] + i / kTcNMax;
  *n = i % kTcNMax;
}

// ---------------------------------------------------------------- activation quantisers

// One warp per grouped row r: x[perm[r] / k] (bf16, exact in fp32) quantised (a token's k
// rows quantise to the same codes). Lane l takes blocks l, l + 32, ...
__global__ void __launch_bounds__(256) nv_quant_x_kernel(Plan p, TcSched S) {
  pdl_wait();
  const int lane = threadIdx.x & 31;
  const int warps = blockDim.x >> 5;
  const int nb = p.d / 16;              // blocks a row
  const int KS = p.d / 64;              // K steps a row
  const int rows = p.T * p.k;
  for (int r = blockIdx.x * warps + (int)(threadIdx.x >> 5); r < rows; r += gridDim.x * warps) {
    const int t = p.perm[r] / p.k;
    const uint4* xr = reinterpret_cast<const uint4*>(p.x + (size_t)t * p.d);
    float amax = 0.f;
    for (int b = lane; b < nb; b += 32) {
      const uint4 a = xr[2 * b], c = xr[2 * b + 1];
      const uint32_t w[8] = {a.x, a.y, a.z, a.w, c.x, c.y, c.z, c.w};
#pragma unroll
      for (int i = 0; i < 8; ++i)
        amax = fmaxf(amax, fmaxf(fabsf(__uint_as_float(w[i] << 16)),
                                 fabsf(__uint_as_float(w[i] & 0xffff0000u))));
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    const float g = __fdiv_rn(amax, kAmaxE2M1 * kAmaxE4M3);
    const float denom = __fmul_rn(kAmaxE2M1, g);
    int mt, n;
    row_tile(p, S, r, &mt, &n);
    uint2* dst = reinterpret_cast<uint2*>(p.xq + (size_t)r * (p.d / 2));
    uint8_t* sf = p.xsf + (size_t)mt * KS * kSfChunk;
    for (int b = lane; b < nb; b += 32) {
      const uint4 a = xr[2 * b], c = xr[2 * b + 1];
      const uint32_t w[8] = {a.x, a.y, a.z, a.w, c.x, c.y, c.z, c.w};
      float v[16];
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        v[2 * q] = __uint_as_float(w[q] << 16);
        v[2 * q + 1] = __uint_as_float(w[q] & 0xffff0000u);
      }
      uint2 cd;
      const uint32_t sc = quant_block(v, g, denom, &cd);
      dst[b] = cd;
      sf[(size_t)(b >> 2) * kSfChunk + sf_pos(n, b & 3)] = (uint8_t)sc;
    }
    if (lane == 0) p.gx[r] = g;
  }
  pdl_trigger();
}

// One warp per grouped row: h (fp32) quantised.
__global__ void __launch_bounds__(256) nv_quant_h_kernel(Plan p, TcSched S) {
  pdl_wait();
  const int lane = threadIdx.x & 31;
  const int warps = blockDim.x >> 5;
  const int nb = p.f / 16;
  const int KS = p.f / 64;
  const int rows = p.T * p.k;
  for (int r = blockIdx.x * warps + (int)(threadIdx.x >> 5); r < rows; r += gridDim.x * warps) {
    const float4* hr = reinterpret_cast<const float4*>(p.h32 + (size_t)r * p.f);
    float amax = 0.f;
    for (int b = lane; b < nb; b += 32) {
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float4 v = hr[4 * b + q];
        amax = fmaxf(amax, fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w))));
      }
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    const float g = __fdiv_rn(amax, kAmaxE2M1 * kAmaxE4M3);
    const float denom = __fmul_rn(kAmaxE2M1, g);
    int mt, n;
    row_tile(p, S, r, &mt, &n);
    uint2* dst = reinterpret_cast<uint2*>(p.hq + (size_t)r * (p.f / 2));
    uint8_t* sf = p.hsf + (size_t)mt * KS * kSfChunk;
    for (int b = lane; b < nb; b += 32) {
      float v[16];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float4 u = hr[4 * b + q];
        v[4 * q] = u.x;
        v[4 * q + 1] = u.y;
        v[4 * q + 2] = u.z;
        v[4 * q + 3] = u.w;
      }
      uint2 c;
      const uint32_t sc = quant_block(v, g, denom, &c);
      dst[b] = c;
      sf[(size_t)(b >> 2) * kSfChunk + sf_pos(n, b & 3)] = (uint8_t)sc;
    }
    if (lane == 0) p.gh[r] = g;
  }
  pdl_trigger();
}

// fp32 rows -> NVFP4 in natural order (codes [rows][K/2], scales [rows][K/16], g [rows]): the
// quantiser of the kernels above, for callers and tests. One warp per row.
__global__ void __launch_bounds__(256) nv_quant_rows_kernel(const float* __restrict__ v, int rows,
                                                            int K, uint8_t* __restrict__ codes,
                                                            uint8_t* __restrict__ scales,
                                                            float* __restrict__ gout) {
  const int lane = threadIdx.x & 31;
  const int warps = blockDim.x >> 5;
  const int nb = K / 16;
  for (int r = blockIdx.x * warps + (int)(threadIdx.x >> 5); r < rows; r += gridDim.x * warps) {
    const float4* vr = reinterpret_cast<const float4*>(v + (size_t)r * K);
    float amax = 0.f;
    for (int b = lane; b < nb; b += 32) {
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float4 u = vr[4 * b + q];
        amax = fmaxf(amax, fmaxf(fmaxf(fabsf(u.x), fabsf(u.y)), fmaxf(fabsf(u.z), fabsf(u.w))));
      }
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    const float g = __fdiv_rn(amax, kAmaxE2M1 * kAmaxE4M3);
    const float denom = __fmul_rn(kAmaxE2M1, g);
    for (int b = lane; b < nb; b += 32) {
      float x[16];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float4 u = vr[4 * b + q];
        x[4 * q] = u.x;
        x[4 * q + 1] = u.y;
        x[4 * q + 2] = u.z;
        x[4 * q + 3] = u.w;
      }
      uint2 c;
      const uint32_t sc = quant_block(x, g, denom, &c);
      reinterpret_cast<uint2*>(codes + (size_t)r * (K / 2))[b] = c;
      scales[(size_t)r * nb + b] = (uint8_t)sc;
    }
    if (lane == 0) gout[r] = g;
  }
}

// Weight scales, natural order [mats][rows][K/16] -> chunks [mats][rows/128][K/64][512]: one
// thread per (row, K step), 4 bytes in, 4 bytes out.
__global__ void __launch_bounds__(256) nv_pack_scales_kernel(const uint32_t* __restrict__ src,
                                                             uint32_t* __restrict__ dst,
                                                             long long n_rows, int KS) {
  const long long total = n_rows * KS;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < total;
       i += (long long)gridDim.x * blockDim.x) {
    const long long row = i / KS;
    const int ks = (int)(i % KS);
    const long long tile = row >> 7;
    const int n = (int)(row & 127);
    const uint32_t v = src[i];  // the four block scales of (row, ks), blocks in byte order
    dst[((tile * KS + ks) * kSfChunk + 16 * (n & 31) + 4 * (n >> 5)) / 4] = v;
  }
}

// ---------------------------------------------------------------- PTX wrappers

// Block-scaled FP4 MMA, D[128 x N] (+)= (A . sfa) (B . sfb)^T, A and B E2M1 in shared
// memory (K-major), scales E4M3 per 16 K values in tensor memory. Warp-level (one elected
// lane issues).
__device__ __forceinline__ void umma_nvf4_warp(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                               uint32_t idesc, uint32_t sfa, uint32_t sfb,
                                               uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred e, p;\n\telect.sync _|e, 0xffffffff;\n\tsetp.ne.b32 p, %6, 0;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%4], "
      "[%5], p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(sfa), "r"(sfb), "r"(accumulate)
      : "memory");
}

// 32 rows x 16 bytes of shared memory -> TMEM lanes 0..31 (and, repeated, 32..63, 64..95,
// 96..127), 4 columns from taddr. Warp-level.
__device__ __forceinline__ void tmem_cp_sf_warp(uint32_t taddr, uint64_t sdesc) {
  asm volatile(
      "{\n\t.reg .pred e;\n\telect.sync _|e, 0xffffffff;\n\t"
      "@e tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;\n\t}" ::"r"(taddr),
      "l"(sdesc)
      : "memory");
}

// Shared-memory descriptor of a scale chunk: no swizzle, K-major, 8-row core matrices of
// 16-byte rows, consecutive (128 bytes apart); one 16-byte column.
__device__ __forceinline__ uint64_t sf_desc(uint32_t saddr) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFF);
  d |= (uint64_t)(128 >> 4) << 32;  // SBO: the next 8 rows
  d |= (uint64_t)1 << 46;           // version (sm_100)
  return d;                         // layout type 0: no swizzle
}

// Instruction descriptor, kind::mxf4nvf4: A and B E2M1 (K-major), D fp32, E4M3 scales
// (scale vector of 4 per K step of 64), M = 128, N = n.
__host__ __device__ constexpr uint32_t umma_idesc_nvf4(int n) {
  return (1u << 7) | (1u << 10) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(kTcM >> 4) << 24);
}

// ---------------------------------------------------------------- the GEMM kernel

template <bool GATE_UP>
__global__ void __launch_bounds__(kNvThreads, 1)
    nv_grouped_kernel(const __grid_constant__ NvMaps maps, Plan p, TcSched S) {
  using C = NvCfg<GATE_UP>;
  constexpr int NM = C::NM;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int K = GATE_UP ? p.d : p.f;
  const int N = GATE_UP ? p.f : p.d;
  const int KS = K / 64;                 // K steps a row
  const int n_stages = K / kNvKS;        // stages a unit
  const int n_tiles = N / kTcM;
  int32_t* sched = reinterpret_cast<int32_t*>(smem + C::NS * C::STAGE);
  uint64_t* bars = reinterpret_cast<uint64_t*>(sched + 4 * (p.E + 2));
  uint64_t* full = bars;                 // [NS]
  uint64_t* empty = full + C::NS;        // [NS]
  uint64_t* acc_full = empty + C::NS;    // [2]
  uint64_t* acc_empty = acc_full + 2;    // [2]
  uint64_t* drain = acc_empty + 2;       // [1]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::NS; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 4);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) tmem_alloc(tmem_slot, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  pdl_wait();
  const int n_active = p.active[0];
  TcSched Ss;
  Ss.slot_rows = sched;
  Ss.slot_row0 = sched + (p.E + 2);
  Ss.slot_expert = sched + 2 * (p.E + 2);
  Ss.mt_prefix = sched + 3 * (p.E + 2);
  Ss.expert_mt = nullptr;
  for (int i = threadIdx.x; i <= n_active; i += blockDim.x) {
    Ss.mt_prefix[i] = S.mt_prefix[i];
    if (i < n_active) {
      Ss.slot_rows[i] = S.slot_rows[i];
      Ss.slot_row0[i] = S.slot_row0[i];
      Ss.slot_expert[i] = S.slot_expert[i];
    }
  }
  __syncthreads();
  const int total = Ss.mt_prefix[n_active] * n_tiles;  // routed units only
  auto fail = [&](int site) {
    set_timeout(p.status, site);
    *abort_flag = 1;
  };

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      const uint8_t* sfw[2];
      for (int mi = 0; mi < NM; ++mi)
        sfw[mi] = reinterpret_cast<const uint8_t*>(p.routed.s[GATE_UP ? mi : 2]);
      const uint8_t* sfx = GATE_UP ? p.xsf : p.hsf;
      int it = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < total && ok && !*abort_flag; u += gridDim.x) {
        const TcUnit t = tc_unit(Ss, n_active, n_tiles, u);
        const int wrow = t.e * N + t.ntile * kTcM;
        const int bx = box_index(t.nrows);
        const int mt = Ss.mt_prefix[t.slot] + t.mtile;
        const uint32_t bytes = NM * C::W_BYTES + maps.box_rows[bx] * 128 + (NM + 1) * C::SF_BYTES;
        for (int st = 0; st < n_stages; ++st, ++it) {
          const int s = it % C::NS, use = it / C::NS;
          if (use > 0 && !mbar_wait(&empty[s], (use - 1) & 1)) {
            ok = false;
            break;
          }
          uint8_t* stage = smem + s * C::STAGE;
          mbar_arrive_expect_tx(&full[s], bytes);
          for (int mi = 0; mi < NM; ++mi)
            tma_load_2d(stage + mi * C::W_BYTES, &maps.w[mi], st * 128, wrow, &full[s]);
          uint8_t* xs = stage + NM * C::W_BYTES;
          tma_load_2d(xs, &maps.act[bx], st * 128, t.row0, &full[s]);
          uint8_t* sfs = xs + C::X_BYTES;
          for (int mi = 0; mi < NM; ++mi)
            bulk_g2s(sfs + mi * C::SF_BYTES,
                     sfw[mi] + ((size_t)(t.e * n_tiles + t.ntile) * KS + st * kNvSteps) * kSfChunk,
                     C::SF_BYTES, &full[s]);
          bulk_g2s(sfs + NM * C::SF_BYTES, sfx + ((size_t)mt * KS + st * kNvSteps) * kSfChunk,
                   C::SF_BYTES, &full[s]);
        }
      }
      if (!ok) fail(40);
      // every issued stage lands before the CTA may exit
      for (int j = (it > C::NS ? it - C::NS : 0); j < it; ++j)
        mbar_wait(&full[j % C::NS], (j / C::NS) & 1);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    int it = 0, tile = 0;
    bool aborted = false;
    for (int u = blockIdx.x; u < total && !aborted; u += gridDim.x, ++tile) {
      const TcUnit t = tc_unit(Ss, n_active, n_tiles, u);
      const int n_mma = (t.nrows + 15) & ~15;
      const uint32_t idesc = umma_idesc_nvf4(n_mma);
      const int b = tile & 1, buse = tile >> 1;
      if (buse > 0 && !mbar_wait(&acc_empty[b], (buse - 1) & 1)) aborted = true;
      aborted = __any_sync(0xffffffffu, aborted || *abort_flag);
      if (aborted) break;
      tc_fence_after();
      const uint32_t dacc = tmem + b * C::ACC_COLS;
      for (int st = 0; st < n_stages; ++st, ++it) {
        const int s = it % C::NS;
        bool ok = mbar_wait(&full[s], (it / C::NS) & 1);
        if (!__all_sync(0xffffffffu, ok)) {
          aborted = true;
          break;
        }
        tc_fence_after();
        const uint8_t* stage = smem + s * C::STAGE;
        const uint8_t* xs = stage + NM * C::W_BYTES;
        const uint8_t* sfs = xs + C::X_BYTES;
        // scales of this stage into TMEM: operand o (weights 0..NM-1, tokens NM), K step kk
        // at column SF_COL0 + 16 o + 4 kk
#pragma unroll
        for (int o = 0; o <= NM; ++o)
#pragma unroll
          for (int kk = 0; kk < kNvSteps; ++kk)
            tmem_cp_sf_warp(tmem + C::SF_COL0 + 16 * o + 4 * kk,
                            sf_desc(smem_u32(sfs + o * C::SF_BYTES + kk * kSfChunk)));
        const uint64_t bdesc = umma_desc_sw128(smem_u32(xs));
#pragma unroll
        for (int mi = 0; mi < NM; ++mi) {
          const uint64_t adesc = umma_desc_sw128(smem_u32(stage + mi * C::W_BYTES));
#pragma unroll
          for (int kk = 0; kk < kNvSteps; ++kk)
            umma_nvf4_warp(dacc + mi * kTcNMax, adesc + (uint64_t)(2 * kk),
                           bdesc + (uint64_t)(2 * kk), idesc,
                           tmem + C::SF_COL0 + 16 * mi + 4 * kk,
                           tmem + C::SF_COL0 + 16 * NM + 4 * kk, (st > 0 || kk > 0) ? 1u : 0u);
        }
        umma_commit_warp(&empty[s]);
      }
      if (aborted) break;
      umma_commit_warp(&acc_full[b]);
    }
    if (aborted) fail(41);
    // all issued MMAs and copies complete before TMEM and shared memory are released
    umma_commit_warp(drain);
    mbar_wait(drain, 0);
  } else {
    // ------------------------------------------------------------ epilogue (warps 2..5)
    const int quarter = warp & 3;          // TMEM lanes 32*quarter .. +31
    const int row = quarter * 32 + lane;   // weight row in the tile
    int tile = 0;
    for (int u = blockIdx.x; u < total && !*abort_flag; u += gridDim.x, ++tile) {
      const TcUnit t = tc_unit(Ss, n_active, n_tiles, u);
      const int b = tile & 1;
      if (!mbar_wait(&acc_full[b], (tile >> 1) & 1)) {
        fail(42);
        break;
      }
      tc_fence_after();
      const uint32_t lane_addr = tmem + ((uint32_t)(quarter * 32) << 16) + b * C::ACC_COLS;
      const int n = t.ntile * kTcM + row;  // output feature
      const float gw0 = p.routed.g[GATE_UP ? 0 : 2][t.e];
      const float gw1 = GATE_UP ? p.routed.g[1][t.e] : 0.f;
      const float* gact = GATE_UP ? p.gx : p.gh;
      for (int m0 = 0; m0 < t.nrows; m0 += 16) {
        float a0[16];
        tmem_ld16(lane_addr + m0, a0);
        if constexpr (GATE_UP) {
          float a1[16];
          tmem_ld16(lane_addr + kTcNMax + m0, a1);
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            if (m0 + j < t.nrows) {
              const int r = t.row0 + m0 + j;
              const float ga = gact[r];
              const float gate = a0[j] * (gw0 * ga);
              const float up = a1[j] * (gw1 * ga);
              p.h32[(size_t)r * p.f + n] = gate / (1.f + expf(-gate)) * up;
            }
          }
        } else {
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            if (m0 + j < t.nrows) {
              const int r = t.row0 + m0 + j;
              p.y_assign[(size_t)r * p.d + n] = a0[j] * (gw0 * gact[r]);
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[b]);
    }
  }

  // ------------------------------------------------------------ teardown
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
  pdl_trigger();
}

template <bool GATE_UP>
int nv_smem_bytes(int E) {
  using C = NvCfg<GATE_UP>;
  return C::NS * C::STAGE + 4 * (E + 2) * (int)sizeof(int32_t) + 256 + 1024;
}

cudaLaunchConfig_t make_cfg(int blocks, int threads, int smem, cudaStream_t st,
                            cudaLaunchAttribute* attr) {
  cudaLaunchConfig_t cfg;
  std::memset(&cfg, 0, sizeof(cfg));
  cfg.gridDim = dim3(blocks);
  cfg.blockDim = dim3(threads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cfg;
}

int sm_count() {
  static int sms = 0;
  static std::once_flag once;
  std::call_once(once, [] {
    int dev = 0;
    if (cudaGetDevice(&dev) == cudaSuccess)
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  });
  return sms;
}

template <bool GATE_UP>
cudaError_t launch_nv(const Plan& p, const TcSched& S, cudaStream_t st) {
  using C = NvCfg<GATE_UP>;
  const int K = GATE_UP ? p.d : p.f;
  const int N = GATE_UP ? p.f : p.d;
  NvMaps maps;
  std::memset(&maps, 0, sizeof(maps));
  for (int mi = 0; mi < C::NM; ++mi) {
    if (!make_map(&maps.w[mi], CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, p.routed.w[GATE_UP ? mi : 2],
                  K / 2, (uint64_t)p.E * N, 128, kTcM, CU_TENSOR_MAP_SWIZZLE_128B))
      return cudaErrorInvalidValue;
  }
  const uint8_t* act = GATE_UP ? p.xq : p.hq;
  const uint64_t rows = (uint64_t)p.T * p.k;
  for (int bx = 0; bx < kBoxes; ++bx) {
    const uint32_t br = (uint32_t)std::min<uint64_t>(16u << bx, rows);
    maps.box_rows[bx] = (int)br;
    if (!make_map(&maps.act[bx], CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, act, K / 2, rows, 128, br,
                  CU_TENSOR_MAP_SWIZZLE_128B))
      return cudaErrorInvalidValue;
  }
  auto kern = nv_grouped_kernel<GATE_UP>;
  const int smem = nv_smem_bytes<GATE_UP>(p.E);
  if (smem > 227 * 1024) return cudaErrorInvalidValue;
  static std::once_flag once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(once, [&] {
    attr_err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024);
  });
  if (attr_err != cudaSuccess) return attr_err;
  const int sms = sm_count();
  if (sms <= 0) return cudaErrorInvalidDevice;
  cudaLaunchAttribute attr[1];
  cudaLaunchConfig_t cfg = make_cfg(sms, kNvThreads, smem, st, attr);
  return cudaLaunchKernelEx(&cfg, kern, maps, p, S);
}

}  // namespace

cudaError_t launch_nv_quant_rows(const float* v, int rows, int K, uint8_t* codes, uint8_t* scales,
                                 float* g, cudaStream_t st) {
  const int blocks = std::max(1, std::min(1184, (rows + 7) / 8));
  nv_quant_rows_kernel<<<blocks, 256, 0, st>>>(v, rows, K, codes, scales, g);
  return cudaGetLastError();
}

size_t nv_tile_cap(int T, int k, int E) {
  const size_t n = (size_t)T * k;
  return n / kTcNMax + 1 + std::min<size_t>((size_t)E, n);
}

bool nv_supported(const Plan& p) {
  return get_encoder() != nullptr && p.d % kNvKS == 0 && p.f % kNvKS == 0 &&
         p.d % kTcM == 0 && p.f % kTcM == 0 && p.d <= 8192 && p.f <= 8192 &&
         nv_smem_bytes<true>(p.E) <= 227 * 1024 && nv_smem_bytes<false>(p.E) <= 227 * 1024;
}

cudaError_t launch_nv_quant_x(const Plan& p, const TcSched& S, cudaStream_t st) {
  const long long rows = (long long)p.T * p.k;
  const int blocks = (int)std::max(1LL, std::min(1184LL, (rows + 7) / 8));
  cudaLaunchAttribute attr[1];
  cudaLaunchConfig_t cfg = make_cfg(blocks, 256, 0, st, attr);
  return cudaLaunchKernelEx(&cfg, nv_quant_x_kernel, p, S);
}

cudaError_t launch_nv_quant_h(const Plan& p, const TcSched& S, cudaStream_t st) {
  const long long rows = (long long)p.T * p.k;
  const int blocks = (int)std::max(1LL, std::min(1184LL, (rows + 7) / 8));
  cudaLaunchAttribute attr[1];
  cudaLaunchConfig_t cfg = make_cfg(blocks, 256, 0, st, attr);
  return cudaLaunchKernelEx(&cfg, nv_quant_h_kernel, p, S);
}

cudaError_t launch_nv_gate_up(const Plan& p, const TcSched& S, cudaStream_t st) {
  return launch_nv<true>(p, S, st);
}
cudaError_t launch_nv_down(const Plan& p, const TcSched& S, cudaStream_t st) {
  return launch_nv<false>(p, S, st);
}

cudaError_t launch_nv_pack_scales(const uint8_t* src, uint8_t* dst, int n_mats, int rows, int K,
                                  cudaStream_t st) {
  const long long n_rows = (long long)n_mats * rows;
  const int KS = K / 64;
  const long long total = n_rows * KS;
  const int blocks = (int)std::max(1LL, std::min(4736LL, (total + 255) / 256));
  nv_pack_scales_kernel<<<blocks, 256, 0, st>>>(reinterpret_cast<const uint32_t*>(src),
                                                reinterpret_cast<uint32_t*>(dst), n_rows, KS);
  return cudaGetLastError();
}

}  // namespace moe
