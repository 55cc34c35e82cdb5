// Grouped expert GEMMs on the 5th-generation tensor cores (tcgen05 + TMEM), for calls with
// many rows per expert (prefill slabs): the dense contraction of each expert's rows with its
// dequantised weights (Qwen3.8-Flash-Next-Dual-GPU README, "Dedicated prefill lane", steps
// 2-4: grouped W4/W8-A16 tensor-core products over expert-major rows, one fp32 output per
// assignment; TandemLLM docs, "17 Qwen3.8-Flash-Next", §17.4: rows sorted by expert, one
// matrix product over each expert's rows).
//
// Orientation ("swap AB"): D[n][m] = sum_k W[n][k] X[m][k]; the weights are the M = 128
// operand (128 rows of one expert matrix), the expert's token rows are N (16..128), K is
// walked in chunks of 64. D lives in TMEM (lane = weight row, column = token).
//
// One persistent CTA per SM, warp roles:
//   warp 0      TMA producer of the raw weight stages [128 rows x 128 bytes] (int4/int8/
//               bf16, 128-byte swizzle) and each unit's group scales
//   warp 1      TMEM owner and MMA issuer (the whole warp, one elected lane issuing):
//               tcgen05.mma kind::f16, fp32 accumulate; warp 14 issues in parallel into a
//               separate accumulator (gate/up: the up projection; down: half the K steps)
//   warps 2-9   dequantisers, two groups of four taking alternate steps of two 64-K chunks:
//               W = fp16(q * s) written straight from registers into TMEM (tcgen05.st),
//               where the MMA reads its A operand; each ready chunk is announced on a named
//               barrier per A stage; shared memory carries only the raw weights and the
//               activations
//   warps 10-13 epilogue: tcgen05.ld of their 32 TMEM lanes; gate/up: h = silu(g) * u ->
//               fp16 rows; down: fp32 rows
//   warp 15     TMA producer of the activation tiles (warp 0 streams the weights)
// Operands are fp16 (kind::f16, fp32 accumulate): the activations (bf16 inputs) convert to
// fp16 exactly in fp16's range, and q * s rounds once with an 11-bit significand, eight
// times finer than bf16. Activations and h outside fp16's range set a device status flag.
// Rings: weights (TMA -> dequant), activations (TMA -> MMA), A (dequant -> MMA, in TMEM;
// announced on a named barrier per stage), accumulator (MMA -> epilogue, in
// TMEM). TMEM columns: the accumulator buffers from column 0 (buffer b: gate at 128 b, up at
// 128 b + 64), then the A stages. Every wait is bounded; a timeout sets the status word and
// every role drains and exits (TMEM is freed by its owner).
//
// Work units (slot, n-tile, m-tile) are ordered with the m-tile fastest, and CTAs take
// them round-robin, so the m-tiles of one weight tile run at the same time on neighbouring
// SMs and re-read that tile from L2 rather than HBM.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <cstring>
#include <mutex>

#include <cuda_fp16.h>

#include "tc_common.cuh"

namespace moe {

constexpr int kTcThreads = 512;  // 16 warps
constexpr int kDqWarps = 8;       // dequantisers (two threads per weight row)
constexpr int kIssuers = 2;       // MMA issuing warps (1 and 14)
// threads of one chunk's ready barrier: a dequantiser group of four warps and the issuers
constexpr int kReadyThreads = 32 * (kDqWarps / 2 + kIssuers);
constexpr int kTcBK = 64;      // K per chunk (one 128-byte swizzle span of bf16)

struct TcMaps {
  CUtensorMap w[2][2];          // [bank: routed, shared][matrix: gate|down, up]
  CUtensorMap act[2][kBoxes];   // [source: grouped rows, shared-expert rows][box]
  int box_rows[2][kBoxes];      // rows per activation box (16 << box, at most the source's)
};

template <int FMT, bool GATE_UP, int ACC> struct TcCfg {
  static constexpr int NM = GATE_UP ? 2 : 1;
  // A weight stage is 128 bytes of each of 128 rows (one 128-byte swizzle span: full L2
  // lines per row and conflict-free reads), i.e. KW = 256 / 128 / 64 K values for int4 /
  // int8 / bf16, walked by the dequantisers in SUB chunks of kTcBK.
  static constexpr int RAW_ROW = 128;                // raw bytes of one row per stage
  static constexpr int KW = RAW_ROW * 8 / FMT;       // K values per stage
  static constexpr int SUB = KW / kTcBK;             // kTcBK chunks per stage
  static constexpr int RAW = kTcM * RAW_ROW;         // one raw matrix stage
  static constexpr int XB = kTcNMax * kTcBK * 2;     // activation stage bytes
  // Ring depths: the weight ring is deep (HBM latency) and is released by the dequantisers
  // as soon as they have read it; the activation ring (mostly L2 hits) by the tensor core.
  static constexpr int WB = NM * RAW;                // weight stage bytes
  static constexpr int W_BUDGET = (GATE_UP ? 128 : 96) * 1024;
  static constexpr int NW = W_BUDGET / WB > 16 ? 16 : W_BUDGET / WB;
  // TMEM: ACC accumulator buffers of 128 columns (two 64-column accumulators each) from
  // column 0, then the A stages. One accumulator buffer leaves room for a deeper gate/up A
  // ring, which lets the dequantisers run ahead of the MMAs; the MMAs of a unit then wait
  // for the epilogue to have read the previous unit. That pause grows with the unit's rows,
  // so calls with many rows per expert take two buffers (measured on B200: prefill 523 vs
  // 578 us with one, a 4096-token call 1232 vs 1322 us with two).
  static constexpr int ACC_BUFS = ACC;
  static constexpr int NX = GATE_UP ? (ACC == 1 ? 6 : 4) : 8;  // activation stages (= A stages)
  static constexpr int A_COLS = NM * (kTcBK / 2);    // TMEM columns of one A stage
  static constexpr int NA = NX;                      // A stages in TMEM
  static constexpr int A_COL0 = ACC_BUFS * 128;
  static_assert(A_COL0 + NA * A_COLS <= 512, "TMEM budget");
  static_assert(NX <= 15, "one named barrier per stage (ids 1..15)");
  // layout (1024-byte aligned pieces first)
  static constexpr int X_OFF = 0;
  static constexpr int R_OFF = X_OFF + NX * XB;
  static constexpr int S_OFF = R_OFF + NW * WB;      // then: unit scales, schedule, barriers
  static_assert(S_OFF + 32 * 1024 <= 227 * 1024, "shared memory budget");
};

// Runtime part of the shared-memory layout: per-unit scale blocks (double buffered) of
// kTcM rows x K/128 bf16 per matrix, the schedule cache and the barriers.
struct TcSmem {
  int sb;                       // bytes of one matrix's scale block
  int sched_off, bar_off, total;
};

template <int FMT, bool GATE_UP, int ACC>
__host__ __device__ inline TcSmem tc_smem(int K, int E) {
  using C = TcCfg<FMT, GATE_UP, ACC>;
  TcSmem m;
  m.sb = (FMT == 16) ? 0 : kTcM * (K / kGroup) * 2;
  m.sched_off = C::S_OFF + 2 * C::NM * m.sb;
  m.bar_off = m.sched_off + 4 * (E + 2) * (int)sizeof(int32_t);
  m.bar_off = (m.bar_off + 15) & ~15;
  m.total = m.bar_off + 512 + 1024;  // barriers and flags, 1024 bytes of alignment slack
  return m;
}


// Warp-level forms: the whole (converged) warp executes them and one elected lane issues.
// Issuing from a converged warp costs a fraction of issuing from a lone lane of a diverged
// warp (about 17 against 46 cycles per M = 128, N = 16 MMA). elect.sync picks the lowest
// active lane, the same thread every time, so the MMAs and their commits stay in one
// thread's issue order.
__device__ __forceinline__ void umma_f16_ts_warp(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc,
                                                 uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred e, p;\n\telect.sync _|e, 0xffffffff;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// 32 consecutive 32-bit columns of this thread's TMEM lane <- registers (one wide
// instruction: every tcgen05 instruction has a sizeable fixed issue cost).
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,"
      "%13,%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
      "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]),
      "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]),
      "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}

__device__ __forceinline__ void tmem_st_wait() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}
// Instruction descriptor: D fp32, A and B fp16, both K-major, M = 128, N = n.
__host__ __device__ constexpr uint32_t umma_idesc_f16(int n) {
  return (1u << 4) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(kTcM >> 4) << 24);
}

// K order of the fp16 operands the tensor core reads. For int4 weights the dequantisers
// produce K pairs interleaved by four inside each aligned group of 8 (operand position 2i holds
// K 8m+i, position 2i+1 holds K 8m+i+4), so the activation rows multiplied with such a bank
// (x rows for gate/up, h rows for down) are stored in that order too; other formats keep K in
// order. A shared permutation of K leaves the contraction unchanged.
__host__ __device__ __forceinline__ bool interleaved_k(int fmt) { return fmt == 4; }

// Operand position of K index n (the position within its aligned group of 8 changes only).
__device__ __forceinline__ int k_position(int n, bool interleave) {
  const int i = n & 7;
  return interleave ? ((n & ~7) | ((i & 3) << 1) | (i >> 2)) : n;
}

// Gathers the activation rows in fp16 (xg[r] = x[perm[r] / k] for the T*k grouped rows, then
// xg[T*k + t] = x[t] for the shared expert; rows from row_begin on) and, in CTA 0, builds the
// unit schedule.
__global__ void __launch_bounds__(256) tc_prep_kernel(Plan p, TcSched S, uint16_t* xg,
                                                      int row_begin) {
  pdl_wait();
  if (blockIdx.x == 0) {
    __shared__ int s_units[kMaxE + 1];
    __shared__ int s_exp[kMaxE + 1];
    __shared__ int s_warp[8];
    const int n_active = p.active[0];
    const int n_slots = n_active + (p.has_shared ? 1 : 0);
    for (int s = threadIdx.x; s < n_slots; s += blockDim.x) {
      int rows, row0, e;
      if (s < n_active) {
        e = p.active[1 + s];
        row0 = p.offsets[e];
        rows = p.offsets[e + 1] - row0;
      } else {
        e = -1;
        row0 = 0;
        rows = p.T;
      }
      S.slot_rows[s] = rows;
      S.slot_row0[s] = row0;
      S.slot_expert[s] = e;
      s_units[s] = (rows + kTcNMax - 1) / kTcNMax;  // m-tiles of the slot
      s_exp[s] = e;
    }
    __syncthreads();
    // exclusive prefix of the m-tiles over the slots: thread i sums a run of `per` slots,
    // the runs are scanned across the block, then each thread writes its run's prefixes
    const int per = (n_slots + blockDim.x - 1) / blockDim.x;
    const int s0 = min(n_slots, (int)threadIdx.x * per), s1 = min(n_slots, s0 + per);
    int local = 0;
    for (int s = s0; s < s1; ++s) local += s_units[s];
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    int incl = local;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    if (lane == 31) s_warp[wid] = incl;
    __syncthreads();
    int base = 0;
    for (int w = 0; w < wid; ++w) base += s_warp[w];
    int run = base + incl - local;
    for (int s = s0; s < s1; ++s) {
      S.mt_prefix[s] = run;
      if (s < n_active) S.expert_mt[s_exp[s]] = run;
      run += s_units[s];
    }
    if (s1 == n_slots && s0 < s1) S.mt_prefix[n_slots] = run;
    if (n_slots == 0 && threadIdx.x == 0) S.mt_prefix[0] = 0;
  }
  {
    // one row per warp, lanes over the row's 16-byte pieces: the source token and the K order
    // are worked out once per row
    const int n = p.T * p.k;
    const int rows = n + (p.has_shared ? p.T : 0);
    const int chunks = p.d / 8;
    const int warps = blockDim.x / 32, lane = threadIdx.x & 31;
    bool range_ok = true;
    for (int r = row_begin + blockIdx.x * warps + (int)(threadIdx.x >> 5); r < rows;
         r += gridDim.x * warps) {
      const int t = (r < n) ? p.perm[r] / p.k : r - n;
      const bool il = interleaved_k((r < n) ? p.routed.fmt : p.shared.fmt);
      const uint4* src = reinterpret_cast<const uint4*>(p.x + (size_t)t * p.d);
      uint4* dst = reinterpret_cast<uint4*>(xg + (size_t)r * p.d);
      for (int c = lane; c < chunks; c += 32) {
        const uint4 v = src[c];
        const uint32_t vv[4] = {v.x, v.y, v.z, v.w};
        float e[8];  // K values 8c .. 8c+7
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          e[2 * q] = __uint_as_float(vv[q] << 16);
          e[2 * q + 1] = __uint_as_float(vv[q] & 0xffff0000u);
          range_ok &= (fabsf(e[2 * q]) <= 65504.f) && (fabsf(e[2 * q + 1]) <= 65504.f);
        }
        uint32_t o[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          __half2 h = il ? __floats2half2_rn(e[q], e[q + 4]) : __floats2half2_rn(e[2 * q], e[2 * q + 1]);
          o[q] = *reinterpret_cast<uint32_t*>(&h);
        }
        dst[c] = make_uint4(o[0], o[1], o[2], o[3]);
      }
    }
    if (!range_ok) set_status(p.status, DEV_RANGE);
  }
  pdl_trigger();
}

// ------------------------------------------------------------------ dequantisation

// Half `half` (K values 32*half .. 32*half+31) of chunk `s` (K values 64*s .. 64*s+63 of the
// stage) of one weight row -> 32 fp16 = W * s, two per register. The row is one 128-byte
// line of a stage written by the TMA with 128-byte swizzling: its 16-byte piece j sits at
// piece j ^ sw7 (sw7 = the row index mod 8).
//
// int4 registers hold K pairs interleaved by four inside each 8-value word: register i of
// word j = (K 8j+i, K 8j+i+4), i = 0..3 (interleaved_k; the activation rows carry the
// same order, so the contraction is unchanged). That order needs only masks: the integer
// pipe, which issues a warp instruction every other cycle, does 5 instructions per 8
// weights instead of 9 for the K-ordered pairs. int8 and bf16 registers hold K in order.
//
// Every conversion is exact up to one final rounding of q * s to fp16 (for scales in fp16's
// normal range): a nibble or byte placed in the mantissa of 1024.0 gives 1024 + u exactly,
// the offset is taken off exactly, and one fp16 multiply rounds q * s.
template <int FMT>
__device__ __forceinline__ void dequant_half_row(const uint8_t* row, int sw7, int s, int half,
                                                 float scale, uint32_t (&outr)[16]) {
  auto piece = [&](int j) {
    return *reinterpret_cast<const uint4*>(row + ((j ^ sw7) << 4));
  };
  auto h2 = [](uint32_t u) { return *reinterpret_cast<__half2*>(&u); };
  auto u32 = [](__half2 h) { return *reinterpret_cast<uint32_t*>(&h); };
  if constexpr (FMT == 4) {
    const uint4 q = piece(2 * s + half);
    const uint32_t w[4] = {q.x, q.y, q.z, q.w};
    const __half2 s2 = __float2half2_rn(scale);
    const __half2 off = __float2half2_rn(1032.f), sixteenth = __float2half2_rn(0.0625f),
                  off16 = __float2half2_rn(-72.f);
#pragma unroll
    for (int j = 0; j < 4; ++j) {  // word j = K values 8j .. 8j+7 of this half, nibble i = K 8j+i
      const uint32_t lo = w[j], hi = w[j] >> 8;
      // (n & 15) ^ 8 = q + 8 (offset binary) in the low mantissa bits of 1024.0, two at a time:
      // nibbles 0/4 (and 2/6 of hi) as 1024 + (q + 8), nibbles 1/5 (3/7) as 1024 + 16 (q + 8)
      const uint32_t a = (lo & 0x000F000Fu) ^ 0x64086408u;
      const uint32_t b = (lo & 0x00F000F0u) ^ 0x64806480u;
      const uint32_t c = (hi & 0x000F000Fu) ^ 0x64086408u;
      const uint32_t d = (hi & 0x00F000F0u) ^ 0x64806480u;
      outr[4 * j + 0] = u32(__hmul2(__hsub2(h2(a), off), s2));             // K 8j+0, 8j+4
      outr[4 * j + 1] = u32(__hmul2(__hfma2(h2(b), sixteenth, off16), s2));  // 8j+1, 8j+5
      outr[4 * j + 2] = u32(__hmul2(__hsub2(h2(c), off), s2));             // 8j+2, 8j+6
      outr[4 * j + 3] = u32(__hmul2(__hfma2(h2(d), sixteenth, off16), s2));  // 8j+3, 8j+7
    }
  } else if constexpr (FMT == 8) {
    const uint4 q0 = piece(4 * s + 2 * half);
    const uint4 q1 = piece(4 * s + 2 * half + 1);
    const uint32_t w[8] = {q0.x, q0.y, q0.z, q0.w, q1.x, q1.y, q1.z, q1.w};
    const __half2 s2 = __float2half2_rn(scale);
    const __half2 off = __float2half2_rn(1152.f);
#pragma unroll
    for (int j = 0; j < 8; ++j) {  // word j = K values 4j .. 4j+3
      const uint32_t u = w[j] ^ 0x80808080u;  // byte = q + 128
      // bytes 0, 1 (2, 3) with 0x64 above each: fp16 pair 1024 + q + 128, exact
      const uint32_t a = __byte_perm(u, 0x64646464u, 0x4140);
      const uint32_t b = __byte_perm(u, 0x64646464u, 0x4342);
      outr[2 * j] = u32(__hmul2(__hsub2(h2(a), off), s2));
      outr[2 * j + 1] = u32(__hmul2(__hsub2(h2(b), off), s2));
    }
  } else {
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint4 v = piece(4 * half + j);
      const uint32_t vv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int i = 0; i < 4; ++i)
        outr[4 * j + i] = u32(__floats2half2_rn(__uint_as_float(vv[i] << 16),
                                                __uint_as_float(vv[i] & 0xffff0000u)));
    }
  }
}

// ------------------------------------------------------------------ the kernel

template <int FMT, bool GATE_UP, int ACC>
__global__ void __launch_bounds__(kTcThreads, 1)
    tc_grouped_kernel(const __grid_constant__ TcMaps maps, Plan p, TcSched S, int part) {
  using C = TcCfg<FMT, GATE_UP, ACC>;
  constexpr int NM = C::NM;
  extern __shared__ uint8_t smem_raw[];
  // 1024-byte alignment for the swizzled tiles
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const TcSmem SL = tc_smem<FMT, GATE_UP, ACC>(GATE_UP ? p.d : p.f, p.E);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + SL.bar_off);
  uint64_t* full_w = bars;                   // [NW]
  uint64_t* empty_w = full_w + C::NW;        // [NW]
  uint64_t* full_x = empty_w + C::NW;        // [NX]
  uint64_t* empty_x = full_x + C::NX;        // [NX]
  uint64_t* acc_full = empty_x + C::NX;      // [2]
  uint64_t* acc_empty = acc_full + 2;        // [2]
  uint64_t* scale_full = acc_empty + 2;      // [2] one per unit parity
  uint64_t* scale_empty = scale_full + 2;    // [2]
  uint64_t* drain = scale_empty + 2;         // [1]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int K = GATE_UP ? p.d : p.f;
  const int N = GATE_UP ? p.f : p.d;
  const int G = K / kGroup;
  const int n_tiles = N / kTcM;
  const int n_chunks = K / kTcBK;
  const int n_wstages = (n_chunks + C::SUB - 1) / C::SUB;  // weight stages a unit

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::NW; ++s) {
      mbar_init(&full_w[s], 1);
      mbar_init(&empty_w[s], kDqWarps);  // dequant warps
    }
    // a chunk's activation stage and A stage are released together by one commit of each
    // MMA issuer (the rings have the same depth and advance in step); a chunk is announced
    // ready to the issuers on named barrier 1 + stage (kReadyThreads threads)
    for (int s = 0; s < C::NX; ++s) {
      mbar_init(&full_x[s], 1);
      mbar_init(&empty_x[s], kIssuers);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], kIssuers);  // one MMA commit per issuer
      mbar_init(&acc_empty[b], 4);      // 4 epilogue warps
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&scale_full[b], 1);
      mbar_init(&scale_empty[b], kDqWarps);
    }
    mbar_init(drain, kIssuers);
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
  const int n_slots = n_active + (p.has_shared ? 1 : 0);
  // schedule -> shared memory (every role looks units up many times)
  TcSched Ss;
  {
    int32_t* sc = reinterpret_cast<int32_t*>(smem + SL.sched_off);
    Ss.slot_rows = sc;
    Ss.slot_row0 = sc + (p.E + 2);
    Ss.slot_expert = sc + 2 * (p.E + 2);
    Ss.mt_prefix = sc + 3 * (p.E + 2);
    for (int i = threadIdx.x; i <= n_slots; i += blockDim.x) {
      Ss.mt_prefix[i] = S.mt_prefix[i];
      if (i < n_slots) {
        Ss.slot_rows[i] = S.slot_rows[i];
        Ss.slot_row0[i] = S.slot_row0[i];
        Ss.slot_expert[i] = S.slot_expert[i];
      }
    }
  }
  __syncthreads();
  // units of this launch: part 0 every slot, 1 the routed experts' slots, 2 the shared
  // expert's slot (one launch per bank when the banks' formats differ); every role walks
  // u_begin + blockIdx.x, + gridDim.x, ... < total
  const int u_begin = (part == 2) ? Ss.mt_prefix[n_active] * n_tiles : 0;
  const int total = (part == 1) ? Ss.mt_prefix[n_active] * n_tiles : Ss.mt_prefix[n_slots] * n_tiles;

  auto fail = [&](int site) {
    set_timeout(p.status, site);
    *abort_flag = 1;
  };

  if (warp == 0) {
    // ------------------------------------------------------------ producers
    // Lane 0 streams the weights (and each unit's scales), gated only by the dequantisers
    // releasing weight stages, so it runs up to NW stages ahead; warp 15 streams the
    // activation tiles, gated by the tensor core releasing them. Coupling both to one loop
    // (or to two lanes of one warp, which then take turns) holds one back by the other.
    if (lane == 0) {
      int it = 0, ui = 0;
      for (int u = u_begin + (int)blockIdx.x; u < total && !*abort_flag; u += gridDim.x, ++ui) {
        const TcUnit t = tc_unit(Ss, n_slots, n_tiles, u);
        const int src = t.shared ? 1 : 0;
        const int wrow = t.e * N + t.ntile * kTcM;
        if constexpr (FMT != 16) {
          // the unit's group scales: kTcM consecutive rows, one contiguous block per matrix
          const int sbuf = ui & 1;
          if (ui >= 2 && !mbar_wait(&scale_empty[sbuf], ((ui >> 1) - 1) & 1)) {
            fail(10);
            break;
          }
          mbar_arrive_expect_tx(&scale_full[sbuf], (uint32_t)(NM * SL.sb));
          const Bank& bank = t.shared ? p.shared : p.routed;
#pragma unroll
          for (int mi = 0; mi < NM; ++mi) {
            const int which = GATE_UP ? mi : 2;
            bulk_g2s(smem + C::S_OFF + (sbuf * NM + mi) * SL.sb, bank.s[which] + (size_t)wrow * G,
                     (uint32_t)SL.sb, &scale_full[sbuf]);
          }
        }
        bool ok = true;
        for (int cw = 0; cw < n_wstages; ++cw, ++it) {
          const int sw = it % C::NW, uw = it / C::NW;
          if (uw > 0 && !mbar_wait(&empty_w[sw], (uw - 1) & 1)) {
            ok = false;
            break;
          }
          // a partial last stage reads past the row end: the TMA fills zeros there and
          // still counts the whole box
          mbar_arrive_expect_tx(&full_w[sw], (uint32_t)C::WB);
#pragma unroll
          for (int mi = 0; mi < NM; ++mi)
            tma_load_2d(smem + C::R_OFF + sw * C::WB + mi * C::RAW, &maps.w[src][mi],
                        cw * C::RAW_ROW, wrow, &full_w[sw]);
        }
        if (!ok) {
          fail(11);
          break;
        }
      }
      // every issued stage lands before the CTA may exit (consumed ones already have)
      for (int j = (it > C::NW ? it - C::NW : 0); j < it; ++j)
        mbar_wait(&full_w[j % C::NW], (j / C::NW) & 1);
    }
    __syncwarp();
  } else if (warp == 1 || warp == 14) {
    // ------------------------------------------------------------ MMA issuers
    // Two converged warps issue, one elected lane each. An issuing warp touches no shared
    // memory inside the K loop: after a tcgen05.mma, the next shared-memory access of the
    // same warp (an mbarrier wait included) stalls until that warp's MMAs have drained,
    // which at N = 16 costs more than the MMAs themselves. So the dequantisers, which wait
    // for the activation stage anyway, announce a ready chunk on a named barrier per stage,
    // and the issuers only bar.sync on it (a named barrier does not stall behind the MMAs).
    // gate/up: issuer i takes matrix i, all K steps; down: issuer i takes the K steps
    // 2i, 2i+1 of every chunk into its own accumulator (the epilogue adds the two).
    // Every chunk's barrier is met by its dequantiser group, also after a failure (the MMAs
    // then run on stale operands and the status word carries the error), so the issuers
    // take every chunk and never wait on a barrier that nobody meets.
    const int iss = (warp == 1) ? 0 : 1;
    const int mi = GATE_UP ? iss : 0;
    const int k0 = GATE_UP ? 0 : 2 * iss, k1 = GATE_UP ? kTcBK / 16 : 2 * iss + 2;
    bool aborted = false;
    int it = 0, tile = 0;
    for (int u = u_begin + (int)blockIdx.x; u < total; u += gridDim.x, ++tile) {
      const TcUnit t = tc_unit(Ss, n_slots, n_tiles, u);
      const int n_mma = (t.nrows + 15) & ~15;
      const uint32_t idesc = umma_idesc_f16(n_mma);
      const int b = tile % C::ACC_BUFS, buse = tile / C::ACC_BUFS;
      aborted = aborted || *abort_flag;
      if (!aborted && buse > 0 && !mbar_wait(&acc_empty[b], (buse - 1) & 1)) {
        fail(12);
        aborted = true;
      }
      aborted = __any_sync(0xffffffffu, aborted);
      tc_fence_after();
      const uint32_t dacc = tmem + b * 128 + iss * kTcNMax;  // this issuer's accumulator
      for (int c = 0; c < n_chunks; ++c, ++it) {
        const int s = it % C::NX;
        named_bar_sync(1 + s, kReadyThreads);
        tc_fence_after();
        // One descriptor and one TMEM address per chunk; the K steps advance them by
        // constants (32 bytes of B = 2 in the descriptor's address field, 8 columns of A).
        const uint64_t bdesc = umma_desc_sw128(smem_u32(smem + C::X_OFF + s * C::XB));
        const uint32_t at = tmem + C::A_COL0 + s * C::A_COLS + mi * (kTcBK / 2);
#pragma unroll
        for (int kk = 0; kk < kTcBK / 16; ++kk)
          if (k0 + kk < k1)
            umma_f16_ts_warp(dacc, at + (k0 + kk) * 8, bdesc + (uint64_t)(2 * (k0 + kk)), idesc,
                             (c > 0 || kk > 0) ? 1u : 0u);
        umma_commit_warp(&empty_x[s]);  // releases the activation stage and the A stage
      }
      umma_commit_warp(&acc_full[b]);
    }
    // all issued MMAs complete before TMEM and shared memory are released
    umma_commit_warp(drain);
    mbar_wait(drain, 0);
  } else if (warp < 2 + kDqWarps) {
    // ------------------------------------------------------------ dequantisers
    // Two groups of four warps take alternate steps of CH consecutive chunks (group g: steps
    // j of a unit with j % 2 == g), so two steps are converted at a time; within a group, warp
    // w covers the weight rows of TMEM lanes 32 * (w % 4) .. +31 (the lanes a warp may
    // write), both K halves. A group converts chunk i into A stage i % NA once the MMAs of
    // chunk i - NA have released it, checks that the chunk's activation stage has landed, and
    // arrives on the chunk's ready barrier. Two chunks a step halve the fixed cost of the
    // waits, the store wait and the arrivals per chunk. A group arrives for every chunk, also
    // after a failure (then without converting and without waiting on the producers), and
    // always after the release of the stage: so the issuers meet each barrier phase exactly
    // once.
    constexpr int CH = C::SUB >= 2 ? 2 : 1;  // chunks a step (K is a multiple of 128)
    const int r = 32 * (warp & 3) + lane;            // weight row in the tile
    const int group = (warp - 2) >> 2;
    const uint32_t lane_base = tmem + ((uint32_t)(32 * (warp & 3)) << 16);
    bool aborted = false;
    int it = 0, ia = 0, ui = 0;
    for (int u = u_begin + (int)blockIdx.x; u < total; u += gridDim.x, ++ui) {
      const int sbuf = ui & 1;
      aborted = aborted || *abort_flag;
      if constexpr (FMT != 16) {
        if (!aborted && !mbar_wait(&scale_full[sbuf], (ui >> 1) & 1)) {
          fail(13);
          aborted = true;
        }
      }
      aborted = __any_sync(0xffffffffu, aborted);
      const uint16_t* sblk = reinterpret_cast<const uint16_t*>(smem + C::S_OFF + sbuf * NM * SL.sb);
      for (int cw = 0; cw < n_wstages; ++cw, ++it) {
        const int sw = it % C::NW;
        // every warp waits for every stage before releasing it (keeps the release phases
        // of the stage in order, also for a group with no chunk in it)
        if (!aborted && !mbar_wait(&full_w[sw], (it / C::NW) & 1)) {
          fail(14);
          aborted = true;
        }
        aborted = __any_sync(0xffffffffu, aborted);
        const int c_end = min(n_chunks, (cw + 1) * C::SUB);
        for (int c = cw * C::SUB; c < c_end; c += CH, ia += CH) {
          if (((c / CH) & 1) != group) continue;
#pragma unroll
          for (int j = 0; j < CH; ++j) {
            const int a = (ia + j) % C::NA;
            // the stage's previous chunk is consumed (waited for also after a failure; the
            // issuers never stop, so this wait ends)
            if (ia + j >= C::NA && !mbar_wait(&empty_x[a], (((ia + j) / C::NA) - 1) & 1)) {
              fail(15);
              aborted = true;
            }
            if (!aborted && !mbar_wait(&full_x[a], ((ia + j) / C::NX) & 1)) {
              fail(16);
              aborted = true;
            }
          }
          aborted = __any_sync(0xffffffffu, aborted);
          if (!aborted) {
#pragma unroll
            for (int j = 0; j < CH; ++j) {
              const int a = (ia + j) % C::NA, cc = c + j;
#pragma unroll
              for (int mi = 0; mi < NM; ++mi) {
                const float sc = (FMT == 16) ? 1.f
                                 : bf16_to_f32(sblk[mi * (SL.sb / 2) + r * G + (cc * kTcBK) / kGroup]);
                const uint8_t* raw_row = smem + C::R_OFF + sw * C::WB + mi * C::RAW + r * C::RAW_ROW;
                uint32_t regs[32];
                uint32_t (&lo)[16] = *reinterpret_cast<uint32_t(*)[16]>(&regs[0]);
                uint32_t (&hi)[16] = *reinterpret_cast<uint32_t(*)[16]>(&regs[16]);
                dequant_half_row<FMT>(raw_row, r & 7, cc - cw * C::SUB, 0, sc, lo);
                dequant_half_row<FMT>(raw_row, r & 7, cc - cw * C::SUB, 1, sc, hi);
                tmem_st32(lane_base + C::A_COL0 + a * C::A_COLS + mi * (kTcBK / 2), regs);
              }
            }
            tmem_st_wait();
          }
          tc_fence_before();  // the stores are complete before the arrivals below
          __syncwarp();
#pragma unroll
          for (int j = 0; j < CH; ++j) named_bar_arrive(1 + (ia + j) % C::NA, kReadyThreads);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty_w[sw]);  // the stage is read
      }
      if constexpr (FMT != 16) {
        __syncwarp();
        if (lane == 0) mbar_arrive(&scale_empty[sbuf]);
      }
    }
  } else if (warp == 15) {
    // ------------------------------------------------------------ activation producer
    if (lane == 0) {
      int it = 0;
      for (int u = u_begin + (int)blockIdx.x; u < total && !*abort_flag; u += gridDim.x) {
        const TcUnit t = tc_unit(Ss, n_slots, n_tiles, u);
        const int bx = box_index(t.nrows);
        const int src = t.shared ? 1 : 0;
        const int box_rows = maps.box_rows[src][bx];
        bool ok = true;
        for (int c = 0; c < n_chunks; ++c, ++it) {
          const int sx = it % C::NX, ux = it / C::NX;
          if (ux > 0 && !mbar_wait(&empty_x[sx], (ux - 1) & 1)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&full_x[sx], (uint32_t)(box_rows * kTcBK * 2));
          tma_load_2d(smem + C::X_OFF + sx * C::XB, &maps.act[src][bx], c * kTcBK, t.row0,
                      &full_x[sx]);
        }
        if (!ok) {
          fail(17);
          break;
        }
      }
      for (int j = (it > C::NX ? it - C::NX : 0); j < it; ++j)
        mbar_wait(&full_x[j % C::NX], (j / C::NX) & 1);
    }
    __syncwarp();
  } else if (warp < 14) {
    // ------------------------------------------------------------ epilogue
    const int quarter = warp & 3;            // TMEM lanes 32*quarter .. +31 (warps 10..13)
    const int row = quarter * 32 + lane;     // weight row in the tile
    int tile = 0;
    for (int u = u_begin + (int)blockIdx.x; u < total && !*abort_flag; u += gridDim.x, ++tile) {
      const TcUnit t = tc_unit(Ss, n_slots, n_tiles, u);
      const int b = tile % C::ACC_BUFS;
      if (!mbar_wait(&acc_full[b], (tile / C::ACC_BUFS) & 1)) {
        fail(18);
        break;
      }
      tc_fence_after();
      const uint32_t lane_addr = tmem + ((uint32_t)(quarter * 32) << 16) + b * 128;
      const int n = t.ntile * kTcM + row;  // output feature
      // gate/up: where feature n sits in the h row (the K order the down GEMM's bank reads)
      const int hn = GATE_UP ? k_position(n, interleaved_k(t.shared ? p.shared.fmt : p.routed.fmt)) : n;
      for (int m0 = 0; m0 < t.nrows; m0 += 16) {
        float g[16];
        tmem_ld16(lane_addr + m0, g);
        if constexpr (GATE_UP) {
          float up[16];
          tmem_ld16(lane_addr + kTcNMax + m0, up);
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            if (m0 + j < t.nrows) {
              const float h = g[j] / (1.f + expf(-g[j])) * up[j];
              const size_t hrow = (t.shared ? (size_t)p.T * p.k : 0) + t.row0 + m0 + j;
              if (!(fabsf(h) <= 65504.f)) set_status(p.status, DEV_RANGE);
              const __half hh = __float2half_rn(h);
              p.h[hrow * p.f + hn] = *reinterpret_cast<const uint16_t*>(&hh);
            }
          }
        } else {
          float g2[16];
          tmem_ld16(lane_addr + kTcNMax + m0, g2);  // the second issuer's K steps
#pragma unroll
          for (int j = 0; j < 16; ++j) g[j] += g2[j];
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            if (m0 + j < t.nrows) {
              float* dst = t.shared ? p.y_shared + (size_t)(t.row0 + m0 + j) * p.d
                                    : p.y_assign + (size_t)(t.row0 + m0 + j) * p.d;
              dst[n] = g[j];
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

// ------------------------------------------------------------------ host side


size_t tc_sched_bytes(int E) { return sizeof(int32_t) * (size_t)(5 * (E + 2)); }

TcSched tc_sched_view(void* base, int E) {
  int32_t* b = static_cast<int32_t*>(base);
  TcSched s;
  s.slot_rows = b;
  s.slot_row0 = b + (E + 2);
  s.slot_expert = b + 2 * (E + 2);
  s.mt_prefix = b + 3 * (E + 2);
  s.expert_mt = b + 4 * (E + 2);
  return s;
}

template <int FMT, bool GATE_UP, int ACC>
static cudaError_t launch_tc_fmt(const Plan& p, const TcSched& S, const uint16_t* xg, int part,
                                 cudaStream_t st) {
  using C = TcCfg<FMT, GATE_UP, ACC>;
  const int K = GATE_UP ? p.d : p.f;
  const int N = GATE_UP ? p.f : p.d;
  const int wbytes_per_row = K * FMT / 8;  // int4: K/2, int8: K, bf16: 2K
  const uint32_t box_w = C::RAW_ROW;
  TcMaps maps;
  std::memset(&maps, 0, sizeof(maps));
  const Bank* banks[2] = {&p.routed, &p.shared};
  // weight maps of the banks this launch reads (FMT is theirs)
  const int nexp[2] = {part == 2 ? 0 : p.E, (p.has_shared && part != 1) ? 1 : 0};
  for (int b = 0; b < 2; ++b) {
    if (nexp[b] == 0) continue;
    for (int mi = 0; mi < C::NM; ++mi) {
      const int which = GATE_UP ? mi : 2;
      if (!make_map(&maps.w[b][mi], CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, banks[b]->w[which],
                    wbytes_per_row, (uint64_t)nexp[b] * N, box_w, kTcM,
                    CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    }
  }
  // activations: grouped rows (gathered x, or h) and the shared expert's rows
  const uint16_t* act_src[2];
  uint64_t act_rows[2];
  if (GATE_UP) {
    act_src[0] = xg;
    act_rows[0] = (uint64_t)p.T * p.k;
    act_src[1] = xg + (size_t)p.T * p.k * p.d;
    act_rows[1] = p.T;
  } else {
    act_src[0] = p.h;
    act_rows[0] = (uint64_t)p.T * p.k;
    act_src[1] = p.h + (size_t)p.T * p.k * p.f;
    act_rows[1] = p.T;
  }
  for (int s = 0; s < 2; ++s) {
    if (s == 1 && !p.has_shared) continue;
    for (int bx = 0; bx < kBoxes; ++bx) {
      const uint32_t rows = (uint32_t)std::min<uint64_t>(16u << bx, act_rows[s]);
      maps.box_rows[s][bx] = (int)rows;
      if (!make_map(&maps.act[s][bx], CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, act_src[s], K,
                    act_rows[s], kTcBK, rows, CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    }
  }
  auto kern = tc_grouped_kernel<FMT, GATE_UP, ACC>;
  const int smem = tc_smem<FMT, GATE_UP, ACC>(K, p.E).total;
  if (smem > 227 * 1024) return cudaErrorInvalidValue;
  static std::once_flag once;
  static cudaError_t attr_err = cudaSuccess;
  static int sms = 0;
  std::call_once(once, [&] {
    attr_err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024);
    int dev = 0;
    if (attr_err == cudaSuccess) attr_err = cudaGetDevice(&dev);
    if (attr_err == cudaSuccess)
      attr_err = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  });
  if (attr_err != cudaSuccess) return attr_err;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(sms);
  cfg.blockDim = dim3(kTcThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, maps, p, S, part);
}

template <bool GATE_UP, int ACC>
static cudaError_t launch_tc_part(const Plan& p, const TcSched& S, const uint16_t* xg, int fmt,
                                  int part, cudaStream_t st) {
  switch (fmt) {
    case 4: return launch_tc_fmt<4, GATE_UP, ACC>(p, S, xg, part, st);
    case 8: return launch_tc_fmt<8, GATE_UP, ACC>(p, S, xg, part, st);
    default: return launch_tc_fmt<16, GATE_UP, ACC>(p, S, xg, part, st);
  }
}

// One launch for both banks when they share a format; otherwise the routed experts and the
// shared expert in two launches, each with its own format.
template <bool GATE_UP, int ACC>
static cudaError_t launch_tc(const Plan& p, const TcSched& S, const uint16_t* xg,
                             cudaStream_t st) {
  if (!p.has_shared || p.shared.fmt == p.routed.fmt)
    return launch_tc_part<GATE_UP, ACC>(p, S, xg, p.routed.fmt, 0, st);
  const cudaError_t err = launch_tc_part<GATE_UP, ACC>(p, S, xg, p.routed.fmt, 1, st);
  if (err != cudaSuccess) return err;
  return launch_tc_part<GATE_UP, ACC>(p, S, xg, p.shared.fmt, 2, st);
}

bool tc_supported(const Plan& p) {
  return get_encoder() != nullptr && p.d % kTcM == 0 && p.f % kTcM == 0 &&
         p.d % kTcBK == 0 && p.f % kTcBK == 0;
}

cudaError_t launch_tc_prep(const Plan& p, const TcSched& S, uint16_t* xg, cudaStream_t st,
                           bool shared_rows_only) {
  const int row_begin = shared_rows_only ? p.T * p.k : 0;
  const long long rows = (long long)p.T * p.k + p.T - row_begin;  // one warp a row, 8 a CTA
  const int blocks = (int)std::max(1LL, std::min<long long>(1184, (rows + 7) / 8));
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(blocks);
  cfg.blockDim = dim3(256);
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, tc_prep_kernel, p, S, xg, row_begin);
}

// Gate/up with two accumulator buffers when the routed experts average 32 rows or more.
cudaError_t launch_tc_gate_up(const Plan& p, const TcSched& S, const uint16_t* xg,
                              cudaStream_t st) {
  if ((long long)p.T * p.k >= 32LL * p.E) return launch_tc<true, 2>(p, S, xg, st);
  return launch_tc<true, 1>(p, S, xg, st);
}
cudaError_t launch_tc_down(const Plan& p, const TcSched& S, cudaStream_t st) {
  return launch_tc<false, 2>(p, S, nullptr, st);
}

cudaError_t launch_tc_shared_gate_up(const Plan& p, const TcSched& S, const uint16_t* xg,
                                     cudaStream_t st) {
  return launch_tc_part<true, 1>(p, S, xg, p.shared.fmt, 2, st);
}
cudaError_t launch_tc_shared_down(const Plan& p, const TcSched& S, cudaStream_t st) {
  return launch_tc_part<false, 2>(p, S, nullptr, p.shared.fmt, 2, st);
}

}  // namespace moe
