// Grouped expert FFN for few rows per expert (decode and verify calls) with int4 weights:
// weight tiles move HBM -> shared memory through the TMA engine (one-dimensional bulk
// copies) in a multi-stage mbarrier pipeline, and 8 consumer warps run the products on the
// tensor cores (mma.sync m16n8k16, fragments from gemv_frag.cuh).
//
// Layout facts used: in the int4 encoding an expert matrix is row-major with K contiguous,
// so ROWS consecutive rows of one expert form ONE contiguous block of ROWS * K / 2 bytes,
// and their group scales [ROWS][K / 128] another. A stage is one such tile of every matrix
// the kernel needs (gate and up for the first kernel, down for the second) plus scales; one
// thread issues two bulk copies per matrix and the copies complete on the stage's mbarrier.
//
// Work: tiles (active expert, ROWS rows) in a flat list; CTA c (one per SM, persistent)
// takes a contiguous range, so consecutive tiles mostly share an expert and its staged
// activation rows. Ranges are balanced by cost, a shared-expert tile (T rows) weighing its
// token chunks: with equal tile counts, the CTAs holding the shared expert's tiles took
// T / 8 times longer than the rest (measured on B200: 16 and 32 rows ran 2x and 4x slower
// than 8 rows per expert tile predicted). Each weight byte is read from HBM once per call; tokens beyond 8 for one
// expert re-use the staged tile from shared memory.
//
// What is computed is the same as gemv_ffn.cu: h = silu(Wg x) * (Wu x) per grouped row
// (Qwen3.8-Flash-Next-Dual-GPU README, "Dedicated prefill lane", step 2), then one fp32
// y = Wd h per assignment (step 4); unselected experts are never read (TandemLLM docs,
// "17 Qwen3.8-Flash-Next", §17.4).
#include <mutex>

#include "gemv_frag.cuh"
#include "pipeline.cuh"

namespace moe {


constexpr int kCons = 16;                    // consumer warps
constexpr int kTmaThreads = 32 * (kCons + 1);  // + one producer warp

// Tile shapes per weight format: int8 rows are twice as long, so its gate/up tiles have
// half the rows (two stages still fit) and its down kernel two stages.
template <int FMT, bool GATE_UP> struct TmaShape {
  static constexpr int ROWS = GATE_UP ? (FMT == 4 ? 32 : 16) : 64;  // weight rows per tile
  static constexpr int NM = GATE_UP ? 2 : 1;      // matrices per tile
  static constexpr int RT = ROWS / 16;            // 16-row MMA tiles per tile
  static constexpr int KS = kCons / RT;           // consumer warps sharing one row tile (K split)
  static constexpr int NS = GATE_UP ? 2 : (FMT == 4 ? 5 : 2);  // pipeline stages
  // int4: the K split of the single-kernel 1-token layer, which computes the same rows
  static_assert(FMT != 4 || KS == (GATE_UP ? kKsGateUp : kKsDown), "shared K split");
};

struct TmaSmem {
  size_t stage_bytes, w_bytes, s_bytes, xs_off, xsum_off, red_off, bar_off, flag_off, total;
};

template <int FMT, bool GATE_UP>
__host__ __device__ inline TmaSmem tma_smem_layout(int K) {
  using Sh = TmaShape<FMT, GATE_UP>;
  TmaSmem m;
  const int G = K / kGroup;
  m.w_bytes = (size_t)Sh::ROWS * K * FMT / 8;  // one matrix tile
  m.s_bytes = (size_t)Sh::ROWS * G * 2;        // its scales (bf16)
  m.stage_bytes = Sh::NM * (m.w_bytes + m.s_bytes);
  size_t o = Sh::NS * m.stage_bytes;
  m.xs_off = o;
  o += (size_t)kTok * (2 * K + 8);
  o = (o + 15) & ~size_t(15);
  m.xsum_off = o;
  o += sizeof(float) * kTok * G;
  m.red_off = o;
  o += sizeof(float) * kCons * 32 * Sh::NM * 4;
  o = (o + 15) & ~size_t(15);
  m.bar_off = o;
  o += sizeof(uint64_t) * 2 * Sh::NS;
  m.flag_off = o;
  o += 16;
  m.total = o;
  return m;
}

// Tile -> expert and rows. Tiles [0, n_active * n_rowtiles) are the active routed experts'
// (ascending ids; all of an expert's rows), then the shared expert's: one tile per (kTok-row
// token chunk, row tile), chunk-major, so every tile carries at most kTok rows and a CTA's
// consecutive shared tiles use the same staged rows. (The shared expert's T rows taken
// whole cost a CTA 3.6x a routed tile at 16 rows, restaging its rows for every chunk.)
struct TileInfo {
  int slot, e, shared, row_begin, nrows, rowtile;
};

__device__ __forceinline__ TileInfo tile_info(const Plan& p, int ti, int n_rowtiles,
                                              int n_active) {
  TileInfo t;
  const int n_rt = n_active * n_rowtiles;
  if (ti < n_rt) {
    t.slot = ti / n_rowtiles;
    t.rowtile = ti % n_rowtiles;
    t.e = p.active[1 + t.slot];
    t.shared = 0;
    t.row_begin = p.offsets[t.e];
    t.nrows = p.offsets[t.e + 1] - t.row_begin;
  } else {
    const int j = ti - n_rt;
    t.slot = n_active;
    t.rowtile = j % n_rowtiles;
    t.e = 0;
    t.shared = 1;
    t.row_begin = (j / n_rowtiles) * kTok;
    t.nrows = min(kTok, p.T - t.row_begin);
  }
  return t;
}

// Tiles of the shared expert: one per (token chunk, row tile).
__host__ __device__ __forceinline__ int shared_tiles(int T, int n_rowtiles) {
  return ((T + kTok - 1) / kTok) * n_rowtiles;
}

// Stage the activation rows of token chunk c0 of tile t (x gathered through perm for the
// gate/up kernel, the h rows of the tile's expert for the down kernel).
template <int FMT, bool GATE_UP>
__device__ __forceinline__ void stage_tile_rows(const Plan& p, const TileInfo& t, int c0, int K,
                                                uint8_t* xs, int S, float* xsum, int ctid) {
  StageArgs sa;
  if (GATE_UP) {
    sa.src = p.x;
    sa.src_stride = p.d;
    sa.perm = t.shared ? nullptr : p.perm;
    sa.k = p.k;
    sa.row0 = t.row_begin + c0;
  } else {
    sa.src = p.h;
    sa.src_stride = p.f;
    sa.perm = nullptr;
    sa.k = 1;
    sa.row0 = (t.shared ? p.T * p.k : 0) + t.row_begin + c0;
  }
  sa.nrows = min(kTok, t.nrows - c0);
  stage_rows<FMT, 32 * kCons>(sa, K, xs, S, xsum, ctid);
}

// part: 0 every tile, 1 the routed experts' tiles, 2 the shared expert's (one launch per
// bank when the banks' formats differ; FMT is the format of the tiles the launch takes).
template <int FMT, bool GATE_UP>
__global__ void __launch_bounds__(kTmaThreads, 1) gemv_tma_kernel(Plan p, int part) {
  using Sh = TmaShape<FMT, GATE_UP>;
  constexpr int NM = Sh::NM;
  constexpr int U = FmtInfo<FMT>::U;  // 16-byte pieces of a row's group a lane reads
  const int K = GATE_UP ? p.d : p.f;
  const int N = GATE_UP ? p.f : p.d;
  const int G = K / kGroup;
  const int S = 2 * K + 8;
  const size_t row_bytes = (size_t)K * FMT / 8;
  const TmaSmem L = tma_smem_layout<FMT, GATE_UP>(K);

  extern __shared__ __align__(128) uint8_t smem[];
  uint8_t* xs = smem + L.xs_off;
  float* xsum = reinterpret_cast<float*>(smem + L.xsum_off);
  float* red = reinterpret_cast<float*>(smem + L.red_off);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L.bar_off);
  uint64_t* empty = full + Sh::NS;
  volatile int* flag = reinterpret_cast<volatile int*>(smem + L.flag_off);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < Sh::NS; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kCons);
    }
    flag[0] = 0;
    fence_barrier_init();
  }
  __syncthreads();
  pdl_wait();     // plan and activations come from the preceding kernels

  const int n_active = p.active[0];
  const int n_rowtiles = N / Sh::ROWS;
  // Contiguous, equal tile ranges over the tiles of this launch (the partition moves no
  // arithmetic: every tile is computed the same way whichever CTA takes it).
  const int n_rt = (part == 2) ? 0 : n_active * n_rowtiles;
  const int n_st = (p.has_shared && part != 1) ? shared_tiles(p.T, n_rowtiles) : 0;
  const int tile0 = (part == 2) ? n_active * n_rowtiles : 0;  // numbering of the full list
  const long long n_tiles = (long long)n_rt + n_st;
  const int t_begin = tile0 + (int)(n_tiles * blockIdx.x / gridDim.x);
  const int t_end = tile0 + (int)(n_tiles * (blockIdx.x + 1) / gridDim.x);

  if (warp == kCons) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int i = 0;
      for (int ti = t_begin; ti < t_end; ++ti, ++i) {
        const int s = i % Sh::NS, u = i / Sh::NS;
        if (u > 0 && !mbar_wait(&empty[s], (u - 1) & 1)) {
          set_timeout(p.status, 30);
          break;
        }
        const TileInfo t = tile_info(p, ti, n_rowtiles, n_active);
        const Bank& bank = t.shared ? p.shared : p.routed;
        uint8_t* st = smem + (size_t)s * L.stage_bytes;
        mbar_arrive_expect_tx(&full[s], (uint32_t)L.stage_bytes);
#pragma unroll
        for (int mi = 0; mi < NM; ++mi) {
          const int which = GATE_UP ? mi : 2;
          const uint8_t* wsrc = static_cast<const uint8_t*>(bank.w[which]) +
                                ((size_t)t.e * N + (size_t)t.rowtile * Sh::ROWS) * row_bytes;
          const uint16_t* ssrc = bank.s[which] + ((size_t)t.e * N + (size_t)t.rowtile * Sh::ROWS) * G;
          bulk_g2s(st + mi * L.w_bytes, wsrc, (uint32_t)L.w_bytes, &full[s]);
          bulk_g2s(st + NM * L.w_bytes + mi * L.s_bytes, ssrc, (uint32_t)L.s_bytes, &full[s]);
        }
      }
      // drain: every issued stage must land before the CTA may exit
      const int issued = i;
      for (int j = (issued > Sh::NS ? issued - Sh::NS : 0); j < issued; ++j)
        mbar_wait(&full[j % Sh::NS], (j / Sh::NS) & 1);
    }
    return;
  }

  // -------------------------------------------------------------- consumers
  const int ctid = threadIdx.x;  // 0 .. 255
  const int rt = warp / Sh::KS, ks = warp % Sh::KS;
  const int grp = lane >> 2, q4 = lane & 3;
  int staged_slot = -1, staged_c0 = -1;  // the staged rows: slot and first grouped row
  int i = 0;
  for (int ti = t_begin; ti < t_end; ++ti, ++i) {
    const int s = i % Sh::NS, u = i / Sh::NS;
    const TileInfo t = tile_info(p, ti, n_rowtiles, n_active);
    // The first token chunk of a new expert is staged before the wait for the tile's
    // weights, so the activation loads overlap the weight copies.
    const bool pre = (staged_slot != t.slot || staged_c0 != t.row_begin);
    if (pre) stage_tile_rows<FMT, GATE_UP>(p, t, 0, K, xs, S, xsum, ctid);
    if (ctid == 0) flag[1] = mbar_wait(&full[s], u & 1) ? 1 : 0;
    named_bar_sync(1, 32 * kCons);
    if (!flag[1]) {
      if (ctid == 0) set_timeout(p.status, 31);
      break;
    }
    if (pre) {
      staged_slot = t.slot;
      staged_c0 = t.row_begin;
    }
    const uint8_t* st = smem + (size_t)s * L.stage_bytes;
    const int la = rt * 16 + grp, lb = la + 8;  // rows inside the tile

    for (int c0 = 0; c0 < t.nrows; c0 += kTok) {
      const int nr = min(kTok, t.nrows - c0);
      if (staged_slot != t.slot || staged_c0 != t.row_begin + c0) {
        named_bar_sync(1, 32 * kCons);  // everyone is done with the previous rows
        stage_tile_rows<FMT, GATE_UP>(p, t, c0, K, xs, S, xsum, ctid);
        named_bar_sync(1, 32 * kCons);
        staged_slot = t.slot;
        staged_c0 = t.row_begin + c0;
      }
      float acc[NM][4];
#pragma unroll
      for (int mi = 0; mi < NM; ++mi)
#pragma unroll
        for (int q = 0; q < 4; ++q) acc[mi][q] = 0.f;
      const uint8_t* xrow = xs + (size_t)grp * S;
      for (int g = ks; g < G; g += Sh::KS) {
        uint4 wa[NM][U], wb[NM][U];
        float fsa[NM], fsb[NM];
#pragma unroll
        for (int mi = 0; mi < NM; ++mi) {
          const uint8_t* wt = st + mi * L.w_bytes;
          // the lane's 32 K values of the group: 16 * U bytes of each of its two rows
#pragma unroll
          for (int u = 0; u < U; ++u) {
            wa[mi][u] = *reinterpret_cast<const uint4*>(wt + la * row_bytes + g * (16 * FMT) +
                                                        q4 * (4 * FMT) + 16 * u);
            wb[mi][u] = *reinterpret_cast<const uint4*>(wt + lb * row_bytes + g * (16 * FMT) +
                                                        q4 * (4 * FMT) + 16 * u);
          }
          const uint16_t* sc = reinterpret_cast<const uint16_t*>(st + NM * L.w_bytes + mi * L.s_bytes);
          fsa[mi] = bf16_to_f32(sc[la * G + g]);
          fsb[mi] = bf16_to_f32(sc[lb * G + g]);
        }
        group_mma<FMT, NM>(wa, wb, fsa, fsb, xrow, xsum, G, g, q4, acc);
      }
      float* myred = red + ((size_t)warp * 32 + lane) * (NM * 4);
#pragma unroll
      for (int mi = 0; mi < NM; ++mi)
#pragma unroll
        for (int q = 0; q < 4; ++q) myred[mi * 4 + q] = acc[mi][q];
      named_bar_sync(1, 32 * kCons);
      // fixed-order sum over the K split, then the epilogue
      for (int o = ctid; o < Sh::ROWS * kTok; o += 32 * kCons) {
        const int row = o / kTok, tok = o % kTok;
        if (tok >= nr) continue;
        const int rtile = row / 16, r16 = row % 16;
        const int l = (r16 % 8) * 4 + tok / 2, q = (r16 / 8) * 2 + (tok % 2);
        float tot[NM];
#pragma unroll
        for (int mi = 0; mi < NM; ++mi) tot[mi] = 0.f;
        for (int k2 = 0; k2 < Sh::KS; ++k2) {
          const float* r = red + ((size_t)(rtile * Sh::KS + k2) * 32 + l) * (NM * 4);
#pragma unroll
          for (int mi = 0; mi < NM; ++mi) tot[mi] += r[mi * 4 + q];
        }
        const int n = t.rowtile * Sh::ROWS + row;
        if constexpr (GATE_UP) {
          const float gte = tot[0], up = tot[1];
          const float hval = gte / (1.f + expf(-gte)) * up;
          const size_t hrow = (t.shared ? (size_t)p.T * p.k : 0) + t.row_begin + c0 + tok;
          p.h[hrow * p.f + n] = f32_to_bf16_rn(hval);
        } else {
          float* dst = t.shared ? p.y_shared + (size_t)(t.row_begin + c0 + tok) * p.d
                                : p.y_assign + (size_t)(t.row_begin + c0 + tok) * p.d;
          dst[n] = tot[0];
        }
      }
      named_bar_sync(1, 32 * kCons);
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);
  }
  pdl_trigger();  // dependents start as this CTA finishes (see route_fused.cu)
}

struct TmaLaunchCache {
  std::mutex mu;
  size_t smem = 0;
  int sms = 0;
};

template <int FMT, bool GATE_UP>
static cudaError_t launch_tma_part(const Plan& p, int part, cudaStream_t st, bool pdl) {
  const int K = GATE_UP ? p.d : p.f;
  const size_t smem = tma_smem_layout<FMT, GATE_UP>(K).total;
  auto kern = gemv_tma_kernel<FMT, GATE_UP>;
  static TmaLaunchCache cache;
  int sms;
  {
    std::lock_guard<std::mutex> lock(cache.mu);
    if (smem > cache.smem) {
      cudaError_t err =
          cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
      if (err != cudaSuccess) return err;
      int dev = 0;
      if ((err = cudaGetDevice(&dev)) != cudaSuccess) return err;
      if ((err = cudaDeviceGetAttribute(&cache.sms, cudaDevAttrMultiProcessorCount, dev)) !=
          cudaSuccess)
        return err;
      cache.smem = smem;
    }
    sms = cache.sms;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(sms);
  cfg.blockDim = dim3(kTmaThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = pdl ? 1 : 0;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, p, part);
}

template <bool GATE_UP>
static cudaError_t launch_tma_fmt(const Plan& p, int fmt, int part, cudaStream_t st, bool pdl) {
  return fmt == 8 ? launch_tma_part<8, GATE_UP>(p, part, st, pdl)
                  : launch_tma_part<4, GATE_UP>(p, part, st, pdl);
}

// One launch when the banks share a format, else the routed experts and the shared expert
// in two launches of their own formats (the second one after the first: same stream).
template <bool GATE_UP>
static cudaError_t launch_tma(const Plan& p, cudaStream_t st, bool pdl) {
  if (!p.has_shared || p.shared.fmt == p.routed.fmt)
    return launch_tma_fmt<GATE_UP>(p, p.routed.fmt, 0, st, pdl);
  const cudaError_t err = launch_tma_fmt<GATE_UP>(p, p.routed.fmt, 1, st, pdl);
  if (err != cudaSuccess) return err;
  return launch_tma_fmt<GATE_UP>(p, p.shared.fmt, 2, st, true);
}


template <int FMT>
static bool tma_fits(const Plan& p) {
  return tma_smem_layout<FMT, true>(p.d).total <= 227 * 1024 &&
         tma_smem_layout<FMT, false>(p.f).total <= 227 * 1024;
}

// int4 and int8 banks (in any pairing); bf16 banks take the register-streaming GEMV.
bool tma_gemv_supported(const Plan& p) {
  auto ok = [&](int fmt) {
    return (fmt == 4 && tma_fits<4>(p)) || (fmt == 8 && tma_fits<8>(p));
  };
  return ok(p.routed.fmt) && (!p.has_shared || ok(p.shared.fmt));
}

cudaError_t launch_tma_gate_up(const Plan& p, cudaStream_t st, bool pdl) {
  return launch_tma<true>(p, st, pdl);
}
cudaError_t launch_tma_down(const Plan& p, cudaStream_t st, bool pdl) {
  return launch_tma<false>(p, st, pdl);
}

}  // namespace moe
