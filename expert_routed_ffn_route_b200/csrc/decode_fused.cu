// The whole layer for a 1-token call in ONE persistent kernel (one CTA per SM, launched
// cooperatively so that every CTA is resident and grid-wide barriers are safe).
//
// A decode token reads ~47 MB of weights in a few microseconds; separate launches for
// routing, gate/up, down and combine cost more than the weight streaming itself. Here the
// phases run back to back inside one grid, and every weight byte that does not depend on
// the routing decision (router rows, the shared expert) is already in flight before that
// decision is known:
//
//   prologue   each CTA issues bulk copies (TMA engine, no multicast) of its slice of the
//              router rows and of its shared-expert gate/up tile, and an L2 prefetch of its
//              shared-expert down rows.
//   route      logits of the CTA's router rows -> workspace; grid barrier B1 (the CTA's
//              shared-expert tile is multiplied while the barrier settles); then EVERY CTA
//              reads the E logits and runs the same stable top-k and softmax over the picks
//              (no second barrier: all CTAs reach the same decision from the same data).
//   gate/up    the CTA's routed gate/up tiles (16 rows of one expert's gate and up, with
//              their group scales) are all requested at once, and the L2 prefetch of its
//              routed down rows follows them; h = silu(Wg x) * (Wu x) per row, rounded to
//              bf16, is written to the workspace. Grid barrier B2.
//   down       the CTA's down units (16 output rows of one expert) were copied into the
//              freed tile buffers before B2; y = Wd h per unit in fp32 -> workspace.
//   combine    per 16-row output tile, the CTA that completes it (an arrival counter per
//              tile, no waiting) sums out = sum_j gate_j * y_j + y_shared in the fixed
//              order j = 0..k-1, then the shared term, and rounds once to bf16.
//
// Products run on the tensor cores (mma.sync m16n8k16, weights as the 16-row A operand,
// the token as column 0 of B), with the int4 codes entering exactly (gemv_frag.cuh) and the
// group scale applied to the fp32 partial of each 128-wide K group. Every K-group partial
// is reduced across warps in a fixed order, so the result is bitwise reproducible.
//
// What is computed is the layer of include/moe_b200.h: stable top-k with ties to the lower
// index (Qwen3.8-Flash-Next-Dual-GPU README, "Independent decode lane"), SwiGLU experts on
// symmetric group-128 int4 weights ("Model artifact and memory placement"), a fixed-order
// reduction of each token's routes without atomics on the data ("Dedicated prefill lane",
// step 5), unselected experts never read (TandemLLM docs, "17 Qwen3.8-Flash-Next", §17.4).
#include <mutex>

#include "gemv_frag.cuh"
#include "pipeline.cuh"

namespace moe {

constexpr int kDfWarps = 20;                 // compute warps
constexpr int kDfCompute = 32 * kDfWarps;
constexpr int kDfThreads = kDfCompute + 32;  // + the producer warp
constexpr int kDfRows = 16;                  // weight rows of a tile / unit (MMA M)
constexpr int kDfMaxTiles = 8;
constexpr int kDfMaxUnits = 24;
constexpr int kDfMaxRouter = 8;


// Smem scratch beyond the buffers: picks, gates and the CTA's tile/unit tables.
struct DfMisc {
  int sel[kMaxK];
  float gate[kMaxK];
  int tile_slot[kDfMaxTiles], tile_rt[kDfMaxTiles];
  int unit_slot[kDfMaxUnits], unit_rt[kDfMaxUnits];
  int n_tiles, n_units, n_split, first_routed, ok, armed_tiles, armed_units, armed_h;
};

// Shared-memory plan of one launch (identical on the host and in every CTA).
struct DfLayout {
  int grid, n_slots, G, Gf;
  int tiles_total, tiles_max, full_per_cta, split_units, units_max, router_max;
  uint32_t tile_bytes, unit_bytes;
  uint32_t off_router, off_h, off_hsum, off_x, off_xsum, off_cand, off_ybuf, off_red, off_bar, off_misc, total;
};

__host__ __device__ inline DfLayout df_layout(int grid, int d, int f, int E, int k,
                                              int has_shared) {
  DfLayout L;
  L.grid = grid;
  L.n_slots = k + has_shared;
  L.G = d / kGroup;
  L.Gf = f / kGroup;
  L.tiles_total = L.n_slots * (f / kDfRows);
  L.tiles_max = (L.tiles_total + grid - 1) / grid;
  // down units: each CTA owns whole 16-row output tiles (all slots of a tile, combined
  // locally); the tiles left over are split by slot across CTAs and combined by the CTA
  // that completes them
  const int n_rt = d / kDfRows;
  L.full_per_cta = n_rt / grid;
  L.split_units = (n_rt - L.full_per_cta * grid) * L.n_slots;
  L.units_max = L.full_per_cta * L.n_slots + (L.split_units + grid - 1) / grid;
  L.router_max = (E + grid - 1) / grid;
  // gate and up rows (int4) then their bf16 scales
  L.tile_bytes = 2u * kDfRows * (d / 2) + 2u * kDfRows * L.G * 2;
  L.unit_bytes = (uint32_t)kDfRows * (f / 2) + (uint32_t)kDfRows * L.Gf * 2;
  // one region holds the gate/up tiles, later the down units; the router rows alias its end
  // when they leave buffer 0 (the shared tile, copied meanwhile) free, else follow it
  const uint32_t router_bytes = (uint32_t)L.router_max * d * 2;
  // the h rows of the call (staged after B2) follow the down units
  L.off_h = L.units_max * L.unit_bytes;
  L.off_hsum = L.off_h + (uint32_t)L.n_slots * f * 2;
  uint32_t region = max(L.tiles_max * L.tile_bytes, L.off_hsum + 4u * L.n_slots * L.Gf);
  region = (region + 15) & ~15u;
  if (router_bytes + (has_shared ? L.tile_bytes : 0u) <= region) {
    L.off_router = region - router_bytes;
  } else {
    L.off_router = region;
    region += router_bytes;
  }
  uint32_t o = region;
  L.off_x = o;
  o += 2u * d;
  L.off_xsum = o;
  o += 4u * L.G;
  o = (o + 15) & ~15u;
  // top-k candidates [ceil(E / 32)][min(k, 32)] (key, index) and their compaction: in the
  // tile region past buffer 0 when it fits (only the shared tile is live at that time)
  const uint32_t cand_bytes = 16u * ((E + 31) / 32) * min(k, 32);
  if (L.tile_bytes + cand_bytes <= region) {
    L.off_cand = L.tile_bytes;
  } else {
    L.off_cand = o;
    o += cand_bytes;
  }
  // y rows of the whole tiles, at the end: past the staged h when it fits
  const uint32_t ybuf_bytes = 4u * L.full_per_cta * L.n_slots * kDfRows;
  const uint32_t yb0 = (L.off_hsum + 4u * L.n_slots * L.Gf + 15) & ~15u;
  if (yb0 + ybuf_bytes <= region) {
    L.off_ybuf = yb0;
  } else {
    L.off_ybuf = o;
    o += ybuf_bytes;
  }
  // K-split partials: [tile][matrix][split part][16 rows], then [unit][split part][16 rows]
  L.off_red = o;
  uint32_t red_gu = (uint32_t)L.tiles_max * 2 * kKsGateUp * kDfRows * 4;
  uint32_t red_dn = (uint32_t)L.units_max * kKsDown * kDfRows * 4;
  o += max(red_gu, red_dn);
  o = (o + 15) & ~15u;
  L.off_bar = o;
  o += 8u * (2 + kDfMaxTiles + kDfMaxUnits);
  L.off_misc = o;
  o += (uint32_t)((sizeof(DfMisc) + 15) & ~size_t(15));
  L.total = o;
  return L;
}

// A wait that every lane of the warp leaves with the same verdict.
__device__ __forceinline__ bool warp_wait(uint64_t* bar) {
  const bool ok = mbar_wait(bar, 0);
  return __all_sync(0xffffffffu, ok);
}

__device__ __forceinline__ void prefetch_l2(const void* src, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}

// ------------------------------------------------------------------ tile products

// One 128-wide K group of a 16-row int4 tile against one activation row held as the
// B operand's column 0 (xb: the lane's 32 activation values of the group, permuted into
// fragment order; zero on lanes that do not carry column 0). Returns, on lanes with q == 0,
// the biased dot products of rows grp and grp + 8 (codes enter as q + 136). The 8 MMAs of
// the group accumulate in one chain, in the order the GEMV kernels use (gemv_frag.cuh), so
// the group product is the same bits as theirs.
__device__ __forceinline__ void t1_group(const uint8_t* tile, uint32_t row_bytes, int g, int grp,
                                         int q, const uint32_t (&xb)[16], float& ra,
                                         float& rb) {
  uint4 wa[1], wb[1];
  wa[0] = *reinterpret_cast<const uint4*>(tile + grp * row_bytes + g * 64 + q * 16);
  wb[0] = *reinterpret_cast<const uint4*>(tile + (grp + 8) * row_bytes + g * 64 + q * 16);
  uint32_t fa[8][2], fb[8][2];
  to_frags<4>(wa, fa);
  to_frags<4>(wb, fb);
  float c[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int m = 0; m < 8; ++m)
    mma_bf16_16x8x16(c, fa[m][0], fb[m][0], fa[m][1], fb[m][1], xb[2 * m], xb[2 * m + 1]);
  ra = c[0];
  rb = c[2];
}

// The lane's 32 activation values [32 q, 32 q + 32) of group g of a bf16 row, in fragment
// order, and their sum (fixed order: within the lane, then across the 4 lanes of the row).
template <bool GLOBAL>
__device__ __forceinline__ float t1_load_act(const uint16_t* row, int g, int q, bool carry,
                                             uint32_t (&xb)[16]) {
  float s = 0.f;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    uint4 v = make_uint4(0, 0, 0, 0);
    if (carry) {
      const uint4* src = reinterpret_cast<const uint4*>(row + g * kGroup + 32 * q + 8 * i);
      v = GLOBAL ? __ldcg(src) : *src;
    }
    const uint32_t vv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      s += __uint_as_float(vv[j] << 16);
      s += __uint_as_float(vv[j] & 0xffff0000u);
    }
    permute_chunk<4>(v);
    xb[4 * i + 0] = v.x;
    xb[4 * i + 1] = v.y;
    xb[4 * i + 2] = v.z;
    xb[4 * i + 3] = v.w;
  }
  s += __shfl_xor_sync(0xffffffffu, s, 1);
  s += __shfl_xor_sync(0xffffffffu, s, 2);
  return s;
}

// ------------------------------------------------------------------ the kernel

// Warps 0..kDfWarps-1 compute; warp kDfWarps (the producer) issues every bulk copy and L2
// prefetch (one lane a copy) and spins on the grid barriers, so no compute warp stalls on
// copy issue or on another CTA.
__global__ void __launch_bounds__(kDfThreads, 1) decode_fused_kernel(Plan p, uint16_t* out,
                                                                     uint32_t* gbar,
                                                                     int32_t* tile_cnt) {
  extern __shared__ __align__(128) uint8_t smem[];
  const int d = p.d, f = p.f, E = p.E, k = p.k;
  const DfLayout L = df_layout(gridDim.x, d, f, E, k, p.has_shared);
  const int G = L.G, Gf = L.Gf, S = L.n_slots;
  const uint32_t rowb_up = d / 2, rowb_dn = f / 2;
  uint16_t* s_x = reinterpret_cast<uint16_t*>(smem + L.off_x);
  float* s_xsum = reinterpret_cast<float*>(smem + L.off_xsum);
  float* red = reinterpret_cast<float*>(smem + L.off_red);
  uint64_t* bar_router = reinterpret_cast<uint64_t*>(smem + L.off_bar);
  uint64_t* bar_h = bar_router + 1;
  uint64_t* bar_tile = bar_router + 2;
  uint64_t* bar_unit = bar_tile + kDfMaxTiles;
  DfMisc* mi = reinterpret_cast<DfMisc*>(smem + L.off_misc);
  const uint16_t* s_router = reinterpret_cast<const uint16_t*>(smem + L.off_router);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const bool producer = (warp == kDfWarps);
  const int grp = lane >> 2, q = lane & 3;
  const int c = blockIdx.x, grid = gridDim.x;
  const int r0 = (int)((long long)E * c / grid), r1 = (int)((long long)E * (c + 1) / grid);
  const int nr = r1 - r0;

  // ---------------------------------------------------------------- prologue
  const int t0 = (int)((long long)L.tiles_total * c / grid);
  const int t1 = (int)((long long)L.tiles_total * (c + 1) / grid);
  // the shared expert's tile of this CTA (at most one: tiles are numbered with the slot
  // fastest, and slot 0 is the shared expert)
  const int sh_i = p.has_shared ? (t0 + S - 1) / S * S : t1;
  const bool has_sh_tile = sh_i < t1;
  if (producer) {
    if (lane == 0) {
      mbar_init(bar_router, 1);
      mbar_init(bar_h, 1);
      for (int i = 0; i < kDfMaxTiles; ++i) mbar_init(&bar_tile[i], 1);
      for (int i = 0; i < kDfMaxUnits; ++i) mbar_init(&bar_unit[i], 1);
      fence_barrier_init();
      mi->ok = 1;
      mi->armed_tiles = has_sh_tile ? 1 : 0;
      mi->armed_units = 0;
      mi->armed_h = 0;
      // the copies that depend on nothing: this CTA's router rows, its shared-expert tile
      const uint32_t rb = (uint32_t)nr * d * 2;
      mbar_arrive_expect_tx(bar_router, rb);
      if (rb) bulk_g2s(smem + L.off_router, p.router_w + (size_t)r0 * d, rb, bar_router);
      if (has_sh_tile) {
        const size_t row = (size_t)(sh_i / S) * kDfRows;
        const uint32_t wbytes = kDfRows * rowb_up, sbytes = kDfRows * G * 2;
        mbar_arrive_expect_tx(&bar_tile[0], L.tile_bytes);
        bulk_g2s(smem, static_cast<const uint8_t*>(p.shared.w[0]) + row * rowb_up, wbytes, &bar_tile[0]);
        bulk_g2s(smem + wbytes, static_cast<const uint8_t*>(p.shared.w[1]) + row * rowb_up, wbytes,
                 &bar_tile[0]);
        bulk_g2s(smem + 2 * wbytes, p.shared.s[0] + row * G, sbytes, &bar_tile[0]);
        bulk_g2s(smem + 2 * wbytes + sbytes, p.shared.s[1] + row * G, sbytes, &bar_tile[0]);
      }
    }
    __syncwarp();
  } else {
    // the activation row (bf16)
    for (int i = tid; i < d / 8; i += kDfCompute)
      reinterpret_cast<uint4*>(s_x)[i] = __ldg(reinterpret_cast<const uint4*>(p.x) + i);
  }
  __syncthreads();  // S1: barriers initialised, x staged

  if (producer) {
    // tile and unit tables, one lane an entry: the shared tile (if any) in position 0,
    // the routed tiles after it in order; units in order
    const int first_routed = has_sh_tile ? 1 : 0;
    const int nt = t1 - t0;
    if (lane < nt) {
      const int i = t0 + lane;
      const int pos = (i == sh_i) ? 0 : first_routed + lane - ((has_sh_tile && i > sh_i) ? 1 : 0);
      mi->tile_slot[pos] = i % S;
      mi->tile_rt[pos] = i / S;
    }
    // units: this CTA's share of the split tiles first, then its whole tiles (slot fastest)
    const int v0 = (int)((long long)L.split_units * c / grid);
    const int v1 = (int)((long long)L.split_units * (c + 1) / grid);
    const int n_split = v1 - v0, n_units = n_split + L.full_per_cta * S;
    for (int i = lane; i < n_units; i += 32) {
      int slot, rt;
      if (i < n_split) {
        slot = (v0 + i) % S;
        rt = L.full_per_cta * grid + (v0 + i) / S;
      } else {
        slot = (i - n_split) % S;
        rt = c * L.full_per_cta + (i - n_split) / S;
      }
      mi->unit_slot[i] = slot;
      mi->unit_rt[i] = rt;
      if (p.has_shared && slot == 0) {  // the shared expert's down rows: into L2 now
        const size_t row = (size_t)rt * kDfRows;
        prefetch_l2(static_cast<const uint8_t*>(p.shared.w[2]) + row * rowb_dn, kDfRows * rowb_dn);
        prefetch_l2(p.shared.s[2] + row * Gf, kDfRows * Gf * 2);
      }
    }
    if (lane == 0) {
      mi->first_routed = first_routed;
      mi->n_tiles = nt;
      mi->n_split = n_split;
      mi->n_units = n_units;
    }
    __syncwarp();
  }

  // ---------------------------------------------------------------- router logits
  if (!producer) {
    // per-group sums of x as the GEMV kernels stage them: a half-warp a group, lane l the 8
    // values of 16-byte chunk l in order, then a fixed tree over the 16 chunks (the value of
    // chunk 0's lane); both half-warps run every pass, so the shuffles stay warp-uniform
    for (int pi = warp; pi < (G + 1) / 2; pi += kDfWarps) {
      const int gi = 2 * pi + (lane >> 4);
      uint4 v = make_uint4(0, 0, 0, 0);
      if (gi < G) v = reinterpret_cast<const uint4*>(s_x + gi * kGroup)[lane & 15];
      const uint32_t vv[4] = {v.x, v.y, v.z, v.w};
      float sm = 0.f;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        sm += __uint_as_float(vv[j] << 16);
        sm += __uint_as_float(vv[j] & 0xffff0000u);
      }
#pragma unroll
      for (int o = 8; o > 0; o >>= 1) sm += __shfl_xor_sync(0xffffffffu, sm, o);
      if (gi < G && (lane & 15) == 0) s_xsum[gi] = sm;
    }
    if (!mbar_wait(bar_router, 0)) {
      set_timeout(p.status, 20);
      mi->ok = 0;
    }
    // logits in the order of the fused routing kernel (route_fused.cu), so a token's logits
    // and gates are the same bits whichever of the two kernels routes it: lane l takes the
    // 16-byte pieces l, l + 32, ... of the row in batches of 8 (pieces past the row are
    // zeros), one fused multiply-add chain over each piece's 8 values in order, then a fixed
    // tree over the lanes, then the bias
    const int n16 = d / 8;
    const uint4* xrow = reinterpret_cast<const uint4*>(s_x);
    for (int r = warp; r < nr; r += kDfWarps) {
      const uint4* wrow = reinterpret_cast<const uint4*>(s_router + (size_t)r * d);
      float acc = 0.f;
      for (int c0 = 0; c0 < n16; c0 += 8 * 32) {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int cc = c0 + lane + 32 * i;
          const uint4 wv = (cc < n16) ? wrow[cc] : make_uint4(0, 0, 0, 0);
          const uint4 xv = (cc < n16) ? xrow[cc] : make_uint4(0, 0, 0, 0);
          const uint32_t ww[4] = {wv.x, wv.y, wv.z, wv.w};
          const uint32_t xx[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4) {
            acc = fmaf(__uint_as_float(xx[q4] << 16), __uint_as_float(ww[q4] << 16), acc);
            acc = fmaf(__uint_as_float(xx[q4] & 0xffff0000u), __uint_as_float(ww[q4] & 0xffff0000u),
                       acc);
          }
        }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
      const int e = r0 + r;
      if (lane == 0) p.logits[e] = acc + (p.router_bias ? p.router_bias[e] : 0.f);
    }
  }
  __syncthreads();  // S2: this CTA's logits are written

  // Items (tile position b, K-split part ks) over the tile range, in tile-major order; warp w
  // takes every kDfWarps-th. An item is part ks of both matrices of its tile: groups ks,
  // ks + kKsGateUp, ..., each added to the part's partial as a fused multiply-add of the
  // row's group scale and (group product - 136 x group sum of x), exactly as the GEMV kernels
  // accumulate a row (gemv_frag.cuh). Partials land in red[b][m][ks][16 rows].
  auto gate_up_items = [&](int b_begin, int b_end) {
    uint32_t xb[16];
    const int n_items = (b_end - b_begin) * kKsGateUp;
    for (int it = warp; it < n_items; it += kDfWarps) {
      const int b = b_begin + it / kKsGateUp, ks = it % kKsGateUp;
      if (!warp_wait(&bar_tile[b])) {
        if (lane == 0) set_timeout(p.status, 21);
        return;
      }
      const uint8_t* tile = smem + (size_t)b * L.tile_bytes;
      const uint16_t* scales = reinterpret_cast<const uint16_t*>(tile + 2 * kDfRows * rowb_up);
      float acc[2][2] = {{0.f, 0.f}, {0.f, 0.f}};  // [matrix][row grp, row grp + 8]
      for (int g = ks; g < G; g += kKsGateUp) {
        t1_load_act<false>(s_x, g, q, grp == 0, xb);
        const float corr = 136.f * s_xsum[g];
#pragma unroll
        for (int m = 0; m < 2; ++m) {
          float ra, rb;
          t1_group(tile + m * kDfRows * rowb_up, rowb_up, g, grp, q, xb, ra, rb);
          const uint16_t* sc = scales + m * kDfRows * G + g;
          acc[m][0] = fmaf(bf16_to_f32(sc[grp * G]), ra - corr, acc[m][0]);
          acc[m][1] = fmaf(bf16_to_f32(sc[(grp + 8) * G]), rb - corr, acc[m][1]);
        }
      }
      if (q == 0) {
        float* red_b = red + (size_t)b * 2 * kKsGateUp * kDfRows;
#pragma unroll
        for (int m = 0; m < 2; ++m) {
          red_b[(m * kKsGateUp + ks) * kDfRows + grp] = acc[m][0];
          red_b[(m * kKsGateUp + ks) * kDfRows + grp + 8] = acc[m][1];
        }
      }
    }
  };

  // ---------------------------------------------------------------- B1 (+ the shared tile)
  __shared__ uint32_t s_arrived;
  if (producer) {
    if (lane == 0) {
      s_arrived = gbar_arrive(gbar);
      if (mi->ok && (!gbar_wait(gbar, s_arrived) || !test_hold_wait(p.test_ctl))) {
        set_timeout(p.status, 22);
        mi->ok = 0;
      }
    }
    __syncwarp();  // the warp reaches the CTA barrier converged
  } else if (mi->ok) {
    gate_up_items(0, mi->first_routed);  // the shared tile, while B1 settles
  }
  __syncthreads();  // S3

  // ---------------------------------------------------------------- top-k (every CTA)
  // "a beats b": a larger logit, or an equal logit and a lower expert index; the k picks
  // are the experts that fewer than k others beat, in that order. Level 1: warp w ranks
  // each chunk of 32 consecutive experts (one per lane, 32 shuffles) and lists the chunk's
  // first kk = min(k, 32) in rank order. Level 2: each listed candidate among the first k
  // of its list counts, by binary search, how many entries of every other list beat it;
  // the sum is its overall rank. Gates: softmax over the picks, summed by a fixed tree.
  if (mi->ok && !producer) {
    const int n_chunks = (E + 31) / 32;
    const int kk = min(k, 32);
    uint32_t* cand = reinterpret_cast<uint32_t*>(smem + L.off_cand);  // [chunk][kk] key, idx
    for (int ch = warp; ch < n_chunks; ch += kDfWarps) {
      const int e = ch * 32 + lane;
      const uint32_t key = (e < E) ? order_key(__ldcg(p.logits + e)) : 0u;
      int rank = 0;
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        const uint32_t kj = __shfl_sync(0xffffffffu, key, j);
        rank += (kj > key) || (kj == key && j < lane);
      }
      if (rank < kk) {
        cand[2 * (ch * kk + rank)] = key;
        cand[2 * (ch * kk + rank) + 1] = (e < E) ? (uint32_t)e : 0xffffffffu;
      }
    }
    named_bar_sync(1, kDfCompute);
    // level 2 (warp 0): the k-th best chunk head bounds the picks from below (the k heads at
    // least as good beat anything it beats), so only candidates it does not beat remain;
    // they are ranked among themselves with shuffles (their overall rank: whatever beats a
    // remaining candidate remains too). More than 32 remaining (heavy ties): a table scan.
    if (warp == 0) {
      auto beats = [](uint32_t ka, uint32_t ia, uint32_t kb, uint32_t ib) {
        return ka > kb || (ka == kb && ia < ib);
      };
      const int n_cand = n_chunks * kk;
      uint32_t tk = 0u, ti = 0xffffffffu;  // the threshold: beats nothing valid by default
      if (n_chunks >= k) {
        const uint32_t hk = (lane < n_chunks) ? cand[2 * (lane * kk)] : 0u;
        const uint32_t hx = (lane < n_chunks) ? cand[2 * (lane * kk) + 1] : 0xffffffffu;
        int hr = 0;
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const uint32_t kj = __shfl_sync(0xffffffffu, hk, j), xj = __shfl_sync(0xffffffffu, hx, j);
          hr += (j < n_chunks) && beats(kj, xj, hk, hx);
        }
        const unsigned at = __ballot_sync(0xffffffffu, lane < n_chunks && hr == k - 1);
        const int tl = __ffs(at) - 1;
        tk = __shfl_sync(0xffffffffu, hk, tl);
        ti = __shfl_sync(0xffffffffu, hx, tl);
      }
      // compact the candidates the threshold does not beat (in table order)
      uint32_t* keep = cand + 2 * n_cand;  // room for n_cand entries after the table
      int n_keep = 0;
      for (int t0 = 0; t0 < n_cand; t0 += 32) {
        const int t = t0 + lane;
        uint32_t ck = 0u, cx = 0xffffffffu;
        if (t < n_cand) {
          ck = cand[2 * t];
          cx = cand[2 * t + 1];
        }
        const bool kp = (t < n_cand) && ck != 0u && !beats(tk, ti, ck, cx);
        const unsigned bal = __ballot_sync(0xffffffffu, kp);
        if (kp) {
          const int at = n_keep + __popc(bal & ((1u << lane) - 1u));
          keep[2 * at] = ck;
          keep[2 * at + 1] = cx;
        }
        n_keep += __popc(bal);
      }
      __syncwarp();
      if (n_keep <= 32) {
        const uint32_t ck = (lane < n_keep) ? keep[2 * lane] : 0u;
        const uint32_t cx = (lane < n_keep) ? keep[2 * lane + 1] : 0xffffffffu;
        int rank = 0;
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const uint32_t kj = __shfl_sync(0xffffffffu, ck, j), xj = __shfl_sync(0xffffffffu, cx, j);
          rank += (j < n_keep) && beats(kj, xj, ck, cx);
        }
        if (lane < n_keep && rank < k) {
          mi->sel[rank] = (int)cx;
          reinterpret_cast<uint32_t*>(mi->gate)[rank] = ck;  // key for now, gate below
        }
      } else {
        for (int t = lane; t < n_keep; t += 32) {
          const uint32_t ck = keep[2 * t], cx = keep[2 * t + 1];
          int rank = 0;
          for (int j = 0; j < n_keep; ++j) rank += beats(keep[2 * j], keep[2 * j + 1], ck, cx);
          if (rank < k) {
            mi->sel[rank] = (int)cx;
            reinterpret_cast<uint32_t*>(mi->gate)[rank] = ck;
          }
        }
      }
    }
    named_bar_sync(1, kDfCompute);
    if (warp == 0) {  // the gates as the routing kernels form them (warp_topk_gate)
      const uint32_t my_key = (lane < k) ? reinterpret_cast<const uint32_t*>(mi->gate)[lane] : 0u;
      const uint32_t top = __shfl_sync(0xffffffffu, my_key, 0);
      const float gate = warp_topk_gate(my_key, top, k, lane);
      __syncwarp();
      if (lane < k) mi->gate[lane] = gate;
    }
  }
  __syncthreads();  // S4: the routing decision
  const bool ok1 = mi->ok;

  // ---------------------------------------------------------------- gate/up tiles
  if (producer) {
    if (ok1) {
      // routed tiles, six copies each (gate and up in halves of 8 rows, then their scales),
      // one lane a copy; every tile's byte count is posted before any of its copies. The
      // router rows they overwrite were consumed before the CTA barrier above.
      const int n_routed = mi->n_tiles - mi->first_routed;
      if (lane < n_routed) mbar_arrive_expect_tx(&bar_tile[mi->first_routed + lane], L.tile_bytes);
      __syncwarp();
      for (int i = lane; i < 6 * n_routed; i += 32) {
        const int b = mi->first_routed + i / 6, part = i % 6;
        const uint32_t wbytes = kDfRows * rowb_up, sbytes = kDfRows * G * 2;
        const int j = mi->tile_slot[b] - p.has_shared;
        const size_t row = (size_t)mi->sel[j] * f + (size_t)mi->tile_rt[b] * kDfRows;
        uint8_t* dst = smem + (size_t)b * L.tile_bytes;
        if (part < 4) {
          const int m = part >> 1, half = part & 1;
          const uint32_t hb = wbytes / 2;
          bulk_g2s(dst + m * wbytes + half * hb,
                   static_cast<const uint8_t*>(p.routed.w[m]) + row * rowb_up + half * hb, hb,
                   &bar_tile[b]);
        } else {
          const int m = part - 4;
          bulk_g2s(dst + 2 * wbytes + m * sbytes, p.routed.s[m] + row * G, sbytes, &bar_tile[b]);
        }
      }
      if (lane == 0) mi->armed_tiles = mi->n_tiles;
      __syncwarp();
      // the routed down rows this CTA will need, into L2 behind the gate/up requests
      for (int i = lane; i < mi->n_units; i += 32) {
        const int slot = mi->unit_slot[i];
        if (p.has_shared && slot == 0) continue;
        const size_t row = (size_t)mi->sel[slot - p.has_shared] * d + (size_t)mi->unit_rt[i] * kDfRows;
        prefetch_l2(static_cast<const uint8_t*>(p.routed.w[2]) + row * rowb_dn, kDfRows * rowb_dn);
        prefetch_l2(p.routed.s[2] + row * Gf, kDfRows * Gf * 2);
      }
    }
    __syncwarp();
  } else if (ok1) {
    if (c == 0) {  // the plan outputs of the call
      if (tid < k) {
        const int e = mi->sel[tid];
        int rank = 0;
        for (int j = 0; j < k; ++j) rank += (mi->sel[j] < e);
        p.topk_idx[tid] = e;
        p.topk_w[tid] = mi->gate[tid];
        p.perm[rank] = tid;
        p.inv[tid] = rank;
      }
      for (int e = tid; e <= E; e += kDfCompute) {
        int cnt = 0;
        for (int j = 0; j < k; ++j) cnt += (mi->sel[j] < e);
        p.offsets[e] = cnt;
      }
    }
    gate_up_items(mi->first_routed, mi->n_tiles);
  }
  __syncthreads();  // S5: every gate/up product of this CTA is in red; tile buffers are free

  if (producer) {
    if (ok1) {
      // down units into the freed tile buffers (from L2 when the prefetch has landed), one
      // lane a unit, while the compute warps finish h
      for (int i = lane; i < mi->n_units; i += 32) {
        const int slot = mi->unit_slot[i];
        const bool sh = p.has_shared && slot == 0;
        const Bank& bk = sh ? p.shared : p.routed;
        const size_t e = sh ? 0 : (size_t)mi->sel[slot - p.has_shared];
        const size_t row = e * d + (size_t)mi->unit_rt[i] * kDfRows;
        const uint32_t wbytes = kDfRows * rowb_dn, sbytes = kDfRows * Gf * 2;
        uint8_t* dst = smem + (size_t)i * L.unit_bytes;
        mbar_arrive_expect_tx(&bar_unit[i], L.unit_bytes);
        bulk_g2s(dst, static_cast<const uint8_t*>(bk.w[2]) + row * rowb_dn, wbytes, &bar_unit[i]);
        bulk_g2s(dst + wbytes, bk.s[2] + row * Gf, sbytes, &bar_unit[i]);
      }
      if (lane == 0) mi->armed_units = mi->n_units;
    }
    __syncwarp();
  } else if (ok1) {
    // h rows of this CTA's tiles: the K-split partials added in part order (as the GEMV
    // kernels add them), SwiGLU, one rounding
    for (int i = tid; i < mi->n_tiles * kDfRows; i += kDfCompute) {
      const int b = i / kDfRows, r = i % kDfRows;
      const float* rg = red + (size_t)(b * 2) * kKsGateUp * kDfRows + r;
      const float* ru = rg + (size_t)kKsGateUp * kDfRows;
      float gs = 0.f, us = 0.f;
      for (int ks = 0; ks < kKsGateUp; ++ks) {
        gs += rg[ks * kDfRows];
        us += ru[ks * kDfRows];
      }
      const float hv = gs / (1.f + expf(-gs)) * us;
      p.h[(size_t)mi->tile_slot[b] * f + (size_t)mi->tile_rt[b] * kDfRows + r] = f32_to_bf16_rn(hv);
    }
  }
  __syncthreads();  // S6: h of this CTA written

  // ---------------------------------------------------------------- B2
  if (producer) {
    // every CTA arrives at every barrier, failed or not, so the word stays consistent
    if (lane == 0) {
      s_arrived = gbar_arrive(gbar);
      if (ok1 && !gbar_wait(gbar, s_arrived)) {
        set_timeout(p.status, 23);
        mi->ok = 0;
      }
      if (mi->ok) {  // every h row of the call, into shared memory in one request
        mbar_arrive_expect_tx(bar_h, (uint32_t)S * f * 2);
        mi->armed_h = 1;
      }
    }
    __syncwarp();
    // the h rows were written through the generic proxy by other CTAs before B2
    asm volatile("fence.proxy.async.global;" ::: "memory");
    if (mi->ok)
      for (int s = lane; s < S; s += 32)
        bulk_g2s(smem + L.off_h + (size_t)s * f * 2, p.h + (size_t)s * f, f * 2, bar_h);
    __syncwarp();
  }
  __syncthreads();  // S7: the B2 verdict
  const bool ok2 = mi->ok;

  // ---------------------------------------------------------------- down units
  // Compute warps: h to fragment order (+ group sums); pass A, the units of split tiles, and
  // their y rows to the workspace; then (the producer meanwhile posts the split-tile
  // arrivals and combines the split tiles it completes) pass B, the whole tiles, combined
  // locally. Both combines sum the gates in rank order, then the shared term, in fp32.
  uint16_t* hw = reinterpret_cast<uint16_t*>(smem + L.off_h);
  float* s_hsum = reinterpret_cast<float*>(smem + L.off_hsum);
  // Items (unit u, K-split part ks) in unit-major order from u_begin; warp w takes every
  // kDfWarps-th (kDfWarps is a multiple of kKsDown, so at most one part of a unit each). Part
  // ks sums groups ks, ks + kKsDown, ... as the GEMV kernels do; partials land in
  // red[u][ks][16 rows].
  static_assert(kDfWarps % kKsDown == 0, "one part of a unit per warp");
  auto down_items = [&](int u_begin, int u_end) {
    uint32_t xb[16];
    for (int u = u_begin; u < u_end; ++u) {
      const int slot = mi->unit_slot[u];
      const uint8_t* unit = smem + (size_t)u * L.unit_bytes;
      const uint16_t* scales = reinterpret_cast<const uint16_t*>(unit + kDfRows * rowb_dn);
      const int ks = ((warp - (u - u_begin) * kKsDown) % kDfWarps + kDfWarps) % kDfWarps;
      if (ks >= kKsDown) continue;
      if (!warp_wait(&bar_unit[u])) {
        if (lane == 0) set_timeout(p.status, 24);
        return;
      }
      float acc0 = 0.f, acc1 = 0.f;
      for (int g = ks; g < Gf; g += kKsDown) {
        const uint16_t* hrow = hw + (size_t)slot * f + g * kGroup + 32 * q;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          uint4 v = make_uint4(0, 0, 0, 0);
          if (grp == 0) v = *reinterpret_cast<const uint4*>(hrow + 8 * i);
          xb[4 * i + 0] = v.x;
          xb[4 * i + 1] = v.y;
          xb[4 * i + 2] = v.z;
          xb[4 * i + 3] = v.w;
        }
        float ra, rb;
        t1_group(unit, rowb_dn, g, grp, q, xb, ra, rb);
        const float corr = 136.f * s_hsum[slot * Gf + g];
        acc0 = fmaf(bf16_to_f32(scales[grp * Gf + g]), ra - corr, acc0);
        acc1 = fmaf(bf16_to_f32(scales[(grp + 8) * Gf + g]), rb - corr, acc1);
      }
      if (q == 0) {
        float* dst = red + ((size_t)u * kKsDown + ks) * kDfRows;
        dst[grp] = acc0;
        dst[grp + 8] = acc1;
      }
    }
  };
  // y of unit u, row r: the K-split partials added in part order
  auto unit_y = [&](int u, int r) {
    const float* src_r = red + (size_t)u * kKsDown * kDfRows + r;
    float y = 0.f;
    for (int ks = 0; ks < kKsDown; ++ks) y += src_r[ks * kDfRows];
    return y;
  };

  if (producer) {
    named_bar_sync(2, kDfThreads);  // the split-tile y rows of this CTA are written
    // Arrivals on the split tiles, one lane a tile (this CTA's split units are consecutive).
    // Every CTA posts its arrivals, failed or not, so the counters return to zero.
    const int ns = mi->n_split;
    const int first_rt = ns ? mi->unit_rt[0] : 0;
    const int rt = first_rt + lane;
    int n = 0;
    for (int i = 0; i < ns; ++i) n += (mi->unit_rt[i] == rt);
    bool mine = false;
    if (n > 0) {
      fence_acq_rel_gpu();
      const int old = atomicAdd(&tile_cnt[rt], n);
      if (old + n == S) {
        tile_cnt[rt] = 0;  // every unit of the tile has arrived: ready for the next call
        mine = ok2 && mi->ok;
        fence_acq_rel_gpu();
      }
    }
    unsigned m = __ballot_sync(0xffffffffu, mine);
    while (m) {  // combine the split tiles this CTA completed
      const int src_lane = __ffs(m) - 1;
      m &= m - 1;
      const int crt = __shfl_sync(0xffffffffu, rt, src_lane);
      if (lane < kDfRows) {
        const size_t nn = (size_t)crt * kDfRows + lane;
        float acc = 0.f;
        for (int j = 0; j < k; ++j)
          acc = fmaf(mi->gate[j], __ldcg(p.y_assign + (size_t)j * d + nn), acc);
        if (p.has_shared) acc += __ldcg(p.y_shared + nn);
        out[nn] = f32_to_bf16_rn(acc);
      }
    }
    __syncwarp();
  } else {
    bool ready = false;
    if (ok2) {
      ready = warp_wait(bar_h);
      if (!ready && lane == 0) set_timeout(p.status, 25);
      // h rows -> fragment order in place, and their per-group sums (a half-warp a group:
      // each lane one 8-value chunk, then a fixed tree over the 16 chunks)
      const int n_groups = S * Gf;
      for (int pi = warp; pi < (n_groups + 1) / 2 && ready; pi += kDfWarps) {
        const int gi = 2 * pi + (lane >> 4);  // both half-warps run every pass
        uint4* chunk = reinterpret_cast<uint4*>(hw + (size_t)min(gi, n_groups - 1) * kGroup) +
                       (lane & 15);
        uint4 v = *chunk;
        const uint32_t vv[4] = {v.x, v.y, v.z, v.w};
        float s = 0.f;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          s += __uint_as_float(vv[j] << 16);
          s += __uint_as_float(vv[j] & 0xffff0000u);
        }
        permute_chunk<4>(v);
        if (gi < n_groups) *chunk = v;
#pragma unroll
        for (int o = 8; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
        if (gi < n_groups && (lane & 15) == 0) s_hsum[gi] = s;
      }
    }
    named_bar_sync(1, kDfCompute);
    if (ok2 && ready) down_items(0, mi->n_split);  // pass A
    named_bar_sync(1, kDfCompute);
    if (ok2) {
      for (int i = tid; i < mi->n_split * kDfRows; i += kDfCompute) {
        const int u = i / kDfRows, r = i % kDfRows;
        const float y = unit_y(u, r);
        const int slot = mi->unit_slot[u];
        const size_t n = (size_t)mi->unit_rt[u] * kDfRows + r;
        if (p.has_shared && slot == 0) p.y_shared[n] = y;
        else p.y_assign[(size_t)(slot - p.has_shared) * d + n] = y;
      }
    }
    named_bar_sync(2, kDfThreads);
    if (ok2 && ready) down_items(mi->n_split, mi->n_units);  // pass B
    named_bar_sync(1, kDfCompute);
    if (ok2) {
      // y of every whole-tile unit row into red's first row of the unit (in place: a row's
      // partials are read before any thread writes that row's slot 0)
      float* ybuf = reinterpret_cast<float*>(smem + L.off_ybuf);  // [units][16]
      for (int i = tid; i < (mi->n_units - mi->n_split) * kDfRows; i += kDfCompute) {
        const int u = mi->n_split + i / kDfRows, r = i % kDfRows;
        ybuf[i] = unit_y(u, r);
      }
    }
    named_bar_sync(1, kDfCompute);
    if (ok2) {
      const float* ybuf = reinterpret_cast<const float*>(smem + L.off_ybuf);
      const int n_full = (mi->n_units - mi->n_split) / S;
      for (int i = tid; i < n_full * kDfRows; i += kDfCompute) {
        const int t = i / kDfRows, r = i % kDfRows;
        const float* yt = ybuf + (size_t)t * S * kDfRows + r;  // slot s at yt[s * 16]
        float acc = 0.f;
        for (int j = 0; j < k; ++j) acc = fmaf(mi->gate[j], yt[(p.has_shared + j) * kDfRows], acc);
        if (p.has_shared) acc += yt[0];
        out[(size_t)mi->unit_rt[mi->n_split + t * S] * kDfRows + r] = f32_to_bf16_rn(acc);
      }
    }
  }
  __syncthreads();

  // ---------------------------------------------------------------- drain
  // No copy may land after the CTA ends: wait (boundedly) for every one that was issued.
  // On the normal path every phase has completed already and each test is immediate.
  if (producer && lane == 0) {
    mbar_wait(bar_router, 0);
    for (int b = 0; b < mi->armed_tiles; ++b) mbar_wait(&bar_tile[b], 0);
    for (int u = 0; u < mi->armed_units; ++u) mbar_wait(&bar_unit[u], 0);
    if (mi->armed_h) mbar_wait(bar_h, 0);
  }
}

// ------------------------------------------------------------------ host side

namespace {
struct DfCache {
  std::mutex mu;
  int dev = -1, sms = 0;
  size_t smem_set = 0;
};
DfCache g_df;

cudaError_t df_sms(int* sms) {
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  std::lock_guard<std::mutex> lock(g_df.mu);
  if (g_df.dev != dev) {
    if ((err = cudaDeviceGetAttribute(&g_df.sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
      return err;
    g_df.dev = dev;
    g_df.smem_set = 0;
  }
  *sms = g_df.sms;
  return cudaSuccess;
}
}  // namespace

bool decode_fused_supported(const Plan& p) {
  if (p.T != 1 || p.routed.fmt != 4 || (p.has_shared && p.shared.fmt != 4)) return false;
  if (p.k > 32 || p.E > kMaxE || p.d % kDfRows || p.f % kDfRows) return false;
  int sms = 0;
  if (df_sms(&sms) != cudaSuccess || sms < 1) return false;
  const DfLayout L = df_layout(sms, p.d, p.f, p.E, p.k, p.has_shared);
  if (L.tiles_max > kDfMaxTiles || L.units_max > kDfMaxUnits || L.router_max > kDfMaxRouter)
    return false;
  if (L.total > 227u * 1024u) return false;
  // bulk copies: 16-byte aligned sources (scales too)
  for (int i = 0; i < 3; ++i) {
    if (reinterpret_cast<uintptr_t>(p.routed.s[i]) % 16) return false;
    if (p.has_shared && reinterpret_cast<uintptr_t>(p.shared.s[i]) % 16) return false;
  }
  return true;
}

cudaError_t launch_decode_fused(const Plan& p, void* out, cudaStream_t st) {
  uint32_t* gbar = p.gbar;
  int32_t* tile_cnt = p.tile_cnt;
  int sms = 0;
  cudaError_t err = df_sms(&sms);
  if (err != cudaSuccess) return err;
  const DfLayout L = df_layout(sms, p.d, p.f, p.E, p.k, p.has_shared);
  {
    std::lock_guard<std::mutex> lock(g_df.mu);
    if (L.total > g_df.smem_set) {
      err = cudaFuncSetAttribute(decode_fused_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)L.total);
      if (err != cudaSuccess) return err;
      g_df.smem_set = L.total;
    }
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(sms);
  cfg.blockDim = dim3(kDfThreads);
  cfg.dynamicSmemBytes = L.total;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, decode_fused_kernel, p, static_cast<uint16_t*>(out), gbar,
                            tile_cnt);
}

}  // namespace moe
