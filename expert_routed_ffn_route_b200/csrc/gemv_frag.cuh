// Fragment helpers shared by the grouped GEMV kernels: quantised weight words -> bf16
// tensor-core A fragments (m16n8k16), and activation rows staged in shared memory in the
// matching order.
//
// A 16-row weight tile times up to 8 tokens is one mma.sync m16n8k16 per 16-wide K step.
// Lane (grp = lane / 4, q = lane % 4) holds rows grp and grp + 8; over one 128-wide K group
// it owns the 32 consecutive K values [32 q, 32 q + 32) of its rows (one 16-byte int4 load
// per row) and feeds them to the 8 MMAs of the group as its four "virtual" k columns
// (2q, 2q+1, 2q+8, 2q+9). The activation operand uses the same real K positions, which
// keeps every dot product exact in its terms, whatever the order of k inside an MMA.
#pragma once

#include "common.cuh"

namespace moe {

constexpr int kTok = 8;       // tokens per MMA (N)

// K split of one weight row's 128-wide groups: split part ks sums groups ks, ks + KS, ...
// (a fused multiply-add chain of scale x (group product - offset correction)), and the
// parts are added in ks order. The GEMV kernels and the single-kernel 1-token layer use the
// same split, so a token's row comes out bit for bit the same whichever of them computes it.
constexpr int kKsGateUp = 8;  // gate/up (K = d)
constexpr int kKsDown = 4;    // down (K = f)

template <int FMT> struct FmtInfo;
template <> struct FmtInfo<4> { static constexpr int U = 1; static constexpr int bits = 4; };
template <> struct FmtInfo<8> { static constexpr int U = 2; static constexpr int bits = 8; };
template <> struct FmtInfo<16> { static constexpr int U = 4; static constexpr int bits = 16; };

// Physical 8-byte unit of logical unit u inside a staged activation row. The XOR spreads
// the four lanes of a quad over distinct banks; together with a row stride of 2K + 8 bytes
// every half-warp's 8-byte reads are conflict free.
__device__ __forceinline__ int phys_unit(int u) { return u ^ (((u >> 4) & 1) << 2); }

__device__ __forceinline__ void mma_bf16_16x8x16(float (&c)[4], uint32_t a0, uint32_t a1,
                                                 uint32_t a2, uint32_t a3, uint32_t b0,
                                                 uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t lop_and_xor(uint32_t a, uint32_t mask, uint32_t xorv) {
  uint32_t r;
  asm("lop3.b32 %0, %1, %2, %3, 0x6A;" : "=r"(r) : "r"(a), "r"(mask), "r"(xorv));  // (a&b)^c
  return r;
}

// A fragments of one weight row for the 8 MMAs of a 128-wide K group.
// fr[m][0] holds the pair for virtual k (2q, 2q+1), fr[m][1] for (2q+8, 2q+9).
template <int FMT>
__device__ __forceinline__ void to_frags(const uint4 (&raw)[FmtInfo<FMT>::U], uint32_t (&fr)[8][2]);

// int4: ((w >> s) & 0x000F000F) ^ 0x43084308 puts nibble n (of two 16-bit halves at once)
// into the mantissa of 128.0 with its sign bit flipped: the bf16 value 128 + (n ^ 8) =
// q + 136, exact, in one LOP3 per register.
template <>
__device__ __forceinline__ void to_frags<4>(const uint4 (&raw)[1], uint32_t (&fr)[8][2]) {
  const uint32_t w[4] = {raw[0].x, raw[0].y, raw[0].z, raw[0].w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    fr[2 * i][0] = lop_and_xor(w[i], 0x000F000Fu, 0x43084308u);        // nibbles 0, 4
    fr[2 * i][1] = lop_and_xor(w[i] >> 4, 0x000F000Fu, 0x43084308u);   // nibbles 1, 5
    fr[2 * i + 1][0] = lop_and_xor(w[i] >> 8, 0x000F000Fu, 0x43084308u);  // 2, 6
    fr[2 * i + 1][1] = lop_and_xor(w[i] >> 12, 0x000F000Fu, 0x43084308u); // 3, 7
  }
}

__device__ __forceinline__ uint32_t i8pair_to_bf16x2(uint32_t w, int lo_byte) {
  const float a = static_cast<float>(static_cast<int8_t>((w >> (8 * lo_byte)) & 0xff));
  const float b = static_cast<float>(static_cast<int8_t>((w >> (8 * lo_byte + 8)) & 0xff));
  return pack_bf16x2(a, b);  // exact: |q| <= 127
}

template <>
__device__ __forceinline__ void to_frags<8>(const uint4 (&raw)[2], uint32_t (&fr)[8][2]) {
  const uint32_t w[8] = {raw[0].x, raw[0].y, raw[0].z, raw[0].w,
                         raw[1].x, raw[1].y, raw[1].z, raw[1].w};
#pragma unroll
  for (int m = 0; m < 8; ++m) {
    fr[m][0] = i8pair_to_bf16x2(w[m], 0);
    fr[m][1] = i8pair_to_bf16x2(w[m], 2);
  }
}

template <>
__device__ __forceinline__ void to_frags<16>(const uint4 (&raw)[4], uint32_t (&fr)[8][2]) {
  const uint32_t w[16] = {raw[0].x, raw[0].y, raw[0].z, raw[0].w, raw[1].x, raw[1].y,
                          raw[1].z, raw[1].w, raw[2].x, raw[2].y, raw[2].z, raw[2].w,
                          raw[3].x, raw[3].y, raw[3].z, raw[3].w};
#pragma unroll
  for (int m = 0; m < 8; ++m) {
    fr[m][0] = w[2 * m];
    fr[m][1] = w[2 * m + 1];
  }
}

// One staged 16-byte chunk (8 bf16 of an activation row) in the order the A fragments use:
// int4 pairs nibble i with nibble i + 4 inside each 8-wide word, so the chunk is stored as
// elements (0,4,1,5,2,6,3,7); the other formats keep the natural order.
template <int FMT>
__device__ __forceinline__ void permute_chunk(uint4& v) {
  if constexpr (FMT == 4) {
    const uint32_t a = v.x, b = v.y, c = v.z, d = v.w;  // (0,1) (2,3) (4,5) (6,7)
    v.x = __byte_perm(a, c, 0x5410);  // 0, 4
    v.y = __byte_perm(a, c, 0x7632);  // 1, 5
    v.z = __byte_perm(b, d, 0x5410);  // 2, 6
    v.w = __byte_perm(b, d, 0x7632);  // 3, 7
  }
}

struct StageArgs {
  const uint16_t* src;   // activation rows (bf16)
  int src_stride;        // elements between rows
  const int32_t* perm;   // grouped row -> assignment (routed gate/up) or NULL
  int k;                 // routed experts a token (assignment -> token)
  int row0, nrows;       // rows [row0, row0 + nrows) of this chunk (grouped numbering)
};

// Stage up to 8 activation rows into shared memory (and per-group sums for int4).
// Loads are issued in batches of 4 items per thread before any of them is used, so a row
// costs two dependent L2 round trips (row index, then data) instead of one per item.
template <int FMT, int NT>
__device__ void stage_rows(const StageArgs& a, int K, uint8_t* xs, int S, float* xsum, int tid) {
  constexpr int B = 4;
  const int chunks = K / 8;  // 16-byte chunks per row (a multiple of 16)
  const int G = K / kGroup;
  const int n_items = a.nrows * chunks;
  for (int i0 = 0; i0 < n_items; i0 += B * NT) {
    const uint16_t* src[B];
#pragma unroll
    for (int j = 0; j < B; ++j) {
      const int i = i0 + j * NT + tid;
      src[j] = nullptr;
      if (i < n_items) {
        const int row = i / chunks;
        int src_row = a.row0 + row;
        if (a.perm) src_row = __ldg(a.perm + src_row) / a.k;
        src[j] = a.src + (size_t)src_row * a.src_stride + 8 * (i - row * chunks);
      }
    }
    uint4 v[B];
#pragma unroll
    for (int j = 0; j < B; ++j)
      v[j] = src[j] ? *reinterpret_cast<const uint4*>(src[j]) : make_uint4(0, 0, 0, 0);
#pragma unroll
    for (int j = 0; j < B; ++j) {
      const int i = i0 + j * NT + tid;
      if (i0 + j * NT >= n_items) break;  // uniform across the CTA
      const int row = i / chunks, c = i - row * chunks;
      if constexpr (FMT == 4) {
        // fixed-order sum of the chunk, then over the 16 chunks of its group (a half-warp)
        const uint32_t vv[4] = {v[j].x, v[j].y, v[j].z, v[j].w};
        float sm = 0.f;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          sm += __uint_as_float(vv[q] << 16);
          sm += __uint_as_float(vv[q] & 0xffff0000u);
        }
#pragma unroll
        for (int o = 8; o > 0; o >>= 1) sm += __shfl_xor_sync(0xffffffffu, sm, o);
        if (i < n_items && (c & 15) == 0) xsum[row * G + c / 16] = sm;
      }
      if (i < n_items) {
        uint4 w = v[j];
        permute_chunk<FMT>(w);
        uint8_t* rowp = xs + (size_t)row * S;
        *reinterpret_cast<uint2*>(rowp + 8 * phys_unit(2 * c)) = make_uint2(w.x, w.y);
        *reinterpret_cast<uint2*>(rowp + 8 * phys_unit(2 * c + 1)) = make_uint2(w.z, w.w);
      }
    }
  }
  // rows nrows..7 are zero (their products are computed and discarded)
  const int z_items = (kTok - a.nrows) * chunks;
  for (int i = tid; i < z_items; i += NT) {
    const int row = a.nrows + i / chunks, c = i % chunks;
    uint8_t* rowp = xs + (size_t)row * S;
    *reinterpret_cast<uint2*>(rowp + 8 * phys_unit(2 * c)) = make_uint2(0, 0);
    *reinterpret_cast<uint2*>(rowp + 8 * phys_unit(2 * c + 1)) = make_uint2(0, 0);
    if (FMT == 4 && (c & 15) == 0) xsum[row * G + c / 16] = 0.f;
  }
}

// Multiply one K group: NM matrices (gate+up or down) on the 8 staged tokens.
template <int FMT, int NM>
__device__ __forceinline__ void group_mma(const uint4 (&ra)[NM][FmtInfo<FMT>::U],
                                          const uint4 (&rb)[NM][FmtInfo<FMT>::U],
                                          const float (&sa)[NM], const float (&sb)[NM],
                                          const uint8_t* xrow, const float* xsum, int G, int g,
                                          int q4, float (&acc)[NM][4]) {
  uint32_t fa[NM][8][2], fb[NM][8][2];
#pragma unroll
  for (int mi = 0; mi < NM; ++mi) {
    to_frags<FMT>(ra[mi], fa[mi]);
    to_frags<FMT>(rb[mi], fb[mi]);
  }
  float c[NM][4];
#pragma unroll
  for (int mi = 0; mi < NM; ++mi)
#pragma unroll
    for (int i = 0; i < 4; ++i) c[mi][i] = 0.f;
  uint2 bfr[8];
#pragma unroll
  for (int m = 0; m < 8; ++m)
    bfr[m] = *reinterpret_cast<const uint2*>(xrow + 8 * phys_unit(32 * g + 8 * q4 + m));
#pragma unroll
  for (int m = 0; m < 8; ++m) {
#pragma unroll
    for (int mi = 0; mi < NM; ++mi)
      mma_bf16_16x8x16(c[mi], fa[mi][m][0], fb[mi][m][0], fa[mi][m][1], fb[mi][m][1],
                       bfr[m].x, bfr[m].y);
  }
  float corr0 = 0.f, corr1 = 0.f;
  if constexpr (FMT == 4) {
    corr0 = 136.f * xsum[(2 * q4) * G + g];
    corr1 = 136.f * xsum[(2 * q4 + 1) * G + g];
  }
#pragma unroll
  for (int mi = 0; mi < NM; ++mi) {
    acc[mi][0] = fmaf(sa[mi], c[mi][0] - corr0, acc[mi][0]);
    acc[mi][1] = fmaf(sa[mi], c[mi][1] - corr1, acc[mi][1]);
    acc[mi][2] = fmaf(sb[mi], c[mi][2] - corr0, acc[mi][2]);
    acc[mi][3] = fmaf(sb[mi], c[mi][3] - corr1, acc[mi][3]);
  }
}

}  // namespace moe
