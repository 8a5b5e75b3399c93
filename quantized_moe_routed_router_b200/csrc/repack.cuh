// Open-time repack: user blobs (rows of Q8_0 / MXFP4 blocks) -> the
// tile-major fragment layout described in layout.cuh.  Runs once per layer
// at ts_moe_open (the pages' repack transcode, gpt-oss state page `read_bias`:
// the install is transcoded once and read back at open).
//
// For lane (g, c) of a warp (g = lane/4, c = lane%4) and a chunk of K, the
// 16 bytes it owns are its m16n8k16 A fragments for the chunk: tile rows g and
// g+8, K offsets 16s + 4c .. 16s + 4c + 3 of each 16-wide step s.  Within a
// step the MMA sees K positions (2c, 2c+1, 2c+8, 2c+9) carry original
// elements (4c, 4c+1, 4c+2, 4c+3); the activation window feeds the same
// order, so the dot product is unchanged.
//   MXFP4 (4 steps, 64 K): word s = bytes {row g: codes(4c,4c+1), row g+8:
//     codes(4c,4c+1), row g: codes(4c+2,4c+3), row g+8: codes(4c+2,4c+3)} --
//     exactly the original packed bytes, one byte per register of the A
//     fragment; scales per quad g: {e(g, blk0), e(g+8, blk0), e(g, blk1), e(g+8, blk1)}.
//   Q8_0 (2 steps, 32 K): per step two words {row g: q(4c), q(4c+1), row g+8:
//     q(4c), q(4c+1)}, {.. q(4c+2), q(4c+3) ..}, each byte stored as q + 128;
//     scales per quad g: {d(g), d(g+8)} fp16.
//   INT4-affine (2 steps, 32 K = one block): per step one word of eight
//     nibbles, low to high {g: e0, g+8: e0, g: e2, g+8: e2, g: e1, g+8: e1,
//     g: e3, g+8: e3} (e_i = element 16s + 4c + i), so that masks of nibbles
//     0/4 and 1/5 (and of the word shifted by 8) land in FP16 mantissas as the
//     A fragment's register pairs; per quad g {d(g), d(g+8), m(g), m(g+8)}.
#pragma once
#include "common.cuh"
#include "layout.cuh"

namespace tsm {

enum : unsigned { BAD_E8M0_NAN = 1u, BAD_Q8_SCALE = 2u, BAD_ROUTER_SCALE = 4u, BAD_I4_SCALE = 8u };

// Nibble `e` (0..31) of an INT4-affine block's code bytes.
TSM_DEV uint32_t i4_code(const uint8_t* qs, int e) { return (qs[e >> 1] >> ((e & 1) * 4)) & 0xFu; }

// PHASE 0: tile t rows 0..7 = gate rows 8t..8t+7, rows 8..15 = up rows
// 8t..8t+7 (matrices [rows][row_bytes]); PHASE 1: tile t rows = rows
// 16t..16t+15 of a [nrows][row_bytes] matrix (down, or the router); tile rows
// at or past nrows repack as zero weights with zero scale.
template <int FMT, int PHASE>
__global__ void repack_kernel(const uint8_t* __restrict__ a, const uint8_t* __restrict__ b, int row_bytes,
                              int nblocks, int tiles, int chunks, int gs, uint8_t* __restrict__ dst, unsigned* bad,
                              int nrows) {
  const int lane = threadIdx.x & 31;
  const int g = lane >> 2, c = lane & 3;
  const long long total = (long long)tiles * chunks;
  const long long nw = (long long)gridDim.x * (blockDim.x >> 5);
  unsigned mybad = 0;
  for (long long u = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); u < total; u += nw) {
    const int t = (int)(u / chunks), ck = (int)(u % chunks);
    const int grp = t / gs, jt = t % gs;
    const int ntg = group_tiles(tiles, gs, grp);
    constexpr int UB = FMT == FMT_INT4_AFFINE ? UNIT_BYTES_I4 : UNIT_BYTES;
    uint8_t* unit = dst + group_offset(gs, chunks, grp, UB) + ((uint64_t)ck * ntg + jt) * UB;
    const uint8_t* rg;
    const uint8_t* rg8;
    bool zg = false, zg8 = false;
    if (PHASE == 0) {
      rg = a + (size_t)(8 * t + g) * row_bytes;
      rg8 = b + (size_t)(8 * t + g) * row_bytes;
    } else {
      zg = 16 * t + g >= nrows;
      zg8 = 16 * t + g + 8 >= nrows;
      rg = a + (size_t)(zg ? 0 : 16 * t + g) * row_bytes;
      rg8 = a + (size_t)(zg8 ? 0 : 16 * t + g + 8) * row_bytes;
    }
    uint32_t w[4];
    if (FMT == FMT_INT4_AFFINE) {
      const uint8_t* qg = rg + ck * 20 + 4;
      const uint8_t* qg8 = rg8 + ck * 20 + 4;
#pragma unroll
      for (int s = 0; s < 2; ++s) {
        const int e0 = 16 * s + 4 * c;
        const uint32_t n[8] = {i4_code(qg, e0),     i4_code(qg8, e0),     i4_code(qg, e0 + 2), i4_code(qg8, e0 + 2),
                               i4_code(qg, e0 + 1), i4_code(qg8, e0 + 1), i4_code(qg, e0 + 3), i4_code(qg8, e0 + 3)};
        uint32_t v = 0;
#pragma unroll
        for (int i = 0; i < 8; ++i) v |= n[i] << (4 * i);
        if (zg) v &= 0xF0F0F0F0u;   // row g nibbles are 0, 2, 4, 6
        if (zg8) v &= 0x0F0F0F0Fu;                      // row g+8 nibbles are 1, 3, 5, 7
        w[s] = v;
      }
      w[2] = w[3] = 0u;
    } else if (FMT == FMT_MXFP4) {
#pragma unroll
      for (int s = 0; s < 4; ++s) {
        const int blk = 2 * ck + s / 2;
        uint32_t v = 0;
        if (blk < nblocks) {
          const int o = blk * 17 + 1 + 8 * (s % 2) + 2 * c;
          v = (uint32_t)rg[o] | ((uint32_t)rg8[o] << 8) | ((uint32_t)rg[o + 1] << 16) | ((uint32_t)rg8[o + 1] << 24);
          if (zg) v &= 0xFF00FF00u;
          if (zg8) v &= 0x00FF00FFu;
        }
        w[s] = v;
      }
    } else {
      const uint8_t* qg = rg + ck * 34 + 2;
      const uint8_t* qg8 = rg8 + ck * 34 + 2;
#pragma unroll
      for (int s = 0; s < 2; ++s) {
        const int o = 16 * s + 4 * c;
        w[2 * s] = ((uint32_t)qg[o] | ((uint32_t)qg[o + 1] << 8) | ((uint32_t)qg8[o] << 16) |
                    ((uint32_t)qg8[o + 1] << 24)) ^ 0x80808080u;
        w[2 * s + 1] = ((uint32_t)qg[o + 2] | ((uint32_t)qg[o + 3] << 8) | ((uint32_t)qg8[o + 2] << 16) |
                        ((uint32_t)qg8[o + 3] << 24)) ^ 0x80808080u;
        if (zg) {  // q = 0 is stored as 0x80
          w[2 * s] = (w[2 * s] & 0xFFFF0000u) | 0x8080u;
          w[2 * s + 1] = (w[2 * s + 1] & 0xFFFF0000u) | 0x8080u;
        }
        if (zg8) {
          w[2 * s] = (w[2 * s] & 0x0000FFFFu) | 0x80800000u;
          w[2 * s + 1] = (w[2 * s + 1] & 0x0000FFFFu) | 0x80800000u;
        }
      }
    }
    if (FMT == FMT_INT4_AFFINE)
      *reinterpret_cast<uint2*>(unit + lane * 8) = make_uint2(w[0], w[1]);
    else
      *reinterpret_cast<uint4*>(unit + lane * 16) = make_uint4(w[0], w[1], w[2], w[3]);
    if (lane < 8) {
      // scales of the quad of rows (lane, lane + 8)
      const uint8_t* sg;
      const uint8_t* sg8;
      bool zs = false, zs8 = false;
      if (PHASE == 0) {
        sg = a + (size_t)(8 * t + lane) * row_bytes;
        sg8 = b + (size_t)(8 * t + lane) * row_bytes;
      } else {
        zs = 16 * t + lane >= nrows;
        zs8 = 16 * t + lane + 8 >= nrows;
        sg = a + (size_t)(zs ? 0 : 16 * t + lane) * row_bytes;
        sg8 = a + (size_t)(zs8 ? 0 : 16 * t + lane + 8) * row_bytes;
      }
      uint32_t sw;
      if (FMT == FMT_INT4_AFFINE) {
        const uint32_t d0 = zs ? 0u : (uint32_t)sg[ck * 20] | ((uint32_t)sg[ck * 20 + 1] << 8);
        const uint32_t d1 = zs8 ? 0u : (uint32_t)sg8[ck * 20] | ((uint32_t)sg8[ck * 20 + 1] << 8);
        const uint32_t m0 = zs ? 0u : (uint32_t)sg[ck * 20 + 2] | ((uint32_t)sg[ck * 20 + 3] << 8);
        const uint32_t m1 = zs8 ? 0u : (uint32_t)sg8[ck * 20 + 2] | ((uint32_t)sg8[ck * 20 + 3] << 8);
        if ((d0 & 0x7C00u) == 0x7C00u || (d1 & 0x7C00u) == 0x7C00u || (m0 & 0x7C00u) == 0x7C00u ||
            (m1 & 0x7C00u) == 0x7C00u)
          mybad |= BAD_I4_SCALE;
        *reinterpret_cast<uint2*>(unit + QUANT_BYTES_I4 + lane * 8) = make_uint2(d0 | (d1 << 16), m0 | (m1 << 16));
        continue;
      } else if (FMT == FMT_MXFP4) {
        uint32_t e[4] = {0, 0, 0, 0};
        if (2 * ck < nblocks) {
          e[0] = sg[(2 * ck) * 17];
          e[1] = sg8[(2 * ck) * 17];
        }
        if (2 * ck + 1 < nblocks) {
          e[2] = sg[(2 * ck + 1) * 17];
          e[3] = sg8[(2 * ck + 1) * 17];
        }
        if (zs) e[0] = e[2] = 0;
        if (zs8) e[1] = e[3] = 0;
        for (int i = 0; i < 4; ++i)
          if (e[i] == 255u) mybad |= BAD_E8M0_NAN;
        sw = e[0] | (e[1] << 8) | (e[2] << 16) | (e[3] << 24);
      } else {
        const uint32_t d0 = zs ? 0u : (uint32_t)sg[ck * 34] | ((uint32_t)sg[ck * 34 + 1] << 8);
        const uint32_t d1 = zs8 ? 0u : (uint32_t)sg8[ck * 34] | ((uint32_t)sg8[ck * 34 + 1] << 8);
        if ((d0 & 0x7C00u) == 0x7C00u || (d1 & 0x7C00u) == 0x7C00u) mybad |= BAD_Q8_SCALE;
        sw = d0 | (d1 << 16);
      }
      *reinterpret_cast<uint32_t*>(unit + QUANT_BYTES + lane * 4) = sw;
    }
  }
  if (mybad) atomicOr(bad, mybad);
}

}  // namespace tsm
