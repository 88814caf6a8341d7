// lores_mma.cuh -- decode-step kernel for heads stored one byte or one nibble per code
// with one scale per value row (G = d_k), sm_100a.
//
// The same step as decode_step_kernel ("Quantizing Recurrent Language Models Is Easier
// Than You Think", summary page: General recurrence form; Key properties item 3;
// Proposition 1; Proposition 3 / Table 6), with the same results bit for bit.  The
// contractions S'k and S'q run on the integer tensor cores: the codes of 16 value rows
// (the A operand, straight from shared memory) times the four base-256 digits of the
// fixed-point alpha k and alpha q (the B operand: 8 columns, digit planes built once per
// tile), mma.sync m16n8k32 s8 (m16n8k16 at d_k = 16) with exact int32 accumulation.  The
// CUDA cores keep the per-entry work: dequantize, x = S' + w k^T, group maximum, dither,
// requantize.
//
// Lane layout (g = lane / 4, t = lane % 4): a strip is 16 rows; lane (g, t) owns rows g
// and g + 8 of the strip and d_k / 4 columns of each, in 16-column chunks at 64 c + 16 t
// (d_k >= 64), or columns 8t.. (d_k = 32) or 4t.. (d_k = 16).  Word m of a lane's row
// (4 columns) is A-operand register a0 / a2 (row g) and a1 / a3 (row g + 8) of k-block
// m / 2: the MMA sums every k-block over 32 columns in an order of its own, which is
// harmless because the sums are exact integers; the B operand of lane (g', t) holds
// digit plane g' at the same columns.  The D fragment gives lane t digit columns 2t and
// 2t + 1: lanes t = 0, 1 hold k's digit sums, t = 2, 3 q's; two shuffles assemble both.
#pragma once
#include <cstdint>

#include "lores_device.cuh"
#include "lores_step.cuh"
#include "lores_pair.cuh"

// CTAs per SM the register allocation is sized for (128 threads each).
#ifndef LORES_MMA_MIN_CTAS
#define LORES_MMA_MIN_CTAS 3
#endif

namespace lores {

// D += A (16 x 32, s8) * B (32 x 8, s8), int32 accumulators.  mma.sync is a warp-wide
// instruction that the whole warp must execute converged: the asm is volatile (not moved
// or duplicated by the compiler) and the caller issues it right after a __syncwarp.
__device__ __forceinline__ void mma_k32(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                        uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile("mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
// D += A (16 x 16, s8) * B (16 x 8, s8)
__device__ __forceinline__ void mma_k16(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t b0) {
  asm volatile("mma.sync.aligned.m16n8k16.row.col.s32.s8.s8.s32 {%0,%1,%2,%3}, {%4,%5}, {%6}, "
      "{%0,%1,%2,%3};"
      : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
      : "r"(a0), "r"(a1), "r"(b0));
}

template <int DK>
struct MmaGeom {
  static constexpr int CPL = DK / 4;                   // columns per lane-row
  static constexpr int NW = CPL / 4;                   // 4-column words per lane-row
  static constexpr int NCH = DK >= 64 ? CPL / 16 : 1;  // 16-column chunks per lane-row
  static constexpr int CH = DK >= 64 ? 16 : CPL;       // columns per chunk
  // first column of chunk c of lane t
  static __device__ __forceinline__ int col(int t, int c) { return DK >= 64 ? 64 * c + 16 * t : CH * t; }
};

// The tile's registers: the B operand (digit plane g at the lane's columns), 2^-E of the
// lane's vector (k for t < 2, q for t >= 2), k.q, beta and scalar alpha, the dither key.
// k (and per-column alpha) stay in the warp's scratch, read per strip.
template <int DK, bool DIAG>
struct MmaTile {
  uint32_t bf[DK / 16];
  double sx;
  float kq, alpha, beta;
  uint32_t tkey;
};

// Tile setup from its k, q (and per-column alpha) in shared or global memory: the digit
// planes of the fixed-point alpha k (planes 0-3) and alpha q (planes 4-7) in the warp's
// scratch (8 d_k bytes), then the lane's B operand; k and alpha are copied after the
// planes (kept: 4 d_k bytes each), where the copy ring cannot overwrite them.
template <int DK, bool DIAG>
__device__ __forceinline__ void mma_tile(const float *k, const float *q, const float *alpha,
                                         float alpha_s, uint8_t *planes, MmaTile<DK, DIAG> &t) {
  using Gm = MmaGeom<DK>;
  const int lane = threadIdx.x & 31, g = lane >> 2, tq = lane & 3;
  __syncwarp();                                     // the previous tile's B loads are done
  const double sk = fixed_point_planes<DK>(k, alpha, DIAG, alpha_s, planes, DK);
  const double sq = fixed_point_planes<DK>(q, alpha, DIAG, alpha_s, planes + 4 * DK, DK);
  __syncwarp();
  const uint8_t *pl = planes + g * DK;
#pragma unroll
  for (int c = 0; c < Gm::NCH; ++c) {
    const uint8_t *src = pl + Gm::col(tq, c);
    if (Gm::CH == 16) {
      const uint4 w = *reinterpret_cast<const uint4 *>(src);
      t.bf[4 * c] = w.x; t.bf[4 * c + 1] = w.y; t.bf[4 * c + 2] = w.z; t.bf[4 * c + 3] = w.w;
    } else if (Gm::CH == 8) {
      const uint2 w = *reinterpret_cast<const uint2 *>(src);
      t.bf[0] = w.x; t.bf[1] = w.y;
    } else {
      t.bf[0] = *reinterpret_cast<const uint32_t *>(src);
    }
  }
  t.sx = tq < 2 ? sk : sq;
  float *kkeep = reinterpret_cast<float *>(planes + 8 * DK);
  float *akeep = kkeep + DK;
  for (int j = lane; j < DK; j += 32) {
    kkeep[j] = k[j];
    if (DIAG) akeep[j] = alpha[j];
  }
  __syncwarp();
}

// A lane's codes of one row: NW words of 4 signed bytes (int4 codes widened), column order.
template <int DK, int BITS>
__device__ __forceinline__ void mma_load_row(const uint8_t *row, int tq, uint32_t (&w)[DK / 16]) {
  using Gm = MmaGeom<DK>;
#pragma unroll
  for (int c = 0; c < Gm::NCH; ++c) {
    const int col = Gm::col(tq, c);
    if (BITS == 8) {
      if (Gm::CH == 16) {
        const uint4 v = *reinterpret_cast<const uint4 *>(row + col);
        w[4 * c] = v.x; w[4 * c + 1] = v.y; w[4 * c + 2] = v.z; w[4 * c + 3] = v.w;
      } else if (Gm::CH == 8) {
        const uint2 v = *reinterpret_cast<const uint2 *>(row + col);
        w[0] = v.x; w[1] = v.y;
      } else {
        w[0] = *reinterpret_cast<const uint32_t *>(row + col);
      }
    } else {
      if (Gm::CH == 16) {
        uint32_t s[4];
        i4_to_s8(*reinterpret_cast<const uint2 *>(row + col / 2), s);
        w[4 * c] = s[0]; w[4 * c + 1] = s[1]; w[4 * c + 2] = s[2]; w[4 * c + 3] = s[3];
      } else if (Gm::CH == 8) {
        const uint32_t nb = *reinterpret_cast<const uint32_t *>(row + col / 2);
        uint32_t s[4];
        i4_to_s8(make_uint2(nb, 0u), s);
        w[0] = s[0]; w[1] = s[1];
      } else {
        const uint32_t nb = *reinterpret_cast<const uint16_t *>(row + col / 2);
        uint32_t s[4];
        i4_to_s8(make_uint2(nb, 0u), s);
        w[0] = s[0];
      }
    }
  }
}

// Signed code bytes (4 per word) -> exact floats in column pairs.
__device__ __forceinline__ void s8_floats(uint32_t w, float2 &lo, float2 &hi) {
  const uint32_t ob = w ^ 0x80808080u;
  const float2 off = byte_bias(128);
  lo = byte_pair_minus(ob, 0, off);
  hi = byte_pair_minus(ob, 2, off);
}

// Store one chunk's codes (CH columns: words of 4 code bytes) of a row, as bytes or nibbles.
// to_stage: the destination is the ring slot (a multi-token call's tokens before the
// last), written with ordinary stores; otherwise global memory, streaming stores.
template <int DK, int BITS, bool to_stage>
__device__ __forceinline__ void mma_store(uint8_t *d, const uint32_t (&wq)[4], bool st) {
  using Gm = MmaGeom<DK>;
  if (!st) return;
  if (BITS == 8) {
    if (Gm::CH == 16) {
      const uint4 v = make_uint4(wq[0], wq[1], wq[2], wq[3]);
      if (to_stage) *reinterpret_cast<uint4 *>(d) = v; else __stcs(reinterpret_cast<uint4 *>(d), v);
    } else if (Gm::CH == 8) {
      const uint2 v = make_uint2(wq[0], wq[1]);
      if (to_stage) *reinterpret_cast<uint2 *>(d) = v; else __stcs(reinterpret_cast<uint2 *>(d), v);
    } else {
      if (to_stage) *reinterpret_cast<unsigned int *>(d) = wq[0];
      else __stcs(reinterpret_cast<unsigned int *>(d), wq[0]);
    }
  } else {
    const uint2 nb = compact_i4(make_uint4(wq[0], Gm::CH >= 8 ? wq[1] : 0u,
                                           Gm::CH == 16 ? wq[2] : 0u, Gm::CH == 16 ? wq[3] : 0u));
    if (Gm::CH == 16) {
      if (to_stage) *reinterpret_cast<uint2 *>(d) = nb; else __stcs(reinterpret_cast<uint2 *>(d), nb);
    } else if (Gm::CH == 8) {
      if (to_stage) *reinterpret_cast<unsigned int *>(d) = nb.x;
      else __stcs(reinterpret_cast<unsigned int *>(d), nb.x);
    } else {
      if (to_stage) *reinterpret_cast<unsigned short *>(d) = (unsigned short)nb.x;
      else __stcs(reinterpret_cast<unsigned short *>(d), (unsigned short)nb.x);
    }
  }
}

// Codes of 4 columns from t = fma(x, inv, 49152 + d/256): byte 1 of each.
__device__ __forceinline__ uint32_t pack4(const float2 &a, const float2 &b) {
  const uint32_t lo = __byte_perm(__float_as_uint(a.x), __float_as_uint(a.y), 0x0051u);
  const uint32_t hi = __byte_perm(__float_as_uint(b.x), __float_as_uint(b.y), 0x0051u);
  return __byte_perm(lo, hi, 0x5410u);
}

// The two rows of a strip (A = row g, B = row g + 8), after the contractions: x = S' + w k^T
// for the lane's columns, each row's group maximum over its four lanes, scales (both rows
// in packed form), dither, codes.  The rows' work interleaves: their dependency chains
// (maximum shuffles, Newton steps) overlap.  s2, w2: the rows' old scales and w; snew:
// their new scales; bad: a row held a non-finite or overflowing entry.  dstA / dstB: the
// rows in global memory, stored if stA / stB.
template <int DK, int BITS, bool DIAG, bool SR, bool TO_STAGE>
__device__ __forceinline__ void mma_rows2(const uint32_t (&cA)[DK / 16], const uint32_t (&cB)[DK / 16],
                                          float2 s2, const float *sa, float alpha_s, float2 w2,
                                          const float *sk, float r, float inv_r,
                                          uint32_t cbA, uint32_t cbB, uint8_t *dstA, uint8_t *dstB,
                                          bool stA, bool stB, float2 &snew, bool &badA,
                                          bool &badB) {
  using Gm = MmaGeom<DK>;
  constexpr int NP = DK / 8;                        // column pairs per lane-row
  const int tq = threadIdx.x & 3;
  float2 xa[NP], xb[NP];
#pragma unroll
  for (int m = 0; m < Gm::NW; ++m) {
    s8_floats(cA[m], xa[2 * m], xa[2 * m + 1]);
    s8_floats(cB[m], xb[2 * m], xb[2 * m + 1]);
  }
  const float2 wA = dup2(w2.x), wB = dup2(w2.y);
  const float2 sA = dup2(s2.x), sB = dup2(s2.y);
  const float2 a2 = __fmul2_rn(s2, dup2(alpha_s));
  const float2 aA = dup2(a2.x), aB = dup2(a2.y);
#pragma unroll
  for (int c = 0; c < Gm::NCH; ++c)
#pragma unroll
    for (int m = 0; m < Gm::CH / 4; ++m) {
      const int e = (Gm::CH / 2) * c + 2 * m;
      const float4 k4 = *reinterpret_cast<const float4 *>(sk + Gm::col(tq, c) + 4 * m);
      const float2 kl = make_float2(k4.x, k4.y), kh = make_float2(k4.z, k4.w);
      if (DIAG) {
        const float4 a4 = *reinterpret_cast<const float4 *>(sa + Gm::col(tq, c) + 4 * m);
        const float2 al = make_float2(a4.x, a4.y), ah = make_float2(a4.z, a4.w);
        xa[e] = __ffma2_rn(wA, kl, __fmul2_rn(xa[e], __fmul2_rn(sA, al)));
        xa[e + 1] = __ffma2_rn(wA, kh, __fmul2_rn(xa[e + 1], __fmul2_rn(sA, ah)));
        xb[e] = __ffma2_rn(wB, kl, __fmul2_rn(xb[e], __fmul2_rn(sB, al)));
        xb[e + 1] = __ffma2_rn(wB, kh, __fmul2_rn(xb[e + 1], __fmul2_rn(sB, ah)));
      } else {
        xa[e] = __ffma2_rn(wA, kl, __fmul2_rn(xa[e], aA));
        xa[e + 1] = __ffma2_rn(wA, kh, __fmul2_rn(xa[e + 1], aA));
        xb[e] = __ffma2_rn(wB, kl, __fmul2_rn(xb[e], aB));
        xb[e + 1] = __ffma2_rn(wB, kh, __fmul2_rn(xb[e + 1], aB));
      }
    }
  // largest |x| of each row's lane columns: trees (the max instructions are opaque to the
  // compiler, so the association is written out), then the row's four lanes
  float ma[NP / 2 > 0 ? NP / 2 : 1], mb[NP / 2 > 0 ? NP / 2 : 1];
#pragma unroll
  for (int e = 0; e < NP / 2; ++e) {
    ma[e] = max_abs_nan(max_abs_nan(max_abs_nan(fabsf(xa[2 * e].x), xa[2 * e].y), xa[2 * e + 1].x),
                        xa[2 * e + 1].y);
    mb[e] = max_abs_nan(max_abs_nan(max_abs_nan(fabsf(xb[2 * e].x), xb[2 * e].y), xb[2 * e + 1].x),
                        xb[2 * e + 1].y);
  }
#pragma unroll
  for (int w = NP / 4; w >= 1; w >>= 1)
#pragma unroll
    for (int e = 0; e < w; ++e) {
      ma[e] = max_nan(ma[e], ma[e + w]);
      mb[e] = max_nan(mb[e], mb[e + w]);
    }
  float2 m2 = make_float2(ma[0], mb[0]);
#pragma unroll
  for (int st = 1; st < 4; st <<= 1) {
    m2.x = max_nan(m2.x, __shfl_xor_sync(kFull, m2.x, st));
    m2.y = max_nan(m2.y, __shfl_xor_sync(kFull, m2.y, st));
  }
  float2 inv2;
  pair_scale(m2, dup2(r), dup2(inv_r), inv2, snew, badA, badB);
  const float2 invA = dup2(inv2.x), invB = dup2(inv2.y);
#pragma unroll
  for (int c = 0; c < Gm::NCH; ++c) {
    // dither words of the chunk's quads of both rows: a chunk of 16 columns is a whole
    // block; chunks of 8 or 4 columns (d_k = 32, 16) take words q0.. of their block
    uint32_t ha[4] = {0u, 0u, 0u, 0u}, hb[4] = {0u, 0u, 0u, 0u};
    if (SR) {
      const int col = Gm::col(tq, c);
      const uint32_t off = 0x9E3779B9u * (uint32_t)(4 * (col / 16));   // block's first quad
      const uint32_t bka = dither_block_key(cbA + off), bkb = dither_block_key(cbB + off);
      const int q0 = (col % 16) / 4;
#pragma unroll
      for (int qd = 0; qd < Gm::CH / 4; ++qd) {
        ha[qd] = dither_word(bka, Gm::CH == 16 ? qd : q0 + qd);
        hb[qd] = dither_word(bkb, Gm::CH == 16 ? qd : q0 + qd);
      }
    }
    uint32_t wa[4], wb[4];
#pragma unroll
    for (int qd = 0; qd < Gm::CH / 4; ++qd) {
      const int e = (Gm::CH / 2) * c + 2 * qd;
      float2 ta0, ta1, tb0, tb1;
      if (SR) {
        ta0 = __ffma2_rn(xa[e], invA, make_float2(__uint_as_float(__byte_perm(ha[qd], 0x47400000u, 0x7650u)),
                                                  __uint_as_float(__byte_perm(ha[qd], 0x47400000u, 0x7651u))));
        ta1 = __ffma2_rn(xa[e + 1], invA, make_float2(__uint_as_float(__byte_perm(ha[qd], 0x47400000u, 0x7652u)),
                                                      __uint_as_float(__byte_perm(ha[qd], 0x47400000u, 0x7653u))));
        tb0 = __ffma2_rn(xb[e], invB, make_float2(__uint_as_float(__byte_perm(hb[qd], 0x47400000u, 0x7650u)),
                                                  __uint_as_float(__byte_perm(hb[qd], 0x47400000u, 0x7651u))));
        tb1 = __ffma2_rn(xb[e + 1], invB, make_float2(__uint_as_float(__byte_perm(hb[qd], 0x47400000u, 0x7652u)),
                                                      __uint_as_float(__byte_perm(hb[qd], 0x47400000u, 0x7653u))));
      } else {
        ta0 = __ffma2_rn(xa[e], invA, dup2(49152.5f));
        ta1 = __ffma2_rn(xa[e + 1], invA, dup2(49152.5f));
        tb0 = __ffma2_rn(xb[e], invB, dup2(49152.5f));
        tb1 = __ffma2_rn(xb[e + 1], invB, dup2(49152.5f));
      }
      wa[qd] = pack4(ta0, ta1);
      wb[qd] = pack4(tb0, tb1);
    }
    const int boff = BITS == 8 ? Gm::col(tq, c) : Gm::col(tq, c) / 2;
    mma_store<DK, BITS, TO_STAGE>(dstA + boff, wa, stA);
    mma_store<DK, BITS, TO_STAGE>(dstB + boff, wb, stB);
  }
}

// One unit (rows [row0, row0 + nrows) of one tile) from a ring slot, strip by strip.
// FULL: the unit is a full row block (full_rows(d_k, BITS) rows, a whole number of
// strips): the strip count and every row's validity are compile-time facts.
// sv: the unit's v rows; go: where its readout rows go; to_stage: write the requantized
// rows and scales back into the slot (a multi-token call's tokens before the last; every
// lane rewrites the bytes it read, and a row's scale is rewritten by the row's lane 0 after
// the row's shuffles, so after all its lanes read it) instead of global memory.
template <int DK, int BITS, bool DIAG, bool DELTA, bool SR, bool FULL, bool TO_STAGE>
__device__ __forceinline__ void mma_unit(const StepParams &p, uint8_t *stage, int b,
                                         const UnitDesc &d, const MmaTile<DK, DIAG> &t,
                                         const float *sk, const float *sa, const float *sv,
                                         float *go) {
  constexpr bool to_stage = TO_STAGE;
  constexpr int RB = DK * BITS / 8;                 // bytes of one row
  const int lane = threadIdx.x & 31, g = lane >> 2, tq = lane & 3;
  const long long tile = (long long)b * p.H + d.head;
  float *ss = reinterpret_cast<float *>(stage + p.st_scales);
  uint8_t *gcodes = to_stage ? stage : p.codes + (long long)b * p.seq_bytes + d.code_off;
  float *gs = to_stage ? ss : p.scales + tile * p.d_v + d.row0;
  constexpr int kFull = full_rows(DK, BITS);
  static_assert(kFull % 16 == 0, "a full row block is a whole number of strips");
  const int nrows = FULL ? kFull : d.nrows;
  uint32_t badmask = 0;                             // bit 2s (+1): row g (g + 8) of strip s
  const int nstrip = FULL ? kFull / 16 : (nrows + 15) >> 4;
#pragma unroll 1
  for (int sp = 0; sp < nstrip; ++sp) {
    const int r0 = 16 * sp + g, r1 = r0 + 8;
    const bool v0 = FULL || r0 < nrows, v1 = FULL || r1 < nrows;
    // rows past the unit read its last row (in bounds; their results are not stored)
    uint32_t c0[DK / 16], c1[DK / 16];
    mma_load_row<DK, BITS>(stage + (v0 ? r0 : nrows - 1) * RB, tq, c0);
    mma_load_row<DK, BITS>(stage + (v1 ? r1 : nrows - 1) * RB, tq, c1);
    int acc[4] = {0, 0, 0, 0};
    __syncwarp();                                   // the MMAs need the whole warp converged
    if (DK == 16) {
      mma_k16(acc, c0[0], c1[0], t.bf[0]);
    } else {
#pragma unroll
      for (int kb = 0; kb < DK / 32; ++kb)
        mma_k32(acc, c0[2 * kb], c1[2 * kb], c0[2 * kb + 1], c1[2 * kb + 1], t.bf[2 * kb],
                t.bf[2 * kb + 1]);
    }
    // lane t holds digit columns 2t, 2t + 1 (t < 2: k, else q); the sums of the two
    // lanes of a vector join into U = lo + 2^16 hi, exact in double
    const int pa = acc[0] + acc[1] * 256, pb = acc[2] + acc[3] * 256;
    const int oa = __shfl_xor_sync(kFull, pa, 1), ob = __shfl_xor_sync(kFull, pb, 1);
    const bool hi = tq & 1;
    const double Ua = fma((double)(hi ? pa : oa), 65536.0, (double)(hi ? oa : pa));
    const double Ub = fma((double)(hi ? pb : ob), 65536.0, (double)(hi ? ob : pb));
    const float sA = ss[v0 ? r0 : 0], sB = ss[v1 ? r1 : 0];
    const float xa = (float)(((double)sA * Ua) * t.sx);
    const float xb = (float)(((double)sB * Ub) * t.sx);
    const float ya = __shfl_xor_sync(kFull, xa, 2), yb = __shfl_xor_sync(kFull, xb, 2);
    // u (the projection S'k) and S'q of both rows
    const float uA = tq < 2 ? xa : ya, uB = tq < 2 ? xb : yb;
    const float qA = tq < 2 ? ya : xa, qB = tq < 2 ? yb : xb;
    const float vA = sv[v0 ? r0 : 0], vB = sv[v1 ? r1 : 0];
    const float wA = DELTA ? __fmul_rn(t.beta, __fsub_rn(vA, uA)) : __fmul_rn(t.beta, vA);
    const float wB = DELTA ? __fmul_rn(t.beta, __fsub_rn(vB, uB)) : __fmul_rn(t.beta, vB);
    if (tq == 0) {
      if (v0 && LORES_IN(p, kRgO, go + r0, 4)) go[r0] = __fmaf_rn(wA, t.kq, qA);
      if (v1 && LORES_IN(p, kRgO, go + r1, 4)) go[r1] = __fmaf_rn(wB, t.kq, qB);
    }
    // dither counter of the row's quad 0: tile key + golden (row d_k/4 + 1)
    const uint32_t cb0 = t.tkey + 0x9E3779B9u * ((uint32_t)(d.row0 + r0) * (uint32_t)(DK / 4) + 1u);
    const uint32_t cb1 = cb0 + 0x9E3779B9u * (uint32_t)(8 * DK / 4);
    float2 sn;
    bool badA, badB;
    // (index-checked build: a row outside the code pool is not stored)
    const bool s0 = v0 && (to_stage || LORES_IN(p, kRgCodes, gcodes + r0 * RB, RB));
    const bool s1 = v1 && (to_stage || LORES_IN(p, kRgCodes, gcodes + r1 * RB, RB));
    mma_rows2<DK, BITS, DIAG, SR, TO_STAGE>(c0, c1, make_float2(sA, sB), sa, t.alpha, make_float2(wA, wB),
                                            sk, d.r, d.inv_r, cb0, cb1, gcodes + r0 * RB,
                                            gcodes + r1 * RB, s0, s1, sn, badA, badB);
    if (tq == 0) {
      if (v0 && (to_stage || LORES_IN(p, kRgScales, gs + r0, 4))) gs[r0] = sn.x;
      if (v1 && (to_stage || LORES_IN(p, kRgScales, gs + r1, 4))) gs[r1] = sn.y;
    }
    badmask |= (badA && v0 ? 1u : 0u) << (2 * sp);
    badmask |= (badB && v1 ? 1u : 0u) << (2 * sp + 1);
  }
  // rare: rows with a non-finite (or overflowing) entry are stored as zero; every lane of
  // the row rewrites its own columns
  if (__any_sync(kFull, badmask != 0u)) {
    using Gm = MmaGeom<DK>;
    for (int sp = 0; sp < nstrip; ++sp)
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        if (!((badmask >> (2 * sp + h)) & 1u)) continue;
        const int r = 16 * sp + g + 8 * h;
        uint8_t *row = gcodes + r * RB;
        if (to_stage || LORES_IN(p, kRgCodes, row, RB))
          for (int c = 0; c < Gm::NCH; ++c)
            for (int by = 0; by < Gm::CH * BITS / 8; ++by) row[(BITS == 8 ? Gm::col(tq, c) : Gm::col(tq, c) / 2) + by] = 0;
        if (tq == 0) {
          if (to_stage || LORES_IN(p, kRgScales, gs + r, 4)) gs[r] = 0.0f;
          atomicOr(p.flag, kFlagNonFinite);
        }
      }
  }
}

// The persistent loop of one warp over the units of one storage class (BITS), as in
// pair_run: warp gw of W takes units [U gw / W, U (gw + 1) / W) of the class's U units in
// (sequence, unit) order through a 2-slot ring of bulk copies; bar0: the first of the
// warp's barrier slots the ring uses.
template <int DK, int BITS, bool DIAG, bool DELTA, bool SR, bool MT>
__device__ __forceinline__ void mma_run(const StepParams &p, const UnitDesc *tbl, uint8_t *wa,
                                        int cta, int nctas, int lo, int hi, int bar0 = 0) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint64_t *bars = reinterpret_cast<uint64_t *>(wa) + bar0;
  float *ow = reinterpret_cast<float *>(wa + 64) + p.opart_floats;
  uint8_t *planes = reinterpret_cast<uint8_t *>(ow + p.ow_floats);
  uint8_t *stages = planes + p.plane_bytes;
  const int per_seq = hi - lo;
  if (per_seq <= 0 || nctas <= 0) return;
  const long long U = (long long)p.B * per_seq;
  const long long W = (long long)nctas * kWarps;
  const long long gw = (long long)cta * kWarps + warp;
  const long long u0 = U * gw / W, u1 = U * (gw + 1) / W;
  if (u0 >= u1) return;
  const int count = (int)(u1 - u0);
  const int H = p.H;
  if (lane == 0) {
    for (int s = 0; s < kStages; ++s) mbar_init(&bars[s], 1);
    fence_mbar_init();
  }
  __syncwarp();
  const PairPos start{(int)(u0 / per_seq), lo + (int)(u0 % per_seq)};
  PairPos fill = start;
  int ftile = -1;
  for (int s = 0; s < kStages && s < count; ++s) {
    const UnitDesc d = tbl[fill.ub];
    const int tl = fill.b * H + d.head;
    pair_issue<DK, DIAG, MT>(p, d, fill.b, fill.ub, tl != ftile, stages + s * p.stage_bytes, &bars[s]);
    ftile = tl;
    fill.next(lo, hi);
  }
  const uint32_t skey = p.step_dev ? step_key_dev(p.seed, *p.step_dev) : p.step_key;
  PairPos cur = start;
  int ctile = -1;
  const float *kkeep = reinterpret_cast<const float *>(planes + 8 * DK);   // the tile's k
  const float *akeep = kkeep + DK;                  // and per-column alpha (DIAG)
  MmaTile<DK, DIAG> t;
  float beta_c = 0.0f, alpha_c = 0.0f;
  if (!MT) {
    const int t0 = cur.b * H + tbl[cur.ub].head;
    beta_c = LORES_LDG(p, kRgBeta, p.beta + t0);
    if (!DIAG) alpha_c = LORES_LDG(p, kRgAlpha, p.alpha + t0);
  }
#pragma unroll 1
  for (int n = 0; n < count; ++n) {
    const int s = n % kStages;
    uint8_t *stage = stages + s * p.stage_bytes;
    PairPos nx = cur;
    nx.next(lo, hi);
    float beta_n = 0.0f, alpha_n = 0.0f;
    if (!MT && n + 1 < count) {
      const int tn = nx.b * H + tbl[nx.ub].head;
      beta_n = LORES_LDG(p, kRgBeta, p.beta + tn);
      if (!DIAG) alpha_n = LORES_LDG(p, kRgAlpha, p.alpha + tn);
    }
    const bool ok = mbar_wait_bounded(&bars[s], (unsigned)((n / kStages) & 1), p.wait_ns);
    if (!__all_sync(kFull, ok)) {
      // give up: record it, let the other slot's copy (if any) land, and leave
      if (lane == 0) {
        atomicOr(p.flag, kFlagTimeout);
        if (n + 1 < count)
          (void)mbar_wait_bounded(&bars[(n + 1) % kStages], (unsigned)(((n + 1) / kStages) & 1),
                                  p.wait_ns);
      }
      __syncwarp();
      return;
    }
    const UnitDesc d = tbl[cur.ub];
    const int tl = cur.b * H + d.head;
    if (MT) {
      // every token of the unit in turn; the unit's codes and scales stay in the slot
      for (int tok = 0; tok < p.T; ++tok) {
        const float *k = p.k + tok * p.tok_qk + (long long)tl * DK;
        const float *q = p.q + tok * p.tok_qk + (long long)tl * DK;
        const float *al = p.alpha + tok * p.tok_a + (long long)tl * DK;
        if (!(LORES_IN(p, kRgK, k, DK * 4) && LORES_IN(p, kRgQ, q, DK * 4) &&
              LORES_IN(p, kRgV, p.v + tok * p.tok_v + (long long)tl * p.d_v + d.row0, d.nrows * 4) &&
              (!DIAG || LORES_IN(p, kRgAlpha, al, DK * 4))))
          continue;                            // index-checked build: vectors out of range
        const float a_s = DIAG ? 0.0f : LORES_LDG(p, kRgAlpha, p.alpha + tok * p.tok_a + tl);
        mma_tile<DK, DIAG>(k, q, al, a_s, planes, t);
        double kqd = 0.0;
#pragma unroll
        for (int j = lane; j < DK; j += 32) kqd = fma((double)__ldg(k + j), (double)__ldg(q + j), kqd);
#pragma unroll
        for (int st = 16; st >= 1; st >>= 1) kqd += __shfl_xor_sync(kFull, kqd, st);
        t.kq = (float)kqd;
        t.tkey = tile_key(step_key_dev(p.seed, p.step0 + (uint64_t)tok), (uint32_t)tl);
        t.beta = LORES_LDG(p, kRgBeta, p.beta + tok * p.tok_b + tl);
        t.alpha = a_s;
        const float *sv = p.v + tok * p.tok_v + (long long)tl * p.d_v + d.row0;
        float *go = p.o + tok * p.tok_o + (long long)tl * p.d_v + d.row0;
        const bool full = d.nrows == full_rows(DK, BITS);
        if (tok + 1 < p.T) {                         // not the last token: back to the slot
          if (full)
            mma_unit<DK, BITS, DIAG, DELTA, SR, true, true>(p, stage, cur.b, d, t, kkeep, akeep, sv, go);
          else
            mma_unit<DK, BITS, DIAG, DELTA, SR, false, true>(p, stage, cur.b, d, t, kkeep, akeep, sv, go);
        } else {
          if (full)
            mma_unit<DK, BITS, DIAG, DELTA, SR, true, false>(p, stage, cur.b, d, t, kkeep, akeep, sv, go);
          else
            mma_unit<DK, BITS, DIAG, DELTA, SR, false, false>(p, stage, cur.b, d, t, kkeep, akeep, sv, go);
        }
        __syncwarp();
      }
    } else if (tl != ctile) {
      // a new tile: its vectors are in this slot (copied out by mma_tile: a later unit of
      // the tile reuses the slot)
      const float *sk = reinterpret_cast<const float *>(stage + p.st_k);
      const float *sq = reinterpret_cast<const float *>(stage + p.st_q);
      const float *sal = reinterpret_cast<const float *>(stage + p.st_a);
      mma_tile<DK, DIAG>(sk, sq, sal, alpha_c, planes, t);
      double kqd = 0.0;
#pragma unroll
      for (int j = lane; j < DK; j += 32) kqd = fma((double)sk[j], (double)sq[j], kqd);
#pragma unroll
      for (int st = 16; st >= 1; st >>= 1) kqd += __shfl_xor_sync(kFull, kqd, st);
      t.kq = (float)kqd;
      t.tkey = tile_key(skey, (uint32_t)tl);
      ctile = tl;
    }
    if (!MT) {
      t.beta = beta_c;
      t.alpha = alpha_c;
      const float *sv = reinterpret_cast<const float *>(stage + p.st_v);
      float *go = p.o + ((long long)tl * p.d_v + d.row0);
      if (d.nrows == full_rows(DK, BITS))
        mma_unit<DK, BITS, DIAG, DELTA, SR, true, false>(p, stage, cur.b, d, t, kkeep, akeep, sv, go);
      else
        mma_unit<DK, BITS, DIAG, DELTA, SR, false, false>(p, stage, cur.b, d, t, kkeep, akeep, sv, go);
    }
    __syncwarp();                                   // every lane is done with this slot
    if (n + kStages < count) {
      fence_proxy_async();
      const UnitDesc dn = tbl[fill.ub];
      const int tf = fill.b * H + dn.head;
      pair_issue<DK, DIAG, MT>(p, dn, fill.b, fill.ub, tf != ftile, stage, &bars[s]);
      ftile = tf;
      fill.next(lo, hi);
    }
    cur = nx;
    beta_c = beta_n;
    alpha_c = alpha_n;
  }
}

// Persistent kernel over the units of heads stored one byte per code (table entries
// [pair_lo[0], pair_hi[0]) of every sequence) and one nibble per code ([pair_lo[1],
// pair_hi[1])), all with one scale per value row.  pair_ctas < 0: every CTA takes both
// classes in turn; else CTAs [0, pair_ctas) take the first class, the others the second.
template <int DK, bool DIAG, bool DELTA, bool SR, bool MT>
__global__ void __launch_bounds__(kThreads, LORES_MMA_MIN_CTAS) decode_mma_kernel(const StepParams p) {
  extern __shared__ __align__(128) uint8_t smem[];
  const int warp = threadIdx.x >> 5;
  UnitDesc *stbl = reinterpret_cast<UnitDesc *>(smem);
  uint8_t *wa = smem + p.table_bytes + warp * p.warp_bytes;
  const UnitDesc *tbl = p.units;
  if (p.table_bytes) {
    for (int i = threadIdx.x; i < p.units_per_seq; i += kThreads) stbl[i] = p.units[i];
    tbl = stbl;
  }
  __syncthreads();                                  // the only CTA-wide barrier
  // pair_ctas < 0: every CTA takes its share of the byte class, then its share of the
  // nibble class, so that an SM runs one class's body at a time (CTAs of both classes side
  // by side on one SM thrash its instruction cache).  Else CTAs [0, pair_ctas) take the
  // byte class and the others the nibble class (about one unit per warp: in turn, the
  // classes would add a unit's latency to a warp's).  The nibble ring takes fresh barriers.
  const int cta = (int)blockIdx.x, grid = (int)gridDim.x;
  const bool both = p.pair_ctas < 0;
  const int c8 = both || cta < p.pair_ctas ? cta : 0;
  const int n8 = both ? grid : (cta < p.pair_ctas ? p.pair_ctas : 0);
  const int c4 = both ? cta : cta - p.pair_ctas;
  const int n4 = both ? grid : (cta < p.pair_ctas ? 0 : grid - p.pair_ctas);
  mma_run<DK, 8, DIAG, DELTA, SR, MT>(p, tbl, wa, c8, n8, p.pair_lo[0], p.pair_hi[0]);
  mma_run<DK, 4, DIAG, DELTA, SR, MT>(p, tbl, wa, c4, n4, p.pair_lo[1], p.pair_hi[1], kStages);
}

template <int DK, bool SR, bool MT>
StepFn pick_mma(bool diag, bool delta) {
  if (diag)
    return delta ? decode_mma_kernel<DK, true, true, SR, MT> : decode_mma_kernel<DK, true, false, SR, MT>;
  return delta ? decode_mma_kernel<DK, false, true, SR, MT> : decode_mma_kernel<DK, false, false, SR, MT>;
}

// One function per key width, each defined in its own compilation of lores_inst.cu.
#define LORES_DECLARE_MMA(dk) StepFn mma_kernels_##dk(bool diag, bool delta, bool sr, bool mt);
LORES_DECLARE_MMA(16)
LORES_DECLARE_MMA(32)
LORES_DECLARE_MMA(64)
LORES_DECLARE_MMA(128)
#undef LORES_DECLARE_MMA

}  // namespace lores
