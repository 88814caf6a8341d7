// lores_pair.cuh -- decode-step kernel for heads stored one byte or one nibble per code
// (value-axis scale groups, one token per call), sm_100a.
//
// The same step as decode_step_kernel in lores_step.cuh ("Quantizing Recurrent Language
// Models Is Easier Than You Think", summary page: General recurrence form; Key properties
// item 3; Proposition 1; Proposition 3 / Table 6), with the same fp32 operations in the
// same order, so the state, scales and readout it writes are bit for bit the ones that
// kernel writes.  What differs is the layout of the work:
//  * a warp takes one contiguous run of work units in (sequence, head, row block) order,
//    so consecutive units mostly share their tile: the tile's k, q and per-column alpha
//    are copied into shared memory (into the ring slot of the tile's first unit) and
//    loaded into registers once per tile, and k.q, the dither key, alpha and beta are
//    formed once per tile, not once per unit;
//  * every lane carries two neighbouring value rows through each pass, so the per-row
//    scalars (scale times decay, u and its shuffle sums, w, the reciprocal of the group
//    maximum, the new scale) run as packed fp32x2 operations on the pair, and the two
//    rows' dependency chains interleave.
// Multi-token calls (MT) keep each unit's codes and scales in its ring slot across the
// tokens.  Heads with fp32 state, dense bit planes or per-channel widths and key-axis scales
// stay on the kernels of lores_step.cuh and lores_key.cuh.
#pragma once
#include <cstdint>

#include "lores_device.cuh"
#include "lores_step.cuh"

// CTAs per SM the register allocation is sized for (128 threads each): 3 leaves the
// compiler 168 registers, enough to interleave two passes of a unit without spills (4
// CTAs at 128 registers measured slower: the pass loop then re-derives its addresses).
#ifndef LORES_PAIR_MIN_CTAS
#define LORES_PAIR_MIN_CTAS 3
#endif

namespace lores {

// Registers of the tile a warp is working on (element pair e holds columns 2e, 2e + 1 of
// the lane's 16), loaded from the ring slot of the tile's first unit.
template <bool DIAG>
struct PairTile {
  float2 kk[8], qq[8], aa[DIAG ? 8 : 1];
  float kq;              // k.q, from a double-precision sum
  float alpha, beta;     // scalar decay (DIAG = false) and beta of the tile
  uint32_t tkey;         // dither key of the tile
};

// Bulk copies of one unit into a ring slot: codes, scales and the v slice, and, for a
// unit that starts a new tile (vec), the tile's k, q and per-column alpha.  Lane 0
// announces the byte count; lanes 0-5 issue one copy each.
template <int DK, bool DIAG, bool MT>
__device__ __forceinline__ void pair_issue(const StepParams &p, const UnitDesc &d, int b, int ub,
                                           bool vec, uint8_t *stage, uint64_t *bar) {
  // multi-token calls stage codes and scales only; every token's vectors come from memory
  vec = vec && !MT;
  const int lane = threadIdx.x & 31;
  const long long tile = (long long)b * p.H + d.head;
  const bool withhold = b == p.fault_b && ub == p.fault_ub;   // failure-path test only
  const unsigned cbytes = (unsigned)(d.nrows * d.rowb);
  const unsigned sbytes = (unsigned)(d.nrows * p.ng * 4);
  const unsigned vbytes = MT ? 0u : (unsigned)(d.nrows * 4);
  constexpr unsigned kVec = DK * 4;
  if (lane == 0)
    mbar_expect_tx(bar, cbytes + sbytes + vbytes + (vec ? (DIAG ? 3u : 2u) * kVec : 0u));
  __syncwarp();
  const void *src = nullptr;
  int dst = 0, rid = kRgCodes;
  unsigned bytes = 0;
  if (lane == 0) { src = p.codes + (long long)b * p.seq_bytes + d.code_off; dst = 0; bytes = cbytes; }
  if (lane == 1) { src = p.scales + (tile * p.d_v + d.row0) * p.ng; dst = p.st_scales; bytes = sbytes; rid = kRgScales; }
  if (!MT && lane == 2) { src = p.v + tile * p.d_v + d.row0; dst = p.st_v; bytes = vbytes; rid = kRgV; }
  if (vec && lane == 3) { src = p.k + tile * DK; dst = p.st_k; bytes = kVec; rid = kRgK; }
  if (vec && lane == 4) { src = p.q + tile * DK; dst = p.st_q; bytes = kVec; rid = kRgQ; }
  if (vec && DIAG && lane == 5) { src = p.alpha + tile * DK; dst = p.st_a; bytes = kVec; rid = kRgAlpha; }
  (void)rid;
  if (bytes && !withhold && LORES_IN(p, rid, src, bytes) && LORES_IN_SMEM(p, stage + dst, bytes))
    bulk_g2s(stage + dst, src, bytes, bar);
}

// 16 codes of one lane's row -> exact floats in column pairs.
template <int BITS>
__device__ __forceinline__ void pair_unpack(const uint8_t *src, float2 (&c)[8]) {
  if (BITS == 8)
    unpack_i8_2(*reinterpret_cast<const uint4 *>(src), c);
  else
    unpack_i4_2(*reinterpret_cast<const uint2 *>(src), c);
}
template <int BITS>
__device__ __forceinline__ void pair_store(uint8_t *dst, const uint32_t (&w)[4], bool to_stage = false) {
  if (to_stage) {                                 // shared memory: an ordinary store
    if (BITS == 8)
      *reinterpret_cast<uint4 *>(dst) = make_uint4(w[0], w[1], w[2], w[3]);
    else
      *reinterpret_cast<uint2 *>(dst) = make_uint2(w[0], w[1]);
  } else if (BITS == 8) {
    __stcs(reinterpret_cast<uint4 *>(dst), make_uint4(w[0], w[1], w[2], w[3]));
  } else {
    __stcs(reinterpret_cast<uint2 *>(dst), make_uint2(w[0], w[1]));
  }
}

// Scale and inverse of two groups at once (the rows' own groups) with largest |x| = m:
// the operations of group_scale, packed.  bad: an entry is inf, NaN or above 2^100.
__device__ __forceinline__ void pair_scale(float2 m, float2 r, float2 inv_r, float2 &inv,
                                           float2 &s, bool &badA, bool &badB) {
  badA = !(m.x <= 0x1p100f);
  badB = !(m.y <= 0x1p100f);
  const bool scA = m.x >= 0x1p-100f && !badA, scB = m.y >= 0x1p-100f && !badB;
  const float2 mm = make_float2(scA ? m.x : 1.0f, scB ? m.y : 1.0f);
  // Newton-Raphson reciprocal from the exponent-reflected seed, three steps (recip_nr)
  float2 y = make_float2(__uint_as_float(0x7F000000u - __float_as_uint(mm.x)),
                         __uint_as_float(0x7F000000u - __float_as_uint(mm.y)));
  const float2 nm = make_float2(-mm.x, -mm.y);
  const float2 one = make_float2(1.0f, 1.0f);
#pragma unroll
  for (int it = 0; it < 3; ++it) {
    const float2 e = __ffma2_rn(nm, y, one);
    y = __ffma2_rn(y, e, y);
  }
  const float2 iv = __fmul2_rn(r, y);
  const float2 sc = __fmul2_rn(m, inv_r);
  inv = make_float2(scA ? iv.x : 0.0f, scB ? iv.y : 0.0f);
  s = make_float2(scA ? sc.x : 0.0f, scB ? sc.y : 0.0f);
}

// One full unit (full_rows(d_k, BITS) rows of one tile) from a ring slot.  Lane layout:
// LPR = d_k/16 lanes own a row, 16 consecutive columns each; a pass covers 2 RPW rows,
// lane (riw, lir) taking rows 2 riw and 2 riw + 1 of the pass.  The pass count and every
// shared- and global-memory offset inside the unit are compile-time constants from the
// lane's base addresses.  GROW: one scale per value row (G = d_k).  Multi-token calls (MT):
// token tok reads its v from memory and writes o at tok * tok_o; tokens before the last
// (to_stage) write the requantized rows and scales back into the slot, each lane the bytes
// it read, a group's scale after the group's shuffles (so after its lanes have read it).
template <int DK, bool DIAG, bool DELTA, bool SR, int BITS, bool GROW, bool MT>
__device__ __forceinline__ void pair_unit(const StepParams &p, uint8_t *stage, int b,
                                          const UnitDesc &d, const PairTile<DIAG> &t,
                                          float *opart, float *ow, int tok, bool to_stage) {
  constexpr int LPR = DK / 16, RPW = 32 / LPR;
  constexpr int RB = DK * BITS / 8;                 // bytes of one row
  constexpr int LB = 2 * BITS;                      // bytes of one lane's 16 codes
  constexpr int kPass = full_rows(DK, BITS) / (2 * RPW);
  static_assert(full_rows(DK, BITS) % (2 * RPW) == 0, "a full unit is a whole number of passes");
  const int lane = threadIdx.x & 31, lir = lane % LPR, riw = lane / LPR;
  const int ng = GROW ? 1 : p.ng;
  const int lpg = GROW ? LPR : p.G / 16;            // lanes per scale group
  const int g = GROW ? 0 : lir / lpg;
  const bool scale_writer = (lir & (lpg - 1)) == 0;
  const int gd[4] = {1 < lpg ? 1 : 0, 2 < lpg ? 2 : 0, 4 < lpg ? 4 : 0, 8 < lpg ? 8 : 0};
  const int r0 = 2 * riw;                           // the lane's first row in pass 0
  const uint8_t *sc = stage + r0 * RB + lir * LB;
  const float *ssr = reinterpret_cast<const float *>(stage + p.st_scales) + r0 * ng + g;
  float *opr = opart + r0 * LPR + lir;
  float *owr = ow + r0;
  const long long tile = (long long)b * p.H + d.head;
  const float *svr = MT ? p.v + tok * p.tok_v + tile * p.d_v + d.row0 + r0
                        : reinterpret_cast<const float *>(stage + p.st_v) + r0;
  // where the requantized rows and scales go: the slot (a multi-token call's tokens before
  // the last) or global memory
  uint8_t *gc = to_stage ? stage + r0 * RB + lir * LB
                         : p.codes + (long long)b * p.seq_bytes + d.code_off + r0 * RB + lir * LB;
  float *gs = to_stage ? reinterpret_cast<float *>(stage + p.st_scales) + r0 * ng + g
                       : p.scales + (tile * p.d_v + d.row0 + r0) * ng + g;
  const float2 r2 = dup2(d.r), inv_r2 = dup2(d.inv_r);
  // dither counter of the lane's first quad in its first row of pass 0; the second row
  // is d_k/4 quads further, the next pass 2 RPW rows further
  const uint32_t cbase0 =
      t.tkey + 0x9E3779B9u * ((uint32_t)(d.row0 + r0) * (uint32_t)(DK / 4) + 4u * lir + 1u);
  constexpr uint32_t kRowCtr = 0x9E3779B9u * (uint32_t)(DK / 4);
  constexpr uint32_t kPassCtr = 0x9E3779B9u * (uint32_t)(2 * RPW * DK / 4);
  uint32_t badmask = 0;                             // bit 2n (+1): row A (B) of pass n bad

#pragma unroll 2
  for (int n = 0; n < kPass; ++n) {
    const int oc = n * 2 * RPW * RB;                // byte offset of the pass's rows
    const int orow = n * 2 * RPW;                   // row offset of the pass

    // ---- dequantize and decay: S'_ij = c_ij * (s_ig * alpha_j) ------------------------
    float2 spA[8], spB[8];
    pair_unpack<BITS>(sc + oc, spA);
    pair_unpack<BITS>(sc + oc + RB, spB);
    const float sA = ssr[orow * ng], sB = ssr[(orow + 1) * ng];
    if (DIAG) {
      const float2 sA2 = dup2(sA), sB2 = dup2(sB);
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        spA[e] = __fmul2_rn(spA[e], __fmul2_rn(sA2, t.aa[e]));
        spB[e] = __fmul2_rn(spB[e], __fmul2_rn(sB2, t.aa[e]));
      }
    } else {
      const float2 a2 = __fmul2_rn(make_float2(sA, sB), dup2(t.alpha));
      const float2 aA = dup2(a2.x), aB = dup2(a2.y);
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        spA[e] = __fmul2_rn(spA[e], aA);
        spB[e] = __fmul2_rn(spB[e], aB);
      }
    }

    // ---- readout shares: this lane's part of S'q for both rows (before x replaces S') ---
    opr[orow * LPR] = dot16_p(spA, t.qq);
    opr[(orow + 1) * LPR] = dot16_p(spB, t.qq);

    // ---- write: w = beta (v - delta (S'k)), x = S' + w k^T ----------------------------
    const float2 v2 = *reinterpret_cast<const float2 *>(svr + orow);
    float2 w2;
    if (DELTA) {
      float2 u2 = make_float2(dot16_p(spA, t.kk), dot16_p(spB, t.kk));
#pragma unroll
      for (int st = 1; st < LPR; st <<= 1)
        u2 = __fadd2_rn(u2, make_float2(__shfl_xor_sync(kFull, u2.x, st),
                                        __shfl_xor_sync(kFull, u2.y, st)));
      w2 = __fmul2_rn(dup2(t.beta), __fadd2_rn(v2, make_float2(-u2.x, -u2.y)));
    } else {
      w2 = __fmul2_rn(dup2(t.beta), v2);
    }
    if (lir == 0) *reinterpret_cast<float2 *>(owr + orow) = w2;
    {
      const float2 wA = dup2(w2.x), wB = dup2(w2.y);
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        spA[e] = __ffma2_rn(wA, t.kk[e], spA[e]);  // now x
        spB[e] = __ffma2_rn(wB, t.kk[e], spB[e]);
      }
    }

    // ---- requantize: group maxima, scales, codes ----------------------------------------
    uint32_t hA[4] = {0u, 0u, 0u, 0u}, hB[4] = {0u, 0u, 0u, 0u};
    if (SR) {
      const uint32_t c = cbase0 + kPassCtr * (uint32_t)n;
      dither_words(c, hA);
      dither_words(c + kRowCtr, hB);
    }
    float2 m2 = make_float2(chunk_absmax(spA), chunk_absmax(spB));
#pragma unroll
    for (int l = 0; (1 << l) < LPR; ++l) {
      m2.x = max_nan(m2.x, __shfl_xor_sync(kFull, m2.x, gd[l]));
      m2.y = max_nan(m2.y, __shfl_xor_sync(kFull, m2.y, gd[l]));
    }
    float2 inv2, s2;
    bool badA, badB;
    pair_scale(m2, r2, inv_r2, inv2, s2, badA, badB);
    uint32_t wA[4], wB[4];
    quantize16<BITS, SR>(spA, dup2(inv2.x), hA, wA);
    quantize16<BITS, SR>(spB, dup2(inv2.y), hB, wB);
    const bool st = MT && to_stage;
    if (st || LORES_IN(p, kRgCodes, gc + oc, LB)) pair_store<BITS>(gc + oc, wA, st);
    if (st || LORES_IN(p, kRgCodes, gc + oc + RB, LB)) pair_store<BITS>(gc + oc + RB, wB, st);
    if (scale_writer) {
      if (GROW) {
        if (st || LORES_IN(p, kRgScales, gs + orow, 8)) *reinterpret_cast<float2 *>(gs + orow) = s2;
      } else {
        if (st || LORES_IN(p, kRgScales, gs + orow * ng, 4)) gs[orow * ng] = s2.x;
        if (st || LORES_IN(p, kRgScales, gs + (orow + 1) * ng, 4)) gs[(orow + 1) * ng] = s2.y;
      }
    }
    badmask |= (badA ? 1u : 0u) << (2 * n);
    badmask |= (badB ? 1u : 0u) << (2 * n + 1);
  }

  // ---- rare: rows with a non-finite (or overflowing) entry are stored as zero -----------
  // A row is bad if any of its groups is; the lane that wrote a word rewrites it.
  if (__any_sync(kFull, badmask != 0u)) {
    const unsigned rowmask = (LPR == 32 ? kFull : ((1u << LPR) - 1u)) << (riw * LPR);
    for (int n = 0; n < kPass; ++n) {
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const unsigned bal = __ballot_sync(kFull, (badmask >> (2 * n + h)) & 1u);
        if ((bal & rowmask) == 0u) continue;
        const uint32_t z[4] = {0u, 0u, 0u, 0u};
        const bool st = MT && to_stage;
        if (st || LORES_IN(p, kRgCodes, gc + n * 2 * RPW * RB + h * RB, LB))
          pair_store<BITS>(gc + n * 2 * RPW * RB + h * RB, z, st);
        if (scale_writer && (st || LORES_IN(p, kRgScales, gs + (n * 2 * RPW + h) * ng, 4)))
          gs[(n * 2 * RPW + h) * ng] = 0.0f;
        if (lir == 0) atomicOr(p.flag, kFlagNonFinite);
      }
    }
  }

  // ---- readout: o_i = sum of the row's lane shares + w_i (k.q) -------------------------
  __syncwarp();
  constexpr int kRows = full_rows(DK, BITS);
  float *go = p.o + (MT ? tok * p.tok_o : 0ll) + tile * p.d_v + d.row0;
#pragma unroll
  for (int r = lane; r < kRows; r += 32) {
    float acc = 0.0f;
    if (LPR >= 4) {
#pragma unroll
      for (int l = 0; l < LPR; l += 4) {
        const float4 v4 = *reinterpret_cast<const float4 *>(opart + r * LPR + l);
        acc = __fadd_rn(__fadd_rn(__fadd_rn(__fadd_rn(acc, v4.x), v4.y), v4.z), v4.w);
      }
    } else {
#pragma unroll
      for (int l = 0; l < LPR; ++l) acc = __fadd_rn(acc, opart[r * LPR + l]);
    }
    if (LORES_IN(p, kRgO, go + r, 4)) go[r] = __fmaf_rn(ow[r], t.kq, acc);
  }
  __syncwarp();
}

// Position of a unit: sequence b, unit ub of the sequence's table, inside the class's
// range [lo, hi) of the table.
struct PairPos {
  int b, ub;
  __device__ __forceinline__ void next(int lo, int hi) {
    if (++ub == hi) {
      ub = lo;
      ++b;
    }
  }
};

// The persistent loop of one warp over the units of one storage class (BITS): the
// class's units are table entries [lo, hi) of every sequence, U = B (hi - lo) in all;
// warp gw of the W warps given to the class takes units [U gw / W, U (gw + 1) / W) in
// (sequence, unit) order, through a 2-slot ring of bulk copies whose producer is the
// warp itself.  Warps never wait on one another.
template <int DK, bool DIAG, bool DELTA, bool SR, bool GROW, int BITS, bool MT>
__device__ __forceinline__ void pair_run(const StepParams &p, const UnitDesc *tbl, uint8_t *wa,
                                         int cta, int nctas, int lo, int hi) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint64_t *bars = reinterpret_cast<uint64_t *>(wa);
  float *opart = reinterpret_cast<float *>(wa + 64);
  float *ow = opart + p.opart_floats;
  uint8_t *stages = reinterpret_cast<uint8_t *>(ow + p.ow_floats) + p.plane_bytes;
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
  PairPos fill = start;                             // the next unit to copy in
  int ftile = -1;                                   // tile of the last unit copied in
  for (int s = 0; s < kStages && s < count; ++s) {
    const UnitDesc d = tbl[fill.ub];
    const int tl = fill.b * H + d.head;
    pair_issue<DK, DIAG, MT>(p, d, fill.b, fill.ub, tl != ftile, stages + s * p.stage_bytes, &bars[s]);
    ftile = tl;
    fill.next(lo, hi);
  }
  const uint32_t skey = p.step_dev ? step_key_dev(p.seed, *p.step_dev) : p.step_key;

  PairPos cur = start;
  int ctile = -1;                                   // tile whose vectors are in registers
  PairTile<DIAG> t;
  // beta and scalar alpha of the current unit's tile, and of the next unit's
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
      // Give up: record it, let the other slot's copy (if any) land, and leave.
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
      // every token of the unit in turn; the unit's rows stay in the slot in between
      const int col0 = (lane % (DK / 16)) * 16;
      for (int tok = 0; tok < p.T; ++tok) {
        const float *k = p.k + tok * p.tok_qk + (long long)tl * DK;
        const float *q = p.q + tok * p.tok_qk + (long long)tl * DK;
        if (!(LORES_IN(p, kRgK, k, DK * 4) && LORES_IN(p, kRgQ, q, DK * 4) &&
              LORES_IN(p, kRgV, p.v + tok * p.tok_v + (long long)tl * p.d_v + d.row0, d.nrows * 4) &&
              (!DIAG || LORES_IN(p, kRgAlpha, p.alpha + tok * p.tok_a + (long long)tl * DK, DK * 4))))
          continue;                            // index-checked build: vectors out of range
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const float4 k4 = __ldg(reinterpret_cast<const float4 *>(k + col0) + c);
          const float4 q4 = __ldg(reinterpret_cast<const float4 *>(q + col0) + c);
          t.kk[2 * c] = make_float2(k4.x, k4.y);
          t.kk[2 * c + 1] = make_float2(k4.z, k4.w);
          t.qq[2 * c] = make_float2(q4.x, q4.y);
          t.qq[2 * c + 1] = make_float2(q4.z, q4.w);
          if (DIAG) {
            const float4 a4 = __ldg(reinterpret_cast<const float4 *>(
                                        p.alpha + tok * p.tok_a + (long long)tl * DK + col0) + c);
            t.aa[2 * c] = make_float2(a4.x, a4.y);
            t.aa[2 * c + 1] = make_float2(a4.z, a4.w);
          }
        }
        double kqd = 0.0;
#pragma unroll
        for (int j = lane; j < DK; j += 32) kqd = fma((double)__ldg(k + j), (double)__ldg(q + j), kqd);
#pragma unroll
        for (int st = 16; st >= 1; st >>= 1) kqd += __shfl_xor_sync(kFull, kqd, st);
        t.kq = (float)kqd;
        t.tkey = tile_key(step_key_dev(p.seed, p.step0 + (uint64_t)tok), (uint32_t)tl);
        t.beta = LORES_LDG(p, kRgBeta, p.beta + tok * p.tok_b + tl);
        t.alpha = DIAG ? 0.0f : LORES_LDG(p, kRgAlpha, p.alpha + tok * p.tok_a + tl);
        pair_unit<DK, DIAG, DELTA, SR, BITS, GROW, MT>(p, stage, cur.b, d, t, opart, ow, tok,
                                                       tok + 1 < p.T);
      }
    } else {
      if (tl != ctile) {
        // a new tile: its vectors are in this slot
        const float *sk = reinterpret_cast<const float *>(stage + p.st_k);
        const int col0 = (lane % (DK / 16)) * 16;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const float4 k4 = *reinterpret_cast<const float4 *>(sk + col0 + 4 * c);
          const float4 q4 = *reinterpret_cast<const float4 *>(sk + DK + col0 + 4 * c);   // q
          t.kk[2 * c] = make_float2(k4.x, k4.y);
          t.kk[2 * c + 1] = make_float2(k4.z, k4.w);
          t.qq[2 * c] = make_float2(q4.x, q4.y);
          t.qq[2 * c + 1] = make_float2(q4.z, q4.w);
          if (DIAG) {
            const float4 a4 = *reinterpret_cast<const float4 *>(sk + 2 * DK + col0 + 4 * c);
            t.aa[2 * c] = make_float2(a4.x, a4.y);
            t.aa[2 * c + 1] = make_float2(a4.z, a4.w);
          }
        }
        // k.q in double (strided columns, warp butterfly): the readout is S'q + w (k.q)
        double kqd = 0.0;
#pragma unroll
        for (int j = lane; j < DK; j += 32) kqd = fma((double)sk[j], (double)sk[DK + j], kqd);
#pragma unroll
        for (int st = 16; st >= 1; st >>= 1) kqd += __shfl_xor_sync(kFull, kqd, st);
        t.kq = (float)kqd;
        t.tkey = tile_key(skey, (uint32_t)tl);
        ctile = tl;
      }
      t.beta = beta_c;
      t.alpha = alpha_c;
      pair_unit<DK, DIAG, DELTA, SR, BITS, GROW, MT>(p, stage, cur.b, d, t, opart, ow, 0, false);
    }
    // pair_unit ends with __syncwarp: every lane is done reading this slot
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
// pair_hi[1])): CTAs [0, pair_ctas) take the first class, the others the second, so every
// CTA runs one code path (the host splits the CTAs in proportion to the state entries).
template <int DK, bool DIAG, bool DELTA, bool SR, bool GROW, bool MT>
__global__ void __launch_bounds__(kThreads, LORES_PAIR_MIN_CTAS) decode_pair_kernel(const StepParams p) {
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
  const int cta = (int)blockIdx.x;
  if (cta < p.pair_ctas)
    pair_run<DK, DIAG, DELTA, SR, GROW, 8, MT>(p, tbl, wa, cta, p.pair_ctas, p.pair_lo[0],
                                               p.pair_hi[0]);
  else
    pair_run<DK, DIAG, DELTA, SR, GROW, 4, MT>(p, tbl, wa, cta - p.pair_ctas,
                                               (int)gridDim.x - p.pair_ctas, p.pair_lo[1],
                                               p.pair_hi[1]);
}

template <int DK, bool SR, bool GROW, bool MT>
StepFn pick_pair(bool diag, bool delta) {
  if (diag)
    return delta ? decode_pair_kernel<DK, true, true, SR, GROW, MT>
                 : decode_pair_kernel<DK, true, false, SR, GROW, MT>;
  return delta ? decode_pair_kernel<DK, false, true, SR, GROW, MT>
               : decode_pair_kernel<DK, false, false, SR, GROW, MT>;
}

// One function per (key width, single / multi-token), each defined in its own compilation
// of lores_inst.cu: heads with several scales per row (heads with one scale per row take
// the tensor-core kernel of lores_mma.cuh, or the general kernel).
#define LORES_DECLARE_PAIR(dk)                                    \
  StepFn pair_kernels_##dk##_0(bool diag, bool delta, bool sr);  \
  StepFn pair_kernels_##dk##_1(bool diag, bool delta, bool sr);
LORES_DECLARE_PAIR(16)
LORES_DECLARE_PAIR(32)
LORES_DECLARE_PAIR(64)
LORES_DECLARE_PAIR(128)
LORES_DECLARE_PAIR(256)
#undef LORES_DECLARE_PAIR

}  // namespace lores
