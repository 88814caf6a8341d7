// lores_step.cuh -- the decode-step kernel of the LoReS quantized recurrent state
// (sm_100a), shared by the single-token and multi-token translation units.
//
// One decode step of a linear-recurrence layer ("Quantizing Recurrent Language Models Is
// Easier Than You Think", summary page: General recurrence form; Key properties item 3;
// Proposition 1; Table 5 text; Proposition 3 / Table 6):
//   S_t = S_{t-1} diag(alpha_t) (I - delta beta_t k_t k_t^T) + beta_t v_t k_t^T,  o_t = S_t q_t
// with S_{t-1} dequantized from b-bit codes and per-(value row, key block) fp32 scales and
// S_t requantized with stochastic rounding, all in one pass over the state.
#pragma once
#include <cstdint>

#include "lores_device.cuh"

namespace lores {

// One work unit: a block of rows of one (sequence, head) tile, processed by one warp.
struct __align__(16) UnitDesc {
  int32_t head;
  int16_t row0;
  int16_t nrows;
  int16_t bits;          // 4..8 (b-bit codes), 32 (fp32 state), or 0: a bit width per key
                         // group (per-channel precision; the lane table has the layout)
  int16_t rowb;          // bytes of one row of the head
  int16_t store;         // storage: 4 nibbles, 8 one byte per code, 32 fp32, 5..7 dense
                         // bit planes, 0 per-lane (lane table)
  int16_t pad;
  int64_t code_off;      // byte offset of row0 of this head inside one sequence's block
  float r;               // largest code, 2^(bits-1) - 1 (bits 4..8)
  float inv_r;           // fl(1/r)
};

// Layout of the 16 columns a lane owns, per (head, 16-column block): the block's bit
// width (its key group's), its byte offset inside a row, r and fl(1/r), and the head's
// row bytes.  Rows store their key groups back to back, group g in G * storage(b_g) / 8
// bytes (4-bit codes as nibbles, 5 to 8 bits one byte each, fp32 heads 4 bytes).
struct __align__(16) LaneFmt {
  float r;
  float inv_r;
  int32_t off;
  int8_t bits;
  int8_t store;          // as UnitDesc::store (dense lanes: off is the nibble part's)
  int16_t rowb;
};

struct StepParams {
  uint8_t *codes;        // [B][seq_bytes]
  float *scales;         // [B][H][d_v][ng]
  const float *q, *k, *v, *alpha, *beta;
  float *o;
  unsigned *flag;
  const UnitDesc *units; // [units_per_seq]
  const LaneFmt *fmt;    // [H][d_k/16]
  long long seq_bytes;
  long long total_units;
  int B, H, d_v, ng, G, units_per_seq;
  uint32_t step_key;
  // shared memory layout: [unit table][warp 0 area][warp 1 area]...; a warp area is
  // [2 mbarriers | pad to 64][readout partials][row w][digit planes][stage 0][stage 1]
  int table_bytes;       // bytes of the unit table copy (0: read the table from global)
  int warp_bytes;        // bytes of one warp area
  int opart_floats;      // readout partials per warp (max rows * lanes per row)
  int ow_floats;         // row w per warp (max rows)
  int plane_bytes;       // exact contractions' scratch per warp: digit planes (8 d_k
                         // bytes), a tile's k and alpha (8 d_k)
  int st_scales, st_k, st_q, st_v, st_a, stage_bytes;   // stage layout
  // multi-token steps: T tokens, token t reads q, k, v, alpha, beta at t * tok_* and
  // writes o at t * tok_o, with the dither of step step0 + t (keys made on the device)
  int T;
  long long tok_qk, tok_v, tok_a, tok_b, tok_o;
  uint64_t seed, step0;
  // single steps replayed from a captured CUDA graph read the step from device memory
  const uint64_t *step_dev;
  // two-rows-per-lane kernel (lores_pair.cuh): per-sequence table ranges of the heads
  // stored one byte per code [pair_lo[0], pair_hi[0]) and one nibble per code
  // [pair_lo[1], pair_hi[1]); CTAs [0, pair_ctas) take the first
  int pair_lo[2], pair_hi[2];
  int pair_ctas;
  // bounded waits give up after wait_ns of GPU time; failure-path testing: the copies of
  // unit fault_ub of sequence fault_b are withheld (fault_b = -1: none)
  unsigned long long wait_ns;
  int fault_b, fault_ub;
  LORES_RANGES           // index-checked build: the extent of every buffer of the launch
};

// Step key of the dither: SplitMix64 (Steele, Lea & Flood 2014; Vigna's constants) of the
// seed xor SplitMix64 of the step, folded to 32 bits (the host computes the same).
__device__ __forceinline__ uint64_t splitmix64_dev(uint64_t z) {
  z += 0x9E3779B97F4A7C15ull;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}
__device__ __forceinline__ uint32_t step_key_dev(uint64_t seed, uint64_t step) {
  const uint64_t k = splitmix64_dev(seed ^ splitmix64_dev(step));
  return (uint32_t)(k ^ (k >> 32));
}

// Storage of b-bit codes: 4-bit codes as nibbles, 5- to 8-bit codes one per byte.
__host__ __device__ constexpr int storage_bits(int bits) {
  return bits == 4 ? 4 : (bits == 32 ? 32 : 8);
}
// Bytes of one row of a tile with `bits`-bit entries stored one byte per code (5..8),
// as nibbles (4) or fp32 (32).
__host__ __device__ constexpr int row_bytes(int dk, int bits) { return dk * storage_bits(bits) / 8; }
// Bytes of one row for a storage class: 4, 8, 32 as above; 5..7 dense bit planes, the
// row padded to a multiple of 8 bytes.
__host__ __device__ constexpr int store_row_bytes(int dk, int store) {
  return (store >= 5 && store <= 7) ? (dk * store / 8 + 7) / 8 * 8 : dk * store / 8;
}

// Rows of a full unit: 4 KB of state, a whole number of warp passes (32/(d_k/16) rows).
// (store: the storage class, see UnitDesc::store)
__host__ __device__ constexpr int full_rows(int dk, int store) {
  return (4096 / store_row_bytes(dk, store)) < (32 / (dk / 16))
             ? (32 / (dk / 16))
             : (4096 / store_row_bytes(dk, store)) -
                   (4096 / store_row_bytes(dk, store)) % (32 / (dk / 16));
}

// -------------------------------------------------------------------------------------
// producer (the whole warp): stage one unit's inputs into the warp's ring slot
// -------------------------------------------------------------------------------------
// Lane 0 announces the byte count on the slot's mbarrier; then lanes 0-5 each issue one
// of the unit's bulk copies (codes, scales, k, q, v slice, per-column alpha) in parallel.
// Multi-token steps (MT) stage only codes and scales; the per-token vectors are read
// from global memory.
template <int DK, bool DIAG, bool MT>
__device__ __forceinline__ void issue_unit(const StepParams &p, const UnitDesc *tbl, int b, int ub,
                                           uint8_t *stage, uint64_t *bar) {
  const int lane = threadIdx.x & 31;
  const UnitDesc d = tbl[ub];
  const long long tile = (long long)b * p.H + d.head;
  const bool withhold = b == p.fault_b && ub == p.fault_ub;   // failure-path test only
  const unsigned cbytes = (unsigned)(d.nrows * d.rowb);
  const unsigned sbytes = d.bits == 32 ? 0u : (unsigned)(d.nrows * p.ng * 4);
  const unsigned vbytes = (unsigned)(d.nrows * 4);
  const unsigned vec = DK * 4;
  if (lane == 0)
    mbar_expect_tx(bar, cbytes + sbytes + (MT ? 0u : vbytes + 2 * vec + (DIAG ? vec : 0u)));
  __syncwarp();
  const void *src = nullptr;
  int dst = 0, rid = kRgCodes;
  unsigned bytes = 0;
  if (lane == 0) { src = p.codes + (long long)b * p.seq_bytes + d.code_off; dst = 0; bytes = cbytes; }
  if (lane == 1) { src = p.scales + (tile * p.d_v + d.row0) * p.ng; dst = p.st_scales; bytes = sbytes; rid = kRgScales; }
  if (!MT && lane == 2) { src = p.k + tile * DK; dst = p.st_k; bytes = vec; rid = kRgK; }
  if (!MT && lane == 3) { src = p.q + tile * DK; dst = p.st_q; bytes = vec; rid = kRgQ; }
  if (!MT && lane == 4) { src = p.v + tile * p.d_v + d.row0; dst = p.st_v; bytes = vbytes; rid = kRgV; }
  if (!MT && DIAG && lane == 5) { src = p.alpha + tile * DK; dst = p.st_a; bytes = vec; rid = kRgAlpha; }
  (void)rid;
  if (bytes && !withhold && LORES_IN(p, rid, src, bytes) && LORES_IN_SMEM(p, stage + dst, bytes))
    bulk_g2s(stage + dst, src, bytes, bar);
}

// -------------------------------------------------------------------------------------
// consumer (the whole warp): rows [row0, row0 + nrows) of one tile from a stage
// -------------------------------------------------------------------------------------
// Lane layout: LPR = d_k/16 lanes own a row, 16 consecutive columns each; a warp pass
// covers RPW = 32/LPR rows.  FULL: every pass is complete (nrows % RPW == 0).
// The readout is reduced per warp: each lane leaves its share of S'q in opart, lane 0
// of the row leaves w in ow, and after the rows each lane forms o for one row as
// sum(opart) + w (k.q).
// Multi-token steps (MT): token t reads its vectors from global memory; tokens before
// the last write the requantized rows back into the stage (each lane rewrites the bytes
// it read; a group's scale is rewritten after the group's lanes have read it), so the
// next token dequantizes them from shared memory; the last token writes global memory.
template <int DK, bool DIAG, bool DELTA, bool SR, int BITS, bool FULL, bool GROW, bool MT,
          bool EXACT>
__device__ __forceinline__ void compute_unit(const StepParams &p, uint8_t *stage, int b,
                                             const UnitDesc &d, float alpha_s, float beta,
                                             float *opart, float *ow, int t) {
  constexpr int LPR = DK / 16;            // lanes per row
  constexpr int RPW = 32 / LPR;           // rows per warp pass
  const int lane = threadIdx.x & 31;
  const int lir = lane % LPR, riw = lane / LPR;
  const int col0 = lir * 16;
  // BITS = 0: a bit width per key group; the lane's width, offset and r come from the
  // lane table (lanes of a warp may differ; cross-lane steps stay convergent)
  constexpr bool DENSE = BITS >= 5 && BITS <= 7;            // dense bit planes
  const int RB = BITS == 0 ? (int)d.rowb : store_row_bytes(DK, BITS);   // bytes per row
  int lsb = BITS, loff = lir * 2 * BITS;                    // lane storage bits, byte offset
  float rq = d.r, rq_inv = d.inv_r;
  if (BITS == 0) {
    const LaneFmt f = p.fmt[d.head * (DK / 16) + lir];
    lsb = f.bits == 4 ? 4 : 8;
    loff = f.off;
    rq = f.r;
    rq_inv = f.inv_r;
  }
  const bool w8 = BITS == 8 || (BITS == 0 && lsb == 8);     // byte codes (else nibbles)
  // GROW: one scale per value row (G = d_k), known at compile time
  const int lpg = GROW ? LPR : p.G / 16;                   // lanes per scale group (power of 2)
  const int g = GROW ? 0 : lir / lpg;                      // this lane's group in the row
  const bool scale_writer = (lir & (lpg - 1)) == 0;
  const int ng = GROW ? 1 : p.ng;
  const long long tile = (long long)b * p.H + d.head;

  const float *sk = MT ? p.k + t * p.tok_qk + tile * DK
                      : reinterpret_cast<const float *>(stage + p.st_k);
  const float *sq = MT ? p.q + t * p.tok_qk + tile * DK
                      : reinterpret_cast<const float *>(stage + p.st_q);
  const float *sv = MT ? p.v + t * p.tok_v + tile * p.d_v + d.row0
                      : reinterpret_cast<const float *>(stage + p.st_v);
  const float *sa = MT ? p.alpha + t * p.tok_a + tile * DK
                      : reinterpret_cast<const float *>(stage + p.st_a);
  float *ss = reinterpret_cast<float *>(stage + p.st_scales);
  const bool to_stage = MT && t + 1 < p.T;   // not the last token: rows go back to the stage
  if (MT && !(LORES_IN(p, kRgK, sk, DK * 4) && LORES_IN(p, kRgQ, sq, DK * 4) &&
              LORES_IN(p, kRgV, sv, d.nrows * 4) && (!DIAG || LORES_IN(p, kRgAlpha, sa, DK * 4))))
    return;                                  // index-checked build: vectors out of range
  // element pair e holds columns (col0 + 2e, col0 + 2e + 1)
  float2 kk[8], qq[8], aa[8];
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    const float4 k4 = *reinterpret_cast<const float4 *>(sk + col0 + 4 * c);
    const float4 q4 = *reinterpret_cast<const float4 *>(sq + col0 + 4 * c);
    kk[2 * c] = make_float2(k4.x, k4.y); kk[2 * c + 1] = make_float2(k4.z, k4.w);
    qq[2 * c] = make_float2(q4.x, q4.y); qq[2 * c + 1] = make_float2(q4.z, q4.w);
    if (DIAG) {
      const float4 a4 = *reinterpret_cast<const float4 *>(sa + col0 + 4 * c);
      aa[2 * c] = make_float2(a4.x, a4.y); aa[2 * c + 1] = make_float2(a4.z, a4.w);
    }
  }
  // k.q in double (strided columns, warp butterfly): the readout is o = S'q + w (k.q),
  // which keeps the step-0 readout (S' = 0) exact even for nearly orthogonal k and q.
  double kqd = 0.0;
#pragma unroll
  for (int j = lane; j < DK; j += 32) kqd = fma((double)sk[j], (double)sq[j], kqd);
#pragma unroll
  for (int st = 16; st >= 1; st >>= 1) kqd += __shfl_xor_sync(kFull, kqd, st);
  const float kq = (float)kqd;
  const uint32_t skey = MT ? step_key_dev(p.seed, p.step0 + (uint64_t)t)
                           : (p.step_dev ? step_key_dev(p.seed, *p.step_dev) : p.step_key);
  const uint32_t tkey = tile_key(skey, (uint32_t)tile);
  // shuffle distances of the group-max levels (0 beyond the group width: own value)
  const int gd1 = 1 < lpg ? 1 : 0, gd2 = 2 < lpg ? 2 : 0, gd4 = 4 < lpg ? 4 : 0,
            gd8 = 8 < lpg ? 8 : 0;

  uint8_t *gcodes = p.codes + (long long)b * p.seq_bytes + d.code_off;
  float *gscales = p.scales + (tile * p.d_v + d.row0) * ng;
  constexpr int kFullPasses = full_rows(DK, BITS == 0 ? 8 : BITS) / RPW;   // FULL: BITS != 0
  // FULL: every pass complete; the pass count is a compile-time constant except for
  // mixed-width rows (BITS = 0), whose unit sizes follow each head's row bytes
  const int npass = FULL ? (BITS == 0 ? d.nrows / RPW : kFullPasses) : (d.nrows + RPW - 1) / RPW;
  // dither counter of the lane's first quad in pass 0: n0 = (row0 + riw) d_k/4 + 4 lir;
  // each pass moves RPW rows, i.e. RPW d_k/4 quads
  const uint32_t cbase0 =
      tkey + 0x9E3779B9u * ((uint32_t)(d.row0 + riw) * (uint32_t)(DK / 4) + (uint32_t)lir * 4u + 1u);
  constexpr uint32_t kCtrPerPass = 0x9E3779B9u * (uint32_t)(RPW * DK / 4);
  uint32_t badmask = 0;                        // bit n: this lane's group was bad in pass n
  // exact contractions (codes one byte or one nibble each, one scale per row): S'k and
  // S'q from the digit planes of the fixed-point alpha k and alpha q, built once per unit
  // (per token)
  constexpr bool kMayExact = EXACT && (BITS == 8 || BITS == 4);
  const bool exact = kMayExact && (GROW || p.G == DK);
  uint8_t *planes = reinterpret_cast<uint8_t *>(ow + p.ow_floats);
  double sx = 0.0, sxq = 0.0;                  // 2^-E of k and q (NaN: non-finite)
  if (kMayExact && exact) {
    __syncwarp();                              // the previous unit's plane reads are done
    if (DELTA) sx = fixed_point_planes_call<DK>(sk, sa, DIAG, alpha_s, planes, DK);
    sxq = fixed_point_planes_call<DK>(sq, sa, DIAG, alpha_s, planes + 4 * DK, DK);
    __syncwarp();
  }

#pragma unroll(FULL ? (BITS == 0 ? 2 : 4) : 1)
  for (int n = 0; n < npass; ++n) {
    const int lr = n * RPW + riw;              // row inside the unit
    const bool active = FULL || lr < d.nrows;
    const int lrr = active ? lr : 0;           // keep shared loads in bounds
    // dither words first: they depend only on the counter, so they fill the latency of
    // the dot-product and group-max shuffles below
    uint32_t hw[4] = {0u, 0u, 0u, 0u};
    if (SR && BITS != 32) dither_words(cbase0 + kCtrPerPass * (uint32_t)n, hw);

    // ---- dequantize and decay: S'_ij = c_ij * (s_ig * alpha_j) ----------------------
    float2 sp[8];
    float u_ex = 0.0f, sq_ex = 0.0f;           // exact contractions: the row's u and S'q
    float s_in = 0.0f;
    if (BITS == 32) {
      const float *srow = reinterpret_cast<const float *>(stage + (size_t)lrr * RB) + col0;
      const float2 as = dup2(alpha_s);
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const float4 s4 = *reinterpret_cast<const float4 *>(srow + 4 * c);
        sp[2 * c] = __fmul2_rn(make_float2(s4.x, s4.y), DIAG ? aa[2 * c] : as);
        sp[2 * c + 1] = __fmul2_rn(make_float2(s4.z, s4.w), DIAG ? aa[2 * c + 1] : as);
      }
    } else {
      float2 cf[8];
      if (DENSE) {
        unpack_dense<DENSE ? BITS : 5>(ld_dense<DENSE ? BITS : 5>(stage + (size_t)lrr * RB, DK, lir), cf);
      } else if (BITS == 0) {
        // per-lane widths: both kinds of lane bring their codes to offset-binary bytes,
        // then take one conversion together
        uint32_t ob[4];
        const uint8_t *src = stage + (size_t)lrr * RB + loff;
        if (w8) {
          const uint4 cw = ld16_a8(src);
          ob[0] = cw.x ^ 0x80808080u; ob[1] = cw.y ^ 0x80808080u;
          ob[2] = cw.z ^ 0x80808080u; ob[3] = cw.w ^ 0x80808080u;
        } else {
          widen_i4_ob(*reinterpret_cast<const uint2 *>(src), ob);
        }
        unpack_ob_2(ob, cf);
      } else if (w8) {
        const uint4 cw = BITS == 0 ? ld16_a8(stage + (size_t)lrr * RB + loff)   // 8-byte aligned
                                   : *reinterpret_cast<const uint4 *>(stage + (size_t)lrr * RB + loff);
        s_in = ss[lrr * ng + g];
        if (kMayExact && exact) {
          // the contractions first, so their digit words and sums are dead before the
          // floats live
          const uint32_t cs[4] = {cw.x, cw.y, cw.z, cw.w};
          exact_row<LPR, DELTA>(cs, planes + col0, DK, s_in, sx, sxq, u_ex, sq_ex);
        }
        unpack_i8_2(cw, cf);
      } else {
        const uint2 cw = *reinterpret_cast<const uint2 *>(stage + (size_t)lrr * RB + loff);
        s_in = ss[lrr * ng + g];
        if (kMayExact && exact) {
          uint32_t cs[4];
          i4_to_s8(cw, cs);
          exact_row<LPR, DELTA>(cs, planes + col0, DK, s_in, sx, sxq, u_ex, sq_ex);
        }
        unpack_i4_2(cw, cf);
      }
      if (DENSE || BITS == 0) s_in = ss[lrr * ng + g];
      const float2 s2 = dup2(s_in);
      const float2 a_row = dup2(__fmul_rn(s_in, alpha_s));
#pragma unroll
      for (int e = 0; e < 8; ++e) sp[e] = __fmul2_rn(cf[e], DIAG ? __fmul2_rn(s2, aa[e]) : a_row);
    }

    // ---- write: w = beta (v - delta (S'k)), x = S' + w k^T ----------------------------
    const float vr = sv[lrr];
    float w;
    if (kMayExact && exact && DELTA) {
      w = __fmul_rn(beta, __fsub_rn(vr, u_ex));
    } else if (DELTA) {
      float u = dot16_p(sp, kk);
#pragma unroll
      for (int st = 1; st < LPR; st <<= 1) u = __fadd_rn(u, __shfl_xor_sync(kFull, u, st));
      w = __fmul_rn(beta, __fsub_rn(vr, u));
    } else {
      w = __fmul_rn(beta, vr);
    }
    float2 x[8];
    const float2 w2 = dup2(w);
#pragma unroll
    for (int e = 0; e < 8; ++e) x[e] = __ffma2_rn(w2, kk[e], sp[e]);

    // ---- readout share: this lane's part of S'q ----------------------------------------
    float opv;
    if (kMayExact && exact) {
      // exact: the row's S'q in its first lane's share, zero in the others
      opv = lir == 0 ? sq_ex : 0.0f;
    } else {
      opv = dot16_p(sp, qq);
    }
    if (active) {
      opart[lr * LPR + lir] = opv;
      if (lir == 0) ow[lr] = w;
    }

    // ---- requantize and store (bad rows are fixed up after the passes) ------------------
    bool gbad;
    if (BITS == 32) {
      float m = 0.0f;
#pragma unroll
      for (int e = 0; e < 8; ++e) m = max_abs_nan(max_abs_nan(m, x[e].x), x[e].y);
      gbad = !(m <= 3.402823466e38f);
      if (active) {
        if (to_stage) {
          float4 *dst = reinterpret_cast<float4 *>(stage + (size_t)lr * RB) + lir * 4;
#pragma unroll
          for (int c = 0; c < 4; ++c)
            dst[c] = make_float4(x[2 * c].x, x[2 * c].y, x[2 * c + 1].x, x[2 * c + 1].y);
        } else {
          float4 *dst = reinterpret_cast<float4 *>(gcodes + (size_t)lr * RB) + lir * 4;
          if (LORES_IN(p, kRgCodes, dst, 64))
#pragma unroll
            for (int c = 0; c < 4; ++c)
              __stcs(dst + c, make_float4(x[2 * c].x, x[2 * c].y, x[2 * c + 1].x, x[2 * c + 1].y));
        }
      }
    } else {
      uint32_t words[4];
      float s_new;
      if (DENSE) {
        constexpr int DB = DENSE ? BITS : 5;
        const float m = group_absmax<LPR>(chunk_absmax(x), gd1, gd2, gd4, gd8);
        float2 inv;
        gbad = group_scale(m, rq, rq_inv, inv, s_new);
        const DenseLane dl = quantize16_dense<DB, SR>(x, inv, hw);
        if (active && (to_stage || LORES_IN(p, kRgCodes, gcodes + (size_t)lr * RB, RB))) {
          st_dense<DB>((to_stage ? stage : gcodes) + (size_t)lr * RB, DK, lir, dl);
          if (scale_writer && (to_stage || LORES_IN(p, kRgScales, gscales + lr * ng + g, 4)))
            (to_stage ? ss : gscales)[lr * ng + g] = s_new;
        }
      } else if (BITS == 0) {
        // group scale with every lane, then each lane packs at its own width
        const float m = group_absmax<LPR>(chunk_absmax(x), gd1, gd2, gd4, gd8);
        float2 inv;
        gbad = group_scale(m, rq, rq_inv, inv, s_new);
        quantize16<8, SR>(x, inv, hw, words);            // code bytes for every lane
        if (!w8) {                                       // nibble lanes compact them
          const uint2 nw = compact_i4(make_uint4(words[0], words[1], words[2], words[3]));
          words[0] = nw.x;
          words[1] = nw.y;
        }
      } else {
        gbad = requantize16_nb<LPR, BITS, SR>(x, rq, rq_inv, gd1, gd2, gd4, gd8, hw, words, s_new);
      }
      if (!DENSE && active) {
        if (to_stage) {
          if (w8 && BITS == 0)
            st16_a8(stage + (size_t)lr * RB + loff, make_uint4(words[0], words[1], words[2], words[3]));
          else if (w8)
            *reinterpret_cast<uint4 *>(stage + (size_t)lr * RB + loff) =
                make_uint4(words[0], words[1], words[2], words[3]);
          else
            *reinterpret_cast<uint2 *>(stage + (size_t)lr * RB + loff) = make_uint2(words[0], words[1]);
          if (scale_writer) ss[lr * ng + g] = s_new;
        } else {
          uint8_t *cdst = gcodes + (size_t)lr * RB + loff;
          if (!LORES_IN(p, kRgCodes, cdst, w8 ? 16 : 8)) {
          } else if (w8 && BITS == 0) {
            uint2 *dst = reinterpret_cast<uint2 *>(cdst);
            __stcs(dst, make_uint2(words[0], words[1]));
            __stcs(dst + 1, make_uint2(words[2], words[3]));
          } else if (w8) {
            __stcs(reinterpret_cast<uint4 *>(cdst), make_uint4(words[0], words[1], words[2], words[3]));
          } else
            __stcs(reinterpret_cast<uint2 *>(cdst), make_uint2(words[0], words[1]));
          if (scale_writer && LORES_IN(p, kRgScales, gscales + lr * ng + g, 4))
            gscales[lr * ng + g] = s_new;
        }
      }
    }
    badmask |= (gbad && active ? 1u : 0u) << n;
  }

  // ---- rare: rows with a non-finite (or overflowing) entry -----------------------------
  // A row is bad if any of its groups is; quantized rows are stored as zero.  The lane
  // that wrote a word rewrites it, so no ordering between lanes is needed.
  if (__any_sync(kFull, badmask != 0u)) {
    const unsigned rowmask = (LPR == 32 ? kFull : ((1u << LPR) - 1u)) << (riw * LPR);
    for (int n = 0; n < npass; ++n) {
      const unsigned bal = __ballot_sync(kFull, (badmask >> n) & 1u);
      const int lr = n * RPW + riw;
      if ((bal & rowmask) == 0u || !(FULL || lr < d.nrows)) continue;
      const bool sok = to_stage || LORES_IN(p, kRgScales, gscales + lr * ng + g, 4);
      if (DENSE) {
        if (to_stage || LORES_IN(p, kRgCodes, gcodes + (size_t)lr * RB, RB))
          st_dense<DENSE ? BITS : 5>((to_stage ? stage : gcodes) + (size_t)lr * RB, DK, lir,
                                     DenseLane{0u, 0u, 0u, 0u});
        if (scale_writer && sok) (to_stage ? ss : gscales)[lr * ng + g] = 0.0f;
      } else if (BITS != 32) {
        uint8_t *dst = (to_stage ? stage : gcodes) + (size_t)lr * RB + loff;
        if (!to_stage && !LORES_IN(p, kRgCodes, dst, w8 ? 16 : 8)) {
        } else if (w8)
          st16_a8(dst, make_uint4(0, 0, 0, 0));
        else
          *reinterpret_cast<uint2 *>(dst) = make_uint2(0, 0);
        if (scale_writer && sok) (to_stage ? ss : gscales)[lr * ng + g] = 0.0f;
      }
      if (lir == 0) atomicOr(p.flag, kFlagNonFinite);
    }
  }

  // ---- readout: o_i = sum of the row's lane shares + w_i (k.q) -------------------------
  __syncwarp();
  float *go = p.o + (MT ? t * p.tok_o : 0ll) + tile * p.d_v + d.row0;
  for (int r = lane; r < d.nrows; r += 32) {
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
    if (LORES_IN(p, kRgO, go + r, 4)) go[r] = __fmaf_rn(ow[r], kq, acc);
  }
  __syncwarp();
}

template <int DK, bool DIAG, bool DELTA, bool SR, int BITS, bool MT, bool EXACT>
__device__ __forceinline__ void compute_any(const StepParams &p, uint8_t *stage, int b,
                                            const UnitDesc &d, float alpha_s, float beta,
                                            float *opart, float *ow, int t) {
  if (BITS == 0) {
    constexpr int RPW = 32 / (DK / 16);
    if (d.nrows % RPW == 0)
      compute_unit<DK, DIAG, DELTA, SR, BITS, true, false, MT, EXACT>(p, stage, b, d, alpha_s, beta, opart, ow, t);
    else
      compute_unit<DK, DIAG, DELTA, SR, BITS, false, false, MT, EXACT>(p, stage, b, d, alpha_s, beta, opart, ow, t);
  } else if (d.nrows == full_rows(DK, BITS)) {
    if (p.G == DK)
      compute_unit<DK, DIAG, DELTA, SR, BITS, true, true, MT, EXACT>(p, stage, b, d, alpha_s, beta, opart, ow, t);
    else
      compute_unit<DK, DIAG, DELTA, SR, BITS, true, false, MT, EXACT>(p, stage, b, d, alpha_s, beta, opart, ow, t);
  } else {
    compute_unit<DK, DIAG, DELTA, SR, BITS, false, false, MT, EXACT>(p, stage, b, d, alpha_s, beta, opart, ow, t);
  }
}
// One unit for one token: the unit's storage class picks the code path.  EXT: 0 the plain
// kernel (int8 / int4 / fp32 units only, the smallest code); 3 the plain kernel with the
// exact contractions for byte and nibble heads with one scale per row; 1 also the dense 5-
// to 7-bit and per-lane (per-channel) paths; 4 the same with the exact contractions; 2 the
// per-lane path without the dense ones, so a handle with per-channel rows and no dense
// heads runs with fewer registers live.  (The exact contractions live only in the
// families that need them: their registers would otherwise cost every other path.)
template <int DK, bool DIAG, bool DELTA, bool SR, bool MT, int EXT>
__device__ __forceinline__ void compute_bits(const StepParams &p, uint8_t *stage, int b,
                                             const UnitDesc &d, float alpha_s, float beta,
                                             float *opart, float *ow, int t) {
  constexpr bool EX = EXT == 3 || EXT == 4;
  constexpr bool DENSE_PATHS = EXT == 1 || EXT == 4;
  if (d.store == 32)
    compute_any<DK, DIAG, DELTA, SR, 32, MT, EX>(p, stage, b, d, alpha_s, beta, opart, ow, t);
  else if (EXT == 0 || EXT == 3 || d.store == 4 || d.store == 8) {
    if (d.store == 4)
      compute_any<DK, DIAG, DELTA, SR, 4, MT, EX>(p, stage, b, d, alpha_s, beta, opart, ow, t);
    else
      compute_any<DK, DIAG, DELTA, SR, 8, MT, EX>(p, stage, b, d, alpha_s, beta, opart, ow, t);
  } else if (d.store == 0) {
    compute_any<DK, DIAG, DELTA, SR, 0, MT, EX>(p, stage, b, d, alpha_s, beta, opart, ow, t);
  } else if constexpr (DENSE_PATHS) {
    if (d.store == 6)
      compute_any<DK, DIAG, DELTA, SR, 6, MT, EX>(p, stage, b, d, alpha_s, beta, opart, ow, t);
    else if (d.store == 5)
      compute_any<DK, DIAG, DELTA, SR, 5, MT, EX>(p, stage, b, d, alpha_s, beta, opart, ow, t);
    else
      compute_any<DK, DIAG, DELTA, SR, 7, MT, EX>(p, stage, b, d, alpha_s, beta, opart, ow, t);
  }
}

// Position of a unit: global unit u = ub * B + b (sequence b is the fast index, so a warp
// striding through units visits the per-sequence unit table in order, and a table sorted
// by bit width keeps each warp on one code path for long runs), advanced by a fixed
// stride without divisions.
struct UnitPos {
  int b, ub;
  __device__ __forceinline__ void advance(int sb, int su, int B) {
    b += sb;
    ub += su;
    if (b >= B) {
      b -= B;
      ++ub;
    }
  }
};

// Persistent kernel: every warp runs its own pipeline over units gw, gw + W, gw + 2W, ...
// (gw = global warp index, W = warps in the grid), with a 2-slot ring of bulk copies
// whose producer is the warp's lane 0.  Warps never wait on one another.
template <int DK, bool DIAG, bool DELTA, bool SR, bool MT, int EXT>
__global__ void __launch_bounds__(kThreads, 4) decode_step_kernel(const StepParams p) {
  extern __shared__ __align__(128) uint8_t smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  UnitDesc *stbl = reinterpret_cast<UnitDesc *>(smem);
  uint8_t *wa = smem + p.table_bytes + warp * p.warp_bytes;
  uint64_t *bars = reinterpret_cast<uint64_t *>(wa);
  float *opart = reinterpret_cast<float *>(wa + 64);
  float *ow = opart + p.opart_floats;
  uint8_t *stages = reinterpret_cast<uint8_t *>(ow + p.ow_floats) + p.plane_bytes;

  const UnitDesc *tbl = p.units;
  const int ups = p.units_per_seq;
  if (p.table_bytes) {
    for (int i = threadIdx.x; i < ups; i += kThreads) stbl[i] = p.units[i];
    tbl = stbl;
  }
  __syncthreads();                                  // the only CTA-wide barrier

  const long long first = (long long)blockIdx.x * kWarps + warp;
  if (first >= p.total_units) return;
  const long long stride = (long long)gridDim.x * kWarps;
  const int B = p.B;
  const int sb = (int)(stride % B), su = (int)(stride / B);
  UnitPos cur{(int)(first % B), (int)(first / B)};

  if (lane == 0) {
    for (int s = 0; s < kStages; ++s) mbar_init(&bars[s], 1);
    fence_mbar_init();
  }
  __syncwarp();
  {
    UnitPos q = cur;
    for (int s = 0; s < kStages && q.ub < ups; ++s) {
      issue_unit<DK, DIAG, MT>(p, tbl, q.b, q.ub, stages + s * p.stage_bytes, &bars[s]);
      q.advance(sb, su, B);
    }
  }
  UnitPos nxt = cur;                                // the unit after `cur`
  nxt.advance(sb, su, B);
  UnitPos fill = nxt;                               // the unit that refills the slot just used
  fill.advance(sb, su, B);

  // per-tile scalars of the current unit; the next unit's are loaded one unit ahead
  float alpha_cur = 0.0f, beta_cur;
  {
    const long long t0 = (long long)cur.b * p.H + tbl[cur.ub].head;
    beta_cur = LORES_LDG(p, kRgBeta, p.beta + t0);
    if (!DIAG) alpha_cur = LORES_LDG(p, kRgAlpha, p.alpha + t0);
  }

  for (int n = 0; cur.ub < ups; ++n) {
    const int s = n % kStages;
    uint8_t *stage = stages + s * p.stage_bytes;
    float alpha_nx = 0.0f, beta_nx = 0.0f;
    if (nxt.ub < ups) {
      const long long tn = (long long)nxt.b * p.H + tbl[nxt.ub].head;
      beta_nx = LORES_LDG(p, kRgBeta, p.beta + tn);
      if (!DIAG) alpha_nx = LORES_LDG(p, kRgAlpha, p.alpha + tn);
    }
    const bool ok = mbar_wait_bounded(&bars[s], (unsigned)((n / kStages) & 1), p.wait_ns);
    if (!__all_sync(kFull, ok)) {
      // Give up: record it, let the other slot's copy (if any) land, and leave.
      if (lane == 0) {
        atomicOr(p.flag, kFlagTimeout);
        if (nxt.ub < ups)
          (void)mbar_wait_bounded(&bars[(n + 1) % kStages], (unsigned)(((n + 1) / kStages) & 1),
                                  p.wait_ns);
      }
      __syncwarp();
      return;
    }
    const UnitDesc d = tbl[cur.ub];
    if (MT) {
      // every token of the unit in turn; the unit's rows stay in the stage in between
      const long long tile = (long long)cur.b * p.H + d.head;
      for (int t = 0; t < p.T; ++t) {
        const float beta_t = LORES_LDG(p, kRgBeta, p.beta + t * p.tok_b + tile);
        const float alpha_t = DIAG ? 0.0f : LORES_LDG(p, kRgAlpha, p.alpha + t * p.tok_a + tile);
        compute_bits<DK, DIAG, DELTA, SR, MT, EXT>(p, stage, cur.b, d, alpha_t, beta_t, opart, ow, t);
      }
    } else {
      compute_bits<DK, DIAG, DELTA, SR, MT, EXT>(p, stage, cur.b, d, alpha_cur, beta_cur, opart, ow, 0);
    }
    // compute_unit ends with __syncwarp: every lane is done reading this slot
    if (fill.ub < ups) {
      fence_proxy_async();
      issue_unit<DK, DIAG, MT>(p, tbl, fill.b, fill.ub, stage, &bars[s]);
    }
    cur = nxt;
    nxt.advance(sb, su, B);
    fill.advance(sb, su, B);
    alpha_cur = alpha_nx;
    beta_cur = beta_nx;
  }
}

using StepFn = void (*)(const StepParams);

// Kernel pickers: every (key width, single/multi-token, storage family) is instantiated
// in its own compilation of lores_inst.cu.
template <int DK, bool SR, bool MT, int EXT>
StepFn pick_step(bool diag, bool delta) {
  if (diag)
    return delta ? decode_step_kernel<DK, true, true, SR, MT, EXT>
                 : decode_step_kernel<DK, true, false, SR, MT, EXT>;
  return delta ? decode_step_kernel<DK, false, true, SR, MT, EXT>
               : decode_step_kernel<DK, false, false, SR, MT, EXT>;
}
// One function per (key width, multi-token, extended) family, each defined in its own
// compilation of lores_inst.cu; kernel_for picks among them.
#define LORES_DECLARE_FAMILY(dk)                                   \
  StepFn step_kernels_##dk##_0_0(bool diag, bool delta, bool sr);  \
  StepFn step_kernels_##dk##_1_0(bool diag, bool delta, bool sr);  \
  StepFn step_kernels_##dk##_0_1(bool diag, bool delta, bool sr);  \
  StepFn step_kernels_##dk##_1_1(bool diag, bool delta, bool sr);  \
  StepFn step_kernels_##dk##_0_2(bool diag, bool delta, bool sr);  \
  StepFn step_kernels_##dk##_1_2(bool diag, bool delta, bool sr);  \
  StepFn step_kernels_##dk##_0_3(bool diag, bool delta, bool sr);  \
  StepFn step_kernels_##dk##_1_3(bool diag, bool delta, bool sr);  \
  StepFn step_kernels_##dk##_0_4(bool diag, bool delta, bool sr);  \
  StepFn step_kernels_##dk##_1_4(bool diag, bool delta, bool sr);
LORES_DECLARE_FAMILY(16)
LORES_DECLARE_FAMILY(32)
LORES_DECLARE_FAMILY(64)
LORES_DECLARE_FAMILY(128)
LORES_DECLARE_FAMILY(256)
#undef LORES_DECLARE_FAMILY

}  // namespace lores
