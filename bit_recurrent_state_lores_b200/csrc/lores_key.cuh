// lores_key.cuh -- the decode step with key-axis scale groups (sm_100a): one fp32 scale
// per key column of a (sequence, head) tile, s_j = max_i |x_ij| / r, the grouping that
// "Quantizing Recurrent Language Models Is Easier Than You Think" (summary page: Scale
// Grouping paragraph; Proposition 1's key-axis error formula) compares value-axis groups
// against.  The recurrence and the per-row arithmetic are the value-axis step's; only
// the scale group differs.
//
// The column maximum couples all rows of a tile, so one CTA handles one whole tile at a
// time: pass 1 updates every row (x = S' + w k^T), keeps w and the readout shares, and
// reduces per-column maxima; pass 2 recomputes x (the same fp32 operations) and writes
// codes with the column scale.  Columns with an inf/NaN/overflow entry are stored as
// zero and flagged; fp32 heads store x as in the value-axis path.  The grid is
// persistent: a CTA walks tiles blockIdx.x, blockIdx.x + gridDim.x, ... and, where two
// stages fit in shared memory, the bulk copies of its next tile land while the current
// one is computed.  The storage class (nibbles, bytes, fp32) and the rounding mode are
// template parameters, so the row loops carry no per-row format branches.
#pragma once
#include <cstdint>

#include "lores_step.cuh"

namespace lores {

struct KeyParams {
  uint8_t *codes;
  float *scales;                // [B][H][d_k]
  const float *q, *k, *v, *alpha, *beta;
  const float *S;               // load_state input [B][H][d_v][d_k], or null
  float *o;
  unsigned *flag;
  const int32_t *head_bits;
  const int64_t *head_off;
  long long seq_bytes;
  long long tiles;              // B * H
  int H, d_v;
  uint32_t step_key;
  uint64_t seed;
  const uint64_t *step_dev;     // step in device memory (CUDA-graph replay), or null
  int delta, diag, stochastic;
  unsigned long long wait_ns;   // bounded waits give up after this much GPU time
  // shared memory: stage s starts at stage0 + s * stage_bytes and holds the tile's codes,
  // scales, k, q, alpha, v at the sm_* offsets inside it; opart, ow, cm are absolute
  int stage0, stage_bytes, nstage;
  int sm_codes, sm_scales, sm_k, sm_q, sm_a, sm_v, sm_opart, sm_ow, sm_cm;
  LORES_RANGES                  // index-checked build: the extent of every buffer of the launch
};

using KeyFn = void (*)(const KeyParams);

// Scales and inverses of the tile's columns from the lanes' running maxima: reduce across
// the row groups of each warp, then across warps through shared memory; then one thread
// per column forms its maximum m, stores the column scale s = m fl(1/r) (0 below 2^-100 or
// for a bad column) to gscales, raises NONFINITE for a bad column (inf, NaN or above
// 2^100), and leaves in smcm[j] the inverse r y (y the Newton reciprocal of m), 0 for a
// tiny column, or a NaN marker for a bad one.  Every thread of the CTA calls this together.
template <int DK>
__device__ __forceinline__ void column_inverses(float (&cm)[16], float *smcm, float r, float inv_r,
                                                float *gscales, unsigned *flag, bool store = true) {
  constexpr int LPR = DK / 16;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int lir = lane % LPR, riw = lane / LPR;
#pragma unroll
  for (int st = LPR; st < 32; st <<= 1)
#pragma unroll
    for (int e = 0; e < 16; ++e) cm[e] = max_nan(cm[e], __shfl_xor_sync(kFull, cm[e], st));
  if (riw == 0)
#pragma unroll
    for (int e = 0; e < 16; ++e) smcm[warp * DK + lir * 16 + e] = cm[e];
  __syncthreads();
  for (int j = threadIdx.x; j < DK; j += kThreads) {
    float m = smcm[j];
    for (int w2 = 1; w2 < kWarps; ++w2) m = max_nan(m, smcm[w2 * DK + j]);
    const bool bad = !(m <= 0x1p100f);
    const bool scaled = !bad && m >= 0x1p-100f;
    if (store) gscales[j] = scaled ? __fmul_rn(m, inv_r) : 0.0f;
    if (bad) atomicOr(flag, kFlagNonFinite);
    smcm[j] = bad ? __uint_as_float(0x7FC00000u) : (scaled ? __fmul_rn(r, recip_nr(m)) : 0.0f);
  }
  __syncthreads();
}

// Bulk copies of tile t's codes, scales and vectors into one stage (one thread).
template <int DK>
__device__ __forceinline__ void issue_key_tile(const KeyParams &p, long long t, uint8_t *st,
                                               uint64_t *bar) {
  const int head = (int)(t % p.H);
  const long long b = t / p.H;
  const int bits = __ldg(p.head_bits + head);
  const unsigned cb = (unsigned)(p.d_v * row_bytes(DK, bits)), sb = bits == 32 ? 0u : DK * 4u;
  const unsigned vec = DK * 4, vb = (unsigned)(p.d_v * 4);
  mbar_expect_tx(bar, cb + sb + 2 * vec + vb + (p.diag ? vec : 0u));
  // (index-checked build: a copy outside its buffer or the stage is not issued)
  auto copy = [&](int off, int rid, const void *src, unsigned bytes) {
    (void)rid;
    if (LORES_IN(p, rid, src, bytes) && LORES_IN_SMEM(p, st + off, bytes)) bulk_g2s(st + off, src, bytes, bar);
  };
  copy(p.sm_codes, kRgCodes, p.codes + b * p.seq_bytes + __ldg(p.head_off + head), cb);
  if (sb) copy(p.sm_scales, kRgScales, p.scales + t * DK, sb);
  copy(p.sm_k, kRgK, p.k + t * DK, vec);
  copy(p.sm_q, kRgQ, p.q + t * DK, vec);
  copy(p.sm_v, kRgV, p.v + t * p.d_v, vb);
  if (p.diag) copy(p.sm_a, kRgAlpha, p.alpha + t * DK, vec);
}

// One tile: STORE is the storage class of the tile's head (4 nibbles, 8 one byte per
// code for 5..8 bits, 32 fp32), SR stochastic rounding, LOAD the state loader (x given).
// Every thread of the CTA calls this together.
template <int DK, int STORE, bool SR, bool LOAD>
__device__ __forceinline__ void key_tile(const KeyParams &p, long long tile, int bits,
                                         const uint8_t *st, float alpha_s, float beta,
                                         uint32_t skey, float *opart, float *ow, float *smcm) {
  constexpr int LPR = DK / 16, RPW = 32 / LPR;
  constexpr int RB = DK * STORE / 8;             // bytes per row
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int lir = lane % LPR, riw = lane / LPR, col0 = lir * 16;
  const int head = (int)(tile % p.H);
  const long long b = tile / p.H;
  uint8_t *gcodes = p.codes + b * p.seq_bytes + __ldg(p.head_off + head);
  const uint8_t *scodes = st + p.sm_codes;
  const float *sk = reinterpret_cast<const float *>(st + p.sm_k);
  const float *sq = reinterpret_cast<const float *>(st + p.sm_q);
  const float *sv = reinterpret_cast<const float *>(st + p.sm_v);

  // element pair e of a lane holds its columns (2e, 2e + 1)
  float2 kk[8], qq[8], aj[8];
  double kqd = 0.0;
  if (!LOAD) {
    const float2 *k2 = reinterpret_cast<const float2 *>(sk + col0);
    const float2 *q2 = reinterpret_cast<const float2 *>(sq + col0);
    const float2 *s2 = reinterpret_cast<const float2 *>(st + p.sm_scales) + lir * 8;
    const float2 *a2 = reinterpret_cast<const float2 *>(st + p.sm_a) + lir * 8;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      kk[e] = k2[e];
      qq[e] = q2[e];
      const float2 al = p.diag ? a2[e] : dup2(alpha_s);
      // entry (i, j) of S_{t-1} diag(alpha) is c_ij * (s_j * alpha_j)
      aj[e] = STORE == 32 ? al : __fmul2_rn(s2[e], al);
    }
    // k.q in double for the readout
    for (int j = lane; j < DK; j += 32) kqd = fma((double)sk[j], (double)sq[j], kqd);
#pragma unroll
    for (int o2 = 16; o2 >= 1; o2 >>= 1) kqd += __shfl_xor_sync(kFull, kqd, o2);
  }
  const uint32_t tkey = tile_key(skey, (uint32_t)tile);

  // S' = c (s alpha) of one row for this lane's 16 columns
  auto row_sp = [&](int lr, float2 (&sp)[8]) {
    if (STORE == 32) {
      const float2 *srow = reinterpret_cast<const float2 *>(scodes + (size_t)lr * RB) + lir * 8;
#pragma unroll
      for (int e = 0; e < 8; ++e) sp[e] = __fmul2_rn(srow[e], aj[e]);
    } else {
      float2 cf[8];
      if (STORE == 4)
        unpack_i4_2(*reinterpret_cast<const uint2 *>(scodes + (size_t)lr * RB + lir * 8), cf);
      else
        unpack_i8_2(*reinterpret_cast<const uint4 *>(scodes + (size_t)lr * RB + lir * 16), cf);
#pragma unroll
      for (int e = 0; e < 8; ++e) sp[e] = __fmul2_rn(cf[e], aj[e]);
    }
  };

  // ---- pass 1: update every row (or take x from S), column maxima ----------------------
  float cm[16];
#pragma unroll
  for (int e = 0; e < 16; ++e) cm[e] = 0.0f;
  bool bad32 = false;
  const int nbase = warp * RPW;
  for (int base = nbase; base < p.d_v; base += kWarps * RPW) {
    const int lr = base + riw;
    const bool active = lr < p.d_v;
    float2 x[8];
    if (LOAD) {
      if (!active) continue;
      const float2 *src = reinterpret_cast<const float2 *>(p.S + (tile * p.d_v + lr) * DK + col0);
      const bool in = LORES_IN(p, kRgS, src, 64);
#pragma unroll
      for (int e = 0; e < 8; ++e) x[e] = in ? src[e] : make_float2(0.0f, 0.0f);
    } else {
      // every lane of the warp takes the shuffles; only real rows keep w and the shares
      const int lrr = active ? lr : 0;
      float2 sp[8];
      row_sp(lrr, sp);
      float w;
      if (p.delta) {
        float u = dot16_p(sp, kk);
#pragma unroll
        for (int o2 = 1; o2 < LPR; o2 <<= 1) u = __fadd_rn(u, __shfl_xor_sync(kFull, u, o2));
        w = __fmul_rn(beta, __fsub_rn(sv[lrr], u));
      } else {
        w = __fmul_rn(beta, sv[lrr]);
      }
      const float opv = dot16_p(sp, qq);
      if (!active) continue;
      opart[lr * LPR + lir] = opv;
      if (lir == 0) ow[lr] = w;
      const float2 w2 = dup2(w);
#pragma unroll
      for (int e = 0; e < 8; ++e) x[e] = __ffma2_rn(w2, kk[e], sp[e]);
    }
    if (STORE == 32) {
      float4 *dst = reinterpret_cast<float4 *>(gcodes + (size_t)lr * RB) + lir * 4;
      if (LORES_IN(p, kRgCodes, dst, 64))
#pragma unroll
        for (int c = 0; c < 4; ++c)
          dst[c] = make_float4(x[2 * c].x, x[2 * c].y, x[2 * c + 1].x, x[2 * c + 1].y);
#pragma unroll
      for (int e = 0; e < 8; ++e) bad32 |= !isfinite(x[e].x) || !isfinite(x[e].y);
    } else {
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        cm[2 * e] = max_abs_nan(cm[2 * e], x[e].x);
        cm[2 * e + 1] = max_abs_nan(cm[2 * e + 1], x[e].y);
      }
    }
  }

  if (!LOAD) {
    // ---- readout of this warp's rows: o_i = the lane shares in lane order + w_i (k.q);
    // the shares and w were written by this warp in pass 1, so no CTA barrier is needed
    __syncwarp();
    const float kq = (float)kqd;
    float *go = p.o + tile * p.d_v;
    for (int k = lane;; k += 32) {
      const int r = (k / RPW) * (kWarps * RPW) + nbase + k % RPW;   // the warp's k-th row
      if (r >= p.d_v) break;
      float acc = 0.0f;
#pragma unroll
      for (int l = 0; l < LPR; ++l) acc = __fadd_rn(acc, opart[r * LPR + l]);
      if (LORES_IN(p, kRgO, go + r, 4)) go[r] = __fmaf_rn(ow[r], kq, acc);
    }
    __syncwarp();
  }
  if (STORE == 32) {
    if (__any_sync(kFull, bad32) && bad32) atomicOr(p.flag, kFlagNonFinite);
  } else {
    const float r = (float)((1 << (bits - 1)) - 1);
    const float inv_r = __fdiv_rn(1.0f, r);
    column_inverses<DK>(cm, smcm, r, inv_r, p.scales + tile * DK, p.flag,
                        LORES_IN(p, kRgScales, p.scales + tile * DK, DK * 4));
    float2 inv[8];
    unsigned badcols = 0;                        // bit e: column col0 + e is bad
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const float4 f = *reinterpret_cast<const float4 *>(smcm + col0 + 4 * c);
      const float fe[4] = {f.x, f.y, f.z, f.w};
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int e = 4 * c + u;
        const bool bad = fe[u] != fe[u];        // the NaN marker of a bad column
        const float ie = bad ? 0.0f : fe[u];
        if (e & 1) inv[e >> 1].y = ie; else inv[e >> 1].x = ie;
        badcols |= (bad ? 1u : 0u) << e;
      }
    }
    // masks that clear the codes of bad columns (bytes, or nibbles: column e of the
    // lane sits in word e/8, nibble e%8)
    uint32_t keep[4];
#pragma unroll
    for (int qd = 0; qd < 4; ++qd) {
      keep[qd] = 0;
      if (STORE == 8) {
#pragma unroll
        for (int e = 0; e < 4; ++e)
          keep[qd] |= ((badcols >> (4 * qd + e)) & 1u) ? 0u : (0xFFu << (8 * e));
      } else if (qd < 2) {
#pragma unroll
        for (int e = 0; e < 8; ++e)
          keep[qd] |= ((badcols >> (8 * qd + e)) & 1u) ? 0u : (0xFu << (4 * e));
      }
    }
    // ---- pass 2: x again (from the codes, or from S), codes ------------------------------
    for (int base = nbase; base < p.d_v; base += kWarps * RPW) {
      const int lr = base + riw;
      if (lr >= p.d_v) continue;
      float2 x[8];
      if (LOAD) {
        const float2 *src = reinterpret_cast<const float2 *>(p.S + (tile * p.d_v + lr) * DK + col0);
        const bool in = LORES_IN(p, kRgS, src, 64);
#pragma unroll
        for (int e = 0; e < 8; ++e) x[e] = in ? src[e] : make_float2(0.0f, 0.0f);
      } else {
        float2 sp[8];
        row_sp(lr, sp);
        const float2 w2 = dup2(ow[lr]);
#pragma unroll
        for (int e = 0; e < 8; ++e) x[e] = __ffma2_rn(w2, kk[e], sp[e]);
      }
      uint32_t h[4] = {0u, 0u, 0u, 0u};
      if (SR)
        dither_words(tkey + 0x9E3779B9u * ((uint32_t)lr * (uint32_t)(DK / 4) + (uint32_t)lir * 4u + 1u), h);
      uint32_t t[16];
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const float2 g =
            SR ? make_float2(
                     __uint_as_float(__byte_perm(h[e >> 1], 0x47400000u, 0x7650u | ((2 * e) & 3))),
                     __uint_as_float(__byte_perm(h[e >> 1], 0x47400000u, 0x7650u | ((2 * e + 1) & 3))))
               : dup2(49152.5f);
        const float2 tt = __ffma2_rn(x[e], inv[e], g);
        t[2 * e] = __float_as_uint(tt.x);
        t[2 * e + 1] = __float_as_uint(tt.y);
      }
      if (STORE == 4) {
        uint2 w = pack_i4(t);
        w.x &= keep[0];
        w.y &= keep[1];
        if (LORES_IN(p, kRgCodes, gcodes + (size_t)lr * RB + lir * 8, 8))
          *reinterpret_cast<uint2 *>(gcodes + (size_t)lr * RB + lir * 8) = w;
      } else {
        uint4 w = pack_i8(t);
        w.x &= keep[0]; w.y &= keep[1]; w.z &= keep[2]; w.w &= keep[3];
        if (LORES_IN(p, kRgCodes, gcodes + (size_t)lr * RB + lir * 16, 16))
          *reinterpret_cast<uint4 *>(gcodes + (size_t)lr * RB + lir * 16) = w;
      }
    }
  }
}

template <int DK, bool SR, bool LOAD>
__global__ void __launch_bounds__(kThreads) decode_step_key_kernel(const KeyParams p) {
  extern __shared__ __align__(128) uint8_t smem[];
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem);
  float *opart = reinterpret_cast<float *>(smem + p.sm_opart);
  float *ow = reinterpret_cast<float *>(smem + p.sm_ow);
  float *smcm = reinterpret_cast<float *>(smem + p.sm_cm);
  const uint32_t skey = p.step_dev ? step_key_dev(p.seed, *p.step_dev) : p.step_key;

  if (!LOAD && threadIdx.x == 0) {
    for (int s = 0; s < p.nstage; ++s) mbar_init(&bars[s], 1);
    fence_mbar_init();
    for (int s = 0; s < p.nstage; ++s) {
      const long long t = blockIdx.x + (long long)s * gridDim.x;
      if (t < p.tiles) issue_key_tile<DK>(p, t, smem + p.stage0 + s * p.stage_bytes, &bars[s]);
    }
  }
  __syncthreads();

  // the first tile's stage: every thread waits, then the CTA agrees it landed
  if (!LOAD && blockIdx.x < p.tiles) {
    const bool ok = mbar_wait_bounded(&bars[0], 0u, p.wait_ns);
    if (!__syncthreads_and(ok)) {
      if (threadIdx.x == 0) {
        atomicOr(p.flag, kFlagTimeout);
        // let every copy in flight land before the CTA exits
        for (int s2 = 0; s2 < p.nstage; ++s2)
          if (blockIdx.x + (long long)s2 * gridDim.x < p.tiles)
            (void)mbar_wait_bounded(&bars[s2], 0u, p.wait_ns);
      }
      return;
    }
  }

  int n = 0;
  for (long long tile = blockIdx.x; tile < p.tiles; tile += gridDim.x, ++n) {
    const int s = n % p.nstage;
    uint8_t *st = smem + p.stage0 + s * p.stage_bytes;
    const int bits = __ldg(p.head_bits + (int)(tile % p.H));
    const float alpha_s = (LOAD || p.diag) ? 1.0f : LORES_LDG(p, kRgAlpha, p.alpha + tile);
    const float beta = LOAD ? 0.0f : LORES_LDG(p, kRgBeta, p.beta + tile);
    if (bits == 32)
      key_tile<DK, 32, SR, LOAD>(p, tile, bits, st, alpha_s, beta, skey, opart, ow, smcm);
    else if (bits == 4)
      key_tile<DK, 4, SR, LOAD>(p, tile, bits, st, alpha_s, beta, skey, opart, ow, smcm);
    else
      key_tile<DK, 8, SR, LOAD>(p, tile, bits, st, alpha_s, beta, skey, opart, ow, smcm);
    if (LOAD) {
      __syncthreads();                         // the column maxima are reused next tile
      continue;
    }
    const long long tnext = tile + gridDim.x;
    const int snext = (n + 1) % p.nstage;
    const unsigned pnext = (unsigned)(((n + 1) / p.nstage) & 1);
    if (p.nstage == 1) {
      // one stage: every thread is done with it before it is refilled with the next tile
      __syncthreads();
      if (threadIdx.x == 0 && tnext < p.tiles) {
        fence_proxy_async();
        issue_key_tile<DK>(p, tnext, st, &bars[0]);
      }
    }
    // Wait for the next tile's stage; the barrier also says that every thread is done
    // with this tile's stage and column maxima, so (two stages) it can be refilled.
    const bool ok = tnext < p.tiles ? mbar_wait_bounded(&bars[snext], pnext, p.wait_ns) : true;
    if (!__syncthreads_and(ok)) {
      if (threadIdx.x == 0) {
        atomicOr(p.flag, kFlagTimeout);
        (void)mbar_wait_bounded(&bars[snext], pnext, p.wait_ns);   // the copy in flight lands first
      }
      return;
    }
    if (p.nstage == 2 && threadIdx.x == 0) {
      const long long tn = tile + 2LL * gridDim.x;
      if (tn < p.tiles) {
        fence_proxy_async();
        issue_key_tile<DK>(p, tn, st, &bars[s]);
      }
    }
  }
}

// One function per key width, defined in its own compilation of lores_inst.cu.
#define LORES_DECLARE_KEY(dk) KeyFn key_kernels_##dk(bool sr, bool load);
LORES_DECLARE_KEY(16)
LORES_DECLARE_KEY(32)
LORES_DECLARE_KEY(64)
LORES_DECLARE_KEY(128)
LORES_DECLARE_KEY(256)
#undef LORES_DECLARE_KEY

}  // namespace lores
