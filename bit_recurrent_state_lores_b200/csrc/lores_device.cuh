// lores_device.cuh -- device building blocks of the LoReS decode step (sm_100a).
//
// Arithmetic of one state row, shared by the decode kernel and the state loader.
// The element order and every fp32 rounding follow the state format definition:
//   entry of S_{t-1} diag(alpha):   c_ij * (s_ig * alpha_j)
//   u_i = (S'k)_i:                  per 16-column block, four fma chains (half h, column
//                                   parity p: columns 8h + p + 2m), summed as
//                                   (c00 + c10) + (c01 + c11); block sums combined
//                                   pairwise, nearest partner first (distance 1, 2, ...)
//   w_i = beta (v_i - u_i)  [delta] or beta v_i;   x_ij = fma(w_i, k_j, S'_ij)
//   requantize per group:           m = max|x|; y = Newton reciprocal of m; inv = r * y;
//                                   s = m * fl(1/r); t = fma(x, inv, 49152 + d/256);
//                                   code = floor(t - 49152)
// ("Quantizing Recurrent Language Models Is Easier Than You Think": General recurrence
// form; Key properties item 3; Proposition 1; Proposition 3.)
#pragma once
#include <cstdint>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

namespace lores {

constexpr int kThreads = 128;          // 4 warps per CTA
constexpr int kWarps = kThreads / 32;
constexpr int kStages = 2;             // smem ring depth per CTA
constexpr unsigned kFull = 0xFFFFFFFFu;

// Flag bits of the handle's sticky device word.
constexpr unsigned kFlagNonFinite = 1u;
constexpr unsigned kFlagTimeout = 2u;
// Index-checked build only: an access fell outside the buffer it belongs to (bit 8 + the
// buffer's RangeId says which; kRgShared: a bulk copy outside the dynamic shared memory)
constexpr unsigned kFlagIndex = 4u;

// Bounded waits: a wait on an mbarrier gives up after the launch's limit in nanoseconds of
// GPU time (%globaltimer; kWaitNs unless a test sets a shorter one), and after kMaxPolls
// polls in any case.
constexpr unsigned kMaxPolls = 1u << 24;
constexpr unsigned long long kWaitNs = 1000000000ull;   // one second

// -------------------------------------------------------------------------------------
// random bits: tile keys from the MurmurHash3 32-bit finalizer (Appleby), dither words
// from multiply-fold rounds of a 16-column block's counter
// -------------------------------------------------------------------------------------
__device__ __forceinline__ uint32_t fmix32(uint32_t h) {
  h ^= h >> 16;
  h *= 0x85EBCA6Bu;
  h ^= h >> 13;
  h *= 0xC2B2AE35u;
  h ^= h >> 16;
  return h;
}

__device__ __forceinline__ uint32_t tile_key(uint32_t step_key, uint32_t tile_index) {
  return fmix32(step_key + 0x85EBCA77u * (tile_index + 1u));
}

// Multiply-fold: low and high halves of the 64-bit product, XORed (one wide multiply
// and one XOR).
__device__ __forceinline__ uint32_t mulfold(uint32_t a, uint32_t b) {
  const unsigned long long p = (unsigned long long)a * b;
  return (uint32_t)p ^ (uint32_t)(p >> 32);
}
// Dither of a 16-column block of a row: its counter c (tile key + golden * (4 block +
// 1), block = row d_k/16 + column/16) is folded once; word q (columns 4q .. 4q + 3 of
// the block, one byte each) folds that again with multiplier q.
__device__ __forceinline__ uint32_t dither_mul(int q) {
  return q == 0 ? 0x846CA68Bu : (q == 1 ? 0xCC9E2D51u : (q == 2 ? 0x1B873593u : 0xE6546B65u));
}
__device__ __forceinline__ uint32_t dither_block_key(uint32_t c) { return mulfold(c, 0x7FEB352Du); }
__device__ __forceinline__ uint32_t dither_word(uint32_t bkey, int q) { return mulfold(bkey, dither_mul(q)); }

// max(m, |x|) that propagates NaN (PTX max.NaN), so a group max is non-finite
// exactly when some entry is.
__device__ __forceinline__ float max_abs_nan(float m, float x) {
  float r;
  asm("max.NaN.f32 %0, %1, %2;" : "=f"(r) : "f"(m), "f"(fabsf(x)));
  return r;
}
__device__ __forceinline__ float max_nan(float a, float b) {
  float r;
  asm("max.NaN.f32 %0, %1, %2;" : "=f"(r) : "f"(a), "f"(b));
  return r;
}

// -------------------------------------------------------------------------------------
// mbarrier + bulk async copy (TMA, non-tensor form; no multicast)
// -------------------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void mbar_init(uint64_t *bar, unsigned count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
               : "memory");
}
__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void fence_proxy_async() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint64_t *bar, unsigned bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, unsigned parity) {
  unsigned ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
// GPU time in nanoseconds.
__device__ __forceinline__ unsigned long long global_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
// Bounded wait; returns false if the phase did not complete within limit_ns nanoseconds
// (the clock is read every 32 polls) or kMaxPolls polls.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t *bar, unsigned parity,
                                                  unsigned long long limit_ns) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = global_ns();
  for (unsigned n = 0; n < kMaxPolls; n += 32) {
#pragma unroll 1
    for (int i = 0; i < 32; ++i)
      if (mbar_try_wait(bar, parity)) return true;
    if (global_ns() - t0 > limit_ns) return false;
  }
  return false;
}
// global -> shared bulk copy completing on `bar`; dst, src 16-byte aligned, bytes % 16 == 0.
__device__ __forceinline__ void bulk_g2s(void *dst, const void *src, unsigned bytes,
                                         uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
          "r"(smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// -------------------------------------------------------------------------------------
// index-checked build (LORES_INDEX_CHECKS): every global access of the decode, loader and
// dequantizer kernels names the buffer it belongs to and its byte count; the access runs
// only if it lies inside that buffer's extent as the host declared it for the launch.
// Otherwise the kernel raises kFlagIndex and the buffer's bit and skips the access (a
// skipped bulk copy leaves its barrier short, so the wait runs out and TIMEOUT is raised
// too).  In the ordinary build LORES_IN is the constant true and costs nothing.
// -------------------------------------------------------------------------------------
enum RangeId : int {
  kRgCodes, kRgScales, kRgQ, kRgK, kRgV, kRgAlpha, kRgBeta, kRgO, kRgS, kRgCount,
  kRgShared = kRgCount
};
struct Ranges {
  const void *base[kRgCount];
  unsigned long long bytes[kRgCount];
};

#ifdef LORES_INDEX_CHECKS
__device__ __forceinline__ bool range_ok(const Ranges &r, int id, const void *ptr,
                                         unsigned long long bytes, unsigned *flag) {
  const unsigned long long lo = reinterpret_cast<unsigned long long>(r.base[id]);
  const unsigned long long a = reinterpret_cast<unsigned long long>(ptr);
  if (a >= lo && a - lo <= r.bytes[id] && bytes <= r.bytes[id] - (a - lo)) return true;
  atomicOr(flag, kFlagIndex | (256u << id));
  return false;
}

// A bulk copy's destination [dst, dst + bytes) inside the launch's dynamic shared memory.
extern __shared__ __align__(16) uint8_t lores_dynamic_smem[];
__device__ __forceinline__ bool smem_range_ok(const void *dst, unsigned bytes, unsigned *flag) {
  unsigned size;
  asm("mov.u32 %0, %%dynamic_smem_size;" : "=r"(size));
  const unsigned lo = smem_u32(lores_dynamic_smem), a = smem_u32(dst);
  if (a >= lo && a - lo <= size && bytes <= size - (a - lo)) return true;
  atomicOr(flag, kFlagIndex | (256u << kRgShared));
  return false;
}

#define LORES_IN(p, id, ptr, bytes) ::lores::range_ok((p).rg, (id), (ptr), (bytes), (p).flag)
#define LORES_IN_SMEM(p, dst, bytes) ::lores::smem_range_ok((dst), (bytes), (p).flag)
#define LORES_RANGES ::lores::Ranges rg;
#define LORES_LDG(p, id, ptr) (LORES_IN(p, id, ptr, 4) ? __ldg(ptr) : 0.0f)
#else
#define LORES_LDG(p, id, ptr) __ldg(ptr)
#define LORES_IN(p, id, ptr, bytes) true
#define LORES_IN_SMEM(p, dst, bytes) true
#define LORES_RANGES
#endif

// 16 code bytes at an address that is only 8-byte aligned (rows of per-channel
// precision heads: key groups of 8 and 16 bytes back to back), as two 8-byte accesses.
__device__ __forceinline__ uint4 ld16_a8(const uint8_t *p) {
  const uint2 a = *reinterpret_cast<const uint2 *>(p);
  const uint2 b = *reinterpret_cast<const uint2 *>(p + 8);
  return make_uint4(a.x, a.y, b.x, b.y);
}
__device__ __forceinline__ void st16_a8(uint8_t *p, uint4 w) {
  *reinterpret_cast<uint2 *>(p) = make_uint2(w.x, w.y);
  *reinterpret_cast<uint2 *>(p + 8) = make_uint2(w.z, w.w);
}

// -------------------------------------------------------------------------------------
// code <-> float
// -------------------------------------------------------------------------------------
// Two fp16 halves of a word, each widened to fp32 and added to `bias` in one
// mixed-precision add (fp16 operand, fp32 operand and result, round to nearest).
__device__ __forceinline__ void halves_plus(uint32_t w, float bias, float &lo, float &hi) {
  asm("{\n\t.reg .f16 l, h;\n\t"
      "mov.b32 {l, h}, %2;\n\t"
      "add.rn.f32.f16 %0, l, %3;\n\t"
      "add.rn.f32.f16 %1, h, %3;\n\t}"
      : "=f"(lo), "=f"(hi)
      : "r"(w), "f"(bias));
}

// Bytes -> exact floats: a byte b dropped into the low mantissa byte of 2^23 (bits
// 0x4B0000bb) is the float 2^23 + b, exactly (the float spacing is 1 there); one packed
// add of -(2^23 + offset) then gives b - offset, exactly, for two bytes at once.
// byte_float(w, k): 2^23 + byte k of w.
__device__ __forceinline__ float byte_float(uint32_t w, int k) {
  return __uint_as_float(__byte_perm(w, 0x4B000000u, 0x7540u | (uint32_t)k));
}
// (byte k of a, byte k of b) - offset as a float pair
__device__ __forceinline__ float2 bytes_minus(uint32_t a, uint32_t b, int k, float2 off) {
  return __fadd2_rn(make_float2(byte_float(a, k), byte_float(b, k)), off);
}
// (byte k, byte k + 1 of w) - offset
__device__ __forceinline__ float2 byte_pair_minus(uint32_t w, int k, float2 off) {
  return __fadd2_rn(make_float2(byte_float(w, k), byte_float(w, k + 1)), off);
}
__device__ __forceinline__ float2 dup2(float v) { return make_float2(v, v); }
// -(2^23 + offset): the packed addend that turns 2^23 + b into b - offset
__device__ __forceinline__ float2 byte_bias(int offset) { return dup2(-(8388608.0f + (float)offset)); }

// 16 int8 codes (two's complement) -> exact floats: bias to offset binary (b = code +
// 128), then b - 128.
__device__ __forceinline__ void unpack_i8(const uint4 &cw, float (&c)[16]) {
  const uint32_t w[4] = {cw.x ^ 0x80808080u, cw.y ^ 0x80808080u, cw.z ^ 0x80808080u,
                         cw.w ^ 0x80808080u};
  const float2 off = byte_bias(128);
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const float2 lo = byte_pair_minus(w[q], 0, off), hi = byte_pair_minus(w[q], 2, off);
    c[4 * q] = lo.x; c[4 * q + 1] = lo.y; c[4 * q + 2] = hi.x; c[4 * q + 3] = hi.y;
  }
}
// 16 int4 codes (two's complement nibbles, even column low) -> exact floats: nibbles to
// offset-binary bytes (even columns in one word, odd in another), then b - 8.
__device__ __forceinline__ void unpack_i4(const uint2 &cw, float (&c)[16]) {
  const uint32_t w[2] = {cw.x, cw.y};
  const float2 off = byte_bias(8);
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const uint32_t ev = (w[h] & 0x0F0F0F0Fu) ^ 0x08080808u;          // columns 0, 2, 4, 6
    const uint32_t od = ((w[h] >> 4) & 0x0F0F0F0Fu) ^ 0x08080808u;   // columns 1, 3, 5, 7
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float2 e = bytes_minus(ev, od, k, off);
      c[8 * h + 2 * k] = e.x;
      c[8 * h + 2 * k + 1] = e.y;
    }
  }
}
// Paired forms: element pair e of a lane holds its columns (2e, 2e + 1), so packed
// fp32x2 instructions (two independent fp32 operations, each rounded to nearest) work
// on natural neighbours.
__device__ __forceinline__ void unpack_i8_2(const uint4 &cw, float2 (&c)[8]) {
  const uint32_t w[4] = {cw.x ^ 0x80808080u, cw.y ^ 0x80808080u, cw.z ^ 0x80808080u,
                         cw.w ^ 0x80808080u};
  const float2 off = byte_bias(128);
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    c[2 * q] = byte_pair_minus(w[q], 0, off);
    c[2 * q + 1] = byte_pair_minus(w[q], 2, off);
  }
}
// int4: column 2k is the low nibble of byte k, column 2k + 1 its high nibble.
__device__ __forceinline__ void unpack_i4_2(const uint2 &cw, float2 (&c)[8]) {
  const uint32_t w[2] = {cw.x, cw.y};
  const float2 off = byte_bias(8);
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const uint32_t ev = (w[h] & 0x0F0F0F0Fu) ^ 0x08080808u;          // columns 0, 2, 4, 6
    const uint32_t od = ((w[h] >> 4) & 0x0F0F0F0Fu) ^ 0x08080808u;   // columns 1, 3, 5, 7
#pragma unroll
    for (int k = 0; k < 4; ++k) c[4 * h + k] = bytes_minus(ev, od, k, off);
  }
}

// Offset-binary bytes (code + 128) of a lane's 16 columns, 4 columns per word in
// column order -> exact floats in column pairs (the int8 path after its bias flip).
__device__ __forceinline__ void unpack_ob_2(const uint32_t (&ob)[4], float2 (&c)[8]) {
  const float2 off = byte_bias(128);
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    c[2 * q] = byte_pair_minus(ob[q], 0, off);
    c[2 * q + 1] = byte_pair_minus(ob[q], 2, off);
  }
}
// 16 int4 codes -> offset-binary bytes (code + 128): nibble n -> (n ^ 8) + 120, no carry
// between bytes ((n ^ 8) <= 15), then even and odd columns interleaved into column order.
__device__ __forceinline__ void widen_i4_ob(const uint2 &cw, uint32_t (&ob)[4]) {
  const uint32_t w[2] = {cw.x, cw.y};
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const uint32_t ev = ((w[h] & 0x0F0F0F0Fu) ^ 0x08080808u) + 0x78787878u;
    const uint32_t od = (((w[h] >> 4) & 0x0F0F0F0Fu) ^ 0x08080808u) + 0x78787878u;
    ob[2 * h] = __byte_perm(ev, od, 0x5140u);       // columns 8h + 0..3
    ob[2 * h + 1] = __byte_perm(ev, od, 0x7362u);   // columns 8h + 4..7
  }
}
// Two's complement code bytes of 16 columns (|code| <= 7) -> int4 nibbles, even column low.
__device__ __forceinline__ uint2 compact_i4(const uint4 &b) {
  const uint32_t w[4] = {b.x, b.y, b.z, b.w};
  uint32_t out[2];
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const uint32_t e = __byte_perm(w[2 * h], w[2 * h + 1], 0x6420u);   // columns 0, 2, 4, 6
    const uint32_t o = __byte_perm(w[2 * h], w[2 * h + 1], 0x7531u);   // columns 1, 3, 5, 7
    out[h] = (e & 0x0F0F0F0Fu) | ((o << 4) & 0xF0F0F0F0u);
  }
  return make_uint2(out[0], out[1]);
}

// t holds 49152 + code + frac in fp32: its byte 1 is the code (two's complement).
__device__ __forceinline__ uint4 pack_i8(const uint32_t (&t)[16]) {
  uint32_t w[4];
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const uint32_t lo = __byte_perm(t[4 * q], t[4 * q + 1], 0x0051u);
    const uint32_t hi = __byte_perm(t[4 * q + 2], t[4 * q + 3], 0x0051u);
    w[q] = __byte_perm(lo, hi, 0x5410u);
  }
  return make_uint4(w[0], w[1], w[2], w[3]);
}
__device__ __forceinline__ uint2 pack_i4(const uint32_t (&t)[16]) {
  uint32_t m[8];
#pragma unroll
  for (int p = 0; p < 8; ++p)
    m[p] = (t[2 * p] & 0x0F00u) | ((t[2 * p + 1] << 4) & 0xF000u);   // byte 1 = (odd<<4)|even
  uint32_t w[2];
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const uint32_t lo = __byte_perm(m[4 * h], m[4 * h + 1], 0x0051u);
    const uint32_t hi = __byte_perm(m[4 * h + 2], m[4 * h + 3], 0x0051u);
    w[h] = __byte_perm(lo, hi, 0x5410u);
  }
  return make_uint2(w[0], w[1]);
}

// Dense 5- to 7-bit codes (B = 5, 6, 7): offset binary u = c + 2^(B-1) split into a 4-bit
// plane (the int4 nibble layout), a 2-bit plane (B >= 6) and a 1-bit plane (B odd).  A
// lane's 16 columns own 8 nibble bytes, one 2-bit word and one 16-bit 1-bit word:
//   2-bit word, byte p: column 8+2p in bits 0-1, 9+2p in 2-3, 2p in 4-5, 2p+1 in 6-7;
//   1-bit word: columns 0,2,4,6 in bits 0-3, 1,3,5,7 in 4-7, 8..14 even in 8-11, odd in 12-15.
// E0/O0/E1/O1 below are the offset-binary bytes of the even/odd columns of the two halves.
struct DenseLane {
  uint32_t nib0, nib1, p2, p1;
};

// Bit `s` of each byte of w, gathered into bits 0-3 (byte p -> bit p).
template <int S>
__device__ __forceinline__ uint32_t gather_bit4(uint32_t w) {
  return (((w >> S) & 0x01010101u) * 0x01020408u) >> 24;
}
// Bits 0-3 of q spread to bit S of bytes 0-3 (bit p -> byte p).
template <int S>
__device__ __forceinline__ uint32_t spread_bit4(uint32_t q) {
  return (((q & 0xFu) * 0x00204081u) & 0x01010101u) << S;
}

// t[e] = 49152 + u_e + fraction (byte 1 of t is u).
template <int B>
__device__ __forceinline__ DenseLane pack_dense(const uint32_t (&t)[16]) {
  auto gather = [&](int a) {                 // byte 1 of t[a], t[a+2], t[a+4], t[a+6]
    const uint32_t lo = __byte_perm(t[a], t[a + 2], 0x0051u);
    const uint32_t hi = __byte_perm(t[a + 4], t[a + 6], 0x0051u);
    return __byte_perm(lo, hi, 0x5410u);
  };
  const uint32_t E0 = gather(0), O0 = gather(1), E1 = gather(8), O1 = gather(9);
  DenseLane d;
  d.nib0 = (E0 & 0x0F0F0F0Fu) | ((O0 << 4) & 0xF0F0F0F0u);
  d.nib1 = (E1 & 0x0F0F0F0Fu) | ((O1 << 4) & 0xF0F0F0F0u);
  d.p2 = 0u;
  d.p1 = 0u;
  if (B >= 6) {
    const uint32_t m = 0x30303030u;
    d.p2 = (E0 & m) | ((O0 & m) << 2) | ((E1 & m) >> 4) | ((O1 & m) >> 2);
  }
  if (B & 1)
    d.p1 = gather_bit4<B - 1>(E0) | (gather_bit4<B - 1>(O0) << 4) |
           (gather_bit4<B - 1>(E1) << 8) | (gather_bit4<B - 1>(O1) << 12);
  return d;
}

// 16 dense codes -> exact floats in column pairs: rebuild the offset-binary bytes u
// (even columns in E, odd in O), drop them into fp16 pairs (1024 + u: the fp16 spacing is
// 1 there) and add -(1024 + 2^(B-1)) in fp32.  (The bit-plane path is short of ALU
// slots, so this route, which puts the conversion on the FMA pipe, suits it better than
// the byte-into-2^23 route of the other paths.)
template <int B>
__device__ __forceinline__ void unpack_dense(const DenseLane &d, float2 (&c)[8]) {
  uint32_t E0 = d.nib0 & 0x0F0F0F0Fu, O0 = (d.nib0 >> 4) & 0x0F0F0F0Fu;
  uint32_t E1 = d.nib1 & 0x0F0F0F0Fu, O1 = (d.nib1 >> 4) & 0x0F0F0F0Fu;
  if (B >= 6) {
    const uint32_t m = 0x30303030u;
    E0 |= d.p2 & m;
    O0 |= (d.p2 >> 2) & m;
    E1 |= (d.p2 << 4) & m;
    O1 |= (d.p2 << 2) & m;
  }
  if (B & 1) {
    E0 |= spread_bit4<B - 1>(d.p1);
    O0 |= spread_bit4<B - 1>(d.p1 >> 4);
    E1 |= spread_bit4<B - 1>(d.p1 >> 8);
    O1 |= spread_bit4<B - 1>(d.p1 >> 12);
  }
  constexpr float bias = -(1024.0f + (float)(1 << (B - 1)));
  const uint32_t x[4] = {__byte_perm(E0, O0, 0x5140u), __byte_perm(E0, O0, 0x7362u),
                         __byte_perm(E1, O1, 0x5140u), __byte_perm(E1, O1, 0x7362u)};
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    halves_plus(__byte_perm(x[q], 0x64646464u, 0x5140u), bias, c[2 * q].x, c[2 * q].y);
    halves_plus(__byte_perm(x[q], 0x64646464u, 0x7362u), bias, c[2 * q + 1].x, c[2 * q + 1].y);
  }
}

// Byte offsets of a lane's dense parts inside a row of d_k columns (lane = 16-column block).
__host__ __device__ constexpr int dense_p2_off(int dk, int lb) { return dk / 2 + 4 * lb; }
__host__ __device__ constexpr int dense_p1_off(int dk, int b, int lb) {
  return dk / 2 + (b >= 6 ? dk / 4 : 0) + 2 * lb;
}
// Load / store a lane's dense parts from a row (8-, 4- and 2-byte aligned accesses).
template <int B>
__device__ __forceinline__ DenseLane ld_dense(const uint8_t *row, int dk, int lb) {
  DenseLane d;
  const uint2 n = *reinterpret_cast<const uint2 *>(row + 8 * lb);
  d.nib0 = n.x;
  d.nib1 = n.y;
  d.p2 = B >= 6 ? *reinterpret_cast<const uint32_t *>(row + dense_p2_off(dk, lb)) : 0u;
  d.p1 = (B & 1) ? *reinterpret_cast<const uint16_t *>(row + dense_p1_off(dk, B, lb)) : 0u;
  return d;
}
template <int B>
__device__ __forceinline__ void st_dense(uint8_t *row, int dk, int lb, const DenseLane &d) {
  *reinterpret_cast<uint2 *>(row + 8 * lb) = make_uint2(d.nib0, d.nib1);
  if (B >= 6) *reinterpret_cast<uint32_t *>(row + dense_p2_off(dk, lb)) = d.p2;
  if (B & 1) *reinterpret_cast<uint16_t *>(row + dense_p1_off(dk, B, lb)) = (uint16_t)d.p1;
}

// -------------------------------------------------------------------------------------
// reductions over the lane's 16 entries
// -------------------------------------------------------------------------------------
// sum_e a_e b_e over the lane's 16 columns in the fixed order: four fma chains from zero,
// chain (h, p) over columns 8h + p + 2m, m = 0..3 ascending (h: half of the 16, p: column
// parity); the lane's sum is (chain(0,0) + chain(1,0)) + (chain(0,1) + chain(1,1)).
// Paired form: chains (h, 0) and (h, 1) run side by side in one packed fma.
__device__ __forceinline__ float dot16_p(const float2 (&a)[8], const float2 (&b)[8]) {
  float2 lo = make_float2(0.0f, 0.0f), hi = make_float2(0.0f, 0.0f);
#pragma unroll
  for (int e = 0; e < 4; ++e) lo = __ffma2_rn(a[e], b[e], lo);
#pragma unroll
  for (int e = 4; e < 8; ++e) hi = __ffma2_rn(a[e], b[e], hi);
  const float2 s = __fadd2_rn(lo, hi);
  return __fadd_rn(s.x, s.y);
}
// The same order with scalar operations.
__device__ __forceinline__ float dot16_b(const float (&a)[16], const float (&b)[16]) {
  float ch[2][2];
#pragma unroll
  for (int h = 0; h < 2; ++h)
#pragma unroll
    for (int p = 0; p < 2; ++p) {
      float acc = 0.0f;
#pragma unroll
      for (int m = 0; m < 4; ++m) acc = __fmaf_rn(a[8 * h + p + 2 * m], b[8 * h + p + 2 * m], acc);
      ch[h][p] = acc;
    }
  return __fadd_rn(__fadd_rn(ch[0][0], ch[1][0]), __fadd_rn(ch[0][1], ch[1][1]));
}

// Newton-Raphson reciprocal of m in [2^-100, 2^100]: seed by reflecting the exponent
// field (bits 0x7F000000 - bits(m), exact for powers of two, within 12.5% otherwise),
// then three steps y <- y + y (1 - m y); relative error < 2^-21.
__device__ __forceinline__ float recip_nr(float m) {
  float y = __uint_as_float(0x7F000000u - __float_as_uint(m));
#pragma unroll
  for (int it = 0; it < 3; ++it) {
    const float e = __fmaf_rn(-m, y, 1.0f);
    y = __fmaf_rn(y, e, y);
  }
  return y;
}

// -------------------------------------------------------------------------------------
// requantize one lane's 16 entries of a value row
// -------------------------------------------------------------------------------------
// Dither words of one 16-column block: cbase = tile key + golden * (n0 + 1), n0 the
// quad index of the block's first column (a multiple of 4).
__device__ __forceinline__ void dither_words(uint32_t cbase, uint32_t (&h)[4]) {
  const uint32_t bk = dither_block_key(cbase);
#pragma unroll
  for (int q = 0; q < 4; ++q) h[q] = dither_word(bk, q);
}

// -------------------------------------------------------------------------------------
// exact projection u = S'k for integer codes with one scale per row
// -------------------------------------------------------------------------------------
// u_i = fl32(fl64(s_i U_i) 2^-E) with U_i = sum_j c_ij Y_j exact, Y_j = rint(alpha_j k_j
// 2^E) (ties to even), E = 29 - floor(log2 max_j |alpha_j k_j|) so |Y_j| <= 2^30 (all
// products zero: E = 0).  Y is kept as four balanced base-256 digits (Y = sum_i 256^i
// d_i, d_i in [-128, 127]) in digit planes: byte j of plane i is d_i of column j.

// Balanced base-256 digits of |Y| <= 2^30.
__device__ __forceinline__ void digits4(int Y, int (&d)[4]) {
  int r = Y;
#pragma unroll
  for (int i = 0; i < 3; ++i) {
    const int di = (int)(int8_t)(r & 0xFF);
    d[i] = di;
    r = (r - di) >> 8;
  }
  d[3] = r;
}
// floor(log2 |x|) of a nonzero finite double (every product of two floats is normal)
__device__ __forceinline__ int ilog2_d(double x) {
  return (int)((__double_as_longlong(x) >> 52) & 0x7FF) - 1023;
}
__device__ __forceinline__ double pow2_d(int e) {   // 2^e, |e| < 1023
  return __longlong_as_double((long long)(e + 1023) << 52);
}

// Digit planes of Y for y (k or q) under decay alpha (alpha_j, or the scalar alpha_s):
// the whole warp; lane l forms quads l and l + 32 (columns 4 quad .. 4 quad + 3).  plane
// points to nplanes_stride * 4 bytes per plane, plane i at plane + i * stride.  Returns
// 2^-E, or NaN if some alpha_j y_j is not finite.
template <int DK>
__device__ __forceinline__ double fixed_point_planes(const float *y, const float *alpha, bool diag,
                                                     float alpha_s, uint8_t *plane, int stride) {
  const int lane = threadIdx.x & 31;
  constexpr int NQ = DK / 4, QPL = (NQ + 31) / 32;
  double pr[QPL][4];
  int emax = -2000;
  bool fin = true;
#pragma unroll
  for (int qi = 0; qi < QPL; ++qi) {
    const int quad = lane + 32 * qi;
    const bool in = quad < NQ;
    const float4 y4 = in ? reinterpret_cast<const float4 *>(y)[quad] : make_float4(0, 0, 0, 0);
    const float4 a4 = (in && diag) ? reinterpret_cast<const float4 *>(alpha)[quad]
                                   : make_float4(alpha_s, alpha_s, alpha_s, alpha_s);
    pr[qi][0] = (double)a4.x * (double)y4.x;
    pr[qi][1] = (double)a4.y * (double)y4.y;
    pr[qi][2] = (double)a4.z * (double)y4.z;
    pr[qi][3] = (double)a4.w * (double)y4.w;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const double v = pr[qi][c];
      fin = fin && isfinite(v);
      if (v != 0.0 && isfinite(v)) emax = max(emax, ilog2_d(v));
    }
  }
#pragma unroll
  for (int st = 16; st >= 1; st >>= 1) emax = max(emax, __shfl_xor_sync(kFull, emax, st));
  fin = __all_sync(kFull, fin);
  const int E = emax == -2000 ? 0 : 29 - emax;
  const double up = pow2_d(E);
#pragma unroll
  for (int qi = 0; qi < QPL; ++qi) {
    const int quad = lane + 32 * qi;
    if (quad < NQ) {
      uint32_t w[4] = {0u, 0u, 0u, 0u};
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        int dg[4];
        digits4(fin ? __double2int_rn(pr[qi][c] * up) : 0, dg);
#pragma unroll
        for (int i = 0; i < 4; ++i) w[i] |= ((uint32_t)dg[i] & 0xFFu) << (8 * c);
      }
#pragma unroll
      for (int i = 0; i < 4; ++i) *reinterpret_cast<uint32_t *>(plane + i * stride + 4 * quad) = w[i];
    }
  }
  return fin ? pow2_d(-E) : __longlong_as_double(0x7FF8000000000000ll);
}

// The same as a real call, for the general kernel: it runs once per unit, and its
// registers must not add to that kernel's inner loop.
template <int DK>
__device__ __noinline__ double fixed_point_planes_call(const float *y, const float *alpha, bool diag,
                                                       float alpha_s, uint8_t *plane, int stride) {
  return fixed_point_planes<DK>(y, alpha, diag, alpha_s, plane, stride);
}

// sum_j c_j Y_j over 16 columns: c as 16 signed bytes (4 words, column order), Y from
// the four digit planes at the same 16 columns; exact.
__device__ __forceinline__ long long exact_dot16(const uint32_t (&c)[4], const uint8_t *plane,
                                                 int stride) {
  long long U = 0;
#pragma unroll
  for (int i = 3; i >= 0; --i) {
    const uint4 dw = *reinterpret_cast<const uint4 *>(plane + i * stride);
    int P = __dp4a((int)c[0], (int)dw.x, 0);
    P = __dp4a((int)c[1], (int)dw.y, P);
    P = __dp4a((int)c[2], (int)dw.z, P);
    P = __dp4a((int)c[3], (int)dw.w, P);
    U = U * 256 + (long long)P;
  }
  return U;
}
// One row's exact u (if DELTA) and S'q from its lanes' 16 codes each (LPR lanes per row,
// every lane of the warp taking part): integer sums over the lane's columns, summed over
// the row's lanes, then fl32(fl64(s U) 2^-E).  planes: digit planes of alpha k at 0 and
// alpha q at 4 stride, at the lane's first column.
template <int LPR, bool DELTA>
__device__ __forceinline__ void exact_row(const uint32_t (&c)[4], const uint8_t *planes, int stride,
                                          float s, double sxk, double sxq, float &u, float &sq) {
  long long Uk = DELTA ? exact_dot16(c, planes, stride) : 0ll;
  long long Uq = exact_dot16(c, planes + 4 * stride, stride);
#pragma unroll
  for (int st = 1; st < LPR; st <<= 1) {
    if (DELTA) Uk += __shfl_xor_sync(kFull, Uk, st);
    Uq += __shfl_xor_sync(kFull, Uq, st);
  }
  u = DELTA ? (float)(((double)s * (double)Uk) * sxk) : 0.0f;
  sq = (float)(((double)s * (double)Uq) * sxq);
}
// 16 int4 codes (nibbles, even column low) -> 16 signed bytes in column order
__device__ __forceinline__ void i4_to_s8(const uint2 &cw, uint32_t (&c)[4]) {
  const uint32_t w[2] = {cw.x, cw.y};
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const uint32_t ev = (w[h] & 0x0F0F0F0Fu) ^ 0x08080808u;          // code + 8, even columns
    const uint32_t od = ((w[h] >> 4) & 0x0F0F0F0Fu) ^ 0x08080808u;   // odd columns
    // (b + 0x78) ^ 0x80 maps b = code + 8 in 0..15 to the code as a signed byte, with no
    // carry between bytes (b + 0x78 <= 0x87)
    c[2 * h] = (__byte_perm(ev, od, 0x5140u) + 0x78787878u) ^ 0x80808080u;
    c[2 * h + 1] = (__byte_perm(ev, od, 0x7362u) + 0x78787878u) ^ 0x80808080u;
  }
}

// Largest |x| over one lane's 16 entries (NaN if any entry is NaN).
__device__ __forceinline__ float chunk_absmax(const float2 (&x)[8]) {
  float mq[4];
#pragma unroll
  for (int c = 0; c < 4; ++c)
    mq[c] = max_abs_nan(max_abs_nan(max_abs_nan(fabsf(x[2 * c].x), x[2 * c].y), x[2 * c + 1].x),
                        x[2 * c + 1].y);
  return max_nan(max_nan(mq[0], mq[1]), max_nan(mq[2], mq[3]));
}

// Group maximum over the lanes of the group: a level at or beyond the group width has
// shuffle distance 0 (the lane's own value).  Every lane of the warp must take part.
template <int LPR>
__device__ __forceinline__ float group_absmax(float m, int gd1, int gd2, int gd4, int gd8) {
  const int dist[4] = {gd1, gd2, gd4, gd8};
#pragma unroll
  for (int l = 0; (1 << l) < LPR; ++l) m = max_nan(m, __shfl_xor_sync(kFull, m, dist[l]));
  return m;
}

// Scale and inverse of a group with largest |x| = m; returns the group's "bad" verdict
// (an entry is inf, NaN or above 2^100).  Below 2^-100 the group is stored as zero.
__device__ __forceinline__ bool group_scale(float m, float r, float inv_r, float2 &inv, float &s) {
  const bool gbad = !(m <= 0x1p100f);
  const bool scaled = m >= 0x1p-100f && !gbad;
  const float y = recip_nr(scaled ? m : 1.0f);
  inv = dup2(scaled ? __fmul_rn(r, y) : 0.0f);
  s = scaled ? __fmul_rn(m, inv_r) : 0.0f;
  return gbad;
}

// Codes of a lane's 16 entries: t = fma(x, inv, 49152 + d/256) (d = byte j mod 4 of the
// quad's hash word; 128 for round to nearest), packed from byte 1 of t.  BITS is the
// storage: 8 (one byte per code, 5- to 8-bit codes; 4 words) or 4 (nibbles; 2 words).
// No cross-lane operation: lanes may take different widths.
template <int BITS, bool SR>
__device__ __forceinline__ void quantize16(const float2 (&x)[8], float2 inv, const uint32_t (&h)[4],
                                           uint32_t (&words)[4]) {
  uint32_t t[16];
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    const float2 g =
        SR ? make_float2(
                 __uint_as_float(__byte_perm(h[e >> 1], 0x47400000u, 0x7650u | ((2 * e) & 3))),
                 __uint_as_float(__byte_perm(h[e >> 1], 0x47400000u, 0x7650u | ((2 * e + 1) & 3))))
           : dup2(49152.5f);
    const float2 tt = __ffma2_rn(x[e], inv, g);
    t[2 * e] = __float_as_uint(tt.x);
    t[2 * e + 1] = __float_as_uint(tt.y);
  }
  if (BITS == 8) {
    const uint4 w = pack_i8(t);
    words[0] = w.x; words[1] = w.y; words[2] = w.z; words[3] = w.w;
  } else {
    const uint2 w = pack_i4(t);
    words[0] = w.x; words[1] = w.y; words[2] = 0u; words[3] = 0u;
  }
}

// Dense codes of a lane's 16 entries: t = fma(x, inv, 49152 + 2^(B-1) + d/256), so byte 1
// of t is the offset-binary u; then the planes.
template <int B, bool SR>
__device__ __forceinline__ DenseLane quantize16_dense(const float2 (&x)[8], float2 inv,
                                                      const uint32_t (&h)[4]) {
  constexpr uint32_t K = 0x47400000u | ((uint32_t)(1 << (B - 1)) << 8);
  uint32_t t[16];
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    const float2 g =
        SR ? make_float2(__uint_as_float(__byte_perm(h[e >> 1], K, 0x7650u | ((2 * e) & 3))),
                         __uint_as_float(__byte_perm(h[e >> 1], K, 0x7650u | ((2 * e + 1) & 3))))
           : dup2(__uint_as_float(K | 0x80u));
    const float2 tt = __ffma2_rn(x[e], inv, g);
    t[2 * e] = __float_as_uint(tt.x);
    t[2 * e + 1] = __float_as_uint(tt.y);
  }
  return pack_dense<B>(t);
}

// Requantize one lane's 16 entries of a value row (a scale group spans G/16 lanes):
// returns this lane's group verdict (true: an entry of the group is inf, NaN or above
// 2^100; the caller then zeroes the row).  r = 2^(b-1) - 1 and inv_r = fl(1/r).
template <int LPR, int BITS, bool SR>
__device__ __forceinline__ bool requantize16_nb(const float2 (&x)[8], float r, float inv_r,
                                                int gd1, int gd2, int gd4, int gd8,
                                                const uint32_t (&h)[4], uint32_t (&words)[4],
                                                float &s_out) {
  const float m = group_absmax<LPR>(chunk_absmax(x), gd1, gd2, gd4, gd8);
  float2 inv;
  const bool gbad = group_scale(m, r, inv_r, inv, s_out);
  quantize16<BITS, SR>(x, inv, h, words);
  return gbad;
}

// Requantizer of the state loader: LPR lanes hold one row (16 consecutive columns
// each); lpg = G/16 lanes share a group.  Returns the row's "non-finite" verdict (same
// on all lanes of the row): a row with an entry that is inf, NaN or above 2^100 is
// stored as zero.  Writes the lane's packed codes into `words` (8-bit storage: 4 words,
// int4: 2 words) and the lane's group scale into `s_out`.  `bits` may differ between
// lanes of one warp; every lane of the warp must call this function together (it
// shuffles and votes across the warp).
template <int LPR>
__device__ __forceinline__ bool requantize16(const float (&x)[16], int bits, int lpg, int lane,
                                             uint32_t tkey, uint32_t n0, int stochastic,
                                             uint32_t (&words)[4], float &s_out, int store = 0) {
  // store 5..7: dense planes (words = nibble word 0, nibble word 1, 2-bit word, 1-bit word)
  const bool dense = store >= 5 && store <= 7;
  const uint32_t kbase = 0x47400000u | (dense ? (1u << (bits - 1)) << 8 : 0u);
  const float r = (float)((1 << (bits - 1)) - 1);        // 2^(b-1) - 1
  const float inv_r = __fdiv_rn(1.0f, r);                 // fl(1/r)
  float mq[4];
#pragma unroll
  for (int c = 0; c < 4; ++c)
    mq[c] = max_abs_nan(max_abs_nan(max_abs_nan(fabsf(x[4 * c]), x[4 * c + 1]), x[4 * c + 2]),
                        x[4 * c + 3]);
  float m = max_nan(max_nan(mq[0], mq[1]), max_nan(mq[2], mq[3]));
  // group max over the lpg lanes of the group: the levels are fixed at compile time
  // (log2 LPR); levels at or beyond the group width keep the lane's own value.
#pragma unroll
  for (int st = 1; st < LPR; st <<= 1) {
    const float mo = __shfl_xor_sync(kFull, m, st);
    m = (st < lpg) ? max_nan(m, mo) : m;
  }
  const bool gbad = !(m <= 0x1p100f);                    // inf, NaN or overflow
  const bool any_bad = __any_sync(kFull, gbad);
  bool row_bad = false;
  if (any_bad) {
    const unsigned bal = __ballot_sync(kFull, gbad);
    const int riw = lane / LPR;
    const unsigned rowmask = (LPR == 32 ? kFull : ((1u << LPR) - 1u)) << (riw * LPR);
    row_bad = (bal & rowmask) != 0u;
  }
  const bool scaled = m >= 0x1p-100f && !gbad;           // below 2^-100: zero group
  const float y = recip_nr(scaled ? m : 1.0f);
  const float inv = scaled ? __fmul_rn(r, y) : 0.0f;
  float s = scaled ? __fmul_rn(m, inv_r) : 0.0f;

  uint32_t t[16];
  if (stochastic) {
    uint32_t h[4];
    dither_words(tkey + 0x9E3779B9u * (n0 + 1u), h);
#pragma unroll
    for (int e = 0; e < 16; ++e) {
      const float g = __uint_as_float(__byte_perm(h[e >> 2], kbase, 0x7650u | (e & 3)));
      t[e] = __float_as_uint(__fmaf_rn(x[e], inv, g));
    }
  } else {
    const float g = __uint_as_float(kbase | 0x80u);
#pragma unroll
    for (int e = 0; e < 16; ++e) t[e] = __float_as_uint(__fmaf_rn(x[e], inv, g));
  }
  if (dense) {
    const DenseLane d = store == 5 ? pack_dense<5>(t) : (store == 6 ? pack_dense<6>(t) : pack_dense<7>(t));
    words[0] = d.nib0; words[1] = d.nib1; words[2] = d.p2; words[3] = d.p1;
  } else if (bits != 4) {
    const uint4 w = pack_i8(t);
    words[0] = w.x; words[1] = w.y; words[2] = w.z; words[3] = w.w;
  } else {
    const uint2 w = pack_i4(t);
    words[0] = w.x; words[1] = w.y; words[2] = 0u; words[3] = 0u;
  }
  if (any_bad && row_bad) {
    words[0] = words[1] = words[2] = words[3] = 0u;
    s = 0.0f;
  }
  s_out = s;
  return row_bad;
}

}  // namespace lores
