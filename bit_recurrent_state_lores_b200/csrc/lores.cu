// lores.cu -- LoReS quantized recurrent-state decode step: kernels and C ABI (sm_100a).
//
// One decode step of a linear-recurrence layer ("Quantizing Recurrent Language Models Is
// Easier Than You Think", summary page: General recurrence form; Key properties item 3;
// Proposition 1; Table 5 text; Proposition 3 / Table 6):
//   S_t = S_{t-1} diag(alpha_t) (I - delta beta_t k_t k_t^T) + beta_t v_t k_t^T,  o_t = S_t q_t
// with S_{t-1} dequantized from int8/int4 codes and per-(value row, key block) fp32
// scales, and S_t requantized with stochastic rounding, all in one pass over the state.
//
// This file: the C ABI (handles, unit planning, launches), the state loader and the
// dequantizer.  The decode-step kernel (a persistent grid whose warps stream row blocks
// of tiles through a bulk-copy ring, d_k/16 lanes per row) is in lores_step.cuh, its row
// arithmetic in lores_device.cuh, the key-axis variant in lores_key.cuh, and their
// instantiations in lores_inst.cu.
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <new>
#include <vector>

#include "lores.h"
#include "lores_device.cuh"
#include "lores_step.cuh"
#include "lores_key.cuh"
#include "lores_pair.cuh"
#include "lores_mma.cuh"

namespace lores {

// -------------------------------------------------------------------------------------
// state loader: quantize an fp32 state [B][H][d_v][d_k] with the step's quantizer
// -------------------------------------------------------------------------------------
struct LoadParams {
  const float *S;
  uint8_t *codes;
  float *scales;
  const LaneFmt *fmt;           // device [H][d_k/16]
  const int64_t *head_off;      // device [H]
  long long seq_bytes;
  long long rows;               // B * H * d_v
  int H, d_v, ng, G;
  uint32_t step_key;
  int stochastic;
  int axis;                     // 0: value-axis groups; 1: one scale per key column
  unsigned *flag;               // the handle's error word
  LORES_RANGES                  // index-checked build: the extent of every buffer of the launch
};

template <int DK>
__global__ void __launch_bounds__(kThreads) load_state_kernel(const LoadParams p) {
  constexpr int LPR = DK / 16, RPW = 32 / LPR;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int lir = lane % LPR, riw = lane / LPR, col0 = lir * 16;
  const long long gr = ((long long)blockIdx.x * kWarps + warp) * RPW + riw;   // global row
  const bool active = gr < p.rows;
  const long long grr = active ? gr : 0;
  const int row = (int)(grr % p.d_v);
  const long long tile = grr / p.d_v;
  const int head = (int)(tile % p.H);
  const long long b = tile / p.H;
  // Rows of one warp may belong to different tiles (and bit widths): every lane runs the
  // quantizer (it shuffles across the warp) and each lane stores per its own row.
  const LaneFmt f = p.fmt[head * (DK / 16) + lir];
  const int bits = f.bits;
  float x[16];
  const float *src = p.S + grr * DK + col0;
  const bool src_in = LORES_IN(p, kRgS, src, 64);
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    const float4 f = src_in ? __ldg(reinterpret_cast<const float4 *>(src) + c) : make_float4(0, 0, 0, 0);
    x[4 * c] = f.x; x[4 * c + 1] = f.y; x[4 * c + 2] = f.z; x[4 * c + 3] = f.w;
  }
  uint8_t *tilecodes = p.codes + b * p.seq_bytes + __ldg(p.head_off + head);
  const int g = col0 / p.G, lpg = p.G / 16;
  const uint32_t tkey = tile_key(p.step_key, (uint32_t)tile);
  const uint32_t n0 = (uint32_t)row * (uint32_t)(DK / 4) + (uint32_t)lir * 4u;
  uint32_t words[4];
  float s_new;
  requantize16<LPR>(x, bits == 32 ? 8 : bits, lpg, lane, tkey, n0, p.stochastic, words, s_new,
                    f.store);
  if (!active) return;
  const bool scale_in = LORES_IN(p, kRgScales, p.scales + grr * p.ng + g, 4);
  if (f.store >= 5 && f.store <= 7) {                 // dense bit planes
    const DenseLane dl{words[0], words[1], words[2], words[3]};
    uint8_t *rowp = tilecodes + (size_t)row * f.rowb;
    if (!LORES_IN(p, kRgCodes, rowp, f.rowb)) return;
    if (f.store == 5) st_dense<5>(rowp, DK, lir, dl);
    else if (f.store == 6) st_dense<6>(rowp, DK, lir, dl);
    else st_dense<7>(rowp, DK, lir, dl);
    if (lir % lpg == 0 && scale_in) p.scales[grr * p.ng + g] = s_new;
    return;
  }
  uint8_t *dst = tilecodes + (size_t)row * f.rowb + f.off;
  if (bits == 32) {
    if (LORES_IN(p, kRgCodes, dst, 64))
#pragma unroll
      for (int c = 0; c < 4; ++c)
        reinterpret_cast<float4 *>(dst)[c] = make_float4(x[4 * c], x[4 * c + 1], x[4 * c + 2], x[4 * c + 3]);
    return;
  }
  // lane blocks are 8-byte aligned (16 with one width per head)
  if (!LORES_IN(p, kRgCodes, dst, bits != 4 ? 16 : 8)) {
  } else if (bits != 4)
    st16_a8(dst, make_uint4(words[0], words[1], words[2], words[3]));
  else
    *reinterpret_cast<uint2 *>(dst) = make_uint2(words[0], words[1]);
  if (lir % lpg == 0 && scale_in) p.scales[grr * p.ng + g] = s_new;
}

// -------------------------------------------------------------------------------------
// dequantize the state into fp32 [B][H][d_v][d_k]
// -------------------------------------------------------------------------------------
template <int DK>
__global__ void __launch_bounds__(kThreads) dequant_kernel(const LoadParams p, float *out) {
  constexpr int LPR = DK / 16;
  const long long t = (long long)blockIdx.x * kThreads + threadIdx.x;
  if (t >= p.rows * LPR) return;
  const long long grr = t / LPR;
  const int lir = (int)(t % LPR), col0 = lir * 16;
  const int row = (int)(grr % p.d_v);
  const long long tile = grr / p.d_v;
  const int head = (int)(tile % p.H);
  const long long b = tile / p.H;
  const LaneFmt f = p.fmt[head * (DK / 16) + lir];
  const int bits = f.bits;
  const uint8_t *lanecodes = p.codes + b * p.seq_bytes + p.head_off[head] + (size_t)row * f.rowb + f.off;
  // (index-checked build: the lane's row must lie in the code pool, its scales in theirs)
  if (!LORES_IN(p, kRgCodes, lanecodes - f.off, f.rowb)) return;
  if (bits != 32 && !(p.axis ? LORES_IN(p, kRgScales, p.scales + tile * DK + col0, 64)
                             : LORES_IN(p, kRgScales, p.scales + grr * p.ng + col0 / p.G, 4)))
    return;
  float y[16];
  if (bits == 32) {
    const float4 *src = reinterpret_cast<const float4 *>(lanecodes);
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const float4 f = src[c];
      y[4 * c] = f.x; y[4 * c + 1] = f.y; y[4 * c + 2] = f.z; y[4 * c + 3] = f.w;
    }
  } else {
    float cf[16];
    if (f.store >= 5 && f.store <= 7) {               // dense bit planes
      const uint8_t *rowp = lanecodes - f.off;
      float2 c2[8];
      if (f.store == 5) unpack_dense<5>(ld_dense<5>(rowp, DK, lir), c2);
      else if (f.store == 6) unpack_dense<6>(ld_dense<6>(rowp, DK, lir), c2);
      else unpack_dense<7>(ld_dense<7>(rowp, DK, lir), c2);
#pragma unroll
      for (int e = 0; e < 8; ++e) { cf[2 * e] = c2[e].x; cf[2 * e + 1] = c2[e].y; }
    } else if (bits != 4) {
      unpack_i8(ld16_a8(lanecodes), cf);          // lane blocks are 8-byte aligned
    } else {
      unpack_i4(*reinterpret_cast<const uint2 *>(lanecodes), cf);
    }
    if (p.axis) {
      const float *sc = p.scales + tile * DK + col0;          // one scale per key column
#pragma unroll
      for (int e = 0; e < 16; ++e) y[e] = __fmul_rn(cf[e], sc[e]);
    } else {
      const float s = p.scales[grr * p.ng + col0 / p.G];
#pragma unroll
      for (int e = 0; e < 16; ++e) y[e] = __fmul_rn(cf[e], s);
    }
  }
  float4 *dst = reinterpret_cast<float4 *>(out + grr * DK + col0);
  if (LORES_IN(p, kRgS, dst, 64))
#pragma unroll
    for (int c = 0; c < 4; ++c) dst[c] = make_float4(y[4 * c], y[4 * c + 1], y[4 * c + 2], y[4 * c + 3]);
}

// Adds n to a device step counter (one thread; captured into a CUDA graph together with
// the steps that read the counter).
__global__ void advance_step_kernel(uint64_t *step, uint64_t n) { *step += n; }

// -------------------------------------------------------------------------------------
// host side
// -------------------------------------------------------------------------------------

// Step key: SplitMix64 (Steele, Lea & Flood 2014; Vigna's constants) of the seed xor
// SplitMix64 of the step, folded to 32 bits.
static uint64_t splitmix64(uint64_t z) {
  z += 0x9E3779B97F4A7C15ull;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}
static uint32_t step_key_of(uint64_t seed, uint64_t step) {
  const uint64_t k = splitmix64(seed ^ splitmix64(step));
  return (uint32_t)(k ^ (k >> 32));
}

using LoadFn = void (*)(const LoadParams);
using DequantFn = void (*)(const LoadParams, float *);

// The decode-step kernel of a configuration: mt = multi-token, ext = extended storage.
// ext: 0 plain kernel, 3 plain with the exact contractions (byte and nibble heads with one
// scale per row), 1 with the dense and per-lane paths, 4 the same with the exact
// contractions, 2 with the per-lane path only
static StepFn kernel_for(int dk, bool mt, int ext, bool diag, bool delta, bool sr) {
#define LORES_PICK_EXT(dk_, m_)                                                       \
  switch (ext) {                                                                      \
    case 1: return step_kernels_##dk_##_##m_##_1(diag, delta, sr);                    \
    case 2: return step_kernels_##dk_##_##m_##_2(diag, delta, sr);                    \
    case 3: return step_kernels_##dk_##_##m_##_3(diag, delta, sr);                    \
    case 4: return step_kernels_##dk_##_##m_##_4(diag, delta, sr);                    \
    default: return step_kernels_##dk_##_##m_##_0(diag, delta, sr);                   \
  }
#define LORES_PICK(dk_)                                                        \
  case dk_:                                                                    \
    if (mt) {                                                                  \
      LORES_PICK_EXT(dk_, 1)                                                   \
    }                                                                          \
    LORES_PICK_EXT(dk_, 0)
  switch (dk) {
    LORES_PICK(16)
    LORES_PICK(32)
    LORES_PICK(64)
    LORES_PICK(128)
    LORES_PICK(256)
  }
#undef LORES_PICK
#undef LORES_PICK_EXT
  return nullptr;
}
// The two-rows-per-lane kernel (heads of one byte or one nibble per code, several scales
// per row).
static StepFn pair_kernel_for(int dk, bool mt, bool diag, bool delta, bool sr) {
#define LORES_PAIR_PICK(dk_)                                                      \
  case dk_:                                                                       \
    return mt ? pair_kernels_##dk_##_1(diag, delta, sr) : pair_kernels_##dk_##_0(diag, delta, sr);
  switch (dk) {
    LORES_PAIR_PICK(16)
    LORES_PAIR_PICK(32)
    LORES_PAIR_PICK(64)
    LORES_PAIR_PICK(128)
    LORES_PAIR_PICK(256)
  }
#undef LORES_PAIR_PICK
  return nullptr;
}
// The tensor-core kernel (heads of one byte or one nibble per code, one scale per row).
static StepFn mma_kernel_for(int dk, bool mt, bool diag, bool delta, bool sr) {
  switch (dk) {
    case 16: return mma_kernels_16(diag, delta, sr, mt);
    case 32: return mma_kernels_32(diag, delta, sr, mt);
    case 64: return mma_kernels_64(diag, delta, sr, mt);
    case 128: return mma_kernels_128(diag, delta, sr, mt);
  }
  return nullptr;
}
static StepFn step_kernel_for(int dk, bool diag, bool delta, bool sr, bool exact) {
  return kernel_for(dk, false, exact ? 3 : 0, diag, delta, sr);
}
static KeyFn key_kernel_for(int dk, bool sr, bool load) {
  switch (dk) {
    case 16: return key_kernels_16(sr, load);
    case 32: return key_kernels_32(sr, load);
    case 64: return key_kernels_64(sr, load);
    case 128: return key_kernels_128(sr, load);
    case 256: return key_kernels_256(sr, load);
  }
  return nullptr;
}
static LoadFn load_kernel_for(int dk) {
  switch (dk) {
    case 16: return load_state_kernel<16>;
    case 32: return load_state_kernel<32>;
    case 64: return load_state_kernel<64>;
    case 128: return load_state_kernel<128>;
    case 256: return load_state_kernel<256>;
  }
  return nullptr;
}
static DequantFn dequant_kernel_for(int dk) {
  switch (dk) {
    case 16: return dequant_kernel<16>;
    case 32: return dequant_kernel<32>;
    case 64: return dequant_kernel<64>;
    case 128: return dequant_kernel<128>;
    case 256: return dequant_kernel<256>;
  }
  return nullptr;
}

}  // namespace lores

using namespace lores;

static_assert(sizeof(UnitDesc) == 32, "unit table entries are 32 bytes (shared-memory copy, "
                                      "allocation-free scratch)");
static_assert(sizeof(LaneFmt) == 16, "lane table entries are 16 bytes");

constexpr int kGuardBytes = 256;
constexpr unsigned char kGuardByte = 0xA5;

struct lores_handle {
  lores_config cfg;
  std::vector<int32_t> bits;       // [H]
  std::vector<int64_t> head_off;   // [H]
  int G = 0, ng = 0;
  long long seq_bytes = 0;
  uint8_t *codes = nullptr;
  float *scales = nullptr;
  unsigned *flag = nullptr;
  UnitDesc *units = nullptr;
  int32_t *d_bits = nullptr;
  int64_t *d_head_off = nullptr;
  LaneFmt *d_fmt = nullptr;        // [H][d_k/16]
  std::vector<LaneFmt> fmt;
  std::vector<int32_t> rowb;       // [H] bytes of one row
  std::vector<int32_t> store;      // [H] storage class (see UnitDesc::store)
  int units_per_seq = 0;
  int grid = 0;
  int smem = 0;
  StepParams sp{};
  StepFn step_fn = nullptr;
  StepFn mt_fn = nullptr;                // multi-token kernel of the same configuration
  bool pair = false;                     // step_fn is the two-rows-per-lane kernel
  bool mma = false;                      // step_fn is the tensor-core kernel
  // key-axis grouping
  int axis = 0;
  KeyParams kp{};
  KeyFn key_fn = nullptr;
  int key_smem = 0;
  KeyFn key_load_fn = nullptr;           // the same kernel as the state loader
  int key_grid = 0;                      // persistent grids of the two
  int key_load_grid = 0;
  // staging for lores_decode_step_host
  float *stage_in = nullptr;
  float *stage_o = nullptr;
  // index-checked build: bytes taken off the end of each buffer's declared extent
  // (lores_debug_trim_range), and the error word the last lores_check_errors read
  unsigned long long trim[kRgCount] = {};
  unsigned last_flags = 0;
};

namespace {

struct DeviceGuard {
  int prev = -1;
  bool ok = false;
  explicit DeviceGuard(int dev) {
    if (cudaGetDevice(&prev) != cudaSuccess) prev = -1;
    ok = cudaSetDevice(dev) == cudaSuccess;
  }
  ~DeviceGuard() {
    if (prev >= 0) cudaSetDevice(prev);
  }
};

inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

lores_status cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return LORES_OK;
  if (e == cudaErrorMemoryAllocation) {
    (void)cudaGetLastError();
    return LORES_ERR_OOM;
  }
  return LORES_ERR_CUDA;
}

void free_all(lores_handle *h) {
  if (h->codes) cudaFree(h->codes - kGuardBytes);
  if (h->scales) cudaFree(reinterpret_cast<uint8_t *>(h->scales) - kGuardBytes);
  cudaFree(h->flag);
  cudaFree(h->units);
  cudaFree(h->d_bits);
  cudaFree(h->d_head_off);
  cudaFree(h->d_fmt);
  cudaFree(h->stage_in);
  cudaFree(h->stage_o);
}

long long scale_count_of(const lores_handle *h) {
  const lores_config &c = h->cfg;
  return h->axis ? (long long)c.batch * c.heads * c.d_k
                 : (long long)c.batch * c.heads * c.d_v * h->ng;
}

LoadParams load_params(const lores_handle *h) {
  LoadParams p{};
  p.codes = h->codes;
  p.scales = h->scales;
  p.fmt = h->d_fmt;
  p.head_off = h->d_head_off;
  p.seq_bytes = h->seq_bytes;
  p.rows = (long long)h->cfg.batch * h->cfg.heads * h->cfg.d_v;
  p.H = h->cfg.heads;
  p.d_v = h->cfg.d_v;
  p.ng = h->ng;
  p.G = h->G;
  p.stochastic = h->cfg.stochastic;
  p.axis = h->axis;
  p.flag = h->flag;
  return p;
}

#ifdef LORES_INDEX_CHECKS
// Extents of the buffers one launch may touch (T tokens of inputs and outputs; S the fp32
// state of lores_load_state, or the output of lores_dequant_state), less the handle's trims.
Ranges ranges_of(const lores_handle *h, const void *q, const void *k, const void *v,
                 const void *alpha, const void *beta, const void *o, const void *S, int T) {
  const lores_config &c = h->cfg;
  const unsigned long long bh = (unsigned long long)c.batch * c.heads, t = (unsigned long long)T;
  Ranges r{};
  auto set = [&](int id, const void *ptr, unsigned long long bytes) {
    r.base[id] = ptr;
    r.bytes[id] = ptr && bytes > h->trim[id] ? bytes - h->trim[id] : 0;
  };
  set(kRgCodes, h->codes, (unsigned long long)c.batch * h->seq_bytes);
  set(kRgScales, h->scales, (unsigned long long)scale_count_of(h) * 4);
  set(kRgQ, q, t * bh * c.d_k * 4);
  set(kRgK, k, t * bh * c.d_k * 4);
  set(kRgV, v, t * bh * c.d_v * 4);
  set(kRgAlpha, alpha, t * (c.decay_diag ? bh * c.d_k : bh) * 4);
  set(kRgBeta, beta, t * bh * 4);
  set(kRgO, o, t * bh * c.d_v * 4);
  set(kRgS, S, bh * c.d_v * c.d_k * 4);
  return r;
}
#define LORES_SET_RANGES(params, ...) ((params).rg = ranges_of(h, __VA_ARGS__))
#else
#define LORES_SET_RANGES(params, ...) ((void)0)
#endif

}  // namespace

extern "C" {

const char *lores_status_string(lores_status s) {
  switch (s) {
    case LORES_OK: return "ok";
    case LORES_ERR_INVALID_ARG: return "invalid argument";
    case LORES_ERR_OOM: return "out of memory";
    case LORES_ERR_CUDA: return "CUDA error";
    case LORES_ERR_NONFINITE: return "non-finite state";
    case LORES_ERR_UNSUPPORTED: return "unsupported configuration";
    case LORES_ERR_TIMEOUT: return "kernel wait timed out";
    case LORES_ERR_CORRUPT: return "memory around the state was overwritten";
    case LORES_ERR_INDEX: return "an access fell outside its buffer (index-checked build)";
  }
  return "unknown status";
}

lores_status lores_assign_bits_by_decay(const float *mean_decay, int32_t H, float frac_high,
                                        int32_t bits_high, int32_t bits_low, int32_t *out_bits) {
  auto okbits = [](int b) { return (b >= 4 && b <= 8) || b == 32; };
  if (!mean_decay || !out_bits || H < 1 || !(frac_high >= 0.0f && frac_high <= 1.0f) ||
      !okbits(bits_high) || !okbits(bits_low))
    return LORES_ERR_INVALID_ARG;
  std::vector<int> order(H);
  for (int h = 0; h < H; ++h) order[h] = h;
  // largest mean decay first; equal decays keep head order (stable sort)
  std::stable_sort(order.begin(), order.end(),
                   [&](int a, int b) { return mean_decay[a] > mean_decay[b]; });
  long long n_high = (long long)((double)frac_high * (double)H + 0.5);
  n_high = std::max(0LL, std::min<long long>(n_high, H));
  for (int h = 0; h < H; ++h) out_bits[h] = bits_low;
  for (long long n = 0; n < n_high; ++n) out_bits[order[n]] = bits_high;
  return LORES_OK;
}

lores_status lores_create(const lores_config *cfg, lores_handle **out) {
  if (!out) return LORES_ERR_INVALID_ARG;
  *out = nullptr;
  if (!cfg) return LORES_ERR_INVALID_ARG;
  const lores_config c = *cfg;
  const int dk = c.d_k, dv = c.d_v;
  if (c.batch < 1 || c.heads < 1 || c.heads > 65536) return LORES_ERR_INVALID_ARG;
  if (!(dk == 16 || dk == 32 || dk == 64 || dk == 128 || dk == 256)) return LORES_ERR_INVALID_ARG;
  if (dv < 4 || dv > 4096 || dv % 4) return LORES_ERR_INVALID_ARG;
  const int G = c.group_size == 0 ? dk : c.group_size;
  if (G < 16 || G % 16 || dk % G) return LORES_ERR_INVALID_ARG;
  if ((c.delta != 0 && c.delta != 1) || (c.decay_diag != 0 && c.decay_diag != 1) ||
      (c.stochastic != 0 && c.stochastic != 1) || c.device < 0)
    return LORES_ERR_INVALID_ARG;
  if (c.scale_axis != 0 && c.scale_axis != 1) return LORES_ERR_INVALID_ARG;
  if (c.scale_axis == 1 && G != dk) return LORES_ERR_INVALID_ARG;   // one scale per column
  std::vector<int32_t> bits(c.heads, 8);
  if (c.head_bits)
    for (int h = 0; h < c.heads; ++h) {
      bits[h] = c.head_bits[h];
      if (!((bits[h] >= 4 && bits[h] <= 8) || bits[h] == 32)) return LORES_ERR_INVALID_ARG;
    }
  // per-channel precision: a width per (head, key group); a head whose groups all share
  // one width is an ordinary head of that width, any other head is "mixed" (bits 0)
  const int ngr = dk / G;
  std::vector<int32_t> gbits((size_t)c.heads * ngr);
  if (c.dense_codes != 0 && c.dense_codes != 1) return LORES_ERR_INVALID_ARG;
  if (c.dense_codes && (c.group_bits || c.scale_axis)) return LORES_ERR_INVALID_ARG;
  if (c.group_bits) {
    if (c.head_bits || c.scale_axis) return LORES_ERR_INVALID_ARG;
    for (int h = 0; h < c.heads; ++h) {
      for (int g = 0; g < ngr; ++g) {
        const int b = c.group_bits[(size_t)h * ngr + g];
        if (b < 4 || b > 8) return LORES_ERR_INVALID_ARG;
        gbits[(size_t)h * ngr + g] = b;
      }
      bits[h] = gbits[(size_t)h * ngr];
      for (int g = 1; g < ngr; ++g)
        if (gbits[(size_t)h * ngr + g] != bits[h]) bits[h] = 0;
    }
  } else {
    for (int h = 0; h < c.heads; ++h)
      for (int g = 0; g < ngr; ++g) gbits[(size_t)h * ngr + g] = bits[h];
  }

  DeviceGuard guard(c.device);
  if (!guard.ok) {
    (void)cudaGetLastError();
    return LORES_ERR_CUDA;
  }
  cudaDeviceProp prop;
  if (cudaGetDeviceProperties(&prop, c.device) != cudaSuccess) return LORES_ERR_CUDA;
  if (prop.major < 10) return LORES_ERR_UNSUPPORTED;

  lores_handle *h = new (std::nothrow) lores_handle();
  if (!h) return LORES_ERR_OOM;
  h->cfg = c;
  h->cfg.head_bits = nullptr;           // the caller's arrays are not kept
  h->cfg.group_bits = nullptr;
  h->bits = bits;
  h->G = G;
  h->ng = dk / G;
  h->axis = c.scale_axis;
  // row layout: key groups back to back, group g in G * storage(b_g) / 8 bytes; the lane
  // table gives each 16-column block its width, offset, r and fl(1/r)
  // dense_codes: heads of 5 to 7 bits store their codes in bit planes (storage class b)
  h->head_off.resize(c.heads);
  h->rowb.assign(c.heads, 0);
  h->store.assign(c.heads, 8);
  h->fmt.resize((size_t)c.heads * (dk / 16));
  long long off = 0;
  for (int hh = 0; hh < c.heads; ++hh) {
    const bool dense = c.dense_codes && bits[hh] >= 5 && bits[hh] <= 7;
    h->store[hh] = bits[hh] == 0 ? 0 : (dense ? bits[hh] : storage_bits(bits[hh]));
    int goff = 0;
    for (int g = 0; g < ngr; ++g) {
      const int b = bits[hh] == 32 ? 32 : gbits[(size_t)hh * ngr + g];
      for (int lb = g * G / 16; lb < (g + 1) * G / 16; ++lb) {
        LaneFmt &f = h->fmt[(size_t)hh * (dk / 16) + lb];
        f.bits = (int8_t)b;
        f.store = (int8_t)(dense ? b : storage_bits(b));
        f.off = dense ? 8 * lb : goff + (lb * 16 - g * G) * storage_bits(b) / 8;
        f.r = b == 32 ? 0.0f : (float)((1 << (b - 1)) - 1);
        f.inv_r = b == 32 ? 0.0f : 1.0f / f.r;
      }
      goff += G * storage_bits(b) / 8;
    }
    if (dense) goff = store_row_bytes(dk, bits[hh]);
    h->rowb[hh] = goff;
    for (int lb = 0; lb < dk / 16; ++lb) h->fmt[(size_t)hh * (dk / 16) + lb].rowb = (int16_t)goff;
    h->head_off[hh] = off;
    off += (long long)dv * goff;
  }
  h->seq_bytes = off;

  // ---- work units: row blocks of one tile, ~4 KB of state each, one warp per unit -----
  // A unit's row count is a multiple of the warp pass (32/LPR rows) where the head's
  // d_v allows; the last unit of a head takes the remainder.  Small batches split
  // units further (down to one pass) until every warp of one wave has work.
  const int LPR = dk / 16, rpw = 32 / LPR;
  // rows of a full unit: 4 KB of state, a whole number of warp passes (full_rows for a
  // head of one width)
  auto rows_for = [&](int rb) {
    const int n = 4096 / rb;
    return std::min(n < rpw ? rpw : n - n % rpw, dv);
  };
  // handles with dense heads take the kernel family with the dense and per-lane paths;
  // handles with per-channel (mixed-width) rows and no dense heads the per-lane family
  bool dense_heads = false, lane_heads = false;
  for (int hh = 0; hh < c.heads; ++hh) {
    dense_heads |= h->store[hh] >= 5 && h->store[hh] <= 7;
    lane_heads |= h->store[hh] == 0;
  }
  // byte or nibble heads with one scale per row take the exact contractions (u and S'q
  // as exact integer sums) wherever the general kernel serves them
  bool exact_heads = false;
  for (int hh = 0; hh < c.heads; ++hh) exact_heads |= G == dk && (h->store[hh] == 8 || h->store[hh] == 4);
  const int ext = dense_heads ? (exact_heads ? 4 : 1) : (lane_heads ? 2 : (exact_heads ? 3 : 0));
  // heads that all store one byte or one nibble per code take the tensor-core kernel with
  // one scale per row (d_k up to 128), or else the two-rows-per-lane kernel when cut into
  // full units; any other handle the general one
  bool pair_heads = ext == 0 || ext == 3;   // no dense or per-lane heads
  for (int hh = 0; hh < c.heads; ++hh) pair_heads &= h->store[hh] == 8 || h->store[hh] == 4;
  const bool mma = pair_heads && G == dk && dk <= 128;
  const StepFn general_fn = kernel_for(dk, false, ext, c.decay_diag, c.delta, c.stochastic);
  const StepFn pair_fn =
      pair_heads && !mma ? pair_kernel_for(dk, false, c.decay_diag, c.delta, c.stochastic) : nullptr;
  const StepFn mma_fn = mma ? mma_kernel_for(dk, false, c.decay_diag, c.delta, c.stochastic) : nullptr;
  StepFn fn = general_fn;
  bool pair = false;
  int split = 1;
  auto build_units = [&](std::vector<UnitDesc> &u) {
    u.clear();
    for (int hh = 0; hh < c.heads; ++hh) {
      const int b = bits[hh];
      const int rb = h->rowb[hh];
      int R = rows_for(rb);
      int Rs = R / split;
      Rs -= Rs % std::min(rpw, R);
      Rs -= Rs % 4;
      R = std::max(Rs, std::min(4, R));
      for (int r0 = 0; r0 < dv; r0 += R) {
        UnitDesc d{};
        d.head = hh;
        d.row0 = (int16_t)r0;
        d.nrows = (int16_t)std::min(R, dv - r0);
        d.bits = (int16_t)b;
        d.rowb = (int16_t)rb;
        d.store = (int16_t)h->store[hh];
        d.code_off = h->head_off[hh] + (long long)r0 * rb;
        d.r = (b == 32 || b == 0) ? 0.0f : (float)((1 << (b - 1)) - 1);
        d.inv_r = (b == 32 || b == 0) ? 0.0f : 1.0f / d.r;
        u.push_back(d);
      }
    }
  };
  std::vector<UnitDesc> units;
  int ctas_per_sm = 1;
  auto bits_rank = [](const UnitDesc &u) {
    return u.store == 8 ? 0 : (u.store == 4 ? 1 : (u.store == 32 ? 2 : 3 + u.store));
  };
  for (;;) {
    build_units(units);
    std::stable_sort(units.begin(), units.end(), [&](const UnitDesc &x, const UnitDesc &y) {
      return bits_rank(x) < bits_rank(y);
    });
    pair = pair_heads && !mma;
    for (const UnitDesc &d : units)      // (storage 8 or 4 checked first: full_rows needs it)
      pair = pair && (d.store == 8 || d.store == 4) && d.nrows == full_rows(dk, d.store);
    fn = mma ? mma_fn : (pair ? pair_fn : general_fn);
    int cmax = 0, smax = 0, vmax = 0, maxrows = 0;
    for (const UnitDesc &d : units) {
      cmax = std::max(cmax, d.nrows * (int)d.rowb);
      if (d.bits != 32) smax = std::max(smax, d.nrows * h->ng * 4);
      vmax = std::max(vmax, d.nrows * 4);
      maxrows = std::max(maxrows, (int)d.nrows);
    }
    auto up16 = [](int x) { return (x + 15) & ~15; };
    const int stage = up16(cmax) + up16(smax) + up16(vmax) + 2 * dk * 4 +
                      (c.decay_diag ? dk * 4 : 0);
    const int opart_floats = ((maxrows * LPR + 31) / 32) * 32;     // 128-byte multiples
    const int ow_floats = ((maxrows + 31) / 32) * 32;
    // digit planes (8 d_k) and a tile's k and alpha (8 d_k): only where exact contractions
    // run (the tensor-core kernel, or the general kernel's exact families)
    const int plane_bytes = (mma || exact_heads) ? 16 * dk : 0;
    const int warp_bytes =
        ((64 + 4 * (opart_floats + ow_floats) + plane_bytes + kStages * stage + 127) / 128) * 128;
    const int table = (int)units.size() * (int)sizeof(UnitDesc) <= 16384
                          ? (((int)units.size() * (int)sizeof(UnitDesc) + 127) / 128) * 128 : 0;
    const int smem = table + kWarps * warp_bytes;
    // the attribute is per kernel and shared by all handles: only ever raise it
    cudaFuncAttributes fa;
    if (cudaFuncGetAttributes(&fa, fn) != cudaSuccess ||
        (fa.maxDynamicSharedSizeBytes < smem &&
         cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
             cudaSuccess)) {
      delete h;
      return LORES_ERR_CUDA;
    }
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&ctas_per_sm, fn, kThreads, smem) !=
            cudaSuccess ||
        ctas_per_sm < 1) {
      delete h;
      return LORES_ERR_CUDA;
    }
    const long long total = (long long)c.batch * (long long)units.size();
    const long long warp_slots = (long long)ctas_per_sm * prop.multiProcessorCount * kWarps;
    if (total >= warp_slots || maxrows <= rpw || maxrows <= 4 || split >= 64) {
      h->smem = smem;
      h->sp.table_bytes = table;
      h->sp.warp_bytes = warp_bytes;
      h->sp.opart_floats = opart_floats;
      h->sp.ow_floats = ow_floats;
      h->sp.plane_bytes = plane_bytes;
      h->sp.st_scales = up16(cmax);
      h->sp.st_v = h->sp.st_scales + up16(smax);
      h->sp.st_k = h->sp.st_v + up16(vmax);
      h->sp.st_q = h->sp.st_k + dk * 4;
      h->sp.st_a = h->sp.st_q + dk * 4;
      h->sp.stage_bytes = stage;
      const long long ctas = (total + kWarps - 1) / kWarps;
      h->grid = (int)std::min<long long>(ctas, (long long)ctas_per_sm * prop.multiProcessorCount);
      if (pair || mma) {
        // the table is sorted bytes first: class 0 = one byte per code, class 1 = nibbles;
        // CTAs are split in proportion to the classes' state entries
        int n8 = 0;
        long long e8 = 0, e4 = 0;
        for (const UnitDesc &d : units) {
          if (d.store == 8) {
            ++n8;
            e8 += (long long)d.nrows * dk;
          } else {
            e4 += (long long)d.nrows * dk;
          }
        }
        if (e8 > 0 && e4 > 0) h->grid = std::max(h->grid, 2);
        long long c8 = (h->grid * e8 + (e8 + e4) / 2) / (e8 + e4);
        if (e8 > 0 && e4 > 0) c8 = std::min<long long>(std::max<long long>(c8, 1), h->grid - 1);
        h->sp.pair_lo[0] = 0;
        h->sp.pair_hi[0] = n8;
        h->sp.pair_lo[1] = n8;
        h->sp.pair_hi[1] = (int)units.size();
        h->sp.pair_ctas = (int)c8;
        // The tensor-core kernel with two or more units per warp: every CTA takes both
        // classes in turn, so an SM runs one body at a time (side by side they thrash its
        // instruction cache).  With fewer, the classes stay in their own CTAs: in turn
        // they would add a unit's latency to a warp's.
        if (mma && e8 > 0 && e4 > 0 && total >= 2 * warp_slots) h->sp.pair_ctas = -1;
      }
      break;
    }
    split *= 2;
  }
  h->units_per_seq = (int)units.size();
  h->step_fn = fn;
  h->pair = pair;
  h->mma = mma;
  // multi-token calls: the tensor-core or two-rows-per-lane kernel's form, or the general one
  h->mt_fn = mma ? mma_kernel_for(dk, true, c.decay_diag, c.delta, c.stochastic)
                 : (pair ? pair_kernel_for(dk, true, c.decay_diag, c.delta, c.stochastic)
                         : kernel_for(dk, true, ext, c.decay_diag, c.delta, c.stochastic));
  {
    cudaFuncAttributes fa;
    if (cudaFuncGetAttributes(&fa, h->mt_fn) != cudaSuccess ||
        (fa.maxDynamicSharedSizeBytes < h->smem &&
         cudaFuncSetAttribute(h->mt_fn, cudaFuncAttributeMaxDynamicSharedMemorySize, h->smem) !=
             cudaSuccess)) {
      delete h;
      return LORES_ERR_CUDA;
    }
  }
  h->sp.T = 1;

  const long long code_bytes = (long long)c.batch * h->seq_bytes;
  const long long scale_count = scale_count_of(h);
  if (h->axis) {
    // key-axis kernel: a CTA holds one whole tile in shared memory at a time, and a second
    // stage for its next tile where both fit
    int rbmax = 0;
    for (int hh = 0; hh < c.heads; ++hh) rbmax = std::max(rbmax, row_bytes(dk, bits[hh]));
    auto up128 = [](int x) { return (x + 127) & ~127; };
    KeyParams &kp = h->kp;
    int so = 0;                                     // offsets inside a stage
    kp.sm_codes = so; so += up128(dv * rbmax);
    kp.sm_scales = so; so += up128(dk * 4);
    kp.sm_k = so; so += up128(dk * 4);
    kp.sm_q = so; so += up128(dk * 4);
    kp.sm_a = so; so += up128(dk * 4);
    kp.sm_v = so; so += up128(dv * 4);
    kp.stage_bytes = so;
    int off = 128;                                  // two mbarriers
    kp.sm_opart = off; off += up128(dv * (dk / 16) * 4);
    kp.sm_ow = off; off += up128(dv * 4);
    kp.sm_cm = off; off += up128(kWarps * dk * 4);
    kp.stage0 = off;
    const int limit = 200 * 1024;
    if (off + so > limit) {
      delete h;
      return LORES_ERR_UNSUPPORTED;                 // tile too large for one CTA
    }
    kp.nstage = off + 2 * so <= limit ? 2 : 1;
    off += kp.nstage * so;
    h->key_smem = off;
    h->key_fn = key_kernel_for(dk, c.stochastic != 0, false);
    h->key_load_fn = key_kernel_for(dk, c.stochastic != 0, true);
    const long long tiles = (long long)c.batch * c.heads;
    int *grids[2] = {&h->key_grid, &h->key_load_grid};
    KeyFn fns[2] = {h->key_fn, h->key_load_fn};
    for (int i = 0; i < 2; ++i) {
      cudaFuncAttributes fa;
      int per_sm = 0;
      if (cudaFuncGetAttributes(&fa, fns[i]) != cudaSuccess ||
          (fa.maxDynamicSharedSizeBytes < off &&
           cudaFuncSetAttribute(fns[i], cudaFuncAttributeMaxDynamicSharedMemorySize, off) !=
               cudaSuccess) ||
          cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fns[i], kThreads, off) !=
              cudaSuccess ||
          per_sm < 1) {
        delete h;
        return LORES_ERR_CUDA;
      }
      *grids[i] = (int)std::min<long long>(tiles, (long long)per_sm * prop.multiProcessorCount);
    }
  }
  cudaError_t e = cudaSuccess;
  // guard bands of kGuardBytes before and after the code pool and the scales, filled
  // with kGuardByte and verified by lores_check_errors: a write outside the state shows
  // up as LORES_ERR_CORRUPT
  uint8_t *cbase = nullptr, *sbase = nullptr;
  if (e == cudaSuccess) e = cudaMalloc(&cbase, (size_t)code_bytes + 2 * kGuardBytes);
  if (e == cudaSuccess) h->codes = cbase + kGuardBytes;
  if (e == cudaSuccess) e = cudaMalloc(&sbase, (size_t)scale_count * 4 + 2 * kGuardBytes);
  if (e == cudaSuccess) h->scales = reinterpret_cast<float *>(sbase + kGuardBytes);
  if (e == cudaSuccess) e = cudaMemset(cbase, kGuardByte, kGuardBytes);
  if (e == cudaSuccess) e = cudaMemset(cbase + kGuardBytes + code_bytes, kGuardByte, kGuardBytes);
  if (e == cudaSuccess) e = cudaMemset(sbase, kGuardByte, kGuardBytes);
  if (e == cudaSuccess)
    e = cudaMemset(sbase + kGuardBytes + scale_count * 4, kGuardByte, kGuardBytes);
  if (e == cudaSuccess) e = cudaMalloc(&h->flag, 16);
  if (e == cudaSuccess) e = cudaMalloc(&h->units, units.size() * sizeof(UnitDesc));
  if (e == cudaSuccess) e = cudaMalloc(&h->d_bits, c.heads * sizeof(int32_t));
  if (e == cudaSuccess) e = cudaMalloc(&h->d_head_off, c.heads * sizeof(int64_t));
  if (e == cudaSuccess) e = cudaMalloc(&h->d_fmt, h->fmt.size() * sizeof(LaneFmt));
  if (e == cudaSuccess) e = cudaMemset(h->codes, 0, (size_t)code_bytes);
  if (e == cudaSuccess) e = cudaMemset(h->scales, 0, (size_t)scale_count * 4);
  if (e == cudaSuccess) e = cudaMemset(h->flag, 0, 16);
  if (e == cudaSuccess)
    e = cudaMemcpy(h->units, units.data(), units.size() * sizeof(UnitDesc), cudaMemcpyHostToDevice);
  if (e == cudaSuccess)
    e = cudaMemcpy(h->d_bits, bits.data(), c.heads * sizeof(int32_t), cudaMemcpyHostToDevice);
  if (e == cudaSuccess)
    e = cudaMemcpy(h->d_head_off, h->head_off.data(), c.heads * sizeof(int64_t),
                   cudaMemcpyHostToDevice);
  if (e == cudaSuccess)
    e = cudaMemcpy(h->d_fmt, h->fmt.data(), h->fmt.size() * sizeof(LaneFmt), cudaMemcpyHostToDevice);
  if (e != cudaSuccess) {
    const lores_status st = cuda_status(e);
    free_all(h);
    delete h;
    return st;
  }

  StepParams &p = h->sp;
  p.codes = h->codes;
  p.scales = h->scales;
  p.flag = h->flag;
  p.wait_ns = kWaitNs;
  p.fault_b = -1;
  p.fault_ub = -1;
  p.units = h->units;
  p.seq_bytes = h->seq_bytes;
  p.total_units = (long long)c.batch * h->units_per_seq;
  p.B = c.batch;
  p.H = c.heads;
  p.d_v = dv;
  p.ng = h->ng;
  p.G = G;
  p.units_per_seq = h->units_per_seq;
  p.fmt = h->d_fmt;
  KeyParams &kp = h->kp;
  kp.codes = h->codes;
  kp.scales = h->scales;
  kp.flag = h->flag;
  kp.head_bits = h->d_bits;
  kp.head_off = h->d_head_off;
  kp.seq_bytes = h->seq_bytes;
  kp.tiles = (long long)c.batch * c.heads;
  kp.H = c.heads;
  kp.d_v = dv;
  kp.delta = c.delta;
  kp.diag = c.decay_diag;
  kp.stochastic = c.stochastic;
  kp.seed = c.seed;
  kp.wait_ns = kWaitNs;
  *out = h;
  return LORES_OK;
}

lores_status lores_destroy(lores_handle *h) {
  if (!h) return LORES_OK;
  DeviceGuard guard(h->cfg.device);
  free_all(h);
  delete h;
  return LORES_OK;
}

static lores_status launch_step(lores_handle *h, const float *q, const float *k, const float *v,
                                const float *alpha, const float *beta, float *o, uint64_t step,
                                const uint64_t *step_dev, void *stream);

lores_status lores_decode_step(lores_handle *h, const float *q, const float *k, const float *v,
                               const float *alpha, const float *beta, float *o, uint64_t step,
                               void *stream) {
  return launch_step(h, q, k, v, alpha, beta, o, step, nullptr, stream);
}

lores_status lores_decode_step_dev(lores_handle *h, const float *q, const float *k, const float *v,
                                   const float *alpha, const float *beta, float *o,
                                   const uint64_t *step, void *stream) {
  if (!step || (reinterpret_cast<uintptr_t>(step) & 7u)) return LORES_ERR_INVALID_ARG;
  return launch_step(h, q, k, v, alpha, beta, o, 0, step, stream);
}

lores_status lores_advance_step(uint64_t *step, uint64_t n, void *stream) {
  if (!step || (reinterpret_cast<uintptr_t>(step) & 7u)) return LORES_ERR_INVALID_ARG;
  advance_step_kernel<<<1, 1, 0, static_cast<cudaStream_t>(stream)>>>(step, n);
  return cuda_status(cudaGetLastError());
}

static lores_status launch_step(lores_handle *h, const float *q, const float *k, const float *v,
                                const float *alpha, const float *beta, float *o, uint64_t step,
                                const uint64_t *step_dev, void *stream) {
  if (!h || !q || !k || !v || !alpha || !beta || !o) return LORES_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) ||
      (h->cfg.decay_diag ? !aligned16(alpha) : (reinterpret_cast<uintptr_t>(alpha) & 3u)) ||
      (reinterpret_cast<uintptr_t>(beta) & 3u) || (reinterpret_cast<uintptr_t>(o) & 3u))
    return LORES_ERR_INVALID_ARG;
  DeviceGuard guard(h->cfg.device);
  if (!guard.ok) return LORES_ERR_CUDA;
  if (h->axis) {
    KeyParams kp = h->kp;
    kp.q = q;
    kp.k = k;
    kp.v = v;
    kp.alpha = alpha;
    kp.beta = beta;
    kp.o = o;
    kp.S = nullptr;
    kp.step_key = step_key_of(h->cfg.seed, step);
    kp.step_dev = step_dev;
    LORES_SET_RANGES(kp, q, k, v, alpha, beta, o, nullptr, 1);
    h->key_fn<<<h->key_grid, kThreads, h->key_smem, static_cast<cudaStream_t>(stream)>>>(kp);
    return cuda_status(cudaGetLastError());
  }
  StepParams p = h->sp;
  p.q = q;
  p.k = k;
  p.v = v;
  p.alpha = alpha;
  p.beta = beta;
  p.o = o;
  p.step_key = step_key_of(h->cfg.seed, step);
  p.seed = h->cfg.seed;
  p.step_dev = step_dev;
  LORES_SET_RANGES(p, q, k, v, alpha, beta, o, nullptr, 1);
  h->step_fn<<<h->grid, kThreads, h->smem, static_cast<cudaStream_t>(stream)>>>(p);
  return cuda_status(cudaGetLastError());
}

lores_status lores_decode_steps(lores_handle *h, int32_t T, const float *q, const float *k,
                                const float *v, const float *alpha, const float *beta, float *o,
                                uint64_t step0, void *stream) {
  if (!h || T < 1 || !q || !k || !v || !alpha || !beta || !o) return LORES_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) ||
      (h->cfg.decay_diag ? !aligned16(alpha) : (reinterpret_cast<uintptr_t>(alpha) & 3u)) ||
      (reinterpret_cast<uintptr_t>(beta) & 3u) || (reinterpret_cast<uintptr_t>(o) & 3u))
    return LORES_ERR_INVALID_ARG;
  const lores_config &c = h->cfg;
  const long long bh = (long long)c.batch * c.heads;
  const long long tok_qk = bh * c.d_k, tok_v = bh * c.d_v, tok_b = bh;
  const long long tok_a = c.decay_diag ? bh * c.d_k : bh;
  if (T == 1 || h->axis) {
    // one token, or key-axis groups (a tile per CTA): one step launch per token
    for (int t = 0; t < T; ++t) {
      const lores_status st =
          lores_decode_step(h, q + t * tok_qk, k + t * tok_qk, v + t * tok_v, alpha + t * tok_a,
                            beta + t * tok_b, o + t * tok_v, step0 + (uint64_t)t, stream);
      if (st != LORES_OK) return st;
    }
    return LORES_OK;
  }
  DeviceGuard guard(c.device);
  if (!guard.ok) return LORES_ERR_CUDA;
  StepParams p = h->sp;
  p.q = q;
  p.k = k;
  p.v = v;
  p.alpha = alpha;
  p.beta = beta;
  p.o = o;
  p.T = T;
  p.tok_qk = tok_qk;
  p.tok_v = tok_v;
  p.tok_a = tok_a;
  p.tok_b = tok_b;
  p.tok_o = tok_v;
  p.seed = c.seed;
  p.step0 = step0;
  LORES_SET_RANGES(p, q, k, v, alpha, beta, o, nullptr, T);
  h->mt_fn<<<h->grid, kThreads, h->smem, static_cast<cudaStream_t>(stream)>>>(p);
  return cuda_status(cudaGetLastError());
}

static lores_status step_host(lores_handle *h, const float *q, const float *k, const float *v,
                              const float *alpha, const float *beta, float *o, uint64_t step,
                              void *stream, bool wait);

lores_status lores_decode_step_host(lores_handle *h, const float *q, const float *k,
                                    const float *v, const float *alpha, const float *beta,
                                    float *o, uint64_t step, void *stream) {
  return step_host(h, q, k, v, alpha, beta, o, step, stream, true);
}

lores_status lores_decode_step_host_async(lores_handle *h, const float *q, const float *k,
                                          const float *v, const float *alpha,
                                          const float *beta, float *o, uint64_t step,
                                          void *stream) {
  return step_host(h, q, k, v, alpha, beta, o, step, stream, false);
}

static lores_status step_host(lores_handle *h, const float *q, const float *k, const float *v,
                              const float *alpha, const float *beta, float *o, uint64_t step,
                              void *stream, bool wait) {
  if (!h || !q || !k || !v || !alpha || !beta || !o) return LORES_ERR_INVALID_ARG;
  DeviceGuard guard(h->cfg.device);
  if (!guard.ok) return LORES_ERR_CUDA;
  const lores_config &c = h->cfg;
  const size_t BH = (size_t)c.batch * c.heads;
  const size_t nk = BH * c.d_k, nv = BH * c.d_v, na = c.decay_diag ? BH * c.d_k : BH;
  // staging: q | k | v | alpha | beta, each region padded to 16 bytes
  auto pad4 = [](size_t n) { return (n + 3) & ~size_t(3); };
  const size_t oq = 0, ok_ = oq + pad4(nk), ov = ok_ + pad4(nk), oa = ov + pad4(nv),
               ob = oa + pad4(na), total = ob + pad4(BH);
  cudaError_t e = cudaSuccess;
  if (!h->stage_in) e = cudaMalloc(&h->stage_in, total * 4);
  if (e == cudaSuccess && !h->stage_o) e = cudaMalloc(&h->stage_o, nv * 4);
  if (e != cudaSuccess) return cuda_status(e);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  float *d = h->stage_in;
  e = cudaMemcpyAsync(d + oq, q, nk * 4, cudaMemcpyHostToDevice, s);
  if (e == cudaSuccess) e = cudaMemcpyAsync(d + ok_, k, nk * 4, cudaMemcpyHostToDevice, s);
  if (e == cudaSuccess) e = cudaMemcpyAsync(d + ov, v, nv * 4, cudaMemcpyHostToDevice, s);
  if (e == cudaSuccess) e = cudaMemcpyAsync(d + oa, alpha, na * 4, cudaMemcpyHostToDevice, s);
  if (e == cudaSuccess) e = cudaMemcpyAsync(d + ob, beta, BH * 4, cudaMemcpyHostToDevice, s);
  if (e != cudaSuccess) return cuda_status(e);
  lores_status st =
      lores_decode_step(h, d + oq, d + ok_, d + ov, d + oa, d + ob, h->stage_o, step, stream);
  if (st != LORES_OK) return st;
  e = cudaMemcpyAsync(o, h->stage_o, nv * 4, cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess && wait) e = cudaStreamSynchronize(s);
  return cuda_status(e);
}

lores_status lores_dequant_state(lores_handle *h, float *out, void *stream) {
  if (!h || !out || !aligned16(out)) return LORES_ERR_INVALID_ARG;
  DeviceGuard guard(h->cfg.device);
  if (!guard.ok) return LORES_ERR_CUDA;
  LoadParams p = load_params(h);
  LORES_SET_RANGES(p, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, out, 1);
  const long long threads = p.rows * (h->cfg.d_k / 16);
  const int blocks = (int)((threads + kThreads - 1) / kThreads);
  dequant_kernel_for(h->cfg.d_k)<<<blocks, kThreads, 0, static_cast<cudaStream_t>(stream)>>>(p, out);
  return cuda_status(cudaGetLastError());
}

lores_status lores_load_state(lores_handle *h, const float *S, uint64_t step, void *stream) {
  if (!h || !S || !aligned16(S)) return LORES_ERR_INVALID_ARG;
  DeviceGuard guard(h->cfg.device);
  if (!guard.ok) return LORES_ERR_CUDA;
  if (h->axis) {
    KeyParams kp = h->kp;
    kp.S = S;
    kp.step_key = step_key_of(h->cfg.seed, step);
    LORES_SET_RANGES(kp, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, S, 1);
    h->key_load_fn<<<h->key_load_grid, kThreads, h->key_smem, static_cast<cudaStream_t>(stream)>>>(kp);
    return cuda_status(cudaGetLastError());
  }
  LoadParams p = load_params(h);
  p.S = S;
  p.step_key = step_key_of(h->cfg.seed, step);
  LORES_SET_RANGES(p, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, S, 1);
  const int rpw = 32 / (h->cfg.d_k / 16);
  const long long warps = (p.rows + rpw - 1) / rpw;
  const int blocks = (int)((warps + kWarps - 1) / kWarps);
  load_kernel_for(h->cfg.d_k)<<<blocks, kThreads, 0, static_cast<cudaStream_t>(stream)>>>(p);
  return cuda_status(cudaGetLastError());
}

lores_status lores_export_codes(lores_handle *h, void *codes, float *scales, void *stream) {
  if (!h) return LORES_ERR_INVALID_ARG;
  DeviceGuard guard(h->cfg.device);
  if (!guard.ok) return LORES_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaSuccess;
  if (codes)
    e = cudaMemcpyAsync(codes, h->codes, (size_t)h->cfg.batch * h->seq_bytes, cudaMemcpyDefault, s);
  if (e == cudaSuccess && scales)
    e = cudaMemcpyAsync(scales, h->scales, (size_t)scale_count_of(h) * 4, cudaMemcpyDefault, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  return cuda_status(e);
}

lores_status lores_load_codes(lores_handle *h, const void *codes, const float *scales,
                              void *stream) {
  if (!h || !codes || !scales) return LORES_ERR_INVALID_ARG;
  DeviceGuard guard(h->cfg.device);
  if (!guard.ok) return LORES_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e =
      cudaMemcpyAsync(h->codes, codes, (size_t)h->cfg.batch * h->seq_bytes, cudaMemcpyDefault, s);
  if (e == cudaSuccess)
    e = cudaMemcpyAsync(h->scales, scales, (size_t)scale_count_of(h) * 4, cudaMemcpyDefault, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  return cuda_status(e);
}

lores_status lores_get_layout(const lores_handle *h, lores_layout *out, int64_t *head_offsets) {
  if (!h || !out) return LORES_ERR_INVALID_ARG;
  out->code_bytes = (int64_t)h->cfg.batch * h->seq_bytes;
  out->seq_code_bytes = h->seq_bytes;
  out->scale_count = scale_count_of(h);
  out->n_groups = h->axis ? 0 : h->ng;
  out->units_per_step = (int32_t)((long long)h->cfg.batch * h->units_per_seq);
  out->grid = h->grid;
  out->smem_bytes = h->smem;
  out->codes_dev = h->codes;
  out->scales_dev = h->scales;
  out->step_kernel = h->axis ? 2 : (h->mma ? 3 : (h->pair ? 1 : 0));
  if (head_offsets)
    for (int hh = 0; hh < h->cfg.heads; ++hh) head_offsets[hh] = h->head_off[hh];
  return LORES_OK;
}

int32_t lores_index_checked(void) {
#ifdef LORES_INDEX_CHECKS
  return 1;
#else
  return 0;
#endif
}

lores_status lores_debug_trim_range(lores_handle *h, int32_t which, uint64_t bytes) {
  if (!h || which < 0 || which >= kRgCount) return LORES_ERR_INVALID_ARG;
#ifdef LORES_INDEX_CHECKS
  h->trim[which] = bytes;
  return LORES_OK;
#else
  (void)bytes;
  return LORES_ERR_UNSUPPORTED;
#endif
}

lores_status lores_debug_last_flags(lores_handle *h, uint32_t *flags) {
  if (!h || !flags) return LORES_ERR_INVALID_ARG;
  *flags = h->last_flags;
  return LORES_OK;
}

lores_status lores_set_fault_injection(lores_handle *h, int32_t seq, int32_t unit,
                                       uint32_t wait_us) {
  if (!h || seq < -1 || seq >= h->cfg.batch) return LORES_ERR_INVALID_ARG;
  if (seq >= 0 && (unit < 0 || unit >= h->units_per_seq)) return LORES_ERR_INVALID_ARG;
  if (seq >= 0 && h->axis) return LORES_ERR_UNSUPPORTED;
  const unsigned long long ns = wait_us ? (unsigned long long)wait_us * 1000ull : kWaitNs;
  h->sp.fault_b = seq;
  h->sp.fault_ub = seq >= 0 ? unit : -1;
  h->sp.wait_ns = ns;
  h->kp.wait_ns = ns;
  return LORES_OK;
}

lores_status lores_check_errors(lores_handle *h, void *stream) {
  if (!h) return LORES_ERR_INVALID_ARG;
  DeviceGuard guard(h->cfg.device);
  if (!guard.ok) return LORES_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  unsigned f = 0;
  cudaError_t e = cudaStreamSynchronize(s);
  if (e == cudaSuccess) e = cudaMemcpy(&f, h->flag, sizeof(unsigned), cudaMemcpyDeviceToHost);
  if (e == cudaSuccess) e = cudaMemset(h->flag, 0, sizeof(unsigned));
  if (e != cudaSuccess) return cuda_status(e);
  h->last_flags = f;
  if (f & kFlagIndex) return LORES_ERR_INDEX;   // (a skipped copy also runs a wait out)
  if (f & kFlagTimeout) return LORES_ERR_TIMEOUT;
  // guard bands around the state
  const long long cb = (long long)h->cfg.batch * h->seq_bytes, sb = scale_count_of(h) * 4;
  const uint8_t *bands[4] = {h->codes - kGuardBytes, h->codes + cb,
                             reinterpret_cast<const uint8_t *>(h->scales) - kGuardBytes,
                             reinterpret_cast<const uint8_t *>(h->scales) + sb};
  for (const uint8_t *band : bands) {
    uint8_t host[kGuardBytes];
    e = cudaMemcpy(host, band, kGuardBytes, cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return cuda_status(e);
    for (int i = 0; i < kGuardBytes; ++i)
      if (host[i] != kGuardByte) return LORES_ERR_CORRUPT;
  }
  if (f & kFlagNonFinite) return LORES_ERR_NONFINITE;
  return LORES_OK;
}

}  // extern "C"

// -------------------------------------------------------------------------------------
// Decode step without any allocation
// -------------------------------------------------------------------------------------
// Some callers cannot let a library allocate device memory: a serving engine that
// plans every buffer from its own pool up front (a cudaMalloc there can stall the
// device and fragment the pool), or an application held to a fixed device-memory
// budget.  For them, lores_decode_step_noalloc runs the same decode kernel on state
// buffers the caller owns, and keeps the kernel's own bookkeeping (the work-unit table
// and the error word) in the fixed array below instead of in allocated memory.  The
// array is part of the module image: every GPU that loads this library holds it until
// the process exits.
namespace {

constexpr int kNoAllocMaxUnits = 2048;                 // work units of one sequence, at most
constexpr size_t kNoAllocTableBytes = kNoAllocMaxUnits * sizeof(UnitDesc);
constexpr size_t kNoAllocScratchBytes = kNoAllocTableBytes + 256;   // table, then error word
constexpr int kNoAllocMaxDevices = 64;

std::mutex g_noalloc_mutex;
void *g_noalloc_scratch_ptr[kNoAllocMaxDevices] = {};
// The work-unit table is planned in host memory of the library (not on the caller's stack,
// which may be small in a worker thread); the lock is held from planning until the
// upload from it has returned.
UnitDesc g_noalloc_units[kNoAllocMaxUnits];
std::mutex g_noalloc_plan_mutex;

}  // namespace

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

namespace {

// Device address of g_noalloc_scratch on `device` (the current device).  In host code the
// array's name only stands in for the symbol, so the address is looked up once per device.
lores_status noalloc_scratch(int device, unsigned char **out) {
  if (device >= kNoAllocMaxDevices) return LORES_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_noalloc_mutex);
  if (!g_noalloc_scratch_ptr[device]) {
    void *ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || !ptr) {
      (void)cudaGetLastError();
      return LORES_ERR_CUDA;
    }
    g_noalloc_scratch_ptr[device] = ptr;
  }
  *out = static_cast<unsigned char *>(g_noalloc_scratch_ptr[device]);
  return LORES_OK;
}

}  // namespace

extern "C" lores_status lores_decode_step_noalloc(const lores_config *cfg, void *codes,
                                                  float *scales, const float *q, const float *k,
                                                  const float *v, const float *alpha,
                                                  const float *beta, float *o, uint64_t step,
                                                  uint32_t *flags_out, void *stream) {
  if (!cfg || !codes || !scales || !q || !k || !v || !alpha || !beta || !o)
    return LORES_ERR_INVALID_ARG;
  const lores_config c = *cfg;
  const int dk = c.d_k, dv = c.d_v;
  if (c.batch < 1 || c.heads < 1 || c.heads > 65536) return LORES_ERR_INVALID_ARG;
  if (!(dk == 16 || dk == 32 || dk == 64 || dk == 128 || dk == 256)) return LORES_ERR_INVALID_ARG;
  if (dv < 4 || dv > 4096 || dv % 4) return LORES_ERR_INVALID_ARG;
  const int G = c.group_size == 0 ? dk : c.group_size;
  if (G < 16 || G % 16 || dk % G) return LORES_ERR_INVALID_ARG;
  if ((c.delta != 0 && c.delta != 1) || (c.decay_diag != 0 && c.decay_diag != 1) ||
      (c.stochastic != 0 && c.stochastic != 1) || c.device < 0)
    return LORES_ERR_INVALID_ARG;
  if (c.scale_axis != 0 || c.group_bits || c.dense_codes)
    return LORES_ERR_UNSUPPORTED;                       // per-head byte/nibble codes,
                                                                          // value-axis groups
  for (int hh = 0; c.head_bits && hh < c.heads; ++hh)
    if (!((c.head_bits[hh] >= 4 && c.head_bits[hh] <= 8) || c.head_bits[hh] == 32))
      return LORES_ERR_INVALID_ARG;
  if (!aligned16(codes) || !aligned16(scales) || !aligned16(q) || !aligned16(k) || !aligned16(v) ||
      (c.decay_diag ? !aligned16(alpha) : (reinterpret_cast<uintptr_t>(alpha) & 3u)) ||
      (reinterpret_cast<uintptr_t>(beta) & 3u) || (reinterpret_cast<uintptr_t>(o) & 3u))
    return LORES_ERR_INVALID_ARG;

  // Work units of one sequence: full units of ~4 KB of state, the last unit of each head
  // takes the remainder (the same plan as a handle at full batch).  A pageable upload has
  // copied the table out of host memory when cudaMemcpyAsync returns, so the lock can be
  // released after it.
  std::lock_guard<std::mutex> plan_lock(g_noalloc_plan_mutex);
  UnitDesc *units = g_noalloc_units;
  int nunits = 0;
  long long seq_bytes = 0;
  int cmax = 0, smax = 0, vmax = 0, maxrows = 0;
  const int ng = dk / G, LPR = dk / 16;
  for (int hh = 0; hh < c.heads; ++hh) {
    const int b = c.head_bits ? c.head_bits[hh] : 8;
    const int R = std::min(full_rows(dk, storage_bits(b)), dv);
    for (int r0 = 0; r0 < dv; r0 += R) {
      if (nunits == kNoAllocMaxUnits) return LORES_ERR_UNSUPPORTED;   // beyond the fixed table
      UnitDesc &d = units[nunits++];
      d = UnitDesc{};
      d.head = hh;
      d.row0 = (int16_t)r0;
      d.nrows = (int16_t)std::min(R, dv - r0);
      d.bits = (int16_t)b;
      d.rowb = (int16_t)row_bytes(dk, b);
      d.store = (int16_t)storage_bits(b);
      d.code_off = seq_bytes + (long long)r0 * row_bytes(dk, b);
      d.r = b == 32 ? 0.0f : (float)((1 << (b - 1)) - 1);
      d.inv_r = b == 32 ? 0.0f : 1.0f / d.r;
      cmax = std::max(cmax, d.nrows * row_bytes(dk, b));
      if (b != 32) smax = std::max(smax, d.nrows * ng * 4);
      vmax = std::max(vmax, d.nrows * 4);
      maxrows = std::max(maxrows, (int)d.nrows);
    }
    seq_bytes += (long long)dv * row_bytes(dk, b);
  }

  DeviceGuard guard(c.device);
  if (!guard.ok) {
    (void)cudaGetLastError();
    return LORES_ERR_CUDA;
  }
  unsigned char *scratch = nullptr;
  lores_status st = noalloc_scratch(c.device, &scratch);
  if (st != LORES_OK) return st;
  int sms = 0;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, c.device) != cudaSuccess)
    return LORES_ERR_CUDA;

  auto up16 = [](int x) { return (x + 15) & ~15; };
  StepParams p{};
  const int stage = up16(cmax) + up16(smax) + up16(vmax) + 2 * dk * 4 + (c.decay_diag ? dk * 4 : 0);
  p.opart_floats = ((maxrows * LPR + 31) / 32) * 32;
  p.ow_floats = ((maxrows + 31) / 32) * 32;
  p.plane_bytes = 16 * dk;
  p.warp_bytes =
      ((64 + 4 * (p.opart_floats + p.ow_floats) + p.plane_bytes + kStages * stage + 127) / 128) * 128;
  p.table_bytes = nunits * (int)sizeof(UnitDesc) <= 16384
                      ? ((nunits * (int)sizeof(UnitDesc) + 127) / 128) * 128 : 0;
  p.st_scales = up16(cmax);
  p.st_v = p.st_scales + up16(smax);
  p.st_k = p.st_v + up16(vmax);
  p.st_q = p.st_k + dk * 4;
  p.st_a = p.st_q + dk * 4;
  p.stage_bytes = stage;
  const int smem = p.table_bytes + kWarps * p.warp_bytes;
  // one scale per row: the byte and nibble heads take the exact contractions
  StepFn fn = step_kernel_for(dk, c.decay_diag, c.delta, c.stochastic, G == dk);
  cudaFuncAttributes fa;
  if (cudaFuncGetAttributes(&fa, fn) != cudaSuccess ||
      (fa.maxDynamicSharedSizeBytes < smem &&
       cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess))
    return LORES_ERR_CUDA;
  int ctas_per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&ctas_per_sm, fn, kThreads, smem) !=
          cudaSuccess ||
      ctas_per_sm < 1)
    return LORES_ERR_CUDA;

  p.codes = static_cast<uint8_t *>(codes);
  p.scales = scales;
  p.q = q;
  p.k = k;
  p.v = v;
  p.alpha = alpha;
  p.beta = beta;
  p.o = o;
  p.units = reinterpret_cast<const UnitDesc *>(scratch);
  p.flag = reinterpret_cast<unsigned *>(scratch + kNoAllocTableBytes);
  p.seq_bytes = seq_bytes;
  p.total_units = (long long)c.batch * nunits;
  p.B = c.batch;
  p.H = c.heads;
  p.d_v = dv;
  p.ng = ng;
  p.G = G;
  p.units_per_seq = nunits;
  p.T = 1;
  p.wait_ns = kWaitNs;
  p.fault_b = -1;
  p.fault_ub = -1;
  p.step_key = step_key_of(c.seed, step);
#ifdef LORES_INDEX_CHECKS
  {
    const unsigned long long bh = (unsigned long long)c.batch * c.heads;
    const void *base[kRgCount] = {codes, scales, q, k, v, alpha, beta, o, nullptr};
    const unsigned long long bytes[kRgCount] = {
        (unsigned long long)c.batch * seq_bytes, bh * dv * ng * 4, bh * dk * 4, bh * dk * 4,
        bh * dv * 4, (c.decay_diag ? bh * dk : bh) * 4, bh * 4, bh * dv * 4, 0};
    for (int i = 0; i < kRgCount; ++i) {
      p.rg.base[i] = base[i];
      p.rg.bytes[i] = bytes[i];
    }
  }
#endif
  const long long ctas = (p.total_units + kWarps - 1) / kWarps;
  const int grid = (int)std::min<long long>(ctas, (long long)ctas_per_sm * sms);

  // The scratch keeps whatever the previous call left: the table is rewritten and the
  // error word cleared on this stream before the launch.
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemcpyAsync(scratch, units, nunits * sizeof(UnitDesc),
                                  cudaMemcpyHostToDevice, s);
  if (e == cudaSuccess) e = cudaMemsetAsync(scratch + kNoAllocTableBytes, 0, sizeof(unsigned), s);
  if (e != cudaSuccess) return cuda_status(e);
  fn<<<grid, kThreads, smem, s>>>(p);
  e = cudaGetLastError();
  if (e == cudaSuccess && flags_out)
    e = cudaMemcpyAsync(flags_out, scratch + kNoAllocTableBytes, sizeof(uint32_t),
                        cudaMemcpyDefault, s);
  return cuda_status(e);
}
