// Fused rotate + sign-adjust + per-token quantization on B200 tensor cores (tcgen05 + TMEM), and a
// one-warp-per-token kernel for rows of 512-2048 channels.
//
// What one token row computes (SignRot abstract and explainer, "The standard fix is rotation" and
// "SignRot asks one crowd to walk across the hall"): y = diag(s) H diag(D) x / sqrt(n), then the
// per-token asymmetric 4-bit grid ("Picture the photographer", "Worked example") or one of its
// variants (8 bits, symmetric).
//
// How it maps onto the hardware. Write the channel index as j = (a, h2, b) with n = 28 * M,
// a in [0, 28), h2 in [0, 4) (top two bits of the length-M axis) and b in [0, M/4), or for
// power-of-two n as j = (r, b) with r in [0, 128). The rotation factors as
//     H = (H_28 kron H_4) kron H_{M/4}      (or H_128 kron H_{n/128})
// and the first factor is a dense 112 x 112 (128 x 128) block with entries +/-1. It is applied as
// a tcgen05 MMA chain per token on the exact bf16 inputs (+/-1 times bf16 is exact; fp32
// accumulation):
//     A  = rowsign (.) (H_28 kron H_4), 128 x 128 bf16, K-major, SMEM (built once per CTA)
//     B  = D (.) x viewed as [K = (c, h2) rows][N = b columns], bf16, MN-major, SMEM
//     Dt = A B in TMEM: lane = (h2', a) row, column = b.
// Each TMEM lane is then one length-M/4 line of the remaining Walsh-Hadamard factor, so the
// remaining FWHT stages run inside one thread's registers (for 256-column lines the stage on the
// top column bit runs inside the MMA accumulation instead), and each thread ends up owning a
// contiguous run of output channels (contiguous packed stores). The per-token min/max is a warp
// reduction plus an exchange between the token's warps through shared memory.
//
// A sign vector from an outlier channel k (signrot_build_sign's form, s_j = sgn(H[j,k] D_k x_k))
// costs nothing per element: s = sigma * H_28[a][c_k] * (-1)^popcount(hi & e_hi) *
// (-1)^popcount(b & e_lo). The row part is folded into A's rows; the column part becomes a
// permutation of the input columns, b -> b ^ e_lo (the TMA box order, and the 16-byte slots and
// words the D pass moves), except its bit 0, which the epilogue applies as a sign on the odd
// columns; sigma is a sign on every output. A general s vector is applied elementwise in the
// epilogue instead.
//
// Kernels (each one's own comment gives its warp roles and pipeline):
//   rotq_stream_kernel  64-128 columns per TMEM lane (n = 7168 .. 14336, 8192 .. 16384), and the
//                       short rows n = 3584, 4096 with four tokens to a 128-column tile
//   rotq_wide_kernel    256 columns per TMEM lane (n = 28672, 32768)
//   rotq_small_kernel   n = 512, 1024, 2048 (F = 1) with s in its outlier form: one warp per token
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cstdint>
#include <mutex>
#include <utility>

#include "signrot_device.cuh"
#include "signrot_internal.h"
#include "tc_ptx.cuh"

namespace signrot {

// Set (bit 0) by any kernel whose bounded wait gave up; read by signrot_device_error.
__device__ unsigned int g_device_error = 0;

namespace {

using namespace ptx;

// Warp roles. Up to 128 columns per token the epilogue runs as two groups of four warps that
// take alternate tokens (12 warps, 168 registers each: three warps share each SM sub-partition's
// 16K-register file); at 256 columns a lane holds more values, so one group (8 warps, up to 255
// registers). Each group's warp w reads TMEM lane quadrant w % 4.
__host__ __device__ constexpr int epi_groups(int ncol) { return ncol <= 128 ? 2 : 1; }
constexpr uint32_t kABytes = 128 * 128 * 2;  // A: 128 x 128 bf16
constexpr uint32_t kBoxBytes = 16 * 128;     // one TMA box: 16 rows x 64 bf16 (128 B) = 2 KB
constexpr float kMagic = 12582912.0f;        // 1.5 * 2^23: fp32 whose ulp is 1

// bit 0: a bounded wait expired; bit 1: the outlier channel index was out of range.
__device__ __forceinline__ void flag_error(unsigned int bit = 1u) { atomicOr(&g_device_error, bit); }

struct TcParams {
  const void* xraw;  // rows, for the streamed variant's bulk copies
  int64_t ldx;
  int32_t T;
  int32_t n;
  int32_t logM;  // F = 28: M = 2^logM; F = 1: unused
  int32_t stages;
  const int8_t* d;
  const int8_t* s;     // general sign vector (kVecSign) or null
  const int32_t* kp;   // outlier channel (pattern sign) or null
  const float* xkp;    // its signed calibration value
  uint8_t* q;
  float* scale;
  float* zero;
  float* y;
  int64_t ldy;
  float clip;
  float inv_sqrt_n;
  H28Masks h;
};

// ---------------------------------------------------------------------------- sign bookkeeping

// Structured sign vector: sigma * g(a) * (-1)^popcount(hi & e_hi) * (-1)^popcount(b & e_lo).
struct SignPlan {
  int32_t c_k;       // F = 28: H_28 column of the outlier (g(a) = H_28[a][c_k])
  uint32_t e_hi;     // bits of the outlier index that index A's rows (h2 or r)
  uint32_t e_lo;     // bits that index the TMEM columns: applied as the column permutation b ^ e_lo
  bool active;
};

// The outlier's index k and value x_k, loaded by every thread before anything else: plain loads
// issued ahead of the CTA's first bulk copies, used only once those are on their way.
struct OutlierRef {
  int32_t k;
  float xk;
};
__device__ __forceinline__ OutlierRef load_outlier(const TcParams& p) {
  OutlierRef o{-1, 0.f};
  if (p.kp != nullptr) {
    o.k = *p.kp;
    o.xk = *p.xkp;
  }
  return o;
}

// The parts of s = sigma * H[:, k] that do not depend on D: its column part e_lo, row part e_hi
// and H_28 column c_k. sigma = sgn(x_k) sgn(D_k), a sign on every output, is applied by the
// epilogue (outlier_sigma), which has time to load D_k.
template <bool kF28, int kNcol>
__device__ __forceinline__ SignPlan make_plan(const TcParams& p, OutlierRef o) {
  SignPlan sp{0, 0u, 0u, false};
  if (p.kp == nullptr) return sp;
  const int k = o.k;
  if (k < 0 || k >= p.n) {  // not a channel: report it and apply no sign adjustment
    flag_error(2u);
    return sp;
  }
  if (o.xk == 0.f) return sp;  // s_j = sgn(+/-0) = +1 everywhere
  sp.active = true;
  constexpr int kLogNcol = kNcol == 16 ? 4 : (kNcol == 32 ? 5 : (kNcol == 64 ? 6 : (kNcol == 128 ? 7 : 8)));
  if (kF28) {
    const int M = 1 << p.logM;
    sp.c_k = k >> p.logM;
    const uint32_t e = static_cast<uint32_t>(k & (M - 1));
    sp.e_hi = e >> kLogNcol;
    sp.e_lo = e & (kNcol - 1);
  } else {
    sp.e_hi = static_cast<uint32_t>(k) >> kLogNcol;
    sp.e_lo = static_cast<uint32_t>(k) & (kNcol - 1);
  }
  return sp;
}

// True when sigma = sgn(x_k) sgn(D_k) is -1 for an active plan: every output changes sign.
__device__ __forceinline__ bool outlier_sigma_neg(const TcParams& p, const SignPlan& sp, OutlierRef o) {
  return sp.active && ((o.xk < 0.f) != (p.d[o.k] < 0));
}

// A[m][8j .. 8j+7] as one 16-byte chunk of bf16 +/-1 (m = TMEM lane / output row, k = K index).
// F = 28: m = 32 h' + a (a < 28), k = 4 c + h2, A = H_28[a][c] (-1)^popc(h' & h2) times the row
// sign of the outlier plan, H_28[a][c_k] (-1)^popc(h' & e_hi); rows a >= 28 and columns c >= 28
// are zero. Power of two: A = (-1)^popc(m & k) times (-1)^popc(m & e_hi).
template <bool kF28>
__device__ __forceinline__ uint4 a_chunk(int m, int j, const SignPlan& sp, const H28Masks& h) {
  uint32_t neg = 0;  // bit e: entry k = 8j + e is -1
  if (kF28) {
    const int hp = m >> 5, a = m & 31;
    if (a >= 28 || j >= 14) return make_uint4(0u, 0u, 0u, 0u);
    const uint32_t row = h.row[a];
    uint32_t s = 0;
    if (sp.active) s = ((row >> sp.c_k) & 1u) ^ (__popc(hp & sp.e_hi) & 1);
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const uint32_t c = 2 * j + (e >> 2), h2 = e & 3;
      neg |= (((row >> c) & 1u) ^ (__popc(hp & h2) & 1) ^ s) << e;
    }
  } else {
    uint32_t s = __popc(m & (8 * j)) & 1;
    if (sp.active) s ^= __popc(m & sp.e_hi) & 1;
#pragma unroll
    for (int e = 0; e < 8; ++e) neg |= ((__popc(m & e) & 1) ^ s) << e;
  }
  uint32_t w[4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
    w[i] = (0x3F80u | (((neg >> (2 * i)) & 1u) << 15)) | ((0x3F80u | (((neg >> (2 * i + 1)) & 1u) << 15)) << 16);
  return make_uint4(w[0], w[1], w[2], w[3]);
}

// K-major 128B-swizzled placement of A[m][k] (8-row x 64-element atoms, K halves 16 KB apart).
__device__ __forceinline__ uint32_t a_offset(int m, int k) {
  return static_cast<uint32_t>((k >> 6) * 16384 + (m >> 3) * 1024 + (m & 7) * 128 +
                               ((((k & 63) >> 3) ^ (m & 7)) << 4) + (k & 7) * 2);
}

__device__ __forceinline__ uint64_t smem_desc(uint32_t addr, uint32_t lbo, uint32_t sbo) {
  return static_cast<uint64_t>((addr & 0x3FFFFu) >> 4) | (static_cast<uint64_t>(lbo >> 4) << 16) |
         (static_cast<uint64_t>(sbo >> 4) << 32) | (1ull << 46) | (2ull << 61);
}


// ---------------------------------------------------------------------------- FWHT in registers

// Butterfly on bit kBit of the column index over pairs p[i] = (w[2i], w[2i+1]).
template <int kPairs, int kBit>
__device__ __forceinline__ void fwht_stage(float2 (&p)[kPairs]) {
  if constexpr (kBit == 0) {
#pragma unroll
    for (int i = 0; i < kPairs; ++i) {
      const float u = p[i].x, v = p[i].y;
      p[i].x = u + v;
      p[i].y = u - v;
    }
  } else {
    constexpr int hs = 1 << (kBit - 1);
#pragma unroll
    for (int i = 0; i < kPairs; ++i) {
      if ((i & hs) == 0) {
        const float2 u = p[i], v = p[i + hs];
        p[i] = __fadd2_rn(u, v);
        p[i + hs] = fsub2(u, v);
      }
    }
  }
}

// All stages over kBits bits of the in-thread column index.
template <int kPairs, int kBits>
__device__ __forceinline__ void fwht_local(float2 (&p)[kPairs]) {
  fwht_stage<kPairs, 0>(p);
  if constexpr (kBits > 1) fwht_stage<kPairs, 1>(p);
  if constexpr (kBits > 2) fwht_stage<kPairs, 2>(p);
  if constexpr (kBits > 3) fwht_stage<kPairs, 3>(p);
  if constexpr (kBits > 4) fwht_stage<kPairs, 4>(p);
  if constexpr (kBits > 5) fwht_stage<kPairs, 5>(p);
  if constexpr (kBits > 6) fwht_stage<kPairs, 6>(p);
}

// D's signs of one 16-byte chunk (8 bf16 columns, D at d8[0..8)) as XOR masks on its four
// 32-bit words.
__device__ __forceinline__ uint4 chunk_sign_masks(uint2 d8) {
  uint32_t w[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint32_t pair = ((i < 2 ? d8.x : d8.y) >> (16 * (i & 1))) & 0xffffu;  // d[2i], d[2i+1]
    w[i] = ((pair & 0x80u) << 8) | ((pair & 0x8000u) << 16);
  }
  return make_uint4(w[0], w[1], w[2], w[3]);
}
__device__ __forceinline__ uint4 chunk_sign_masks(const int8_t* d8) {
  uint32_t w[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) w[i] = (d8[2 * i] < 0 ? 0x8000u : 0u) | (d8[2 * i + 1] < 0 ? 0x80000000u : 0u);
  return make_uint4(w[0], w[1], w[2], w[3]);
}

// Streamed D pass for one token: each lane takes its kPerD fixed 16-byte chunks of the linear row
// (32 chunks apart; the last one only when `last` is set), flips D's signs, moves the chunk's words
// by kW (the permutation's bits 1 and 2; bit 0 is left to the epilogue) and stores the chunk at its
// place in the swizzled MMA tile. Chunks go in batches of kBatch loads, then kBatch stores: the
// two buffers are different, but the compiler cannot know it and would otherwise wait out every
// load.
template <int kW, int kPerD, int kBatch>
__device__ __forceinline__ void stream_d_pass(const uint4* src, uint8_t* tile, const uint4 (&mask)[kPerD],
                                              const uint32_t (&dst)[kPerD], bool last) {
#pragma unroll
  for (int u0 = 0; u0 < kPerD; u0 += kBatch) {
    constexpr int kB = kBatch;
    uint4 v[kB];
#pragma unroll
    for (int b = 0; b < kB; ++b)
      if (u0 + b < kPerD && (u0 + b < kPerD - 1 || last)) v[b] = src[32 * (u0 + b)];
#pragma unroll
    for (int b = 0; b < kB; ++b) {
      if (u0 + b < kPerD && (u0 + b < kPerD - 1 || last)) {
        const uint4 m = mask[u0 + b];
        const uint32_t w[4] = {v[b].x ^ m.x, v[b].y ^ m.y, v[b].z ^ m.z, v[b].w ^ m.w};
        *reinterpret_cast<uint4*>(tile + dst[u0 + b]) = make_uint4(w[kW], w[1 ^ kW], w[2 ^ kW], w[3 ^ kW]);
      }
    }
  }
}

// TMEM -> registers: kN pairs (2 * kN consecutive columns from taddr) into p[kOff .. kOff + kN).
template <int kOff, int kN, int kPairs>
__device__ __forceinline__ void tmem_load_pairs(uint32_t taddr, float2 (&p)[kPairs]) {
  static_assert(kN % 16 == 0 && kOff + kN <= kPairs, "whole 32-column loads only");
  if constexpr (kN == 64) {
    uint32_t r[128];
    tmem_ld128(taddr, r);
#pragma unroll
    for (int i = 0; i < 64; ++i) p[kOff + i] = make_float2(__uint_as_float(r[2 * i]), __uint_as_float(r[2 * i + 1]));
  } else {
#pragma unroll
    for (int c = 0; c < kN; c += 16) {
      uint32_t r[32];
      tmem_ld32(taddr + 2 * c, r);
#pragma unroll
      for (int i = 0; i < 16; ++i)
        p[kOff + c + i] = make_float2(__uint_as_float(r[2 * i]), __uint_as_float(r[2 * i + 1]));
    }
  }
}


// Elementwise general sign vector: bit r of sbits flips the sign of column r.
template <int kPairs>
__device__ __forceinline__ void apply_sign_bits(float2 (&p)[kPairs], const uint32_t* sbits_in) {
  // The words are the same for every token; hiding that from the compiler keeps it from hoisting
  // all 2*kPairs masks out of the token loop into registers.
  uint32_t sbits[(2 * kPairs + 31) / 32];
#pragma unroll
  for (int w = 0; w < (2 * kPairs + 31) / 32; ++w) {
    sbits[w] = sbits_in[w];
    asm volatile("" : "+r"(sbits[w]));
  }
#pragma unroll
  for (int i = 0; i < kPairs; ++i) {
    const int r0 = 2 * i, r1 = 2 * i + 1;
    const uint32_t m0 = (sbits[r0 >> 5] << (31 - (r0 & 31))) & 0x80000000u;
    const uint32_t m1 = (sbits[r1 >> 5] << (31 - (r1 & 31))) & 0x80000000u;
    p[i].x = __uint_as_float(__float_as_uint(p[i].x) ^ m0);
    p[i].y = __uint_as_float(__float_as_uint(p[i].y) ^ m1);
  }
}

// Extremes of the even (.x) and odd (.y) columns kept apart, so that a sign flip of every odd
// column can be applied to the result instead of the values.
template <int kPairs>
__device__ __forceinline__ void local_minmax_xy(const float2 (&p)[kPairs], float& lx, float& hx, float& ly, float& hy) {
  float l0 = p[0].x, h0 = p[0].x, l1 = p[0].y, h1 = p[0].y;
#pragma unroll
  for (int i = 1; i + 1 < kPairs; i += 2) {
    l0 = fmin3(l0, p[i].x, p[i + 1].x);
    h0 = fmax3(h0, p[i].x, p[i + 1].x);
    l1 = fmin3(l1, p[i].y, p[i + 1].y);
    h1 = fmax3(h1, p[i].y, p[i + 1].y);
  }
  if ((kPairs & 1) == 0) {
    l0 = fminf(l0, p[kPairs - 1].x);
    h0 = fmaxf(h0, p[kPairs - 1].x);
    l1 = fminf(l1, p[kPairs - 1].y);
    h1 = fmaxf(h1, p[kPairs - 1].y);
  }
  lx = l0; hx = h0; ly = l1; hy = h1;
}


// Eight consecutive codes -> one u32 of nibbles (element 2i low nibble). u holds the bit
// patterns of fma(w, c, zero + 1.5*2^23), whose low byte is the code: 0..15 on the asymmetric grid,
// where one multiply-add per pair combines them; -7..7 (two's complement) on the symmetric grid,
// whose negative codes carry set high bits into the byte and are masked to their nibble first.
template <bool kSigned = false>
__device__ __forceinline__ uint32_t pack8(const uint32_t (&u)[8]) {
  if constexpr (kSigned) {
    uint32_t b[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) b[i] = ((u[2 * i + 1] & 15u) << 4) | (u[2 * i] & 15u);
    return __byte_perm(b[0] | (b[1] << 8), b[2] | (b[3] << 8), 0x5410);
  } else {
    const uint32_t b01 = u[1] * 16u + u[0], b23 = u[3] * 16u + u[2];
    const uint32_t b45 = u[5] * 16u + u[4], b67 = u[7] * 16u + u[6];
    const uint32_t w0 = b23 * 256u + b01, w1 = b67 * 256u + b45;
    return __byte_perm(w0, w1, 0x5410);
  }
}

// Quantize 16 pairs (32 consecutive columns) into one 16-byte store of packed nibbles. Each
// fma(w, c, zm) lands in [lo_m, hi_m] around 1.5 * 2^23 after clamping, where the fp32 ulp is 1,
// so its low bits are the code (two's complement for the symmetric grid's negative codes).
template <bool kClamp, bool kSigned, int kWords = 4>
__device__ __forceinline__ void quant_words(const float2* p, float2 c2, float zm, float lo_m, float hi_m,
                                            uint32_t (&words)[kWords]) {
  const float2 z2 = make_float2(zm, zm);
#pragma unroll
  for (int g = 0; g < kWords; ++g) {
    uint32_t u[8];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      float2 t = __ffma2_rn(p[4 * g + k], c2, z2);
      if (kClamp) {
        t.x = fminf(fmaxf(t.x, lo_m), hi_m);
        t.y = fminf(fmaxf(t.y, lo_m), hi_m);
      }
      u[2 * k] = __float_as_uint(t.x);
      u[2 * k + 1] = __float_as_uint(t.y);
    }
    words[g] = pack8<kSigned>(u);
  }
}
template <bool kClamp, bool kSigned>
__device__ __forceinline__ uint4 quant16(const float2* p, float2 c2, float zm, float lo_m, float hi_m) {
  uint32_t w[4];
  quant_words<kClamp, kSigned, 4>(p, c2, zm, lo_m, hi_m, w);
  return make_uint4(w[0], w[1], w[2], w[3]);
}
// Eight pairs (16 columns) into one 8-byte store.
template <bool kClamp, bool kSigned>
__device__ __forceinline__ uint2 quant8(const float2* p, float2 c2, float zm, float lo_m, float hi_m) {
  uint32_t w[2];
  quant_words<kClamp, kSigned, 2>(p, c2, zm, lo_m, hi_m, w);
  return make_uint2(w[0], w[1]);
}

// The 8-bit form: 8 pairs (16 consecutive columns) into one 16-byte store, one code per byte.
template <bool kClamp>
__device__ __forceinline__ uint4 quant16_bytes(const float2* p, float2 c2, float zm, float lo_m, float hi_m) {
  const float2 z2 = make_float2(zm, zm);
  uint32_t words[4];
#pragma unroll
  for (int g = 0; g < 4; ++g) {
    float2 t0 = __ffma2_rn(p[2 * g], c2, z2), t1 = __ffma2_rn(p[2 * g + 1], c2, z2);
    if (kClamp) {
      t0.x = fminf(fmaxf(t0.x, lo_m), hi_m);
      t0.y = fminf(fmaxf(t0.y, lo_m), hi_m);
      t1.x = fminf(fmaxf(t1.x, lo_m), hi_m);
      t1.y = fminf(fmaxf(t1.y, lo_m), hi_m);
    }
    const uint32_t w01 = __byte_perm(__float_as_uint(t0.x), __float_as_uint(t0.y), 0x0040);
    const uint32_t w23 = __byte_perm(__float_as_uint(t1.x), __float_as_uint(t1.y), 0x0040);
    words[g] = __byte_perm(w01, w23, 0x5410);
  }
  return make_uint4(words[0], words[1], words[2], words[3]);
}

// Quantize + store one run of 2*kPairs consecutive channels at q_out (16 B aligned): kBits = 4,
// two codes per byte (element 2i low nibble); kBits = 8, one per byte. c2 holds the multipliers of
// the even and the odd channels.
template <int kPairs, int kBits, bool kSigned>
__device__ __forceinline__ void quant_store(const float2 (&p)[kPairs], float2 c2, float zm, bool clamp, float lo_m,
                                            float hi_m, uint8_t* q_out) {
  uint4* dst = reinterpret_cast<uint4*>(q_out);
  if constexpr (kBits == 4 && kPairs == 8) {  // 16 columns: 8 bytes of codes
    *reinterpret_cast<uint2*>(q_out) = clamp ? quant8<true, kSigned>(p, c2, zm, lo_m, hi_m)
                                             : quant8<false, kSigned>(p, c2, zm, lo_m, hi_m);
  } else if constexpr (kBits == 4) {
    static_assert(kPairs % 16 == 0, "whole 16-byte runs of codes");
    if (clamp) {
#pragma unroll
      for (int i = 0; i < kPairs / 16; ++i) dst[i] = quant16<true, kSigned>(p + 16 * i, c2, zm, lo_m, hi_m);
    } else {
#pragma unroll
      for (int i = 0; i < kPairs / 16; ++i) dst[i] = quant16<false, kSigned>(p + 16 * i, c2, zm, lo_m, hi_m);
    }
  } else {
    if (clamp) {
#pragma unroll
      for (int i = 0; i < kPairs / 8; ++i) dst[i] = quant16_bytes<true>(p + 8 * i, c2, zm, lo_m, hi_m);
    } else {
#pragma unroll
      for (int i = 0; i < kPairs / 8; ++i) dst[i] = quant16_bytes<false>(p + 8 * i, c2, zm, lo_m, hi_m);
    }
  }
}

template <int kPairs>
__device__ __forceinline__ void store_y(const float2 (&p)[kPairs], float rs, float* y_out, float rs_odd) {
  float4* dst = reinterpret_cast<float4*>(y_out);
#pragma unroll
  for (int i = 0; i < kPairs / 2; ++i)
    dst[i] = make_float4(p[2 * i].x * rs, p[2 * i].y * rs_odd, p[2 * i + 1].x * rs, p[2 * i + 1].y * rs_odd);
}
template <int kPairs>
__device__ __forceinline__ void store_y(const float2 (&p)[kPairs], float rs, float* y_out) {
  store_y<kPairs>(p, rs, y_out, rs);
}

struct TokenGrid {
  float c;      // w -> y / scale
  float zm;     // zero + 1.5 * 2^23
  bool clamp;   // some code of this token falls outside [code_min, code_max] before clamping
  float scale;
  float zero;
  float lo_m, hi_m;  // 1.5 * 2^23 + code_min, 1.5 * 2^23 + code_max: the clamp bounds of fma(w, c, zm)
};

// Asymmetric grid with codes 0 .. qmax (15 or 255) over [clip * min y, clip * max y].
__device__ __forceinline__ TokenGrid token_grid(float lo_w, float hi_w, float rs, float clip, float qmax) {
  // The grid sits on every token's critical path, so it avoids IEEE divisions: scale is the exact
  // fp32 quotient (u - l) / qmax; zero = rne(-l / scale) comes from -l * (1 / scale),
  // which lies within a few ulps of the exact fp32 quotient -- only when that puts it within a
  // guard band of a half-integer could the two round differently, and only then is the exact
  // division taken. 1 / scale itself (for the codes) is the hardware approximation.
  const float lo_y = __fmul_rn(lo_w, rs), hi_y = __fmul_rn(hi_w, rs);
  const float l = __fmul_rn(lo_y, clip), u = __fmul_rn(hi_y, clip);
  TokenGrid tg;
  float inv;
  if (u == l) {
    tg.scale = 1.f;
    tg.zero = rintf(-l);
    inv = 1.f;
  } else {
    const float d = __fsub_rn(u, l);
    if (qmax == 15.f) {
      // (u - l) / 15 rounded to nearest: x * fp32(1/15) with one FMA correction step, which
      // equals the IEEE quotient for every finite fp32 x except -0 (checked on the GPU over all
      // 2^32 patterns; here x = u - l > 0, and an infinite range keeps its quotient, infinity)
      const float q0 = __fmul_rn(d, 1.0f / 15.0f);
      tg.scale = isinf(d) ? d : __fmaf_rn(__fmaf_rn(-q0, 15.0f, d), 1.0f / 15.0f, q0);
    } else {
      tg.scale = __fdiv_rn(d, qmax);
    }
    asm("rcp.approx.f32 %0, %1;" : "=f"(inv) : "f"(tg.scale));
    const float z0 = __fmul_rn(-l, inv);
    tg.zero = rintf(z0);
    const float off = fabsf(__fsub_rn(z0, tg.zero));      // distance to the nearest integer
    const float guard = fmaf(fabsf(z0), 0x1p-19f, 0x1p-40f);  // ~16 ulps of z0
    if (!(0.5f - off > guard)) tg.zero = rintf(__fdiv_rn(-l, tg.scale));
  }
  tg.c = __fmul_rn(rs, inv);
  tg.zm = __fadd_rn(tg.zero, kMagic);
  tg.lo_m = kMagic;
  tg.hi_m = kMagic + qmax;
  // codes are monotone in w, so the row's extremes decide whether any code needs clamping;
  // a zero-point too large for the 1.5 * 2^23 trick also takes the clamped path
  const int c_lo = static_cast<int>(__float_as_uint(fmaf(lo_w, tg.c, tg.zm)) - __float_as_uint(kMagic));
  const int c_hi = static_cast<int>(__float_as_uint(fmaf(hi_w, tg.c, tg.zm)) - __float_as_uint(kMagic));
  tg.clamp = !(c_lo >= 0 && c_hi <= static_cast<int>(qmax)) || fabsf(tg.zero) > 4194304.f;
  return tg;
}

// Symmetric grid: codes -L .. L (L = 7 or 127), scale = max |y| / L (1 for an all-zero row),
// code = clamp(rne(y / scale), -L, L); no zero-point.
__device__ __forceinline__ TokenGrid token_grid_sym(float lo_w, float hi_w, float rs, float L) {
  const float lo_y = __fmul_rn(lo_w, rs), hi_y = __fmul_rn(hi_w, rs);
  const float amax = fmaxf(fabsf(lo_y), fabsf(hi_y));
  TokenGrid tg;
  tg.scale = amax == 0.f ? 1.f : __fdiv_rn(amax, L);
  float inv;
  asm("rcp.approx.f32 %0, %1;" : "=f"(inv) : "f"(tg.scale));
  tg.c = __fmul_rn(rs, inv);
  tg.zero = 0.f;
  tg.zm = kMagic;
  tg.lo_m = kMagic - L;
  tg.hi_m = kMagic + L;
  const int c_lo = static_cast<int>(__float_as_uint(fmaf(lo_w, tg.c, kMagic)) - __float_as_uint(kMagic));
  const int c_hi = static_cast<int>(__float_as_uint(fmaf(hi_w, tg.c, kMagic)) - __float_as_uint(kMagic));
  tg.clamp = !(c_lo >= -static_cast<int>(L) && c_hi <= static_cast<int>(L));
  return tg;
}

// What a fused kernel writes per token: the check path's fp32 y, or codes of one grid.
enum : int { kModeY = 0, kModeA4 = 1, kModeA8 = 2, kModeS4 = 3, kModeS8 = 4 };
__host__ __device__ constexpr int mode_bits(int m) { return (m == kModeA8 || m == kModeS8) ? 8 : 4; }
__host__ __device__ constexpr bool mode_sym(int m) { return m == kModeS4 || m == kModeS8; }

// The token's grid from its extremes (lo, hi of the raw transform w; y = w / sqrt(n)).
template <int kMode>
__device__ __forceinline__ TokenGrid mode_grid(float lo, float hi, const TcParams& p) {
  constexpr int kBits = mode_bits(kMode);
  return mode_sym(kMode) ? token_grid_sym(lo, hi, p.inv_sqrt_n, kBits == 4 ? 7.f : 127.f)
                         : token_grid(lo, hi, p.inv_sqrt_n, p.clip, kBits == 4 ? 15.f : 255.f);
}

// One thread's run of 2 * kPairs output channels starting at channel j0: codes on grid g (or y).
// sneg / odd_neg: every output / every odd column comes out of the transform negated (see
// rotq_stream_kernel).
template <int kPairs, int kMode>
__device__ __forceinline__ void emit_run(const float2 (&v)[kPairs], const TokenGrid& g, bool sneg, bool odd_neg,
                                         bool active, const TcParams& p, int t, int64_t j0) {
  if (!active) return;
  const float rs = p.inv_sqrt_n;
  if constexpr (kMode == kModeY) {
    store_y<kPairs>(v, sneg ? -rs : rs, p.y + static_cast<int64_t>(t) * p.ldy + j0, (sneg != odd_neg) ? -rs : rs);
  } else {
    constexpr int kBits = mode_bits(kMode);
    quant_store<kPairs, kBits, mode_sym(kMode)>(
        v, make_float2(sneg ? -g.c : g.c, (sneg != odd_neg) ? -g.c : g.c), g.zm, g.clamp, g.lo_m, g.hi_m,
        p.q + static_cast<int64_t>(t) * (p.n * kBits / 8) + j0 * kBits / 8);
  }
}

// The end of one token for one thread's run of 2 * kPairs output channels starting at channel j0:
// grid from the token's extremes, codes (or y) stored. writer: this thread also stores the
// token's scale and zero-point.
template <int kPairs, int kMode>
__device__ __forceinline__ void finish_token(const float2 (&v)[kPairs], float lo, float hi, bool sneg, bool odd_neg,
                                             bool active, bool writer, const TcParams& p, int t, int64_t j0) {
  TokenGrid g{};
  if constexpr (kMode != kModeY) {
    g = mode_grid<kMode>(lo, hi, p);
    if (writer) {
      p.scale[t] = g.scale;
      if (!mode_sym(kMode)) p.zero[t] = g.zero;
    }
  }
  emit_run<kPairs, kMode>(v, g, sneg, odd_neg, active, p, t, j0);
}

// ------------------------------------------------------------- the top column bit on the MMA
//
// Y_h = A B_0 + (-1)^h A B_1 for h = 0, 1, where B_g is the g-th column half of the staged tile
// (kHalfBytes apart; kLbo is the tile's stride between 64-column blocks) and each Y_h has its own
// TMEM accumulator (d_tmem + h * n_half columns): the column butterfly on the top bit, done
// inside the fp32 accumulation. -B comes from the descriptor's negate-B bit (exact). Within each
// accumulator, the half holding input columns 0 .. half - 1 (g_first) goes first at every K
// step: when the outlier permutation swaps the halves, Y_1 is then accumulated as the term by
// term negation of its unswapped sum, and the swap stays an exact sign flip.
template <int kKSteps, uint32_t kHalfBytes, uint32_t kLbo>
__device__ __forceinline__ void fold_mmas(uint32_t d_tmem, uint32_t n_half, uint32_t a_base, uint32_t b_base,
                                          int g_first, uint32_t idesc) {
  constexpr uint32_t kNegB = 1u << 14;
  const uint32_t b_first = b_base + static_cast<uint32_t>(g_first) * kHalfBytes;
  const uint32_t b_second = b_base + static_cast<uint32_t>(g_first ^ 1) * kHalfBytes;
  const uint32_t id_first1 = g_first ? idesc | kNegB : idesc, id_second1 = g_first ? idesc : idesc | kNegB;
#pragma unroll
  for (int ks = 0; ks < kKSteps; ++ks) {
    const uint64_t ad = smem_desc(a_base + (ks >> 2) * 16384 + (ks & 3) * 32, 16, 1024);
    const uint64_t b0 = smem_desc(b_first + ks * 2048, kLbo, 1024);
    const uint64_t b1 = smem_desc(b_second + ks * 2048, kLbo, 1024);
    mma_bf16(d_tmem, ad, b0, idesc, ks > 0 ? 1u : 0u);
    mma_bf16(d_tmem, ad, b1, idesc, 1u);
    mma_bf16(d_tmem + n_half, ad, b0, id_first1, ks > 0 ? 1u : 0u);
    mma_bf16(d_tmem + n_half, ad, b1, id_second1, 1u);
  }
}

// ------------------------------------------------------------------------------------- kernel

// ------------------------------------------------------------- streamed variant (<= 128 columns)
//
// mbar_wait by every lane of the warp, with one verdict for all of them (a lane whose wait ran out
// makes the whole warp leave its loop together).
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity) {
  return __all_sync(0xffffffffu, mbar_wait(bar, parity));
}

// The same pipeline with the token row fetched by plain 1-D bulk copies into a linear shared-
// memory ring (the tensor-map boxes above gather 16 separate 128-byte pieces each, which streams
// ~14% slower from HBM). Three D-pass warps each own a third of the row: they stream it in with
// their own bulk copies and do the whole layout change in one read and one write per 16-byte chunk
// (linear row -> XOR D -> column permutation -> the MMA's swizzled tile), with their D sign masks
// and destinations held in registers, refilling their part of a ring slot as soon as they have
// converted it. A fourth warp issues the MMAs; three tiles let the D warps run two tokens ahead of
// it. Twelve warps in all: a thirteenth would cap every thread at 128 registers.

constexpr int kStreamDWarps = 3;
constexpr int kStreamTiles = 3;
__host__ __device__ constexpr int stream_threads(int ncol) { return 32 * (4 * epi_groups(ncol) + kStreamDWarps + 1); }

template <int kNcol, bool kF28, bool kVecSign, int kMode, int kTok>
__global__ void __launch_bounds__(stream_threads(kNcol), 1) rotq_stream_kernel(TcParams p) {
  static_assert(kNcol <= 128, "the streamed variant keeps a token's lane line in registers");
  // kTok tokens share one MMA tile (short rows): token v of a tile owns tile columns
  // [v * kTokCols, (v + 1) * kTokCols) and the same K rows; kTok = 1 is one token per tile.
  static_assert(kTok == 1 || (kNcol == 128 && kTok == 4), "tile of 128 columns for short rows");
  constexpr int kTokCols = kNcol / kTok;
  constexpr int kTokPairs = kTokCols / 2;
  constexpr int kKRows = kF28 ? 112 : 128;
  constexpr int kKSteps = kKRows / 16;
  constexpr int kChunksN = kNcol / 64;
  constexpr uint32_t kChunkBytes = kKRows * 128;
  constexpr uint32_t kRowBytes = kChunksN * kChunkBytes;  // = 2n: one bf16 token row
  constexpr int kRowChunks = static_cast<int>(kRowBytes / 16);
  constexpr int kTokChunks = kRowChunks / kTok;            // one token's row
  constexpr int kDW = kStreamDWarps;
  constexpr int kLaneChunks = kRowChunks / 32;             // chunks per lane position, over all D warps
  static_assert(kRowChunks % 32 == 0, "D-pass lanes own whole chunks");
  constexpr int kPerD = (kLaneChunks + kDW - 1) / kDW;     // D warp w: kPerD or kPerD - 1 per lane
  constexpr int kDBatch = 7;
  constexpr int kPairs = kNcol / 2;
  constexpr uint32_t kIdesc = (1u << 4) | (1u << 7) | (1u << 10) | (1u << 16) |
                              (static_cast<uint32_t>(kNcol >> 3) << 17) | (static_cast<uint32_t>(128 >> 4) << 24);
  constexpr int kGroups = epi_groups(kNcol);
  constexpr int kEpiWarps = 4 * kGroups;  // warps [0, kEpiWarps): epilogue
  constexpr int kDWarp0 = kEpiWarps;      // then the D warps and the MMA warp
  constexpr int kMmaWarp = kDWarp0 + kDW;
  constexpr int kThreads = stream_threads(kNcol);
  constexpr int kTBufs = 2 * kGroups;
  constexpr int kTiles = kStreamTiles;
  constexpr uint32_t kTmemCols = kTBufs * kNcol < 32 ? 32 : kTBufs * kNcol;
  static_assert(kTBufs * kNcol <= 512, "TMEM holds 512 columns");

  extern __shared__ uint8_t smem_raw[];
  // 1024-byte aligned base for the 128-byte swizzle atoms; offsetting the pointer (not casting
  // through an integer) keeps the compiler's knowledge that every access below is to shared memory
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const int S = p.stages;
  uint8_t* a_smem = smem;
  uint8_t* btile = smem + kABytes;             // kTiles swizzled MMA tiles
  uint8_t* lin = btile + kTiles * kRowBytes;   // S linear rows
  uint64_t* bars = reinterpret_cast<uint64_t*>(lin + S * kRowBytes);
  uint64_t* lfull = bars;                      // [slot][D warp]
  uint64_t* bfull = bars + S * kDW;            // [tile]
  uint64_t* bempty = bfull + kTiles;
  uint64_t* tfull = bempty + kTiles;           // [TMEM buffer]
  uint64_t* tempty = tfull + kTBufs;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tempty + kTBufs);
  float* red = reinterpret_cast<float*>(tmem_slot + 4);  // [buffer][4 quadrants][token][lo, hi]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int i = 0; i < S * kDW; ++i) mbar_init(smem_u32(&lfull[i]), 1);
    for (int i = 0; i < kTiles; ++i) {
      mbar_init(smem_u32(&bfull[i]), kDW);
      mbar_init(smem_u32(&bempty[i]), 1);
    }
    for (int i = 0; i < kTBufs; ++i) {
      mbar_init(smem_u32(&tfull[i]), 1);
      mbar_init(smem_u32(&tempty[i]), 4);
    }
    fence_mbar_init();
  }
  __syncthreads();
  // everything above touched only this CTA's shared memory; inputs may come from the grid before
  griddep_wait();
  griddep_launch_dependents();
  const OutlierRef orf = load_outlier(p);  // issued ahead of the bulk copies
  const int ntiles = (p.T + kTok - 1) / kTok;

  // D warp w's share of the row: lane chunks [c0, c0 + 32 * per) of the kRowChunks
  const bool dwarp = warp >= kDWarp0 && warp < kMmaWarp;
  const int dw = dwarp ? warp - kDWarp0 : 0;
  const int per = kLaneChunks / kDW + (dw < kLaneChunks % kDW ? 1 : 0);
  const int c0 = 32 * (dw * (kLaneChunks / kDW) + (dw < kLaneChunks % kDW ? dw : kLaneChunks % kDW));
  const uint32_t part_bytes = static_cast<uint32_t>(per) * 32u * 16u;
  const char* xpart = static_cast<const char*>(p.xraw) + c0 * 16;
  // one D warp's copy of its share of tile u into ring slot st (one copy per token its share
  // touches; rows past the last token are not read, and their slot bytes are never stored)
  auto stream_in = [&](int st, int u) {
    const uint32_t fb = smem_u32(&lfull[st * kDW + dw]);
    if constexpr (kTok == 1) {
      mbar_arrive_expect_tx(fb, part_bytes);
      bulk_load(smem_u32(lin + st * kRowBytes + c0 * 16), xpart + static_cast<int64_t>(u) * p.ldx * 2, part_bytes, fb);
    } else {
      const int e0 = c0 + 32 * per;
      uint32_t bytes = 0;
#pragma unroll
      for (int v = 0; v < kTok; ++v) {
        const int a = c0 > v * kTokChunks ? c0 : v * kTokChunks;
        const int b = e0 < (v + 1) * kTokChunks ? e0 : (v + 1) * kTokChunks;
        if (a < b && kTok * u + v < p.T) bytes += static_cast<uint32_t>(b - a) * 16u;
      }
      mbar_arrive_expect_tx(fb, bytes);
#pragma unroll
      for (int v = 0; v < kTok; ++v) {
        const int a = c0 > v * kTokChunks ? c0 : v * kTokChunks;
        const int b = e0 < (v + 1) * kTokChunks ? e0 : (v + 1) * kTokChunks;
        const int t = kTok * u + v;
        if (a < b && t < p.T)
          bulk_load(smem_u32(lin + st * kRowBytes + a * 16),
                    static_cast<const char*>(p.xraw) + static_cast<int64_t>(t) * p.ldx * 2 + (a - v * kTokChunks) * 16,
                    static_cast<uint32_t>(b - a) * 16u, fb);
      }
    }
  };
  // The D warps' sign words are loaded (8 bytes per chunk when D is 8-byte aligned) before the
  // bulk copies are issued, so that they do not queue behind every CTA's first copies; the mask
  // arithmetic on them comes after the copies are on their way.
  const int M = kF28 ? (1 << p.logM) : 0;
  const bool last = per == kPerD;  // this warp also takes its lanes' kPerD-th chunk
  const bool d_aligned = (reinterpret_cast<uintptr_t>(p.d) & 7u) == 0;
  uint2 draw[kPerD];
  if (dwarp && d_aligned) {
#pragma unroll
    for (int u = 0; u < kPerD; ++u) {
      const int L = (u < per ? c0 + 32 * u : c0) + lane;
      const int Lt = L % kTokChunks;  // chunk within its token's row
      const int k = Lt / (kTokCols / 8), b0 = (Lt % (kTokCols / 8)) * 8;
      const int j0 = kF28 ? (k >> 2) * M + (k & 3) * kTokCols + b0 : k * kTokCols + b0;
      draw[u] = *reinterpret_cast<const uint2*>(p.d + j0);
    }
  }
  int issued = 0;  // bulk copies this D warp has started (lane 0)
  if (dwarp && lane == 0) {
    for (int st = 0; st < S; ++st) {
      const int u = blockIdx.x + st * gridDim.x;
      if (u >= ntiles) break;
      stream_in(st, u);
      ++issued;
    }
  }

  const SignPlan sp = make_plan<kF28, kTokCols>(p, orf);
  const uint32_t col_xor = sp.active ? sp.e_lo : 0u;
  uint4 mask[kPerD];
  uint32_t dst[kPerD];
  // Short rows (several tokens per tile) with an outlier plan: the outlier channel k is left out of
  // the MMA (its element is zeroed in the tile) and its exact contribution, sgn(x_k) x_{t,k} on
  // every sign-adjusted output, is added once after the butterflies. The massive value then never
  // passes through the fp32 sums, whose rounding at its magnitude would otherwise move a row's
  // codes near rounding ties. kill[v]: byte offset in the tile of token v's element k when this
  // lane writes it, else ~0.
  // kill, packed: bits 0-15 the element's byte offset in its chunk row (K row * 128 + offset inside
  // the 16-byte chunk), bits 16-17 the permuted chunk within the token's 32 columns, bits 18-20
  // the K row's swizzle phase, bits 24+ one bit per token v whose element k this lane writes.
  uint32_t kill = 0;
  if (kTok > 1 && dwarp && sp.active) {
    const int kk = orf.k;
    const int rk = kF28 ? 4 * (kk >> p.logM) + ((kk & (M - 1)) / kTokCols) : kk / kTokCols;  // K row
    const int bk = kk % kTokCols;                                                            // input column
    const int ltk = rk * (kTokCols / 8) + (bk >> 3);                                         // chunk in its row
    const int kw = static_cast<int>((col_xor >> 1) & 3u), ek = bk & 7;
    static_assert(kTok == 1 || kTokCols == 32, "packed kill state assumes 32-column tokens");
#pragma unroll
    for (int v = 0; v < kTok; ++v) {
      const int L = v * kTokChunks + ltk;
      if (L >= c0 && L < c0 + 32 * per && (L - c0) % 32 == lane) kill |= 1u << (24 + v);
    }
    const uint32_t col = static_cast<uint32_t>((bk & ~7) ^ static_cast<int>(col_xor & ~7u));  // < 32
    kill |= static_cast<uint32_t>(rk * 128 + ((((ek >> 1) ^ kw) << 2) | ((ek & 1) << 1))) | ((col >> 3) << 16) |
            ((static_cast<uint32_t>(rk) & 7u) << 18);
  }
  if (dwarp) {
#pragma unroll
    for (int u = 0; u < kPerD; ++u) {
      const int L = (u < per ? c0 + 32 * u : c0) + lane;
      const int Lt = L % kTokChunks, vtok = L / kTokChunks;
      const int k = Lt / (kTokCols / 8), b0 = (Lt % (kTokCols / 8)) * 8;
      const int j0 = kF28 ? (k >> 2) * M + (k & 3) * kTokCols + b0 : k * kTokCols + b0;
      if (d_aligned) {
        asm volatile("" : "+r"(draw[u].x), "+r"(draw[u].y));  // keeps the use after the copies
        mask[u] = chunk_sign_masks(draw[u]);
      } else {
        mask[u] = chunk_sign_masks(p.d + j0);
      }
      const int bp = vtok * kTokCols + (b0 ^ static_cast<int>(col_xor & ~7u));  // where this chunk's columns go
      const int nbp = bp >> 6, segp = (bp >> 3) & 7;
      dst[u] = static_cast<uint32_t>(nbp) * kChunkBytes + k * 128 + ((segp ^ (k & 7)) << 4);
    }
  } else {
    // ... while the other warps build A: rowsign (.) (H_28 kron H_4) or rowsign (.) H_128, K-major SW128
    const int a_tid = threadIdx.x < kDWarp0 * 32 ? threadIdx.x : threadIdx.x - kDW * 32;
    for (int idx = a_tid; idx < 128 * 16; idx += kThreads - kDW * 32) {
      const int m = idx >> 4, j = idx & 15;
      *reinterpret_cast<uint4*>(a_smem + a_offset(m, 8 * j)) = a_chunk<kF28>(m, j, sp, p.h);
    }
  }
  if (warp == kMmaWarp) {
    tmem_alloc(smem_u32(tmem_slot), kTmemCols);
    tmem_relinquish();
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == kMmaWarp) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t a_base = smem_u32(a_smem);
      int i = 0;
      for (int u = blockIdx.x; u < ntiles; u += gridDim.x, ++i) {
        const int bb = i % kTiles, tb = i % kTBufs;
        if (!mbar_wait(smem_u32(&bfull[bb]), (i / kTiles) & 1) ||
            !mbar_wait(smem_u32(&tempty[tb]), ((i / kTBufs) & 1) ^ 1)) {
          flag_error();
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + tb * kNcol;
        const uint32_t b_base = smem_u32(btile + bb * kRowBytes);
#pragma unroll
        for (int ks = 0; ks < kKSteps; ++ks) {
          const uint64_t ad = smem_desc(a_base + (ks >> 2) * 16384 + (ks & 3) * 32, 16, 1024);
          const uint64_t bd = smem_desc(b_base + ks * 2048, kChunkBytes, 1024);
          mma_bf16(d_tmem, ad, bd, kIdesc, ks > 0 ? 1u : 0u);
        }
        mma_commit(smem_u32(&bempty[bb]));
        mma_commit(smem_u32(&tfull[tb]));
      }
      // the last MMAs finish before the TMEM is freed
      if (i > 0 && !mbar_wait(smem_u32(&tfull[(i - 1) % kTBufs]), ((i - 1) / kTBufs) & 1)) flag_error();
    }
  } else if (dwarp) {
    // ------------------------------------------------------------------ D pass: linear -> tile
    int i = 0;
    for (int u = blockIdx.x; u < ntiles; u += gridDim.x, ++i) {
      const int st = i % S, bb = i % kTiles;
      if (!warp_wait(smem_u32(&lfull[st * kDW + dw]), (i / S) & 1) ||
          !warp_wait(smem_u32(&bempty[bb]), ((i / kTiles) & 1) ^ 1)) {
        flag_error();
        break;
      }
      const uint4* src = reinterpret_cast<const uint4*>(lin + st * kRowBytes) + c0 + lane;
      uint8_t* tile = btile + bb * kRowBytes;
      switch ((col_xor >> 1) & 3u) {
        case 0: stream_d_pass<0, kPerD, kDBatch>(src, tile, mask, dst, last); break;
        case 1: stream_d_pass<1, kPerD, kDBatch>(src, tile, mask, dst, last); break;
        case 2: stream_d_pass<2, kPerD, kDBatch>(src, tile, mask, dst, last); break;
        default: stream_d_pass<3, kPerD, kDBatch>(src, tile, mask, dst, last); break;
      }
      if constexpr (kTok > 1) {
#pragma unroll
        for (int v = 0; v < kTok; ++v) {
          if ((kill >> (24 + v)) & 1u) {  // the chunk was written above by this lane
            // token v's 32 columns start at column 32 v: 64-column block v / 2, 16-byte slot 4 (v % 2)
            const uint32_t segp = 4u * (v & 1) + ((kill >> 16) & 3u);
            *reinterpret_cast<uint16_t*>(tile + (v >> 1) * kChunkBytes + (kill & 0xffffu) +
                                         ((segp ^ ((kill >> 18) & 7u)) << 4)) = 0;
          }
        }
      }
      // the tile writes must reach the MMA (async proxy), and this slot's reads must be done
      // before the next bulk copy overwrites it
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(smem_u32(&bfull[bb]));
        const int un = u + S * gridDim.x;
        if (un < ntiles) {
          stream_in(st, un);
          ++issued;
        }
      }
    }
    if (lane == 0) {
      // on an early exit, let this warp's copies still in flight land before the CTA ends
      for (int j = i; j < issued; ++j)
        if (!mbar_wait(smem_u32(&lfull[(j % S) * kDW + dw]), (j / S) & 1)) { flag_error(); break; }
    }
  } else {
    // ------------------------------------------------------------------ epilogue
    const int quad = warp & 3, group = warp >> 2;
    const bool active = !kF28 || lane < 28;
    // this thread's run of kTokCols output channels (the same channels in every token of a tile)
    const int64_t j0 = kF28 ? static_cast<int64_t>(lane) * M + quad * kTokCols
                            : static_cast<int64_t>(quad * 32 + lane) * kTokCols;
    uint32_t sbits[kVecSign ? kNcol / 32 : 1];
    if (kVecSign) {
#pragma unroll
      for (int w = 0; w < kNcol / 32; ++w) {
        uint32_t b = 0;
        if (active)
          for (int r = 0; r < 32; ++r) b |= (p.s[j0 + (32 * w + r) % kTokCols] < 0 ? 1u : 0u) << r;
        sbits[w] = b;
      }
    }
    // the outlier permutation's bit 0 is not applied to the input: every odd column of the
    // transform comes out negated (H P_1 = diag((-1)^j) H), which min/max and quantization undo
    const bool sneg = outlier_sigma_neg(p, sp, orf);  // every output negated
    const bool odd_neg = (col_xor & 1u) != 0;
    // A warp whose wait runs out stops working but keeps taking its group's barrier, once per tile
    // like the others, so that no warp of the group is left waiting there.
    bool live = true;
    int i = group;
    for (int u = blockIdx.x + group * gridDim.x; u < ntiles; u += kGroups * gridDim.x, i += kGroups) {
      const int tb = i % kTBufs;
      if (live && !warp_wait(smem_u32(&tfull[tb]), (i / kTBufs) & 1)) {
        flag_error();
        live = false;
      }
      if (!live) {
        named_barrier_sync(1 + group, 128);
        continue;
      }
      tc_fence_after();
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(quad * 32) << 16) + tb * kNcol;
      float2 v[kPairs];
      tmem_load_pairs<0, kPairs>(taddr, v);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&tempty[tb]));
      fwht_local<kPairs, (kTokCols == 16 ? 4 : (kTokCols == 32 ? 5 : (kTokCols == 64 ? 6 : 7)))>(v);
      if (kVecSign) apply_sign_bits<kPairs>(v, sbits);
      // short rows: the tokens' outlier values, left out of the MMA (see kill); their contribution
      // sgn(x_k) x_{t,k} to every sign-adjusted output is added after the extremes are known
      float dlt[kTok];
#pragma unroll
      for (int tk = 0; tk < kTok; ++tk) {
        const int t = kTok * u + tk;
        dlt[tk] = 0.f;
        if (kTok > 1 && sp.active && t < p.T) {
          const float xv = __uint_as_float(
              static_cast<uint32_t>(reinterpret_cast<const uint16_t*>(p.xraw)[static_cast<int64_t>(t) * p.ldx + orf.k]) << 16);
          dlt[tk] = orf.xk < 0.f ? -xv : xv;
        }
      }
      float lo[kTok], hi[kTok];
#pragma unroll
      for (int tk = 0; tk < kTok; ++tk) {
        lo[tk] = pos_inf();
        hi[tk] = -pos_inf();
        if (active) {
          float lx, hx, ly, hy;
          local_minmax_xy<kTokPairs>(*reinterpret_cast<const float2(*)[kTokPairs]>(v + tk * kTokPairs), lx, hx, ly, hy);
          lo[tk] = fminf(lx, odd_neg ? -hy : ly);
          hi[tk] = fmaxf(hx, odd_neg ? -ly : hy);
        }
        lo[tk] = warp_min(lo[tk]);
        hi[tk] = warp_max(hi[tk]);
      }
      float* rb = red + (tb * 4) * kTok * 2;  // [quadrant][token][lo, hi] of this buffer
      if (lane == 0) {
#pragma unroll
        for (int tk = 0; tk < kTok; ++tk) {
          rb[(quad * kTok + tk) * 2] = lo[tk];
          rb[(quad * kTok + tk) * 2 + 1] = hi[tk];
        }
      }
      named_barrier_sync(1 + group, 128);  // the group's four quadrant extremes are in
#pragma unroll
      for (int tk = 0; tk < kTok; ++tk) {
#pragma unroll
        for (int w = 0; w < 4; ++w) {
          lo[tk] = fminf(lo[tk], rb[(w * kTok + tk) * 2]);
          hi[tk] = fmaxf(hi[tk], rb[(w * kTok + tk) * 2 + 1]);
        }
        if (sneg) {
          const float t_lo = lo[tk];
          lo[tk] = -hi[tk];
          hi[tk] = -t_lo;
        }
        if constexpr (kTok > 1) {
          // each output rounds once, RN(v + shift); rounding is monotone, so the extremes shift alike
          lo[tk] = __fadd_rn(lo[tk], dlt[tk]);
          hi[tk] = __fadd_rn(hi[tk], dlt[tk]);
          const float2 d2 = make_float2(sneg ? -dlt[tk] : dlt[tk], (sneg != odd_neg) ? -dlt[tk] : dlt[tk]);
#pragma unroll
          for (int i = 0; i < kTokPairs; ++i) v[tk * kTokPairs + i] = __fadd2_rn(v[tk * kTokPairs + i], d2);
        }
        const int t = kTok * u + tk;
        if (t < p.T)
          finish_token<kTokPairs, kMode>(*reinterpret_cast<const float2(*)[kTokPairs]>(v + tk * kTokPairs), lo[tk],
                                         hi[tk], sneg, odd_neg, active, quad == 0 && lane == 0, p, t, j0);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

// ------------------------------------------------------------------ 256 columns: half-row epilogue
//
// A 256-column row per token is 56-64 KB, so the input is staged by tensor-map TMA boxes straight
// into the swizzled MMA tile (three stages fit beside A), and two D warps convert each stage in
// place: sign flips, the word permutation, and the permutation of the 16-byte slots inside each
// 128-byte row (column bits 3-5; bits 6-7 pick the TMA box, bit 0 is folded into the epilogue).
// The column butterfly on bit 7 runs on the tensor cores too: two N = 128 MMA chains per token,
// each accumulating over both 128-column halves of the tile, write Y_0 = A X_0 + A X_1 and
// Y_1 = A X_0 - A X_1 to TMEM (twice the MMA work of one N = 256 chain, which the tensor pipe has
// to spare, for one fewer add per value and a single TMEM load per thread). Eight epilogue
// warps share a token: the warp for half h and lane quadrant q loads its 128 values of Y_h, then
// runs the remaining seven butterfly stages, min/max, the 8-warp exchange and quantization. (A token's 28,672-32,768 fp32 values fill the register file, so two tokens' epilogues
// cannot overlap here; a version with two groups of four warps on alternate tokens, each parking
// half of its 256-column line in TMEM, held the TMEM buffer through the whole epilogue and ran
// slower: 40 % of the HBM roofline against 50 % at n = 28672.)

constexpr int kWideEpiWarps = 8;
constexpr int kWideDWarps = 2;
constexpr int kWideThreads = 32 * (kWideEpiWarps + kWideDWarps + 2);
constexpr int kWideTBufs = 2;

// One stage of the in-place D pass (packed sign words, see chunk_sign_bits): chunk ch is read,
// its signs flipped and words moved by kW, and written to slot ch ^ seg_xor of the same 128-byte
// row. A row's 8 chunks belong to 8 lanes of one warp and one batch, read before any is written.
template <int kW, int kPerD, int kDT, int kBatch>
__device__ __forceinline__ void inplace_d_pass_bits(uint4* base, const uint32_t (&bits_in)[kPerD], int td,
                                                    uint32_t seg_xor) {
  uint32_t bits[kPerD];
#pragma unroll
  for (int u = 0; u < kPerD; ++u) {
    bits[u] = bits_in[u];
    asm volatile("" : "+r"(bits[u]));
  }
#pragma unroll
  for (int u0 = 0; u0 < kPerD; u0 += kBatch) {
    uint4 v[kBatch];
#pragma unroll
    for (int b = 0; b < kBatch; ++b)
      if (u0 + b < kPerD) v[b] = base[(u0 + b) * kDT + td];
    __syncwarp();
#pragma unroll
    for (int b = 0; b < kBatch; ++b) {
      if (u0 + b < kPerD) {
        const uint32_t m = bits[u0 + b];
        const uint32_t w[4] = {v[b].x ^ (m & 0x80008000u), v[b].y ^ ((m << 1) & 0x80008000u),
                               v[b].z ^ ((m << 2) & 0x80008000u), v[b].w ^ ((m << 3) & 0x80008000u)};
        base[((u0 + b) * kDT + td) ^ static_cast<int>(seg_xor)] = make_uint4(w[kW], w[1 ^ kW], w[2 ^ kW], w[3 ^ kW]);
      }
    }
    __syncwarp();
  }
}

template <bool kF28, bool kVecSign, int kMode>
__global__ void __launch_bounds__(kWideThreads, 1) rotq_wide_kernel(const __grid_constant__ CUtensorMap tmap,
                                                                    TcParams p) {
  constexpr int kNcol = 256, kHalf = 128, kPairs = 64;
  constexpr int kKRows = kF28 ? 112 : 128;
  constexpr int kKSteps = kKRows / 16;
  constexpr int kChunksN = kNcol / 64;
  constexpr int kBoxesPerChunk = kKRows / 16;
  constexpr uint32_t kChunkBytes = kKRows * 128;
  constexpr uint32_t kStageBytes = kChunksN * kChunkBytes;
  constexpr int kStageChunks = static_cast<int>(kStageBytes / 16);
  constexpr int kDT = kWideDWarps * 32;
  constexpr int kPerD = kStageChunks / kDT;
  static_assert(kStageChunks % kDT == 0, "D lanes own whole chunks");
  constexpr int kDBatch = 4;
  constexpr uint32_t kIdesc = (1u << 4) | (1u << 7) | (1u << 10) | (1u << 16) |
                              (static_cast<uint32_t>(kHalf >> 3) << 17) | (static_cast<uint32_t>(128 >> 4) << 24);
  constexpr int kDWarp0 = kWideEpiWarps;
  constexpr int kTmaWarp = kDWarp0 + kWideDWarps;
  constexpr int kMmaWarp = kTmaWarp + 1;
  constexpr int kThreads = kWideThreads;
  constexpr int kTBufs = kWideTBufs;
  constexpr uint32_t kTmemCols = kTBufs * kNcol;
  static_assert(kTmemCols <= 512, "TMEM holds 512 columns");

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const int S = p.stages;
  uint8_t* a_smem = smem;
  uint8_t* ring = smem + kABytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(ring + S * kStageBytes);
  uint64_t* full = bars;
  uint64_t* dready = bars + S;
  uint64_t* empty = bars + 2 * S;
  uint64_t* tfull = bars + 3 * S;
  uint64_t* tempty = tfull + kTBufs;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tempty + kTBufs);
  float* red = reinterpret_cast<float*>(tmem_slot + 4);  // [token parity][half][quadrant][lo, hi]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  griddep_wait();  // inputs may come from the grid before
  griddep_launch_dependents();
  const OutlierRef orf = load_outlier(p);
  const SignPlan sp = make_plan<kF28, kNcol>(p, orf);
  const uint32_t col_xor = sp.active ? sp.e_lo : 0u;
  const uint32_t seg_xor = (col_xor >> 3) & 7u;
  const int box_xor = static_cast<int>(col_xor >> 6);
  const int M = kF28 ? (1 << p.logM) : 0;

  if (threadIdx.x == 0) {
    for (int i = 0; i < S; ++i) {
      mbar_init(smem_u32(&full[i]), 1);
      mbar_init(smem_u32(&dready[i]), kWideDWarps);
      mbar_init(smem_u32(&empty[i]), 1);
    }
    for (int i = 0; i < kTBufs; ++i) {
      mbar_init(smem_u32(&tfull[i]), 1);
      mbar_init(smem_u32(&tempty[i]), kWideEpiWarps);
    }
    fence_mbar_init();
  }
  const bool dwarp = warp >= kDWarp0 && warp < kTmaWarp;
  const int td = threadIdx.x - kDWarp0 * 32;
  uint32_t bits[kPerD];
  const bool d_aligned = (reinterpret_cast<uintptr_t>(p.d) & 7u) == 0;
  if (dwarp) {
    // D signs of this lane's chunks, in the staged tile's order: chunk ch holds row (K index)
    // ch % (kKRows * 8) / 8, input columns of box (nb ^ box_xor), segment (slot ^ row) & 7
#pragma unroll
    for (int u = 0; u < kPerD; ++u) {
      const int ch = u * kDT + td;
      const int nb = ch / (kKRows * 8), rem = ch % (kKRows * 8);
      const int row = rem >> 3, slot = rem & 7;
      const int b0 = (nb ^ box_xor) * 64 + ((slot ^ (row & 7)) << 3);
      const int j0 = kF28 ? (row >> 2) * M + (row & 3) * kNcol + b0 : row * kNcol + b0;
      uint32_t b = 0;
      if (d_aligned) {
        const uint2 w = *reinterpret_cast<const uint2*>(p.d + j0);  // 8 signs in one load
#pragma unroll
        for (int e = 0; e < 8; ++e) b |= (((e < 4 ? w.x : w.y) >> (8 * (e & 3) + 7)) & 1u) << (15 + 16 * (e & 1) - (e >> 1));
      } else {
#pragma unroll
        for (int e = 0; e < 8; ++e) b |= (p.d[j0 + e] < 0 ? 1u : 0u) << (15 + 16 * (e & 1) - (e >> 1));
      }
      bits[u] = b;
    }
  } else {
    const int a_tid = threadIdx.x < kDWarp0 * 32 ? threadIdx.x : threadIdx.x - kWideDWarps * 32;
    for (int idx = a_tid; idx < 128 * 16; idx += kThreads - kWideDWarps * 32) {
      const int m = idx >> 4, j = idx & 15;
      *reinterpret_cast<uint4*>(a_smem + a_offset(m, 8 * j)) = a_chunk<kF28>(m, j, sp, p.h);
    }
  }
  if (warp == kMmaWarp) {
    tmem_alloc(smem_u32(tmem_slot), kTmemCols);
    tmem_relinquish();
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == kTmaWarp) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      prefetch_tmap(&tmap);
      int i = 0;
      for (int t = blockIdx.x; t < p.T; t += gridDim.x, ++i) {
        const int st = i % S;
        if (!mbar_wait(smem_u32(&empty[st]), ((i / S) & 1) ^ 1)) { flag_error(); break; }
        const uint32_t fb = smem_u32(&full[st]);
        mbar_arrive_expect_tx(fb, kStageBytes);
        const uint32_t dst0 = smem_u32(ring + st * kStageBytes);
#pragma unroll 1
        for (int nb = 0; nb < kChunksN; ++nb) {
#pragma unroll 1
          for (int bx = 0; bx < kBoxesPerChunk; ++bx) {
            const uint32_t dst = dst0 + nb * kChunkBytes + bx * kBoxBytes;
            if (kF28)
              tma_load_4d(dst, &tmap, (nb ^ box_xor) * 64, 0, bx * 4, t, fb);
            else
              tma_load_3d(dst, &tmap, (nb ^ box_xor) * 64, bx * 16, t, fb);
          }
        }
      }
      // do not leave the CTA with copies in flight: wait (bounded) for the last stages issued
      const int issued = i;
      for (int j = issued - S > 0 ? issued - S : 0; j < issued; ++j)
        if (!mbar_wait(smem_u32(&full[j % S]), (j / S) & 1)) { flag_error(); break; }
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t a_base = smem_u32(a_smem);
      const int g_first = box_xor >> 1;  // the tile half that holds input columns 0..127
      int i = 0;
      for (int t = blockIdx.x; t < p.T; t += gridDim.x, ++i) {
        const int st = i % S, tb = i % kTBufs;
        if (!mbar_wait(smem_u32(&dready[st]), (i / S) & 1) ||
            !mbar_wait(smem_u32(&tempty[tb]), ((i / kTBufs) & 1) ^ 1)) {
          flag_error();
          break;
        }
        tc_fence_after();
        const uint32_t b_base = smem_u32(ring + st * kStageBytes);
        // Y_h = A B_0 + (-1)^h A B_1 (B_g = tile columns 128g .. 128g + 127), see fold_mmas
        fold_mmas<kKSteps, 2 * kChunkBytes, kChunkBytes>(tmem_base + tb * kNcol, kHalf, a_base, b_base, g_first,
                                                          kIdesc);
        mma_commit(smem_u32(&empty[st]));
        mma_commit(smem_u32(&tfull[tb]));
      }
      if (i > 0 && !mbar_wait(smem_u32(&tfull[(i - 1) % kTBufs]), ((i - 1) / kTBufs) & 1)) flag_error();
    }
  } else if (dwarp) {
    // ------------------------------------------------------------------ D pass, in place
    int i = 0;
    for (int t = blockIdx.x; t < p.T; t += gridDim.x, ++i) {
      const int st = i % S;
      if (!warp_wait(smem_u32(&full[st]), (i / S) & 1)) { flag_error(); break; }
      uint4* base = reinterpret_cast<uint4*>(ring + st * kStageBytes);
      switch ((col_xor >> 1) & 3u) {
        case 0: inplace_d_pass_bits<0, kPerD, kDT, kDBatch>(base, bits, td, seg_xor); break;
        case 1: inplace_d_pass_bits<1, kPerD, kDT, kDBatch>(base, bits, td, seg_xor); break;
        case 2: inplace_d_pass_bits<2, kPerD, kDT, kDBatch>(base, bits, td, seg_xor); break;
        default: inplace_d_pass_bits<3, kPerD, kDT, kDBatch>(base, bits, td, seg_xor); break;
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&dready[st]));
    }
  } else {
    // ------------------------------------------------------------------ epilogue: one half row per thread
    const int quad = warp & 3, half = warp >> 2;
    const bool active = !kF28 || lane < 28;
    const int64_t j0 = (kF28 ? static_cast<int64_t>(lane) * M + quad * kNcol
                             : static_cast<int64_t>(quad * 32 + lane) * kNcol) + half * kHalf;
    uint32_t sbits[kVecSign ? kHalf / 32 : 1];
    if (kVecSign) {
#pragma unroll
      for (int w = 0; w < kHalf / 32; ++w) {
        uint32_t b = 0;
        if (active)
          for (int r = 0; r < 32; ++r) b |= (p.s[j0 + 32 * w + r] < 0 ? 1u : 0u) << r;
        sbits[w] = b;
      }
    }
    const bool sneg = outlier_sigma_neg(p, sp, orf);  // every output negated
    const bool odd_neg = (col_xor & 1u) != 0;  // see rotq_stream_kernel
    bool live = true;
    int i = 0;
    for (int t = blockIdx.x; t < p.T; t += gridDim.x, ++i) {
      const int tb = i % kTBufs;
      if (live && !warp_wait(smem_u32(&tfull[tb]), (i / kTBufs) & 1)) {
        flag_error();
        live = false;
      }
      if (!live) {
        named_barrier_sync(1, 32 * kWideEpiWarps);
        continue;
      }
      tc_fence_after();
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(quad * 32) << 16) + tb * kNcol + half * kHalf;
      float2 v[kPairs];
      tmem_load_pairs<0, kPairs, kPairs>(taddr, v);  // Y_half: one 128-column load, one wait
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&tempty[tb]));
      fwht_local<kPairs, 7>(v);
      if (kVecSign) apply_sign_bits<kPairs>(v, sbits);
      float lo = pos_inf(), hi = -pos_inf();
      if (active) {
        float lx, hx, ly, hy;
        local_minmax_xy<kPairs>(v, lx, hx, ly, hy);
        lo = fminf(lx, odd_neg ? -hy : ly);
        hi = fmaxf(hx, odd_neg ? -ly : hy);
      }
      lo = warp_min(lo);
      hi = warp_max(hi);
      // exchange slots alternate per token: a slot is rewritten only after the next token's
      // barrier, which every epilogue warp passes after reading it
      float* rslot = red + (i & 1) * 16;
      if (lane == 0) {
        rslot[(half * 4 + quad) * 2] = lo;
        rslot[(half * 4 + quad) * 2 + 1] = hi;
      }
      named_barrier_sync(1, 32 * kWideEpiWarps);  // the token's eight partial extremes are in
#pragma unroll
      for (int w = 0; w < 8; ++w) {
        lo = fminf(lo, rslot[w * 2]);
        hi = fmaxf(hi, rslot[w * 2 + 1]);
      }
      if (sneg) {
        const float t_lo = lo;
        lo = -hi;
        hi = -t_lo;
      }
      finish_token<kPairs, kMode>(v, lo, hi, sneg, odd_neg, active, warp == 0 && lane == 0, p, t, j0);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

// ------------------------------------------------------------- short rows: one warp per token
//
// n = 512, 1024, 2048 (F = 1), fp32 or bf16 rows, s in its outlier form (BASELINE config C1:
// n = 1024, fp32, a massive outlier on every token). One warp per token: lane l holds channels
// [l V, l V + V) (V = n / 32); the low log2(V) Walsh stages run in the lane's registers, the five
// high ones across lanes (shfl.xor). The sums are fp64 and y = s w / sqrt(n) is rounded once to
// fp32, so y is the correctly rounded fp32 of the exact rotation up to a rare double rounding.
// That matters for the token's extremes: on rows like C1's every output sits near
// |x_k| / sqrt(n) with a spread of ~1, so |y| / scale reaches ~700, and an extreme one ulp off
// (what fp32 sums give) moves the scale by ~5e-6 and every code by ~3e-3 of a step -- past the
// rounding-tie window on ~1 % of the elements. With fp64 sums the scale is the oracle's.
constexpr int kSmallWarps = 4;

template <int kV, bool kF32In, int kMode>
__global__ void __launch_bounds__(32 * kSmallWarps) rotq_small_kernel(TcParams p) {
  static_assert(kV == 16 || kV == 32 || kV == 64, "512, 1024 or 2048 channels");
  constexpr int kPairs = kV / 2;
  const int lane = threadIdx.x & 31;
  const int gw = static_cast<int>(blockIdx.x) * kSmallWarps + static_cast<int>(threadIdx.x >> 5);
  const int nw = static_cast<int>(gridDim.x) * kSmallWarps;
  griddep_wait();  // inputs may come from the grid before
  griddep_launch_dependents();
  const OutlierRef o = load_outlier(p);
  const int k = o.k;
  if (p.kp != nullptr && (k < 0 || k >= p.n)) flag_error(2u);  // not a channel: no sign adjustment
  const bool pattern = p.kp != nullptr && k >= 0 && k < p.n && o.xk != 0.f;
  const int j0 = lane * kV;
  // D of this lane's channels, and s with 1/sqrt(n) folded in (s_j = sgn(H[j,k] D_k x_k) =
  // (-1)^popcount(j & k) sgn(D_k) sgn(x_k))
  uint64_t dbits = 0, sbits = 0;
#pragma unroll
  for (int v = 0; v < kV; ++v)
    if (p.d[j0 + v] < 0) dbits |= 1ull << v;
  if (pattern) {
    const uint32_t sig = ((o.xk < 0.f) != (p.d[k] < 0)) ? 1u : 0u;
#pragma unroll
    for (int v = 0; v < kV; ++v)
      if (((__popc(static_cast<uint32_t>((j0 + v) & k)) & 1u) ^ sig) != 0u) sbits |= 1ull << v;
  }
  const double rs = 1.0 / sqrt(static_cast<double>(p.n));

  for (int t = gw; t < p.T; t += nw) {
    double a[kV];
    if constexpr (kF32In) {
      const float4* xr = reinterpret_cast<const float4*>(static_cast<const float*>(p.xraw) +
                                                         static_cast<int64_t>(t) * p.ldx + j0);
#pragma unroll
      for (int i = 0; i < kV / 4; ++i) {
        const float4 f = xr[i];
        a[4 * i] = f.x;
        a[4 * i + 1] = f.y;
        a[4 * i + 2] = f.z;
        a[4 * i + 3] = f.w;
      }
    } else {
      const uint4* xr = reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(p.xraw) +
                                                       static_cast<int64_t>(t) * p.ldx + j0);
#pragma unroll
      for (int i = 0; i < kV / 8; ++i) {
        const uint4 w = xr[i];
        const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          a[8 * i + 2 * e] = __uint_as_float(u[e] << 16);
          a[8 * i + 2 * e + 1] = __uint_as_float(u[e] & 0xffff0000u);
        }
      }
    }
#pragma unroll
    for (int v = 0; v < kV; ++v)  // x' = D x
      if ((dbits >> v) & 1ull) a[v] = -a[v];
    // the stages on the lane-local bits of j
#pragma unroll
    for (int h = 1; h < kV; h <<= 1) {
#pragma unroll
      for (int v = 0; v < kV; ++v) {
        if ((v & h) == 0) {
          const double u = a[v], w = a[v + h];
          a[v] = u + w;
          a[v + h] = u - w;
        }
      }
    }
    // the stages on the lane bits: the lower lane keeps u + w, the upper one u - w
#pragma unroll
    for (int b = 0; b < 5; ++b) {
      const bool upper = (lane >> b) & 1;
#pragma unroll
      for (int v = 0; v < kV; ++v) {
        const double w = __shfl_xor_sync(0xffffffffu, a[v], 1 << b);
        a[v] = upper ? w - a[v] : a[v] + w;
      }
    }
    // y = s w / sqrt(n), rounded once to fp32
    float2 y[kPairs];
#pragma unroll
    for (int i = 0; i < kPairs; ++i) {
      const double y0 = ((sbits >> (2 * i)) & 1ull) ? -a[2 * i] * rs : a[2 * i] * rs;
      const double y1 = ((sbits >> (2 * i + 1)) & 1ull) ? -a[2 * i + 1] * rs : a[2 * i + 1] * rs;
      y[i] = make_float2(__double2float_rn(y0), __double2float_rn(y1));
    }
    float lx, hx, ly, hy;
    local_minmax_xy<kPairs>(y, lx, hx, ly, hy);
    const float lo = warp_min(fminf(lx, ly)), hi = warp_max(fmaxf(hx, hy));
    finish_token<kPairs, kMode>(y, lo, hi, false, false, true, lane == 0, p, t, j0);  // p.inv_sqrt_n = 1
  }
}

// ------------------------------------------------------------------------------------- host

// Per kernel instantiation: its shared-memory attribute, set once per device, and the device's SM
// count, queried once per device. Decode-sized calls (a handful of tokens) take a few microseconds
// on the device, so the host side of a launch must not repeat these driver calls every time.
struct KernelSetup {
  static constexpr int kMaxDevices = 64;
  std::atomic<int> sms[kMaxDevices] = {};  // 0 = not prepared on that device yet

  cudaError_t prepare(const void* kern, int smem, int* sms_out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < kMaxDevices) {
      const int cached = sms[dev].load(std::memory_order_acquire);
      if (cached > 0) {
        *sms_out = cached;
        return cudaSuccess;
      }
    }
    if ((e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem)) != cudaSuccess) return e;
    int count = 0;
    if ((e = cudaDeviceGetAttribute(&count, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
    if (dev >= 0 && dev < kMaxDevices) sms[dev].store(count, std::memory_order_release);
    *sms_out = count;
    return cudaSuccess;
  }
};

// Launch with programmatic stream serialization: the kernel may be scheduled while the previous
// kernel in the stream is finishing; it waits (griddepcontrol.wait) before reading any input.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), int grid, int threads, size_t smem, cudaStream_t st, Args&&... args) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(threads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() { return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(tensor_map_encoder()); }

template <bool kF28, bool kVecSign, int kMode>
cudaError_t launch_wide(const CUtensorMap& tmap, const TcParams& p0, cudaStream_t st) {
  constexpr int kKRows = kF28 ? 112 : 128;
  constexpr uint32_t kStageBytes = 4 * kKRows * 128;
  constexpr uint32_t kSmemBudget = 227 * 1024 - 1024 - kABytes - 1024;
  TcParams p = p0;
  p.stages = static_cast<int>(kSmemBudget / kStageBytes);
  if (p.stages > 8) p.stages = 8;
  if (p.stages < 2) return cudaErrorNotSupported;
  const size_t smem = 1024 + kABytes + static_cast<size_t>(p.stages) * kStageBytes + 1024;
  auto kern = rotq_wide_kernel<kF28, kVecSign, kMode>;
  static KernelSetup setup;
  int sms = 0;
  cudaError_t e = setup.prepare(reinterpret_cast<const void*>(kern), static_cast<int>(smem), &sms);
  if (e != cudaSuccess) return e;
  const int grid = p.T < sms ? p.T : sms;
  e = launch_pdl(kern, grid, kWideThreads, smem, st, tmap, p);
  count_launch();
  return e;
}

template <bool kF28, bool kVecSign>
cudaError_t dispatch_wide_mode(const CUtensorMap& tmap, const TcParams& p, int mode, cudaStream_t st) {
  switch (mode) {
    case kModeY: return launch_wide<kF28, kVecSign, kModeY>(tmap, p, st);
    case kModeA4: return launch_wide<kF28, kVecSign, kModeA4>(tmap, p, st);
    case kModeA8: return launch_wide<kF28, kVecSign, kModeA8>(tmap, p, st);
    case kModeS4: return launch_wide<kF28, kVecSign, kModeS4>(tmap, p, st);
    default: return launch_wide<kF28, kVecSign, kModeS8>(tmap, p, st);
  }
}

template <bool kF28>
cudaError_t dispatch_wide(const CUtensorMap& tmap, const TcParams& p, bool vec_sign, int mode, cudaStream_t st) {
  return vec_sign ? dispatch_wide_mode<kF28, true>(tmap, p, mode, st) : dispatch_wide_mode<kF28, false>(tmap, p, mode, st);
}

template <int kNcol, bool kF28, bool kVecSign, int kMode, int kTok>
cudaError_t launch_stream(const TcParams& p0, cudaStream_t st) {
  constexpr int kKRows = kF28 ? 112 : 128;
  constexpr uint32_t kRowBytes = (kNcol / 64) * kKRows * 128;
  constexpr uint32_t kTail = kTok > 1 ? 2048 : 1024;  // barriers, TMEM address, extremes exchange
  constexpr uint32_t kSmemBudget = 227 * 1024 - 1024 - kABytes - kStreamTiles * kRowBytes - kTail;
  TcParams p = p0;
  p.stages = static_cast<int>(kSmemBudget / kRowBytes);
  if (p.stages > 8) p.stages = 8;
  if (p.stages < 2) return cudaErrorNotSupported;
  const size_t smem = 1024 + kABytes + kStreamTiles * kRowBytes + static_cast<size_t>(p.stages) * kRowBytes + kTail;
  auto kern = rotq_stream_kernel<kNcol, kF28, kVecSign, kMode, kTok>;
  static KernelSetup setup;
  int sms = 0;
  cudaError_t e = setup.prepare(reinterpret_cast<const void*>(kern), static_cast<int>(smem), &sms);
  if (e != cudaSuccess) return e;
  const int ntiles = (p.T + kTok - 1) / kTok;
  const int grid = ntiles < sms ? ntiles : sms;
  e = launch_pdl(kern, grid, stream_threads(kNcol), smem, st, p);
  count_launch();
  return e;
}

template <int kNcol, bool kF28, bool kVecSign, int kTok>
cudaError_t dispatch_stream_mode(const TcParams& p, int mode, cudaStream_t st) {
  switch (mode) {
    case kModeY: return launch_stream<kNcol, kF28, kVecSign, kModeY, kTok>(p, st);
    case kModeA4: return launch_stream<kNcol, kF28, kVecSign, kModeA4, kTok>(p, st);
    case kModeA8: return launch_stream<kNcol, kF28, kVecSign, kModeA8, kTok>(p, st);
    case kModeS4: return launch_stream<kNcol, kF28, kVecSign, kModeS4, kTok>(p, st);
    default: return launch_stream<kNcol, kF28, kVecSign, kModeS8, kTok>(p, st);
  }
}

template <int kNcol, bool kF28, int kTok = 1>
cudaError_t dispatch_stream(const TcParams& p, bool vec_sign, int mode, cudaStream_t st) {
  return vec_sign ? dispatch_stream_mode<kNcol, kF28, true, kTok>(p, mode, st)
                  : dispatch_stream_mode<kNcol, kF28, false, kTok>(p, mode, st);
}

}  // namespace

template <int kV, bool kF32In>
cudaError_t launch_small_mode(const TcParams& p, int mode, cudaStream_t st) {
  const void* kerns[5] = {reinterpret_cast<const void*>(rotq_small_kernel<kV, kF32In, kModeY>),
                          reinterpret_cast<const void*>(rotq_small_kernel<kV, kF32In, kModeA4>),
                          reinterpret_cast<const void*>(rotq_small_kernel<kV, kF32In, kModeA8>),
                          reinterpret_cast<const void*>(rotq_small_kernel<kV, kF32In, kModeS4>),
                          reinterpret_cast<const void*>(rotq_small_kernel<kV, kF32In, kModeS8>)};
  static KernelSetup setup[5];
  int sms = 0;
  cudaError_t e = setup[mode].prepare(kerns[mode], 0, &sms);
  if (e != cudaSuccess) return e;
  const int64_t ctas = (static_cast<int64_t>(p.T) + kSmallWarps - 1) / kSmallWarps;
  const int grid = static_cast<int>(ctas < 16LL * sms ? ctas : 16LL * sms);
  switch (mode) {
    case kModeY: e = launch_pdl(rotq_small_kernel<kV, kF32In, kModeY>, grid, 32 * kSmallWarps, 0, st, p); break;
    case kModeA4: e = launch_pdl(rotq_small_kernel<kV, kF32In, kModeA4>, grid, 32 * kSmallWarps, 0, st, p); break;
    case kModeA8: e = launch_pdl(rotq_small_kernel<kV, kF32In, kModeA8>, grid, 32 * kSmallWarps, 0, st, p); break;
    case kModeS4: e = launch_pdl(rotq_small_kernel<kV, kF32In, kModeS4>, grid, 32 * kSmallWarps, 0, st, p); break;
    default: e = launch_pdl(rotq_small_kernel<kV, kF32In, kModeS8>, grid, 32 * kSmallWarps, 0, st, p); break;
  }
  count_launch();
  return e;
}

// Rows of 512-2048 channels (F = 1) with s in its outlier form: one warp per token.
cudaError_t launch_small(const RotateArgs& a, const H28Masks& h, cudaStream_t st) {
  const bool f32 = a.dtype == kF32;
  const int es = f32 ? 4 : 2;
  if (reinterpret_cast<uintptr_t>(a.x) % 16 != 0 || (a.ld * es) % 16 != 0) return cudaErrorNotSupported;
  const bool quant = a.q != nullptr;
  const int mode = !quant ? kModeY : (a.sym ? (a.bits == 8 ? kModeS8 : kModeS4) : (a.bits == 8 ? kModeA8 : kModeA4));
  if (quant && reinterpret_cast<uintptr_t>(a.q) % 16 != 0) return cudaErrorNotSupported;
  if (!quant && (reinterpret_cast<uintptr_t>(a.y) % 16 != 0 || a.ldy % 4 != 0)) return cudaErrorNotSupported;
  TcParams p{};
  p.xraw = a.x;
  p.ldx = a.ld;
  p.T = static_cast<int32_t>(a.T);
  p.n = a.shape.n;
  p.logM = a.shape.logM;
  p.d = a.d;
  p.s = nullptr;
  p.kp = a.kp;
  p.xkp = a.xkp;
  p.q = a.q;
  p.scale = a.scale;
  p.zero = a.zero;
  p.y = a.y;
  p.ldy = a.ldy;
  p.clip = a.clip;
  p.inv_sqrt_n = 1.f;  // the kernel stores y = s w / sqrt(n) itself: the grid's multiplier is 1
  p.h = h;
  switch (a.shape.n) {
    case 512: return f32 ? launch_small_mode<16, true>(p, mode, st) : launch_small_mode<16, false>(p, mode, st);
    case 1024: return f32 ? launch_small_mode<32, true>(p, mode, st) : launch_small_mode<32, false>(p, mode, st);
    default: return f32 ? launch_small_mode<64, true>(p, mode, st) : launch_small_mode<64, false>(p, mode, st);
  }
}

constexpr bool kShortRowTiles = true;

cudaError_t launch_rotate_fast(const RotateArgs& a, const H28Masks& h, cudaStream_t st) {
  if (a.T > 0 && a.T <= 0x7fffffff && a.shape.F == 1 && a.kp != nullptr &&
      (a.shape.n == 512 || a.shape.n == 1024 || a.shape.n == 2048)) {
    cudaError_t e = launch_small(a, h, st);
    if (e != cudaErrorNotSupported) return e;
  }
  if (a.dtype != kBF16 || a.T <= 0 || a.T > 0x7fffffff) return cudaErrorNotSupported;
  if (a.shape.F != 1 && a.shape.F != 28) return cudaErrorNotSupported;
  const bool f28 = a.shape.F == 28;
  const int ncol = f28 ? (1 << a.shape.logM) / 4 : a.shape.n / 128;
  if (ncol != 32 && ncol != 64 && ncol != 128 && ncol != 256) return cudaErrorNotSupported;
  if (reinterpret_cast<uintptr_t>(a.x) % 16 != 0 || a.ld % 8 != 0) return cudaErrorNotSupported;
  const bool quant = a.q != nullptr;
  const int mode = !quant ? kModeY : (a.sym ? (a.bits == 8 ? kModeS8 : kModeS4) : (a.bits == 8 ? kModeA8 : kModeA4));
  if (quant && reinterpret_cast<uintptr_t>(a.q) % 16 != 0) return cudaErrorNotSupported;
  if (!quant && (reinterpret_cast<uintptr_t>(a.y) % 16 != 0 || a.ldy % 4 != 0)) return cudaErrorNotSupported;
  TcParams p{};
  p.xraw = a.x;
  p.ldx = a.ld;
  p.T = static_cast<int32_t>(a.T);
  p.n = a.shape.n;
  p.logM = a.shape.logM;
  p.d = a.d;
  p.s = a.s;
  p.kp = a.kp;
  p.xkp = a.xkp;
  p.q = a.q;
  p.scale = a.scale;
  p.zero = a.zero;
  p.y = a.y;
  p.ldy = a.ldy;
  p.clip = a.clip;
  p.inv_sqrt_n = a.inv_sqrt_n;
  p.h = h;
  const bool vec = a.s != nullptr && a.kp == nullptr;
  // Up to 128 columns per token: the streamed kernel (32 columns: 4 tokens share a 128-column
  // tile); 256 columns: the TMA-staged wide kernel. Shorter rows take the generic kernel.
  // Short rows with a materialised sign vector take the generic (exact) kernel: only the outlier
  // form tells the kernel which channel to keep out of the fp32 sums (see kill in
  // rotq_stream_kernel), and a sign vector built from the outlier gives exactly the rows (one
  // crowd far from zero, a narrow spread) where those sums' rounding would reach the codes.
  if (ncol == 32 && vec) return cudaErrorNotSupported;
  if (kShortRowTiles && ncol == 32)
    return f28 ? dispatch_stream<128, true, 4>(p, vec, mode, st) : dispatch_stream<128, false, 4>(p, vec, mode, st);
  if (ncol < 64) return cudaErrorNotSupported;
  if (ncol == 64) return f28 ? dispatch_stream<64, true>(p, vec, mode, st) : dispatch_stream<64, false>(p, vec, mode, st);
  if (ncol == 128) return f28 ? dispatch_stream<128, true>(p, vec, mode, st) : dispatch_stream<128, false>(p, vec, mode, st);

  auto encode = encode_fn();
  if (encode == nullptr) return cudaErrorNotSupported;
  CUtensorMap tmap;
  CUresult r;
  const cuuint32_t elem_strides[4] = {1, 1, 1, 1};
  if (f28) {
    const int M = 1 << a.shape.logM;
    const cuuint64_t dims[4] = {static_cast<cuuint64_t>(ncol), 4, 28, static_cast<cuuint64_t>(a.T)};
    const cuuint64_t strides[3] = {static_cast<cuuint64_t>(ncol) * 2, static_cast<cuuint64_t>(M) * 2,
                                   static_cast<cuuint64_t>(a.ld) * 2};
    const cuuint32_t box[4] = {64, 4, 4, 1};
    r = encode(&tmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(a.x), dims, strides, box, elem_strides,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  } else {
    const cuuint64_t dims[3] = {static_cast<cuuint64_t>(ncol), 128, static_cast<cuuint64_t>(a.T)};
    const cuuint64_t strides[2] = {static_cast<cuuint64_t>(ncol) * 2, static_cast<cuuint64_t>(a.ld) * 2};
    const cuuint32_t box[3] = {64, 16, 1};
    r = encode(&tmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(a.x), dims, strides, box, elem_strides,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  }
  if (r != CUDA_SUCCESS) return cudaErrorNotSupported;
  return f28 ? dispatch_wide<true>(tmap, p, vec, mode, st) : dispatch_wide<false>(tmap, p, vec, mode, st);
}

void* tensor_map_encoder() {
  static void* fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &ptr, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = ptr;
  });
  return fn;
}

cudaError_t read_device_error(uint32_t* out, bool clear) {
  cudaError_t e = cudaMemcpyFromSymbol(out, g_device_error, sizeof(uint32_t));
  if (e != cudaSuccess || !clear) return e;
  const uint32_t zero = 0;
  return cudaMemcpyToSymbol(g_device_error, &zero, sizeof(uint32_t));
}

}  // namespace signrot
