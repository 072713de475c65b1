// Device helpers shared by the rotation kernels.
#pragma once

#include <cstdint>

#include <cuda_runtime.h>

#include "signrot_internal.h"

namespace signrot {

// 1 iff H_344[i][j] == -1 (Paley construction I over GF(343), element e = c0 + 7 c1 + 49 c2):
// row 0 is all +1, column 0 below it all -1, and H[1+e][1+f] = [e == f] + chi(e - f).
__host__ __device__ __forceinline__ int h344_neg(const GF343Squares& sq, int i, int j) {
  if (i == 0) return 0;
  if (j == 0) return 1;
  if (i == j) return 0;
  const int e = i - 1, f = j - 1;
  const int d0 = (e % 7 - f % 7 + 7) % 7;
  const int d1 = ((e / 7) % 7 - (f / 7) % 7 + 7) % 7;
  const int d2 = (e / 49 - f / 49 + 7) % 7;
  const int d = d0 + 7 * d1 + 49 * d2;
  return ((sq.bits[d >> 5] >> (d & 31)) & 1u) ? 0 : 1;
}

__device__ __forceinline__ float load_as_float(const uint16_t* p) {
  return __uint_as_float(static_cast<uint32_t>(*p) << 16);  // bf16 -> fp32 is exact
}
__device__ __forceinline__ float load_as_float(const float* p) { return *p; }

__device__ __forceinline__ float pos_inf() { return __int_as_float(0x7f800000); }

// Row-wide min/max over a CTA; every thread returns the CTA result. red holds 64 floats.
__device__ __forceinline__ void block_minmax(float& lo, float& hi, float* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, o));
    hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, o));
  }
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31, nw = blockDim.x >> 5;
  if (l == 0) {
    red[w] = lo;
    red[32 + w] = hi;
  }
  __syncthreads();
  if (w == 0) {
    lo = l < nw ? red[l] : pos_inf();
    hi = l < nw ? red[32 + l] : -pos_inf();
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, o));
      hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, o));
    }
    if (l == 0) {
      red[0] = lo;
      red[32] = hi;
    }
  }
  __syncthreads();
  lo = red[0];
  hi = red[32];
}

// Asymmetric per-token 4-bit grid over [c*lo, c*hi] (the explainer's "16 levels, spaced evenly
// from the smallest to the largest value of one token"; "Worked example": step = range / 15).
struct QuantGrid {
  float scale;  // (hi - lo) / 15, or 1 for a constant row
  float zero;   // rne(-lo / scale), integer-valued
  float inv;    // fp32(1 / scale)
};

__device__ __forceinline__ QuantGrid make_grid(float lo, float hi, float clip, float qmax = 15.f) {
  const float l = __fmul_rn(lo, clip), u = __fmul_rn(hi, clip);
  QuantGrid g;
  if (u == l) {
    g.scale = 1.f;
    g.zero = rintf(-l);
  } else {
    g.scale = __fdiv_rn(__fsub_rn(u, l), qmax);
    g.zero = rintf(__fdiv_rn(-l, g.scale));
  }
  g.inv = __frcp_rn(g.scale);
  return g;
}

// code = clamp(rne(y / scale) + zero, 0, qmax) with a true IEEE division (the formula as written).
__device__ __forceinline__ uint32_t quant_code_div(float y, const QuantGrid& g, float qmax = 15.f) {
  const float v = __fadd_rn(rintf(__fdiv_rn(y, g.scale)), g.zero);
  return static_cast<uint32_t>(fminf(fmaxf(v, 0.f), qmax));
}

// Symmetric grid, codes -L .. L: scale = max |y| / L (1 for an all-zero row) ...
__device__ __forceinline__ float sym_scale(float lo, float hi, float L) {
  const float amax = fmaxf(fabsf(lo), fabsf(hi));
  return amax == 0.f ? 1.f : __fdiv_rn(amax, L);
}
// ... and code = clamp(rne(y / scale), -L, L), true IEEE division.
__device__ __forceinline__ int32_t sym_code_div(float y, float scale, float L) {
  return static_cast<int32_t>(fminf(fmaxf(rintf(__fdiv_rn(y, scale)), -L), L));
}

// code = clamp(rne(y / scale) + zero, 0, 15), with y / scale taken as y * fp32(1/scale).
__device__ __forceinline__ uint32_t quant_code(float y, const QuantGrid& g) {
  const float v = __fadd_rn(rintf(__fmul_rn(y, g.inv)), g.zero);
  return static_cast<uint32_t>(fminf(fmaxf(v, 0.f), 15.f));
}

}  // namespace signrot
