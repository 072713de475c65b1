// Calibration (abstract: "a single calibration forward pass"; explainer, "SignRot asks one crowd
// to walk across the hall": the channel with the largest absolute activation) and the sign
// adjustment vector built from it.
//
// The per-channel state is one 64-bit key, so folding a chunk of tokens is a single atomicMax
// per (CTA, channel):
//   key = |x| as fp32 bits << 32  |  (2^31 - 1 - t) << 1  |  sign bit of x
// The high word orders by magnitude (non-negative fp32 bit patterns are monotone), the middle
// field makes the FIRST token win a tie, and the low bit keeps the value's sign so the signed
// x_k can be rebuilt from |x| and it.
#include <cstdint>

#include "signrot_internal.h"
#include "signrot_device.cuh"

namespace signrot {
namespace {

constexpr int kFoldThreads = 256;
constexpr int kVec = 8;            // channels per thread (one 16 B bf16 load, two for fp32)
constexpr int kTokensPerCta = 64;  // tokens folded by one CTA before its atomics

__device__ __forceinline__ unsigned long long calib_key(float v, int64_t t) {
  const uint32_t mag = __float_as_uint(v) & 0x7fffffffu;
  const uint32_t sign = __float_as_uint(v) >> 31;
  const uint32_t order = (0x7fffffffu - static_cast<uint32_t>(t)) << 1;
  return (static_cast<unsigned long long>(mag) << 32) | order | sign;
}

template <typename Tin>
__global__ void __launch_bounds__(kFoldThreads) calib_fold_kernel(CalibArgs a) {
  const Tin* __restrict__ x = static_cast<const Tin*>(a.x);
  const int64_t i0 = (static_cast<int64_t>(blockIdx.x) * kFoldThreads + threadIdx.x) * kVec;
  if (i0 >= a.n) return;
  const int nv = a.n - i0 < kVec ? static_cast<int>(a.n - i0) : kVec;
  unsigned long long best[kVec];
#pragma unroll
  for (int v = 0; v < kVec; ++v) best[v] = 0ull;
  // token blocks of kTokensPerCta, grid-strided along y (gridDim.y is capped at 65535)
  for (int64_t t0 = static_cast<int64_t>(blockIdx.y) * kTokensPerCta; t0 < a.T;
       t0 += static_cast<int64_t>(gridDim.y) * kTokensPerCta) {
    const int64_t t1 = t0 + kTokensPerCta < a.T ? t0 + kTokensPerCta : a.T;
    for (int64_t t = t0; t < t1; ++t) {
      const Tin* row = x + t * a.ld + i0;
      const int64_t tg = a.t_offset + t;
#pragma unroll
      for (int v = 0; v < kVec; ++v) {
        if (v < nv) {
          const unsigned long long key = calib_key(load_as_float(row + v), tg);
          best[v] = key > best[v] ? key : best[v];
        }
      }
    }
  }
#pragma unroll
  for (int v = 0; v < kVec; ++v)
    if (v < nv && best[v] != 0ull) atomicMax(a.ws + i0 + v, best[v]);
}

// One CTA: channel with the largest |x| (lowest index on ties), then its signed value.
__global__ void __launch_bounds__(1024) calib_argmax_kernel(const unsigned long long* __restrict__ ws,
                                                            int32_t n, int32_t* k_out, float* xk_out) {
  __shared__ unsigned long long red[32];
  unsigned long long best = 0ull;
  for (int i = threadIdx.x; i < n; i += blockDim.x) {
    const unsigned long long mag = ws[i] >> 32;
    const unsigned long long key = (mag << 32) | (0xffffffffu - static_cast<uint32_t>(i));
    best = key > best ? key : best;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const unsigned long long other = __shfl_xor_sync(0xffffffffu, best, o);
    best = other > best ? other : best;
  }
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = best;
  __syncthreads();
  if (threadIdx.x < 32) {
    best = threadIdx.x < (blockDim.x >> 5) ? red[threadIdx.x] : 0ull;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const unsigned long long other = __shfl_xor_sync(0xffffffffu, best, o);
      best = other > best ? other : best;
    }
    if (threadIdx.x == 0) {
      const int32_t k = static_cast<int32_t>(0xffffffffu - static_cast<uint32_t>(best & 0xffffffffull));
      const unsigned long long w = ws[k];
      const uint32_t mag = static_cast<uint32_t>(w >> 32);
      const uint32_t sign = static_cast<uint32_t>(w & 1ull);
      *k_out = k;
      *xk_out = __uint_as_float(mag | (sign << 31));
    }
  }
}

// s_j = +1 if H[j][k] * D_k * x_k >= 0 else -1, H[(a,b),(c,e)] = H_F[a][c] (-1)^popcount(b & e).
__global__ void build_sign_kernel(Shape sh, const int32_t* __restrict__ kp, const float* __restrict__ xkp,
                                  const int8_t* __restrict__ d, int8_t* __restrict__ s, H28Masks h,
                                  GF343Squares sq) {
  const int j = blockIdx.x * blockDim.x + threadIdx.x;
  if (j >= sh.n) return;
  const int k = *kp;
  const float xk = *xkp;
  if (k < 0 || k >= sh.n) {  // not a channel index: no sign adjustment
    s[j] = 1;
    return;
  }
  const int M1 = (1 << sh.logM) - 1;
  const int a = j >> sh.logM, b = j & M1;
  const int c = k >> sh.logM, e = k & M1;
  int neg = __popc(b & e) & 1;
  if (sh.F == 28) neg ^= static_cast<int>((h.row[a] >> c) & 1u);
  if (sh.F == 344) neg ^= h344_neg(sq, a, c);
  const float hv = neg ? -1.f : 1.f;
  const float v = hv * static_cast<float>(d[k]) * xk;  // exact: +/-1 factors
  s[j] = v >= 0.f ? int8_t(1) : int8_t(-1);
}

}  // namespace

cudaError_t launch_calibrate_fold(const CalibArgs& a, cudaStream_t st) {
  if (a.T == 0) return cudaSuccess;
  const int64_t per_cta = static_cast<int64_t>(kFoldThreads) * kVec;
  const int64_t blocks_t = (a.T + kTokensPerCta - 1) / kTokensPerCta;
  const dim3 grid(static_cast<unsigned>((a.n + per_cta - 1) / per_cta),
                  static_cast<unsigned>(blocks_t < 65535 ? blocks_t : 65535));
  if (a.dtype == kBF16)
    calib_fold_kernel<uint16_t><<<grid, kFoldThreads, 0, st>>>(a);
  else
    calib_fold_kernel<float><<<grid, kFoldThreads, 0, st>>>(a);
  count_launch();
  return cudaGetLastError();
}

cudaError_t launch_calibrate_argmax(const unsigned long long* ws, int32_t n, int32_t* k_out,
                                    float* xk_out, cudaStream_t st) {
  calib_argmax_kernel<<<1, 1024, 0, st>>>(ws, n, k_out, xk_out);
  count_launch();
  return cudaGetLastError();
}

cudaError_t launch_build_sign(Shape shape, const int32_t* k, const float* xk, const int8_t* d,
                              int8_t* s_out, const H28Masks& h, const GF343Squares& sq, cudaStream_t st) {
  const int threads = 256;
  const int grid = (shape.n + threads - 1) / threads;
  build_sign_kernel<<<grid, threads, 0, st>>>(shape, k, xk, d, s_out, h, sq);
  count_launch();
  return cudaGetLastError();
}

}  // namespace signrot
