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
#include "tc_ptx.cuh"

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
  ptx::griddep_launch_dependents();
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

// bf16 rows, 16-byte aligned, n % 8 == 0: the same keys from a streaming loop that keeps
// kUnroll 16-byte loads in flight per thread. Inside one CTA's token block (fewer than 2^16
// tokens) a 32-bit key orders exactly like the 64-bit one:
//   key32 = |x| bf16 bits (15) << 17  |  (0xffff - (t - t0)) << 1  |  sign bit of x
// and costs a shift, an OR and a max per element; each thread widens its 8 winners to 64-bit
// keys once, before the atomics.
constexpr int kUnroll = 8;

__device__ __forceinline__ void fold_word(uint32_t w, uint32_t tp, uint32_t& b_lo, uint32_t& b_hi) {
  const uint32_t k_lo = (w << 17) | tp | ((w >> 15) & 1u);
  const uint32_t k_hi = ((w << 1) & 0xfffe0000u) | tp | (w >> 31);
  b_lo = max(b_lo, k_lo);
  b_hi = max(b_hi, k_hi);
}

__device__ __forceinline__ void fold_row(const uint4& w, uint32_t tp, uint32_t (&best)[kVec]) {
  fold_word(w.x, tp, best[0], best[1]);
  fold_word(w.y, tp, best[2], best[3]);
  fold_word(w.z, tp, best[4], best[5]);
  fold_word(w.w, tp, best[6], best[7]);
}

__global__ void __launch_bounds__(kFoldThreads) calib_fold_bf16_kernel(CalibArgs a, int32_t tokens_per_cta) {
  ptx::griddep_launch_dependents();  // the argmax may be scheduled now; it waits for this grid
  const int64_t i0 = (static_cast<int64_t>(blockIdx.x) * kFoldThreads + threadIdx.x) * kVec;
  if (i0 >= a.n) return;
  const int64_t t0 = static_cast<int64_t>(blockIdx.y) * tokens_per_cta;
  const int64_t t1 = t0 + tokens_per_cta < a.T ? t0 + tokens_per_cta : a.T;
  const uint16_t* __restrict__ x = static_cast<const uint16_t*>(a.x) + i0;
  uint32_t best[kVec];
#pragma unroll
  for (int v = 0; v < kVec; ++v) best[v] = 0u;
  int64_t t = t0;
  for (; t + kUnroll <= t1; t += kUnroll) {
    uint4 w[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) w[u] = __ldcs(reinterpret_cast<const uint4*>(x + (t + u) * a.ld));
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) fold_row(w[u], (0xffffu - static_cast<uint32_t>(t + u - t0)) << 1, best);
  }
  for (; t < t1; ++t) {
    const uint4 w = __ldcs(reinterpret_cast<const uint4*>(x + t * a.ld));
    fold_row(w, (0xffffu - static_cast<uint32_t>(t - t0)) << 1, best);
  }
  if (t1 <= t0) return;
#pragma unroll
  for (int v = 0; v < kVec; ++v) {
    const uint32_t mag = (best[v] >> 17) << 16;  // fp32 bits of |x|
    const int64_t tg = a.t_offset + t0 + (0xffffu - ((best[v] >> 1) & 0xffffu));
    const uint32_t order = (0x7fffffffu - static_cast<uint32_t>(tg)) << 1;
    atomicMax(a.ws + i0 + v, (static_cast<unsigned long long>(mag) << 32) | order | (best[v] & 1u));
  }
}

// One CTA: channel with the largest |x| (lowest index on ties), then its signed value.
__global__ void __launch_bounds__(1024) calib_argmax_kernel(const unsigned long long* __restrict__ ws,
                                                            int32_t n, int32_t* k_out, float* xk_out) {
  __shared__ unsigned long long red[32];
  ptx::griddep_wait();  // the fold grid before this one has finished and its atomics are visible
  unsigned long long best = 0ull;
  for (int base = threadIdx.x; base < n; base += blockDim.x * 8) {
    unsigned long long w[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int i = base + u * static_cast<int>(blockDim.x);
      w[u] = i < n ? __ldcg(ws + i) : 0ull;
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int i = base + u * static_cast<int>(blockDim.x);
      const unsigned long long key = ((w[u] >> 32) << 32) | (0xffffffffu - static_cast<uint32_t>(i));
      if (i < n) best = key > best ? key : best;
    }
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
  const bool vec = a.dtype == kBF16 && a.n % kVec == 0 && a.ld % kVec == 0 &&
                   reinterpret_cast<uintptr_t>(a.x) % 16 == 0;
  if (vec) {
    // grid: channel tiles of kFoldThreads * kVec along x; along y, token blocks sized so that the
    // grid fills every SM at its occupancy, no block is shorter than 64 tokens (to bound the
    // atomics per channel) or longer than 65534 (the 32-bit key's token field)
    int dev = 0, sms = 0, per_sm = 0;
    cudaError_t e;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
    if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
    if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, calib_fold_bf16_kernel, kFoldThreads, 0)) !=
        cudaSuccess)
      return e;
    const int64_t per_cta = static_cast<int64_t>(kFoldThreads) * kVec;
    const int64_t gx = (a.n + per_cta - 1) / per_cta;
    const int64_t slots = static_cast<int64_t>(sms) * (per_sm > 0 ? per_sm : 1);
    const int64_t target = slots / gx > 0 ? slots / gx : 1;  // one wave
    int64_t gy = (a.T + 63) / 64;
    if (gy > target) gy = target;
    if (gy < 1) gy = 1;
    int64_t tpc = (a.T + gy - 1) / gy;
    if (tpc > 65534) tpc = 65534;
    gy = (a.T + tpc - 1) / tpc;
    if (gy > 65535) return cudaErrorInvalidValue;  // unreachable: T < 2^31
    calib_fold_bf16_kernel<<<dim3(static_cast<unsigned>(gx), static_cast<unsigned>(gy)), kFoldThreads, 0, st>>>(
        a, static_cast<int32_t>(tpc));
    count_launch();
    return cudaGetLastError();
  }
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
  // programmatic dependent launch: scheduled while the fold drains, it waits for the fold's
  // completion (griddepcontrol.wait) before reading the keys
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(1);
  cfg.blockDim = dim3(1024);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, calib_argmax_kernel, ws, n, k_out, xk_out);
  count_launch();
  return e != cudaSuccess ? e : cudaGetLastError();
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
