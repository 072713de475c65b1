// Generic rotate / rotate+quantize kernel: one CTA per token row, the row staged in shared
// memory. Covers every supported n, fp32 or bf16 input and any element-aligned rows; the fused
// tensor-core kernel (rotate_tc.cu) takes the bf16 shapes it is built for.
//
// Per row (SignRot explainer, "The standard fix is rotation" and "SignRot asks one crowd to walk
// across the hall"; abstract: fast Walsh-Hadamard transform):
//   1. x' = D (.) x                 (exact sign flips)
//   2. H_F across the stride-M axis (dense 28 x 28 or 344 x 344 block, F > 1 only)
//   3. FWHT of length M along the contiguous axis, radix-2 stages
//   4. y = s (.) w / sqrt(n), rounded once to fp32
//   5. check path: store y; quantized path: row min/max, the asymmetric (scale, zero) or symmetric
//      (scale) grid, codes packed two per byte (4 bits) or one per byte (8 bits).
// The rotation accumulates in fp64 (fp32 only for n = 32768, whose fp64 row would not fit in
// shared memory), so y is the correctly rounded fp32 of the exact rotation up to a rare double
// rounding, and the quantizer then takes the same fp32 steps as the formula in the header
// (true divisions, ties to even). This path is the slow, exact-decision reference on the device.
#include <cstdint>

#include "signrot_internal.h"
#include "signrot_device.cuh"

namespace signrot {
namespace {

constexpr int kThreads = 512;

template <typename Acc>
__device__ __forceinline__ Acc neg_if(Acc v, bool neg) {
  return neg ? -v : v;
}

template <typename Tin, typename Acc, bool kQuant>
__global__ void __launch_bounds__(kThreads) rotate_generic_kernel(RotateArgs a, H28Masks h, GF343Squares sq,
                                                                  double sqrt_n) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  Acc* buf = reinterpret_cast<Acc*>(smem_raw);
  float* ybuf = reinterpret_cast<float*>(smem_raw);  // fp32 y, aliases buf after step 4
  __shared__ float red[64];
  const int n = a.shape.n;
  const int logM = a.shape.logM;
  const int M = 1 << logM;
  const bool f344 = a.shape.F == 344;
  // F = 344: the mixed row goes to a second buffer (the block is too large to hold a column in
  // registers), and the block's sign masks sit after it: bit c % 32 of hm[r * 11 + c / 32] is
  // set iff H_344[r][c] == -1.
  Acc* mixed = f344 ? buf + n : buf;
  uint32_t* hm = reinterpret_cast<uint32_t*>(smem_raw + 2 * static_cast<size_t>(n) * sizeof(Acc));
  if (f344) {
    for (int w = threadIdx.x; w < 344 * 11; w += blockDim.x) {
      const int r = w / 11, c0 = (w % 11) * 32;
      uint32_t bits = 0;
      for (int cc = 0; cc < 32 && c0 + cc < 344; ++cc) bits |= static_cast<uint32_t>(h344_neg(sq, r, c0 + cc)) << cc;
      hm[w] = bits;
    }
    __syncthreads();
  }
  const Tin* __restrict__ x = static_cast<const Tin*>(a.x);
  // sign vector from the outlier channel: s_j = sgn(H[j,k] D_k x_k), +1 everywhere if x_k = 0
  bool pattern = false;
  int c_k = 0, e_k = 0, sig_neg = 0;
  if (a.kp != nullptr) {
    const int k = *a.kp;
    const float xk = *a.xkp;
    pattern = xk != 0.f && k >= 0 && k < n;  // an out-of-range k applies no sign adjustment
    if (pattern) {
      c_k = k >> logM;
      e_k = k & (M - 1);
      sig_neg = ((xk < 0.f) != (a.d[k] < 0)) ? 1 : 0;
    }
  }

  for (int64_t t = blockIdx.x; t < a.T; t += gridDim.x) {
    const Tin* xr = x + t * a.ld;
    for (int j = threadIdx.x; j < n; j += blockDim.x)
      buf[j] = neg_if(static_cast<Acc>(load_as_float(xr + j)), a.d[j] < 0);
    __syncthreads();

    if (a.shape.F == 28) {
      for (int b = threadIdx.x; b < M; b += blockDim.x) {
        Acc v[28];
#pragma unroll
        for (int c = 0; c < 28; ++c) v[c] = buf[c * M + b];
        for (int r = 0; r < 28; ++r) {
          const uint32_t m = h.row[r];
          Acc acc = 0;
#pragma unroll
          for (int c = 0; c < 28; ++c) acc += neg_if(v[c], (m >> c) & 1u);
          buf[r * M + b] = acc;
        }
      }
      __syncthreads();
    } else if (f344) {
      // eight output rows of one column per work item; c ascending, a fixed summation order
      for (int item = threadIdx.x; item < M * 43; item += blockDim.x) {
        const int b = item % M, r0 = (item / M) * 8;
        Acc acc[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[i] = 0;
        for (int w = 0; w < 11; ++w) {
          uint32_t m[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) m[i] = hm[(r0 + i) * 11 + w];
          const int cn = w < 10 ? 32 : 344 - 320;
          for (int cc = 0; cc < cn; ++cc) {
            const Acc v = buf[(w * 32 + cc) * M + b];
#pragma unroll
            for (int i = 0; i < 8; ++i) acc[i] += neg_if(v, (m[i] >> cc) & 1u);
          }
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) mixed[(r0 + i) * M + b] = acc[i];
      }
      __syncthreads();
    }

    for (int hs = 1; hs < M; hs <<= 1) {
      for (int p = threadIdx.x; p < (n >> 1); p += blockDim.x) {
        const int row = p >> (logM - 1);
        const int r = p & ((M >> 1) - 1);
        const int i = ((r & ~(hs - 1)) << 1) | (r & (hs - 1));
        Acc* base = mixed + row * M;
        const Acc u = base[i], v = base[i + hs];
        base[i] = u + v;
        base[i + hs] = u - v;
      }
      __syncthreads();
    }

    // y in fp32: one rounding of s_j * w_j / sqrt(n)
    float lo = pos_inf(), hi = -pos_inf();
    constexpr int kPer = (sizeof(Acc) + sizeof(float) - 1) / sizeof(float);  // y overwrites buf in place
    for (int j0 = 0; j0 < n; j0 += blockDim.x * kPer) {
      float yv[kPer];
#pragma unroll
      for (int e = 0; e < kPer; ++e) {
        const int j = j0 + threadIdx.x * kPer + e;
        yv[e] = 0.f;
        if (j < n) {
          bool neg;
          if (pattern) {
            neg = ((__popc((j & (M - 1)) & e_k) & 1) ^ sig_neg) != 0;
            if (a.shape.F == 28) neg ^= ((h.row[j >> logM] >> c_k) & 1u) != 0;
            if (f344) neg ^= ((hm[(j >> logM) * 11 + (c_k >> 5)] >> (c_k & 31)) & 1u) != 0;
          } else {
            neg = a.s != nullptr && a.s[j] < 0;
          }
          const Acc w = neg_if(mixed[j], neg);
          yv[e] = sizeof(Acc) == 8 ? static_cast<float>(static_cast<double>(w) / sqrt_n)
                                   : static_cast<float>(w) * a.inv_sqrt_n;
        }
      }
      __syncthreads();
#pragma unroll
      for (int e = 0; e < kPer; ++e) {
        const int j = j0 + threadIdx.x * kPer + e;
        if (j < n) {
          if (kQuant) {
            ybuf[j] = yv[e];
            lo = fminf(lo, yv[e]);
            hi = fmaxf(hi, yv[e]);
          } else {
            a.y[t * a.ldy + j] = yv[e];
          }
        }
      }
      __syncthreads();
    }
    if (kQuant) {
      block_minmax(lo, hi, red);
      if (a.sym) {
        const float L = a.bits == 8 ? 127.f : 7.f;
        const float scale = sym_scale(lo, hi, L);
        if (threadIdx.x == 0) a.scale[t] = scale;
        if (a.bits == 8) {
          int8_t* qr = reinterpret_cast<int8_t*>(a.q) + t * n;
          for (int j = threadIdx.x; j < n; j += blockDim.x) qr[j] = static_cast<int8_t>(sym_code_div(ybuf[j], scale, L));
        } else {
          uint8_t* qr = a.q + t * (n >> 1);
          for (int i = threadIdx.x; i < (n >> 1); i += blockDim.x) {
            const uint32_t c0 = static_cast<uint32_t>(sym_code_div(ybuf[2 * i], scale, L)) & 15u;
            const uint32_t c1 = static_cast<uint32_t>(sym_code_div(ybuf[2 * i + 1], scale, L)) & 15u;
            qr[i] = static_cast<uint8_t>(c0 | (c1 << 4));
          }
        }
      } else {
        const float qmax = a.bits == 8 ? 255.f : 15.f;
        const QuantGrid g = make_grid(lo, hi, a.clip, qmax);
        if (threadIdx.x == 0) {
          a.scale[t] = g.scale;
          a.zero[t] = g.zero;
        }
        if (a.bits == 8) {
          uint8_t* qr = a.q + t * n;
          for (int j = threadIdx.x; j < n; j += blockDim.x) qr[j] = static_cast<uint8_t>(quant_code_div(ybuf[j], g, qmax));
        } else {
          uint8_t* qr = a.q + t * (n >> 1);
          for (int i = threadIdx.x; i < (n >> 1); i += blockDim.x) {
            const uint32_t c0 = quant_code_div(ybuf[2 * i], g);
            const uint32_t c1 = quant_code_div(ybuf[2 * i + 1], g);
            qr[i] = static_cast<uint8_t>(c0 | (c1 << 4));
          }
        }
      }
    }
    __syncthreads();
  }
}

template <typename Tin, typename Acc, bool kQuant>
cudaError_t launch_typed(const RotateArgs& a, const H28Masks& h, const GF343Squares& sq, cudaStream_t st) {
  const size_t row = static_cast<size_t>(a.shape.n) * sizeof(Acc);
  const size_t smem = a.shape.F == 344 ? 2 * row + 344 * 11 * sizeof(uint32_t) : row;
  auto kern = rotate_generic_kernel<Tin, Acc, kQuant>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 0, per_sm = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
  if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kThreads, smem)) != cudaSuccess)
    return e;
  const int64_t cap = static_cast<int64_t>(sms) * (per_sm > 0 ? per_sm : 1);
  const int grid = static_cast<int>(a.T < cap ? a.T : cap);
  kern<<<grid, kThreads, smem, st>>>(a, h, sq, sqrt(static_cast<double>(a.shape.n)));
  count_launch();
  return cudaGetLastError();
}

template <typename Tin, typename Acc>
cudaError_t launch_acc(const RotateArgs& a, const H28Masks& h, const GF343Squares& sq, cudaStream_t st) {
  return a.q != nullptr ? launch_typed<Tin, Acc, true>(a, h, sq, st) : launch_typed<Tin, Acc, false>(a, h, sq, st);
}

}  // namespace

cudaError_t launch_rotate_generic(const RotateArgs& a, const H28Masks& h, const GF343Squares& sq,
                                  cudaStream_t st) {
  // fp64 row (two of them and the sign masks for F = 344, n <= 11008) fits in shared memory
  const bool wide = a.shape.n <= 28672;
  if (a.dtype == kBF16)
    return wide ? launch_acc<uint16_t, double>(a, h, sq, st) : launch_acc<uint16_t, float>(a, h, sq, st);
  return wide ? launch_acc<float, double>(a, h, sq, st) : launch_acc<float, float>(a, h, sq, st);
}

}  // namespace signrot
