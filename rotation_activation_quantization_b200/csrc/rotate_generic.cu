// Generic rotate / rotate+quantize kernel: one CTA per token row, the row staged in shared
// memory as fp32. Covers every supported n and any element-aligned input; the fused fast
// kernels (rotate_fast.cu) take the shapes they are built for.
//
// Per row (SignRot explainer, "The standard fix is rotation" and "SignRot asks one crowd to walk
// across the hall"; abstract: fast Walsh-Hadamard transform):
//   1. x' = D (.) x                 (exact sign flips)
//   2. H_28 across the stride-M axis (dense 28 x 28 block, F = 28 only)
//   3. FWHT of length M along the contiguous axis, radix-2 stages
//   4. y = s (.) w * fp32(1/sqrt(n))
//   5. check path: store y; quantized path: row min/max, scale, zero, codes, nibble pack.
#include <cstdint>

#include "signrot_internal.h"
#include "signrot_device.cuh"

namespace signrot {
namespace {

constexpr int kThreads = 512;

template <typename Tin, bool kQuant>
__global__ void __launch_bounds__(kThreads) rotate_generic_kernel(RotateArgs a, H28Masks h) {
  extern __shared__ float buf[];
  __shared__ float red[64];
  const int n = a.shape.n;
  const int logM = a.shape.logM;
  const int M = 1 << logM;
  const Tin* __restrict__ x = static_cast<const Tin*>(a.x);

  for (int64_t t = blockIdx.x; t < a.T; t += gridDim.x) {
    const Tin* xr = x + t * a.ld;
    for (int j = threadIdx.x; j < n; j += blockDim.x) {
      float v = load_as_float(xr + j);
      buf[j] = a.d[j] < 0 ? -v : v;
    }
    __syncthreads();

    if (a.shape.F == 28) {
      for (int b = threadIdx.x; b < M; b += blockDim.x) {
        float v[28];
#pragma unroll
        for (int c = 0; c < 28; ++c) v[c] = buf[c * M + b];
        for (int r = 0; r < 28; ++r) {
          const uint32_t m = h.row[r];
          float acc = 0.f;
#pragma unroll
          for (int c = 0; c < 28; ++c) acc += ((m >> c) & 1u) ? -v[c] : v[c];
          buf[r * M + b] = acc;
        }
      }
      __syncthreads();
    }

    for (int hs = 1; hs < M; hs <<= 1) {
      for (int p = threadIdx.x; p < (n >> 1); p += blockDim.x) {
        const int row = p >> (logM - 1);
        const int r = p & ((M >> 1) - 1);
        const int i = ((r & ~(hs - 1)) << 1) | (r & (hs - 1));
        float* base = buf + row * M;
        const float u = base[i], v = base[i + hs];
        base[i] = u + v;
        base[i + hs] = u - v;
      }
      __syncthreads();
    }

    float lo = __int_as_float(0x7f800000), hi = -lo;
    for (int j = threadIdx.x; j < n; j += blockDim.x) {
      float w = buf[j];
      if (a.s != nullptr && a.s[j] < 0) w = -w;
      const float yv = w * a.inv_sqrt_n;
      if (kQuant) {
        buf[j] = yv;
        lo = fminf(lo, yv);
        hi = fmaxf(hi, yv);
      } else {
        a.y[t * a.ldy + j] = yv;
      }
    }
    if (kQuant) {
      block_minmax(lo, hi, red);
      QuantGrid g = make_grid(lo, hi, a.clip);
      if (threadIdx.x == 0) {
        a.scale[t] = g.scale;
        a.zero[t] = g.zero;
      }
      uint8_t* qr = a.q + t * (n >> 1);
      for (int i = threadIdx.x; i < (n >> 1); i += blockDim.x) {
        const uint32_t c0 = quant_code(buf[2 * i], g);
        const uint32_t c1 = quant_code(buf[2 * i + 1], g);
        qr[i] = static_cast<uint8_t>(c0 | (c1 << 4));
      }
    }
    __syncthreads();
  }
}

template <typename Tin, bool kQuant>
cudaError_t launch_typed(const RotateArgs& a, const H28Masks& h, cudaStream_t st) {
  const size_t smem = static_cast<size_t>(a.shape.n) * sizeof(float);
  auto kern = rotate_generic_kernel<Tin, kQuant>;
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
  kern<<<grid, kThreads, smem, st>>>(a, h);
  count_launch();
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_rotate_generic(const RotateArgs& a, const H28Masks& h, cudaStream_t st) {
  const bool quant = a.q != nullptr;
  if (a.dtype == kBF16)
    return quant ? launch_typed<uint16_t, true>(a, h, st) : launch_typed<uint16_t, false>(a, h, st);
  return quant ? launch_typed<float, true>(a, h, st) : launch_typed<float, false>(a, h, st);
}

}  // namespace signrot
