// The consumer of the packed codes: the W4A4 down projection on tcgen05 (kind::i8).
//
// SignRot explainer, "SignRot asks one crowd to walk across the hall": the rotation and the sign
// flip are folded into the weights offline (W' = W R^T, so W' (R x) = W x); "The flip alone does
// nothing for a symmetric quantizer": the asymmetric activation grid costs one correction in the
// matrix multiply, the zero-point times a precomputed column sum of the (quantized) weights:
//
//     out[t, o] = scale_t * wscale_o * (sum_j q_tj Q_oj - zero_t * c_o),   c_o = sum_j Q_oj
//
// with q_tj the token's codes 0..15 (two per byte), Q_oj the weights' symmetric 4-bit codes -7..7
// (held one per byte, the tensor core's operand width), scale/zero the activation grid and wscale
// the weights' per-output-channel scale. Activations on the symmetric grid (signed codes -7..7,
// no zero-point: the explainer's comparison grid) take the same kernel without the correction.
//
// Tensor-core mapping. The MMA takes 8-bit signed operands. The activation converter turns each
// packed byte into two signed bytes a = 16 (q - 8) -- the code's nibble moved to the high half of
// the byte with its top bit flipped, three logic operations per four codes -- so the s32
// accumulator holds acc16 = 16 sum_j (q_tj - 8) Q_oj exactly (weight codes in [-8, 7]: |acc16| <=
// 1024 K), acc16 >> 4 is the exact sum (below 2^24 in magnitude, so
// exact in fp32, for K <= 2^18), and
//     sum_j q_tj Q_oj - zero_t c_o = (acc16 >> 4) + (8 - zero_t) c_o,
// one fp32 FMA of exact operands (a single rounding), then the two scales.
//
// Tile: 128 tokens x 256 outputs per CTA, K in blocks of 128 bytes (one 128-byte swizzle atom).
// Warp roles (320 threads, one CTA per SM, persistent over tiles):
//   warp 0     TMA producer: weight block [256 x 128] (swizzled, straight into the MMA tile) and
//              packed activation block [128 x 64 bytes]
//   warps 1-4  converters: packed codes -> the MMA's swizzled s8 activation tile
//   warp 5     TMEM allocator and MMA issuer (4 x M128 N256 K32 per K block)
//   warps 6-9  epilogue (TMEM lane quadrant = warp % 4): accumulator -> fp32 outputs
// Pipeline: TMA -> loaded[s] -> convert -> ready[s] -> MMA -> empty[s]; the accumulator is double
// buffered in TMEM (2 x 256 columns) so one tile's epilogue overlaps the next tile's K loop.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cstdint>

#include "signrot_internal.h"
#include "tc_ptx.cuh"

namespace signrot {

__device__ unsigned int g_gemm_error = 0;

namespace {

using namespace ptx;

constexpr int kGM = 128;                     // tokens per tile (TMEM lanes)
constexpr int kGN = 256;                     // outputs per tile (TMEM columns per buffer)
constexpr int kGK = 128;                     // K bytes per block
constexpr int kGStages = 4;
constexpr uint32_t kBBytes = kGN * kGK;      // 32 KB weight block
constexpr uint32_t kABytes8 = kGM * kGK;     // 16 KB s8 activation block
constexpr uint32_t kPBytes = kGM * kGK / 2;  // 8 KB packed activation block
constexpr int kConvWarps = 4;
constexpr int kConvThreads = 32 * kConvWarps;
constexpr int kConvPer = static_cast<int>(kPBytes / 16) / kConvThreads;  // packed 16-byte chunks per thread
constexpr int kMmaWarpG = 1 + kConvWarps;                                // then four epilogue warps
constexpr int kGThreads = 32 * (kMmaWarpG + 1 + 4);
constexpr uint32_t kGIdesc = (2u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(kGN >> 3) << 17) |
                             (static_cast<uint32_t>(kGM >> 4) << 24);  // s32 <- s8 x s8, both K-major
constexpr size_t kGSmem = 1024 + kGStages * (kBBytes + kABytes8 + kPBytes) + 1024;

__device__ __forceinline__ void gemm_error() { atomicOr(&g_gemm_error, 1u); }

__device__ __forceinline__ uint64_t sw128_desc(uint32_t addr) {
  return static_cast<uint64_t>((addr & 0x3FFFFu) >> 4) | (static_cast<uint64_t>(16 >> 4) << 16) |
         (static_cast<uint64_t>(1024 >> 4) << 32) | (1ull << 46) | (2ull << 61);
}

// Four packed bytes (codes 2i low, 2i+1 high) -> eight s8 values 16 (code - 8), in element order.
// (Symmetric codes, two's complement nibbles c in [-8, 7], are first XORed with 8 in every nibble:
// c ^ 8 read unsigned is c + 8, so the same step gives 16 c.)
__device__ __forceinline__ uint2 unpack8(uint32_t w) {
  const uint32_t odd = (w & 0xF0F0F0F0u) ^ 0x80808080u;
  const uint32_t even = ((w << 4) & 0xF0F0F0F0u) ^ 0x80808080u;
  return make_uint2(__byte_perm(even, odd, 0x5140), __byte_perm(even, odd, 0x7362));
}

struct GemmParams {
  const float* scale;
  const float* zero;
  const float* wscale;
  const int32_t* colsum;
  float* out;
  int64_t ldo;
  int32_t T, N, K;
  int32_t tiles_m, tiles;
};

__global__ void __launch_bounds__(kGThreads, 1) w4a4_gemm_kernel(const __grid_constant__ CUtensorMap tmap_w,
                                                                   const __grid_constant__ CUtensorMap tmap_q,
                                                                   GemmParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint8_t* bbuf = smem;                               // [stage] 32 KB weight blocks
  uint8_t* abuf = bbuf + kGStages * kBBytes;          // [stage] 16 KB s8 activation blocks
  uint8_t* pbuf = abuf + kGStages * kABytes8;         // [stage] 8 KB packed activation blocks
  uint64_t* bars = reinterpret_cast<uint64_t*>(pbuf + kGStages * kPBytes);
  uint64_t* loaded = bars;
  uint64_t* ready = bars + kGStages;
  uint64_t* empty = bars + 2 * kGStages;
  uint64_t* tfull = bars + 3 * kGStages;
  uint64_t* tempty = tfull + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tempty + 2);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int kblocks = p.K / kGK;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kGStages; ++s) {
      mbar_init(smem_u32(&loaded[s]), 1);
      mbar_init(smem_u32(&ready[s]), kConvWarps);
      mbar_init(smem_u32(&empty[s]), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(smem_u32(&tfull[b]), 1);
      mbar_init(smem_u32(&tempty[b]), 4);
    }
    fence_mbar_init();
  }
  __syncthreads();
  griddep_wait();  // inputs may come from the grid before (the quantizer)
  griddep_launch_dependents();
  if (warp == kMmaWarpG) {
    tmem_alloc(smem_u32(tmem_slot), 2 * kGN);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      prefetch_tmap(&tmap_w);
      prefetch_tmap(&tmap_q);
      int it = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < p.tiles && ok; tile += gridDim.x) {
        const int m0 = (tile % p.tiles_m) * kGM, n0 = (tile / p.tiles_m) * kGN;
        for (int kb = 0; kb < kblocks; ++kb, ++it) {
          const int s = it % kGStages;
          if (!mbar_wait(smem_u32(&empty[s]), ((it / kGStages) & 1) ^ 1)) {
            gemm_error();
            ok = false;
            break;
          }
          const uint32_t fb = smem_u32(&loaded[s]);
          mbar_arrive_expect_tx(fb, kBBytes + kPBytes);
          tma_load_2d(smem_u32(bbuf + s * kBBytes), &tmap_w, kb * kGK, n0, fb);
          tma_load_2d(smem_u32(pbuf + s * kPBytes), &tmap_q, kb * (kGK / 2), m0, fb);
        }
      }
      // do not leave with copies in flight: the last stages issued must have landed
      for (int j = it - kGStages > 0 ? it - kGStages : 0; j < it; ++j)
        if (!mbar_wait(smem_u32(&loaded[j % kGStages]), (j / kGStages) & 1)) { gemm_error(); break; }
    }
  } else if (warp <= kConvWarps) {
    // ------------------------------------------------------------------ converters
    // Packed row m holds 64 bytes = 4 chunks of 16; chunk c gives s8 bytes [32c, 32c + 32) of the
    // K-major 128-byte row m, i.e. 16-byte slots 2c and 2c + 1, swizzled by (m & 7).
    const int ct = threadIdx.x - 32;  // 0 .. kConvThreads - 1
    const uint32_t nib_xor = p.zero == nullptr ? 0x88888888u : 0u;
    int it = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < p.tiles && ok; tile += gridDim.x) {
      for (int kb = 0; kb < kblocks; ++kb, ++it) {
        const int s = it % kGStages;
        if (!__all_sync(0xffffffffu, mbar_wait(smem_u32(&loaded[s]), (it / kGStages) & 1))) {
          gemm_error();
          ok = false;
          break;
        }
        const uint4* src = reinterpret_cast<const uint4*>(pbuf + s * kPBytes);
        uint8_t* dst = abuf + s * kABytes8;
        uint4 v[kConvPer];
#pragma unroll
        for (int u = 0; u < kConvPer; ++u) v[u] = src[u * kConvThreads + ct];
#pragma unroll
        for (int u = 0; u < kConvPer; ++u) {
          const int chunk = u * kConvThreads + ct, m = chunk >> 2, c = chunk & 3;
          const uint2 a0 = unpack8(v[u].x ^ nib_xor), a1 = unpack8(v[u].y ^ nib_xor);
          const uint2 a2 = unpack8(v[u].z ^ nib_xor), a3 = unpack8(v[u].w ^ nib_xor);
          uint8_t* row = dst + (m >> 3) * 1024 + (m & 7) * 128;
          *reinterpret_cast<uint4*>(row + (((2 * c) ^ (m & 7)) << 4)) = make_uint4(a0.x, a0.y, a1.x, a1.y);
          *reinterpret_cast<uint4*>(row + (((2 * c + 1) ^ (m & 7)) << 4)) = make_uint4(a2.x, a2.y, a3.x, a3.y);
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&ready[s]));
      }
    }
  } else if (warp == kMmaWarpG) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int it = 0, lt = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < p.tiles && ok; tile += gridDim.x, ++lt) {
        const int b = lt & 1;
        if (!mbar_wait(smem_u32(&tempty[b]), ((lt >> 1) & 1) ^ 1)) {
          gemm_error();
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + b * kGN;
        for (int kb = 0; kb < kblocks; ++kb, ++it) {
          const int s = it % kGStages;
          if (!mbar_wait(smem_u32(&ready[s]), (it / kGStages) & 1)) {
            gemm_error();
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a0 = smem_u32(abuf + s * kABytes8), b0 = smem_u32(bbuf + s * kBBytes);
#pragma unroll
          for (int ks = 0; ks < kGK / 32; ++ks)
            mma_i8(d_tmem, sw128_desc(a0 + ks * 32), sw128_desc(b0 + ks * 32), kGIdesc, (kb | ks) != 0 ? 1u : 0u);
          mma_commit(smem_u32(&empty[s]));
        }
        if (ok) mma_commit(smem_u32(&tfull[b]));
      }
      // the last MMAs finish before the TMEM is freed
      if (lt > 0 && ok && !mbar_wait(smem_u32(&tfull[(lt - 1) & 1]), ((lt - 1) >> 1) & 1)) gemm_error();
    }
  } else {
    // ------------------------------------------------------------------ epilogue
    const int quad = warp & 3;
    int lt = 0;
    for (int tile = blockIdx.x; tile < p.tiles; tile += gridDim.x, ++lt) {
      const int b = lt & 1;
      const int m0 = (tile % p.tiles_m) * kGM, n0 = (tile / p.tiles_m) * kGN;
      if (!__all_sync(0xffffffffu, mbar_wait(smem_u32(&tfull[b]), (lt >> 1) & 1))) {
        gemm_error();
        break;
      }
      tc_fence_after();
      const int t = m0 + quad * 32 + lane;
      const bool row_ok = t < p.T;
      const float st = row_ok ? p.scale[t] : 0.f;
      // unsigned codes: (acc16 >> 4) + (8 - zero) c_o; symmetric signed codes: acc16 >> 4
      const float a8z = (row_ok && p.zero != nullptr) ? 8.f - p.zero[t] : 0.f;
      float* orow = p.out + static_cast<int64_t>(row_ok ? t : 0) * p.ldo;
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(quad * 32) << 16) + b * kGN;
#pragma unroll 1
      for (int c0 = 0; c0 < kGN; c0 += 32) {
        uint32_t r[32];
        tmem_ld32(taddr + c0, r);
        const int nb = n0 + c0;
        if (row_ok && nb < p.N) {
          float o[32];
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            const int col = nb + e < p.N ? nb + e : p.N - 1;
            const float cs = static_cast<float>(__ldg(p.colsum + col));
            // acc16 is a multiple of 16: the arithmetic shift is the exact integer sum
            const float v = __fmaf_rn(a8z, cs, __int2float_rn(static_cast<int32_t>(r[e]) >> 4));
            o[e] = __fmul_rn(__fmul_rn(v, st), __ldg(p.wscale + col));
          }
          if (nb + 32 <= p.N && (reinterpret_cast<uintptr_t>(orow + nb) & 15u) == 0) {
#pragma unroll
            for (int e = 0; e < 32; e += 4)
              *reinterpret_cast<float4*>(orow + nb + e) = make_float4(o[e], o[e + 1], o[e + 2], o[e + 3]);
          } else {
#pragma unroll
            for (int e = 0; e < 32; ++e)
              if (nb + e < p.N) orow[nb + e] = o[e];
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&tempty[b]));
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarpG) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 2 * kGN);
  }
}

// Weight preparation (offline): symmetric 4-bit codes packed two per byte (two's complement
// nibbles, element 2i low, as signrot_rotate_quant_sym writes them) -> one signed byte each, and
// each row's code sum c_o. One CTA per output row; the sum is a fixed-order tree (deterministic).
constexpr int kPrepThreads = 256;

__global__ void __launch_bounds__(kPrepThreads) w4a4_prepare_kernel(const uint8_t* __restrict__ wq4, int64_t ldw4,
                                                                   int32_t K, int8_t* __restrict__ wq8, int64_t ldw8,
                                                                   int32_t* __restrict__ colsum) {
  __shared__ int32_t red[kPrepThreads / 32];
  const int64_t row = blockIdx.x;
  const uint8_t* src = wq4 + row * ldw4;
  int8_t* dst = wq8 + row * ldw8;
  int32_t sum = 0;
  for (int i = threadIdx.x; i < K / 2; i += kPrepThreads) {
    const uint32_t byte = src[i];
    const int32_t lo = static_cast<int32_t>((byte & 15u) ^ 8u) - 8;
    const int32_t hi = static_cast<int32_t>((byte >> 4) ^ 8u) - 8;
    dst[2 * i] = static_cast<int8_t>(lo);
    dst[2 * i + 1] = static_cast<int8_t>(hi);
    sum += lo + hi;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = sum;
  __syncthreads();
  if (threadIdx.x == 0) {
    int32_t total = 0;
    for (int w = 0; w < kPrepThreads / 32; ++w) total += red[w];
    colsum[row] = total;
  }
}

struct GemmSetup {
  std::atomic<int> sms[64] = {};
};

}  // namespace

cudaError_t launch_w4a4_gemm(const GemmArgs& a, cudaStream_t st) {
  auto encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(tensor_map_encoder());
  if (encode == nullptr) return cudaErrorNotSupported;
  CUtensorMap tw, tq;
  const cuuint32_t es[2] = {1, 1};
  {
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(a.K), static_cast<cuuint64_t>(a.N)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(a.ldw)};
    const cuuint32_t box[2] = {kGK, kGN};
    if (encode(&tw, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<int8_t*>(a.wq), dims, strides, box, es,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  {
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(a.K / 2), static_cast<cuuint64_t>(a.T)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(a.ldq)};
    const cuuint32_t box[2] = {kGK / 2, kGM};
    if (encode(&tq, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(a.q), dims, strides, box, es,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  GemmParams p{};
  p.scale = a.scale;
  p.zero = a.zero;
  p.wscale = a.wscale;
  p.colsum = a.colsum;
  p.out = a.out;
  p.ldo = a.ldo;
  p.T = static_cast<int32_t>(a.T);
  p.N = a.N;
  p.K = a.K;
  p.tiles_m = static_cast<int32_t>((a.T + kGM - 1) / kGM);
  p.tiles = p.tiles_m * ((a.N + kGN - 1) / kGN);

  static GemmSetup setup;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  int sms = dev < 64 ? setup.sms[dev].load(std::memory_order_acquire) : 0;
  if (sms == 0) {
    if ((e = cudaFuncSetAttribute(w4a4_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  static_cast<int>(kGSmem))) != cudaSuccess)
      return e;
    if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
    if (dev < 64) setup.sms[dev].store(sms, std::memory_order_release);
  }
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(p.tiles < sms ? p.tiles : sms);
  cfg.blockDim = dim3(kGThreads);
  cfg.dynamicSmemBytes = kGSmem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, w4a4_gemm_kernel, tw, tq, p);
  count_launch();
  return e;
}

cudaError_t launch_w4a4_prepare(const uint8_t* wq4, int64_t ldw4, int32_t N, int32_t K, int8_t* wq8, int64_t ldw8,
                                int32_t* colsum, cudaStream_t st) {
  w4a4_prepare_kernel<<<N, kPrepThreads, 0, st>>>(wq4, ldw4, K, wq8, ldw8, colsum);
  count_launch();
  return cudaGetLastError();
}

cudaError_t read_gemm_error(uint32_t* out, bool clear) {
  cudaError_t e = cudaMemcpyFromSymbol(out, g_gemm_error, sizeof(uint32_t));
  if (e != cudaSuccess || !clear) return e;
  const uint32_t zero = 0;
  return cudaMemcpyToSymbol(g_gemm_error, &zero, sizeof(uint32_t));
}

}  // namespace signrot
