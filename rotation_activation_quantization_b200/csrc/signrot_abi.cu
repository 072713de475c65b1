// The C ABI (include/signrot.h): argument validation, shape factorisation, dispatch to the
// kernels, and error reporting. No device memory is allocated here.
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>

#include <atomic>

#include <cuda_runtime.h>

#include "signrot.h"
#include "signrot_internal.h"

namespace signrot {
namespace {
std::atomic<uint64_t> g_launches{0};
}
void count_launch(int n) { g_launches.fetch_add(static_cast<uint64_t>(n), std::memory_order_relaxed); }
}  // namespace signrot

namespace {

thread_local char g_last_error[512] = "";

signrot_status fail(signrot_status st, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_last_error, sizeof(g_last_error), fmt, ap);
  va_end(ap);
  return st;
}

signrot_status cuda_fail(cudaError_t e, const char* what) {
  return fail(SIGNROT_ERR_CUDA, "%s: %s (%s)", what, cudaGetErrorName(e), cudaGetErrorString(e));
}

bool factor_n(int32_t n, signrot::Shape* sh) {
  if (n <= 0) return false;
  const auto pow2 = [](int32_t v) { return v > 0 && (v & (v - 1)) == 0; };
  const auto lg = [](int32_t v) {
    int m = 0;
    while ((1 << m) < v) ++m;
    return m;
  };
  if (pow2(n) && n >= 2 && n <= (1 << 15)) {
    *sh = {n, 1, lg(n)};
    return true;
  }
  if (n % 28 == 0 && pow2(n / 28) && n / 28 <= (1 << 10)) {
    *sh = {n, 28, lg(n / 28)};
    return true;
  }
  if (n % 344 == 0 && pow2(n / 344) && n / 344 <= 32) {
    *sh = {n, 344, lg(n / 344)};
    return true;
  }
  return false;
}

#define SIGNROT_N_FORMS "2^m (1<=m<=15), 28*2^m (0<=m<=10) or 344*2^m (0<=m<=5)"


struct H28State {
  int8_t h[28][28];
  signrot::H28Masks masks;
};

const H28State& h28_state() {
  static H28State st;
  static std::once_flag once;
  std::call_once(once, [] {
    signrot::paley_h28(st.h);
    for (int a = 0; a < 28; ++a) {
      uint32_t m = 0;
      for (int c = 0; c < 28; ++c)
        if (st.h[a][c] < 0) m |= 1u << c;
      st.masks.row[a] = m;
    }
  });
  return st;
}

const signrot::GF343Squares& gf343_state() {
  static signrot::GF343Squares sq;
  static std::once_flag once;
  std::call_once(once, [] { sq = signrot::gf343_squares(); });
  return sq;
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// Two copy/compute streams and their join events per device, created on first use and kept for
// the life of the process (the host-buffer entry point allocates nothing per call).
struct HostStreams {
  cudaStream_t s[2];
  cudaEvent_t start;
  cudaEvent_t done[2];
};

HostStreams* host_streams(int dev) {
  static std::mutex mu;
  static HostStreams* per_dev[64] = {};
  if (dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> guard(mu);
  if (per_dev[dev] == nullptr) {
    auto* h = new HostStreams{};
    bool ok = cudaStreamCreateWithFlags(&h->s[0], cudaStreamNonBlocking) == cudaSuccess &&
              cudaStreamCreateWithFlags(&h->s[1], cudaStreamNonBlocking) == cudaSuccess &&
              cudaEventCreateWithFlags(&h->start, cudaEventDisableTiming) == cudaSuccess &&
              cudaEventCreateWithFlags(&h->done[0], cudaEventDisableTiming) == cudaSuccess &&
              cudaEventCreateWithFlags(&h->done[1], cudaEventDisableTiming) == cudaSuccess;
    if (!ok) {
      delete h;
      return nullptr;
    }
    per_dev[dev] = h;
  }
  return per_dev[dev];
}

signrot_status check_rows(const void* x, int32_t dtype, int64_t T, int32_t n, int64_t ld,
                          signrot::Shape* sh) {
  if (dtype != SIGNROT_BF16 && dtype != SIGNROT_F32)
    return fail(SIGNROT_ERR_INVALID_ARG, "dtype %d is neither SIGNROT_BF16 nor SIGNROT_F32", dtype);
  if (T < 0) return fail(SIGNROT_ERR_INVALID_ARG, "T = %lld < 0", static_cast<long long>(T));
  if (!factor_n(n, sh))
    return fail(SIGNROT_ERR_UNSUPPORTED_N, "n = %d is not " SIGNROT_N_FORMS, n);
  if (ld < n) return fail(SIGNROT_ERR_INVALID_ARG, "ld = %lld < n = %d", static_cast<long long>(ld), n);
  if (T > 0 && x == nullptr) return fail(SIGNROT_ERR_INVALID_ARG, "x is NULL");
  if (!aligned(x, dtype == SIGNROT_BF16 ? 2 : 4))
    return fail(SIGNROT_ERR_ALIGNMENT, "x is not aligned to its element size");
  return SIGNROT_OK;
}

signrot_status run_rotate(signrot::RotateArgs& a, cudaStream_t st) {
  const auto& h = h28_state().masks;
  a.inv_sqrt_n = static_cast<float>(1.0 / std::sqrt(static_cast<double>(a.shape.n)));
  cudaError_t e = signrot::launch_rotate_fast(a, h, st);
  if (e == cudaErrorNotSupported) {
    (void)cudaGetLastError();
    e = signrot::launch_rotate_generic(a, h, gf343_state(), st);
  }
  if (e != cudaSuccess) return cuda_fail(e, "rotate launch");
  return SIGNROT_OK;
}

signrot_status rotate_impl(const void* x, int32_t dtype, int64_t T, int32_t n, int64_t ld,
                           const int8_t* d, const int8_t* s, const int32_t* kp, const float* xkp,
                           float* y, int64_t ldy, void* stream) {
  g_last_error[0] = '\0';
  signrot::Shape sh;
  signrot_status st = check_rows(x, dtype, T, n, ld, &sh);
  if (st != SIGNROT_OK) return st;
  if (d == nullptr) return fail(SIGNROT_ERR_INVALID_ARG, "d is NULL");
  if (T > 0 && y == nullptr) return fail(SIGNROT_ERR_INVALID_ARG, "y is NULL");
  if (ldy < n) return fail(SIGNROT_ERR_INVALID_ARG, "ldy < n");
  if (!aligned(y, 4)) return fail(SIGNROT_ERR_ALIGNMENT, "y is not 4-byte aligned");
  if (!aligned(kp, 4) || !aligned(xkp, 4)) return fail(SIGNROT_ERR_ALIGNMENT, "k or xk misaligned");
  if (T == 0) return SIGNROT_OK;
  signrot::RotateArgs a{};
  a.x = x;
  a.dtype = dtype;
  a.T = T;
  a.ld = ld;
  a.shape = sh;
  a.d = d;
  a.s = s;
  a.kp = kp;
  a.xkp = xkp;
  a.y = y;
  a.ldy = ldy;
  a.clip = 1.f;
  return run_rotate(a, static_cast<cudaStream_t>(stream));
}

signrot_status rotate_quant_impl(const void* x, int32_t dtype, int64_t T, int32_t n, int64_t ld,
                                 const int8_t* d, const int8_t* s, const int32_t* kp, const float* xkp,
                                 int32_t bits, float clip, uint8_t* q, float* scale, float* zero,
                                 void* stream, bool sym = false) {
  g_last_error[0] = '\0';
  signrot::Shape sh;
  signrot_status st = check_rows(x, dtype, T, n, ld, &sh);
  if (st != SIGNROT_OK) return st;
  if (bits != 4 && bits != 8) return fail(SIGNROT_ERR_UNSUPPORTED, "bits = %d; 4 and 8 are supported", bits);
  if (!(clip > 0.f && clip <= 1.f)) return fail(SIGNROT_ERR_UNSUPPORTED, "clip must lie in (0, 1]");
  if (d == nullptr) return fail(SIGNROT_ERR_INVALID_ARG, "d is NULL");
  if (T > 0 && (q == nullptr || scale == nullptr || (!sym && zero == nullptr)))
    return fail(SIGNROT_ERR_INVALID_ARG, sym ? "q and scale must be device pointers"
                                             : "q, scale and zero must be device pointers");
  if (!aligned(scale, 4) || !aligned(zero, 4))
    return fail(SIGNROT_ERR_ALIGNMENT, "scale / zero not 4-byte aligned");
  if (!aligned(kp, 4) || !aligned(xkp, 4)) return fail(SIGNROT_ERR_ALIGNMENT, "k or xk misaligned");
  if (T == 0) return SIGNROT_OK;
  signrot::RotateArgs a{};
  a.x = x;
  a.dtype = dtype;
  a.T = T;
  a.ld = ld;
  a.shape = sh;
  a.d = d;
  a.s = s;
  a.kp = kp;
  a.xkp = xkp;
  a.q = q;
  a.scale = scale;
  a.zero = sym ? nullptr : zero;
  a.clip = clip;
  a.bits = bits;
  a.sym = sym;
  return run_rotate(a, static_cast<cudaStream_t>(stream));
}

}  // namespace

extern "C" {

signrot_status signrot_calibrate(const void* x, int32_t dtype, int64_t T, int32_t n, int64_t ld,
                                 int64_t t_offset, uint64_t* ws, int32_t accumulate,
                                 int32_t* k_out, float* xk_out, void* stream) {
  signrot_status st = signrot::check_calibrate_args(x, dtype, T, n, ld, t_offset, k_out, xk_out);
  if (st != SIGNROT_OK) return st;
  if (ws == nullptr) return fail(SIGNROT_ERR_INVALID_ARG, "ws must be a device pointer");
  if (!aligned(ws, 8)) return fail(SIGNROT_ERR_ALIGNMENT, "ws is not 8-byte aligned");
  auto s = static_cast<cudaStream_t>(stream);
  cudaError_t e;
  if (!accumulate) {
    e = cudaMemsetAsync(ws, 0, sizeof(uint64_t) * static_cast<size_t>(n), s);
    if (e != cudaSuccess) return cuda_fail(e, "workspace reset");
  }
  signrot::CalibArgs a{x, dtype, T, n, ld, t_offset, reinterpret_cast<unsigned long long*>(ws)};
  if ((e = signrot::launch_calibrate_fold(a, s)) != cudaSuccess) return cuda_fail(e, "calibrate fold");
  e = signrot::launch_calibrate_argmax(reinterpret_cast<const unsigned long long*>(ws), n, k_out, xk_out, s);
  if (e != cudaSuccess) return cuda_fail(e, "calibrate argmax");
  return SIGNROT_OK;
}

signrot_status signrot_build_sign(int32_t n, const int32_t* k, const float* xk, const int8_t* d,
                                  int8_t* s_out, void* stream) {
  g_last_error[0] = '\0';
  signrot::Shape sh;
  if (!factor_n(n, &sh))
    return fail(SIGNROT_ERR_UNSUPPORTED_N, "n = %d is not " SIGNROT_N_FORMS, n);
  if (k == nullptr || xk == nullptr || d == nullptr || s_out == nullptr)
    return fail(SIGNROT_ERR_INVALID_ARG, "k, xk, d and s_out must be device pointers");
  if (!aligned(k, 4) || !aligned(xk, 4)) return fail(SIGNROT_ERR_ALIGNMENT, "k or xk misaligned");
  cudaError_t e = signrot::launch_build_sign(sh, k, xk, d, s_out, h28_state().masks, gf343_state(),
                                             static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "build_sign launch");
  return SIGNROT_OK;
}

signrot_status signrot_rotate(const void* x, int32_t dtype, int64_t T, int32_t n, int64_t ld,
                              const int8_t* d, const int8_t* s, float* y, int64_t ldy,
                              void* stream) {
  return rotate_impl(x, dtype, T, n, ld, d, s, nullptr, nullptr, y, ldy, stream);
}

signrot_status signrot_rotate_outlier(const void* x, int32_t dtype, int64_t T, int32_t n, int64_t ld,
                                      const int8_t* d, const int32_t* k, const float* xk, float* y,
                                      int64_t ldy, void* stream) {
  if (k == nullptr || xk == nullptr) return fail(SIGNROT_ERR_INVALID_ARG, "k and xk must be device pointers");
  return rotate_impl(x, dtype, T, n, ld, d, nullptr, k, xk, y, ldy, stream);
}

signrot_status signrot_rotate_quant(const void* x, int32_t dtype, int64_t T, int32_t n, int64_t ld,
                                    const int8_t* d, const int8_t* s, int32_t bits, float clip,
                                    uint8_t* q, float* scale, float* zero, void* stream) {
  return rotate_quant_impl(x, dtype, T, n, ld, d, s, nullptr, nullptr, bits, clip, q, scale, zero, stream);
}

signrot_status signrot_rotate_quant_outlier(const void* x, int32_t dtype, int64_t T, int32_t n,
                                            int64_t ld, const int8_t* d, const int32_t* k,
                                            const float* xk, int32_t bits, float clip, uint8_t* q,
                                            float* scale, float* zero, void* stream) {
  if (k == nullptr || xk == nullptr) return fail(SIGNROT_ERR_INVALID_ARG, "k and xk must be device pointers");
  return rotate_quant_impl(x, dtype, T, n, ld, d, nullptr, k, xk, bits, clip, q, scale, zero, stream);
}

signrot_status signrot_rotate_quant_sym(const void* x, int32_t dtype, int64_t T, int32_t n, int64_t ld,
                                        const int8_t* d, const int8_t* s, int32_t bits, uint8_t* q, float* scale,
                                        void* stream) {
  return rotate_quant_impl(x, dtype, T, n, ld, d, s, nullptr, nullptr, bits, 1.f, q, scale, nullptr, stream, true);
}

signrot_status signrot_rotate_quant_sym_outlier(const void* x, int32_t dtype, int64_t T, int32_t n, int64_t ld,
                                                const int8_t* d, const int32_t* k, const float* xk, int32_t bits,
                                                uint8_t* q, float* scale, void* stream) {
  if (k == nullptr || xk == nullptr) return fail(SIGNROT_ERR_INVALID_ARG, "k and xk must be device pointers");
  return rotate_quant_impl(x, dtype, T, n, ld, d, nullptr, k, xk, bits, 1.f, q, scale, nullptr, stream, true);
}

size_t signrot_host_bytes_per_token(int32_t n, int32_t dtype) {
  if (n <= 0) return 0;
  const size_t in_row = static_cast<size_t>(n) * (dtype == SIGNROT_F32 ? 4 : 2);
  return in_row + static_cast<size_t>(n) / 2 + 8;
}

signrot_status signrot_rotate_quant_host(const void* x_host, int32_t dtype, int64_t T, int32_t n,
                                         int64_t ld, const int8_t* d, const int8_t* s,
                                         const int32_t* k, const float* xk, int32_t bits, float clip,
                                         uint8_t* q_host, float* scale_host, float* zero_host,
                                         void* workspace, size_t workspace_bytes, void* stream) {
  g_last_error[0] = '\0';
  signrot::Shape sh;
  signrot_status st = check_rows(x_host, dtype, T, n, ld, &sh);
  if (st != SIGNROT_OK) return st;
  if (bits != 4) return fail(SIGNROT_ERR_UNSUPPORTED, "bits = %d; only 4 is supported", bits);
  if (!(clip > 0.f && clip <= 1.f)) return fail(SIGNROT_ERR_UNSUPPORTED, "clip must lie in (0, 1]");
  if (d == nullptr) return fail(SIGNROT_ERR_INVALID_ARG, "d is NULL");
  if ((k == nullptr) != (xk == nullptr)) return fail(SIGNROT_ERR_INVALID_ARG, "give both k and xk, or neither");
  if (k != nullptr && s != nullptr) return fail(SIGNROT_ERR_INVALID_ARG, "s and (k, xk) are exclusive");
  if (T > 0 && (q_host == nullptr || scale_host == nullptr || zero_host == nullptr || workspace == nullptr))
    return fail(SIGNROT_ERR_INVALID_ARG, "q_host, scale_host, zero_host and workspace are required");
  if (!aligned(workspace, 16)) return fail(SIGNROT_ERR_ALIGNMENT, "workspace must be 16-byte aligned");
  if (T == 0) return SIGNROT_OK;
  const size_t esz = dtype == SIGNROT_F32 ? 4 : 2;
  const size_t in_row = static_cast<size_t>(n) * esz, q_row = static_cast<size_t>(n) / 2;
  const size_t per_token = signrot_host_bytes_per_token(n, dtype);
  const size_t slack = 64;  // 16-byte alignment of the three buffers in a slot
  if (workspace_bytes < 2 * (per_token + slack))
    return fail(SIGNROT_ERR_INVALID_ARG, "workspace of %zu bytes holds no token (need >= %zu)", workspace_bytes,
                2 * (per_token + slack));
  const int64_t chunk_cap = static_cast<int64_t>((workspace_bytes / 2 - slack) / per_token);
  const int64_t chunk = chunk_cap < T ? chunk_cap : T;
  const auto up16 = [](size_t v) { return (v + 15) & ~size_t(15); };
  const size_t off_q = up16(static_cast<size_t>(chunk) * in_row);
  const size_t off_s = up16(off_q + static_cast<size_t>(chunk) * q_row);
  const size_t off_z = up16(off_s + static_cast<size_t>(chunk) * 4);
  const size_t slot_bytes = up16(off_z + static_cast<size_t>(chunk) * 4);

  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  HostStreams* hs = host_streams(dev);
  if (hs == nullptr) return fail(SIGNROT_ERR_CUDA, "could not create the copy streams");
  auto caller = static_cast<cudaStream_t>(stream);
  if ((e = cudaEventRecord(hs->start, caller)) != cudaSuccess) return cuda_fail(e, "event record");
  for (int i = 0; i < 2; ++i)
    if ((e = cudaStreamWaitEvent(hs->s[i], hs->start, 0)) != cudaSuccess) return cuda_fail(e, "stream wait");

  const auto* xb = static_cast<const uint8_t*>(x_host);
  auto* ws = static_cast<uint8_t*>(workspace);
  for (int64_t t0 = 0, c = 0; t0 < T; t0 += chunk, ++c) {
    const int64_t tc = T - t0 < chunk ? T - t0 : chunk;
    cudaStream_t cs = hs->s[c & 1];
    uint8_t* slot = ws + (c & 1) * slot_bytes;
    e = cudaMemcpy2DAsync(slot, in_row, xb + static_cast<size_t>(t0) * ld * esz, static_cast<size_t>(ld) * esz, in_row,
                          static_cast<size_t>(tc), cudaMemcpyHostToDevice, cs);
    if (e != cudaSuccess) return cuda_fail(e, "rows to device");
    signrot::RotateArgs a{};
    a.x = slot;
    a.dtype = dtype;
    a.T = tc;
    a.ld = n;
    a.shape = sh;
    a.d = d;
    a.s = s;
    a.kp = k;
    a.xkp = xk;
    a.q = slot + off_q;
    a.scale = reinterpret_cast<float*>(slot + off_s);
    a.zero = reinterpret_cast<float*>(slot + off_z);
    a.clip = clip;
    if ((st = run_rotate(a, cs)) != SIGNROT_OK) return st;
    if ((e = cudaMemcpyAsync(q_host + static_cast<size_t>(t0) * q_row, a.q, static_cast<size_t>(tc) * q_row,
                             cudaMemcpyDeviceToHost, cs)) != cudaSuccess ||
        (e = cudaMemcpyAsync(scale_host + t0, a.scale, static_cast<size_t>(tc) * 4, cudaMemcpyDeviceToHost, cs)) !=
            cudaSuccess ||
        (e = cudaMemcpyAsync(zero_host + t0, a.zero, static_cast<size_t>(tc) * 4, cudaMemcpyDeviceToHost, cs)) !=
            cudaSuccess)
      return cuda_fail(e, "codes to host");
  }
  for (int i = 0; i < 2; ++i) {
    if ((e = cudaEventRecord(hs->done[i], hs->s[i])) != cudaSuccess) return cuda_fail(e, "event record");
    if ((e = cudaStreamWaitEvent(caller, hs->done[i], 0)) != cudaSuccess) return cuda_fail(e, "stream wait");
  }
  return SIGNROT_OK;
}

signrot_status signrot_device_error(int32_t* code, int32_t clear) {
  g_last_error[0] = '\0';
  if (code == nullptr) return fail(SIGNROT_ERR_INVALID_ARG, "code is NULL");
  uint32_t v = 0, g = 0;
  cudaError_t e = signrot::read_device_error(&v, clear != 0);
  if (e != cudaSuccess) return cuda_fail(e, "device error word");
  if ((e = signrot::read_gemm_error(&g, clear != 0)) != cudaSuccess) return cuda_fail(e, "device error word");
  *code = static_cast<int32_t>(v | g);
  return SIGNROT_OK;
}

signrot_status signrot_w4a4_prepare_weights(const uint8_t* wq4, int32_t N, int32_t K, int64_t ldw4, int8_t* wq8,
                                            int64_t ldw8, int32_t* colsum, void* stream) {
  g_last_error[0] = '\0';
  if (N < 0 || K <= 0 || K % 2 != 0) return fail(SIGNROT_ERR_INVALID_ARG, "N = %d, K = %d: need N >= 0, K even", N, K);
  if (ldw4 < K / 2 || ldw8 < K) return fail(SIGNROT_ERR_INVALID_ARG, "row strides below the row lengths");
  if (N > 0 && (wq4 == nullptr || wq8 == nullptr || colsum == nullptr))
    return fail(SIGNROT_ERR_INVALID_ARG, "wq4, wq8 and colsum must be device pointers");
  if (!aligned(colsum, 4)) return fail(SIGNROT_ERR_ALIGNMENT, "colsum is not 4-byte aligned");
  if (N == 0) return SIGNROT_OK;
  cudaError_t e = signrot::launch_w4a4_prepare(wq4, ldw4, N, K, wq8, ldw8, colsum, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "weight preparation launch");
  return SIGNROT_OK;
}

signrot_status signrot_w4a4_matmul(const uint8_t* q, int64_t T, int32_t K, int64_t ldq, const float* scale,
                                   const float* zero, const int8_t* wq8, int32_t N, int64_t ldw, const float* wscale,
                                   const int32_t* colsum, float* out, int64_t ldo, void* stream) {
  g_last_error[0] = '\0';
  if (T < 0 || N < 0) return fail(SIGNROT_ERR_INVALID_ARG, "T and N must be >= 0");
  if (K <= 0 || K % 128 != 0 || K > (1 << 18))
    return fail(SIGNROT_ERR_UNSUPPORTED, "K = %d: the W4A4 product needs K a multiple of 128, at most 2^18", K);
  if (T > 0x7fffffffLL) return fail(SIGNROT_ERR_INVALID_ARG, "T too large");
  if (ldq < K / 2 || ldw < K || ldo < N) return fail(SIGNROT_ERR_INVALID_ARG, "row strides below the row lengths");
  if (T == 0 || N == 0) return SIGNROT_OK;
  if (q == nullptr || scale == nullptr || wq8 == nullptr || wscale == nullptr || colsum == nullptr || out == nullptr)
    return fail(SIGNROT_ERR_INVALID_ARG, "q, scale, wq8, wscale, colsum and out must be device pointers");
  if (!aligned(q, 16) || !aligned(wq8, 16) || ldq % 16 != 0 || ldw % 16 != 0)
    return fail(SIGNROT_ERR_ALIGNMENT, "q and wq8 must start on 16 bytes, with row strides multiples of 16 bytes");
  if (!aligned(scale, 4) || !aligned(zero, 4) || !aligned(wscale, 4) || !aligned(colsum, 4) || !aligned(out, 4))
    return fail(SIGNROT_ERR_ALIGNMENT, "scale, zero, wscale, colsum and out must be 4-byte aligned");
  signrot::GemmArgs a{};
  a.q = q;
  a.ldq = ldq;
  a.scale = scale;
  a.zero = zero;
  a.wq = wq8;
  a.ldw = ldw;
  a.wscale = wscale;
  a.colsum = colsum;
  a.out = out;
  a.ldo = ldo;
  a.T = T;
  a.N = N;
  a.K = K;
  cudaError_t e = signrot::launch_w4a4_gemm(a, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "W4A4 product launch");
  return SIGNROT_OK;
}

signrot_status signrot_get_h28(int8_t* out) {
  if (out == nullptr) return fail(SIGNROT_ERR_INVALID_ARG, "out is NULL");
  std::memcpy(out, h28_state().h, 28 * 28);
  return SIGNROT_OK;
}

signrot_status signrot_get_h344(int8_t* out) {
  if (out == nullptr) return fail(SIGNROT_ERR_INVALID_ARG, "out is NULL");
  signrot::paley_h344(out);
  return SIGNROT_OK;
}

int32_t signrot_supported_n(int32_t n) {
  signrot::Shape sh;
  return factor_n(n, &sh) ? 1 : 0;
}

const char* signrot_status_string(signrot_status status) {
  switch (status) {
    case SIGNROT_OK: return "ok";
    case SIGNROT_ERR_INVALID_ARG: return "invalid argument";
    case SIGNROT_ERR_UNSUPPORTED_N: return "unsupported row length n";
    case SIGNROT_ERR_ALIGNMENT: return "misaligned pointer";
    case SIGNROT_ERR_CUDA: return "CUDA runtime error";
    case SIGNROT_ERR_UNSUPPORTED: return "unsupported option";
    default: return "unknown status";
  }
}

const char* signrot_last_error(void) { return g_last_error; }

uint64_t signrot_kernel_launches(void) { return signrot::g_launches.load(std::memory_order_relaxed); }

}  // extern "C"

void signrot::set_last_error(const char* msg) {
  std::snprintf(g_last_error, sizeof(g_last_error), "%s", msg);
}

signrot_status signrot::check_calibrate_args(const void* x, int32_t dtype, int64_t T, int32_t n, int64_t ld,
                                             int64_t t_offset, const int32_t* k_out, const float* xk_out) {
  g_last_error[0] = '\0';
  signrot::Shape sh;
  signrot_status st = check_rows(x, dtype, T, n, ld, &sh);
  if (st != SIGNROT_OK) return st;
  if (k_out == nullptr || xk_out == nullptr) return fail(SIGNROT_ERR_INVALID_ARG, "k_out and xk_out must be device pointers");
  if (!aligned(k_out, 4) || !aligned(xk_out, 4)) return fail(SIGNROT_ERR_ALIGNMENT, "k_out and xk_out must be 4-byte aligned");
  if (t_offset < 0 || t_offset + T > 0x7fffffffLL)
    return fail(SIGNROT_ERR_INVALID_ARG, "token indices t_offset + t must stay below 2^31 - 1");
  return SIGNROT_OK;
}
