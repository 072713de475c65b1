// Internal launch interface between the C ABI (signrot_abi.cu) and the kernels.
#pragma once

#include <cstdint>

#include <cuda_runtime.h>

namespace signrot {

// Counts every kernel launch the library issues (read by signrot_kernel_launches).
void count_launch(int n = 1);

// Sets the message signrot_last_error returns on this host thread.
void set_last_error(const char* msg);

// The argument checks signrot_calibrate makes on everything but its workspace (rows, n, outputs,
// token offsets); clears the last-error message first, sets it on failure. No CUDA call.
int32_t check_calibrate_args(const void* x, int32_t dtype, int64_t T, int32_t n, int64_t ld, int64_t t_offset,
                             const int32_t* k_out, const float* xk_out);

// Library-owned Paley matrices (paley.cpp), row-major, entries +/-1.
void paley_h28(int8_t h[28][28]);
void paley_h344(int8_t* h);  // [344 * 344]

// H_28 as sign masks: bit c of row[a] is set iff H_28[a][c] == -1. Passed by value in kernel
// parameters (constant bank), so no per-device state has to be initialised.
struct H28Masks {
  uint32_t row[28];
};

// The nonzero squares of GF(343) = GF(7)[t]/(t^3 + t + 1) (bit e set iff element e is one),
// element e = c0 + 7 c1 + 49 c2. With them H_344[1+e][1+f] = -1 iff e != f and e - f (digitwise
// mod 7) is a non-square; row 0 is all +1 and column 0 below it all -1. Passed by value.
struct GF343Squares {
  uint32_t bits[11];
};
GF343Squares gf343_squares();

enum : int32_t { kBF16 = 0, kF32 = 1 };

// n = F * 2^logM, F in {1, 28, 344}.
struct Shape {
  int32_t n;
  int32_t F;
  int32_t logM;
};

struct RotateArgs {
  const void* x;
  int32_t dtype;
  int64_t T;
  int64_t ld;
  Shape shape;
  const int8_t* d;  // [n] +/-1
  const int8_t* s;  // [n] +/-1 or null
  // sign vector given by its outlier channel instead (s_j = sgn(H[j,k] D_k x_k)), read on device
  const int32_t* kp;
  const float* xkp;
  // check path (fp32 y) -- y != null
  float* y;
  int64_t ldy;
  // quantized path -- q != null
  uint8_t* q;
  float* scale;
  float* zero;  // asymmetric grid only
  float clip;   // asymmetric grid only
  int32_t bits = 4;  // 4: two codes per byte; 8: one per byte
  bool sym = false;  // symmetric grid (codes -L..L, no zero-point) instead of the asymmetric one
  float inv_sqrt_n;  // fp32(1 / sqrt(n))
};

// Generic row kernel: any supported n, any element-aligned x. One CTA per row (grid-stride).
cudaError_t launch_rotate_generic(const RotateArgs& a, const H28Masks& h, const GF343Squares& sq,
                                  cudaStream_t st);

// Fast fused kernels for the shapes they cover; return cudaErrorNotSupported when the shape or
// the alignment is not theirs (the caller then uses the generic kernel).
cudaError_t launch_rotate_fast(const RotateArgs& a, const H28Masks& h, cudaStream_t st);

// Reads (and optionally clears) the device error word set by a kernel whose bounded wait expired.
cudaError_t read_device_error(uint32_t* out, bool clear);
cudaError_t read_gemm_error(uint32_t* out, bool clear);  // the same, for the W4A4 GEMM

// The driver's cuTensorMapEncodeTiled (PFN_cuTensorMapEncodeTiled_v12000), looked up once; null if
// the driver does not provide it.
void* tensor_map_encoder();

// W4A4 down projection (w4a4_gemm.cu): out[t, o] = scale_t wscale_o (sum_j q_tj Q_oj - zero_t c_o).
struct GemmArgs {
  const uint8_t* q;      // [T, K/2] packed activation codes 0..15, element 2i low nibble
  int64_t ldq;           // bytes between rows of q
  const float* scale;    // [T]
  const float* zero;     // [T] or null (symmetric activations: zero = 0)
  const int8_t* wq;      // [N, K] weight codes, one per byte
  int64_t ldw;           // bytes between rows of wq
  const float* wscale;   // [N]
  const int32_t* colsum; // [N]: c_o = sum_j wq[o, j]
  float* out;            // [T, N] fp32
  int64_t ldo;           // elements between rows of out
  int64_t T;
  int32_t N, K;
};
cudaError_t launch_w4a4_gemm(const GemmArgs& a, cudaStream_t st);
cudaError_t launch_w4a4_prepare(const uint8_t* wq4, int64_t ldw4, int32_t N, int32_t K, int8_t* wq8, int64_t ldw8,
                                int32_t* colsum, cudaStream_t st);

struct CalibArgs {
  const void* x;
  int32_t dtype;
  int64_t T;
  int32_t n;
  int64_t ld;
  int64_t t_offset;
  unsigned long long* ws;
};
cudaError_t launch_calibrate_fold(const CalibArgs& a, cudaStream_t st);
cudaError_t launch_calibrate_argmax(const unsigned long long* ws, int32_t n, int32_t* k_out,
                                    float* xk_out, cudaStream_t st);
cudaError_t launch_build_sign(Shape shape, const int32_t* k, const float* xk, const int8_t* d,
                              int8_t* s_out, const H28Masks& h, const GF343Squares& sq, cudaStream_t st);

}  // namespace signrot
