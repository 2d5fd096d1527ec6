// Shared device/host helpers of libmoe (sm_100a only).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>
#include <stdint.h>

#include "moe.h"

#if defined(__CUDA_ARCH__) && (__CUDA_ARCH__ < 1000)
#error "libmoe targets sm_100a (B200) only"
#endif

namespace moe {

// ---------------------------------------------------------------- host side
void set_error(const char* fmt, ...);
void count_launch();

#define MOE_CHECK_ARG(cond, ...)                     \
  do {                                               \
    if (!(cond)) {                                   \
      ::moe::set_error(__VA_ARGS__);                 \
      return MOE_ERR_INVALID_ARG;                    \
    }                                                \
  } while (0)

#define MOE_CHECK_LAUNCH(what)                                                   \
  do {                                                                           \
    ::moe::count_launch();                                                       \
    cudaError_t e_ = cudaGetLastError();                                         \
    if (e_ != cudaSuccess) {                                                     \
      ::moe::set_error("%s: %s", what, cudaGetErrorString(e_));                  \
      return MOE_ERR_CUDA;                                                       \
    }                                                                            \
  } while (0)

#define MOE_TRY(expr)                         \
  do {                                        \
    moe_status_t s_ = (expr);                 \
    if (s_ != MOE_OK) return s_;              \
  } while (0)

// tensor-core router (grouped_gemm.cu): logits, top-k (k <= 8), gates,
// in-block ranks and per-128-token-block histograms
moe_status_t router_tc(const void* x, const void* wsplit, const float* bias, int T, int d, int E,
                       int k, float* logits, int32_t* topk, float* gates, int32_t* rank,
                       int32_t* hist, int32_t* status, cudaStream_t s);

// moe_grouped_gemm_dgrad with an optional rank-1 epilogue term (EPI_NONE):
// dA[row, n] += row_scale[row] * col_vec[e * K + n] on the rows of group e
moe_status_t grouped_gemm_dgrad(int dt, const void* dC, const uint8_t* dC_sc, const void* B,
                                const uint8_t* B_sc, const void* B3, const uint8_t* B3_sc,
                                const int32_t* poff, int E, int A_pad_max, int N, int K,
                                int epilogue, const void* aux, void* dA, const float* row_scale,
                                const float* col_vec, int32_t* dev_status, cudaStream_t s);

// moe_grouped_gemm_wgrad whose per-group reduction stops after the group's
// last real row (offsets: unpadded group offsets, E + 1 ints, or null)
moe_status_t grouped_gemm_wgrad(int dt, const void* A, const uint8_t* A_sc, const void* dC,
                                const uint8_t* dC_sc, const int32_t* poff, const int32_t* offsets,
                                int E, int A_pad_max, int K, int N, void* dB, void* dB3,
                                int32_t* dev_status, cudaStream_t s);

// Weight-gradient grouped GEMM (BF16) on SM pairs (grouped_gemm_pair.cu):
// dB[e] = A_e^T dC_e (+ dB3 from dC's second N half), reduced over group e
// up to its last real row; A the padded buffer.  K % 256 == 0, N % 256 == 0.
moe_status_t grouped_gemm_wgrad_pair(const void* A, const void* dC, const int32_t* poff,
                                     const int32_t* offsets,
                                     int E, int A_pad_max, int K, int N, void* dB, void* dB3,
                                     int32_t* dev_status, cudaStream_t s);

// Tokens-N grouped GEMM (BF16; grouped_gemm_tn.cu): weights on the MMA's M
// side, an expert's real rows split evenly over token blocks of <= 256 on
// the N side, padding rows after the last real row written as zeros.
// epilogue MOE_EPI_SWIGLU: C = h [A_pad, N], aux = [XW | XW3]; MOE_EPI_NONE:
// C = X W (MN-major weights [E, K, N]) or, with w_kmajor, C = X[:, :K/2] W^T
// + X[:, K/2:] W3^T (weights [E, N, K/2]; W3 null: C = X W^T) plus the
// optional rank-1 term row_scale[row] * col_vec[e * N + n].  offsets: the
// unpadded group offsets, or null (every padded row counts as real).
moe_status_t gemm_tn(int epilogue, const void* X, const void* W, const void* W3, int w_kmajor,
                     const int32_t* poff, const int32_t* offsets, int E, int A_pad_max, int N,
                     int K, void* C, void* aux, const float* row_scale, const float* col_vec,
                     int32_t* dev_status, cudaStream_t s);

// out[cols, rows] = in[rows, cols]^T (fp32)
moe_status_t transpose_f32(const float* in, int rows, int cols, float* out, cudaStream_t s);

// The driver's tensor-map encoder, looked up once per process (thread-safe);
// null if the driver does not provide it.
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder();

// Raise a kernel's dynamic shared-memory limit to `bytes` on the current
// device.  The attribute is per device, so it is set once per (kernel,
// device) under a lock, and recorded only when the call succeeds.
moe_status_t set_smem_limit(const void* kernel, size_t bytes, const char* what);

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline size_t round_up(size_t v, size_t a) { return (v + a - 1) / a * a; }
int num_sms();

// ---------------------------------------------------------------- device side
__device__ __forceinline__ void report(int32_t* status, int32_t bit) {
  if (status) atomicOr(status, bit);
}

// 8 bf16 <-> 8 fp32 through one 16-byte vector
__device__ __forceinline__ void unpack8(const uint4& v, float* f) {
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float2 t = __bfloat1622float2(h[i]);
    f[2 * i] = t.x;
    f[2 * i + 1] = t.y;
  }
}

__device__ __forceinline__ uint4 pack8(const float* f) {
  uint4 v;
  __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&v);
#pragma unroll
  for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(f[2 * i], f[2 * i + 1]);
  return v;
}

__device__ __forceinline__ uint32_t pack2(float a, float b) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}

__device__ __forceinline__ uint4 ldg_stream(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

}  // namespace moe
