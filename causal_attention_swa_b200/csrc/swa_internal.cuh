// swa_internal.cuh -- declarations shared by the translation units of
// libswa.so (launchers, device helpers).  Not part of the public ABI.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/swa.h"

namespace swa {

// Error codes a kernel writes into the device error word (first writer wins).
enum DeviceError : unsigned {
  kDevOk = 0,
  kDevTimeoutFull = 1,   // a wait for a "full" (data landed) barrier ran out
  kDevTimeoutEmpty = 2,  // a wait for an "empty" (slot released) barrier ran out
  kDevTimeoutMma = 3,    // a wait for an MMA completion ran out
  kDevTimeoutOther = 4,
  kDevSmemAlign = 5,     // dynamic shared memory not 1024-byte aligned (kernel did nothing)
};

__host__ __device__ __forceinline__ int64_t pad128(int64_t n) { return (n + 127) / 128 * 128; }
__host__ __device__ __forceinline__ int64_t imin64(int64_t a, int64_t b) { return a < b ? a : b; }

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

// Device-side element conversion.
__device__ __forceinline__ float to_f(float x) { return x; }
__device__ __forceinline__ float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }
template <typename T> __device__ __forceinline__ T from_f(float x);
template <> __device__ __forceinline__ float from_f<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}

// ------------------------------------------------- shared C-ABI bookkeeping
// (swa_api.cu): error message, argument checks, device error word and the
// per-thread launch count, for entry points defined in other files.
swa_status api_fail(swa_status st, const char* msg);
swa_status api_cuda_fail(cudaError_t e, const char* where);
swa_status api_check_attn_shape(int64_t B, int64_t H, int64_t N, int64_t D, swa_dtype dt);
unsigned* api_error_word(swa_status* st);
void api_begin_call();
void api_end_call(int launches);

// ---------------------------------------------------------------- launchers
// Each returns the launch's cudaError_t and adds the number of kernels it
// enqueued to *launches.

cudaError_t launch_scan_nonfinite(swa_dtype dt, const void* x, int64_t heads,
                                  int64_t elems_per_head, int* flags, cudaStream_t s,
                                  int* launches);

// Per-head information of a bf16 call: kHeadInfoInts int32 per head (zeroed
// by the caller): [0] bit 0 = V holds an infinity or NaN, bit 1 = dout does;
// [1], [2], [3] = the largest biased exponent of the finite values of V, of
// Q and K, of dout.
constexpr int kHeadInfoInts = 4;

// Fills fields 0 (bit 0) and 1 from a scan of V (the forward's needs).
cudaError_t launch_scan_v_info(const void* v, int64_t heads, int64_t elems_per_head,
                               int* info, cudaStream_t s, int* launches);

// Merge of a partial attention result over a disjoint key set into a
// float32 accumulator (attn_merge.cu): out_part [rows][64] of dt, lse_part
// [rows]; out_acc [rows][64] float32, lse_acc [rows] (in/out; ignored on
// input when `first`); out_final (nullable) receives the merged rows in dt.
cudaError_t launch_attn_merge(swa_dtype dt, const void* out_part, const float* lse_part,
                              float* out_acc, float* lse_acc, void* out_final, int64_t rows,
                              int first, cudaStream_t s, int* launches);

// float32 -> bf16 of n values (n a multiple of 8; 16-byte aligned buffers).
cudaError_t launch_f32_to_bf16(const float* src, void* dst, int64_t n, cudaStream_t s,
                               int* launches);

// The prep pass over [BH][N][64] bf16 tensors: f16 copies of v (and of q and
// k if q is non-null, of dout if non-null) into v16 (q16, k16, do16); with
// `out` non-null (dout then too) delta = dout . out and nlse2 = -lse log2 e
// per row, [BH][Npad] with padding rows 0 and -inf; the per-head info; if
// vrows is non-null, per 128-row tile of V the mask of its rows that hold an
// infinity or NaN ([BH][Npad / 128][4] uint32, every word written).
cudaError_t launch_attn_convert(const void* q, const void* k, const void* v, const void* dout,
                                const void* out, const float* lse, void* q16, void* k16,
                                void* v16, void* do16, float* delta, float* nlse2, int* info,
                                unsigned* vrows, int64_t BH, int64_t N, cudaStream_t s,
                                int* launches);

cudaError_t launch_attn_fwd_simt(swa_dtype dt, const void* q, const void* k, const void* v,
                                 void* out, float* lse, int64_t BH, int64_t N, int causal,
                                 float scale, cudaStream_t s, int* launches);

// delta[h][i] and nlse2[h][i] = -lse * log2 e, both [BH][Npad] (Npad = N
// rounded up to 128; padding rows 0 and -inf).
cudaError_t launch_attn_bwd_prep(swa_dtype dt, const void* out, const void* dout,
                                 const float* lse, float* delta, float* nlse2, int64_t BH,
                                 int64_t N, int64_t Npad, cudaStream_t s, int* launches);

cudaError_t launch_attn_bwd_simt(swa_dtype dt, const void* q, const void* k, const void* v,
                                 const void* dout, const float* lse, const float* delta,
                                 int64_t dstride, void* dq, void* dk, void* dv, int64_t BH,
                                 int64_t N, int causal, float scale, cudaStream_t s,
                                 int* launches);

size_t nw_partials_bytes(int64_t M, int64_t S);
// targets [M, dims], sources [S, dims] (dims = 1, 2 or 3).
cudaError_t launch_nw_partial(const float* targets, int64_t M, const float* sources,
                              const float* vals, int64_t S, int dims, float h, float* partials,
                              cudaStream_t s, int* launches);
cudaError_t launch_nw_finalize(int64_t M, int64_t S, const float* partials, float* out,
                               cudaStream_t s, int* launches);

// Backward of the regrid (nw_grad.cu): workspace bytes and the four launches.
size_t nw_bwd_workspace_bytes(int64_t M, int64_t S);
cudaError_t launch_nw_bwd(const float* targets, int64_t M, const float* sources,
                          const float* vals, int64_t S, int dims, float h, const float* gout,
                          float* dtargets, float* dsources, float* dvals, float* ws,
                          cudaStream_t s, int* launches);

}  // namespace swa
