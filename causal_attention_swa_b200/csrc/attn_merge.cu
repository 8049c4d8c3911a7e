// attn_merge.cu -- merge of two partial attention results over disjoint key
// sets (sequence sharding: a rank's queries meet the key blocks of the
// other ranks one at a time).
//
// The method's output is a softmax-weighted average over the existing
// pairs ("Show HN: Automatic deduction of FlashAttention kernel from ~25
// lines of SQL", page 2, the view ATTENTION_WINDOW: out_i = sum_j w_ij v_j /
// z_i with w = exp(s - max)).  Split the keys j of row i into two disjoint
// sets with partial results (out_a, lse_a) and (out_b, lse_b), lse = max +
// ln z of its set.  Then, exactly,
//   lse = ln(e^lse_a + e^lse_b)
//   out = e^(lse_a - lse) out_a + e^(lse_b - lse) out_b
// (the two weights are the sets' shares of the row's normaliser), the same
// rescaling FlashAttention applies between key blocks.  A set that holds
// no key of the row has lse = -inf and weight 0; its term is left out
// rather than multiplied (its out may hold anything).
//
// One row of 64 values per 8 threads (16 bytes of the partial each); the
// accumulator is float32 [rows][64] plus lse [rows] (natural log).  HBM
// bound: 128 + 256 + 256 bytes per bf16 row (partial in, accumulator in and
// out), plus 128 when the final result is written.
#include <cuda_bf16.h>

#include "swa_internal.cuh"

namespace swa {
namespace {

constexpr int kMergeThreads = 256;  // 32 rows per block

template <typename T>
struct Vec8;  // eight values of the partial / final output: 16 or 32 bytes

template <>
struct Vec8<__nv_bfloat16> {
  static __device__ __forceinline__ void load(const void* base, int64_t row, int part,
                                              float (&x)[8]) {
    const uint4 u = reinterpret_cast<const uint4*>(base)[row * 8 + part];
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      x[2 * e] = __uint_as_float(w[e] << 16);
      x[2 * e + 1] = __uint_as_float(w[e] & 0xFFFF0000u);
    }
  }
  static __device__ __forceinline__ void store(void* base, int64_t row, int part,
                                               const float (&x)[8]) {
    uint32_t w[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const __nv_bfloat162 h = __floats2bfloat162_rn(x[2 * e], x[2 * e + 1]);
      w[e] = *reinterpret_cast<const uint32_t*>(&h);
    }
    reinterpret_cast<uint4*>(base)[row * 8 + part] = make_uint4(w[0], w[1], w[2], w[3]);
  }
};

template <>
struct Vec8<float> {
  static __device__ __forceinline__ void load(const void* base, int64_t row, int part,
                                              float (&x)[8]) {
    const float4* p = reinterpret_cast<const float4*>(base) + (row * 8 + part) * 2;
    const float4 a = p[0], b = p[1];
    x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
    x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
  }
  static __device__ __forceinline__ void store(void* base, int64_t row, int part,
                                               const float (&x)[8]) {
    float4* p = reinterpret_cast<float4*>(base) + (row * 8 + part) * 2;
    p[0] = make_float4(x[0], x[1], x[2], x[3]);
    p[1] = make_float4(x[4], x[5], x[6], x[7]);
  }
};

template <typename T>
__global__ void __launch_bounds__(kMergeThreads)
attn_merge_kernel(const void* __restrict__ out_part, const float* __restrict__ lse_part,
                  float* __restrict__ out_acc, float* __restrict__ lse_acc,
                  void* __restrict__ out_final, int64_t rows, int first) {
  const int64_t row = (int64_t)blockIdx.x * (kMergeThreads / 8) + (threadIdx.x >> 3);
  const int part = threadIdx.x & 7;  // columns 8 part .. 8 part + 7
  const bool valid = row < rows;
  // the eight threads of a row all read lse_acc[row] before one of them
  // overwrites it (__syncwarp below; no thread leaves early)
  float p[8] = {}, a[8] = {};
  float lse = -INFINITY;
  if (valid) {
    Vec8<T>::load(out_part, row, part, p);
    const float lb = lse_part[row];
    if (first) {
      lse = lb;
#pragma unroll
      for (int e = 0; e < 8; ++e) a[e] = p[e];
    } else {
      const float la = lse_acc[row];
      Vec8<float>::load(out_acc, row, part, a);
      const float m = fmaxf(la, lb);
      if (m == -INFINITY) {  // neither set holds a key of this row yet
        lse = -INFINITY;
      } else {
        lse = m + logf(expf(la - m) + expf(lb - m));
        const float wa = expf(la - lse), wb = expf(lb - lse);
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const float ta = wa > 0.f ? wa * a[e] : 0.f;  // an empty set's term is left out
          const float tb = wb > 0.f ? wb * p[e] : 0.f;
          a[e] = ta + tb;
        }
      }
    }
  }
  __syncwarp();
  if (!valid) return;
  Vec8<float>::store(out_acc, row, part, a);
  if (part == 0) lse_acc[row] = lse;
  if (out_final != nullptr) Vec8<T>::store(out_final, row, part, a);
}

// float32 -> bf16 (round to nearest even), eight values per thread.
__global__ void __launch_bounds__(256)
f32_to_bf16_kernel(const float4* __restrict__ src, uint4* __restrict__ dst, int64_t n8) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n8) return;
  const float4 a = src[2 * i], b = src[2 * i + 1];
  const float x[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
  uint32_t w[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(x[2 * e], x[2 * e + 1]);
    w[e] = *reinterpret_cast<const uint32_t*>(&h);
  }
  dst[i] = make_uint4(w[0], w[1], w[2], w[3]);
}

}  // namespace

cudaError_t launch_f32_to_bf16(const float* src, void* dst, int64_t n, cudaStream_t s,
                               int* launches) {
  const int64_t n8 = n / 8;
  f32_to_bf16_kernel<<<(unsigned)((n8 + 255) / 256), 256, 0, s>>>(
      reinterpret_cast<const float4*>(src), static_cast<uint4*>(dst), n8);
  *launches += 1;
  return cudaGetLastError();
}

cudaError_t launch_attn_merge(swa_dtype dt, const void* out_part, const float* lse_part,
                              float* out_acc, float* lse_acc, void* out_final, int64_t rows,
                              int first, cudaStream_t s, int* launches) {
  const int64_t blocks = (rows + kMergeThreads / 8 - 1) / (kMergeThreads / 8);
  if (dt == SWA_BF16)
    attn_merge_kernel<__nv_bfloat16><<<(unsigned)blocks, kMergeThreads, 0, s>>>(
        out_part, lse_part, out_acc, lse_acc, out_final, rows, first);
  else
    attn_merge_kernel<float><<<(unsigned)blocks, kMergeThreads, 0, s>>>(
        out_part, lse_part, out_acc, lse_acc, out_final, rows, first);
  *launches += 1;
  return cudaGetLastError();
}

}  // namespace swa
