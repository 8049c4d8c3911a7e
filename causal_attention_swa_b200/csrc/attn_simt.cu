// attn_simt.cu -- pair-by-pair attention kernels on CUDA cores (float32
// arithmetic), plus the small HBM-bound helpers of the attention path.
//
// These kernels visit exactly the existing pairs of the join (j <= i when
// causal, "Show HN: Automatic deduction of FlashAttention kernel from ~25
// lines of SQL", view ATTENTION_WINDOW and check_masks_are_absent_rows): a
// masked pair is skipped by a branch, never multiplied by a zero weight, so
// non-finite values in V or dout propagate exactly as IEEE sums over the
// existing pairs.  They are the float32 path.
//
// Forward: one thread per query row keeps q (pre-scaled into the log2
// domain), the output accumulator and the running (max, sum) in registers,
// and streams 32-key K/V tiles through shared memory; the online softmax
// rescales once per 16-key chunk, and leaves an accumulator that is already
// +-inf or NaN as it is (a weight > 0 keeps its class; a rescale factor that
// underflows to 0 must not turn it into 0 * inf = NaN).
// Backward: delta_i = dout_i . out_i (prep kernel, also lse * log2 e, both
// padded to whole 128-row blocks for the tensor-core kernel); a key-major kernel
// accumulates dk_j, dv_j over the rows i that see j; a query-major kernel
// accumulates dq_i.  Two threads share a row (32 dims each, interleaved in
// float4 groups so the pair reads distinct banks) and combine their partial
// dot products with one shuffle.
#include "swa_internal.cuh"

namespace swa {
namespace {

constexpr int D = 64;

// ------------------------------------------------------------------ helpers

template <typename T>
__device__ __forceinline__ void load_rows_f32(float (*dst)[D], const T* __restrict__ src,
                                              int64_t row0, int nvalid, int rows, int tid,
                                              int nthreads) {
  for (int e = tid; e < rows * D; e += nthreads) {
    int r = e / D, c = e % D;
    dst[r][c] = (r < nvalid) ? to_f(src[(row0 + r) * D + c]) : 0.f;
  }
}

// dims owned by half h of a row pair: d = 8*u + 4*h + c, u in [0,8), c in [0,4)
__device__ __forceinline__ int pair_dim(int u, int h, int c) { return 8 * u + 4 * h + c; }

template <typename T>
__device__ __forceinline__ void load_half_row(float (&r)[32], const T* __restrict__ src,
                                              int h, float mul) {
#pragma unroll
  for (int u = 0; u < 8; ++u)
#pragma unroll
    for (int c = 0; c < 4; ++c) r[4 * u + c] = to_f(src[pair_dim(u, h, c)]) * mul;
}

__device__ __forceinline__ float dot_half(const float* __restrict__ srow, const float (&r)[32],
                                          int h) {
  float acc = 0.f;
#pragma unroll
  for (int u = 0; u < 8; ++u) {
    float4 a = *reinterpret_cast<const float4*>(srow + 8 * u + 4 * h);
    acc = fmaf(a.x, r[4 * u + 0], acc);
    acc = fmaf(a.y, r[4 * u + 1], acc);
    acc = fmaf(a.z, r[4 * u + 2], acc);
    acc = fmaf(a.w, r[4 * u + 3], acc);
  }
  return acc;
}

__device__ __forceinline__ void axpy_half(float (&acc)[32], float a, const float* __restrict__ srow,
                                          int h) {
#pragma unroll
  for (int u = 0; u < 8; ++u) {
    float4 x = *reinterpret_cast<const float4*>(srow + 8 * u + 4 * h);
    acc[4 * u + 0] = fmaf(a, x.x, acc[4 * u + 0]);
    acc[4 * u + 1] = fmaf(a, x.y, acc[4 * u + 1]);
    acc[4 * u + 2] = fmaf(a, x.z, acc[4 * u + 2]);
    acc[4 * u + 3] = fmaf(a, x.w, acc[4 * u + 3]);
  }
}

// ------------------------------------------------------------------ forward

constexpr int kFwdRows = 128;  // query rows (= threads) per block
constexpr int kFwdKeys = 32;   // keys per shared-memory tile
constexpr int kChunk = 16;     // keys per online-softmax rescale

template <typename T>
__global__ void __launch_bounds__(kFwdRows)
attn_fwd_simt_kernel(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
                     T* __restrict__ out, float* __restrict__ lse, int64_t N, int causal,
                     float scale_log2) {
  const int64_t head = blockIdx.y;
  __shared__ __align__(16) float Ks[kFwdKeys][D];
  __shared__ __align__(16) float Vs[kFwdKeys][D];

  const int tid = threadIdx.x;
  const int64_t row0 = (int64_t)blockIdx.x * kFwdRows;
  const int64_t i = row0 + tid;
  const bool row_ok = i < N;
  const T* qh = q + head * N * D;
  const T* kh = k + head * N * D;
  const T* vh = v + head * N * D;

  float qr[D], o[D];
#pragma unroll
  for (int d = 0; d < D; ++d) {
    qr[d] = row_ok ? to_f(qh[i * D + d]) * scale_log2 : 0.f;
    o[d] = 0.f;
  }
  float m = -INFINITY;  // running max of the log2-domain scores
  float l = 0.f;        // running sum of 2^(s - m)

  const int64_t key_end = causal ? imin64(N, row0 + kFwdRows) : N;
  for (int64_t t0 = 0; t0 < key_end; t0 += kFwdKeys) {
    const int nk = (int)imin64(kFwdKeys, key_end - t0);
    __syncthreads();
    load_rows_f32(Ks, kh, t0, nk, kFwdKeys, tid, kFwdRows);
    load_rows_f32(Vs, vh, t0, nk, kFwdKeys, tid, kFwdRows);
    __syncthreads();
#pragma unroll 1
    for (int c0 = 0; c0 < kFwdKeys; c0 += kChunk) {
      float s[kChunk];
      unsigned valid = 0;
      float mc = -INFINITY;
#pragma unroll
      for (int jj = 0; jj < kChunk; ++jj) {
        const int64_t j = t0 + c0 + jj;
        const bool ok = row_ok && (c0 + jj < nk) && (!causal || j <= i);
        float acc = 0.f;
        if (ok) {
          const float* kr = Ks[c0 + jj];
#pragma unroll
          for (int d4 = 0; d4 < D; d4 += 4) {
            float4 kk = *reinterpret_cast<const float4*>(kr + d4);
            acc = fmaf(qr[d4 + 0], kk.x, acc);
            acc = fmaf(qr[d4 + 1], kk.y, acc);
            acc = fmaf(qr[d4 + 2], kk.z, acc);
            acc = fmaf(qr[d4 + 3], kk.w, acc);
          }
          valid |= 1u << jj;
          mc = fmaxf(mc, acc);
        }
        s[jj] = acc;
      }
      if (valid == 0) continue;  // no existing pair for this row in the chunk
      if (mc > m) {
        const float alpha = exp2f(m - mc);  // 0 on the first chunk (m = -inf)
        l *= alpha;
#pragma unroll
        for (int d = 0; d < D; ++d) o[d] = isfinite(o[d]) ? o[d] * alpha : o[d];
        m = mc;
      }
#pragma unroll
      for (int jj = 0; jj < kChunk; ++jj) {
        if (valid & (1u << jj)) {
          const float p = exp2f(s[jj] - m);
          l += p;
          const float* vr = Vs[c0 + jj];
#pragma unroll
          for (int d4 = 0; d4 < D; d4 += 4) {
            float4 vv = *reinterpret_cast<const float4*>(vr + d4);
            o[d4 + 0] = fmaf(p, vv.x, o[d4 + 0]);
            o[d4 + 1] = fmaf(p, vv.y, o[d4 + 1]);
            o[d4 + 2] = fmaf(p, vv.z, o[d4 + 2]);
            o[d4 + 3] = fmaf(p, vv.w, o[d4 + 3]);
          }
        }
      }
    }
  }
  if (row_ok) {
    T* orow = out + (head * N + i) * D;
    const float inv = 1.f / l;
#pragma unroll
    for (int d = 0; d < D; ++d) orow[d] = from_f<T>(o[d] * inv);
    lse[head * N + i] = m * kLn2 + logf(l);
  }
}

// ------------------------------------------------------------------ backward

// Backward row statistics, 8 threads per row, into two [heads][Npad]
// float32 arrays (Npad = N rounded up to 128):
//   delta[h][i] = sum_d dout_id * out_id      (0 for the padding rows)
//   nlse2[h][i] = -lse_i * log2(e)            (-inf for the padding rows)
template <typename T>
__global__ void __launch_bounds__(256)
attn_bwd_prep_kernel(const T* __restrict__ out, const T* __restrict__ dout,
                     const float* __restrict__ lse, float* __restrict__ delta,
                     float* __restrict__ nlse2, int64_t N, int64_t Npad, int64_t rows_pad) {
  const int64_t g = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int64_t rp = g >> 3;
  const int part = (int)(g & 7);
  const int64_t head = rp / Npad, i = rp - head * Npad;
  const bool real = rp < rows_pad && i < N;
  float acc = 0.f;
  if (real) {
    const int64_t r = head * N + i;
    const T* o = out + r * D + part * 8;
    const T* d = dout + r * D + part * 8;
#pragma unroll
    for (int c = 0; c < 8; ++c) acc = fmaf(to_f(d[c]), to_f(o[c]), acc);
  }
  acc += __shfl_xor_sync(0xffffffffu, acc, 4);
  acc += __shfl_xor_sync(0xffffffffu, acc, 2);
  acc += __shfl_xor_sync(0xffffffffu, acc, 1);
  if (rp < rows_pad && part == 0) {
    delta[rp] = real ? acc : 0.f;
    nlse2[rp] = real ? -lse[head * N + i] * kLog2e : -INFINITY;
  }
}

constexpr int kBwdRows = 64;  // rows per block, two threads per row
constexpr int kBwdTile = 32;  // streamed rows per shared-memory tile

// dk_j, dv_j: key-major; rows i that see key j are streamed.
template <typename T>
__global__ void __launch_bounds__(2 * kBwdRows)
attn_bwd_dkdv_simt_kernel(const T* __restrict__ q, const T* __restrict__ k,
                          const T* __restrict__ v, const T* __restrict__ dout,
                          const float* __restrict__ lse, const float* __restrict__ delta,
                          T* __restrict__ dk, T* __restrict__ dv, int64_t N, int64_t dstride,
                          int causal, float scale, float scale_log2) {
  const int64_t head = blockIdx.y;
  __shared__ __align__(16) float Qs[kBwdTile][D];
  __shared__ __align__(16) float Ds[kBwdTile][D];
  __shared__ float Ls[kBwdTile];
  __shared__ float Es[kBwdTile];

  const int tid = threadIdx.x;
  const int h = tid & 1;
  const int64_t key0 = (int64_t)blockIdx.x * kBwdRows;
  const int64_t j = key0 + (tid >> 1);
  const bool key_ok = j < N;
  const int64_t base = head * N;

  float kr[32], vr[32], dkr[32], dvr[32];
  if (key_ok) {
    load_half_row(kr, k + (base + j) * D, h, scale_log2);
    load_half_row(vr, v + (base + j) * D, h, 1.f);
  } else {
#pragma unroll
    for (int e = 0; e < 32; ++e) { kr[e] = 0.f; vr[e] = 0.f; }
  }
#pragma unroll
  for (int e = 0; e < 32; ++e) { dkr[e] = 0.f; dvr[e] = 0.f; }

  const int64_t i_begin = causal ? key0 : 0;
  for (int64_t t0 = i_begin; t0 < N; t0 += kBwdTile) {
    const int nq = (int)imin64(kBwdTile, N - t0);
    __syncthreads();
    load_rows_f32(Qs, q + base * D, t0, nq, kBwdTile, tid, 2 * kBwdRows);
    load_rows_f32(Ds, dout + base * D, t0, nq, kBwdTile, tid, 2 * kBwdRows);
    if (tid < kBwdTile) {
      Ls[tid] = tid < nq ? lse[base + t0 + tid] * kLog2e : 0.f;
      Es[tid] = tid < nq ? delta[head * dstride + t0 + tid] : 0.f;
    }
    __syncthreads();
#pragma unroll 2
    for (int r = 0; r < kBwdTile; ++r) {
      const int64_t i = t0 + r;
      const bool ok = key_ok && r < nq && (!causal || i >= j);
      float s = dot_half(Qs[r], kr, h);
      s += __shfl_xor_sync(0xffffffffu, s, 1);
      float dp = dot_half(Ds[r], vr, h);
      dp += __shfl_xor_sync(0xffffffffu, dp, 1);
      if (ok) {
        const float p = exp2f(s - Ls[r]);
        const float ds = p * (dp - Es[r]);
        axpy_half(dvr, p, Ds[r], h);
        axpy_half(dkr, ds, Qs[r], h);
      }
    }
  }
  if (key_ok) {
    T* dkrow = dk + (base + j) * D;
    T* dvrow = dv + (base + j) * D;
#pragma unroll
    for (int u = 0; u < 8; ++u)
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        dkrow[pair_dim(u, h, c)] = from_f<T>(dkr[4 * u + c] * scale);
        dvrow[pair_dim(u, h, c)] = from_f<T>(dvr[4 * u + c]);
      }
  }
}

// dq_i: query-major; keys j in J(i) are streamed.
template <typename T>
__global__ void __launch_bounds__(2 * kBwdRows)
attn_bwd_dq_simt_kernel(const T* __restrict__ q, const T* __restrict__ k,
                        const T* __restrict__ v, const T* __restrict__ dout,
                        const float* __restrict__ lse, const float* __restrict__ delta,
                        T* __restrict__ dq, int64_t N, int64_t dstride, int causal,
                        float scale, float scale_log2) {
  const int64_t head = blockIdx.y;
  __shared__ __align__(16) float Ks[kBwdTile][D];
  __shared__ __align__(16) float Vs[kBwdTile][D];

  const int tid = threadIdx.x;
  const int h = tid & 1;
  const int64_t row0 = (int64_t)blockIdx.x * kBwdRows;
  const int64_t i = row0 + (tid >> 1);
  const bool row_ok = i < N;
  const int64_t base = head * N;

  float qr[32], dor[32], dqr[32];
  float lrow = 0.f, erow = 0.f;
  if (row_ok) {
    load_half_row(qr, q + (base + i) * D, h, scale_log2);
    load_half_row(dor, dout + (base + i) * D, h, 1.f);
    lrow = lse[base + i] * kLog2e;
    erow = delta[head * dstride + i];
  } else {
#pragma unroll
    for (int e = 0; e < 32; ++e) { qr[e] = 0.f; dor[e] = 0.f; }
  }
#pragma unroll
  for (int e = 0; e < 32; ++e) dqr[e] = 0.f;

  const int64_t key_end = causal ? imin64(N, row0 + kBwdRows) : N;
  for (int64_t t0 = 0; t0 < key_end; t0 += kBwdTile) {
    const int nk = (int)imin64(kBwdTile, key_end - t0);
    __syncthreads();
    load_rows_f32(Ks, k + base * D, t0, nk, kBwdTile, tid, 2 * kBwdRows);
    load_rows_f32(Vs, v + base * D, t0, nk, kBwdTile, tid, 2 * kBwdRows);
    __syncthreads();
#pragma unroll 2
    for (int r = 0; r < kBwdTile; ++r) {
      const int64_t j = t0 + r;
      const bool ok = row_ok && r < nk && (!causal || j <= i);
      float s = dot_half(Ks[r], qr, h);
      s += __shfl_xor_sync(0xffffffffu, s, 1);
      float dp = dot_half(Vs[r], dor, h);
      dp += __shfl_xor_sync(0xffffffffu, dp, 1);
      if (ok) {
        const float p = exp2f(s - lrow);
        const float ds = p * (dp - erow);
        axpy_half(dqr, ds, Ks[r], h);
      }
    }
  }
  if (row_ok) {
    T* dqrow = dq + (base + i) * D;
#pragma unroll
    for (int u = 0; u < 8; ++u)
#pragma unroll
      for (int c = 0; c < 4; ++c) dqrow[pair_dim(u, h, c)] = from_f<T>(dqr[4 * u + c] * scale);
  }
}

// ------------------------------------------------------------- nonfinite scan

// flags[head] = 1 if any element of that head is +-inf or NaN.  Each thread
// checks 16-byte vectors; heads hold a whole number of vectors (N*64 elements).
template <int kElemBytes>
__global__ void __launch_bounds__(256)
scan_nonfinite_kernel(const uint4* __restrict__ x, int64_t total_vec, int64_t vec_per_head,
                      int* __restrict__ flags) {
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; idx < total_vec;
       idx += stride) {
    const uint4 u = x[idx];
    const unsigned w[4] = {u.x, u.y, u.z, u.w};
    bool bad = false;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      if (kElemBytes == 2) {
        bad |= (w[e] & 0x7F80u) == 0x7F80u;
        bad |= (w[e] & 0x7F800000u) == 0x7F800000u;
      } else {
        bad |= (w[e] & 0x7F800000u) == 0x7F800000u;
      }
    }
    if (bad) flags[idx / vec_per_head] = 1;
  }
}

// Per-head information of a bf16 attention call: four int32 per head h
// (zeroed first), info[4h + 0] bit 0 = V holds an infinity or NaN, bit 1 =
// dout does; info[4h + 1], [4h + 2], [4h + 3] = the largest biased exponent
// of the finite values of V, of Q and K, and of dout.

// bf16x8 helpers: the largest biased exponent among the finite values, and
// whether any value is +-inf or NaN.
__device__ __forceinline__ unsigned maxexp8(const uint4& u) {
  const unsigned w[4] = {u.x, u.y, u.z, u.w};
  unsigned m = 0u;
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const unsigned lo = (w[e] >> 7) & 0xFFu, hi = (w[e] >> 23) & 0xFFu;
    m = max(m, lo == 0xFFu ? 0u : lo);
    m = max(m, hi == 0xFFu ? 0u : hi);
  }
  return m;
}
__device__ __forceinline__ bool nonfinite8(const uint4& u) {
  const unsigned w[4] = {u.x, u.y, u.z, u.w};
  bool bad = false;
#pragma unroll
  for (int e = 0; e < 4; ++e)
    bad |= ((w[e] & 0x7F80u) == 0x7F80u) | ((w[e] & 0x7F800000u) == 0x7F800000u);
  return bad;
}
// bf16x8 -> f16x8, round to nearest even (infinities and NaN keep their class).
__device__ __forceinline__ uint4 to_f16x8(const uint4& u) {
  const unsigned w[4] = {u.x, u.y, u.z, u.w};
  unsigned r[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const float lo = __uint_as_float(w[e] << 16), hi = __uint_as_float(w[e] & 0xFFFF0000u);
    asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r[e]) : "f"(hi), "f"(lo));
  }
  return make_uint4(r[0], r[1], r[2], r[3]);
}
__device__ __forceinline__ float dot8(const uint4& a, const uint4& b) {
  const unsigned x[4] = {a.x, a.y, a.z, a.w}, y[4] = {b.x, b.y, b.z, b.w};
  float acc = 0.f;
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    acc = fmaf(__uint_as_float(x[e] << 16), __uint_as_float(y[e] << 16), acc);
    acc = fmaf(__uint_as_float(x[e] & 0xFFFF0000u), __uint_as_float(y[e] & 0xFFFF0000u), acc);
  }
  return acc;
}

// Block-level reduction of the four info fields of one head, then one
// global atomic per field.
__device__ __forceinline__ void flush_info(unsigned fl, unsigned ve, unsigned qke, unsigned de,
                                           int* info_h, unsigned* sh) {
  fl = __reduce_or_sync(0xffffffffu, fl);
  ve = __reduce_max_sync(0xffffffffu, ve);
  qke = __reduce_max_sync(0xffffffffu, qke);
  de = __reduce_max_sync(0xffffffffu, de);
  if ((threadIdx.x & 31) == 0) {
    atomicOr(&sh[0], fl);
    atomicMax(&sh[1], ve);
    atomicMax(&sh[2], qke);
    atomicMax(&sh[3], de);
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    if (sh[0]) atomicOr(&info_h[0], (int)sh[0]);
    if (sh[1]) atomicMax(&info_h[1], (int)sh[1]);
    if (sh[2]) atomicMax(&info_h[2], (int)sh[2]);
    if (sh[3]) atomicMax(&info_h[3], (int)sh[3]);
  }
}

// Forward scan of V: info fields 0 (bit 0) and 1.  Grid (x: blocks over the
// head's 16-byte vectors, y: head).
__global__ void __launch_bounds__(256)
scan_v_info_kernel(const uint4* __restrict__ v, int64_t vec_per_head, int* __restrict__ info) {
  __shared__ unsigned sh[4];
  if (threadIdx.x < 4) sh[threadIdx.x] = 0u;
  __syncthreads();
  const int64_t head = blockIdx.y;
  const uint4* vh = v + head * vec_per_head;
  unsigned nonfinite = 0u, maxexp = 0u;
  for (int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; idx < vec_per_head;
       idx += (int64_t)gridDim.x * blockDim.x) {
    const uint4 u = vh[idx];
    nonfinite |= nonfinite8(u) ? 1u : 0u;
    maxexp = max(maxexp, maxexp8(u));
  }
  flush_info(nonfinite, maxexp, 0u, 0u, info + 4 * head, sh);
}

// Prep pass of the bf16 backward.  8 threads per row (16 bytes of each
// tensor per thread) over the padded rows [BH][Npad] (Npad = N rounded up to
// 128), 128 rows per block, so a block never spans two heads:
//   * f16 copies (round to nearest even; exact below 2^15 in magnitude) of
//     v and, when given, q and k, and dout -- the operands of the f16
//     instances (the forward reads only v's);
//   * when `out` is given: delta = sum_d dout_d out_d and nlse2 = -lse log2 e
//     (padding rows: 0 and -inf);
//   * the per-head info (all four fields; dout's only when dout is given);
//   * when `vrows` is given: per 128-row tile of V, a 128-bit mask of its
//     rows that hold an infinity or NaN ([BH][Npad / 128][4] uint32; bit
//     r % 32 of word r / 32 for row r of the tile), every word written.
constexpr int kConvRows = 128;
__global__ void __launch_bounds__(256)
attn_convert_kernel(const uint4* __restrict__ q, const uint4* __restrict__ k,
                    const uint4* __restrict__ v, const uint4* __restrict__ dout,
                    const uint4* __restrict__ out, const float* __restrict__ lse,
                    uint4* __restrict__ q16, uint4* __restrict__ k16, uint4* __restrict__ v16,
                    uint4* __restrict__ do16, float* __restrict__ delta,
                    float* __restrict__ nlse2, int* __restrict__ info,
                    unsigned* __restrict__ vrows, int64_t N, int64_t Npad) {
  __shared__ unsigned sh[4];
  __shared__ unsigned rows_nf[kConvRows / 32];  // this tile's rows with a non-finite V entry
  if (threadIdx.x < 4) sh[threadIdx.x] = 0u;
  if (threadIdx.x < kConvRows / 32) rows_nf[threadIdx.x] = 0u;
  __syncthreads();
  const int64_t rp0 = (int64_t)blockIdx.x * kConvRows;
  const int64_t head = rp0 / Npad;
  const int part = threadIdx.x & 7;
  unsigned fl = 0u, ve = 0u, qke = 0u, de = 0u;
#pragma unroll 1
  for (int it = 0; it < kConvRows / 32; ++it) {
    const int64_t rp = rp0 + it * 32 + (threadIdx.x >> 3);
    const int64_t i = rp - head * Npad;
    const bool real = i < N;
    float acc = 0.f;
    if (real) {
      const int64_t vec = (head * N + i) * 8 + part;
      uint4 x;
      if (q != nullptr) {
        x = q[vec];
        q16[vec] = to_f16x8(x);
        qke = max(qke, maxexp8(x));
        x = k[vec];
        k16[vec] = to_f16x8(x);
        qke = max(qke, maxexp8(x));
      }
      x = v[vec];
      v16[vec] = to_f16x8(x);
      ve = max(ve, maxexp8(x));
      if (nonfinite8(x)) {
        fl |= 1u;
        const int r = it * 32 + (threadIdx.x >> 3);  // row within the tile
        atomicOr(&rows_nf[r >> 5], 1u << (r & 31));
      }
      if (dout != nullptr) {
        x = dout[vec];
        do16[vec] = to_f16x8(x);
        de = max(de, maxexp8(x));
        fl |= nonfinite8(x) ? 2u : 0u;
        if (out != nullptr) acc = dot8(x, out[vec]);
      }
    }
    if (out != nullptr) {
      acc += __shfl_xor_sync(0xffffffffu, acc, 4);
      acc += __shfl_xor_sync(0xffffffffu, acc, 2);
      acc += __shfl_xor_sync(0xffffffffu, acc, 1);
      if (part == 0) {
        delta[rp] = real ? acc : 0.f;
        nlse2[rp] = real ? -lse[head * N + i] * kLog2e : -INFINITY;
      }
    }
  }
  flush_info(fl, ve, qke, de, info + 4 * head, sh);  // (its __syncthreads covers rows_nf)
  if (vrows != nullptr && threadIdx.x < kConvRows / 32)
    vrows[(int64_t)blockIdx.x * (kConvRows / 32) + threadIdx.x] = rows_nf[threadIdx.x];
}

template <typename T>
cudaError_t fwd_simt(const void* q, const void* k, const void* v, void* out, float* lse,
                     int64_t BH, int64_t N, int causal, float scale, cudaStream_t s) {
  dim3 grid((unsigned)((N + kFwdRows - 1) / kFwdRows), (unsigned)BH);
  attn_fwd_simt_kernel<T><<<grid, kFwdRows, 0, s>>>(
      (const T*)q, (const T*)k, (const T*)v, (T*)out, lse, N, causal, scale * kLog2e);
  return cudaGetLastError();
}

template <typename T>
cudaError_t bwd_simt(const void* q, const void* k, const void* v, const void* dout,
                     const float* lse, const float* delta, int64_t dstride, void* dq, void* dk,
                     void* dv, int64_t BH, int64_t N, int causal, float scale, cudaStream_t s) {
  dim3 grid((unsigned)((N + kBwdRows - 1) / kBwdRows), (unsigned)BH);
  attn_bwd_dkdv_simt_kernel<T><<<grid, 2 * kBwdRows, 0, s>>>(
      (const T*)q, (const T*)k, (const T*)v, (const T*)dout, lse, delta, (T*)dk, (T*)dv, N,
      dstride, causal, scale, scale * kLog2e);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  attn_bwd_dq_simt_kernel<T><<<grid, 2 * kBwdRows, 0, s>>>(
      (const T*)q, (const T*)k, (const T*)v, (const T*)dout, lse, delta, (T*)dq, N, dstride,
      causal, scale, scale * kLog2e);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_scan_nonfinite(swa_dtype dt, const void* x, int64_t heads,
                                  int64_t elems_per_head, int* flags, cudaStream_t s,
                                  int* launches) {
  const int eb = dt == SWA_BF16 ? 2 : 4;
  const int64_t vec_per_head = elems_per_head * eb / 16;
  const int64_t total = vec_per_head * heads;
  int64_t blocks = (total + 255) / 256;
  if (blocks > 148 * 8) blocks = 148 * 8;
  if (blocks < 1) blocks = 1;
  if (eb == 2)
    scan_nonfinite_kernel<2><<<(unsigned)blocks, 256, 0, s>>>((const uint4*)x, total,
                                                              vec_per_head, flags);
  else
    scan_nonfinite_kernel<4><<<(unsigned)blocks, 256, 0, s>>>((const uint4*)x, total,
                                                              vec_per_head, flags);
  *launches += 1;
  return cudaGetLastError();
}

cudaError_t launch_scan_v_info(const void* v, int64_t heads, int64_t elems_per_head,
                               int* info, cudaStream_t s, int* launches) {
  const int64_t vec_per_head = elems_per_head * 2 / 16;
  int64_t bx = (vec_per_head + 256 * 4 - 1) / (256 * 4);  // about four vectors per thread
  if (bx > 1024) bx = 1024;
  if (bx < 1) bx = 1;
  dim3 grid((unsigned)bx, (unsigned)heads);
  scan_v_info_kernel<<<grid, 256, 0, s>>>((const uint4*)v, vec_per_head, info);
  *launches += 1;
  return cudaGetLastError();
}

cudaError_t launch_attn_convert(const void* q, const void* k, const void* v, const void* dout,
                                const void* out, const float* lse, void* q16, void* k16,
                                void* v16, void* do16, float* delta, float* nlse2, int* info,
                                unsigned* vrows, int64_t BH, int64_t N, cudaStream_t s,
                                int* launches) {
  const int64_t Npad = pad128(N);
  const int64_t blocks = BH * Npad / kConvRows;
  attn_convert_kernel<<<(unsigned)blocks, 256, 0, s>>>(
      (const uint4*)q, (const uint4*)k, (const uint4*)v, (const uint4*)dout, (const uint4*)out,
      lse, (uint4*)q16, (uint4*)k16, (uint4*)v16, (uint4*)do16, delta, nlse2, info, vrows, N,
      Npad);
  *launches += 1;
  return cudaGetLastError();
}

cudaError_t launch_attn_fwd_simt(swa_dtype dt, const void* q, const void* k, const void* v,
                                 void* out, float* lse, int64_t BH, int64_t N, int causal,
                                 float scale, cudaStream_t s, int* launches) {
  *launches += 1;
  if (dt == SWA_BF16)
    return fwd_simt<__nv_bfloat16>(q, k, v, out, lse, BH, N, causal, scale, s);
  return fwd_simt<float>(q, k, v, out, lse, BH, N, causal, scale, s);
}

cudaError_t launch_attn_bwd_prep(swa_dtype dt, const void* out, const void* dout,
                                 const float* lse, float* delta, float* nlse2, int64_t BH,
                                 int64_t N, int64_t Npad, cudaStream_t s, int* launches) {
  const int64_t rows_pad = BH * Npad;
  const unsigned blocks = (unsigned)((rows_pad * 8 + 255) / 256);
  if (dt == SWA_BF16)
    attn_bwd_prep_kernel<__nv_bfloat16><<<blocks, 256, 0, s>>>(
        (const __nv_bfloat16*)out, (const __nv_bfloat16*)dout, lse, delta, nlse2, N, Npad,
        rows_pad);
  else
    attn_bwd_prep_kernel<float><<<blocks, 256, 0, s>>>((const float*)out, (const float*)dout,
                                                       lse, delta, nlse2, N, Npad, rows_pad);
  *launches += 1;
  return cudaGetLastError();
}

cudaError_t launch_attn_bwd_simt(swa_dtype dt, const void* q, const void* k, const void* v,
                                 const void* dout, const float* lse, const float* delta,
                                 int64_t dstride, void* dq, void* dk, void* dv, int64_t BH,
                                 int64_t N, int causal, float scale, cudaStream_t s,
                                 int* launches) {
  *launches += 2;
  if (dt == SWA_BF16)
    return bwd_simt<__nv_bfloat16>(q, k, v, dout, lse, delta, dstride, dq, dk, dv, BH, N, causal,
                                   scale, s);
  return bwd_simt<float>(q, k, v, dout, lse, delta, dstride, dq, dk, dv, BH, N, causal, scale,
                         s);
}

}  // namespace swa
