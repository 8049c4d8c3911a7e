// nw_grad.cu -- backward of the Nadaraya-Watson regrid on CUDA cores.
//
// The regrid of "Show HN: Automatic deduction of FlashAttention kernel from
// ~25 lines of SQL" (query NADARAYA_WATSON) is the same softmax-weighted
// average over a join as attention -- P_pq = w_pq / Z_p with
// w_pq = exp(-|t_p - s_q|^2 / h^2), out_p = sum_q P_pq v_q -- and its
// gradient has attention's shape (the page's einfold docstring: one rule
// for any softmax-weighted average whose scores come from a join).  For an
// upstream gradient g_p = dL/dout_p:
//   dv_q  = sum_p g_p P_pq
//   dt_p  = (-2/h^2) (g_p / Z_p) sum_q w_pq (v_q - out_p) (t_p - s_q)
//   ds_q  = (+2/h^2) sum_p (g_p / Z_p) w_pq (v_q - out_p) (t_p - s_q)
// Two passes, each over the whole pair grid with one MUFU ex2 per pair (the
// bandwidth and the base change folded into the staged coordinates as in
// the forward, c = sqrt(log2 e) / h, so w = 2^-|c (t - s)|^2):
//   target pass  threads hold targets; per (source chunk, target) partial
//                sums Z, C = sum w v, A = sum w v c(t - s), B = sum w c(t - s);
//                its final sum (fixed order) gives out_p = C / Z, dt_p =
//                (-2/h^2)(g_p/Z_p)(A - out_p B)/c, and a_p = g_p / Z_p;
//   source pass  threads hold sources; per (target chunk, source) partial
//                sums E = sum a w and F = sum a w (v_q - out_p) c(s - t) (the
//                difference taken per pair, as the definition has it: with
//                values near out_p the sum of the two products would cancel
//                in float32); its final sum gives dv_q = E and
//                ds_q = -(2/h^2) F / c  (t - s = -(s - t)).
// Deterministic: every partial goes to its own slot and the final sums add
// them in chunk order.
#include "swa_internal.cuh"

namespace swa {
namespace {

constexpr int kThreads = 256;
constexpr int kPer = 4;                       // points per thread
constexpr int kPerBlock = kThreads * kPer;    // 1024 owned points per block
constexpr int kTargetBlocks = 148 * 8;
constexpr int kStage = 2048;                  // staged points at a time
constexpr int64_t kMaxChunks = 65535;
constexpr int kSlot = 8;                      // floats per (chunk, point) partial

__device__ __forceinline__ float ex2_neg(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(-x));
  return y;
}

struct Plan {
  int64_t tiles, nchunks, chunk;
};

// owned points [0, n_own) in tiles of kPerBlock; streamed points [0, n_str)
// in chunks sized so that the grid fills the GPU (and grid.y <= 65535)
Plan plan(int64_t n_own, int64_t n_str) {
  Plan pl;
  pl.tiles = (n_own + kPerBlock - 1) / kPerBlock;
  int64_t want = (kTargetBlocks + pl.tiles - 1) / pl.tiles;
  if (want < 1) want = 1;
  int64_t chunk = (n_str + want - 1) / want;
  if (chunk > kStage) chunk = kStage;
  const int64_t min_chunk = (n_str + kMaxChunks - 1) / kMaxChunks;
  if (chunk < min_chunk) chunk = min_chunk;
  if (chunk < 1) chunk = 1;
  pl.chunk = chunk;
  pl.nchunks = (n_str + chunk - 1) / chunk;
  return pl;
}

// Target pass: partials[chunk][target][kSlot] = (Z, C, A_0..A_{D-1}, B_0..B_{D-1}).
template <int DIMS>
__global__ void __launch_bounds__(kThreads)
nw_bwd_target_kernel(const float* __restrict__ targets, int64_t M,
                     const float* __restrict__ sources, const float* __restrict__ vals,
                     int64_t S, float c, int64_t chunk, float* __restrict__ partials) {
  extern __shared__ float4 src[];  // (-s c per coordinate, then v)
  const int tid = threadIdx.x;
  const int64_t c0 = (int64_t)blockIdx.y * chunk;
  const int64_t c1 = imin64(c0 + chunk, S);
  const int64_t p0 = (int64_t)blockIdx.x * kPerBlock + tid;
  float tc[kPer][DIMS], z[kPer], cv[kPer], a[kPer][DIMS], b[kPer][DIMS];
#pragma unroll
  for (int u = 0; u < kPer; ++u) {
    const int64_t p = p0 + (int64_t)u * kThreads;
#pragma unroll
    for (int d = 0; d < DIMS; ++d) {
      tc[u][d] = p < M ? targets[p * DIMS + d] * c : 0.f;
      a[u][d] = b[u][d] = 0.f;
    }
    z[u] = cv[u] = 0.f;
  }
  for (int64_t s0 = c0; s0 < c1; s0 += kStage) {
    const int ns = (int)imin64(kStage, c1 - s0);
    if (s0 != c0) __syncthreads();
    for (int e = tid; e < ns; e += kThreads) {
      float f[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int d = 0; d < DIMS; ++d) f[d] = -(sources[(s0 + e) * DIMS + d] * c);
      f[DIMS] = vals[s0 + e];
      src[e] = make_float4(f[0], f[1], f[2], f[3]);
    }
    __syncthreads();
#pragma unroll 2
    for (int e = 0; e < ns; ++e) {
      const float4 sv = src[e];
      const float sf[4] = {sv.x, sv.y, sv.z, sv.w};
      const float v = sf[DIMS];
#pragma unroll
      for (int u = 0; u < kPer; ++u) {
        float dd[DIMS], d2 = 0.f;
#pragma unroll
        for (int d = 0; d < DIMS; ++d) {
          dd[d] = tc[u][d] + sf[d];  // c (t - s)
          d2 = fmaf(dd[d], dd[d], d2);
        }
        const float w = ex2_neg(d2);
        const float wv = w * v;
        z[u] += w;
        cv[u] += wv;
#pragma unroll
        for (int d = 0; d < DIMS; ++d) {
          a[u][d] = fmaf(wv, dd[d], a[u][d]);
          b[u][d] = fmaf(w, dd[d], b[u][d]);
        }
      }
    }
  }
#pragma unroll
  for (int u = 0; u < kPer; ++u) {
    const int64_t p = p0 + (int64_t)u * kThreads;
    if (p >= M) continue;
    float* slot = partials + ((int64_t)blockIdx.y * M + p) * kSlot;
    float f[kSlot] = {z[u], cv[u], 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int d = 0; d < DIMS; ++d) {
      f[2 + d] = a[u][d];
      f[2 + DIMS + d] = b[u][d];
    }
    reinterpret_cast<float4*>(slot)[0] = make_float4(f[0], f[1], f[2], f[3]);
    reinterpret_cast<float4*>(slot)[1] = make_float4(f[4], f[5], f[6], f[7]);
  }
}

// Final sum of the target pass, one thread per target, chunks in order:
// out_p, dt_p, and (a_p = g_p / Z_p, out_p) for the source pass.
template <int DIMS>
__global__ void __launch_bounds__(256)
nw_bwd_target_final_kernel(const float* __restrict__ partials, int nchunks, int64_t M,
                           const float* __restrict__ gout, float dt_scale,
                           float* __restrict__ dtargets, float2* __restrict__ ao) {
  const int64_t p = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (p >= M) return;
  float f[kSlot] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  for (int ch = 0; ch < nchunks; ++ch) {
    const float4* slot = reinterpret_cast<const float4*>(partials + ((int64_t)ch * M + p) * kSlot);
    const float4 x = slot[0], y = slot[1];
    f[0] += x.x; f[1] += x.y; f[2] += x.z; f[3] += x.w;
    f[4] += y.x; f[5] += y.y; f[6] += y.z; f[7] += y.w;
  }
  const float zp = f[0], out = f[1] / zp, ap = gout[p] / zp;
#pragma unroll
  for (int d = 0; d < DIMS; ++d)
    dtargets[p * DIMS + d] = dt_scale * ap * (f[2 + d] - out * f[2 + DIMS + d]);
  ao[p] = make_float2(ap, out);
}

// Source pass: partials[chunk][source][kSlot] = (E, F_0..F_{D-1}).
template <int DIMS>
__global__ void __launch_bounds__(kThreads)
nw_bwd_source_kernel(const float* __restrict__ targets, int64_t M,
                     const float* __restrict__ sources, const float* __restrict__ vals,
                     int64_t S, float c, const float2* __restrict__ ao, int64_t chunk,
                     float* __restrict__ partials) {
  extern __shared__ float4 tgt[];  // (-t c per coordinate, then a_p); out_p after them
  float* tgt_o = reinterpret_cast<float*>(tgt + imin64(chunk, kStage));
  const int tid = threadIdx.x;
  const int64_t c0 = (int64_t)blockIdx.y * chunk;
  const int64_t c1 = imin64(c0 + chunk, M);
  const int64_t q0 = (int64_t)blockIdx.x * kPerBlock + tid;
  float sc[kPer][DIMS], vq[kPer], e_[kPer], fs[kPer][DIMS];
#pragma unroll
  for (int u = 0; u < kPer; ++u) {
    const int64_t q = q0 + (int64_t)u * kThreads;
#pragma unroll
    for (int d = 0; d < DIMS; ++d) {
      sc[u][d] = q < S ? sources[q * DIMS + d] * c : 0.f;
      fs[u][d] = 0.f;
    }
    vq[u] = q < S ? vals[q] : 0.f;
    e_[u] = 0.f;
  }
  for (int64_t t0 = c0; t0 < c1; t0 += kStage) {
    const int nt = (int)imin64(kStage, c1 - t0);
    if (t0 != c0) __syncthreads();
    for (int e = tid; e < nt; e += kThreads) {
      const float2 x = ao[t0 + e];
      float f[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int d = 0; d < DIMS; ++d) f[d] = -(targets[(t0 + e) * DIMS + d] * c);
      f[DIMS] = x.x;
      tgt[e] = make_float4(f[0], f[1], f[2], f[3]);
      tgt_o[e] = x.y;
    }
    __syncthreads();
#pragma unroll 2
    for (int e = 0; e < nt; ++e) {
      const float4 tv = tgt[e];
      const float tf[4] = {tv.x, tv.y, tv.z, tv.w};
      const float ap = tf[DIMS], op = tgt_o[e];
#pragma unroll
      for (int u = 0; u < kPer; ++u) {
        float dd[DIMS], d2 = 0.f;
#pragma unroll
        for (int d = 0; d < DIMS; ++d) {
          dd[d] = sc[u][d] + tf[d];  // c (s - t)
          d2 = fmaf(dd[d], dd[d], d2);
        }
        const float w = ex2_neg(d2);
        const float aw = ap * w;
        const float kk = aw * (vq[u] - op);
        e_[u] += aw;
#pragma unroll
        for (int d = 0; d < DIMS; ++d) fs[u][d] = fmaf(kk, dd[d], fs[u][d]);
      }
    }
  }
#pragma unroll
  for (int u = 0; u < kPer; ++u) {
    const int64_t q = q0 + (int64_t)u * kThreads;
    if (q >= S) continue;
    float* slot = partials + ((int64_t)blockIdx.y * S + q) * kSlot;
    float f[kSlot] = {e_[u], 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int d = 0; d < DIMS; ++d) f[1 + d] = fs[u][d];
    reinterpret_cast<float4*>(slot)[0] = make_float4(f[0], f[1], f[2], f[3]);
    reinterpret_cast<float4*>(slot)[1] = make_float4(f[4], f[5], f[6], f[7]);
  }
}

template <int DIMS>
__global__ void __launch_bounds__(256)
nw_bwd_source_final_kernel(const float* __restrict__ partials, int nchunks, int64_t S,
                           float ds_scale, float* __restrict__ dsources,
                           float* __restrict__ dvals) {
  const int64_t q = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (q >= S) return;
  float f[kSlot] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  for (int ch = 0; ch < nchunks; ++ch) {
    const float4* slot = reinterpret_cast<const float4*>(partials + ((int64_t)ch * S + q) * kSlot);
    const float4 x = slot[0], y = slot[1];
    f[0] += x.x; f[1] += x.y; f[2] += x.z; f[3] += x.w;
    f[4] += y.x; f[5] += y.y; f[6] += y.z; f[7] += y.w;
  }
#pragma unroll
  for (int d = 0; d < DIMS; ++d) dsources[q * DIMS + d] = ds_scale * f[1 + d];
  dvals[q] = f[0];
}

template <int DIMS>
cudaError_t nw_bwd(const float* targets, int64_t M, const float* sources, const float* vals,
                   int64_t S, float h, const float* gout, float* dtargets, float* dsources,
                   float* dvals, float* ws, cudaStream_t s, int* launches) {
  const float c = sqrtf(kLog2e) / h;
  // (t - s) = c (t - s) / c: the scales of dt and ds absorb 1/c
  const float grad_scale = 2.f / (h * h) / c;
  const Plan pt = plan(M, S), ps = plan(S, M);
  float2* ao = reinterpret_cast<float2*>(ws);
  float* partials = ws + 2 * ((M + 1) / 2 * 2);
  cudaError_t e;
  nw_bwd_target_kernel<DIMS><<<dim3((unsigned)pt.tiles, (unsigned)pt.nchunks), kThreads,
                               (size_t)imin64(pt.chunk, kStage) * sizeof(float4), s>>>(
      targets, M, sources, vals, S, c, pt.chunk, partials);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  nw_bwd_target_final_kernel<DIMS><<<(unsigned)((M + 255) / 256), 256, 0, s>>>(
      partials, (int)pt.nchunks, M, gout, -grad_scale, dtargets, ao);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  const size_t smem = (size_t)imin64(ps.chunk, kStage) * (sizeof(float4) + sizeof(float));
  nw_bwd_source_kernel<DIMS><<<dim3((unsigned)ps.tiles, (unsigned)ps.nchunks), kThreads,
                               smem, s>>>(targets, M, sources, vals, S, c, ao, ps.chunk,
                                          partials);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  nw_bwd_source_final_kernel<DIMS><<<(unsigned)((S + 255) / 256), 256, 0, s>>>(
      partials, (int)ps.nchunks, S, -grad_scale, dsources, dvals);
  *launches += 4;
  return cudaGetLastError();
}

}  // namespace

size_t nw_bwd_workspace_bytes(int64_t M, int64_t S) {
  const Plan pt = plan(M, S), ps = plan(S, M);
  const int64_t part = (pt.nchunks * M > ps.nchunks * S ? pt.nchunks * M : ps.nchunks * S);
  return (size_t)(2 * ((M + 1) / 2 * 2) + part * kSlot) * sizeof(float);
}

cudaError_t launch_nw_bwd(const float* targets, int64_t M, const float* sources,
                          const float* vals, int64_t S, int dims, float h, const float* gout,
                          float* dtargets, float* dsources, float* dvals, float* ws,
                          cudaStream_t s, int* launches) {
  if (dims == 1)
    return nw_bwd<1>(targets, M, sources, vals, S, h, gout, dtargets, dsources, dvals, ws, s,
                     launches);
  if (dims == 2)
    return nw_bwd<2>(targets, M, sources, vals, S, h, gout, dtargets, dsources, dvals, ws, s,
                     launches);
  return nw_bwd<3>(targets, M, sources, vals, S, h, gout, dtargets, dsources, dvals, ws, s,
                   launches);
}

}  // namespace swa
