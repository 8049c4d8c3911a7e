// nw_regrid.cu -- Nadaraya-Watson regrid on CUDA cores.
//
// "Show HN: Automatic deduction of FlashAttention kernel from ~25 lines of
// SQL", query NADARAYA_WATSON: w_pq = exp(-((tx-sx)^2 + (ty-sy)^2) / h^2)
// ("bandwidth h = 0.5", divisor 0.25), out_p = sum_q w_pq v_q / sum_q w_pq.
// Every weight is <= 1, so no running max is needed.  The kernels take
// points of DIMS = 1, 2 or 3 coordinates (the squared distance summed over
// them); the pages' points, and the benchmark's, have two.
//
// Work split: the (targets x sources) pair grid is cut into target tiles of
// kTargetsPerBlock (kPerThread targets per thread, kept in registers) and
// source chunks sized so the grid fills every SM several times over.  A
// block stages its chunk as float4 (-x*c, -y*c, v, 0) in shared memory,
// where c = sqrt(log2 e)/h folds the bandwidth and the base change into the
// coordinates, so each pair costs 2 FADD, FMUL, FFMA, one MUFU ex2 (with the
// sign folded into its operand), FADD and FFMA -- the FP32 steps issued two
// targets at a time as packed f32x2 instructions (bitwise the same sums),
// which leaves MUFU as the one limit.  A chunk longer than the shared-memory
// stage (2048 sources) is staged in turns, so any S fits the grid.  Partial
// (sum w, sum w v) per (chunk, target) go to a float2 workspace; a second
// kernel adds them in a fixed order (deterministic) and divides: eight
// threads per target each add every eighth chunk, then the eight sums are
// added in order.  0/0 gives NaN.
#include "swa_internal.cuh"

namespace swa {
namespace {

constexpr int kThreads = 256;
constexpr int kPerThread = 8;
constexpr int kTargetsPerBlock = kThreads * kPerThread;
constexpr int kTargetBlocks = 148 * 8;   // blocks the grid aims for (SMs x resident blocks)
constexpr int kStage = 2048;             // sources staged at a time (32 KB of shared memory)
constexpr int64_t kMaxChunks = 65535;    // grid.y limit

__device__ __forceinline__ float ex2_neg(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(-x));
  return y;
}

template <int DIMS>
__global__ void __launch_bounds__(kThreads)
nw_partial_kernel(const float* __restrict__ targets, int64_t M,
                  const float* __restrict__ sources, const float* __restrict__ vals,
                  int64_t S, float c, int64_t chunk, float2* __restrict__ partials) {
  static_assert(DIMS >= 1 && DIMS <= 3, "1 to 3 coordinates");
  extern __shared__ float4 src[];
  const int tid = threadIdx.x;
  const int64_t c0 = (int64_t)blockIdx.y * chunk;
  const int64_t c1 = imin64(c0 + chunk, S);

  // targets in pairs: lane .x of pair u is target 2u, lane .y target 2u + 1
  constexpr int kPairs = kPerThread / 2;
  float2 tc[DIMS][kPairs], sw[kPairs], swv[kPairs];
  const int64_t p0 = (int64_t)blockIdx.x * kTargetsPerBlock + tid;
#pragma unroll
  for (int u = 0; u < kPairs; ++u) {
    const int64_t pa = p0 + (int64_t)(2 * u) * kThreads, pb = pa + kThreads;
#pragma unroll
    for (int d = 0; d < DIMS; ++d)
      tc[d][u] = make_float2(pa < M ? targets[pa * DIMS + d] * c : 0.f,
                             pb < M ? targets[pb * DIMS + d] * c : 0.f);
    sw[u] = make_float2(0.f, 0.f);
    swv[u] = make_float2(0.f, 0.f);
  }
  for (int64_t s0 = c0; s0 < c1; s0 += kStage) {
    const int ns = (int)imin64(kStage, c1 - s0);
    if (s0 != c0) __syncthreads();  // the previous stage is no longer read
    for (int e = tid; e < ns; e += kThreads) {
      // (-s c per coordinate, then v): the value sits right after the coordinates
      float f[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int d = 0; d < DIMS; ++d) f[d] = -(sources[(s0 + e) * DIMS + d] * c);
      f[DIMS] = vals[s0 + e];
      src[e] = make_float4(f[0], f[1], f[2], f[3]);
    }
    __syncthreads();
#pragma unroll 4
    for (int e = 0; e < ns; ++e) {
      const float4 sv = src[e];
      const float sf[4] = {sv.x, sv.y, sv.z, sv.w};
      const float2 v2 = make_float2(sf[DIMS], sf[DIMS]);
#pragma unroll
      for (int u = 0; u < kPairs; ++u) {
        // squared scaled distance: (t0 - s0)^2 first, then + (t_d - s_d)^2
        float2 d2;
#pragma unroll
        for (int d = 0; d < DIMS; ++d) {
          const float2 dd = __fadd2_rn(tc[d][u], make_float2(sf[d], sf[d]));
          d2 = d == 0 ? __fmul2_rn(dd, dd) : __ffma2_rn(dd, dd, d2);
        }
        const float2 w = make_float2(ex2_neg(d2.x), ex2_neg(d2.y));
        sw[u] = __fadd2_rn(sw[u], w);
        swv[u] = __ffma2_rn(w, v2, swv[u]);
      }
    }
  }
#pragma unroll
  for (int u = 0; u < kPairs; ++u) {
    const int64_t pa = p0 + (int64_t)(2 * u) * kThreads, pb = pa + kThreads;
    if (pa < M) partials[(int64_t)blockIdx.y * M + pa] = make_float2(sw[u].x, swv[u].x);
    if (pb < M) partials[(int64_t)blockIdx.y * M + pb] = make_float2(sw[u].y, swv[u].y);
  }
}

// Block = 32 lanes x 8 chunk groups; lane t holds kFinVec consecutive
// targets (2: one 16-byte load of two (sum w, sum w v) pairs, when M is
// even; else 1).  Thread (g, t) adds chunks g, g + 8, ... (each chunk's 32
// lanes read 256 or 512 contiguous bytes), then thread (0, t) adds the eight
// group sums in order: the result does not depend on timing.
constexpr int kFinLanes = 32;
constexpr int kFinGroups = 8;
template <int kFinVec>
__global__ void __launch_bounds__(kFinLanes * kFinGroups)
nw_finalize_kernel(const float2* __restrict__ partials, int nchunks, int64_t M,
                   float* __restrict__ out) {
  __shared__ float4 part[kFinGroups][kFinLanes];
  const int t = threadIdx.x % kFinLanes, g = threadIdx.x / kFinLanes;
  const int64_t p = ((int64_t)blockIdx.x * kFinLanes + t) * kFinVec;  // first target
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);  // (sw, swv) of targets p, p + 1
  if (p < M) {
#pragma unroll 8
    for (int ch = g; ch < nchunks; ch += kFinGroups) {
      if constexpr (kFinVec == 2) {
        const float4 a = *reinterpret_cast<const float4*>(partials + (int64_t)ch * M + p);
        acc.x += a.x;
        acc.y += a.y;
        acc.z += a.z;
        acc.w += a.w;
      } else {
        const float2 a = partials[(int64_t)ch * M + p];
        acc.x += a.x;
        acc.y += a.y;
      }
    }
  }
  part[g][t] = acc;
  __syncthreads();
  if (g == 0 && p < M) {
    float4 sum = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int i = 0; i < kFinGroups; ++i) {
      sum.x += part[i][t].x;
      sum.y += part[i][t].y;
      sum.z += part[i][t].z;
      sum.w += part[i][t].w;
    }
    out[p] = sum.y / sum.x;
    if (kFinVec == 2) out[p + 1] = sum.w / sum.z;  // M even: p + 1 < M
  }
}

struct Plan {
  int64_t mtiles, nchunks, chunk;
};

Plan plan(int64_t M, int64_t S) {
  Plan pl;
  pl.mtiles = (M + kTargetsPerBlock - 1) / kTargetsPerBlock;
  int64_t want = (kTargetBlocks + pl.mtiles - 1) / pl.mtiles;
  if (want < 1) want = 1;
  int64_t chunk = (S + want - 1) / want;
  if (chunk > kStage) chunk = kStage;         // one stage per block when S allows
  const int64_t min_chunk = (S + kMaxChunks - 1) / kMaxChunks;
  if (chunk < min_chunk) chunk = min_chunk;   // else several stages: grid.y <= 65535
  if (chunk < 1) chunk = 1;
  pl.chunk = chunk;
  pl.nchunks = (S + chunk - 1) / chunk;
  return pl;
}

}  // namespace

size_t nw_partials_bytes(int64_t M, int64_t S) {
  const Plan pl = plan(M, S);
  return (size_t)(pl.nchunks * M) * sizeof(float2);
}

cudaError_t launch_nw_partial(const float* targets, int64_t M, const float* sources,
                              const float* vals, int64_t S, int dims, float h, float* partials,
                              cudaStream_t s, int* launches) {
  const Plan pl = plan(M, S);
  const float c = sqrtf(kLog2e) / h;
  dim3 grid((unsigned)pl.mtiles, (unsigned)pl.nchunks);
  const size_t smem = (size_t)imin64(pl.chunk, kStage) * sizeof(float4);
  float2* part = reinterpret_cast<float2*>(partials);
  if (dims == 1)
    nw_partial_kernel<1><<<grid, kThreads, smem, s>>>(targets, M, sources, vals, S, c, pl.chunk,
                                                      part);
  else if (dims == 2)
    nw_partial_kernel<2><<<grid, kThreads, smem, s>>>(targets, M, sources, vals, S, c, pl.chunk,
                                                      part);
  else
    nw_partial_kernel<3><<<grid, kThreads, smem, s>>>(targets, M, sources, vals, S, c, pl.chunk,
                                                      part);
  *launches += 1;
  return cudaGetLastError();
}

cudaError_t launch_nw_finalize(int64_t M, int64_t S, const float* partials, float* out,
                               cudaStream_t s, int* launches) {
  const Plan pl = plan(M, S);
  const auto* part = reinterpret_cast<const float2*>(partials);
  constexpr unsigned kBlock = kFinLanes * kFinGroups;
  if (M % 2 == 0)  // every chunk row starts on a 16-byte boundary
    nw_finalize_kernel<2><<<(unsigned)((M / 2 + kFinLanes - 1) / kFinLanes), kBlock, 0, s>>>(
        part, (int)pl.nchunks, M, out);
  else
    nw_finalize_kernel<1><<<(unsigned)((M + kFinLanes - 1) / kFinLanes), kBlock, 0, s>>>(
        part, (int)pl.nchunks, M, out);
  *launches += 1;
  return cudaGetLastError();
}

}  // namespace swa
