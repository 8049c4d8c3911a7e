// nw_regrid.cu -- Nadaraya-Watson regrid on CUDA cores.
//
// "Show HN: Automatic deduction of FlashAttention kernel from ~25 lines of
// SQL", query NADARAYA_WATSON: w_pq = exp(-((tx-sx)^2 + (ty-sy)^2) / h^2)
// ("bandwidth h = 0.5", divisor 0.25), out_p = sum_q w_pq v_q / sum_q w_pq.
// Every weight is <= 1, so no running max is needed.
//
// Work split: the (targets x sources) pair grid is cut into target tiles of
// kTargetsPerBlock (kPerThread targets per thread, kept in registers) and
// source chunks sized so the grid fills every SM several times over.  A
// block stages its chunk as float4 (-x*c, -y*c, v, 0) in shared memory,
// where c = sqrt(log2 e)/h folds the bandwidth and the base change into the
// coordinates, so each pair costs 2 FADD, FMUL, FFMA, one MUFU ex2 (with the
// sign folded into its operand), FADD and FFMA -- the FP32 steps issued two
// targets at a time as packed f32x2 instructions (bitwise the same sums),
// which leaves MUFU as the one limit.  Partial (sum w, sum w v)
// per (chunk, target) go to a float2 workspace; a second kernel adds them in
// chunk order (deterministic) and divides.  0/0 gives NaN.
#include "swa_internal.cuh"

namespace swa {
namespace {

constexpr int kThreads = 256;
constexpr int kPerThread = 8;
constexpr int kTargetsPerBlock = kThreads * kPerThread;
constexpr int kTargetBlocks = 148 * 8;   // blocks the grid aims for (SMs x resident blocks)
constexpr int kMaxChunk = 2048;          // sources per block (32 KB of shared memory)

__device__ __forceinline__ float ex2_neg(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(-x));
  return y;
}

__global__ void __launch_bounds__(kThreads)
nw_partial_kernel(const float* __restrict__ targets, int64_t M,
                  const float* __restrict__ sources, const float* __restrict__ vals,
                  int64_t S, float c, int64_t chunk, float2* __restrict__ partials) {
  extern __shared__ float4 src[];
  const int tid = threadIdx.x;
  const int64_t s0 = (int64_t)blockIdx.y * chunk;
  const int ns = (int)imin64(chunk, S - s0);
  for (int e = tid; e < ns; e += kThreads) {
    const float2 xy = reinterpret_cast<const float2*>(sources)[s0 + e];
    src[e] = make_float4(-(xy.x * c), -(xy.y * c), vals[s0 + e], 0.f);
  }
  __syncthreads();

  // targets in pairs: lane .x of pair u is target 2u, lane .y target 2u + 1
  constexpr int kPairs = kPerThread / 2;
  float2 tx[kPairs], ty[kPairs], sw[kPairs], swv[kPairs];
  const int64_t p0 = (int64_t)blockIdx.x * kTargetsPerBlock + tid;
#pragma unroll
  for (int u = 0; u < kPairs; ++u) {
    float2 a = make_float2(0.f, 0.f), b = make_float2(0.f, 0.f);
    const int64_t pa = p0 + (int64_t)(2 * u) * kThreads, pb = pa + kThreads;
    if (pa < M) a = reinterpret_cast<const float2*>(targets)[pa];
    if (pb < M) b = reinterpret_cast<const float2*>(targets)[pb];
    tx[u] = make_float2(a.x * c, b.x * c);
    ty[u] = make_float2(a.y * c, b.y * c);
    sw[u] = make_float2(0.f, 0.f);
    swv[u] = make_float2(0.f, 0.f);
  }
#pragma unroll 4
  for (int e = 0; e < ns; ++e) {
    const float4 sv = src[e];
    const float2 nsx = make_float2(sv.x, sv.x), nsy = make_float2(sv.y, sv.y);
    const float2 v2 = make_float2(sv.z, sv.z);
#pragma unroll
    for (int u = 0; u < kPairs; ++u) {
      const float2 dx = __fadd2_rn(tx[u], nsx);
      const float2 dy = __fadd2_rn(ty[u], nsy);
      const float2 d2 = __ffma2_rn(dy, dy, __fmul2_rn(dx, dx));
      const float2 w = make_float2(ex2_neg(d2.x), ex2_neg(d2.y));
      sw[u] = __fadd2_rn(sw[u], w);
      swv[u] = __ffma2_rn(w, v2, swv[u]);
    }
  }
#pragma unroll
  for (int u = 0; u < kPairs; ++u) {
    const int64_t pa = p0 + (int64_t)(2 * u) * kThreads, pb = pa + kThreads;
    if (pa < M) partials[(int64_t)blockIdx.y * M + pa] = make_float2(sw[u].x, swv[u].x);
    if (pb < M) partials[(int64_t)blockIdx.y * M + pb] = make_float2(sw[u].y, swv[u].y);
  }
}

__global__ void __launch_bounds__(256)
nw_finalize_kernel(const float2* __restrict__ partials, int nchunks, int64_t M,
                   float* __restrict__ out) {
  const int64_t p = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (p >= M) return;
  float sw = 0.f, swv = 0.f;
  for (int ch = 0; ch < nchunks; ++ch) {
    const float2 a = partials[(int64_t)ch * M + p];
    sw += a.x;
    swv += a.y;
  }
  out[p] = swv / sw;
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
  if (chunk > kMaxChunk) chunk = kMaxChunk;
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
                              const float* vals, int64_t S, float h, float* partials,
                              cudaStream_t s, int* launches) {
  const Plan pl = plan(M, S);
  const float c = sqrtf(kLog2e) / h;
  dim3 grid((unsigned)pl.mtiles, (unsigned)pl.nchunks);
  const size_t smem = (size_t)pl.chunk * sizeof(float4);
  nw_partial_kernel<<<grid, kThreads, smem, s>>>(targets, M, sources, vals, S, c, pl.chunk,
                                                 reinterpret_cast<float2*>(partials));
  *launches += 1;
  return cudaGetLastError();
}

cudaError_t launch_nw_finalize(int64_t M, int64_t S, const float* partials, float* out,
                               cudaStream_t s, int* launches) {
  const Plan pl = plan(M, S);
  nw_finalize_kernel<<<(unsigned)((M + 255) / 256), 256, 0, s>>>(
      reinterpret_cast<const float2*>(partials), (int)pl.nchunks, M, out);
  *launches += 1;
  return cudaGetLastError();
}

}  // namespace swa
