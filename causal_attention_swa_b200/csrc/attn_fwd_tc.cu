// attn_fwd_tc.cu -- causal / non-causal attention forward on the sm_100a
// tensor cores (tcgen05.mma kind::f16, bf16 operands, f32 accumulators in
// TMEM, TMA-staged K/V).
//
// The method: "Show HN: Automatic deduction of FlashAttention kernel from
// ~25 lines of SQL" (page 2, the demo's docstring): FlashAttention streams
// blocks of keys past blocks of queries under a running softmax, so the
// N x N scores are never stored; the math is the view ATTENTION_WINDOW
// (scores = q.k/8 over the pairs with q.t >= k.t, w = exp(s - row max),
// out = sum w/z v).
//
// Block = two 128-row query tiles of one head (256 rows) and 384 threads:
//   warps 0-3  softmax for query tile 0 (thread r owns row r = TMEM lane r)
//   warps 4-7  softmax for query tile 1
//   warp  8    TMA producer: Q0, Q1 once, then K_j, V_j into 3 stages
//   warp  9    MMA issuer (one thread) and TMEM owner
//   warps 10-11 idle
// Registers: launched at 168 per thread (384 x 168); the softmax
// warpgroups take 224 (a full row of S stays in registers), the
// producer/MMA warpgroup gives up to 56: 256 x 224 + 128 x 56 = 384 x 168.
// TMEM (512 columns): S0 [0,128) S1 [128,256) O0 [256,320) O1 [320,384);
// P_t (bf16, two per column) overwrites the first 64 columns of S_t and is
// the A operand of O_t += P_t V_j straight from TMEM.
// Per key tile j the MMA warp issues, for t = 0, 1:  O_t += P_t,j V_j, then
// S_t,j+1 = Q_t K_j+1^T.  tcgen05 MMAs of one thread execute in issue
// order, so S_t,j+1 may overwrite P_t,j, and the commit that announces
// S_t,j+1 also covers O_t's update with P_t,j -- the softmax warps may then
// rescale O_t in TMEM before publishing P_t,j+1.  The two query tiles
// ping-pong: while one softmax warpgroup waits for its next S, the other
// computes.
// Online softmax in the log2 domain with a lazy rescale: the reference max
// of a row moves (and O, l are rescaled) only when the new row max exceeds
// it by more than 8, so P <= 2^8 (exact after the final division by l).
// Causal: key tiles past the diagonal are never loaded; inside the
// diagonal tile (and past N on a ragged tail) a masked score is replaced by
// -inf before the max, so its weight is exactly 0; V is all-finite in the
// heads this kernel takes (the caller's scan), so 0 * v = 0 and the product
// is the same as skipping the pair.
// Every mbarrier wait is bounded; on expiry the block records an error code
// in the device error word, all roles leave their loops, and TMEM is freed.
#include <cudaTypedefs.h>

#include "attn_tc.cuh"
#include "tc_ptx.cuh"

namespace swa {
namespace {

using namespace tc;

constexpr int BM = 128;                 // query rows per tile (MMA M)
constexpr int BN = 128;                 // keys per K/V tile
constexpr int HD = 64;                  // head dimension
constexpr int kStages = 3;              // K/V pipeline depth
constexpr int kTileBytes = BM * HD * 2; // 16 KB per bf16 tile
constexpr int kThreads = 384;
constexpr int kSoftmaxRegs = 224;
constexpr int kOtherRegs = 56;
static_assert(256 * kSoftmaxRegs + 128 * kOtherRegs <= kThreads * 168, "register split");
constexpr int kTmaWarp = 8;
constexpr int kMmaWarp = 9;
constexpr uint32_t kTmemCols = 512;
constexpr float kRescaleThreshold = 8.0f;

struct __align__(1024) Smem {
  uint8_t q[2][kTileBytes];
  uint8_t k[kStages][kTileBytes];
  uint8_t v[kStages][kTileBytes];
  uint64_t q_full;
  uint64_t k_full[kStages];
  uint64_t v_full[kStages];
  uint64_t kv_empty[kStages];
  uint64_t s_full[2];
  uint64_t p_full[2];
  uint64_t o_final[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
};

constexpr size_t kSmemBytes = sizeof(Smem) + 1024;

__device__ __forceinline__ uint32_t col_s(int t) { return t ? 128u : 0u; }
__device__ __forceinline__ uint32_t col_o(int t) { return t ? 320u : 256u; }

__device__ __forceinline__ bool wait_unbounded_by_abort(uint64_t* bar, uint32_t parity) {
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity)) {
    if (clock64() - t0 > kWaitCycles) return false;
  }
  return true;
}

__global__ void __launch_bounds__(kThreads, 1)
attn_fwd_tc_kernel(const __grid_constant__ CUtensorMap tm_q,
                   const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, __nv_bfloat16* __restrict__ out,
                   float* __restrict__ lse, int N, int BH, int n_ctiles, int causal,
                   float scale_log2, const int* __restrict__ flags, unsigned* __restrict__ err) {
  // Longest first: every head's latest (heaviest) query tiles, then the next.
  const int head = blockIdx.x % BH;
  const int c = n_ctiles - 1 - blockIdx.x / BH;
  if (flags[head] != 0) return;         // a non-finite head: the pair-by-pair kernel's

  extern __shared__ uint8_t smem_raw[];
  Smem& sm = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                      ~static_cast<uintptr_t>(1023));
  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;

  const int n_key_tiles = (N + BN - 1) / BN;
  int n_t[2];
#pragma unroll
  for (int t = 0; t < 2; ++t) {
    const int g = 2 * c + t;
    if (g * BM >= N) n_t[t] = 0;
    else n_t[t] = causal ? min(g + 1, n_key_tiles) : n_key_tiles;
  }
  const int n_kv = max(n_t[0], n_t[1]);

  if (tid == 0) {
    mbar_init(&sm.q_full, 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&sm.k_full[s], 1);
      mbar_init(&sm.v_full[s], 1);
      mbar_init(&sm.kv_empty[s], 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(&sm.s_full[t], 1);
      mbar_init(&sm.p_full[t], 128);
      mbar_init(&sm.o_final[t], 1);
    }
    mbar_init(&sm.drain, 1);
    sm.abort = 0;
    fence_mbar_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(&sm.tmem_base, kTmemCols);
    tmem_relinquish();
  }
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  const uint32_t tmem = sm.tmem_base;
  volatile int* abort = &sm.abort;

  if (warp >= 8) regs_decrease<kOtherRegs>();

  if (warp == kTmaWarp) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      prefetch_tmap(&tm_q);
      prefetch_tmap(&tm_k);
      prefetch_tmap(&tm_v);
      mbar_arrive_expect_tx(&sm.q_full, 2 * kTileBytes);
      tma_load_3d(sm.q[0], &tm_q, &sm.q_full, 0, (2 * c) * BM, head);
      tma_load_3d(sm.q[1], &tm_q, &sm.q_full, 0, (2 * c + 1) * BM, head);
      for (int j = 0; j < n_kv; ++j) {
        const int s = j % kStages;
        const int round = j / kStages;
        if (round > 0 && !mbar_wait(&sm.kv_empty[s], (round - 1) & 1, abort, err,
                                    kDevTimeoutEmpty))
          break;
        mbar_arrive_expect_tx(&sm.k_full[s], kTileBytes);
        tma_load_3d(sm.k[s], &tm_k, &sm.k_full[s], 0, j * BN, head);
        mbar_arrive_expect_tx(&sm.v_full[s], kTileBytes);
        tma_load_3d(sm.v[s], &tm_v, &sm.v_full[s], 0, j * BN, head);
      }
    }
    __syncwarp();
  } else if (warp == kMmaWarp) {
    // --------------------------------------------------------- MMA issuer
    {  // the whole warp runs the issue loop; one elected lane issues
      constexpr uint32_t idesc_s = idesc_bf16_f32(BM, BN, 0, 0);  // Q, K both K-major
      constexpr uint32_t idesc_o = idesc_bf16_f32(BM, HD, 0, 1);  // V is MN-major (dims contiguous)
      int k_ready = -1;
      bool ok = mbar_wait(&sm.q_full, 0, abort, err, kDevTimeoutFull);
      auto wait_k = [&](int j) -> bool {
        if (j <= k_ready) return true;
        if (!mbar_wait(&sm.k_full[j % kStages], (j / kStages) & 1, abort, err, kDevTimeoutFull))
          return false;
        k_ready = j;
        return true;
      };
      auto issue_s = [&](int t, int j) {
        const uint32_t a0 = smem_u32(sm.q[t]);
        const uint32_t b0 = smem_u32(sm.k[j % kStages]);
#pragma unroll
        for (int kk = 0; kk < HD / 16; ++kk)
          mma_ss_elect(tmem + col_s(t), desc_sw128(a0 + kk * 32, 16, 1024),
                 desc_sw128(b0 + kk * 32, 16, 1024), idesc_s, kk > 0 ? 1u : 0u);
        mma_commit_elect(&sm.s_full[t]);
      };
      auto issue_pv = [&](int t, int j) {
        const uint32_t b0 = smem_u32(sm.v[j % kStages]);
#pragma unroll
        for (int kk = 0; kk < BN / 16; ++kk)
          mma_ts_elect(tmem + col_o(t), tmem + col_s(t) + kk * 8,
                 desc_sw128(b0 + kk * 2048, 8192, 1024), idesc_o,
                 (j > 0 || kk > 0) ? 1u : 0u);
      };
      if (ok) ok = wait_k(0);
      if (ok) {
        fence_after_sync();
        for (int t = 0; t < 2; ++t)
          if (n_t[t] > 0) issue_s(t, 0);
      }
      for (int j = 0; ok && j < n_kv; ++j) {
        const int s = j % kStages;
        if (!mbar_wait(&sm.v_full[s], (j / kStages) & 1, abort, err, kDevTimeoutFull)) break;
        for (int t = 0; t < 2 && ok; ++t) {
          if (j >= n_t[t]) continue;
          if (!mbar_wait(&sm.p_full[t], j & 1, abort, err, kDevTimeoutOther)) { ok = false; break; }
          fence_after_sync();
          issue_pv(t, j);
          if (j + 1 < n_t[t]) {
            if (!wait_k(j + 1)) { ok = false; break; }
            issue_s(t, j + 1);
          } else {
            mma_commit_elect(&sm.o_final[t]);
          }
        }
        mma_commit_elect(&sm.kv_empty[s]);
      }
      // every MMA this thread issued has finished before TMEM is released
      mma_commit_elect(&sm.drain);
      wait_unbounded_by_abort(&sm.drain, 0);
    }
    __syncwarp();
  } else if (warp < 8) {
    // ------------------------------------------------------------ softmax
    regs_increase<kSoftmaxRegs>();
    const int t = warp >> 2;
    const int wt = warp & 3;
    const int r = wt * 32 + lane;
    const int g = 2 * c + t;
    const int row = g * BM + r;
    const uint32_t lane_off = static_cast<uint32_t>(wt * 32) << 16;
    const uint32_t tS = tmem + lane_off + col_s(t);
    const uint32_t tO = tmem + lane_off + col_o(t);
    float m_used = -INFINITY;  // reference max (log2 domain)
    float l = 0.f;
    bool ok = true;
    for (int j = 0; j < n_t[t]; ++j) {
      if (!mbar_wait(&sm.s_full[t], j & 1, abort, err, kDevTimeoutMma)) { ok = false; break; }
      fence_after_sync();
      float x[BN];
      {
        uint32_t u[BN / 16][16];
#pragma unroll
        for (int i = 0; i < BN / 16; ++i) tmem_ld16(tS + i * 16, u[i]);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < BN / 16; ++i)
#pragma unroll
          for (int e = 0; e < 16; ++e) x[i * 16 + e] = __uint_as_float(u[i][e]) * scale_log2;
      }
      const bool need_mask = (j * BN + BN > N) || (causal && j == g);
      if (need_mask) {
#pragma unroll
        for (int e = 0; e < BN; ++e) {
          const int key = j * BN + e;
          if (key >= N || (causal && key > row)) x[e] = -INFINITY;
        }
      }
      float mxp[8];
#pragma unroll
      for (int a = 0; a < 8; ++a) mxp[a] = x[a];
#pragma unroll
      for (int e = 8; e < BN; ++e) mxp[e & 7] = fmaxf(mxp[e & 7], x[e]);
      const float mx = fmaxf(fmaxf(fmaxf(mxp[0], mxp[1]), fmaxf(mxp[2], mxp[3])),
                             fmaxf(fmaxf(mxp[4], mxp[5]), fmaxf(mxp[6], mxp[7])));
      const float m_new = fmaxf(m_used, mx);
      const bool need = (j == 0) || (m_new > m_used + kRescaleThreshold);
      if (j > 0 && __any_sync(0xffffffffu, need)) {
        const float alpha = need ? ex2(m_used - m_new) : 1.f;
#pragma unroll
        for (int i = 0; i < HD / 16; ++i) {
          uint32_t u[16];
          tmem_ld16(tO + i * 16, u);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 16; ++e) u[e] = __float_as_uint(__uint_as_float(u[e]) * alpha);
          tmem_st16(tO + i * 16, u);
        }
        l *= alpha;
      }
      if (need) m_used = m_new;
      float rsp[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int i = 0; i < BN / 32; ++i) {
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const float p0 = ex2(x[i * 32 + 2 * e] - m_used);
          const float p1 = ex2(x[i * 32 + 2 * e + 1] - m_used);
          rsp[e & 3] += p0 + p1;
          pk[e] = pack_bf16(p0, p1);
        }
        tmem_st16(tS + i * 16, pk);
      }
      tmem_wait_st();
      fence_before_sync();
      mbar_arrive(&sm.p_full[t]);
      l += (rsp[0] + rsp[1]) + (rsp[2] + rsp[3]);
    }
    if (ok && n_t[t] > 0 && mbar_wait(&sm.o_final[t], 0, abort, err, kDevTimeoutMma)) {
      fence_after_sync();
      const float inv = 1.f / l;
      uint32_t packed[HD / 2];
#pragma unroll
      for (int i = 0; i < HD / 16; ++i) {
        uint32_t u[16];
        tmem_ld16(tO + i * 16, u);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 8; ++e)
          packed[i * 8 + e] = pack_bf16(__uint_as_float(u[2 * e]) * inv,
                                        __uint_as_float(u[2 * e + 1]) * inv);
      }
      if (row < N) {
        uint4* dst = reinterpret_cast<uint4*>(out + ((size_t)head * N + row) * HD);
#pragma unroll
        for (int i = 0; i < HD / 8; ++i)
          dst[i] = make_uint4(packed[4 * i], packed[4 * i + 1], packed[4 * i + 2],
                              packed[4 * i + 3]);
        lse[(size_t)head * N + row] = (m_used + __log2f(l)) * kLn2;
      }
    }
  }

  fence_before_sync();
  __syncthreads();
  if (warp == kMmaWarp) {
    fence_after_sync();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// --------------------------------------------------------------------- host

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

}  // namespace

// [BH][N][64] bf16 viewed as a 3-D tensor (64, N, BH); 64 x rows x 1 boxes,
// 128-byte swizzle; rows past N read as zeros.
cudaError_t make_tmap_bf16_rows(CUtensorMap* map, const void* base, int64_t BH, int64_t N,
                                int box_rows) {
  auto fn = encode_fn();
  if (!fn) return cudaErrorNotSupported;
  cuuint64_t dims[3] = {64, (cuuint64_t)N, (cuuint64_t)BH};
  cuuint64_t strides[2] = {64 * 2, (cuuint64_t)N * 64 * 2};
  cuuint32_t box[3] = {64, (cuuint32_t)box_rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims,
                  strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

cudaError_t launch_attn_fwd_tc(const void* q, const void* k, const void* v, void* out,
                               float* lse, int64_t B, int64_t H, int64_t N, int causal,
                               float scale, const int* flags, unsigned* err, cudaStream_t s,
                               int* launches) {
  const int64_t BH = B * H;
  CUtensorMap tq, tk, tv;
  cudaError_t e;
  if ((e = make_tmap_bf16_rows(&tq, q, BH, N, BM)) != cudaSuccess) return e;
  if ((e = make_tmap_bf16_rows(&tk, k, BH, N, BN)) != cudaSuccess) return e;
  if ((e = make_tmap_bf16_rows(&tv, v, BH, N, BN)) != cudaSuccess) return e;
  e = cudaFuncSetAttribute(attn_fwd_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)kSmemBytes);
  if (e != cudaSuccess) return e;
  const int n_ctiles = (int)((N + 2 * BM - 1) / (2 * BM));
  const int64_t grid = (int64_t)n_ctiles * BH;
  attn_fwd_tc_kernel<<<(unsigned)grid, kThreads, kSmemBytes, s>>>(
      tq, tk, tv, static_cast<__nv_bfloat16*>(out), lse, (int)N, (int)BH, n_ctiles, causal,
      scale * kLog2e, flags, err);
  *launches += 1;
  return cudaGetLastError();
}

}  // namespace swa
