// attn_bwd_tc.cu -- attention backward on the sm_100a tensor cores
// (tcgen05.mma kind::f16: bf16 operands, f32 accumulators in TMEM).
//
// The method: the GRADIENT query of "Show HN: Automatic deduction of
// FlashAttention kernel from ~25 lines of SQL" (page 2) -- one backward pass
// for dq, dk and dv of a loss that reads the attention view -- in the
// FlashAttention form that recomputes P from the saved row logsumexp:
//   P_ij = exp(s_ij - lse_i)            dP_ij = dout_i . v_j
//   dS_ij = P_ij (dP_ij - delta_i)      delta_i = dout_i . out_i (prep kernel)
//   dv_j += P_ij dout_i   dk_j += scale dS_ij q_i   dq_i += scale dS_ij k_j
// over the pairs that exist (j <= i when causal).
//
// Block = one 128-key block j of one head (K_j, V_j stay in shared memory)
// and 576 threads; it walks the 128-query blocks i that see j:
//   warps 0-15  compute, four warpgroups: thread t of warpgroup w owns key
//               j0 + t (TMEM lane t) and queries 32w..32w+31 of each block.
//               From S^T and dP^T (one batched TMEM load per block) it forms
//               P^T (bf16, written back over its own dP^T columns for the
//               dV MMA) and dS (float32 -> bf16 hi + lo, into shared
//               memory); then it drains columns 16w..16w+15 of the previous
//               block's dQ (TMEM lane = query) into the float32 dQ
//               accumulator with vector red.add; at the end warpgroup w
//               stores columns 16w..16w+15 of its key's dv and dk
//   warp  16    TMA producer: K_j, V_j once; Q_i, dO_i, lse_i, delta_i into a
//               2-stage ring
//   warp  17    MMA issuer (one thread), TMEM owner
// Per query block, seven MMAs (M = 128, K = 64 or 128):
//   S^T = K_j Q_i^T              (A = K smem K-major, B = Q smem K-major)
//   dP^T = V_j dO_i^T            (A = V, B = dO, both K-major)
//   dV += P^T dO_i               (A = P^T from TMEM, B = dO MN-major)
//   dK += dS_hi^T Q_i + dS_lo^T Q_i   (A = dS tiles read K-major, B = Q MN-major)
//   dQ_i = dS_hi K_j + dS_lo K_j      (A = the same tiles read MN-major, B = K)
// dS is carried as hi + lo bf16 pairs (hi = bf16(dS), lo = bf16(dS - hi)),
// so dk and dq see dS to ~16 bits: a single bf16 rounding of dS, amplified
// by the cancellation in sum_j dS_ij k_j (sum_j dS_ij = 0), costs dq about
// 2% of its row RMS at N = 2048.  One [128 keys][128 queries] tile layout
// (rows = keys, 128-byte swizzle, two 64-query halves) is both the K-major
// A operand of dK and the MN-major A operand of dQ; it is double-buffered
// by query block, so block i's dS is written while block i-1's dK and dQ
// MMAs still read the other buffer.
// TMEM (512 columns): S^T buffers [0,128) and [128,256) (the block's dQ in
// the first 64 columns once S^T is consumed), dP^T [256,384) (warpgroup w
// writes the P^T of its 32 queries over its own columns 32w..32w+15 after
// loading them; the dV MMA takes each 16-query group's A from there),
// dV [384,448), dK [448,512).  MMAs of one thread execute in issue order,
// so a later MMA may overwrite TMEM an earlier one reads.
// Causal: only query blocks i >= j are visited; in the diagonal block (and
// past N on a ragged tail) P and dS of a masked pair are set to 0 by select.
// This kernel takes only heads whose V and dout are all finite, so 0 times
// a finite value is the same as skipping the pair.
// Every mbarrier wait is bounded (device error word on expiry).
#include "attn_tc.cuh"
#include "tc_ptx.cuh"

namespace swa {
namespace {

using namespace tc;

constexpr int BK = 128;                 // keys per block
constexpr int BQ = 128;                 // queries per block
constexpr int HD = 64;
constexpr int kTileBytes = 128 * HD * 2;
constexpr int kComputeThreads = 512;    // four warpgroups
constexpr int kTmaWarp = 16;
constexpr int kMmaWarp = 17;
constexpr int kThreads = 576;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColDP = 256, kColDV = 384, kColDK = 448;
constexpr int kHeadGroup = 4;      // heads scheduled together (their dQ, Q, dO share L2)

__device__ __forceinline__ uint32_t col_s(int b) { return b ? 128u : 0u; }

// Shared memory (227 KB of the 227 KB a block may use): the dynamic base is
// expected 1024-byte aligned (the kernel checks and reports otherwise).
struct __align__(1024) Smem {
  uint8_t k[kTileBytes];
  uint8_t v[kTileBytes];
  uint8_t q[2][kTileBytes];
  uint8_t dout[2][kTileBytes];
  uint8_t ds_hi[2][2][kTileBytes];  // [buffer][query half]: [128 keys][64 queries]
  uint8_t ds_lo[2][2][kTileBytes];
  float lse[2][BQ];                 // lse_i * log2(e) of each staged query block (+inf past N)
  float delta[2][BQ];               // delta_i of each staged query block (0 past N)
  uint64_t kv_full;
  uint64_t qd_full[2];
  uint64_t qd_empty[2];
  uint64_t s_full[2];
  uint64_t dp_full;
  uint64_t sm_done;
  uint64_t dq_full;
  uint64_t dq_empty;
  uint64_t acc_full;
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
};

constexpr size_t kSmemBytes = sizeof(Smem);
static_assert(kSmemBytes <= 232448, "shared memory");

__device__ __forceinline__ bool wait_drain(uint64_t* bar, uint32_t parity) {
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity)) {
    if (clock64() - t0 > kWaitCycles) return false;
  }
  return true;
}

__global__ void __launch_bounds__(kThreads, 1)
attn_bwd_tc_kernel(const __grid_constant__ CUtensorMap tm_q,
                   const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v,
                   const __grid_constant__ CUtensorMap tm_do, const float* __restrict__ lse2,
                   const float* __restrict__ delta, __nv_bfloat16* __restrict__ dk,
                   __nv_bfloat16* __restrict__ dv, float* __restrict__ dqacc, int N, int BH,
                   int causal, float scale, float scale_log2, const int* __restrict__ flags,
                   unsigned* __restrict__ err) {
  // Block order: groups of kHeadGroup heads; inside a group the longest key
  // blocks (j = 0 sees every query block) first, heads interleaved.
  const int n_blocks = (N + BQ - 1) / BQ;
  const int Npad = n_blocks * BQ;
  const int group = blockIdx.x / (kHeadGroup * n_blocks);
  const int g_heads = min(kHeadGroup, BH - group * kHeadGroup);
  const int r = blockIdx.x - group * kHeadGroup * n_blocks;
  const int jb = r / g_heads;
  const int head = group * kHeadGroup + r % g_heads;
  if (flags[head] != 0) return;

  extern __shared__ __align__(1024) uint8_t smem_raw[];
  if (smem_u32(smem_raw) & 1023u) {  // the swizzled tiles need 1024-byte alignment
    if (threadIdx.x == 0) atomicCAS(err, 0u, (unsigned)kDevSmemAlign);
    return;
  }
  Smem& sm = *reinterpret_cast<Smem*>(smem_raw);
  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int ib0 = causal ? jb : 0;
  const int n_q = n_blocks - ib0;
  const int j0 = jb * BK;

  if (tid == 0) {
    mbar_init(&sm.kv_full, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&sm.qd_full[s], 1);
      mbar_init(&sm.qd_empty[s], 1);
      mbar_init(&sm.s_full[s], 1);
    }
    mbar_init(&sm.dp_full, 1);
    mbar_init(&sm.sm_done, kComputeThreads);
    mbar_init(&sm.dq_full, 1);
    mbar_init(&sm.dq_empty, kComputeThreads);
    mbar_init(&sm.acc_full, 1);
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

  if (warp == kTmaWarp) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      prefetch_tmap(&tm_q);
      prefetch_tmap(&tm_k);
      prefetch_tmap(&tm_v);
      prefetch_tmap(&tm_do);
      mbar_arrive_expect_tx(&sm.kv_full, 2 * kTileBytes);
      tma_load_3d(sm.k, &tm_k, &sm.kv_full, 0, j0, head);
      tma_load_3d(sm.v, &tm_v, &sm.kv_full, 0, j0, head);
      for (int it = 0; it < n_q; ++it) {
        const int s = it & 1;
        const int round = it >> 1;
        if (round > 0 &&
            !mbar_wait(&sm.qd_empty[s], (round - 1) & 1, abort, err, kDevTimeoutEmpty))
          break;
        const int i0 = (ib0 + it) * BQ;
        mbar_arrive_expect_tx(&sm.qd_full[s], 2 * kTileBytes + 2 * BQ * 4);
        tma_load_3d(sm.q[s], &tm_q, &sm.qd_full[s], 0, i0, head);
        tma_load_3d(sm.dout[s], &tm_do, &sm.qd_full[s], 0, i0, head);
        bulk_load(sm.lse[s], lse2 + (size_t)head * Npad + i0, BQ * 4, &sm.qd_full[s]);
        bulk_load(sm.delta[s], delta + (size_t)head * Npad + i0, BQ * 4, &sm.qd_full[s]);
      }
    }
    __syncwarp();
  } else if (warp == kMmaWarp) {
    // --------------------------------------------------------- MMA issuer
    {  // the whole warp runs the issue loop; one elected lane issues
      constexpr uint32_t id_kk = idesc_bf16_f32(128, 128, 0, 0);  // S^T, dP^T: both K-major
      constexpr uint32_t id_mn = idesc_bf16_f32(128, 64, 0, 1);   // dV, dK: B MN-major
      constexpr uint32_t id_dq = idesc_bf16_f32(128, 64, 1, 1);   // dQ: A and B MN-major
      const uint32_t k_s = smem_u32(sm.k), v_s = smem_u32(sm.v);
      // Runs of MMAs from one asm block; descriptor steps in 16-byte units:
      // K-major operands +32 B (2) per K = 16 step, MN-major +2048 B (128).
      auto issue_kk = [&](uint32_t d_col, uint32_t a0, uint32_t b0) {
        mma_ss_run<4, 2, 0, 2>(tmem + d_col, desc_sw128(a0, 16, 1024), desc_sw128(b0, 16, 1024),
                               id_kk, 0u);
      };
      // dK += dS^T Q_i from one dS tile pair: A rows = keys, K = queries
      // (K-major; queries 64-127 in the second half tile)
      // (step 4 jumps to the second half tile: +16 KB = 1024 units in all)
      auto issue_dk = [&](const uint8_t (*ds)[kTileBytes], uint32_t q0, bool first) {
        mma_ss_run<8, 2, kTileBytes / 16 - 8, 128>(
            tmem + kColDK, desc_sw128(smem_u32(ds[0]), 16, 1024), desc_sw128(q0, 8192, 1024),
            id_mn, first ? 0u : 1u);
      };
      // dQ_i (+)= dS K_j from one dS tile pair: A M = queries (MN-major, the
      // two 64-query halves 16 KB apart), K = keys
      auto issue_dq = [&](const uint8_t (*ds)[kTileBytes], uint32_t col, bool first) {
        mma_ss_run<8, 128, 0, 128>(tmem + col, desc_sw128(smem_u32(ds[0]), kTileBytes, 1024),
                                   desc_sw128(k_s, 8192, 1024), id_dq, first ? 0u : 1u);
      };
      bool ok = mbar_wait(&sm.kv_full, 0, abort, err, kDevTimeoutFull) &&
                mbar_wait(&sm.qd_full[0], 0, abort, err, kDevTimeoutFull);
      if (ok) {
        issue_kk(col_s(0), k_s, smem_u32(sm.q[0]));
        mma_commit_elect(&sm.s_full[0]);
        issue_kk(kColDP, v_s, smem_u32(sm.dout[0]));
        mma_commit_elect(&sm.dp_full);
      }
      for (int it = 0; ok && it < n_q; ++it) {
        const int b = it & 1;
        const bool next = it + 1 < n_q;
        // the other S^T buffer holds dQ_it-1 until the compute warps drained it
        if (it >= 1 && !mbar_wait(&sm.dq_empty, (it - 1) & 1, abort, err, kDevTimeoutOther)) break;
        if (next) {
          if (!mbar_wait(&sm.qd_full[b ^ 1], ((it + 1) >> 1) & 1, abort, err, kDevTimeoutFull))
            break;
          issue_kk(col_s(b ^ 1), k_s, smem_u32(sm.q[b ^ 1]));
          mma_commit_elect(&sm.s_full[b ^ 1]);
        }
        if (!mbar_wait(&sm.sm_done, it & 1, abort, err, kDevTimeoutOther)) break;
        fence_after_sync();
        // dV += P^T dO_i: 16-query group kk's P^T is in dP^T columns 32(kk/2) + 8(kk%2)
        mma_ts_run8<128, 8, 32, 40, 64, 72, 96, 104>(
            tmem + kColDV, tmem + kColDP, desc_sw128(smem_u32(sm.dout[b]), 8192, 1024), id_mn,
            it > 0 ? 1u : 0u);
        if (next) {
          issue_kk(kColDP, v_s, smem_u32(sm.dout[b ^ 1]));
          mma_commit_elect(&sm.dp_full);
        }
        const uint32_t q0 = smem_u32(sm.q[b]);
        issue_dk(sm.ds_hi[b], q0, it == 0);
        issue_dk(sm.ds_lo[b], q0, false);
        issue_dq(sm.ds_hi[b], col_s(b), true);
        issue_dq(sm.ds_lo[b], col_s(b), false);
        mma_commit_elect(&sm.dq_full);
        mma_commit_elect(&sm.qd_empty[b]);
      }
      mma_commit_elect(&sm.acc_full);
      mma_commit_elect(&sm.drain);
      wait_drain(&sm.drain, 0);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------- compute
    const int w = warp >> 2;        // warpgroup: queries 32w..32w+31
    const int tl = (warp & 3) * 32 + lane;  // TMEM lane: key row here, query row in dQ
    const int jg = j0 + tl;
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const int qw = 32 * w;                  // first query of this warpgroup in a block
    const int half = w >> 1;
    const uint32_t chunk0 = 4u * (uint32_t)(w & 1);  // first 16-byte chunk in the half-tile row
    // dQ of the block before: rows = queries, this warpgroup's 16 columns
    auto drain_dq = [&](int itp) -> bool {
      if (!mbar_wait(&sm.dq_full, itp & 1, abort, err, kDevTimeoutMma)) return false;
      fence_after_sync();
      uint32_t a[16];
      tmem_ld16(tmem + lane_off + col_s(itp & 1) + 16 * w, a);
      tmem_wait_ld();
      fence_before_sync();
      mbar_arrive(&sm.dq_empty);
      const int row = (ib0 + itp) * BQ + tl;
      if (row < N) {
        float* dst = dqacc + ((size_t)head * N + row) * HD + 16 * w;
#pragma unroll
        for (int c = 0; c < 4; ++c)
          red_add_v4(dst + 4 * c, __uint_as_float(a[4 * c]), __uint_as_float(a[4 * c + 1]),
                     __uint_as_float(a[4 * c + 2]), __uint_as_float(a[4 * c + 3]));
      }
      return true;
    };
    bool ok = true;
    for (int it = 0; it < n_q; ++it) {
      const int b = it & 1;
      const int ib = ib0 + it;
      const int i0 = ib * BQ;
      const bool need_mask = (causal && ib == jb) || (i0 + BQ > N) || (j0 + BK > N);
      // S^T_i done implies Q_i's stage (with lse and delta) has landed
      if (!mbar_wait(&sm.s_full[b], (it >> 1) & 1, abort, err, kDevTimeoutMma) ||
          !mbar_wait(&sm.dp_full, it & 1, abort, err, kDevTimeoutMma)) {
        ok = false;
        break;
      }
      fence_after_sync();
      uint32_t sv[32], dpv[32];
      tmem_ld16(tmem + lane_off + col_s(b) + qw, *reinterpret_cast<uint32_t(*)[16]>(sv));
      tmem_ld16(tmem + lane_off + col_s(b) + qw + 16, *reinterpret_cast<uint32_t(*)[16]>(sv + 16));
      tmem_ld16(tmem + lane_off + kColDP + qw, *reinterpret_cast<uint32_t(*)[16]>(dpv));
      tmem_ld16(tmem + lane_off + kColDP + qw + 16,
                *reinterpret_cast<uint32_t(*)[16]>(dpv + 16));
      tmem_wait_ld();
      uint32_t wp[16], wh[16], wl[16];
      const float4* l4 = reinterpret_cast<const float4*>(&sm.lse[b][qw]);
      const float4* d4 = reinterpret_cast<const float4*>(&sm.delta[b][qw]);
#pragma unroll
      for (int e4 = 0; e4 < 8; ++e4) {
        const float4 lv = l4[e4], dl = d4[e4];
        const float la[4] = {lv.x, lv.y, lv.z, lv.w};
        const float da[4] = {dl.x, dl.y, dl.z, dl.w};
        float p[4], ds[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int e = 4 * e4 + u;
          p[u] = ex2(fmaf(__uint_as_float(sv[e]), scale_log2, -la[u]));
          ds[u] = p[u] * (__uint_as_float(dpv[e]) - da[u]);
          if (need_mask) {
            const int ig = i0 + qw + e;
            if (ig >= N || jg >= N || (causal && ig < jg)) {
              p[u] = 0.f;
              ds[u] = 0.f;
            }
          }
        }
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const int w2 = 2 * e4 + u;
          wp[w2] = pack_bf16(p[2 * u], p[2 * u + 1]);
          wh[w2] = pack_bf16(ds[2 * u], ds[2 * u + 1]);
          wl[w2] = pack_bf16(ds[2 * u] - bf16lo(wh[w2]), ds[2 * u + 1] - bf16hi(wh[w2]));
        }
      }
      // P^T of this warpgroup's 32 queries over its own (already loaded) dP^T columns
      tmem_st16(tmem + lane_off + kColDP + qw, wp);
      // dS row of this key into buffer b: query q is element q % 64 of half
      // q / 64; 16-byte chunk k (8 queries) of a half-tile row sits at chunk
      // k ^ (key & 7) (128-byte swizzle)
      {
        const uint32_t hi_row = smem_u32(sm.ds_hi[b][half]) + tl * 128;
        const uint32_t lo_row = smem_u32(sm.ds_lo[b][half]) + tl * 128;
#pragma unroll
        for (int g = 0; g < 4; ++g) {
          const uint32_t off = ((chunk0 + g) ^ (uint32_t)(tl & 7)) << 4;
          st_shared_v4(hi_row + off, wh[4 * g], wh[4 * g + 1], wh[4 * g + 2], wh[4 * g + 3]);
          st_shared_v4(lo_row + off, wl[4 * g], wl[4 * g + 1], wl[4 * g + 2], wl[4 * g + 3]);
        }
      }
      if (it >= 1 && !drain_dq(it - 1)) {
        ok = false;
        break;
      }
      tmem_wait_st();
      fence_proxy_async_smem();
      fence_before_sync();
      mbar_arrive(&sm.sm_done);
    }
    if (ok && n_q > 0) ok = drain_dq(n_q - 1);
    // ---- columns 16w..16w+15 of this key's dv and dk
    if (ok && mbar_wait(&sm.acc_full, 0, abort, err, kDevTimeoutMma)) {
      fence_after_sync();
      uint32_t av[16], ak[16];
      tmem_ld16(tmem + lane_off + kColDV + 16 * w, av);
      tmem_ld16(tmem + lane_off + kColDK + 16 * w, ak);
      tmem_wait_ld();
      if (jg < N) {
        uint4* dvd = reinterpret_cast<uint4*>(dv + ((size_t)head * N + jg) * HD + 16 * w);
        uint4* dkd = reinterpret_cast<uint4*>(dk + ((size_t)head * N + jg) * HD + 16 * w);
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          dvd[h] = make_uint4(
              pack_bf16(__uint_as_float(av[8 * h + 0]), __uint_as_float(av[8 * h + 1])),
              pack_bf16(__uint_as_float(av[8 * h + 2]), __uint_as_float(av[8 * h + 3])),
              pack_bf16(__uint_as_float(av[8 * h + 4]), __uint_as_float(av[8 * h + 5])),
              pack_bf16(__uint_as_float(av[8 * h + 6]), __uint_as_float(av[8 * h + 7])));
          dkd[h] = make_uint4(pack_bf16(__uint_as_float(ak[8 * h + 0]) * scale,
                                        __uint_as_float(ak[8 * h + 1]) * scale),
                              pack_bf16(__uint_as_float(ak[8 * h + 2]) * scale,
                                        __uint_as_float(ak[8 * h + 3]) * scale),
                              pack_bf16(__uint_as_float(ak[8 * h + 4]) * scale,
                                        __uint_as_float(ak[8 * h + 5]) * scale),
                              pack_bf16(__uint_as_float(ak[8 * h + 6]) * scale,
                                        __uint_as_float(ak[8 * h + 7]) * scale));
        }
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

// dq = bf16(scale * dq accumulator) for the heads the tensor-core kernel took.
__global__ void __launch_bounds__(256)
attn_dq_convert_kernel(const float4* __restrict__ acc, uint4* __restrict__ dq, int64_t rows_per_head,
                       int64_t total8, float scale, const int* __restrict__ flags) {
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  const int64_t per_head8 = rows_per_head * (HD / 8);
  for (int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; idx < total8; idx += stride) {
    if (flags[idx / per_head8] != 0) continue;
    const float4 a = acc[2 * idx], c = acc[2 * idx + 1];
    dq[idx] = make_uint4(pack_bf16(a.x * scale, a.y * scale), pack_bf16(a.z * scale, a.w * scale),
                         pack_bf16(c.x * scale, c.y * scale), pack_bf16(c.z * scale, c.w * scale));
  }
}

}  // namespace

cudaError_t launch_attn_bwd_tc(const void* q, const void* k, const void* v, const void* dout,
                               const float* lse2, const float* delta, void* dk, void* dv,
                               float* dqacc, int64_t B, int64_t H, int64_t N, int causal,
                               float scale, const int* flags, unsigned* err, cudaStream_t s,
                               int* launches) {
  const int64_t BH = B * H;
  CUtensorMap tq, tk, tv, tdo;
  cudaError_t e;
  if ((e = make_tmap_bf16_rows(&tq, q, BH, N, BQ)) != cudaSuccess) return e;
  if ((e = make_tmap_bf16_rows(&tk, k, BH, N, BK)) != cudaSuccess) return e;
  if ((e = make_tmap_bf16_rows(&tv, v, BH, N, BK)) != cudaSuccess) return e;
  if ((e = make_tmap_bf16_rows(&tdo, dout, BH, N, BQ)) != cudaSuccess) return e;
  e = cudaFuncSetAttribute(attn_bwd_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)kSmemBytes);
  if (e != cudaSuccess) return e;
  const int64_t n_blocks = (N + BK - 1) / BK;
  attn_bwd_tc_kernel<<<(unsigned)(n_blocks * BH), kThreads, kSmemBytes, s>>>(
      tq, tk, tv, tdo, lse2, delta, static_cast<__nv_bfloat16*>(dk),
      static_cast<__nv_bfloat16*>(dv), dqacc, (int)N, (int)BH, causal, scale, scale * kLog2e,
      flags, err);
  *launches += 1;
  return cudaGetLastError();
}

cudaError_t launch_attn_dq_convert(const float* dqacc, void* dq, int64_t BH, int64_t N,
                                   float scale, const int* flags, cudaStream_t s,
                                   int* launches) {
  const int64_t total8 = BH * N * HD / 8;
  int64_t blocks = (total8 + 255) / 256;
  if (blocks > 148 * 16) blocks = 148 * 16;
  attn_dq_convert_kernel<<<(unsigned)blocks, 256, 0, s>>>(
      reinterpret_cast<const float4*>(dqacc), static_cast<uint4*>(dq), N, total8, scale, flags);
  *launches += 1;
  return cudaGetLastError();
}

}  // namespace swa
