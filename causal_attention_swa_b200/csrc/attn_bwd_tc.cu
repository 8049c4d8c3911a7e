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
// Operands: the kernels are instantiated for f16 and for bf16 operands.  The
// f16 instance reads f16 copies of q, k, v and dout (made by the caller's
// prep pass, exact for values below 2^15 in magnitude) and takes P and dS as
// f16 (10 fraction bits), which keeps the end-to-end gradient of
// 1/2 sum out^2 inside the bf16 path's tolerance with one dS per dQ product;
// the bf16 instance (heads with larger values) takes P and dS^T as bf16 and
// dS for dQ as bf16 hi + lo (below).  Each launch takes the heads of its type.
// Two kernels, neither with atomics:
//   attn_bwd_dkdv_kernel  block = one 128-key block j; it walks the query
//                         blocks i that see j and keeps dV_j, dK_j in TMEM
//   attn_bwd_dq_kernel    block = one 128-query block i; it walks the key
//                         blocks j that i sees and keeps dQ_i in TMEM
// Each recomputes S and dP for its pairs (two of the products are done
// twice), in exchange for no float32 dQ accumulator in memory, no reduce
// traffic and no conversion pass.
//
// Both kernels: 576 threads = warps 0-15 compute (four warpgroups), warp 16
// TMA producer, warp 17 MMA issuer (one elected lane) and TMEM owner.  The
// compute warps copy S and dP of a block into registers and release dP's
// TMEM columns at once (dp_free), so the MMA warp computes the next block's
// dP (and S, double-buffered) while they form P and dS: the tensor pipe
// works under the exponentials instead of waiting for them.
//
// dkdv: thread t of warpgroup w owns key j0 + t (TMEM lane t) and queries
// 32w..32w+31 of a block.  Per query block four products (M = 128):
//   S^T = K_j Q_i^T      (A = K smem K-major, B = Q smem K-major)
//   dP^T = V_j dO_i^T    (A = V, B = dO, both K-major)
//   dV += P^T dO_i       (A = P^T from TMEM, B = dO MN-major)
//   dK += dS^T Q_i       (A = dS^T from TMEM, B = Q MN-major)
// P^T and dS^T (bf16) go back over the warpgroup's own, already loaded S^T
// columns 32w..32w+15 and 32w+16..32w+31.
// dq: thread t of warpgroup w owns query i0 + t (TMEM lane t) and keys
// 32w..32w+31 of a block.  Per key block:
//   S = Q_i K_j^T, dP = dO_i V_j^T   (A from TMEM, B K-major)
//   dQ += dS_hi K_j + dS_lo K_j      (A = dS from TMEM, B = K MN-major)
// with dS_hi and dS_lo over the warpgroup's own S columns likewise.
// Operands that a thread computes never pass through shared memory: an SS
// MMA of N = 64 reads 6 KB of shared memory per 32 tensor cycles, above the
// 128 bytes per clock the SM's shared memory delivers, while A from TMEM
// costs none of it.  A later S MMA may overwrite those TMEM columns because
// one thread's MMAs execute in issue order.
// In the bf16 instance dS is carried as hi + lo bf16 (hi = bf16(dS),
// lo = bf16(dS - hi)) for dq: sum_j dS_ij = 0, and a single bf16 rounding of
// dS, amplified by that cancellation in sum_j dS_ij k_j, costs dq about 2% of
// its row RMS at N = 2048.  An f16 dS (three more fraction bits) needs no lo.
// Causal: a key block meets only the query blocks i >= j; inside a diagonal
// block (and past N on a ragged tail) P and dS of a masked pair are set to
// 0 by select, so dS never carries a masked pair into dK or dQ.
// Non-finite V or dout (absent rows, "check_masks_are_absent_rows": a masked
// pair must never enter a product).  Every product over existing pairs is
// the IEEE one: S, dP, dS and the dK, dQ sums run on the values as given
// (tcgen05 propagates infinities and NaN), and for dq the lo word of a
// non-finite dS is 0 (hi - hi would be NaN).  The one product that meets
// masked pairs is dV += P^T dO_i of the diagonal block: its zero weights
// meet dout rows of queries before the key.  For a head whose V or dout
// holds an infinity or NaN (the scan's flag), the dK/dV kernel therefore
// loads the diagonal block's dO a second time into a buffer of its own,
// the producer warp replaces its non-finite entries by 0 (recording, per
// column d, the last query row of the block holding +inf, -inf and NaN),
// and dV of that block reads the clean copy; the epilogue then merges the
// IEEE class those rows give dV_jd (rows i >= j of the block, each with a
// weight > 0) into the value the other blocks accumulated.
// Every mbarrier wait is bounded (device error word on expiry).
#include <type_traits>

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
constexpr int kQStages = 4;             // dkdv's Q/dO ring depth
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColDP = 256;

// Per-head information (four int32 per head, from the prep pass):
//   [0] bit 0: V holds an infinity or NaN; bit 1: dout does
//   [1] [2] [3] largest biased exponent of the finite values of V, of Q and
//       K, and of dout.
// A head takes the f16 instance when all three exponents are below 2^15's.
constexpr int kInfoInts = 4;
constexpr int kF16ExpLimit = 127 + 15;
__device__ __forceinline__ bool head_is_f16(const int* info, int head) {
  const int* hi = info + kInfoInts * head;
  return max(hi[1], max(hi[2], hi[3])) < kF16ExpLimit;
}

// A 16-bit value (f16 or bf16) that is +-inf or NaN, and its class
// (0 = +inf, 1 = -inf, 2 = NaN).
template <bool kF16>
__device__ __forceinline__ bool nonfinite16(uint32_t b) {
  return kF16 ? (b & 0x7C00u) == 0x7C00u : (b & 0x7F80u) == 0x7F80u;
}
template <bool kF16>
__device__ __forceinline__ int class16(uint32_t b) {
  return (b & (kF16 ? 0x03FFu : 0x7Fu)) ? 2 : ((b & 0x8000u) ? 1 : 0);
}

__device__ __forceinline__ uint32_t col_s(int b) { return b ? 128u : 0u; }

__device__ __forceinline__ bool wait_drain(uint64_t* bar, uint32_t parity) {
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity)) {
    if (clock64() - t0 > kWaitCycles) return false;
  }
  return true;
}

// Block -> (head, block index) in groups of `group_heads` heads (head_group()
// on the host: the operands a head's blocks stream stay in L2); inside a
// group the heaviest blocks first, heads interleaved.  heavy_low: block
// index 0 is the heaviest (dkdv: key block 0 meets every query block);
// else the last one is (dq: the last query block sees every key block).
__device__ __forceinline__ void block_order(int n_blocks, int BH, int group_heads,
                                            bool heavy_low, int* head, int* blk) {
  const int group = blockIdx.x / (group_heads * n_blocks);
  const int g_heads = min(group_heads, BH - group * group_heads);
  const int r = blockIdx.x - group * group_heads * n_blocks;
  const int rank = r / g_heads;
  *head = group * group_heads + r % g_heads;
  *blk = heavy_low ? rank : n_blocks - 1 - rank;
}

// =================================================================== dK, dV

struct __align__(1024) SmemKV {
  uint8_t k[kTileBytes];
  uint8_t v[kTileBytes];
  uint8_t q[kQStages][kTileBytes];
  uint8_t dout[kQStages][kTileBytes];
  uint8_t dout_diag[kTileBytes];  // non-finite heads: the diagonal block's dO, cleaned
  float nlse[kQStages][BQ];      // -lse_i * log2(e) of each staged query block (-inf past N)
  float delta[kQStages][BQ];     // delta_i (0 past N)
  int last_cls[3][HD];           // per column: last diagonal-block row with +inf, -inf, NaN
  uint64_t diag_full;
  uint64_t diag_clean;
  uint64_t kv_full;
  uint64_t qd_full[kQStages];
  uint64_t qd_empty[kQStages];
  uint64_t dp_full;  // dP^T (and the S^T issued before it) of the next block
  uint64_t dp_free;
  uint64_t sm_done;
  uint64_t acc_full;
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
};
constexpr size_t kSmemKV = sizeof(SmemKV);
static_assert(kSmemKV <= 232448, "shared memory");
constexpr uint32_t kColDV = 384, kColDK = 448;

template <bool kF16>
__global__ void __launch_bounds__(kThreads, 1)
attn_bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tm_q,
                     const __grid_constant__ CUtensorMap tm_k,
                     const __grid_constant__ CUtensorMap tm_v,
                     const __grid_constant__ CUtensorMap tm_do, const float* __restrict__ nlse2,
                     const float* __restrict__ delta, __nv_bfloat16* __restrict__ dk,
                     __nv_bfloat16* __restrict__ dv, float* __restrict__ dk_acc,
                     float* __restrict__ dv_acc, int N, int BH, int group_heads, int causal,
                     float scale,
                     float scale_log2, const int* __restrict__ info, unsigned* __restrict__ err) {
  pdl_prologue();  // the next launch (independent outputs) overlaps this one's tail
  const int n_blocks = (N + BQ - 1) / BQ;
  const int Npad = n_blocks * BQ;
  int head, jb;
  block_order(n_blocks, BH, group_heads, true, &head, &jb);
  if (head_is_f16(info, head) != kF16) return;  // the other instance's head
  // a head with a non-finite V or dout: dV of the diagonal block reads a
  // cleaned copy of its dO (non-causal: no masked pair meets dO at all)
  const bool clean_diag = info[kInfoInts * head] != 0 && causal;

  extern __shared__ __align__(1024) uint8_t smem_raw[];
  if (smem_u32(smem_raw) & 1023u) {  // the swizzled tiles need 1024-byte alignment
    if (threadIdx.x == 0) atomicCAS(err, 0u, (unsigned)kDevSmemAlign);
    return;
  }
  SmemKV& sm = *reinterpret_cast<SmemKV*>(smem_raw);
  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int ib0 = causal ? jb : 0;
  const int n_q = n_blocks - ib0;
  const int j0 = jb * BK;

  if (tid == 0) {
    mbar_init(&sm.kv_full, 1);
    for (int s = 0; s < kQStages; ++s) {
      mbar_init(&sm.qd_full[s], 1);
      mbar_init(&sm.qd_empty[s], 1);
    }
    mbar_init(&sm.dp_full, 1);
    mbar_init(&sm.dp_free, kComputeThreads / 32);  // one arrival per compute warp
    mbar_init(&sm.sm_done, kComputeThreads / 32);
    mbar_init(&sm.acc_full, 1);
    mbar_init(&sm.drain, 1);
    mbar_init(&sm.diag_full, 1);
    mbar_init(&sm.diag_clean, 1);
    sm.abort = 0;
    fence_mbar_init();
  }
  if (tid < 3 * HD) (&sm.last_cls[0][0])[tid] = -1;
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
    if (clean_diag) {
      // the diagonal block's dO once more, into a buffer of its own; every
      // lane then cleans it (non-finite -> 0, rows recorded per column)
      if (lane == 0) {
        mbar_arrive_expect_tx(&sm.diag_full, kTileBytes);
        tma_load_3d(sm.dout_diag, &tm_do, &sm.diag_full, 0, j0, head);
      }
      __syncwarp();
      if (mbar_wait_parked(&sm.diag_full, 0, abort, err, kDevTimeoutFull)) {
        uint4* base = reinterpret_cast<uint4*>(sm.dout_diag);
        for (int c = lane; c < kTileBytes / 16; c += 32) {
          const uint4 x = base[c];
          uint32_t w[4] = {x.x, x.y, x.z, x.w};
          const int r = c >> 3;                      // query row of the block
          const int d0 = ((c & 7) ^ (r & 7)) * 8;    // first column (swizzle undone)
          bool changed = false;
#pragma unroll
          for (int e = 0; e < 4; ++e)
#pragma unroll
            for (int p = 0; p < 2; ++p) {
              const uint32_t bits = (w[e] >> (16 * p)) & 0xFFFFu;
              if (nonfinite16<kF16>(bits)) {
                atomicMax(&sm.last_cls[class16<kF16>(bits)][d0 + 2 * e + p], j0 + r);
                w[e] &= ~(0xFFFFu << (16 * p));
                changed = true;
              }
            }
          if (changed) base[c] = make_uint4(w[0], w[1], w[2], w[3]);
        }
      }
      fence_proxy_async_smem();  // the dV MMA (async proxy) reads the cleaned tile
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.diag_clean);
    }
    if (lane == 0) {
      prefetch_tmap(&tm_q);
      prefetch_tmap(&tm_k);
      prefetch_tmap(&tm_v);
      prefetch_tmap(&tm_do);
      mbar_arrive_expect_tx(&sm.kv_full, 2 * kTileBytes);
      tma_load_3d(sm.k, &tm_k, &sm.kv_full, 0, j0, head);
      tma_load_3d(sm.v, &tm_v, &sm.kv_full, 0, j0, head);
      for (int it = 0; it < n_q; ++it) {
        const int s = it % kQStages;
        const int round = it / kQStages;
        if (round > 0 && !mbar_wait_parked(&sm.qd_empty[s], (round - 1) & 1, abort, err,
                                           kDevTimeoutEmpty))
          break;
        const int i0 = (ib0 + it) * BQ;
        mbar_arrive_expect_tx(&sm.qd_full[s], 2 * kTileBytes + 2 * BQ * 4);
        tma_load_3d(sm.q[s], &tm_q, &sm.qd_full[s], 0, i0, head);
        tma_load_3d(sm.dout[s], &tm_do, &sm.qd_full[s], 0, i0, head);
        bulk_load(sm.nlse[s], nlse2 + (size_t)head * Npad + i0, BQ * 4, &sm.qd_full[s]);
        bulk_load(sm.delta[s], delta + (size_t)head * Npad + i0, BQ * 4, &sm.qd_full[s]);
      }
    }
    __syncwarp();
  } else if (warp == kMmaWarp) {
    // --------------------------------------------------------- MMA issuer
    {  // the whole warp runs the issue loop; one elected lane issues
      constexpr uint32_t fmt = kF16 ? 0u : 1u;
      constexpr uint32_t id_kk = idesc_f32acc(128, 128, 0, 0, fmt);  // S^T, dP^T: both K-major
      constexpr uint32_t id_mn = idesc_f32acc(128, 64, 0, 1, fmt);   // dV, dK: B MN-major
      const uint32_t k_s = smem_u32(sm.k), v_s = smem_u32(sm.v);
      // descriptor steps in 16-byte units: K-major +32 B (2) per K = 16
      // step, MN-major +2048 B (128)
      auto issue_kk = [&](uint32_t d_col, uint32_t a0, uint32_t b0) {
        mma_ss_run<4, 2, 0, 2>(tmem + d_col, desc_sw128(a0, 16, 1024), desc_sw128(b0, 16, 1024),
                               id_kk, 0u);
      };
      auto wait_qd = [&](int it) {
        return mbar_wait_parked(&sm.qd_full[it % kQStages], (it / kQStages) & 1, abort, err,
                                kDevTimeoutFull);
      };
      bool ok = mbar_wait_parked(&sm.kv_full, 0, abort, err, kDevTimeoutFull) && n_q > 0 &&
                wait_qd(0);
      if (ok) {
        fence_after_sync();
        issue_kk(col_s(0), k_s, smem_u32(sm.q[0]));
        issue_kk(kColDP, v_s, smem_u32(sm.dout[0]));
        mma_commit_elect(&sm.dp_full);
      }
      for (int it = 0; ok && it < n_q; ++it) {
        const int b = it & 1;
        const int st = it % kQStages;
        if (it + 1 < n_q) {
          const int sn = (it + 1) % kQStages;
          // S^T_it+1 over P^T_it-1 and dS^T_it-1: the dV and dK MMAs that
          // read them were issued before
          if (!wait_qd(it + 1)) break;
          fence_after_sync();
          issue_kk(col_s(b ^ 1), k_s, smem_u32(sm.q[sn]));
          // dP^T_it+1 once the compute warps hold dP^T_it in registers
          if (!mbar_wait_parked(&sm.dp_free, it & 1, abort, err, kDevTimeoutOther)) break;
          fence_after_sync();
          issue_kk(kColDP, v_s, smem_u32(sm.dout[sn]));
          mma_commit_elect(&sm.dp_full);
        }
        if (!mbar_wait_parked(&sm.sm_done, it & 1, abort, err, kDevTimeoutOther)) break;
        const bool diag = clean_diag && it == 0;  // dV of the diagonal block: the clean dO
        if (diag && !mbar_wait_parked(&sm.diag_clean, 0, abort, err, kDevTimeoutOther)) break;
        fence_after_sync();
        // dV += P^T dO_i: 16-query group kk's P^T is in S^T columns 32(kk/2) + 8(kk%2)
        mma_ts_run8<128, 8, 32, 40, 64, 72, 96, 104>(
            tmem + kColDV, tmem + col_s(b),
            desc_sw128(smem_u32(diag ? sm.dout_diag : sm.dout[st]), 8192, 1024), id_mn,
            it > 0 ? 1u : 0u);
        // dK += dS^T Q_i: dS^T of 16-query group kk 16 columns further on
        mma_ts_run8<128, 8, 32, 40, 64, 72, 96, 104>(
            tmem + kColDK, tmem + col_s(b) + 16, desc_sw128(smem_u32(sm.q[st]), 8192, 1024),
            id_mn, it > 0 ? 1u : 0u);
        mma_commit_elect(&sm.qd_empty[st]);
      }
      mma_commit_elect(&sm.acc_full);
      mma_commit_elect(&sm.drain);
      wait_drain(&sm.drain, 0);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------- compute
    const int w = warp >> 2;                 // warpgroup: queries 32w..32w+31
    const int tl = (warp & 3) * 32 + lane;   // TMEM lane = key row
    const int jg = j0 + tl;
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const int qw = 32 * w;
    bool ok = true;
    for (int it = 0; it < n_q; ++it) {
      const int b = it & 1;
      const int st = it % kQStages;
      const int ib = ib0 + it;
      const int i0 = ib * BQ;
      const bool need_mask = (causal && ib == jb) || (i0 + BQ > N) || (j0 + BK > N);
      // dP^T_i done implies S^T_i (issued before it) is done and Q_i's
      // stage (with lse and delta) has landed
      if (!mbar_wait_spin(&sm.dp_full, it & 1, abort, err, kDevTimeoutMma)) {
        ok = false;
        break;
      }
      fence_after_sync();
      // queries qw..qw+15 first; qw+16..qw+31 load while the first half is
      // worked, and the first half's stores drain under the second half
      uint32_t s0[16], d0[16], s1[16], d1[16];
      tmem_ld16(tmem + lane_off + col_s(b) + qw, s0);
      tmem_ld16(tmem + lane_off + kColDP + qw, d0);
      tmem_wait_ld();
      tmem_ld16(tmem + lane_off + col_s(b) + qw + 16, s1);
      tmem_ld16(tmem + lane_off + kColDP + qw + 16, d1);
      // two queries at a time in packed f32x2 arithmetic:
      //   p = 2^(s c - lse log2 e),  dS = p (dP - delta)
      uint32_t wp[16], wd[16];
      const float4* l4 = reinterpret_cast<const float4*>(&sm.nlse[st][qw]);
      const float4* d4 = reinterpret_cast<const float4*>(&sm.delta[st][qw]);
      const float2 c2 = make_float2(scale_log2, scale_log2);
      const float2 m1 = make_float2(-1.f, -1.f);
      // the mask flag is a compile-time constant of each instance, so the
      // unmasked blocks' code carries no per-pair tests
      auto math = [&](auto mask_tag, const uint32_t (&sv)[16], const uint32_t (&dpv)[16],
                      int h) {
        constexpr bool kMask = decltype(mask_tag)::value;
#pragma unroll
        for (int e4 = 0; e4 < 4; ++e4) {
          const float4 lv = l4[4 * h + e4], dl = d4[4 * h + e4];
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            const int e = 4 * e4 + 2 * u;
            const float2 nl = u ? make_float2(lv.z, lv.w) : make_float2(lv.x, lv.y);
            const float2 de = u ? make_float2(dl.z, dl.w) : make_float2(dl.x, dl.y);
            const float2 a = __ffma2_rn(
                make_float2(__uint_as_float(sv[e]), __uint_as_float(sv[e + 1])), c2, nl);
            float2 p = make_float2(ex2(a.x), ex2(a.y));
            const float2 dd = __ffma2_rn(
                de, m1, make_float2(__uint_as_float(dpv[e]), __uint_as_float(dpv[e + 1])));
            float2 ds = __fmul2_rn(p, dd);
            if constexpr (kMask) {
              const int ig = i0 + qw + 16 * h + e;
              if (ig >= N || jg >= N || (causal && ig < jg)) p.x = ds.x = 0.f;
              if (ig + 1 >= N || jg >= N || (causal && ig + 1 < jg)) p.y = ds.y = 0.f;
            }
            wp[8 * h + 2 * e4 + u] = pack_p<kF16>(p.x, p.y);
            wd[8 * h + 2 * e4 + u] = pack_p<kF16>(ds.x, ds.y);
          }
        }
      };
      if (need_mask) math(std::true_type{}, s0, d0, 0);
      else math(std::false_type{}, s0, d0, 0);
      // P^T and dS^T of these 16 queries over the warpgroup's own S^T
      // columns: P^T at 32w + 0..7, dS^T at 32w + 16..23 (the latter only
      // once the second half's load has landed)
      const uint32_t tw = tmem + lane_off + col_s(b) + qw;
      tmem_st8(tw, *reinterpret_cast<const uint32_t(*)[8]>(wp));
      tmem_wait_ld_tied(s1, d1);
      fence_before_sync();
      warp_arrive(&sm.dp_free);  // dP^T's columns may take the next block's
      tmem_st8(tw + 16, *reinterpret_cast<const uint32_t(*)[8]>(wd));
      if (need_mask) math(std::true_type{}, s1, d1, 1);
      else math(std::false_type{}, s1, d1, 1);
      tmem_st8(tw + 8, *reinterpret_cast<const uint32_t(*)[8]>(wp + 8));
      tmem_st8(tw + 24, *reinterpret_cast<const uint32_t(*)[8]>(wd + 8));
      tmem_wait_st();
      fence_before_sync();
      warp_arrive(&sm.sm_done);
    }
    // ---- columns 16w..16w+15 of this key's dv and dk
    if (ok && mbar_wait_spin(&sm.acc_full, 0, abort, err, kDevTimeoutMma)) {
      fence_after_sync();
      uint32_t av[16], ak[16];
      tmem_ld16(tmem + lane_off + kColDV + 16 * w, av);
      tmem_ld16(tmem + lane_off + kColDK + 16 * w, ak);
      tmem_wait_ld();
      if (clean_diag && mbar_wait_spin(&sm.diag_clean, 0, abort, err, kDevTimeoutOther)) {
        // merge the IEEE class of the diagonal block's rows i >= jg into dv
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const int d = 16 * w + e;
          const float x = __uint_as_float(av[e]);
          const bool pinf = sm.last_cls[0][d] >= jg || x == INFINITY;
          const bool ninf = sm.last_cls[1][d] >= jg || x == -INFINITY;
          const bool nan = sm.last_cls[2][d] >= jg || x != x || (pinf && ninf);
          if (nan) av[e] = 0x7FC00000u;
          else if (pinf) av[e] = 0x7F800000u;
          else if (ninf) av[e] = 0xFF800000u;
        }
      }
      if (jg < N && dv_acc != nullptr) {
        // accumulate mode: add this call's dv, dk (float32) to the caller's sums
        float4* va = reinterpret_cast<float4*>(dv_acc + ((size_t)head * N + jg) * HD + 16 * w);
        float4* ka = reinterpret_cast<float4*>(dk_acc + ((size_t)head * N + jg) * HD + 16 * w);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          float4 x = va[i], y = ka[i];
          x.x += __uint_as_float(av[4 * i]);
          x.y += __uint_as_float(av[4 * i + 1]);
          x.z += __uint_as_float(av[4 * i + 2]);
          x.w += __uint_as_float(av[4 * i + 3]);
          y.x += __uint_as_float(ak[4 * i]) * scale;
          y.y += __uint_as_float(ak[4 * i + 1]) * scale;
          y.z += __uint_as_float(ak[4 * i + 2]) * scale;
          y.w += __uint_as_float(ak[4 * i + 3]) * scale;
          va[i] = x;
          ka[i] = y;
        }
      } else if (jg < N) {
        uint4* dvd = reinterpret_cast<uint4*>(dv + ((size_t)head * N + jg) * HD + 16 * w);
        uint4* dkd = reinterpret_cast<uint4*>(dk + ((size_t)head * N + jg) * HD + 16 * w);
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          uint32_t pv[4], pk[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            pv[e] = pack_bf16(__uint_as_float(av[8 * h + 2 * e]),
                              __uint_as_float(av[8 * h + 2 * e + 1]));
            pk[e] = pack_bf16(__uint_as_float(ak[8 * h + 2 * e]) * scale,
                              __uint_as_float(ak[8 * h + 2 * e + 1]) * scale);
          }
          dvd[h] = make_uint4(pv[0], pv[1], pv[2], pv[3]);
          dkd[h] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
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

// ======================================================================= dQ

// Every role of this kernel polls its barriers (mbar_wait_spin): each of
// its waits sits on the block's critical path.
// Q_i and dO_i, the A operands of S and dP in every key block, sit in TMEM
// (columns [448, 480) and [480, 512), written once by the compute warps from
// their own rows), so those MMAs read only K_j and V_j from shared memory.
constexpr int kKVStagesQ = 4;

struct __align__(1024) SmemQ {
  uint8_t k[kKVStagesQ][kTileBytes];
  uint8_t v[kKVStagesQ][kTileBytes];
  uint64_t qt_ready;  // Q_i and dO_i are in TMEM
  uint64_t kv_full[kKVStagesQ];
  uint64_t kv_empty[kKVStagesQ];
  uint64_t dp_full;  // dP (and the S issued before it) of the next block
  uint64_t dp_free;
  uint64_t sm_done;
  uint64_t acc_full;
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
};
constexpr size_t kSmemQ = sizeof(SmemQ);
static_assert(kSmemQ <= 232448, "shared memory");
constexpr uint32_t kColDQ = 384, kColQ = 448, kColDO = 480;

template <bool kF16>
__global__ void __launch_bounds__(kThreads, 1)
attn_bwd_dq_kernel(const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const uint16_t* __restrict__ q,
                   const uint16_t* __restrict__ dout, const float* __restrict__ nlse2,
                   const float* __restrict__ delta, __nv_bfloat16* __restrict__ dq,
                   float* __restrict__ dq_acc, int N, int BH, int group_heads, int causal,
                   float scale,
                   float scale_log2, const int* __restrict__ info, unsigned* __restrict__ err) {
  pdl_prologue();  // the next launch (independent outputs) overlaps this one's tail
  const int n_blocks = (N + BQ - 1) / BQ;
  const int Npad = n_blocks * BQ;
  int head, ib;
  block_order(n_blocks, BH, group_heads, false, &head, &ib);
  if (head_is_f16(info, head) != kF16) return;  // the other instance's head
  const bool nonfinite = info[kInfoInts * head] != 0;  // V or dout holds an infinity or NaN

  extern __shared__ __align__(1024) uint8_t smem_raw[];
  if (smem_u32(smem_raw) & 1023u) {
    if (threadIdx.x == 0) atomicCAS(err, 0u, (unsigned)kDevSmemAlign);
    return;
  }
  SmemQ& sm = *reinterpret_cast<SmemQ*>(smem_raw);
  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int n_k = causal ? ib + 1 : n_blocks;
  const int i0 = ib * BQ;

  if (tid == 0) {
    mbar_init(&sm.qt_ready, kComputeThreads / 32);
    for (int s = 0; s < kKVStagesQ; ++s) {
      mbar_init(&sm.kv_full[s], 1);
      mbar_init(&sm.kv_empty[s], 1);
    }
    mbar_init(&sm.dp_full, 1);
    mbar_init(&sm.dp_free, kComputeThreads / 32);  // one arrival per compute warp
    mbar_init(&sm.sm_done, kComputeThreads / 32);
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
      prefetch_tmap(&tm_k);
      prefetch_tmap(&tm_v);
      for (int jt = 0; jt < n_k; ++jt) {
        const int s = jt % kKVStagesQ;
        const int round = jt / kKVStagesQ;
        if (round > 0 && !mbar_wait_spin(&sm.kv_empty[s], (round - 1) & 1, abort, err,
                                         kDevTimeoutEmpty))
          break;
        mbar_arrive_expect_tx(&sm.kv_full[s], 2 * kTileBytes);
        tma_load_3d(sm.k[s], &tm_k, &sm.kv_full[s], 0, jt * BK, head);
        tma_load_3d(sm.v[s], &tm_v, &sm.kv_full[s], 0, jt * BK, head);
      }
    }
    __syncwarp();
  } else if (warp == kMmaWarp) {
    // --------------------------------------------------------- MMA issuer
    {
      constexpr uint32_t fmt = kF16 ? 0u : 1u;
      constexpr uint32_t id_kk = idesc_f32acc(128, 128, 0, 0, fmt);  // S, dP: both K-major
      constexpr uint32_t id_mn = idesc_f32acc(128, 64, 0, 1, fmt);   // dQ: B (K_j) MN-major
      // S = Q K_j^T and dP = dO V_j^T with A from TMEM (8 columns per 16
      // dims) and B K-major (+32 B per 16 dims)
      auto issue_kk = [&](uint32_t d_col, uint32_t a_col, uint32_t b0) {
        mma_ts_run4<8, 2>(tmem + d_col, tmem + a_col, desc_sw128(b0, 16, 1024), id_kk, 0u);
      };
      // dQ (+)= dS K_j with dS from TMEM: 16-key group kk's hi words at
      // S columns 32(kk/2) + 8(kk%2), lo words 16 columns further on; B = K_j
      // rows (+2048 B per 16 keys)
      auto issue_dq = [&](uint32_t a_col, uint32_t k0, bool first) {
        mma_ts_run8<128, 8, 32, 40, 64, 72, 96, 104>(tmem + kColDQ, tmem + a_col,
                                                     desc_sw128(k0, 8192, 1024), id_mn,
                                                     first ? 0u : 1u);
      };
      auto wait_kv = [&](int jt) {
        return mbar_wait_spin(&sm.kv_full[jt % kKVStagesQ], (jt / kKVStagesQ) & 1, abort,
                              err, kDevTimeoutFull);
      };
      bool ok = mbar_wait_spin(&sm.qt_ready, 0, abort, err, kDevTimeoutOther) && n_k > 0 &&
                wait_kv(0);
      if (ok) {
        fence_after_sync();
        issue_kk(col_s(0), kColQ, smem_u32(sm.k[0]));
        issue_kk(kColDP, kColDO, smem_u32(sm.v[0]));
        mma_commit_elect(&sm.dp_full);
      }
      for (int jt = 0; ok && jt < n_k; ++jt) {
        const int b = jt & 1;
        const int st = jt % kKVStagesQ;
        if (jt + 1 < n_k) {
          const int sn = (jt + 1) % kKVStagesQ;
          // S_jt+1 over dS_jt-1: the dQ MMAs that read it were issued before
          if (!wait_kv(jt + 1)) break;
          fence_after_sync();
          issue_kk(col_s(b ^ 1), kColQ, smem_u32(sm.k[sn]));
          if (!mbar_wait_spin(&sm.dp_free, jt & 1, abort, err, kDevTimeoutOther)) break;
          fence_after_sync();
          issue_kk(kColDP, kColDO, smem_u32(sm.v[sn]));
          mma_commit_elect(&sm.dp_full);
        }
        if (!mbar_wait_spin(&sm.sm_done, jt & 1, abort, err, kDevTimeoutOther)) break;
        fence_after_sync();
        const uint32_t k0 = smem_u32(sm.k[st]);
        issue_dq(col_s(b), k0, jt == 0);
        if constexpr (!kF16) issue_dq(col_s(b) + 16, k0, false);  // + the lo words
        mma_commit_elect(&sm.kv_empty[st]);
      }
      mma_commit_elect(&sm.acc_full);
      mma_commit_elect(&sm.drain);
      wait_drain(&sm.drain, 0);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------- compute
    const int w = warp >> 2;                 // warpgroup: keys 32w..32w+31 of a block
    const int tl = (warp & 3) * 32 + lane;   // TMEM lane = query row
    const int ig = i0 + tl;
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const int kw = 32 * w;
    const float nl = nlse2[(size_t)head * Npad + ig];  // -inf past N
    const float dl = delta[(size_t)head * Npad + ig];  // 0 past N
    const float2 c2 = make_float2(scale_log2, scale_log2);
    const float2 nl2 = make_float2(nl, nl);
    const float2 dl2 = make_float2(dl, dl);
    const float2 m1 = make_float2(-1.f, -1.f);
    {  // this thread's 16 dims (16w..16w+15) of Q_i and dO_i into TMEM (0 past N)
      uint32_t qa[8], da[8];
      if (ig < N) {
        const size_t off = ((size_t)head * N + ig) * HD + 16 * w;
        const uint4* qs = reinterpret_cast<const uint4*>(q + off);  // 16-bit words as given
        const uint4* os = reinterpret_cast<const uint4*>(dout + off);
        const uint4 q0 = qs[0], q1 = qs[1], e0 = os[0], e1 = os[1];
        qa[0] = q0.x; qa[1] = q0.y; qa[2] = q0.z; qa[3] = q0.w;
        qa[4] = q1.x; qa[5] = q1.y; qa[6] = q1.z; qa[7] = q1.w;
        da[0] = e0.x; da[1] = e0.y; da[2] = e0.z; da[3] = e0.w;
        da[4] = e1.x; da[5] = e1.y; da[6] = e1.z; da[7] = e1.w;
      } else {
#pragma unroll
        for (int e = 0; e < 8; ++e) qa[e] = da[e] = 0u;
      }
      tmem_st8(tmem + lane_off + kColQ + 8 * w, qa);
      tmem_st8(tmem + lane_off + kColDO + 8 * w, da);
      tmem_wait_st();
      fence_before_sync();
      warp_arrive(&sm.qt_ready);
    }
    bool ok = true;
    for (int jt = 0; jt < n_k; ++jt) {
      const int b = jt & 1;
      const int j0 = jt * BK;
      const bool need_mask = (causal && jt == ib) || (j0 + BK > N) || (i0 + BQ > N);
      // dP_jt done implies S_jt (issued before it) is done
      if (!mbar_wait_spin(&sm.dp_full, jt & 1, abort, err, kDevTimeoutMma)) {
        ok = false;
        break;
      }
      fence_after_sync();
      // keys kw..kw+15 first; kw+16..kw+31 load while the first half is
      // worked, and the first half's dS stores drain under the second half
      uint32_t s0[16], d0[16], s1[16], d1[16];
      tmem_ld16(tmem + lane_off + col_s(b) + kw, s0);
      tmem_ld16(tmem + lane_off + kColDP + kw, d0);
      tmem_wait_ld();
      tmem_ld16(tmem + lane_off + col_s(b) + kw + 16, s1);
      tmem_ld16(tmem + lane_off + kColDP + kw + 16, d1);
      // two keys at a time in packed f32x2 arithmetic; lo = dS - hi is exact
      uint32_t wh[16], wl[16];
      auto math = [&](auto mask_tag, auto nonfinite_tag, const uint32_t (&sv)[16],
                      const uint32_t (&dpv)[16], int h) {
        constexpr bool kMask = decltype(mask_tag)::value;
        [[maybe_unused]] constexpr bool kNonFinite = decltype(nonfinite_tag)::value;
#pragma unroll
        for (int e2 = 0; e2 < 8; ++e2) {
          const int e = 2 * e2;
          const float2 a = __ffma2_rn(
              make_float2(__uint_as_float(sv[e]), __uint_as_float(sv[e + 1])), c2, nl2);
          const float2 p = make_float2(ex2(a.x), ex2(a.y));
          const float2 dd = __ffma2_rn(
              dl2, m1, make_float2(__uint_as_float(dpv[e]), __uint_as_float(dpv[e + 1])));
          float2 ds = __fmul2_rn(p, dd);
          if constexpr (kMask) {
            const int jg = j0 + kw + 16 * h + e;
            if (jg >= N || ig >= N || (causal && jg > ig)) ds.x = 0.f;
            if (jg + 1 >= N || ig >= N || (causal && jg + 1 > ig)) ds.y = 0.f;
          }
          const int wi = 8 * h + e2;
          if constexpr (kF16) {
            wh[wi] = pack_f16(ds.x, ds.y);
          } else {
            wh[wi] = pack_bf16(ds.x, ds.y);
            float2 lo = __ffma2_rn(make_float2(bf16lo(wh[wi]), bf16hi(wh[wi])), m1, ds);
            if constexpr (kNonFinite) {  // inf - inf: the hi word carries the class alone
              if (!isfinite(ds.x)) lo.x = 0.f;
              if (!isfinite(ds.y)) lo.y = 0.f;
            }
            wl[wi] = pack_bf16(lo.x, lo.y);
          }
        }
      };
      auto math_any = [&](const uint32_t (&sv)[16], const uint32_t (&dpv)[16], int h) {
        if (nonfinite) {
          if (need_mask) math(std::true_type{}, std::true_type{}, sv, dpv, h);
          else math(std::false_type{}, std::true_type{}, sv, dpv, h);
        } else {
          if (need_mask) math(std::true_type{}, std::false_type{}, sv, dpv, h);
          else math(std::false_type{}, std::false_type{}, sv, dpv, h);
        }
      };
      math_any(s0, d0, 0);
      // dS of these 16 keys over the warpgroup's own S columns: hi at
      // 32w + 0..7, lo at 32w + 16..23 (once the second half's load landed)
      const uint32_t tw = tmem + lane_off + col_s(b) + kw;
      tmem_st8(tw, *reinterpret_cast<const uint32_t(*)[8]>(wh));
      tmem_wait_ld_tied(s1, d1);
      fence_before_sync();
      warp_arrive(&sm.dp_free);  // dP's columns may take dP_jt+1
      if constexpr (!kF16) tmem_st8(tw + 16, *reinterpret_cast<const uint32_t(*)[8]>(wl));
      math_any(s1, d1, 1);
      tmem_st8(tw + 8, *reinterpret_cast<const uint32_t(*)[8]>(wh + 8));
      if constexpr (!kF16) tmem_st8(tw + 24, *reinterpret_cast<const uint32_t(*)[8]>(wl + 8));
      tmem_wait_st();
      fence_before_sync();
      warp_arrive(&sm.sm_done);
    }
    // ---- columns 16w..16w+15 of this query's dq
    if (ok && mbar_wait_spin(&sm.acc_full, 0, abort, err, kDevTimeoutMma)) {
      fence_after_sync();
      uint32_t a[16];
      tmem_ld16(tmem + lane_off + kColDQ + 16 * w, a);
      tmem_wait_ld();
      if (ig < N && dq_acc != nullptr) {
        // accumulate mode: add this call's dq (float32) to the caller's sums
        float4* dqa = reinterpret_cast<float4*>(dq_acc + ((size_t)head * N + ig) * HD + 16 * w);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          float4 x = dqa[i];
          x.x += __uint_as_float(a[4 * i]) * scale;
          x.y += __uint_as_float(a[4 * i + 1]) * scale;
          x.z += __uint_as_float(a[4 * i + 2]) * scale;
          x.w += __uint_as_float(a[4 * i + 3]) * scale;
          dqa[i] = x;
        }
      } else if (ig < N) {
        uint4* dst = reinterpret_cast<uint4*>(dq + ((size_t)head * N + ig) * HD + 16 * w);
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          uint32_t pq[4];
#pragma unroll
          for (int e = 0; e < 4; ++e)
            pq[e] = pack_bf16(__uint_as_float(a[8 * h + 2 * e]) * scale,
                              __uint_as_float(a[8 * h + 2 * e + 1]) * scale);
          dst[h] = make_uint4(pq[0], pq[1], pq[2], pq[3]);
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

template <bool kF16>
cudaError_t launch_bwd_instance(const void* q, const void* k, const void* v, const void* dout,
                                const float* nlse2, const float* delta, void* dq, void* dk,
                                void* dv, const BwdAcc& acc, int64_t BH, int64_t N, int causal,
                                float scale, const int* info, unsigned* err, cudaStream_t s,
                                bool after, int* launches) {
  CUtensorMap tq, tk, tv, tdo;
  cudaError_t e;
  if ((e = make_tmap_bf16_rows(&tq, q, BH, N, BQ)) != cudaSuccess) return e;
  if ((e = make_tmap_bf16_rows(&tk, k, BH, N, BK)) != cudaSuccess) return e;
  if ((e = make_tmap_bf16_rows(&tv, v, BH, N, BK)) != cudaSuccess) return e;
  if ((e = make_tmap_bf16_rows(&tdo, dout, BH, N, BQ)) != cudaSuccess) return e;
  e = cudaFuncSetAttribute(attn_bwd_dkdv_kernel<kF16>,
                           cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemKV);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(attn_bwd_dq_kernel<kF16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)kSmemQ);
  if (e != cudaSuccess) return e;
  const int64_t n_blocks = (N + BK - 1) / BK;
  // dkdv, dq and the other instance's pair write disjoint outputs and read
  // only what was complete before the first of them: each after the first
  // may start in the tail of the one before
  const dim3 grid((unsigned)(n_blocks * BH));
  e = launch_after(after, attn_bwd_dkdv_kernel<kF16>, grid, dim3(kThreads), kSmemKV, s, tq, tk,
                   tv, tdo, nlse2, delta, static_cast<__nv_bfloat16*>(dk),
                   static_cast<__nv_bfloat16*>(dv), acc.dk, acc.dv, (int)N, (int)BH,
                   head_group(BH, N), causal, scale, scale * kLog2e, info, err);
  if (e != cudaSuccess) return e;
  *launches += 1;
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  e = launch_after(true, attn_bwd_dq_kernel<kF16>, grid, dim3(kThreads), kSmemQ, s, tk, tv,
                   static_cast<const uint16_t*>(q), static_cast<const uint16_t*>(dout), nlse2,
                   delta, static_cast<__nv_bfloat16*>(dq), acc.dq, (int)N, (int)BH,
                   head_group(BH, N), causal, scale, scale * kLog2e, info, err);
  if (e != cudaSuccess) return e;
  *launches += 1;
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attn_bwd_tc(const BwdOperands& f16, const BwdOperands& bf16,
                               const float* nlse2, const float* delta, void* dq, void* dk,
                               void* dv, const BwdAcc& acc, int64_t B, int64_t H, int64_t N,
                               int causal, float scale, const int* info, unsigned* err,
                               cudaStream_t s, int* launches) {
  const int64_t BH = B * H;
  cudaError_t e = launch_bwd_instance<true>(f16.q, f16.k, f16.v, f16.dout, nlse2, delta, dq, dk,
                                            dv, acc, BH, N, causal, scale, info, err, s, false,
                                            launches);
  if (e != cudaSuccess) return e;
  return launch_bwd_instance<false>(bf16.q, bf16.k, bf16.v, bf16.dout, nlse2, delta, dq, dk, dv,
                                    acc, BH, N, causal, scale, info, err, s, true, launches);
}

}  // namespace swa
