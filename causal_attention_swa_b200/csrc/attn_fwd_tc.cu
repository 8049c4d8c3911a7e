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
// Block = two 128-row query tiles of one head (256 rows) and 640 threads:
//   warps 0-7   softmax for query tile 0, warps 8-15 for query tile 1; in
//               each group, warps 4h + w (w = 0..3) take TMEM lanes
//               32w..32w+31 (rows) and score columns 64h..64h+63, so a row
//               is shared by two threads that agree on its max each tile
//   warp  16    TMA producer: Q0, Q1 once, then K_j, V_j into 4 stages
//   warp  17    MMA issuer for query tile 0 (one elected lane), TMEM owner
//   warp  18    MMA issuer for query tile 1
//   warp  19    idle (gives its registers to the softmax warps of its scheduler)
// Each query tile has an issuer of its own, so neither tile's MMAs queue
// behind the other tile's barriers; each issuer releases a K/V stage on a
// barrier of its own and the producer waits for the issuers that read it.
// Registers: launched at 96 per thread (640 x 96); the softmax warps take
// 104 and warps 16-19 give up to 40, one of them on each scheduler (the
// registers of a warp stay in its scheduler's file).  The launcher checks
// that the kernel was built with exactly 96: a larger claim than the
// scheduler holds would stall setmaxnreg.inc.
// TMEM (512 columns): S0 [0,128) S1 [128,256) P0 [256,320) P1 [320,384)
// O0 [384,448) O1 [448,512).  P_t (bf16, two per column) has columns of its
// own and is the A operand of O_t += P_t V_j straight from TMEM.
// The softmax warps copy S_t,j into registers and release its columns
// (s_free) first, so the MMA warp computes S_t,j+1 while they exponentiate
// S_t,j: the tensor work hides under the softmax instead of alternating
// with it.  Per key tile j the MMA warp issues S_t,j+1 = Q_t K_j+1^T once
// s_free[t] fires and O_t += P_t,j V_j once p_full[t] fires, then commits
// pv_done[t]; the softmax warps wait on pv_done before they rescale O_t or
// overwrite P_t, and store P_t only after computing all of it, by which
// time O_t += P_t,j-1 V_j-1 has long finished.
// Every wait parks the waiting warp (try_wait with a suspend hint), so idle
// roles take no issue slots from the softmax warps that share a scheduler.
// At D = 64 the exponentials bound the kernel: a score costs one MUFU ex2
// (16 per clock per SM) and 4 * 64 MMA flops (about 8000 per clock per SM),
// so ex2 time is about twice the MMA time.  A single warp cannot keep its
// scheduler's MUFU busy (the FMA -> ex2 -> convert chains are too short),
// so every scheduler runs four softmax warps.
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
constexpr int kStages = 4;              // K/V pipeline depth
constexpr int kTileBytes = BM * HD * 2; // 16 KB per bf16 tile
constexpr int kSoftmaxWarps = 16;
constexpr int kThreads = (kSoftmaxWarps + 4) * 32;  // 640: five warps per scheduler
// 16384 registers per scheduler / (5 warps * 32 threads), rounded down to 8
constexpr int kLaunchRegs = 96;
constexpr int kSoftmaxRegs = 104;
constexpr int kOtherRegs = 40;
// Warp w runs on scheduler w % 4 and setmaxnreg moves registers only
// between the warps of one scheduler: each scheduler holds four softmax
// warps and one of warps 16-19, which gives up what the four take.
static_assert(4 * kSoftmaxRegs + kOtherRegs <= 5 * kLaunchRegs, "register split per scheduler");
constexpr int kTmaWarp = kSoftmaxWarps;
constexpr int kMmaWarp = kSoftmaxWarps + 1;  // issuer of tile 0; kMmaWarp + 1 issues tile 1
constexpr int kHalf = BN / 2;                // score columns per softmax thread
constexpr uint32_t kTmemCols = 512;
constexpr float kRescaleThreshold = 8.0f;
constexpr float kFastRange = 64.0f;  // P < 2^64 against a stale max still fits


struct __align__(1024) Smem {
  uint8_t q[2][kTileBytes];
  uint8_t k[kStages][kTileBytes];
  uint8_t v[kStages][kTileBytes];
  uint64_t q_full;
  uint64_t k_full[kStages];
  uint64_t v_full[kStages];
  uint64_t kv_empty[2][kStages];  // per issuer
  uint64_t s_full[2];
  uint64_t s_free[2];
  uint64_t p_full[2];
  uint64_t pv_done[2];
  uint64_t pair[2][4];          // the two threads of a row: tile t, lanes 32w..
  float part[2][2][2][BM];      // [tile][parity][half][row]: partial row max / sum
  uint64_t drain[2];
  uint32_t tmem_base;
  int abort;
};

constexpr size_t kSmemBytes = sizeof(Smem) + 1024;

__device__ __forceinline__ uint32_t col_s(int t) { return t ? 128u : 0u; }
__device__ __forceinline__ uint32_t col_p(int t) { return t ? 320u : 256u; }
__device__ __forceinline__ uint32_t col_o(int t) { return t ? 448u : 384u; }

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
      mbar_init(&sm.kv_empty[0][s], 1);
      mbar_init(&sm.kv_empty[1][s], 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(&sm.s_full[t], 1);
      mbar_init(&sm.s_free[t], 256);
      mbar_init(&sm.p_full[t], 256);
      mbar_init(&sm.pv_done[t], 1);
      for (int w = 0; w < 4; ++w) mbar_init(&sm.pair[t][w], 64);
    }
    mbar_init(&sm.drain[0], 1);
    mbar_init(&sm.drain[1], 1);
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

  if (warp >= kSoftmaxWarps) regs_decrease<kOtherRegs>();

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
        // the stage held tile j - kStages: wait for each issuer that read it
        bool ok = true;
        for (int t = 0; t < 2 && ok && round > 0; ++t)
          if (j - kStages < n_t[t])
            ok = mbar_wait_parked(&sm.kv_empty[t][s], (round - 1) & 1, abort, err,
                                  kDevTimeoutEmpty);
        if (!ok) break;
        mbar_arrive_expect_tx(&sm.k_full[s], kTileBytes);
        tma_load_3d(sm.k[s], &tm_k, &sm.k_full[s], 0, j * BN, head);
        mbar_arrive_expect_tx(&sm.v_full[s], kTileBytes);
        tma_load_3d(sm.v[s], &tm_v, &sm.v_full[s], 0, j * BN, head);
      }
    }
    __syncwarp();
  } else if (warp == kMmaWarp || warp == kMmaWarp + 1) {
    // ------------------------------------------------ MMA issuer of tile t
    {  // the whole warp runs the issue loop; one elected lane issues
      const int t = warp - kMmaWarp;
      constexpr uint32_t idesc_s = idesc_bf16_f32(BM, BN, 0, 0);  // Q, K both K-major
      constexpr uint32_t idesc_o = idesc_bf16_f32(BM, HD, 0, 1);  // V is MN-major (dims contiguous)
      const uint64_t q_desc = desc_sw128(smem_u32(sm.q[t]), 16, 1024);
      auto issue_s = [&](int j) {
        // one asm block of 4 MMAs; K steps of 32 B = 2 descriptor units
        mma_ss_run<4, 2, 0, 2>(tmem + col_s(t), q_desc,
                               desc_sw128(smem_u32(sm.k[j % kStages]), 16, 1024), idesc_s, 0u);
        mma_commit_elect(&sm.s_full[t]);
      };
      auto issue_pv = [&](int j) {
        // 8 MMAs: P columns 8k, V rows 16k (+2048 B = 128 units)
        mma_ts_run8<128, 8, 16, 24, 32, 40, 48, 56>(
            tmem + col_o(t), tmem + col_p(t), desc_sw128(smem_u32(sm.v[j % kStages]), 8192, 1024),
            idesc_o, j > 0 ? 1u : 0u);
        mma_commit_elect(&sm.pv_done[t]);
        mma_commit_elect(&sm.kv_empty[t][j % kStages]);
      };
      auto wait_k = [&](int j) {
        return mbar_wait_parked(&sm.k_full[j % kStages], (j / kStages) & 1, abort, err,
                                kDevTimeoutFull);
      };
      bool ok = n_t[t] > 0 && mbar_wait_parked(&sm.q_full, 0, abort, err, kDevTimeoutFull) &&
                wait_k(0);
      if (ok) {
        fence_after_sync();
        issue_s(0);
      }
      for (int j = 0; ok && j < n_t[t]; ++j) {
        // S_t,j+1 as soon as the softmax warps hold S_t,j in registers
        if (j + 1 < n_t[t]) {
          if (!mbar_wait_parked(&sm.s_free[t], j & 1, abort, err, kDevTimeoutOther) ||
              !wait_k(j + 1))
            break;
          fence_after_sync();
          issue_s(j + 1);
        }
        if (!mbar_wait_parked(&sm.v_full[j % kStages], (j / kStages) & 1, abort, err,
                              kDevTimeoutFull) ||
            !mbar_wait_parked(&sm.p_full[t], j & 1, abort, err, kDevTimeoutOther))
          break;
        fence_after_sync();
        issue_pv(j);
      }
      // every MMA this warp issued has finished before TMEM is released
      mma_commit_elect(&sm.drain[t]);
      wait_unbounded_by_abort(&sm.drain[t], 0);
    }
    __syncwarp();
  } else if (warp < kSoftmaxWarps) {
    // ------------------------------------------------------------ softmax
    regs_increase<kSoftmaxRegs>();
    const int t = warp >> 3;        // query tile
    const int h = (warp >> 2) & 1;  // score columns 64h..64h+63
    const int wt = warp & 3;        // TMEM lanes 32wt..32wt+31
    const int r = wt * 32 + lane;
    const int g = 2 * c + t;
    const int row = g * BM + r;
    const uint32_t lane_off = static_cast<uint32_t>(wt * 32) << 16;
    const uint32_t tS = tmem + lane_off + col_s(t) + kHalf * h;
    const uint32_t tP = tmem + lane_off + col_p(t) + (kHalf / 2) * h;
    const uint32_t tO = tmem + lane_off + col_o(t) + (HD / 2) * h;
    uint64_t* pair = &sm.pair[t][wt];
    int pair_phase = 0;
    // publish v for the row, wait for the partner thread's value
    auto exchange = [&](float v, float& other) -> bool {
      const int slot = pair_phase & 1;
      sm.part[t][slot][h][r] = v;
      mbar_arrive(pair);
      if (!mbar_wait_parked(pair, pair_phase & 1, abort, err, kDevTimeoutOther)) return false;
      other = sm.part[t][slot][h ^ 1][r];
      ++pair_phase;
      return true;
    };
    float m_used = -INFINITY;  // reference max (log2 domain), the same in both
                               // threads of the row
    float l = 0.f;             // this thread's share of the row sum
    bool ok = true;
    bool s_ready = false;  // S_t,j already seen complete by the probe of tile j-1
    for (int j = 0; j < n_t[t]; ++j) {
      if (!s_ready && !mbar_wait_parked(&sm.s_full[t], j & 1, abort, err, kDevTimeoutMma)) {
        ok = false;
        break;
      }
      fence_after_sync();
      float x[kHalf];
      {
        uint32_t u[kHalf / 16][16];
#pragma unroll
        for (int i = 0; i < kHalf / 16; ++i) tmem_ld16(tS + i * 16, u[i]);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < kHalf / 16; ++i)
#pragma unroll
          for (int e = 0; e < 16; ++e) x[i * 16 + e] = __uint_as_float(u[i][e]);
      }
      fence_before_sync();
      mbar_arrive(&sm.s_free[t]);  // S_t,j is in registers: its columns may take S_t,j+1
      const bool need_mask = (j * BN + BN > N) || (causal && j == g);
      if (need_mask) {
#pragma unroll
        for (int e = 0; e < kHalf; ++e) {
          const int key = j * BN + kHalf * h + e;
          if (key >= N || (causal && key > row)) x[e] = -INFINITY;
        }
      }
      // 8 chains of three-input maxima over this thread's 64 scores
      float mxp[8];
#pragma unroll
      for (int a = 0; a < 8; ++a) mxp[a] = fmax3(x[a], x[a + 8], x[a + 16]);
#pragma unroll
      for (int a = 0; a < 8; ++a) mxp[a] = fmax3(mxp[a], x[a + 24], x[a + 32]);
#pragma unroll
      for (int a = 0; a < 8; ++a) mxp[a] = fmax3(mxp[a], x[a + 40], x[a + 48]);
#pragma unroll
      for (int a = 0; a < 8; ++a) mxp[a] = fmaxf(mxp[a], x[a + 56]);
      const float mine = fmaxf(fmax3(mxp[0], mxp[1], mxp[2]),
                               fmax3(fmax3(mxp[3], mxp[4], mxp[5]), mxp[6], mxp[7]));
      // Publish this thread's max now, read the partner's when it is needed:
      // before the ex2 loop only if a score of this thread could lie far
      // above m_used (the first tile, a jump of more than kFastRange, a
      // NaN); else after it, when the partner has long published.  Both
      // threads derive the same m_new from (m_used, both maxima); a P
      // computed against m_used is then moved to m_new (rare: the partner
      // raised the max by more than the lazy threshold) by one rounding.
      const float mine_l2 = mine * scale_log2;  // scale_log2 > 0 commutes with the max
      const int slot = pair_phase & 1;
      const uint32_t par = static_cast<uint32_t>(pair_phase & 1);
      ++pair_phase;
      sm.part[t][slot][h][r] = mine_l2;
      mbar_arrive(pair);
      float m_new = m_used;
      bool pair_seen = false;  // set by an earlier successful probe
      auto fetch_and_decide = [&]() -> bool {
        if (!pair_seen && !mbar_wait_parked(pair, par, abort, err, kDevTimeoutOther))
          return false;
        const float theirs = sm.part[t][slot][h ^ 1][r];
        // the same operand order in both threads of the row
        const float cand = h == 0 ? fmaxf(mine_l2, theirs) : fmaxf(theirs, mine_l2);
        const float mc = fmaxf(m_used, cand);
        if (j == 0 || mc > m_used + kRescaleThreshold) m_new = mc;
        return true;
      };
      const bool early = __any_sync(0xffffffffu, j == 0 || !(mine_l2 <= m_used + kFastRange));
      if (early && !fetch_and_decide()) { ok = false; break; }
      const float m_exp = m_new;  // the reference the ex2 loop uses
      // O_t += P_t,j-1 V_j-1 (issued at the end of the last tile) is probed
      // now and waited for, if still needed, only after the ex2 loop
      const bool pv_ready = j == 0 || mbar_test_wait(&sm.pv_done[t], (j - 1) & 1);
      float2 rsp[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
      const float2 sc2 = make_float2(scale_log2, scale_log2);
      const float2 nm2 = make_float2(-m_exp, -m_exp);
      uint32_t pk[kHalf / 32][16];
      auto exps = [&](int i) {
#pragma unroll
        for (int e = 16 * i; e < 16 * i + 16; ++e) {
          const float2 a = __ffma2_rn(make_float2(x[2 * e], x[2 * e + 1]), sc2, nm2);
          const float2 pe = make_float2(ex2(a.x), ex2(a.y));
          rsp[e & 1] = __fadd2_rn(rsp[e & 1], pe);
          pk[i][e & 15] = pack_bf16(pe.x, pe.y);
        }
      };
      exps(0);
      // the partner published with this thread: probe between the halves
      if (!early) pair_seen = mbar_test_wait(pair, par);
      exps(1);
      if (!early && !fetch_and_decide()) { ok = false; break; }
      if (__any_sync(0xffffffffu, m_exp != m_new)) {  // rare: the partner moved the max
        const float beta = ex2(m_exp - m_new);
#pragma unroll
        for (int i = 0; i < kHalf / 32; ++i)
#pragma unroll
          for (int e = 0; e < 16; ++e)
            pk[i][e] = pack_bf16(bf16lo(pk[i][e]) * beta, bf16hi(pk[i][e]) * beta);
        rsp[0].x *= beta; rsp[0].y *= beta; rsp[1].x *= beta; rsp[1].y *= beta;
      }
      // O_t += P_t,j-1 V_j-1 must finish before O_t is rescaled or P_t is
      // overwritten: by now it normally has.
      if (j > 0) {
        if (!pv_ready &&
            !mbar_wait_parked(&sm.pv_done[t], (j - 1) & 1, abort, err, kDevTimeoutMma)) {
          ok = false;
          break;
        }
        fence_after_sync();
        if (__any_sync(0xffffffffu, m_new != m_used)) {
          const float alpha = ex2(m_used - m_new);
#pragma unroll
          for (int i = 0; i < HD / 32; ++i) {
            uint32_t u[16];
            tmem_ld16(tO + i * 16, u);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 16; ++e) u[e] = __float_as_uint(__uint_as_float(u[e]) * alpha);
            tmem_st16(tO + i * 16, u);
          }
          l *= alpha;
        }
      }
      m_used = m_new;
#pragma unroll
      for (int i = 0; i < kHalf / 32; ++i) tmem_st16(tP + i * 16, pk[i]);
      // S_t,j+1 was issued early in this tile: probe it while the stores land
      s_ready = j + 1 < n_t[t] && mbar_test_wait(&sm.s_full[t], (j + 1) & 1);
      tmem_wait_st();
      fence_before_sync();
      mbar_arrive(&sm.p_full[t]);
      l += (rsp[0].x + rsp[0].y) + (rsp[1].x + rsp[1].y);
    }
    float l_other = 0.f;
    if (ok && n_t[t] > 0 && exchange(l, l_other) &&
        mbar_wait_parked(&sm.pv_done[t], (n_t[t] - 1) & 1, abort, err, kDevTimeoutMma)) {
      fence_after_sync();
      const float inv = 1.f / (h == 0 ? l + l_other : l_other + l);
      uint32_t packed[HD / 4];
#pragma unroll
      for (int i = 0; i < HD / 32; ++i) {
        uint32_t u[16];
        tmem_ld16(tO + i * 16, u);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 8; ++e)
          packed[i * 8 + e] = pack_bf16(__uint_as_float(u[2 * e]) * inv,
                                        __uint_as_float(u[2 * e + 1]) * inv);
      }
      if (row < N) {
        uint4* dst = reinterpret_cast<uint4*>(out + ((size_t)head * N + row) * HD + (HD / 2) * h);
#pragma unroll
        for (int i = 0; i < HD / 16; ++i)
          dst[i] = make_uint4(packed[4 * i], packed[4 * i + 1], packed[4 * i + 2],
                              packed[4 * i + 3]);
        if (h == 0) lse[(size_t)head * N + row] = (m_used + __log2f(l + l_other)) * kLn2;
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
  // looked up once; the initialisation of a function-local static is thread-safe
  static const PFN_cuTensorMapEncodeTiled_v12000 fn = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    return cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                       cudaSuccess && q == cudaDriverEntryPointSuccess
               ? reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p)
               : nullptr;
  }();
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
  cudaFuncAttributes fa;
  e = cudaFuncGetAttributes(&fa, attn_fwd_tc_kernel);
  if (e != cudaSuccess) return e;
  if (fa.numRegs != kLaunchRegs) return cudaErrorInvalidKernelImage;  // register split unsafe
  const int n_ctiles = (int)((N + 2 * BM - 1) / (2 * BM));
  const int64_t grid = (int64_t)n_ctiles * BH;
  attn_fwd_tc_kernel<<<(unsigned)grid, kThreads, kSmemBytes, s>>>(
      tq, tk, tv, static_cast<__nv_bfloat16*>(out), lse, (int)N, (int)BH, n_ctiles, causal,
      scale * kLog2e, flags, err);
  *launches += 1;
  return cudaGetLastError();
}

}  // namespace swa
