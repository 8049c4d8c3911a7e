// attn_fwd_tc.cu -- causal / non-causal attention forward on the sm_100a
// tensor cores (tcgen05.mma kind::f16: bf16 Q K^T, f16 or bf16 P V; f32
// accumulators in TMEM; TMA-staged K/V).
//
// The method: "Show HN: Automatic deduction of FlashAttention kernel from
// ~25 lines of SQL" (page 2, the demo's docstring): FlashAttention streams
// blocks of keys past blocks of queries under a running softmax, so the
// N x N scores are never stored; the math is the view ATTENTION_WINDOW
// (scores = q.k/8 over the pairs with q.t >= k.t, w = exp(s - row max),
// out = sum w/z v).
//
// Block = two 128-row query tiles of one head (256 rows) and 384 threads:
//   warps 0-3   softmax for query tile 0, warps 4-7 for query tile 1; warp w
//               takes TMEM lanes 32(w%4)..+31, one row per thread, all 128
//               score columns of the key tile
//   warp  8     TMA producer: Q0, Q1 once, then K_j, V_j into 4 stages
//   warp  9     MMA issuer for query tile 0 (one elected lane), TMEM owner
//   warp  10    MMA issuer for query tile 1
//   warp  11    V cleaner (heads whose V holds an infinity or NaN): rewrites
//               each staged V tile in place (a non-finite entry -> 0, its row
//               recorded), then releases it to the issuers; it also gives its
//               registers to the softmax warps of its scheduler
// Each query tile has an issuer of its own, so neither tile's MMAs queue
// behind the other tile's barriers; each issuer releases a K/V stage on a
// barrier of its own and the producer waits for the issuers that read it.
// Registers: launched at 168 per thread (384 x 168); the softmax warps take
// 232 and warps 8-11 give up to 40, one of them on each scheduler (the
// registers of a warp stay in its scheduler's file).  The launcher checks
// that the kernel was built with exactly 168: a larger claim than the
// scheduler holds would stall setmaxnreg.inc.
// TMEM (512 columns): S0 [0,128) S1 [128,256) P0 [256,320) P1 [320,384)
// O0 [384,448) O1 [448,512).  P_t (16-bit, two per column) has columns of
// its own and is the A operand of O_t += P_t V_j straight from TMEM.
// The softmax warps copy S_t,j into registers and release its columns
// (s_free) first, so the MMA warp computes S_t,j+1 while they exponentiate
// S_t,j: the tensor work hides under the softmax instead of alternating
// with it.  Per key tile j the MMA warp issues S_t,j+1 = Q_t K_j+1^T once
// s_free[t] fires and O_t += P_t,j V_j once p_full[t] fires, then commits
// pv_done[t]; the softmax warps wait on pv_done before they rescale O_t or
// overwrite P_t, and store P_t only after computing all of it, by which
// time O_t += P_t,j-1 V_j-1 has long finished.
// Every wait polls its barrier (try_wait without a suspend hint): a parked
// warp wakes late enough to cost the forward about 2%, and the polls of the
// idle roles did not slow the softmax warps that share their schedulers.
// At D = 64 the exponentials bound the kernel: a score costs one MUFU ex2
// (16 per clock per SM) and 4 * 64 MMA flops (about 8000 per clock per SM),
// so ex2 time is about twice the MMA time.  A warp whose ex2 loop runs over
// 128 independent scores keeps its scheduler's MUFU ~88% busy alone (~99%
// with the second softmax warp), so one thread per row suffices; it also
// needs no exchange of partial row maxima between threads.
// Online softmax in the log2 domain with a lazy rescale: the reference max
// of a row moves (and O, l are rescaled) only when the new row max exceeds
// it by more than 8, so P <= 2^8 (exact after the final division by l).
// Precision of O += P V: P enters the MMA as f16 (10 fraction bits) with V
// read from an f16 copy of V (the caller's prep pass writes it), for every
// head whose finite V values lie below 2^15 in magnitude (f16 holds them
// exactly, up to f16's subnormal spacing of 2^-24); a head with larger
// values keeps both in bf16 (V as given).  A bf16 P (7 fraction bits) is
// exact enough for the output itself, but the output is what the gradient
// of loss = 1/2 sum out^2 feeds back as dout, and the rounding of few-key
// rows (early rows) reaches the gradient amplified by the cancellation in
// sum_j dS_ij k_j; with the f16 P the end-to-end gradient stays inside the
// bf16 path's tolerance.  Rows
// that see few keys (the first rows of a causal head) average no rounding
// away, so on the diagonal tile -- the last key tile of every causal query
// tile -- P also enters as the sum of two 16-bit words: its rounding
// residual goes into that tile's S columns (free then: no later S is
// computed for the query tile) and a second P V product adds it.  The
// kernel is instantiated for both operand types; each launch takes the
// heads of its type (the per-head scan of V decides).
// For the gradient of loss = 1/2 sum out^2 (dout = out) the epilogue can
// also write what the backward reads: an f16 copy of the float32 output,
// delta_i = sum_d out_id^2 in float32, and -lse_i log2 e, the last two
// padded to whole 128-row blocks.
// Causal: key tiles past the diagonal are never loaded; inside the
// diagonal tile (and past N on a ragged tail) a masked score is replaced by
// -inf before the max, so its weight is exactly 0.
// Non-finite V (absent rows: a masked pair must never enter a product,
// "check_masks_are_absent_rows"): a masked weight of a diagonal tile meets
// the V rows of keys after the query, and 0 * inf would be NaN.  For a head
// whose V holds an infinity or NaN (the scan's flag) the cleaner warp
// replaces every non-finite V entry by 0 before the MMA reads the tile and
// records, per column d, the first key row holding +inf, -inf and NaN; the
// epilogue then sets out[i, d] to the IEEE class that the sum over the
// existing pairs j in J(i) takes (every existing weight is > 0): NaN if a
// NaN, or both infinities, lie in rows J(i), else the infinity that does,
// else the finite value computed from the sanitised V.
// Every mbarrier wait is bounded; on expiry the block records an error code
// in the device error word, all roles leave their loops, and TMEM is freed.
#include <cudaTypedefs.h>

#include <climits>

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
constexpr int kSoftmaxWarps = 8;
constexpr int kThreads = (kSoftmaxWarps + 4) * 32;  // 384: three warps per scheduler
// 16384 registers per scheduler / (3 warps * 32 threads), rounded down to 8
constexpr int kLaunchRegs = 168;
// A softmax thread holds its row's 128 scores plus the loop's state.  The
// other warps (TMA, MMA issue, the V cleaner) fit in 40.
constexpr int kSoftmaxRegs = 232;
constexpr int kOtherRegs = 40;
// Warp w runs on scheduler w % 4 and setmaxnreg moves registers only
// between the warps of one scheduler: each scheduler holds two softmax
// warps (one per query tile) and one of warps 8-11, which gives up what the
// two take.
static_assert(2 * kSoftmaxRegs + kOtherRegs <= 3 * kLaunchRegs, "register split per scheduler");
constexpr int kTmaWarp = kSoftmaxWarps;
constexpr int kMmaWarp = kSoftmaxWarps + 1;  // issuer of tile 0; kMmaWarp + 1 issues tile 1
constexpr uint32_t kTmemCols = 512;
constexpr float kRescaleThreshold = 8.0f;
constexpr int kCleanWarp = kSoftmaxWarps + 3;  // warp 11
// Per-head information (kHeadInfoInts int32 per head): bit 0 of [0] is set if
// V holds an infinity or NaN, [1] is the largest biased exponent of its
// finite values.  f16 operands are used when that exponent is below 2^15's.
constexpr int kF16ExpLimit = 127 + 15;


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
  uint64_t v_ready[kStages];    // the cleaner has rewritten the stage's V tile
  uint64_t cls_done;            // the cleaner has recorded every tile's classes
  int first_cls[3][HD];         // per column: first key row with +inf, -inf, NaN
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

// The V cleaner's unit: one 16-byte chunk c (row c / 8 of the staged tile,
// 128-byte swizzle) of a head whose V holds an infinity or NaN.  A
// non-finite 16-bit entry (f16 in the f16 instance, bf16 in the other)
// becomes 0 and its key row goes into first_cls (per column: first row with
// +inf, -inf, NaN).
template <bool kF16>
__device__ __forceinline__ void clean_v_chunk(uint4* base, int c, int key0,
                                              int (*first_cls)[HD]) {
  constexpr uint32_t kExp = kF16 ? 0x7C00u : 0x7F80u;   // exponent field all ones
  constexpr uint32_t kMan = kF16 ? 0x03FFu : 0x007Fu;   // fraction: non-zero = NaN
  const uint4 x = base[c];
  uint32_t w[4] = {x.x, x.y, x.z, x.w};
  bool any = false;
#pragma unroll
  for (int e = 0; e < 4; ++e)
    any |= ((w[e] & kExp) == kExp) | (((w[e] >> 16) & kExp) == kExp);
  if (!any) return;
  const int r = c >> 3;                      // row of the tile
  const int d0 = ((c & 7) ^ (r & 7)) * 8;    // its first column (swizzle undone)
#pragma unroll
  for (int e = 0; e < 4; ++e)
#pragma unroll
    for (int p = 0; p < 2; ++p) {
      const uint32_t b = (w[e] >> (16 * p)) & 0xFFFFu;
      if ((b & kExp) == kExp) {
        const int cls = (b & kMan) ? 2 : ((b & 0x8000u) ? 1 : 0);
        atomicMin(&first_cls[cls][d0 + 2 * e + p], key0 + r);
        w[e] &= ~(0xFFFFu << (16 * p));
      }
    }
  base[c] = make_uint4(w[0], w[1], w[2], w[3]);
}

// Cleans one staged V tile (128 rows of 128 bytes).  With the prep pass's
// row mask of the tile (rows holding a non-finite entry) only those rows are
// read, 8 lanes per row; without it, every chunk.
template <bool kF16>
__device__ __forceinline__ void clean_v_tile(uint8_t* tile, int lane, int key0,
                                             const uint4* rowmask, int (*first_cls)[HD]) {
  uint4* base = reinterpret_cast<uint4*>(tile);
  if (rowmask != nullptr) {
    const uint4 m4 = *rowmask;
    const uint32_t words[4] = {m4.x, m4.y, m4.z, m4.w};
#pragma unroll 1
    for (int wd = 0; wd < 4; ++wd)
      for (uint32_t m = words[wd]; m != 0u; m &= m - 1u) {  // warp-uniform
        const int r = 32 * wd + (__ffs(m) - 1);
        if (lane < 8) clean_v_chunk<kF16>(base, r * 8 + lane, key0, first_cls);
      }
    return;
  }
#pragma unroll 2
  for (int c = lane; c < kTileBytes / 16; c += 32) clean_v_chunk<kF16>(base, c, key0, first_cls);
}

template <bool kF16>
__global__ void __launch_bounds__(kThreads, 1)
attn_fwd_tc_kernel(const __grid_constant__ CUtensorMap tm_q,
                   const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, __nv_bfloat16* __restrict__ out,
                   float* __restrict__ lse, int N, int BH, int n_ctiles, int head_group,
                   int causal,
                   float scale_log2, const int* __restrict__ vinfo,
                   const uint4* __restrict__ vrows, int all_bf16,
                   uint16_t* __restrict__ do16, float* __restrict__ delta,
                   float* __restrict__ nlse2, unsigned* __restrict__ err) {
  pdl_prologue();  // the other instance's launch overlaps this one's tail
  // Heads in groups of head_group (head_group() on the host), whose K and V
  // stay in L2 while the group's blocks run; inside a group the heaviest
  // (latest) query tiles first, heads interleaved.
  const int group = blockIdx.x / (head_group * n_ctiles);
  const int g_heads = min(head_group, BH - group * head_group);
  const int rr = blockIdx.x - group * head_group * n_ctiles;
  const int head = group * head_group + rr % g_heads;
  const int c = n_ctiles - 1 - rr / g_heads;
  const bool nonfinite = (vinfo[kHeadInfoInts * head] & 1) != 0;
  const bool f16_head = !all_bf16 && vinfo[kHeadInfoInts * head + 1] < kF16ExpLimit;
  if (f16_head != kF16) return;  // the other instance's head
  // the cleaner rewrites the V tiles of a head with non-finite values
  const bool convert = nonfinite;

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
      mbar_init(&sm.s_free[t], kSoftmaxWarps / 2);  // one arrival per softmax warp of tile t
      mbar_init(&sm.p_full[t], kSoftmaxWarps / 2);
      mbar_init(&sm.pv_done[t], 1);
    }
    mbar_init(&sm.drain[0], 1);
    mbar_init(&sm.drain[1], 1);
    for (int s = 0; s < kStages; ++s) mbar_init(&sm.v_ready[s], 1);
    mbar_init(&sm.cls_done, 1);
    sm.abort = 0;
    fence_mbar_init();
  }
  if (tid < 3 * HD) (&sm.first_cls[0][0])[tid] = INT_MAX;
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
            ok = mbar_wait_spin(&sm.kv_empty[t][s], (round - 1) & 1, abort, err,
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
      // V is MN-major (dims contiguous); P and V are f16 or bf16 together
      constexpr uint32_t idesc_o = kF16 ? idesc_f16_f32(BM, HD, 0, 1) : idesc_bf16_f32(BM, HD, 0, 1);
      const uint64_t q_desc = desc_sw128(smem_u32(sm.q[t]), 16, 1024);
      auto issue_s = [&](int j) {
        // one asm block of 4 MMAs; K steps of 32 B = 2 descriptor units
        mma_ss_run<4, 2, 0, 2>(tmem + col_s(t), q_desc,
                               desc_sw128(smem_u32(sm.k[j % kStages]), 16, 1024), idesc_s, 0u);
        mma_commit_elect(&sm.s_full[t]);
      };
      auto issue_pv = [&](int j) {
        const uint64_t v_desc = desc_sw128(smem_u32(sm.v[j % kStages]), 8192, 1024);
        // 8 MMAs: P columns 8k, V rows 16k (+2048 B = 128 units)
        mma_ts_run8<128, 8, 16, 24, 32, 40, 48, 56>(tmem + col_o(t), tmem + col_p(t), v_desc,
                                                    idesc_o, j > 0 ? 1u : 0u);
        if (causal && j == n_t[t] - 1)  // the diagonal tile: + P's residual (in S's columns)
          mma_ts_run8<128, 8, 16, 24, 32, 40, 48, 56>(tmem + col_o(t), tmem + col_s(t), v_desc,
                                                      idesc_o, 1u);
        mma_commit_elect(&sm.pv_done[t]);
        mma_commit_elect(&sm.kv_empty[t][j % kStages]);
      };
      auto wait_k = [&](int j) {
        return mbar_wait_spin(&sm.k_full[j % kStages], (j / kStages) & 1, abort, err,
                              kDevTimeoutFull);
      };
      bool ok = n_t[t] > 0 && mbar_wait_spin(&sm.q_full, 0, abort, err, kDevTimeoutFull) &&
                wait_k(0);
      if (ok) {
        fence_after_sync();
        issue_s(0);
      }
      for (int j = 0; ok && j < n_t[t]; ++j) {
        // S_t,j+1 as soon as the softmax warps hold S_t,j in registers
        if (j + 1 < n_t[t]) {
          if (!mbar_wait_spin(&sm.s_free[t], j & 1, abort, err, kDevTimeoutOther) ||
              !wait_k(j + 1))
            break;
          fence_after_sync();
          issue_s(j + 1);
        }
        if (!mbar_wait_spin(convert ? &sm.v_ready[j % kStages] : &sm.v_full[j % kStages],
                            (j / kStages) & 1, abort, err, kDevTimeoutFull) ||
            !mbar_wait_spin(&sm.p_full[t], j & 1, abort, err, kDevTimeoutOther))
          break;
        fence_after_sync();
        issue_pv(j);
      }
      // every MMA this warp issued has finished before TMEM is released
      mma_commit_elect(&sm.drain[t]);
      wait_unbounded_by_abort(&sm.drain[t], 0);
    }
    __syncwarp();
  } else if (warp == kCleanWarp) {
    // ------------------------------------------------------------ cleaner
    if (convert) {
      for (int j = 0; j < n_kv; ++j) {
        const int s = j % kStages;
        if (!mbar_wait_spin(&sm.v_full[s], (j / kStages) & 1, abort, err, kDevTimeoutFull))
          break;
        const uint4* rowmask =
            vrows != nullptr ? vrows + (size_t)head * ((N + BN - 1) / BN) + j : nullptr;
        clean_v_tile<kF16>(sm.v[s], lane, j * BN, rowmask, sm.first_cls);
        fence_proxy_async_smem();  // the MMA (async proxy) reads what was written
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.v_ready[s]);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.cls_done);
    }
    __syncwarp();
  } else if (warp < kSoftmaxWarps) {
    // ------------------------------------------------------------ softmax
    regs_increase<kSoftmaxRegs>();
    const int t = warp >> 2;   // query tile
    const int wt = warp & 3;   // TMEM lanes 32wt..32wt+31 (the warp's subpartition)
    const int r = wt * 32 + lane;
    const int g = 2 * c + t;
    const int row = g * BM + r;
    const uint32_t lane_off = static_cast<uint32_t>(wt * 32) << 16;
    const uint32_t tS = tmem + lane_off + col_s(t);
    const uint32_t tP = tmem + lane_off + col_p(t);
    const uint32_t tO = tmem + lane_off + col_o(t);
    float m_used = -INFINITY;  // reference max of the row (log2 domain)
    float l = 0.f;             // row sum against m_used
    bool ok = true;
    bool s_ready = false;  // S_t,j already seen complete by the probe of tile j-1
    const float2 sc2 = make_float2(scale_log2, scale_log2);
    for (int j = 0; j < n_t[t]; ++j) {
      if (!s_ready && !mbar_wait_spin(&sm.s_full[t], j & 1, abort, err, kDevTimeoutMma)) {
        ok = false;
        break;
      }
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
          for (int e = 0; e < 16; ++e) x[i * 16 + e] = __uint_as_float(u[i][e]);
      }
      fence_before_sync();
      warp_arrive(&sm.s_free[t]);  // S_t,j is in registers: its columns may take S_t,j+1
      const bool need_mask = (j * BN + BN > N) || (causal && j == g);
      if (need_mask) {
#pragma unroll
        for (int e = 0; e < BN; ++e) {
          const int key = j * BN + e;
          if (key >= N || (causal && key > row)) x[e] = -INFINITY;
        }
      }
      // 16 chains of three-input maxima over the row's 128 scores
      float mxp[16];
#pragma unroll
      for (int a = 0; a < 16; ++a) mxp[a] = fmax3(x[a], x[a + 16], x[a + 32]);
#pragma unroll
      for (int a = 0; a < 16; ++a) mxp[a] = fmax3(mxp[a], x[a + 48], x[a + 64]);
#pragma unroll
      for (int a = 0; a < 16; ++a) mxp[a] = fmax3(mxp[a], x[a + 80], x[a + 96]);
#pragma unroll
      for (int a = 0; a < 16; ++a) mxp[a] = fmaxf(mxp[a], x[a + 112]);
#pragma unroll
      for (int a = 0; a < 5; ++a) mxp[a] = fmax3(mxp[3 * a], mxp[3 * a + 1], mxp[3 * a + 2]);
      const float mine = fmax3(fmax3(mxp[0], mxp[1], mxp[2]), fmaxf(mxp[3], mxp[4]), mxp[15]);
      // Lazy rescale: the reference moves only when the row max exceeds it
      // by more than kRescaleThreshold (always on the first tile), so every
      // P = 2^(s - m_used) <= 2^8.
      const float mc = fmaxf(m_used, mine * scale_log2);  // scale_log2 > 0 commutes with max
      const float m_new = (j == 0 || mc > m_used + kRescaleThreshold) ? mc : m_used;
      // O_t += P_t,j-1 V_j-1 (issued at the end of the last tile) reads P_t:
      // probed now, waited for (if still needed) after the ex2 loop
      const bool pv_ready = j == 0 || mbar_test_wait(&sm.pv_done[t], (j - 1) & 1);
      const float2 nm2 = make_float2(-m_new, -m_new);
      float2 rsp[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
      uint32_t pk[BN / 32][16];
#pragma unroll
      for (int e = 0; e < BN / 2; ++e) {
        const float2 a = __ffma2_rn(make_float2(x[2 * e], x[2 * e + 1]), sc2, nm2);
        const float2 pe = make_float2(ex2(a.x), ex2(a.y));
        rsp[e & 1] = __fadd2_rn(rsp[e & 1], pe);
        pk[e >> 4][e & 15] = pack_p<kF16>(pe.x, pe.y);
      }
      if (j > 0) {
        if (!pv_ready &&
            !mbar_wait_spin(&sm.pv_done[t], (j - 1) & 1, abort, err, kDevTimeoutMma)) {
          ok = false;
          break;
        }
        fence_after_sync();
        // O_t is complete: move it to the new reference (rare)
        if (__any_sync(0xffffffffu, m_new != m_used)) {
          const float alpha = ex2(m_used - m_new);  // 1 in rows whose reference stays
#pragma unroll 1
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
      }
      m_used = m_new;
#pragma unroll
      for (int i = 0; i < BN / 32; ++i) tmem_st16(tP + i * 16, pk[i]);
      if (causal && j == n_t[t] - 1) {
        // the diagonal tile: P's rounding residual P - hi(P), 16 keys per 8
        // columns, over the row's own S columns (each chunk is read before
        // it is written); a second P V product adds it
#pragma unroll 1
        for (int cidx = 0; cidx < BN / 16; ++cidx) {
          uint32_t u[16];
          tmem_ld16(tS + 16 * cidx, u);
          tmem_wait_ld();
          uint32_t lo[8];
#pragma unroll
          for (int e2 = 0; e2 < 8; ++e2) {
            float2 sv = make_float2(__uint_as_float(u[2 * e2]), __uint_as_float(u[2 * e2 + 1]));
            const int key = j * BN + 16 * cidx + 2 * e2;
            if (key >= N || key > row) sv.x = -INFINITY;
            if (key + 1 >= N || key + 1 > row) sv.y = -INFINITY;
            const float2 a = __ffma2_rn(sv, sc2, nm2);
            const float2 pe = make_float2(ex2(a.x), ex2(a.y));
            const uint32_t hi = pack_p<kF16>(pe.x, pe.y);
            lo[e2] = pack_p<kF16>(pe.x - unpack_lo<kF16>(hi), pe.y - unpack_hi<kF16>(hi));
          }
          tmem_st8(tS + 8 * cidx, lo);
        }
      }
      // S_t,j+1 was issued early in this tile: probe it while the stores land
      s_ready = j + 1 < n_t[t] && mbar_test_wait(&sm.s_full[t], (j + 1) & 1);
      tmem_wait_st();
      fence_before_sync();
      warp_arrive(&sm.p_full[t]);
      l += (rsp[0].x + rsp[0].y) + (rsp[1].x + rsp[1].y);
    }
    if (ok && n_t[t] > 0 &&
        mbar_wait_spin(&sm.pv_done[t], (n_t[t] - 1) & 1, abort, err, kDevTimeoutMma)) {
      fence_after_sync();
      const float inv = 1.f / l;
      float o[HD];  // out_row, float32
#pragma unroll
      for (int i = 0; i < HD / 16; ++i) {
        uint32_t u[16];
        tmem_ld16(tO + i * 16, u);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 16; ++e) o[i * 16 + e] = __uint_as_float(u[e]) * inv;
      }
      if (nonfinite && mbar_wait_spin(&sm.cls_done, 0, abort, err, kDevTimeoutOther)) {
        // IEEE class of sum_{j in J(row)} P_ij v_jd with every P_ij > 0
        const int last = causal ? row : N - 1;
#pragma unroll
        for (int d = 0; d < HD; ++d) {
          const bool pinf = sm.first_cls[0][d] <= last, ninf = sm.first_cls[1][d] <= last;
          const bool nan = sm.first_cls[2][d] <= last || (pinf && ninf);
          if (nan) o[d] = __uint_as_float(0x7FC00000u);
          else if (pinf) o[d] = INFINITY;
          else if (ninf) o[d] = -INFINITY;
        }
      }
      const float lse2 = m_used + __log2f(l);  // lse * log2 e
      if (row < N) {
        uint4* dst = reinterpret_cast<uint4*>(out + ((size_t)head * N + row) * HD);
#pragma unroll
        for (int i = 0; i < HD / 8; ++i)
          dst[i] = make_uint4(pack_bf16(o[8 * i], o[8 * i + 1]), pack_bf16(o[8 * i + 2], o[8 * i + 3]),
                              pack_bf16(o[8 * i + 4], o[8 * i + 5]),
                              pack_bf16(o[8 * i + 6], o[8 * i + 7]));
        lse[(size_t)head * N + row] = lse2 * kLn2;
      }
      if (do16 != nullptr) {
        // what the backward of loss = 1/2 sum out^2 reads: dout = out as f16,
        // delta = sum_d out_d^2, -lse log2 e (rows past N: 0 and -inf)
        float sq = 0.f;
#pragma unroll
        for (int d = 0; d < HD; ++d) sq = fmaf(o[d], o[d], sq);
        const int64_t Npad = pad128(N);
        if (row < N) {
          uint4* dst = reinterpret_cast<uint4*>(do16 + ((size_t)head * N + row) * HD);
#pragma unroll
          for (int i = 0; i < HD / 8; ++i)
            dst[i] = make_uint4(pack_f16(o[8 * i], o[8 * i + 1]), pack_f16(o[8 * i + 2], o[8 * i + 3]),
                                pack_f16(o[8 * i + 4], o[8 * i + 5]),
                                pack_f16(o[8 * i + 6], o[8 * i + 7]));
        }
        if (row < Npad) {
          const bool real = row < N;
          delta[(size_t)head * Npad + row] = real ? sq : 0.f;
          nlse2[(size_t)head * Npad + row] = real ? -lse2 : -INFINITY;
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

template <bool kF16>
cudaError_t launch_fwd_instance(const CUtensorMap& tq, const CUtensorMap& tk,
                                const CUtensorMap& tv, void* out, float* lse, int64_t BH,
                                int64_t N, int causal, float scale, const int* vinfo,
                                const unsigned* vrows, int all_bf16, const FwdSaved& saved,
                                unsigned* err, cudaStream_t s, bool after) {
  cudaError_t e = cudaFuncSetAttribute(attn_fwd_tc_kernel<kF16>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)kSmemBytes);
  if (e != cudaSuccess) return e;
  cudaFuncAttributes fa;
  e = cudaFuncGetAttributes(&fa, attn_fwd_tc_kernel<kF16>);
  if (e != cudaSuccess) return e;
  if (fa.numRegs != kLaunchRegs) return cudaErrorInvalidKernelImage;  // register split unsafe
  const int n_ctiles = (int)((N + 2 * BM - 1) / (2 * BM));
  const int64_t grid = (int64_t)n_ctiles * BH;
  e = launch_after(after, attn_fwd_tc_kernel<kF16>, dim3((unsigned)grid), dim3(kThreads),
                   kSmemBytes, s, tq, tk, tv, static_cast<__nv_bfloat16*>(out), lse, (int)N,
                   (int)BH, n_ctiles, head_group(BH, N), causal, scale * kLog2e, vinfo,
                   reinterpret_cast<const uint4*>(vrows), all_bf16,
                   static_cast<uint16_t*>(saved.do16), saved.delta, saved.nlse2, err);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

cudaError_t launch_attn_fwd_tc(const void* q, const void* k, const void* v, const void* v16,
                               void* out, float* lse, int64_t B, int64_t H, int64_t N,
                               int causal, float scale, const int* vinfo, const unsigned* vrows,
                               const FwdSaved& saved, unsigned* err, cudaStream_t s,
                               int* launches) {
  const int64_t BH = B * H;
  CUtensorMap tq, tk, tv, tv16;
  cudaError_t e;
  if ((e = make_tmap_bf16_rows(&tq, q, BH, N, BM)) != cudaSuccess) return e;
  if ((e = make_tmap_bf16_rows(&tk, k, BH, N, BN)) != cudaSuccess) return e;
  if ((e = make_tmap_bf16_rows(&tv, v, BH, N, BN)) != cudaSuccess) return e;
  const int all_bf16 = v16 == nullptr ? 1 : 0;
  if (!all_bf16) {
    // f16-operand heads (the usual case) first; the bf16 instance's blocks of
    // those heads exit at once, and the other way round
    if ((e = make_tmap_bf16_rows(&tv16, v16, BH, N, BN)) != cudaSuccess) return e;
    if ((e = launch_fwd_instance<true>(tq, tk, tv16, out, lse, BH, N, causal, scale, vinfo,
                                       vrows, 0, saved, err, s, false)) != cudaSuccess)
      return e;
    *launches += 1;
  }
  // behind the f16 instance (disjoint heads, no data between them) it may
  // start in that launch's tail; alone it follows the prep pass as usual
  if ((e = launch_fwd_instance<false>(tq, tk, tv, out, lse, BH, N, causal, scale, vinfo,
                                      vrows, all_bf16, saved, err, s, !all_bf16)) != cudaSuccess)
    return e;
  *launches += 1;
  return cudaSuccess;
}

}  // namespace swa
