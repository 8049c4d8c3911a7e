// qkv_proj.cu -- the QKV projection in front of attention on the sm_100a
// tensor cores: q = x Wq, k = x Wk, v = x Wv ("Wiki notes", page 5,
// mini_attention), written straight into attention's [B, H, N, 64] layout.
//
// x is [B*N, C] (rows = tokens), w is [3*H*64, C] (one row per output
// feature: Wq's features h*64 + d, then Wk's, then Wv's -- the layout of a
// linear layer's weight, so both operands are K-major).  Output tile =
// 128 tokens x 256 features (four heads of one of q, k, v); the K loop walks
// C in steps of 64 (one 128-byte swizzle row per operand row).  N = 256
// because shared memory carries both the MMA's operand reads and the TMA
// writes that refill the stages, 128 bytes per clock in all: per tensor-pipe
// cycle an N = 128 product needs 128 bytes of reads and 128 of writes, an
// N = 256 one 96 and 96, which lifts that bound from one half of the tensor
// peak to two thirds.
//
// Persistent: one block per SM walks the tiles t = blockIdx.x + i gridDim.x
// (all tiles cost the same).  Block = 6 warps: warp 0 TMA producer (x and w
// tiles into a 4-stage ring that runs on across tiles), warp 1 MMA issuer
// (one elected lane) and TMEM owner, warps 2-5 epilogue (a warp reaches the
// TMEM lanes of its subpartition, 32 (w mod 4)..; lane = token; each thread
// converts its token's 256 features to bf16 and stores four 128-byte head
// rows).  Two TMEM accumulators of 256 columns alternate between tiles, so
// a tile's epilogue runs under the next tile's main loop.  Rows past B*N and
// features past 3*H*64 read as zeros (TMA fill) and are not written.  Every
// wait is bounded (device error word).
#include <cudaTypedefs.h>

#include "attn_tc.cuh"
#include "tc_ptx.cuh"

namespace swa {
namespace {

using namespace tc;

constexpr int TM = 128;                  // tokens per tile (MMA M)
constexpr int TN = 256;                  // features per tile (MMA N)
constexpr int TK = 64;                   // input channels per stage
constexpr int HD = 64;
constexpr int kStages = 4;
constexpr int kXBytes = TM * TK * 2;     // 16 KB
constexpr int kWBytes = TN * TK * 2;     // 32 KB: two 128-row loads
constexpr int kThreads = 192;
constexpr int kEpilogueWarps = 4;

struct __align__(1024) SmemP {
  uint8_t x[kStages][kXBytes];
  uint8_t w[kStages][kWBytes];
  uint64_t full[kStages];
  uint64_t empty[kStages];
  uint64_t acc_full[2];   // accumulator b holds a finished tile
  uint64_t acc_empty[2];  // the epilogue has read accumulator b out
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
};
constexpr size_t kSmemP = sizeof(SmemP) + 1024;
static_assert(kSmemP <= 232448, "shared memory");

__global__ void __launch_bounds__(kThreads, 1)
qkv_proj_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_w,
                __nv_bfloat16* __restrict__ q, __nv_bfloat16* __restrict__ k,
                __nv_bfloat16* __restrict__ v, int N, int H, int rows, int features, int k_tiles,
                int f_tiles, int n_tiles, unsigned* __restrict__ err) {
  extern __shared__ uint8_t smem_raw[];
  SmemP& sm = *reinterpret_cast<SmemP*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                        ~static_cast<uintptr_t>(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&sm.full[s], 1);
      mbar_init(&sm.empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&sm.acc_full[b], 1);
      mbar_init(&sm.acc_empty[b], kEpilogueWarps);
    }
    mbar_init(&sm.drain, 1);
    sm.abort = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&sm.tmem_base, 2 * TN);
    tmem_relinquish();
  }
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  const uint32_t tmem = sm.tmem_base;
  volatile int* abort = &sm.abort;

  if (warp == 0) {
    if (lane == 0) {
      prefetch_tmap(&tm_x);
      prefetch_tmap(&tm_w);
      int g = 0;  // stages filled so far, over all tiles
      bool ok = true;
      for (int t = blockIdx.x; ok && t < n_tiles; t += gridDim.x) {
        const int m0 = (t / f_tiles) * TM, f0 = (t % f_tiles) * TN;
        for (int kt = 0; kt < k_tiles; ++kt, ++g) {
          const int s = g % kStages, round = g / kStages;
          if (round > 0 &&
              !mbar_wait_parked(&sm.empty[s], (round - 1) & 1, abort, err, kDevTimeoutEmpty)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&sm.full[s], kXBytes + kWBytes);
          tma_load_3d(sm.x[s], &tm_x, &sm.full[s], kt * TK, m0, 0);
          tma_load_3d(sm.w[s], &tm_w, &sm.full[s], kt * TK, f0, 0);
          tma_load_3d(sm.w[s] + kWBytes / 2, &tm_w, &sm.full[s], kt * TK, f0 + 128, 0);
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    constexpr uint32_t idesc = idesc_bf16_f32(TM, TN, 0, 0);  // both K-major
    int g = 0, it = 0;
    bool ok = true;
    for (int t = blockIdx.x; ok && t < n_tiles; t += gridDim.x, ++it) {
      const int b = it & 1;
      // accumulator b's last tile (two tiles ago) has been read out
      if (it >= 2 &&
          !mbar_wait_parked(&sm.acc_empty[b], (it / 2 - 1) & 1, abort, err, kDevTimeoutOther))
        break;
      fence_after_sync();
      for (int kt = 0; kt < k_tiles; ++kt, ++g) {
        const int s = g % kStages;
        if (!mbar_wait_parked(&sm.full[s], (g / kStages) & 1, abort, err, kDevTimeoutFull)) {
          ok = false;
          break;
        }
        fence_after_sync();
        // 4 MMAs of K = 16 (32 bytes = 2 descriptor units along the swizzled row)
        mma_ss_run<4, 2, 0, 2>(tmem + b * TN, desc_sw128(smem_u32(sm.x[s]), 16, 1024),
                               desc_sw128(smem_u32(sm.w[s]), 16, 1024), idesc,
                               kt > 0 ? 1u : 0u);
        mma_commit_elect(&sm.empty[s]);
      }
      if (ok) mma_commit_elect(&sm.acc_full[b]);
    }
    mma_commit_elect(&sm.drain);
    const long long t0 = clock64();
    while (!mbar_try_wait(&sm.drain, 0) && clock64() - t0 < kWaitCycles) {
    }
    __syncwarp();
  } else {
    // epilogue: TMEM lane = token row of the tile (warps 2, 3, 4, 5 take the
    // subpartitions 2, 3, 0, 1)
    const int r = (warp & 3) * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const int per = H * HD;  // features of each of q, k, v
    int it = 0;
    for (int t = blockIdx.x; t < n_tiles; t += gridDim.x, ++it) {
      const int b = it & 1;
      if (!mbar_wait_parked(&sm.acc_full[b], (it / 2) & 1, abort, err, kDevTimeoutMma)) break;
      fence_after_sync();
      const int m = (t / f_tiles) * TM + r, f0 = (t % f_tiles) * TN;
      const int bb = m / N, n = m - bb * N;
#pragma unroll 1
      for (int gh = 0; gh < TN / HD; ++gh) {  // four 64-feature groups: one head each
        uint32_t packed[HD / 2];
#pragma unroll
        for (int i = 0; i < HD / 16; ++i) {
          uint32_t u[16];
          tmem_ld16(tmem + lane_off + b * TN + gh * HD + i * 16, u);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 8; ++e)
            packed[i * 8 + e] = pack_bf16(__uint_as_float(u[2 * e]), __uint_as_float(u[2 * e + 1]));
        }
        const int f = f0 + gh * HD;
        if (m < rows && f < features) {
          const int which = f / per, h = (f - which * per) / HD;
          __nv_bfloat16* dst = which == 0 ? q : (which == 1 ? k : v);
          uint4* row = reinterpret_cast<uint4*>(dst + (((size_t)bb * H + h) * N + n) * HD);
#pragma unroll
          for (int i = 0; i < HD / 8; ++i)
            row[i] = make_uint4(packed[4 * i], packed[4 * i + 1], packed[4 * i + 2],
                                packed[4 * i + 3]);
        }
      }
      // every load of accumulator b has completed: the MMA warp may reuse it
      fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.acc_empty[b]);
    }
  }
  fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    fence_after_sync();
    tmem_dealloc(tmem, 2 * TN);
  }
}

// [rows][cols] bf16 row-major as a 3-D map (cols, rows, 1), 64 x 128 boxes,
// 128-byte swizzle; out-of-range rows and columns read as zeros.  cols must
// be a multiple of 8 (16-byte row stride).
cudaError_t make_tmap_matrix(CUtensorMap* map, const void* base, int64_t rows, int64_t cols) {
  void* fnp = nullptr;
  cudaDriverEntryPointQueryResult qr;
  if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fnp, cudaEnableDefault, &qr) !=
          cudaSuccess || qr != cudaDriverEntryPointSuccess)
    return cudaErrorNotSupported;
  auto fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fnp);
  cuuint64_t dims[3] = {(cuuint64_t)cols, (cuuint64_t)rows, 1};
  cuuint64_t strides[2] = {(cuuint64_t)cols * 2, (cuuint64_t)rows * cols * 2};
  cuuint32_t box[3] = {TK, 128, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims,
                  strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_qkv_proj(const void* x, const void* w, void* q, void* k, void* v, int64_t B,
                            int64_t N, int64_t C, int64_t H, unsigned* err, cudaStream_t s,
                            int* launches) {
  const int64_t rows = B * N, features = 3 * H * HD;
  CUtensorMap tx, tw;
  cudaError_t e;
  if ((e = make_tmap_matrix(&tx, x, rows, C)) != cudaSuccess) return e;
  if ((e = make_tmap_matrix(&tw, w, features, C)) != cudaSuccess) return e;
  e = cudaFuncSetAttribute(qkv_proj_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)kSmemP);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
    return e;
  const int64_t m_tiles = (rows + TM - 1) / TM, f_tiles = (features + TN - 1) / TN;
  const int64_t n_tiles = m_tiles * f_tiles;
  const unsigned grid = (unsigned)(n_tiles < sms ? n_tiles : sms);
  qkv_proj_kernel<<<grid, kThreads, kSmemP, s>>>(
      tx, tw, static_cast<__nv_bfloat16*>(q), static_cast<__nv_bfloat16*>(k),
      static_cast<__nv_bfloat16*>(v), (int)N, (int)H, (int)rows, (int)features, (int)(C / TK),
      (int)f_tiles, (int)n_tiles, err);
  *launches += 1;
  return cudaGetLastError();
}

}  // namespace swa
