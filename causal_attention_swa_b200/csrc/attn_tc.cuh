// attn_tc.cuh -- launchers of the tensor-core (tcgen05) attention kernels.
// They take every head of a bf16 call; heads whose V (or, in the backward,
// dout) holds an infinity or NaN get the kernels' non-finite handling.
#pragma once

#include <cuda.h>

#include <utility>

#include "swa_internal.cuh"

namespace swa {

// Launches `kernel` on stream s, with programmatic stream serialisation when
// `after` is set: it may start once every block of the previous grid has
// begun (the kernels call pdl_prologue()), instead of after that grid ends.
// Only for a grid that reads nothing the previous grid writes.
template <typename... KArgs, typename... Args>
cudaError_t launch_after(bool after, void (*kernel)(KArgs...), dim3 grid, dim3 block,
                         size_t smem, cudaStream_t s, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = after ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// [BH][N][64] of a 16-bit type (bf16 or f16: the copy does not convert) as
// a 3-D TMA tensor map (64, N, BH) with 64 x box_rows x 1 boxes and 128-byte
// swizzle; rows past N read as zeros.
cudaError_t make_tmap_bf16_rows(CUtensorMap* map, const void* base, int64_t BH, int64_t N,
                                int box_rows);

// Heads whose blocks are scheduled together.  Every block of a head streams
// 256 N bytes of its 16-bit rows (K and V in the forward and dq, Q and dO
// in dK/dV).  When all heads' rows fit in 64 MB of the 126 MB L2, one group:
// the whole grid runs heaviest blocks first (no late group whose heavy
// blocks form a tail).  Else groups of four heads, whose rows stay in L2
// while the group's blocks run (groups of 16 at 2x16x16384 left the time
// unchanged and raised DRAM traffic 1.6x).  Inside a group blocks run
// heaviest first, heads interleaved.
inline int head_group(int64_t BH, int64_t N) {
  const int64_t per_head = 256 * (N > 0 ? N : 1);
  if (BH * per_head <= (int64_t(64) << 20)) return static_cast<int>(BH);
  return static_cast<int>(BH < 4 ? BH : 4);
}

// What the forward saves for the backward of loss = 1/2 sum out^2 (all
// null for a plain forward): do16 [BH][N][64] f16 copy of out; delta and
// nlse2 [BH][Npad] float32 (sum_d out_d^2 and -lse log2 e; padding rows 0
// and -inf).
struct FwdSaved {
  void* do16 = nullptr;
  float* delta = nullptr;
  float* nlse2 = nullptr;
};

// vinfo: the per-head information of the prep pass.  v16: an f16 copy of v
// (launch_attn_convert); with v16 the f16-operand instance takes the heads
// within f16's range and the bf16 instance the others (two launches);
// without it every head takes bf16 operands (one launch).  vrows (nullable):
// the prep pass's per-tile masks of V rows with a non-finite entry, which
// let the V cleaner of a flagged head skip clean rows.
cudaError_t launch_attn_fwd_tc(const void* q, const void* k, const void* v, const void* v16,
                               void* out, float* lse, int64_t B, int64_t H, int64_t N,
                               int causal, float scale, const int* vinfo, const unsigned* vrows,
                               const FwdSaved& saved, unsigned* err, cudaStream_t s,
                               int* launches);

// The four 16-bit operand tensors of a backward instance, [BH][N][64] each.
struct BwdOperands {
  const void* q;
  const void* k;
  const void* v;
  const void* dout;
};

// Backward: a key-major kernel writes dk and dv, a query-major kernel writes
// dq (both directly in bf16, no accumulator in memory); f16-operand heads
// read `f16` (copies), the others `bf16`.  Four launches.  nlse2 = -lse *
// log2 e and delta are [BH][Npad] float32; info holds four int32 per head
// (non-finite flags of V and dout, largest exponents of V, Q/K and dout).
// Accumulate mode of the backward (all null: write bf16 dq, dk, dv): float32
// [BH][N][64] sums to which each call adds its dq, dk, dv instead.
struct BwdAcc {
  float* dq = nullptr;
  float* dk = nullptr;
  float* dv = nullptr;
};

cudaError_t launch_attn_bwd_tc(const BwdOperands& f16, const BwdOperands& bf16,
                               const float* nlse2, const float* delta, void* dq, void* dk,
                               void* dv, const BwdAcc& acc, int64_t B, int64_t H, int64_t N,
                               int causal, float scale, const int* info, unsigned* err,
                               cudaStream_t s, int* launches);

}  // namespace swa

namespace swa {

// q, k, v [B][H][N][64] bf16 = x [B*N][C] times the rows of w [3*H*64][C]
// (q's features, then k's, then v's); C a multiple of 64.  One launch.
cudaError_t launch_qkv_proj(const void* x, const void* w, void* q, void* k, void* v, int64_t B,
                            int64_t N, int64_t C, int64_t H, unsigned* err, cudaStream_t s,
                            int* launches);

}  // namespace swa
