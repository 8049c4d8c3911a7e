// attn_tc.cuh -- launchers of the tensor-core (tcgen05) attention kernels.
// They handle only the heads whose flag is 0 (V, and for the backward dout,
// all finite); the pair-by-pair kernels take the others.
#pragma once

#include <cuda.h>

#include "swa_internal.cuh"

namespace swa {

// [BH][N][64] bf16 as a 3-D TMA tensor map (64, N, BH) with 64 x box_rows x 1
// boxes and 128-byte swizzle; rows past N read as zeros.
cudaError_t make_tmap_bf16_rows(CUtensorMap* map, const void* base, int64_t BH, int64_t N,
                                int box_rows);

cudaError_t launch_attn_fwd_tc(const void* q, const void* k, const void* v, void* out,
                               float* lse, int64_t B, int64_t H, int64_t N, int causal,
                               float scale, const int* flags, unsigned* err, cudaStream_t s,
                               int* launches);

// Backward of the finite heads: a key-major kernel writes dk and dv, a
// query-major kernel writes dq (both directly in bf16, no accumulator in
// memory).  nlse2 = -lse * log2 e and delta are the prep kernel's [BH][Npad]
// arrays.
cudaError_t launch_attn_bwd_tc(const void* q, const void* k, const void* v, const void* dout,
                               const float* nlse2, const float* delta, void* dq, void* dk,
                               void* dv, int64_t B, int64_t H, int64_t N, int causal,
                               float scale, const int* flags, unsigned* err, cudaStream_t s,
                               int* launches);

}  // namespace swa
