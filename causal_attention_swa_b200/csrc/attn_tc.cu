// attn_tc.cu -- backward of the finite heads of the bf16 path.  Routed to
// the CUDA-core kernels until the tcgen05 backward is in place.
#include "attn_tc.cuh"

namespace swa {

cudaError_t launch_attn_bwd_tc(const void* q, const void* k, const void* v, const void* dout,
                               const float* lse, const float* delta, void* dq, void* dk,
                               void* dv, float* dqacc, int64_t B, int64_t H, int64_t N,
                               int causal, float scale, const int* flags, unsigned* err,
                               cudaStream_t s, int* launches) {
  (void)err;
  (void)dqacc;
  return launch_attn_bwd_simt(SWA_BF16, q, k, v, dout, lse, delta, dq, dk, dv, B * H, N, causal,
                              scale, flags, 0, s, launches);
}

}  // namespace swa
