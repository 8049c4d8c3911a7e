// swa_noalloc.cu -- swa_attn_fwd_noalloc: the attention forward for callers
// that cannot allocate device memory.
//
// Some callers cannot call cudaMalloc or accept a workspace: a plugin whose
// host application owns every device allocation and hands it only the
// input and output buffers, or a latency-critical path that must not pay
// for cudaMalloc / cudaFree and their implicit device synchronisation.  For
// them this entry point keeps the forward's only scratch memory -- four
// int32 per head from the scan of V (whether it holds an infinity or NaN,
// and the largest exponent of its finite values) -- in a file-scope device
// array instead of a caller workspace.
//
// The array holds kSwaNoallocMaxHeads = 4096 heads (4 x 4096 int32, 64 KB).
// Every GPU that loads the library holds it until the process exits.  Host code may not use the
// array's name as a device address (on the host it names a stand-in), so on
// the first call on each device, with that device current, the entry point
// looks the address up with cudaGetSymbolAddress and caches it; that first
// call should therefore come before any stream capture.  All calls share
// the array and it keeps the last call's contents: each call clears the
// entries it uses before the scan, and calls that overlap on the GPU (other
// streams, other host threads) race on it.
#include <mutex>

#include "attn_tc.cuh"
#include "swa_internal.cuh"

namespace {

constexpr int64_t kSwaNoallocMaxHeads = 4096;

static __device__ __align__(256) int g_noalloc_head_flags[swa::kHeadInfoInts *
                                                          kSwaNoallocMaxHeads];

// Device address of g_noalloc_head_flags for the current device.
int* noalloc_flags(swa_status* st) {
  static std::mutex mu;
  static int* cache[64] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess || dev < 0 || dev >= 64) {
    *st = swa::api_cuda_fail(e == cudaSuccess ? cudaErrorInvalidDevice : e, "cudaGetDevice");
    return nullptr;
  }
  std::lock_guard<std::mutex> lock(mu);
  if (!cache[dev]) {
    int* p = nullptr;
    e = cudaGetSymbolAddress((void**)&p, g_noalloc_head_flags);
    if (e != cudaSuccess) {
      *st = swa::api_cuda_fail(e, "cudaGetSymbolAddress(noalloc head flags)");
      return nullptr;
    }
    cache[dev] = p;
  }
  *st = SWA_OK;
  return cache[dev];
}

bool aligned16(const void* p) { return p != nullptr && ((uintptr_t)p & 15u) == 0; }

}  // namespace

extern "C" swa_status swa_attn_fwd_noalloc(const void* q, const void* k, const void* v,
                                           void* out, float* lse, int64_t B, int64_t H,
                                           int64_t N, int64_t D, int causal, swa_dtype dt,
                                           void* stream) {
  swa::api_begin_call();
  swa_status st = swa::api_check_attn_shape(B, H, N, D, dt);
  if (st != SWA_OK) return st;
  if (B * H > kSwaNoallocMaxHeads)
    return swa::api_fail(SWA_ERR_UNSUPPORTED,
                         "swa_attn_fwd_noalloc: B*H exceeds the 4096 heads its static "
                         "scratch holds");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(lse))
    return swa::api_fail(SWA_ERR_INVALID_ARGUMENT,
                         "q, k, v, out, lse must be non-null and 16-byte aligned");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int64_t BH = B * H;
  const float scale = 1.0f / sqrtf((float)D);
  const int c = causal ? 1 : 0;
  unsigned* err = swa::api_error_word(&st);
  if (!err) return st;
  int launches = 0;
  cudaError_t e;
  if (dt == SWA_F32) {
    e = swa::launch_attn_fwd_simt(dt, q, k, v, out, lse, BH, N, c, scale, s, &launches);
    if (e != cudaSuccess) return swa::api_cuda_fail(e, "attn_fwd_simt");
  } else {
    int* vinfo = noalloc_flags(&st);
    if (!vinfo) return st;
    e = cudaMemsetAsync(vinfo, 0, (size_t)BH * swa::kHeadInfoInts * sizeof(int), s);
    if (e != cudaSuccess) return swa::api_cuda_fail(e, "cudaMemsetAsync(noalloc scratch)");
    e = swa::launch_scan_v_info(v, BH, N * D, vinfo, s, &launches);
    if (e != cudaSuccess) return swa::api_cuda_fail(e, "scan_v_info");
    e = swa::launch_attn_fwd_tc(q, k, v, nullptr, out, lse, B, H, N, c, scale, vinfo, nullptr,
                                swa::FwdSaved{}, err, s, &launches);
    if (e != cudaSuccess) return swa::api_cuda_fail(e, "attn_fwd_tc");
  }
  swa::api_end_call(launches);
  return SWA_OK;
}
