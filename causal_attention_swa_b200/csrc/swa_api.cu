// swa_api.cu -- the C ABI of libswa.so (include/swa.h): argument checks,
// workspace carving, per-head dispatch and the device error word.  No
// allocation happens here: every buffer, workspaces included, is the
// caller's.
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "swa_internal.cuh"
#include "attn_tc.cuh"

// Device error word: kernels whose bounded waits run out record a code here
// (first writer wins) instead of trapping; swa_get_device_error() reports
// and clears it.
static __device__ unsigned g_swa_error_word;

namespace {

thread_local char t_msg[512];
thread_local int t_launches;

struct Prof {
  swa_kernel which = SWA_KERNEL_NONE;
  cudaEvent_t start = nullptr, stop = nullptr;
};
thread_local Prof t_prof;

// Records the hook's start/stop events around one launcher call when it
// names this kernel.
struct ProfScope {
  bool on;
  cudaStream_t s;
  ProfScope(swa_kernel k, cudaStream_t stream) : on(t_prof.which == k), s(stream) {
    if (on) cudaEventRecord(t_prof.start, s);
  }
  ~ProfScope() {
    if (on) cudaEventRecord(t_prof.stop, s);
  }
};

swa_status fail(swa_status st, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(t_msg, sizeof(t_msg), fmt, ap);
  va_end(ap);
  return st;
}

swa_status cuda_fail(cudaError_t e, const char* where) {
  return fail(SWA_ERR_CUDA, "%s: %s", where, cudaGetErrorString(e));
}

bool aligned16(const void* p) { return p != nullptr && ((uintptr_t)p & 15u) == 0; }

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Device address of g_swa_error_word for the current device (host code may
// not take the symbol's address directly).
unsigned* device_error_word(swa_status* st) {
  static std::mutex mu;
  static unsigned* cache[64] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess || dev < 0 || dev >= 64) {
    *st = cuda_fail(e == cudaSuccess ? cudaErrorInvalidDevice : e, "cudaGetDevice");
    return nullptr;
  }
  std::lock_guard<std::mutex> lock(mu);
  if (!cache[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_swa_error_word);
    if (e != cudaSuccess) {
      *st = cuda_fail(e, "cudaGetSymbolAddress(error word)");
      return nullptr;
    }
    cache[dev] = static_cast<unsigned*>(p);
  }
  *st = SWA_OK;
  return cache[dev];
}

constexpr int64_t kMaxElems = (int64_t)1 << 40;

swa_status check_attn_shape(int64_t B, int64_t H, int64_t N, int64_t D, swa_dtype dt) {
  if (dt != SWA_F32 && dt != SWA_BF16) return fail(SWA_ERR_INVALID_ARGUMENT, "unknown dtype %d", (int)dt);
  if (B < 1 || H < 1 || N < 1) return fail(SWA_ERR_INVALID_ARGUMENT, "B, H, N must be >= 1 (got %lld, %lld, %lld)",
                                           (long long)B, (long long)H, (long long)N);
  if (D != 64) return fail(SWA_ERR_UNSUPPORTED, "only D = 64 is implemented (got %lld)", (long long)D);
  if (B * H > 65535) return fail(SWA_ERR_UNSUPPORTED, "B*H must be <= 65535 (got %lld)", (long long)(B * H));
  if (N > ((int64_t)1 << 30)) return fail(SWA_ERR_UNSUPPORTED, "N must be <= 2^30 (got %lld)", (long long)N);
  if (B * H * N > kMaxElems / D) return fail(SWA_ERR_UNSUPPORTED, "tensor too large");
  return SWA_OK;
}

// Per 128-row tile of V, the mask of its rows that hold an infinity or NaN:
// [BH][Npad / 128][4] uint32 (written whole by the prep pass).
size_t vrows_bytes(int64_t B, int64_t H, int64_t N) {
  return round_up((size_t)(B * H) * (size_t)(swa::pad128(N) / 128) * 16, 256);
}

// Forward workspace (bf16 only), in this order:
//   info   [BH][4] int32            per-head information of the prep pass
//   vrows  [BH][Npad/128][4] uint32 non-finite row masks of V's tiles
//   v16    [BH][N][64] f16          the f16 copy of V (the f16 instance's operand)
struct FwdWs {
  size_t info, vrows, total;
};

FwdWs fwd_ws(int64_t B, int64_t H, int64_t N, int64_t D, swa_dtype dt) {
  FwdWs w{0, 0, 0};
  if (dt != SWA_BF16) return w;
  w.info = round_up((size_t)(B * H) * swa::kHeadInfoInts * sizeof(int), 256);
  w.vrows = vrows_bytes(B, H, N);
  w.total = w.info + w.vrows + round_up((size_t)(B * H * N * D) * 2, 256);
  return w;
}

// Backward (and gradient) workspace, in this order:
//   info   [BH][4] int32        per-head information
//   vrows  [BH][Npad/128][4] uint32  non-finite row masks of V's tiles (the
//                               gradient's forward reads them)
//   delta  [BH][Npad] float32   dout . out per row (Npad = N rounded up to 128)
//   nlse2  [BH][Npad] float32   -lse log2 e per row
//   q16, k16, v16, do16  [BH][N][64] f16 each (bf16 only): the f16 operands
struct BwdWs {
  size_t info, vrows, delta, nlse2, copy, total;
};

BwdWs bwd_ws(int64_t B, int64_t H, int64_t N, int64_t D, swa_dtype dt) {
  BwdWs w;
  w.info = round_up((size_t)(B * H) * swa::kHeadInfoInts * sizeof(int), 256);
  w.vrows = dt == SWA_BF16 ? vrows_bytes(B, H, N) : 0;
  w.delta = round_up((size_t)(B * H * swa::pad128(N)) * sizeof(float), 256);
  w.nlse2 = w.delta;
  w.copy = dt == SWA_BF16 ? round_up((size_t)(B * H * N * D) * 2, 256) : 0;
  w.total = w.info + w.vrows + w.delta + w.nlse2 + 4 * w.copy;
  return w;
}

struct BwdPtrs {
  int* info;
  unsigned* vrows;
  float* delta;
  float* nlse2;
  void* q16;
  void* k16;
  void* v16;
  void* do16;
};

BwdPtrs carve(void* workspace, const BwdWs& w) {
  char* b = static_cast<char*>(workspace);
  BwdPtrs p;
  p.info = reinterpret_cast<int*>(b);
  p.vrows = reinterpret_cast<unsigned*>(b + w.info);
  p.delta = reinterpret_cast<float*>(b + w.info + w.vrows);
  p.nlse2 = reinterpret_cast<float*>(b + w.info + w.vrows + w.delta);
  char* c = b + w.info + w.vrows + w.delta + w.nlse2;
  p.q16 = c;
  p.k16 = c + w.copy;
  p.v16 = c + 2 * w.copy;
  p.do16 = c + 3 * w.copy;
  return p;
}

}  // namespace

namespace swa {

swa_status api_fail(swa_status st, const char* msg) { return fail(st, "%s", msg); }
swa_status api_cuda_fail(cudaError_t e, const char* where) { return cuda_fail(e, where); }
swa_status api_check_attn_shape(int64_t B, int64_t H, int64_t N, int64_t D, swa_dtype dt) {
  return check_attn_shape(B, H, N, D, dt);
}
unsigned* api_error_word(swa_status* st) { return device_error_word(st); }
void api_begin_call() {
  t_msg[0] = 0;
  t_launches = 0;
}
void api_end_call(int launches) { t_launches = launches; }

}  // namespace swa

extern "C" {

size_t swa_attn_fwd_workspace_size(int64_t B, int64_t H, int64_t N, int64_t D, swa_dtype dt) {
  if (B < 1 || H < 1 || N < 1 || D < 1) return 0;
  return fwd_ws(B, H, N, D, dt).total;
}

swa_status swa_attn_fwd(const void* q, const void* k, const void* v, void* out, float* lse,
                        int64_t B, int64_t H, int64_t N, int64_t D, int causal,
                        swa_dtype dt, void* workspace, size_t workspace_bytes, void* stream) {
  t_msg[0] = 0;
  t_launches = 0;
  swa_status st = check_attn_shape(B, H, N, D, dt);
  if (st != SWA_OK) return st;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(lse))
    return fail(SWA_ERR_INVALID_ARGUMENT, "q, k, v, out, lse must be non-null and 16-byte aligned");
  const FwdWs ws = fwd_ws(B, H, N, D, dt);
  const size_t need = ws.total;
  if (need && (!aligned16(workspace) || workspace_bytes < need))
    return fail(SWA_ERR_INVALID_ARGUMENT, "workspace must be 16-byte aligned and >= %zu bytes", need);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int64_t BH = B * H;
  const float scale = 1.0f / sqrtf((float)D);
  unsigned* err = device_error_word(&st);
  if (!err) return st;
  int launches = 0;
  cudaError_t e;
  if (dt == SWA_F32) {
    e = swa::launch_attn_fwd_simt(dt, q, k, v, out, lse, BH, N, causal ? 1 : 0, scale, s,
                                  &launches);
    if (e != cudaSuccess) return cuda_fail(e, "attn_fwd_simt");
  } else {
    // prep: the f16 copy of V and the per-head V information (non-finite
    // values, range); then the tensor-core kernels for every head
    int* vinfo = static_cast<int*>(workspace);
    unsigned* vrows = reinterpret_cast<unsigned*>(static_cast<char*>(workspace) + ws.info);
    void* v16 = static_cast<char*>(workspace) + ws.info + ws.vrows;
    e = cudaMemsetAsync(vinfo, 0, (size_t)BH * swa::kHeadInfoInts * sizeof(int), s);
    if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync(vinfo)");
    e = swa::launch_attn_convert(nullptr, nullptr, v, nullptr, nullptr, nullptr, nullptr,
                                 nullptr, v16, nullptr, nullptr, nullptr, vinfo, vrows, BH, N, s,
                                 &launches);
    if (e != cudaSuccess) return cuda_fail(e, "attn_convert");
    {
      ProfScope ps(SWA_KERNEL_ATTN_FWD, s);
      e = swa::launch_attn_fwd_tc(q, k, v, v16, out, lse, B, H, N, causal ? 1 : 0, scale,
                                  vinfo, vrows, swa::FwdSaved{}, err, s, &launches);
    }
    if (e != cudaSuccess) return cuda_fail(e, "attn_fwd_tc");
  }
  t_launches = launches;
  return SWA_OK;
}

size_t swa_attn_bwd_workspace_size(int64_t B, int64_t H, int64_t N, int64_t D, swa_dtype dt) {
  if (B < 1 || H < 1 || N < 1 || D < 1) return 0;
  return bwd_ws(B, H, N, D, dt).total;
}

}  // extern "C"

namespace {

// The backward with bf16 (or float32) dq, dk, dv, or -- acc non-null, bf16
// only -- with dq, dk, dv added to float32 sums.
swa_status attn_bwd_impl(const void* q, const void* k, const void* v, const void* out,
                         const void* dout, const float* lse, void* dq, void* dk, void* dv,
                         const swa::BwdAcc& acc, int64_t B, int64_t H, int64_t N, int64_t D,
                         int causal, swa_dtype dt, void* workspace, size_t workspace_bytes,
                         void* stream) {
  t_msg[0] = 0;
  t_launches = 0;
  swa_status st = check_attn_shape(B, H, N, D, dt);
  if (st != SWA_OK) return st;
  const bool accumulate = acc.dq != nullptr;
  if (accumulate && dt != SWA_BF16)
    return fail(SWA_ERR_UNSUPPORTED, "the accumulating backward takes bf16 inputs only");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(dout) ||
      !aligned16(lse))
    return fail(SWA_ERR_INVALID_ARGUMENT,
                "q, k, v, out, dout, lse must be non-null and 16-byte aligned");
  if (accumulate ? (!aligned16(acc.dq) || !aligned16(acc.dk) || !aligned16(acc.dv))
                 : (!aligned16(dq) || !aligned16(dk) || !aligned16(dv)))
    return fail(SWA_ERR_INVALID_ARGUMENT, "dq, dk, dv must be non-null and 16-byte aligned");
  const BwdWs ws = bwd_ws(B, H, N, D, dt);
  if (!aligned16(workspace) || workspace_bytes < ws.total)
    return fail(SWA_ERR_INVALID_ARGUMENT, "workspace must be 16-byte aligned and >= %zu bytes",
                ws.total);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int64_t BH = B * H;
  const float scale = 1.0f / sqrtf((float)D);
  unsigned* err = device_error_word(&st);
  if (!err) return st;
  const BwdPtrs w = carve(workspace, ws);
  const int64_t Npad = swa::pad128(N);
  const int c = causal ? 1 : 0;
  int launches = 0;
  cudaError_t e;
  if (dt == SWA_F32) {
    e = swa::launch_attn_bwd_prep(dt, out, dout, lse, w.delta, w.nlse2, BH, N, Npad, s,
                                  &launches);
    if (e != cudaSuccess) return cuda_fail(e, "attn_bwd_prep");
    e = swa::launch_attn_bwd_simt(dt, q, k, v, dout, lse, w.delta, Npad, dq, dk, dv, BH, N, c,
                                  scale, s, &launches);
    if (e != cudaSuccess) return cuda_fail(e, "attn_bwd_simt");
  } else {
    // prep: f16 operand copies, delta, -lse log2 e, per-head information;
    // then the tensor-core kernels for every head (f16 or bf16 operands per
    // head; the information switches on their non-finite handling)
    e = cudaMemsetAsync(w.info, 0, (size_t)BH * swa::kHeadInfoInts * sizeof(int), s);
    if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync(info)");
    e = swa::launch_attn_convert(q, k, v, dout, out, lse, w.q16, w.k16, w.v16, w.do16, w.delta,
                                 w.nlse2, w.info, nullptr, BH, N, s, &launches);
    if (e != cudaSuccess) return cuda_fail(e, "attn_convert");
    {
      ProfScope ps(SWA_KERNEL_ATTN_BWD, s);
      e = swa::launch_attn_bwd_tc(swa::BwdOperands{w.q16, w.k16, w.v16, w.do16},
                                  swa::BwdOperands{q, k, v, dout}, w.nlse2, w.delta, dq, dk, dv,
                                  acc, B, H, N, c, scale, w.info, err, s, &launches);
    }
    if (e != cudaSuccess) return cuda_fail(e, "attn_bwd_tc");
  }
  t_launches = launches;
  return SWA_OK;
}

}  // namespace

extern "C" {

swa_status swa_attn_bwd(const void* q, const void* k, const void* v, const void* out,
                        const void* dout, const float* lse, void* dq, void* dk, void* dv,
                        int64_t B, int64_t H, int64_t N, int64_t D, int causal, swa_dtype dt,
                        void* workspace, size_t workspace_bytes, void* stream) {
  return attn_bwd_impl(q, k, v, out, dout, lse, dq, dk, dv, swa::BwdAcc{}, B, H, N, D, causal,
                       dt, workspace, workspace_bytes, stream);
}

swa_status swa_attn_bwd_acc(const void* q, const void* k, const void* v, const void* out,
                            const void* dout, const float* lse, float* dq_acc, float* dk_acc,
                            float* dv_acc, int64_t B, int64_t H, int64_t N, int64_t D,
                            int causal, swa_dtype dt, void* workspace, size_t workspace_bytes,
                            void* stream) {
  if (dq_acc == nullptr || dk_acc == nullptr || dv_acc == nullptr) {
    t_msg[0] = 0;
    t_launches = 0;
    return fail(SWA_ERR_INVALID_ARGUMENT, "dq_acc, dk_acc, dv_acc must be non-null");
  }
  swa::BwdAcc acc;
  acc.dq = dq_acc;
  acc.dk = dk_acc;
  acc.dv = dv_acc;
  return attn_bwd_impl(q, k, v, out, dout, lse, nullptr, nullptr, nullptr, acc, B, H, N, D,
                       causal, dt, workspace, workspace_bytes, stream);
}

size_t swa_attn_grad_workspace_size(int64_t B, int64_t H, int64_t N, int64_t D, swa_dtype dt) {
  if (B < 1 || H < 1 || N < 1 || D < 1) return 0;
  return bwd_ws(B, H, N, D, dt).total;
}

swa_status swa_attn_grad(const void* q, const void* k, const void* v, void* out, float* lse,
                         void* dq, void* dk, void* dv, int64_t B, int64_t H, int64_t N,
                         int64_t D, int causal, swa_dtype dt, void* workspace,
                         size_t workspace_bytes, void* stream) {
  t_msg[0] = 0;
  t_launches = 0;
  swa_status st = check_attn_shape(B, H, N, D, dt);
  if (st != SWA_OK) return st;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(lse) ||
      !aligned16(dq) || !aligned16(dk) || !aligned16(dv))
    return fail(SWA_ERR_INVALID_ARGUMENT,
                "q, k, v, out, lse, dq, dk, dv must be non-null and 16-byte aligned");
  const BwdWs ws = bwd_ws(B, H, N, D, dt);
  if (!aligned16(workspace) || workspace_bytes < ws.total)
    return fail(SWA_ERR_INVALID_ARGUMENT, "workspace must be 16-byte aligned and >= %zu bytes",
                ws.total);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int64_t BH = B * H;
  const float scale = 1.0f / sqrtf((float)D);
  unsigned* err = device_error_word(&st);
  if (!err) return st;
  const BwdPtrs w = carve(workspace, ws);
  const int64_t Npad = swa::pad128(N);
  const int c = causal ? 1 : 0;
  int launches = 0;
  cudaError_t e;
  if (dt == SWA_F32) {
    e = swa::launch_attn_fwd_simt(dt, q, k, v, out, lse, BH, N, c, scale, s, &launches);
    if (e != cudaSuccess) return cuda_fail(e, "attn_fwd_simt");
    e = swa::launch_attn_bwd_prep(dt, out, out, lse, w.delta, w.nlse2, BH, N, Npad, s,
                                  &launches);
    if (e != cudaSuccess) return cuda_fail(e, "attn_bwd_prep");
    e = swa::launch_attn_bwd_simt(dt, q, k, v, out, lse, w.delta, Npad, dq, dk, dv, BH, N, c,
                                  scale, s, &launches);
    if (e != cudaSuccess) return cuda_fail(e, "attn_bwd_simt");
  } else {
    // prep (f16 copies of q, k, v; per-head information), the forward --
    // which also saves an f16 copy of out, delta = |out_i|^2 and -lse log2 e
    // from its float32 accumulator -- and the backward with dout = out
    e = cudaMemsetAsync(w.info, 0, (size_t)BH * swa::kHeadInfoInts * sizeof(int), s);
    if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync(info)");
    e = swa::launch_attn_convert(q, k, v, nullptr, nullptr, nullptr, w.q16, w.k16, w.v16,
                                 nullptr, nullptr, nullptr, w.info, w.vrows, BH, N, s, &launches);
    if (e != cudaSuccess) return cuda_fail(e, "attn_convert");
    swa::FwdSaved saved;
    saved.do16 = w.do16;
    saved.delta = w.delta;
    saved.nlse2 = w.nlse2;
    {
      ProfScope ps(SWA_KERNEL_ATTN_FWD, s);
      e = swa::launch_attn_fwd_tc(q, k, v, w.v16, out, lse, B, H, N, c, scale, w.info, w.vrows,
                                  saved, err, s, &launches);
    }
    if (e != cudaSuccess) return cuda_fail(e, "attn_fwd_tc");
    {
      ProfScope ps(SWA_KERNEL_ATTN_BWD, s);
      e = swa::launch_attn_bwd_tc(swa::BwdOperands{w.q16, w.k16, w.v16, w.do16},
                                  swa::BwdOperands{q, k, v, out}, w.nlse2, w.delta, dq, dk, dv,
                                  swa::BwdAcc{}, B, H, N, c, scale, w.info, err, s, &launches);
    }
    if (e != cudaSuccess) return cuda_fail(e, "attn_bwd_tc");
  }
  t_launches = launches;
  return SWA_OK;
}

size_t swa_nw_workspace_size(int64_t M, int64_t S) {
  if (M < 1 || S < 1) return 0;
  return round_up(swa::nw_partials_bytes(M, S), 256);
}

namespace {

swa_status check_nw(const float* targets, int64_t M, const float* sources, const float* vals,
                    int64_t S, int dims, float h) {
  if (M < 1 || S < 1)
    return fail(SWA_ERR_INVALID_ARGUMENT, "M and S must be >= 1 (got %lld, %lld)", (long long)M,
                (long long)S);
  if (M > ((int64_t)1 << 31) || S > ((int64_t)1 << 31))
    return fail(SWA_ERR_UNSUPPORTED, "M and S must be <= 2^31");
  if (dims < 1 || dims > 3)
    return fail(SWA_ERR_UNSUPPORTED, "points must have 1, 2 or 3 coordinates (got %d)", dims);
  if (!(h > 0.f) || !isfinite(h))
    return fail(SWA_ERR_INVALID_ARGUMENT, "bandwidth h must be finite and > 0");
  if (!aligned16(targets) || !aligned16(sources) || !aligned16(vals))
    return fail(SWA_ERR_INVALID_ARGUMENT,
                "targets, sources, vals must be non-null and 16-byte aligned");
  return SWA_OK;
}

swa_status nw_forward(const float* targets, int64_t M, const float* sources, const float* vals,
                      int64_t S, int dims, float h, float* out, void* workspace,
                      size_t workspace_bytes, void* stream) {
  t_msg[0] = 0;
  t_launches = 0;
  swa_status st = check_nw(targets, M, sources, vals, S, dims, h);
  if (st != SWA_OK) return st;
  if (!aligned16(out)) return fail(SWA_ERR_INVALID_ARGUMENT, "out must be non-null and 16-byte aligned");
  const size_t need = swa_nw_workspace_size(M, S);
  if (!aligned16(workspace) || workspace_bytes < need)
    return fail(SWA_ERR_INVALID_ARGUMENT, "workspace must be 16-byte aligned and >= %zu bytes",
                need);
  int launches = 0;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e;
  {
    ProfScope ps(SWA_KERNEL_NW, s);  // the whole call: pair grid and final sum
    e = swa::launch_nw_partial(targets, M, sources, vals, S, dims, h,
                               static_cast<float*>(workspace), s, &launches);
    if (e != cudaSuccess) return cuda_fail(e, "nw_partial");
    e = swa::launch_nw_finalize(M, S, static_cast<const float*>(workspace), out, s, &launches);
  }
  if (e != cudaSuccess) return cuda_fail(e, "nw_finalize");
  t_launches = launches;
  return SWA_OK;
}

}  // namespace

swa_status swa_nw_regrid(const float* targets, int64_t M, const float* sources,
                         const float* vals, int64_t S, float h, float* out, void* workspace,
                         size_t workspace_bytes, void* stream) {
  return nw_forward(targets, M, sources, vals, S, 2, h, out, workspace, workspace_bytes, stream);
}

swa_status swa_nw_regrid_nd(const float* targets, int64_t M, const float* sources,
                            const float* vals, int64_t S, int dims, float h, float* out,
                            void* workspace, size_t workspace_bytes, void* stream) {
  return nw_forward(targets, M, sources, vals, S, dims, h, out, workspace, workspace_bytes,
                    stream);
}

size_t swa_nw_regrid_bwd_workspace_size(int64_t M, int64_t S, int dims) {
  if (M < 1 || S < 1 || dims < 1 || dims > 3) return 0;
  return round_up(swa::nw_bwd_workspace_bytes(M, S), 256);
}

swa_status swa_nw_regrid_bwd(const float* targets, int64_t M, const float* sources,
                             const float* vals, int64_t S, int dims, float h, const float* gout,
                             float* dtargets, float* dsources, float* dvals, void* workspace,
                             size_t workspace_bytes, void* stream) {
  t_msg[0] = 0;
  t_launches = 0;
  swa_status st = check_nw(targets, M, sources, vals, S, dims, h);
  if (st != SWA_OK) return st;
  if (!aligned16(gout) || !aligned16(dtargets) || !aligned16(dsources) || !aligned16(dvals))
    return fail(SWA_ERR_INVALID_ARGUMENT,
                "gout, dtargets, dsources, dvals must be non-null and 16-byte aligned");
  const size_t need = swa_nw_regrid_bwd_workspace_size(M, S, dims);
  if (!aligned16(workspace) || workspace_bytes < need)
    return fail(SWA_ERR_INVALID_ARGUMENT, "workspace must be 16-byte aligned and >= %zu bytes",
                need);
  int launches = 0;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e;
  {
    ProfScope ps(SWA_KERNEL_NW_BWD, s);
    e = swa::launch_nw_bwd(targets, M, sources, vals, S, dims, h, gout, dtargets, dsources, dvals,
                           static_cast<float*>(workspace), s, &launches);
  }
  if (e != cudaSuccess) return cuda_fail(e, "nw_bwd");
  t_launches = launches;
  return SWA_OK;
}

swa_status swa_qkv_proj(const void* x, const void* w, void* q, void* k, void* v, int64_t B,
                        int64_t N, int64_t C, int64_t H, int64_t D, swa_dtype dt, void* stream) {
  t_msg[0] = 0;
  t_launches = 0;
  if (dt != SWA_BF16) return fail(SWA_ERR_UNSUPPORTED, "the projection takes bf16 only");
  swa_status st = check_attn_shape(B, H, N, D, dt);
  if (st != SWA_OK) return st;
  if (C < 64 || C % 64 != 0)
    return fail(SWA_ERR_UNSUPPORTED, "C must be a positive multiple of 64 (got %lld)",
                (long long)C);
  if (C > (1 << 20) || B * N > ((int64_t)1 << 31))
    return fail(SWA_ERR_UNSUPPORTED, "C <= 2^20 and B*N <= 2^31 are supported");
  if (!aligned16(x) || !aligned16(w) || !aligned16(q) || !aligned16(k) || !aligned16(v))
    return fail(SWA_ERR_INVALID_ARGUMENT, "x, w, q, k, v must be non-null and 16-byte aligned");
  unsigned* err = device_error_word(&st);
  if (!err) return st;
  int launches = 0;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e;
  {
    ProfScope ps(SWA_KERNEL_QKV, s);
    e = swa::launch_qkv_proj(x, w, q, k, v, B, N, C, H, err, s, &launches);
  }
  if (e != cudaSuccess) return cuda_fail(e, "qkv_proj");
  t_launches = launches;
  return SWA_OK;
}

swa_status swa_attn_merge(const void* out_part, const float* lse_part, float* out_acc,
                          float* lse_acc, void* out_final, int64_t rows, int64_t D, int first,
                          swa_dtype dt, void* stream) {
  t_msg[0] = 0;
  t_launches = 0;
  if (dt != SWA_BF16 && dt != SWA_F32) return fail(SWA_ERR_INVALID_ARGUMENT, "unknown dtype");
  if (D != 64) return fail(SWA_ERR_UNSUPPORTED, "D must be 64 (got %lld)", (long long)D);
  if (rows < 1 || rows > ((int64_t)1 << 31))
    return fail(SWA_ERR_INVALID_ARGUMENT, "rows must be in [1, 2^31] (got %lld)",
                (long long)rows);
  if (!aligned16(out_part) || !aligned16(lse_part) || !aligned16(out_acc) ||
      !aligned16(lse_acc) || (out_final != nullptr && !aligned16(out_final)))
    return fail(SWA_ERR_INVALID_ARGUMENT,
                "out_part, lse_part, out_acc, lse_acc must be non-null and 16-byte aligned "
                "(out_final too, when given)");
  int launches = 0;
  cudaError_t e = swa::launch_attn_merge(dt, out_part, lse_part, out_acc, lse_acc, out_final,
                                         rows, first ? 1 : 0, static_cast<cudaStream_t>(stream),
                                         &launches);
  if (e != cudaSuccess) return cuda_fail(e, "attn_merge");
  t_launches = launches;
  return SWA_OK;
}

swa_status swa_f32_to_bf16(const float* src, void* dst, int64_t n, void* stream) {
  t_msg[0] = 0;
  t_launches = 0;
  if (n < 8 || n % 8 != 0 || n > ((int64_t)1 << 40))
    return fail(SWA_ERR_INVALID_ARGUMENT, "n must be a positive multiple of 8 (got %lld)",
                (long long)n);
  if (!aligned16(src) || !aligned16(dst))
    return fail(SWA_ERR_INVALID_ARGUMENT, "src, dst must be non-null and 16-byte aligned");
  int launches = 0;
  cudaError_t e = swa::launch_f32_to_bf16(src, dst, n, static_cast<cudaStream_t>(stream),
                                          &launches);
  if (e != cudaSuccess) return cuda_fail(e, "f32_to_bf16");
  t_launches = launches;
  return SWA_OK;
}

swa_status swa_get_device_error(void* stream) {
  t_msg[0] = 0;
  swa_status st;
  unsigned* err = device_error_word(&st);
  if (!err) return st;
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
  unsigned word = 0;
  e = cudaMemcpy(&word, err, sizeof(word), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e, "read error word");
  if (word != 0) {
    const unsigned zero = 0;
    e = cudaMemcpy(err, &zero, sizeof(zero), cudaMemcpyHostToDevice);
    if (e != cudaSuccess) return cuda_fail(e, "clear error word");
    return fail(SWA_ERR_DEVICE_TIMEOUT, "a kernel gave up a bounded wait (device code %u)", word);
  }
  return SWA_OK;
}

const char* swa_status_string(swa_status status) {
  switch (status) {
    case SWA_OK: return "SWA_OK";
    case SWA_ERR_INVALID_ARGUMENT: return "SWA_ERR_INVALID_ARGUMENT";
    case SWA_ERR_UNSUPPORTED: return "SWA_ERR_UNSUPPORTED";
    case SWA_ERR_CUDA: return "SWA_ERR_CUDA";
    case SWA_ERR_DEVICE_TIMEOUT: return "SWA_ERR_DEVICE_TIMEOUT";
  }
  return "SWA_ERR_UNKNOWN";
}

const char* swa_last_error_message(void) { return t_msg; }

int swa_last_launch_count(void) { return t_launches; }

void swa_profile_kernel(swa_kernel which, void* start_event, void* stop_event) {
  if (which == SWA_KERNEL_NONE || !start_event || !stop_event) {
    t_prof = Prof{};
    return;
  }
  t_prof.which = which;
  t_prof.start = static_cast<cudaEvent_t>(start_event);
  t_prof.stop = static_cast<cudaEvent_t>(stop_event);
}

}  // extern "C"
