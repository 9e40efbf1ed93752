// rwkv7_api.cu -- the extern "C" entry points declared in include/rwkv7.h:
// host-side argument checks, kernel choice and launches.  Nothing here
// allocates, synchronises or touches the data; every step of the computation
// runs in the kernels.
#include "../../include/rwkv7.h"
#include "common.cuh"
#include "launch.h"

namespace rwkv7 {

__device__ int g_error_word = 0;

namespace {

constexpr int kVersion = 100;  // 0.1.0

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

template <typename... P> bool all_aligned(const P *...ps) { return (aligned16(ps) && ...); }
template <typename... P> bool none_null(const P *...ps) { return ((ps != nullptr) && ...); }

rwkv7_status from_cuda(cudaError_t e) { return e == cudaSuccess ? RWKV7_OK : RWKV7_ERR_CUDA; }

// Device address of the error word on the current device (looked up once per device).
int *error_word_ptr() {
  static int *cache[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return nullptr;
  if (dev >= 0 && dev < 64 && cache[dev] != nullptr) return cache[dev];
  void *p = nullptr;
  if (cudaGetSymbolAddress(&p, g_error_word) != cudaSuccess) return nullptr;
  if (dev >= 0 && dev < 64) cache[dev] = static_cast<int *>(p);
  return static_cast<int *>(p);
}

// Kernel choice for bf16 prefill.  AUTO takes the chunked tensor-core kernel
// once a sequence spans two chunks; shorter ones are latency-bound either way
// and the sequential scan has no set-up cost.
constexpr long long kChunkMinT = 128;
bool use_chunk(int path, long long max_T) {
  return path == RWKV7_PATH_CHUNK || (path == RWKV7_PATH_AUTO && max_T >= kChunkMinT);
}

// Checks shared by every prefill entry point.  `need_ops` is false when no
// token is processed (T == 0), in which case operand pointers may be NULL.
template <typename TIn>
rwkv7_status check_prefill(int B, long long tokens, int H, int N, const TIn *r, const TIn *w, const TIn *k,
                           const TIn *v, const TIn *a, const TIn *b, const float *s_in, const TIn *y,
                           const float *s_out) {
  if (N != kN) return RWKV7_ERR_UNSUPPORTED;
  if (B <= 0 || H <= 0 || tokens < 0) return RWKV7_ERR_INVALID;
  if (s_out == nullptr) return RWKV7_ERR_INVALID;
  const bool need_ops = tokens > 0;
  if (need_ops && !none_null(r, w, k, v, a, b, y)) return RWKV7_ERR_INVALID;
  if (!all_aligned(r, w, k, v, a, b, y, s_in, s_out)) return RWKV7_ERR_ALIGN;
  if (static_cast<long long>(B) > 65535) return RWKV7_ERR_INVALID;  // grid.y limit of the launches
  return RWKV7_OK;
}

}  // namespace
}  // namespace rwkv7

using namespace rwkv7;

extern "C" {

const char *rwkv7_status_string(rwkv7_status status) {
  switch (status) {
    case RWKV7_OK: return "ok";
    case RWKV7_ERR_INVALID: return "invalid argument";
    case RWKV7_ERR_ALIGN: return "pointer not 16-byte aligned";
    case RWKV7_ERR_CUDA: return "CUDA error";
    case RWKV7_ERR_TIMEOUT: return "device wait timed out";
    case RWKV7_ERR_UNSUPPORTED: return "unsupported size (head size must be 64)";
  }
  return "unknown status";
}

int rwkv7_version(void) { return kVersion; }

rwkv7_status rwkv7_get_last_error(void) {
  if (cudaDeviceSynchronize() != cudaSuccess) return RWKV7_ERR_CUDA;
  int word = 0;
  const int zero = 0;
  if (cudaMemcpyFromSymbol(&word, g_error_word, sizeof(int)) != cudaSuccess) return RWKV7_ERR_CUDA;
  if (word != 0 && cudaMemcpyToSymbol(g_error_word, &zero, sizeof(int)) != cudaSuccess) return RWKV7_ERR_CUDA;
  if (cudaGetLastError() != cudaSuccess) return RWKV7_ERR_CUDA;
  return word == kDevErrNone ? RWKV7_OK : RWKV7_ERR_TIMEOUT;
}

rwkv7_status rwkv7_wkv_prefill(int B, int T, int H, int N, const float *r, const float *w, const float *k,
                               const float *v, const float *a, const float *b, const float *s_in, float *y,
                               float *s_out, rwkv7_stream_t stream) {
  const rwkv7_status st = check_prefill(B, T, H, N, r, w, k, v, a, b, s_in, y, s_out);
  if (st != RWKV7_OK) return st;
  return from_cuda(launch_scan<float>(r, w, k, v, a, b, s_in, y, s_out, nullptr, B, T,
                                      static_cast<long long>(B) * T, H, reinterpret_cast<cudaStream_t>(stream)));
}

rwkv7_status rwkv7_wkv_prefill_bf16_path(int path, int B, int T, int H, int N, const uint16_t *r, const uint16_t *w,
                                         const uint16_t *k, const uint16_t *v, const uint16_t *a, const uint16_t *b,
                                         const float *s_in, uint16_t *y, float *s_out, rwkv7_stream_t stream) {
  if (path != RWKV7_PATH_AUTO && path != RWKV7_PATH_SCAN && path != RWKV7_PATH_CHUNK) return RWKV7_ERR_INVALID;
  const rwkv7_status st = check_prefill(B, T, H, N, r, w, k, v, a, b, s_in, y, s_out);
  if (st != RWKV7_OK) return st;
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  const long long total = static_cast<long long>(B) * T;
  if (use_chunk(path, T))
    return from_cuda(launch_chunk(r, w, k, v, a, b, s_in, y, s_out, nullptr, B, T, total, H, error_word_ptr(), cs));
  return from_cuda(launch_scan<uint16_t>(r, w, k, v, a, b, s_in, y, s_out, nullptr, B, T, total, H, cs));
}

rwkv7_status rwkv7_wkv_prefill_bf16(int B, int T, int H, int N, const uint16_t *r, const uint16_t *w,
                                    const uint16_t *k, const uint16_t *v, const uint16_t *a, const uint16_t *b,
                                    const float *s_in, uint16_t *y, float *s_out, rwkv7_stream_t stream) {
  return rwkv7_wkv_prefill_bf16_path(RWKV7_PATH_AUTO, B, T, H, N, r, w, k, v, a, b, s_in, y, s_out, stream);
}

rwkv7_status rwkv7_wkv_prefill_varlen_bf16(int path, int B, int total_T, int max_T, int H, int N,
                                           const int32_t *cu_seqlens, const uint16_t *r, const uint16_t *w,
                                           const uint16_t *k, const uint16_t *v, const uint16_t *a,
                                           const uint16_t *b, const float *s_in, uint16_t *y, float *s_out,
                                           rwkv7_stream_t stream) {
  if (path != RWKV7_PATH_AUTO && path != RWKV7_PATH_SCAN && path != RWKV7_PATH_CHUNK) return RWKV7_ERR_INVALID;
  if (max_T < 0 || cu_seqlens == nullptr || !aligned16(cu_seqlens)) {
    if (cu_seqlens != nullptr && !aligned16(cu_seqlens) && max_T >= 0) return RWKV7_ERR_ALIGN;
    return RWKV7_ERR_INVALID;
  }
  const rwkv7_status st = check_prefill(B, total_T, H, N, r, w, k, v, a, b, s_in, y, s_out);
  if (st != RWKV7_OK) return st;
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  if (use_chunk(path, max_T))
    return from_cuda(
        launch_chunk(r, w, k, v, a, b, s_in, y, s_out, cu_seqlens, B, 0, total_T, H, error_word_ptr(), cs));
  return from_cuda(launch_scan<uint16_t>(r, w, k, v, a, b, s_in, y, s_out, cu_seqlens, B, 0, total_T, H, cs));
}

rwkv7_status rwkv7_wkv_decode(int B, int H, int N, const float *r, const float *w, const float *k, const float *v,
                              const float *a, const float *b, float *s_inout, float *y, rwkv7_stream_t stream) {
  if (N != kN) return RWKV7_ERR_UNSUPPORTED;
  if (B <= 0 || H <= 0 || !none_null(r, w, k, v, a, b, s_inout, y)) return RWKV7_ERR_INVALID;
  if (!all_aligned(r, w, k, v, a, b, s_inout, y)) return RWKV7_ERR_ALIGN;
  return from_cuda(launch_decode<float>(r, w, k, v, a, b, s_inout, y, B, H, reinterpret_cast<cudaStream_t>(stream)));
}

rwkv7_status rwkv7_wkv_decode_bf16(int B, int H, int N, const uint16_t *r, const uint16_t *w, const uint16_t *k,
                                   const uint16_t *v, const uint16_t *a, const uint16_t *b, float *s_inout,
                                   uint16_t *y, rwkv7_stream_t stream) {
  if (N != kN) return RWKV7_ERR_UNSUPPORTED;
  if (B <= 0 || H <= 0 || !none_null(r, w, k, v, a, b, s_inout, y)) return RWKV7_ERR_INVALID;
  if (!all_aligned(r, w, k, v, a, b, s_inout, y)) return RWKV7_ERR_ALIGN;
  return from_cuda(launch_decode_ext(r, w, k, v, a, b, false, nullptr, false, nullptr, nullptr, s_inout, y, B, H,
                                     reinterpret_cast<cudaStream_t>(stream)));
}

rwkv7_status rwkv7_wkv_prefill_ext_bf16(int path, int B, int T, int H, int N, const uint16_t *r, const uint16_t *w,
                                        const uint16_t *k, const uint16_t *v, const uint16_t *a, const uint16_t *b,
                                        const rwkv7_options *opt, const float *s_in, uint16_t *y, float *s_out,
                                        rwkv7_stream_t stream) {
  if (path != RWKV7_PATH_AUTO && path != RWKV7_PATH_SCAN && path != RWKV7_PATH_CHUNK) return RWKV7_ERR_INVALID;
  const bool native = opt != nullptr && opt->model_native != 0;
  const bool ln = opt != nullptr && opt->group_norm != 0;
  const float *k_k = native ? opt->k_k : nullptr;
  const float *ln_w = ln ? opt->ln_w : nullptr, *ln_b = ln ? opt->ln_b : nullptr;
  const int schedule = opt != nullptr ? opt->chunk_schedule : 0;
  if (schedule < 0 || schedule > 2) return RWKV7_ERR_INVALID;
  // model-native calls have no b: the shared checks see a in its place
  const rwkv7_status st = check_prefill(B, T, H, N, r, w, k, v, a, native ? a : b, s_in, y, s_out);
  if (st != RWKV7_OK) return st;
  if (!all_aligned(k_k, ln_w, ln_b)) return RWKV7_ERR_ALIGN;
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  const long long total = static_cast<long long>(B) * T;
  if (use_chunk(path, T))
    return from_cuda(launch_chunk_ext(r, w, k, v, a, b, native, k_k, ln, ln_w, ln_b, s_in, y, s_out, nullptr, B, T,
                                      total, H, schedule, nullptr, error_word_ptr(), cs));
  return from_cuda(
      launch_scan_ext(r, w, k, v, a, b, native, k_k, ln, ln_w, ln_b, s_in, y, s_out, nullptr, B, T, total, H, cs));
}

rwkv7_status rwkv7_wkv_decode_ext_bf16(int B, int H, int N, const uint16_t *r, const uint16_t *w, const uint16_t *k,
                                       const uint16_t *v, const uint16_t *a, const uint16_t *b,
                                       const rwkv7_options *opt, float *s_inout, uint16_t *y,
                                       rwkv7_stream_t stream) {
  const bool native = opt != nullptr && opt->model_native != 0;
  const bool ln = opt != nullptr && opt->group_norm != 0;
  const float *k_k = native ? opt->k_k : nullptr;
  const float *ln_w = ln ? opt->ln_w : nullptr, *ln_b = ln ? opt->ln_b : nullptr;
  if (N != kN) return RWKV7_ERR_UNSUPPORTED;
  if (B <= 0 || H <= 0 || !none_null(r, w, k, v, a, s_inout, y) || (!native && b == nullptr))
    return RWKV7_ERR_INVALID;
  if (!all_aligned(r, w, k, v, a, b, s_inout, y, k_k, ln_w, ln_b)) return RWKV7_ERR_ALIGN;
  return from_cuda(launch_decode_ext(r, w, k, v, a, b, native, k_k, ln, ln_w, ln_b, s_inout, y, B, H,
                                     reinterpret_cast<cudaStream_t>(stream)));
}

rwkv7_status rwkv7_wkv_prefill_fused_bf16(int path, int B, int T, int H, int N, const uint16_t *r,
                                          const uint16_t *xw, const uint16_t *k, const uint16_t *v,
                                          const uint16_t *xa, const float *k_k, const float *s_in, uint16_t *y,
                                          float *s_out, rwkv7_stream_t stream) {
  const rwkv7_options opt{1, k_k, 0, nullptr, nullptr, 0};
  return rwkv7_wkv_prefill_ext_bf16(path, B, T, H, N, r, xw, k, v, xa, nullptr, &opt, s_in, y, s_out, stream);
}

rwkv7_status rwkv7_wkv_decode_fused_bf16(int B, int H, int N, const uint16_t *r, const uint16_t *xw,
                                         const uint16_t *k, const uint16_t *v, const uint16_t *xa, const float *k_k,
                                         float *s_inout, uint16_t *y, rwkv7_stream_t stream) {
  const rwkv7_options opt{1, k_k, 0, nullptr, nullptr, 0};
  return rwkv7_wkv_decode_ext_bf16(B, H, N, r, xw, k, v, xa, nullptr, &opt, s_inout, y, stream);
}

rwkv7_status rwkv7_wkv_decode_bf16_bf16state(int B, int H, int N, const uint16_t *r, const uint16_t *w,
                                             const uint16_t *k, const uint16_t *v, const uint16_t *a,
                                             const uint16_t *b, uint16_t *s_inout, uint16_t *y,
                                             rwkv7_stream_t stream) {
  if (N != kN) return RWKV7_ERR_UNSUPPORTED;
  if (B <= 0 || H <= 0 || !none_null(r, w, k, v, a, b, s_inout, y)) return RWKV7_ERR_INVALID;
  if (!all_aligned(r, w, k, v, a, b, s_inout, y)) return RWKV7_ERR_ALIGN;
  return from_cuda(launch_decode_bf16state(r, w, k, v, a, b, s_inout, y, B, H, reinterpret_cast<cudaStream_t>(stream)));
}

rwkv7_status rwkv7_wkv_prefill_save_bf16(int path, int B, int T, int H, int N, const uint16_t *r,
                                         const uint16_t *w, const uint16_t *k, const uint16_t *v, const uint16_t *a,
                                         const uint16_t *b, const float *s_in, uint16_t *y, float *s_out,
                                         float *states, rwkv7_stream_t stream) {
  if (path != RWKV7_PATH_AUTO && path != RWKV7_PATH_SCAN && path != RWKV7_PATH_CHUNK) return RWKV7_ERR_INVALID;
  const rwkv7_status st = check_prefill(B, T, H, N, r, w, k, v, a, b, s_in, y, s_out);
  if (st != RWKV7_OK) return st;
  if (T > 0 && states == nullptr) return RWKV7_ERR_INVALID;
  if (!aligned16(states)) return RWKV7_ERR_ALIGN;
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  if (use_chunk(path, T))
    return from_cuda(launch_chunk_ext(r, w, k, v, a, b, false, nullptr, false, nullptr, nullptr, s_in, y, s_out,
                                      nullptr, B, T, static_cast<long long>(B) * T, H, 0, states, error_word_ptr(),
                                      cs));
  return from_cuda(launch_scan_save(r, w, k, v, a, b, s_in, y, s_out, states, B, T, H, cs));
}

rwkv7_status rwkv7_wkv_backward_bf16(int B, int T, int H, int N, const uint16_t *r, const uint16_t *w,
                                     const uint16_t *k, const uint16_t *v, const uint16_t *a, const uint16_t *b,
                                     const float *states, const uint16_t *dy, const float *ds_out, float *dr,
                                     float *dw, float *dk, float *dv, float *da, float *db, float *ds_in,
                                     rwkv7_stream_t stream) {
  if (N != kN) return RWKV7_ERR_UNSUPPORTED;
  if (B <= 0 || H <= 0 || T < 0 || B > 65535 || H > 0xffff) return RWKV7_ERR_INVALID;
  if (T > 0 && !none_null(r, w, k, v, a, b, states, dy, dr, dw, dk, dv, da, db)) return RWKV7_ERR_INVALID;
  if (!all_aligned(r, w, k, v, a, b, dy, dr, dw, dk, dv, da, db) || !all_aligned(states, ds_out, ds_in))
    return RWKV7_ERR_ALIGN;
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  const size_t bytes = sizeof(float) * static_cast<size_t>(B) * T * H * kN;
  if (T > 0) {
    // the column sums arrive from several row groups: these five are accumulated
    for (float *g : {dr, dw, dk, da, db})
      if (cudaMemsetAsync(g, 0, bytes, cs) != cudaSuccess) return RWKV7_ERR_CUDA;
  } else if (ds_in != nullptr) {
    const size_t sb = sizeof(float) * static_cast<size_t>(B) * H * kN * kN;
    const cudaError_t e = ds_out ? cudaMemcpyAsync(ds_in, ds_out, sb, cudaMemcpyDeviceToDevice, cs)
                                 : cudaMemsetAsync(ds_in, 0, sb, cs);
    return from_cuda(e);
  } else {
    return RWKV7_OK;
  }
  return from_cuda(launch_backward(r, w, k, v, a, b, states, dy, ds_out, dr, dw, dk, dv, da, db, ds_in, B, T, H, cs));
}

}  // extern "C"
