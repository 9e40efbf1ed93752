// rwkv7_api.cu -- the extern "C" entry points declared in include/rwkv7.h:
// host-side argument checks, kernel choice and launches.  Nothing here
// allocates memory or synchronises; apart from the host-buffer prefill, which
// queues copies between the caller's host and device buffers around the
// launches, nothing here touches the data: every step of the computation runs
// in the kernels.
#include <mutex>

#include "../../include/rwkv7.h"
#include "common.cuh"
#include "launch.h"

namespace rwkv7 {

__device__ int g_error_word = 0;

namespace {

constexpr int kVersion = 200;  // 0.2.0: adds the host-buffer prefill

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

template <typename... P> bool all_aligned(const P *...ps) { return (aligned16(ps) && ...); }
template <typename... P> bool none_null(const P *...ps) { return ((ps != nullptr) && ...); }

rwkv7_status from_cuda(cudaError_t e) { return e == cudaSuccess ? RWKV7_OK : RWKV7_ERR_CUDA; }

// Device address of the error word on the current device (looked up once per device; the cache is
// shared by host threads, so it is read and filled under a lock).
int *error_word_ptr() {
  static int *cache[64] = {};
  static std::mutex mu;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return nullptr;
  const bool cached = dev >= 0 && dev < 64;
  std::lock_guard<std::mutex> lock(mu);
  if (cached && cache[dev] != nullptr) return cache[dev];
  void *p = nullptr;
  if (cudaGetSymbolAddress(&p, g_error_word) != cudaSuccess) return nullptr;
  if (cached) cache[dev] = static_cast<int *>(p);
  return static_cast<int *>(p);
}

// Kernel choice for bf16 prefill.  AUTO takes the chunked tensor-core kernel from
// 48 tokens on.  Measured on B200 (scan / chunk, us per call): B1 H12 T32 15.8 / 16.3,
// T64 20.9 / 21.0, T96 29.1 / 21.1; B8 H12 T32 15.7 / 16.4, T48 22.1 / 16.6, T64
// 27.7 / 16.6; B64 H32 T32 181 / 164, T48 270 / 166, T64 355 / 167; B256 H16 T16
// 189 / 317, T48 528 / 321, T127 1371 / 538.  Below that the sequential scan is as
// fast or faster: its per-token chain is short and it has no set-up.
constexpr long long kChunkMinT = 48;
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

int *device_error_word() { return error_word_ptr(); }

// The two internal streams of the host-buffer prefill on the current device (kernels; device -> host
// copies), created on first use and kept for the life of the process, so a call does not pay for
// creating and destroying streams.  Calls on one device share them: their work is ordered on them,
// and each call's own order comes from its events.
cudaError_t host_prefill_streams(cudaStream_t &ks, cudaStream_t &os) {
  static cudaStream_t cache[64][2] = {};
  static std::mutex mu;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(mu);
  for (int i = 0; i < 2; ++i)
    if (cache[dev][i] == nullptr) {
      e = cudaStreamCreateWithFlags(&cache[dev][i], cudaStreamNonBlocking);
      if (e != cudaSuccess) {
        cache[dev][i] = nullptr;
        return e;
      }
    }
  ks = cache[dev][0];
  os = cache[dev][1];
  return cudaSuccess;
}
bool prefill_uses_chunk(int path, long long max_T) { return use_chunk(path, max_T); }

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
    case RWKV7_ERR_DOMAIN: return "decay product of a chunk outside the chunked kernel's range (outputs invalid)";
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
  if (word == kDevErrNone) return RWKV7_OK;
  // A launch that gave up may have left chain flags raised (a later replay of a captured launch has
  // the same epoch and would take them for its own), and the word keeps only the first error of a
  // sequence of launches: after any recorded error, zero all flags before anything runs again.
  if (clear_chain_flags() != cudaSuccess) return RWKV7_ERR_CUDA;
  return word == kDevErrDomain ? RWKV7_ERR_DOMAIN : RWKV7_ERR_TIMEOUT;
}

rwkv7_status rwkv7_test_set_wait_hooks(unsigned max_polls, long long skip_publish_pair) {
  set_chunk_test_hooks(max_polls, skip_publish_pair);
  return RWKV7_OK;
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

rwkv7_status rwkv7_wkv_prefill_host_bf16(int path, int B, int T, int H, int N, const uint16_t *r, const uint16_t *w,
                                         const uint16_t *k, const uint16_t *v, const uint16_t *a, const uint16_t *b,
                                         const float *s_in, uint16_t *y, float *s_out, uint16_t *dev_r,
                                         uint16_t *dev_w, uint16_t *dev_k, uint16_t *dev_v, uint16_t *dev_a,
                                         uint16_t *dev_b, float *dev_s_in, uint16_t *dev_y, float *dev_s_out,
                                         int slices, rwkv7_stream_t stream) {
  if (path != RWKV7_PATH_AUTO && path != RWKV7_PATH_SCAN && path != RWKV7_PATH_CHUNK) return RWKV7_ERR_INVALID;
  rwkv7_status st = check_prefill(B, T, H, N, r, w, k, v, a, b, s_in, y, s_out);
  if (st != RWKV7_OK) return st;
  st = check_prefill(B, T, H, N, dev_r, dev_w, dev_k, dev_v, dev_a, dev_b, dev_s_in, dev_y, dev_s_out);
  if (st != RWKV7_OK) return st;
  if (slices < 0 || (s_in != nullptr && dev_s_in == nullptr)) return RWKV7_ERR_INVALID;
  // default: 4 slices (B200 over PCIe, B8 T4096 H12: 4.79 / 5.07 / 5.17 / 5.09 / 5.10 M tokens/s end
  // to end with 1 / 2 / 4 / 8 / 16 slices; the host -> device copies bound it)
  const int ns = slices == 0 ? (B < 4 ? B : 4) : (slices < B ? slices : B);
  const bool chunk = use_chunk(path, T);
  cudaStream_t user = reinterpret_cast<cudaStream_t>(stream);
  const uint16_t *hops[6] = {r, w, k, v, a, b};
  uint16_t *dops[6] = {dev_r, dev_w, dev_k, dev_v, dev_a, dev_b};
  const long long row_elems = static_cast<long long>(T) * H * kN;  // operand elements per batch row
  const long long row_state = static_cast<long long>(H) * kN * kN;  // state elements per batch row
  // host -> device copies on `stream`; the prefill on `ks`; device -> host copies on `os`
  cudaStream_t ks = nullptr, os = nullptr;
  cudaEvent_t ev_in = nullptr, ev_k = nullptr, ev_done = nullptr;
  cudaError_t e = host_prefill_streams(ks, os);
  if (e == cudaSuccess) e = cudaEventCreateWithFlags(&ev_done, cudaEventDisableTiming);
  for (int i = 0; i < ns && e == cudaSuccess; ++i) {
    const int b0 = static_cast<int>(static_cast<long long>(B) * i / ns);
    const int b1 = static_cast<int>(static_cast<long long>(B) * (i + 1) / ns);
    const int nb = b1 - b0;
    const size_t op_bytes = static_cast<size_t>(nb * row_elems) * sizeof(uint16_t);
    const size_t st_bytes = static_cast<size_t>(nb * row_state) * sizeof(float);
    const long long oo = b0 * row_elems, so = b0 * row_state;
    // one event pair per slice, released by the runtime once the work that records them is done
    e = cudaEventCreateWithFlags(&ev_in, cudaEventDisableTiming);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&ev_k, cudaEventDisableTiming);
    for (int q = 0; q < 6 && e == cudaSuccess && op_bytes > 0; ++q)
      e = cudaMemcpyAsync(dops[q] + oo, hops[q] + oo, op_bytes, cudaMemcpyHostToDevice, user);
    if (e == cudaSuccess && s_in != nullptr)
      e = cudaMemcpyAsync(dev_s_in + so, s_in + so, st_bytes, cudaMemcpyHostToDevice, user);
    if (e == cudaSuccess) e = cudaEventRecord(ev_in, user);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(ks, ev_in, 0);
    if (e == cudaSuccess) {
      const uint16_t *dr = dev_r + oo, *dw = dev_w + oo, *dk = dev_k + oo, *dv = dev_v + oo, *da = dev_a + oo,
                     *db = dev_b + oo;
      const float *dsi = s_in != nullptr ? dev_s_in + so : nullptr;
      const long long total = static_cast<long long>(nb) * T;
      e = chunk ? launch_chunk(dr, dw, dk, dv, da, db, dsi, dev_y + oo, dev_s_out + so, nullptr, nb, T, total, H,
                               error_word_ptr(), ks)
                : launch_scan<uint16_t>(dr, dw, dk, dv, da, db, dsi, dev_y + oo, dev_s_out + so, nullptr, nb, T, total,
                                        H, ks);
    }
    if (e == cudaSuccess) e = cudaEventRecord(ev_k, ks);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(os, ev_k, 0);
    if (e == cudaSuccess && op_bytes > 0)
      e = cudaMemcpyAsync(y + oo, dev_y + oo, op_bytes, cudaMemcpyDeviceToHost, os);
    if (e == cudaSuccess) e = cudaMemcpyAsync(s_out + so, dev_s_out + so, st_bytes, cudaMemcpyDeviceToHost, os);
    if (ev_in != nullptr) cudaEventDestroy(ev_in);
    if (ev_k != nullptr) cudaEventDestroy(ev_k);
    ev_in = ev_k = nullptr;
  }
  // `stream` waits for the last device -> host copy (the copies on `os` run in order)
  if (e == cudaSuccess) e = cudaEventRecord(ev_done, os);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(user, ev_done, 0);
  if (ev_done != nullptr) cudaEventDestroy(ev_done);
  return from_cuda(e);
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
  return from_cuda(launch_decode_ext(r, w, k, v, a, b, false, nullptr, false, nullptr, nullptr, false, s_inout, y, B,
                                     H, reinterpret_cast<cudaStream_t>(stream)));
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
  if (schedule < 0 || schedule > 3) return RWKV7_ERR_INVALID;
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
  const bool early = opt != nullptr && opt->independent_state != 0;
  return from_cuda(launch_decode_ext(r, w, k, v, a, b, native, k_k, ln, ln_w, ln_b, early, s_inout, y, B, H,
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
  return from_cuda(
      launch_decode_bf16state(r, w, k, v, a, b, false, s_inout, y, B, H, reinterpret_cast<cudaStream_t>(stream)));
}

rwkv7_status rwkv7_wkv_decode_ext_bf16state(int B, int H, int N, const uint16_t *r, const uint16_t *w,
                                            const uint16_t *k, const uint16_t *v, const uint16_t *a,
                                            const uint16_t *b, const rwkv7_options *opt, uint16_t *s_inout,
                                            uint16_t *y, rwkv7_stream_t stream) {
  if (opt != nullptr && (opt->model_native != 0 || opt->group_norm != 0)) return RWKV7_ERR_INVALID;
  if (N != kN) return RWKV7_ERR_UNSUPPORTED;
  if (B <= 0 || H <= 0 || !none_null(r, w, k, v, a, b, s_inout, y)) return RWKV7_ERR_INVALID;
  if (!all_aligned(r, w, k, v, a, b, s_inout, y)) return RWKV7_ERR_ALIGN;
  const bool early = opt != nullptr && opt->independent_state != 0;
  return from_cuda(
      launch_decode_bf16state(r, w, k, v, a, b, early, s_inout, y, B, H, reinterpret_cast<cudaStream_t>(stream)));
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
