// rwkv7_noalloc.cu -- the host-buffer bf16 prefill for callers that cannot allocate device memory.
//
// rwkv7_wkv_prefill_host_bf16 stages its host operands through device buffers that the caller
// allocates.  This entry point stages them instead through one array that the library itself
// holds in static device memory (reserved once per GPU when the library's module is loaded, kept
// until the process exits), so a call allocates nothing.  It copies the operands (and the initial
// state) into that array, runs the same prefill kernels as the other entry points on it, and copies
// y and the final state back, all on the caller's stream.
#include <mutex>

#include "../../include/rwkv7.h"
#include "common.cuh"
#include "launch.h"

namespace rwkv7 {

// The staging array.  Its size is the public limit RWKV7_NOALLOC_STAGING_BYTES; every call of the
// entry point reuses it, and it keeps whatever the previous call left in it.
static __device__ __align__(256) unsigned char g_noalloc_staging[RWKV7_NOALLOC_STAGING_BYTES];

namespace {

constexpr int kMaxDevices = 64;
constexpr size_t kRegionAlign = 256;

size_t round_up(size_t x) { return (x + kRegionAlign - 1) / kRegionAlign * kRegionAlign; }

// Device address of the staging array on the current device.  In host code the array's name only
// identifies the symbol; the address a kernel may use is looked up with cudaGetSymbolAddress, once
// per device (with that device current) on the first call, and cached.
unsigned char *staging_base(cudaError_t *err) {
  static std::mutex mu;
  static unsigned char *cache[kMaxDevices] = {};
  int dev = 0;
  *err = cudaGetDevice(&dev);
  if (*err != cudaSuccess) return nullptr;
  if (dev < 0 || dev >= kMaxDevices) {
    *err = cudaErrorInvalidDevice;
    return nullptr;
  }
  std::lock_guard<std::mutex> lock(mu);
  if (cache[dev] == nullptr) {
    void *p = nullptr;
    *err = cudaGetSymbolAddress(&p, g_noalloc_staging);
    if (*err != cudaSuccess) return nullptr;
    cache[dev] = static_cast<unsigned char *>(p);
  }
  return cache[dev];
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace
}  // namespace rwkv7

using namespace rwkv7;

extern "C" rwkv7_status rwkv7_wkv_prefill_host_noalloc_bf16(int path, int B, int T, int H, int N, const uint16_t *r,
                                                             const uint16_t *w, const uint16_t *k, const uint16_t *v,
                                                             const uint16_t *a, const uint16_t *b, const float *s_in,
                                                             uint16_t *y, float *s_out, rwkv7_stream_t stream) {
  if (path != RWKV7_PATH_AUTO && path != RWKV7_PATH_SCAN && path != RWKV7_PATH_CHUNK) return RWKV7_ERR_INVALID;
  if (N != kN) return RWKV7_ERR_UNSUPPORTED;
  if (B <= 0 || H <= 0 || T < 0 || B > 65535 || s_out == nullptr) return RWKV7_ERR_INVALID;
  const uint16_t *hops[6] = {r, w, k, v, a, b};
  if (T > 0) {
    for (const uint16_t *p : hops)
      if (p == nullptr) return RWKV7_ERR_INVALID;
    if (y == nullptr) return RWKV7_ERR_INVALID;
  }
  for (const void *p : {static_cast<const void *>(r), static_cast<const void *>(w), static_cast<const void *>(k),
                        static_cast<const void *>(v), static_cast<const void *>(a), static_cast<const void *>(b),
                        static_cast<const void *>(s_in), static_cast<const void *>(y),
                        static_cast<const void *>(s_out)})
    if (!aligned16(p)) return RWKV7_ERR_ALIGN;

  // staging layout: r, w, k, v, a, b, y, s_in (when given), s_out; each region 256-byte aligned
  const size_t op_bytes = sizeof(uint16_t) * static_cast<size_t>(B) * static_cast<size_t>(T) * H * kN;
  const size_t st_bytes = sizeof(float) * static_cast<size_t>(B) * H * kN * kN;
  const size_t need = 7 * round_up(op_bytes) + (s_in != nullptr ? 2 : 1) * round_up(st_bytes);
  if (need > static_cast<size_t>(RWKV7_NOALLOC_STAGING_BYTES)) return RWKV7_ERR_INVALID;

  cudaError_t e = cudaSuccess;
  unsigned char *base = staging_base(&e);
  if (base == nullptr) return RWKV7_ERR_CUDA;
  uint16_t *dops[7];
  for (int q = 0; q < 7; ++q) dops[q] = reinterpret_cast<uint16_t *>(base + q * round_up(op_bytes));
  unsigned char *st = base + 7 * round_up(op_bytes);
  float *dev_s_in = s_in != nullptr ? reinterpret_cast<float *>(st) : nullptr;
  float *dev_s_out = reinterpret_cast<float *>(s_in != nullptr ? st + round_up(st_bytes) : st);

  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  for (int q = 0; q < 6 && e == cudaSuccess && op_bytes > 0; ++q)
    e = cudaMemcpyAsync(dops[q], hops[q], op_bytes, cudaMemcpyHostToDevice, cs);
  if (e == cudaSuccess && s_in != nullptr) e = cudaMemcpyAsync(dev_s_in, s_in, st_bytes, cudaMemcpyHostToDevice, cs);
  if (e == cudaSuccess) {
    const long long total = static_cast<long long>(B) * T;
    e = prefill_uses_chunk(path, T)
            ? launch_chunk(dops[0], dops[1], dops[2], dops[3], dops[4], dops[5], dev_s_in, dops[6], dev_s_out,
                           nullptr, B, T, total, H, device_error_word(), cs)
            : launch_scan<uint16_t>(dops[0], dops[1], dops[2], dops[3], dops[4], dops[5], dev_s_in, dops[6],
                                    dev_s_out, nullptr, B, T, total, H, cs);
  }
  if (e == cudaSuccess && op_bytes > 0) e = cudaMemcpyAsync(y, dops[6], op_bytes, cudaMemcpyDeviceToHost, cs);
  if (e == cudaSuccess) e = cudaMemcpyAsync(s_out, dev_s_out, st_bytes, cudaMemcpyDeviceToHost, cs);
  return e == cudaSuccess ? RWKV7_OK : RWKV7_ERR_CUDA;
}
