// common.cuh -- small device helpers shared by the kernels of this library.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace rwkv7 {

constexpr int kN = 64;  // head size; the pages fix it at 64 (compile-time -D_N_=64)

// Device error word: kernels that give up on a bounded wait store a nonzero
// code through the pointer they are given (the library's word, defined in
// rwkv7_api.cu); the host reads and clears it in rwkv7_get_last_error().
// kDevErrDomain: a chunked-prefill kernel met a chunk whose decay product lies outside what it can
// factorise (its results for that call are not valid).
enum DeviceError : int { kDevErrNone = 0, kDevErrTimeout = 1, kDevErrDomain = 2 };

__device__ __forceinline__ void report_device_error(int *word, int code) {
  if (word != nullptr) atomicCAS(word, 0, code);
}

// ---- element conversions ---------------------------------------------------
__device__ __forceinline__ float bf16_bits_to_float(uint16_t b) {
  return __uint_as_float(static_cast<uint32_t>(b) << 16);
}
__device__ __forceinline__ uint16_t float_to_bf16_bits(float f) {
  __nv_bfloat16 h = __float2bfloat16_rn(f);
  return *reinterpret_cast<uint16_t *>(&h);
}

// Storage-type traits: float32 or bfloat16 bit patterns.
template <typename T> struct Elem;
template <> struct Elem<float> {
  static __device__ __forceinline__ float load(const float *p) { return *p; }
  static __device__ __forceinline__ void store(float *p, float v) { *p = v; }
  // four consecutive elements (16-byte aligned for float)
  static __device__ __forceinline__ void load4(const float *p, float out[4]) {
    float4 v = *reinterpret_cast<const float4 *>(p);
    out[0] = v.x; out[1] = v.y; out[2] = v.z; out[3] = v.w;
  }
};
template <> struct Elem<uint16_t> {
  static __device__ __forceinline__ float load(const uint16_t *p) { return bf16_bits_to_float(*p); }
  static __device__ __forceinline__ void store(uint16_t *p, float v) { *p = float_to_bf16_bits(v); }
  // four consecutive elements (8-byte aligned)
  static __device__ __forceinline__ void load4(const uint16_t *p, float out[4]) {
    uint2 v = *reinterpret_cast<const uint2 *>(p);
    out[0] = __uint_as_float(v.x << 16);
    out[1] = __uint_as_float(v.x & 0xffff0000u);
    out[2] = __uint_as_float(v.y << 16);
    out[3] = __uint_as_float(v.y & 0xffff0000u);
  }
};

// ---- the x070 operand prologue for model-native inputs --------------------------
// RWKV-7 G0 7.2B walkthrough, lshu.cn/news/198401, section 7.1: the decay comes from its
// pre-activation x as exp(-exp(-softplus(-x) - 0.5)), which equals exp(-e^-0.5 sigmoid(x)) because
// exp(-softplus(-x)) = sigmoid(x); the in-context learning rate is sigmoid(x_a); the key scaled by
// k_k and L2-normalised over the head gives kk, and the recurrence takes a = -kk, b = kk * rate
// (k itself enters unchanged).  Computed in float32 from the bf16 inputs.
__device__ __forceinline__ float x070_sigmoid(float x) { return __fdividef(1.f, 1.f + __expf(-x)); }
__device__ __forceinline__ float x070_decay(float xw) { return __expf(-0.60653065971263342f * x070_sigmoid(xw)); }
// 1 / max(||x||, 1e-12) from the sum of squares (the divisor of the L2 normalisation)
__device__ __forceinline__ float x070_inv_norm(float sumsq) { return rsqrtf(fmaxf(sumsq, 1e-24f)); }

// ---- the x070 ln_x epilogue: GroupNorm with one group per head, eps 64e-5 ----------
// (lshu.cn/news/198401, section 7.1).  y_n = (y - mean) / sqrt(var + eps) * ln_w + ln_b over the 64
// channels of a token-head, variance with divisor 64.
constexpr float kLnEps = 64e-5f;

// Mean and variance of the 64 values held two per lane (x0, x1) by a full warp.
__device__ __forceinline__ void warp_mean_var64(float x0, float x1, float &mean, float &var) {
  float s = x0 + x1;
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
  mean = s * (1.f / 64.f);
  const float d0 = x0 - mean, d1 = x1 - mean;
  float q = d0 * d0 + d1 * d1;
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) q += __shfl_xor_sync(0xffffffffu, q, off);
  var = q * (1.f / 64.f);
}

// ---- cp.async (16-byte, L2-only) ---------------------------------------------
// Programmatic dependent launch.  pdl_wait: the grid launched before this one in the stream (if
// this launch allowed overlap with it) has completed and its memory is visible; a no-op otherwise.
// pdl_trigger: the next grid in the stream may start launching once every CTA of this grid has
// called it or exited (it still waits in its own pdl_wait before touching memory).
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;\n" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory"); }

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void cp_async16(void *smem_dst, const void *gmem_src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(smem_u32(smem_dst)), "l"(gmem_src)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
template <int N> __device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory");
}

// Sequence bounds for row b: fixed-length batches use start = b*T, len = T;
// ragged batches read them from the device offsets.  A row whose offsets are
// out of range gets len = -1 and is skipped by the caller.
struct SeqBounds {
  long long start;
  int len;
};
__device__ __forceinline__ SeqBounds seq_bounds(const int32_t *cu_seqlens, int b, int T, long long total_T) {
  SeqBounds sb;
  if (cu_seqlens == nullptr) {
    sb.start = static_cast<long long>(b) * T;
    sb.len = T;
  } else {
    const long long lo = cu_seqlens[b], hi = cu_seqlens[b + 1];
    if (lo < 0 || hi < lo || hi > total_T) {
      sb.start = 0;
      sb.len = -1;
    } else {
      sb.start = lo;
      sb.len = static_cast<int>(hi - lo);
    }
  }
  return sb;
}

}  // namespace rwkv7
