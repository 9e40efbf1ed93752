// wkv7_decode.cu -- one-token step of the x070 recurrence ("RNN mode"),
// updating the float32 state in place.
//
// Operation (RWKV-7 G0 7.2B walkthrough, lshu.cn/news/198401, sections 3.2
// and 7.1: wkv7s is the single-step form of the same update):
//   sa = S a;  S = S diag(w) + sa b^T + v k^T;  y = S r.
//
// The step is bound by HBM: every (b, h) reads and writes its 16 KiB state
// once and touches only 7 vectors of 64 elements besides.  One CTA of 256
// threads owns one (b, h).  Thread t holds columns 4*(t%16) .. +3 of rows
// t/16 + 16*m (m = 0..3): four 16-byte loads per thread, issued together,
// and a warp covers two whole 256-byte rows per load.  The row sums S a and
// S r are finished with four xor-shuffles inside each 16-lane half-warp.
//
// The reduced-precision variant keeps the state in HBM as bfloat16 (8 KiB per head instead of 16):
// it is widened to float32 on load, updated in float32, and rounded to nearest-even bf16 on store.
// The pages keep the state in fp32 (RWKV-LM README copy, oa0.com/c/1004164), so this is an
// opt-in trade of state precision for half the decode traffic, not the default.
//
// The fused variant takes model-native inputs (decay pre-activation x_w in place of w, the key k,
// the learning-rate pre-activation x_a in place of a, and the per-channel key scale k_k) and forms
// w, a = -kk and b = kk * sigmoid(x_a) in-kernel; the key norm is one more 16-lane reduction.
#include <mutex>

#include "common.cuh"
#include "launch.h"

namespace rwkv7 {

template <typename TIn, typename TS = float> struct DecodeArgs {
  const TIn *r, *w, *k, *v, *a, *b;  // fused: w = x_w, a = x_a, b unused
  TS *s;
  TIn *y;
  const float *k_k;  // fused: [H, 64] key scale, nullptr = ones
  int H;
  const float *ln_w, *ln_b;  // group-norm epilogue: [H, 64] weight / bias, nullptr = ones / zeros
};

__device__ __forceinline__ float4 ld_state(const float *p) { return *reinterpret_cast<const float4 *>(p); }
__device__ __forceinline__ void st_state(float *p, float4 x) { *reinterpret_cast<float4 *>(p) = x; }
// bf16 state: four elements in 8 bytes
__device__ __forceinline__ float4 ld_state(const uint16_t *p) {
  const uint2 u = *reinterpret_cast<const uint2 *>(p);
  return make_float4(__uint_as_float(u.x << 16), __uint_as_float(u.x & 0xffff0000u), __uint_as_float(u.y << 16),
                     __uint_as_float(u.y & 0xffff0000u));
}
__device__ __forceinline__ uint32_t bf16x2_rn(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;\n" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}
__device__ __forceinline__ void st_state(uint16_t *p, float4 x) {
  *reinterpret_cast<uint2 *>(p) = make_uint2(bf16x2_rn(x.x, x.y), bf16x2_rn(x.z, x.w));
}

// kEarly (the caller's promise that no step still running before this one writes this step's state):
// the state loads go out before the wait for the previous grid, so they overlap its last wave.
template <typename TIn, bool kFused, bool kLN, bool kEarly, typename TS = float>
__global__ void __launch_bounds__(256, 5) wkv7_decode_kernel(DecodeArgs<TIn, TS> A) {
  const long long pair = blockIdx.x;  // b * H + h
  const int tid = threadIdx.x;
  // the step before may still be finishing (its launch allowed this grid to start early): every CTA
  // of this grid has started once all have passed the trigger, and none reads memory the step before
  // may write (the operands; the state too, without kEarly) before the wait
  pdl_trigger();
  if (!kEarly) pdl_wait();
  const int c4 = tid & 15;   // column chunk: columns 4*c4 .. 4*c4+3
  const int rg = tid >> 4;   // rows rg + 16*m
  TS *S = A.s + pair * (kN * kN);

  // the state loads go out first, so everything below overlaps them
  float4 st[4];
#pragma unroll
  for (int m = 0; m < 4; ++m) st[m] = ld_state(S + (rg + 16 * m) * kN + 4 * c4);
  if (kEarly) pdl_wait();

  // then every other load, before any arithmetic waits on one: a single memory round trip per CTA
  const long long vb = pair * kN;
  float ww[4], kk[4], aa[4], bb[4], rr[4], vv[4];
  Elem<TIn>::load4(A.k + vb + 4 * c4, kk);
  Elem<TIn>::load4(A.w + vb + 4 * c4, ww);  // fused: x_w
  Elem<TIn>::load4(A.a + vb + 4 * c4, aa);  // fused: x_a
  if (!kFused) Elem<TIn>::load4(A.b + vb + 4 * c4, bb);
  Elem<TIn>::load4(A.r + vb + 4 * c4, rr);
#pragma unroll
  for (int m = 0; m < 4; ++m) vv[m] = Elem<TIn>::load(A.v + vb + rg + 16 * m);
  float4 ksc = make_float4(1.f, 1.f, 1.f, 1.f);  // fused: the key scale of this thread's channels
  if (kFused && A.k_k != nullptr)
    ksc = *reinterpret_cast<const float4 *>(A.k_k + static_cast<int>(pair % A.H) * kN + 4 * c4);
  float sa[4];
  if (kFused) {
    // x070 prologue: kk = normalise(k * k_k) over the 64 channels, a = -kk, b = kk * rate, decay from
    // x_w.  S a = -(S kx) / |kx| with kx = k * k_k: the row sums of S kx and |kx|^2 share the shuffles.
    const float kscale[4] = {ksc.x, ksc.y, ksc.z, ksc.w};
    float kx[4], ss = 0.f;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      kx[e] = kk[e] * kscale[e];
      ss = fmaf(kx[e], kx[e], ss);
    }
#pragma unroll
    for (int m = 0; m < 4; ++m) {
      float p = st[m].x * kx[0];
      p = fmaf(st[m].y, kx[1], p);
      p = fmaf(st[m].z, kx[2], p);
      p = fmaf(st[m].w, kx[3], p);
      sa[m] = p;
    }
#pragma unroll
    for (int off = 8; off >= 1; off >>= 1) {
      ss += __shfl_xor_sync(0xffffffffu, ss, off);
#pragma unroll
      for (int m = 0; m < 4; ++m) sa[m] += __shfl_xor_sync(0xffffffffu, sa[m], off);
    }
    const float inv = x070_inv_norm(ss);
#pragma unroll
    for (int m = 0; m < 4; ++m) sa[m] *= -inv;
    // the decays and learning rates of this thread's 4 channels: lanes l and l ^ 16 hold the same
    // channels, so each forms two of each (lane bit 4 picks which two) and they swap the rest
    const bool upper = (tid & 16) != 0;
    float dw[2], dr[2];
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      dw[e] = x070_decay(upper ? ww[2 + e] : ww[e]);
      dr[e] = x070_sigmoid(upper ? aa[2 + e] : aa[e]);
    }
    float rate[4];
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const float ow = __shfl_xor_sync(0xffffffffu, dw[e], 16), orr = __shfl_xor_sync(0xffffffffu, dr[e], 16);
      ww[e] = upper ? ow : dw[e];
      ww[2 + e] = upper ? dw[e] : ow;
      rate[e] = upper ? orr : dr[e];
      rate[2 + e] = upper ? dr[e] : orr;
    }
#pragma unroll
    for (int e = 0; e < 4; ++e) bb[e] = kx[e] * inv * rate[e];
  } else {
#pragma unroll
    for (int m = 0; m < 4; ++m) {
      float p = st[m].x * aa[0];
      p = fmaf(st[m].y, aa[1], p);
      p = fmaf(st[m].z, aa[2], p);
      p = fmaf(st[m].w, aa[3], p);
      sa[m] = p;
    }
#pragma unroll
    for (int off = 8; off >= 1; off >>= 1)
#pragma unroll
      for (int m = 0; m < 4; ++m) sa[m] += __shfl_xor_sync(0xffffffffu, sa[m], off);
  }
  float yv[4];
#pragma unroll
  for (int m = 0; m < 4; ++m) {
    float4 x = st[m];
    x.x = fmaf(x.x, ww[0], fmaf(sa[m], bb[0], vv[m] * kk[0]));
    x.y = fmaf(x.y, ww[1], fmaf(sa[m], bb[1], vv[m] * kk[1]));
    x.z = fmaf(x.z, ww[2], fmaf(sa[m], bb[2], vv[m] * kk[2]));
    x.w = fmaf(x.w, ww[3], fmaf(sa[m], bb[3], vv[m] * kk[3]));
    st[m] = x;
    float p = x.x * rr[0];
    p = fmaf(x.y, rr[1], p);
    p = fmaf(x.z, rr[2], p);
    p = fmaf(x.w, rr[3], p);
    yv[m] = p;
  }
#pragma unroll
  for (int m = 0; m < 4; ++m) st_state(S + (rg + 16 * m) * kN + 4 * c4, st[m]);
#pragma unroll
  for (int off = 8; off >= 1; off >>= 1)
#pragma unroll
    for (int m = 0; m < 4; ++m) yv[m] += __shfl_xor_sync(0xffffffffu, yv[m], off);
  if (!kLN) {
    if (c4 == 0) {
#pragma unroll
      for (int m = 0; m < 4; ++m) Elem<TIn>::store(A.y + vb + rg + 16 * m, yv[m]);
    }
  } else {
    // ln_x: GroupNorm over the head's 64 channels of y, by warp 0 (two channels per lane)
    __shared__ float s_y[kLN ? kN : 1];
    if (c4 == 0) {
#pragma unroll
      for (int m = 0; m < 4; ++m) s_y[rg + 16 * m] = yv[m];
    }
    __syncthreads();
    if (tid < 32) {
      const float y0 = s_y[tid], y1 = s_y[tid + 32];
      float mean, var;
      warp_mean_var64(y0, y1, mean, var);
      const float rs = rsqrtf(var + kLnEps);
      const int h = static_cast<int>(pair % A.H);
      const float w0 = A.ln_w ? A.ln_w[h * kN + tid] : 1.f, w1 = A.ln_w ? A.ln_w[h * kN + tid + 32] : 1.f;
      const float b0 = A.ln_b ? A.ln_b[h * kN + tid] : 0.f, b1 = A.ln_b ? A.ln_b[h * kN + tid + 32] : 0.f;
      Elem<TIn>::store(A.y + vb + tid, fmaf((y0 - mean) * rs, w0, b0));
      Elem<TIn>::store(A.y + vb + tid + 32, fmaf((y1 - mean) * rs, w1, b1));
    }
  }
}

// Launches a decode step allowing programmatic overlap with the grid before it in the stream: its CTAs
// may be placed while that grid drains, and wait (pdl_wait) before reading the state it wrote.
template <typename... KArgs, typename... Args>
static cudaError_t launch_overlapped(void (*kernel)(KArgs...), unsigned grid, unsigned block, cudaStream_t stream,
                                     Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(block);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, args...);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

// Whether a grid of `ctas` CTAs of `kernel` is larger than what the current device runs at once (its
// SM count times the kernel's resident CTAs per SM; cached per device and kernel).  Only then can no
// more than one earlier step still be running when a step's CTAs start: the step before cannot place
// all its CTAs, and so cannot release the next launch, until the one before it has finished.  Smaller
// grids could chain several waiting steps, so the early state loads are used only above this size.
// False when the device cannot be queried.
static bool exceeds_resident(const void *kernel, int threads, long long ctas) {
  constexpr int kMaxDev = 64, kMaxKernels = 16;
  static const void *keys[kMaxDev][kMaxKernels] = {};
  static long long vals[kMaxDev][kMaxKernels] = {};
  static std::mutex mu;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDev) return false;
  std::lock_guard<std::mutex> lock(mu);
  int slot = 0;
  for (; slot < kMaxKernels && keys[dev][slot] != nullptr; ++slot)
    if (keys[dev][slot] == kernel) return ctas > vals[dev][slot];
  int per_sm = 0, sms = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, threads, 0) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || per_sm <= 0 || sms <= 0) {
    (void)cudaGetLastError();  // clear a failed query; the launch then waits first, which is always correct
    return false;
  }
  const long long resident = static_cast<long long>(per_sm) * sms;
  if (slot < kMaxKernels) {
    keys[dev][slot] = kernel;
    vals[dev][slot] = resident;
  }
  return ctas > resident;
}

template <typename TIn>
cudaError_t launch_decode(const TIn *r, const TIn *w, const TIn *k, const TIn *v, const TIn *a, const TIn *b,
                          float *s, TIn *y, int B, int H, cudaStream_t stream) {
  DecodeArgs<TIn> A{r, w, k, v, a, b, s, y, nullptr, H, nullptr, nullptr};
  const long long pairs = static_cast<long long>(B) * H;
  if (pairs > 0x7fffffffLL) return cudaErrorInvalidValue;
  return launch_overlapped(wkv7_decode_kernel<TIn, false, false, false>, static_cast<unsigned>(pairs), 256, stream, A);
}

cudaError_t launch_decode_ext(const uint16_t *r, const uint16_t *w, const uint16_t *k, const uint16_t *v,
                              const uint16_t *a, const uint16_t *b, bool model_native, const float *k_k,
                              bool group_norm, const float *ln_w, const float *ln_b, bool early_state, float *s,
                              uint16_t *y, int B, int H, cudaStream_t stream) {
  DecodeArgs<uint16_t> A{r, w, k, v, a, b, s, y, k_k, H, ln_w, ln_b};
  const long long pairs = static_cast<long long>(B) * H;
  if (pairs > 0x7fffffffLL) return cudaErrorInvalidValue;
  const unsigned g = static_cast<unsigned>(pairs);
  if (early_state) {
    // the residency check takes the variant about to launch
    const void *kern = model_native && group_norm ? reinterpret_cast<const void *>(wkv7_decode_kernel<uint16_t, true, true, true>)
                       : model_native             ? reinterpret_cast<const void *>(wkv7_decode_kernel<uint16_t, true, false, true>)
                       : group_norm               ? reinterpret_cast<const void *>(wkv7_decode_kernel<uint16_t, false, true, true>)
                                                  : reinterpret_cast<const void *>(wkv7_decode_kernel<uint16_t, false, false, true>);
    early_state = exceeds_resident(kern, 256, pairs);
  }
  if (early_state) {
    if (model_native && group_norm)
      return launch_overlapped(wkv7_decode_kernel<uint16_t, true, true, true>, g, 256, stream, A);
    if (model_native) return launch_overlapped(wkv7_decode_kernel<uint16_t, true, false, true>, g, 256, stream, A);
    if (group_norm) return launch_overlapped(wkv7_decode_kernel<uint16_t, false, true, true>, g, 256, stream, A);
    return launch_overlapped(wkv7_decode_kernel<uint16_t, false, false, true>, g, 256, stream, A);
  }
  if (model_native && group_norm)
    return launch_overlapped(wkv7_decode_kernel<uint16_t, true, true, false>, g, 256, stream, A);
  if (model_native) return launch_overlapped(wkv7_decode_kernel<uint16_t, true, false, false>, g, 256, stream, A);
  if (group_norm) return launch_overlapped(wkv7_decode_kernel<uint16_t, false, true, false>, g, 256, stream, A);
  return launch_overlapped(wkv7_decode_kernel<uint16_t, false, false, false>, g, 256, stream, A);
}

// The bf16-state step: one CTA of 128 threads per (b, h); thread t holds columns 8*(t%8) .. +7 of
// rows t/8 + 16*m (m = 0..3), so each state load and store is 16 bytes (8 bf16) as in the float32
// kernel, and the row sums are three xor-shuffles inside 8 lanes.
__device__ __forceinline__ void unpack8(uint4 u, float (&o)[8]) {
  o[0] = __uint_as_float(u.x << 16);
  o[1] = __uint_as_float(u.x & 0xffff0000u);
  o[2] = __uint_as_float(u.y << 16);
  o[3] = __uint_as_float(u.y & 0xffff0000u);
  o[4] = __uint_as_float(u.z << 16);
  o[5] = __uint_as_float(u.z & 0xffff0000u);
  o[6] = __uint_as_float(u.w << 16);
  o[7] = __uint_as_float(u.w & 0xffff0000u);
}

template <bool kEarly>
__global__ void __launch_bounds__(128) wkv7_decode_bf16state_kernel(DecodeArgs<uint16_t, uint16_t> A) {
  pdl_trigger();
  if (!kEarly) pdl_wait();
  const long long pair = blockIdx.x;
  const int tid = threadIdx.x;
  const int c8 = tid & 7, rg = tid >> 3;
  uint16_t *S = A.s + pair * (kN * kN);
  uint4 raw[4];
#pragma unroll
  for (int m = 0; m < 4; ++m) raw[m] = *reinterpret_cast<const uint4 *>(S + (rg + 16 * m) * kN + 8 * c8);
  if (kEarly) pdl_wait();
  const long long vb = pair * kN;
  float ww[8], kk[8], aa[8], bb[8], rr[8];
  unpack8(*reinterpret_cast<const uint4 *>(A.w + vb + 8 * c8), ww);
  unpack8(*reinterpret_cast<const uint4 *>(A.k + vb + 8 * c8), kk);
  unpack8(*reinterpret_cast<const uint4 *>(A.a + vb + 8 * c8), aa);
  unpack8(*reinterpret_cast<const uint4 *>(A.b + vb + 8 * c8), bb);
  unpack8(*reinterpret_cast<const uint4 *>(A.r + vb + 8 * c8), rr);
  float st[4][8], sa[4], yv[4], vv[4];
#pragma unroll
  for (int m = 0; m < 4; ++m) {
    unpack8(raw[m], st[m]);
    float p = 0.f;
#pragma unroll
    for (int e = 0; e < 8; ++e) p = fmaf(st[m][e], aa[e], p);
    sa[m] = p;
    vv[m] = bf16_bits_to_float(A.v[vb + rg + 16 * m]);
  }
#pragma unroll
  for (int off = 4; off >= 1; off >>= 1)
#pragma unroll
    for (int m = 0; m < 4; ++m) sa[m] += __shfl_xor_sync(0xffffffffu, sa[m], off);
#pragma unroll
  for (int m = 0; m < 4; ++m) {
    float p = 0.f;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      st[m][e] = fmaf(st[m][e], ww[e], fmaf(sa[m], bb[e], vv[m] * kk[e]));
      p = fmaf(st[m][e], rr[e], p);
    }
    yv[m] = p;
    *reinterpret_cast<uint4 *>(S + (rg + 16 * m) * kN + 8 * c8) =
        make_uint4(bf16x2_rn(st[m][0], st[m][1]), bf16x2_rn(st[m][2], st[m][3]), bf16x2_rn(st[m][4], st[m][5]),
                   bf16x2_rn(st[m][6], st[m][7]));
  }
#pragma unroll
  for (int off = 4; off >= 1; off >>= 1)
#pragma unroll
    for (int m = 0; m < 4; ++m) yv[m] += __shfl_xor_sync(0xffffffffu, yv[m], off);
  if (c8 == 0) {
#pragma unroll
    for (int m = 0; m < 4; ++m) Elem<uint16_t>::store(A.y + vb + rg + 16 * m, yv[m]);
  }
}

cudaError_t launch_decode_bf16state(const uint16_t *r, const uint16_t *w, const uint16_t *k, const uint16_t *v,
                                    const uint16_t *a, const uint16_t *b, bool early_state, uint16_t *s, uint16_t *y,
                                    int B, int H, cudaStream_t stream) {
  DecodeArgs<uint16_t, uint16_t> A{r, w, k, v, a, b, s, y, nullptr, H, nullptr, nullptr};
  const long long pairs = static_cast<long long>(B) * H;
  if (pairs > 0x7fffffffLL) return cudaErrorInvalidValue;
  const unsigned g = static_cast<unsigned>(pairs);
  if (early_state && exceeds_resident(reinterpret_cast<const void *>(wkv7_decode_bf16state_kernel<true>), 128, pairs))
    return launch_overlapped(wkv7_decode_bf16state_kernel<true>, g, 128, stream, A);
  return launch_overlapped(wkv7_decode_bf16state_kernel<false>, g, 128, stream, A);
}

template cudaError_t launch_decode<float>(const float *, const float *, const float *, const float *, const float *,
                                          const float *, float *, float *, int, int, cudaStream_t);
template cudaError_t launch_decode<uint16_t>(const uint16_t *, const uint16_t *, const uint16_t *, const uint16_t *,
                                             const uint16_t *, const uint16_t *, float *, uint16_t *, int, int,
                                             cudaStream_t);

}  // namespace rwkv7
