// wkv7_scan.cu -- sequential-scan prefill: the x070 recurrence token by token
// with the float32 state held in registers.
//
// Operation (RWKV-7 G0 7.2B walkthrough, lshu.cn/news/198401, section 7.1):
//   sa = S a_t;  S = S diag(w_t) + sa b_t^T + v_t k_t^T;  y_t = S r_t.
//
// Rows of S are independent of each other: row i needs only its own values,
// v_t[i] and the shared vectors r, w, k, a, b.  So a (b, h) pair is split
// into 64 / ROWS row groups, one CTA each, and every row is spread over
// LANES lanes (8: 8 columns each).  The two per-token
// dot products (S a and S r) are finished with xor-shuffles inside those lanes.
//
// Column ownership: lane q holds the 4-column chunks starting at 4*q + 4*LANES*m,
// so the lanes of a row read adjacent chunks of shared memory and the rows of a
// warp read the same addresses (broadcast).
//
// Per-token operands are staged into shared memory in tiles of TT tokens
// with cp.async, double-buffered, and y is staged per tile and written back
// as contiguous runs of ROWS elements.
//
// The fused variant takes model-native inputs (x_w in place of w, x_a in place of a, no b, and the
// per-channel key scale k_k) and forms w, a = -kk and b = kk * sigmoid(x_a) per token in registers;
// the key norm is one more reduction over the row's lanes, which hold all 64 columns of the row.
//
// The group-norm variant (x070 ln_x on y) runs one CTA of 256 threads per (b, h) (ROWS = 64), so
// every token's 64 channels of y meet in one tile of shared memory; one warp per token normalises
// them on the way out.
#include "common.cuh"
#include "launch.h"

namespace rwkv7 {

// Lanes per state row (every variant: the per-row arithmetic, and so the state, is then the same with
// and without the group-norm epilogue, whose variant holds all 64 rows in one CTA).  Measured on
// B200 at B8 T4096 H12 (bf16 / float32 / model-native operands): 4 lanes 2.11 / 2.34 / 4.15 ms,
// 8 lanes 1.53 / 1.98 / 3.21 ms, 16 lanes 1.70 / 1.90 / 3.30 ms.
constexpr int kScanLanes = 8;

template <typename TIn, int ROWS, int LANES = 4> struct ScanCfg {
  static constexpr int kThreads = ROWS * LANES;
  static constexpr int kTT = sizeof(TIn) == 2 ? 32 : 16;  // tokens per tile (24+ KB per buffer)
  static constexpr int kVecElems = 5 * kN;                 // r, w, k, a, b
  static constexpr int kTokElems = kVecElems + ROWS;       // + this CTA's slice of v
  static constexpr int kBufElems = kTT * kTokElems;
  static constexpr int kEPC = 16 / static_cast<int>(sizeof(TIn));  // elements per 16-byte chunk
  static constexpr int kChunksVec = kN / kEPC;
  static constexpr int kChunksV = ROWS / kEPC;
  static constexpr int kChunksTok = 5 * kChunksVec + kChunksV;
  static constexpr size_t kSmemBytes = 2 * kBufElems * sizeof(TIn) + kTT * ROWS * sizeof(float);
  static_assert((kTokElems * sizeof(TIn)) % 16 == 0, "token stride must keep 16-byte alignment");
  static_assert(ROWS % kEPC == 0, "row slice must be whole 16-byte chunks");
};

template <typename TIn> struct ScanArgs {
  const TIn *r, *w, *k, *v, *a, *b;  // fused: w = x_w, a = x_a, b unused
  const float *s_in;
  TIn *y;
  float *s_out;
  const int32_t *cu_seqlens;  // nullptr: fixed length T
  int T;
  long long total_T;
  int H;
  const float *k_k;  // fused: [H, 64] key scale, nullptr = ones
  const float *ln_w, *ln_b;  // group-norm epilogue: [H, 64] weight / bias, nullptr = ones / zeros
  float *states;  // nullptr, or [B, H, ceil(T / 64), 64, 64]: the state before every 64th token (dense T)
};

template <typename TIn, int ROWS, bool kFused, int LANES>
__device__ __forceinline__ void scan_load_tile(const ScanArgs<TIn> &A, TIn *buf, long long tok0, int ntok, int h,
                                               int row0) {
  using C = ScanCfg<TIn, ROWS, LANES>;
  const int total = ntok * C::kChunksTok;
  for (int c = threadIdx.x; c < total; c += C::kThreads) {
    const int tt = c / C::kChunksTok, cc = c - tt * C::kChunksTok;
    const long long base = ((tok0 + tt) * A.H + h) * kN;
    TIn *dst = buf + tt * C::kTokElems;
    if (cc < 5 * C::kChunksVec) {
      const int vid = cc / C::kChunksVec, part = cc - vid * C::kChunksVec;
      if (kFused && vid == 4) continue;  // no b
      const TIn *src = vid == 0 ? A.r : vid == 1 ? A.w : vid == 2 ? A.k : vid == 3 ? A.a : A.b;
      cp_async16(dst + vid * kN + part * C::kEPC, src + base + part * C::kEPC);
    } else {
      const int part = cc - 5 * C::kChunksVec;
      cp_async16(dst + C::kVecElems + part * C::kEPC, A.v + base + row0 + part * C::kEPC);
    }
  }
}

// LANES lanes share a state row: lane q holds the 4-column chunks starting at 4 q + 4 LANES m
// (m = 0 .. 16 / LANES - 1), CPL = 64 / LANES columns in all.
template <typename TIn, int ROWS, bool kFused, bool kLN, int LANES = 4>
__global__ void __launch_bounds__(ScanCfg<TIn, ROWS, LANES>::kThreads) wkv7_scan_kernel(ScanArgs<TIn> A) {
  static_assert(!kLN || ROWS == kN, "the group-norm epilogue needs all 64 rows in one CTA");
  static_assert(LANES == 4 || LANES == 8 || LANES == 16, "4, 8 or 16 lanes per row");
  using C = ScanCfg<TIn, ROWS, LANES>;
  constexpr int CPL = kN / LANES;  // columns per lane
  constexpr int NM = CPL / 4;      // 4-column chunks per lane
  constexpr int kSplits = kN / ROWS;
  extern __shared__ __align__(16) uint8_t smem_raw[];
  TIn *bufs = reinterpret_cast<TIn *>(smem_raw);
  float *ys = reinterpret_cast<float *>(smem_raw + 2 * C::kBufElems * sizeof(TIn));

  const int h = blockIdx.x / kSplits;
  const int row0 = (blockIdx.x - h * kSplits) * ROWS;
  const int bidx = blockIdx.y;
  const SeqBounds sb = seq_bounds(A.cu_seqlens, bidx, A.T, A.total_T);
  if (sb.len < 0) return;

  const int tid = threadIdx.x;
  const int rloc = tid / LANES, q = tid % LANES;
  const int row = row0 + rloc;
  const long long sbase = (static_cast<long long>(bidx) * A.H + h) * (kN * kN) + static_cast<long long>(row) * kN;

  float s[CPL];
#pragma unroll
  for (int m = 0; m < NM; ++m) {
    float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
    if (A.s_in != nullptr) x = *reinterpret_cast<const float4 *>(A.s_in + sbase + 4 * LANES * m + 4 * q);
    s[4 * m + 0] = x.x; s[4 * m + 1] = x.y; s[4 * m + 2] = x.z; s[4 * m + 3] = x.w;
  }

  float kkr[CPL];  // fused: key scale of this thread's columns
#pragma unroll
  for (int m = 0; m < NM; ++m)
#pragma unroll
    for (int e = 0; e < 4; ++e) kkr[4 * m + e] = (kFused && A.k_k) ? A.k_k[h * kN + 4 * LANES * m + 4 * q + e] : 1.f;

  const int ntiles = (sb.len + C::kTT - 1) / C::kTT;
  if (ntiles > 0) {
    scan_load_tile<TIn, ROWS, kFused, LANES>(A, bufs, sb.start, min(C::kTT, sb.len), h, row0);
    cp_async_commit();
  }
  for (int tile = 0; tile < ntiles; ++tile) {
    const int t0 = tile * C::kTT;
    const int ntok = min(C::kTT, sb.len - t0);
    if (tile + 1 < ntiles) {
      const int t1 = t0 + C::kTT;
      scan_load_tile<TIn, ROWS, kFused, LANES>(A, bufs + ((tile + 1) & 1) * C::kBufElems, sb.start + t1,
                                        min(C::kTT, sb.len - t1), h, row0);
      cp_async_commit();
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();

    const TIn *buf = bufs + (tile & 1) * C::kBufElems;
#pragma unroll 2
    for (int tt = 0; tt < ntok; ++tt) {
      const TIn *tok = buf + tt * C::kTokElems;
      float rr[CPL], ww[CPL], kk[CPL], aa[CPL], bb[CPL];
#pragma unroll
      for (int m = 0; m < NM; ++m) {
        const int col = 4 * LANES * m + 4 * q;
        Elem<TIn>::load4(tok + 0 * kN + col, rr + 4 * m);
        Elem<TIn>::load4(tok + 1 * kN + col, ww + 4 * m);
        Elem<TIn>::load4(tok + 2 * kN + col, kk + 4 * m);
        Elem<TIn>::load4(tok + 3 * kN + col, aa + 4 * m);
        if (!kFused) Elem<TIn>::load4(tok + 4 * kN + col, bb + 4 * m);
      }
      const float vi = Elem<TIn>::load(tok + C::kVecElems + rloc);
      if (A.states != nullptr && ((t0 + tt) & 63) == 0) {
        // checkpoint for the backward: this thread's 16 columns of the state before the token
        const int nck = (A.T + 63) >> 6;
        float *ck = A.states + ((static_cast<long long>(bidx) * A.H + h) * nck + ((t0 + tt) >> 6)) * (kN * kN) +
                    static_cast<long long>(row) * kN;
#pragma unroll
        for (int m = 0; m < NM; ++m)
          *reinterpret_cast<float4 *>(ck + 4 * LANES * m + 4 * q) =
              make_float4(s[4 * m + 0], s[4 * m + 1], s[4 * m + 2], s[4 * m + 3]);
      }
      if (kFused) {
        // x070 prologue: kk = normalise(k * k_k) over the row's 64 columns, a = -kk, b = kk * rate
        float ss = 0.f;
#pragma unroll
        for (int c = 0; c < CPL; ++c) ss = fmaf(kk[c] * kkr[c], kk[c] * kkr[c], ss);
#pragma unroll
        for (int off = 1; off < LANES; off <<= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
        const float inv = x070_inv_norm(ss);
#pragma unroll
        for (int c = 0; c < CPL; ++c) {
          const float kkv = kk[c] * kkr[c] * inv;
          bb[c] = kkv * x070_sigmoid(aa[c]);
          aa[c] = -kkv;
          ww[c] = x070_decay(ww[c]);
        }
      }

      // sa = S a (state before this token), four partial sums, then the row's lanes
      float p0 = 0.f, p1 = 0.f, p2 = 0.f, p3 = 0.f;
#pragma unroll
      for (int c = 0; c < CPL; c += 4) {
        p0 = fmaf(s[c + 0], aa[c + 0], p0);
        p1 = fmaf(s[c + 1], aa[c + 1], p1);
        p2 = fmaf(s[c + 2], aa[c + 2], p2);
        p3 = fmaf(s[c + 3], aa[c + 3], p3);
      }
      float sa = (p0 + p1) + (p2 + p3);
#pragma unroll
      for (int off = 1; off < LANES; off <<= 1) sa += __shfl_xor_sync(0xffffffffu, sa, off);

      // S = S diag(w) + sa b^T + v k^T
#pragma unroll
      for (int c = 0; c < CPL; ++c) s[c] = fmaf(s[c], ww[c], fmaf(sa, bb[c], vi * kk[c]));

      // y = S r (updated state)
      p0 = p1 = p2 = p3 = 0.f;
#pragma unroll
      for (int c = 0; c < CPL; c += 4) {
        p0 = fmaf(s[c + 0], rr[c + 0], p0);
        p1 = fmaf(s[c + 1], rr[c + 1], p1);
        p2 = fmaf(s[c + 2], rr[c + 2], p2);
        p3 = fmaf(s[c + 3], rr[c + 3], p3);
      }
      float y = (p0 + p1) + (p2 + p3);
#pragma unroll
      for (int off = 1; off < LANES; off <<= 1) y += __shfl_xor_sync(0xffffffffu, y, off);
      if (q == 0) ys[tt * ROWS + rloc] = y;
    }
    __syncthreads();
    if (!kLN) {
      for (int e = tid; e < ntok * ROWS; e += C::kThreads) {
        const int tt = e / ROWS, rr_ = e - tt * ROWS;
        const long long yi = ((sb.start + t0 + tt) * A.H + h) * kN + row0 + rr_;
        Elem<TIn>::store(A.y + yi, ys[e]);
      }
    } else {
      // ln_x: one warp per token, channels lane and lane + 32
      const int lane = tid & 31;
      const float w0 = A.ln_w ? A.ln_w[h * kN + lane] : 1.f, w1 = A.ln_w ? A.ln_w[h * kN + lane + 32] : 1.f;
      const float b0 = A.ln_b ? A.ln_b[h * kN + lane] : 0.f, b1 = A.ln_b ? A.ln_b[h * kN + lane + 32] : 0.f;
      for (int tt = tid >> 5; tt < ntok; tt += C::kThreads / 32) {
        const float y0 = ys[tt * ROWS + lane], y1 = ys[tt * ROWS + lane + 32];
        float mean, var;
        warp_mean_var64(y0, y1, mean, var);
        const float rs = rsqrtf(var + kLnEps);
        const long long yi = ((sb.start + t0 + tt) * A.H + h) * kN;
        Elem<TIn>::store(A.y + yi + lane, fmaf((y0 - mean) * rs, w0, b0));
        Elem<TIn>::store(A.y + yi + lane + 32, fmaf((y1 - mean) * rs, w1, b1));
      }
    }
    // the next iteration's first __syncthreads orders these reads of ys
    // before the next tile's writes to it
  }

#pragma unroll
  for (int m = 0; m < NM; ++m)
    *reinterpret_cast<float4 *>(A.s_out + sbase + 4 * LANES * m + 4 * q) =
        make_float4(s[4 * m + 0], s[4 * m + 1], s[4 * m + 2], s[4 * m + 3]);
}

template <typename TIn, int ROWS, bool kFused = false, bool kLN = false, int LANES = kScanLanes>
static cudaError_t launch_scan_rows(const ScanArgs<TIn> &A, int B, cudaStream_t stream) {
  using C = ScanCfg<TIn, ROWS, LANES>;
  auto kern = wkv7_scan_kernel<TIn, ROWS, kFused, kLN, LANES>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(C::kSmemBytes));
  if (e != cudaSuccess) return e;
  dim3 grid(A.H * (kN / ROWS), B);
  kern<<<grid, C::kThreads, C::kSmemBytes, stream>>>(A);
  return cudaGetLastError();
}

template <typename TIn>
cudaError_t launch_scan(const TIn *r, const TIn *w, const TIn *k, const TIn *v, const TIn *a, const TIn *b,
                        const float *s_in, TIn *y, float *s_out, const int32_t *cu_seqlens, int B, int T,
                        long long total_T, int H, cudaStream_t stream) {
  ScanArgs<TIn> A{r, w, k, v, a, b, s_in, y, s_out, cu_seqlens, T, total_T, H, nullptr, nullptr, nullptr, nullptr};
  return launch_scan_rows<TIn, 16>(A, B, stream);
}

cudaError_t launch_scan_save(const uint16_t *r, const uint16_t *w, const uint16_t *k, const uint16_t *v,
                             const uint16_t *a, const uint16_t *b, const float *s_in, uint16_t *y, float *s_out,
                             float *states, int B, int T, int H, cudaStream_t stream) {
  ScanArgs<uint16_t> A{r, w, k, v, a, b, s_in, y, s_out, nullptr, T, static_cast<long long>(B) * T, H,
                       nullptr, nullptr, nullptr, states};
  return launch_scan_rows<uint16_t, 16>(A, B, stream);
}

cudaError_t launch_scan_ext(const uint16_t *r, const uint16_t *w, const uint16_t *k, const uint16_t *v,
                            const uint16_t *a, const uint16_t *b, bool model_native, const float *k_k,
                            bool group_norm, const float *ln_w, const float *ln_b, const float *s_in, uint16_t *y,
                            float *s_out, const int32_t *cu_seqlens, int B, int T, long long total_T, int H,
                            cudaStream_t stream) {
  ScanArgs<uint16_t> A{r, w, k, v, a, b, s_in, y, s_out, cu_seqlens, T, total_T, H, k_k, ln_w, ln_b, nullptr};
  if (model_native && group_norm) return launch_scan_rows<uint16_t, 64, true, true>(A, B, stream);
  if (model_native) return launch_scan_rows<uint16_t, 16, true, false>(A, B, stream);
  if (group_norm) return launch_scan_rows<uint16_t, 64, false, true>(A, B, stream);
  return launch_scan_rows<uint16_t, 16, false, false>(A, B, stream);
}

template cudaError_t launch_scan<float>(const float *, const float *, const float *, const float *, const float *,
                                        const float *, const float *, float *, float *, const int32_t *, int, int,
                                        long long, int, cudaStream_t);
template cudaError_t launch_scan<uint16_t>(const uint16_t *, const uint16_t *, const uint16_t *, const uint16_t *,
                                           const uint16_t *, const uint16_t *, const float *, uint16_t *, float *,
                                           const int32_t *, int, int, long long, int, cudaStream_t);

}  // namespace rwkv7
