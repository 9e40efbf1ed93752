// wkv7_backward.cu -- gradients of the x070 recurrence for training (sequential form).
//
// The forward (RWKV-7 G0 7.2B walkthrough, lshu.cn/news/198401, section 7.1) is, per (b, h),
//   sa = S a_t;   S' = S diag(w_t) + sa b_t^T + v_t k_t^T;   y_t = S' r_t.
// The pages give no backward; this is the chain rule applied to that loop, for a loss whose
// gradients dy (per token) and ds_out (final state) are given.  Walking the tokens backwards with
// G = dL/dS' (starting from ds_out):
//   G += dy_t r_t^T;   dr_t = S'^T dy_t;   dv_t = G k_t;   dk_t = G^T v_t;
//   db_t = G^T sa;     g = G b_t;          dw_t = colsum(G .* S);   da_t = S^T g;
//   G <- G diag(w_t) + g a_t^T            (= dL/dS, carried to the token before),
// and ds_in = G at the start.
//
// Rows of S (value channels) are independent in the forward and in the walk back: row i of G and
// of S only meet the shared vectors.  A (b, h) pair is split into 4 row groups of 16 rows, one CTA
// of 128 threads each; every row is spread over 8 lanes holding 8 columns.  Row sums (sa, g, dv)
// are three xor-shuffles inside the 8 lanes; the column sums (dr, dk, db, dw, da: sums over rows)
// go through shared memory: every thread stores its 5 x 8 partial products, then 80 threads each
// sum one 4-column group over the 16 rows (float4 loads), then float32 atomics across the 4 row
// groups (the caller zeroes those outputs first).
//
// The states S before every token are recomputed from the checkpoints the forward saved (the state
// before every 64th token): per 64-token chunk, walked from the last, a forward pass from the
// checkpoint keeps the state before each 8-token sub-block in shared memory; then each sub-block,
// from the last, recomputes its 9 states into registers and walks its tokens back.  Per-token
// operands are staged 8 tokens at a time by cp.async, double-buffered, in the order the schedule
// visits them.
#include "common.cuh"
#include "launch.h"

namespace rwkv7 {
namespace bwd {

// A thread layout: 16 state rows per CTA (4 CTAs per (b, h)), kLanes lanes per row, each holding
// 64 / kLanes columns: 128 threads at 8 lanes, 256 at 16 (twice the warps for the same rows, to hide
// the latency of the per-token chain).
template <int kLanes> struct Layout {
  static constexpr int kRows = 16;
  static constexpr int kCols = kN / kLanes;              // 8 or 4
  static constexpr int kThreads = kRows * kLanes;        // 128 or 256
};
#ifndef RWKV7_BWD_LANES
#define RWKV7_BWD_LANES 16
#endif
constexpr int kBwdLanes = RWKV7_BWD_LANES;  // the layout the library launches
constexpr int kSub = 8;                   // tokens per sub-block
constexpr int kChunk = 64;                // tokens per saved state
constexpr int kSubs = kChunk / kSub;      // sub-blocks per chunk
constexpr int kTokVec = 7;                // staged per token: r, w, k, a, b, v, dy (64 bf16 each)
constexpr int kStageElems = kSub * kTokVec * kN;
enum { V_R = 0, V_W = 1, V_K = 2, V_A = 3, V_B = 4, V_V = 5, V_DY = 6 };

template <int kLanes> __host__ __device__ constexpr size_t smem_subck() { return sizeof(float) * kSubs * Layout<kLanes>::kRows * kN; }
constexpr size_t kSmemStage = sizeof(uint16_t) * 2 * kStageElems;   // 14 KB
// the column partials of one token: [row][5][64] at 8 lanes; at 16 lanes the two rows a warp holds are
// summed first ([row pair][5][64]) and the buffer is doubled, alternating by token
template <int kLanes> __host__ __device__ constexpr int part_rows() { return kLanes == 16 ? Layout<kLanes>::kRows / 2 : Layout<kLanes>::kRows; }
template <int kLanes> __host__ __device__ constexpr int part_bufs() { return kLanes == 16 ? 2 : 1; }
template <int kLanes> __host__ __device__ constexpr size_t smem_part() {
  return sizeof(float) * part_bufs<kLanes>() * part_rows<kLanes>() * 5 * kN;
}
template <int kLanes> __host__ __device__ constexpr size_t smem_bytes() { return smem_subck<kLanes>() + kSmemStage + smem_part<kLanes>(); }

struct Args {
  const uint16_t *r, *w, *k, *v, *a, *b, *dy;
  const float *states;  // [B, H, ceil(T/64), 64, 64]
  const float *ds_out;  // [B, H, 64, 64] or nullptr
  float *dr, *dw, *dk, *dv, *da, *db;  // [B, T, H, 64]; dr dw dk da db accumulated
  float *ds_in;                        // [B, H, 64, 64] or nullptr
  int T, H;
};

// One visit of the schedule: sub-block s of chunk c, in the forward pass (fwd) or the walk back.
struct Visit {
  int c, s, fwd;
};
// Chunks from the last; each contributes its forward sub-blocks 0..n-1, then n-1..0 backwards.
__device__ __forceinline__ Visit visit_at(int kk, int nck, int nsub_last) {
  Visit v;
  int j, nsub;
  if (kk < 2 * nsub_last) {
    v.c = nck - 1;
    j = kk;
    nsub = nsub_last;
  } else {
    const int k2 = kk - 2 * nsub_last;
    v.c = nck - 2 - k2 / (2 * kSubs);
    j = k2 % (2 * kSubs);
    nsub = kSubs;
  }
  v.fwd = j < nsub ? 1 : 0;
  v.s = v.fwd ? j : 2 * nsub - 1 - j;
  return v;
}

template <int kThreads>
__device__ __forceinline__ void stage_visit(const Args &A, uint16_t *buf, long long tok0, int ntok, int h) {
  const int total = ntok * kTokVec * 8;  // 16-byte pieces
  for (int c = threadIdx.x; c < total; c += kThreads) {
    const int tt = c / (kTokVec * 8), rem = c - tt * (kTokVec * 8);
    const int vid = rem >> 3, part = rem & 7;
    const uint16_t *src = vid == V_R   ? A.r
                          : vid == V_W ? A.w
                          : vid == V_K ? A.k
                          : vid == V_A ? A.a
                          : vid == V_B ? A.b
                          : vid == V_V ? A.v
                                       : A.dy;
    cp_async16(buf + (tt * kTokVec + vid) * kN + part * 8, src + ((tok0 + tt) * A.H + h) * kN + part * 8);
  }
}

// kC consecutive bf16 values (kC = 8: one 16-byte load, 4: one 8-byte load) as floats
template <int kC> __device__ __forceinline__ void ldc(const uint16_t *p, float (&o)[kC]) {
  if constexpr (kC == 8) {
    const uint4 u = *reinterpret_cast<const uint4 *>(p);
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      o[2 * i] = __uint_as_float(w[i] << 16);
      o[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
  } else {
    static_assert(kC == 4, "4 or 8 columns per thread");
    const uint2 u = *reinterpret_cast<const uint2 *>(p);
    o[0] = __uint_as_float(u.x << 16);
    o[1] = __uint_as_float(u.x & 0xffff0000u);
    o[2] = __uint_as_float(u.y << 16);
    o[3] = __uint_as_float(u.y & 0xffff0000u);
  }
}

// sum over the kLanes lanes that hold one row
template <int kLanes> __device__ __forceinline__ float rowsum(float x) {
#pragma unroll
  for (int off = 1; off < kLanes; off <<= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
  return x;
}

// One forward token on this thread's columns (c0 ..) of row `row`: S <- S diag(w) + (S a) b^T + v k^T.
template <int kLanes, int kC>
__device__ __forceinline__ void fwd_token(float (&S)[kC], const uint16_t *tk, int c0, int row) {
  float w8[kC], k8[kC], a8[kC], b8[kC];
  ldc<kC>(tk + V_W * kN + c0, w8);
  ldc<kC>(tk + V_K * kN + c0, k8);
  ldc<kC>(tk + V_A * kN + c0, a8);
  ldc<kC>(tk + V_B * kN + c0, b8);
  const float vi = bf16_bits_to_float(tk[V_V * kN + row]);
  float sa = 0.f;
#pragma unroll
  for (int e = 0; e < kC; ++e) sa = fmaf(S[e], a8[e], sa);
  sa = rowsum<kLanes>(sa);
#pragma unroll
  for (int e = 0; e < kC; ++e) S[e] = fmaf(S[e], w8[e], fmaf(sa, b8[e], vi * k8[e]));
}

// (3 CTAs per SM: a grid of 4 CTAs per (b, h) is all resident up to 111 pairs)
template <int kLanes>
__global__ void __launch_bounds__(Layout<kLanes>::kThreads, 3) wkv7_backward_kernel(const Args A) {
  constexpr int kRows = Layout<kLanes>::kRows, kC = Layout<kLanes>::kCols, kThreads = Layout<kLanes>::kThreads;
  extern __shared__ __align__(16) uint8_t smem_raw[];
  float *subck = reinterpret_cast<float *>(smem_raw);
  uint16_t *stage = reinterpret_cast<uint16_t *>(smem_raw + smem_subck<kLanes>());
  float *part = reinterpret_cast<float *>(smem_raw + smem_subck<kLanes>() + kSmemStage);

  constexpr int kSplits = kN / kRows;
  const int h = blockIdx.x / kSplits;
  const int row0 = (blockIdx.x - h * kSplits) * kRows;
  const int bidx = blockIdx.y;
  const int tid = threadIdx.x;
  const int rl = tid / kLanes, c0 = kC * (tid % kLanes);
  const int row = row0 + rl;  // state row (value channel) of this thread
  const int T = A.T;
  const long long pair = static_cast<long long>(bidx) * A.H + h;
  const long long tok_base = static_cast<long long>(bidx) * T;  // token row of t = 0
  const int nck = (T + kChunk - 1) / kChunk;
  const int nsub_last = nck > 0 ? (T - (nck - 1) * kChunk + kSub - 1) / kSub : 0;
  const int nvisits = nck > 0 ? 2 * nsub_last + 2 * kSubs * (nck - 1) : 0;

  float G[kC];  // dL/dS for this thread's columns of its row
#pragma unroll
  for (int e = 0; e < kC; ++e) G[e] = A.ds_out ? A.ds_out[pair * (kN * kN) + row * kN + c0 + e] : 0.f;
  float S[kC];  // running state of the forward passes
#pragma unroll
  for (int e = 0; e < kC; ++e) S[e] = 0.f;

  if (nvisits > 0) {
    const Visit v0 = visit_at(0, nck, nsub_last);
    const int t0 = v0.c * kChunk + v0.s * kSub;
    stage_visit<kThreads>(A, stage, tok_base + t0, min(kSub, T - t0), h);
    cp_async_commit();
  }
  for (int kk = 0; kk < nvisits; ++kk) {
    const Visit vis = visit_at(kk, nck, nsub_last);
    if (kk + 1 < nvisits) {
      const Visit vn = visit_at(kk + 1, nck, nsub_last);
      const int tn = vn.c * kChunk + vn.s * kSub;
      stage_visit<kThreads>(A, stage + ((kk + 1) & 1) * kStageElems, tok_base + tn, min(kSub, T - tn), h);
      cp_async_commit();
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();
    const uint16_t *buf = stage + (kk & 1) * kStageElems;
    const int t0 = vis.c * kChunk + vis.s * kSub;
    const int Ls = min(kSub, T - t0);
    float *sck = subck + (vis.s * kRows + rl) * kN + c0;

    if (vis.fwd) {
      // forward from the chunk's checkpoint, keeping the state before each sub-block
      if (vis.s == 0) {
        const float *ck = A.states + (pair * nck + vis.c) * (kN * kN) + row * kN + c0;
#pragma unroll
        for (int e = 0; e < kC; ++e) S[e] = ck[e];
      }
#pragma unroll
      for (int e = 0; e < kC; ++e) sck[e] = S[e];
      for (int u = 0; u < Ls; ++u) fwd_token<kLanes, kC>(S, buf + u * kTokVec * kN, c0, row);
    } else {
      // this sub-block's states: St[u] before token t0 + u, St[u + 1] after it
      float St[kSub + 1][kC];
#pragma unroll
      for (int e = 0; e < kC; ++e) St[0][e] = sck[e];
#pragma unroll
      for (int u = 0; u < kSub; ++u) {
#pragma unroll
        for (int e = 0; e < kC; ++e) St[u + 1][e] = St[u][e];
        if (u < Ls) fwd_token<kLanes, kC>(St[u + 1], buf + u * kTokVec * kN, c0, row);
      }
#pragma unroll
      for (int u = kSub - 1; u >= 0; --u) {
        if (u >= Ls) continue;  // uniform across the CTA
        const uint16_t *tk = buf + u * kTokVec * kN;
        float r8[kC], w8[kC], k8[kC], a8[kC], b8[kC];
        ldc<kC>(tk + V_R * kN + c0, r8);
        ldc<kC>(tk + V_W * kN + c0, w8);
        ldc<kC>(tk + V_K * kN + c0, k8);
        ldc<kC>(tk + V_A * kN + c0, a8);
        ldc<kC>(tk + V_B * kN + c0, b8);
        const float vi = bf16_bits_to_float(tk[V_V * kN + row]);
        const float dyi = bf16_bits_to_float(tk[V_DY * kN + row]);
        // y_t = S' r_t
#pragma unroll
        for (int e = 0; e < kC; ++e) G[e] = fmaf(dyi, r8[e], G[e]);
        float p[5][kC];  // column partials: dr, dk, db, dw, da
        float dv = 0.f, sa = 0.f, g = 0.f;
#pragma unroll
        for (int e = 0; e < kC; ++e) {
          p[0][e] = St[u + 1][e] * dyi;
          dv = fmaf(G[e], k8[e], dv);
          p[1][e] = G[e] * vi;
          sa = fmaf(St[u][e], a8[e], sa);
          g = fmaf(G[e], b8[e], g);
          p[3][e] = G[e] * St[u][e];
        }
        dv = rowsum<kLanes>(dv);
        sa = rowsum<kLanes>(sa);
        g = rowsum<kLanes>(g);
#pragma unroll
        for (int e = 0; e < kC; ++e) {
          p[2][e] = G[e] * sa;
          p[4][e] = St[u][e] * g;
          G[e] = fmaf(G[e], w8[e], g * a8[e]);
        }
        // column sums: the partials to shared memory (at 16 lanes, the warp's two rows summed first, by
        // an xor-shuffle over lane bit 4), then one 4-column group over the CTA's rows per thread (80 of
        // them), then the row groups through float32 atomics
        const long long tok = tok_base + t0 + u;
        constexpr int kPR = part_rows<kLanes>();
        float *pbuf = part + (part_bufs<kLanes>() == 2 ? (u & 1) : 0) * (kPR * 5 * kN);
        int prow = rl;
        bool writes = true;
        if constexpr (kLanes == 16) {
#pragma unroll
          for (int q = 0; q < 5; ++q)
#pragma unroll
            for (int e = 0; e < kC; ++e) p[q][e] += __shfl_xor_sync(0xffffffffu, p[q][e], 16);
          prow = rl >> 1;
          writes = (tid & 16) == 0;
        }
        if (writes) {
#pragma unroll
          for (int q = 0; q < 5; ++q) {
            float *dst = pbuf + (prow * 5 + q) * kN + c0;
#pragma unroll
            for (int x = 0; x < kC; x += 4)
              *reinterpret_cast<float4 *>(dst + x) = make_float4(p[q][x], p[q][x + 1], p[q][x + 2], p[q][x + 3]);
          }
        }
        if (tid % kLanes == 0) A.dv[(tok * A.H + h) * kN + row] = dv;
        __syncthreads();
        if (tid < 5 * kN / 4) {
          const int q = tid >> 4, c4 = (tid & 15) * 4;
          float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
          for (int rr = 0; rr < kPR; ++rr) {
            const float4 x = *reinterpret_cast<const float4 *>(pbuf + (rr * 5 + q) * kN + c4);
            acc.x += x.x;
            acc.y += x.y;
            acc.z += x.z;
            acc.w += x.w;
          }
          float *g = (q == 0 ? A.dr : q == 1 ? A.dk : q == 2 ? A.db : q == 3 ? A.dw : A.da) + (tok * A.H + h) * kN + c4;
          atomicAdd(g + 0, acc.x);
          atomicAdd(g + 1, acc.y);
          atomicAdd(g + 2, acc.z);
          atomicAdd(g + 3, acc.w);
        }
        // the partials are rewritten by the next token (one buffer) or by the token after it, which
        // every thread reaches only through the next token's barrier (two buffers)
        if constexpr (part_bufs<kLanes>() == 1) __syncthreads();
      }
    }
    // every thread is done with this staging buffer before the next visit refills it
    __syncthreads();
  }
  if (A.ds_in != nullptr)
#pragma unroll
    for (int e = 0; e < kC; ++e) A.ds_in[pair * (kN * kN) + row * kN + c0 + e] = G[e];
}

}  // namespace bwd

cudaError_t launch_backward(const uint16_t *r, const uint16_t *w, const uint16_t *k, const uint16_t *v,
                            const uint16_t *a, const uint16_t *b, const float *states, const uint16_t *dy,
                            const float *ds_out, float *dr, float *dw, float *dk, float *dv, float *da, float *db,
                            float *ds_in, int B, int T, int H, cudaStream_t stream) {
  using namespace bwd;
  Args A{r, w, k, v, a, b, dy, states, ds_out, dr, dw, dk, dv, da, db, ds_in, T, H};
  constexpr int kLanes = kBwdLanes;
  using L = Layout<kLanes>;
  cudaError_t e = cudaFuncSetAttribute(wkv7_backward_kernel<kLanes>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem_bytes<kLanes>()));
  if (e != cudaSuccess) return e;
  dim3 grid(H * (kN / L::kRows), B);
  wkv7_backward_kernel<kLanes><<<grid, L::kThreads, smem_bytes<kLanes>(), stream>>>(A);
  return cudaGetLastError();
}

}  // namespace rwkv7
