// wkv7_chunk.cu -- chunked prefill of the x070 recurrence on the tcgen05 tensor
// cores (the pages' "GPT mode": the parallel, sequence-at-once evaluation that
// yields the RNN-mode state; RWKV-LM README copy, oa0.com/c/1004164, and
// RWKV-7 G0 7.2B walkthrough, lshu.cn/news/198401, sections 3.2 and 7.1).
//
// Per (b, h) and chunk of C = 64 tokens, with Gamma_t = prod_{u<=t} w_u inside
// the chunk (t = 0..63), the recurrence S <- S diag(w) + (S a) b^T + v k^T,
// y = S r unrolls to (WY / UT form; rows are tokens, columns channels):
//
//   A~ = a*Gamma_{t-1}  R~ = r*Gamma_t  B^ = b/Gamma_t  K^ = k/Gamma_t
//   B- = b*Gamma_C/Gamma_t  K- = k*Gamma_C/Gamma_t  (Gamma_C: whole chunk)
//   MMA1 (tf32)  [Mrb Mrk; Lab Lak] = [R~; A~] [B^; K^]^T, causally masked
//   CUDA cores   Tinv = (I - Lab)^-1 (unit lower triangular)
//   MMA3 (bf16)  [W~ U~]^T = [A~^T; Lak^T] Tinv^T
//   MMA2 (tf32)  [Q P; E F] = [R~ Mrk; 0 K-^T] + [Mrb; B-^T] [W~ U~]
//   MMA4 (tf32)  [Y; X] = [Q P; E F] [S0^T; V],   S_C^T = diag(Gamma_C) S0^T + X
//
// Every tf32 operand is K-major: the 128-byte-swizzled MN-major layout is not
// valid for 32-bit operands (a tf32 MMA given one produced zeros on B200).
//
// The products whose rounding reaches y directly (MMA1, the per-chunk state
// transition MMA4 and its inputs) run in tf32; MMA3 runs in bf16.  The state
// is carried in float32 registers across chunks; only its tf32 copy feeds
// MMA4.  The decay term diag(Gamma_C) S0^T is applied in float32.
//
// One CTA of 256 threads owns one (b, h) and walks its chunks in order; the
// next chunk's six 64x64 bf16 tiles are fetched by TMA while the current one
// is processed.  TMEM (512 columns) holds every MMA accumulator; MMA2 and MMA4
// read their A operand straight from TMEM.
//
// Domain: the decay is referenced to the chunk start, so 1/Gamma_t must stay
// finite in float32: every w must satisfy w >= 0.27 (0.27^64 > 1.2e-38).  The
// model's decay exp(-e^-0.5 sigmoid(x)) is always >= 0.5452.
#include <cuda.h>

#include "common.cuh"
#include "launch.h"
#include "tc_ptx.cuh"

namespace rwkv7 {
namespace chunk {

constexpr int C = 64;
constexpr int kThreads = 256;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kMaxPolls = 1u << 22;

// TMEM column map
constexpr uint32_t TM_D1 = 0;    // 128 cols: [Mrb Mrk] (lanes 0-63), [Lab Lak] (lanes 64-127)
constexpr uint32_t TM_D2 = 128;  // 128 cols: [Q P] / [E F]
constexpr uint32_t TM_D3 = 256;  // 64 cols: [W~ U~]^T (lane = column index of W~|U~, col = token)
constexpr uint32_t TM_D4 = 320;  // 64 cols: Y (lanes 0-63), X (lanes 64-127)
constexpr uint32_t TM_A2 = 384;  // 64 cols: Mrb (lanes 0-63), B-^T (lanes 64-127)

// shared memory map (bytes from a 1024-aligned base)
constexpr uint32_t kTile = C * kN * 2;            // one bf16 64x64 tile
constexpr uint32_t OFF_RAW = 0;                   // r w k a b v tiles, row-major [token][channel]
constexpr uint32_t OFF_A1 = OFF_RAW + 6 * kTile;  // tf32 K-major [R~; A~] 128x64 (32 KB)
constexpr uint32_t OFF_B1 = OFF_A1 + 32768;       // tf32 K-major [B^; K^] 128x64 (32 KB)
constexpr uint32_t OFF_A3 = OFF_B1 + 32768;       // bf16 MN-major [A~^T; Lak^T], M=128 x K=64 (16 KB)
constexpr uint32_t OFF_B4S = OFF_A3 + 16384;      // tf32 K-major S0^T part of the chain B: row i, K = j (16 KB)
constexpr uint32_t OFF_B4V = OFF_B4S + 16384;     // tf32 K-major V part of the chain B: row i, K = m (16 KB)
constexpr uint32_t OFF_MISC = OFF_B4V + 16384;
// regions reused once MMA1 has consumed A1 / B1
constexpr int LDL = 68;                           // row stride (floats) of Lab: conflict-free as an mma A operand
constexpr int LDT = 72;                           // row stride (floats) of Tinv: conflict-free as an mma B operand
constexpr uint32_t OFF_LS = OFF_A1;               // float [64][LDL]
constexpr uint32_t OFF_ZS = OFF_A1 + 64 * LDL * 4;  // float [3 warps][16][24]
constexpr uint32_t OFF_B2 = OFF_A1;               // tf32 K-major [W~ U~]^T 128x64 (after the inverse)
constexpr uint32_t OFF_TS = OFF_B1;               // float [64][LDT]
constexpr uint32_t OFF_B3 = OFF_B1 + 19456;       // bf16 K-major Tinv 64x64 (8 KB), 1024-aligned
constexpr uint32_t MISC_GC = 256;                 // float [64]   Gamma at the chunk end
constexpr uint32_t MISC_TOT = 512;                // float [16][64] per-token-group decay products
constexpr uint32_t kSmemBytes = OFF_MISC + MISC_TOT + 16 * 64 * 4 + 1024;

static_assert(OFF_ZS + 3 * 16 * 24 * 4 <= OFF_B1, "inverse scratch overflows A1");
static_assert(OFF_TS + 64 * LDT * 4 <= OFF_B3 && OFF_B3 + 8192 <= OFF_A3, "inverse scratch overflows B1");

struct Maps {
  CUtensorMap m[6];  // r, w, k, a, b, v: dims {64, H, tokens}, box {64, 1, 64}
};

struct Args {
  uint16_t *y;
  const float *s_in;
  float *s_out;
  const int32_t *cu_seqlens;
  int T;
  long long total_T;
  int H;
  int *err;
};

enum { RAW_R = 0, RAW_W = 1, RAW_K = 2, RAW_A = 3, RAW_B = 4, RAW_V = 5 };

// byte offset of element (row, k) in a K-major tf32 operand with `rows` rows
__device__ __forceinline__ uint32_t kmaj_tf32(uint32_t rows, uint32_t row, uint32_t k) {
  return (k >> 5) * (rows * 128u) + tc::sw128(row, (k & 31u) >> 2) + (k & 3u) * 4u;
}
// byte offset of element (k, mn) in an MN-major bf16 operand with `krows` K rows
__device__ __forceinline__ uint32_t mnmaj_bf16(uint32_t krows, uint32_t k, uint32_t mn) {
  return (mn >> 6) * (krows * 128u) + tc::sw128(k, (mn & 63u) >> 3) + (mn & 7u) * 2u;
}

// four consecutive bf16 channels of one token row of a raw tile
__device__ __forceinline__ void raw4(const uint8_t *smem, int tile, int t, int j0, float (&o)[4]) {
  const uint2 u = *reinterpret_cast<const uint2 *>(smem + OFF_RAW + tile * kTile + (t * kN + j0) * 2);
  o[0] = __uint_as_float(u.x << 16);
  o[1] = __uint_as_float(u.x & 0xffff0000u);
  o[2] = __uint_as_float(u.y << 16);
  o[3] = __uint_as_float(u.y & 0xffff0000u);
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  return static_cast<uint32_t>(float_to_bf16_bits(lo)) | (static_cast<uint32_t>(float_to_bf16_bits(hi)) << 16);
}

__device__ __forceinline__ void st_tf32x4(uint8_t *p, float a, float b, float c, float d) {
  *reinterpret_cast<uint4 *>(p) = make_uint4(tc::to_tf32(a), tc::to_tf32(b), tc::to_tf32(c), tc::to_tf32(d));
}

// Writes 32 consecutive float32 values as tf32 into one 128-byte swizzled row.
__device__ __forceinline__ void store_row_tf32(uint8_t *region_row_block, uint32_t row, const float (&v)[32]) {
#pragma unroll
  for (int c = 0; c < 8; ++c)
    st_tf32x4(region_row_block + tc::sw128(row, c), v[4 * c], v[4 * c + 1], v[4 * c + 2], v[4 * c + 3]);
}

// B4S holds S0^T as the K-major B operand of the chain product: row = value
// channel i, K = key channel j.  A state thread owns S^T[j][32*ch + x].
__device__ __forceinline__ void store_state_tf32(uint8_t *sB4S, int j, int ch, const float (&st)[32]) {
#pragma unroll
  for (int x = 0; x < 32; ++x)
    *reinterpret_cast<uint32_t *>(sB4S + kmaj_tf32(64, 32 * ch + x, j)) = tc::to_tf32(st[x]);
}

__global__ void __launch_bounds__(kThreads, 1) wkv7_chunk_kernel(const __grid_constant__ Maps maps, const Args A) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *sA1 = smem + OFF_A1;
  uint8_t *sB1 = smem + OFF_B1;
  uint8_t *sA3 = smem + OFF_A3;
  uint8_t *sB4S = smem + OFF_B4S;
  uint8_t *sB4V = smem + OFF_B4V;
  uint8_t *sB3 = smem + OFF_B3;
  uint8_t *sB2 = smem + OFF_B2;
  float *Ls = reinterpret_cast<float *>(smem + OFF_LS);
  float *Ts = reinterpret_cast<float *>(smem + OFF_TS);
  float *Zs = reinterpret_cast<float *>(smem + OFF_ZS);
  uint64_t *bar_tma = reinterpret_cast<uint64_t *>(smem + OFF_MISC);
  uint64_t *bar_mma = bar_tma + 1;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + OFF_MISC + 16);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + OFF_MISC + 20);
  float *GCs = reinterpret_cast<float *>(smem + OFF_MISC + MISC_GC);
  float *tot = reinterpret_cast<float *>(smem + OFF_MISC + MISC_TOT);

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int q = warp & 3;    // TMEM lane quadrant of this warp
  const int ch = warp >> 2;  // which half of a 64-column block this warp handles
  const int h = blockIdx.x;
  const int bidx = blockIdx.y;
  const SeqBounds sb = seq_bounds(A.cu_seqlens, bidx, A.T, A.total_T);
  if (sb.len < 0) return;
  const int nchunks = (sb.len + C - 1) / C;
  const bool hi_lanes = q >= 2;  // owns TMEM lanes 64..127
  const int j = tid & 63;        // for hi-lane threads: the key channel of its lane
  const long long pair = static_cast<long long>(bidx) * A.H + h;
  // operand-construction layout: 4 channels x 4 tokens per thread
  const int cq = 8 * (warp & 1) + (lane & 7), tg = 4 * (warp >> 1) + (lane >> 3);
  const int j0 = 4 * cq, t0 = 4 * tg;

  if (tid == 0) {
    tc::mbar_init(bar_tma, 1);
    tc::mbar_init(bar_mma, 1);
    tc::fence_mbar_init();
    *abort_flag = 0;
    for (int i = 0; i < 6; ++i) tc::prefetch_tensormap(&maps.m[i]);
  }
  if (warp == 0) {
    tc::tmem_alloc(tmem_slot, kTmemCols);
    tc::tmem_relinquish();
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t lane_base = static_cast<uint32_t>(32 * q) << 16;

  // state: hi-lane threads hold S^T[j][32*ch .. 32*ch+31] in float32
  float st[32];
  if (hi_lanes) {
#pragma unroll
    for (int x = 0; x < 32; ++x)
      st[x] = A.s_in ? A.s_in[pair * (kN * kN) + static_cast<long long>(32 * ch + x) * kN + j] : 0.f;
    store_state_tf32(sB4S, j, ch, st);
  }

  uint32_t tma_phase = 0, mma_phase = 0;
  bool tma_pending = false;
  if (tid == 0 && nchunks > 0) {
    tc::mbar_arrive_expect_tx(bar_tma, 6 * kTile);
    for (int i = 0; i < 6; ++i)
      tc::tma_load_3d(smem + OFF_RAW + i * kTile, &maps.m[i], bar_tma, 0, h, static_cast<int>(sb.start));
    tma_pending = true;
  }

  auto wait_mma = [&]() {
    if (tid == 0) {
      if (!tc::mbar_wait_bounded(bar_mma, mma_phase, kMaxPolls)) {
        *abort_flag = 1;
        report_device_error(A.err, kDevErrTimeout);
      }
    }
    mma_phase ^= 1u;
  };

  for (int c = 0; c < nchunks; ++c) {
    const int Lc = min(C, sb.len - c * C);
    // ---- this chunk's tiles have landed ---------------------------------------------------
    if (tid == 0) {
      if (!tc::mbar_wait_bounded(bar_tma, tma_phase, kMaxPolls)) {
        *abort_flag = 1;
        report_device_error(A.err, kDevErrTimeout);
      } else {
        tma_pending = false;
      }
      tma_phase ^= 1u;
    }
    __syncthreads();
    if (*abort_flag) break;

    // ---- P1: decay products and operands (4 channels x 4 tokens per thread) ---------------
    float G[4][4];  // Gamma_t for t = t0..t0+3 (rows) and channels j0..j0+3 (cols)
    {
      float wv[4][4];
#pragma unroll
      for (int tt = 0; tt < 4; ++tt) {
        if (t0 + tt < Lc) {
          raw4(smem, RAW_W, t0 + tt, j0, wv[tt]);
        } else {
#pragma unroll
          for (int e = 0; e < 4; ++e) wv[tt][e] = 1.f;
        }
      }
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        G[0][e] = wv[0][e];
        G[1][e] = G[0][e] * wv[1][e];
        G[2][e] = G[1][e] * wv[2][e];
        G[3][e] = G[2][e] * wv[3][e];
      }
      *reinterpret_cast<float4 *>(tot + tg * 64 + j0) = make_float4(G[3][0], G[3][1], G[3][2], G[3][3]);
    }
    __syncthreads();
    {
      float pre[4] = {1.f, 1.f, 1.f, 1.f};
#pragma unroll
      for (int g = 0; g < 15; ++g) {
        if (g < tg) {
          const float4 u = *reinterpret_cast<const float4 *>(tot + g * 64 + j0);
          pre[0] *= u.x;
          pre[1] *= u.y;
          pre[2] *= u.z;
          pre[3] *= u.w;
        }
      }
      float rr[4][4], kk[4][4], aa[4][4], bb[4][4], vv[4][4];
#pragma unroll
      for (int tt = 0; tt < 4; ++tt) {
        if (t0 + tt < Lc) {
          raw4(smem, RAW_R, t0 + tt, j0, rr[tt]);
          raw4(smem, RAW_K, t0 + tt, j0, kk[tt]);
          raw4(smem, RAW_A, t0 + tt, j0, aa[tt]);
          raw4(smem, RAW_B, t0 + tt, j0, bb[tt]);
          raw4(smem, RAW_V, t0 + tt, j0, vv[tt]);
        } else {
#pragma unroll
          for (int e = 0; e < 4; ++e) rr[tt][e] = kk[tt][e] = aa[tt][e] = bb[tt][e] = vv[tt][e] = 0.f;
        }
      }
      float Gp[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) Gp[e] = pre[e];  // Gamma_{t0 - 1}
#pragma unroll
      for (int tt = 0; tt < 4; ++tt) {
        const int t = t0 + tt;
        float Gt[4], inv[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          Gt[e] = pre[e] * G[tt][e];
          inv[e] = tc::rcp_approx(Gt[e]);
        }
        const uint32_t kofs = (j0 >> 5) * (128 * 128) + ((j0 & 31) >> 2);  // katom base + chunk index
        uint8_t *a1r = sA1 + (j0 >> 5) * (128 * 128);
        uint8_t *b1r = sB1 + (j0 >> 5) * (128 * 128);
        const uint32_t chunk = (j0 & 31) >> 2;
        (void)kofs;
        st_tf32x4(a1r + tc::sw128(t, chunk), rr[tt][0] * Gt[0], rr[tt][1] * Gt[1], rr[tt][2] * Gt[2],
                  rr[tt][3] * Gt[3]);
        const float At0 = aa[tt][0] * Gp[0], At1 = aa[tt][1] * Gp[1], At2 = aa[tt][2] * Gp[2],
                    At3 = aa[tt][3] * Gp[3];
        st_tf32x4(a1r + tc::sw128(64 + t, chunk), At0, At1, At2, At3);
        st_tf32x4(b1r + tc::sw128(t, chunk), bb[tt][0] * inv[0], bb[tt][1] * inv[1], bb[tt][2] * inv[2],
                  bb[tt][3] * inv[3]);
        st_tf32x4(b1r + tc::sw128(64 + t, chunk), kk[tt][0] * inv[0], kk[tt][1] * inv[1], kk[tt][2] * inv[2],
                  kk[tt][3] * inv[3]);
        // A3: A~^T as the MN-major bf16 A operand of MMA3 (M = channel, K = token)
        *reinterpret_cast<uint2 *>(sA3 + mnmaj_bf16(64, t, j0)) =
            make_uint2(pack_bf16x2(At0, At1), pack_bf16x2(At2, At3));
#pragma unroll
        for (int e = 0; e < 4; ++e) Gp[e] = Gt[e];
      }
      if (tg == 15) *reinterpret_cast<float4 *>(GCs + j0) = make_float4(Gp[0], Gp[1], Gp[2], Gp[3]);
      // V -> B4V (row = value channel, K = token), bf16 values are exact in tf32
#pragma unroll
      for (int e = 0; e < 4; ++e)
        *reinterpret_cast<uint4 *>(sB4V + kmaj_tf32(64, j0 + e, t0)) =
            make_uint4(__float_as_uint(vv[0][e]), __float_as_uint(vv[1][e]), __float_as_uint(vv[2][e]),
                       __float_as_uint(vv[3][e]));
    }
    tc::fence_proxy_async_smem();
    __syncthreads();

    // ---- MMA1 (tf32): D1 = [R~; A~] [B^; K^]^T, and the next chunk's tiles ---------------------
    if (tid == 0) {
      if (c + 1 < nchunks) {
        tc::mbar_arrive_expect_tx(bar_tma, 6 * kTile);
        for (int i = 0; i < 6; ++i)
          tc::tma_load_3d(smem + OFF_RAW + i * kTile, &maps.m[i], bar_tma, 0, h,
                          static_cast<int>(sb.start + static_cast<long long>(c + 1) * C));
        tma_pending = true;
      }
      tc::tc_fence_after();
      constexpr uint32_t idesc = tc::instr_desc(tc::kFmtTF32, 128, 128, false, false);
      const uint32_t a0 = smem_u32(sA1), b0 = smem_u32(sB1);
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
        const uint32_t off = (ks >> 2) * (128 * 128) + (ks & 3) * 32;
        tc::mma_ss(1, tmem + TM_D1, tc::smem_desc(a0 + off, 16, 1024), tc::smem_desc(b0 + off, 16, 1024), idesc,
                   ks > 0);
      }
      tc::mma_commit(bar_mma);
    }
    // D2 and A2 set-up from the operands (overlaps MMA1, which only reads A1 / B1)
    if (!hi_lanes) {
      // lanes t = 0..63: Q-part of D2 starts at R~[t][32ch .. 32ch+31] (read back from A1)
      const int t = q * 32 + lane;
      float rt[32];
      const uint8_t *rowblk = sA1 + ch * (128 * 128);
#pragma unroll
      for (int cc = 0; cc < 8; ++cc) {
        const uint4 u = *reinterpret_cast<const uint4 *>(rowblk + tc::sw128(t, cc));
        rt[4 * cc + 0] = __uint_as_float(u.x);
        rt[4 * cc + 1] = __uint_as_float(u.y);
        rt[4 * cc + 2] = __uint_as_float(u.z);
        rt[4 * cc + 3] = __uint_as_float(u.w);
      }
      tc::tmem_st32(tmem + lane_base + TM_D2 + 32 * ch, rt);
    } else {
      // lanes 64+j: B-^T[j][m] = Gamma_C[j] B^[m][j] -> A2; K-^T[j][m] = Gamma_C[j] K^[m][j] -> F-part of D2
      const float gc = GCs[j];
      float bv[32], kv[32], zero[32];
#pragma unroll
      for (int x = 0; x < 32; ++x) {
        const int m = 32 * ch + x;
        bv[x] = gc * __uint_as_float(*reinterpret_cast<const uint32_t *>(sB1 + kmaj_tf32(128, m, j)));
        kv[x] = gc * __uint_as_float(*reinterpret_cast<const uint32_t *>(sB1 + kmaj_tf32(128, 64 + m, j)));
        zero[x] = 0.f;
      }
      tc::tmem_st32(tmem + lane_base + TM_A2 + 32 * ch, bv);
      tc::tmem_st32(tmem + lane_base + TM_D2 + 64 + 32 * ch, kv);
      tc::tmem_st32(tmem + lane_base + TM_D2 + 32 * ch, zero);
    }
    tc::tmem_st_wait();
    wait_mma();
    tc::tc_fence_before();
    __syncthreads();
    if (*abort_flag) break;
    tc::tc_fence_after();

    // ---- P3: masks ------------------------------------------------------------------------------
    {
      const int t = q * 32 + lane - (hi_lanes ? 64 : 0);  // token row of this lane
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        float v[32];
        tc::tmem_ld32(tmem + lane_base + TM_D1 + 64 * ch + 32 * half, v);
        if (!hi_lanes) {
          // lanes 0..63: Mrb (ch 0) / Mrk (ch 1), keep m <= t
#pragma unroll
          for (int x = 0; x < 32; ++x)
            if (32 * half + x > t) v[x] = 0.f;
          tc::tmem_st32(tmem + lane_base + (ch == 0 ? TM_A2 : TM_D2 + 64) + 32 * half, v);
        } else {
          // lanes 64..127: Lab (ch 0) / Lak (ch 1), keep m < t
#pragma unroll
          for (int x = 0; x < 32; ++x)
            if (32 * half + x >= t) v[x] = 0.f;
          if (ch == 0) {
#pragma unroll
            for (int x = 0; x < 32; x += 4)
              *reinterpret_cast<float4 *>(Ls + t * LDL + 32 * half + x) = make_float4(v[x], v[x + 1], v[x + 2], v[x + 3]);
          } else {
            // A3 rows M = 64 + m' (Lak^T), K = t: bf16, one 128-byte row per thread
#pragma unroll
            for (int cc = 0; cc < 4; ++cc) {
              uint4 u;
              u.x = pack_bf16x2(v[8 * cc + 0], v[8 * cc + 1]);
              u.y = pack_bf16x2(v[8 * cc + 2], v[8 * cc + 3]);
              u.z = pack_bf16x2(v[8 * cc + 4], v[8 * cc + 5]);
              u.w = pack_bf16x2(v[8 * cc + 6], v[8 * cc + 7]);
              *reinterpret_cast<uint4 *>(sA3 + 64 * 128 + tc::sw128(t, 4 * half + cc)) = u;
            }
          }
        }
      }
      if (!hi_lanes) tc::tmem_st_wait();
    }
    tc::fence_proxy_async_smem();
    tc::tc_fence_before();
    __syncthreads();

    // ---- P4: Tinv = (I - Lab)^-1 -------------------------------------------------------------------
    if (warp < 2) {
      // diagonal 16x16 blocks: x = (I - L_ss)^-1 e_c by forward substitution (x_r = [r == c] + sum_{q<r} L_rq x_q)
      const int s = 2 * warp + (lane >> 4), cix = lane & 15, base = 16 * s;
      float x[16];
#pragma unroll
      for (int r = 0; r < 16; ++r) {
        float acc = (r == cix) ? 1.f : 0.f;
#pragma unroll
        for (int qq = 0; qq < r; ++qq) acc = fmaf(Ls[(base + r) * LDL + base + qq], x[qq], acc);
        x[r] = acc;
      }
#pragma unroll
      for (int r = 0; r < 16; ++r) Ts[(base + r) * LDT + base + cix] = x[r];
    } else {
      // zero the blocks above the block diagonal
      for (int e = tid - 64; e < 6 * 256; e += kThreads - 64) {
        const int blk = e >> 8, rr = (e >> 4) & 15, cc = e & 15;
        const int sr = blk < 3 ? 0 : (blk < 5 ? 1 : 2);
        const int sc = blk < 3 ? blk + 1 : (blk < 5 ? blk - 1 : 3);
        Ts[(16 * sr + rr) * LDT + 16 * sc + cc] = 0.f;
      }
    }
    __syncthreads();
    if (warp < 3) {
      // block column m = warp: T_sm = D_s sum_{q=m}^{s-1} L_sq T_qm, rows s = m+1..3, on warp-level tf32 mma
      const int m = warp;
      float *Zw = Zs + warp * (16 * 24);
#pragma unroll
      for (int s = 1; s < 4; ++s) {
        if (s > m) {
          float z[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
          for (int qq = 0; qq < 3; ++qq)
            if (qq >= m && qq < s)
              tc::block16_mma(z, Ls + (16 * s) * LDL + 16 * qq, LDL, Ts + (16 * qq) * LDT + 16 * m, LDT, lane);
          tc::block16_store(Zw, 24, z, lane);
          __syncwarp();
          float tb[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
          tc::block16_mma(tb, Ts + (16 * s) * LDT + 16 * s, LDT, Zw, 24, lane);
          tc::block16_store(Ts + (16 * s) * LDT + 16 * m, LDT, tb, lane);
          __syncwarp();
        }
      }
    }
    __syncthreads();
    {
      // Tinv -> B3 (bf16, K-major: row t, K = m)
      const int t = tid >> 2, m0 = (tid & 3) * 16;
#pragma unroll
      for (int cc = 0; cc < 2; ++cc) {
        const float *src = Ts + t * LDT + m0 + 8 * cc;
        uint4 u;
        u.x = pack_bf16x2(src[0], src[1]);
        u.y = pack_bf16x2(src[2], src[3]);
        u.z = pack_bf16x2(src[4], src[5]);
        u.w = pack_bf16x2(src[6], src[7]);
        *reinterpret_cast<uint4 *>(sB3 + tc::sw128(t, (m0 >> 3) + cc)) = u;
      }
    }
    tc::fence_proxy_async_smem();
    __syncthreads();

    // ---- MMA3 (bf16): D3 = [A~^T; Lak^T] Tinv^T ---------------------------------------------------
    if (tid == 0) {
      tc::tc_fence_after();
      constexpr uint32_t idesc = tc::instr_desc(tc::kFmtBF16, 128, 64, true, false);
      const uint32_t a0 = smem_u32(sA3), b0 = smem_u32(sB3);
#pragma unroll
      for (int ks = 0; ks < 4; ++ks)
        tc::mma_ss(0, tmem + TM_D3, tc::smem_desc(a0 + ks * 2048, 64 * 128, 1024),
                   tc::smem_desc(b0 + ks * 32, 16, 1024), idesc, ks > 0);
      tc::mma_commit(bar_mma);
    }
    wait_mma();
    __syncthreads();
    if (*abort_flag) break;
    tc::tc_fence_after();

    // ---- P6: D3 -> B2 (tf32 K-major: row n = column of [W~ U~], K = token) ---------------------------
    {
      float v[32];
      tc::tmem_ld32(tmem + lane_base + TM_D3 + 32 * ch, v);
      store_row_tf32(sB2 + ch * (128 * 128), q * 32 + lane, v);
    }
    tc::fence_proxy_async_smem();
    tc::tc_fence_before();
    __syncthreads();

    // ---- MMA2 (tf32, A from TMEM): D2 += [Mrb; B-^T] [W~ U~]; then MMA4 ------------------------------
    if (tid == 0) {
      tc::tc_fence_after();
      constexpr uint32_t idesc2 = tc::instr_desc(tc::kFmtTF32, 128, 128, false, false);
      const uint32_t b2 = smem_u32(sB2);
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
        const uint32_t off = (ks >> 2) * (128 * 128) + (ks & 3) * 32;
        tc::mma_ts_tf32(tmem + TM_D2, tmem + TM_A2 + 8 * ks, tc::smem_desc(b2 + off, 16, 1024), idesc2, 1);
      }
      tc::mma_commit(bar_mma);
    }
    wait_mma();
    __syncthreads();
    if (*abort_flag) break;

    // ---- MMA4 (tf32, A from TMEM): D4 = [Q P; E F] [S0^T; V] ------------------------------------------
    if (tid == 0) {
      tc::tc_fence_after();
      constexpr uint32_t idesc4 = tc::instr_desc(tc::kFmtTF32, 128, 64, false, false);
      const uint32_t bs = smem_u32(sB4S), bvv = smem_u32(sB4V);
#pragma unroll
      for (int ks = 0; ks < 16; ++ks) {
        const uint32_t base = ks < 8 ? bs : bvv;
        const uint32_t kk = ks & 7;
        const uint32_t off = (kk >> 2) * (64 * 128) + (kk & 3) * 32;
        tc::mma_ts_tf32(tmem + TM_D4, tmem + TM_D2 + 8 * ks, tc::smem_desc(base + off, 16, 1024), idesc4, ks > 0);
      }
      tc::mma_commit(bar_mma);
    }
    wait_mma();
    __syncthreads();
    if (*abort_flag) break;
    tc::tc_fence_after();

    // ---- P8: outputs and state ------------------------------------------------------------------------
    {
      float v[32];
      tc::tmem_ld32(tmem + lane_base + TM_D4 + 32 * ch, v);
      if (!hi_lanes) {
        const int t = q * 32 + lane;
        if (t < Lc) {
          const long long tok = sb.start + static_cast<long long>(c) * C + t;
          uint16_t *dst = A.y + (tok * A.H + h) * kN + 32 * ch;
#pragma unroll
          for (int cc = 0; cc < 4; ++cc) {
            uint4 u;
            u.x = pack_bf16x2(v[8 * cc + 0], v[8 * cc + 1]);
            u.y = pack_bf16x2(v[8 * cc + 2], v[8 * cc + 3]);
            u.z = pack_bf16x2(v[8 * cc + 4], v[8 * cc + 5]);
            u.w = pack_bf16x2(v[8 * cc + 6], v[8 * cc + 7]);
            *reinterpret_cast<uint4 *>(dst + 8 * cc) = u;
          }
        }
      } else {
        const float gc = GCs[j];
#pragma unroll
        for (int x = 0; x < 32; ++x) st[x] = fmaf(gc, st[x], v[x]);
        store_state_tf32(sB4S, j, ch, st);
      }
    }
    tc::fence_proxy_async_smem();
    tc::tc_fence_before();
  }

  __syncthreads();
  if (tid == 0 && tma_pending) {
    // an aborted run may leave one tile load in flight: let it land (bounded)
    (void)tc::mbar_wait_bounded(bar_tma, tma_phase, kMaxPolls);
  }
  if (hi_lanes) {
#pragma unroll
    for (int x = 0; x < 32; ++x) A.s_out[pair * (kN * kN) + static_cast<long long>(32 * ch + x) * kN + j] = st[x];
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  if (warp == 0) tc::tmem_dealloc(tmem, kTmemCols);
}

// ---- host side -----------------------------------------------------------------------------------

typedef CUresult (*PFN_encodeTiled)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                    const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                    CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static PFN_encodeTiled get_encode() {
  static PFN_encodeTiled fn = nullptr;
  static bool tried = false;
  if (!tried) {
    tried = true;
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_encodeTiled>(p);
  }
  return fn;
}

static bool make_map(CUtensorMap *map, const void *base, long long tokens, int H) {
  PFN_encodeTiled enc = get_encode();
  if (enc == nullptr) return false;
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(kN), static_cast<cuuint64_t>(H),
                              static_cast<cuuint64_t>(tokens)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(kN) * 2, static_cast<cuuint64_t>(H) * kN * 2};
  const cuuint32_t box[3] = {static_cast<cuuint32_t>(kN), 1, static_cast<cuuint32_t>(C)};
  const cuuint32_t estr[3] = {1, 1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace chunk

cudaError_t launch_chunk(const uint16_t *r, const uint16_t *w, const uint16_t *k, const uint16_t *v,
                         const uint16_t *a, const uint16_t *b, const float *s_in, uint16_t *y, float *s_out,
                         const int32_t *cu_seqlens, int B, int T, long long total_T, int H, int *err_word,
                         cudaStream_t stream) {
  using namespace chunk;
  if (total_T > 0x7fffffffLL || H > 0xffff || B > 65535) return cudaErrorInvalidValue;
  Maps maps;
  const void *ops[6] = {r, w, k, a, b, v};
  const long long tokens = total_T > 0 ? total_T : 1;
  for (int i = 0; i < 6; ++i) {
    // a zero-token call still needs a valid map; it never issues a load
    if (!make_map(&maps.m[i], ops[i] ? ops[i] : static_cast<const void *>(s_out), tokens, H))
      return cudaErrorInvalidValue;
  }
  Args args{y, s_in, s_out, cu_seqlens, T, total_T, H, err_word};
  cudaError_t e = cudaFuncSetAttribute(wkv7_chunk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(kSmemBytes));
  if (e != cudaSuccess) return e;
  dim3 grid(H, B);
  wkv7_chunk_kernel<<<grid, kThreads, kSmemBytes, stream>>>(maps, args);
  return cudaGetLastError();
}

}  // namespace rwkv7
