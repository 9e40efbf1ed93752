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
constexpr uint32_t kTile = C * kN * 2;           // one bf16 64x64 tile
constexpr uint32_t OFF_RAW = 0;                  // r w k a b v tiles, row-major [token][channel]
constexpr uint32_t OFF_A1 = OFF_RAW + 6 * kTile; // tf32 K-major 128x64 (32 KB); later B3 + Lab
constexpr uint32_t OFF_B1 = OFF_A1 + 32768;      // tf32 K-major 128x64 (32 KB); later Tinv, then B2
constexpr uint32_t OFF_A3 = OFF_B1 + 32768;      // bf16 MN-major M=128 x K=64 (16 KB)
constexpr uint32_t OFF_B4 = OFF_A3 + 16384;      // tf32 K-major N=64 (value i) x K=128 (key j | token m) (32 KB)
constexpr uint32_t OFF_MISC = OFF_B4 + 32768;
constexpr uint32_t OFF_B3 = OFF_A1;              // bf16 K-major 64x64 (8 KB)
constexpr uint32_t OFF_LS = OFF_A1 + 8192;       // float [64][65]  (Lab, strictly lower)
constexpr uint32_t OFF_TS = OFF_B1;              // float [64][65]  (Tinv in float32)
constexpr uint32_t OFF_ZS = OFF_B1 + 64 * 65 * 4;  // float [3][16][17]
constexpr uint32_t OFF_B2 = OFF_B1;              // tf32 K-major 128x64 (32 KB)
constexpr uint32_t kSmemBytes = OFF_MISC + 2048 + 1024;  // + misc + alignment slack
constexpr int LDS = 65;                          // padded row stride of Ls / Ts

static_assert(OFF_LS + 64 * LDS * 4 <= OFF_B1, "Lab scratch overflows its region");
static_assert(OFF_ZS + 3 * 16 * 17 * 4 <= OFF_A3, "Tinv scratch overflows its region");

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

// address helpers (byte offsets inside a region)
__device__ __forceinline__ uint32_t kmaj_tf32(uint32_t rows, uint32_t row, uint32_t k) {
  return (k >> 5) * (rows * 128u) + tc::sw128(row, (k & 31u) >> 2) + (k & 3u) * 4u;
}
__device__ __forceinline__ uint32_t mnmaj_bf16(uint32_t krows, uint32_t k, uint32_t mn) {
  return (mn >> 6) * (krows * 128u) + tc::sw128(k, (mn & 63u) >> 3) + (mn & 7u) * 2u;
}

__device__ __forceinline__ float raw_at(const uint16_t *raw, int tile, int t, int j) {
  return bf16_bits_to_float(raw[tile * (C * kN) + t * kN + j]);
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  return static_cast<uint32_t>(float_to_bf16_bits(lo)) | (static_cast<uint32_t>(float_to_bf16_bits(hi)) << 16);
}

// Writes 32 consecutive float32 values as tf32 into one 128-byte swizzled row.
__device__ __forceinline__ void store_row_tf32(uint8_t *region_row_block, uint32_t row, const float (&v)[32]) {
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    uint4 q;
    q.x = tc::to_tf32(v[4 * c + 0]);
    q.y = tc::to_tf32(v[4 * c + 1]);
    q.z = tc::to_tf32(v[4 * c + 2]);
    q.w = tc::to_tf32(v[4 * c + 3]);
    *reinterpret_cast<uint4 *>(region_row_block + tc::sw128(row, c)) = q;
  }
}

// B4 holds [S0^T; V] as the K-major B operand of the chain product: row n is
// the value channel i, K runs over key channels j (0..63) then tokens m
// (64..127).  A channel thread owns S^T[j][32*ch + x] = S[32*ch + x][j], i.e.
// column K = j of rows 32*ch .. 32*ch+31.
__device__ __forceinline__ void store_state_tf32(uint8_t *sB4, int j, int ch, const float (&st)[32]) {
#pragma unroll
  for (int x = 0; x < 32; ++x)
    *reinterpret_cast<uint32_t *>(sB4 + kmaj_tf32(64, 32 * ch + x, j)) = tc::to_tf32(st[x]);
}

__global__ void __launch_bounds__(kThreads, 1) wkv7_chunk_kernel(const __grid_constant__ Maps maps, const Args A) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint16_t *raw = reinterpret_cast<const uint16_t *>(smem + OFF_RAW);
  uint8_t *sA1 = smem + OFF_A1;
  uint8_t *sB1 = smem + OFF_B1;
  uint8_t *sA3 = smem + OFF_A3;
  uint8_t *sB4 = smem + OFF_B4;
  uint8_t *sB3 = smem + OFF_B3;
  uint8_t *sB2 = smem + OFF_B2;
  float *Ls = reinterpret_cast<float *>(smem + OFF_LS);
  float *Ts = reinterpret_cast<float *>(smem + OFF_TS);
  float *Zs = reinterpret_cast<float *>(smem + OFF_ZS);
  uint64_t *bar_tma = reinterpret_cast<uint64_t *>(smem + OFF_MISC);
  uint64_t *bar_mma = bar_tma + 1;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + OFF_MISC + 16);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + OFF_MISC + 20);
  float *gtot = reinterpret_cast<float *>(smem + OFF_MISC + 64);  // [2][64]

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int q = warp & 3;    // TMEM lane quadrant of this warp
  const int ch = warp >> 2;  // which half of the columns this warp handles
  const int h = blockIdx.x;
  const int bidx = blockIdx.y;
  const SeqBounds sb = seq_bounds(A.cu_seqlens, bidx, A.T, A.total_T);
  if (sb.len < 0) return;
  const int nchunks = (sb.len + C - 1) / C;
  const bool chan_thread = q >= 2;          // channel-major role (owns TMEM lanes 64..127)
  const int j = tid & 63;                   // channel of a channel-major thread
  const long long pair = static_cast<long long>(bidx) * A.H + h;

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

  // state: channel threads hold S^T[j][32*ch .. 32*ch+31] in float32
  float st[32];
  if (chan_thread) {
#pragma unroll
    for (int x = 0; x < 32; ++x)
      st[x] = A.s_in ? A.s_in[pair * (kN * kN) + static_cast<long long>(32 * ch + x) * kN + j] : 0.f;
    store_state_tf32(sB4, j, ch, st);
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
    // ---- P0: this chunk's tiles have landed --------------------------------------------
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

    // ---- P1: decay products and operands ------------------------------------------------
    float G[32];   // channel threads: local cumulative products of w over their 32 tokens
    float GC = 1.f;
    if (chan_thread) {
      const int t0 = 32 * ch;
      float p = 1.f;
#pragma unroll
      for (int tt = 0; tt < 32; ++tt) {
        const int t = t0 + tt;
        const float wv = t < Lc ? raw_at(raw, RAW_W, t, j) : 1.f;
        p *= wv;
        G[tt] = p;
      }
      gtot[ch * 64 + j] = p;
    } else {
      // V (token m, value channel i) -> B4 element (row i, K = 64 + m); bf16 is exact in tf32.
      // Lanes walk the 32 channels in a rotated order to spread shared-memory banks.
      const int rid = (ch * 64) + q * 32 + lane;  // 0..127
      const int m = rid & 63, ih = rid >> 6;
#pragma unroll 8
      for (int x = 0; x < 32; ++x) {
        const int i = 32 * ih + ((x + lane) & 31);
        const float vv = m < Lc ? raw_at(raw, RAW_V, m, i) : 0.f;
        *reinterpret_cast<uint32_t *>(sB4 + kmaj_tf32(64, i, 64 + m)) = __float_as_uint(vv);
      }
    }
    __syncthreads();
    if (chan_thread) {
      const float g0 = gtot[j], g1 = gtot[64 + j];
      GC = g0 * g1;
      const float pre = ch ? g0 : 1.f;
      float Bbar[32], Kbar[32];
#pragma unroll
      for (int tt = 0; tt < 32; ++tt) {
        const int t = 32 * ch + tt;
        const bool valid = t < Lc;
        const float Gt = pre * G[tt];
        const float Gp = tt == 0 ? pre : pre * G[tt - 1];
        const float rv = valid ? raw_at(raw, RAW_R, t, j) : 0.f;
        const float kv = valid ? raw_at(raw, RAW_K, t, j) : 0.f;
        const float av = valid ? raw_at(raw, RAW_A, t, j) : 0.f;
        const float bv = valid ? raw_at(raw, RAW_B, t, j) : 0.f;
        const float inv = __frcp_rn(Gt);
        const float At = av * Gp;
        *reinterpret_cast<uint32_t *>(sA1 + kmaj_tf32(128, t, j)) = tc::to_tf32(rv * Gt);
        *reinterpret_cast<uint32_t *>(sA1 + kmaj_tf32(128, 64 + t, j)) = tc::to_tf32(At);
        *reinterpret_cast<uint32_t *>(sB1 + kmaj_tf32(128, t, j)) = tc::to_tf32(bv * inv);
        *reinterpret_cast<uint32_t *>(sB1 + kmaj_tf32(128, 64 + t, j)) = tc::to_tf32(kv * inv);
        *reinterpret_cast<uint16_t *>(sA3 + mnmaj_bf16(64, t, j)) = float_to_bf16_bits(At);
        const float ratio = GC * inv;
        Bbar[tt] = bv * ratio;
        Kbar[tt] = kv * ratio;
      }
      float zeros[32];
#pragma unroll
      for (int x = 0; x < 32; ++x) zeros[x] = 0.f;
      tc::tmem_st32(tmem + lane_base + TM_A2 + 32 * ch, Bbar);
      tc::tmem_st32(tmem + lane_base + TM_D2 + 64 + 32 * ch, Kbar);
      tc::tmem_st32(tmem + lane_base + TM_D2 + 32 * ch, zeros);
      tc::tmem_st_wait();
    }
    tc::fence_proxy_async_smem();
    __syncthreads();
    if (!chan_thread) {
      // Q-part init of D2: row t gets R~[t][32ch .. 32ch+31], read back from A1
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
      tc::tmem_st_wait();
    }
    tc::tc_fence_before();
    __syncthreads();

    // ---- MMA1 (tf32): D1 = [R~; A~] [B^; K^]^T ----------------------------------------------
    if (tid == 0) {
      tc::tc_fence_after();
      // the raw tiles are consumed: prefetch the next chunk
      if (c + 1 < nchunks) {
        tc::mbar_arrive_expect_tx(bar_tma, 6 * kTile);
        for (int i = 0; i < 6; ++i)
          tc::tma_load_3d(smem + OFF_RAW + i * kTile, &maps.m[i], bar_tma, 0, h,
                          static_cast<int>(sb.start + static_cast<long long>(c + 1) * C));
        tma_pending = true;
      }
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
    wait_mma();
    __syncthreads();
    if (*abort_flag) break;
    tc::tc_fence_after();

    // ---- P3: masks --------------------------------------------------------------------------
    {
      const int t = q * 32 + lane - (chan_thread ? 64 : 0);  // token row of this lane
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        float v[32];
        tc::tmem_ld32(tmem + lane_base + TM_D1 + 64 * ch + 32 * half, v);
        if (!chan_thread) {
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
            for (int x = 0; x < 32; ++x) Ls[t * LDS + 32 * half + x] = v[x];
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
      if (!chan_thread) tc::tmem_st_wait();
    }
    tc::fence_proxy_async_smem();
    tc::tc_fence_before();
    __syncthreads();

    // ---- P4: Tinv = (I - Lab)^-1 --------------------------------------------------------------
    if (tid < 64) {
      // diagonal 16x16 blocks, one column per thread, forward substitution
      const int s = tid >> 4, cix = tid & 15, base = 16 * s;
      float x[16];
#pragma unroll
      for (int r = 0; r < 16; ++r) {
        float acc = (r == cix) ? 1.f : 0.f;
        if (r > cix) {
#pragma unroll
          for (int qq = 0; qq < 16; ++qq)
            if (qq >= cix && qq < r) acc = fmaf(Ls[(base + r) * LDS + base + qq], x[qq], acc);
        }
        x[r] = acc;
      }
#pragma unroll
      for (int r = 0; r < 16; ++r) Ts[(base + r) * LDS + base + cix] = x[r];
    } else {
      // zero the blocks above the block diagonal
      for (int e = tid - 64; e < 6 * 256; e += kThreads - 64) {
        const int blk = e >> 8, rr = (e >> 4) & 15, cc = e & 15;
        const int sr = blk < 3 ? 0 : (blk < 5 ? 1 : 2);
        const int sc = blk < 3 ? blk + 1 : (blk < 5 ? blk - 1 : 3);
        Ts[(16 * sr + rr) * LDS + 16 * sc + cc] = 0.f;
      }
    }
    __syncthreads();
    {
      const int r = tid >> 4, cix = tid & 15;
      for (int s = 1; s < 4; ++s) {
        for (int m = 0; m < s; ++m) {
          float acc = 0.f;
          for (int qq = 16 * m; qq < 16 * s; ++qq) acc = fmaf(Ls[(16 * s + r) * LDS + qq], Ts[qq * LDS + 16 * m + cix], acc);
          Zs[(m * 16 + r) * 17 + cix] = acc;
        }
        __syncthreads();
        for (int m = 0; m < s; ++m) {
          float acc = 0.f;
#pragma unroll
          for (int p = 0; p < 16; ++p) acc = fmaf(Ts[(16 * s + r) * LDS + 16 * s + p], Zs[(m * 16 + p) * 17 + cix], acc);
          Ts[(16 * s + r) * LDS + 16 * m + cix] = acc;
        }
        __syncthreads();
      }
    }
    {
      // Tinv -> B3 (bf16, K-major: row t, K = m)
      const int t = tid >> 2, m0 = (tid & 3) * 16;
#pragma unroll
      for (int cc = 0; cc < 2; ++cc) {
        const float *src = Ts + t * LDS + m0 + 8 * cc;
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

    // ---- MMA3 (bf16): D3 = [A~^T; Lak^T] Tinv^T ---------------------------------------------
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

    // ---- P6: D3 -> B2 (tf32 K-major: row n = column of [W~ U~], K = token) -------------------
    {
      float v[32];
      tc::tmem_ld32(tmem + lane_base + TM_D3 + 32 * ch, v);
      store_row_tf32(sB2 + ch * (128 * 128), q * 32 + lane, v);
    }
    tc::fence_proxy_async_smem();
    tc::tc_fence_before();
    __syncthreads();

    // ---- MMA2 (tf32, A from TMEM): D2 += [Mrb; B-^T] [W~ U~] ----------------------------------
    if (tid == 0) {
      tc::tc_fence_after();
      constexpr uint32_t idesc = tc::instr_desc(tc::kFmtTF32, 128, 128, false, false);
      const uint32_t b0 = smem_u32(sB2);
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
        const uint32_t off = (ks >> 2) * (128 * 128) + (ks & 3) * 32;
        tc::mma_ts_tf32(tmem + TM_D2, tmem + TM_A2 + 8 * ks, tc::smem_desc(b0 + off, 16, 1024), idesc, 1);
      }
      tc::mma_commit(bar_mma);
    }
    wait_mma();
    __syncthreads();
    if (*abort_flag) break;

    // ---- MMA4 (tf32, A from TMEM): D4 = [Q P; E F] [S0^T; V] ----------------------------------
    if (tid == 0) {
      tc::tc_fence_after();
      constexpr uint32_t idesc = tc::instr_desc(tc::kFmtTF32, 128, 64, false, false);
      const uint32_t b0 = smem_u32(sB4);
#pragma unroll
      for (int ks = 0; ks < 16; ++ks) {
        const uint32_t off = (ks >> 2) * (64 * 128) + (ks & 3) * 32;
        tc::mma_ts_tf32(tmem + TM_D4, tmem + TM_D2 + 8 * ks, tc::smem_desc(b0 + off, 16, 1024), idesc, ks > 0);
      }
      tc::mma_commit(bar_mma);
    }
    wait_mma();
    __syncthreads();
    if (*abort_flag) break;
    tc::tc_fence_after();

    // ---- P8: outputs and state ---------------------------------------------------------------
    {
      float v[32];
      tc::tmem_ld32(tmem + lane_base + TM_D4 + 32 * ch, v);
      if (!chan_thread) {
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
#pragma unroll
        for (int x = 0; x < 32; ++x) st[x] = fmaf(GC, st[x], v[x]);
        store_state_tf32(sB4, j, ch, st);
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
  if (chan_thread) {
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
