// wkv7_pipe.cu -- chunked prefill of the x070 recurrence on the tcgen05 tensor cores as a
// warp-specialised pipeline with three chunks in flight per SM (the pages' "GPT mode": the
// parallel, sequence-at-once evaluation that yields the RNN-mode state; RWKV-LM README copy,
// oa0.com/c/1004164, and RWKV-7 G0 7.2B walkthrough, lshu.cn/news/198401, sections 3.2 and 7.1).
//
// Per (b, h) and chunk of C = 64 tokens, with Gamma_t = prod_{u<=t} w_u inside the chunk, the
// recurrence S <- S diag(w) + (S a) b^T + v k^T, y = S r unrolls to (WY / UT form; rows are tokens,
// columns channels):
//
//   A~ = a*Gamma_{t-1}  R~ = r*Gamma_t  B^ = b/Gamma_t  K^ = k/Gamma_t
//   B- = b*Gamma_C/Gamma_t  K- = k*Gamma_C/Gamma_t  (Gamma_C: whole chunk)
//   MMA1  (tf32)  [Mrb Mrk; Lab Lak] = [R~; A~] [B^; K^]^T, causally masked (strict for L*)
//   inverse       Tinv = (I - Lab)^-1 (unit lower triangular)
//   MMA3  (bf16)  [W~ U~]^T = [A~^T; Lak^T] Tinv^T
//   MMA2  (bf16)  [Q P; E F] = [R~ Mrk; 0 K-^T] + [Mrb; B-^T] [W~ U~]
//   MMA4a (tf32)  D4 = [P; F] V                     (no state involved)
//   MMA4b (tf32)  D4 += [Q; E] S0^T = [Y; X],   S_C^T = diag(Gamma_C) S0^T + X
//
// Everything up to MMA4a is independent of the chunk's start state, so one CTA per SM runs the
// chunks of its (b, h) pairs through a pipeline: while chunk n is in the state chain (MMA4b, the
// state update, y), chunk n+1 is in the masks / inverse stage and chunk n+2 in the operand
// preparation.  Warp roles (448 threads):
//   warp 0      lane 0 issues every MMA (one tcgen05.mma holds the issuing thread for about as long
//               as the tensor pipe needs for it, 70-120 cycles at these shapes, so the tensor pipe,
//               about 2.35 K cycles per chunk, is the limit)
//   warp 1      lane 0 loads the operand tiles by TMA into a ring of 8 slots
//   warps 2-3   the state chain: TMEM lanes 64..127, the float32 state of column j in registers
//   warps 4-7   operand preparation: decay products, [R~; A~] (tf32, into TMEM: MMA1 reads its A
//               operand there), [B^; K^] (tf32, shared memory, two buffers), V^T
//   warps 8-11  the causal masks, the D2 set-up, the inverse, D3 -> B2
//   warps 12-13 y: TMEM lanes 0..63, one token row per thread
//
// Every tf32 operand is K-major (a tf32 MMA given a 128-byte-swizzled MN-major operand produced
// zeros on B200).  The products whose rounding reaches y directly (MMA1, MMA4) run in tf32; MMA3 and
// MMA2 in bf16.  The state is kept in float32 registers; only its tf32 copy feeds MMA4b, and
// diag(Gamma_C) S0^T is applied in float32.
//
// Domain: the factors B^, K^ divide by Gamma_t.  A chunk whose decay product Gamma_C falls below
// 2^-100 in some channel (or is not a number) is flagged by the preparation; its tensor-core results
// are discarded and the state warps run that chunk token by token in float32 (exact for every w in
// [0, 1], about 20x slower than a tensor-core chunk).  The model's decays never trigger it:
// exp(-e^-0.5 sigmoid(x)) >= 0.5452, and 0.5452^64 > 2^-57.
#include <cuda.h>

#include <mutex>

#include "common.cuh"
#include "launch.h"
#include "tc_ptx.cuh"

namespace rwkv7 {
namespace pipe {

constexpr int C = 64;
constexpr int NS = 8;                       // raw-tile ring slots
constexpr uint32_t kTile = C * kN * 2;      // one bf16 64 x 64 tile
constexpr int kThreads = 14 * 32;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kMaxPolls = 1u << 22;    // bounded mbarrier waits at exit
constexpr uint32_t kSuspendNs = 1000000;    // a waiting thread sleeps up to 1 ms per poll
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // a wait gives up after 2 s
constexpr float kGammaMin = 7.8886090522101181e-31f;  // 2^-100

// warp roles
constexpr int W_MMA = 0, W_TMA = 1, W_ST = 2, W_PREP = 4, W_S2 = 8, W_Y = 12;

// TMEM columns
constexpr uint32_t TM_X = 0;     // 2 x 128, slot n & 1: D1 of chunk n, then its D2
constexpr uint32_t TM_D4 = 256;  // 2 x 64, slot n & 1: D3 of chunk n, then its D4
constexpr uint32_t TM_A2 = 384;  // 2 x 32, slot n & 1: A operand [Mrb; B-^T] of MMA2 (bf16 pairs)
constexpr uint32_t TM_A1 = 448;  // 64: A operand [R~; A~] of MMA1 (tf32), one chunk at a time

// shared memory map (bytes from a 1024-aligned base)
constexpr uint32_t OFF_RAW = 0;                    // NS tiles [token][channel], 128-byte swizzled
constexpr uint32_t OFF_B1 = OFF_RAW + NS * kTile;  // 2 x tf32 K-major [B^; K^] 128 x 64, slot n & 1
constexpr uint32_t OFF_VT = OFF_B1 + 2 * 32768;    // tf32 K-major V^T: row vrow(i), K = token
constexpr uint32_t OFF_B4S = OFF_VT + 16384;       // tf32 K-major S0: row vrow(i), K = j (fallback: float [64][64])
constexpr uint32_t OFF_A3 = OFF_B4S + 16384;       // bf16 MN-major [A~^T; Lak^T]
constexpr uint32_t OFF_B3 = OFF_A3 + 16384;        // bf16 K-major Tinv (row t, K = t'); B2 from here on
constexpr int LDL = 68;   // row stride (floats) of Lab: conflict-free as an mma A operand
constexpr int LDTB = 24;  // row stride of the 16x16 fp32 blocks of Tinv
constexpr int LDZ = 20;   // row stride of the 16x16 scratch products
constexpr uint32_t OFF_ZS = OFF_B3 + 8192;                 // float [6][16][LDZ] (7680 B, then 512 B unused)
constexpr uint32_t OFF_B2 = OFF_B3;                        // bf16 K-major [W~ U~]^T over B3 and Zs (16 KB)
constexpr uint32_t OFF_LS = OFF_B3 + 16384;                // float [64][LDL]
constexpr uint32_t OFF_TS = OFF_LS + 64 * LDL * 4;         // float [6][16][LDTB]
constexpr uint32_t OFF_MISC = OFF_TS + 6 * 16 * LDTB * 4;
constexpr uint32_t MISC_WORDS = 320;   // tmem slot, abort flag, group decisions
constexpr uint32_t MISC_GC = 512;      // float [4][64]: Gamma_C by ring slot n % 4
constexpr uint32_t MISC_GFLAG = 1536;  // uint32 [4]: nonzero = chunk out of the factorised domain
constexpr uint32_t MISC_TOT = 1600;    // float [8][64]: decay products of the token octets (preparation)
constexpr uint32_t MISC_FB = 3648;     // float [2][6][64]: per-token vectors of the token-by-token path
constexpr uint32_t MISC_END = MISC_FB + 2 * 6 * 64 * 4;
constexpr uint32_t kSmemBytes = OFF_MISC + MISC_END + 1024;
static_assert(kSmemBytes <= 232448, "shared memory over the sm_100 limit");
static_assert(OFF_B3 % 1024 == 0 && OFF_A3 % 1024 == 0 && OFF_B2 % 1024 == 0, "operand alignment");
static_assert(OFF_ZS + 6 * 16 * LDZ * 4 <= OFF_B2 + 16384, "B2 covers B3 and Zs");

// mbarriers (count 1 unless noted)
enum {
  B_RAW_FULL = 0,     // [NS] tile landed (tx bytes)
  B_RAW_EMPTY = 8,    // [NS] preparation done with the slot
  B_AB_FULL = 16,     // A1 (TMEM), B1 slot, Gamma_C written (preparation of chunk n)
  B_A1_EMPTY = 17,    // A1 read by the mask stage of chunk n (count 4: one per warp of the stage)
  B_VT_FULL = 18,     // V^T of chunk n written
  B_M1 = 19,          // MMA1 of chunk n done
  B_B3 = 20,          // A3, B3 written
  B_M3 = 21,          // MMA3 done
  B_B2 = 22,          // B2 written, D2 set up (TMEM), A2 written
  B_M2 = 23,          // MMA2 done (B2 = B3 + Zs free)
  B_M4A = 24,         // MMA4a done (V^T free)
  B_S_FULL = 25,      // S0 of chunk n in B4S
  B_M4 = 26,          // [2] MMA4b of chunk n done, slot n & 1
  B_D4_EMPTY = 28,    // [2] D4 slot read out (count 2: state warps, y warps)
  B_GC = 30,          // [4] Gamma_C and the domain flag of chunk n, slot n % 4
  B_B1_EMPTY = 34,    // [2] B1 slot read by MMA1 and the mask stage of chunk n
  B_DRAIN = 36,       // every MMA of the CTA done (one commit at the end)
  kNumBars = 37
};
static_assert(kNumBars * 8 <= MISC_WORDS, "barrier area");

// named barriers (0 is __syncthreads)
constexpr int NB_PREP = 1, NB_S2 = 2, NB_LS = 3, NB_ST = 4, NB_Y = 5;

// Named barriers in their non-aligned form (barrier.sync / barrier.arrive), so a warp whose lanes arrive
// from different branches (a group leader that polled an mbarrier) is still counted correctly; callers
// reconverge with __syncwarp() before any .sync.aligned instruction.
__device__ __forceinline__ void nbar_sync(int id, int n) {
  asm volatile("barrier.sync %0, %1;\n" ::"r"(id), "r"(n) : "memory");
}
__device__ __forceinline__ void nbar_arrive(int id, int n) {
  asm volatile("barrier.arrive %0, %1;\n" ::"r"(id), "r"(n) : "memory");
}

struct Maps {
  CUtensorMap m[6];  // w, r, a, b, k, v: dims {64, H, tokens}, box {64, 1, 64}, 128-byte swizzle
};

struct Args {
  const uint16_t *op[6];  // w, r, a, b, k, v: [tokens, H, 64] (the token-by-token path reads them)
  uint16_t *y;
  const float *s_in;
  float *s_out;
  const int32_t *cu_seqlens;
  int T;
  long long total_T;
  int H;
  long long BH;
  int *err;
  const float *k_k;          // model-native inputs: [H, 64] key scale, nullptr = ones
  const float *ln_w, *ln_b;  // group-norm epilogue: [H, 64], nullptr = ones / zeros
  float *states;             // nullptr, or [B, H, nck, 64, 64]: the state before every chunk (dense T)
  int nck;
};
enum { OP_W = 0, OP_R = 1, OP_A = 2, OP_B = 3, OP_K = 4, OP_V = 5 };

// The chunk sequence of one CTA: pairs blockIdx.x, blockIdx.x + gridDim.x, ... (b, h) with a
// non-empty sequence, each pair's chunks in order.  Every role walks the same sequence.
struct ChunkIt {
  long long pair, start, tok0;
  int h, c, nck, len, Lc;
};
__device__ __noinline__ bool pair_load(const Args &A, long long pair, ChunkIt &it) {
  const int b = static_cast<int>(pair / A.H);
  const SeqBounds sb = seq_bounds(A.cu_seqlens, b, A.T, A.total_T);
  if (sb.len <= 0) return false;
  it.pair = pair;
  it.h = static_cast<int>(pair - static_cast<long long>(b) * A.H);
  it.start = sb.start;
  it.len = sb.len;
  it.nck = (sb.len + C - 1) / C;
  it.c = 0;
  it.tok0 = sb.start;
  it.Lc = min(C, sb.len);
  return true;
}
__device__ __noinline__ bool pairs_from(const Args &A, long long pair, ChunkIt &it) {
  for (; pair < A.BH; pair += gridDim.x)
    if (pair_load(A, pair, it)) return true;
  return false;
}
__device__ __forceinline__ bool it_first(const Args &A, ChunkIt &it) { return pairs_from(A, blockIdx.x, it); }
__device__ __forceinline__ bool it_next(const Args &A, ChunkIt &it) {
  if (it.c + 1 < it.nck) {
    ++it.c;
    it.tok0 = it.start + static_cast<long long>(it.c) * C;
    it.Lc = min(C, it.len - it.c * C);
    return true;
  }
  return pairs_from(A, it.pair + gridDim.x, it);
}

// ---- layouts ---------------------------------------------------------------------------------------
// byte offset of element (row, k) in a K-major 32-bit operand with `rows` rows
__device__ __forceinline__ uint32_t kmaj_tf32(uint32_t rows, uint32_t row, uint32_t k) {
  return (k >> 5) * (rows * 128u) + tc::sw128(row, (k & 31u) >> 2) + (k & 3u) * 4u;
}
// Row of value channel i in V^T, S0 and the columns of D4: within each 32-channel half, channel
// 4l + e sits in row 8e + l, so the preparation's 16-byte V^T stores of one quarter-warp (channels 4l
// + e, l = 0..7) hit 8 distinct bank groups of the 128-byte swizzle.
__host__ __device__ constexpr int vrow(int i) { return (i & 32) | ((i & 3) << 3) | ((i >> 2) & 7); }
__host__ __device__ constexpr int vinv(int p) { return (p & 32) | ((p & 7) << 2) | ((p >> 3) & 3); }

// One column k = j of 32 consecutive rows row0 .. row0+31 (row0 a multiple of 8) of a K-major 32-bit
// operand whose K-atoms hold `rows` rows: row row0 + x sits at p[x & 7] + x * 128.
struct ColPtrs {
  uint8_t *p[8];
};
__device__ __forceinline__ ColPtrs col_ptrs(uint8_t *region, uint32_t rows, uint32_t row0, uint32_t j) {
  ColPtrs c;
  uint8_t *base = region + (j >> 5) * (rows * 128u) + row0 * 128u + (j & 3u) * 4u;
  const uint32_t chunk = (j & 31u) >> 2;
#pragma unroll
  for (uint32_t r = 0; r < 8; ++r) c.p[r] = base + ((chunk ^ r) << 4);
  return c;
}

// four consecutive bf16 channels (j0 % 4 == 0) of token row t of a 128-byte-swizzled tile
__device__ __forceinline__ void raw4(const uint8_t *tile, int t, int j0, float (&o)[4]) {
  const uint32_t byte = static_cast<uint32_t>(j0) * 2u;
  const uint2 u = *reinterpret_cast<const uint2 *>(tile + tc::sw128(t, byte >> 4) + (byte & 15u));
  o[0] = __uint_as_float(u.x << 16);
  o[1] = __uint_as_float(u.x & 0xffff0000u);
  o[2] = __uint_as_float(u.y << 16);
  o[3] = __uint_as_float(u.y & 0xffff0000u);
}
// two floats -> one bf16x2 word (round to nearest even; lo in the low half)
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;\n" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}
// float32 -> tf32 operand bits, rounded to nearest with ties away from zero: half an ulp of the 10-bit
// mantissa is added to the magnitude bits; the tensor core ignores the 13 low bits of a tf32 operand,
// so they need not be cleared.
__device__ __forceinline__ uint32_t tf32r(float x) { return __float_as_uint(x) + 0x1000u; }
__device__ __forceinline__ void st_tf32x4(uint8_t *p, float a, float b, float c, float d) {
  *reinterpret_cast<uint4 *>(p) = make_uint4(tf32r(a), tf32r(b), tf32r(c), tf32r(d));
}
// 32 consecutive float32 values of one 128-byte-swizzled row
__device__ __forceinline__ void load_row(const uint8_t *blk, uint32_t row, float (&v)[32]) {
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    const float4 u = *reinterpret_cast<const float4 *>(blk + tc::sw128(row, c));
    v[4 * c] = u.x;
    v[4 * c + 1] = u.y;
    v[4 * c + 2] = u.z;
    v[4 * c + 3] = u.w;
  }
}
// 32 values -> 16 TMEM columns of bf16 pairs
__device__ __forceinline__ void tmem_st_bf16x32(uint32_t taddr, const float (&v)[32]) {
  float p[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) p[i] = __uint_as_float(pack_bf16x2(v[2 * i], v[2 * i + 1]));
  tc::tmem_st16(taddr, p);
}
// four bf16 pairs from 8 floats (round to nearest even)
__device__ __forceinline__ uint4 pack8(const float (&v)[8]) {
  return make_uint4(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]), pack_bf16x2(v[4], v[5]), pack_bf16x2(v[6], v[7]));
}
// 8 bf16 of a 16-byte chunk -> floats
__device__ __forceinline__ void unpack8(const uint4 &u, float (&v)[8]) {
  v[0] = __uint_as_float(u.x << 16);
  v[1] = __uint_as_float(u.x & 0xffff0000u);
  v[2] = __uint_as_float(u.y << 16);
  v[3] = __uint_as_float(u.y & 0xffff0000u);
  v[4] = __uint_as_float(u.z << 16);
  v[5] = __uint_as_float(u.z & 0xffff0000u);
  v[6] = __uint_as_float(u.w << 16);
  v[7] = __uint_as_float(u.w & 0xffff0000u);
}
// 16 floats -> 8 bf16 pairs as the register image of 8 TMEM columns
__device__ __forceinline__ void pack16(const float (&v)[16], float (&p)[8]) {
#pragma unroll
  for (int i = 0; i < 8; ++i) p[i] = __uint_as_float(pack_bf16x2(v[2 * i], v[2 * i + 1]));
}
// the 16-byte bf16 chunk of v[8h .. 8h + 7]
__device__ __forceinline__ uint4 pack_half(const float (&v)[16], int h) {
  return make_uint4(pack_bf16x2(v[8 * h], v[8 * h + 1]), pack_bf16x2(v[8 * h + 2], v[8 * h + 3]),
                    pack_bf16x2(v[8 * h + 4], v[8 * h + 5]), pack_bf16x2(v[8 * h + 6], v[8 * h + 7]));
}
__device__ __forceinline__ void keep16(float (&v)[16], int col0, int lim) {
#pragma unroll
  for (int x = 0; x < 16; ++x) v[x] = col0 + x <= lim ? v[x] : 0.f;
}
// keep v[x] where col0 + x <= lim (causal mask); zero the rest
__device__ __forceinline__ void keep8(float (&v)[8], int col0, int lim) {
#pragma unroll
  for (int x = 0; x < 8; ++x) v[x] = col0 + x <= lim ? v[x] : 0.f;
}
// keep v[x] where x <= lim (inclusive causal mask on a 32-column half); zero the rest
__device__ __forceinline__ void keep_upto(float (&v)[32], int lim) {
#pragma unroll
  for (int x = 0; x < 32; ++x) v[x] = x <= lim ? v[x] : 0.f;
}
__device__ __forceinline__ void zero32(float (&v)[32]) {
#pragma unroll
  for (int x = 0; x < 32; ++x) v[x] = 0.f;
}

// ---- bounded waits -----------------------------------------------------------------------------------
struct Ctl {
  volatile int *abort;
  int *err;
};
__device__ __noinline__ void fail(const Ctl &ctl) {
  *ctl.abort = 1;
  report_device_error(ctl.err, kDevErrTimeout);
}
// Waits for the phase with `parity`, sleeping in the barrier between polls; false once the CTA aborts
// or after kWaitLimitNs.
__device__ __noinline__ bool wait_slow(uint64_t *bar, uint32_t parity, volatile int *abort) {
  const uint64_t t0 = tc::globaltimer_ns();
  for (;;) {
    if (tc::mbar_try_wait_hint(bar, parity, kSuspendNs)) return true;
    if (*abort || tc::globaltimer_ns() - t0 > kWaitLimitNs) return false;
  }
}
__device__ __forceinline__ bool wait_or_abort(uint64_t *bar, uint32_t parity, volatile int *abort) {
  return tc::mbar_test_wait(bar, parity) || wait_slow(bar, parity, abort);
}
// A group of warps waits for barriers: its leader polls (bounded), publishes the outcome in one of
// two slots (alternating per call; a slot is rewritten only after every member passed the next
// call's barrier), then the group synchronises, so all members take the same branch.
struct Group {
  int id, n;
  bool leader;
  volatile int *slot;
  uint32_t calls;
};
__device__ __forceinline__ bool gwait(Group &g, const Ctl &ctl, uint64_t *b0, uint32_t p0, uint64_t *b1 = nullptr,
                                      uint32_t p1 = 0, uint64_t *b2 = nullptr, uint32_t p2 = 0,
                                      uint64_t *b3 = nullptr, uint32_t p3 = 0) {
  const uint32_t s = g.calls++ & 1u;
  if (g.leader) {
    bool ok = wait_or_abort(b0, p0, ctl.abort);
    if (ok && b1) ok = wait_or_abort(b1, p1, ctl.abort);
    if (ok && b2) ok = wait_or_abort(b2, p2, ctl.abort);
    if (ok && b3) ok = wait_or_abort(b3, p3, ctl.abort);
    if (!ok) fail(ctl);
    g.slot[s] = ok ? 1 : 0;
  }
  nbar_sync(g.id, g.n);
  __syncwarp();
  return g.slot[s] != 0;
}

// ---- the inverse ----------------------------------------------------------------------------------
__device__ __forceinline__ float *ts_block(float *Ts, int r, int c) {
  return Ts + ((r == c) ? r : (r == 1 ? 4 : 5)) * (16 * LDTB);
}
// Stores a 16x16 mma-layout accumulator as bf16 into the K-major bf16 Tinv (rows row0.., K col0..).
__device__ __forceinline__ void block16_store_bf16(uint8_t *op, int row0, int col0, const float (&acc)[2][4],
                                                   int lane) {
  const int g = lane >> 2, t = lane & 3;
#pragma unroll
  for (int nt = 0; nt < 2; ++nt) {
    const int col = col0 + 8 * nt + 2 * t;
    *reinterpret_cast<uint32_t *>(op + tc::sw128(row0 + g, col >> 3) + (col & 7) * 2) =
        pack_bf16x2(acc[nt][0], acc[nt][1]);
    *reinterpret_cast<uint32_t *>(op + tc::sw128(row0 + g + 8, col >> 3) + (col & 7) * 2) =
        pack_bf16x2(acc[nt][2], acc[nt][3]);
  }
}
// The four 16x16 diagonal blocks D_s = (I - L_ss)^-1 by forward substitution, into Ts (float32), run
// by two warps: lanes 0-15 of warp w solve block 2w, lanes 16-31 block 2w + 1, one column c per lane:
// x_r = [r == c] + sum_{q<r} L_rq x_q, row by row, each row of L read with 16-byte loads as it is
// needed (the sum split over two accumulators to halve the dependent chain).
__device__ __forceinline__ void invert_diagonal(const float *Ls, float *Ts, int w, int lane) {
  const int blk = 2 * w + (lane >> 4), base = 16 * blk, cix = lane & 15;
  float x[16];
  x[0] = cix == 0 ? 1.f : 0.f;
#pragma unroll
  for (int r = 1; r < 16; ++r) {
    const float *row = Ls + (base + r) * LDL + base;
    float acc0 = (r == cix) ? 1.f : 0.f, acc1 = 0.f;
#pragma unroll
    for (int q4 = 0; q4 < (r + 3) / 4; ++q4) {
      const float4 u = *reinterpret_cast<const float4 *>(row + 4 * q4);
      const float uu[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int q = 4 * q4 + e;
        if (q < r) {
          if (q & 1)
            acc1 = fmaf(uu[e], x[q], acc1);
          else
            acc0 = fmaf(uu[e], x[q], acc0);
        }
      }
    }
    x[r] = acc0 + acc1;
  }
  float *D = ts_block(Ts, blk, blk);
#pragma unroll
  for (int r = 0; r < 16; ++r) D[r * LDTB + cix] = x[r];
}
// The blocks below the diagonal, from the diagonal ones (the block identity for a lower
// block-triangular M = I - L: (M^-1)_BA = (M^-1)_BB L_BA (M^-1)_AA), first (1,0) and (3,2), then the
// lower-left 32x32 block, each 16x16 product on warp-level tf32 mma.  All four warps of the stage;
// B3 (which B2 of the previous chunk overlays) is written whole: the diagonal blocks from Ts, the zero
// blocks above them and the products; ends with Tinv complete in B3.
__device__ __forceinline__ void invert_offdiag(const float *Ls, float *Ts, float *Zs, uint8_t *sB3, int warp,
                                               int lane) {
  {
    const int e = warp * 32 + lane;
    // the six 16x16 blocks above the block diagonal: 16 rows x 2 chunks each
    for (int k = e; k < 6 * 32; k += 128) {
      const int blk = k >> 5, rr = (k >> 1) & 15, half = k & 1;
      const int sr = blk < 3 ? 0 : (blk < 5 ? 1 : 2);
      const int sc = blk < 3 ? blk + 1 : (blk < 5 ? blk - 1 : 3);
      *reinterpret_cast<uint4 *>(sB3 + tc::sw128(16 * sr + rr, 2 * sc + half)) = make_uint4(0u, 0u, 0u, 0u);
    }
    // the diagonal blocks as bf16: row 16 s + (e >> 3), eight columns 16 s + 8 (e & 1) .. per thread
    for (int k = e; k < 4 * 32; k += 128) {
      const int sblk = k >> 5, rr = (k >> 1) & 15, half = k & 1;
      const float *D = ts_block(Ts, sblk, sblk) + rr * LDTB + 8 * half;
      uint4 w4;
      w4.x = pack_bf16x2(D[0], D[1]);
      w4.y = pack_bf16x2(D[2], D[3]);
      w4.z = pack_bf16x2(D[4], D[5]);
      w4.w = pack_bf16x2(D[6], D[7]);
      *reinterpret_cast<uint4 *>(sB3 + tc::sw128(16 * sblk + rr, 2 * sblk + half)) = w4;
    }
  }
  if (warp < 2) {
    // T_{s+1,s} = D_{s+1} L_{s+1,s} D_s for s = 0, 2
    const int s = 2 * warp;
    float *Z = Zs + warp * (16 * LDZ);
    float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
    tc::block16_mma(acc, Ls + (16 * (s + 1)) * LDL + 16 * s, LDL, ts_block(Ts, s, s), LDTB, lane);
    tc::block16_store(Z, LDZ, acc, lane);
    __syncwarp();
    float t2[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
    tc::block16_mma(t2, ts_block(Ts, s + 1, s + 1), LDTB, Z, LDZ, lane);
    tc::block16_store(ts_block(Ts, s + 1, s), LDTB, t2, lane);
    block16_store_bf16(sB3, 16 * (s + 1), 16 * s, t2, lane);
  }
  nbar_sync(NB_S2, 128);
  // lower-left 32x32 block, one warp per 16x16 tile (s, m), s in {2, 3}, m in {0, 1}
  const int s = 2 + (warp >> 1), m = warp & 1;
  {
    // X_sm = sum_{q=m}^{1} L_sq T_qm
    float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
    for (int q = 0; q < 2; ++q)
      if (q >= m) tc::block16_mma(acc, Ls + (16 * s) * LDL + 16 * q, LDL, ts_block(Ts, q, m), LDTB, lane);
    tc::block16_store(Zs + (2 + warp) * (16 * LDZ), LDZ, acc, lane);
  }
  nbar_sync(NB_S2, 128);
  {
    // T_sm = sum_{p=2}^{s} T_sp X_pm
    float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
    for (int p = 2; p < 4; ++p)
      if (p <= s) tc::block16_mma(acc, ts_block(Ts, s, p), LDTB, Zs + (2 + 2 * (p - 2) + m) * (16 * LDZ), LDZ, lane);
    block16_store_bf16(sB3, 16 * s, 16 * m, acc, lane);
  }
}

// ---- the token-by-token path of a flagged chunk ------------------------------------------------------
// Run by the 64 state threads (named barrier NB_ST).  On entry S (float [64][64], row i = value
// channel, column j) holds the chunk's start state; on exit its end state.  Thread i owns row i:
// sa = S a, S = S diag(w) + sa b^T + v k^T, y = S r token by token in float32, with the token's
// vectors staged in `vec` (two buffers of w, k, a, b, r, v).
template <bool kFused, bool kLN>
__device__ __noinline__ void chunk_by_tokens(const Args &A, long long tok0, int h, int Lc, float *S, float *vec,
                                             int i) {
  float s[64];
#pragma unroll
  for (int j = 0; j < 64; ++j) s[j] = S[i * 64 + j];
  const float kkw = kFused && A.k_k ? A.k_k[h * kN + i] : 1.f;
  const float lw = kLN ? (A.ln_w ? A.ln_w[h * kN + i] : 1.f) : 1.f;
  const float lb = kLN ? (A.ln_b ? A.ln_b[h * kN + i] : 0.f) : 0.f;
  for (int t = 0; t < Lc; ++t) {
    float *vb = vec + (t & 1) * (6 * 64);
    const long long e = ((tok0 + t) * A.H + h) * kN + i;
    float wv = bf16_bits_to_float(A.op[OP_W][e]);
    const float kv = bf16_bits_to_float(A.op[OP_K][e]);
    float av = bf16_bits_to_float(A.op[OP_A][e]);
    float bv = kFused ? 0.f : bf16_bits_to_float(A.op[OP_B][e]);
    if (kFused) {
      // w = decay(x_w); kk = k k_k / |k k_k|; a = -kk; b = kk sigmoid(x_a) (the a slot holds x_a)
      wv = x070_decay(wv);
      const float kx = kv * kkw;
      vb[5 * 64 + i] = kx * kx;  // the v slot first carries the squares of the norm
      nbar_sync(NB_ST, 64);
      float ss = 0.f;
#pragma unroll 8
      for (int q = 0; q < 64; ++q) ss += vb[5 * 64 + q];
      const float kk = kx * x070_inv_norm(ss);
      bv = kk * x070_sigmoid(av);
      av = -kk;
      nbar_sync(NB_ST, 64);
    }
    vb[0 * 64 + i] = wv;
    vb[1 * 64 + i] = kv;
    vb[2 * 64 + i] = av;
    vb[3 * 64 + i] = bv;
    vb[4 * 64 + i] = bf16_bits_to_float(A.op[OP_R][e]);
    const float vi = bf16_bits_to_float(A.op[OP_V][e]);
    nbar_sync(NB_ST, 64);
    float sa = 0.f;
#pragma unroll
    for (int j = 0; j < 64; ++j) sa = fmaf(s[j], vb[2 * 64 + j], sa);
    float y = 0.f;
#pragma unroll
    for (int j = 0; j < 64; ++j) {
      s[j] = fmaf(s[j], vb[0 * 64 + j], fmaf(sa, vb[3 * 64 + j], vi * vb[1 * 64 + j]));
      y = fmaf(s[j], vb[4 * 64 + j], y);
    }
    if (kLN) {
      vb[5 * 64 + i] = y;
      nbar_sync(NB_ST, 64);
      float mu = 0.f;
#pragma unroll 8
      for (int q = 0; q < 64; ++q) mu += vb[5 * 64 + q];
      mu *= (1.f / 64.f);
      float var = 0.f;
#pragma unroll 8
      for (int q = 0; q < 64; ++q) var = fmaf(vb[5 * 64 + q] - mu, vb[5 * 64 + q] - mu, var);
      var *= (1.f / 64.f);
      y = fmaf((y - mu) * rsqrtf(var + kLnEps), lw, lb);
    }
    A.y[e] = float_to_bf16_bits(y);
  }
  nbar_sync(NB_ST, 64);
#pragma unroll
  for (int j = 0; j < 64; ++j) S[i * 64 + j] = s[j];
}

// The rare steps of the state chain, on the state held in S (float32 [i][j]; thread j of the 64
// state threads owns column j): a flagged chunk `fl` run token by token; the end state of pair `done` to
// s_out; the start state of pair `next` (s_in or zero) into S; S as checkpoint `ck` of states (each
// skipped when null / negative).
template <bool kFused, bool kLN>
__device__ __noinline__ void state_edge(const Args &A, long long done, long long next, long long ck,
                                        const ChunkIt *fl, float *S, float *vec, int j) {
  if (fl != nullptr) {
    nbar_sync(NB_ST, 64);
    chunk_by_tokens<kFused, kLN>(A, fl->tok0, fl->h, fl->Lc, S, vec, j);
    nbar_sync(NB_ST, 64);
  }
  if (done >= 0) {
    float *o = A.s_out + done * (kN * kN) + j;
#pragma unroll 4
    for (int i = 0; i < kN; ++i) o[i * kN] = S[i * 64 + j];
  }
  if (next >= 0) {
    const float *in = A.s_in ? A.s_in + next * (kN * kN) + j : nullptr;
#pragma unroll 4
    for (int i = 0; i < kN; ++i) S[i * 64 + j] = in ? in[i * kN] : 0.f;
  }
  if (ck >= 0) {
    float *o = A.states + ck * (kN * kN) + j;
#pragma unroll 4
    for (int i = 0; i < kN; ++i) o[i * kN] = S[i * 64 + j];
  }
}

// ---- the kernel ------------------------------------------------------------------------------------
// kFused: model-native inputs -- the w and a tiles hold x_w and x_a, no b tile is loaded; w =
// decay(x_w), a = -kk and b = kk * sigmoid(x_a) with kk = k * k_k / |k * k_k| are formed by the
// preparation.  kLN: the x070 ln_x epilogue (GroupNorm over each token-head's 64 channels, eps 64e-5)
// is applied to y before it is stored.
template <bool kFused, bool kLN>
__global__ void __launch_bounds__(kThreads, 1) wkv7_pipe_kernel(const __grid_constant__ Maps maps, const Args A) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *misc = smem + OFF_MISC;
  uint64_t *bars = reinterpret_cast<uint64_t *>(misc);
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(misc + MISC_WORDS);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(misc + MISC_WORDS + 4);
  volatile int *slots = reinterpret_cast<volatile int *>(misc + MISC_WORDS + 16);  // [5 groups][2]
  float *gcs = reinterpret_cast<float *>(misc + MISC_GC);
  volatile uint32_t *gflag = reinterpret_cast<volatile uint32_t *>(misc + MISC_GFLAG);
  float *tot = reinterpret_cast<float *>(misc + MISC_TOT);
  uint8_t *sVT = smem + OFF_VT;
  uint8_t *sB4S = smem + OFF_B4S;
  uint8_t *sA3 = smem + OFF_A3;
  uint8_t *sB2 = smem + OFF_B2;
  uint8_t *sB3 = smem + OFF_B3;
  float *Ls = reinterpret_cast<float *>(smem + OFF_LS);
  float *Ts = reinterpret_cast<float *>(smem + OFF_TS);
  float *Zs = reinterpret_cast<float *>(smem + OFF_ZS);
  auto bar = [&](int i) { return bars + i; };

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const Ctl ctl{abort_flag, A.err};
  constexpr int kTiles = kFused ? 5 : 6;
  // operand (map) of the i-th tile of a chunk, in the order the preparation reads them
  auto tile_op = [](int i) { return kFused ? (i < 3 ? i : i + 1) : i; };

  if (tid == 0) {
    for (int i = 0; i < kNumBars; ++i)
      tc::mbar_init(bar(i), (i == B_D4_EMPTY || i == B_D4_EMPTY + 1) ? 2 : (i == B_A1_EMPTY ? 4 : 1));
    tc::fence_mbar_init();
    *abort_flag = 0;
  }
  if (warp == W_MMA) {
    tc::tmem_alloc(tmem_slot, kTmemCols);
    tc::tmem_relinquish();
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == W_MMA) {
    // ===== MMA issue ==================================================================================
    // MMAs of one thread run in issue order, so an MMA may read what an earlier one wrote with no wait
    // in between, and overwrite what an earlier one read.
    if (lane == 0) {
      long long total = 0;
      {
        ChunkIt it;
        for (bool ok = it_first(A, it); ok; ok = it_next(A, it)) ++total;
      }
      const uint32_t sb = smem_u32(smem);
      const uint64_t dB1[2] = {tc::smem_desc(sb + OFF_B1, 16, 1024), tc::smem_desc(sb + OFF_B1 + 32768, 16, 1024)};
      const uint64_t dA3 = tc::smem_desc(sb + OFF_A3, 64 * 128, 1024), dB3 = tc::smem_desc(sb + OFF_B3, 16, 1024);
      const uint64_t dB2 = tc::smem_desc(sb + OFF_B2, 16, 1024);
      const uint64_t dVT = tc::smem_desc(sb + OFF_VT, 16, 1024), dS = tc::smem_desc(sb + OFF_B4S, 16, 1024);
      constexpr uint32_t id1 = tc::instr_desc(tc::kFmtTF32, 128, 128, false, false);
      constexpr uint32_t id3 = tc::instr_desc(tc::kFmtBF16, 128, 64, true, false);
      constexpr uint32_t id2 = tc::instr_desc(tc::kFmtBF16, 128, 128, false, false);
      constexpr uint32_t id4 = tc::instr_desc(tc::kFmtTF32, 128, 64, false, false);
      // MMA1 (tf32, A from TMEM): D1 = [R~; A~] [B^; K^]^T into the X slot of chunk c
      auto mma1 = [&](long long c) {
        const uint32_t sl = static_cast<uint32_t>(c & 1);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
          const uint32_t off = (ks >> 2) * (128 * 128) + (ks & 3) * 32;
          tc::mma_ts_tf32(tmem + TM_X + 128 * sl, tmem + TM_A1 + 8 * ks, dB1[sl] + (off >> 4), id1, ks > 0);
        }
        tc::mma_commit(bar(B_M1));
      };
      // The next chunk of each MMA kind; each is issued as soon as its inputs are there, the later
      // stages first.  MMA1 of chunk c reuses the X slot of chunk c - 2 (its MMA4b must have been
      // issued), MMA3 of chunk c the D4 slot of chunk c - 2 (read out) and B2 of chunk c - 1 (MMA2 of
      // chunk c - 1 issued before it).
      long long i1 = 0, i3 = 0, i2 = 0, i4 = 0;
      bool ok = true;
      uint64_t t_idle = 0;
      while (i4 < total) {
        if (i4 < i2 && tc::mbar_test_wait(bar(B_S_FULL), static_cast<uint32_t>(i4 & 1))) {
          // MMA4b (tf32, A from TMEM): D4 += [Q; E] S0^T
          tc::tc_fence_after();
          const uint32_t sl = static_cast<uint32_t>(i4 & 1);
#pragma unroll
          for (int ks = 0; ks < 8; ++ks) {
            const uint32_t off = (ks >> 2) * (64 * 128) + (ks & 3) * 32;
            tc::mma_ts_tf32(tmem + TM_D4 + 64 * sl, tmem + TM_X + 128 * sl + 8 * ks, dS + (off >> 4), id4, 1);
          }
          tc::mma_commit(bar(B_M4 + sl));
          ++i4;
          t_idle = 0;
        } else if (i2 < i3 && tc::mbar_test_wait(bar(B_B2), static_cast<uint32_t>(i2 & 1)) &&
                   tc::mbar_test_wait(bar(B_VT_FULL), static_cast<uint32_t>(i2 & 1))) {
          // MMA2 (bf16, A from TMEM): D2 += [Mrb; B-^T] [W~ U~]; MMA4a (tf32): D4 = [P; F] V
          tc::tc_fence_after();
          const uint32_t sl = static_cast<uint32_t>(i2 & 1);
#pragma unroll
          for (int ks = 0; ks < 4; ++ks)
            tc::mma_ts_bf16(tmem + TM_X + 128 * sl, tmem + TM_A2 + 32 * sl + 8 * ks, dB2 + ((ks * 32) >> 4), id2, 1);
          tc::mma_commit(bar(B_M2));
#pragma unroll
          for (int ks = 0; ks < 8; ++ks) {
            const uint32_t off = (ks >> 2) * (64 * 128) + (ks & 3) * 32;
            tc::mma_ts_tf32(tmem + TM_D4 + 64 * sl, tmem + TM_X + 128 * sl + 64 + 8 * ks, dVT + (off >> 4), id4,
                            ks > 0);
          }
          tc::mma_commit(bar(B_M4A));
          ++i2;
          t_idle = 0;
        } else if (i3 < i1 && i3 <= i2 && tc::mbar_test_wait(bar(B_B3), static_cast<uint32_t>(i3 & 1)) &&
                   (i3 < 2 || tc::mbar_test_wait(bar(B_D4_EMPTY + (i3 & 1)), static_cast<uint32_t>(((i3 >> 1) + 1) & 1)))) {
          // MMA3 (bf16): D3 = [A~^T; Lak^T] Tinv^T, into the D4 slot of the chunk
          tc::tc_fence_after();
          const uint32_t sl = static_cast<uint32_t>(i3 & 1);
#pragma unroll
          for (int ks = 0; ks < 4; ++ks)
            tc::mma_ss(0, tmem + TM_D4 + 64 * sl, dA3 + ((ks * 2048) >> 4), dB3 + ((ks * 32) >> 4), id3, ks > 0);
          tc::mma_commit(bar(B_M3));
          ++i3;
          t_idle = 0;
        } else if (i1 < total && i1 <= i4 + 1 && tc::mbar_test_wait(bar(B_AB_FULL), static_cast<uint32_t>(i1 & 1))) {
          tc::tc_fence_after();
          mma1(i1);
          ++i1;
          t_idle = 0;
        } else {
          // nothing ready: sleep on the barrier the pipeline most likely waits for (up to 0.5 us; it wakes
          // when that barrier completes), bounded in time
          uint64_t *wb;
          uint32_t wp;
          if (i4 < i2) {
            wb = bar(B_S_FULL);
            wp = static_cast<uint32_t>(i4 & 1);
          } else if (i2 < i3) {
            wb = bar(B_B2);
            wp = static_cast<uint32_t>(i2 & 1);
          } else if (i3 < i1) {
            wb = bar(B_B3);
            wp = static_cast<uint32_t>(i3 & 1);
          } else {
            wb = bar(B_AB_FULL);
            wp = static_cast<uint32_t>(i1 & 1);
          }
          (void)tc::mbar_try_wait_hint(wb, wp, 500);
          const uint64_t now = tc::globaltimer_ns();
          if (t_idle == 0) {
            t_idle = now;
          } else if (*abort_flag || now - t_idle > kWaitLimitNs) {
            ok = false;
            break;
          }
        }
      }
      if (!ok) fail(ctl);
      // every MMA issued here completes before the CTA exits (a commit tracks all earlier MMAs of the
      // thread; bounded)
      tc::mma_commit(bar(B_DRAIN));
      (void)tc::mbar_wait_bounded(bar(B_DRAIN), 0, kMaxPolls);
    }
  } else if (warp == W_TMA) {
    // ===== TMA loads of the operand tiles =============================================================
    if (lane == 0) {
      for (int i = 0; i < 6; ++i) tc::prefetch_tensormap(&maps.m[i]);
      uint32_t tcount = 0;
      ChunkIt it;
      bool ok = true;
      for (bool more = it_first(A, it); more && ok; more = it_next(A, it)) {
        for (int i = 0; i < kTiles; ++i) {
          const uint32_t s = tcount % NS, k = tcount / NS;
          if (!wait_or_abort(bar(B_RAW_EMPTY + s), (k & 1) ^ 1, abort_flag)) {
            fail(ctl);
            ok = false;
            break;
          }
          tc::mbar_arrive_expect_tx(bar(B_RAW_FULL + s), kTile);
          tc::tma_load_3d(smem + OFF_RAW + s * kTile, &maps.m[tile_op(i)], bar(B_RAW_FULL + s), 0, it.h,
                          static_cast<int>(it.tok0));
          ++tcount;
        }
      }
      // the last loads land before the CTA exits (bounded)
      for (uint32_t q = tcount > NS ? tcount - NS : 0; q < tcount; ++q)
        (void)tc::mbar_wait_bounded(bar(B_RAW_FULL + q % NS), (q / NS) & 1, kMaxPolls);
    }
  } else if (warp >= W_PREP && warp < W_PREP + 4) {
    // ===== operand preparation ========================================================================
    // Phase 1 (4 channels x 8 tokens per thread): the decay products, staged as float32 in the chunk's
    // B1 slot: Gamma_t in rows 0..63, Gamma_{t-1} in rows 64..127; Gamma_C and the domain flag.  Phase 2
    // (one token row per thread; warp q of the four owns TMEM lanes 32q..32q+31), each thread over its
    // own staged row only: warps 0-1 write R~ row t into A1 (TMEM lanes 0..63) and B^ row t over
    // Gamma_t; warps 2-3 write A~ row t (lanes 64..127) and K^ row t over Gamma_{t-1} (Gamma_t =
    // Gamma_{t-1} w_t).  Phase 3 (phase 1's layout): V^T.
    const int ptid = tid - 32 * W_PREP;
    const int pq = warp - W_PREP;              // TMEM lane quadrant of this warp
    const int cq = ptid & 15, to = ptid >> 4;  // phase 1 / 3: channel quad, token octet
    const int j0 = 4 * cq, tb = 8 * to;
    const int tr = 32 * (pq & 1) + lane;       // phase 2: token row
    const uint32_t lane_base = static_cast<uint32_t>(32 * pq) << 16;
    Group g{NB_PREP, 128, ptid == 0, slots + 0, 0};
    uint32_t tcount = 0;
    long long n = 0;
    ChunkIt it;
    for (bool more = it_first(A, it); more; more = it_next(A, it), ++n, tcount += kTiles) {
      const int Lc = it.Lc;
      const uint32_t sl = static_cast<uint32_t>(n & 1);
      uint8_t *b1 = smem + OFF_B1 + 32768 * sl;
      auto slot = [&](int i) { return (tcount + i) % NS; };
      auto ph = [&](int i) { return ((tcount + i) / NS) & 1u; };
      auto tile = [&](int i) { return smem + OFF_RAW + slot(i) * kTile; };
      // ---- phase 1: decay products (w tile; the B1 slot once chunk n - 2 is done with it)
      if (!gwait(g, ctl, bar(B_RAW_FULL + slot(0)), ph(0), bar(B_B1_EMPTY + sl), static_cast<uint32_t>(((n >> 1) & 1) ^ 1)))
        break;
      {
        float G[8][4];
#pragma unroll
        for (int tt = 0; tt < 8; ++tt) {
          if (tb + tt < Lc) {
            raw4(tile(0), tb + tt, j0, G[tt]);
            if (kFused) {
#pragma unroll
              for (int e = 0; e < 4; ++e) G[tt][e] = x070_decay(G[tt][e]);  // the tile holds x_w
            }
          } else {
#pragma unroll
            for (int e = 0; e < 4; ++e) G[tt][e] = 1.f;
          }
        }
#pragma unroll
        for (int tt = 1; tt < 8; ++tt)
#pragma unroll
          for (int e = 0; e < 4; ++e) G[tt][e] *= G[tt - 1][e];
        *reinterpret_cast<float4 *>(tot + to * 64 + j0) = make_float4(G[7][0], G[7][1], G[7][2], G[7][3]);
        nbar_sync(NB_PREP, 128);
        float p0[4] = {1.f, 1.f, 1.f, 1.f}, gc[4] = {1.f, 1.f, 1.f, 1.f};
#pragma unroll
        for (int o = 0; o < 8; ++o) {
          const float4 u = *reinterpret_cast<const float4 *>(tot + o * 64 + j0);
          const float uu[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            if (o < to) p0[e] *= uu[e];
            gc[e] *= uu[e];
          }
        }
        uint8_t *g1 = b1 + (j0 >> 5) * (128 * 128);
        const uint32_t chk = (j0 & 31) >> 2;
#pragma unroll
        for (int tt = 0; tt < 8; ++tt) {
          *reinterpret_cast<float4 *>(g1 + tc::sw128(tb + tt, chk)) =
              make_float4(p0[0] * G[tt][0], p0[1] * G[tt][1], p0[2] * G[tt][2], p0[3] * G[tt][3]);
          if (tt == 0) {
            *reinterpret_cast<float4 *>(g1 + tc::sw128(64 + tb, chk)) = make_float4(p0[0], p0[1], p0[2], p0[3]);
          } else {
            *reinterpret_cast<float4 *>(g1 + tc::sw128(64 + tb + tt, chk)) = make_float4(
                p0[0] * G[tt - 1][0], p0[1] * G[tt - 1][1], p0[2] * G[tt - 1][2], p0[3] * G[tt - 1][3]);
          }
        }
        bool bad = false;
#pragma unroll
        for (int e = 0; e < 4; ++e) bad |= !(gc[e] >= kGammaMin);
        const unsigned anyb = __any_sync(0xffffffffu, bad);
        if (lane == 0) reinterpret_cast<volatile uint8_t *>(gflag)[(n & 3) * 4 + pq] = anyb ? 1 : 0;
        if (to == 0) *reinterpret_cast<float4 *>(gcs + (n & 3) * 64 + j0) = make_float4(gc[0], gc[1], gc[2], gc[3]);
        __syncwarp();
      }
      // ---- phase 2: the other tiles; A1 once the mask stage of chunk n - 1 has read it
      if (!gwait(g, ctl, bar(B_RAW_FULL + slot(1)), ph(1), bar(B_RAW_FULL + slot(2)), ph(2),
                 bar(B_RAW_FULL + slot(3)), ph(3), bar(B_A1_EMPTY), static_cast<uint32_t>((n & 1) ^ 1)))
        break;
      if (!kFused && !gwait(g, ctl, bar(B_RAW_FULL + slot(4)), ph(4))) break;
      const int tk_k = kFused ? 3 : 4, tk_v = kFused ? 4 : 5;
      {
        const bool live = tr < Lc;
        const float *kkw = A.k_k ? A.k_k + it.h * kN : nullptr;
        float kscale = 1.f;  // model-native: 1 / |k k_k| of this token
        if (kFused) {
          float ss = 0.f;
#pragma unroll 1
          for (int c = 0; c < 8; ++c) {
            float kv[8];
            unpack8(*reinterpret_cast<const uint4 *>(tile(tk_k) + tc::sw128(tr, c)), kv);
#pragma unroll
            for (int x = 0; x < 8; ++x) {
              const float kx = kv[x] * (kkw ? kkw[8 * c + x] : 1.f);
              ss = fmaf(kx, kx, ss);
            }
          }
          kscale = x070_inv_norm(ss);
        }
        const uint32_t a1 = tmem + TM_A1 + lane_base;
        if (pq < 2) {
          // R~ = r Gamma_t (A1), B^ = b / Gamma_t (B1 row t, over Gamma_t); model-native b = kk sigmoid(x_a)
#pragma unroll 1
          for (int c = 0; c < 8; ++c) {
            uint8_t *gp = b1 + (c >> 2) * (128 * 128) + tr * 128;
            const uint32_t o0 = ((2 * (c & 3)) ^ (tr & 7)) << 4, o1 = ((2 * (c & 3) + 1) ^ (tr & 7)) << 4;
            const float4 ga = *reinterpret_cast<const float4 *>(gp + o0), gb = *reinterpret_cast<const float4 *>(gp + o1);
            const float gam[8] = {ga.x, ga.y, ga.z, ga.w, gb.x, gb.y, gb.z, gb.w};
            float rr[8], bb[8];
            unpack8(*reinterpret_cast<const uint4 *>(tile(1) + tc::sw128(tr, c)), rr);
            unpack8(*reinterpret_cast<const uint4 *>(tile(kFused ? 2 : 3) + tc::sw128(tr, c)), bb);
            if (kFused) {
              float kv[8];
              unpack8(*reinterpret_cast<const uint4 *>(tile(tk_k) + tc::sw128(tr, c)), kv);
#pragma unroll
              for (int x = 0; x < 8; ++x) bb[x] = kv[x] * (kkw ? kkw[8 * c + x] : 1.f) * kscale * x070_sigmoid(bb[x]);
            }
            float v[8];
            uint32_t bw[8];
#pragma unroll
            for (int x = 0; x < 8; ++x) {
              v[x] = live ? __uint_as_float(tf32r(rr[x] * gam[x])) : 0.f;
              bw[x] = live ? tf32r(bb[x] * tc::rcp_approx(gam[x])) : 0u;
            }
            *reinterpret_cast<uint4 *>(gp + o0) = make_uint4(bw[0], bw[1], bw[2], bw[3]);
            *reinterpret_cast<uint4 *>(gp + o1) = make_uint4(bw[4], bw[5], bw[6], bw[7]);
            tc::tmem_st8(a1 + 8 * c, v);
          }
        } else {
          // A~ = a Gamma_{t-1} (A1), K^ = k / Gamma_t (B1 row 64 + t, over Gamma_{t-1}); model-native
          // a = -kk
#pragma unroll 1
          for (int c = 0; c < 8; ++c) {
            uint8_t *gp = b1 + (c >> 2) * (128 * 128) + (64 + tr) * 128;
            const uint32_t o0 = ((2 * (c & 3)) ^ (tr & 7)) << 4, o1 = ((2 * (c & 3) + 1) ^ (tr & 7)) << 4;
            const float4 ga = *reinterpret_cast<const float4 *>(gp + o0), gb = *reinterpret_cast<const float4 *>(gp + o1);
            const float gpv[8] = {ga.x, ga.y, ga.z, ga.w, gb.x, gb.y, gb.z, gb.w};
            float wv[8], aa[8], kv[8];
            unpack8(*reinterpret_cast<const uint4 *>(tile(0) + tc::sw128(tr, c)), wv);
            unpack8(*reinterpret_cast<const uint4 *>(tile(tk_k) + tc::sw128(tr, c)), kv);
            if (kFused) {
#pragma unroll
              for (int x = 0; x < 8; ++x) {
                wv[x] = x070_decay(wv[x]);  // the tile holds x_w
                aa[x] = -(kv[x] * (kkw ? kkw[8 * c + x] : 1.f) * kscale);
              }
            } else {
              unpack8(*reinterpret_cast<const uint4 *>(tile(2) + tc::sw128(tr, c)), aa);
            }
            float v[8];
            uint32_t kw[8];
#pragma unroll
            for (int x = 0; x < 8; ++x) {
              v[x] = live ? __uint_as_float(tf32r(aa[x] * gpv[x])) : 0.f;
              kw[x] = live ? tf32r(kv[x] * tc::rcp_approx(gpv[x] * wv[x])) : 0u;
            }
            *reinterpret_cast<uint4 *>(gp + o0) = make_uint4(kw[0], kw[1], kw[2], kw[3]);
            *reinterpret_cast<uint4 *>(gp + o1) = make_uint4(kw[4], kw[5], kw[6], kw[7]);
            tc::tmem_st8(a1 + 8 * c, v);
          }
        }
      }
      tc::tmem_st_wait();
      tc::fence_proxy_async_smem();
      tc::tc_fence_before();
      nbar_sync(NB_PREP, 128);
      if (ptid == 0) {
        tc::mbar_arrive(bar(B_AB_FULL));
        tc::mbar_arrive(bar(B_GC + (n & 3)));
        for (int i = 0; i < tk_v; ++i) tc::mbar_arrive(bar(B_RAW_EMPTY + slot(i)));
      }
      __syncwarp();
      // ---- phase 3: V^T (row vrow(channel), K = token; bf16 values are exact in tf32), once MMA4a of the
      // previous chunk is done with it
      if (!gwait(g, ctl, bar(B_RAW_FULL + slot(tk_v)), ph(tk_v), bar(B_M4A), static_cast<uint32_t>((n & 1) ^ 1)))
        break;
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        float vv[4][4];
#pragma unroll
        for (int tt = 0; tt < 4; ++tt) {
          if (tb + 4 * hh + tt < Lc) {
            raw4(tile(tk_v), tb + 4 * hh + tt, j0, vv[tt]);
          } else {
#pragma unroll
            for (int e = 0; e < 4; ++e) vv[tt][e] = 0.f;
          }
        }
#pragma unroll
        for (int e = 0; e < 4; ++e)
          *reinterpret_cast<uint4 *>(sVT + kmaj_tf32(64, vrow(j0 + e), tb + 4 * hh)) =
              make_uint4(__float_as_uint(vv[0][e]), __float_as_uint(vv[1][e]), __float_as_uint(vv[2][e]),
                         __float_as_uint(vv[3][e]));
      }
      tc::fence_proxy_async_smem();
      nbar_sync(NB_PREP, 128);
      if (ptid == 0) {
        tc::mbar_arrive(bar(B_VT_FULL));
        tc::mbar_arrive(bar(B_RAW_EMPTY + slot(tk_v)));
      }
      __syncwarp();
    }
  } else if (warp >= W_S2 && warp < W_S2 + 4) {
    // ===== causal masks, D2 set-up, inverse, D3 -> B2 ==================================================
    const int q = warp - W_S2;  // TMEM lane quadrant (warp % 4 == q)
    const int dh = q & 1;       // the 32-column half that holds this quadrant's diagonal
    const uint32_t lane_base = static_cast<uint32_t>(32 * q) << 16;
    Group g{NB_S2, 128, q == 0 && lane == 0, slots + 2, 0};
    long long n = 0;
    ChunkIt it;
    for (bool more = it_first(A, it); more; more = it_next(A, it), ++n) {
      const uint32_t sl = static_cast<uint32_t>(n & 1);
      const uint32_t X = tmem + TM_X + 128 * sl + lane_base;
      const uint32_t A2 = tmem + TM_A2 + 32 * sl + lane_base;
      const uint32_t A1 = tmem + TM_A1 + lane_base;
      uint8_t *b1 = smem + OFF_B1 + 32768 * sl;
      if (!gwait(g, ctl, bar(B_M1), sl, bar(B_AB_FULL), sl)) break;
      tc::tc_fence_after();
      const int t = 32 * dh + lane;  // the token row of this thread's TMEM lane (and, lanes 64..127, key channel j)
      if (q >= 2) {
        // A~ row t (A1) -> the A~^T block of A3 (bf16; MMA3 of the previous chunk is done with A3)
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          float v[16];
          tc::tmem_ld16(A1 + 16 * c, v);
          *reinterpret_cast<uint4 *>(sA3 + tc::sw128(t, 2 * c)) = pack_half(v, 0);
          *reinterpret_cast<uint4 *>(sA3 + tc::sw128(t, 2 * c + 1)) = pack_half(v, 1);
        }
        tc::tc_fence_before();
        if (lane == 0) tc::mbar_arrive(bar(B_A1_EMPTY));
        __syncwarp();
        // rows of Lab (strictly lower, m < t) -> Ls
#pragma unroll 1
        for (int c = 0; c < 2 * (dh + 1); ++c) {
          float v[16];
          tc::tmem_ld16(X + 16 * c, v);
          keep16(v, 16 * c, t - 1);
          float *row = Ls + t * LDL + 16 * c;
#pragma unroll
          for (int x = 0; x < 16; x += 4) *reinterpret_cast<float4 *>(row + x) = make_float4(v[x], v[x + 1], v[x + 2], v[x + 3]);
        }
        nbar_arrive(NB_LS, 128);
        // rows of Lak (strictly lower) -> the Lak^T block of A3
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          float v[16];
          if (c < 2 * (dh + 1)) {
            tc::tmem_ld16(X + 64 + 16 * c, v);
            keep16(v, 16 * c, t - 1);
          } else {
#pragma unroll
            for (int x = 0; x < 16; ++x) v[x] = 0.f;
          }
          *reinterpret_cast<uint4 *>(sA3 + 64 * 128 + tc::sw128(t, 2 * c)) = pack_half(v, 0);
          *reinterpret_cast<uint4 *>(sA3 + 64 * 128 + tc::sw128(t, 2 * c + 1)) = pack_half(v, 1);
        }
        // the D2 set-up of lanes 64..127 (Lab and Lak have been read): E-part = 0, F-part = K-^T[j][m] =
        // Gamma_C[j] K^[m][j] (column j of the B1 slot's K^ rows); A2's lower half B-^T[j][m] =
        // Gamma_C[j] B^[m][j] (column j of its B^ rows)
        const float gcj = gcs[(n & 3) * 64 + t];
        const uint8_t *colb = b1 + (t >> 5) * (128 * 128) + (t & 3) * 4;
        const uint32_t cchunk = (t & 31) >> 2;
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          float kv[16], bv[16], z[16], bp[8];
#pragma unroll
          for (int x = 0; x < 16; ++x) {
            const uint32_t sw = (cchunk ^ (x & 7)) << 4;  // row 16c + x (and 64 + 16c + x) has (row & 7) == x & 7
            kv[x] = gcj * *reinterpret_cast<const float *>(colb + (64 + 16 * c + x) * 128 + sw);
            bv[x] = gcj * *reinterpret_cast<const float *>(colb + (16 * c + x) * 128 + sw);
            z[x] = 0.f;
          }
          tc::tmem_st16(X + 64 + 16 * c, kv);
          tc::tmem_st16(X + 16 * c, z);
          pack16(bv, bp);
          tc::tmem_st8(A2 + 8 * c, bp);
        }
        tc::tmem_st_wait();
      } else {
        // rows of Mrb (inclusive, m <= t) -> A2 upper half; R~ row t (A1) over them: the Q-part of D2
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          float v[16], bp[8];
          if (c < 2 * (dh + 1)) {
            tc::tmem_ld16(X + 16 * c, v);
            keep16(v, 16 * c, t);
          } else {
#pragma unroll
            for (int x = 0; x < 16; ++x) v[x] = 0.f;
          }
          pack16(v, bp);
          tc::tmem_st8(A2 + 8 * c, bp);
          tc::tmem_ld16(A1 + 16 * c, v);
          tc::tmem_st16(X + 16 * c, v);
        }
        tc::tc_fence_before();
        if (lane == 0) tc::mbar_arrive(bar(B_A1_EMPTY));
        __syncwarp();
        // rows of Mrk (inclusive) masked in place: the P-part
#pragma unroll 1
        for (int c = 2 * dh; c < 4; ++c) {
          float v[16];
          if (c < 2 * (dh + 1)) {
            tc::tmem_ld16(X + 64 + 16 * c, v);
            keep16(v, 16 * c, t);
          } else {
#pragma unroll
            for (int x = 0; x < 16; ++x) v[x] = 0.f;
          }
          tc::tmem_st16(X + 64 + 16 * c, v);
        }
        tc::tmem_st_wait();
        // the diagonal blocks of the inverse, once Lab is in Ls
        nbar_sync(NB_LS, 128);
        invert_diagonal(Ls, Ts, q, lane);
      }
      // B2 of the previous chunk overlays B3 and Zs: MMA2 of chunk n - 1 must be done with it
      if (!gwait(g, ctl, bar(B_M2), sl ^ 1u)) break;
      // the B1 slot has been read (MMA1 is done): the preparation of chunk n + 2 may overwrite it
      if (q == 0 && lane == 0) tc::mbar_arrive(bar(B_B1_EMPTY + sl));
      __syncwarp();
      invert_offdiag(Ls, Ts, Zs, sB3, q, lane);
      tc::fence_proxy_async_smem();
      tc::tc_fence_before();
      nbar_sync(NB_S2, 128);
      if (q == 0 && lane == 0) tc::mbar_arrive(bar(B_B3));
      __syncwarp();
      // D3 -> B2 (bf16, K-major: row = TMEM lane = column of [W~ U~], K = token)
      if (!gwait(g, ctl, bar(B_M3), sl)) break;
      tc::tc_fence_after();
      {
        const uint32_t nrow = 32 * q + lane;
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          float v[16];
          tc::tmem_ld16(tmem + TM_D4 + 64 * sl + lane_base + 16 * c, v);
          *reinterpret_cast<uint4 *>(sB2 + tc::sw128(nrow, 2 * c)) = pack_half(v, 0);
          *reinterpret_cast<uint4 *>(sB2 + tc::sw128(nrow, 2 * c + 1)) = pack_half(v, 1);
        }
      }
      tc::fence_proxy_async_smem();
      tc::tc_fence_before();
      nbar_sync(NB_S2, 128);
      if (q == 0 && lane == 0) tc::mbar_arrive(bar(B_B2));
      __syncwarp();
    }
  } else if (warp >= W_ST && warp < W_ST + 2) {
    // ===== the state chain ============================================================================
    const int j = tid - 32 * W_ST;  // key channel = TMEM lane 64 + j
    const uint32_t lane_base = static_cast<uint32_t>(64 + 32 * (warp - W_ST)) << 16;
    Group g{NB_ST, 64, j == 0, slots + 6, 0};
    // empty sequences (T = 0, or empty rows of a ragged batch) have no chunk: their end state is the
    // start state
    for (long long pr = blockIdx.x; pr < A.BH; pr += gridDim.x) {
      const int b = static_cast<int>(pr / A.H);
      if (seq_bounds(A.cu_seqlens, b, A.T, A.total_T).len != 0) continue;
      for (int i = 0; i < kN; ++i)
        A.s_out[pr * (kN * kN) + i * kN + j] = A.s_in ? A.s_in[pr * (kN * kN) + i * kN + j] : 0.f;
    }
    float s[64];  // s[p] = S[vinv(p)][j]
    // The state passes through B4S as float32 [i][j] (each thread its own column j, so no barrier is
    // needed between a thread's own writes and reads) around the rare steps done out of line.
    float *S = reinterpret_cast<float *>(sB4S);
    auto dump = [&]() {
#pragma unroll
      for (int p = 0; p < 64; ++p) S[vinv(p) * 64 + j] = s[p];
    };
    auto reload = [&]() {
#pragma unroll
      for (int p = 0; p < 64; ++p) s[p] = S[vinv(p) * 64 + j];
    };
    // S0 as the tf32 B operand of MMA4b (row p, K = j), then the MMA warp is told; B4S was last read
    // by MMA4b of the previous chunk, which is done.  This layout overlaps the other threads' float32
    // columns, so every state thread must be done reading those first.
    auto publish = [&]() {
      nbar_sync(NB_ST, 64);
      const uint32_t base = smem_u32(sB4S) + (j >> 5) * (64 * 128) + (j & 3) * 4;
      const uint32_t chunk = (j & 31) >> 2;
#pragma unroll
      for (int x = 0; x < 64; ++x)
        asm volatile("st.shared.u32 [%0], %1;\n" ::"r"(base + x * 128 + ((chunk ^ (x & 7)) << 4)), "r"(tf32r(s[x]))
                     : "memory");
      tc::fence_proxy_async_smem();
      nbar_sync(NB_ST, 64);
      if (j == 0) tc::mbar_arrive(bar(B_S_FULL));
      __syncwarp();
    };
    long long n = 0;
    ChunkIt it;
    bool more = it_first(A, it);
    if (more) {
      state_edge<kFused, kLN>(A, -1, it.pair, A.states ? it.pair * A.nck : -1, nullptr, S, nullptr, j);
      reload();
    }
    for (; more; ++n) {
      publish();
      const uint32_t sl = static_cast<uint32_t>(n & 1);
      if (!gwait(g, ctl, bar(B_M4 + sl), static_cast<uint32_t>((n >> 1) & 1), bar(B_GC + (n & 3)),
                 static_cast<uint32_t>((n >> 2) & 1)))
        break;
      tc::tc_fence_after();
      const bool flagged = gflag[n & 3] != 0;
      if (!flagged) {
        // S_C^T = diag(Gamma_C) S0^T + X (lanes 64..127 of D4; column p = value channel vinv(p))
        const float gcj = gcs[(n & 3) * 64 + j];
        const uint32_t d4 = tmem + TM_D4 + 64 * sl + lane_base;
        float v[32];
        tc::tmem_ld32(d4, v);
#pragma unroll
        for (int x = 0; x < 32; ++x) s[x] = fmaf(gcj, s[x], v[x]);
        tc::tmem_ld32(d4 + 32, v);
#pragma unroll
        for (int x = 0; x < 32; ++x) s[32 + x] = fmaf(gcj, s[32 + x], v[x]);
      }
      tc::tc_fence_before();
      const ChunkIt cur = it;
      more = it_next(A, it);
      const bool edge = !more || it.pair != cur.pair;
      if (flagged || edge || A.states != nullptr) {
        // out of line: a flagged chunk token by token (B4S is idle until the next S0); the finished
        // pair's end state out, the next pair's start state in; the next checkpoint
        dump();
        state_edge<kFused, kLN>(A, edge ? cur.pair : -1, more && edge ? it.pair : -1,
                                more && A.states ? it.pair * A.nck + it.c : -1, flagged ? &cur : nullptr, S,
                                reinterpret_cast<float *>(misc + MISC_FB), j);
        reload();
      }
      nbar_sync(NB_ST, 64);
      if (j == 0) tc::mbar_arrive(bar(B_D4_EMPTY + sl));
      __syncwarp();
    }
  } else if (warp >= W_Y && warp < W_Y + 2) {
    // ===== y ==========================================================================================
    const int t = tid - 32 * W_Y;  // token row = TMEM lane t
    const uint32_t lane_base = static_cast<uint32_t>(32 * (warp - W_Y)) << 16;
    Group g{NB_Y, 64, t == 0, slots + 8, 0};
    long long n = 0;
    ChunkIt it;
    for (bool more = it_first(A, it); more; more = it_next(A, it), ++n) {
      const uint32_t sl = static_cast<uint32_t>(n & 1);
      if (!gwait(g, ctl, bar(B_M4 + sl), static_cast<uint32_t>((n >> 1) & 1), bar(B_GC + (n & 3)),
                 static_cast<uint32_t>((n >> 2) & 1)))
        break;
      tc::tc_fence_after();
      if (gflag[n & 3] == 0) {
        float v[64];
        {
          float u[32];
          tc::tmem_ld32(tmem + TM_D4 + 64 * sl + lane_base, u);
#pragma unroll
          for (int x = 0; x < 32; ++x) v[x] = u[x];
          tc::tmem_ld32(tmem + TM_D4 + 64 * sl + lane_base + 32, u);
#pragma unroll
          for (int x = 0; x < 32; ++x) v[32 + x] = u[x];
        }
        if (kLN) {
          float mu = 0.f;
#pragma unroll
          for (int x = 0; x < 64; ++x) mu += v[x];
          mu *= (1.f / 64.f);
          float var = 0.f;
#pragma unroll
          for (int x = 0; x < 64; ++x) var = fmaf(v[x] - mu, v[x] - mu, var);
          const float rs = rsqrtf(var * (1.f / 64.f) + kLnEps);
          const float *lw = A.ln_w ? A.ln_w + it.h * kN : nullptr;
          const float *lb = A.ln_b ? A.ln_b + it.h * kN : nullptr;
#pragma unroll
          for (int i = 0; i < 64; ++i)
            v[vrow(i)] = fmaf((v[vrow(i)] - mu) * rs, lw ? lw[i] : 1.f, lb ? lb[i] : 0.f);
        }
        if (t < it.Lc) {
          uint16_t *dst = A.y + ((it.tok0 + t) * A.H + it.h) * kN;
#pragma unroll
          for (int cc = 0; cc < 8; ++cc) {
            uint4 w4;
            w4.x = pack_bf16x2(v[vrow(8 * cc + 0)], v[vrow(8 * cc + 1)]);
            w4.y = pack_bf16x2(v[vrow(8 * cc + 2)], v[vrow(8 * cc + 3)]);
            w4.z = pack_bf16x2(v[vrow(8 * cc + 4)], v[vrow(8 * cc + 5)]);
            w4.w = pack_bf16x2(v[vrow(8 * cc + 6)], v[vrow(8 * cc + 7)]);
            *reinterpret_cast<uint4 *>(dst + 8 * cc) = w4;
          }
        }
      }
      tc::tc_fence_before();
      nbar_sync(NB_Y, 64);
      if (t == 0) tc::mbar_arrive(bar(B_D4_EMPTY + sl));
      __syncwarp();
    }
  }
  __syncwarp();
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  if (warp == W_MMA) tc::tmem_dealloc(tmem, kTmemCols);
}

// ---- host side -----------------------------------------------------------------------------------

typedef CUresult (*PFN_encodeTiled)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                    const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                    CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// The driver's tensor-map encoder, looked up once (thread-safe static initialisation).
static PFN_encodeTiled get_encode() {
  static const PFN_encodeTiled fn = []() -> PFN_encodeTiled {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      return reinterpret_cast<PFN_encodeTiled>(p);
    return nullptr;
  }();
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
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

static int sm_count() {
  static std::mutex mu;
  static int cache[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
  std::lock_guard<std::mutex> lock(mu);
  if (cache[dev] == 0) {
    int sms = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess) cache[dev] = sms;
  }
  return cache[dev];
}

template <bool kFused, bool kLN>
static cudaError_t launch_variant(const Maps &maps, const Args &args, int grid, cudaStream_t stream) {
  cudaError_t e = cudaFuncSetAttribute(wkv7_pipe_kernel<kFused, kLN>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(kSmemBytes));
  if (e != cudaSuccess) return e;
  wkv7_pipe_kernel<kFused, kLN><<<grid, kThreads, kSmemBytes, stream>>>(maps, args);
  return cudaGetLastError();
}

}  // namespace pipe

cudaError_t launch_chunk_pipe(const uint16_t *r, const uint16_t *w, const uint16_t *k, const uint16_t *v,
                              const uint16_t *a, const uint16_t *b, bool model_native, const float *k_k,
                              bool group_norm, const float *ln_w, const float *ln_b, const float *s_in, uint16_t *y,
                              float *s_out, const int32_t *cu_seqlens, int B, int T, long long total_T, int H,
                              float *states, int *err_word, cudaStream_t stream) {
  using namespace pipe;
  if (states != nullptr && cu_seqlens != nullptr) return cudaErrorInvalidValue;
  if (total_T > 0x7fffffffLL || H > 0xffff || B > 65535) return cudaErrorInvalidValue;
  const long long BH = static_cast<long long>(B) * H;
  if (BH <= 0) return cudaSuccess;
  Maps maps;
  const uint16_t *ops[6] = {w, r, a, model_native ? nullptr : b, k, v};  // model-native: no b tile
  const long long tokens = total_T > 0 ? total_T : 1;
  for (int i = 0; i < 6; ++i) {
    // a zero-token call still needs a valid map; it never issues a load
    if (!make_map(&maps.m[i], ops[i] ? static_cast<const void *>(ops[i]) : static_cast<const void *>(s_out), tokens, H))
      return cudaErrorInvalidValue;
  }
  Args args{};
  for (int i = 0; i < 6; ++i) args.op[i] = ops[i];
  args.y = y;
  args.s_in = s_in;
  args.s_out = s_out;
  args.cu_seqlens = cu_seqlens;
  args.T = T;
  args.total_T = total_T;
  args.H = H;
  args.BH = BH;
  args.err = err_word;
  args.k_k = k_k;
  args.ln_w = ln_w;
  args.ln_b = ln_b;
  args.states = states;
  args.nck = (T + C - 1) / C;
  const int sms = sm_count();
  if (sms <= 0) return cudaErrorInvalidValue;
  const int grid = static_cast<int>(BH < sms ? BH : sms);
  if (model_native && group_norm) return launch_variant<true, true>(maps, args, grid, stream);
  if (model_native) return launch_variant<true, false>(maps, args, grid, stream);
  if (group_norm) return launch_variant<false, true>(maps, args, grid, stream);
  return launch_variant<false, false>(maps, args, grid, stream);
}

}  // namespace rwkv7
