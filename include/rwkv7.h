/*
 * rwkv7.h -- C ABI of the RWKV-7 (x070) state-recurrence library for NVIDIA
 * B200 (sm_100a).
 *
 * The operation (RWKV-7 G0 7.2B walkthrough, lshu.cn/news/198401, section 7.1,
 * "the two core operators of x070"): for every batch row b and head h an
 * N x N float32 state S (N = 64; row i = value channel, column j = key
 * channel) is updated token by token as
 *
 *     sa   = S a_t                                   (state before the update)
 *     S    = S diag(w_t) + sa b_t^T + v_t k_t^T
 *     y_t  = S r_t                                   (state after the update)
 *
 * "Prefill" runs this over a whole sequence at once (the pages' GPT mode,
 * kernel wkv7); "decode" runs one token and updates the state in place (the
 * pages' RNN mode, kernel wkv7s).  The RWKV-LM README copy (oa0.com/c/1004164)
 * notes that the state and w must be kept in fp32 because w can be very close
 * to 1: the state is float32 everywhere here and all accumulation is float32.
 *
 * Layouts (row-major, contiguous, no padding):
 *   prefill operands r, w, k, v, a, b and output y : [B, T, H, N]
 *   varlen operands and y (packed tokens)          : [total_T, H, N]
 *   decode operands and y                          : [B, H, N]
 *   states s_in, s_out, s_inout                    : [B, H, N, N] float32,
 *                                                    element (b,h,i,j) at ((b*H+h)*N+i)*N+j
 *   "_bf16" entry points take the operands and write y as bfloat16 bit
 *   patterns (uint16_t); the others use float32.
 *
 * Ownership and execution:
 *   - Every pointer is a device pointer owned by the caller (except the host
 *     buffers of rwkv7_wkv_prefill_host_bf16); the library allocates no memory
 *     per call and keeps no pointer after returning.
 *   - Calls only enqueue work on `stream` (NULL = the legacy default stream)
 *     and return; they never synchronise, so they can be captured into a CUDA
 *     graph.  Results are ready once the stream reaches that point.  (The
 *     host-buffer prefill also uses two streams of its own, ordered after
 *     `stream` and joined back into it.)
 *   - s_in may be NULL (zero initial state) and may equal s_out (in place).
 *     y must not overlap any other argument.
 *   - Every pointer must be 16-byte aligned.
 *
 * Errors: a call returns RWKV7_OK once its kernels are enqueued.  Arguments are
 * checked on the host first and nothing is launched when one is wrong:
 *   N != 64                                  -> RWKV7_ERR_UNSUPPORTED
 *   B, H <= 0, T < 0, a NULL required pointer -> RWKV7_ERR_INVALID
 *   a pointer that is not 16-byte aligned     -> RWKV7_ERR_ALIGN
 *   a failed launch                           -> RWKV7_ERR_CUDA
 * Kernels that wait on an mbarrier or on another CTA give up after a bounded
 * number of polls, record the fact in a device error word and return;
 * rwkv7_get_last_error() reads and clears that word (it synchronises the
 * current device).  When the word holds an error it also resets the chunked
 * kernel's chain flags, so after a timeout, replays of a captured launch are
 * valid again only once it has been called.
 * No C++ exception crosses this interface.
 */
#ifndef RWKV7_H
#define RWKV7_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define RWKV7_API __attribute__((visibility("default")))
#else
#define RWKV7_API
#endif

/* Same type as cudaStream_t, declared without the CUDA headers. */
struct CUstream_st;
typedef struct CUstream_st *rwkv7_stream_t;

typedef enum rwkv7_status {
  RWKV7_OK = 0,
  RWKV7_ERR_INVALID = 1,
  RWKV7_ERR_ALIGN = 2,
  RWKV7_ERR_CUDA = 3,
  RWKV7_ERR_TIMEOUT = 4,
  RWKV7_ERR_UNSUPPORTED = 5,
  RWKV7_ERR_DOMAIN = 6
} rwkv7_status;

/* Prefill kernels: AUTO picks by T and dtype (bf16 with T >= 48 -> CHUNK,
 * otherwise SCAN); SCAN is the sequential kernel (state in registers); CHUNK
 * is the chunked tensor-core kernel (bf16 only).
 * Decay domain of CHUNK: the chunked form divides by the product of up to 64
 * consecutive decays, so it factorises a 64-token chunk only while that
 * product stays >= 2^-100 in every channel (true whenever every w >= 0.34; the
 * model's decay exp(-e^-0.5 sigmoid(x)) always lies in [0.5452, 1)).  A chunk
 * outside that range (w near 0, or exactly 0) is detected on the device and run
 * token by token in float32 instead, on every schedule, so CHUNK, AUTO and SCAN
 * are exact for every w in [0, 1].  (With model-native inputs the decay cannot
 * leave the range; there such a chunk would be reported by
 * rwkv7_get_last_error() as RWKV7_ERR_DOMAIN.) */
typedef enum rwkv7_prefill_path {
  RWKV7_PATH_AUTO = 0,
  RWKV7_PATH_SCAN = 1,
  RWKV7_PATH_CHUNK = 2
} rwkv7_prefill_path;

/* ---- prefill ("GPT mode", wkv7) ------------------------------------------
 * Runs T tokens of every (b, h) from s_in (NULL = zero) and writes y for
 * every token and the final state to s_out.  T == 0 copies s_in (or zeros)
 * to s_out and writes no y.  Float32 operands; uses the sequential kernel. */
RWKV7_API rwkv7_status rwkv7_wkv_prefill(int B, int T, int H, int N, const float *r, const float *w,
                               const float *k, const float *v, const float *a, const float *b,
                               const float *s_in, float *y, float *s_out, rwkv7_stream_t stream);

/* Same, bfloat16 operands and y (bit patterns), float32 state.  The kernel is
 * chosen as for RWKV7_PATH_AUTO (see the decay domain above: exact for every
 * w in [0, 1]). */
RWKV7_API rwkv7_status rwkv7_wkv_prefill_bf16(int B, int T, int H, int N, const uint16_t *r,
                                    const uint16_t *w, const uint16_t *k, const uint16_t *v,
                                    const uint16_t *a, const uint16_t *b, const float *s_in,
                                    uint16_t *y, float *s_out, rwkv7_stream_t stream);

/* bfloat16 prefill with an explicit kernel choice (for cross-checks and
 * timing).  `path` is an rwkv7_prefill_path value; an unknown value returns
 * RWKV7_ERR_INVALID. */
RWKV7_API rwkv7_status rwkv7_wkv_prefill_bf16_path(int path, int B, int T, int H, int N, const uint16_t *r,
                                         const uint16_t *w, const uint16_t *k, const uint16_t *v,
                                         const uint16_t *a, const uint16_t *b, const float *s_in,
                                         uint16_t *y, float *s_out, rwkv7_stream_t stream);

/* Ragged batch in packed layout (the long-context workload at the 7.2B width
 * with per-row lengths, as a serving batch of unequal prompts; the pages'
 * GPT mode, RWKV-7 G0 7.2B walkthrough, lshu.cn/news/198401, section 3.2, runs
 * each row as its own sequence): B sequences, row b owns the tokens
 * cu_seqlens[b] .. cu_seqlens[b+1]-1 of the [total_T, H, N] operands.
 * cu_seqlens is a DEVICE array of B+1 non-decreasing int32 offsets with
 * cu_seqlens[0] = 0 and cu_seqlens[B] = total_T (not checked on the host,
 * since it lives on the device; rows whose offsets fall outside
 * [0, total_T] are skipped and leave their y and s_out untouched).
 * `max_T` is an upper bound on the longest row (used for scheduling; rows
 * longer than it are still processed completely).  s_in / s_out are
 * [B, H, N, N]. */
RWKV7_API rwkv7_status rwkv7_wkv_prefill_varlen_bf16(int path, int B, int total_T, int max_T, int H, int N,
                                           const int32_t *cu_seqlens, const uint16_t *r,
                                           const uint16_t *w, const uint16_t *k,
                                           const uint16_t *v, const uint16_t *a,
                                           const uint16_t *b, const float *s_in, uint16_t *y,
                                           float *s_out, rwkv7_stream_t stream);

/* ---- decode ("RNN mode", wkv7s) ------------------------------------------
 * One token for every (b, h): operands [B, H, N], state [B, H, N, N] updated
 * in place, y [B, H, N]. */
RWKV7_API rwkv7_status rwkv7_wkv_decode(int B, int H, int N, const float *r, const float *w, const float *k,
                              const float *v, const float *a, const float *b, float *s_inout,
                              float *y, rwkv7_stream_t stream);

RWKV7_API rwkv7_status rwkv7_wkv_decode_bf16(int B, int H, int N, const uint16_t *r, const uint16_t *w,
                                   const uint16_t *k, const uint16_t *v, const uint16_t *a,
                                   const uint16_t *b, float *s_inout, uint16_t *y,
                                   rwkv7_stream_t stream);

/* ---- model-native inputs (operand prologue fused into the kernels) ------------
 *
 * The same recurrence, but the caller passes what the x070 time-mix produces before its operand
 * prologue (RWKV-7 G0 7.2B walkthrough, lshu.cn/news/198401, section 7.1), and the kernels form
 * the operands in float32:
 *   w = exp(-exp(-softplus(-xw) - 0.5))          (decay in (0.5452, 1))
 *   kk = normalize(k * k_k) over the 64 channels   (x / max(|x|, 1e-12))
 *   a = -kk,  b = kk * sigmoid(xa)
 * and k enters the recurrence as given.  Five token tensors instead of six.
 *
 * r, xw, k, v, xa: bf16 bit patterns [B,T,H,64] (prefill) / [B,H,64] (decode), 16-byte aligned.
 * k_k: float32 [H,64] key scale, or NULL for ones (16-byte aligned when given; device memory).
 * Everything else (state, y, ownership, errors, paths) as for the bf16 entry points above; the
 * CHUNK path has no extra domain condition here, since every decay is >= 0.5452. */
RWKV7_API rwkv7_status rwkv7_wkv_prefill_fused_bf16(int path, int B, int T, int H, int N, const uint16_t *r,
                                                    const uint16_t *xw, const uint16_t *k, const uint16_t *v,
                                                    const uint16_t *xa, const float *k_k, const float *s_in,
                                                    uint16_t *y, float *s_out, rwkv7_stream_t stream);

RWKV7_API rwkv7_status rwkv7_wkv_decode_fused_bf16(int B, int H, int N, const uint16_t *r, const uint16_t *xw,
                                                   const uint16_t *k, const uint16_t *v, const uint16_t *xa,
                                                   const float *k_k, float *s_inout, uint16_t *y,
                                                   rwkv7_stream_t stream);

/* ---- options: model-native inputs and the ln_x epilogue, in any combination ----
 *
 * A host struct read during the call; zero-initialise it for none of the parts, or pass NULL.
 *   model_native = 1: the w and a arguments hold the pre-activations x_w and x_a, b is ignored (may
 *                     be NULL) and k_k is the key scale (see the fused entry points above).
 *   group_norm = 1:   the x070 ln_x epilogue (RWKV-7 G0 7.2B walkthrough, lshu.cn/news/198401,
 *                     section 7.1: GroupNorm with one group per head, eps 64e-5) is applied to y:
 *                     y = (y - mean) / sqrt(var + 64e-5) * ln_w + ln_b over each token-head's 64
 *                     channels (variance with divisor 64).  ln_w / ln_b: float32 [H,64] device
 *                     buffers, 16-byte aligned, NULL meaning ones / zeros.
 * The state is not affected by group_norm.
 *   chunk_schedule:   how the CHUNK path spreads its work (prefill only; results are the same up
 *                     to float32 rounding order):
 *                     0 = chosen from the shape;
 *                     1 = one CTA per (b, h), walking its chunks with the state on chip;
 *                     2 = every chunk of every (b, h) is a task, spread over all SMs; each chunk
 *                         takes its start state from s_out, where the previous chunk of the same
 *                         (b, h) left it (flags in library-owned device memory order the two).
 *                         Needs B*H <= 65536 (else RWKV7_ERR_CUDA).  Up to 4 such launches may
 *                         run at once on a device: successive launches take 4 flag slots in
 *                         turn.  A launch captured in a CUDA graph keeps the slot of its capture
 *                         for every replay, so graphs replayed at the same time must have been
 *                         captured into different slots (captures that are not 4 launches apart);
 *                         every launch leaves the flags zeroed unless it times out (see Errors).
 *                         Choice 0 never takes this schedule while `stream` is capturing.
 *                     3 = a warp-specialised pipeline: one persistent CTA per SM walks its (b, h)
 *                         pairs' chunks with three chunks in flight (operand preparation, masks
 *                         and inverse, state chain on separate warps).  Needs H <= 65535.
 *                     Every schedule is exact for every decay in [0, 1] (see the decay domain
 *                     above).
 *   independent_state = 1 (decode only, library scheduling with no counterpart on the pages; the
 *                     prefill ignores it): the caller promises that the decode step queued just
 *                     before this one on `stream` does not write this step's state.  The decode
 *                     kernels start under programmatic dependent launch: a step's CTAs may start
 *                     while the step before is finishing, and they read nothing that step writes
 *                     before it has completed.  With this option they load their state before that
 *                     wait, so the state loads overlap the previous step's last wave.  Results are
 *                     the same; only the timing changes.  The option takes effect only when B*H
 *                     exceeds the CTAs the device runs at once (the library checks; smaller steps
 *                     wait first as without it): with steps of that size queued back to back, no
 *                     step older than the one before is still running when a step's CTAs start.
 *                     A model whose layers each keep their own state, stepped in turn, qualifies.
 *                     Consecutive steps of one state do not: with the option set they could read a
 *                     state that is not yet written.  Left 0, every step waits first, which is
 *                     always correct.
 */
typedef struct rwkv7_options {
  int model_native;
  const float *k_k;
  int group_norm;
  const float *ln_w;
  const float *ln_b;
  int chunk_schedule;
  int independent_state;
} rwkv7_options;

/* ---- prefill from and to host memory ------------------------------------------------------
 *
 * The pages run the model from host-side code (the RWKV-LM README copy, oa0.com/c/1004164, and the
 * walkthrough's GPT / RNN modes, lshu.cn/news/198401, section 3.2) but give no call of this kind; it
 * is the end-to-end form of the prefill for a caller whose tokens and state live in host memory.
 * The bf16 prefill of rwkv7_wkv_prefill_bf16_path for operands that live in host memory: r, w, k,
 * v, a, b ([B,T,H,64] bf16), s_in ([B,H,64,64] float32, NULL = zero state), y and s_out are HOST
 * pointers; dev_r .. dev_b, dev_s_in, dev_y, dev_s_out are DEVICE buffers of the same shapes that
 * the call uses as staging (dev_s_in may be NULL when s_in is).  The batch is cut into `slices`
 * runs of whole rows b (0 = chosen by the call, at most B); per slice the call copies the slice's
 * operands (and initial state) host -> device, runs the prefill on it once they have landed, and
 * copies its y and final state device -> host, on two internal streams ordered after `stream`, so
 * the copies of one slice overlap the compute and the copies of others.  On return the work is
 * queued; `stream` waits for all of it (synchronise `stream` before reading y / s_out).  For the
 * copies to overlap, the host buffers must be page-locked (cudaHostAlloc / cudaHostRegister);
 * pageable buffers give the same results without overlap.  Every pointer must be 16-byte aligned.
 * The two internal streams are created on a device's first call and kept until the process exits
 * (calls on one device share them, so their work is ordered; each call creates and releases only a
 * few events).  Not meant for CUDA graph capture: the work forks onto those streams.
 * Errors as for the device entry point; a failure leaves the outputs undefined. */
RWKV7_API rwkv7_status rwkv7_wkv_prefill_host_bf16(int path, int B, int T, int H, int N, const uint16_t *r,
                                                   const uint16_t *w, const uint16_t *k, const uint16_t *v,
                                                   const uint16_t *a, const uint16_t *b, const float *s_in,
                                                   uint16_t *y, float *s_out, uint16_t *dev_r, uint16_t *dev_w,
                                                   uint16_t *dev_k, uint16_t *dev_v, uint16_t *dev_a,
                                                   uint16_t *dev_b, float *dev_s_in, uint16_t *dev_y,
                                                   float *dev_s_out, int slices, rwkv7_stream_t stream);

/* ---- prefill from and to host memory, allocating nothing ----------------------------------
 *
 * The pages have no counterpart of this call: it exists for callers that hold their data in host
 * memory and cannot allocate device memory.  Examples: a plain C program or a binding from another
 * language that reaches the GPU only through this library and does not link the CUDA runtime, so it
 * has no way to create device buffers; a process whose device memory is handed out by an allocator
 * it does not control; a serving loop that must not call cudaMalloc / cudaFree, which can
 * synchronise the whole device.  rwkv7_wkv_prefill_host_bf16 needs device staging buffers from its
 * caller; this call instead stages through one array of RWKV7_NOALLOC_STAGING_BYTES in the
 * library's static device memory (every GPU that loads the library holds it until the process
 * exits) and allocates nothing: no cudaMalloc, no cudaFree, no stream or event.
 *
 * r, w, k, v, a, b ([B,T,H,64] bf16), s_in ([B,H,64,64] float32, NULL = zero state), y and s_out are
 * HOST pointers, 16-byte aligned.  On `stream` the call copies the operands (and s_in) into the
 * array, runs the prefill that `path` selects (as rwkv7_wkv_prefill_bf16_path), and copies y and the
 * final state back; synchronise `stream` before reading y / s_out.  Page-locked host buffers make
 * the copies asynchronous; pageable ones give the same results.
 *   Size limit: with P = B*T*H*64*2 bytes (one operand) and Q = B*H*64*64*4 bytes (one state), each
 *   rounded up to a multiple of 256, the call needs 7*P + Q bytes (7*P + 2*Q when s_in is given).
 *   A call that needs more than RWKV7_NOALLOC_STAGING_BYTES returns RWKV7_ERR_INVALID and enqueues
 *   nothing.
 *   Shared array: every call uses the same array, which keeps the previous call's contents (nothing
 *   in it has to start at zero: each call writes every byte it reads).  Calls whose work overlaps
 *   on the GPU (other streams, other host threads) race on it; calls on one stream are ordered.
 *   Set-up: the first call on a device looks up the array's device address (cudaGetSymbolAddress,
 *   with that device current) and caches it; make that first call before any stream capture.
 * Other errors as for rwkv7_wkv_prefill_host_bf16. */
#define RWKV7_NOALLOC_STAGING_BYTES (32u * 1024u * 1024u)
RWKV7_API rwkv7_status rwkv7_wkv_prefill_host_noalloc_bf16(int path, int B, int T, int H, int N,
                                                           const uint16_t *r, const uint16_t *w,
                                                           const uint16_t *k, const uint16_t *v,
                                                           const uint16_t *a, const uint16_t *b,
                                                           const float *s_in, uint16_t *y, float *s_out,
                                                           rwkv7_stream_t stream);

/* bf16 prefill with options (NULL = none); other arguments as for rwkv7_wkv_prefill_bf16_path. */
RWKV7_API rwkv7_status rwkv7_wkv_prefill_ext_bf16(int path, int B, int T, int H, int N, const uint16_t *r,
                                                  const uint16_t *w, const uint16_t *k, const uint16_t *v,
                                                  const uint16_t *a, const uint16_t *b, const rwkv7_options *opt,
                                                  const float *s_in, uint16_t *y, float *s_out,
                                                  rwkv7_stream_t stream);

/* bf16 decode step with options (NULL = none); other arguments as for rwkv7_wkv_decode_bf16. */
RWKV7_API rwkv7_status rwkv7_wkv_decode_ext_bf16(int B, int H, int N, const uint16_t *r, const uint16_t *w,
                                                 const uint16_t *k, const uint16_t *v, const uint16_t *a,
                                                 const uint16_t *b, const rwkv7_options *opt, float *s_inout,
                                                 uint16_t *y, rwkv7_stream_t stream);

/* ---- reduced-precision decode state ------------------------------------------------------
 *
 * The decode step with the state kept in HBM as bfloat16 [B, H, 64, 64] (s_inout: bf16 bit patterns,
 * updated in place): each step widens it to float32, applies the update above in float32, writes y,
 * and rounds the new state to nearest-even bf16.  Half the state traffic of rwkv7_wkv_decode_bf16
 * (quantised states are explored in the RWKV-8 preview, trdm.cn/news/547794).
 * The pages keep the state in fp32 because w can be very close to 1 (RWKV-LM README copy,
 * oa0.com/c/1004164); with a bf16 state every step adds up to 2^-8 relative rounding to it, so
 * long decodes drift from the float32-state result: an opt-in for memory-bound serving, not the
 * default.  Other arguments, errors and ownership as for rwkv7_wkv_decode_bf16. */
RWKV7_API rwkv7_status rwkv7_wkv_decode_bf16_bf16state(int B, int H, int N, const uint16_t *r, const uint16_t *w,
                                                       const uint16_t *k, const uint16_t *v, const uint16_t *a,
                                                       const uint16_t *b, uint16_t *s_inout, uint16_t *y,
                                                       rwkv7_stream_t stream);

/* The same step with options (NULL = none): only independent_state applies (see rwkv7_options);
 * model_native or group_norm set returns RWKV7_ERR_INVALID.  Other arguments, errors and ownership
 * as for rwkv7_wkv_decode_bf16_bf16state. */
RWKV7_API rwkv7_status rwkv7_wkv_decode_ext_bf16state(int B, int H, int N, const uint16_t *r, const uint16_t *w,
                                                      const uint16_t *k, const uint16_t *v, const uint16_t *a,
                                                      const uint16_t *b, const rwkv7_options *opt,
                                                      uint16_t *s_inout, uint16_t *y, rwkv7_stream_t stream);

/* ---- training: forward with checkpoints, and the backward ----------------------------------
 *
 * The gradients of a loss L with respect to the operands and the initial state, given dL/dy
 * (dy) and dL/ds_out (ds_out).  The pages give no backward; it is the chain rule applied to the
 * recurrence above (RWKV-7 G0 7.2B walkthrough, lshu.cn/news/198401, section 7.1): walking the
 * tokens from the last, with G = dL/dS' for the state S' after token t and S the state before it,
 *   G += dy_t r_t^T;  dr_t = S'^T dy_t;  dv_t = G k_t;  dk_t = G^T v_t;  db_t = G^T (S a_t);
 *   g = G b_t;  dw_t[j] = sum_i G[i][j] S[i][j];  da_t = S^T g;  G <- G diag(w_t) + g a_t^T,
 * and ds_in = G at the start.
 *
 * rwkv7_wkv_prefill_save_bf16: rwkv7_wkv_prefill_bf16_path that also writes the state before every
 *   64th token: states float32 [B, H, ceil(T/64), 64, 64] (device, 16-byte aligned, caller-owned;
 *   states[b,h,c] = the state before token 64c, so states[b,h,0] = s_in or zeros).
 * rwkv7_wkv_backward_bf16: r, w, k, v, a, b, dy bf16 [B,T,H,64] (the forward's operands and dL/dy);
 *   states from the forward above; ds_out float32 [B,H,64,64] or NULL (zero).  Outputs float32
 *   [B,T,H,64]: dr, dw, dk, dv, da, db (all required; dr, dw, dk, da, db are zeroed on the stream
 *   and accumulated, so they must not alias each other or an input); ds_in float32 [B,H,64,64] or
 *   NULL.  Dense batches only (no cu_seqlens).  Same status codes as the other entry points; the
 *   library allocates nothing. */
RWKV7_API rwkv7_status rwkv7_wkv_prefill_save_bf16(int path, int B, int T, int H, int N, const uint16_t *r,
                                                   const uint16_t *w, const uint16_t *k, const uint16_t *v,
                                                   const uint16_t *a, const uint16_t *b, const float *s_in,
                                                   uint16_t *y, float *s_out, float *states,
                                                   rwkv7_stream_t stream);

RWKV7_API rwkv7_status rwkv7_wkv_backward_bf16(int B, int T, int H, int N, const uint16_t *r, const uint16_t *w,
                                               const uint16_t *k, const uint16_t *v, const uint16_t *a,
                                               const uint16_t *b, const float *states, const uint16_t *dy,
                                               const float *ds_out, float *dr, float *dw, float *dk, float *dv,
                                               float *da, float *db, float *ds_in, rwkv7_stream_t stream);

/* ---- test hook ------------------------------------------------------------------------------
 *
 * For tests of the failure path only (the pages have no counterpart): sets, for every later launch
 * of the chunked kernel in this process, the bound of each device wait to `max_polls` polls (0 =
 * the production bound, about 2^22) and, in the task-parallel schedule, names a (b, h) pair
 * `skip_publish_pair` = b*H + h whose first chunk never raises its chain flag (-1 = none), so that
 * the wait of its second chunk runs out.  Such a launch returns with RWKV7_ERR_TIMEOUT recorded
 * (rwkv7_get_last_error) and its y and s_out are not valid.  Not thread-safe with concurrent
 * launches; call rwkv7_test_set_wait_hooks(0, -1) to restore production behaviour.  Always
 * returns RWKV7_OK. */
RWKV7_API rwkv7_status rwkv7_test_set_wait_hooks(unsigned max_polls, long long skip_publish_pair);

/* ---- status ----------------------------------------------------------------
 * Library plumbing with no counterpart on the pages: how a caller learns that a call was refused
 * (the return codes above) or that a kernel gave up or met inputs outside its range (the device
 * error word below).  RWKV7_ERR_DOMAIN follows from the pages' own fp32 note on w (RWKV-LM README
 * copy, oa0.com/c/1004164): the chunked form divides by decay products, which only float32 range
 * limits. */

/* Static English description of a status code (never NULL). */
RWKV7_API const char *rwkv7_status_string(rwkv7_status status);

/* Reads and clears the device error word of the current device (RWKV7_OK,
 * RWKV7_ERR_TIMEOUT or RWKV7_ERR_DOMAIN: the first error recorded since the
 * last call), and reports a pending CUDA error as RWKV7_ERR_CUDA.
 * Synchronises the current device.  When it reports an error it also zeroes the
 * chunked kernel's chain flags (see chunk_schedule 2). */
RWKV7_API rwkv7_status rwkv7_get_last_error(void);

/* Library version as major*10000 + minor*100 + patch. */
RWKV7_API int rwkv7_version(void);

#ifdef __cplusplus
}
#endif

#endif /* RWKV7_H */
