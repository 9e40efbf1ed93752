// launch.h -- internal launchers behind the C ABI (not exported).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace rwkv7 {

// The library's device error word on the current device (looked up once per device), and the
// kernel choice of the bf16 prefill entry points for a path value and the longest sequence.
int *device_error_word();
bool prefill_uses_chunk(int path, long long max_T);

// Test hooks of the chunked prefill (process-wide): the bound of every device wait (0 = the
// production bound) and a (b, h) pair whose first chunk never raises its flag in the task-parallel
// schedule (-1 = none), so its successor's bounded wait runs out.
void set_chunk_test_hooks(uint32_t max_polls, long long skip_publish_pair);
// Zeroes the task-parallel schedule's flag words on the current device (synchronous).
cudaError_t clear_chain_flags();

// Sequential scan over [B,T,H,64] (cu_seqlens == nullptr) or a packed ragged
// batch (cu_seqlens = device offsets, total_T tokens).  TIn: float or
// uint16_t (bfloat16 bits).
template <typename TIn>
cudaError_t launch_scan(const TIn *r, const TIn *w, const TIn *k, const TIn *v, const TIn *a, const TIn *b,
                        const float *s_in, TIn *y, float *s_out, const int32_t *cu_seqlens, int B, int T,
                        long long total_T, int H, cudaStream_t stream);

// The bf16 scan with the optional parts: model-native inputs (w, a slots hold x_w, x_a; b unused;
// key scale k_k [H,64] float32 or nullptr for ones) and the GroupNorm epilogue on y (ln_w, ln_b
// [H,64] float32 or nullptr for ones / zeros).
cudaError_t launch_scan_ext(const uint16_t *r, const uint16_t *w, const uint16_t *k, const uint16_t *v,
                            const uint16_t *a, const uint16_t *b, bool model_native, const float *k_k,
                            bool group_norm, const float *ln_w, const float *ln_b, const float *s_in, uint16_t *y,
                            float *s_out, const int32_t *cu_seqlens, int B, int T, long long total_T, int H,
                            cudaStream_t stream);

// The bf16 scan (dense T) that also writes the state before every 64th token into states
// [B, H, ceil(T/64), 64, 64] (the checkpoints the backward starts from).
cudaError_t launch_scan_save(const uint16_t *r, const uint16_t *w, const uint16_t *k, const uint16_t *v,
                             const uint16_t *a, const uint16_t *b, const float *s_in, uint16_t *y, float *s_out,
                             float *states, int B, int T, int H, cudaStream_t stream);

// Gradients of the recurrence (see wkv7_backward.cu); dr, dw, dk, da, db must be zero on entry
// (they are accumulated), dv and ds_in (optional) are written.
cudaError_t launch_backward(const uint16_t *r, const uint16_t *w, const uint16_t *k, const uint16_t *v,
                            const uint16_t *a, const uint16_t *b, const float *states, const uint16_t *dy,
                            const float *ds_out, float *dr, float *dw, float *dk, float *dv, float *da, float *db,
                            float *ds_in, int B, int T, int H, cudaStream_t stream);

// One decode step over [B,H,64], state updated in place.
template <typename TIn>
cudaError_t launch_decode(const TIn *r, const TIn *w, const TIn *k, const TIn *v, const TIn *a, const TIn *b,
                          float *s, TIn *y, int B, int H, cudaStream_t stream);

// The bf16 step with the state stored as bf16 [B,H,64,64] (widened to float32 for the update, rounded
// to nearest-even on store).
// early_state: the state loads go out before the wait for the previous grid on the stream (the caller
// promises that no step still running before this one writes this step's state).
cudaError_t launch_decode_bf16state(const uint16_t *r, const uint16_t *w, const uint16_t *k, const uint16_t *v,
                                    const uint16_t *a, const uint16_t *b, bool early_state, uint16_t *s, uint16_t *y,
                                    int B, int H, cudaStream_t stream);

// The bf16 step with the optional parts: model-native inputs (w, a slots hold x_w, x_a; b unused;
// key scale k_k [H,64] float32 or nullptr for ones) and the GroupNorm epilogue on y (ln_w, ln_b
// [H,64] float32 or nullptr for ones / zeros); early_state as for launch_decode_bf16state.
cudaError_t launch_decode_ext(const uint16_t *r, const uint16_t *w, const uint16_t *k, const uint16_t *v,
                              const uint16_t *a, const uint16_t *b, bool model_native, const float *k_k,
                              bool group_norm, const float *ln_w, const float *ln_b, bool early_state, float *s,
                              uint16_t *y, int B, int H, cudaStream_t stream);

// The chunked prefill as a warp-specialised pipeline (one persistent CTA per SM walking its (b, h)
// pairs' chunks with three chunks in flight); same arguments as launch_chunk_ext without the schedule.
cudaError_t launch_chunk_pipe(const uint16_t *r, const uint16_t *w, const uint16_t *k, const uint16_t *v,
                              const uint16_t *a, const uint16_t *b, bool model_native, const float *k_k,
                              bool group_norm, const float *ln_w, const float *ln_b, const float *s_in, uint16_t *y,
                              float *s_out, const int32_t *cu_seqlens, int B, int T, long long total_T, int H,
                              float *states, int *err_word, cudaStream_t stream);

// Chunked tensor-core prefill (bfloat16 operands), same layouts as
// launch_scan.  err_word: device word that bounded waits report into.
cudaError_t launch_chunk(const uint16_t *r, const uint16_t *w, const uint16_t *k, const uint16_t *v,
                         const uint16_t *a, const uint16_t *b, const float *s_in, uint16_t *y, float *s_out,
                         const int32_t *cu_seqlens, int B, int T, long long total_T, int H, int *err_word,
                         cudaStream_t stream);

// The chunked prefill with the optional parts: model-native inputs (w, a slots hold x_w, x_a; b
// unused; key scale k_k [H,64] float32 or nullptr for ones) and the GroupNorm epilogue on y (ln_w,
// ln_b [H,64] float32 or nullptr for ones / zeros).  schedule: 0 = chosen from the shape, 1 = one
// CTA per (b, h), 2 = chunks of every pair spread over all SMs (cudaErrorInvalidValue when the
// shape does not allow it).  states: nullptr, or [B,H,ceil(T/64),64,64] float32 receiving the state
// before every chunk (dense T only).
cudaError_t launch_chunk_ext(const uint16_t *r, const uint16_t *w, const uint16_t *k, const uint16_t *v,
                             const uint16_t *a, const uint16_t *b, bool model_native, const float *k_k,
                             bool group_norm, const float *ln_w, const float *ln_b, const float *s_in, uint16_t *y,
                             float *s_out, const int32_t *cu_seqlens, int B, int T, long long total_T, int H,
                             int schedule, float *states, int *err_word, cudaStream_t stream);

}  // namespace rwkv7
