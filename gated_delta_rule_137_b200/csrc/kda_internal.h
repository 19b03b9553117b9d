// kda_internal.h — declarations shared by the library's translation units (not
// part of the public C ABI, which is include/kda.h).
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

#include "../../include/kda.h"
#include "sm100_ptx.cuh"

namespace kda {

// Head dimension the tensor-core prefill kernel is built for; other sizes are
// zero-padded to it (exact: padded channels carry log_alpha = 0 and zero data).
constexpr int kD = 128;
// Tokens per chunk of the chunked prefill.
constexpr int kChunk = 64;

// Workspace layout of kda_chunk_fwd / kda_mixer_fwd: the first 256 bytes hold the
// device status word; staging buffers (if any) follow at 256-byte boundaries.
constexpr size_t kStatusBytes = 256;

inline size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

struct PrefillArgs {
  const void* q;          // [total_T, H, 128], bf16 or fp32 (in_f32)
  const void* k;          // [total_T, H, 128]
  const void* v;          // [total_T, H, 128]
  const float* log_alpha; // fp32 [total_T, H, 128]
  const float* beta;      // fp32 [total_T, H]
  const float* h0;        // fp32 [N, H, 128, 128] or null
  const int32_t* cu;      // int32 [N+1] or null (equal lengths)
  const void* gate;       // bf16 [total_T, H, 128] or null (sigmoid output gate)
  const float* conv_w;    // fp32 [3, H*128, 4] or null: q, k, v are the raw mixer inputs and
                          // go through conv4 (+ L2 norm of q, k) inside the kernel
  void* out;              // [total_T, H, 128], bf16 or fp32 (out_f32)
  float* ht;              // fp32 [N, H, 128, 128] or null
  uint32_t* status;       // device status word
  int64_t total_T;
  int N, H;
  bool in_f32;            // q, k, v are fp32 (else bf16)
  bool out_f32;           // out is fp32 (else bf16)
  void* split_ws;         // split_workspace_bytes() of scratch for the two-pass prefill, or
                          // null for the single-pass kernel
  const void* a_pre;      // bf16 [total_T, H, 128] or null: the decay gate's pre-activation, with
  const float* a_scale;   // fp32 [H]: log_alpha = -a_scale[h] * softplus(a_pre) (log_alpha null);
                          // two-pass full mixer only
  float* map_M;           // segment maps (two-pass only): when set, the recurrence writes no
  float* map_B;           // outputs; half of its value-column slices run from the identity with zero
                          // values (their final states are M [N, H, 128, 128]), the other half from
                          // zero with the real values (B); out, ht and h0 are not used
  const int32_t* slots;   // int32 [N] or null: sequence n's final state goes to ht slot slots[n]
  int pool_size;          // (ht then holds pool_size states); a slot outside [0, pool_size) is
                          // flagged (kFlagBadIndex) and that state is not written
};

#ifdef __CUDACC__
// The index of sequence n's final state in a.ht: n, or its pool slot; -1 (nothing is
// written) for a slot outside the pool, which the thread with `flag` reports.
__device__ __forceinline__ int64_t final_state_index(const PrefillArgs& a, int n, bool flag) {
  if (!a.slots) return n;
  const int s = __ldg(a.slots + n);
  if (s >= 0 && s < a.pool_size) return s;
  if (flag && a.status) atomicOr(a.status, kFlagBadIndex);
  return -1;
}
#endif

// ---- two-pass prefill (kda_split.cu) ---------------------------------------------------
// Pass 1 writes one item of kItemBytes per (chunk, head) — the state-independent part
// of the chunk; pass 2 runs the recurrence over them. Scratch: the per-sequence chunk
// offsets, then the items.
// The split pays when there are few (sequence, head) chains: the single-pass kernel
// then has to cut each chain into value-column slices that all redo the chunk's
// state-free work. With more than kSplitMaxChains chains it runs whole chains per CTA
// with nothing repeated, and stays the faster form; it is used there, and above
// kSplitMaxItemBytes of items (it needs no scratch).
constexpr size_t kItemBytes = 147968;
constexpr size_t kSplitMaxItemBytes = size_t{32} << 30;
// Upper bound on the number of 64-token chunks over all sequences (each sequence adds at
// most one partial chunk; every chunk holds at least one token).
inline int64_t split_max_chunks(int64_t total_T, int N) {
  const int64_t c = total_T / kChunk + N;
  return c < total_T ? c : total_T;
}
// per-sequence first chunks [N + 1], then one flag: some item was handed over as raw rows
inline size_t split_plan_bytes(int N) { return align256((static_cast<size_t>(N) + 2) * sizeof(int32_t)); }
constexpr int64_t kSplitMaxChains = 74;  // half of the 148 SMs: beyond it no slicing is needed
inline size_t split_workspace_bytes(int64_t total_T, int N, int H, bool any_chains = false) {
  if (total_T <= 0 || N <= 0) return 0;
  if (!any_chains && static_cast<int64_t>(N) * H > kSplitMaxChains) return 0;
  const size_t items = static_cast<size_t>(split_max_chunks(total_T, N)) * static_cast<size_t>(H) * kItemBytes;
  if (items > kSplitMaxItemBytes) return 0;
  return split_plan_bytes(N) + items;
}
cudaError_t launch_prefill_split(const PrefillArgs& a, cudaStream_t stream);
// The recurrence alone over the plan and items a previous launch_prefill_split left in
// a.split_ws (same sequences): outputs and final states from a new initial state.
cudaError_t launch_recur_only(const PrefillArgs& a, cudaStream_t stream);
// cu_seqlens (or N equal lengths) -> chunk_start[N + 1]: the first 64-token chunk of each
// sequence, [N] = total; -1 there and the status flag on bad cu_seqlens.
cudaError_t launch_plan(const int32_t* cu, int64_t total_T, int N, int32_t* chunk_start, uint32_t* status,
                        cudaStream_t stream);

// Backward of the recurrence (kda_backward.cu).
size_t bwd_workspace_bytes(int64_t total_T, int N, int H);
cudaError_t launch_backward(const void* q, const void* k, const void* v, bool bf16, const float* log_alpha,
                            const float* beta, const float* h0, const int32_t* cu, int64_t total_T, int N, int H,
                            const void* d_out, const float* d_final, float* dq, float* dk, float* dv, float* dla,
                            float* dbeta, float* dh0, void* ws, uint32_t* status, cudaStream_t stream);

// Sets the message kda_last_error() returns on this host thread.
void set_last_error(const char* msg);

cudaError_t launch_decode_step(const void* q, const void* k, const void* v, bool bf16, const float* log_alpha,
                               const float* beta, float* state, int N, int H, int dk, int dv, void* out,
                               cudaStream_t stream);

// Serving decode of the full mixer, K tokens per sequence (d = 128, bf16 raw inputs and
// out); with checkpoints the pools are left unchanged.
cudaError_t launch_mixer_decode(const void* q_raw, const void* k_raw, const void* v_raw, const float* conv_w,
                                const float* log_alpha, const float* beta, const void* gate, float* state_pool,
                                void* conv_pool, const int32_t* state_indices, int pool_size, int N, int K, int H,
                                void* out, float* state_ckpt, void* conv_ckpt, uint32_t* status, cudaStream_t stream);
cudaError_t launch_mixer_decode_commit(const float* state_ckpt, const void* conv_ckpt, const int32_t* accepted,
                                       float* state_pool, void* conv_pool, const int32_t* state_indices,
                                       int pool_size, int N, int K, int H, uint32_t* status, cudaStream_t stream);

// out[i] = M[i] S[i] + B[i] for `count` 128 x 128 fp32 matrices (S, B may be null: zero).
cudaError_t launch_state_affine(const float* M, const float* S, const float* B, float* out, int64_t count,
                                cudaStream_t stream);
// S <- M_j S + B_j for j = 0 .. maps-1 (MB: [maps][2][count][128][128]; S0 null: zero).
// The serving hand-off after a pooled mixer prefill: each sequence's last three raw q, k,
// v rows (zeros before its start) into conv_pool[slot] ([pool, H, 3, 3, 128] bf16); with
// copy_states, also state_pool[slot] <- h0[n] (or zero), for calls with no tokens.
cudaError_t launch_pool_store(const void* q_raw, const void* k_raw, const void* v_raw, const int32_t* cu,
                              int64_t total_T, int N, int H, const int32_t* slots, int pool_size, void* conv_pool,
                              bool copy_states, const float* h0, float* state_pool, uint32_t* status,
                              cudaStream_t stream);
cudaError_t launch_state_fold(const float* MB, int maps, const float* S0, float* out, int64_t count,
                              cudaStream_t stream);

// Tensor-core chunked prefill on d = 128 operands (bf16 or fp32 q/k/v/out).
cudaError_t launch_prefill_d128(const PrefillArgs& a, cudaStream_t stream);

// Staging for head dims below 128: zero-pads q/k/v (in their own dtype), log_alpha
// and the initial state to d = 128, and copies the results back.
cudaError_t launch_stage_in(const void* q, const void* k, const void* v, bool bf16, const float* log_alpha,
                            const float* h0, int64_t total_T, int N, int H, int dk, int dv, void* q_p, void* k_p,
                            void* v_p, float* la_p, float* h0_p, cudaStream_t stream);
cudaError_t launch_stage_out(const void* out_p, const float* ht_p, bool bf16, int64_t total_T, int N, int H, int dk,
                             int dv, void* out, float* ht, cudaStream_t stream);

// Two-stage form of the full mixer: conv4 + L2 pre-stage into fp32 scratch buffers,
// then the recurrence (used where the scratch is provided by the caller's side).
kda_status mixer_fwd_staged(const void* q_raw, const void* k_raw, const void* v_raw, const float* conv_w,
                            const float* log_alpha, const float* beta, const void* gate, const float* initial_state,
                            const int32_t* cu_seqlens, int64_t total_T, int N, int H, void* out, float* final_state,
                            void* scratch, cudaStream_t stream);
inline size_t mixer_staged_scratch_bytes(int64_t total_T, int H) {
  return kStatusBytes + 3 * align256(static_cast<size_t>(total_T) * H * kD * sizeof(float));
}

// Pre-stage of the two-stage mixer: causal depthwise conv (width 4) on q, k, v, L2
// norm of q and k, written in fp32 (no intermediate rounding).
cudaError_t launch_conv_l2(const void* q_raw, const void* k_raw, const void* v_raw, const float* conv_w,
                           const int32_t* cu, int64_t total_T, int N, int H, int d, void* q_o, void* k_o, void* v_o,
                           uint32_t* status, cudaStream_t stream);

}  // namespace kda
