// kda_abi.cu — the extern "C" boundary of libkda.so: argument validation on the
// host, workspace sizing, status strings, and dispatch to the kernels.
#include <cstdarg>
#include <cstdio>
#include <cstring>

#include "kda_internal.h"

namespace {

thread_local char g_last_error[512] = "";

kda_status fail(kda_status s, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_last_error, sizeof(g_last_error), fmt, ap);
  va_end(ap);
  return s;
}

kda_status ok() {
  g_last_error[0] = '\0';
  return KDA_OK;
}

kda_status cuda_fail(cudaError_t e, const char* what) {
  return fail(KDA_ERR_CUDA, "%s: %s (%s)", what, cudaGetErrorName(e), cudaGetErrorString(e));
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

size_t elem_size(kda_dtype dt) { return dt == KDA_DT_F32 ? 4 : 2; }

bool ranges_overlap(const void* a, size_t na, const void* b, size_t nb) {
  if (!a || !b || na == 0 || nb == 0) return false;
  const uintptr_t a0 = reinterpret_cast<uintptr_t>(a), b0 = reinterpret_cast<uintptr_t>(b);
  return a0 < b0 + nb && b0 < a0 + na;
}

// Staging buffers of kda_chunk_fwd when a head dim is below 128 (zero padding in
// the input dtype; element size es).
struct StageLayout {
  size_t q, k, v, la, h0, out, ht, total;
};

StageLayout stage_layout(int64_t total_T, int N, int H, size_t es) {
  StageLayout L{};
  const size_t tok = static_cast<size_t>(total_T) * H * kda::kD;
  const size_t st = static_cast<size_t>(N) * H * kda::kD * kda::kD * sizeof(float);
  size_t off = kda::kStatusBytes;
  L.q = off;   off = kda::align256(off + tok * es);
  L.k = off;   off = kda::align256(off + tok * es);
  L.v = off;   off = kda::align256(off + tok * es);
  L.la = off;  off = kda::align256(off + tok * 4);
  L.h0 = off;  off = kda::align256(off + st);
  L.out = off; off = kda::align256(off + tok * es);
  L.ht = off;  off = kda::align256(off + st);
  L.total = off;
  return L;
}

bool needs_staging(int dk, int dv) { return dk != kda::kD || dv != kda::kD; }

kda_status check_common(int64_t total_T, int N, int H, int dk, int dv) {
  if (total_T < 0 || total_T > (int64_t{1} << 31) - 1024)
    return fail(KDA_ERR_INVALID_ARG, "total_T=%lld out of range [0, 2^31-1024]", static_cast<long long>(total_T));
  if (N < 0) return fail(KDA_ERR_INVALID_ARG, "N=%d must be >= 0", N);
  if (H < 1 || H > 65535) return fail(KDA_ERR_INVALID_ARG, "H=%d must be in [1, 65535]", H);
  if (dk < 1 || dk > KDA_MAX_HEAD_DIM || dv < 1 || dv > KDA_MAX_HEAD_DIM)
    return fail(KDA_ERR_INVALID_ARG, "dk=%d, dv=%d must be in [1, %d]", dk, dv, KDA_MAX_HEAD_DIM);
  return KDA_OK;
}

}  // namespace

namespace kda {
void set_last_error(const char* msg) { snprintf(g_last_error, sizeof(g_last_error), "%s", msg); }

kda_status mixer_fwd_staged(const void* q_raw, const void* k_raw, const void* v_raw, const float* conv_w,
                            const float* log_alpha, const float* beta, const void* gate, const float* initial_state,
                            const int32_t* cu_seqlens, int64_t total_T, int N, int H, void* out, float* final_state,
                            void* scratch, cudaStream_t stream);
}  // namespace kda

extern "C" {

const char* kda_status_string(kda_status s) {
  switch (s) {
    case KDA_OK: return "KDA_OK";
    case KDA_ERR_INVALID_ARG: return "KDA_ERR_INVALID_ARG";
    case KDA_ERR_UNSUPPORTED: return "KDA_ERR_UNSUPPORTED";
    case KDA_ERR_WORKSPACE: return "KDA_ERR_WORKSPACE";
    case KDA_ERR_CUDA: return "KDA_ERR_CUDA";
    case KDA_ERR_RANGE: return "KDA_ERR_RANGE";
  }
  return "KDA_ERR_UNKNOWN";
}

const char* kda_last_error(void) { return g_last_error; }

const char* kda_version(void) { return "0.1.0"; }

size_t kda_chunk_fwd_workspace(int64_t total_T, int N, int H, int dk, int dv, kda_dtype qkv_dtype) {
  if (check_common(total_T, N, H, dk, dv) != KDA_OK) return 0;
  if (qkv_dtype != KDA_DT_F32 && qkv_dtype != KDA_DT_BF16) return 0;
  const size_t base = needs_staging(dk, dv) ? stage_layout(total_T, N, H, elem_size(qkv_dtype)).total
                                           : kda::kStatusBytes;
  return base + kda::split_workspace_bytes(total_T, N, H);
}

kda_status kda_chunk_fwd(const void* q, const void* k, const void* v, kda_dtype qkv_dtype, const float* log_alpha,
                         const float* beta, const float* initial_state, const int32_t* cu_seqlens, int64_t total_T,
                         int N, int H, int dk, int dv, void* out, float* final_state, void* workspace,
                         size_t workspace_bytes, kda_stream_t stream_) {
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  kda_status st = check_common(total_T, N, H, dk, dv);
  if (st != KDA_OK) return st;
  if (qkv_dtype != KDA_DT_F32 && qkv_dtype != KDA_DT_BF16)
    return fail(KDA_ERR_INVALID_ARG, "qkv_dtype=%d is neither KDA_DT_F32 nor KDA_DT_BF16", static_cast<int>(qkv_dtype));
  if (N == 0) {
    if (total_T != 0) return fail(KDA_ERR_INVALID_ARG, "N=0 with total_T=%lld", static_cast<long long>(total_T));
    return ok();
  }
  if (!cu_seqlens && total_T % N != 0)
    return fail(KDA_ERR_INVALID_ARG, "cu_seqlens is NULL but total_T=%lld is not a multiple of N=%d",
                static_cast<long long>(total_T), N);
  if (total_T > 0 && (!q || !k || !v || !log_alpha || !beta || !out))
    return fail(KDA_ERR_INVALID_ARG, "q, k, v, log_alpha, beta and out must be non-NULL");
  const void* ptrs[] = {q, k, v, log_alpha, beta, initial_state, out, final_state, workspace};
  const char* names[] = {"q", "k", "v", "log_alpha", "beta", "initial_state", "out", "final_state", "workspace"};
  for (int i = 0; i < 9; ++i)
    if (ptrs[i] && !aligned16(ptrs[i])) return fail(KDA_ERR_INVALID_ARG, "%s is not 16-byte aligned", names[i]);
  if (cu_seqlens && (reinterpret_cast<uintptr_t>(cu_seqlens) & 3u))
    return fail(KDA_ERR_INVALID_ARG, "cu_seqlens is not 4-byte aligned");
  const size_t es = elem_size(qkv_dtype);
  const size_t n_out = static_cast<size_t>(total_T) * H * dv * es;
  const size_t n_st = static_cast<size_t>(N) * H * dk * dv * sizeof(float);
  if (final_state && initial_state && final_state != initial_state &&
      ranges_overlap(final_state, n_st, initial_state, n_st))
    return fail(KDA_ERR_INVALID_ARG, "final_state partially overlaps initial_state");
  if (ranges_overlap(out, n_out, q, static_cast<size_t>(total_T) * H * dk * es) ||
      ranges_overlap(out, n_out, k, static_cast<size_t>(total_T) * H * dk * es) ||
      ranges_overlap(out, n_out, v, static_cast<size_t>(total_T) * H * dv * es) ||
      ranges_overlap(out, n_out, final_state, n_st) || ranges_overlap(out, n_out, initial_state, n_st))
    return fail(KDA_ERR_INVALID_ARG, "out overlaps an input or a state buffer");
  const size_t need = kda_chunk_fwd_workspace(total_T, N, H, dk, dv, qkv_dtype);
  if (!workspace || workspace_bytes < need)
    return fail(KDA_ERR_WORKSPACE, "workspace of %zu bytes given, %zu needed", workspace ? workspace_bytes : 0, need);

  char* ws = static_cast<char*>(workspace);
  uint32_t* status = reinterpret_cast<uint32_t*>(ws);
  cudaError_t e = cudaMemsetAsync(status, 0, sizeof(uint32_t), stream);
  if (e != cudaSuccess) return cuda_fail(e, "clearing the status word");

  kda::PrefillArgs a{};
  a.beta = beta;
  a.cu = cu_seqlens;
  a.status = status;
  a.total_T = total_T;
  a.N = N;
  a.H = H;
  a.in_f32 = a.out_f32 = (qkv_dtype == KDA_DT_F32);
  if (kda::split_workspace_bytes(total_T, N, H) > 0)
    a.split_ws = ws + (needs_staging(dk, dv) ? stage_layout(total_T, N, H, es).total : kda::kStatusBytes);
  if (!needs_staging(dk, dv)) {
    a.q = q; a.k = k; a.v = v; a.log_alpha = log_alpha; a.h0 = initial_state;
    a.out = out; a.ht = final_state;
    e = kda::launch_prefill_d128(a, stream);
    if (e != cudaSuccess) return cuda_fail(e, "prefill kernel launch");
    return ok();
  }
  const StageLayout L = stage_layout(total_T, N, H, es);
  a.q = ws + L.q; a.k = ws + L.k; a.v = ws + L.v;
  a.log_alpha = reinterpret_cast<float*>(ws + L.la);
  a.h0 = initial_state ? reinterpret_cast<float*>(ws + L.h0) : nullptr;
  a.out = ws + L.out;
  a.ht = final_state ? reinterpret_cast<float*>(ws + L.ht) : nullptr;
  e = kda::launch_stage_in(q, k, v, qkv_dtype == KDA_DT_BF16, log_alpha, initial_state, total_T, N, H, dk, dv,
                           ws + L.q, ws + L.k, ws + L.v, reinterpret_cast<float*>(ws + L.la),
                           initial_state ? reinterpret_cast<float*>(ws + L.h0) : nullptr, stream);
  if (e != cudaSuccess) return cuda_fail(e, "staging kernel launch");
  e = kda::launch_prefill_d128(a, stream);
  if (e != cudaSuccess) return cuda_fail(e, "prefill kernel launch");
  e = kda::launch_stage_out(ws + L.out, a.ht, qkv_dtype == KDA_DT_BF16, total_T, N, H, dk, dv, out, final_state,
                            stream);
  if (e != cudaSuccess) return cuda_fail(e, "unstaging kernel launch");
  return ok();
}

kda_status kda_decode_step(const void* q, const void* k, const void* v, kda_dtype qkv_dtype, const float* log_alpha,
                           const float* beta, float* state, int N, int H, int dk, int dv, void* out,
                           kda_stream_t stream_) {
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  kda_status st = check_common(0, N, H, dk, dv);
  if (st != KDA_OK) return st;
  if (qkv_dtype != KDA_DT_F32 && qkv_dtype != KDA_DT_BF16)
    return fail(KDA_ERR_INVALID_ARG, "qkv_dtype=%d is neither KDA_DT_F32 nor KDA_DT_BF16", static_cast<int>(qkv_dtype));
  if (dv % 4 != 0) return fail(KDA_ERR_UNSUPPORTED, "decode needs dv %% 4 == 0 (dv=%d)", dv);
  if (N == 0) return ok();
  if (!q || !k || !v || !log_alpha || !beta || !state || !out)
    return fail(KDA_ERR_INVALID_ARG, "all pointers must be non-NULL");
  if (!aligned16(state) || !aligned16(out)) return fail(KDA_ERR_INVALID_ARG, "state and out must be 16-byte aligned");
  const void* small[] = {q, k, v, log_alpha, beta};
  for (const void* p : small)
    if (reinterpret_cast<uintptr_t>(p) & 3u) return fail(KDA_ERR_INVALID_ARG, "q/k/v/log_alpha/beta must be 4-byte aligned");
  const size_t n_st = static_cast<size_t>(N) * H * dk * dv * sizeof(float);
  const size_t n_out = static_cast<size_t>(N) * H * dv * elem_size(qkv_dtype);
  if (ranges_overlap(out, n_out, state, n_st)) return fail(KDA_ERR_INVALID_ARG, "out overlaps state");
  cudaError_t e = kda::launch_decode_step(q, k, v, qkv_dtype == KDA_DT_BF16, log_alpha, beta, state, N, H, dk, dv,
                                          out, stream);
  if (e != cudaSuccess) return cuda_fail(e, "decode kernel launch");
  return ok();
}

}  // extern "C"
namespace {
// Checks shared by the serving mixer decode entry points (K tokens per sequence).
kda_status check_mixer_decode(const void* q_raw, const void* k_raw, const void* v_raw, const float* conv_w,
                              const float* log_alpha, const float* beta, const void* gate, const float* state_pool,
                              const void* conv_pool, const int32_t* state_indices, int pool_size, int N, int K, int H,
                              int dk, int dv, const void* out, const void* status) {
  kda_status st = check_common(0, N, H, dk, dv);
  if (st != KDA_OK) return st;
  if (dk != kda::kD || dv != kda::kD)
    return fail(KDA_ERR_UNSUPPORTED, "the mixer decode is built for dk = dv = 128 (got %d, %d)", dk, dv);
  if (K < 0) return fail(KDA_ERR_INVALID_ARG, "K=%d must be >= 0", K);
  if (pool_size < 1) return fail(KDA_ERR_INVALID_ARG, "pool_size=%d must be >= 1", pool_size);
  if (!state_indices && N > pool_size)
    return fail(KDA_ERR_INVALID_ARG, "state_indices is NULL but N=%d exceeds pool_size=%d", N, pool_size);
  const void* ptrs[] = {q_raw, k_raw, v_raw, conv_w, log_alpha, beta, state_pool, conv_pool, out};
  const char* names[] = {"q_raw", "k_raw", "v_raw", "conv_w", "log_alpha", "beta", "state_pool", "conv_pool", "out"};
  for (int i = 0; i < 9; ++i) {
    if (!ptrs[i]) return fail(KDA_ERR_INVALID_ARG, "%s must be non-NULL", names[i]);
    if (!aligned16(ptrs[i])) return fail(KDA_ERR_INVALID_ARG, "%s is not 16-byte aligned", names[i]);
  }
  if (gate && !aligned16(gate)) return fail(KDA_ERR_INVALID_ARG, "gate is not 16-byte aligned");
  if (status && (reinterpret_cast<uintptr_t>(status) & 3u)) return fail(KDA_ERR_INVALID_ARG, "status is not 4-byte aligned");
  if (state_indices && (reinterpret_cast<uintptr_t>(state_indices) & 3u))
    return fail(KDA_ERR_INVALID_ARG, "state_indices is not 4-byte aligned");
  const size_t n_out = static_cast<size_t>(N) * K * H * dv * 2;
  const size_t n_state = static_cast<size_t>(pool_size) * H * dk * dv * sizeof(float);
  const size_t n_conv = static_cast<size_t>(pool_size) * H * 9 * dk * 2;
  if (ranges_overlap(out, n_out, state_pool, n_state) || ranges_overlap(out, n_out, conv_pool, n_conv) ||
      ranges_overlap(state_pool, n_state, conv_pool, n_conv))
    return fail(KDA_ERR_INVALID_ARG, "out, state_pool and conv_pool must not overlap");
  return KDA_OK;
}
}  // namespace
extern "C" {
kda_status kda_mixer_decode_step(const void* q_raw, const void* k_raw, const void* v_raw, const float* conv_w,
                                 const float* log_alpha, const float* beta, const void* gate, float* state_pool,
                                 void* conv_pool, const int32_t* state_indices, int pool_size, int N, int H, int dk,
                                 int dv, void* out, void* status, kda_stream_t stream_) {
  kda_status st = check_mixer_decode(q_raw, k_raw, v_raw, conv_w, log_alpha, beta, gate, state_pool, conv_pool,
                                     state_indices, pool_size, N, 1, H, dk, dv, out, status);
  if (st != KDA_OK || N == 0) return st == KDA_OK ? ok() : st;
  cudaError_t e = kda::launch_mixer_decode(q_raw, k_raw, v_raw, conv_w, log_alpha, beta, gate, state_pool, conv_pool,
                                           state_indices, pool_size, N, 1, H, out, nullptr, nullptr,
                                           static_cast<uint32_t*>(status), reinterpret_cast<cudaStream_t>(stream_));
  if (e != cudaSuccess) return cuda_fail(e, "mixer decode kernel launch");
  return ok();
}
kda_status kda_mixer_decode_tokens(const void* q_raw, const void* k_raw, const void* v_raw, const float* conv_w,
                                   const float* log_alpha, const float* beta, const void* gate, float* state_pool,
                                   void* conv_pool, const int32_t* state_indices, int pool_size, int N, int K, int H,
                                   int dk, int dv, void* out, float* state_ckpt, void* conv_ckpt, void* status,
                                   kda_stream_t stream_) {
  kda_status st = check_mixer_decode(q_raw, k_raw, v_raw, conv_w, log_alpha, beta, gate, state_pool, conv_pool,
                                     state_indices, pool_size, N, K, H, dk, dv, out, status);
  if (st != KDA_OK) return st;
  if ((state_ckpt == nullptr) != (conv_ckpt == nullptr))
    return fail(KDA_ERR_INVALID_ARG, "state_ckpt and conv_ckpt must both be given or both be NULL");
  if (state_ckpt && (!aligned16(state_ckpt) || !aligned16(conv_ckpt)))
    return fail(KDA_ERR_INVALID_ARG, "state_ckpt and conv_ckpt must be 16-byte aligned");
  if (N == 0 || K == 0) return ok();
  cudaError_t e = kda::launch_mixer_decode(q_raw, k_raw, v_raw, conv_w, log_alpha, beta, gate, state_pool, conv_pool,
                                           state_indices, pool_size, N, K, H, out, state_ckpt, conv_ckpt,
                                           static_cast<uint32_t*>(status), reinterpret_cast<cudaStream_t>(stream_));
  if (e != cudaSuccess) return cuda_fail(e, "mixer decode kernel launch");
  return ok();
}
kda_status kda_mixer_decode_commit(const float* state_ckpt, const void* conv_ckpt, const int32_t* accepted,
                                   float* state_pool, void* conv_pool, const int32_t* state_indices, int pool_size,
                                   int N, int K, int H, int d, void* status, kda_stream_t stream_) {
  kda_status st = check_common(0, N, H, d, d);
  if (st != KDA_OK) return st;
  if (d != kda::kD) return fail(KDA_ERR_UNSUPPORTED, "the mixer decode is built for d = 128 (got %d)", d);
  if (K < 1 || pool_size < 1) return fail(KDA_ERR_INVALID_ARG, "K=%d and pool_size=%d must be >= 1", K, pool_size);
  if (!state_indices && N > pool_size)
    return fail(KDA_ERR_INVALID_ARG, "state_indices is NULL but N=%d exceeds pool_size=%d", N, pool_size);
  const void* ptrs[] = {state_ckpt, conv_ckpt, accepted, state_pool, conv_pool};
  const char* names[] = {"state_ckpt", "conv_ckpt", "accepted", "state_pool", "conv_pool"};
  for (int i = 0; i < 5; ++i)
    if (!ptrs[i]) return fail(KDA_ERR_INVALID_ARG, "%s must be non-NULL", names[i]);
  if (!aligned16(state_ckpt) || !aligned16(conv_ckpt) || !aligned16(state_pool) || !aligned16(conv_pool))
    return fail(KDA_ERR_INVALID_ARG, "checkpoints and pools must be 16-byte aligned");
  if ((reinterpret_cast<uintptr_t>(accepted) & 3u) || (state_indices && (reinterpret_cast<uintptr_t>(state_indices) & 3u)))
    return fail(KDA_ERR_INVALID_ARG, "accepted and state_indices must be 4-byte aligned");
  if (N == 0) return ok();
  cudaError_t e = kda::launch_mixer_decode_commit(state_ckpt, conv_ckpt, accepted, state_pool, conv_pool,
                                                  state_indices, pool_size, N, K, H, static_cast<uint32_t*>(status),
                                                  reinterpret_cast<cudaStream_t>(stream_));
  if (e != cudaSuccess) return cuda_fail(e, "mixer decode commit kernel launch");
  return ok();
}
kda_status kda_state_affine(const float* M, const float* S, const float* B, float* out, int64_t count, int d,
                            kda_stream_t stream_) {
  if (count < 0) return fail(KDA_ERR_INVALID_ARG, "count=%lld must be >= 0", static_cast<long long>(count));
  if (d != kda::kD) return fail(KDA_ERR_UNSUPPORTED, "kda_state_affine is built for d = 128 (got %d)", d);
  if (count > (int64_t{1} << 31) - 1) return fail(KDA_ERR_INVALID_ARG, "count too large");
  if (count == 0) return ok();
  if (!M || !out) return fail(KDA_ERR_INVALID_ARG, "M and out must be non-NULL");
  const void* ptrs[] = {M, S, B, out};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return fail(KDA_ERR_INVALID_ARG, "M, S, B and out must be 16-byte aligned");
  const size_t n = static_cast<size_t>(count) * d * d * sizeof(float);
  if (ranges_overlap(out, n, M, n) || ranges_overlap(out, n, S, n))
    return fail(KDA_ERR_INVALID_ARG, "out must not overlap M or S");
  if (B && B != out && ranges_overlap(out, n, B, n)) return fail(KDA_ERR_INVALID_ARG, "out partially overlaps B");
  cudaError_t e = kda::launch_state_affine(M, S, B, out, count, reinterpret_cast<cudaStream_t>(stream_));
  if (e != cudaSuccess) return cuda_fail(e, "state affine kernel launch");
  return ok();
}
kda_status kda_state_fold(const float* MB, int maps, const float* S0, float* out, int64_t count, int d,
                          kda_stream_t stream_) {
  if (count < 0 || maps < 0) return fail(KDA_ERR_INVALID_ARG, "count=%lld and maps=%d must be >= 0",
                                         static_cast<long long>(count), maps);
  if (d != kda::kD) return fail(KDA_ERR_UNSUPPORTED, "kda_state_fold is built for d = 128 (got %d)", d);
  if (count > (int64_t{1} << 31) - 1) return fail(KDA_ERR_INVALID_ARG, "count too large");
  if (count == 0) return ok();
  if (!out || (maps > 0 && !MB)) return fail(KDA_ERR_INVALID_ARG, "MB and out must be non-NULL");
  const void* ptrs[] = {MB, S0, out};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return fail(KDA_ERR_INVALID_ARG, "MB, S0 and out must be 16-byte aligned");
  const size_t n = static_cast<size_t>(count) * d * d * sizeof(float);
  if (maps > 0 && ranges_overlap(out, n, MB, 2 * static_cast<size_t>(maps) * n))
    return fail(KDA_ERR_INVALID_ARG, "out must not overlap the maps");
  if (S0 && S0 != out && ranges_overlap(out, n, S0, n)) return fail(KDA_ERR_INVALID_ARG, "out partially overlaps S0");
  cudaError_t e = kda::launch_state_fold(MB, maps, S0, out, count, reinterpret_cast<cudaStream_t>(stream_));
  if (e != cudaSuccess) return cuda_fail(e, "state fold kernel launch");
  return ok();
}
size_t kda_mixer_fwd_workspace(int64_t total_T, int N, int H, int dk, int dv) {
  if (check_common(total_T, N, H, dk, dv) != KDA_OK) return 0;
  if (dk != kda::kD || dv != kda::kD) return 0;
  // status word + the two-pass prefill's scratch (the conv/L2 stage runs inside it)
  return kda::kStatusBytes + kda::split_workspace_bytes(total_T, N, H);
}

namespace {

// Checks shared by the fused and the two-stage mixer entry points.
kda_status check_mixer(const void* q_raw, const void* k_raw, const void* v_raw, const float* conv_w,
                       const float* log_alpha, const float* beta, const void* gate, const float* initial_state,
                       const int32_t* cu_seqlens, int64_t total_T, int N, int H, int dk, int dv, void* out,
                       float* final_state) {
  kda_status st = check_common(total_T, N, H, dk, dv);
  if (st != KDA_OK) return st;
  if (dk != kda::kD || dv != kda::kD)
    return fail(KDA_ERR_UNSUPPORTED, "the fused mixer is built for dk = dv = 128 (got %d, %d)", dk, dv);
  if (N == 0 && total_T != 0) return fail(KDA_ERR_INVALID_ARG, "N=0 with total_T=%lld", static_cast<long long>(total_T));
  if (N > 0 && !cu_seqlens && total_T % N != 0)
    return fail(KDA_ERR_INVALID_ARG, "cu_seqlens is NULL but total_T=%lld is not a multiple of N=%d",
                static_cast<long long>(total_T), N);
  if (total_T > 0 && (!q_raw || !k_raw || !v_raw || !conv_w || !log_alpha || !beta || !out))
    return fail(KDA_ERR_INVALID_ARG, "q_raw, k_raw, v_raw, conv_w, log_alpha, beta and out must be non-NULL");
  const void* ptrs[] = {q_raw, k_raw, v_raw, conv_w, log_alpha, beta, gate, initial_state, out, final_state};
  const char* names[] = {"q_raw", "k_raw", "v_raw", "conv_w", "log_alpha", "beta", "gate",
                         "initial_state", "out", "final_state"};
  for (int i = 0; i < 10; ++i)
    if (ptrs[i] && !aligned16(ptrs[i])) return fail(KDA_ERR_INVALID_ARG, "%s is not 16-byte aligned", names[i]);
  if (cu_seqlens && (reinterpret_cast<uintptr_t>(cu_seqlens) & 3u))
    return fail(KDA_ERR_INVALID_ARG, "cu_seqlens is not 4-byte aligned");
  const size_t n_st = static_cast<size_t>(N) * H * dk * dv * sizeof(float);
  if (final_state && initial_state && final_state != initial_state &&
      ranges_overlap(final_state, n_st, initial_state, n_st))
    return fail(KDA_ERR_INVALID_ARG, "final_state partially overlaps initial_state");
  return KDA_OK;
}

}  // namespace

kda_status kda_mixer_fwd(const void* q_raw, const void* k_raw, const void* v_raw, const float* conv_w,
                         const float* log_alpha, const float* beta, const void* gate, const float* initial_state,
                         const int32_t* cu_seqlens, int64_t total_T, int N, int H, int dk, int dv, void* out,
                         float* final_state, void* workspace, size_t workspace_bytes, kda_stream_t stream_) {
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  kda_status st = check_mixer(q_raw, k_raw, v_raw, conv_w, log_alpha, beta, gate, initial_state, cu_seqlens,
                              total_T, N, H, dk, dv, out, final_state);
  if (st != KDA_OK) return st;
  if (N == 0) return ok();
  if (workspace && !aligned16(workspace)) return fail(KDA_ERR_INVALID_ARG, "workspace is not 16-byte aligned");
  const size_t need = kda_mixer_fwd_workspace(total_T, N, H, dk, dv);
  if (!workspace || workspace_bytes < need)
    return fail(KDA_ERR_WORKSPACE, "workspace of %zu bytes given, %zu needed", workspace ? workspace_bytes : 0, need);
  uint32_t* status = static_cast<uint32_t*>(workspace);
  cudaError_t e = cudaMemsetAsync(status, 0, sizeof(uint32_t), stream);
  if (e != cudaSuccess) return cuda_fail(e, "clearing the status word");
  kda::PrefillArgs a{};
  a.q = q_raw; a.k = k_raw; a.v = v_raw; a.log_alpha = log_alpha; a.beta = beta; a.h0 = initial_state;
  a.cu = cu_seqlens; a.gate = gate; a.conv_w = conv_w; a.out = out; a.ht = final_state; a.status = status;
  a.total_T = total_T; a.N = N; a.H = H;
  a.in_f32 = false;  // raw bf16 q, k, v
  a.out_f32 = false;
  if (kda::split_workspace_bytes(total_T, N, H) > 0) a.split_ws = static_cast<char*>(workspace) + kda::kStatusBytes;
  e = kda::launch_prefill_d128(a, stream);
  if (e != cudaSuccess) return cuda_fail(e, "prefill kernel launch");
  return ok();
}

kda_status kda_mixer_fwd_pooled(const void* q_raw, const void* k_raw, const void* v_raw, const float* conv_w,
                                const float* log_alpha, const float* beta, const void* gate,
                                const float* initial_state, const int32_t* cu_seqlens, int64_t total_T, int N, int H,
                                int dk, int dv, void* out, float* state_pool, void* conv_pool,
                                const int32_t* state_indices, int pool_size, void* workspace, size_t workspace_bytes,
                                kda_stream_t stream_) {
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  kda_status st = check_mixer(q_raw, k_raw, v_raw, conv_w, log_alpha, beta, gate, initial_state, cu_seqlens,
                              total_T, N, H, dk, dv, out, nullptr);
  if (st != KDA_OK) return st;
  if (pool_size < 1) return fail(KDA_ERR_INVALID_ARG, "pool_size=%d must be >= 1", pool_size);
  if (!state_indices && N > pool_size)
    return fail(KDA_ERR_INVALID_ARG, "state_indices is NULL but N=%d exceeds pool_size=%d", N, pool_size);
  if (!state_pool || !conv_pool) return fail(KDA_ERR_INVALID_ARG, "state_pool and conv_pool must be non-NULL");
  if (!aligned16(state_pool) || !aligned16(conv_pool))
    return fail(KDA_ERR_INVALID_ARG, "state_pool and conv_pool must be 16-byte aligned");
  if (state_indices && (reinterpret_cast<uintptr_t>(state_indices) & 3u))
    return fail(KDA_ERR_INVALID_ARG, "state_indices is not 4-byte aligned");
  const size_t n_state = static_cast<size_t>(pool_size) * H * dk * dv * sizeof(float);
  const size_t n_conv = static_cast<size_t>(pool_size) * H * 9 * dk * 2;
  const size_t n_out = static_cast<size_t>(total_T) * H * dv * 2;
  const size_t n_h0 = static_cast<size_t>(N) * H * dk * dv * sizeof(float);
  if (ranges_overlap(state_pool, n_state, conv_pool, n_conv) || ranges_overlap(out, n_out, state_pool, n_state) ||
      ranges_overlap(out, n_out, conv_pool, n_conv) ||
      (initial_state && ranges_overlap(initial_state, n_h0, state_pool, n_state)))
    return fail(KDA_ERR_INVALID_ARG, "out, initial_state, state_pool and conv_pool must not overlap");
  if (N == 0) return ok();
  if (workspace && !aligned16(workspace)) return fail(KDA_ERR_INVALID_ARG, "workspace is not 16-byte aligned");
  const size_t need = kda_mixer_fwd_workspace(total_T, N, H, dk, dv);
  if (!workspace || workspace_bytes < need)
    return fail(KDA_ERR_WORKSPACE, "workspace of %zu bytes given, %zu needed", workspace ? workspace_bytes : 0, need);
  uint32_t* status = static_cast<uint32_t*>(workspace);
  cudaError_t e = cudaMemsetAsync(status, 0, sizeof(uint32_t), stream);
  if (e != cudaSuccess) return cuda_fail(e, "clearing the status word");
  kda::PrefillArgs a{};
  a.q = q_raw; a.k = k_raw; a.v = v_raw; a.log_alpha = log_alpha; a.beta = beta; a.h0 = initial_state;
  a.cu = cu_seqlens; a.gate = gate; a.conv_w = conv_w; a.out = out; a.ht = state_pool; a.status = status;
  a.total_T = total_T; a.N = N; a.H = H;
  a.slots = state_indices;  // NULL: slot n, and the pool holds at least N states
  a.pool_size = pool_size;
  a.in_f32 = false;
  a.out_f32 = false;
  if (kda::split_workspace_bytes(total_T, N, H) > 0) a.split_ws = static_cast<char*>(workspace) + kda::kStatusBytes;
  if (total_T > 0) {
    e = kda::launch_prefill_d128(a, stream);
    if (e != cudaSuccess) return cuda_fail(e, "prefill kernel launch");
  }
  e = kda::launch_pool_store(q_raw, k_raw, v_raw, cu_seqlens, total_T, N, H, state_indices, pool_size, conv_pool,
                             total_T == 0, initial_state, state_pool, status, stream);
  if (e != cudaSuccess) return cuda_fail(e, "pool store kernel launch");
  return ok();
}

size_t kda_mixer_fwd_gate_workspace(int64_t total_T, int N, int H, int dk, int dv) {
  if (check_common(total_T, N, H, dk, dv) != KDA_OK) return 0;
  if (dk != kda::kD || dv != kda::kD) return 0;
  if (total_T == 0 || N == 0) return kda::kStatusBytes;
  const size_t split = kda::split_workspace_bytes(total_T, N, H, /*any_chains=*/true);
  return split ? kda::kStatusBytes + split : 0;
}
kda_status kda_mixer_fwd_gate(const void* q_raw, const void* k_raw, const void* v_raw, const float* conv_w,
                              const void* a_pre, const float* a_scale, const float* beta, const void* gate,
                              const float* initial_state, const int32_t* cu_seqlens, int64_t total_T, int N, int H,
                              int dk, int dv, void* out, float* final_state, void* workspace, size_t workspace_bytes,
                              kda_stream_t stream_) {
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  // a_pre stands where log_alpha stands in the shared checks (same shape, 16-byte aligned)
  kda_status st = check_mixer(q_raw, k_raw, v_raw, conv_w, static_cast<const float*>(a_pre), beta, gate,
                              initial_state, cu_seqlens, total_T, N, H, dk, dv, out, final_state);
  if (st != KDA_OK) return st;
  if (total_T > 0 && !a_scale) return fail(KDA_ERR_INVALID_ARG, "a_scale must be non-NULL");
  if (a_scale && (reinterpret_cast<uintptr_t>(a_scale) & 3u)) return fail(KDA_ERR_INVALID_ARG, "a_scale is not 4-byte aligned");
  if (N == 0) return ok();
  if (workspace && !aligned16(workspace)) return fail(KDA_ERR_INVALID_ARG, "workspace is not 16-byte aligned");
  const size_t need = kda_mixer_fwd_gate_workspace(total_T, N, H, dk, dv);
  if (need == 0) return fail(KDA_ERR_UNSUPPORTED, "the two-pass scratch for these sizes exceeds the supported 32 GiB");
  if (!workspace || workspace_bytes < need)
    return fail(KDA_ERR_WORKSPACE, "workspace of %zu bytes given, %zu needed", workspace ? workspace_bytes : 0, need);
  uint32_t* status = static_cast<uint32_t*>(workspace);
  cudaError_t e = cudaMemsetAsync(status, 0, sizeof(uint32_t), stream);
  if (e != cudaSuccess) return cuda_fail(e, "clearing the status word");
  kda::PrefillArgs a{};
  a.q = q_raw; a.k = k_raw; a.v = v_raw; a.log_alpha = nullptr; a.beta = beta; a.h0 = initial_state;
  a.cu = cu_seqlens; a.gate = gate; a.conv_w = conv_w; a.out = out; a.ht = final_state; a.status = status;
  a.total_T = total_T; a.N = N; a.H = H;
  a.in_f32 = false;
  a.out_f32 = false;
  a.a_pre = a_pre;
  a.a_scale = a_scale;
  if (total_T > 0) a.split_ws = static_cast<char*>(workspace) + kda::kStatusBytes;
  e = kda::launch_prefill_d128(a, stream);
  if (e != cudaSuccess) return cuda_fail(e, "prefill kernel launch");
  return ok();
}
size_t kda_chunk_bwd_workspace(int64_t total_T, int N, int H, int dk, int dv) {
  if (check_common(total_T, N, H, dk, dv) != KDA_OK) return 0;
  if (dk != kda::kD || dv != kda::kD) return 0;
  return kda::kStatusBytes + kda::bwd_workspace_bytes(total_T, N, H);
}

kda_status kda_chunk_bwd(const void* q, const void* k, const void* v, kda_dtype qkv_dtype, const float* log_alpha,
                         const float* beta, const float* initial_state, const int32_t* cu_seqlens, int64_t total_T,
                         int N, int H, int dk, int dv, const void* d_out, const float* d_final_state, float* dq,
                         float* dk_out, float* dv_out, float* d_log_alpha, float* d_beta, float* d_initial_state,
                         void* workspace, size_t workspace_bytes, kda_stream_t stream_) {
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  kda_status st = check_common(total_T, N, H, dk, dv);
  if (st != KDA_OK) return st;
  if (dk != kda::kD || dv != kda::kD) return fail(KDA_ERR_UNSUPPORTED, "the backward needs dk == dv == 128");
  if (qkv_dtype != KDA_DT_F32 && qkv_dtype != KDA_DT_BF16)
    return fail(KDA_ERR_INVALID_ARG, "qkv_dtype=%d is neither KDA_DT_F32 nor KDA_DT_BF16", static_cast<int>(qkv_dtype));
  if (N == 0) {
    if (total_T != 0) return fail(KDA_ERR_INVALID_ARG, "N=0 with total_T=%lld", static_cast<long long>(total_T));
    return ok();
  }
  if (!cu_seqlens && total_T % N != 0)
    return fail(KDA_ERR_INVALID_ARG, "cu_seqlens is NULL but total_T=%lld is not a multiple of N=%d",
                static_cast<long long>(total_T), N);
  if (total_T > 0 && (!q || !k || !v || !log_alpha || !beta || !d_out || !dq || !dk_out || !dv_out ||
                      !d_log_alpha || !d_beta))
    return fail(KDA_ERR_INVALID_ARG, "inputs, d_out and the token gradients must be non-NULL");
  const void* ptrs[] = {q, k, v, log_alpha, initial_state, d_out, d_final_state, dq, dk_out, dv_out,
                        d_log_alpha, d_initial_state, workspace};
  const char* names[] = {"q", "k", "v", "log_alpha", "initial_state", "d_out", "d_final_state", "dq", "dk",
                         "dv", "d_log_alpha", "d_initial_state", "workspace"};
  for (int i = 0; i < 13; ++i)
    if (ptrs[i] && !aligned16(ptrs[i])) return fail(KDA_ERR_INVALID_ARG, "%s is not 16-byte aligned", names[i]);
  if ((beta && (reinterpret_cast<uintptr_t>(beta) & 3u)) || (d_beta && (reinterpret_cast<uintptr_t>(d_beta) & 3u)))
    return fail(KDA_ERR_INVALID_ARG, "beta and d_beta must be 4-byte aligned");
  if (cu_seqlens && (reinterpret_cast<uintptr_t>(cu_seqlens) & 3u))
    return fail(KDA_ERR_INVALID_ARG, "cu_seqlens is not 4-byte aligned");
  {  // the gradients are written while the inputs are read: no output may overlap any
     // input or another output
    const size_t es = elem_size(qkv_dtype);
    const size_t tok = static_cast<size_t>(total_T) * H * kda::kD;
    const size_t n_st = static_cast<size_t>(N) * H * kda::kD * kda::kD * sizeof(float);
    const size_t n_tb = static_cast<size_t>(total_T) * H * sizeof(float);
    const void* in[] = {q, k, v, d_out, log_alpha, beta, initial_state, d_final_state, cu_seqlens};
    const size_t in_n[] = {tok * es, tok * es, tok * es, tok * es, tok * 4, n_tb, n_st, n_st,
                           (static_cast<size_t>(N) + 1) * sizeof(int32_t)};
    const void* outp[] = {dq, dk_out, dv_out, d_log_alpha, d_beta, d_initial_state};
    const size_t out_n[] = {tok * 4, tok * 4, tok * 4, tok * 4, n_tb, n_st};
    const char* out_names[] = {"dq", "dk", "dv", "d_log_alpha", "d_beta", "d_initial_state"};
    for (int i = 0; i < 6; ++i) {
      for (int j = 0; j < 9; ++j)
        if (ranges_overlap(outp[i], out_n[i], in[j], in_n[j]))
          return fail(KDA_ERR_INVALID_ARG, "%s overlaps an input", out_names[i]);
      for (int j = i + 1; j < 6; ++j)
        if (ranges_overlap(outp[i], out_n[i], outp[j], out_n[j]))
          return fail(KDA_ERR_INVALID_ARG, "%s overlaps %s", out_names[i], out_names[j]);
    }
  }
  const size_t need = kda_chunk_bwd_workspace(total_T, N, H, dk, dv);
  if (!workspace || workspace_bytes < need)
    return fail(KDA_ERR_WORKSPACE, "workspace of %zu bytes given, %zu needed", workspace ? workspace_bytes : 0, need);
  uint32_t* status = static_cast<uint32_t*>(workspace);
  cudaError_t e = cudaMemsetAsync(status, 0, sizeof(uint32_t), stream);
  if (e != cudaSuccess) return cuda_fail(e, "clearing the status word");
  e = kda::launch_backward(q, k, v, qkv_dtype == KDA_DT_BF16, log_alpha, beta, initial_state, cu_seqlens, total_T, N,
                           H, d_out, d_final_state, dq, dk_out, dv_out, d_log_alpha, d_beta, d_initial_state,
                           static_cast<char*>(workspace) + kda::kStatusBytes, status, stream);
  if (e != cudaSuccess) return cuda_fail(e, "backward kernel launch");
  return ok();
}

kda_status kda_workspace_status(void* workspace, kda_stream_t stream_, uint32_t* flags) {
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  if (!workspace) return fail(KDA_ERR_INVALID_ARG, "workspace is NULL");
  uint32_t word = 0;
  cudaError_t e = cudaMemcpyAsync(&word, workspace, sizeof(word), cudaMemcpyDeviceToHost, stream);
  if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
  if (e == cudaSuccess) e = cudaMemsetAsync(workspace, 0, sizeof(word), stream);
  if (e != cudaSuccess) return cuda_fail(e, "reading the status word");
  if (flags) *flags = word;
  if (word) return fail(KDA_ERR_RANGE, "device status word 0x%08x", word);
  return ok();
}

}  // extern "C"

namespace {
kda_status check_segment(const void* q, const void* k, const void* v, kda_dtype dt, const float* log_alpha,
                         const float* beta, const int32_t* cu_seqlens, int64_t total_T, int N, int H, int dk, int dv) {
  kda_status st = check_common(total_T, N, H, dk, dv);
  if (st != KDA_OK) return st;
  if (dk != kda::kD || dv != kda::kD)
    return fail(KDA_ERR_UNSUPPORTED, "the segment calls are built for dk = dv = 128 (got %d, %d)", dk, dv);
  if (dt != KDA_DT_F32 && dt != KDA_DT_BF16)
    return fail(KDA_ERR_INVALID_ARG, "qkv_dtype=%d is neither KDA_DT_F32 nor KDA_DT_BF16", static_cast<int>(dt));
  if (N < 1 || total_T < 1) return fail(KDA_ERR_INVALID_ARG, "a segment needs N >= 1 and total_T >= 1");
  if (!cu_seqlens && total_T % N != 0)
    return fail(KDA_ERR_INVALID_ARG, "cu_seqlens is NULL but total_T=%lld is not a multiple of N=%d",
                static_cast<long long>(total_T), N);
  if (cu_seqlens && (reinterpret_cast<uintptr_t>(cu_seqlens) & 3u))
    return fail(KDA_ERR_INVALID_ARG, "cu_seqlens is not 4-byte aligned");
  const void* ptrs[] = {q, k, v, log_alpha, beta};
  const char* names[] = {"q", "k", "v", "log_alpha", "beta"};
  for (int i = 0; i < 5; ++i) {
    if (!ptrs[i]) return fail(KDA_ERR_INVALID_ARG, "%s must be non-NULL", names[i]);
    if (!aligned16(ptrs[i])) return fail(KDA_ERR_INVALID_ARG, "%s is not 16-byte aligned", names[i]);
  }
  return KDA_OK;
}
}  // namespace

extern "C" size_t kda_segment_maps_workspace(int64_t total_T, int N, int H, int dk, int dv) {
  if (check_common(total_T, N, H, dk, dv) != KDA_OK || dk != kda::kD || dv != kda::kD) return 0;
  const size_t s = kda::split_workspace_bytes(total_T, N, H, /*any_chains=*/true);
  return s ? kda::kStatusBytes + s : 0;
}

extern "C" kda_status kda_segment_maps(const void* q, const void* k, const void* v, kda_dtype qkv_dtype,
                                       const float* log_alpha, const float* beta, const int32_t* cu_seqlens,
                                       int64_t total_T, int N, int H, int dk, int dv, float* M, float* B,
                                       void* workspace, size_t workspace_bytes, kda_stream_t stream_) {
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  kda_status st = check_segment(q, k, v, qkv_dtype, log_alpha, beta, cu_seqlens, total_T, N, H, dk, dv);
  if (st != KDA_OK) return st;
  if (!M || !B || !aligned16(M) || !aligned16(B))
    return fail(KDA_ERR_INVALID_ARG, "M and B must be non-NULL and 16-byte aligned");
  const size_t n_st = static_cast<size_t>(N) * H * kda::kD * kda::kD * sizeof(float);
  if (ranges_overlap(M, n_st, B, n_st)) return fail(KDA_ERR_INVALID_ARG, "M and B overlap");
  const size_t need = kda_segment_maps_workspace(total_T, N, H, dk, dv);
  if (need == 0) return fail(KDA_ERR_UNSUPPORTED, "the items of this segment would pass 32 GiB");
  if (!workspace || workspace_bytes < need || !aligned16(workspace))
    return fail(KDA_ERR_WORKSPACE, "workspace of %zu bytes given, %zu needed (16-byte aligned)",
                workspace ? workspace_bytes : 0, need);
  char* ws = static_cast<char*>(workspace);
  uint32_t* status = reinterpret_cast<uint32_t*>(ws);
  cudaError_t e = cudaMemsetAsync(status, 0, sizeof(uint32_t), stream);
  if (e != cudaSuccess) return cuda_fail(e, "clearing the status word");
  kda::PrefillArgs a{};
  a.q = q; a.k = k; a.v = v; a.log_alpha = log_alpha; a.beta = beta; a.cu = cu_seqlens;
  a.status = status; a.total_T = total_T; a.N = N; a.H = H;
  a.in_f32 = a.out_f32 = (qkv_dtype == KDA_DT_F32);
  a.split_ws = ws + kda::kStatusBytes;
  a.map_M = M; a.map_B = B;
  e = kda::launch_prefill_split(a, stream);
  if (e != cudaSuccess) return cuda_fail(e, "segment map kernels launch");
  return ok();
}

extern "C" kda_status kda_segment_prefill(void* workspace, size_t workspace_bytes, kda_dtype qkv_dtype,
                                          const float* initial_state, const int32_t* cu_seqlens, int64_t total_T,
                                          int N, int H, int dk, int dv, void* out, float* final_state,
                                          kda_stream_t stream_) {
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  kda_status st = check_common(total_T, N, H, dk, dv);
  if (st != KDA_OK) return st;
  if (dk != kda::kD || dv != kda::kD)
    return fail(KDA_ERR_UNSUPPORTED, "the segment calls are built for dk = dv = 128 (got %d, %d)", dk, dv);
  if (qkv_dtype != KDA_DT_F32 && qkv_dtype != KDA_DT_BF16)
    return fail(KDA_ERR_INVALID_ARG, "qkv_dtype=%d is neither KDA_DT_F32 nor KDA_DT_BF16", static_cast<int>(qkv_dtype));
  if (N < 1 || total_T < 1) return fail(KDA_ERR_INVALID_ARG, "a segment needs N >= 1 and total_T >= 1");
  if (!out || !aligned16(out)) return fail(KDA_ERR_INVALID_ARG, "out must be non-NULL and 16-byte aligned");
  const void* opt[] = {initial_state, final_state};
  for (const void* x : opt)
    if (x && !aligned16(x)) return fail(KDA_ERR_INVALID_ARG, "initial_state and final_state must be 16-byte aligned");
  if (cu_seqlens && (reinterpret_cast<uintptr_t>(cu_seqlens) & 3u))
    return fail(KDA_ERR_INVALID_ARG, "cu_seqlens is not 4-byte aligned");
  const size_t n_st = static_cast<size_t>(N) * H * kda::kD * kda::kD * sizeof(float);
  if (final_state && initial_state && final_state != initial_state &&
      ranges_overlap(final_state, n_st, initial_state, n_st))
    return fail(KDA_ERR_INVALID_ARG, "final_state partially overlaps initial_state");
  const size_t need = kda_segment_maps_workspace(total_T, N, H, dk, dv);
  if (!workspace || workspace_bytes < need || !aligned16(workspace))
    return fail(KDA_ERR_WORKSPACE, "the workspace of the segment's kda_segment_maps call is needed (%zu bytes)", need);
  char* ws = static_cast<char*>(workspace);
  kda::PrefillArgs a{};
  a.cu = cu_seqlens; a.status = reinterpret_cast<uint32_t*>(ws); a.total_T = total_T; a.N = N; a.H = H;
  a.h0 = initial_state; a.out = out; a.ht = final_state;
  a.in_f32 = a.out_f32 = (qkv_dtype == KDA_DT_F32);
  a.split_ws = ws + kda::kStatusBytes;
  cudaError_t e = kda::launch_recur_only(a, stream);
  if (e != cudaSuccess) return cuda_fail(e, "segment prefill kernel launch");
  return ok();
}

namespace {
// One thread waits on an mbarrier that nothing arrives at, with the library's bounded
// wait: the wait runs out after budget_ns, raises the timeout bit in *status and the
// kernel returns.
__global__ void wait_timeout_probe_kernel(uint32_t* status, uint64_t budget_ns) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    kda::mbar_init(&bar, 1);
    kda::fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) kda::mbar_wait_for(&bar, 0, status, budget_ns);
  __syncthreads();
}
}  // namespace

extern "C" kda_status kda_selftest_wait_timeout(void* workspace, size_t workspace_bytes, uint32_t budget_us,
                                                kda_stream_t stream_) {
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  if (!workspace || workspace_bytes < kda::kStatusBytes)
    return fail(KDA_ERR_WORKSPACE, "a workspace of at least %zu bytes is needed", kda::kStatusBytes);
  if (!aligned16(workspace)) return fail(KDA_ERR_INVALID_ARG, "workspace is not 16-byte aligned");
  if (budget_us < 1 || budget_us > 2000000u)
    return fail(KDA_ERR_INVALID_ARG, "budget_us=%u must be in [1, 2000000]", budget_us);
  uint32_t* status = static_cast<uint32_t*>(workspace);
  cudaError_t e = cudaMemsetAsync(status, 0, sizeof(uint32_t), stream);
  if (e != cudaSuccess) return cuda_fail(e, "clearing the status word");
  wait_timeout_probe_kernel<<<1, 32, 0, stream>>>(status, static_cast<uint64_t>(budget_us) * 1000u);
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "wait probe kernel launch");
  return ok();
}

namespace kda {

// Two-stage form of the full mixer (conv4 + L2 pre-stage into fp32 buffers in
// `scratch`, then the recurrence on them). `scratch` holds
// mixer_staged_scratch_bytes(total_T, H) bytes.
kda_status mixer_fwd_staged(const void* q_raw, const void* k_raw, const void* v_raw, const float* conv_w,
                            const float* log_alpha, const float* beta, const void* gate, const float* initial_state,
                            const int32_t* cu_seqlens, int64_t total_T, int N, int H, void* out, float* final_state,
                            void* scratch, cudaStream_t stream) {
  kda_status st = check_mixer(q_raw, k_raw, v_raw, conv_w, log_alpha, beta, gate, initial_state, cu_seqlens,
                              total_T, N, H, kD, kD, out, final_state);
  if (st != KDA_OK) return st;
  if (N == 0) return ok();
  char* ws = static_cast<char*>(scratch);
  uint32_t* status = reinterpret_cast<uint32_t*>(ws);
  cudaError_t e = cudaMemsetAsync(status, 0, sizeof(uint32_t), stream);
  if (e != cudaSuccess) return cuda_fail(e, "clearing the status word");
  const size_t tok = align256(static_cast<size_t>(total_T) * H * kD * sizeof(float));
  char* qn = ws + kStatusBytes;
  char* kn = qn + tok;
  char* vn = kn + tok;
  e = launch_conv_l2(q_raw, k_raw, v_raw, conv_w, cu_seqlens, total_T, N, H, kD, qn, kn, vn, status, stream);
  if (e != cudaSuccess) return cuda_fail(e, "conv/L2 kernel launch");
  PrefillArgs a{};
  a.q = qn; a.k = kn; a.v = vn; a.log_alpha = log_alpha; a.beta = beta; a.h0 = initial_state; a.cu = cu_seqlens;
  a.gate = gate; a.out = out; a.ht = final_state; a.status = status; a.total_T = total_T; a.N = N; a.H = H;
  a.in_f32 = true;   // conv/L2 outputs stay fp32
  a.out_f32 = false;
  e = launch_prefill_d128(a, stream);
  if (e != cudaSuccess) return cuda_fail(e, "prefill kernel launch");
  return ok();
}

}  // namespace kda
