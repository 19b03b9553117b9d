// kda_noalloc.cu — kda_mixer_fwd_noalloc: the full-mixer prefill for callers that
// cannot hand the library a workspace.
//
// Some callers are not allowed to allocate device memory at the point where they
// run the mixer: a plugin inside a host framework that owns every device
// allocation through its own pool, or a latency-critical serving loop where a
// cudaMalloc (and the device-wide synchronisation it can imply) is not acceptable.
// This entry point takes only inputs and outputs. It runs the two-stage form of the
// mixer, whose scratch (the fp32 conv/L2 outputs and the device status word) lives in
// one file-scope __device__ array of fixed size that every GPU which loads the
// library keeps until the process exits.
//
// Contract:
//   * scratch capacity: total_T * H <= kNoallocMaxTokenHeads (16384 token-heads,
//     e.g. 512 tokens of the 32-head model); larger problems are rejected with
//     KDA_ERR_UNSUPPORTED before anything is launched;
//   * the first call on each device (with that device current) looks up the
//     array's device address with cudaGetSymbolAddress; make that first call
//     before any stream capture;
//   * every call on a device shares the same array and leaves its contents for the
//     next call; the status word is cleared at the start of each call. Calls that
//     overlap on the GPU (different streams, no ordering between them) race on the
//     array and give undefined results;
//   * with CUDA's lazy module loading (the default) the first call on a device is
//     also when the driver loads the library's device code and so reserves the
//     array; a call with total_T = 0 and N = 0 does that set-up and launches nothing, so it
//     can serve as a warm-up while the device still has room;
//   * the device status word (bad cu_seqlens, a wait that ran out of time) lives in
//     the array too; kda_mixer_fwd_noalloc_status reads and clears it;
//   * it allocates nothing: no cudaMalloc, cudaFree or allocating library call.
#include <cstdio>
#include <mutex>

#include "kda_internal.h"

namespace {

constexpr int64_t kNoallocMaxTokenHeads = 16384;
constexpr size_t kNoallocTensorBytes = static_cast<size_t>(kNoallocMaxTokenHeads) * kda::kD * sizeof(float);
constexpr size_t kNoallocScratchBytes = kda::kStatusBytes + 3 * kNoallocTensorBytes;  // 24 MiB + 256 B

// The scratch itself. In host code this name is only a stand-in for the symbol:
// its device address comes from cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoallocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_setup_mutex;
void* g_scratch_addr[kMaxDevices] = {};

kda_status noalloc_fail(kda_status s, const char* msg) {
  kda::set_last_error(msg);
  return s;
}

// Device address of the scratch array on the current device (looked up once).
cudaError_t scratch_on_current_device(unsigned char** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_addr[dev] = p;
  }
  *out = static_cast<unsigned char*>(g_scratch_addr[dev]);
  return cudaSuccess;
}

}  // namespace

extern "C" KDA_API kda_status kda_mixer_fwd_noalloc(const void* q_raw, const void* k_raw, const void* v_raw,
                                                    const float* conv_w, const float* log_alpha, const float* beta,
                                                    const void* gate, const float* initial_state,
                                                    const int32_t* cu_seqlens, int64_t total_T, int N, int H, int dk,
                                                    int dv, void* out, float* final_state, kda_stream_t stream_) {
  // total_T is bounded on its own first, so that total_T * H cannot overflow
  if (total_T < 0 || H < 1 || total_T > kNoallocMaxTokenHeads || total_T * H > kNoallocMaxTokenHeads) {
    char msg[256];
    snprintf(msg, sizeof(msg),
             "kda_mixer_fwd_noalloc: total_T * H = %lld exceeds the static scratch capacity of %lld token-heads "
             "(%zu bytes); use kda_mixer_fwd with a workspace",
             static_cast<long long>(total_T) * H, static_cast<long long>(kNoallocMaxTokenHeads),
             kNoallocScratchBytes);
    return noalloc_fail(total_T < 0 || H < 1 ? KDA_ERR_INVALID_ARG : KDA_ERR_UNSUPPORTED, msg);
  }
  if (dk != kda::kD || dv != kda::kD || kda_mixer_fwd_workspace(total_T, N, H, dk, dv) == 0)
    return noalloc_fail(KDA_ERR_INVALID_ARG, "kda_mixer_fwd_noalloc: sizes rejected (dk = dv = 128 required)");
  if (kda::mixer_staged_scratch_bytes(total_T, H) > kNoallocScratchBytes)
    return noalloc_fail(KDA_ERR_UNSUPPORTED, "kda_mixer_fwd_noalloc: scratch too small");
  unsigned char* scratch = nullptr;
  const cudaError_t e = scratch_on_current_device(&scratch);
  if (e != cudaSuccess) {
    char msg[256];
    snprintf(msg, sizeof(msg), "kda_mixer_fwd_noalloc: cudaGetSymbolAddress failed: %s", cudaGetErrorString(e));
    return noalloc_fail(KDA_ERR_CUDA, msg);
  }
  // The two-stage form of the mixer (conv/L2 outputs kept in fp32 in the static array,
  // then the recurrence); it computes what kda_mixer_fwd computes, within rounding.
  return kda::mixer_fwd_staged(q_raw, k_raw, v_raw, conv_w, log_alpha, beta, gate, initial_state, cu_seqlens,
                               total_T, N, H, out, final_state, scratch, reinterpret_cast<cudaStream_t>(stream_));
}

extern "C" KDA_API kda_status kda_mixer_fwd_noalloc_status(kda_stream_t stream_, uint32_t* flags) {
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  unsigned char* scratch = nullptr;
  cudaError_t e = scratch_on_current_device(&scratch);
  uint32_t word = 0;
  if (e == cudaSuccess) e = cudaMemcpyAsync(&word, scratch, sizeof(word), cudaMemcpyDeviceToHost, stream);
  if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
  if (e == cudaSuccess) e = cudaMemsetAsync(scratch, 0, sizeof(word), stream);
  if (e != cudaSuccess) {
    char msg[256];
    snprintf(msg, sizeof(msg), "kda_mixer_fwd_noalloc_status: %s", cudaGetErrorString(e));
    return noalloc_fail(KDA_ERR_CUDA, msg);
  }
  if (flags) *flags = word;
  if (word) {
    char msg[128];
    snprintf(msg, sizeof(msg), "kda_mixer_fwd_noalloc: device status word 0x%08x", word);
    return noalloc_fail(KDA_ERR_RANGE, msg);
  }
  kda::set_last_error("");
  return KDA_OK;
}
