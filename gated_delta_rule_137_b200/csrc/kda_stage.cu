// kda_stage.cu — the small memory-bound kernels around the tensor-core prefill:
//   * staging of head dims below 128 into zero-padded d = 128 buffers of the same
//     dtype, and the copy of the results back (zero padding is exact: padded key channels carry
//     log_alpha = 0 and zero q/k, padded value columns carry zero v, so padded
//     state rows/columns stay zero and the real outputs do not change);
//   * the mixer pre-stage drawn in the KDA panel of the Ling-3.0-flash article
//     (section "KDA: constant-size memory over a very long context"): a causal
//     depthwise convolution of width 4 (page "Ling 3.0 Flash", field
//     short_conv_kernel_size) on q, k and v, then an L2 norm of q and k.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "kda_internal.h"

namespace kda {

namespace {

template <typename T>
__device__ __forceinline__ T zero_of();
template <>
__device__ __forceinline__ float zero_of<float>() { return 0.f; }
template <>
__device__ __forceinline__ __nv_bfloat16 zero_of<__nv_bfloat16>() { return __float2bfloat16_rn(0.f); }

// Pads rows of dk (dv) elements to 128 in the same dtype (an exact copy).
template <typename T>
__global__ void stage_in_kernel(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
                                const float* __restrict__ la, int64_t rows, int dk, int dv, T* __restrict__ qp,
                                T* __restrict__ kp, T* __restrict__ vp, float* __restrict__ lap) {
  // rows = total_T * H; element (row, c) of the padded [rows, 128] buffers
  const size_t n = static_cast<size_t>(rows) * kD;
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const size_t r = i / kD;
    const int c = static_cast<int>(i % kD);
    const bool kin = c < dk, vin = c < dv;
    qp[i] = kin ? q[r * dk + c] : zero_of<T>();
    kp[i] = kin ? k[r * dk + c] : zero_of<T>();
    vp[i] = vin ? v[r * dv + c] : zero_of<T>();
    lap[i] = kin ? la[r * dk + c] : 0.f;
  }
}

__global__ void stage_state_in_kernel(const float* __restrict__ h0, int64_t nh, int dk, int dv, float* __restrict__ hp) {
  const size_t n = static_cast<size_t>(nh) * kD * kD;
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const size_t m = i / (kD * kD);
    const int c = static_cast<int>((i / kD) % kD), j = static_cast<int>(i % kD);
    hp[i] = (c < dk && j < dv) ? h0[(m * dk + c) * dv + j] : 0.f;
  }
}

template <typename T>
__global__ void stage_out_kernel(const T* __restrict__ op, int64_t rows, int dv, T* __restrict__ out) {
  const size_t n = static_cast<size_t>(rows) * dv;
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const size_t r = i / dv;
    const int j = static_cast<int>(i % dv);
    out[i] = op[r * kD + j];
  }
}

__global__ void stage_state_out_kernel(const float* __restrict__ hp, int64_t nh, int dk, int dv, float* __restrict__ ht) {
  const size_t n = static_cast<size_t>(nh) * dk * dv;
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const size_t m = i / (static_cast<size_t>(dk) * dv);
    const int c = static_cast<int>((i / dv) % dk), j = static_cast<int>(i % dv);
    ht[i] = hp[(m * kD + c) * kD + j];
  }
}

unsigned grid_for(size_t n) {
  const size_t b = (n + 255) / 256;
  return static_cast<unsigned>(b < 16384 ? (b ? b : 1) : 16384);
}

// One warp per (token, head, tensor): lane l owns channels 4l..4l+3 of the head.
constexpr int kConvWarps = 8;

__global__ void __launch_bounds__(kConvWarps * 32)
    conv_l2_kernel(const __nv_bfloat16* __restrict__ qr, const __nv_bfloat16* __restrict__ kr,
                   const __nv_bfloat16* __restrict__ vr, const float* __restrict__ w, const int32_t* __restrict__ cu,
                   int64_t total_T, int N, int H, float* __restrict__ qo, float* __restrict__ ko,
                   float* __restrict__ vo, uint32_t* status) {
  const int64_t gw = static_cast<int64_t>(blockIdx.x) * kConvWarps + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  const int64_t items = total_T * H * 3;
  if (gw >= items) return;
  const int tensor = static_cast<int>(gw % 3);
  const int64_t th = gw / 3;
  const int h = static_cast<int>(th % H);
  const int64_t t = th / H;

  // first token of the sequence that holds t
  int64_t bos;
  if (cu) {
    int lo = 0, hi = N;  // find the last n with cu[n] <= t
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (cu[mid] <= t) lo = mid; else hi = mid;
    }
    bos = cu[lo];
    if (bos > t || bos < 0) {
      if (lane == 0) atomicOr(status, kFlagBadSeqlens);
      return;
    }
  } else {
    const int64_t L = total_T / N;
    bos = (t / L) * L;
  }

  const __nv_bfloat16* x = tensor == 0 ? qr : (tensor == 1 ? kr : vr);
  float* y = tensor == 0 ? qo : (tensor == 1 ? ko : vo);
  const int c0 = lane * 4;
  const size_t ch = static_cast<size_t>(h) * kD + c0;             // channel index within H*128
  const float* wt = w + (static_cast<size_t>(tensor) * H * kD + ch) * 4;  // [3, H*128, 4]
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const int64_t src = t - 3 + j;
    if (src < bos) continue;
    const uint2 raw = *reinterpret_cast<const uint2*>(x + static_cast<size_t>(src) * H * kD + ch);
    const __nv_bfloat16* xb = reinterpret_cast<const __nv_bfloat16*>(&raw);
#pragma unroll
    for (int c = 0; c < 4; ++c) acc[c] = fmaf(wt[c * 4 + j], __bfloat162float(xb[c]), acc[c]);
  }
  float scale = 1.f;
  if (tensor < 2) {
    float ss = acc[0] * acc[0] + acc[1] * acc[1] + acc[2] * acc[2] + acc[3] * acc[3];
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
    scale = rsqrtf(ss + 1e-6f);
  }
  *reinterpret_cast<float4*>(y + static_cast<size_t>(t) * H * kD + ch) =
      make_float4(acc[0] * scale, acc[1] * scale, acc[2] * scale, acc[3] * scale);
}

}  // namespace

cudaError_t launch_stage_in(const void* q, const void* k, const void* v, bool bf16, const float* log_alpha,
                            const float* h0, int64_t total_T, int N, int H, int dk, int dv, void* q_p, void* k_p,
                            void* v_p, float* la_p, float* h0_p, cudaStream_t stream) {
  const int64_t rows = total_T * H;
  if (rows > 0) {
    const unsigned g = grid_for(static_cast<size_t>(rows) * kD);
    if (bf16)
      stage_in_kernel<__nv_bfloat16><<<g, 256, 0, stream>>>(
          static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(k),
          static_cast<const __nv_bfloat16*>(v), log_alpha, rows, dk, dv, static_cast<__nv_bfloat16*>(q_p),
          static_cast<__nv_bfloat16*>(k_p), static_cast<__nv_bfloat16*>(v_p), la_p);
    else
      stage_in_kernel<float><<<g, 256, 0, stream>>>(
          static_cast<const float*>(q), static_cast<const float*>(k), static_cast<const float*>(v), log_alpha, rows,
          dk, dv, static_cast<float*>(q_p), static_cast<float*>(k_p), static_cast<float*>(v_p), la_p);
  }
  if (h0 && h0_p) {
    const int64_t nh = static_cast<int64_t>(N) * H;
    stage_state_in_kernel<<<grid_for(static_cast<size_t>(nh) * kD * kD), 256, 0, stream>>>(h0, nh, dk, dv, h0_p);
  }
  return cudaGetLastError();
}

cudaError_t launch_stage_out(const void* out_p, const float* ht_p, bool bf16, int64_t total_T, int N, int H, int dk,
                             int dv, void* out, float* ht, cudaStream_t stream) {
  const int64_t rows = total_T * H;
  if (rows > 0) {
    const unsigned g = grid_for(static_cast<size_t>(rows) * dv);
    if (bf16)
      stage_out_kernel<__nv_bfloat16><<<g, 256, 0, stream>>>(static_cast<const __nv_bfloat16*>(out_p), rows, dv,
                                                             static_cast<__nv_bfloat16*>(out));
    else
      stage_out_kernel<float><<<g, 256, 0, stream>>>(static_cast<const float*>(out_p), rows, dv,
                                                     static_cast<float*>(out));
  }
  if (ht && ht_p) {
    const int64_t nh = static_cast<int64_t>(N) * H;
    stage_state_out_kernel<<<grid_for(static_cast<size_t>(nh) * dk * dv), 256, 0, stream>>>(ht_p, nh, dk, dv, ht);
  }
  return cudaGetLastError();
}

cudaError_t launch_conv_l2(const void* q_raw, const void* k_raw, const void* v_raw, const float* conv_w,
                           const int32_t* cu, int64_t total_T, int N, int H, int /*d*/, void* q_o, void* k_o,
                           void* v_o, uint32_t* status, cudaStream_t stream) {
  const int64_t items = total_T * H * 3;
  if (items == 0) return cudaSuccess;
  const int64_t blocks = (items + kConvWarps - 1) / kConvWarps;
  conv_l2_kernel<<<static_cast<unsigned>(blocks), kConvWarps * 32, 0, stream>>>(
      static_cast<const __nv_bfloat16*>(q_raw), static_cast<const __nv_bfloat16*>(k_raw),
      static_cast<const __nv_bfloat16*>(v_raw), conv_w, cu, total_T, N, H, static_cast<float*>(q_o),
      static_cast<float*>(k_o), static_cast<float*>(v_o), status);
  return cudaGetLastError();
}

}  // namespace kda
