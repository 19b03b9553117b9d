// kda_affine.cu — out[i] = M[i] S[i] + B[i] for a batch of 128 x 128 fp32 matrices.
//
// The KDA state after a stretch of tokens is affine in the state before it
// (S_end = M S_start + B, M acting on the key rows): the recurrence of the
// Ling-3.0-flash article, section "KDA: constant-size memory over a very long
// context", multiplies the state by (I - b k k^T) Diag(a) on the left and adds
// b k v^T. Composing such maps lets the segments of one long sequence be prefilled
// in parallel (context parallelism): this kernel applies one map to a state.
//
// fp32 FMA on CUDA cores (the matrices are few and small: 2 MFLOP each). One CTA of
// 256 threads per 32-row band of one output stages S in shared memory; thread t takes
// row t / 8 of the band and 16 consecutive columns. state_fold_kernel applies a chain of
// maps in one launch.
#include <cuda_runtime.h>

#include "kda_internal.h"

namespace kda {

namespace {

constexpr int kAffD = 128;

__global__ void __launch_bounds__(256) state_affine_kernel(const float* __restrict__ M, const float* __restrict__ S,
                                                           const float* B, float* out) {
  extern __shared__ float4 s_S4[];  // S of this matrix, [128][128] fp32 (64 KB)
  const size_t mat = static_cast<size_t>(blockIdx.x) * kAffD * kAffD;
  const int row = blockIdx.y * 32 + (threadIdx.x >> 3);
  const int c0 = (threadIdx.x & 7) * 16;
  float acc[16];
#pragma unroll
  for (int e = 0; e < 16; e += 4) {
    const float4 b = B ? *reinterpret_cast<const float4*>(B + mat + static_cast<size_t>(row) * kAffD + c0 + e)
                       : make_float4(0.f, 0.f, 0.f, 0.f);
    acc[e] = b.x; acc[e + 1] = b.y; acc[e + 2] = b.z; acc[e + 3] = b.w;
  }
  if (S) {
    const float4* Sg = reinterpret_cast<const float4*>(S + mat);
    for (int e = threadIdx.x; e < kAffD * kAffD / 4; e += blockDim.x) s_S4[e] = __ldg(Sg + e);
    __syncthreads();
    const float* s_S = reinterpret_cast<const float*>(s_S4);
    const float* Mr = M + mat + static_cast<size_t>(row) * kAffD;
    for (int k = 0; k < kAffD; k += 4) {
      const float4 m4 = __ldg(reinterpret_cast<const float4*>(Mr + k));
      const float mk[4] = {m4.x, m4.y, m4.z, m4.w};
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
#pragma unroll
        for (int e = 0; e < 16; e += 4) {
          const float4 sv = *reinterpret_cast<const float4*>(s_S + (k + kk) * kAffD + c0 + e);
          acc[e] = fmaf(mk[kk], sv.x, acc[e]);
          acc[e + 1] = fmaf(mk[kk], sv.y, acc[e + 1]);
          acc[e + 2] = fmaf(mk[kk], sv.z, acc[e + 2]);
          acc[e + 3] = fmaf(mk[kk], sv.w, acc[e + 3]);
        }
      }
    }
  }
#pragma unroll
  for (int e = 0; e < 16; e += 4)
    *reinterpret_cast<float4*>(out + mat + static_cast<size_t>(row) * kAffD + c0 + e) =
        make_float4(acc[e], acc[e + 1], acc[e + 2], acc[e + 3]);
}

// Folds `maps` affine maps into start states: S <- M_j S + B_j for j = 0 .. maps-1. MB holds
// the maps as [maps][2][count][128][128] (M then B of each map, the layout of the ranks'
// all-gathered maps). The columns of S evolve independently, so one CTA of 256 threads
// takes 32 columns of one state through every map with that slice in shared memory;
// thread t holds row t / 2, columns 16 (t % 2) .. +15.
__global__ void __launch_bounds__(256) state_fold_kernel(const float* __restrict__ MB, int maps, int64_t count,
                                                         const float* S0, float* out) {
  __shared__ float4 s_S4[2][kAffD * 32 / 4];  // two buffers of the [128][32] slice
  const size_t mat = static_cast<size_t>(blockIdx.x) * kAffD * kAffD;
  const int col0 = blockIdx.y * 32;
  const int row = threadIdx.x >> 1, c0 = (threadIdx.x & 1) * 16;
  const size_t map_elems = static_cast<size_t>(count) * kAffD * kAffD;
  for (int e = threadIdx.x; e < kAffD * 8; e += blockDim.x) {  // the start slice (zero without S0)
    const int r = e >> 3, c4 = (e & 7) * 4;
    s_S4[0][e] = S0 ? __ldg(reinterpret_cast<const float4*>(S0 + mat + static_cast<size_t>(r) * kAffD + col0 + c4))
                    : make_float4(0.f, 0.f, 0.f, 0.f);
  }
  __syncthreads();
  int cur = 0;
  for (int j = 0; j < maps; ++j) {
    const float* M = MB + (2 * static_cast<size_t>(j)) * map_elems + mat;
    const float* B = M + map_elems;
    float acc[16];
#pragma unroll
    for (int e = 0; e < 16; e += 4) {
      const float4 b = __ldg(reinterpret_cast<const float4*>(B + static_cast<size_t>(row) * kAffD + col0 + c0 + e));
      acc[e] = b.x; acc[e + 1] = b.y; acc[e + 2] = b.z; acc[e + 3] = b.w;
    }
    const float* sS = reinterpret_cast<const float*>(s_S4[cur]);
    const float* Mr = M + static_cast<size_t>(row) * kAffD;
    for (int k = 0; k < kAffD; k += 4) {
      const float4 m4 = __ldg(reinterpret_cast<const float4*>(Mr + k));
      const float mk[4] = {m4.x, m4.y, m4.z, m4.w};
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
#pragma unroll
        for (int e = 0; e < 16; e += 4) {
          const float4 sv = *reinterpret_cast<const float4*>(sS + (k + kk) * 32 + c0 + e);
          acc[e] = fmaf(mk[kk], sv.x, acc[e]);
          acc[e + 1] = fmaf(mk[kk], sv.y, acc[e + 1]);
          acc[e + 2] = fmaf(mk[kk], sv.z, acc[e + 2]);
          acc[e + 3] = fmaf(mk[kk], sv.w, acc[e + 3]);
        }
      }
    }
    float* sN = reinterpret_cast<float*>(s_S4[cur ^ 1]);
#pragma unroll
    for (int e = 0; e < 16; e += 4)
      *reinterpret_cast<float4*>(sN + row * 32 + c0 + e) = make_float4(acc[e], acc[e + 1], acc[e + 2], acc[e + 3]);
    __syncthreads();
    cur ^= 1;
  }
  const float* sS = reinterpret_cast<const float*>(s_S4[cur]);
#pragma unroll
  for (int e = 0; e < 16; e += 4)
    *reinterpret_cast<float4*>(out + mat + static_cast<size_t>(row) * kAffD + col0 + c0 + e) =
        *reinterpret_cast<const float4*>(sS + row * 32 + c0 + e);
}

}  // namespace

cudaError_t launch_state_fold(const float* MB, int maps, const float* S0, float* out, int64_t count,
                              cudaStream_t stream) {
  if (count == 0) return cudaSuccess;
  state_fold_kernel<<<dim3(static_cast<unsigned>(count), kAffD / 32), 256, 0, stream>>>(MB, maps, count, S0, out);
  return cudaGetLastError();
}

cudaError_t launch_state_affine(const float* M, const float* S, const float* B, float* out, int64_t count,
                                cudaStream_t stream) {
  if (count == 0) return cudaSuccess;
  constexpr int kSmem = kAffD * kAffD * 4;
  static cudaError_t attr = cudaFuncSetAttribute(state_affine_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
  if (attr != cudaSuccess) return attr;
  state_affine_kernel<<<dim3(static_cast<unsigned>(count), kAffD / 32), 256, S ? kSmem : 0, stream>>>(M, S, B, out);
  return cudaGetLastError();
}

}  // namespace kda
