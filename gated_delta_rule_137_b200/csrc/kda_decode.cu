// kda_decode.cu — one KDA decode token per (sequence, head), fp32 state in place.
//
// Per (n, h), with S the d_k x d_v state (rows = key channels):
//   S' = Diag(alpha) S,  a = S'^T k,  b = S'^T q,  u = beta (v - a),
//   S <- S' + k u^T,     out = S^T q = b + u (k . q)
// (the KDA recurrence of the Ling-3.0-flash article, section "KDA: constant-size
// memory over a very long context", for a single token).
//
// The step is bound by HBM: each 64 KiB state is read once and written once, and
// the arithmetic is ~7 flops per state element. One CTA owns one (n, h) state;
// its 8 warps each stream 16 rows with 128-bit loads (lane = 4 adjacent value
// columns), so all 64 KiB are in flight before any arithmetic. Column sums over
// the 128 key rows reduce within a thread, then across the 8 warps through shared
// memory. Loads/stores use the streaming (evict-first) cache hint: the state is
// touched once per step and is far larger than L2.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "kda_internal.h"

namespace kda {

namespace {

constexpr int kDecodeWarps = 8;
constexpr int kRowsPerWarp = 16;  // 8 x 16 = 128 = KDA_MAX_HEAD_DIM rows

template <typename T>
__device__ __forceinline__ float to_f32(T x);
template <>
__device__ __forceinline__ float to_f32<float>(float x) { return x; }
template <>
__device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T>
__device__ __forceinline__ void store4(T* dst, float4 v);
template <>
__device__ __forceinline__ void store4<float>(float* dst, float4 v) {
  *reinterpret_cast<float4*>(dst) = v;
}
template <>
__device__ __forceinline__ void store4<__nv_bfloat16>(__nv_bfloat16* dst, float4 v) {
  uint2 p;
  p.x = pack_bf16x2(v.x, v.y);
  p.y = pack_bf16x2(v.z, v.w);
  *reinterpret_cast<uint2*>(dst) = p;
}

template <typename T>
__global__ void __launch_bounds__(kDecodeWarps * 32, 2)
    decode_step_kernel(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
                       const float* __restrict__ log_alpha, const float* __restrict__ beta,
                       float* __restrict__ state, T* __restrict__ out, int dk, int dv) {
  const int nh = blockIdx.x;  // n * H + h
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int col = lane * 4;
  const bool col_ok = col < dv;

  __shared__ float s_k[KDA_MAX_HEAD_DIM], s_q[KDA_MAX_HEAD_DIM], s_alpha[KDA_MAX_HEAD_DIM],
      s_v[KDA_MAX_HEAD_DIM];
  __shared__ float4 s_red[2][kDecodeWarps][32];

  float* S = state + static_cast<size_t>(nh) * dk * dv;

  // 1) put the whole state slice of this warp in flight
  float4 s[kRowsPerWarp];
#pragma unroll
  for (int r = 0; r < kRowsPerWarp; ++r) {
    const int row = warp * kRowsPerWarp + r;
    if (col_ok && row < dk)
      s[r] = __ldcs(reinterpret_cast<const float4*>(S + static_cast<size_t>(row) * dv + col));
    else
      s[r] = make_float4(0.f, 0.f, 0.f, 0.f);
  }

  // 2) the token's small vectors
  {
    const int i = threadIdx.x;
    if (i < KDA_MAX_HEAD_DIM) {
      const bool ok = i < dk;
      const size_t o = static_cast<size_t>(nh) * dk + i;
      s_k[i] = ok ? to_f32(k[o]) : 0.f;
      s_q[i] = ok ? to_f32(q[o]) : 0.f;
      s_alpha[i] = ok ? expf(log_alpha[o]) : 0.f;
    } else {
      const int j = i - KDA_MAX_HEAD_DIM;
      s_v[j] = (j < dv) ? to_f32(v[static_cast<size_t>(nh) * dv + j]) : 0.f;
    }
  }
  __syncthreads();

  // 3) decay the rows and accumulate the two column sums a = S'^T k, b = S'^T q
  float4 pa = make_float4(0.f, 0.f, 0.f, 0.f), pb = pa;
#pragma unroll
  for (int r = 0; r < kRowsPerWarp; ++r) {
    const int row = warp * kRowsPerWarp + r;
    const float al = s_alpha[row], kr = s_k[row], qr = s_q[row];
    s[r].x *= al; s[r].y *= al; s[r].z *= al; s[r].w *= al;
    pa.x = fmaf(kr, s[r].x, pa.x); pa.y = fmaf(kr, s[r].y, pa.y);
    pa.z = fmaf(kr, s[r].z, pa.z); pa.w = fmaf(kr, s[r].w, pa.w);
    pb.x = fmaf(qr, s[r].x, pb.x); pb.y = fmaf(qr, s[r].y, pb.y);
    pb.z = fmaf(qr, s[r].z, pb.z); pb.w = fmaf(qr, s[r].w, pb.w);
  }
  s_red[0][warp][lane] = pa;
  s_red[1][warp][lane] = pb;

  // k . q (every warp computes it; 128 entries, 4 per lane)
  float kq = 0.f;
#pragma unroll
  for (int i = lane; i < KDA_MAX_HEAD_DIM; i += 32) kq = fmaf(s_k[i], s_q[i], kq);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) kq += __shfl_xor_sync(0xffffffffu, kq, off);
  __syncthreads();

  float4 a = make_float4(0.f, 0.f, 0.f, 0.f), b = a;
#pragma unroll
  for (int w = 0; w < kDecodeWarps; ++w) {
    const float4 x = s_red[0][w][lane], y = s_red[1][w][lane];
    a.x += x.x; a.y += x.y; a.z += x.z; a.w += x.w;
    b.x += y.x; b.y += y.y; b.z += y.z; b.w += y.w;
  }
  const float bt = beta[nh];
  float4 u;
  u.x = bt * (s_v[(col + 0) & 127] - a.x);
  u.y = bt * (s_v[(col + 1) & 127] - a.y);
  u.z = bt * (s_v[(col + 2) & 127] - a.z);
  u.w = bt * (s_v[(col + 3) & 127] - a.w);

  if (warp == 0 && col_ok) {
    float4 o;
    o.x = fmaf(u.x, kq, b.x); o.y = fmaf(u.y, kq, b.y);
    o.z = fmaf(u.z, kq, b.z); o.w = fmaf(u.w, kq, b.w);
    store4<T>(out + static_cast<size_t>(nh) * dv + col, o);
  }

  // 4) write S' + k u^T back in place
#pragma unroll
  for (int r = 0; r < kRowsPerWarp; ++r) {
    const int row = warp * kRowsPerWarp + r;
    if (col_ok && row < dk) {
      const float kr = s_k[row];
      float4 x = s[r];
      x.x = fmaf(kr, u.x, x.x); x.y = fmaf(kr, u.y, x.y);
      x.z = fmaf(kr, u.z, x.z); x.w = fmaf(kr, u.w, x.w);
      __stcs(reinterpret_cast<float4*>(S + static_cast<size_t>(row) * dv + col), x);
    }
  }
}

// ---- serving decode step of the full mixer ------------------------------------------
// Per (n, h) with slot p = state_indices[n] (n when the indices are NULL): the conv
// history of slot p holds the last three raw q, k, v rows (bf16, oldest first). Thread
// c < 128 convolves channel c of q and k over (history, this token), thread 128 + c
// channel c of v; q and k are L2-normalised over the head's 128 channels; then the
// decode step of decode_step_kernel on the slot's state, the sigmoid gate on the
// output, and the history rolls by one row. (Ling-3.0-flash article, KDA panel: conv4,
// L2 norm, the recurrence, the output gate; one token at a time.)
constexpr int kMixD = 128;

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
  return x;
}

__global__ void __launch_bounds__(kDecodeWarps * 32, 2)
    mixer_decode_kernel(const __nv_bfloat16* __restrict__ q_raw, const __nv_bfloat16* __restrict__ k_raw,
                        const __nv_bfloat16* __restrict__ v_raw, const float* __restrict__ conv_w,
                        const float* __restrict__ log_alpha, const float* __restrict__ beta,
                        const __nv_bfloat16* __restrict__ gate, float* __restrict__ state_pool,
                        __nv_bfloat16* __restrict__ conv_pool, const int32_t* __restrict__ state_indices,
                        int pool_size, int H, __nv_bfloat16* __restrict__ out, uint32_t* status) {
  const int nh = blockIdx.x;  // n * H + h
  const int n = nh / H, h = nh % H;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int col = lane * 4;
  const int slot = state_indices ? state_indices[n] : n;
  if (slot < 0 || slot >= pool_size) {  // the whole CTA takes this branch
    if (threadIdx.x == 0 && status) atomicOr(status, kFlagBadIndex);
    return;
  }
  float* S = state_pool + (static_cast<size_t>(slot) * H + h) * kMixD * kMixD;
  __nv_bfloat16* hist = conv_pool + (static_cast<size_t>(slot) * H + h) * (3 * 3 * kMixD);  // [q,k,v][row][c]

  __shared__ float s_k[kMixD], s_q[kMixD], s_alpha[kMixD], s_v[kMixD];
  __shared__ float s_ss[2][4];
  __shared__ float4 s_red[2][kDecodeWarps][32];

  // 1) the state slice of this warp in flight
  float4 s[kRowsPerWarp];
#pragma unroll
  for (int r = 0; r < kRowsPerWarp; ++r)
    s[r] = __ldcs(reinterpret_cast<const float4*>(S + static_cast<size_t>(warp * kRowsPerWarp + r) * kMixD + col));

  // 2) conv4 over (history, token); roll the history; L2 norm of q and k
  const int i = threadIdx.x, c = i & (kMixD - 1);
  const size_t tok = static_cast<size_t>(nh) * kMixD + c;
  auto conv = [&](int t, const __nv_bfloat16* raw) -> float {
    __nv_bfloat16* hr = hist + t * 3 * kMixD + c;
    const __nv_bfloat16 x0 = hr[0], x1 = hr[kMixD], x2 = hr[2 * kMixD], x3 = raw[tok];
    const float4 w = __ldg(reinterpret_cast<const float4*>(conv_w + ((static_cast<size_t>(t) * H + h) * kMixD + c) * 4));
    hr[0] = x1;
    hr[kMixD] = x2;
    hr[2 * kMixD] = x3;
    return fmaf(w.x, __bfloat162float(x0),
                fmaf(w.y, __bfloat162float(x1), fmaf(w.z, __bfloat162float(x2), w.w * __bfloat162float(x3))));
  };
  float yq = 0.f, yk = 0.f;
  if (i < kMixD) {
    yq = conv(0, q_raw);
    yk = conv(1, k_raw);
    s_alpha[c] = expf(log_alpha[tok]);
    const float sq = warp_sum(yq * yq), sk = warp_sum(yk * yk);
    if (lane == 0) {
      s_ss[0][warp] = sq;
      s_ss[1][warp] = sk;
    }
  } else {
    s_v[c] = conv(2, v_raw);
  }
  __syncthreads();
  if (i < kMixD) {
    const float fq = rsqrtf(s_ss[0][0] + s_ss[0][1] + s_ss[0][2] + s_ss[0][3] + 1e-6f);
    const float fk = rsqrtf(s_ss[1][0] + s_ss[1][1] + s_ss[1][2] + s_ss[1][3] + 1e-6f);
    s_q[c] = yq * fq;
    s_k[c] = yk * fk;
  }
  __syncthreads();

  // 3) decay the rows and accumulate a = S'^T k, b = S'^T q (as decode_step_kernel)
  float4 pa = make_float4(0.f, 0.f, 0.f, 0.f), pb = pa;
#pragma unroll
  for (int r = 0; r < kRowsPerWarp; ++r) {
    const int row = warp * kRowsPerWarp + r;
    const float al = s_alpha[row], kr = s_k[row], qr = s_q[row];
    s[r].x *= al; s[r].y *= al; s[r].z *= al; s[r].w *= al;
    pa.x = fmaf(kr, s[r].x, pa.x); pa.y = fmaf(kr, s[r].y, pa.y);
    pa.z = fmaf(kr, s[r].z, pa.z); pa.w = fmaf(kr, s[r].w, pa.w);
    pb.x = fmaf(qr, s[r].x, pb.x); pb.y = fmaf(qr, s[r].y, pb.y);
    pb.z = fmaf(qr, s[r].z, pb.z); pb.w = fmaf(qr, s[r].w, pb.w);
  }
  s_red[0][warp][lane] = pa;
  s_red[1][warp][lane] = pb;
  float kq = 0.f;
#pragma unroll
  for (int j = lane; j < kMixD; j += 32) kq = fmaf(s_k[j], s_q[j], kq);
  kq = warp_sum(kq);
  __syncthreads();

  float4 a = make_float4(0.f, 0.f, 0.f, 0.f), b = a;
#pragma unroll
  for (int w = 0; w < kDecodeWarps; ++w) {
    const float4 x = s_red[0][w][lane], y = s_red[1][w][lane];
    a.x += x.x; a.y += x.y; a.z += x.z; a.w += x.w;
    b.x += y.x; b.y += y.y; b.z += y.z; b.w += y.w;
  }
  const float bt = beta[nh];
  float4 u;
  u.x = bt * (s_v[col + 0] - a.x);
  u.y = bt * (s_v[col + 1] - a.y);
  u.z = bt * (s_v[col + 2] - a.z);
  u.w = bt * (s_v[col + 3] - a.w);

  if (warp == 0) {
    float o[4] = {fmaf(u.x, kq, b.x), fmaf(u.y, kq, b.y), fmaf(u.z, kq, b.z), fmaf(u.w, kq, b.w)};
    const size_t oo = static_cast<size_t>(nh) * kMixD + col;
    if (gate) {
#pragma unroll
      for (int e = 0; e < 4; ++e) o[e] *= 1.f / (1.f + expf(-__bfloat162float(gate[oo + e])));
    }
    store4<__nv_bfloat16>(out + oo, make_float4(o[0], o[1], o[2], o[3]));
  }

  // 4) S' + k u^T back into the slot
#pragma unroll
  for (int r = 0; r < kRowsPerWarp; ++r) {
    const int row = warp * kRowsPerWarp + r;
    const float kr = s_k[row];
    float4 x = s[r];
    x.x = fmaf(kr, u.x, x.x); x.y = fmaf(kr, u.y, x.y);
    x.z = fmaf(kr, u.z, x.z); x.w = fmaf(kr, u.w, x.w);
    __stcs(reinterpret_cast<float4*>(S + static_cast<size_t>(row) * kMixD + col), x);
  }
}

}  // namespace

cudaError_t launch_mixer_decode_step(const void* q_raw, const void* k_raw, const void* v_raw, const float* conv_w,
                                     const float* log_alpha, const float* beta, const void* gate, float* state_pool,
                                     void* conv_pool, const int32_t* state_indices, int pool_size, int N, int H,
                                     void* out, uint32_t* status, cudaStream_t stream) {
  const unsigned grid = static_cast<unsigned>(N) * static_cast<unsigned>(H);
  if (grid == 0) return cudaSuccess;
  mixer_decode_kernel<<<grid, kDecodeWarps * 32, 0, stream>>>(
      static_cast<const __nv_bfloat16*>(q_raw), static_cast<const __nv_bfloat16*>(k_raw),
      static_cast<const __nv_bfloat16*>(v_raw), conv_w, log_alpha, beta, static_cast<const __nv_bfloat16*>(gate),
      state_pool, static_cast<__nv_bfloat16*>(conv_pool), state_indices, pool_size, H,
      static_cast<__nv_bfloat16*>(out), status);
  return cudaGetLastError();
}

cudaError_t launch_decode_step(const void* q, const void* k, const void* v, bool bf16, const float* log_alpha,
                               const float* beta, float* state, int N, int H, int dk, int dv, void* out,
                               cudaStream_t stream) {
  const unsigned grid = static_cast<unsigned>(N) * static_cast<unsigned>(H);
  if (grid == 0) return cudaSuccess;
  const dim3 block(kDecodeWarps * 32);
  if (bf16) {
    decode_step_kernel<__nv_bfloat16><<<grid, block, 0, stream>>>(
        static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(k),
        static_cast<const __nv_bfloat16*>(v), log_alpha, beta, state, static_cast<__nv_bfloat16*>(out), dk, dv);
  } else {
    decode_step_kernel<float><<<grid, block, 0, stream>>>(
        static_cast<const float*>(q), static_cast<const float*>(k), static_cast<const float*>(v), log_alpha, beta,
        state, static_cast<float*>(out), dk, dv);
  }
  return cudaGetLastError();
}

}  // namespace kda
