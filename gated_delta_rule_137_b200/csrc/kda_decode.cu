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

// ---- serving decode of the full mixer ---------------------------------------------------
// Per (n, h) with slot p = state_indices[n] (n when the indices are NULL): the conv
// history of slot p holds the last three raw q, k, v rows (bf16, oldest first). For each
// of the K tokens in order: thread c < 128 convolves channel c of q and k over (history,
// token) and thread 128 + c channel c of v, rolling the history in registers; q and k are
// L2-normalised over the head's 128 channels; the KDA decode step updates the state
// (held in registers across the K tokens); the output gets the sigmoid gate. The state
// and history after token j go to the checkpoints if given (the pools are then left
// as they were), else the final ones go back into the pools. (Ling-3.0-flash article,
// KDA panel: conv4, L2 norm, the recurrence, the output gate; one token at a time.)
constexpr int kMixD = 128;

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
  return x;
}

struct MixerDecodeArgs {
  const __nv_bfloat16* q_raw;  // [N, K, H, d]
  const __nv_bfloat16* k_raw;
  const __nv_bfloat16* v_raw;
  const float* conv_w;         // [3, H*d, 4]
  const float* log_alpha;      // [N, K, H, d]
  const float* beta;           // [N, K, H]
  const __nv_bfloat16* gate;   // [N, K, H, d] or null
  float* state_pool;           // [P, H, d, d]
  __nv_bfloat16* conv_pool;    // [P, H, 3, 3, d]
  const int32_t* state_indices;
  float* state_ckpt;           // [N, K, H, d, d] or null
  __nv_bfloat16* conv_ckpt;    // [N, K, H, 3, 3, d] or null
  __nv_bfloat16* out;          // [N, K, H, d]
  uint32_t* status;
  int pool_size, K, H;
};

// kSingle: one token and no checkpoints (the serving step), compiled without the token
// loop's bookkeeping.
template <bool kSingle>
__global__ void __launch_bounds__(kDecodeWarps * 32, 2) mixer_decode_kernel(const MixerDecodeArgs a) {
  const int nh = blockIdx.x;  // n * H + h
  const int H = a.H, K = kSingle ? 1 : a.K;
  float* const state_ckpt = kSingle ? nullptr : a.state_ckpt;
  const int n = nh / H, h = nh % H;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int col = lane * 4;
  const int slot = a.state_indices ? a.state_indices[n] : n;
  if (slot < 0 || slot >= a.pool_size) {  // the whole CTA takes this branch
    if (threadIdx.x == 0 && a.status) atomicOr(a.status, kFlagBadIndex);
    return;
  }
  float* S = a.state_pool + (static_cast<size_t>(slot) * H + h) * kMixD * kMixD;
  __nv_bfloat16* hist = a.conv_pool + (static_cast<size_t>(slot) * H + h) * (3 * 3 * kMixD);  // [q,k,v][row][c]

  __shared__ float s_k[kMixD], s_q[kMixD], s_alpha[kMixD], s_v[kMixD];
  __shared__ float s_ss[2][4];
  __shared__ float4 s_red[2][kDecodeWarps][32];

  // the state slice of this warp, in flight first; it stays in registers for all K tokens
  float4 s[kRowsPerWarp];
#pragma unroll
  for (int r = 0; r < kRowsPerWarp; ++r)
    s[r] = __ldcs(reinterpret_cast<const float4*>(S + static_cast<size_t>(warp * kRowsPerWarp + r) * kMixD + col));

  // this thread's channel: history rows (oldest first) and conv weights of q, k (i < 128) or v
  const int i = threadIdx.x, c = i & (kMixD - 1);
  const int t0 = i < kMixD ? 0 : 2;    // first tensor of this thread: q (then k) or v
  const int nt = i < kMixD ? 2 : 1;
  float hx[2][3] = {{0.f, 0.f, 0.f}, {0.f, 0.f, 0.f}};
#pragma unroll
  for (int u = 0; u < 2; ++u) {
    if (u >= nt) break;
    const __nv_bfloat16* hr = hist + (t0 + u) * 3 * kMixD + c;
    hx[u][0] = __bfloat162float(hr[0]);
    hx[u][1] = __bfloat162float(hr[kMixD]);
    hx[u][2] = __bfloat162float(hr[2 * kMixD]);
  }
  const float* cwp = a.conv_w + (static_cast<size_t>(t0) * H + h) * kMixD * 4 + c * 4;  // + u * H * d * 4
  const __nv_bfloat16* raw0 = i < kMixD ? a.q_raw : a.v_raw;  // this thread's tensors: q, k or v

  for (int j = 0; j < K; ++j) {
    const size_t tok = ((static_cast<size_t>(n) * K + j) * H + h) * kMixD + c;  // [n][j][h][c]
    // conv4 over (history, token); roll the history; L2 norm of q and k
    float y[2] = {0.f, 0.f};
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      if (u >= nt) break;
      const float x3 = __bfloat162float((u == 0 ? raw0 : a.k_raw)[tok]);
      const float4 cw = __ldg(reinterpret_cast<const float4*>(cwp + static_cast<size_t>(u) * H * kMixD * 4));
      y[u] = fmaf(cw.x, hx[u][0], fmaf(cw.y, hx[u][1], fmaf(cw.z, hx[u][2], cw.w * x3)));
      hx[u][0] = hx[u][1];
      hx[u][1] = hx[u][2];
      hx[u][2] = x3;
    }
    if (i < kMixD) {
      s_alpha[c] = expf(a.log_alpha[tok]);
      const float sq = warp_sum(y[0] * y[0]), sk = warp_sum(y[1] * y[1]);
      if (lane == 0) {
        s_ss[0][warp] = sq;
        s_ss[1][warp] = sk;
      }
    } else {
      s_v[c] = y[0];
    }
    __syncthreads();
    if (i < kMixD) {
      s_q[c] = y[0] * rsqrtf(s_ss[0][0] + s_ss[0][1] + s_ss[0][2] + s_ss[0][3] + 1e-6f);
      s_k[c] = y[1] * rsqrtf(s_ss[1][0] + s_ss[1][1] + s_ss[1][2] + s_ss[1][3] + 1e-6f);
    }
    __syncthreads();

    // decay the rows and accumulate a = S'^T k, b = S'^T q (as decode_step_kernel)
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
    for (int e = lane; e < kMixD; e += 32) kq = fmaf(s_k[e], s_q[e], kq);
    kq = warp_sum(kq);
    __syncthreads();

    float4 ra = make_float4(0.f, 0.f, 0.f, 0.f), rb = ra;
#pragma unroll
    for (int w = 0; w < kDecodeWarps; ++w) {
      const float4 x = s_red[0][w][lane], z = s_red[1][w][lane];
      ra.x += x.x; ra.y += x.y; ra.z += x.z; ra.w += x.w;
      rb.x += z.x; rb.y += z.y; rb.z += z.z; rb.w += z.w;
    }
    const float bt = a.beta[(static_cast<size_t>(n) * K + j) * H + h];
    float4 uu;
    uu.x = bt * (s_v[col + 0] - ra.x);
    uu.y = bt * (s_v[col + 1] - ra.y);
    uu.z = bt * (s_v[col + 2] - ra.z);
    uu.w = bt * (s_v[col + 3] - ra.w);
    if (warp == 0) {
      float o[4] = {fmaf(uu.x, kq, rb.x), fmaf(uu.y, kq, rb.y), fmaf(uu.z, kq, rb.z), fmaf(uu.w, kq, rb.w)};
      const size_t oo = ((static_cast<size_t>(n) * K + j) * H + h) * kMixD + col;
      if (a.gate) {
#pragma unroll
        for (int e = 0; e < 4; ++e) o[e] *= 1.f / (1.f + expf(-__bfloat162float(a.gate[oo + e])));
      }
      store4<__nv_bfloat16>(a.out + oo, make_float4(o[0], o[1], o[2], o[3]));
    }
    // S' + k u^T
#pragma unroll
    for (int r = 0; r < kRowsPerWarp; ++r) {
      const float kr = s_k[warp * kRowsPerWarp + r];
      s[r].x = fmaf(kr, uu.x, s[r].x); s[r].y = fmaf(kr, uu.y, s[r].y);
      s[r].z = fmaf(kr, uu.z, s[r].z); s[r].w = fmaf(kr, uu.w, s[r].w);
    }
    if (state_ckpt) {  // the state and history after token j
      float* C = state_ckpt + ((static_cast<size_t>(n) * K + j) * H + h) * kMixD * kMixD;
#pragma unroll
      for (int r = 0; r < kRowsPerWarp; ++r)
        __stcs(reinterpret_cast<float4*>(C + static_cast<size_t>(warp * kRowsPerWarp + r) * kMixD + col), s[r]);
      __nv_bfloat16* hc = a.conv_ckpt + ((static_cast<size_t>(n) * K + j) * H + h) * (3 * 3 * kMixD) + c;
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        if (u >= nt) break;
#pragma unroll
        for (int m = 0; m < 3; ++m) hc[((t0 + u) * 3 + m) * kMixD] = __float2bfloat16_rn(hx[u][m]);
      }
    }
    if (!kSingle) __syncthreads();  // s_k, s_q, s_v, s_alpha are rewritten by the next token
  }

  if (!state_ckpt) {  // no checkpoints: the state and history after the K tokens go back
#pragma unroll
    for (int r = 0; r < kRowsPerWarp; ++r)
      __stcs(reinterpret_cast<float4*>(S + static_cast<size_t>(warp * kRowsPerWarp + r) * kMixD + col), s[r]);
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      if (u >= nt) break;
#pragma unroll
      for (int m = 0; m < 3; ++m) hist[((t0 + u) * 3 + m) * kMixD + c] = __float2bfloat16_rn(hx[u][m]);
    }
  }
}

// K = 2..4 tokens of one (sequence, head) with a single pass over the state (256 threads,
// 8 warps of 16 state rows, two CTAs per SM): the K-token
// block of the recurrence in the WY form the chunked prefill uses (chunk size K), with
// every product on the CUDA cores. Per key channel r, with tokens j = 0..K-1,
//   c_j = alpha_0 ... alpha_j,   D(i, j) = alpha_{i+1} ... alpha_j   (D(j, j) = 1),
//   S'_j = Diag(c_j) S_0 + sum_{i<j} Diag(D(i, j)) k_i u_i^T   (the state before token j
//          is read, after its decay),
//   a_j = S'_j^T k_j = S_0^T (c_j k_j) + sum_{i<j} G_ji u_i,   G_ji = sum_r k_j k_i D(i, j),
//   u_j = beta_j (v_j - a_j),
//   o_j = S_j^T q_j = S_0^T (c_j q_j) + sum_{i<=j} Q_ji u_i,   Q_ji = sum_r q_j k_i D(i, j),
//   S_j = Diag(c_j) S_0 + sum_{i<=j} Diag(D(i, j)) k_i u_i^T.
// One pass over S_0 gives the 2K column sums S_0^T (c_j k_j), S_0^T (c_j q_j); the K x K
// terms come from the token vectors alone, so the tokens' dependency runs through
// K x 4 numbers per thread instead of the state. The conv, L2 norm and gate are those of
// mixer_decode_kernel; the state after every token is written only with checkpoints.
constexpr int kBlockWarps = 8;  // 256 threads, 16 state rows per warp, two CTAs per SM
constexpr int kBlockRows = kMixD / kBlockWarps;
template <int KB>
struct BlockSmem {
  static constexpr int kC1 = (2 * KB + 3) & ~3;  // per key row: c_j k_j, c_j q_j (padded)
  static constexpr int kC2 = (KB + 1 + 3) & ~3;  // per key row: c_{K-1}, D(j, K-1) k_j
  static constexpr int kCk = KB * (KB + 1);      // per key row and token j: c_j, D(i, j) k_i (i <= j)
  static constexpr int kPairs = KB * KB;         // G_ji (i < j) and Q_ji (i <= j)
  float v[KB][kMixD];
  float ss[KB][2][4];
  float pair[kPairs][4];
  float pairT[kPairs];
  alignas(16) float c1[kMixD][kC1];
  alignas(16) float c2[kMixD][kC2];
  float ck[kMixD][kCk];
  float4 red[2 * KB][kBlockWarps][32];
  float4 sum[2 * KB][32];
};

// G_ji (i < j) at index j * K + i, Q_ji (i <= j) at index i * K + j (the upper triangle)
template <int KB>
__host__ __device__ constexpr int g_index(int j, int i) { return j * KB + i; }
template <int KB>
__host__ __device__ constexpr int q_index(int j, int i) { return i * KB + j; }

template <int KB>
__global__ void __launch_bounds__(kBlockWarps * 32, 2) mixer_decode_block_kernel(const MixerDecodeArgs a) {
  using SM = BlockSmem<KB>;
  extern __shared__ __align__(16) uint8_t block_smem_raw[];
  SM& sm = *reinterpret_cast<SM*>(block_smem_raw);
  const int nh = blockIdx.x;  // n * H + h
  const int H = a.H;
  const int n = nh / H, h = nh % H;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int col = lane * 4;
  const int slot = a.state_indices ? a.state_indices[n] : n;
  if (slot < 0 || slot >= a.pool_size) {  // the whole CTA takes this branch
    if (threadIdx.x == 0 && a.status) atomicOr(a.status, kFlagBadIndex);
    return;
  }
  float* S = a.state_pool + (static_cast<size_t>(slot) * H + h) * kMixD * kMixD;
  __nv_bfloat16* hist = a.conv_pool + (static_cast<size_t>(slot) * H + h) * (3 * 3 * kMixD);

  // ---- the K tokens' conv (q, k: threads 0..127; v: 128..255), L2 sums, decays --------
  const int i = threadIdx.x, c = i & (kMixD - 1);
  const int t0 = i < kMixD ? 0 : 2;
  const int nt = i < kMixD ? 2 : (i < 2 * kMixD ? 1 : 0);  // threads 256.. join at the state pass
  float y[2][KB];
  const float* cwp = a.conv_w + (static_cast<size_t>(t0) * H + h) * kMixD * 4 + c * 4;
  const __nv_bfloat16* raw0 = i < kMixD ? a.q_raw : a.v_raw;
  // raw row m of this thread's tensor u: the three of the history, then the K tokens' (read
  // again for the history written at the end, so that they need no registers meanwhile)
  auto raw_row = [&](int u, int m) -> __nv_bfloat16 {
    if (m < 3) return hist[((t0 + u) * 3 + m) * kMixD + c];
    const __nv_bfloat16* src = u == 0 ? raw0 : a.k_raw;
    return src[((static_cast<size_t>(n) * KB + (m - 3)) * H + h) * kMixD + c];
  };
#pragma unroll
  for (int u = 0; u < 2; ++u) {
    if (u >= nt) break;
    float xr[3 + KB];
#pragma unroll
    for (int m = 0; m < 3 + KB; ++m) xr[m] = __bfloat162float(raw_row(u, m));
    const float4 cw = __ldg(reinterpret_cast<const float4*>(cwp + static_cast<size_t>(u) * H * kMixD * 4));
#pragma unroll
    for (int j = 0; j < KB; ++j)
      y[u][j] = fmaf(cw.x, xr[j], fmaf(cw.y, xr[j + 1], fmaf(cw.z, xr[j + 2], cw.w * xr[j + 3])));
  }
  float al[KB];
  if (i < kMixD) {
#pragma unroll
    for (int j = 0; j < KB; ++j) {
      al[j] = expf(a.log_alpha[((static_cast<size_t>(n) * KB + j) * H + h) * kMixD + c]);
      const float sq = warp_sum(y[0][j] * y[0][j]), sk = warp_sum(y[1][j] * y[1][j]);
      if (lane == 0) {
        sm.ss[j][0][warp] = sq;
        sm.ss[j][1][warp] = sk;
      }
    }
  } else if (i < 2 * kMixD) {
#pragma unroll
    for (int j = 0; j < KB; ++j) sm.v[j][c] = y[0][j];
  }
  float bt[KB];
#pragma unroll
  for (int j = 0; j < KB; ++j) bt[j] = a.beta[(static_cast<size_t>(n) * KB + j) * H + h];
  __syncthreads();

  // ---- per key channel: the coefficient rows and the K x K terms (threads 0..127) --------
  if (i < kMixD) {
    float q[KB], k[KB], cc[KB];
#pragma unroll
    for (int j = 0; j < KB; ++j) {
      q[j] = y[0][j] * rsqrtf(sm.ss[j][0][0] + sm.ss[j][0][1] + sm.ss[j][0][2] + sm.ss[j][0][3] + 1e-6f);
      k[j] = y[1][j] * rsqrtf(sm.ss[j][1][0] + sm.ss[j][1][1] + sm.ss[j][1][2] + sm.ss[j][1][3] + 1e-6f);
      cc[j] = j == 0 ? al[0] : cc[j - 1] * al[j];
      sm.c1[c][j] = cc[j] * k[j];
      sm.c1[c][KB + j] = cc[j] * q[j];
    }
    sm.c2[c][0] = cc[KB - 1];
#pragma unroll
    for (int j = 0; j < KB; ++j) {
      // D(i, j) for i = j, j-1, .., 0: the decays after token i up to token j
      float d = 1.f;
      sm.ck[c][j * (KB + 1)] = cc[j];
#pragma unroll
      for (int ii = j; ii >= 0; --ii) {
        sm.ck[c][j * (KB + 1) + 1 + ii] = d * k[ii];
        const float qp = warp_sum(q[j] * k[ii] * d);
        if (lane == 0) sm.pair[q_index<KB>(j, ii)][warp] = qp;
        if (ii < j) {
          const float gp = warp_sum(k[j] * k[ii] * d);
          if (lane == 0) sm.pair[g_index<KB>(j, ii)][warp] = gp;
        }
        if (ii > 0) d *= al[ii];
      }
      if (j == KB - 1) {
        float e = 1.f;
#pragma unroll
        for (int ii = KB - 1; ii >= 0; --ii) {
          sm.c2[c][1 + ii] = e * k[ii];
          if (ii > 0) e *= al[ii];
        }
      }
    }
  }
  // the state slice of this warp (loaded once the token vectors are done with their
  // registers; the other resident CTAs keep HBM busy meanwhile)
  float4 s[kBlockRows];
#pragma unroll
  for (int r = 0; r < kBlockRows; ++r)
    s[r] = __ldcs(reinterpret_cast<const float4*>(S + static_cast<size_t>(warp * kBlockRows + r) * kMixD + col));
  __syncthreads();
  if (threadIdx.x < SM::kPairs)
    sm.pairT[threadIdx.x] = sm.pair[threadIdx.x][0] + sm.pair[threadIdx.x][1] + sm.pair[threadIdx.x][2] +
                            sm.pair[threadIdx.x][3];

  // ---- one pass over S_0 (held in registers): the 2K column sums, K at a time so that
  //      the accumulators fit beside the state -----------------------------------------
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    float4 acc[KB];
#pragma unroll
    for (int v = 0; v < KB; ++v) acc[v] = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int r = 0; r < kBlockRows; ++r) {
      const float* cr = sm.c1[warp * kBlockRows + r] + half * KB;
#pragma unroll
      for (int v = 0; v < KB; ++v) {
        const float w = cr[v];
        acc[v].x = fmaf(w, s[r].x, acc[v].x); acc[v].y = fmaf(w, s[r].y, acc[v].y);
        acc[v].z = fmaf(w, s[r].z, acc[v].z); acc[v].w = fmaf(w, s[r].w, acc[v].w);
      }
    }
#pragma unroll
    for (int v = 0; v < KB; ++v) sm.red[half * KB + v][warp][lane] = acc[v];
  }
  __syncthreads();
  for (int v = warp; v < 2 * KB; v += kBlockWarps) {
    float4 t = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int w = 0; w < kBlockWarps; ++w) {
      const float4 x = sm.red[v][w][lane];
      t.x += x.x; t.y += x.y; t.z += x.z; t.w += x.w;
    }
    sm.sum[v][lane] = t;
  }
  __syncthreads();

  // ---- the K tokens' u and o for this lane's four value columns ---------------------------
  float4 uu[KB];
#pragma unroll
  for (int j = 0; j < KB; ++j) {
    float4 t = sm.sum[j][lane];  // S_0^T (c_j k_j)
#pragma unroll
    for (int ii = 0; ii < j; ++ii) {
      const float g = sm.pairT[g_index<KB>(j, ii)];
      t.x = fmaf(g, uu[ii].x, t.x); t.y = fmaf(g, uu[ii].y, t.y);
      t.z = fmaf(g, uu[ii].z, t.z); t.w = fmaf(g, uu[ii].w, t.w);
    }
    const float4 vv = *reinterpret_cast<const float4*>(&sm.v[j][col]);
    uu[j] = make_float4(bt[j] * (vv.x - t.x), bt[j] * (vv.y - t.y), bt[j] * (vv.z - t.z), bt[j] * (vv.w - t.w));
  }
  if (warp < KB) {  // warp j writes token j's output row
    const int j = warp;
    float4 o = sm.sum[KB + j][lane];  // S_0^T (c_j q_j)
#pragma unroll
    for (int ii = 0; ii < KB; ++ii) {
      if (ii > j) break;
      const float qv = sm.pairT[q_index<KB>(j, ii)];
      o.x = fmaf(qv, uu[ii].x, o.x); o.y = fmaf(qv, uu[ii].y, o.y);
      o.z = fmaf(qv, uu[ii].z, o.z); o.w = fmaf(qv, uu[ii].w, o.w);
    }
    float ov[4] = {o.x, o.y, o.z, o.w};
    const size_t oo = ((static_cast<size_t>(n) * KB + j) * H + h) * kMixD + col;
    if (a.gate) {
#pragma unroll
      for (int e = 0; e < 4; ++e) ov[e] *= 1.f / (1.f + expf(-__bfloat162float(a.gate[oo + e])));
    }
    store4<__nv_bfloat16>(a.out + oo, make_float4(ov[0], ov[1], ov[2], ov[3]));
  }

  // ---- the states after the tokens: every one with checkpoints, else the last -------------
  if (a.state_ckpt) {
#pragma unroll
    for (int j = 0; j < KB; ++j) {
      float* C = a.state_ckpt + ((static_cast<size_t>(n) * KB + j) * H + h) * kMixD * kMixD;
#pragma unroll
      for (int r = 0; r < kBlockRows; ++r) {
        const int row = warp * kBlockRows + r;
        const float* ck = sm.ck[row] + j * (KB + 1);
        float4 x = make_float4(ck[0] * s[r].x, ck[0] * s[r].y, ck[0] * s[r].z, ck[0] * s[r].w);
#pragma unroll
        for (int ii = 0; ii <= j; ++ii) {
          const float w = ck[1 + ii];
          x.x = fmaf(w, uu[ii].x, x.x); x.y = fmaf(w, uu[ii].y, x.y);
          x.z = fmaf(w, uu[ii].z, x.z); x.w = fmaf(w, uu[ii].w, x.w);
        }
        __stcs(reinterpret_cast<float4*>(C + static_cast<size_t>(row) * kMixD + col), x);
      }
      __nv_bfloat16* hc = a.conv_ckpt + ((static_cast<size_t>(n) * KB + j) * H + h) * (3 * 3 * kMixD) + c;
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        if (u >= nt) break;
#pragma unroll
        for (int m = 0; m < 3; ++m) hc[((t0 + u) * 3 + m) * kMixD] = raw_row(u, j + 1 + m);
      }
    }
  } else {
#pragma unroll
    for (int r = 0; r < kBlockRows; ++r) {
      const int row = warp * kBlockRows + r;
      const float* c2 = sm.c2[row];
      float4 x = make_float4(c2[0] * s[r].x, c2[0] * s[r].y, c2[0] * s[r].z, c2[0] * s[r].w);
#pragma unroll
      for (int ii = 0; ii < KB; ++ii) {
        const float w = c2[1 + ii];
        x.x = fmaf(w, uu[ii].x, x.x); x.y = fmaf(w, uu[ii].y, x.y);
        x.z = fmaf(w, uu[ii].z, x.z); x.w = fmaf(w, uu[ii].w, x.w);
      }
      __stcs(reinterpret_cast<float4*>(S + static_cast<size_t>(row) * kMixD + col), x);
    }
    // the last three raw rows (read before any is written: for K < 3 some come from the history)
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      if (u >= nt) break;
      __nv_bfloat16 last[3];
#pragma unroll
      for (int m = 0; m < 3; ++m) last[m] = raw_row(u, KB + m);
#pragma unroll
      for (int m = 0; m < 3; ++m) hist[((t0 + u) * 3 + m) * kMixD + c] = last[m];
    }
  }
}

template <int KB>
cudaError_t launch_block(const MixerDecodeArgs& a, unsigned grid, cudaStream_t stream) {
  constexpr int kSmem = static_cast<int>(sizeof(BlockSmem<KB>));
  static cudaError_t attr = cudaFuncSetAttribute(mixer_decode_block_kernel<KB>,
                                                 cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
  if (attr != cudaSuccess) return attr;
  mixer_decode_block_kernel<KB><<<grid, kBlockWarps * 32, kSmem, stream>>>(a);
  return cudaGetLastError();
}

// Commit after speculative decoding: slot <- the checkpoint after token accepted[n] - 1
// (accepted[n] = 0 keeps the slot as it is). One CTA per (n, h) copies 64 KiB of state
// and the 2.25 KiB history.
__global__ void __launch_bounds__(256) mixer_decode_commit_kernel(
    const float* __restrict__ state_ckpt, const __nv_bfloat16* __restrict__ conv_ckpt,
    const int32_t* __restrict__ accepted, float* __restrict__ state_pool, __nv_bfloat16* __restrict__ conv_pool,
    const int32_t* __restrict__ state_indices, int pool_size, int K, int H, uint32_t* status) {
  const int nh = blockIdx.x, n = nh / H, h = nh % H;
  const int slot = state_indices ? state_indices[n] : n;
  const int acc = accepted[n];
  if (slot < 0 || slot >= pool_size || acc < 0 || acc > K) {
    if (threadIdx.x == 0 && status) atomicOr(status, kFlagBadIndex);
    return;
  }
  if (acc == 0) return;
  const size_t src = (static_cast<size_t>(n) * K + (acc - 1)) * H + h;
  const size_t dst = static_cast<size_t>(slot) * H + h;
  const float4* cs = reinterpret_cast<const float4*>(state_ckpt + src * kMixD * kMixD);
  float4* ps = reinterpret_cast<float4*>(state_pool + dst * kMixD * kMixD);
  for (int e = threadIdx.x; e < kMixD * kMixD / 4; e += blockDim.x) __stcs(ps + e, __ldcs(cs + e));
  const uint4* ch = reinterpret_cast<const uint4*>(conv_ckpt + src * 9 * kMixD);
  uint4* ph = reinterpret_cast<uint4*>(conv_pool + dst * 9 * kMixD);
  for (int e = threadIdx.x; e < 9 * kMixD / 8; e += blockDim.x) ph[e] = ch[e];
}

}  // namespace

cudaError_t launch_mixer_decode(const void* q_raw, const void* k_raw, const void* v_raw, const float* conv_w,
                                const float* log_alpha, const float* beta, const void* gate, float* state_pool,
                                void* conv_pool, const int32_t* state_indices, int pool_size, int N, int K, int H,
                                void* out, float* state_ckpt, void* conv_ckpt, uint32_t* status, cudaStream_t stream) {
  const unsigned grid = static_cast<unsigned>(N) * static_cast<unsigned>(H);
  if (grid == 0 || K == 0) return cudaSuccess;
  MixerDecodeArgs a{static_cast<const __nv_bfloat16*>(q_raw), static_cast<const __nv_bfloat16*>(k_raw),
                    static_cast<const __nv_bfloat16*>(v_raw), conv_w, log_alpha, beta,
                    static_cast<const __nv_bfloat16*>(gate), state_pool, static_cast<__nv_bfloat16*>(conv_pool),
                    state_indices, state_ckpt, static_cast<__nv_bfloat16*>(conv_ckpt),
                    static_cast<__nv_bfloat16*>(out), status, pool_size, K, H};
  // K = 2..4: the block form (one pass over the state); longer runs of tokens step through
  // them one at a time
  if (K == 2) return launch_block<2>(a, grid, stream);
  if (K == 3) return launch_block<3>(a, grid, stream);
  if (K == 4) return launch_block<4>(a, grid, stream);
  if (K == 1 && !state_ckpt)
    mixer_decode_kernel<true><<<grid, kDecodeWarps * 32, 0, stream>>>(a);
  else
    mixer_decode_kernel<false><<<grid, kDecodeWarps * 32, 0, stream>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_mixer_decode_commit(const float* state_ckpt, const void* conv_ckpt, const int32_t* accepted,
                                       float* state_pool, void* conv_pool, const int32_t* state_indices,
                                       int pool_size, int N, int K, int H, uint32_t* status, cudaStream_t stream) {
  const unsigned grid = static_cast<unsigned>(N) * static_cast<unsigned>(H);
  if (grid == 0) return cudaSuccess;
  mixer_decode_commit_kernel<<<grid, 256, 0, stream>>>(state_ckpt, static_cast<const __nv_bfloat16*>(conv_ckpt),
                                                       accepted, state_pool, static_cast<__nv_bfloat16*>(conv_pool),
                                                       state_indices, pool_size, K, H, status);
  return cudaGetLastError();
}

namespace {
// After a pooled mixer prefill: one CTA of 128 threads per (sequence, head), thread c =
// channel c. Writes the sequence's last three raw q, k, v rows (oldest first, zeros before
// its start) into its conv_pool slot, the layout the decode step reads; with copy_states
// (a call with no tokens), the slot's state becomes h0[n] or zero.
__global__ void __launch_bounds__(128) pool_store_kernel(const __nv_bfloat16* __restrict__ q,
                                                         const __nv_bfloat16* __restrict__ k,
                                                         const __nv_bfloat16* __restrict__ v, const int32_t* cu,
                                                         int64_t total_T, int N, int H, const int32_t* slots,
                                                         int pool_size, __nv_bfloat16* conv_pool, bool copy_states,
                                                         const float* h0, float* state_pool, uint32_t* status) {
  const int n = blockIdx.x / H, h = blockIdx.x % H, c = threadIdx.x;
  int64_t bos, eos;
  if (cu) {
    bos = __ldg(cu + n);
    eos = __ldg(cu + n + 1);
  } else {
    const int64_t len = total_T / N;
    bos = n * len;
    eos = bos + len;
  }
  if (bos < 0 || eos < bos || eos > total_T) return;  // bad cu_seqlens: the prefill's plan flags them
  const int slot = slots ? __ldg(slots + n) : n;
  if (slot < 0 || slot >= pool_size) {
    if (c == 0 && status) atomicOr(status, kFlagBadIndex);
    return;
  }
  const __nv_bfloat16* src[3] = {q, k, v};
  __nv_bfloat16* dst = conv_pool + (static_cast<size_t>(slot) * H + h) * 9 * kD + c;
#pragma unroll
  for (int w = 0; w < 3; ++w)
#pragma unroll
    for (int r = 0; r < 3; ++r) {
      const int64_t t = eos - 3 + r;
      dst[(w * 3 + r) * kD] = t >= bos ? src[w][(static_cast<size_t>(t) * H + h) * kD + c] : __float2bfloat16(0.f);
    }
  if (copy_states) {
    float4* S = reinterpret_cast<float4*>(state_pool + (static_cast<size_t>(slot) * H + h) * kD * kD);
    const float4* S0 = h0 ? reinterpret_cast<const float4*>(h0 + (static_cast<size_t>(n) * H + h) * kD * kD) : nullptr;
    for (int i = c; i < kD * kD / 4; i += 128) S[i] = S0 ? S0[i] : make_float4(0.f, 0.f, 0.f, 0.f);
  }
}
}  // namespace

cudaError_t launch_pool_store(const void* q_raw, const void* k_raw, const void* v_raw, const int32_t* cu,
                              int64_t total_T, int N, int H, const int32_t* slots, int pool_size, void* conv_pool,
                              bool copy_states, const float* h0, float* state_pool, uint32_t* status,
                              cudaStream_t stream) {
  const unsigned grid = static_cast<unsigned>(N) * static_cast<unsigned>(H);
  if (grid == 0) return cudaSuccess;
  pool_store_kernel<<<grid, 128, 0, stream>>>(
      static_cast<const __nv_bfloat16*>(q_raw), static_cast<const __nv_bfloat16*>(k_raw),
      static_cast<const __nv_bfloat16*>(v_raw), cu, total_T, N, H, slots, pool_size,
      static_cast<__nv_bfloat16*>(conv_pool), copy_states, h0, state_pool, status);
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
