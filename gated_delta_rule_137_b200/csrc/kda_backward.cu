// kda_backward.cu — gradients of the KDA recurrence (training), one CTA per (sequence,
// head), fp32 on CUDA cores.
//
// Recurrence (Ling-3.0-flash article, section "KDA: constant-size memory over a very
// long context"), one token written with P = Diag(alpha) S_prev, w = P^T k,
// u = beta (v - w):  S = P + k u^T,  o = S^T q.  Walking the tokens backwards with G the
// gradient of S:
//   G += q do^T;  dq = S do;  du = G^T k;  dv = beta du;  dbeta = du . (v - w);
//   dw = -beta du;  dk = G u + P dw;  dP = G + k dw^T;
//   dlog_alpha_i = sum_j dP_ij P_ij;  G <- Diag(alpha) dP.
//
// The states the walk needs are recomputed: pass 1 runs the forward with the state in
// registers and stores it at the start of every 64-token chunk; pass 2 takes the chunks
// in reverse, recomputes one from its checkpoint (keeping the state before each token,
// and u and v - w, in a per-CTA scratch) and walks its tokens backwards. The checkpoints
// come every 16 tokens so that the scratch a CTA writes and reads back (16 states of
// 64 KB) stays in L2; the grid is persistent, each CTA taking (sequence, head) chains in
// turn, so the scratch is bounded by the number of SMs.
//
// Layout as in the decode kernels: 256 threads, warp w holds state rows 16w..16w+15,
// lane l columns 4l..4l+3. Column sums (over rows) go through shared memory across the
// 8 warps; row sums (over columns) are a reduce-scatter inside the warp.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "kda_internal.h"

namespace kda {

namespace {

constexpr int kBD = 128;          // head dim
constexpr int kBRows = 16;        // rows per warp
constexpr int kBChunk = 16;       // checkpoint interval (tokens): a CTA's scratch (1 MB) stays in L2
constexpr int kBPerChunk = 64 / kBChunk;  // checkpoints per 64-token chunk of the plan
constexpr int kBwdMaxCtas = 148;  // persistent grid: one CTA per SM (the registers allow no more)

__device__ __forceinline__ float bload(const float* p) { return __ldg(p); }
__device__ __forceinline__ float bload(const __nv_bfloat16* p) { return __bfloat162float(*p); }

// Row sums of a warp's 16 x 128 block: v[r] is this lane's partial (its 4 columns) for
// row r. Returns the full sum of row `row` (set here), which lanes l and l ^ 1 share.
__device__ __forceinline__ float row_sums16(const float (&v)[16], int lane, int& row) {
  const bool b4 = lane & 16, b3 = lane & 8, b2 = lane & 4, b1 = lane & 2;
  float a[8];
  #pragma unroll
  for (int r = 0; r < 8; ++r) {
    const float keep = b4 ? v[r + 8] : v[r], send = b4 ? v[r] : v[r + 8];
    a[r] = keep + __shfl_xor_sync(0xffffffffu, send, 16);
  }
  float b[4];
  #pragma unroll
  for (int r = 0; r < 4; ++r) {
    const float keep = b3 ? a[r + 4] : a[r], send = b3 ? a[r] : a[r + 4];
    b[r] = keep + __shfl_xor_sync(0xffffffffu, send, 8);
  }
  float c[2];
  #pragma unroll
  for (int r = 0; r < 2; ++r) {
    const float keep = b2 ? b[r + 2] : b[r], send = b2 ? b[r] : b[r + 2];
    c[r] = keep + __shfl_xor_sync(0xffffffffu, send, 4);
  }
  const float keep = b1 ? c[1] : c[0], send = b1 ? c[0] : c[1];
  float d = keep + __shfl_xor_sync(0xffffffffu, send, 2);
  d += __shfl_xor_sync(0xffffffffu, d, 1);
  row = (b4 ? 8 : 0) + (b3 ? 4 : 0) + (b2 ? 2 : 0) + (b1 ? 1 : 0);
  return d;
}

struct BwdArgs {
  const void *q, *k, *v, *d_out;  // [T, H, 128] in TIn
  const float* log_alpha;         // [T, H, 128]
  const float* beta;              // [T, H]
  const float* h0;                // [N, H, 128, 128] or null
  const float* d_final;           // [N, H, 128, 128] or null
  const int32_t* cu;              // [N + 1] or null
  const int32_t* chunk_start;     // [N + 1] from the plan kernel
  float *dq, *dk, *dv, *dla, *dbeta, *dh0;
  float* ckpt;                    // [4 x 64-token chunks][H][128][128]: one state per 16 tokens
  float* scratch;                 // per CTA: [16][128][128] states + [16][2][128] u, v - w
  uint32_t* status;
  int64_t total_T;
  int N, H;
};

constexpr size_t kBwdScratchFloats = static_cast<size_t>(kBChunk) * kBD * kBD + static_cast<size_t>(kBChunk) * 2 * kBD;

template <typename TIn>
__global__ void __launch_bounds__(256, 1) kda_bwd_kernel(const BwdArgs a) {
  if (__ldg(a.chunk_start + a.N) < 0) return;  // bad cu_seqlens (flagged by the plan kernel)
  const int H = a.H;
  const int64_t chains = static_cast<int64_t>(a.N) * a.H;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, tid = threadIdx.x;
  const int col = lane * 4, row0 = warp * kBRows;
  const TIn* qg = static_cast<const TIn*>(a.q);
  const TIn* kg = static_cast<const TIn*>(a.k);
  const TIn* vg = static_cast<const TIn*>(a.v);
  const TIn* dog = static_cast<const TIn*>(a.d_out);
  float* scrS = a.scratch + static_cast<size_t>(blockIdx.x) * kBwdScratchFloats;  // [16][128][128]
  float* scrU = scrS + static_cast<size_t>(kBChunk) * kBD * kBD;                  // [16][2][128]: u, v - w

  __shared__ float s_k[kBD], s_q[kBD], s_al[kBD];   // row vectors of the current token
  __shared__ float s_v[kBD], s_do[kBD];             // column vectors
  __shared__ float s_beta;
  __shared__ float4 s_red[8][32];

  for (int64_t nh = blockIdx.x; nh < chains; nh += gridDim.x) {
    const int n = static_cast<int>(nh / H), h = static_cast<int>(nh % H);
    int64_t bos, eos;
    if (a.cu) {
      bos = __ldg(a.cu + n);
      eos = __ldg(a.cu + n + 1);
    } else {
      const int64_t L = a.total_T / a.N;
      bos = static_cast<int64_t>(n) * L;
      eos = bos + L;
    }
    const int nch = static_cast<int>((eos - bos + kBChunk - 1) / kBChunk);
    const int64_t cbase = static_cast<int64_t>(__ldg(a.chunk_start + n)) * kBPerChunk;

    auto tok_off = [&](int64_t t) { return (static_cast<size_t>(t) * H + h) * kBD; };
    auto state_at = [&](float* base, int r) { return base + static_cast<size_t>(row0 + r) * kBD + col; };

    float4 S[kBRows];
    {
      const float* h0 = a.h0 ? a.h0 + static_cast<size_t>(nh) * kBD * kBD : nullptr;
      #pragma unroll
      for (int r = 0; r < kBRows; ++r)
        S[r] = h0 ? *reinterpret_cast<const float4*>(h0 + static_cast<size_t>(row0 + r) * kBD + col)
                  : make_float4(0.f, 0.f, 0.f, 0.f);
    }

    // one forward token step on S (registers); returns u and v - w for this lane's columns
    auto fwd_step = [&](int64_t t, float4& u_out, float4& vw_out) {
      const size_t o = tok_off(t);
      if (tid < kBD) {
        s_k[tid] = bload(kg + o + tid);
        s_al[tid] = expf(a.log_alpha[o + tid]);
      } else {
        s_v[tid - kBD] = bload(vg + o + tid - kBD);
      }
      if (tid == 0) s_beta = a.beta[static_cast<size_t>(t) * H + h];
      __syncthreads();
      float4 pw = make_float4(0.f, 0.f, 0.f, 0.f);
      #pragma unroll
      for (int r = 0; r < kBRows; ++r) {
        const float al = s_al[row0 + r], kr = s_k[row0 + r];
        S[r].x *= al; S[r].y *= al; S[r].z *= al; S[r].w *= al;
        pw.x = fmaf(kr, S[r].x, pw.x); pw.y = fmaf(kr, S[r].y, pw.y);
        pw.z = fmaf(kr, S[r].z, pw.z); pw.w = fmaf(kr, S[r].w, pw.w);
      }
      s_red[warp][lane] = pw;
      __syncthreads();
      float4 w = make_float4(0.f, 0.f, 0.f, 0.f);
      #pragma unroll
      for (int x = 0; x < 8; ++x) {
        const float4 p = s_red[x][lane];
        w.x += p.x; w.y += p.y; w.z += p.z; w.w += p.w;
      }
      const float bt = s_beta;
      vw_out = make_float4(s_v[col] - w.x, s_v[col + 1] - w.y, s_v[col + 2] - w.z, s_v[col + 3] - w.w);
      u_out = make_float4(bt * vw_out.x, bt * vw_out.y, bt * vw_out.z, bt * vw_out.w);
      #pragma unroll
      for (int r = 0; r < kBRows; ++r) {
        const float kr = s_k[row0 + r];
        S[r].x = fmaf(kr, u_out.x, S[r].x); S[r].y = fmaf(kr, u_out.y, S[r].y);
        S[r].z = fmaf(kr, u_out.z, S[r].z); S[r].w = fmaf(kr, u_out.w, S[r].w);
      }
      __syncthreads();  // s_k / s_al / s_v / s_red are rewritten by the next step
    };

    // ---- pass 1: forward, a checkpoint at the start of every chunk ------------------------
    for (int c = 0; c < nch; ++c) {
      float* ck = a.ckpt + (static_cast<size_t>(cbase + c) * H + h) * kBD * kBD;
      #pragma unroll
      for (int r = 0; r < kBRows; ++r) *reinterpret_cast<float4*>(state_at(ck, r)) = S[r];
      const int64_t t0 = bos + static_cast<int64_t>(c) * kBChunk;
      const int clen = static_cast<int>(eos - t0 < kBChunk ? eos - t0 : kBChunk);
      float4 u, vw;
      for (int i = 0; i < clen; ++i) fwd_step(t0 + i, u, vw);
    }

    // ---- pass 2: chunks in reverse; recompute, then walk the tokens backwards -----------------
    float4 G[kBRows];
    {
      const float* df = a.d_final ? a.d_final + static_cast<size_t>(nh) * kBD * kBD : nullptr;
      #pragma unroll
      for (int r = 0; r < kBRows; ++r)
        G[r] = df ? *reinterpret_cast<const float4*>(df + static_cast<size_t>(row0 + r) * kBD + col)
                  : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    for (int c = nch - 1; c >= 0; --c) {
      const float* ck = a.ckpt + (static_cast<size_t>(cbase + c) * H + h) * kBD * kBD;
      #pragma unroll
      for (int r = 0; r < kBRows; ++r) S[r] = *reinterpret_cast<const float4*>(state_at(const_cast<float*>(ck), r));
      const int64_t t0 = bos + static_cast<int64_t>(c) * kBChunk;
      const int clen = static_cast<int>(eos - t0 < kBChunk ? eos - t0 : kBChunk);
      for (int i = 0; i < clen; ++i) {  // the state before token i, and u, v - w of token i
        float* sp = scrS + static_cast<size_t>(i) * kBD * kBD;
        #pragma unroll
        for (int r = 0; r < kBRows; ++r) *reinterpret_cast<float4*>(state_at(sp, r)) = S[r];
        float4 u, vw;
        fwd_step(t0 + i, u, vw);
        if (warp == 0) {
          *reinterpret_cast<float4*>(scrU + (static_cast<size_t>(i) * 2) * kBD + col) = u;
          *reinterpret_cast<float4*>(scrU + (static_cast<size_t>(i) * 2 + 1) * kBD + col) = vw;
        }
      }
      __syncthreads();  // the scratch rows of u, v - w written by warp 0 are read by every warp

      // S now holds the state after the chunk: the state after its last token
      for (int i = clen - 1; i >= 0; --i) {
        const int64_t t = t0 + i;
        const size_t o = tok_off(t);
        if (tid < kBD) {
          s_k[tid] = bload(kg + o + tid);
          s_q[tid] = bload(qg + o + tid);
          s_al[tid] = expf(a.log_alpha[o + tid]);
        } else {
          s_do[tid - kBD] = bload(dog + o + tid - kBD);
        }
        if (tid == 0) s_beta = a.beta[static_cast<size_t>(t) * H + h];
        float4 Sp[kBRows];  // the state before token t
        const float* sp = scrS + static_cast<size_t>(i) * kBD * kBD;
        #pragma unroll
        for (int r = 0; r < kBRows; ++r) Sp[r] = *reinterpret_cast<const float4*>(state_at(const_cast<float*>(sp), r));
        const float4 u = *reinterpret_cast<const float4*>(scrU + (static_cast<size_t>(i) * 2) * kBD + col);
        const float4 vw = *reinterpret_cast<const float4*>(scrU + (static_cast<size_t>(i) * 2 + 1) * kBD + col);
        __syncthreads();
        const float4 dov = make_float4(s_do[col], s_do[col + 1], s_do[col + 2], s_do[col + 3]);
        const float bt = s_beta;

        // G += q do^T;  dq = S do (rows);  du partial = G^T k
        float rs[kBRows];
        float4 pdu = make_float4(0.f, 0.f, 0.f, 0.f);
        #pragma unroll
        for (int r = 0; r < kBRows; ++r) {
          const float qr = s_q[row0 + r], kr = s_k[row0 + r];
          G[r].x = fmaf(qr, dov.x, G[r].x); G[r].y = fmaf(qr, dov.y, G[r].y);
          G[r].z = fmaf(qr, dov.z, G[r].z); G[r].w = fmaf(qr, dov.w, G[r].w);
          rs[r] = S[r].x * dov.x + S[r].y * dov.y + S[r].z * dov.z + S[r].w * dov.w;
          pdu.x = fmaf(kr, G[r].x, pdu.x); pdu.y = fmaf(kr, G[r].y, pdu.y);
          pdu.z = fmaf(kr, G[r].z, pdu.z); pdu.w = fmaf(kr, G[r].w, pdu.w);
        }
        int rr;
        float sum = row_sums16(rs, lane, rr);
        if (!(lane & 1)) a.dq[o + row0 + rr] = sum;
        s_red[warp][lane] = pdu;
        __syncthreads();
        float4 du = make_float4(0.f, 0.f, 0.f, 0.f);
        #pragma unroll
        for (int x = 0; x < 8; ++x) {
          const float4 p = s_red[x][lane];
          du.x += p.x; du.y += p.y; du.z += p.z; du.w += p.w;
        }
        if (warp == 0) {  // dv = beta du;  dbeta = du . (v - w)
          *reinterpret_cast<float4*>(a.dv + o + col) = make_float4(bt * du.x, bt * du.y, bt * du.z, bt * du.w);
          float db = du.x * vw.x + du.y * vw.y + du.z * vw.z + du.w * vw.w;
          #pragma unroll
          for (int off = 16; off > 0; off >>= 1) db += __shfl_xor_sync(0xffffffffu, db, off);
          if (lane == 0) a.dbeta[static_cast<size_t>(t) * H + h] = db;
        }
        const float4 dw = make_float4(-bt * du.x, -bt * du.y, -bt * du.z, -bt * du.w);

        // P = Diag(alpha) S_prev;  dk = G u + P dw;  dP = G + k dw^T;  dla = rowsum(dP * P);  G = alpha dP
        float rk[kBRows], rl[kBRows];
        #pragma unroll
        for (int r = 0; r < kBRows; ++r) {
          const float al = s_al[row0 + r], kr = s_k[row0 + r];
          const float4 P = make_float4(al * Sp[r].x, al * Sp[r].y, al * Sp[r].z, al * Sp[r].w);
          rk[r] = G[r].x * u.x + G[r].y * u.y + G[r].z * u.z + G[r].w * u.w +
                  P.x * dw.x + P.y * dw.y + P.z * dw.z + P.w * dw.w;
          const float4 dP = make_float4(fmaf(kr, dw.x, G[r].x), fmaf(kr, dw.y, G[r].y), fmaf(kr, dw.z, G[r].z),
                                        fmaf(kr, dw.w, G[r].w));
          rl[r] = dP.x * P.x + dP.y * P.y + dP.z * P.z + dP.w * P.w;
          G[r] = make_float4(al * dP.x, al * dP.y, al * dP.z, al * dP.w);
          S[r] = Sp[r];  // the state after token t - 1
        }
        sum = row_sums16(rk, lane, rr);
        if (!(lane & 1)) a.dk[o + row0 + rr] = sum;
        sum = row_sums16(rl, lane, rr);
        if (!(lane & 1)) a.dla[o + row0 + rr] = sum;
        __syncthreads();  // shared vectors and s_red are rewritten by the next token
      }
    }
    if (a.dh0) {
      float* d0 = a.dh0 + static_cast<size_t>(nh) * kBD * kBD;
      #pragma unroll
      for (int r = 0; r < kBRows; ++r) *reinterpret_cast<float4*>(state_at(d0, r)) = G[r];
    }
  }  // chains
}

}  // namespace

size_t bwd_workspace_bytes(int64_t total_T, int N, int H) {
  if (total_T < 0 || N <= 0 || H <= 0) return 0;
  if (total_T == 0) return split_plan_bytes(N);  // only the plan: no chain has a token
  const int64_t ckpts = split_max_chunks(total_T, N) * kBPerChunk;
  const int64_t chains = static_cast<int64_t>(N) * H;
  const int64_t ctas = chains < kBwdMaxCtas ? chains : kBwdMaxCtas;
  return split_plan_bytes(N) + align256(static_cast<size_t>(ckpts) * H * kBD * kBD * sizeof(float)) +
         static_cast<size_t>(ctas) * kBwdScratchFloats * sizeof(float);
}

cudaError_t launch_backward(const void* q, const void* k, const void* v, bool bf16, const float* log_alpha,
                            const float* beta, const float* h0, const int32_t* cu, int64_t total_T, int N, int H,
                            const void* d_out, const float* d_final, float* dq, float* dk, float* dv, float* dla,
                            float* dbeta, float* dh0, void* ws, uint32_t* status, cudaStream_t stream) {
  uint8_t* w = static_cast<uint8_t*>(ws);
  int32_t* cs = reinterpret_cast<int32_t*>(w);
  cudaError_t e = launch_plan(cu, total_T, N, cs, status, stream);  // 64-token chunks per sequence
  if (e != cudaSuccess) return e;
  const int64_t ckpts = split_max_chunks(total_T, N) * kBPerChunk;
  float* ckpt = reinterpret_cast<float*>(w + split_plan_bytes(N));
  float* scratch = reinterpret_cast<float*>(w + split_plan_bytes(N) +
                                            align256(static_cast<size_t>(ckpts) * H * kBD * kBD * sizeof(float)));
  BwdArgs a{q, k, v, d_out, log_alpha, beta, h0, d_final, cu, cs, dq, dk, dv, dla, dbeta, dh0,
            ckpt, scratch, status, total_T, N, H};
  const int64_t chains = static_cast<int64_t>(N) * H;
  const unsigned grid = static_cast<unsigned>(chains < kBwdMaxCtas ? chains : kBwdMaxCtas);
  if (bf16)
    kda_bwd_kernel<__nv_bfloat16><<<grid, 256, 0, stream>>>(a);
  else
    kda_bwd_kernel<float><<<grid, 256, 0, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace kda
