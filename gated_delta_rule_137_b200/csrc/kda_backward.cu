// kda_backward.cu — gradients of the KDA recurrence (training), fp32 on CUDA cores.
//
// Recurrence (Ling-3.0-flash article, section "KDA: constant-size memory over a very
// long context"), one token written with P = Diag(alpha) S_prev, w = P^T k,
// u = beta (v - w):  S = P + k u^T,  o = S^T q.  Walking the tokens backwards with G the
// gradient of S:
//   G += q do^T;  dq = S do;  du = G^T k;  dv = beta du;  dbeta = du . (v - w);
//   dw = -beta du;  dk = G u + P dw;  dP = G + k dw^T;
//   dlog_alpha_i = sum_j dP_ij P_ij;  G <- Diag(alpha) dP.
//
// Every column j of S (and of G) evolves on its own: w_j, u_j, du_j, dv_j, dw_j and the
// updates of S[:, j] and G[:, j] read only column j and the token's row vectors (k, q,
// alpha). Only dq, dk, dlog_alpha and dbeta sum over the columns. So a (sequence, head)
// chain is cut into 4 slices of 32 value columns, one CTA each, the 4 CTAs of a chain
// forming a thread-block cluster; their per-slice row sums meet through distributed
// shared memory and are added in a fixed order (the result does not depend on timing).
//
// The states the backward walk needs are recomputed: pass 1 runs the forward and stores
// the state at the start of every 8 tokens; pass 2 takes these stretches in reverse,
// recomputes one from its checkpoint (keeping the state before each of its tokens, and
// u and v - w, in shared memory) and walks its tokens backwards. Per token the inputs of
// the next token are fetched while the current one computes (two buffers in shared
// memory), from L2: each stretch's inputs, and in pass 2 its checkpoint, are prefetched
// into L2 one stretch ahead.
//
// Thread layout: 256 threads, warp w holds state rows 16w..16w+15, lane l column l of
// the slice. Column sums (over rows) go through shared memory across the 8 warps; row
// sums (over the slice's columns) are a reduce-scatter across the 32 lanes.
#include <cooperative_groups.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "kda_internal.h"
#include "sm100_ptx.cuh"

namespace cg = cooperative_groups;

namespace kda {

namespace {

constexpr int kBD = 128;                  // head dim (rows of the state, and all its columns)
constexpr int kBCols = 32;                // value columns of one slice
constexpr int kBSlices = kBD / kBCols;    // CTAs (cluster size) per chain
constexpr int kBRows = 16;                // rows per warp
constexpr int kBStretch = 8;              // checkpoint interval (tokens)
constexpr int kBPerChunk = 64 / kBStretch;  // checkpoints per 64-token chunk of the plan
constexpr int kBThreads = 256;
constexpr int kBMaxClusters = 37;         // 148 SMs / 4: an upper bound on resident clusters

__device__ __forceinline__ float bload(const float* p) { return __ldg(p); }
__device__ __forceinline__ float bload(const __nv_bfloat16* p) { return __bfloat162float(*p); }

// Row sums of a warp's 16 x 32 block: v[r] is this lane's element of row r. Returns the
// full sum of row `row` (set here), which lanes l and l ^ 1 share.
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
  const int32_t* chunk_start;     // [N + 1] from the plan kernel (64-token chunks)
  float *dq, *dk, *dv, *dla, *dbeta, *dh0;
  float* ckpt;                    // [8 x 64-token chunks][H][128][128]: the state every 8 tokens
  int64_t total_T;
  int N, H;
};

// Shared memory of one CTA (dynamic).
struct BwdSmem {
  float st[kBStretch][kBD][kBCols];      // state before each token of the stretch (this slice)
  float part[2][kBStretch][3][kBD];      // per-slice row sums dq, dk, dla (double-buffered)
  float part_beta[2][kBStretch];         // per-slice dbeta
  float u[kBStretch][kBCols], vw[kBStretch][kBCols];
  float red[8][kBCols];                  // column sums across the 8 warps
  float k[2][kBD], q[2][kBD], al[2][kBD];  // row vectors of the token (two buffers)
  float v[2][kBCols], dout[2][kBCols];   // this slice's columns of v and d_out
  float beta[2];
};

// The inputs of one token, held in registers between fetch and publish.
struct TokRegs {
  float k, q, la;  // row tid (tid < 128)
  float x, y;      // v, d_out of column tid - 128 of the slice (128 <= tid < 160); beta (tid == 160)
};

template <typename TIn, bool kAll>
__device__ __forceinline__ TokRegs fetch_token(const BwdArgs& a, int64_t t, int h, int c0, int tid) {
  TokRegs r{0.f, 0.f, 0.f, 0.f, 0.f};
  const size_t o = (static_cast<size_t>(t) * a.H + h) * kBD;
  if (tid < kBD) {
    r.k = bload(static_cast<const TIn*>(a.k) + o + tid);
    r.la = __ldg(a.log_alpha + o + tid);
    if (kAll) r.q = bload(static_cast<const TIn*>(a.q) + o + tid);
  } else if (tid < kBD + kBCols) {
    r.x = bload(static_cast<const TIn*>(a.v) + o + c0 + tid - kBD);
    if (kAll) r.y = bload(static_cast<const TIn*>(a.d_out) + o + c0 + tid - kBD);
  } else if (tid == kBD + kBCols) {
    r.x = __ldg(a.beta + static_cast<size_t>(t) * a.H + h);
  }
  return r;
}

template <bool kAll>
__device__ __forceinline__ void publish_token(BwdSmem& s, int b, const TokRegs& r, int tid) {
  if (tid < kBD) {
    s.k[b][tid] = r.k;
    s.al[b][tid] = expf(r.la);
    if (kAll) s.q[b][tid] = r.q;
  } else if (tid < kBD + kBCols) {
    s.v[b][tid - kBD] = r.x;
    if (kAll) s.dout[b][tid - kBD] = r.y;
  } else if (tid == kBD + kBCols) {
    s.beta[b] = r.x;
  }
}

// Brings a stretch's token inputs into L2 ahead of use (the rows are read from HBM
// otherwise, one token ahead, which does not cover the latency): per token the k, log
// alpha (and, for pass 2, q) rows of the head, this slice's 32 columns of v (and d_out),
// and beta.
template <typename TIn, bool kAll>
__device__ __forceinline__ void prefetch_stretch(const BwdArgs& a, int64_t t0, int len, int h, int c0, int tid) {
  if (tid >= kBStretch * 6) return;
  const int i = tid / 6, which = tid % 6;
  if (i >= len) return;
  const size_t tok = static_cast<size_t>(t0 + i) * a.H + h;
  const size_t o = tok * kBD;
  switch (which) {
    case 0: bulk_prefetch_l2(static_cast<const TIn*>(a.k) + o, kBD * sizeof(TIn)); break;
    case 1: bulk_prefetch_l2(a.log_alpha + o, kBD * sizeof(float)); break;
    case 2: bulk_prefetch_l2(static_cast<const TIn*>(a.v) + o + c0, kBCols * sizeof(TIn)); break;
    case 3: asm volatile("prefetch.global.L2 [%0];" ::"l"(a.beta + tok)); break;
    case 4: if (kAll) bulk_prefetch_l2(static_cast<const TIn*>(a.q) + o, kBD * sizeof(TIn)); break;
    default: if (kAll) bulk_prefetch_l2(static_cast<const TIn*>(a.d_out) + o + c0, kBCols * sizeof(TIn)); break;
  }
}

// Brings this slice's 128 x 32 block of a checkpoint into L2 (one 128-byte row segment
// per thread of the upper half of the CTA). `state` is the checkpoint's [128][128] base.
__device__ __forceinline__ void prefetch_ckpt(const float* state, int c0, int tid) {
  if (tid >= kBD) bulk_prefetch_l2(state + static_cast<size_t>(tid - kBD) * kBD + c0, kBCols * sizeof(float));
}

template <typename TIn>
__global__ void __cluster_dims__(kBSlices, 1, 1) __launch_bounds__(kBThreads, 1) kda_bwd_kernel(const BwdArgs a) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  BwdSmem& s = *reinterpret_cast<BwdSmem*>(smem_raw);
  cg::cluster_group cluster = cg::this_cluster();
  const int slice = static_cast<int>(cluster.block_rank());
  const int c0 = slice * kBCols;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, tid = threadIdx.x;
  const int row0 = warp * kBRows;
  const int H = a.H;
  const int64_t chains = static_cast<int64_t>(a.N) * a.H;
  const int64_t cluster_id = blockIdx.x / kBSlices, n_clusters = gridDim.x / kBSlices;
  const bool bad = __ldg(a.chunk_start + a.N) < 0;  // bad cu_seqlens (flagged by the plan kernel)
  const float* peer_part[kBSlices];
  const float* peer_beta[kBSlices];
#pragma unroll
  for (int p = 0; p < kBSlices; ++p) {
    peer_part[p] = cluster.map_shared_rank(&s.part[0][0][0][0], p);
    peer_beta[p] = cluster.map_shared_rank(&s.part_beta[0][0], p);
  }
  int pb = 0;  // partial-sum buffer of the current stretch

  for (int64_t nh = bad ? chains : cluster_id; nh < chains; nh += n_clusters) {
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
    const int nst = static_cast<int>((eos - bos + kBStretch - 1) / kBStretch);
    const int64_t cbase = static_cast<int64_t>(__ldg(a.chunk_start + n)) * kBPerChunk;
    auto ckpt_of = [&](int c) { return a.ckpt + (static_cast<size_t>(cbase + c) * H + h) * kBD * kBD + c0 + lane; };

    float S[kBRows];
    {
      const float* h0 = a.h0 ? a.h0 + static_cast<size_t>(nh) * kBD * kBD + c0 + lane : nullptr;
#pragma unroll
      for (int r = 0; r < kBRows; ++r) S[r] = h0 ? __ldg(h0 + (row0 + r) * kBD) : 0.f;
    }

    // one forward token step on S from buffer b; when i >= 0 keeps the state before it,
    // and u, v - w, as token i of the stretch. Ends after the column-sum barrier.
    auto fwd_compute = [&](int b, int i) {
      if (i >= 0) {
#pragma unroll
        for (int r = 0; r < kBRows; ++r) s.st[i][row0 + r][lane] = S[r];
      }
      float pw = 0.f;
#pragma unroll
      for (int r = 0; r < kBRows; ++r) {
        S[r] *= s.al[b][row0 + r];
        pw = fmaf(s.k[b][row0 + r], S[r], pw);
      }
      s.red[warp][lane] = pw;
      __syncthreads();
      float w = 0.f;
#pragma unroll
      for (int x = 0; x < 8; ++x) w += s.red[x][lane];
      const float vw = s.v[b][lane] - w, u = s.beta[b] * vw;
#pragma unroll
      for (int r = 0; r < kBRows; ++r) S[r] = fmaf(s.k[b][row0 + r], u, S[r]);
      if (i >= 0 && warp == 0) {
        s.u[i][lane] = u;
        s.vw[i][lane] = vw;
      }
    };

    // ---- pass 1: forward, a checkpoint at the start of every stretch ------------------------
    int b = 0;
    if (nst > 0) {
      publish_token<false>(s, b, fetch_token<TIn, false>(a, bos, h, c0, tid), tid);
      __syncthreads();
    }
    if (nst > 0) prefetch_stretch<TIn, false>(a, bos, nst > 1 ? kBStretch : static_cast<int>(eos - bos), h, c0, tid);
    for (int c = 0; c < nst; ++c) {
      float* ck = ckpt_of(c);
#pragma unroll
      for (int r = 0; r < kBRows; ++r) ck[(row0 + r) * kBD] = S[r];
      const int64_t t0 = bos + static_cast<int64_t>(c) * kBStretch;
      const int len = static_cast<int>(eos - t0 < kBStretch ? eos - t0 : kBStretch);
      if (c + 1 < nst) {  // the next stretch (the last may be partial)
        const int64_t t1 = t0 + kBStretch;
        prefetch_stretch<TIn, false>(a, t1, static_cast<int>(eos - t1 < kBStretch ? eos - t1 : kBStretch), h, c0, tid);
      }
      for (int i = 0; i < len; ++i) {
        const int64_t tn = t0 + i + 1;
        TokRegs nx{};
        if (tn < eos) nx = fetch_token<TIn, false>(a, tn, h, c0, tid);
        fwd_compute(b, -1);
        if (tn < eos) publish_token<false>(s, b ^ 1, nx, tid);
        __syncthreads();
        b ^= 1;
      }
    }

    // ---- pass 2: stretches in reverse; recompute, then walk the tokens backwards --------------
    float G[kBRows];
    {
      const float* df = a.d_final ? a.d_final + static_cast<size_t>(nh) * kBD * kBD + c0 + lane : nullptr;
#pragma unroll
      for (int r = 0; r < kBRows; ++r) G[r] = df ? __ldg(df + (row0 + r) * kBD) : 0.f;
    }
    if (nst > 0) {
      const int64_t t0 = bos + static_cast<int64_t>(nst - 1) * kBStretch;
      publish_token<true>(s, b, fetch_token<TIn, true>(a, t0, h, c0, tid), tid);
      __syncthreads();
    }
    if (nst > 0) {
      const int64_t tl = bos + static_cast<int64_t>(nst - 1) * kBStretch;
      prefetch_stretch<TIn, true>(a, tl, static_cast<int>(eos - tl), h, c0, tid);
    }
    for (int c = nst - 1; c >= 0; --c) {
      const float* ck = ckpt_of(c);
#pragma unroll
      for (int r = 0; r < kBRows; ++r) S[r] = ck[(row0 + r) * kBD];
      const int64_t t0 = bos + static_cast<int64_t>(c) * kBStretch;
      const int len = static_cast<int>(eos - t0 < kBStretch ? eos - t0 : kBStretch);
      if (c > 0) {  // the stretch before (full) and its checkpoint, used after this one
        prefetch_stretch<TIn, true>(a, t0 - kBStretch, kBStretch, h, c0, tid);
        prefetch_ckpt(a.ckpt + (static_cast<size_t>(cbase + c - 1) * H + h) * kBD * kBD, c0, tid);
      }
      // recompute tokens t0 .. t0 + len - 1; the last one's inputs stay in their buffer,
      // since the backward walk starts with the same token
      for (int i = 0; i < len; ++i) {
        const bool more = i + 1 < len;
        TokRegs nx{};
        if (more) nx = fetch_token<TIn, true>(a, t0 + i + 1, h, c0, tid);
        fwd_compute(b, i);
        if (more) publish_token<true>(s, b ^ 1, nx, tid);
        __syncthreads();
        if (more) b ^= 1;
      }
      // S holds the state after the stretch's last token
      for (int i = len - 1; i >= 0; --i) {
        const int64_t t = t0 + i;
        // next: token t - 1, or, after the stretch's first token, the first token of the
        // stretch before it (full, 8 tokens), whose recompute comes next
        const bool more = i > 0 || c > 0;
        TokRegs nx{};
        if (more) nx = fetch_token<TIn, true>(a, i > 0 ? t - 1 : t0 - kBStretch, h, c0, tid);
        const float dov = s.dout[b][lane], bt = s.beta[b];
        const float u = s.u[i][lane], vw = s.vw[i][lane];

        // G += q do^T;  dq = S do;  du = G^T k (column sum)
        float rs[kBRows];
        float pdu = 0.f;
#pragma unroll
        for (int r = 0; r < kBRows; ++r) {
          G[r] = fmaf(s.q[b][row0 + r], dov, G[r]);
          rs[r] = S[r] * dov;
          pdu = fmaf(s.k[b][row0 + r], G[r], pdu);
        }
        int rr;
        float sum = row_sums16(rs, lane, rr);
        if (!(lane & 1)) s.part[pb][i][0][row0 + rr] = sum;
        s.red[warp][lane] = pdu;
        __syncthreads();
        float du = 0.f;
#pragma unroll
        for (int x = 0; x < 8; ++x) du += s.red[x][lane];
        if (warp == 0) {  // dv = beta du (complete: column-local);  dbeta partial = du . (v - w)
          a.dv[(static_cast<size_t>(t) * H + h) * kBD + c0 + lane] = bt * du;
          float db = du * vw;
#pragma unroll
          for (int off = 16; off > 0; off >>= 1) db += __shfl_xor_sync(0xffffffffu, db, off);
          if (lane == 0) s.part_beta[pb][i] = db;
        }
        const float dw = -bt * du;

        // P = Diag(alpha) S_prev;  dk = G u + P dw;  dP = G + k dw^T;  dla = rowsum(dP * P);  G = alpha dP
        float rk[kBRows], rl[kBRows];
#pragma unroll
        for (int r = 0; r < kBRows; ++r) {
          const float al = s.al[b][row0 + r], kr = s.k[b][row0 + r];
          const float sp = s.st[i][row0 + r][lane];
          const float P = al * sp;
          rk[r] = fmaf(G[r], u, P * dw);
          const float dP = fmaf(kr, dw, G[r]);
          rl[r] = dP * P;
          G[r] = al * dP;
          S[r] = sp;  // the state after token t - 1
        }
        sum = row_sums16(rk, lane, rr);
        if (!(lane & 1)) s.part[pb][i][1][row0 + rr] = sum;
        sum = row_sums16(rl, lane, rr);
        if (!(lane & 1)) s.part[pb][i][2][row0 + rr] = sum;
        if (more) publish_token<true>(s, b ^ 1, nx, tid);
        __syncthreads();
        if (more) b ^= 1;
      }

      // the stretch's row sums of all 4 slices: slice p adds up rows 32p .. 32p + 31
      cluster.sync();
      for (int e = tid; e < len * 3 * kBCols; e += kBThreads) {
        const int i = e / (3 * kBCols), which = (e / kBCols) % 3, row = c0 + e % kBCols;
        const int off = ((pb * kBStretch + i) * 3 + which) * kBD + row;
        float acc = 0.f;
#pragma unroll
        for (int p = 0; p < kBSlices; ++p) acc += peer_part[p][off];
        float* dst = which == 0 ? a.dq : which == 1 ? a.dk : a.dla;
        dst[(static_cast<size_t>(t0 + i) * H + h) * kBD + row] = acc;
      }
      if (slice == 0 && tid < len) {
        float acc = 0.f;
#pragma unroll
        for (int p = 0; p < kBSlices; ++p) acc += peer_beta[p][pb * kBStretch + tid];
        a.dbeta[static_cast<size_t>(t0 + tid) * H + h] = acc;
      }
      pb ^= 1;  // the next stretch writes the other buffer while peers may still read this one
    }
    if (a.dh0) {
      float* d0 = a.dh0 + static_cast<size_t>(nh) * kBD * kBD + c0 + lane;
#pragma unroll
      for (int r = 0; r < kBRows; ++r) d0[(row0 + r) * kBD] = G[r];
    }
  }
  cluster.sync();  // no CTA leaves while a peer may still read its partial sums
}

}  // namespace

size_t bwd_workspace_bytes(int64_t total_T, int N, int H) {
  if (total_T < 0 || N <= 0 || H <= 0) return 0;
  if (total_T == 0) return split_plan_bytes(N);  // only the plan: no chain has a token
  const int64_t ckpts = split_max_chunks(total_T, N) * kBPerChunk;
  return split_plan_bytes(N) + align256(static_cast<size_t>(ckpts) * H * kBD * kBD * sizeof(float));
}

cudaError_t launch_backward(const void* q, const void* k, const void* v, bool bf16, const float* log_alpha,
                            const float* beta, const float* h0, const int32_t* cu, int64_t total_T, int N, int H,
                            const void* d_out, const float* d_final, float* dq, float* dk, float* dv, float* dla,
                            float* dbeta, float* dh0, void* ws, uint32_t* status, cudaStream_t stream) {
  uint8_t* w = static_cast<uint8_t*>(ws);
  int32_t* cs = reinterpret_cast<int32_t*>(w);
  cudaError_t e = launch_plan(cu, total_T, N, cs, status, stream);  // 64-token chunks per sequence
  if (e != cudaSuccess) return e;
  float* ckpt = reinterpret_cast<float*>(w + split_plan_bytes(N));
  BwdArgs a{q, k, v, d_out, log_alpha, beta, h0, d_final, cu, cs, dq, dk, dv, dla, dbeta, dh0, ckpt, total_T, N, H};
  const size_t smem = sizeof(BwdSmem);
  auto kern = bf16 ? kda_bwd_kernel<__nv_bfloat16> : kda_bwd_kernel<float>;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  // persistent grid: as many 4-CTA clusters as are resident at once (a cluster must fit in
  // one GPC, so fewer than 148 / 4), each taking chains in turn
  int resident = 0;
  {
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(kBMaxClusters * kBSlices);
    cfg.blockDim = dim3(kBThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr{};
    attr.id = cudaLaunchAttributeClusterDimension;
    attr.val.clusterDim.x = kBSlices;
    attr.val.clusterDim.y = 1;
    attr.val.clusterDim.z = 1;
    cfg.attrs = &attr;
    cfg.numAttrs = 1;
    if (cudaOccupancyMaxActiveClusters(&resident, kern, &cfg) != cudaSuccess || resident < 1) {
      (void)cudaGetLastError();
      resident = 1;
    }
  }
  const int64_t chains = static_cast<int64_t>(N) * H;
  const int64_t cap = resident < kBMaxClusters ? resident : kBMaxClusters;
  const unsigned clusters = static_cast<unsigned>(chains < cap ? chains : cap);
  kern<<<clusters * kBSlices, kBThreads, smem, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace kda
