// kda_prefill.cu — chunked KDA prefill on sm_100a tensor cores.
//
// The recurrence (Ling-3.0-flash article, section "KDA: constant-size memory over a
// very long context"):  S_t = (I - b_t k_t k_t^T) Diag(a_t) S_{t-1} + b_t k_t v_t^T,
// o_t = S_t^T q_t, with a_t = exp(log_alpha_t) per key channel.
//
// Chunked form (64-token chunks, per (sequence, head)); inside a chunk that starts
// from state S, with g_r the running sum of log_alpha up to and including token r:
//   Kt = K*e^g,  Qt = Q*e^g,  Kh = K*e^-g
//   A  = strict_lower(Kt Kh^T) scaled by beta on rows,  P = lower(Qt Kh^T)
//   T  = (I + A)^-1 Diag(beta),  W = T Kt,  U~ = T V
//   U  = U~ - W S,   O = Qt S + P U,   S' = Diag(e^g_last) (S + Kh^T U)
// (the last line folds the usual K*e^(g_last-g) factor into Kh and a row scale).
//
// Mapping onto one CTA of 128 threads (thread i <-> TMEM lane i):
//   * the CTA owns one (sequence, head) chain and a slice of DV value columns;
//     the fp32 state slice S [128 x DV] lives in registers (thread c = key row c)
//     and is copied to shared memory as an MMA operand once per chunk;
//   * every GEMM is tcgen05.mma kind::tf32 (fp32 operands in shared memory read
//     with a 10-bit mantissa, fp32 accumulate in TMEM), M = 128, with 64-row
//     operands stacked in pairs:
//       [Kt; Qt] Kh^T     -> D0 = [A_raw; P_raw]     (M128 N64  K128)
//       [T; P] Kt         -> D0 = [W; -]             (M128 N128 K64)
//       [T; P] V          -> D3 = [U~; -]            (M128 NDV  K64)
//       [-W; Qt] S        -> D1 = [-W S; Qt S]       (M128 NDV  K128)
//       Kh^T U            -> D2                      (M128 NDV  K64)
//       [T; P] U  (+= D1) -> D1 = [-; Qt S + P U]    (M128 NDV  K64)
//     ("-" rows are by-products that are never read). Every operand is stored
//     K-major (the K index contiguous within 128-byte swizzled rows), so Kt and Kh
//     are written twice, token-major and channel-major, and V, S, U transposed.
//     bf16 operands would cost about 2% of RMS in the worst output element on top
//     of the bf16 store; tf32 keeps the operand error well below the store's own
//     rounding;
//   * the 64x64 unit-lower-triangular inverse is done in fp32 on CUDA cores:
//     16x16 diagonal blocks by substitution, then two levels of block doubling
//     X21 = -X22 (A21 X11);
//   * V arrives by TMA (no multicast) and is widened/transposed to fp32 in shared
//     memory; q, k, log_alpha, beta are read with coalesced read-only loads by the
//     thread that owns each key channel.
// Supported decay range: e^{-g} must stay finite, so the decay summed over one
// chunk is limited to kMaxChunkDecay nats per channel (status flag otherwise).
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <mutex>

#include "kda_internal.h"

namespace kda {

namespace {

constexpr int kThreads = 256;  // 8 warps; warps w and w+4 share TMEM lane quarter w
constexpr float kMaxChunkDecay = 80.f;
constexpr int kLd = 68;  // row stride (floats) of the fp32 solve scratch (16-B aligned rows)

// ---- shared memory plan (bytes from a 1024-aligned base); fp32 K-major tiles -------
//  region   size        holds (in chunk order)
//  KQ       64 KB       [Kt; Qt] (128 tok-rows x 128 ch)  ->  [-W; Qt]
//  KH       32 KB       Kh (64 tok-rows x 128 ch)  ->  solve scratch  ->  S^T (with KTT)
//  KTT      32 KB       Kt^T (128 ch-rows x 64 tok)  ->  S^T (second half)
//  KHT      32 KB       Kh^T (128 ch-rows x 64 tok)
//  TP       32 KB       bf16 V from TMA  ->  [T; P] (128 rows x 64 tok)
//  VT       DV*256 B    V^T (DV rows x 64 tok)  ->  U^T
template <int DV>
struct Smem {
  static constexpr int kKQ = 0;
  static constexpr int kKH = 65536;
  static constexpr int kKTT = kKH + 32768;
  static constexpr int kKHT = kKTT + 32768;
  static constexpr int kTP = kKHT + 32768;
  static constexpr int kVT = kTP + 32768;
  static constexpr int kST = kKH;                    // DV*512 <= 64 KB, spans KH and KTT
  static constexpr int kStage = kTP;                 // 64 x DV bf16
  static constexpr int kScratch = kKH;               // A/X [64][kLd] + Y [32][kLd]
  static constexpr int kTot = kVT;                   // per-warp decay totals [8][128] (gate pass only)
  static constexpr int kBeta = kVT + DV * 256;       // fp32 [64]
  static constexpr int kBar = kBeta + 256;           // 2 mbarriers
  static constexpr int kTmemSlot = kBar + 16;
  static constexpr int kTotal = kTmemSlot + 16;
  static constexpr int kAlloc = kTotal + 1024;       // slack for the 1024-B alignment
  static_assert(DV * 512 <= 65536, "S^T must fit in KH + KTT");
  static_assert((64 + 32) * kLd * 4 <= 32768, "solve scratch must fit in KH");
};

template <int DV>
struct Tmem {
  static constexpr uint32_t kCols = (128 + 3 * DV) <= 256 ? 256u : 512u;
  static constexpr uint32_t kD0 = 0;                 // [A; P], then [W; -]   (128 cols)
  static constexpr uint32_t kD1 = 128;               // [-W S; Qt S] -> O     (DV cols)
  static constexpr uint32_t kD2 = 128 + DV;          // Kh^T U                (DV cols)
  static constexpr uint32_t kD3 = 128 + 2 * DV;      // [U~; -]               (DV cols)
};

// K-major fp32 operand tile with `rows` rows (M or N), K step kk (8 columns per step).
__device__ __forceinline__ uint64_t kdesc(uint32_t base, int kk, uint32_t rows) {
  return sdesc(base + (kk >> 2) * rows * 128u + (kk & 3) * 32u, 16u, 1024u, kSwz128);
}

__device__ __forceinline__ float bf2f(__nv_bfloat16 x) { return __bfloat162float(x); }

// read-only loads of an input element as fp32
__device__ __forceinline__ float ld_in(const __nv_bfloat16* p) { return __bfloat162float(__ldg(p)); }
__device__ __forceinline__ float ld_in(const float* p) { return __ldg(p); }
__device__ __forceinline__ float as_f32(__nv_bfloat16 x) { return __bfloat162float(x); }
__device__ __forceinline__ float as_f32(float x) { return x; }

// 4 consecutive input elements (8-byte bf16 or 16-byte fp32 read-only load)
__device__ __forceinline__ void ld4_in(const __nv_bfloat16* p, float* o) {
  const uint2 raw = __ldg(reinterpret_cast<const uint2*>(p));
  const __nv_bfloat16* b = reinterpret_cast<const __nv_bfloat16*>(&raw);
  o[0] = __bfloat162float(b[0]); o[1] = __bfloat162float(b[1]);
  o[2] = __bfloat162float(b[2]); o[3] = __bfloat162float(b[3]);
}
__device__ __forceinline__ void ld4_in(const float* p, float* o) {
  const float4 x = __ldg(reinterpret_cast<const float4*>(p));
  o[0] = x.x; o[1] = x.y; o[2] = x.z; o[3] = x.w;
}

// 16 consecutive output values of one row (TOut = bf16 or fp32)
__device__ __forceinline__ void store16(__nv_bfloat16* dst, const float* o) {
  uint4 p0, p1;
  p0.x = pack_bf16x2(o[0], o[1]);   p0.y = pack_bf16x2(o[2], o[3]);
  p0.z = pack_bf16x2(o[4], o[5]);   p0.w = pack_bf16x2(o[6], o[7]);
  p1.x = pack_bf16x2(o[8], o[9]);   p1.y = pack_bf16x2(o[10], o[11]);
  p1.z = pack_bf16x2(o[12], o[13]); p1.w = pack_bf16x2(o[14], o[15]);
  reinterpret_cast<uint4*>(dst)[0] = p0;
  reinterpret_cast<uint4*>(dst)[1] = p1;
}
__device__ __forceinline__ void store16(float* dst, const float* o) {
#pragma unroll
  for (int i = 0; i < 16; i += 4) *reinterpret_cast<float4*>(dst + i) = make_float4(o[i], o[i + 1], o[i + 2], o[i + 3]);
}

__device__ __forceinline__ void st_tf32(uint8_t* base, uint32_t off, float v) {
  *reinterpret_cast<float*>(base + off) = to_tf32(v);
}
// 4 consecutive fp32 of one row (4-aligned column) as one 16-byte store, tf32-rounded.
__device__ __forceinline__ void st4_tf32(uint8_t* base, uint32_t off, float a, float b, float c, float d) {
  *reinterpret_cast<float4*>(base + off) = make_float4(to_tf32(a), to_tf32(b), to_tf32(c), to_tf32(d));
}

// CTA-wide OR of a predicate (every thread gets the same answer).
__device__ __forceinline__ bool cta_any(bool x) { return __syncthreads_or(x ? 1 : 0) != 0; }

// C (n x n, row stride kLd) = scale * A (n x n) * B (n x n), all fp32 in shared
// memory; n in {16, 32}; `count` independent products are spread over the CTA.
// Thread tile: 2 rows x 4 columns.
__device__ __forceinline__ void small_gemm(int n, int count, const float* const* As, const float* const* Bs,
                                           float* const* Cs, float scale) {
  const int tiles_per = (n / 2) * (n / 4);
  for (int w = threadIdx.x; w < count * tiles_per; w += kThreads) {
    const int p = w / tiles_per, t = w % tiles_per;
    const int r0 = (t / (n / 4)) * 2, c0 = (t % (n / 4)) * 4;
    const float* A = As[p];
    const float* B = Bs[p];
    float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
    for (int k = 0; k < n; ++k) {
      const float a0 = A[r0 * kLd + k], a1 = A[(r0 + 1) * kLd + k];
      const float4 b = *reinterpret_cast<const float4*>(B + k * kLd + c0);
      acc[0][0] = fmaf(a0, b.x, acc[0][0]); acc[0][1] = fmaf(a0, b.y, acc[0][1]);
      acc[0][2] = fmaf(a0, b.z, acc[0][2]); acc[0][3] = fmaf(a0, b.w, acc[0][3]);
      acc[1][0] = fmaf(a1, b.x, acc[1][0]); acc[1][1] = fmaf(a1, b.y, acc[1][1]);
      acc[1][2] = fmaf(a1, b.z, acc[1][2]); acc[1][3] = fmaf(a1, b.w, acc[1][3]);
    }
    float* C = Cs[p];
#pragma unroll
    for (int i = 0; i < 2; ++i)
      *reinterpret_cast<float4*>(C + (r0 + i) * kLd + c0) =
          make_float4(scale * acc[i][0], scale * acc[i][1], scale * acc[i][2], scale * acc[i][3]);
  }
}

template <int DV, typename TIn, typename TOut>
__global__ void __launch_bounds__(kThreads, 1)
    kda_prefill_kernel(const __grid_constant__ CUtensorMap tm_v, const PrefillArgs a) {
  using SM = Smem<DV>;
  using TM = Tmem<DV>;
  constexpr int kSlices = kD / DV;
  static_assert(64 * DV * sizeof(TIn) <= 32768, "V staging must fit in the TP region");

  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sb = smem_u32(sm);
  float* sA = reinterpret_cast<float*>(sm + SM::kScratch);    // [64][kLd]: A, then X in place
  float* sY = sA + 64 * kLd;                                  // [32][kLd]
  float* sBeta = reinterpret_cast<float*>(sm + SM::kBeta);
  float* sTot = reinterpret_cast<float*>(sm + SM::kTot);      // [8][128]
  uint64_t* bar_mma = reinterpret_cast<uint64_t*>(sm + SM::kBar);
  uint64_t* bar_tma = bar_mma + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + SM::kTmemSlot);

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int lq = warp & 3;          // TMEM lane quarter this warp may access
  const int half = warp >> 2;       // which half of a row's columns this warp handles
  const int row = lq * 32 + lane;   // TMEM lane = accumulator row of this thread
  const bool owner = warp < 4;      // warps 0-3 own the state rows (row == tid)
  const int slice = blockIdx.x % kSlices;
  const int nh = blockIdx.x / kSlices;
  const int H = a.H;
  const int h = nh % H;
  const int n = nh / H;
  const int col0 = slice * DV;      // first value column owned by this CTA

  // ---- sequence bounds ------------------------------------------------------------
  int64_t bos, eos;
  if (a.cu) {
    bos = a.cu[n];
    eos = a.cu[n + 1];
    if (bos < 0 || eos < bos || eos > a.total_T || (n == 0 && bos != 0) || (n == a.N - 1 && eos != a.total_T)) {
      if (tid == 0) atomicOr(a.status, kFlagBadSeqlens);
      return;
    }
  } else {
    const int64_t L = a.total_T / a.N;
    bos = static_cast<int64_t>(n) * L;
    eos = bos + L;
  }

  // ---- setup: barriers, TMEM ---------------------------------------------------------
  if (tid == 0) {
    mbar_init(bar_mma, 1);
    mbar_init(bar_tma, 1);
    fence_mbar_init();
    tma_prefetch_desc(&tm_v);
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, TM::kCols);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = *tmem_slot;
  const uint32_t lane_off = static_cast<uint32_t>(lq * 32) << 16;

  // ---- the state slice in registers of warps 0-3: thread c holds S[c][col0 .. col0+DV)
  float S[DV];
#pragma unroll
  for (int j = 0; j < DV; ++j) S[j] = 0.f;
  if (owner && a.h0) {
    const float* h0 = a.h0 + ((static_cast<size_t>(n) * H + h) * kD + tid) * kD + col0;
#pragma unroll
    for (int j = 0; j < DV; j += 4) {
      const float4 x = *reinterpret_cast<const float4*>(h0 + j);
      S[j] = x.x; S[j + 1] = x.y; S[j + 2] = x.z; S[j + 3] = x.w;
    }
  }

  const TIn* __restrict__ qg = static_cast<const TIn*>(a.q);
  const TIn* __restrict__ kg = static_cast<const TIn*>(a.k);
  const float* __restrict__ lag = a.log_alpha;
  const __nv_bfloat16* gateg = static_cast<const __nv_bfloat16*>(a.gate);
  TOut* outg = static_cast<TOut*>(a.out);
  const int64_t tok_stride = static_cast<int64_t>(H) * kD;  // elements between tokens

  constexpr uint32_t kIdAP = idesc_tf32(128, 64, false, false);
  constexpr uint32_t kIdW = idesc_tf32(128, 128, false, false);
  constexpr uint32_t kIdV = idesc_tf32(128, DV, false, false);

  uint32_t mma_phase = 0, tma_phase = 0;
  bool failed = false;

  // all threads wait for the last commit; false (everywhere) if it never came
  auto wait_mma = [&]() -> bool {
    const bool ok = mbar_wait(bar_mma, mma_phase, a.status);
    mma_phase ^= 1u;
    if (cta_any(!ok)) return false;
    tc_fence_after_sync();
    return true;
  };

  for (int64_t t0 = bos; t0 < eos && !failed; t0 += kChunk) {
    const int len = static_cast<int>(eos - t0 < kChunk ? eos - t0 : kChunk);

    // -- 1. V tile by TMA into the staging area (the TP region, free until step 5) -----
    if (tid == 0) {
      mbar_arrive_expect_tx(bar_tma, 64u * DV * static_cast<uint32_t>(sizeof(TIn)));
      tma_load_3d(sm + SM::kStage, &tm_v, col0, h, static_cast<int>(t0), bar_tma);
    }
    // warm L2 with the next chunk's q, k, log_alpha rows
    if (t0 + kChunk < eos && lane < 8) {
      const int64_t nt = t0 + kChunk;
      const int r = warp * 8 + lane;
      if (nt + r < eos) {
        const size_t o = static_cast<size_t>(nt + r) * tok_stride + static_cast<size_t>(h) * kD;
#pragma unroll
        for (int c = 0; c < kD; c += 32) prefetch_l2(lag + o + c);
        prefetch_l2(kg + o);
        prefetch_l2(kg + o + 64);
        prefetch_l2(qg + o);
        prefetch_l2(qg + o + 64);
      }
    }

    // -- 2. gates. Warp w takes tokens 8w..8w+7, lane l key channels 4l..4l+3 ----------
    float gamma_last = 1.f;  // e^{g_last} of key channel `tid` (owner warps)
    {
      if (tid < 64) sBeta[tid] = tid < len ? __ldg(a.beta + (t0 + tid) * H + h) : 0.f;
      const int c0 = lane * 4, r0 = warp * 8;
      float la[8][4], kv[8][4], qv[8][4];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const bool in = r0 + i < len;
        const size_t o = static_cast<size_t>(t0 + (in ? r0 + i : 0)) * tok_stride + static_cast<size_t>(h) * kD + c0;
        const float4 l4 = __ldg(reinterpret_cast<const float4*>(lag + o));
        float k4[4], q4[4];
        ld4_in(kg + o, k4);
        ld4_in(qg + o, q4);
        la[i][0] = in ? l4.x : 0.f; la[i][1] = in ? l4.y : 0.f; la[i][2] = in ? l4.z : 0.f; la[i][3] = in ? l4.w : 0.f;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          kv[i][e] = in ? k4[e] : 0.f;
          qv[i][e] = in ? q4[e] : 0.f;
        }
      }
      // running sums within this warp's 8 tokens, then the other warps' totals before them
      float tot[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int e = 0; e < 4; ++e) { tot[e] += la[i][e]; la[i][e] = tot[e]; }
      *reinterpret_cast<float4*>(sTot + warp * kD + c0) = make_float4(tot[0], tot[1], tot[2], tot[3]);
      __syncthreads();
      float pre[4] = {0.f, 0.f, 0.f, 0.f};
      for (int w = 0; w < warp; ++w) {
        const float4 t4 = *reinterpret_cast<const float4*>(sTot + w * kD + c0);
        pre[0] += t4.x; pre[1] += t4.y; pre[2] += t4.z; pre[3] += t4.w;
      }
      if (owner) {
        float gl = 0.f;
#pragma unroll
        for (int w = 0; w < 8; ++w) gl += sTot[w * kD + tid];
        if (-gl > kMaxChunkDecay) atomicOr(a.status, kFlagDecayRange);
        gamma_last = __expf(gl);
      }
      float kt[8][4], kh[8][4];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        float qt[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float g = pre[e] + la[i][e];
          const float eg = __expf(g), eng = __expf(-g);
          kt[i][e] = kv[i][e] * eg;
          kh[i][e] = kv[i][e] * eng;
          qt[e] = qv[i][e] * eg;
        }
        const int r = r0 + i;
        st4_tf32(sm + SM::kKQ, f32_offset(r, c0, 128), kt[i][0], kt[i][1], kt[i][2], kt[i][3]);   // Kt [tok][ch]
        st4_tf32(sm + SM::kKQ, f32_offset(64 + r, c0, 128), qt[0], qt[1], qt[2], qt[3]);          // Qt [tok][ch]
        st4_tf32(sm + SM::kKH, f32_offset(r, c0, 64), kh[i][0], kh[i][1], kh[i][2], kh[i][3]);    // Kh [tok][ch]
      }
      // channel-major copies: channel c0+e, tokens r0..r0+7; lanes rotate e so that one
      // store instruction touches 8 different swizzle rows (no 16-way bank conflict)
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int e = (j + lane) & 3;
        float x[8], y[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          x[i] = e == 0 ? kt[i][0] : e == 1 ? kt[i][1] : e == 2 ? kt[i][2] : kt[i][3];
          y[i] = e == 0 ? kh[i][0] : e == 1 ? kh[i][1] : e == 2 ? kh[i][2] : kh[i][3];
        }
        const int c = c0 + e;
        st4_tf32(sm + SM::kKTT, f32_offset(c, r0, 128), x[0], x[1], x[2], x[3]);       // Kt^T [ch][tok]
        st4_tf32(sm + SM::kKTT, f32_offset(c, r0 + 4, 128), x[4], x[5], x[6], x[7]);
        st4_tf32(sm + SM::kKHT, f32_offset(c, r0, 128), y[0], y[1], y[2], y[3]);       // Kh^T [ch][tok]
        st4_tf32(sm + SM::kKHT, f32_offset(c, r0 + 4, 128), y[4], y[5], y[6], y[7]);
      }
    }

    // -- 3. V landed: widen/transpose to V^T fp32 (rows past the sequence end -> 0) -------
    {
      const bool ok = mbar_wait(bar_tma, tma_phase, a.status);
      tma_phase ^= 1u;
      if (cta_any(!ok)) { failed = true; break; }
      const TIn* st = reinterpret_cast<const TIn*>(sm + SM::kStage);
      for (int i = tid; i < DV * 16; i += kThreads) {
        const int j = i % DV, t4 = (i / DV) * 4;
        float x[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) x[e] = (t4 + e < len) ? as_f32(st[(t4 + e) * DV + j]) : 0.f;
        st4_tf32(sm + SM::kVT, f32_offset(j, t4, DV), x[0], x[1], x[2], x[3]);
      }
    }
    fence_proxy_async_smem();
    __syncthreads();

    // -- 4. D0 = [A_raw; P_raw] = [Kt; Qt] Kh^T --------------------------------------------
    if (tid == 0) {
      tc_fence_after_sync();
#pragma unroll
      for (int kk = 0; kk < 16; ++kk)
        umma_tf32(tmem + TM::kD0, kdesc(sb + SM::kKQ, kk, 128), kdesc(sb + SM::kKH, kk, 64), kIdAP, kk > 0);
      umma_commit(bar_mma);
    }
    if (!wait_mma()) { failed = true; break; }

    // -- 5. A (rows 0..63: beta-scaled, strictly lower), P (rows 64..127: lower) ---------
    //       each warp takes 32 of the 64 columns of its rows
    {
      const int cb = half * 32;
      float d[32];
      tmem_ld16(tmem + lane_off + TM::kD0 + cb, *reinterpret_cast<float(*)[16]>(d));
      tmem_ld16(tmem + lane_off + TM::kD0 + cb + 16, *reinterpret_cast<float(*)[16]>(d + 16));
      tmem_ld_wait();
      if (lq < 2) {
        const int r = row;
        const float br = sBeta[r];
#pragma unroll
        for (int i = 0; i < 32; i += 4) {
          const int c = cb + i;
          *reinterpret_cast<float4*>(sA + r * kLd + c) =
              make_float4(c < r ? br * d[i] : 0.f, c + 1 < r ? br * d[i + 1] : 0.f, c + 2 < r ? br * d[i + 2] : 0.f,
                          c + 3 < r ? br * d[i + 3] : 0.f);
        }
      } else {
        const int r = row - 64;
#pragma unroll
        for (int i = 0; i < 32; i += 4) {
          const int c = cb + i;
          st4_tf32(sm + SM::kTP, f32_offset(64 + r, c, 128), c <= r ? d[i] : 0.f, c + 1 <= r ? d[i + 1] : 0.f,
                   c + 2 <= r ? d[i + 2] : 0.f, c + 3 <= r ? d[i + 3] : 0.f);
        }
      }
    }
    tc_fence_before_sync();
    __syncthreads();

    // -- 6. X = (I + A)^-1 in fp32 (in place over A), T = X Diag(beta) ---------------------
    {
      float x[16];
      if (tid < 64) {  // 16x16 diagonal blocks: thread (b, j) solves column j of block b
        const int b = tid >> 4, j = tid & 15;
        const float* Ab = sA + (16 * b) * kLd + 16 * b;
#pragma unroll
        for (int r = 0; r < 16; ++r) {
          float acc = (r == j) ? 1.f : 0.f;
#pragma unroll
          for (int i = 0; i < r; ++i) acc = fmaf(-Ab[r * kLd + i], x[i], acc);
          x[r] = acc;
        }
      }
      __syncthreads();
      if (tid < 64) {
        const int b = tid >> 4, j = tid & 15;
#pragma unroll
        for (int r = 0; r < 16; ++r) sA[(16 * b + r) * kLd + 16 * b + j] = x[r];
      }
      __syncthreads();
      // doubling: for each diagonal pair [[X1, 0], [A21, X2]] -> X21 = -X2 (A21 X1)
#pragma unroll 1
      for (int s = 16; s < 64; s *= 2) {
        const int pairs = 64 / (2 * s);
        const float* As_[2];
        const float* Bs_[2];
        float* Cs_[2];
        for (int p = 0; p < pairs; ++p) {
          const int o = 2 * s * p;
          As_[p] = sA + (o + s) * kLd + o;   // A21
          Bs_[p] = sA + o * kLd + o;         // X1
          Cs_[p] = sY + p * 16;              // Y (pairs of 16 side by side, or one 32)
        }
        small_gemm(s, pairs, As_, Bs_, Cs_, 1.f);
        __syncthreads();
        for (int p = 0; p < pairs; ++p) {
          const int o = 2 * s * p;
          As_[p] = sA + (o + s) * kLd + o + s;  // X2
          Bs_[p] = sY + p * 16;                 // Y
          Cs_[p] = sA + (o + s) * kLd + o;      // X21 over A21
        }
        small_gemm(s, pairs, As_, Bs_, Cs_, -1.f);
        __syncthreads();
      }
    }
    if (tid < 128) {  // T row r, columns 32*hc .. +31
      const int r = tid & 63, hc = tid >> 6;
#pragma unroll
      for (int i = 32 * hc; i < 32 * hc + 32; i += 4) {
        const float4 xr = *reinterpret_cast<const float4*>(sA + r * kLd + i);
        st4_tf32(sm + SM::kTP, f32_offset(r, i, 128), i <= r ? xr.x * sBeta[i] : 0.f,
                 i + 1 <= r ? xr.y * sBeta[i + 1] : 0.f, i + 2 <= r ? xr.z * sBeta[i + 2] : 0.f,
                 i + 3 <= r ? xr.w * sBeta[i + 3] : 0.f);
      }
    }
    fence_proxy_async_smem();
    __syncthreads();

    // -- 7. D0 = [W; -] = [T; P] Kt   and   D3 = [U~; -] = [T; P] V -------------------------
    if (tid == 0) {
      tc_fence_after_sync();
#pragma unroll
      for (int kk = 0; kk < 8; ++kk)
        umma_tf32(tmem + TM::kD0, kdesc(sb + SM::kTP, kk, 128), kdesc(sb + SM::kKTT, kk, 128), kIdW, kk > 0);
#pragma unroll
      for (int kk = 0; kk < 8; ++kk)
        umma_tf32(tmem + TM::kD3, kdesc(sb + SM::kTP, kk, 128), kdesc(sb + SM::kVT, kk, DV), kIdV, kk > 0);
      umma_commit(bar_mma);
    }
    if (!wait_mma()) { failed = true; break; }

    // -- 8. -W -> rows 0..63 of KQ (over Kt), 64 columns per warp;  S -> S^T operand ------
    if (lq < 2) {
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int cb = half * 64 + 16 * j;
        float w[16];
        tmem_ld16(tmem + lane_off + TM::kD0 + cb, w);
        tmem_ld_wait();
#pragma unroll
        for (int e = 0; e < 16; e += 4)
          st4_tf32(sm + SM::kKQ, f32_offset(row, cb + e, 128), -w[e], -w[e + 1], -w[e + 2], -w[e + 3]);
      }
    }
    if (owner) {
#pragma unroll
      for (int j = 0; j < DV; ++j) st_tf32(sm + SM::kST, f32_offset(j, tid, DV), S[j]);
    }
    fence_proxy_async_smem();
    tc_fence_before_sync();
    __syncthreads();

    // -- 9. D1 = [-W S; Qt S] ----------------------------------------------------------------
    if (tid == 0) {
      tc_fence_after_sync();
#pragma unroll
      for (int kk = 0; kk < 16; ++kk)
        umma_tf32(tmem + TM::kD1, kdesc(sb + SM::kKQ, kk, 128), kdesc(sb + SM::kST, kk, DV), kIdV, kk > 0);
      umma_commit(bar_mma);
    }
    if (!wait_mma()) { failed = true; break; }

    // -- 10. U = U~ - W S -> U^T operand (over V^T), DV/2 columns per warp ----------------------
    if (lq < 2) {
#pragma unroll
      for (int j = 0; j < DV / 2; j += 16) {
        const int cb = half * (DV / 2) + j;
        float ut[16], ws[16];
        tmem_ld16(tmem + lane_off + TM::kD3 + cb, ut);
        tmem_ld16(tmem + lane_off + TM::kD1 + cb, ws);
        tmem_ld_wait();
#pragma unroll
        for (int e = 0; e < 16; ++e) st_tf32(sm + SM::kVT, f32_offset(cb + e, row, DV), ut[e] + ws[e]);
      }
    }
    fence_proxy_async_smem();
    tc_fence_before_sync();
    __syncthreads();

    // -- 11. D2 = Kh^T U ;  D1 += [T; P] U  ->  O = Qt S + P U in rows 64..127 ----------------
    if (tid == 0) {
      tc_fence_after_sync();
#pragma unroll
      for (int kk = 0; kk < 8; ++kk)
        umma_tf32(tmem + TM::kD2, kdesc(sb + SM::kKHT, kk, 128), kdesc(sb + SM::kVT, kk, DV), kIdV, kk > 0);
#pragma unroll
      for (int kk = 0; kk < 8; ++kk)
        umma_tf32(tmem + TM::kD1, kdesc(sb + SM::kTP, kk, 128), kdesc(sb + SM::kVT, kk, DV), kIdV, 1u);
      umma_commit(bar_mma);
    }
    if (!wait_mma()) { failed = true; break; }

    // -- 12. S <- e^{g_last} (S + D2) (owners);  out rows <- O (* sigmoid(gate)) ---------
    if (owner) {
#pragma unroll
      for (int j = 0; j < DV; j += 16) {
        float d2[16];
        tmem_ld16(tmem + lane_off + TM::kD2 + j, d2);
        tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 16; ++i) S[j + i] = gamma_last * (S[j + i] + d2[i]);
      }
    }
    if (lq >= 2) {
      const int r = row - 64;
#pragma unroll
      for (int j = 0; j < DV / 2; j += 16) {
        const int cb = half * (DV / 2) + j;
        float o[16];
        tmem_ld16(tmem + lane_off + TM::kD1 + cb, o);
        tmem_ld_wait();
        if (r < len) {
          const size_t off = static_cast<size_t>(t0 + r) * tok_stride + static_cast<size_t>(h) * kD + col0 + cb;
          if (gateg) {
            const uint4 g0 = *reinterpret_cast<const uint4*>(gateg + off);
            const uint4 g1 = *reinterpret_cast<const uint4*>(gateg + off + 8);
            const __nv_bfloat16* gb0 = reinterpret_cast<const __nv_bfloat16*>(&g0);
            const __nv_bfloat16* gb1 = reinterpret_cast<const __nv_bfloat16*>(&g1);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              o[i] *= 1.f / (1.f + __expf(-bf2f(gb0[i])));
              o[8 + i] *= 1.f / (1.f + __expf(-bf2f(gb1[i])));
            }
          }
          store16(outg + off, o);
        }
      }
    }
    tc_fence_before_sync();
    __syncthreads();
  }

  // ---- final state -------------------------------------------------------------------
  if (!failed && a.ht && owner) {
    float* ht = a.ht + ((static_cast<size_t>(n) * H + h) * kD + tid) * kD + col0;
#pragma unroll
    for (int j = 0; j < DV; j += 4) *reinterpret_cast<float4*>(ht + j) = make_float4(S[j], S[j + 1], S[j + 2], S[j + 3]);
  }

  // ---- teardown ----------------------------------------------------------------------
  tc_fence_before_sync();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after_sync();
    tmem_dealloc(tmem, TM::kCols);
  }
}

// final_state = initial_state (or 0) for calls with no tokens at all
__global__ void copy_states_kernel(const float* __restrict__ h0, float* __restrict__ ht, size_t n4) {
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < n4;
       i += static_cast<size_t>(gridDim.x) * blockDim.x)
    reinterpret_cast<float4*>(ht)[i] = h0 ? reinterpret_cast<const float4*>(h0)[i] : make_float4(0.f, 0.f, 0.f, 0.f);
}

// ---- TMA descriptor encoding through the driver entry point ----------------------------
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// [total_T, H, 128] (bf16 or fp32) viewed as (d, head, token); box = (box_d, 1, 64),
// rows land unswizzled (box_d elements each)
bool encode_value_map(CUtensorMap* m, const void* ptr, int64_t total_T, int H, int box_d, bool f32) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t es = f32 ? 4 : 2;
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(kD), static_cast<cuuint64_t>(H),
                              static_cast<cuuint64_t>(total_T)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(kD) * es, static_cast<cuuint64_t>(H) * kD * es};
  const cuuint32_t box[3] = {static_cast<cuuint32_t>(box_d), 1u, static_cast<cuuint32_t>(kChunk)};
  const cuuint32_t estr[3] = {1u, 1u, 1u};
  const CUresult r = fn(m, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3,
                        const_cast<void*>(ptr), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <int DV, typename TIn, typename TOut>
cudaError_t launch_dv(const PrefillArgs& a, cudaStream_t stream) {
  CUtensorMap tm;
  if (!encode_value_map(&tm, a.v, a.total_T, a.H, DV, sizeof(TIn) == 4)) return cudaErrorInvalidValue;
  auto kern = kda_prefill_kernel<DV, TIn, TOut>;
  static std::once_flag once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(once, [&] {
    attr_err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Smem<DV>::kAlloc);
  });
  if (attr_err != cudaSuccess) return attr_err;
  const unsigned grid = static_cast<unsigned>(a.N) * static_cast<unsigned>(a.H) * (kD / DV);
  kern<<<grid, kThreads, Smem<DV>::kAlloc, stream>>>(tm, a);
  return cudaGetLastError();
}

template <typename TIn, typename TOut>
cudaError_t launch_types(const PrefillArgs& a, cudaStream_t stream) {
  // value-column slices per chain: split more when there are few (sequence, head)
  // chains, so that the grid still covers the 148 SMs
  const int64_t chains = static_cast<int64_t>(a.N) * a.H;
  if (chains <= 74) return launch_dv<32, TIn, TOut>(a, stream);
  if (chains <= 296) return launch_dv<64, TIn, TOut>(a, stream);
  return launch_dv<128, TIn, TOut>(a, stream);
}

}  // namespace

cudaError_t launch_prefill_d128(const PrefillArgs& a, cudaStream_t stream) {
  if (a.N == 0) return cudaSuccess;
  if (a.total_T == 0) {
    if (!a.ht) return cudaSuccess;
    const size_t n4 = static_cast<size_t>(a.N) * a.H * kD * kD / 4;
    copy_states_kernel<<<static_cast<unsigned>((n4 + 255) / 256 < 4096 ? (n4 + 255) / 256 : 4096), 256, 0, stream>>>(
        a.h0, a.ht, n4);
    return cudaGetLastError();
  }
  if (!a.in_f32) return a.out_f32 ? cudaErrorInvalidValue : launch_types<__nv_bfloat16, __nv_bfloat16>(a, stream);
  return a.out_f32 ? launch_types<float, float>(a, stream) : launch_types<float, __nv_bfloat16>(a, stream);
}

}  // namespace kda
