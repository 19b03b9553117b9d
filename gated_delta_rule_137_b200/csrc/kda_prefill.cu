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
// Mapping onto one CTA of 512 threads (warp w reads TMEM lanes 32 (w % 4) .. and value
// column part w / 4):
//   * the CTA owns one (sequence, head) chain and a slice of DV value columns; the fp32
//     state slice S [128 x DV] lives in TMEM (lane c = key row c) and is copied to
//     shared memory as an MMA operand once per chunk;
//   * every GEMM is tcgen05.mma kind::tf32 (fp32 operands in shared memory read
//     with a 10-bit mantissa, fp32 accumulate in TMEM), M = 128, with 64-row
//     operands stacked in pairs:
//       [Kt; Qt] Kh^T     -> D0 = [A_raw; P_raw]     (M128 N64  K128)
//       [T; P] Kt         -> D0 = [W; -]             (M128 N128 K64)
//       [T; P] V          -> D3 = [U~; -]            (M128 NDV  K64)
//       [-W; Qt] S        -> D1 = [-W S; Qt S]       (M128 NDV  K128)
//       Kh^T U            -> D2                      (M128 NDV  K64)
//       [T; P] U  (+= D1) -> D1 = [-; Qt S + P U]    (M128 NDV  K64)
//     ("-" rows are by-products that are never read). Kt, Kh and V are written once
//     more as whole lines of MN-major tiles (128B swizzle with 32-byte atoms), the B
//     operands Kt and V and the A operand Kh^T, so nothing is transposed on the CUDA
//     cores for them; S^T and U^T are written K-major by the epilogues (MN-major lines
//     measured slower there). bf16 operands would cost about 2% of RMS in the worst
//     output element on top of the bf16 store; tf32 keeps the operand error well below
//     the store's own rounding;
//   * the 64x64 unit-lower-triangular inverse is done in fp32 on CUDA cores:
//     16x16 diagonal blocks by substitution, then two levels of block doubling
//     X21 = -X22 (A21 X11);
//   * V arrives by TMA (no multicast) and is widened to fp32 operand lines in shared
//     memory; q, k, log_alpha, beta are read with coalesced read-only loads by the
//     thread that owns each key channel.
// Decay range: the factorised products need e^{-g} finite, so a chunk whose decay summed
// over its tokens passes kMaxChunkDecay nats in some key channel is walked token by
// token instead (walk_chunk: the recurrence itself on the state slice, exact for any
// decay); kMaxChunkDecay also keeps the tf32 form within its parity bar. Both forms give
// the same result up to rounding; the walk is slower.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "kda_tile.cuh"

namespace kda {

namespace {

constexpr int kThreads = 512;  // 16 warps; warp w reads TMEM lanes 32*(w%4).. and column part w/4
// ---- shared memory plan (bytes from a 1024-aligned base); fp32 operand tiles ------
//  region   size        holds (in chunk order)
//  KQ       64 KB       [Kt; Qt] (128 tok-rows x 128 ch)  ->  [-W; Qt]
//  KH       32 KB       Kh (64 tok-rows x 128 ch)  ->  solve scratch  ->  S^T (with KTT)
//  KTT      32 KB       Kt as MN-major lines (64 tok x 128 ch)  ->  S^T (second half)
//  KHT      32 KB       Kh as MN-major lines (64 tok x 128 ch)
//  TP       32 KB       bf16 V from TMA  ->  [T; P] (128 rows x 64 tok)
//  VT       DV*256 B    V as MN-major lines (64 tok x DV)  ->  U^T
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
  static constexpr int kTot = kVT;                   // per-warp decay totals [16][128] (gate pass only)
  static constexpr int kBeta = kVT + DV * 256;       // fp32 [64]
  static constexpr int kGamma = kBeta + 256;         // fp32 [2][128]: e^{g_last} of the last two chunks
  static constexpr int kBar = kGamma + 1024;         // 2 mbarriers
  static constexpr int kTmemSlot = kBar + 16;
  static constexpr int kTotal = kTmemSlot + 16;
  static constexpr int kAlloc = kTotal + 1024;       // slack for the 1024-B alignment
  static_assert(DV * 512 <= 65536, "S^T must fit in KH + KTT");
  static_assert((64 + 32) * kLd * 4 <= 32768, "solve scratch must fit in KH");
  static_assert(16 * 128 * 4 <= DV * 256, "decay totals must fit in VT");
};

template <int DV>
struct Tmem {
  static constexpr uint32_t kCols = (128 + 3 * DV) <= 256 ? 256u : 512u;
  static constexpr uint32_t kD0 = 0;                 // [A; P], then [W; -]   (128 cols)
  static constexpr uint32_t kD1 = 128;               // [-W S; Qt S] -> O     (DV cols)
  static constexpr uint32_t kD2 = 128 + DV;          // the state S (+= Kh^T U) (DV cols)
  static constexpr uint32_t kD3 = 128 + 2 * DV;      // [U~; -]               (DV cols)
};

// kConv: q, k, v are the raw inputs of the full mixer; the kernel applies the causal
// depthwise conv of width 4 (zero history at each sequence start) to all three and
// the L2 norm x / sqrt(sum x^2 + 1e-6) to q and k, in fp32, before the recurrence.
template <int DV, typename TIn, typename TOut, bool kConv>
__global__ void __launch_bounds__(kThreads, 1)
    kda_prefill_kernel(const __grid_constant__ CUtensorMap tm_v, const PrefillArgs a) {
  using SM = Smem<DV>;
  using TM = Tmem<DV>;
  constexpr int kSlices = kD / DV;
  constexpr int kPart = DV / 4;          // value columns per warp in the TMEM epilogues
  constexpr int kHist = kConv ? 3 : 0;   // tokens of history the conv needs
  constexpr int kVRows = kChunk + kHist; // rows of the V tile brought by TMA
  constexpr int kGRows = 4 + kHist;      // q/k rows each thread loads in the gate pass
  static_assert(kVRows * DV * sizeof(TIn) <= 32768, "V staging must fit in the TP region");

  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sb = smem_u32(sm);
  float* sA = reinterpret_cast<float*>(sm + SM::kScratch);    // [64][kLd]: A, then X in place
  float* sY = sA + 64 * kLd;                                  // [32][kLd]
  float* sBeta = reinterpret_cast<float*>(sm + SM::kBeta);
  float* sGamma = reinterpret_cast<float*>(sm + SM::kGamma);  // [2][128]
  float* sTot = reinterpret_cast<float*>(sm + SM::kTot);      // [16][128]
  uint64_t* bar_mma = reinterpret_cast<uint64_t*>(sm + SM::kBar);
  uint64_t* bar_tma = bar_mma + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + SM::kTmemSlot);

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int lq = warp & 3;          // TMEM lane quarter this warp may access
  const int cp = warp >> 2;         // which quarter of a row's columns this warp handles
  const int row = lq * 32 + lane;   // TMEM lane = accumulator row of this thread
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
  if (tid < 128) sGamma[128 + tid] = 1.f;  // "previous chunk" scale for the first chunk
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = *tmem_slot;
  const uint32_t lane_off = static_cast<uint32_t>(lq * 32) << 16;

  // ---- the state slice lives in TMEM (D2): lane c = key row c, DV columns ----------
  {
    const float* h0 = a.h0 ? a.h0 + ((static_cast<size_t>(n) * H + h) * kD + row) * kD + col0 : nullptr;
#pragma unroll
    for (int j = 0; j < kPart; j += 8) {
      const int c = cp * kPart + j;
      float x[8];
      if (h0) {
        const float4 u = *reinterpret_cast<const float4*>(h0 + c);
        const float4 w = *reinterpret_cast<const float4*>(h0 + c + 4);
        x[0] = u.x; x[1] = u.y; x[2] = u.z; x[3] = u.w; x[4] = w.x; x[5] = w.y; x[6] = w.z; x[7] = w.w;
      } else {
#pragma unroll
        for (int e = 0; e < 8; ++e) x[e] = 0.f;
      }
      tmem_st8(tmem + lane_off + TM::kD2 + c, x);
    }
    tmem_st_wait();
  }

  const TIn* __restrict__ qg = static_cast<const TIn*>(a.q);
  const TIn* __restrict__ kg = static_cast<const TIn*>(a.k);
  const float* __restrict__ lag = a.log_alpha;
  const __nv_bfloat16* gateg = static_cast<const __nv_bfloat16*>(a.gate);
  TOut* outg = static_cast<TOut*>(a.out);
  const int64_t tok_stride = static_cast<int64_t>(H) * kD;  // elements between tokens

  constexpr uint32_t kIdAP = idesc_tf32(128, 64, false, false);
  constexpr uint32_t kIdW = idesc_tf32(128, 128, false, true);
  constexpr uint32_t kIdVb = idesc_tf32(128, DV, false, true);   // B = V (MN-major)
  constexpr uint32_t kIdV = idesc_tf32(128, DV, false, false);   // B = S^T, U^T (K-major)
  constexpr uint32_t kIdVmn = idesc_tf32(128, DV, true, false);  // A = Kh^T (MN-major)

  uint32_t mma_phase = 0, tma_phase = 0;
  bool failed = false;
  int gslot = 1;  // sGamma slot of the last chunk's e^{g_last} (slot 1 holds 1.0 initially)

  // Every thread waits for the last commit on its own. A wait that runs out of time
  // raises the status flag and marks this thread; the CTA agrees on it once per chunk
  // and stops (after draining the tensor pipe, see the teardown).
  bool lost = false;
  auto wait_mma = [&]() {
    if (!lost && !mbar_wait(bar_mma, mma_phase, a.status)) lost = true;
    mma_phase ^= 1u;
    tc_fence_after_sync();
  };

  // Gate inputs of one chunk for this thread (warp w: tokens 4w..4w+3, lane l: key
  // channels 4l..4l+3). The next chunk's are loaded while this chunk's MMAs run.
  const int c0 = lane * 4, r0 = warp * 4;
  float4 la4[4];   // raw loads, masked where used (keeps the loads in flight)
  uint32_t kraw[kGRows][sizeof(TIn)], qraw[kGRows][sizeof(TIn)];  // 4 elements: 2 words (bf16) or 4 (fp32)
  auto load_gate = [&](int64_t tc, int lc) {
    // q/k row m is chunk row r0 - kHist + m; rows outside [bos, tc + lc) read row tc
    // (always in bounds) and are replaced by zero where used
#pragma unroll
    for (int m = 0; m < kGRows; ++m) {
      const int rr = r0 - kHist + m;
      const bool in = rr < lc && tc + rr >= bos;
      const size_t o = static_cast<size_t>(in ? tc + rr : tc) * tok_stride + static_cast<size_t>(h) * kD + c0;
      if constexpr (sizeof(TIn) == 2) {
        const uint2 kk2 = __ldg(reinterpret_cast<const uint2*>(kg + o));
        const uint2 qq2 = __ldg(reinterpret_cast<const uint2*>(qg + o));
        kraw[m][0] = kk2.x; kraw[m][1] = kk2.y; qraw[m][0] = qq2.x; qraw[m][1] = qq2.y;
      } else {
        const uint4 kk4 = __ldg(reinterpret_cast<const uint4*>(kg + o));
        const uint4 qq4 = __ldg(reinterpret_cast<const uint4*>(qg + o));
        kraw[m][0] = kk4.x; kraw[m][1] = kk4.y; kraw[m][2] = kk4.z; kraw[m][3] = kk4.w;
        qraw[m][0] = qq4.x; qraw[m][1] = qq4.y; qraw[m][2] = qq4.z; qraw[m][3] = qq4.w;
      }
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const bool in = r0 + i < lc;
      const size_t o = static_cast<size_t>(tc + (in ? r0 + i : 0)) * tok_stride + static_cast<size_t>(h) * kD + c0;
      la4[i] = __ldg(reinterpret_cast<const float4*>(lag + o));
    }
  };
  // element e (0..3) of a raw 4-element load
  auto unpack = [&](const uint32_t* w, int e) -> float {
    if constexpr (sizeof(TIn) == 2) {
      const uint32_t x = w[e >> 1];
      return __uint_as_float((e & 1) ? (x & 0xFFFF0000u) : (x << 16));
    } else {
      return __uint_as_float(w[e]);
    }
  };
  if (bos < eos) load_gate(bos, static_cast<int>(eos - bos < kChunk ? eos - bos : kChunk));

  for (int64_t t0 = bos; t0 < eos && !failed; t0 += kChunk) {
    const int len = static_cast<int>(eos - t0 < kChunk ? eos - t0 : kChunk);
    const int gnew = gslot ^ 1;  // slot for this chunk's e^{g_last}
    bool strong;                 // the chunk's decay passes kMaxChunkDecay in some channel

    // -- 1. V tile by TMA into the staging area (the TP region, free until step 5) -----
    if (tid == 0) {
      mbar_arrive_expect_tx(bar_tma, static_cast<uint32_t>(kVRows * DV * sizeof(TIn)));
      tma_load_3d(sm + SM::kStage, &tm_v, col0, h, static_cast<int>(t0) - kHist, bar_tma);
    }
    // warm L2 with the next chunk's q, k, log_alpha rows
    if (t0 + kChunk < eos && lane < 4) {
      const int64_t nt = t0 + kChunk;
      const int r = warp * 4 + lane;
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

    // -- 2. gates. Warp w takes tokens 4w..4w+3, lane l key channels 4l..4l+3 ----------
    {
      if (tid < 64) sBeta[tid] = tid < len ? __ldg(a.beta + (t0 + tid) * H + h) : 0.f;
      float la[4][4], kv[4][4], qv[4][4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const bool in = r0 + i < len;
        la[i][0] = in ? la4[i].x : 0.f; la[i][1] = in ? la4[i].y : 0.f;
        la[i][2] = in ? la4[i].z : 0.f; la[i][3] = in ? la4[i].w : 0.f;
      }
      if constexpr (kConv) {
        // y[t, c] = sum_j w[c, j] x[t - 3 + j, c] (x = 0 before the sequence start), then
        // x / sqrt(sum_c y^2 + 1e-6) over the head's 128 channels (this warp holds them all)
        float wq[4][4], wk[4][4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float4 a4 = __ldg(reinterpret_cast<const float4*>(a.conv_w + ((0 * H + h) * kD + c0 + e) * 4));
          const float4 b4 = __ldg(reinterpret_cast<const float4*>(a.conv_w + ((1 * H + h) * kD + c0 + e) * 4));
          wq[e][0] = a4.x; wq[e][1] = a4.y; wq[e][2] = a4.z; wq[e][3] = a4.w;
          wk[e][0] = b4.x; wk[e][1] = b4.y; wk[e][2] = b4.z; wk[e][3] = b4.w;
        }
        bool rin[kGRows];
#pragma unroll
        for (int m = 0; m < kGRows; ++m) rin[m] = (r0 - kHist + m) < len && t0 + (r0 - kHist + m) >= bos;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          float sq = 0.f, sk = 0.f;
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            float yq = 0.f, yk = 0.f;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const int m = i + j;
              yq = fmaf(wq[e][j], rin[m] ? unpack(qraw[m], e) : 0.f, yq);
              yk = fmaf(wk[e][j], rin[m] ? unpack(kraw[m], e) : 0.f, yk);
            }
            qv[i][e] = yq;
            kv[i][e] = yk;
            sq = fmaf(yq, yq, sq);
            sk = fmaf(yk, yk, sk);
          }
#pragma unroll
          for (int off = 16; off > 0; off >>= 1) {
            sq += __shfl_xor_sync(0xffffffffu, sq, off);
            sk += __shfl_xor_sync(0xffffffffu, sk, off);
          }
          const bool in = r0 + i < len;
          const float fq = in ? rsqrtf(sq + 1e-6f) : 0.f, fk = in ? rsqrtf(sk + 1e-6f) : 0.f;
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            qv[i][e] *= fq;
            kv[i][e] *= fk;
          }
        }
      } else {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const bool in = r0 + i < len;
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            kv[i][e] = in ? unpack(kraw[i], e) : 0.f;
            qv[i][e] = in ? unpack(qraw[i], e) : 0.f;
          }
        }
      }
      // running sums within this warp's 4 tokens, then the totals of the warps before it
      float tot[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int e = 0; e < 4; ++e) { tot[e] += la[i][e]; la[i][e] = tot[e]; }
      *reinterpret_cast<float4*>(sTot + warp * kD + c0) = make_float4(tot[0], tot[1], tot[2], tot[3]);
      __syncthreads();
      float pre[4] = {0.f, 0.f, 0.f, 0.f};
      for (int w = 0; w < warp; ++w) {
        const float4 t4 = *reinterpret_cast<const float4*>(sTot + w * kD + c0);
        pre[0] += t4.x; pre[1] += t4.y; pre[2] += t4.z; pre[3] += t4.w;
      }
      // the chunk's decay per channel decides its form: factorised (e^g, e^-g finite) or
      // the exact token walk
      float gl = 0.f;
      if (tid < 128) {
#pragma unroll
        for (int w = 0; w < 16; ++w) gl += sTot[w * kD + tid];
      }
      strong = __syncthreads_or(tid < 128 && -gl > kMaxChunkDecay) != 0;
      // e^{g_last} scales the state at the next chunk; after a walk the state is exact
      if (tid < 128) sGamma[gnew * 128 + tid] = strong ? 1.f : __expf(gl);
      if (strong) {  // k, q (after conv / L2) and the raw log_alpha, row-major, for the walk
        float* sKr = reinterpret_cast<float*>(sm + SM::kKQ);
        float* sLAr = reinterpret_cast<float*>(sm + SM::kKH);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int r = r0 + i;
          const bool in = r < len;
          *reinterpret_cast<float4*>(sKr + r * kD + c0) = make_float4(kv[i][0], kv[i][1], kv[i][2], kv[i][3]);
          *reinterpret_cast<float4*>(sKr + (64 + r) * kD + c0) = make_float4(qv[i][0], qv[i][1], qv[i][2], qv[i][3]);
          *reinterpret_cast<float4*>(sLAr + r * kD + c0) = in ? la4[i] : make_float4(0.f, 0.f, 0.f, 0.f);
        }
      } else {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          float kt[4], kh[4], qt[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float g = pre[e] + la[i][e];
            const float eg = __expf(g), eng = __expf(-g);
            kt[e] = kv[i][e] * eg;
            kh[e] = to_tf32(kv[i][e] * eng);
            qt[e] = qv[i][e] * eg;
          }
          const int r = r0 + i;
          st4_f32(sm + SM::kKQ, f32_offset(r, c0, 128), kt[0], kt[1], kt[2], kt[3]);           // Kt [tok][ch]
          st4_tf32(sm + SM::kKQ, f32_offset(64 + r, c0, 128), qt[0], qt[1], qt[2], qt[3]);     // Qt [tok][ch]
          st4_f32(sm + SM::kKH, f32_offset(r, c0, 64), kh[0], kh[1], kh[2], kh[3]);            // Kh [tok][ch]
          // the same rows as lines of the MN-major operands: Kt of T Kt, Kh (Kh^T) of Kh^T U
          st4_f32(sm + SM::kKTT, mn_offset(r, c0, 64), kt[0], kt[1], kt[2], kt[3]);
          st4_f32(sm + SM::kKHT, mn_offset(r, c0, 64), kh[0], kh[1], kh[2], kh[3]);
        }
      }  // factorised form
    }

    // -- 3. V landed: widen to fp32 operand lines (rows past the sequence end -> 0) --------
    {
      if (!lost && !mbar_wait(bar_tma, tma_phase, a.status)) lost = true;
      tma_phase ^= 1u;
      __syncthreads();  // every thread is done with the decay totals (they share V's space)
      const TIn* st = reinterpret_cast<const TIn*>(sm + SM::kStage);  // row m = token t0 - kHist + m
      for (int i = tid; i < DV * 16; i += kThreads) {
        const int j = i % DV, t4 = (i / DV) * 4;
        float x[4];
        if constexpr (kConv) {
          const float4 w4 = __ldg(reinterpret_cast<const float4*>(a.conv_w + ((2 * H + h) * kD + col0 + j) * 4));
          const float w[4] = {w4.x, w4.y, w4.z, w4.w};
          float xs[7];
#pragma unroll
          for (int m = 0; m < 7; ++m) xs[m] = (t0 - kHist + t4 + m >= bos) ? as_f32(st[(t4 + m) * DV + j]) : 0.f;
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            float y = 0.f;
#pragma unroll
            for (int tap = 0; tap < 4; ++tap) y = fmaf(w[tap], xs[e + tap], y);
            x[e] = (t4 + e < len) ? y : 0.f;
          }
        } else {
#pragma unroll
          for (int e = 0; e < 4; ++e) x[e] = (t4 + e < len) ? as_f32(st[(t4 + e) * DV + j]) : 0.f;
        }
        if (strong) {  // the walk reads V row-major in fp32
          float* vr = reinterpret_cast<float*>(sm + SM::kVT);
#pragma unroll
          for (int e = 0; e < 4; ++e) vr[(t4 + e) * DV + j] = x[e];
        } else {  // lines of the MN-major B operand of T V (a warp writes 32 columns of a token)
#pragma unroll
          for (int e = 0; e < 4; ++e) st_tf32(sm + SM::kVT, mn_offset(t4 + e, j, kChunk), x[e]);
        }
      }
    }
    fence_proxy_async_smem();
    __syncthreads();

    // -- a chunk the factorised form cannot carry: the exact token walk on the state slice --
    if (strong) {
      WalkArgs wa;
      wa.sK = reinterpret_cast<const float*>(sm + SM::kKQ);
      wa.sQ = wa.sK + 64 * kD;
      wa.sLA = reinterpret_cast<const float*>(sm + SM::kKH);
      wa.sBeta = sBeta;
      wa.sV = reinterpret_cast<const float*>(sm + SM::kVT);
      wa.scr = reinterpret_cast<float*>(sm + SM::kKTT);
      wa.sST = nullptr;
      wa.out = outg + static_cast<size_t>(t0) * tok_stride + static_cast<size_t>(h) * kD + col0;
      wa.gate = gateg ? gateg + static_cast<size_t>(t0) * tok_stride + static_cast<size_t>(h) * kD + col0 : nullptr;
      wa.out_stride = tok_stride;
      wa.tmem_state = tmem + lane_off + TM::kD2;
      wa.scale = sGamma[gslot * 128 + row];  // the true state is e^{g_last}(prev) * D2
      wa.len = len;
      walk_chunk<DV, TOut>(wa);
      if (t0 + kChunk < eos) {  // next chunk's gate inputs
        const int64_t nt = t0 + kChunk;
        load_gate(nt, static_cast<int>(eos - nt < kChunk ? eos - nt : kChunk));
      }
      gslot = gnew;
      tc_fence_before_sync();
      failed = cta_any(lost);
      tc_fence_after_sync();
      continue;
    }

    // -- 4. D0 = [A_raw; P_raw] = [Kt; Qt] Kh^T --------------------------------------------
    if (tid == 0) {
      tc_fence_after_sync();
      const uint64_t a0 = kdesc0(sb + SM::kKQ), b0 = kdesc0(sb + SM::kKH);
#pragma unroll
      for (int kk = 0; kk < 16; ++kk)
        umma_tf32(tmem + TM::kD0, a0 + kstep(kk, 128), b0 + kstep(kk, 64), kIdAP, kk > 0);
      umma_commit(bar_mma);
    }
    wait_mma();

    // -- 5. A (rows 0..63: beta-scaled, strictly lower), P (rows 64..127: lower) ---------
    {
      const int cb = cp * 16;
      float d[16];
      tmem_ld16(tmem + lane_off + TM::kD0 + cb, d);
      tmem_ld_wait();
      if (lq < 2) {
        const int r = row;
        const float br = sBeta[r];
#pragma unroll
        for (int i = 0; i < 16; i += 4) {
          const int c = cb + i;
          *reinterpret_cast<float4*>(sA + r * kLd + c) =
              make_float4(c < r ? br * d[i] : 0.f, c + 1 < r ? br * d[i + 1] : 0.f, c + 2 < r ? br * d[i + 2] : 0.f,
                          c + 3 < r ? br * d[i + 3] : 0.f);
        }
      } else {
        const int r = row - 64;
#pragma unroll
        for (int i = 0; i < 16; i += 4) {
          const int c = cb + i;
          st4_tf32(sm + SM::kTP, f32_offset(64 + r, c, 128), c <= r ? d[i] : 0.f, c + 1 <= r ? d[i + 1] : 0.f,
                   c + 2 <= r ? d[i + 2] : 0.f, c + 3 <= r ? d[i + 3] : 0.f);
        }
      }
    }
    tc_fence_before_sync();
    __syncthreads();

    // -- 6. X = (I + A)^-1 in fp32 (in place over A), T = X Diag(beta) ---------------------
    invert_unit_lower_64(sA, sY);
    {  // T row r, columns 8*part .. +7
      const int r = tid & 63, c = (tid >> 6) * 8;
#pragma unroll
      for (int i = c; i < c + 8; i += 4) {
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
      const uint64_t a0 = kdesc0(sb + SM::kTP);
#pragma unroll
      for (int kk = 0; kk < 8; ++kk)
        umma_tf32(tmem + TM::kD0, a0 + kstep(kk, 128), mndesc(sb + SM::kKTT, kChunk, kk), kIdW, kk > 0);
#pragma unroll
      for (int kk = 0; kk < 8; ++kk)
        umma_tf32(tmem + TM::kD3, a0 + kstep(kk, 128), mndesc(sb + SM::kVT, kChunk, kk), kIdVb, kk > 0);
      umma_commit(bar_mma);
    }
    wait_mma();

    // -- 8. -W -> rows 0..63 of KQ (over Kt);  S <- e^{g_last}(previous chunk) S in TMEM
    //       and as the S^T operand -------------------------------------------------------
    if (lq < 2) {
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const int cb = cp * 32 + 16 * j;
        float w[16];
        tmem_ld16(tmem + lane_off + TM::kD0 + cb, w);
        tmem_ld_wait();
#pragma unroll
        for (int e = 0; e < 16; e += 4)
          st4_f32(sm + SM::kKQ, f32_offset(row, cb + e, 128), -w[e], -w[e + 1], -w[e + 2], -w[e + 3]);
      }
    }
    {
      const float gm = sGamma[gslot * 128 + row];
#pragma unroll
      for (int j = 0; j < kPart; j += 8) {
        const int c = cp * kPart + j;
        float x[8];
        tmem_ld8(tmem + lane_off + TM::kD2 + c, x);
        tmem_ld_wait();
#pragma unroll
        for (int e = 0; e < 8; ++e) x[e] *= gm;
#pragma unroll
        for (int e = 0; e < 8; ++e) *reinterpret_cast<float*>(sm + SM::kST + f32_offset(c + e, row, DV)) = x[e];
        tmem_st8(tmem + lane_off + TM::kD2 + c, x);
      }
      tmem_st_wait();
    }
    fence_proxy_async_smem();
    tc_fence_before_sync();
    __syncthreads();

    // -- 9. D1 = [-W S; Qt S] ----------------------------------------------------------------
    if (tid == 0) {
      tc_fence_after_sync();
      const uint64_t a0 = kdesc0(sb + SM::kKQ);
#pragma unroll
      for (int kk = 0; kk < 16; ++kk)
        umma_tf32(tmem + TM::kD1, a0 + kstep(kk, 128), kdesc0(sb + SM::kST) + kstep(kk, DV), kIdV, kk > 0);
      umma_commit(bar_mma);
    }
    if (t0 + kChunk < eos) {  // next chunk's gate inputs, in flight during the MMAs
      const int64_t nt = t0 + kChunk;
      load_gate(nt, static_cast<int>(eos - nt < kChunk ? eos - nt : kChunk));
    }
    wait_mma();

    // -- 10. U = U~ - W S -> U^T operand (over V) -----------------------------------------------
    if (lq < 2) {
#pragma unroll
      for (int j = 0; j < kPart; j += 8) {
        const int c = cp * kPart + j;
        float ut[8], ws[8];
        tmem_ld8(tmem + lane_off + TM::kD3 + c, ut);
        tmem_ld8(tmem + lane_off + TM::kD1 + c, ws);
        tmem_ld_wait();
#pragma unroll
        for (int e = 0; e < 8; ++e) st_tf32(sm + SM::kVT, f32_offset(c + e, row, DV), ut[e] + ws[e]);
      }
    }
    fence_proxy_async_smem();
    tc_fence_before_sync();
    __syncthreads();

    // -- 11. D2 = S + Kh^T U ;  D1 += [T; P] U  ->  O = Qt S + P U in rows 64..127 ------------
    if (tid == 0) {
      tc_fence_after_sync();
      const uint64_t t0d = kdesc0(sb + SM::kTP);
#pragma unroll
      for (int kk = 0; kk < 8; ++kk)
        umma_tf32(tmem + TM::kD2, mndesc(sb + SM::kKHT, kChunk, kk), kdesc0(sb + SM::kVT) + kstep(kk, DV), kIdVmn, 1u);
#pragma unroll
      for (int kk = 0; kk < 8; ++kk)
        umma_tf32(tmem + TM::kD1, t0d + kstep(kk, 128), kdesc0(sb + SM::kVT) + kstep(kk, DV), kIdV, 1u);
      umma_commit(bar_mma);
    }
    wait_mma();
    gslot = gnew;

    // -- 12. out rows <- O (* sigmoid(gate)) ------------------------------------------------------
    if (lq >= 2) {
      const int r = row - 64;
#pragma unroll
      for (int j = 0; j < kPart; j += 8) {
        const int c = cp * kPart + j;
        float o[8];
        tmem_ld8(tmem + lane_off + TM::kD1 + c, o);
        tmem_ld_wait();
        if (r < len) {
          const size_t off = static_cast<size_t>(t0 + r) * tok_stride + static_cast<size_t>(h) * kD + col0 + c;
          if (gateg) {
            const uint4 g0 = *reinterpret_cast<const uint4*>(gateg + off);
            const __nv_bfloat16* gb0 = reinterpret_cast<const __nv_bfloat16*>(&g0);
#pragma unroll
            for (int i = 0; i < 8; ++i) o[i] *= 1.f / (1.f + __expf(-bf2f(gb0[i])));
          }
          store8(outg + off, o);
        }
      }
    }
    tc_fence_before_sync();
    failed = cta_any(lost);
  }

  // ---- final state: e^{g_last} of the last chunk times D2 --------------------------------
  const int64_t hn = a.ht ? final_state_index(a, n, tid == 0) : -1;
  if (!failed && hn >= 0) {
    const float gm = sGamma[gslot * 128 + row];
    float* ht = a.ht + ((static_cast<size_t>(hn) * H + h) * kD + row) * kD + col0;
#pragma unroll
    for (int j = 0; j < kPart; j += 8) {
      const int c = cp * kPart + j;
      float x[8];
      tmem_ld8(tmem + lane_off + TM::kD2 + c, x);
      tmem_ld_wait();
      *reinterpret_cast<float4*>(ht + c) = make_float4(gm * x[0], gm * x[1], gm * x[2], gm * x[3]);
      *reinterpret_cast<float4*>(ht + c + 4) = make_float4(gm * x[4], gm * x[5], gm * x[6], gm * x[7]);
    }
  }

  // ---- teardown: after a lost wait, let the tensor pipe and the TMA unit drain (bounded)
  //      before the TMEM goes back -------------------------------------------------------
  if (failed && tid == 0) {
    umma_commit(bar_mma);
    mbar_wait(bar_mma, mma_phase, a.status);
    mbar_wait(bar_tma, tma_phase, a.status);
  }
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

template <int DV, typename TIn, typename TOut, bool kConv>
cudaError_t launch_dv(const PrefillArgs& a, cudaStream_t stream) {
  CUtensorMap tm;
  if (!encode_value_map(&tm, a.v, a.total_T, a.H, DV, kChunk + (kConv ? 3 : 0), sizeof(TIn) == 4))
    return cudaErrorInvalidValue;
  auto kern = kda_prefill_kernel<DV, TIn, TOut, kConv>;
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

template <typename TIn, typename TOut, bool kConv>
cudaError_t launch_types(const PrefillArgs& a, cudaStream_t stream) {
  // value-column slices per chain: split when there are few (sequence, head) chains,
  // as far as a single wave of CTAs over the 148 SMs allows (one CTA per SM)
  const int64_t chains = static_cast<int64_t>(a.N) * a.H;
  if (4 * chains <= 148) return launch_dv<32, TIn, TOut, kConv>(a, stream);
  if (2 * chains <= 148) return launch_dv<64, TIn, TOut, kConv>(a, stream);
  return launch_dv<128, TIn, TOut, kConv>(a, stream);
}

}  // namespace

cudaError_t launch_prefill_d128(const PrefillArgs& a, cudaStream_t stream) {
  if (a.N == 0) return cudaSuccess;
  if (a.total_T == 0) {
    if (!a.ht || a.slots) return cudaSuccess;  // pooled states: launch_pool_store copies them
    const size_t n4 = static_cast<size_t>(a.N) * a.H * kD * kD / 4;
    copy_states_kernel<<<static_cast<unsigned>((n4 + 255) / 256 < 4096 ? (n4 + 255) / 256 : 4096), 256, 0, stream>>>(
        a.h0, a.ht, n4);
    return cudaGetLastError();
  }
  if (a.split_ws) return launch_prefill_split(a, stream);
  if (a.a_pre) return cudaErrorInvalidValue;  // the pre-activation gate has only the two-pass form
  if (a.conv_w) {  // the fused full mixer: raw bf16 q/k/v, bf16 out
    if (a.in_f32 || a.out_f32) return cudaErrorInvalidValue;
    return launch_types<__nv_bfloat16, __nv_bfloat16, true>(a, stream);
  }
  if (!a.in_f32) return a.out_f32 ? cudaErrorInvalidValue : launch_types<__nv_bfloat16, __nv_bfloat16, false>(a, stream);
  return a.out_f32 ? launch_types<float, float, false>(a, stream) : launch_types<float, __nv_bfloat16, false>(a, stream);
}

}  // namespace kda
