// kda_split.cu — chunked KDA prefill in two passes on sm_100a tensor cores.
//
// The recurrence (Ling-3.0-flash article, section "KDA: constant-size memory over a
// very long context"):  S_t = (I - b_t k_t k_t^T) Diag(a_t) S_{t-1} + b_t k_t v_t^T,
// o_t = S_t^T q_t. Chunked form (64-token chunks; g = running sum of log_alpha within
// the chunk):
//   Kt = K*e^g,  Qt = Q*e^g,  Kh = K*e^-g
//   A  = strict_lower(Kt Kh^T) scaled by beta on rows,  P = lower(Qt Kh^T)
//   T  = (I + A)^-1 Diag(beta),  W = T Kt,  U~ = T V
//   U  = U~ - W S,   O = Qt S + P U,   S' = Diag(e^g_last) (S + Kh^T U)
// Only the last three lines depend on the state S; everything above them is
// independent across chunks. So the work is split:
//
//   plan  (kda_plan_kernel): cu_seqlens -> first global chunk index of each sequence;
//   pass 1 (kda_intra_kernel): persistent CTAs walk every (chunk, head) of the batch.
//     Computes the state-free part and writes one item per (chunk, head):
//       [-W; Qt]  128 x 128 fp32 tile   (A operand of D1 = [-W; Qt] S, K-major)
//       P         rows 64..127 of a 128 x 64 tile (A operand of D1 += [.; P] U, K-major)
//       Kh        64 token lines of 128 channels: the MN-major A operand Kh^T of
//                 D2 += Kh^T U (128B swizzle with 32-byte atoms)
//       U~        64 x 128 fp32 (64-row swizzled layout, read back row by row)
//       e^g_last  128 fp32
//     The three tiles are written in the exact layouts the MMAs read, so pass 2 moves
//     them into shared memory with plain bulk copies;
//   pass 2 (kda_recur_kernel): one CTA per (sequence, head, slice of DV value columns)
//     walks its chunks in order with the fp32 state slice in TMEM. Per chunk:
//       group 1:  D1 = [-W; Qt] S                         (M128 NDV K128)
//       U = U~ + D1[0:64] -> U^T operand (tf32)
//       group 2:  D2 += Kh^T U ;  D1 += [.; P] U          (M128 NDV K64, twice)
//       S <- e^g_last * D2 (TMEM and the S^T operand);  O = D1[64:128] -> out
//     D1 alternates between two TMEM buffers so that a chunk's output rows are read
//     while the next chunk's first MMA group runs; the next chunk's tiles are bulk-
//     loaded as soon as the MMA that read the previous ones has completed.
//
// Precision: operands are fp32 in shared memory read as tf32 by kind::tf32 MMAs, with
// fp32 accumulation; the operands whose truncation would cost accuracy (Qt, Kh, P, T,
// V, U) are rounded to nearest tf32 when written. The 64x64 inverse is fp32-accurate.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "kda_tile.cuh"

namespace kda {

namespace {

// ---- item layout (bytes from the start of one (chunk, head) item) ------------------
constexpr uint32_t kItemQW = 0;          // [-W; Qt] tile, 64 KB
constexpr uint32_t kItemP = 65536;       // P: rows 64..127 of K blocks 0 and 1, 2 x 8 KB
constexpr uint32_t kItemKHT = 81920;     // Kh (the MN-major A operand Kh^T), 32 KB
constexpr uint32_t kItemU = 114688;      // U~ 64 x 128 fp32 in the 64-row tile layout, 32 KB
constexpr uint32_t kItemGamma = 147456;  // e^g_last [128] fp32
static_assert(kItemGamma + 512 == kItemBytes, "item layout");

struct SplitPlan {
  const int32_t* chunk_start;  // [N + 1]: first global chunk of each sequence; [N] = total (-1: bad seqlens)
  int32_t* any_raw;            // set by pass 1 when it hands any item over as raw rows (cleared by the plan)
  uint8_t* items;              // [chunks][H] items of kItemBytes
};

// ================================ plan ===============================================
// One block of 1024 threads: per-sequence chunk counts, exclusive scan.
__global__ void __launch_bounds__(1024) kda_plan_kernel(const int32_t* __restrict__ cu, int64_t total_T, int N,
                                                        int32_t* __restrict__ cs, uint32_t* status) {
  __shared__ int32_t s_scan[1024];
  __shared__ int32_t s_carry;
  __shared__ int s_bad;
  const int tid = threadIdx.x;
  if (tid == 0) {
    s_carry = 0;
    s_bad = 0;
  }
  __syncthreads();
  for (int base = 0; base < N; base += 1024) {
    const int n = base + tid;
    int32_t c = 0;
    if (n < N) {
      int64_t bos, eos;
      if (cu) {
        bos = cu[n];
        eos = cu[n + 1];
      } else {
        const int64_t L = total_T / N;
        bos = static_cast<int64_t>(n) * L;
        eos = bos + L;
      }
      if (bos < 0 || eos < bos || eos > total_T || (n == 0 && bos != 0) || (n == N - 1 && eos != total_T))
        s_bad = 1;
      else
        c = static_cast<int32_t>((eos - bos + kChunk - 1) / kChunk);
    }
    s_scan[tid] = c;
    __syncthreads();
    for (int off = 1; off < 1024; off <<= 1) {  // inclusive Hillis-Steele scan
      const int32_t x = tid >= off ? s_scan[tid - off] : 0;
      __syncthreads();
      s_scan[tid] += x;
      __syncthreads();
    }
    if (n < N) cs[n] = s_carry + s_scan[tid] - c;
    __syncthreads();
    if (tid == 1023) s_carry += s_scan[1023];
    __syncthreads();
  }
  if (tid == 0) {
    cs[N] = s_bad ? -1 : s_carry;
    cs[N + 1] = 0;  // no item handed over as raw rows yet (pass 1 sets it)
    if (s_bad) atomicOr(status, kFlagBadSeqlens);
  }
}

// ================================ pass 1 =============================================
// Persistent: each CTA walks the items it = blockIdx.x + k * gridDim.x (item = global
// chunk it / H, head it % H). Two warp groups work on consecutive items at once:
//   front (warps 0..7):  gate inputs, [Kt; Qt] and Kh, the [A; P] MMA, Kt (and V) as
//                        MN-major operand lines                                   (item k+1)
//   back  (warps 8..15): A and P out of TMEM, the triangular inverse, T into TMEM (V for
//                        the mixer),
//                        the W / U~ MMA with A read from TMEM, -W, U~, P into the item (item k)
// Each buffer the groups share is handed over through an mbarrier (bounded waits).
constexpr int kIntraThreads = 512;
constexpr int kGroupThreads = 256;
constexpr uint32_t kBarFront = 1, kBarBack = 2;  // named barrier ids of the two groups

//  region  size     holds
//  KQ      64 KB    [Kt; Qt] (128 x 128); the gate pass's decay totals first     (front)
//  KH      32 KB    Kh (64 tok x 128 ch); the mixer's decay running sums first   (front)
//  KTT     32 KB    Kt as MN-major lines (64 tok x 128 ch): front writes, back's W MMA
//                   reads; then staged -W
//  VT      32 KB    V as MN-major lines (64 tok x 128 dv), then staged U~
//  KHT     32 KB    Kh as MN-major lines, staged for the bulk store into the item (front)
//  SCR     25.5 KB  inverse scratch: A/X [64][kLd] + Y [32][kLd]                  (back)
//  CONVW   4 KB     the mixer's q, k conv taps of the item's head                 (front)
struct IntraSmem {
  static constexpr int kKQ = 0;
  static constexpr int kKH = 65536;
  static constexpr int kKTT = 98304;
  static constexpr int kVT = 131072;
  static constexpr int kKHT = 163840;
  static constexpr int kScr = 196608;
  static constexpr int kTot = kKQ;                   // [16][128] fp32
  static constexpr int kBeta = kScr + 96 * kLd * 4;  // fp32 [2][64]
  static constexpr int kBar = kBeta + 512;
  static constexpr int kNumBars = 8;
  static constexpr int kTmemSlot = kBar + 8 * kNumBars;
  static constexpr int kStrong = kTmemSlot + 16;     // int [2]: the item is walked token by token
  static constexpr int kConvW = kStrong + 16;       // fp32 [2][4][128]: q, k conv taps (tap, channel)
  static constexpr int kTotal = kConvW + 4096;
  static constexpr int kAlloc = kTotal + 1024;
  static_assert(kAlloc <= 232448, "shared memory plan exceeds the per-block limit");
};
enum : int {
  kBApFull = 0,  // [A; P] MMA done: back may read it, front may rewrite KQ / KH   (commit)
  kBApFree,      // back has read [A; P] out of TMEM                                (back arrives)
  kBVtFull,      // front has written Kt (and V)                                    (front arrives)
  kBWuDone,      // W / U~ MMA done                                                 (commit)
  kBWFree,       // back is done with KTT (W MMA read it, staged -W stored from it)  (back arrives)
  kBDrain        // teardown after a lost wait
};
constexpr uint32_t kTmAP = 0;    // D [A; P]             64 columns
constexpr uint32_t kTmT = 64;    // A operand T (rows 0..63), 64 columns
constexpr uint32_t kTmW = 128;   // D [W; -]             128 columns
constexpr uint32_t kTmU = 256;   // D [U~; -]            128 columns
constexpr uint32_t kTmP = 384;   // P kept for the epilogue (rows 64..127), 64 columns
constexpr uint32_t kIntraCols = 512;

// position of one item
struct ItemPos {
  int64_t t0, bos;
  int len, h;
  uint8_t* item;
};
__device__ __forceinline__ ItemPos item_pos(int64_t it, const PrefillArgs& a, const SplitPlan& p) {
  ItemPos o;
  const int gch = static_cast<int>(it / a.H);
  o.h = static_cast<int>(it % a.H);
  int lo = 0, hi = a.N - 1;  // sequence: the last n with chunk_start[n] <= gch
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (__ldg(p.chunk_start + mid) <= gch) lo = mid; else hi = mid - 1;
  }
  int64_t eos;
  if (a.cu) {
    o.bos = __ldg(a.cu + lo);
    eos = __ldg(a.cu + lo + 1);
  } else {
    const int64_t L = a.total_T / a.N;
    o.bos = static_cast<int64_t>(lo) * L;
    eos = o.bos + L;
  }
  o.t0 = o.bos + static_cast<int64_t>(gch - __ldg(p.chunk_start + lo)) * kChunk;
  o.len = static_cast<int>(eos - o.t0 < kChunk ? eos - o.t0 : kChunk);
  o.item = p.items + static_cast<size_t>(it) * kItemBytes;
  return o;
}

// ---- raw rows of an item handed to the recurrence's token walk ----------------------
// Out of line: the rare path, kept away from the register allocation and the
// instruction footprint of the factorised pass.
struct RawRowsFront {
  const void* q;
  const void* k;
  const float* log_alpha;
  const void* a_pre;
  const float* a_scale;
  const float* conv_w;
  uint8_t* item;
  int64_t t0, bos;
  int len, h, H, fw;
};
// One warp of the front group: chunk rows 8 fw .. 8 fw + 7, lane l = key channels 4l .. 4l+3.
// Writes k and q (after the conv and L2 norm for the mixer) into the item's [-W; Qt] space
// as [64][128] fp32 each, and the raw log_alpha into its Kh^T space; rows past the chunk
// are zero.
template <typename TIn, bool kConv, bool kPre>
__device__ __noinline__ void raw_rows_front(const RawRowsFront r) {
  const int lane = threadIdx.x & 31, c0 = lane * 4;
  const TIn* qg = static_cast<const TIn*>(r.q);
  const TIn* kg = static_cast<const TIn*>(r.k);
  const int64_t ts = static_cast<int64_t>(r.H) * kD;
  const size_t hc = static_cast<size_t>(r.h) * kD + c0;
  float* ik = reinterpret_cast<float*>(r.item + kItemQW);
  float* il = reinterpret_cast<float*>(r.item + kItemKHT);
  for (int i = 0; i < 8; ++i) {
    const int t = 8 * r.fw + i;
    const bool in = t < r.len;  // uniform over the warp
    float kv[4] = {0.f, 0.f, 0.f, 0.f}, qv[4] = {0.f, 0.f, 0.f, 0.f}, l[4] = {0.f, 0.f, 0.f, 0.f};
    if (in) {
      if constexpr (kConv) {  // y = sum_j w[c, j] x[t - 3 + j, c], zero before the sequence start
        for (int j = 0; j < 4; ++j) {
          const int64_t tt = r.t0 + t - 3 + j;
          if (tt < r.bos) continue;
          float xq[4], xk[4];
          ld4_in(qg + static_cast<size_t>(tt) * ts + hc, xq);
          ld4_in(kg + static_cast<size_t>(tt) * ts + hc, xk);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            qv[e] = fmaf(__ldg(r.conv_w + ((0 * r.H + r.h) * kD + c0 + e) * 4 + j), xq[e], qv[e]);
            kv[e] = fmaf(__ldg(r.conv_w + ((1 * r.H + r.h) * kD + c0 + e) * 4 + j), xk[e], kv[e]);
          }
        }
      } else {
        ld4_in(qg + static_cast<size_t>(r.t0 + t) * ts + hc, qv);
        ld4_in(kg + static_cast<size_t>(r.t0 + t) * ts + hc, kv);
      }
      if constexpr (kPre) {  // log alpha = -scale * softplus(a)
        const float sc = __ldg(r.a_scale + r.h);
        float x[4];
        ld4_in(static_cast<const __nv_bfloat16*>(r.a_pre) + static_cast<size_t>(r.t0 + t) * ts + hc, x);
#pragma unroll
        for (int e = 0; e < 4; ++e) l[e] = -sc * softplus_fast(x[e]);
      } else {
        ld4_in(r.log_alpha + static_cast<size_t>(r.t0 + t) * ts + hc, l);
      }
    }
    if constexpr (kConv) {  // x / sqrt(sum x^2 + 1e-6) over the head's 128 channels (the warp holds them)
      float sq = 0.f, sk = 0.f;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        sq = fmaf(qv[e], qv[e], sq);
        sk = fmaf(kv[e], kv[e], sk);
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) {
        sq += __shfl_xor_sync(0xffffffffu, sq, off);
        sk += __shfl_xor_sync(0xffffffffu, sk, off);
      }
      const float fq = rsqrtf(sq + 1e-6f), fk = rsqrtf(sk + 1e-6f);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        qv[e] *= fq;
        kv[e] *= fk;
      }
    }
    *reinterpret_cast<float4*>(ik + t * kD + c0) = make_float4(kv[0], kv[1], kv[2], kv[3]);
    *reinterpret_cast<float4*>(ik + (64 + t) * kD + c0) = make_float4(qv[0], qv[1], qv[2], qv[3]);
    *reinterpret_cast<float4*>(il + t * kD + c0) = make_float4(l[0], l[1], l[2], l[3]);
  }
}

struct RawRowsBack {
  const void* v;
  const float* conv_w;
  uint8_t* item;
  int64_t t0, bos;
  int len, h, H, btid;
};
// The back group (256 threads): v rows (after the conv for the mixer) into the item's U~
// space as [64][128] fp32; rows past the chunk are zero.
template <typename TIn, bool kConv>
__device__ __noinline__ void raw_rows_back(const RawRowsBack r) {
  const TIn* vh = static_cast<const TIn*>(r.v) + static_cast<size_t>(r.h) * kD;
  const int64_t ts = static_cast<int64_t>(r.H) * kD;
  float* iv = reinterpret_cast<float*>(r.item + kItemU);
  for (int idx = r.btid; idx < kChunk * 32; idx += 256) {  // (token, 4 value columns)
    const int t = idx >> 5, j4 = 4 * (idx & 31);
    float x[4] = {0.f, 0.f, 0.f, 0.f};
    if (t < r.len) {
      if constexpr (kConv) {
        for (int j = 0; j < 4; ++j) {
          const int64_t tt = r.t0 + t - 3 + j;
          if (tt < r.bos) continue;
          float xv[4];
          ld4_in(vh + static_cast<size_t>(tt) * ts + j4, xv);
#pragma unroll
          for (int e = 0; e < 4; ++e) x[e] = fmaf(__ldg(r.conv_w + ((2 * r.H + r.h) * kD + j4 + e) * 4 + j), xv[e], x[e]);
        }
      } else {
        ld4_in(vh + static_cast<size_t>(r.t0 + t) * ts + j4, x);
      }
    }
    *reinterpret_cast<float4*>(iv + t * kD + j4) = make_float4(x[0], x[1], x[2], x[3]);
  }
}

// kConv: q, k, v are the raw inputs of the full mixer; the causal depthwise conv of
// width 4 (zero history at each sequence start) is applied to all three and the L2
// norm x / sqrt(sum x^2 + 1e-6) to q and k, in fp32, before anything else.
// kPre: the decay gate arrives as its bf16 pre-activation and a per-head scale,
// log_alpha = -a_scale[h] * softplus(a_pre), made here as it is loaded.
template <typename TIn, bool kConv, bool kPre = false>
__global__ void __launch_bounds__(kIntraThreads, 1)
    kda_intra_kernel(const PrefillArgs a, const SplitPlan p) {
  using SM = IntraSmem;
  constexpr int kHist = kConv ? 3 : 0;    // tokens of history the conv needs
  constexpr int kGRows = 4 + kHist;       // q/k rows a thread loads per 4-token group
  // which group builds the V rows: the front one, except for the mixer, whose gate pass
  // (conv and L2 norm of q and k) already makes the front group the longer one
  constexpr bool kVFront = !kConv;
  // the conv's gate pass holds its taps and 7 raw rows per group in registers: the decay's
  // running sums wait in shared memory meanwhile, in the bytes of KH that the same thread's
  // Kh rows overwrite later (no other thread touches them in between)
  constexpr bool kParkLa = kConv;

  const int H = a.H;
  const int total_chunks = __ldg(p.chunk_start + a.N);
  if (total_chunks <= 0) return;  // nothing to do, or bad cu_seqlens (-1, flagged by the plan)
  const int64_t total_items = static_cast<int64_t>(total_chunks) * H;
  if (static_cast<int64_t>(blockIdx.x) >= total_items) return;
  const int n_mine = static_cast<int>((total_items - 1 - blockIdx.x) / gridDim.x + 1);

  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sb = smem_u32(sm);
  float* sBeta = reinterpret_cast<float*>(sm + SM::kBeta);  // [2][64]
  float* sTot = reinterpret_cast<float*>(sm + SM::kTot);    // [16][128]
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + SM::kBar);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + SM::kTmemSlot);
  int* sStrong = reinterpret_cast<int*>(sm + SM::kStrong);

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int lq = warp & 3;         // TMEM lane quarter this warp may access
  const int row = lq * 32 + lane;  // TMEM lane of this thread

  if (tid == 0) {
    for (int i = 0; i < SM::kNumBars; ++i) mbar_init(bars + i, 1);
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, kIntraCols);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = *tmem_slot;
  const uint32_t lane_off = static_cast<uint32_t>(lq * 32) << 16;
  const int64_t tok_stride = static_cast<int64_t>(H) * kD;

  bool lost = false;

  if (warp < 8) {
    // ================================= front group =================================
    const int fw = warp;  // tokens 8fw .. 8fw+7: two groups of 4 (grp = 2fw + s)
    const int ftid = tid;
    const int c0 = lane * 4;  // key channels c0 .. c0+3
    const TIn* __restrict__ qg = static_cast<const TIn*>(a.q);
    const TIn* __restrict__ kg = static_cast<const TIn*>(a.k);
    const TIn* __restrict__ vg = static_cast<const TIn*>(a.v);
    uint32_t ph_apfull = 0, ph_apfree = 0, ph_wfree = 0;
    auto fsync = [] { group_sync(kBarFront, kGroupThreads); };

    for (int k = 0; k < n_mine; ++k) {
      const int64_t it = blockIdx.x + static_cast<int64_t>(k) * gridDim.x;
      const ItemPos ip = item_pos(it, a, p);
      const int64_t t0 = ip.t0, bos = ip.bos;
      const int len = ip.len, h = ip.h;
      uint8_t* item = ip.item;
      float* sB = sBeta + (k & 1) * 64;

      // warm L2 with the next item's inputs (64 rows: 4 lines of log_alpha, 2 each of k, q, v)
      if (k + 1 < n_mine) {
        const ItemPos nx = item_pos(it + gridDim.x, a, p);
        const int r = ftid >> 2, part = ftid & 3;
        if (r < nx.len) {
          const size_t o = static_cast<size_t>(nx.t0 + r) * tok_stride + static_cast<size_t>(nx.h) * kD;
          constexpr int kLine = 128 / sizeof(TIn);  // elements per 128-B line
          if constexpr (kPre)
            prefetch_l2(static_cast<const __nv_bfloat16*>(a.a_pre) + o + (part & 1) * 64);
          else
            prefetch_l2(a.log_alpha + o + part * 32);
          prefetch_l2((part < 2 ? kg : qg) + o + (part & 1) * kLine);
          prefetch_l2(vg + o + (part & 1) * kLine + (part >> 1) * (sizeof(TIn) == 4 ? 2 * kLine : 0));
        }
      }
      // KQ (the totals' space) and KH are free once the previous [A; P] MMA is done. One
      // thread waits on each mbarrier; the group follows it through a named barrier.
      if (k > 0) {
        if (ftid == 0 && !lost && !mbar_wait(bars + kBApFull, ph_apfull, a.status)) lost = true;
        ph_apfull ^= 1u;
        fsync();
      }
      if (ftid < 64) sB[ftid] = ftid < len ? __ldg(a.beta + (t0 + ftid) * H + h) : 0.f;
      float4 wtap;  // the conv taps of channel ftid & 127 of q (ftid < 128) or k
      if constexpr (kConv)
        wtap = __ldg(reinterpret_cast<const float4*>(a.conv_w + (((ftid >> 7) * H + h) * kD + (ftid & 127)) * 4));

      // raw q/k rows of both 4-token groups, in flight together with log_alpha (no conv:
      // the conv's extra history rows are loaded per group below)
      uint32_t kpre[2][4][sizeof(TIn)], qpre[2][4][sizeof(TIn)];
      if constexpr (!kConv) {
#pragma unroll
        for (int s = 0; s < 2; ++s)
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int rr = 4 * (2 * fw + s) + i;
            const size_t o = static_cast<size_t>(rr < len ? t0 + rr : t0) * tok_stride + static_cast<size_t>(h) * kD + c0;
            if constexpr (sizeof(TIn) == 2) {
              const uint2 kk2 = __ldg(reinterpret_cast<const uint2*>(kg + o));
              const uint2 qq2 = __ldg(reinterpret_cast<const uint2*>(qg + o));
              kpre[s][i][0] = kk2.x; kpre[s][i][1] = kk2.y; qpre[s][i][0] = qq2.x; qpre[s][i][1] = qq2.y;
            } else {
              const uint4 kk4 = __ldg(reinterpret_cast<const uint4*>(kg + o));
              const uint4 qq4 = __ldg(reinterpret_cast<const uint4*>(qg + o));
              kpre[s][i][0] = kk4.x; kpre[s][i][1] = kk4.y; kpre[s][i][2] = kk4.z; kpre[s][i][3] = kk4.w;
              qpre[s][i][0] = qq4.x; qpre[s][i][1] = qq4.y; qpre[s][i][2] = qq4.z; qpre[s][i][3] = qq4.w;
            }
          }
      }

      // -- gate pass A: running sums of log_alpha inside each 4-token group -------------
      float la[2][4][4], tot[2][4];
#pragma unroll
      for (int s = 0; s < 2; ++s) {
        const int r0 = 4 * (2 * fw + s);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const bool in = r0 + i < len;
          const size_t o = static_cast<size_t>(t0 + (in ? r0 + i : 0)) * tok_stride + static_cast<size_t>(h) * kD + c0;
          if constexpr (kPre) {
            // log alpha = -scale * softplus(x)
            const float sc = __ldg(a.a_scale + h);
            float x[4];
            ld4_in(static_cast<const __nv_bfloat16*>(a.a_pre) + o, x);
#pragma unroll
            for (int e = 0; e < 4; ++e)
              la[s][i][e] = in ? -sc * softplus_fast(x[e]) : 0.f;
          } else {
            const float4 l4 = __ldg(reinterpret_cast<const float4*>(a.log_alpha + o));
            la[s][i][0] = in ? l4.x : 0.f; la[s][i][1] = in ? l4.y : 0.f;
            la[s][i][2] = in ? l4.z : 0.f; la[s][i][3] = in ? l4.w : 0.f;
          }
        }
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          tot[s][e] = 0.f;
#pragma unroll
          for (int i = 0; i < 4; ++i) { tot[s][e] += la[s][i][e]; la[s][i][e] = tot[s][e]; }
        }
        if constexpr (kParkLa) {
#pragma unroll
          for (int i = 0; i < 4; ++i)
            st4_f32(sm + SM::kKH, f32_offset(r0 + i, c0, 64), la[s][i][0], la[s][i][1], la[s][i][2], la[s][i][3]);
        }
        *reinterpret_cast<float4*>(sTot + (2 * fw + s) * kD + c0) = make_float4(tot[s][0], tot[s][1], tot[s][2], tot[s][3]);
      }
      if constexpr (kConv) {
        float* w = reinterpret_cast<float*>(sm + SM::kConvW) + (ftid >> 7) * 512 + (ftid & 127);
        w[0] = wtap.x; w[128] = wtap.y; w[256] = wtap.z; w[384] = wtap.w;
      }
      fsync();
      float pre[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
      for (int g = 0; g < 2 * fw; ++g) {
        const float4 t4 = *reinterpret_cast<const float4*>(sTot + g * kD + c0);
        pre[0][0] += t4.x; pre[0][1] += t4.y; pre[0][2] += t4.z; pre[0][3] += t4.w;
      }
#pragma unroll
      for (int e = 0; e < 4; ++e) pre[1][e] = pre[0][e] + tot[0][e];
      float gl = 0.f;
      if (ftid < 128) {
#pragma unroll
        for (int g = 0; g < 16; ++g) gl += sTot[g * kD + ftid];
      }
      if (ftid == 0) bulk_wait_read();  // the previous item's Qt and Kh have left KQ and KHT
      // The totals are read (KQ may be written) and the group votes: a chunk whose decay
      // passes kMaxChunkDecay in some channel is handed to the recurrence as its raw rows
      // (k, q after conv / L2, log_alpha, v, beta) and walked there token by token;
      // e^g_last[0] = -1 marks such an item.
      const bool strong = group_any(kBarFront, kGroupThreads, ftid < 128 && -gl > kMaxChunkDecay);
      if (ftid < 128)
        reinterpret_cast<float*>(item + kItemGamma)[ftid] = strong ? (ftid == 0 ? -1.f : 0.f) : __expf(gl);
      if (ftid == 0) {
        sStrong[k & 1] = strong ? 1 : 0;  // for the back group (ordered by kBApFull)
        if (strong) *p.any_raw = 1;       // the recurrence runs its walking loop
      }
      if (strong && ftid < 64) reinterpret_cast<float*>(item + kItemP)[ftid] = sB[ftid];

      // -- gate pass B: q, k (conv, L2 norm), Kt, Qt, Kh -----------------------------------
      if (strong) {  // raw rows for the token walk (out of line: the rare path)
        RawRowsFront rr{a.q, a.k, a.log_alpha, a.a_pre, a.a_scale, a.conv_w, item, t0, bos, len, h, H, fw};
        raw_rows_front<TIn, kConv, kPre>(rr);
      } else {
        // q/k row m of group s is chunk row r0 - kHist + m; rows outside [bos, t0 + len) read
        // row t0 (always in bounds) and are replaced by zero where used. With the conv, the
        // second group's history rows are the first group's last rows: carried, not reloaded.
        uint32_t kraw[kGRows][sizeof(TIn)], qraw[kGRows][sizeof(TIn)];
        bool rin[kGRows];
#pragma unroll
        for (int s = 0; s < 2; ++s) {
          const int r0 = 4 * (2 * fw + s);
#pragma unroll
          for (int m = 0; m < kGRows; ++m) {
            const int rr = r0 - kHist + m;
            if (kConv && s == 1 && m < kHist) {
#pragma unroll
              for (int w = 0; w < static_cast<int>(sizeof(TIn)); ++w) {
                kraw[m][w] = kraw[m + 4][w];
                qraw[m][w] = qraw[m + 4][w];
              }
              rin[m] = rin[m + 4];
              continue;
            }
            rin[m] = rr < len && t0 + rr >= bos;
            if constexpr (!kConv) {
#pragma unroll
              for (int w = 0; w < static_cast<int>(sizeof(TIn)); ++w) {
                kraw[m][w] = kpre[s][m][w];
                qraw[m][w] = qpre[s][m][w];
              }
              continue;
            }
            const size_t o = static_cast<size_t>(rin[m] ? t0 + rr : t0) * tok_stride + static_cast<size_t>(h) * kD + c0;
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
          auto unpack = [&](const uint32_t* w, int e) -> float {
            if constexpr (sizeof(TIn) == 2) {
              const uint32_t x = w[e >> 1];
              return __uint_as_float((e & 1) ? (x & 0xFFFF0000u) : (x << 16));
            } else {
              return __uint_as_float(w[e]);
            }
          };
          float kv[4][4], qv[4][4];
          if constexpr (kConv) {
            // y[t, c] = sum_j w[c, j] x[t - 3 + j, c] (x = 0 before the sequence start), then
            // x / sqrt(sum_c y^2 + 1e-6) over the head's 128 channels (this warp holds them all)
            // taps from shared memory, [tensor][tap][channel]
            const float* sw = reinterpret_cast<const float*>(sm + SM::kConvW) + c0;
            float wq[4][4], wk[4][4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const float4 a4 = *reinterpret_cast<const float4*>(sw + j * 128);
              const float4 b4 = *reinterpret_cast<const float4*>(sw + 512 + j * 128);
              wq[0][j] = a4.x; wq[1][j] = a4.y; wq[2][j] = a4.z; wq[3][j] = a4.w;
              wk[0][j] = b4.x; wk[1][j] = b4.y; wk[2][j] = b4.z; wk[3][j] = b4.w;
            }
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
            for (int i = 0; i < 4; ++i)
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                kv[i][e] = rin[i] ? unpack(kraw[i], e) : 0.f;
                qv[i][e] = rin[i] ? unpack(qraw[i], e) : 0.f;
              }
          }
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            float kt[4], qt[4], kh[4];
            const int r = r0 + i;
            float lr[4];
            if constexpr (kParkLa) {
              const float4 l4 = *reinterpret_cast<const float4*>(sm + SM::kKH + f32_offset(r, c0, 64));
              lr[0] = l4.x; lr[1] = l4.y; lr[2] = l4.z; lr[3] = l4.w;
            } else {
#pragma unroll
              for (int e = 0; e < 4; ++e) lr[e] = la[s][i][e];
            }
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float g = pre[s][e] + lr[e];
              const float eg = __expf(g), eng = __expf(-g);
              kt[e] = kv[i][e] * eg;
              kh[e] = to_tf32(kv[i][e] * eng);
              qt[e] = to_tf32(qv[i][e] * eg);
            }
            st4_f32(sm + SM::kKQ, f32_offset(r, c0, 128), kt[0], kt[1], kt[2], kt[3]);       // Kt [tok][ch]
            st4_f32(sm + SM::kKQ, f32_offset(64 + r, c0, 128), qt[0], qt[1], qt[2], qt[3]);  // Qt [tok][ch]
            st4_f32(sm + SM::kKH, f32_offset(r, c0, 64), kh[0], kh[1], kh[2], kh[3]);        // Kh [tok][ch]
            // the same rows for the item: Kh as the MN-major A operand (Kh^T) of the state update
            st4_f32(sm + SM::kKHT, mn_offset(r, c0, 64), kh[0], kh[1], kh[2], kh[3]);
          }
        }
      }  // factorised form
      fence_proxy_async_smem();
      fsync();
      if (ftid == 0 && !strong) {  // Qt: rows 64..127 of each 32-column block of the tile; Kh whole
#pragma unroll
        for (int kb = 0; kb < 4; ++kb)
          bulk_store(item + kItemQW + kb * 16384 + 8192, sm + SM::kKQ + kb * 16384 + 8192, 8192);
        bulk_store(item + kItemKHT, sm + SM::kKHT, 32768);
        bulk_commit_group();
      }

      // -- D[A; P] = [Kt; Qt] Kh^T, once the back group has read the previous one out ------
      if (ftid == 0) {
        if (k > 0) {
          if (!lost && !mbar_wait(bars + kBApFree, ph_apfree, a.status)) lost = true;
          ph_apfree ^= 1u;
        }
        tc_fence_after_sync();
        if (strong) {
          mbar_arrive(bars + kBApFull);  // nothing to multiply: the back group only passes it on
        } else {
          constexpr uint32_t kIdAP = idesc_tf32(128, 64, false, false);
          const uint64_t a0 = kdesc0(sb + SM::kKQ), b0 = kdesc0(sb + SM::kKH);
#pragma unroll
          for (int kk = 0; kk < 16; ++kk)
            umma_tf32(tmem + kTmAP, a0 + kstep(kk, 128), b0 + kstep(kk, 64), kIdAP, kk > 0);
          umma_commit(bars + kBApFull);
        }
      }

      // the V rows this thread turns into operand lines below (4-token x 4-column blocks, all
      // their rows in flight at once; they were warmed into L2): for plain bf16 inputs they
      // are loaded before waiting for VT; with the conv's extra rows (or fp32 inputs) after
      // it, where fewer registers are live
      constexpr int kW = sizeof(TIn);  // 32-bit words per 4 elements
      constexpr bool kEarlyV = !kConv && kW == 2;
      uint32_t vraw[2][kGRows][kW];
      auto load_v = [&] {
        const TIn* vh = vg + static_cast<size_t>(h) * kD;
#pragma unroll
        for (int bb = 0; bb < 2; ++bb) {
          const int blk = ftid + bb * kGroupThreads, t4 = 4 * (blk >> 5), j4 = 4 * (blk & 31);
#pragma unroll
          for (int m = 0; m < kGRows; ++m) {
            const int rr = t4 - kHist + m;
            const bool in = rr < len && t0 + rr >= bos;
            const TIn* src = vh + static_cast<size_t>(in ? t0 + rr : t0) * tok_stride + j4;
            if constexpr (kW == 2) {
              const uint2 x = __ldg(reinterpret_cast<const uint2*>(src));
              vraw[bb][m][0] = in ? x.x : 0u; vraw[bb][m][1] = in ? x.y : 0u;
            } else {
              const uint4 x = __ldg(reinterpret_cast<const uint4*>(src));
              vraw[bb][m][0] = in ? x.x : 0u; vraw[bb][m][1] = in ? x.y : 0u;
              vraw[bb][m][2] = in ? x.z : 0u; vraw[bb][m][3] = in ? x.w : 0u;
            }
          }
        }
      };
      if (kEarlyV && !strong) load_v();

      // -- Kt and V, once the back group's previous W / U~ MMA and its staging have let go of
      //    KTT and VT --------------------------------------------------------------------------
      if (k > 0) {
        if (ftid == 0 && !lost && !mbar_wait(bars + kBWFree, ph_wfree, a.status)) lost = true;
        ph_wfree ^= 1u;
        fsync();
      }
      for (int i = ftid; i < (strong ? 0 : kChunk * 32); i += kGroupThreads) {
        // Kt (rows 0..63 of KQ) -> the MN-major B operand of T Kt, 4 channels at a time
        const int r = i >> 5, c = 4 * (i & 31);
        *reinterpret_cast<float4*>(sm + SM::kKTT + mn_offset(r, c, 64)) =
            *reinterpret_cast<const float4*>(sm + SM::kKQ + f32_offset(r, c, 128));
      }
      // V rows (tf32; conv for the mixer) as the MN-major B operand of T V: each thread takes
      // 4-token x 4-column blocks (their rows loaded above)
      if (kVFront && !strong) {
        if constexpr (!kEarlyV) load_v();
#pragma unroll
        for (int bb = 0; bb < 2; ++bb) {
          const int blk = ftid + bb * kGroupThreads, t4 = 4 * (blk >> 5), j4 = 4 * (blk & 31);
          auto elem = [&](int jr, int m) -> float {  // column j4 + jr of loaded row m
            if constexpr (kW == 2) {
              const uint32_t x = vraw[bb][m][jr >> 1];
              return __uint_as_float((jr & 1) ? (x & 0xFFFF0000u) : (x << 16));
            } else {
              return __uint_as_float(vraw[bb][m][jr]);
            }
          };
          float4 wv[kConv ? 4 : 1];  // conv taps of columns j4 .. j4 + 3
          if constexpr (kConv) {
#pragma unroll
            for (int jr = 0; jr < 4; ++jr)
              wv[jr] = __ldg(reinterpret_cast<const float4*>(a.conv_w + ((2 * H + h) * kD + j4 + jr) * 4));
          }
          // V rows t4 .. t4 + 3 as whole lines of the MN-major B operand of T V
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            float y[4];
#pragma unroll
            for (int jr = 0; jr < 4; ++jr) {
              if constexpr (kConv) {
                const float4 w4 = wv[jr];
                const float yc = fmaf(w4.x, elem(jr, e), fmaf(w4.y, elem(jr, e + 1),
                                                              fmaf(w4.z, elem(jr, e + 2), w4.w * elem(jr, e + 3))));
                y[jr] = (t4 + e < len) ? yc : 0.f;
              } else {
                y[jr] = elem(jr, e);
              }
            }
            st4_tf32(sm + SM::kVT, mn_offset(t4 + e, j4, 64), y[0], y[1], y[2], y[3]);
          }
        }
      }

      fence_proxy_async_smem();
      fsync();
      if (ftid == 0) mbar_arrive(bars + kBVtFull);
      if (group_any(kBarFront, kGroupThreads, lost)) {
        lost = true;
        break;
      }
    }
  } else {
    // ================================= back group ==================================
    const int bw = warp - 8;
    const int btid = tid - kGroupThreads;
    const int half = bw >> 2;  // which half of a row's columns this warp handles
    float* sA = reinterpret_cast<float*>(sm + SM::kScr);  // [64][kLd]: A, then X in place
    float* sY = sA + 64 * kLd;                            // [32][kLd]
    uint32_t ph_apfull = 0, ph_vtfull = 0, ph_wu = 0;
    auto bsync = [] { group_sync(kBarBack, kGroupThreads); };
    constexpr uint32_t kIdN128Bmn = idesc_tf32(128, 128, false, true);  // B (Kt, V) MN-major

    for (int k = 0; k < n_mine; ++k) {
      const int64_t it = blockIdx.x + static_cast<int64_t>(k) * gridDim.x;
      const ItemPos ip = item_pos(it, a, p);
      uint8_t* item = ip.item;
      const float* sB = sBeta + (k & 1) * 64;

      // -- A (rows 0..63: beta-scaled, strictly lower) -> scratch; P (rows 64..127: lower) -> item
      if (btid == 0 && !lost && !mbar_wait(bars + kBApFull, ph_apfull, a.status)) lost = true;
      ph_apfull ^= 1u;
      bsync();
      tc_fence_after_sync();
      if (sStrong[k & 1]) {
        // -- an item handed over as raw rows (walked by the recurrence): no solve; the v rows
        //    (conv for the mixer) go to the item's U~ space in fp32, and the hand-overs with
        //    the front group run as for any item ---------------------------------------------
        tc_fence_before_sync();
        bsync();
        if (btid == 0) mbar_arrive(bars + kBApFree);
        RawRowsBack rb{a.v, a.conv_w, item, ip.t0, ip.bos, ip.len, ip.h, H, btid};
        raw_rows_back<TIn, kConv>(rb);
        if (btid == 0) {
          if (!lost && !mbar_wait(bars + kBVtFull, ph_vtfull, a.status)) lost = true;
          ph_vtfull ^= 1u;
          mbar_arrive(bars + kBWuDone);
          if (!lost && !mbar_wait(bars + kBWuDone, ph_wu, a.status)) lost = true;
          mbar_arrive(bars + kBWFree);
        }
        ph_wu ^= 1u;
        if (group_any(kBarBack, kGroupThreads, lost)) {
          lost = true;
          break;
        }
        continue;
      }
      {
        const int cb = half * 32;
        float d[32];
        tmem_ld16(tmem + lane_off + kTmAP + cb, *reinterpret_cast<float(*)[16]>(d));
        tmem_ld16(tmem + lane_off + kTmAP + cb + 16, *reinterpret_cast<float(*)[16]>(d + 16));
        tmem_ld_wait();
        if (lq < 2) {
          const int r = row;
          const float br = sB[r];
#pragma unroll
          for (int i = 0; i < 32; i += 4) {
            const int c = cb + i;
            *reinterpret_cast<float4*>(sA + r * kLd + c) =
                make_float4(c < r ? br * d[i] : 0.f, c + 1 < r ? br * d[i + 1] : 0.f,
                            c + 2 < r ? br * d[i + 2] : 0.f, c + 3 < r ? br * d[i + 3] : 0.f);
          }
        } else {  // P row r (lower, tf32) kept in TMEM until the epilogue stages it
          const int r = row - 64;
#pragma unroll
          for (int i = 0; i < 32; i += 8) {
            float x[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) x[e] = (cb + i + e <= r) ? to_tf32(d[i + e]) : 0.f;
            tmem_st8(tmem + lane_off + kTmP + cb + i, x);
          }
          tmem_st_wait();
        }
      }
      tc_fence_before_sync();
      bsync();
      if (btid == 0) mbar_arrive(bars + kBApFree);

      // -- X = (I + A)^-1; T = X Diag(beta) into TMEM rows 0..63 (the W / U~ MMA's A) ---------
      // the mixer's V rows (with the conv's history rows) in flight during the inverse
      constexpr int kWb = sizeof(TIn);  // 32-bit words per 4 elements
      uint32_t vraw[2][kGRows][kWb];
      if constexpr (!kVFront) {
        const TIn* vh = static_cast<const TIn*>(a.v) + static_cast<size_t>(ip.h) * kD;
#pragma unroll
        for (int bb = 0; bb < 2; ++bb) {
          const int t4 = 4 * (2 * (btid >> 5) + bb), j4 = 4 * (btid & 31);  // two consecutive groups
#pragma unroll
          for (int m = 0; m < kGRows; ++m) {
            if (bb == 1 && m < kHist) {  // the second group's history rows: the first group's last
#pragma unroll
              for (int w = 0; w < kWb; ++w) vraw[1][m][w] = vraw[0][m + 4][w];
              continue;
            }
            const int rr = t4 - kHist + m;
            const bool in = rr < ip.len && ip.t0 + rr >= ip.bos;
            const TIn* src = vh + static_cast<size_t>(in ? ip.t0 + rr : ip.t0) * tok_stride + j4;
            if constexpr (kWb == 2) {
              const uint2 x = __ldg(reinterpret_cast<const uint2*>(src));
              vraw[bb][m][0] = in ? x.x : 0u; vraw[bb][m][1] = in ? x.y : 0u;
            } else {
              const uint4 x = __ldg(reinterpret_cast<const uint4*>(src));
              vraw[bb][m][0] = in ? x.x : 0u; vraw[bb][m][1] = in ? x.y : 0u;
              vraw[bb][m][2] = in ? x.z : 0u; vraw[bb][m][3] = in ? x.w : 0u;
            }
          }
        }
      }
      invert_unit_lower_64(sA, sY, bw, bsync);
      if (lq < 2) {
        const int r = row;
#pragma unroll
        for (int j = 0; j < 32; j += 8) {
          const int c = half * 32 + j;
          float x[8];
          const float4 x0 = *reinterpret_cast<const float4*>(sA + r * kLd + c);
          const float4 x1 = *reinterpret_cast<const float4*>(sA + r * kLd + c + 4);
          const float xr[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
#pragma unroll
          for (int e = 0; e < 8; ++e) x[e] = (c + e <= r) ? to_tf32(xr[e] * sB[c + e]) : 0.f;
          tmem_st8(tmem + lane_off + kTmT + c, x);
        }
        tmem_st_wait();
      }
      tc_fence_before_sync();
      bsync();

      // -- the V rows with their conv (the mixer) as lines of the MN-major B operand of T V:
      //    each thread takes 4-token x 4-column blocks, all of whose rows are loaded before
      //    any is used (the rows were warmed into L2) ------------------------------------------
      if constexpr (!kVFront) {
#pragma unroll
        for (int bb = 0; bb < 2; ++bb) {
          const int t4 = 4 * (2 * (btid >> 5) + bb), j4 = 4 * (btid & 31);  // two consecutive groups
          auto elem = [&](int jr, int m) -> float {  // column j4 + jr of loaded row m
            if constexpr (kWb == 2) {
              const uint32_t x = vraw[bb][m][jr >> 1];
              return __uint_as_float((jr & 1) ? (x & 0xFFFF0000u) : (x << 16));
            } else {
              return __uint_as_float(vraw[bb][m][jr]);
            }
          };
          float4 wv[kConv ? 4 : 1];  // conv taps of columns j4 .. j4 + 3
          if constexpr (kConv) {
#pragma unroll
            for (int jr = 0; jr < 4; ++jr)
              wv[jr] = __ldg(reinterpret_cast<const float4*>(a.conv_w + ((2 * H + ip.h) * kD + j4 + jr) * 4));
          }
          // V rows t4 .. t4 + 3 as whole lines of the MN-major B operand of T V
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            float y[4];
#pragma unroll
            for (int jr = 0; jr < 4; ++jr) {
              if constexpr (kConv) {
                const float4 w4 = wv[jr];
                const float yc = fmaf(w4.x, elem(jr, e), fmaf(w4.y, elem(jr, e + 1),
                                                              fmaf(w4.z, elem(jr, e + 2), w4.w * elem(jr, e + 3))));
                y[jr] = (t4 + e < ip.len) ? yc : 0.f;
              } else {
                y[jr] = elem(jr, e);
              }
            }
            st4_tf32(sm + SM::kVT, mn_offset(t4 + e, j4, 64), y[0], y[1], y[2], y[3]);
          }
        }
      }
      fence_proxy_async_smem();
      bsync();

      // -- D[W; -] = T Kt, D[U~; -] = T V, once the front group has written Kt and V ---------
      if (btid == 0) {
        if (!lost && !mbar_wait(bars + kBVtFull, ph_vtfull, a.status)) lost = true;
        ph_vtfull ^= 1u;
        tc_fence_after_sync();
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          umma_tf32_ta(tmem + kTmW, tmem + kTmT + kk * 8, mndesc(sb + SM::kKTT, 64, kk), kIdN128Bmn, kk > 0);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          umma_tf32_ta(tmem + kTmU, tmem + kTmT + kk * 8, mndesc(sb + SM::kVT, 64, kk), kIdN128Bmn, kk > 0);
        umma_commit(bars + kBWuDone);
      }
      if (btid == 0 && !lost && !mbar_wait(bars + kBWuDone, ph_wu, a.status)) lost = true;
      ph_wu ^= 1u;
      bsync();
      tc_fence_after_sync();

      // -- -W, U~ (over the Kt and V tiles, which the MMA has read) and P (over the scratch) staged
      //    as 64-row tiles, then bulk-stored into the item --------------------------------------
      if (lq < 2) {
        const int r = row;
#pragma unroll
        for (int j = 0; j < 64; j += 16) {
          const int c = half * 64 + j;
          float w[16], u[16];
          tmem_ld16(tmem + lane_off + kTmW + c, w);
          tmem_ld16(tmem + lane_off + kTmU + c, u);
          tmem_ld_wait();
#pragma unroll
          for (int e = 0; e < 16; e += 4) {
            st4_f32(sm + SM::kKTT, f32_offset(r, c + e, 64), -w[e], -w[e + 1], -w[e + 2], -w[e + 3]);
            st4_f32(sm + SM::kVT, f32_offset(r, c + e, 64), u[e], u[e + 1], u[e + 2], u[e + 3]);
          }
        }
      } else {
        const int r = row - 64;
#pragma unroll
        for (int j = 0; j < 32; j += 16) {
          const int c = half * 32 + j;
          float x[16];
          tmem_ld16(tmem + lane_off + kTmP + c, x);
          tmem_ld_wait();
#pragma unroll
          for (int e = 0; e < 16; e += 4)
            st4_f32(sm + SM::kScr, f32_offset(r, c + e, 64), x[e], x[e + 1], x[e + 2], x[e + 3]);
        }
      }
      fence_proxy_async_smem();
      tc_fence_before_sync();
      bsync();
      if (btid == 0) {
#pragma unroll
        for (int kb = 0; kb < 4; ++kb)  // -W: rows 0..63 of each 32-column block of the tile
          bulk_store(item + kItemQW + kb * 16384, sm + SM::kKTT + kb * 8192, 8192);
        bulk_store(item + kItemU, sm + SM::kVT, 32768);
        bulk_store(item + kItemP, sm + SM::kScr, 16384);
        bulk_commit_group();
        bulk_wait_read();  // the Kt and V tiles and the scratch are free again
        mbar_arrive(bars + kBWFree);
      }
      if (group_any(kBarBack, kGroupThreads, lost)) {
        lost = true;
        break;
      }
    }
  }

  // ---- teardown: bulk stores complete; after a lost wait, let the tensor pipe drain
  //      (bounded) before the TMEM goes back ----------------------------------------------
  if (tid == 0 || tid == kGroupThreads) bulk_wait_all();  // the items' bulk stores are done
  const bool any_lost = __syncthreads_or(lost ? 1 : 0) != 0;
  if (any_lost && tid == 0) {
    umma_commit(bars + kBDrain);
    mbar_wait(bars + kBDrain, 0, a.status);
  }
  tc_fence_before_sync();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after_sync();
    tmem_dealloc(tmem, kIntraCols);
  }
}

// ================================ pass 2 =============================================
// 17 warps: warps 0..15 run the epilogues (warp w reads TMEM lanes 32*(w%4).. and value
// column part w/4); warp 16 waits for the tiles and issues the MMAs, so that an issue
// that blocks on the tensor pipe never holds up an epilogue.
constexpr int kRecEpiThreads = 512;
constexpr int kRecThreads = kRecEpiThreads + 32;
constexpr uint32_t kRecBarU = 1;  // named barrier: U^T written (epilogue warps + the issuer warp)

//  region   size        holds
//  QW       64 KB       [-W; Qt] of the current chunk
//  PT       2 x 32 KB   P of chunks i, i+1 (alternating) in rows 64..127 (K blocks at +8K,
//                       +24K); the chunk's e^g_last in the unused rows at +0
//  KHT      32 KB       Kh (the MN-major A operand Kh^T)
//  ST       DV*512 B    S^T (DV x 128), the B operand of group 1
//  UT       DV*256 B    U^T (DV x 64), the B operand of group 2
template <int DV>
struct RecSmem {
  static constexpr int kQW = 0;
  static constexpr int kPT = 65536;
  static constexpr int kKHT = 131072;
  static constexpr int kST = 163840;
  static constexpr int kUT = kST + DV * 512;
  static constexpr int kBar = kUT + DV * 256;  // 5 mbarriers
  static constexpr int kTmemSlot = kBar + 48;
  static constexpr int kTotal = kTmemSlot + 16;
  static constexpr int kAlloc = kTotal + 1024;
  static_assert(kAlloc <= 232448, "shared memory plan exceeds the per-block limit");
};

// Per chunk, with S the state slice (TMEM D2 and the S^T operand in shared memory):
//   issuer:   QW landed -> G1: D1 = [-W; Qt] S -> (G1 done) next chunk's QW on its way
//   epilogue: (G1 done) U = U~ + D1[0:64] -> U^T operand                  [barrier U]
//   issuer:   PK landed -> G2a: D2 += Kh^T U ; G2b: D1 += [.; P] U (output rows, read a
//             chunk later) -> (G2a done) next chunk's P, Kh^T, e^g_last on their way
//   epilogue: (G2a done) S <- e^g_last D2 (TMEM and S^T)                 [end barrier]
// The state chain waits only for G1, the U epilogue, G2a and the S epilogue.
// kRaw: some items were handed over as raw rows and are walked token by token; without
// it the loop is the plain tensor-core chain (the kernel picks the form from the flag
// pass 1 leaves, so that the common case carries none of the walk's code).
template <int DV, typename TOut, bool kRaw>
__device__ __forceinline__ void recur_body(const PrefillArgs& a, const SplitPlan& p) {
  using SM = RecSmem<DV>;
  constexpr int kSlices = kD / DV;
  constexpr int kPart = DV / 4;  // value columns per thread in the TMEM epilogues
  constexpr uint32_t kCols = 3 * DV <= 128 ? 128u : (3 * DV <= 256 ? 256u : 512u);
  constexpr uint32_t kD2 = 0;    // the state S (DV columns)
  constexpr uint32_t kD1 = DV;   // two buffers of DV columns: [-W S; Qt S] -> [-; O]

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const bool issuer_warp = warp == 16;
  const bool issuer = issuer_warp && lane == 0;
  const int lq = warp & 3;
  const int cp = warp >> 2;
  const int row = lq * 32 + lane;
  // segment maps: slices [0, kSlices) run from the identity with zero values (M), slices
  // [kSlices, 2 kSlices) from zero with the real values (B); no outputs
  const bool maps = a.map_M != nullptr;
  const int nslices = maps ? 2 * kSlices : kSlices;
  const bool map_m = maps && static_cast<int>(blockIdx.x % nslices) < kSlices;
  const int slice = (blockIdx.x % nslices) % kSlices;
  const int nh = blockIdx.x / nslices;
  const int H = a.H;
  const int h = nh % H;
  const int n = nh / H;
  const int col0 = slice * DV;

  const int32_t* cs = p.chunk_start;
  if (__ldg(cs + a.N) < 0) return;  // bad cu_seqlens: flagged by the plan kernel
  const int c_begin = __ldg(cs + n), c_end = __ldg(cs + n + 1);
  int64_t bos, eos;
  if (a.cu) {
    bos = __ldg(a.cu + n);
    eos = __ldg(a.cu + n + 1);
  } else {
    const int64_t L = a.total_T / a.N;
    bos = static_cast<int64_t>(n) * L;
    eos = bos + L;
  }

  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sb = smem_u32(sm);
  uint64_t* bar_g1 = reinterpret_cast<uint64_t*>(sm + SM::kBar);  // G1 done
  uint64_t* bar_qw = bar_g1 + 1;                                    // QW landed
  uint64_t* bar_pk = bar_g1 + 2;                                    // P, Kh^T, e^g_last landed
  uint64_t* bar_o = bar_g1 + 3;   // the chunk's P U is done: its output rows may be read
  uint64_t* bar_g2 = bar_g1 + 4;  // G2a done: the state may be updated
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + SM::kTmemSlot);

  if (tid == 0) {
    for (int i = 0; i < 5; ++i) mbar_init(bar_g1 + i, 1);
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, kCols);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = *tmem_slot;
  const uint32_t lane_off = static_cast<uint32_t>(lq * 32) << 16;

  auto item_of = [&](int c) -> const uint8_t* { return p.items + (static_cast<size_t>(c) * H + h) * kItemBytes; };
  // loads issued / waited per barrier (the issuer issues; the counts tell the teardown
  // what may still be in flight)
  int qw_issued = 0, pk_issued = 0;
  auto load_qw = [&](int c) {
    mbar_arrive_expect_tx(bar_qw, 65536u);
    bulk_load(sm + SM::kQW, item_of(c) + kItemQW, 65536u, bar_qw);
    ++qw_issued;
  };
  auto load_pk = [&](int c, int slot) {  // P and e^g_last into PT[slot], Kh^T
    const uint8_t* it = item_of(c);
    uint8_t* pt = sm + SM::kPT + slot * 32768;
    mbar_arrive_expect_tx(bar_pk, 16384u + 32768u + 512u);
    bulk_load(pt + 8192, it + kItemP, 8192u, bar_pk);
    bulk_load(pt + 24576, it + kItemP + 8192, 8192u, bar_pk);
    bulk_load(sm + SM::kKHT, it + kItemKHT, 32768u, bar_pk);
    bulk_load(pt, it + kItemGamma, 512u, bar_pk);
    ++pk_issued;
  };
  if (issuer && c_begin < c_end) {
    load_qw(c_begin);
    load_pk(c_begin, 0);
    if (c_begin + 1 < c_end) bulk_prefetch_l2(item_of(c_begin + 1), kItemBytes);
  }

  // ---- the state slice: TMEM D2 (lane c = key row c) and the S^T operand ---------------
  if (!issuer_warp) {
    const float* h0 =
        a.h0 && !maps ? a.h0 + ((static_cast<size_t>(n) * H + h) * kD + row) * kD + col0 : nullptr;
#pragma unroll
    for (int j = 0; j < kPart; j += 8) {
      const int c = cp * kPart + j;
      float x[8];
      if (map_m) {  // the identity (key row = value column)
#pragma unroll
        for (int e = 0; e < 8; ++e) x[e] = (row == col0 + c + e) ? 1.f : 0.f;
      } else if (h0) {
        const float4 u = *reinterpret_cast<const float4*>(h0 + c);
        const float4 w = *reinterpret_cast<const float4*>(h0 + c + 4);
        x[0] = u.x; x[1] = u.y; x[2] = u.z; x[3] = u.w; x[4] = w.x; x[5] = w.y; x[6] = w.z; x[7] = w.w;
      } else {
#pragma unroll
        for (int e = 0; e < 8; ++e) x[e] = 0.f;
      }
#pragma unroll
      for (int e = 0; e < 8; ++e) *reinterpret_cast<float*>(sm + SM::kST + f32_offset(c + e, row, DV)) = x[e];
      tmem_st8(tmem + lane_off + kD2 + c, x);
    }
    tmem_st_wait();
  }

  // U~ of the next chunk for this thread (rows 0..63: row, columns col0 + cp*kPart ..);
  // zero for the identity slices of the segment maps (zero values)
  float ut[kPart];
#pragma unroll
  for (int e = 0; e < kPart; ++e) ut[e] = 0.f;
  auto load_ut = [&](int c) {
    if (map_m) return;
    const uint8_t* src = item_of(c) + kItemU;
#pragma unroll
    for (int e = 0; e < kPart / 4; ++e) {
      const float4 x = __ldg(reinterpret_cast<const float4*>(src + f32_offset(row, col0 + cp * kPart + 4 * e, 64)));
      ut[4 * e] = x.x; ut[4 * e + 1] = x.y; ut[4 * e + 2] = x.z; ut[4 * e + 3] = x.w;
    }
  };
  if (!issuer_warp && lq < 2 && c_begin < c_end) load_ut(c_begin);

  const __nv_bfloat16* gateg = static_cast<const __nv_bfloat16*>(a.gate);
  TOut* outg = static_cast<TOut*>(a.out);
  const int64_t tok_stride = static_cast<int64_t>(H) * kD;
  // output rows of a finished chunk: rows 64..127 of its D1 buffer (* sigmoid(gate))
  auto out_rows = [&](uint32_t d1, int64_t tt0, int tlen) {
    if (maps) return;
    const int r = row - 64;
#pragma unroll
    for (int j = 0; j < kPart; j += 8) {
      const int c = cp * kPart + j;
      float o[8];
      tmem_ld8(d1 + lane_off + c, o);
      tmem_ld_wait();
      if (r < tlen) {
        const size_t off = static_cast<size_t>(tt0 + r) * tok_stride + static_cast<size_t>(h) * kD + col0 + c;
        if (gateg) {
          const uint4 g0 = *reinterpret_cast<const uint4*>(gateg + off);
          const __nv_bfloat16* gb0 = reinterpret_cast<const __nv_bfloat16*>(&g0);
#pragma unroll
          for (int i = 0; i < 8; ++i) o[i] *= 1.f / (1.f + __expf(-bf2f(gb0[i])));
        }
        store8(outg + off, o);
      }
    }
  };

  fence_proxy_async_smem();
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();

  // B (S^T, U^T) is K-major; A is [-W; Qt] and P (K-major) or Kh^T (MN-major: Kh's rows)
  constexpr uint32_t kIdV = idesc_tf32(128, DV, false, false);
  constexpr uint32_t kIdVmn = idesc_tf32(128, DV, true, false);
  bool lost = false, failed = false;
  // completions seen per barrier (each thread counts those it waits for)
  uint32_t g1_phase = 0, g2_phase = 0, o_phase = 0;
  int qw_waited = 0, pk_waited = 0;
  auto wait_bar = [&](uint64_t* bar, uint32_t& phase) {
    if (!lost && !mbar_wait(bar, phase, a.status)) lost = true;
    phase ^= 1u;
  };
  auto wait_loads = [&](uint64_t* bar, int& waited) {
    if (!lost && !mbar_wait(bar, static_cast<uint32_t>(waited & 1), a.status)) lost = true;
    ++waited;
  };

  int64_t prev_t0 = -1;
  int prev_len = 0;
  int b = 0;
  // items that pass 1 left as raw rows (e^g_last[0] = -1) are walked token by token
  auto item_raw = [&](int c) {
    return __ldg(reinterpret_cast<const float*>(item_of(c) + kItemGamma)) < 0.f;
  };
  bool raw = false;
  if constexpr (kRaw) raw = c_begin < c_end && item_raw(c_begin);
  for (int c = c_begin; c < c_end && !failed; ++c) {
    const int i = c - c_begin;
    const int64_t t0 = bos + static_cast<int64_t>(i) * kChunk;
    const int len = static_cast<int>(eos - t0 < kChunk ? eos - t0 : kChunk);
    const uint32_t d1 = tmem + kD1 + b * DV;
    bool raw_next = false;
    if constexpr (kRaw) raw_next = c + 1 < c_end && item_raw(c + 1);

    if (kRaw && raw) {
      // -- the exact token walk: k | q in QW, log_alpha in KHT, beta in this chunk's PT slot
      //    (P's bytes), v staged from the item into the other PT slot; the state slice moves
      //    TMEM -> registers -> TMEM and the S^T operand
      if (!issuer_warp && prev_t0 >= 0 && lq >= 2) {  // the previous chunk's output rows first
        wait_bar(bar_o, o_phase);
        tc_fence_after_sync();
        out_rows(tmem + kD1 + (b ^ 1) * DV, prev_t0, prev_len);
      }
      prev_t0 = -1;
      if (issuer) {
        wait_loads(bar_qw, qw_waited);
        wait_loads(bar_pk, pk_waited);
      }
      tc_fence_before_sync();
      failed = cta_any(lost);  // the raw rows have landed (or a wait gave up)
      tc_fence_after_sync();
      // the epilogue warps count the PK phase the issuer waited for (their next wait names
      // the right parity)
      if (!issuer_warp) ++pk_waited;
      if (failed) break;
      if (!issuer_warp) {
        // the chunk's v slice (DV columns) into the other PT slot, row-major, for the walk
        const float* vsrc = reinterpret_cast<const float*>(item_of(c) + kItemU) + col0;
        float* sv = reinterpret_cast<float*>(sm + SM::kPT + ((i + 1) & 1) * 32768);
        for (int idx = tid; idx < 64 * (DV / 4); idx += kRecEpiThreads) {
          const int t = idx / (DV / 4), c4 = 4 * (idx % (DV / 4));
          *reinterpret_cast<float4*>(sv + t * DV + c4) =
              map_m ? make_float4(0.f, 0.f, 0.f, 0.f) : __ldg(reinterpret_cast<const float4*>(vsrc + t * kD + c4));
        }
        WalkArgs wa;
        wa.sK = reinterpret_cast<const float*>(sm + SM::kQW);
        wa.sQ = wa.sK + 64 * kD;
        wa.sLA = reinterpret_cast<const float*>(sm + SM::kKHT);
        wa.sBeta = reinterpret_cast<const float*>(sm + SM::kPT + (i & 1) * 32768 + 8192);
        wa.sV = sv;
        wa.scr = reinterpret_cast<float*>(sm + SM::kUT);
        wa.sST = reinterpret_cast<float*>(sm + SM::kST);
        wa.out = maps ? nullptr : outg + static_cast<size_t>(t0) * tok_stride + static_cast<size_t>(h) * kD + col0;
        wa.gate = gateg ? gateg + static_cast<size_t>(t0) * tok_stride + static_cast<size_t>(h) * kD + col0 : nullptr;
        wa.out_stride = tok_stride;
        wa.tmem_state = tmem + lane_off + kD2;
        wa.scale = 1.f;
        wa.len = len;
        walk_chunk<DV, TOut>(wa);
        fence_proxy_async_smem();
      }
      tc_fence_before_sync();
      failed = cta_any(lost);  // QW, KHT and the PT slots are read: the next chunk's tiles may land
      tc_fence_after_sync();
      if (issuer && c + 1 < c_end) {
        load_qw(c + 1);
        load_pk(c + 1, (i + 1) & 1);
        if (c + 2 < c_end) bulk_prefetch_l2(item_of(c + 2), kItemBytes);
      }
      if (!issuer_warp && lq < 2 && c + 1 < c_end) load_ut(c + 1);
      raw = raw_next;
      continue;
    }

    if (issuer_warp) {
      // ================================ the MMA issuer ====================================
      if (issuer) {
        wait_loads(bar_qw, qw_waited);
        tc_fence_after_sync();
        const uint64_t a0 = kdesc0(sb + SM::kQW), b0 = kdesc0(sb + SM::kST);
#pragma unroll
        for (int kk = 0; kk < 16; ++kk) umma_tf32(d1, a0 + kstep(kk, 128), b0 + kstep(kk, DV), kIdV, kk > 0);
        umma_commit(bar_g1);
        wait_bar(bar_g1, g1_phase);  // QW has been read: the next chunk's [-W; Qt] on its way
        if (c + 1 < c_end) {
          load_qw(c + 1);
          if (c + 2 < c_end) bulk_prefetch_l2(item_of(c + 2), kItemBytes);
        }
      }
      group_sync(kRecBarU, kRecThreads);  // U^T is written
      if (issuer) {
        wait_loads(bar_pk, pk_waited);
        tc_fence_after_sync();
        const uint64_t pa = kdesc0(sb + SM::kPT + (i & 1) * 32768), ub = kdesc0(sb + SM::kUT);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          umma_tf32(tmem + kD2, mndesc(sb + SM::kKHT, kChunk, kk), ub + kstep(kk, DV), kIdVmn, 1u);
        umma_commit(bar_g2);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) umma_tf32(d1, pa + kstep(kk, 128), ub + kstep(kk, DV), kIdV, 1u);
        umma_commit(bar_o);
        // Kh^T and the other PT slot (last read by the P U of the previous chunk, which the
        // G2a commit covers) are free: the next chunk's P, Kh^T, e^g_last on their way
        wait_bar(bar_g2, g2_phase);
        if (c + 1 < c_end) load_pk(c + 1, (i + 1) & 1);
      }
    } else {
      // ================================ the epilogue warps ================================
      if (prev_t0 >= 0 && lq >= 2) {  // the previous chunk's output rows, while G1 runs
        wait_bar(bar_o, o_phase);
        tc_fence_after_sync();
        out_rows(tmem + kD1 + (b ^ 1) * DV, prev_t0, prev_len);
      }
      if (lq < 2) {  // U = U~ + D1[0:64] -> U^T operand
        wait_bar(bar_g1, g1_phase);
        tc_fence_after_sync();
#pragma unroll
        for (int j = 0; j < kPart; j += 8) {
          const int cc = cp * kPart + j;
          float ws[8];
          tmem_ld8(d1 + lane_off + cc, ws);
          tmem_ld_wait();
          // U row `row` into the U^T operand of group 2
#pragma unroll
          for (int e = 0; e < 8; ++e) st_tf32(sm + SM::kUT, f32_offset(cc + e, row, DV), ut[j + e] + ws[e]);
        }
        if (c + 1 < c_end) load_ut(c + 1);
        fence_proxy_async_smem();
      }
      tc_fence_before_sync();
      group_sync(kRecBarU, kRecThreads);  // U^T is written
      // S <- e^g_last D2 (TMEM and S^T), once G2a is done and this chunk's e^g_last has landed
      wait_loads(bar_pk, pk_waited);
      wait_bar(bar_g2, g2_phase);
      tc_fence_after_sync();
      const float gm = reinterpret_cast<const float*>(sm + SM::kPT + (i & 1) * 32768)[row];
#pragma unroll
      for (int j = 0; j < kPart; j += 8) {
        const int cc = cp * kPart + j;
        float x[8];
        tmem_ld8(tmem + lane_off + kD2 + cc, x);
        tmem_ld_wait();
#pragma unroll
        for (int e = 0; e < 8; ++e) x[e] *= gm;
#pragma unroll
        for (int e = 0; e < 8; ++e) *reinterpret_cast<float*>(sm + SM::kST + f32_offset(cc + e, row, DV)) = x[e];
        tmem_st8(tmem + lane_off + kD2 + cc, x);
      }
      tmem_st_wait();
      fence_proxy_async_smem();
    }
    tc_fence_before_sync();
    failed = cta_any(lost);  // the state is written (S^T and TMEM): the next chunk's G1 may go
    tc_fence_after_sync();
    prev_t0 = t0;
    prev_len = len;
    b ^= 1;
    raw = raw_next;
  }
  if (!failed && !issuer_warp && prev_t0 >= 0 && lq >= 2) {
    wait_bar(bar_o, o_phase);
    tc_fence_after_sync();
    out_rows(tmem + kD1 + (b ^ 1) * DV, prev_t0, prev_len);
  }

  // ---- final state ---------------------------------------------------------------------------
  float* ht_base = maps ? (map_m ? a.map_M : a.map_B) : a.ht;
  const int64_t hn = ht_base && !maps ? final_state_index(a, n, threadIdx.x == 0) : n;
  if (!failed && !issuer_warp && ht_base && hn >= 0) {
    float* ht = ht_base + ((static_cast<size_t>(hn) * H + h) * kD + row) * kD + col0;
#pragma unroll
    for (int j = 0; j < kPart; j += 8) {
      const int c = cp * kPart + j;
      float x[8];
      tmem_ld8(tmem + lane_off + kD2 + c, x);
      tmem_ld_wait();
      *reinterpret_cast<float4*>(ht + c) = make_float4(x[0], x[1], x[2], x[3]);
      *reinterpret_cast<float4*>(ht + c + 4) = make_float4(x[4], x[5], x[6], x[7]);
    }
  }

  // ---- teardown: after a lost wait, let the tensor pipe and the bulk loads drain (bounded)
  //      before the TMEM and the shared memory go back --------------------------------------
  if (failed && issuer) {
    umma_commit(bar_o);
    mbar_wait(bar_o, o_phase, a.status);
    for (; qw_waited < qw_issued; ++qw_waited) mbar_wait(bar_qw, static_cast<uint32_t>(qw_waited & 1), a.status);
    for (; pk_waited < pk_issued; ++pk_waited) mbar_wait(bar_pk, static_cast<uint32_t>(pk_waited & 1), a.status);
  }
  tc_fence_before_sync();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after_sync();
    tmem_dealloc(tmem, kCols);
  }
}
template <int DV, typename TOut>
__global__ void __launch_bounds__(kRecThreads, 1) kda_recur_kernel(const PrefillArgs a, const SplitPlan p) {
  if (__ldg(p.any_raw))
    recur_body<DV, TOut, true>(a, p);
  else
    recur_body<DV, TOut, false>(a, p);
}

// ================================ host =================================================
template <typename TIn, bool kConv, bool kPre = false>
cudaError_t launch_intra(const PrefillArgs& a, const SplitPlan& p, int64_t max_chunks, cudaStream_t stream) {
  auto kern = kda_intra_kernel<TIn, kConv, kPre>;
  static std::once_flag once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(once, [&] {
    attr_err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, IntraSmem::kAlloc);
  });
  if (attr_err != cudaSuccess) return attr_err;
  // persistent: one CTA per SM (the shared memory plan allows no more), each walking items
  int dev = 0, sms = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  const int64_t items = max_chunks * a.H;
  const unsigned grid = static_cast<unsigned>(items < sms ? items : sms);
  kern<<<grid, kIntraThreads, IntraSmem::kAlloc, stream>>>(a, p);
  return cudaGetLastError();
}

template <int DV, typename TOut>
cudaError_t launch_recur_dv(const PrefillArgs& a, const SplitPlan& p, cudaStream_t stream) {
  auto kern = kda_recur_kernel<DV, TOut>;
  static std::once_flag once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(once, [&] {
    attr_err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, RecSmem<DV>::kAlloc);
  });
  if (attr_err != cudaSuccess) return attr_err;
  const unsigned grid = static_cast<unsigned>(a.N) * static_cast<unsigned>(a.H) * (kD / DV) * (a.map_M ? 2u : 1u);
  kern<<<grid, kRecThreads, RecSmem<DV>::kAlloc, stream>>>(a, p);
  return cudaGetLastError();
}

template <typename TOut>
cudaError_t launch_recur(const PrefillArgs& a, const SplitPlan& p, cudaStream_t stream) {
  // value-column slices per chain: as many as a single wave of CTAs over the 148 SMs
  // allows (one CTA per SM); beyond 74 chains (only the gate-from-pre-activation mixer
  // takes the two passes there) 64-column slices in several waves
  // (the segment maps run twice the slices: both halves of a single wave where they fit)
  const int64_t chains = static_cast<int64_t>(a.N) * a.H * (a.map_M ? 2 : 1);
  if (4 * chains <= 148) return launch_recur_dv<32, TOut>(a, p, stream);
  return launch_recur_dv<64, TOut>(a, p, stream);  // more than 74 chains: several waves
}

}  // namespace

cudaError_t launch_plan(const int32_t* cu, int64_t total_T, int N, int32_t* chunk_start, uint32_t* status,
                        cudaStream_t stream) {
  kda_plan_kernel<<<1, 1024, 0, stream>>>(cu, total_T, N, chunk_start, status);
  return cudaGetLastError();
}

cudaError_t launch_recur_only(const PrefillArgs& a, cudaStream_t stream) {
  uint8_t* ws = static_cast<uint8_t*>(a.split_ws);
  SplitPlan p{reinterpret_cast<const int32_t*>(ws), reinterpret_cast<int32_t*>(ws) + a.N + 1,
              ws + split_plan_bytes(a.N)};
  return a.out_f32 ? launch_recur<float>(a, p, stream) : launch_recur<__nv_bfloat16>(a, p, stream);
}

cudaError_t launch_prefill_split(const PrefillArgs& a, cudaStream_t stream) {
  uint8_t* ws = static_cast<uint8_t*>(a.split_ws);
  SplitPlan p{reinterpret_cast<const int32_t*>(ws), reinterpret_cast<int32_t*>(ws) + a.N + 1,
              ws + split_plan_bytes(a.N)};
  cudaError_t e = launch_plan(a.cu, a.total_T, a.N, reinterpret_cast<int32_t*>(ws), a.status, stream);
  if (e != cudaSuccess) return e;
  const int64_t max_chunks = split_max_chunks(a.total_T, a.N);
  if (a.a_pre) {  // the full mixer with the decay gate made from its pre-activation
    if (!a.conv_w || !a.a_scale || a.in_f32 || a.out_f32) return cudaErrorInvalidValue;
    e = launch_intra<__nv_bfloat16, true, true>(a, p, max_chunks, stream);
  } else if (a.conv_w) {
    if (a.in_f32 || a.out_f32) return cudaErrorInvalidValue;
    e = launch_intra<__nv_bfloat16, true>(a, p, max_chunks, stream);
  } else {
    e = a.in_f32 ? launch_intra<float, false>(a, p, max_chunks, stream)
                 : launch_intra<__nv_bfloat16, false>(a, p, max_chunks, stream);
  }
  if (e != cudaSuccess) return e;
  return a.out_f32 ? launch_recur<float>(a, p, stream) : launch_recur<__nv_bfloat16>(a, p, stream);
}

}  // namespace kda
