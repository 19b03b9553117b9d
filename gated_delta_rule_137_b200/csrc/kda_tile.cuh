// kda_tile.cuh — device helpers shared by the prefill kernels: operand-tile
// descriptors, vector loads/stores of inputs and outputs, tf32 rounding stores into
// 128B-swizzled fp32 tiles, the fp32-accurate 64x64 unit-lower-triangular inverse,
// and the host-side TMA descriptor encoding. Internal to the library.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <mutex>

#include "kda_internal.h"

namespace kda {
namespace {

// Largest decay, summed over one chunk's tokens in any key channel, that a chunk may
// carry into the factorised (tensor-core) form; stronger-decaying chunks are walked token
// by token (walk_chunk below). Two limits meet here: e^-g must stay finite in fp32 (below
// about 88 nats), and the tf32 operands keep the form within the 2e-2 RMS parity bar only
// while the chunk forgets little. Measured against the fp64 oracle: final-state errors of
// 0.3-0.4% of RMS at 5 nats, up to 1.4% at 18 nats when every channel decays that much,
// and up to 3% between 40 and 80 nats (the state is then made of the last few tokens'
// writes, so the relative error of each tf32 product shows undiluted).
constexpr float kMaxChunkDecay = 20.f;
constexpr int kLd = 68;  // row stride (floats) of the fp32 solve scratch (16-B aligned rows)

// K-major fp32 operand tile with `rows` rows (M or N): descriptor of K step 0, and the
// constant to add for K step kk (8 columns per step: 32 B within a 128-B row, then
// the next 32-column block `rows` rows further). The start-address field holds
// address / 16 in its low 14 bits and shared memory is < 256 KB, so the sum never
// carries out of the field.
__device__ __forceinline__ uint64_t kdesc0(uint32_t base) { return sdesc(base, 16u, 1024u, kSwz128); }
__host__ __device__ constexpr uint64_t kstep(int kk, uint32_t rows) {
  return static_cast<uint64_t>(((kk >> 2) * rows * 128u + (kk & 3) * 32u) >> 4);
}

// softplus(x) = max(x, 0) + log(1 + e^-|x|) with the fast exp / log intrinsics: 1 + e^-|x|
// lies in (1, 2], where the sum rounds to within 1.2e-7 and the log's absolute error is
// about 4e-7, so the result is within 1e-6 of the exact value for every x (a decay made
// from it moves by less than 1e-6 nats per token).
__device__ __forceinline__ float softplus_fast(float x) { return fmaxf(x, 0.f) + __logf(1.f + __expf(-fabsf(x))); }

// MN-major fp32 operand tile of `krows` K lines (mn_offset): descriptor of K step kk
// (8 lines, 1024 B, per tf32 instruction).
__device__ __forceinline__ uint64_t mndesc(uint32_t base, uint32_t krows, int kk) {
  return sdesc(base + static_cast<uint32_t>(kk) * 1024u, krows * 128u, 512u, kSwz128A32);
}

// Eight consecutive elements (mn .. mn + 7, mn a multiple of 8) of line k of an MN-major
// tile, as two 16-byte stores (tf32-rounded if `tf32`). When the 32 lanes of a warp write
// 32 consecutive lines at the same mn, rows with bit 2 set store their upper half first,
// so that each quarter-warp's 16-byte stores land on 8 different bank groups.
__device__ __forceinline__ void st8_line(uint8_t* tile, uint32_t k, uint32_t mn, uint32_t krows, const float (&x)[8],
                                         bool tf32) {
  const bool swap = (k >> 2) & 1u;
  float y[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) y[e] = tf32 ? to_tf32(x[e]) : x[e];
  const float4 lo = make_float4(y[0], y[1], y[2], y[3]), hi = make_float4(y[4], y[5], y[6], y[7]);
  *reinterpret_cast<float4*>(tile + mn_offset(k, mn + (swap ? 4u : 0u), krows)) = swap ? hi : lo;
  *reinterpret_cast<float4*>(tile + mn_offset(k, mn + (swap ? 0u : 4u), krows)) = swap ? lo : hi;
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

// 8 consecutive output values of one row (TOut = bf16 or fp32)
__device__ __forceinline__ void store8(__nv_bfloat16* dst, const float* o) {
  uint4 p;
  p.x = pack_bf16x2(o[0], o[1]); p.y = pack_bf16x2(o[2], o[3]);
  p.z = pack_bf16x2(o[4], o[5]); p.w = pack_bf16x2(o[6], o[7]);
  *reinterpret_cast<uint4*>(dst) = p;
}
__device__ __forceinline__ void store8(float* dst, const float* o) {
  *reinterpret_cast<float4*>(dst) = make_float4(o[0], o[1], o[2], o[3]);
  *reinterpret_cast<float4*>(dst + 4) = make_float4(o[4], o[5], o[6], o[7]);
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

// 4 consecutive fp32 of one row as one 16-byte store, not rounded: operands whose
// tf32 truncation costs no accuracy (Kt, W, S) skip the rounding.
__device__ __forceinline__ void st4_f32(uint8_t* base, uint32_t off, float a, float b, float c, float d) {
  *reinterpret_cast<float4*>(base + off) = make_float4(a, b, c, d);
}

// CTA-wide OR of a predicate (every thread gets the same answer).
__device__ __forceinline__ bool cta_any(bool x) { return __syncthreads_or(x ? 1 : 0) != 0; }

// ---- small fp32-accurate products for the triangular solve (warp-level mma.sync) ----
// x = hi + lo with hi, lo representable in tf32; the 3-term product hi*hi + hi*lo + lo*hi
// keeps close to fp32 accuracy on the tensor pipe.
__device__ __forceinline__ void split_tf32(float x, uint32_t& hi, uint32_t& lo) {
  const float h = to_tf32(x);
  hi = __float_as_uint(h);
  lo = __float_as_uint(to_tf32(x - h));
}

__device__ __forceinline__ void mma_m16n8k8_tf32(float (&d)[4], const uint32_t (&a)[4], const uint32_t (&b)[2]) {
  asm volatile(
      "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

// One warp: C (16 x 8) = scale * A (16 x K, row stride kLd) * B (K x 8, row stride kLd),
// fp32 in shared memory, K a multiple of 8; C stored with row stride kLd.
__device__ __forceinline__ void warp_gemm_16x8(const float* A, const float* B, int K, float* C, float scale) {
  const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  for (int k = 0; k < K; k += 8) {
    uint32_t ah[4], al[4], bh[2], bl[2];
    split_tf32(A[g * kLd + k + t], ah[0], al[0]);
    split_tf32(A[(g + 8) * kLd + k + t], ah[1], al[1]);
    split_tf32(A[g * kLd + k + t + 4], ah[2], al[2]);
    split_tf32(A[(g + 8) * kLd + k + t + 4], ah[3], al[3]);
    split_tf32(B[(k + t) * kLd + g], bh[0], bl[0]);
    split_tf32(B[(k + t + 4) * kLd + g], bh[1], bl[1]);
    mma_m16n8k8_tf32(acc, al, bh);
    mma_m16n8k8_tf32(acc, ah, bl);
    mma_m16n8k8_tf32(acc, ah, bh);
  }
  *reinterpret_cast<float2*>(C + g * kLd + 2 * t) = make_float2(scale * acc[0], scale * acc[1]);
  *reinterpret_cast<float2*>(C + (g + 8) * kLd + 2 * t) = make_float2(scale * acc[2], scale * acc[3]);
}


// ---- X = (I + A)^-1 for a strictly lower 64x64 A in fp32 ----------------------------
// sA: A in [64][kLd] on entry, X in place on return; sY: [32][kLd] scratch. Called by
// every thread of a group of at least 8 warps; `gw` is the caller's warp index within
// the group and `sync()` a barrier over the group (warps 0..7 work; all take it).
// 16x16 diagonal blocks by forward substitution in registers, then two levels of block
// doubling: [[X1, 0], [A21, X2]]^-1 has lower-left block -X2 (A21 X1).
template <typename Sync>
__device__ __forceinline__ void invert_unit_lower_64(float* sA, float* sY, int gw, Sync sync) {
  const int lane = threadIdx.x & 31;
  // warp b < 4 owns diagonal block b; lane (r = lane % 16, half hh) holds row r,
  // columns 8hh..8hh+7
  if (gw < 4) {
    const int b = gw, r = lane & 15, hh = lane >> 4;
    float* Arow = sA + (16 * b + r) * kLd + 16 * b;
    float av[16], x[8];
#pragma unroll
    for (int i = 0; i < 16; ++i) av[i] = Arow[i];
#pragma unroll
    for (int j = 0; j < 8; ++j) x[j] = (8 * hh + j == r) ? 1.f : 0.f;
#pragma unroll
    for (int i = 0; i < 15; ++i) {  // row i is final: rows below subtract A[r][i] * row i
      const float c = (r > i) ? av[i] : 0.f;
#pragma unroll
      for (int j = 0; j < 8; ++j) x[j] = fmaf(-c, __shfl_sync(0xffffffffu, x[j], i + 16 * hh), x[j]);
    }
    __syncwarp();
    *reinterpret_cast<float4*>(Arow + 8 * hh) = make_float4(x[0], x[1], x[2], x[3]);
    *reinterpret_cast<float4*>(Arow + 8 * hh + 4) = make_float4(x[4], x[5], x[6], x[7]);
  }
  sync();
  // 16 -> 32 on the two diagonal pairs (warp = pair * 2 + 8-column tile) ...
  if (gw < 4) {
    const int p = gw >> 1, nt = gw & 1, o = 32 * p;
    warp_gemm_16x8(sA + (o + 16) * kLd + o, sA + o * kLd + o + 8 * nt, 16, sY + 16 * p + 8 * nt, 1.f);
  }
  sync();
  if (gw < 4) {
    const int p = gw >> 1, nt = gw & 1, o = 32 * p;
    warp_gemm_16x8(sA + (o + 16) * kLd + o + 16, sY + 16 * p + 8 * nt, 16, sA + (o + 16) * kLd + o + 8 * nt, -1.f);
  }
  sync();
  // ... then 32 -> 64 (warp = 16-row tile * 4 + 8-column tile)
  if (gw < 8) {
    const int mt = gw >> 2, nt = gw & 3;
    warp_gemm_16x8(sA + (32 + 16 * mt) * kLd, sA + 8 * nt, 32, sY + (16 * mt) * kLd + 8 * nt, 1.f);
  }
  sync();
  if (gw < 8) {
    const int mt = gw >> 2, nt = gw & 3;
    warp_gemm_16x8(sA + (32 + 16 * mt) * kLd + 32, sY + 8 * nt, 32, sA + (32 + 16 * mt) * kLd + 8 * nt, -1.f);
  }
  sync();
}
// Whole-CTA form (threadIdx.x / 32 is the warp index, __syncthreads the barrier).
__device__ __forceinline__ void invert_unit_lower_64(float* sA, float* sY) {
  invert_unit_lower_64(sA, sY, static_cast<int>(threadIdx.x >> 5), [] { __syncthreads(); });
}

// ---- the exact token-by-token walk of one chunk ------------------------------------
// The chunked form multiplies K e^g by K e^-g; a chunk whose decay summed over its
// tokens passes kMaxChunkDecay nats in some key channel would overflow e^-g or lose the
// parity bar to tf32 rounding. Such a chunk is walked token by token instead, with the
// recurrence itself in fp32 (no factorised exponentials, so any decay is exact):
//     S' = Diag(alpha_t) S;  w = S'^T k_t;  b = S'^T q_t;  u = beta_t (v_t - w);
//     S = S' + k_t u^T;      o_t = S^T q_t = b + u (k_t . q_t).

// 16 values per lane; returns to lane l the sum over the warp of value l >> 1 (lanes
// 2m and 2m + 1 both get value m). Halving exchanges: 8 + 4 + 2 + 1 + 1 shuffles.
__device__ __forceinline__ float warp_reduce_scatter16(const float (&v)[16]) {
  const int lane = threadIdx.x & 31;
  const bool h16 = (lane & 16) != 0, h8 = (lane & 8) != 0, h4 = (lane & 4) != 0, h2 = (lane & 2) != 0;
  float a8[8], a4[4], a2[2];
#pragma unroll
  for (int i = 0; i < 8; ++i)
    a8[i] = (h16 ? v[i + 8] : v[i]) + __shfl_xor_sync(0xffffffffu, h16 ? v[i] : v[i + 8], 16);
#pragma unroll
  for (int i = 0; i < 4; ++i)
    a4[i] = (h8 ? a8[i + 4] : a8[i]) + __shfl_xor_sync(0xffffffffu, h8 ? a8[i] : a8[i + 4], 8);
#pragma unroll
  for (int i = 0; i < 2; ++i)
    a2[i] = (h4 ? a4[i + 2] : a4[i]) + __shfl_xor_sync(0xffffffffu, h4 ? a4[i] : a4[i + 2], 4);
  float x = (h2 ? a2[1] : a2[0]) + __shfl_xor_sync(0xffffffffu, h2 ? a2[0] : a2[1], 2);
  return x + __shfl_xor_sync(0xffffffffu, x, 1);
}

// Scratch of walk_chunk, in floats: k.q per token, then two buffers of per-warp partial
// sums (16 per 8-column group per warp).
template <int KP>
struct WalkScratch {
  static constexpr int kKQ = 0;
  static constexpr int kRed = 64;
  static constexpr int kRedBuf = (KP / 8) * 256;
  static constexpr int kFloats = kRed + 2 * kRedBuf;
};

// Where one chunk's walk reads and writes. Thread (warp w, lane l) of the 512-thread CTA
// holds row r = 32 (w % 4) + l (key channel r) of the state slice and value columns
// cp*KP .. cp*KP + KP - 1 of the CTA's DV columns, cp = w / 4, KP = DV / 4.
struct WalkArgs {
  const float* sK;             // shared [64][128] (token, channel): k of the chunk
  const float* sQ;             // shared [64][128]: q
  const float* sLA;            // shared [64][128]: log_alpha
  const float* sBeta;          // shared [64]
  const float* sV;             // shared [64][DV]: v, the CTA's value columns
  float* scr;                  // shared, WalkScratch<DV / 4>::kFloats floats
  float* sST;                  // shared S^T operand tile to refresh (f32_offset(col, row, DV)), or null
  void* out;                   // global: out[t0][h][col0]; rows out_stride elements apart (null: none)
  const __nv_bfloat16* gate;   // global: gate[t0][h][col0] (same strides), or null
  int64_t out_stride;
  uint32_t tmem_state;         // TMEM address of the state slice's column 0 for this thread's lanes
  float scale;                 // the state is scale * (TMEM contents) on entry
  int len;                     // tokens of the chunk (<= 64)
};

// Named barrier of the 512 threads that walk (a CTA may hold more warps, which do not).
constexpr uint32_t kWalkBar = 2;
__device__ __forceinline__ void walk_sync() { group_sync(kWalkBar, 512); }

// Walks tokens 0..len-1 of one chunk through the recurrence. Threads 0..511 of the CTA
// call it (they synchronise on kWalkBar); on return the TMEM state slice (and sST, if
// given) hold the state after the chunk and out (x sigmoid(gate)) holds its rows. Kept
// out of line: it is the rare path, and inlining it would weigh on the register
// allocation of the kernels' tensor-core loops.
template <int DV, typename TOut>
__device__ __noinline__ void walk_chunk(const WalkArgs& wa) {
  constexpr int KP = DV / 4;
  using WS = WalkScratch<KP>;
  static_assert(KP % 8 == 0, "column parts come in groups of 8");
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int lq = warp & 3, cp = warp >> 2;
  const int r = lq * 32 + lane;
  const float* sK = wa.sK;
  const float* sQ = wa.sQ;
  float* scr = wa.scr;
  float s[KP];
#pragma unroll
  for (int j = 0; j < KP; j += 8) {
    float x[8];
    tmem_ld8(wa.tmem_state + cp * KP + j, x);
    tmem_ld_wait();
#pragma unroll
    for (int e = 0; e < 8; ++e) s[j + e] = wa.scale * x[e];
  }
  float* sKQ = scr + WS::kKQ;
  for (int t = warp; t < wa.len; t += 16) {  // k_t . q_t
    float x = 0.f;
#pragma unroll
    for (int c = lane; c < 128; c += 32) x = fmaf(sK[t * 128 + c], sQ[t * 128 + c], x);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
    if (lane == 0) sKQ[t] = x;
  }
  walk_sync();
  TOut* out = static_cast<TOut*>(wa.out);
  for (int t = 0; t < wa.len; ++t) {
    const float al = __expf(wa.sLA[t * 128 + r]), kr = sK[t * 128 + r], qr = sQ[t * 128 + r];
    float* red = scr + WS::kRed + (t & 1) * WS::kRedBuf;
#pragma unroll
    for (int g = 0; g < KP / 8; ++g) {
      float p[16];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        s[g * 8 + j] *= al;
        p[j] = s[g * 8 + j] * kr;
        p[8 + j] = s[g * 8 + j] * qr;
      }
      const float x = warp_reduce_scatter16(p);
      if (!(lane & 1)) red[g * 256 + (cp * 4 + lq) * 16 + (lane >> 1)] = x;
    }
    walk_sync();  // (the other buffer takes the next token: one barrier per token)
    const float bt = wa.sBeta[t], kq = sKQ[t];
    const float* vr = wa.sV + t * DV + cp * KP;
#pragma unroll
    for (int g = 0; g < KP / 8; ++g) {
      float w[8], b[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) w[j] = b[j] = 0.f;
#pragma unroll
      for (int q4 = 0; q4 < 4; ++q4) {
        const float* pr = red + g * 256 + (cp * 4 + q4) * 16;
#pragma unroll
        for (int j = 0; j < 8; j += 4) {
          const float4 x = *reinterpret_cast<const float4*>(pr + j);
          const float4 y = *reinterpret_cast<const float4*>(pr + 8 + j);
          w[j] += x.x; w[j + 1] += x.y; w[j + 2] += x.z; w[j + 3] += x.w;
          b[j] += y.x; b[j + 1] += y.y; b[j + 2] += y.z; b[j + 3] += y.w;
        }
      }
      float o[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const float u = bt * (vr[g * 8 + j] - w[j]);
        o[j] = fmaf(u, kq, b[j]);
        s[g * 8 + j] = fmaf(kr, u, s[g * 8 + j]);
      }
      if (out && lq == 0 && lane == 0) {  // one thread per column part writes the row
        const size_t off = static_cast<size_t>(t) * wa.out_stride + cp * KP + g * 8;
        if (wa.gate) {
#pragma unroll
          for (int e = 0; e < 8; ++e) o[e] *= 1.f / (1.f + __expf(-bf2f(wa.gate[off + e])));
        }
        store8(out + off, o);
      }
    }
  }
#pragma unroll
  for (int j = 0; j < KP; j += 8) {
    float x[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      x[e] = s[j + e];
      if (wa.sST) wa.sST[f32_offset(cp * KP + j + e, r, DV) >> 2] = x[e];
    }
    tmem_st8(wa.tmem_state + cp * KP + j, x);
  }
  tmem_st_wait();
  walk_sync();  // the scratch and the chunk's inputs are free again
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

// [total_T, H, 128] (bf16 or fp32) viewed as (d, head, token); box = (box_d, 1, rows),
// rows land unswizzled (box_d elements each)
bool encode_value_map(CUtensorMap* m, const void* ptr, int64_t total_T, int H, int box_d, int rows, bool f32) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t es = f32 ? 4 : 2;
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(kD), static_cast<cuuint64_t>(H),
                              static_cast<cuuint64_t>(total_T)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(kD) * es, static_cast<cuuint64_t>(H) * kD * es};
  const cuuint32_t box[3] = {static_cast<cuuint32_t>(box_d), 1u, static_cast<cuuint32_t>(rows)};
  const cuuint32_t estr[3] = {1u, 1u, 1u};
  const CUresult r = fn(m, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3,
                        const_cast<void*>(ptr), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

}  // namespace
}  // namespace kda
