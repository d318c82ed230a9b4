// Mixed-precision block-sparse attention on the 5th-generation tensor cores (K3).
//
// "DraftAttention2: Fast Video Diffusion with Low-Resolution-Guided Mixed-Precision
// Attention", Abstract: one attention kernel with precision-specific phases that share
// data movement, softmax statistics and output accumulation. "DraftAttention: Fast Video
// Diffusion via Low-Resolution Attention Guidance", Abstract: the output is restored to
// the original token order after the block-sparse attention.
//
// Per work item (b, h, query block i): the FP8 phase visits list8[i], the mixed phase
// listm[i] (E4M3 scores, E2M1 P V), then the FP4 phase list4[i], each in ascending block
// order, with ONE running row max m, ONE running sum l and ONE fp32 accumulator O in tensor
// memory. For each visited block j (S at the block's score precision, P V at its P V
// precision):
//   S = Q' K_j'^T            tcgen05.mma kind::f8f6f4 (E4M3) or kind::mxf4nvf4 (E2M1 with
//                            E4M3 scales per 16 along d), fp32 in TMEM
//   m_new = max(m, rowmax(S * s_q s_k sm_scale)), padded keys masked
//   l = l 2^(m-m_new) + sum p,  p = 2^(S' - m_new)  (log2 domain)
//   O = O 2^(m-m_new)        (only when the max moved, done in TMEM by the softmax warps)
//   P~ = E4M3(448 p) or E2M1(448 p / sigma) with sigma = E4M3(amax16 / 6) per 16 keys,
//                            written to tensor memory by the softmax threads
//   O += P~ V_j'             same MMA kind as the block (A = P~ read from tensor memory),
//                            accumulating into the one O.
// Epilogue: out = O s_v / (448 l) in bf16, written to the tokens' original positions.
//
// Two query tiles (work items) per CTA, processed as a ping-pong: while one tile's
// softmax warpgroup runs its exponential loop, the other's does its per-block
// bookkeeping, so the SM's special-function units and issue slots stay busy. 384 threads,
// one CTA per SM, persistent over work items in head-major order (one head's K/V stay in
// L2); round k of a CTA takes its work items 2k (tile A) and 2k+1 (tile B):
//   warps 0-3   softmax + epilogue of tile A: thread r owns query row r (TMEM lane r)
//   warps 4-7   softmax + epilogue of tile B
//   warp 8      MMA issue for tile A (one thread) and TMEM allocation
//   warp 9      producer: 1-D bulk copies of the pre-tiled Q/K/V operand tiles and scales
//   warp 10     MMA issue for tile B (one thread)
//   warp 11     idle
// Tensor memory: O of each tile, ONE S region the two tiles take in turns, scale factors
// and each tile's P~. Each tile's issuer runs S(0), then per block t: S(t+1), PV(t); the S region is
// taken in the order S_A(t), S_B(t), S_A(t+1), ..., each S waiting until the softmax of
// the previous owner has read its own. K/V stages are filled in that S order and released
// after their P V.
// Every mbarrier wait is bounded; a wait that runs out sets the workspace error word; the
// producer and the issuers stop issuing work, the producer waits for its copies in flight
// and the issuers for their MMAs, the softmax warps run through the rest of their round
// without waiting, and the kernel frees its tensor memory and exits.
#include <type_traits>

#include "common.cuh"
#include "tc.cuh"

namespace da2 {
namespace {

constexpr int kThreads = 384;
constexpr int kMmaWarp = 8;
constexpr int kLoadWarp = 9;
constexpr int kStages = 4;
constexpr int kPrefetch = 8;   // KV blocks the producer warms in L2 ahead of its copies
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLog2_448 = 8.807354922057604f;     // log2(448)

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float max3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}
// Pairs of fp32 values in one 64-bit register for the packed f32x2 instructions (two
// lanes per instruction, each rounded as the scalar instruction would round it).
typedef unsigned long long f32x2;
__device__ __forceinline__ f32x2 pk2(float lo, float hi) {
  f32x2 r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void upk2(f32x2 v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ f32x2 fma2(f32x2 a, f32x2 b, f32x2 c) {
  f32x2 d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ f32x2 mul2(f32x2 a, f32x2 b) {
  f32x2 d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ f32x2 add2(f32x2 a, f32x2 b) {
  f32x2 d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ float lg2(float x) {
  float y;
  asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// TMEM columns (512 allocated): O of tile A and B, the shared S region, scale factors,
// and each tile's quantised P (row r in lane r, 4 bytes of consecutive keys per column;
// the A operand of its P V MMAs).
constexpr uint32_t kColO0 = 0, kColO1 = 128, kColS = 256;
constexpr uint32_t kColSFQ = 384, kColSFK = 400, kColSFP = 416, kColSFV = 432;   // + 8 * tile
constexpr uint32_t kColP = 448;                                                   // + 32 * tile

// shared memory carve-up (bytes)
constexpr uint32_t kQ8 = 0, kQ4 = 16384, kSFQ = 24576, kQBytes = 25600;   // per tile
constexpr uint32_t kStage0 = 2 * kQBytes;
constexpr uint32_t kStK = 0, kStV = 16384, kStSFK = 32768, kStSFV = 33792, kStageBytes = 34816;
constexpr uint32_t kMask = kStage0 + kStages * kStageBytes;   // 5 slot-validity masks x 4 words
constexpr uint32_t kEdge = kMask + 128;            // edge class of every block (u8 [N <= 4096])
constexpr int kNoBlock = 4;                        // mask class of a -1 list entry: no valid key
constexpr uint32_t kBar = kEdge + 4096;
constexpr uint32_t kSmemBytes = kBar + 256;
static_assert(kSmemBytes <= 232448, "shared memory budget");

struct TileBars {
  uint64_t s_full, s_free, p_full, p_free, q_full, q_empty, o_full, o_free;
};
struct Bars {
  uint64_t kv_full[kStages], kv_empty[kStages];
  TileBars tb[2];
  uint64_t done;
  uint32_t tmem;
};
static_assert(sizeof(Bars) <= 256, "barrier area");

__device__ __forceinline__ uint64_t gtime() {
  uint64_t t;
  asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
  return t;
}

// Bounded wait, slow path: polls until the phase completes or `limit_ns` have passed (2 s
// in use: nothing here legitimately waits that long), then records the timeout in the
// error word and returns false. Once any wait of the launch has run out, every later wait
// returns at once, so a broken pipeline drains quickly instead of timing out wait by wait.
__device__ __noinline__ bool wait_bar_slow(uint64_t* bar, uint32_t parity, uint32_t* err,
                                           unsigned long long limit_ns, bool honour_abort) {
  const uint64_t t0 = gtime();
  while (true) {
    for (int i = 0; i < 32; ++i)
      if (tc::mbar_try_wait(bar, parity)) return true;
    if (honour_abort && (*reinterpret_cast<volatile uint32_t*>(err) & kErrWaitTimeout)) return false;
    if (gtime() - t0 > limit_ns) {
      set_error(err, kErrWaitTimeout);
      return false;
    }
  }
}
// Fast path inline: one non-blocking test of the phase.
__device__ __forceinline__ bool wait_bar(uint64_t* bar, uint32_t parity, uint32_t* err,
                                         unsigned long long limit_ns, bool honour_abort = true) {
  if (tc::mbar_test_wait(bar, parity)) return true;
  return wait_bar_slow(bar, parity, err, limit_ns, honour_abort);
}

__device__ __forceinline__ int block_valid_rows(const Geo& g, int n, int& hv, int& wv) {
  const int fpf = g.ny * g.nx;
  const int rem = n % fpf, by = rem / g.nx, bx = rem - by * g.nx;
  hv = min(g.ph, g.Hf - by * g.ph);
  wv = min(g.pw, g.Wf - bx * g.pw);
  return hv * wv;
}

// O row *= alpha in TMEM (D columns from taddr). Out of line: after the first few blocks
// the running max rarely moves, and the unrolled body would sit in the hot loop's code.
template <int D>
__device__ __noinline__ void rescale_o(uint32_t taddr, float alpha) {
#pragma unroll
  for (int h0 = 0; h0 < D; h0 += 32) {
    uint32_t orr[32];
    tc::tmem_ld16(taddr + h0, orr);
    tc::tmem_ld16(taddr + h0 + 16, orr + 16);
    tc::tmem_wait_ld16(orr);
    tc::tmem_wait_ld16(orr + 16);
#pragma unroll
    for (int e = 0; e < 32; ++e) orr[e] = __float_as_uint(__uint_as_float(orr[e]) * alpha);
    tc::tmem_st16(taddr + h0, orr);
    tc::tmem_st16(taddr + h0 + 16, orr + 16);
  }
  tc::tmem_wait_st();
}

// One KV block of one query row of a tile (softmax warps; FP8 selects the block's
// precision). The S row is read once from the shared S region (which is released at once)
// -> group maxima -> row max -> alpha -> one fused loop computing p448 = 2^(S c + log2 448
// - m_new), the row sum and the quantised P (E4M3, or E2M1 with an E4M3 scale per 16
// keys), stored with tcgen05.st into the tile's P columns of tensor memory (after the
// tile's previous P V has landed) -> O rescale by alpha in TMEM when the max moved -> P
// ready.
// gx counts this tile's blocks over the whole launch. A wait that runs out does not stop
// the block (checking here costs the loop several percent): after a timeout every later
// wait returns at once, so the rest of the round runs through without waiting and the
// warpgroup stops at the round's epilogue.
template <int D, int BS, bool FP8>
__device__ __forceinline__ void softmax_block(const Ws& w, TileBars* tb, uint8_t* sm, uint32_t colP,
                                              uint32_t tmem, uint32_t lane_base, uint32_t colO, int r,
                                              float c, int ecls, uint32_t gx, int t, float& m, float& l,
                                              unsigned long long wait_ns) {
  constexpr int NG = BS / 16;
  constexpr int KV4 = BS < 64 ? 64 : BS;
  wait_bar(&tb->s_full, gx & 1, w.err, wait_ns);
  tc::fence_after_sync();
  uint32_t sr[BS];
#pragma unroll
  for (int c0 = 0; c0 < BS; c0 += 32) tc::tmem_ld32(tmem + lane_base + kColS + c0, sr + c0);
#pragma unroll
  for (int c0 = 0; c0 < BS; c0 += 16) tc::tmem_wait_ld16(sr + c0);
  tc::fence_before_sync();
  tc::mbar_arrive(&tb->s_free);                          // the S region may be reused
  float* s = reinterpret_cast<float*>(sr);
  if (ecls != 0) {                                        // padded slots of an edge block
    const uint32_t* mw = reinterpret_cast<const uint32_t*>(sm + kMask) + ecls * 4;
#pragma unroll
    for (int q = 0; q < BS / 32; ++q) {
      const uint32_t bits = mw[q];
#pragma unroll
      for (int e = 0; e < 32; ++e)
        if (!((bits >> e) & 1u)) s[32 * q + e] = -INFINITY;
    }
  }
  // group maxima of the raw dot products (c > 0, so they order like S)
  float gm[NG];
#pragma unroll
  for (int q = 0; q < NG; ++q) {
    const float* x = s + 16 * q;
    gm[q] = fmaxf(max3(max3(x[0], x[1], x[2]), max3(x[3], x[4], x[5]), max3(x[6], x[7], x[8])),
                  max3(max3(x[9], x[10], x[11]), max3(x[12], x[13], x[14]), x[15]));
  }
  float mh = gm[0];
#pragma unroll
  for (int q = 1; q < NG; ++q) mh = fmaxf(mh, gm[q]);
  const float m_new = fmaxf(m, mh * c);
  // a row whose blocks so far held no valid key keeps m = -inf: alpha 1, and the bias
  // stays finite so that its p are 0
  const bool none = m_new == -INFINITY;
  const float alpha = none ? 1.0f : ex2(m - m_new);
  const float bias = kLog2_448 - (none ? 0.0f : m_new);
  // The quantised P stays in registers until the exponential loop is done: only then does
  // the row wait for its tile's previous P V (which frees the P columns and O), so that
  // wait overlaps the loop.
  auto wait_p_free = [&]() {
    if (t > 0) {
      wait_bar(&tb->p_free, (gx - 1) & 1, w.err, wait_ns);
      tc::fence_after_sync();
    }
  };
  // row-sum partials: keys 4i+0/4i+1 in sA, 4i+2/4i+3 in sB
  f32x2 sA = pk2(0.0f, 0.0f), sB = pk2(0.0f, 0.0f);
  const f32x2 c2 = pk2(c, c);
  if constexpr (FP8) {
    const f32x2 b2 = pk2(bias, bias);
    uint32_t wd[BS / 4];
#pragma unroll
    for (int q = 0; q < NG; ++q) {
#pragma unroll
      for (int e = 0; e < 16; e += 4) {
        float x0, x1, x2, x3;
        upk2(fma2(pk2(s[16 * q + e], s[16 * q + e + 1]), c2, b2), x0, x1);
        upk2(fma2(pk2(s[16 * q + e + 2], s[16 * q + e + 3]), c2, b2), x2, x3);
        const float p0 = ex2(x0), p1 = ex2(x1), p2 = ex2(x2), p3 = ex2(x3);
        sA = add2(sA, pk2(p0, p1));
        sB = add2(sB, pk2(p2, p3));
        wd[4 * q + e / 4] = (uint32_t)f32x2_to_e4m3x2(p0, p1) | ((uint32_t)f32x2_to_e4m3x2(p2, p3) << 16);
      }
    }
    wait_p_free();
    if constexpr (NG >= 4) {
#pragma unroll
      for (int q = 0; q < NG; q += 4) tc::tmem_st16(tmem + lane_base + colP + 4 * q, wd + 4 * q);
    } else {
#pragma unroll
      for (int q = 0; q < NG; ++q) tc::tmem_st4(tmem + lane_base + colP + 4 * q, wd + 4 * q);
    }
  } else {
    uint32_t sfw[KV4 / 64];
#pragma unroll
    for (int q = 0; q < KV4 / 64; ++q) sfw[q] = 0u;
    // Group scales first (independent chains): sigma = E4M3(448 p_max / 6), p_max from the
    // group max. The E2M1 operand y = p448 / sigma is then taken as one exp2 with the
    // group's shift -log2(sigma) folded into the bias, and the row sum gets sigma times
    // the group's sum of y. A group with sigma = 0 keeps shift 0: its p448 are below a
    // quarter, so their E2M1 codes are 0, and its sum is p448 itself.
    float gb[NG], gs[NG];
#pragma unroll
    for (int q = 0; q < NG; q += 2) {                       // two groups at a time
      float z0, z1;
      upk2(fma2(pk2(gm[q], gm[q + 1]), pk2(c, c), pk2(bias, bias)), z0, z1);
      upk2(mul2(pk2(ex2(z0), ex2(z1)), pk2(1.0f / 6.0f, 1.0f / 6.0f)), z0, z1);
      const uint32_t sc2 = f32x2_to_e4m3x2(z0, z1);          // group q in the low byte
      uint32_t h2;
      asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"((uint16_t)sc2));
      const float2 sg = __half22float2(*reinterpret_cast<const __half2*>(&h2));
      gb[q] = sg.x > 0.0f ? bias - lg2(sg.x) : bias;
      gb[q + 1] = sg.y > 0.0f ? bias - lg2(sg.y) : bias;
      gs[q] = sg.x > 0.0f ? sg.x : 1.0f;
      gs[q + 1] = sg.y > 0.0f ? sg.y : 1.0f;
      sfw[q >> 2] |= sc2 << (8 * (q & 3));
    }
    uint32_t pw[2 * NG];
#pragma unroll
    for (int q = 0; q < NG; ++q) {
      const f32x2 b2 = pk2(gb[q], gb[q]);
      float y[16];
      f32x2 yA = pk2(0.0f, 0.0f), yB = pk2(0.0f, 0.0f);
#pragma unroll
      for (int e = 0; e < 16; e += 4) {
        float x0, x1, x2, x3;
        upk2(fma2(pk2(s[16 * q + e], s[16 * q + e + 1]), c2, b2), x0, x1);
        upk2(fma2(pk2(s[16 * q + e + 2], s[16 * q + e + 3]), c2, b2), x2, x3);
        y[e] = ex2(x0);
        y[e + 1] = ex2(x1);
        y[e + 2] = ex2(x2);
        y[e + 3] = ex2(x3);
        yA = add2(yA, pk2(y[e], y[e + 1]));
        yB = add2(yB, pk2(y[e + 2], y[e + 3]));
      }
      float a0, a1, b0, b1;
      upk2(yA, a0, a1);
      upk2(yB, b0, b1);
      const float gsum = (a0 + a1) + (b0 + b1);
      if (q & 1) sB = add2(sB, pk2(gs[q] * gsum, 0.0f));
      else sA = add2(sA, pk2(gs[q] * gsum, 0.0f));
      pw[2 * q] = f32x8_to_e2m1x8(y);
      pw[2 * q + 1] = f32x8_to_e2m1x8(y + 8);
    }
    wait_p_free();
#pragma unroll
    for (int q = 0; q < NG; q += 2) tc::tmem_st4(tmem + lane_base + colP + 2 * q, pw + 2 * q);
#pragma unroll
    for (int gk = BS; gk < KV4; gk += 16)                  // zero keys past the block (32-token blocks)
      tc::tmem_st2(tmem + lane_base + colP + gk / 8, 0u, 0u);
    // This row's scale word for each 64-key step, where the MMA reads it: lane r, column
    // 4 kb + (r / 32) of the tile's P scale columns (the layout that copying a replicated
    // 32-row scale atom leaves there).
    const uint32_t sfp = kColSFP + (colP - kColP) / 4;   // + 8 * tile
#pragma unroll
    for (int q = 0; q < KV4 / 64; ++q) tc::tmem_st1(tmem + lane_base + sfp + 4 * q + (r >> 5), sfw[q]);
  }
  float s0, s1, s2, s3;
  upk2(sA, s0, s1);
  upk2(sB, s2, s3);
  l = fmaf(l, alpha, (s0 + s1) + (s2 + s3));
  // O row *= alpha (the previous P V of this tile has landed: waited above)
  if (t > 0 && __any_sync(0xffffffffu, alpha != 1.0f)) rescale_o<D>(tmem + lane_base + colO, alpha);
  m = m_new;
  tc::tmem_wait_st();                                     // P and its scales are in TMEM
  tc::fence_before_sync();
  tc::mbar_arrive(&tb->p_full);
}

template <int D, int BS>
__global__ void __launch_bounds__(kThreads, 1) k_attention_tc(Geo g, Ws w, __nv_bfloat16* __restrict__ out) {
  extern __shared__ __align__(1024) uint8_t sm[];
  Bars* bars = reinterpret_cast<Bars*>(sm + kBar);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int N = g.N, BH = g.B * g.H;
  // phases: blocks t < n8 FP8, n8 <= t < n8m mixed (E4M3 scores, E2M1 P V), then FP4
  // with the adaptive budget every row runs n4max FP4 entries; -1 entries are no block
  // (a fully masked block that contributes nothing)
  const int n8 = g.n8, n8m = g.n8 + g.nm, nb = g.n8 + g.nm + g.n4max;
  const int total = BH * N;
  constexpr int KV4 = BS < 64 ? 64 : BS;
  // work items of this CTA: blockIdx.x + m gridDim.x; round k takes m = 2k (A), 2k+1 (B)
  const int my_items = (int)blockIdx.x < total ? (total - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;
  const int rounds = (my_items + 1) / 2;
  auto item_of = [&](int k, int x) { return (int)blockIdx.x + (2 * k + x) * (int)gridDim.x; };
  auto has_tile = [&](int k, int x) { return 2 * k + x < my_items; };

  // ---- set-up: barriers, zeroed Q tiles (rows >= bs stay zero), edge tables, TMEM ----
  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      tc::mbar_init(&bars->kv_full[s], 1);
      tc::mbar_init(&bars->kv_empty[s], 1);
    }
    for (int x = 0; x < 2; ++x) {
      TileBars* tb = &bars->tb[x];
      tc::mbar_init(&tb->s_full, 1);
      tc::mbar_init(&tb->s_free, 128);
      tc::mbar_init(&tb->p_full, 128);
      tc::mbar_init(&tb->p_free, 1);
      tc::mbar_init(&tb->q_full, 1);
      tc::mbar_init(&tb->q_empty, 1);
      tc::mbar_init(&tb->o_full, 1);
      tc::mbar_init(&tb->o_free, 128);
    }
    tc::mbar_init(&bars->done, 2);
    tc::fence_mbar_init();
  }
  for (uint32_t o = tid * 16; o < kStage0; o += kThreads * 16)
    *reinterpret_cast<uint4*>(sm + o) = make_uint4(0u, 0u, 0u, 0u);
  // Edge tables: class of each block (bit 1: last window row is short, bit 0: last window
  // column is short) and, per class, which of the BS slots hold real tokens.
  {
    const int hl = g.Hf - (g.ny - 1) * g.ph, wl = g.Wf - (g.nx - 1) * g.pw;
    uint8_t* ecl = sm + kEdge;
    for (int n = tid; n < N; n += kThreads) {
      const int rem = n % (g.ny * g.nx), by = rem / g.nx, bx = rem - by * g.nx;
      ecl[n] = (uint8_t)(((by == g.ny - 1 && hl < g.ph) ? 2 : 0) | ((bx == g.nx - 1 && wl < g.pw) ? 1 : 0));
    }
    if (tid < 20) {                                      // class 4 (no block) keeps no slot
      const int cls = tid >> 2, q = tid & 3;
      const int hv = (cls & 2) ? hl : g.ph, wv = (cls & 1) ? wl : g.pw;
      uint32_t bits = 0u;
      for (int e = 0; e < 32; ++e) {
        const int k = 32 * q + e, ky = k / g.pw, kx = k - ky * g.pw;
        if (cls < kNoBlock && k < BS && ky < hv && kx < wv) bits |= 1u << e;
      }
      reinterpret_cast<uint32_t*>(sm + kMask)[tid] = bits;
    }
  }
  if (warp == kMmaWarp) {
    tc::tmem_alloc(&bars->tmem, 512);
    tc::tmem_relinquish();
  }
  tc::fence_proxy_async_smem();
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = bars->tmem;

  if (warp >= 8) {
  if (warp == kLoadWarp) {
    // ===================== producer =====================
    if (lane == 0 && nb > 0) {
      uint32_t gkv = 0;
      auto list_j = [&](const int16_t* l8, const int16_t* lm, const int16_t* l4, int t) {
        const int j = t < n8 ? l8[t] : (t < n8m ? lm[t - n8] : l4[t - n8m]);
        return (j < 0 || j >= N) ? 0 : j;
      };
      // K at 8 bits for FP8 and mixed blocks, V at 8 bits for FP8 blocks only
      auto kv_prefetch = [&](int bh, int j, int t) {
        const size_t kj = (size_t)bh * N + j;
        if (t < n8m) tc::prefetch_l2(w.k8 + kj * w.tile8_qk, BS * D);
        else tc::prefetch_l2(w.k4 + kj * w.tile4_qk, BS * D / 2);
        if (t < n8) tc::prefetch_l2(w.v8 + kj * w.tile8_v, BS * D);
        else tc::prefetch_l2(w.v4 + kj * w.tile4_v, D * KV4 / 2);
      };
      bool dead = false;                // a wait ran out: issue nothing more
      int q_rounds[2] = {0, 0};         // Q tiles loaded per tile
      const bool stall = (g.flags & DA2_FLAG_TEST_STALL) != 0;   // test hook: stage 0 never fills
      for (int k = 0; k < rounds && !dead; ++k) {
        const int nx = has_tile(k, 1) ? 2 : 1;
        int bhx[2], ix[2];
        const int16_t* l8x[2];
        const int16_t* lmx[2];
        const int16_t* l4x[2];
        for (int x = 0; x < nx && !dead; ++x) {
          const int item = item_of(k, x);
          bhx[x] = item / N;
          ix[x] = item - bhx[x] * N;
          const size_t qi = (size_t)bhx[x] * N + ix[x];
          l8x[x] = w.list8 + qi * w.n8s;
          lmx[x] = w.listm + qi * w.nms;
          l4x[x] = w.list4 + qi * w.n4s;
          TileBars* tb = &bars->tb[x];
          if (!wait_bar(&tb->q_empty, (k & 1) ^ 1, w.err, g.wait_ns)) { dead = true; break; }
          const uint32_t qbytes = BS * D + BS * D / 2 + (uint32_t)w.sf_qk;
          uint8_t* qs = sm + x * kQBytes;
          tc::mbar_arrive_expect_tx(&tb->q_full, qbytes);
          tc::bulk_g2s(qs + kQ8, w.q8 + qi * w.tile8_qk, BS * D, &tb->q_full);
          tc::bulk_g2s(qs + kQ4, w.q4 + qi * w.tile4_qk, BS * D / 2, &tb->q_full);
          tc::bulk_g2s(qs + kSFQ, w.sfq4 + qi * w.sf_qk, (uint32_t)w.sf_qk, &tb->q_full);
          ++q_rounds[x];
        }
        if (dead) break;
        for (int t = 0; t < kPrefetch / 2 && t < nb; ++t)
          for (int x = 0; x < nx; ++x) kv_prefetch(bhx[x], list_j(l8x[x], lmx[x], l4x[x], t), t);
        for (int t = 0; t < nb && !dead; ++t) {
          const bool k8 = t < n8m, v8 = t < n8;
          for (int x = 0; x < nx; ++x) {
            if (t + kPrefetch / 2 < nb)
              kv_prefetch(bhx[x], list_j(l8x[x], lmx[x], l4x[x], t + kPrefetch / 2), t + kPrefetch / 2);
            const int j = list_j(l8x[x], lmx[x], l4x[x], t);
            const size_t kj = (size_t)bhx[x] * N + j;
            const uint32_t s = gkv % kStages, ks = gkv / kStages;
            if (stall && gkv == 0) {      // withhold the first K/V tile: its consumer's wait runs out
              ++gkv;
              continue;
            }
            if (!wait_bar(&bars->kv_empty[s], (ks & 1) ^ 1, w.err, g.wait_ns)) { dead = true; break; }
            uint8_t* st = sm + kStage0 + s * kStageBytes;
            const uint32_t kbytes = k8 ? BS * D : BS * D / 2 + (uint32_t)w.sf_qk;
            const uint32_t vbytes = v8 ? BS * D : D * KV4 / 2 + (uint32_t)w.sf_v;
            tc::mbar_arrive_expect_tx(&bars->kv_full[s], kbytes + vbytes);
            if (k8) {
              tc::bulk_g2s(st + kStK, w.k8 + kj * w.tile8_qk, BS * D, &bars->kv_full[s]);
            } else {
              tc::bulk_g2s(st + kStK, w.k4 + kj * w.tile4_qk, BS * D / 2, &bars->kv_full[s]);
              tc::bulk_g2s(st + kStSFK, w.sfk4 + kj * w.sf_qk, (uint32_t)w.sf_qk, &bars->kv_full[s]);
            }
            if (v8) {
              tc::bulk_g2s(st + kStV, w.v8 + kj * w.tile8_v, BS * D, &bars->kv_full[s]);
            } else {
              tc::bulk_g2s(st + kStV, w.v4 + kj * w.tile4_v, D * KV4 / 2, &bars->kv_full[s]);
              tc::bulk_g2s(st + kStSFV, w.sfv4 + kj * w.sf_v, (uint32_t)w.sf_v, &bars->kv_full[s]);
            }
            ++gkv;
          }
        }
      }
      // Every copy issued above has landed before this thread leaves (normally they were
      // consumed long ago; after an aborted wait they may still be in flight).
      for (uint32_t s = 0; s < (uint32_t)kStages && s < gkv; ++s) {
        const uint32_t last = s + ((gkv - 1 - s) / kStages) * kStages;
        wait_bar(&bars->kv_full[s], (last / kStages) & 1, w.err, g.wait_ns, false);
      }
      for (int x = 0; x < 2; ++x)
        if (q_rounds[x] > 0) wait_bar(&bars->tb[x].q_full, (q_rounds[x] - 1) & 1, w.err, g.wait_ns, false);
    }
  } else if (warp == kMmaWarp || warp == kMmaWarp + 2) {
    // ============ MMA issue: one thread per tile (warp 8: tile A, warp 10: tile B) ============
    const int x = warp == kMmaWarp ? 0 : 1;
    if (lane == 0 && nb > 0) {
      const uint32_t id8_s = tc::idesc_e4m3(128, BS), id4_s = tc::idesc_nvf4(128, BS);
      const uint32_t id8_o = tc::idesc_e4m3(128, D), id4_o = tc::idesc_nvf4(128, D);
      TileBars* tb = &bars->tb[x];
      const uint8_t* qs = sm + x * kQBytes;
      const uint32_t aP = tmem + kColP + 32 * x;          // P: the A operand of P V, in TMEM
      const uint32_t dO = tmem + (x ? kColO1 : kColO0);
      bool dead = false;                // a wait ran out: issue nothing more
      for (int k = 0; k < rounds && !dead; ++k) {
        if (!has_tile(k, x)) break;     // only tile B can be missing, in the last round only
        const int nx = has_tile(k, 1) ? 2 : 1;
        const uint32_t gbase = (uint32_t)k * (uint32_t)nb;   // blocks each tile had in earlier rounds
        const uint32_t kvbase = 2u * gbase;                  // K/V stages of earlier rounds (2 tiles each)
        dead = !wait_bar(&tb->q_full, k & 1, w.err, g.wait_ns);
        tc::fence_after_sync();
        if (!dead && nb > n8m)                               // blocks with E2M1 scores follow
          for (int kb = 0; kb < D / 64; ++kb)
            tc::cp_sf_atom(tmem + kColSFQ + 8 * x + kb * 4, qs + kSFQ + kb * 512);
        // The S region is taken in the order A0 B0 A1 B1 ... (A0 A1 ... when B is absent),
        // continuing across rounds; S of this tile's block t waits until the softmax of the
        // previous owner has read its S.
        auto issue_s = [&](int t) -> bool {
          if (x == 1) {
            if (!wait_bar(&bars->tb[0].s_free, (gbase + t) & 1, w.err, g.wait_ns)) return false;
          } else if (t > 0) {
            if (!wait_bar(&bars->tb[nx - 1].s_free, (gbase + t - 1) & 1, w.err, g.wait_ns)) return false;
          } else if (k > 0) {
            if (!wait_bar(&bars->tb[1].s_free, (gbase - 1) & 1, w.err, g.wait_ns)) return false;
          }
          const uint32_t seq = kvbase + (uint32_t)(nx * t + x);   // K/V stage sequence number
          const uint32_t s = seq % kStages;
          if (!wait_bar(&bars->kv_full[s], (seq / kStages) & 1, w.err, g.wait_ns)) return false;
          tc::fence_after_sync();
          const uint8_t* st = sm + kStage0 + s * kStageBytes;
          if (t < n8m) {                                      // FP8 and mixed blocks: E4M3 scores
#pragma unroll
            for (int kk = 0; kk < D / 32; ++kk)
              tc::mma_e4m3(tmem + kColS, tc::sdesc(qs + kQ8 + kk * 256, 128, D * 8),
                           tc::sdesc(st + kStK + kk * 256, 128, D * 8), id8_s, kk > 0);
          } else {
            for (int kb = 0; kb < D / 64; ++kb)
              tc::cp_sf_atom(tmem + kColSFK + 8 * x + kb * 4, st + kStSFK + kb * 512);
#pragma unroll
            for (int kk = 0; kk < D / 64; ++kk)
              tc::mma_nvf4(tmem + kColS, tc::sdesc(qs + kQ4 + kk * 256, 128, D * 4),
                           tc::sdesc(st + kStK + kk * 256, 128, D * 4), id4_s,
                           tmem + kColSFQ + 8 * x + kk * 4, tmem + kColSFK + 8 * x + kk * 4, kk > 0);
          }
          tc::mma_commit(&tb->s_full);
          return true;
        };
        // O += P V of this tile's block t
        auto issue_pv = [&](int t) -> bool {
          if (!wait_bar(&tb->p_full, (gbase + (uint32_t)t) & 1, w.err, g.wait_ns)) return false;
          if (t == 0 && k > 0 && !wait_bar(&tb->o_free, (k - 1) & 1, w.err, g.wait_ns)) return false;
          tc::fence_after_sync();
          const uint32_t s = (kvbase + (uint32_t)(nx * t + x)) % kStages;
          const uint8_t* st = sm + kStage0 + s * kStageBytes;
          const uint32_t acc0 = t > 0 ? 1u : 0u;
          if (t < n8) {
#pragma unroll
            for (int kk = 0; kk < BS / 32; ++kk)
              tc::mma_e4m3_ta(dO, aP + kk * 8, tc::sdesc(st + kStV + kk * 256, 128, BS * 8), id8_o,
                              acc0 | (kk > 0));
          } else {
            for (int kb = 0; kb < KV4 / 64; ++kb)
              tc::cp_sf_atom(tmem + kColSFV + 8 * x + kb * 4, st + kStSFV + kb * 512);
#pragma unroll
            for (int kk = 0; kk < KV4 / 64; ++kk)
              tc::mma_nvf4_ta(dO, aP + kk * 8, tc::sdesc(st + kStV + kk * 256, 128, KV4 * 4), id4_o,
                              tmem + kColSFP + 8 * x + kk * 4, tmem + kColSFV + 8 * x + kk * 4,
                              acc0 | (kk > 0));
          }
          tc::mma_commit(&tb->p_free);
          tc::mma_commit(&bars->kv_empty[s]);
          return true;
        };
        // This tile's next S is issued as soon as the S region comes free, ahead of the
        // current block's P V, so that it is ready when the softmax finishes the block.
        dead = dead || !issue_s(0);
        for (int t = 0; t < nb && !dead; ++t) {
          if (t + 1 < nb) dead = !issue_s(t + 1);
          if (!dead) dead = !issue_pv(t);
        }
        if (!dead) {
          tc::mma_commit(&tb->q_empty);
          tc::mma_commit(&tb->o_full);
        }
      }
      tc::mma_commit(&bars->done);
      wait_bar(&bars->done, 0, w.err, g.wait_ns, false);   // both issuers' MMAs retired before TMEM is freed
    }
  }
  } else {
    // ============ softmax + epilogue (warps 0-3: tile A, 4-7: tile B) ============
    const int x = warp >> 2;
    const int r = (warp & 3) * 32 + lane;               // query row = TMEM lane
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t colO = x ? kColO1 : kColO0;
    TileBars* tb = &bars->tb[x];
    const uint32_t colP = kColP + 32 * x;
    const int fpf = g.ny * g.nx;
    uint32_t gx = 0;                                     // blocks of this tile so far
    bool dead = false;                                   // a wait ran out: stop
    for (int k = 0; k < rounds && !dead; ++k) {
      if (!has_tile(k, x)) break;
      const int item = item_of(k, x);
      const int bh = item / N, i = item - bh * N;
      const size_t qi = (size_t)bh * N + i;
      int hq, wq;
      block_valid_rows(g, i, hq, wq);
      const int wy = r / g.pw, wx = r - wy * g.pw;
      const bool row_ok = r < BS && wy < hq && wx < wq;
      __nv_bfloat16* orow = nullptr;
      if (row_ok) {
        const int f = i / fpf, rem = i - f * fpf, by = rem / g.nx, bx = rem - by * g.nx;
        const size_t tk = (size_t)f * g.Hf * g.Wf + (size_t)(by * g.ph + wy) * g.Wf + bx * g.pw + wx;
        orow = out + tok_off(g, bh, tk);
      }
      if (nb == 0) {
        if (row_ok)
          for (int c = 0; c < D; c += 8) *reinterpret_cast<uint4*>(orow + c) = make_uint4(0u, 0u, 0u, 0u);
        continue;
      }
      const float sq = w.sq[qi];

      float m = -INFINITY, l = 0.0f;
      // Block index j and key scale s_k[j] of every visited block, fetched 32 blocks at a
      // time (lane i holds block 32 ch + i) and broadcast by shuffles: the list entries of
      // chunk ch + 2 and the scales of chunk ch + 1 are loaded at the start of chunk ch,
      // so no block waits on a global load.
      const float cq = sq * g.sm_scale * kLog2e;
      const float* skh = w.sk + (size_t)bh * N;
      // list entries are fetched 32 blocks at a time; the three lists' addresses follow
      // from the work item when needed (fewer live registers in the block loop)
      auto list_j = [&](int t) -> int {
        int j = 0;
        if (t < n8) j = w.list8[qi * w.n8s + t];
        else if (t < n8m) j = w.listm[qi * w.nms + (t - n8)];
        else if (t < nb) j = w.list4[qi * w.n4s + (t - n8m)];
        return j < 0 ? -1 : (j >= N ? 0 : j);            // -1: no block
      };
      int jA = list_j(lane), jB = list_j(32 + lane), jC = list_j(64 + lane);
      float sA = skh[jA < 0 ? 0 : jA], sB = skh[jB < 0 ? 0 : jB];
      // one loop per P precision (FP8 blocks, then mixed and FP4 blocks), each with a
      // single softmax body
      auto step = [&](auto fp8, int t) {
        const int ln = t & 31;
        const int j = __shfl_sync(0xffffffffu, jA, ln);
        const float c = cq * __shfl_sync(0xffffffffu, sA, ln);
        if (ln == 31) {                                   // next chunk
          jA = jB;
          sA = sB;
          jB = jC;
          sB = skh[jB < 0 ? 0 : jB];
          jC = list_j(t + 65 + lane);
        }
        const int ecls = j < 0 ? kNoBlock : sm[kEdge + j];
        softmax_block<D, BS, decltype(fp8)::value>(w, tb, sm, colP, tmem, lane_base, colO, r, c, ecls, gx, t, m,
                                                     l, g.wait_ns);
      };
      int t = 0;
      for (; t < n8; ++t, ++gx) step(std::true_type{}, t);
      for (; t < nb; ++t, ++gx) step(std::false_type{}, t);
      // ---- epilogue: O / l, V channel scale, bf16, original token order ----
      if (!wait_bar(&tb->o_full, k & 1, w.err, g.wait_ns)) {
        dead = true;
        break;
      }
      tc::fence_after_sync();
      const float inv = l > 0.0f ? 1.0f / l : 0.0f;     // l holds 448 * row sum
      const float* sv = w.sv + (size_t)bh * D;
#pragma unroll
      for (int h0 = 0; h0 < D; h0 += 64) {
        uint32_t rr[64];
#pragma unroll
        for (int c0 = 0; c0 < 64; c0 += 16) tc::tmem_ld16(tmem + lane_base + colO + h0 + c0, rr + c0);
#pragma unroll
        for (int c0 = 0; c0 < 64; c0 += 16) tc::tmem_wait_ld16(rr + c0);
        if (row_ok) {
#pragma unroll
          for (int c0 = 0; c0 < 64; c0 += 8) {
            uint32_t pk[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int cc = h0 + c0 + 2 * e;
              const float a = __uint_as_float(rr[c0 + 2 * e]) * __ldg(sv + cc) * inv;
              const float bq = __uint_as_float(rr[c0 + 2 * e + 1]) * __ldg(sv + cc + 1) * inv;
              const __nv_bfloat162 hh = __floats2bfloat162_rn(a, bq);
              pk[e] = *reinterpret_cast<const uint32_t*>(&hh);
            }
            *reinterpret_cast<uint4*>(orow + h0 + c0) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
          }
        }
      }
      tc::fence_before_sync();
      tc::mbar_arrive(&tb->o_free);
    }
  }
  tc::fence_before_sync();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, 512);
  }
}

template <int D, int BS>
cudaError_t launch_tc(const Geo& g, const Ws& w, __nv_bfloat16* out, cudaStream_t st) {
  cudaError_t e = cudaFuncSetAttribute(k_attention_tc<D, BS>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)kSmemBytes);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int total = g.B * g.H * g.N;
  const int grid = total < sms ? total : sms;
  k_attention_tc<D, BS><<<grid, kThreads, kSmemBytes, st>>>(g, w, out);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attention_tc(const Geo& g, const Ws& w, void* out, cudaStream_t st) {
  auto* o = static_cast<__nv_bfloat16*>(out);
  if (g.d == 128) {
    if (g.bs == 128) return launch_tc<128, 128>(g, w, o, st);
    if (g.bs == 64) return launch_tc<128, 64>(g, w, o, st);
    return launch_tc<128, 32>(g, w, o, st);
  }
  if (g.bs == 128) return launch_tc<64, 128>(g, w, o, st);
  if (g.bs == 64) return launch_tc<64, 64>(g, w, o, st);
  return launch_tc<64, 32>(g, w, o, st);
}

}  // namespace da2
