// Draft attention maps and the shared ranking (K2).
//
// "DraftAttention2: Fast Video Diffusion with Low-Resolution-Guided Mixed-Precision
// Attention", Abstract: the low-resolution draft attention map, built from average- and
// max-pooled queries and keys, estimates block importance; one shared ranking per query
// block gives its most important KV blocks high precision, the next ones low precision
// and skips the rest under configurable budgets. "DraftAttention: Fast Video Diffusion via
// Low-Resolution Attention Guidance", Abstract: the draft map is the attention of the
// pooled queries over the pooled keys.
//
// Up to 1024 key blocks: the two logit maps of every (b, h) run on the tensor cores into a
// scratch (k_draft_logits_tc), then k_draft_rank turns each query block's two rows into row
// softmaxes, averages them into the score, and ranks the row with an exact radix select
// over the score bits (ties broken by the lower block index), writing tags and the
// ascending index lists of the kept classes (FP8, mixed, FP4). Above 1024 key blocks one
// kernel (k_draft_select) forms the logits with fp32 FMAs and ranks in the same way.
#include "common.cuh"
#include "split_tiles.cuh"
#include "tc.cuh"

namespace da2 {

// One pass of an 8-bit radix select within one warp: from the 256-bin histogram of the keys
// under the current prefix, the digit that holds the remaining-th largest of them and how
// many keys lie in the digits above it.
__device__ __forceinline__ void radix_pick(const uint32_t* hist, int remaining, int lane, uint32_t& digit,
                                           uint32_t& above) {
  // lane l owns digits 255-8l .. 255-8l-7 (descending)
  uint32_t c[8];
  uint32_t s = 0u;
#pragma unroll
  for (int t = 0; t < 8; ++t) { c[t] = hist[255 - 8 * lane - t]; s += c[t]; }
  uint32_t incl = s;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  const uint32_t excl = incl - s;
  const bool mine = excl < (uint32_t)remaining && (uint32_t)remaining <= incl;
  digit = 0u;
  above = 0u;
  if (mine) {
    uint32_t acc = excl;
#pragma unroll
    for (int t = 0; t < 8; ++t) {
      if (acc + c[t] >= (uint32_t)remaining) { digit = 255u - 8u * lane - t; above = acc; break; }
      acc += c[t];
    }
  }
  const uint32_t found = __ballot_sync(0xffffffffu, mine);
  const int src = found ? __ffs(found) - 1 : 0;   // always found when 1 <= remaining <= keys counted
  digit = __shfl_sync(0xffffffffu, digit, src);
  above = __shfl_sync(0xffffffffu, above, src);
}

// k-th largest 32-bit key of `keys[0..n)` (1 <= kth <= n) by an 8-bit radix select within
// one warp. Returns the key value T and how many of the keys equal to T belong to the top
// kth (the rest of the top kth are strictly greater than T). hist: 256 words.
__device__ void warp_radix_select(const uint32_t* keys, int n, int kth, uint32_t* hist,
                                  uint32_t& T, int& need) {
  const int lane = threadIdx.x & 31;
  uint32_t prefix = 0u, pmask = 0u;
  int remaining = kth;
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int b = lane; b < 256; b += 32) hist[b] = 0u;
    __syncwarp();
    for (int j = lane; j < n; j += 32) {
      const uint32_t u = keys[j];
      if ((u & pmask) == prefix) atomicAdd(&hist[(u >> shift) & 255u], 1u);
    }
    __syncwarp();
    uint32_t digit, above;
    radix_pick(hist, remaining, lane, digit, above);
    prefix |= digit << shift;
    pmask |= 0xFFu << shift;
    remaining -= (int)above;
    __syncwarp();
  }
  T = prefix;
  need = remaining;
}

// The same select for two ranks at once (1 <= ka, kb <= n): each pass reads the keys once,
// counting into one histogram while the two cuts' digit prefixes agree and into two once
// they differ (a key then matches at most one prefix). hist: 512 words.
__device__ void warp_radix_select2(const uint32_t* keys, int n, int ka, int kb, uint32_t* hist,
                                   uint32_t& Ta, int& needa, uint32_t& Tb, int& needb) {
  const int lane = threadIdx.x & 31;
  uint32_t* ha = hist;
  uint32_t* hb = hist + 256;
  uint32_t pa = 0u, pb = 0u, pmask = 0u;
  int ra = ka, rb = kb;
  for (int shift = 24; shift >= 0; shift -= 8) {
    const bool same = pa == pb;
    for (int b = lane; b < (same ? 256 : 512); b += 32) hist[b] = 0u;
    __syncwarp();
    for (int j = lane; j < n; j += 32) {
      const uint32_t u = keys[j];
      const uint32_t m = u & pmask, dg = (u >> shift) & 255u;
      if (m == pa) atomicAdd(&ha[dg], 1u);
      else if (m == pb) atomicAdd(&hb[dg], 1u);
    }
    __syncwarp();
    uint32_t da, aa, db, ab;
    radix_pick(ha, ra, lane, da, aa);
    radix_pick(same ? ha : hb, rb, lane, db, ab);
    pa |= da << shift;
    pb |= db << shift;
    pmask |= 0xFFu << shift;
    ra -= (int)aa;
    rb -= (int)ab;
    __syncwarp();
  }
  Ta = pa;
  needa = ra;
  Tb = pb;
  needb = rb;
}

// The k-th largest for one or two ranks (a rank of 0 is no cut and leaves its outputs).
__device__ __forceinline__ void radix_cuts(const uint32_t* keys, int n, int ka, int kb, uint32_t* hist,
                                           uint32_t& Ta, int& needa, uint32_t& Tb, int& needb) {
  if (ka > 0 && kb > 0) warp_radix_select2(keys, n, ka, kb, hist, Ta, needa, Tb, needb);
  else if (ka > 0) warp_radix_select(keys, n, ka, hist, Ta, needa);
  else if (kb > 0) warp_radix_select(keys, n, kb, hist, Tb, needb);
}

constexpr int kHistWords = 512;   // per warp: the two histograms of warp_radix_select2

constexpr int kDraftThreads = 512, kDraftWarps = kDraftThreads / 32;

// The shared ranking of one score row (one warp; keys = the N scores' bit patterns, which
// order like the non-negative scores): the radix-select cuts, then tags and the ascending
// lists of the kept classes. h: the warp's kHistWords histogram words; row: (b, h, query block).
// MIX: a mixed class (nm > 0); ADAPT: the adaptive FP4 budget (tau > 0, n4max > n4). Without
// them the row needs neither their cuts nor their per-key tests.
template <bool MIX, bool ADAPT>
__device__ __forceinline__ void rank_keys_row_t(const Geo& g, const Ws& w, const uint32_t* keys, uint32_t* h, size_t row,
                                int lane) {
  const int N = g.N;
  const int n8m = g.n8 + g.nm, nk = g.n8 + g.nm + g.n4;   // the ranking's cuts
  const int nkx = g.n8 + g.nm + g.n4max;                    // last rank the adaptive budget may reach
  const uint32_t tau_bits = __float_as_uint(g.tau);       // scores are non-negative: bits order like values
  // the three cuts of the ranking: n8-th, (n8 + nm)-th and nk-th largest score
  // (and the adaptive cap's nkx-th), selected two at a time
  uint32_t T8 = 0xFFFFFFFFu, Tm = 0xFFFFFFFFu, Tk = 0xFFFFFFFFu, Tx = 0xFFFFFFFFu;
  int need8 = 0, needm = 0, needk = 0, needx = 0;
  radix_cuts(keys, N, g.n8, nk, h, T8, need8, Tk, needk);
  if (MIX || ADAPT) radix_cuts(keys, N, MIX ? n8m : 0, ADAPT ? nkx : 0, h, Tm, needm, Tx, needx);
  int eq8 = 0, eqm = 0, eqk = 0, eqx = 0, c8 = 0, cm = 0, c4 = 0;
  uint8_t* trow = w.tags + row * N;
  int16_t* l8 = w.list8 + row * w.n8s;
  int16_t* lmx = w.listm + row * w.nms;
  int16_t* l4 = w.list4 + row * w.n4s;
  const uint32_t lt = (1u << lane) - 1u;
  for (int j0 = 0; j0 < N; j0 += 32) {
    const int j = j0 + lane;
    const bool ok = j < N;
    const uint32_t key = ok ? keys[j] : 0u;
    // keys equal to a cut value belong above it in block order, as many as the cut needs
    const uint32_t e8 = __ballot_sync(0xffffffffu, ok && g.n8 > 0 && key == T8);
    const uint32_t em = MIX ? __ballot_sync(0xffffffffu, ok && key == Tm) : 0u;
    const uint32_t ek = __ballot_sync(0xffffffffu, ok && nk > 0 && key == Tk);
    const uint32_t ex = ADAPT ? __ballot_sync(0xffffffffu, ok && key == Tx) : 0u;
    const bool in8 = ok && g.n8 > 0 && (key > T8 || (key == T8 && eq8 + __popc(e8 & lt) < need8));
    const bool in8m = in8 || (MIX && ok && (key > Tm || (key == Tm && eqm + __popc(em & lt) < needm)));
    const bool ink = ok && nk > 0 && (key > Tk || (key == Tk && eqk + __popc(ek & lt) < needk));
    // adaptive budget: a block ranked after the fixed cut, within the cap, whose score
    // reaches the threshold joins FP4 (those form a prefix of the ranks, scores being
    // sorted within the ranking)
    const bool inx = ADAPT && ok && (key > Tx || (key == Tx && eqx + __popc(ex & lt) < needx));
    const bool rec = inx && !ink && key >= tau_bits;
    eq8 += __popc(e8);
    eqk += __popc(ek);
    if (MIX) eqm += __popc(em);
    if (ADAPT) eqx += __popc(ex);
    const bool inm = in8m && !in8;
    const bool in4 = (ink && !in8m) || rec;
    const uint32_t b8 = __ballot_sync(0xffffffffu, in8), b4 = __ballot_sync(0xffffffffu, in4);
    const uint32_t bm = MIX ? __ballot_sync(0xffffffffu, inm) : 0u;
    const int p8 = c8 + __popc(b8 & lt), p4 = c4 + __popc(b4 & lt);
    if (in8 && p8 < g.n8) l8[p8] = (int16_t)j;
    if (in4 && p4 < g.n4max) l4[p4] = (int16_t)j;
    if (MIX) {
      const int pm = cm + __popc(bm & lt);
      if (inm && pm < g.nm) lmx[pm] = (int16_t)j;
      cm += __popc(bm);
    }
    c8 += __popc(b8);
    c4 += __popc(b4);
    if (ok) trow[j] = in8 ? 2 : (inm ? 3 : (in4 ? 1 : 0));
  }
  for (int p = c4 + lane; p < g.n4max; p += 32) l4[p] = (int16_t)-1;   // no block
  if (lane == 0 && (c8 != g.n8 || cm != g.nm || c4 < g.n4 || c4 > g.n4max)) set_error(w.err, kErrBadIndex);
}

__device__ __forceinline__ void rank_keys_row(const Geo& g, const Ws& w, const uint32_t* keys, uint32_t* h,
                                              size_t row, int lane) {
  const bool mix = g.nm > 0, adapt = g.tau > 0.0f && g.n4max > g.n4;
  if (mix) {
    if (adapt) rank_keys_row_t<true, true>(g, w, keys, h, row, lane);
    else rank_keys_row_t<true, false>(g, w, keys, h, row, lane);
  } else {
    if (adapt) rank_keys_row_t<false, true>(g, w, keys, h, row, lane);
    else rank_keys_row_t<false, false>(g, w, keys, h, row, lane);
  }
}

// Per-row ranking of the draft scores (one warp per row): the two row softmaxes of the
// average- and max-pooled logits (in la / lm, R rows of N), their mean as the score, then
// the shared ranking of the row.
__device__ void rank_rows(const Geo& g, const Ws& w, float* la, float* lm, uint32_t* hist, int bh, int i0,
                          int rows, int warp, int lane, int nwarps) {
  const int N = g.N;
  uint32_t* h = hist + warp * kHistWords;
  for (int r = warp; r < rows; r += nwarps) {
    float* ra = la + r * N;
    float* rm = lm + r * N;
    // two row softmaxes, averaged
    float mxa = -INFINITY, mxm = -INFINITY;
    for (int j = lane; j < N; j += 32) { mxa = fmaxf(mxa, ra[j]); mxm = fmaxf(mxm, rm[j]); }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      mxa = fmaxf(mxa, __shfl_xor_sync(0xffffffffu, mxa, o));
      mxm = fmaxf(mxm, __shfl_xor_sync(0xffffffffu, mxm, o));
    }
    float sa = 0.0f, sm = 0.0f;
    for (int j = lane; j < N; j += 32) {
      const float ea = expf(ra[j] - mxa), em = expf(rm[j] - mxm);
      ra[j] = ea;
      rm[j] = em;
      sa += ea;
      sm += em;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      sa += __shfl_xor_sync(0xffffffffu, sa, o);
      sm += __shfl_xor_sync(0xffffffffu, sm, o);
    }
    const float ia = 1.0f / sa, im = 1.0f / sm;
    const size_t row = (size_t)bh * N + (i0 + r);
    for (int j = lane; j < N; j += 32) {
      const float sc = 0.5f * (ra[j] * ia + rm[j] * im);
      ra[j] = sc;
      if (g.flags & DA2_FLAG_EXPORT_SCORES) w.scores[row * N + j] = sc;
    }
    __syncwarp();
    rank_keys_row(g, w, reinterpret_cast<const uint32_t*>(ra), h, row, lane);
  }
}


template <int D>
__global__ void __launch_bounds__(kDraftThreads) k_draft_select(Geo g, Ws w, int R) {
  extern __shared__ __align__(16) float dsm[];
  const int N = g.N;
  float* qa = dsm;                 // [R][D]
  float* qm = qa + R * D;          // [R][D]
  float* la = qm + R * D;          // [R][N]  avg logits, later the score
  float* lm = la + R * N;          // [R][N]  max logits
  uint32_t* hist = reinterpret_cast<uint32_t*>(lm + R * N);  // [warps][kHistWords]
  const int bh = blockIdx.y, i0 = blockIdx.x * R;
  const int rows = min(R, N - i0);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

  const float* qavg = w.qavg + ((size_t)bh * N + i0) * D;
  const float* qmax = w.qmax + ((size_t)bh * N + i0) * D;
  for (int u = tid; u < R * D / 4; u += kDraftThreads) {
    const bool ok = u < rows * D / 4;
    reinterpret_cast<float4*>(qa)[u] = ok ? reinterpret_cast<const float4*>(qavg)[u] : make_float4(0, 0, 0, 0);
    reinterpret_cast<float4*>(qm)[u] = ok ? reinterpret_cast<const float4*>(qmax)[u] : make_float4(0, 0, 0, 0);
  }
  __syncthreads();

  const bool mass = !(g.flags & DA2_FLAG_NO_MASS_CORRECTION);
  const int fpf = g.ny * g.nx;
  const float* kavg = w.kavg + (size_t)bh * N * D;
  const float* kmax = w.kmax + (size_t)bh * N * D;
  for (int j = tid; j < N; j += kDraftThreads) {
    float aa[16], am[16];
#pragma unroll
    for (int r = 0; r < 16; ++r) { aa[r] = 0.0f; am[r] = 0.0f; }
    const float4* ka = reinterpret_cast<const float4*>(kavg + (size_t)j * D);
    const float4* km = reinterpret_cast<const float4*>(kmax + (size_t)j * D);
    for (int c4 = 0; c4 < D / 4; ++c4) {
      const float4 a = __ldg(ka + c4), m = __ldg(km + c4);
#pragma unroll
      for (int r = 0; r < 16; ++r) {
        if (r < R) {
          const float4 x = reinterpret_cast<const float4*>(qa + r * D)[c4];
          const float4 y = reinterpret_cast<const float4*>(qm + r * D)[c4];
          aa[r] = fmaf(x.x, a.x, aa[r]); aa[r] = fmaf(x.y, a.y, aa[r]);
          aa[r] = fmaf(x.z, a.z, aa[r]); aa[r] = fmaf(x.w, a.w, aa[r]);
          am[r] = fmaf(y.x, m.x, am[r]); am[r] = fmaf(y.y, m.y, am[r]);
          am[r] = fmaf(y.z, m.z, am[r]); am[r] = fmaf(y.w, m.w, am[r]);
        }
      }
    }
    float lc = 0.0f;
    if (mass) {
      const int rem = j % fpf, by = rem / g.nx, bx = rem - by * g.nx;
      const int hv = min(g.ph, g.Hf - by * g.ph), wv = min(g.pw, g.Wf - bx * g.pw);
      lc = logf((float)(hv * wv));
    }
#pragma unroll
    for (int r = 0; r < 16; ++r)
      if (r < R) {
        la[r * N + j] = fmaf(g.sm_scale, aa[r], lc);
        lm[r * N + j] = fmaf(g.sm_scale, am[r], lc);
      }
  }
  __syncthreads();

  rank_rows(g, w, la, lm, hist, bh, i0, rows, warp, lane, kDraftWarps);
}

// ---- draft logits on the tensor cores (N <= 1024) ----
// The two draft maps are dense contractions per head, L_map = Q_map K_map^T ([N, d] x [d, N]),
// run as tcgen05 MMAs of kind::tf32 on operands that the preparation kernel has already split
// into tf32 high parts and their remainders and laid out in the MMA's core-matrix chunks
// (split_tiles.cuh); each K step of 8 channels accumulates hi_a hi_b + hi_a lo_b + lo_a hi_b
// in fp32 (every product of tf32 significands is exact; the dropped lo_a lo_b and the
// remainders' truncation to tf32 stay below 2^-20 of |a b|).
// One CTA takes 128 query blocks (TMEM lanes) of one (b, h) and a range of 128-key tiles,
// one map after the other. Warp 0 (one thread) bulk-copies the map's query chunks once and
// the key chunks through a four-stage ring; warp 1 (one thread) issues the MMAs into one of
// two 128-column TMEM accumulators; warps 2-5 (TMEM lane quarters 2, 3, 0, 1) read a finished
// accumulator out as logits sm_scale * acc + ln c_j into the [B*H][N][2][np] fp32 scratch
// that the ranking kernel reads.
constexpr int kTcRows = 128, kTcKeys = 128, kTcStages = 4, kTcThreads = 192;

__host__ __device__ constexpr uint32_t idesc_tf32(int M, int N) {
  // D fp32, A and B tf32, both K-major, N / 8, M / 16
  return (1u << 4) | (2u << 7) | (2u << 10) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}
__device__ __forceinline__ void mma_tf32(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                         uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate));
}
__device__ __forceinline__ unsigned long long draft_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
// Bounded wait on an mbarrier phase; a wait that runs out sets the error word and returns
// false (the caller stops issuing work).
__device__ __forceinline__ bool draft_wait(uint64_t* bar, uint32_t parity, uint32_t* err,
                                           unsigned long long limit_ns) {
  if (tc::mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = draft_ns();
  while (!tc::mbar_try_wait(bar, parity)) {
    if (draft_ns() - t0 > limit_ns) {
      set_error(err, kErrWaitTimeout);
      return false;
    }
  }
  return true;
}

template <int D>
__global__ void __launch_bounds__(kTcThreads, 1) k_draft_logits_tc(Geo g, Ws w, const uint8_t* __restrict__ qt,
                                                                  const uint8_t* __restrict__ kt,
                                                                  float* dlog, int NP, int tiles_per_cta) {
  constexpr int NKC = D / kSplitKC;                       // 16-channel chunks
  constexpr uint32_t CHUNK = 2 * kSplitPart;              // hi + lo of one chunk, 16 KB
  constexpr uint32_t A_BYTES = NKC * CHUNK;               // all chunks of the queries
  extern __shared__ __align__(1024) uint8_t dsm_tc[];
  uint8_t* a_sm = dsm_tc;                                 // [kc][part][8 KB]
  uint8_t* b_sm = dsm_tc + A_BYTES;                       // [stage][part][8 KB]
  float* lcs = reinterpret_cast<float*>(b_sm + kTcStages * CHUNK);   // ln c_j, [1024]
  uint64_t* bars = reinterpret_cast<uint64_t*>(lcs + 1024);
  uint64_t* a_full = bars;                                // queries of the map in place
  uint64_t* a_empty = bars + 1;                           // MMAs done with them
  uint64_t* b_full = bars + 2;                            // [kTcStages]
  uint64_t* b_empty = b_full + kTcStages;                 // [kTcStages]
  uint64_t* acc_full = b_empty + kTcStages;               // [2]
  uint64_t* acc_empty = acc_full + 2;                     // [2]
  __shared__ uint32_t tmem_holder;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int N = g.N, bh = blockIdx.y, rtile = blockIdx.x, i0 = rtile * kTcRows;
  const int RT = (N + kSplitRows - 1) / kSplitRows;
  const int NT = (N + kTcKeys - 1) / kTcKeys;
  const int t0 = blockIdx.z * tiles_per_cta, t1 = min(NT, t0 + tiles_per_cta);
  if (t0 >= t1) return;
  const int nt = t1 - t0, U = 2 * nt;                     // accumulator tiles of this CTA
  if (warp == 0) {
    tc::tmem_alloc(&tmem_holder, 2 * kTcKeys);
    tc::tmem_relinquish();
  }
  if (tid == 0) {
    tc::mbar_init(a_full, 1);
    tc::mbar_init(a_empty, 1);
    for (int i = 0; i < kTcStages; ++i) {
      tc::mbar_init(&b_full[i], 1);
      tc::mbar_init(&b_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      tc::mbar_init(&acc_full[i], 1);
      tc::mbar_init(&acc_empty[i], 4);                    // one arrival per read-out warp
    }
    tc::fence_mbar_init();
  }
  const bool mass = !(g.flags & DA2_FLAG_NO_MASS_CORRECTION);
  const int fpf = g.ny * g.nx;
  for (int j = tid; j < N; j += kTcThreads) {
    float lc = 0.0f;
    if (mass) {
      const int rem = j % fpf, by = rem / g.nx, bx = rem - by * g.nx;
      const int hv = min(g.ph, g.Hf - by * g.ph), wv = min(g.pw, g.Wf - bx * g.pw);
      lc = logf((float)(hv * wv));
    }
    lcs[j] = lc;
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = tmem_holder;

  if (warp == 0) {
    // ---- copies: per map the query chunks, then the key chunks of every tile ----
    if (lane == 0) {
      int idx = 0;
      for (int m = 0; m < 2; ++m) {
        if (m > 0 && !draft_wait(a_empty, 0, w.err, g.wait_ns)) break;
        tc::mbar_arrive_expect_tx(a_full, A_BYTES);
        for (int kc = 0; kc < NKC; ++kc)
          tc::bulk_g2s(a_sm + kc * CHUNK, qt + split_chunk_off(bh, RT, rtile, m, kc, NKC), CHUNK, a_full);
        bool ok = true;
        for (int tt = 0; tt < nt && ok; ++tt)
          for (int kc = 0; kc < NKC; ++kc, ++idx) {
            const int s = idx % kTcStages;
            if (idx >= kTcStages && !draft_wait(&b_empty[s], (uint32_t)(idx / kTcStages - 1) & 1u, w.err, g.wait_ns)) {
              ok = false;
              break;
            }
            tc::mbar_arrive_expect_tx(&b_full[s], CHUNK);
            tc::bulk_g2s(b_sm + s * CHUNK, kt + split_chunk_off(bh, RT, t0 + tt, m, kc, NKC), CHUNK, &b_full[s]);
          }
        if (!ok) break;
      }
    }
  } else if (warp == 1) {
    // ---- MMAs: 3 per K step of 8 channels, 6 per 16-channel chunk ----
    if (lane == 0) {
      const uint32_t idesc = idesc_tf32(kTcRows, kTcKeys);
      int idx = 0;
      bool ok = true;
      for (int m = 0; m < 2 && ok; ++m) {
        ok = draft_wait(a_full, (uint32_t)m & 1u, w.err, g.wait_ns);
        tc::fence_after_sync();
        for (int tt = 0; tt < nt && ok; ++tt) {
          const int u = m * nt + tt, buf = u & 1;
          if (u >= 2 && !(ok = draft_wait(&acc_empty[buf], (uint32_t)((u >> 1) - 1) & 1u, w.err, g.wait_ns))) break;
          tc::fence_after_sync();
          const uint32_t d_tmem = tmem + (uint32_t)(buf * kTcKeys);
          for (int kc = 0; kc < NKC; ++kc, ++idx) {
            const int s = idx % kTcStages;
            if (!(ok = draft_wait(&b_full[s], (uint32_t)(idx / kTcStages) & 1u, w.err, g.wait_ns))) break;
            tc::fence_after_sync();
            const uint8_t* ah = a_sm + kc * CHUNK;
            const uint8_t* bhp = b_sm + s * CHUNK;
#pragma unroll
            for (int ks = 0; ks < kSplitKC / 8; ++ks) {
              const uint64_t adh = tc::sdesc(ah + ks * 256, 128, kSplitKC * 4 * 8);
              const uint64_t adl = tc::sdesc(ah + kSplitPart + ks * 256, 128, kSplitKC * 4 * 8);
              const uint64_t bdh = tc::sdesc(bhp + ks * 256, 128, kSplitKC * 4 * 8);
              const uint64_t bdl = tc::sdesc(bhp + kSplitPart + ks * 256, 128, kSplitKC * 4 * 8);
              mma_tf32(d_tmem, adh, bdh, idesc, (kc | ks) != 0 ? 1u : 0u);
              mma_tf32(d_tmem, adh, bdl, idesc, 1u);
              mma_tf32(d_tmem, adl, bdh, idesc, 1u);
            }
            tc::mma_commit(&b_empty[s]);
          }
          if (ok) tc::mma_commit(&acc_full[buf]);
        }
        if (ok) tc::mma_commit(a_empty);                  // this map's MMAs are all issued
      }
    }
  } else {
    // ---- read-out: warp w owns TMEM lanes 32 (w % 4) .. + 31, i.e. query rows ----
    const int q = warp & 3;
    const int row = i0 + 32 * q + lane;
    for (int u = 0; u < U; ++u) {
      const int buf = u & 1, m = u / nt, t = t0 + u % nt;
      if (!draft_wait(&acc_full[buf], (uint32_t)(u >> 1) & 1u, w.err, g.wait_ns)) break;
      tc::fence_after_sync();
      float* out = dlog + (((size_t)bh * N + row) * 2 + m) * NP;
#pragma unroll
      for (int cc = 0; cc < kTcKeys / 32; ++cc) {
        uint32_t r[32];
        tc::tmem_ld32(tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(buf * kTcKeys + 32 * cc), r);
        tc::tmem_wait_ld();
        const int j0 = t * kTcKeys + 32 * cc;
        if (row < N) {
          if (j0 + 32 <= N) {
#pragma unroll
            for (int e = 0; e < 32; e += 4) {
              float4 o;
              o.x = fmaf(g.sm_scale, __uint_as_float(r[e]), lcs[j0 + e]);
              o.y = fmaf(g.sm_scale, __uint_as_float(r[e + 1]), lcs[j0 + e + 1]);
              o.z = fmaf(g.sm_scale, __uint_as_float(r[e + 2]), lcs[j0 + e + 2]);
              o.w = fmaf(g.sm_scale, __uint_as_float(r[e + 3]), lcs[j0 + e + 3]);
              *reinterpret_cast<float4*>(out + j0 + e) = o;
            }
          } else {
#pragma unroll
            for (int e = 0; e < 32; ++e)
              if (j0 + e < N) out[j0 + e] = fmaf(g.sm_scale, __uint_as_float(r[e]), lcs[j0 + e]);
          }
        }
      }
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&acc_empty[buf]);
    }
  }
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 0) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, 2 * kTcKeys);
  }
}

size_t logits_tc_smem_bytes(int d) {
  return (size_t)(d / kSplitKC) * 2 * kSplitPart + (size_t)kTcStages * 2 * kSplitPart + 1024 * 4 + 16 * 8;
}

// e^t for t <= 0 (a logit minus its row max) as 2^(t log2 e) on the special-function unit
// (ex2.approx.ftz.f32): two instructions instead of the accurate expf's range reduction.
// Its relative error, a few units in the last place, stays far inside the ranking's
// tolerance; results below 2^-126 flush to zero.
__device__ __forceinline__ float exp_sfu(float t) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(t * 1.4426950408889634f));
  return y;
}

// Ranking of the draft scores from the logits scratch: one warp per query block, 16 per CTA.
// Only one N-float row per warp sits in shared memory (the average map's exponentials, then
// the scores): the maxima and the max map's exponentials are read from the scratch, the
// latter twice, so that three CTAs (48 warps) fit on an SM at N = 630. The scores are
// formed as in rank_rows except for the exponentials, taken here by exp_sfu.
constexpr int kRankRows = 16;
__global__ void __launch_bounds__(kRankRows * 32) k_draft_rank(Geo g, Ws w, const float* dlog, int NP) {
  extern __shared__ __align__(16) float rsm[];
  const int N = g.N;
  const int bh = blockIdx.y, warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int i = blockIdx.x * kRankRows + warp;
  if (i >= N) return;
  float* ra = rsm + warp * N;
  uint32_t* h = reinterpret_cast<uint32_t*>(rsm + kRankRows * N) + warp * kHistWords;
  const size_t row = (size_t)bh * N + i;
  const float* la = dlog + row * 2 * NP;
  const float* lm = la + NP;
  float mxa = -INFINITY, mxm = -INFINITY;
  for (int j = lane; j < N; j += 32) { mxa = fmaxf(mxa, la[j]); mxm = fmaxf(mxm, lm[j]); }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    mxa = fmaxf(mxa, __shfl_xor_sync(0xffffffffu, mxa, o));
    mxm = fmaxf(mxm, __shfl_xor_sync(0xffffffffu, mxm, o));
  }
  float sa = 0.0f, sm = 0.0f;
  for (int j = lane; j < N; j += 32) {
    const float ea = exp_sfu(la[j] - mxa), em = exp_sfu(lm[j] - mxm);
    ra[j] = ea;
    sa += ea;
    sm += em;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    sa += __shfl_xor_sync(0xffffffffu, sa, o);
    sm += __shfl_xor_sync(0xffffffffu, sm, o);
  }
  const float ia = 1.0f / sa, im = 1.0f / sm;
  for (int j = lane; j < N; j += 32) {
    const float em = exp_sfu(lm[j] - mxm);
    const float sc = 0.5f * (ra[j] * ia + em * im);
    ra[j] = sc;
    if (g.flags & DA2_FLAG_EXPORT_SCORES) w.scores[row * N + j] = sc;
  }
  __syncwarp();
  rank_keys_row(g, w, reinterpret_cast<const uint32_t*>(ra), h, row, lane);
}

size_t rank_smem_bytes(const Geo& g) {
  return (size_t)kRankRows * g.N * 4 + (size_t)kRankRows * kHistWords * 4;
}

size_t draft_smem_bytes(const Geo& g, int R) {
  return (size_t)(2 * R * g.d + 2 * R * g.N) * 4 + kDraftWarps * kHistWords * 4;
}

int draft_rows_per_cta(const Geo& g) {
  int R = 16;
  while (R > 1 && draft_smem_bytes(g, R) > 200 * 1024) --R;
  return R;
}

cudaError_t launch_draft_select(const Geo& g, const Ws& w, const uint8_t* qt, const uint8_t* kt,
                                float* dlog, int np, cudaStream_t st) {
  // up to 1024 key blocks: the logits on the tensor cores into the scratch, then the ranking
  if (g.N <= 1024) {
    const int NT = (g.N + kTcKeys - 1) / kTcKeys;
    const int per = NT < 3 ? NT : 3;                     // key tiles per CTA (A/B: 3 beats 1, 2 and all)
    const dim3 g1((g.N + kTcRows - 1) / kTcRows, g.B * g.H, (NT + per - 1) / per);
    const size_t s1 = logits_tc_smem_bytes(g.d);
    cudaError_t e;
    if (g.d == 128) {
      e = cudaFuncSetAttribute(k_draft_logits_tc<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)s1);
      if (e != cudaSuccess) return e;
      k_draft_logits_tc<128><<<g1, kTcThreads, s1, st>>>(g, w, qt, kt, dlog, np, per);
    } else {
      e = cudaFuncSetAttribute(k_draft_logits_tc<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)s1);
      if (e != cudaSuccess) return e;
      k_draft_logits_tc<64><<<g1, kTcThreads, s1, st>>>(g, w, qt, kt, dlog, np, per);
    }
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const size_t s2 = rank_smem_bytes(g);
    e = cudaFuncSetAttribute(k_draft_rank, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)s2);
    if (e != cudaSuccess) return e;
    k_draft_rank<<<dim3((g.N + kRankRows - 1) / kRankRows, g.B * g.H), kRankRows * 32, s2, st>>>(g, w, dlog, np);
    return cudaGetLastError();
  }
  const int R = draft_rows_per_cta(g);
  const size_t smem = draft_smem_bytes(g, R);
  dim3 grid((g.N + R - 1) / R, g.B * g.H);
  cudaError_t e;
  if (g.d == 128) {
    e = cudaFuncSetAttribute(k_draft_select<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    k_draft_select<128><<<grid, kDraftThreads, smem, st>>>(g, w, R);
  } else {
    e = cudaFuncSetAttribute(k_draft_select<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    k_draft_select<64><<<grid, kDraftThreads, smem, st>>>(g, w, R);
  }
  return cudaGetLastError();
}

}  // namespace da2
