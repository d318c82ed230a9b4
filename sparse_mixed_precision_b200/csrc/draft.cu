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
// One CTA takes R query blocks of one (b, h): it forms both draft logit rows against all N
// key blocks (fp32 FMA), turns each into a row softmax, averages the two maps into the
// score, and each warp ranks its rows with an exact radix select over the score bits
// (ties broken by the lower block index), then writes tags and the ascending index lists of
// the kept classes (FP8, mixed, FP4).
#include "common.cuh"

namespace da2 {

// k-th largest 32-bit key of `keys[0..n)` (1 <= kth <= n) by an 8-bit radix select within
// one warp. Returns the key value T and how many of the keys equal to T belong to the top
// kth (the rest of the top kth are strictly greater than T).
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
    uint32_t digit = 0u, above = 0u;
    if (mine) {
      uint32_t acc = excl;
#pragma unroll
      for (int t = 0; t < 8; ++t) {
        if (acc + c[t] >= (uint32_t)remaining) { digit = 255u - 8u * lane - t; above = acc; break; }
        acc += c[t];
      }
    }
    const uint32_t found = __ballot_sync(0xffffffffu, mine);
    const int src = found ? __ffs(found) - 1 : 0;   // always found when 1 <= kth <= n
    digit = __shfl_sync(0xffffffffu, digit, src);
    above = __shfl_sync(0xffffffffu, above, src);
    prefix |= digit << shift;
    pmask |= 0xFFu << shift;
    remaining -= (int)above;
    __syncwarp();
  }
  T = prefix;
  need = remaining;
}

constexpr int kDraftThreads = 512, kDraftWarps = kDraftThreads / 32;

// Per-row ranking of the draft scores (one warp per row): the two row softmaxes of the
// average- and max-pooled logits (in la / lm, R rows of N), their mean as the score, and the
// radix-select cuts of the shared ranking; writes tags and the ascending lists.
__device__ void rank_rows(const Geo& g, const Ws& w, float* la, float* lm, uint32_t* hist, int bh, int i0,
                          int rows, int warp, int lane, int nwarps) {
  const int N = g.N;
  const int n8m = g.n8 + g.nm, nk = g.n8 + g.nm + g.n4;   // the ranking's cuts
  const bool adaptive = g.tau > 0.0f && g.n4max > g.n4;
  const int nkx = g.n8 + g.nm + g.n4max;                    // last rank the adaptive budget may reach
  const uint32_t tau_bits = __float_as_uint(g.tau);       // scores are non-negative: bits order like values
  uint32_t* h = hist + warp * 256;
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
    const uint32_t* keys = reinterpret_cast<const uint32_t*>(ra);
    // the three cuts of the ranking: n8-th, (n8 + nm)-th and nk-th largest score
    uint32_t T8 = 0xFFFFFFFFu, Tm = 0xFFFFFFFFu, Tk = 0xFFFFFFFFu;
    int need8 = 0, needm = 0, needk = 0;
    if (g.n8 > 0) warp_radix_select(keys, N, g.n8, h, T8, need8);
    if (g.nm > 0) warp_radix_select(keys, N, n8m, h, Tm, needm);
    if (nk > 0) warp_radix_select(keys, N, nk, h, Tk, needk);
    uint32_t Tx = 0xFFFFFFFFu;
    int needx = 0;
    if (adaptive) warp_radix_select(keys, N, nkx, h, Tx, needx);
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
      const uint32_t em = __ballot_sync(0xffffffffu, ok && g.nm > 0 && key == Tm);
      const uint32_t ek = __ballot_sync(0xffffffffu, ok && nk > 0 && key == Tk);
      const uint32_t ex = __ballot_sync(0xffffffffu, ok && adaptive && key == Tx);
      const bool in8 = ok && g.n8 > 0 && (key > T8 || (key == T8 && eq8 + __popc(e8 & lt) < need8));
      const bool in8m = in8 || (ok && g.nm > 0 && (key > Tm || (key == Tm && eqm + __popc(em & lt) < needm)));
      const bool ink = ok && nk > 0 && (key > Tk || (key == Tk && eqk + __popc(ek & lt) < needk));
      // adaptive budget: a block ranked after the fixed cut, within the cap, whose score
      // reaches the threshold joins FP4 (those form a prefix of the ranks, scores being
      // sorted within the ranking)
      const bool inx = ok && adaptive && (key > Tx || (key == Tx && eqx + __popc(ex & lt) < needx));
      const bool rec = inx && !ink && key >= tau_bits;
      eq8 += __popc(e8);
      eqm += __popc(em);
      eqk += __popc(ek);
      eqx += __popc(ex);
      const bool inm = in8m && !in8;
      const bool in4 = (ink && !in8m) || rec;
      const uint32_t b8 = __ballot_sync(0xffffffffu, in8), bm = __ballot_sync(0xffffffffu, inm),
                     b4 = __ballot_sync(0xffffffffu, in4);
      const int p8 = c8 + __popc(b8 & lt), pm = cm + __popc(bm & lt), p4 = c4 + __popc(b4 & lt);
      if (in8 && p8 < g.n8) l8[p8] = (int16_t)j;
      if (inm && pm < g.nm) lmx[pm] = (int16_t)j;
      if (in4 && p4 < g.n4max) l4[p4] = (int16_t)j;
      c8 += __popc(b8);
      cm += __popc(bm);
      c4 += __popc(b4);
      if (ok) trow[j] = in8 ? 2 : (inm ? 3 : (in4 ? 1 : 0));
    }
    for (int p = c4 + lane; p < g.n4max; p += 32) l4[p] = (int16_t)-1;   // no block
    if (lane == 0 && (c8 != g.n8 || cm != g.nm || c4 < g.n4 || c4 > g.n4max)) set_error(w.err, kErrBadIndex);
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
  uint32_t* hist = reinterpret_cast<uint32_t*>(lm + R * N);  // [warps][256]
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

// Register-tiled draft logits for up to 1024 key blocks: a CTA of KL = blockDim.x threads
// takes 16 query blocks of one (b, h); thread t owns key blocks t and t + KL and all 16 query
// rows, one map after the other, as packed pairs of rows (f32x2 FMA). The pooled queries sit
// in shared memory transposed ([map][channel][row], read as float4 by every thread alike);
// each thread streams its own two pooled key rows (16-byte loads through L1). Then the same
// per-row ranking as the general kernel. At 64 registers a thread and about 111 KB of
// shared memory (up to 630 key blocks) two CTAs share an SM, so that the latency of one
// CTA's phases is hidden by the other's warps.
constexpr int kTileRows = 16;

__device__ __forceinline__ unsigned long long pk2f(float lo, float hi) {
  unsigned long long r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void upk2f(unsigned long long v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ unsigned long long fma2f(unsigned long long a, unsigned long long b,
                                                    unsigned long long c) {
  unsigned long long d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}

template <int D>
__global__ void __launch_bounds__(kDraftThreads, 2) k_draft_tiled(Geo g, Ws w) {
  extern __shared__ __align__(16) float dsm[];
  constexpr int R = kTileRows;
  const int N = g.N;
  const int KL = ((N + 1) / 2 + 31) / 32 * 32;    // key lanes: keys t and t + KL (t < KL)
  float* qT = dsm;                                // [2][D][R]
  float* la = qT + 2 * D * R;                     // [R][N]
  float* lm = la + R * N;                         // [R][N]
  uint32_t* hist = reinterpret_cast<uint32_t*>(lm + R * N);   // [warps][256]
  const int bh = blockIdx.y, i0 = blockIdx.x * R;
  const int rows = min(R, N - i0);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

  const float* qavg = w.qavg + ((size_t)bh * N + i0) * D;
  const float* qmax = w.qmax + ((size_t)bh * N + i0) * D;
  for (int u = tid; u < R * D; u += blockDim.x) {
    const int r = u / D, c = u - r * D;
    const bool ok = r < rows;
    qT[c * R + r] = ok ? __ldg(qavg + u) : 0.0f;
    qT[(D + c) * R + r] = ok ? __ldg(qmax + u) : 0.0f;
  }
  const float* kavg = w.kavg + (size_t)bh * N * D;
  const float* kmax = w.kmax + (size_t)bh * N * D;
  __syncthreads();                                // the transposed query rows are in place
  // this thread's two key blocks (a lane past the last block recomputes the last one);
  // threads t >= KL only rank. One map at a time: 2 keys x 8 row pairs of accumulators.
  const int ja = tid < N ? tid : N - 1, jb = tid + KL < N ? tid + KL : N - 1;
  const bool mass = !(g.flags & DA2_FLAG_NO_MASS_CORRECTION);
  const int fpf = g.ny * g.nx;
  float lc[2] = {0.0f, 0.0f};
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const int j = tid + i * KL;
    if (mass && j < N) {
      const int rem = j % fpf, by = rem / g.nx, bx = rem - by * g.nx;
      const int hv = min(g.ph, g.Hf - by * g.ph), wv = min(g.pw, g.Wf - bx * g.pw);
      lc[i] = logf((float)(hv * wv));
    }
  }
  if (tid < KL) {
#pragma unroll 1
    for (int m = 0; m < 2; ++m) {
      const float* kb = m == 0 ? kavg : kmax;
      const float4* kp[2] = {reinterpret_cast<const float4*>(kb + (size_t)ja * D),
                             reinterpret_cast<const float4*>(kb + (size_t)jb * D)};
      const float* qm = qT + m * D * R;
      unsigned long long acc[2][R / 2];
#pragma unroll
      for (int i = 0; i < 2; ++i)
#pragma unroll
        for (int p = 0; p < R / 2; ++p) acc[i][p] = 0ull;
      // acc += q[c] k[c] over the channels of one float4 of each key, c ascending
      auto step = [&](int c4, const float4 (&kv)[2]) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float4* qp = reinterpret_cast<const float4*>(qm + (4 * c4 + e) * R);
          unsigned long long kk[2];
#pragma unroll
          for (int i = 0; i < 2; ++i) {
            const float k1 = e == 0 ? kv[i].x : (e == 1 ? kv[i].y : (e == 2 ? kv[i].z : kv[i].w));
            kk[i] = pk2f(k1, k1);
          }
#pragma unroll
          for (int f = 0; f < R / 4; ++f) {
            const float4 x = qp[f];
            const unsigned long long q0 = pk2f(x.x, x.y), q1 = pk2f(x.z, x.w);
#pragma unroll
            for (int i = 0; i < 2; ++i) {
              acc[i][2 * f] = fma2f(q0, kk[i], acc[i][2 * f]);
              acc[i][2 * f + 1] = fma2f(q1, kk[i], acc[i][2 * f + 1]);
            }
          }
        }
      };
#pragma unroll 2
      for (int c4 = 0; c4 < D / 4; ++c4) {
        const float4 kv[2] = {__ldg(kp[0] + c4), __ldg(kp[1] + c4)};
        step(c4, kv);
      }
      float* lo = m == 0 ? la : lm;
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        const int j = tid + i * KL;
        if (j >= N) continue;
#pragma unroll
        for (int p = 0; p < R / 2; ++p) {
          float a0, a1;
          upk2f(acc[i][p], a0, a1);
          lo[(2 * p) * N + j] = fmaf(g.sm_scale, a0, lc[i]);
          lo[(2 * p + 1) * N + j] = fmaf(g.sm_scale, a1, lc[i]);
        }
      }
    }
  }
  __syncthreads();
  rank_rows(g, w, la, lm, hist, bh, i0, rows, warp, lane, blockDim.x / 32);
}

size_t tiled_smem_bytes(const Geo& g) {
  return (size_t)(2 * g.d * kTileRows + 2 * kTileRows * g.N) * 4 + (size_t)kDraftWarps * 256 * 4;
}

size_t draft_smem_bytes(const Geo& g, int R) {
  return (size_t)(2 * R * g.d + 2 * R * g.N) * 4 + kDraftWarps * 256 * 4;
}

int draft_rows_per_cta(const Geo& g) {
  int R = 16;
  while (R > 1 && draft_smem_bytes(g, R) > 200 * 1024) --R;
  return R;
}

cudaError_t launch_draft_select(const Geo& g, const Ws& w, cudaStream_t st) {
  // up to 1024 key blocks (and shared memory to spare): the register-tiled kernel
  if (g.N <= 2 * kDraftThreads && tiled_smem_bytes(g) <= 232448) {
    const int KL = kDraftThreads;                  // 16 warps: one per query row when ranking
    const size_t smem = tiled_smem_bytes(g);
    dim3 grid((g.N + kTileRows - 1) / kTileRows, g.B * g.H);
    cudaError_t e;
    if (g.d == 128) {
      e = cudaFuncSetAttribute(k_draft_tiled<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
      if (e != cudaSuccess) return e;
      e = cudaFuncSetAttribute(k_draft_tiled<128>, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
      if (e != cudaSuccess) return e;
      k_draft_tiled<128><<<grid, KL, smem, st>>>(g, w);
    } else {
      e = cudaFuncSetAttribute(k_draft_tiled<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
      if (e != cudaSuccess) return e;
      e = cudaFuncSetAttribute(k_draft_tiled<64>, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
      if (e != cudaSuccess) return e;
      k_draft_tiled<64><<<grid, KL, smem, st>>>(g, w);
    }
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
