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

  const int n8m = g.n8 + g.nm, nk = g.n8 + g.nm + g.n4;   // the ranking's cuts
  uint32_t* h = hist + warp * 256;
  for (int r = warp; r < rows; r += kDraftWarps) {
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
    int eq8 = 0, eqm = 0, eqk = 0, c8 = 0, cm = 0, c4 = 0;
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
      const bool in8 = ok && g.n8 > 0 && (key > T8 || (key == T8 && eq8 + __popc(e8 & lt) < need8));
      const bool in8m = in8 || (ok && g.nm > 0 && (key > Tm || (key == Tm && eqm + __popc(em & lt) < needm)));
      const bool ink = ok && nk > 0 && (key > Tk || (key == Tk && eqk + __popc(ek & lt) < needk));
      eq8 += __popc(e8);
      eqm += __popc(em);
      eqk += __popc(ek);
      const bool inm = in8m && !in8;
      const bool in4 = ink && !in8m;
      const uint32_t b8 = __ballot_sync(0xffffffffu, in8), bm = __ballot_sync(0xffffffffu, inm),
                     b4 = __ballot_sync(0xffffffffu, in4);
      const int p8 = c8 + __popc(b8 & lt), pm = cm + __popc(bm & lt), p4 = c4 + __popc(b4 & lt);
      if (in8 && p8 < g.n8) l8[p8] = (int16_t)j;
      if (inm && pm < g.nm) lmx[pm] = (int16_t)j;
      if (in4 && p4 < g.n4) l4[p4] = (int16_t)j;
      c8 += __popc(b8);
      cm += __popc(bm);
      c4 += __popc(b4);
      if (ok) trow[j] = in8 ? 2 : (inm ? 3 : (in4 ? 1 : 0));
    }
    if (lane == 0 && (c8 != g.n8 || cm != g.nm || c4 != g.n4)) set_error(w.err, kErrBadIndex);
  }
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
