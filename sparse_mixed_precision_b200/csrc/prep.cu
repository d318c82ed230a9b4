// Operand preparation (HBM-bound): V channel amax pre-pass and the fused prepare kernel.
//
// "DraftAttention2: Fast Video Diffusion with Low-Resolution-Guided Mixed-Precision
// Attention", Abstract: draft queries/keys are spatial 2D average- and max-pooled, and a
// fused operand-preparation step feeds the mixed-precision attention kernel.
// "DraftAttention: Fast Video Diffusion via Low-Resolution Attention Guidance", Abstract:
// per-frame downsampling; tokens are reordered so that each pooled region is contiguous.
//
// One CTA prepares one (b, h, block) of one tensor: it stages the window's tokens (bf16,
// 128-bit loads, padded slots zero) in shared memory once, then writes the pooled draft
// vectors (Q, K), the E4M3 copy and the E2M1 copy with its E4M3 group scales in the tile
// layouts the attention kernel loads directly (see include/da2.h).
#include "common.cuh"

namespace da2 {

__device__ __forceinline__ uint4 ld_stream_u4(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "l"(p));
  return r;
}

__device__ __forceinline__ void bf16x8_to_f32(uint4 u, float* f) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

// ---- K0: amax of V over all tokens, per (b, h, channel) ----
// grid (chunks, B*H); vamax must be zero on entry (non-negative floats compare as uints).
// BTHD: q, k, v token-major [B,T,H,d] (token stride H*D) instead of [B,H,T,d] (stride D).
template <int D, bool BTHD>
__global__ void __launch_bounds__(256) k_vamax(Geo g, const __nv_bfloat16* __restrict__ v,
                                               float* __restrict__ vamax, int chunk) {
  const int T = g.T;
  constexpr int VPR = D / 8;          // 16-byte vectors per token
  constexpr int RSTEP = 256 / VPR;    // tokens per sweep
  __shared__ float red[RSTEP][D + 1];
  const int bh = blockIdx.y;
  const int t0 = blockIdx.x * chunk, t1 = min(T, t0 + chunk);
  const int cv = threadIdx.x % VPR, tr = threadIdx.x / VPR;
  float m[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) m[i] = 0.0f;
  const __nv_bfloat16* base = v + tok_off(g, bh, 0) + cv * 8;
  const size_t ts = BTHD ? (size_t)g.H * D : (size_t)D;
  int t = t0 + tr;
  for (; t + 3 * RSTEP < t1; t += 4 * RSTEP) {        // four loads in flight per thread
    uint4 u[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) u[j] = ld_stream_u4(base + (size_t)(t + j * RSTEP) * ts);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      float f[8];
      bf16x8_to_f32(u[j], f);
#pragma unroll
      for (int i = 0; i < 8; ++i) m[i] = fmaxf(m[i], fabsf(f[i]));
    }
  }
  for (; t < t1; t += RSTEP) {
    float f[8];
    bf16x8_to_f32(ld_stream_u4(base + (size_t)t * ts), f);
#pragma unroll
    for (int i = 0; i < 8; ++i) m[i] = fmaxf(m[i], fabsf(f[i]));
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) red[tr][cv * 8 + i] = m[i];
  __syncthreads();
  for (int c = threadIdx.x; c < D; c += 256) {
    float a = 0.0f;
    for (int r = 0; r < RSTEP; ++r) a = fmaxf(a, red[r][c]);
    atomicMax(reinterpret_cast<unsigned int*>(vamax + (size_t)bh * D + c), __float_as_uint(a));
  }
}

// Pairs of fp32 values for the packed f32x2 multiply (each lane rounded as fmul.rn).
typedef unsigned long long f32x2;
__device__ __forceinline__ f32x2 pk2(float lo, float hi) {
  f32x2 r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void upk2(f32x2 v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ f32x2 mul2(f32x2 a, f32x2 b) {
  f32x2 d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
// y[i] * s for 16 values, two per packed multiply.
__device__ __forceinline__ void scale16(const float* x, float s, float* y) {
  const f32x2 s2 = pk2(s, s);
#pragma unroll
  for (int i = 0; i < 16; i += 2) upk2(mul2(pk2(x[i], x[i + 1]), s2), y[i], y[i + 1]);
}

// a / 6 correctly rounded for finite a >= 0, in three FMA-pipe steps: q0 = a * fl(1/6), the
// exact residual r = a - 6 q0 (one fma), q = q0 + r * fl(1/6). The quotient a / 6 = (a / 2) / 3
// lies, in units of its own ulp, at a fraction 0, 1/3 or 2/3 from the fp32 grid, never
// within the correction's residual error of a rounding midpoint, so q equals the IEEE
// quotient (values below 2^-126 only reach E4M3 code 0 either way).
__device__ __forceinline__ float div6_rn(float a) {
  const float c = 0.16666667163372040f;       // fl(1/6)
  const float q0 = __fmul_rn(a, c);
  const float r = __fmaf_rn(-6.0f, q0, a);
  return __fmaf_rn(r, c, q0);
}

// Quantise one group of 16 values y (already divided by their outer scale) to E2M1 with an
// E4M3 group scale: sigma = E4M3(amax16 / 6); codes = E2M1(y * (1/sigma)), the correctly
// rounded reciprocal taken from a table over the 128 non-negative E4M3 codes (filled with
// __frcp_rn of each code's value); a group whose sigma is zero is all zero codes. Writes 8
// bytes of packed codes and returns sigma's byte.
__device__ __forceinline__ uint8_t quant_fp4_group16_tab(const float* y, uint32_t* packed2,
                                                         const float* rcp_tab) {
  float amax = 0.0f;
#pragma unroll
  for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(y[i]));
  const uint8_t sc = f32_to_e4m3(div6_rn(amax));
  if (sc != 0) {
    const float r = rcp_tab[sc & 0x7F];
    float z[16];
    scale16(y, r, z);
    packed2[0] = f32x8_to_e2m1x8(z);
    packed2[1] = f32x8_to_e2m1x8(z + 8);
  } else {
    packed2[0] = 0u;
    packed2[1] = 0u;
  }
  return sc;
}

// ---- K1: fused preparation of one (b, h, block) of Q, K (pool + quantise) or V ----
// grid (N, B*H, 3); blockIdx.z: 0 = Q, 1 = K, 2 = V.
template <int D, bool BTHD>
__global__ void __launch_bounds__(256) k_prepare(Geo g, Ws w, const __nv_bfloat16* __restrict__ q,
                                                 const __nv_bfloat16* __restrict__ k,
                                                 const __nv_bfloat16* __restrict__ v) {
  constexpr int RS = D + 8;           // smem row stride (bf16), padded against bank conflicts
  constexpr int VPR = D / 8;
  extern __shared__ __align__(16) uint8_t smem[];
  __nv_bfloat16* X = reinterpret_cast<__nv_bfloat16*>(smem);
  const int bs = g.bs;
  uint8_t* sfbuf = smem + (size_t)bs * RS * 2;             // up to 1 KB of group scales
  float* red = reinterpret_cast<float*>(sfbuf + 1024);      // reduction scratch / V scales
  float* rcp_tab = red + 128;                               // 1/value of each E4M3 code

  const int n = blockIdx.x, bh = blockIdx.y, which = blockIdx.z;
  const int tid = threadIdx.x;
  const __nv_bfloat16* src = which == 0 ? q : (which == 1 ? k : v);
  const int fpf = g.ny * g.nx;
  const int f = n / fpf, rem = n - f * fpf, by = rem / g.nx, bx = rem - by * g.nx;
  const int y0 = by * g.ph, x0 = bx * g.pw;
  const int hv = min(g.ph, g.Hf - y0), wv = min(g.pw, g.Wf - x0);

  // stage the window (padded slots zero)
  const __nv_bfloat16* sbase = src + tok_off(g, bh, 0);
  const size_t ts = BTHD ? (size_t)g.H * D : (size_t)D;
  {
    // slot s = wy*pw + wx advances by a fixed step per iteration: step the window
    // coordinates instead of dividing every time
    constexpr int DS = 256 / VPR;
    const int cv = tid % VPR;
    int s0 = tid / VPR;
    int wy = s0 / g.pw, wx = s0 - wy * g.pw;
    const int dy = DS / g.pw, dx = DS - dy * g.pw;
    for (int sl = s0; sl < bs; sl += DS) {
      uint4 val = make_uint4(0u, 0u, 0u, 0u);
      if (wy < hv && wx < wv) {
        const size_t t = (size_t)f * g.Hf * g.Wf + (size_t)(y0 + wy) * g.Wf + (x0 + wx);
        val = ld_stream_u4(sbase + t * ts + cv * 8);
      }
      *reinterpret_cast<uint4*>(X + sl * RS + cv * 8) = val;
      wx += dx;
      wy += dy;
      if (wx >= g.pw) { wx -= g.pw; ++wy; }
    }
  }
  const int sfbytes = which < 2 ? (int)w.sf_qk : (int)w.sf_v;
  for (int i = tid; i < sfbytes / 4; i += 256) reinterpret_cast<uint32_t*>(sfbuf)[i] = 0u;
  if (tid < 128) rcp_tab[tid] = tid > 0 ? __frcp_rn(e4m3_to_f32((uint8_t)tid)) : 0.0f;
  __syncthreads();

  if (which < 2) {
    // ---- draft pooling: fp32 running sum in slot order, then IEEE divide; exact max ----
    // threads [0, D/2): sums of channel pairs; [D/2, D): maxima of channel pairs
    float* avg_out = (which == 0 ? w.qavg : w.kavg) + ((size_t)bh * g.N + n) * D;
    float* max_out = (which == 0 ? w.qmax : w.kmax) + ((size_t)bh * g.N + n) * D;
    if (tid < D) {
      const bool do_sum = tid < D / 2;
      const int c2 = 2 * (tid % (D / 2));
      float a0 = do_sum ? 0.0f : -INFINITY, a1 = a0;
      for (int wy = 0; wy < hv; ++wy) {
        const __nv_bfloat16* row = X + wy * g.pw * RS + c2;
        if (do_sum) {
#pragma unroll 4
          for (int wx = 0; wx < wv; ++wx) {
            const uint32_t u = *reinterpret_cast<const uint32_t*>(row + wx * RS);
            a0 = __fadd_rn(a0, __uint_as_float(u << 16));
            a1 = __fadd_rn(a1, __uint_as_float(u & 0xFFFF0000u));
          }
        } else {
#pragma unroll 4
          for (int wx = 0; wx < wv; ++wx) {
            const uint32_t u = *reinterpret_cast<const uint32_t*>(row + wx * RS);
            a0 = fmaxf(a0, __uint_as_float(u << 16));
            a1 = fmaxf(a1, __uint_as_float(u & 0xFFFF0000u));
          }
        }
      }
      if (do_sum) {
        const float cnt = (float)(hv * wv);
        *reinterpret_cast<float2*>(avg_out + c2) = make_float2(__fdiv_rn(a0, cnt), __fdiv_rn(a1, cnt));
      } else {
        *reinterpret_cast<float2*>(max_out + c2) = make_float2(a0, a1);
      }
    }
    // ---- block amax -> outer scale ----
    float am = 0.0f;
    for (int u = tid; u < bs * VPR; u += 256) {
      const int s = u / VPR, cv = u - s * VPR;
      float fv[8];
      bf16x8_to_f32(*reinterpret_cast<const uint4*>(X + s * RS + cv * 8), fv);
#pragma unroll
      for (int i = 0; i < 8; ++i) am = fmaxf(am, fabsf(fv[i]));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, o));
    if ((tid & 31) == 0) red[tid >> 5] = am;
    __syncthreads();
    am = red[0];
#pragma unroll
    for (int i = 1; i < 8; ++i) am = fmaxf(am, red[i]);
    const float inv = am > 0.0f ? __fdiv_rn(kE4M3Max, am) : 1.0f;
    if (tid == 0) (which == 0 ? w.sq : w.sk)[(size_t)bh * g.N + n] = am > 0.0f ? __fdiv_rn(am, kE4M3Max) : 1.0f;

    // ---- E4M3 and E2M1 copies, one 16-channel chunk of one token per step ----
    uint8_t* t8 = (which == 0 ? w.q8 : w.k8) + ((size_t)bh * g.N + n) * w.tile8_qk;
    uint8_t* t4 = (which == 0 ? w.q4 : w.k4) + ((size_t)bh * g.N + n) * w.tile4_qk;
    constexpr int KC = D / 16;
    for (int u = tid; u < bs * KC; u += 256) {
      const int rg = u / (8 * KC), within = u - rg * 8 * KC;
      const int kc = within >> 3, rr = within & 7;
      const int r = rg * 8 + rr;
      float y[16];
      float xf[16];
      bf16x8_to_f32(*reinterpret_cast<const uint4*>(X + r * RS + kc * 16), xf);
      bf16x8_to_f32(*reinterpret_cast<const uint4*>(X + r * RS + kc * 16 + 8), xf + 8);
      scale16(xf, inv, y);
      uint32_t p8[4];
#pragma unroll
      for (int i = 0; i < 4; ++i)
        p8[i] = (uint32_t)f32x2_to_e4m3x2(y[4 * i], y[4 * i + 1]) |
                ((uint32_t)f32x2_to_e4m3x2(y[4 * i + 2], y[4 * i + 3]) << 16);
      *reinterpret_cast<uint4*>(t8 + (size_t)u * 16) = make_uint4(p8[0], p8[1], p8[2], p8[3]);
      uint32_t p4[2];
      const uint8_t sc = quant_fp4_group16_tab(y, p4, rcp_tab);
      *reinterpret_cast<uint2*>(t4 + kmajor_off(r, kc * 8, D / 2)) = make_uint2(p4[0], p4[1]);
      sfbuf[sf_off(kc >> 2, r, kc & 3)] = sc;
    }
    __syncthreads();
    uint8_t* sfo = (which == 0 ? w.sfq4 : w.sfk4) + ((size_t)bh * g.N + n) * w.sf_qk;
    for (int i = tid; i < sfbytes / 16; i += 256)
      reinterpret_cast<uint4*>(sfo)[i] = reinterpret_cast<const uint4*>(sfbuf)[i];
  } else {
    // ---- V: per-channel outer scale from the amax pre-pass; tiles are channel-major ----
    const float* am = w.vamax + (size_t)bh * D;
    float* vinv = red;                                      // D inverse channel scales
    for (int c = tid; c < D; c += 256) {
      const float a = am[c];
      vinv[c] = a > 0.0f ? __fdiv_rn(kE4M3Max, a) : 1.0f;
      if (n == 0) w.sv[(size_t)bh * D + c] = a > 0.0f ? __fdiv_rn(a, kE4M3Max) : 1.0f;
    }
    __syncthreads();
    uint8_t* t8 = w.v8 + ((size_t)bh * g.N + n) * w.tile8_v;
    uint8_t* t4 = w.v4 + ((size_t)bh * g.N + n) * w.tile4_v;
    const int SC = bs / 16, SC4 = g.kv4 / 16;
    // one unit = channels c, c + 1 of one 16-slot group; a warp takes 32 consecutive channel
    // pairs of one group, so its 32-bit reads cover 128 contiguous bytes of each staged row
    constexpr int CP = D / 2;
    for (int u = tid; u < CP * SC4; u += 256) {
      const int sc = u / CP, c = 2 * (u - sc * CP);
      const float inv0 = vinv[c], inv1 = vinv[c + 1];
      float y0[16], y1[16];
      if (sc < SC) {
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const uint32_t pr = *reinterpret_cast<const uint32_t*>(X + (sc * 16 + i) * RS + c);
          upk2(mul2(pk2(__uint_as_float(pr << 16), __uint_as_float(pr & 0xFFFF0000u)), pk2(inv0, inv1)),
               y0[i], y1[i]);
        }
        uint32_t p8[4], q8[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          p8[i] = (uint32_t)f32x2_to_e4m3x2(y0[4 * i], y0[4 * i + 1]) |
                  ((uint32_t)f32x2_to_e4m3x2(y0[4 * i + 2], y0[4 * i + 3]) << 16);
          q8[i] = (uint32_t)f32x2_to_e4m3x2(y1[4 * i], y1[4 * i + 1]) |
                  ((uint32_t)f32x2_to_e4m3x2(y1[4 * i + 2], y1[4 * i + 3]) << 16);
        }
        *reinterpret_cast<uint4*>(t8 + kmajor_off(c, sc * 16, bs)) = make_uint4(p8[0], p8[1], p8[2], p8[3]);
        *reinterpret_cast<uint4*>(t8 + kmajor_off(c + 1, sc * 16, bs)) = make_uint4(q8[0], q8[1], q8[2], q8[3]);
      } else {
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          y0[i] = 0.0f;
          y1[i] = 0.0f;
        }
      }
      uint32_t p4[2];
      const uint8_t s40 = quant_fp4_group16_tab(y0, p4, rcp_tab);
      *reinterpret_cast<uint2*>(t4 + kmajor_off(c, sc * 8, g.kv4 / 2)) = make_uint2(p4[0], p4[1]);
      const uint8_t s41 = quant_fp4_group16_tab(y1, p4, rcp_tab);
      *reinterpret_cast<uint2*>(t4 + kmajor_off(c + 1, sc * 8, g.kv4 / 2)) = make_uint2(p4[0], p4[1]);
      sfbuf[sf_off(sc >> 2, c, sc & 3)] = s40;
      sfbuf[sf_off(sc >> 2, c + 1, sc & 3)] = s41;
    }
    __syncthreads();
    uint8_t* sfo = w.sfv4 + ((size_t)bh * g.N + n) * w.sf_v;
    for (int i = tid; i < sfbytes / 16; i += 256)
      reinterpret_cast<uint4*>(sfo)[i] = reinterpret_cast<const uint4*>(sfbuf)[i];
  }
}

size_t prepare_smem_bytes(const Geo& g) {
  return (size_t)g.bs * (g.d + 8) * 2 + 1024 + 4 * 128 + 4 * 128;
}

cudaError_t launch_prepare(const Geo& g, const Ws& w, const void* q, const void* k,
                           const void* v, cudaStream_t st) {
  const int BH = g.B * g.H;
  cudaError_t e = cudaMemsetAsync(w.vamax, 0, sizeof(float) * BH * g.d, st);
  if (e != cudaSuccess) return e;
  e = cudaMemsetAsync(w.err, 0, sizeof(uint32_t), st);
  if (e != cudaSuccess) return e;
  const int chunk = 2048;
  dim3 g0((g.T + chunk - 1) / chunk, BH);
  const size_t smem = prepare_smem_bytes(g);
  dim3 g1(g.N, BH, 3);
  const auto* qb = static_cast<const __nv_bfloat16*>(q);
  const auto* kb = static_cast<const __nv_bfloat16*>(k);
  const auto* vb = static_cast<const __nv_bfloat16*>(v);
  if (g.d == 128 && !g.bthd) {
    k_vamax<128, false><<<g0, 256, 0, st>>>(g, vb, w.vamax, chunk);
    k_prepare<128, false><<<g1, 256, smem, st>>>(g, w, qb, kb, vb);
  } else if (g.d == 128) {
    k_vamax<128, true><<<g0, 256, 0, st>>>(g, vb, w.vamax, chunk);
    k_prepare<128, true><<<g1, 256, smem, st>>>(g, w, qb, kb, vb);
  } else if (!g.bthd) {
    k_vamax<64, false><<<g0, 256, 0, st>>>(g, vb, w.vamax, chunk);
    k_prepare<64, false><<<g1, 256, smem, st>>>(g, w, qb, kb, vb);
  } else {
    k_vamax<64, true><<<g0, 256, 0, st>>>(g, vb, w.vamax, chunk);
    k_prepare<64, true><<<g1, 256, smem, st>>>(g, w, qb, kb, vb);
  }
  return cudaGetLastError();
}

}  // namespace da2
