// Operand preparation (HBM-bound): V channel amax, pooling and quantisation of Q and K, and
// quantisation of V, in two kernels.
//
// "DraftAttention2: Fast Video Diffusion with Low-Resolution-Guided Mixed-Precision
// Attention", Abstract: draft queries/keys are spatial 2D average- and max-pooled, and a
// fused operand-preparation step feeds the mixed-precision attention kernel.
// "DraftAttention: Fast Video Diffusion via Low-Resolution Attention Guidance", Abstract:
// per-frame downsampling; tokens are reordered so that each pooled region is contiguous.
//
// A block item stages the window's tokens of one (b, h, block) of one tensor (bf16,
// 16-byte copies, padded slots zero) in shared memory once, then writes the pooled draft
// vectors (Q, K), the E4M3 copy and the E2M1 copy with its E4M3 group scales in the tile
// layouts the attention kernel loads directly (see include/da2.h).
#include "common.cuh"
#include "split_tiles.cuh"

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

// 16-byte global -> shared copy that bypasses L1 (cp.async.cg); src_bytes 0 writes zeros.
__device__ __forceinline__ void cp_async16(void* dst, const void* src, uint32_t src_bytes) {
  const uint32_t d = static_cast<uint32_t>(__cvta_generic_to_shared(dst));
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(d), "l"(src), "r"(src_bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

// lo += bf16 low half of w, hi += bf16 high half, each one fp32 add rounded to nearest (the
// bf16 operand widens exactly, so this is the fp32 sum of the widened values).
__device__ __forceinline__ void acc_bf16x2(uint32_t w, float& lo, float& hi) {
  asm("{\n\t.reg .b16 l, h;\n\tmov.b32 {l, h}, %2;\n\t"
      "add.rn.f32.bf16 %0, l, %0;\n\tadd.rn.f32.bf16 %1, h, %1;\n\t}"
      : "+f"(lo), "+f"(hi) : "r"(w));
}
// Elementwise max / min of two bf16 pairs (exact; a NaN operand yields the other).
__device__ __forceinline__ uint32_t bmax2(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("max.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}
__device__ __forceinline__ uint32_t bmin2(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("min.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

// The preparation runs as two kernels. The first takes, per (b, h), the V amax chunks of
// the head spread evenly among its Q and K blocks: the chunks are pure reads and use the
// memory bandwidth that the instruction-bound Q/K blocks leave free. The second quantises
// the V blocks once every channel amax is final.

// V channel amax over tokens [t0, t1) of head bh, merged into vamax (non-negative floats
// order like their bit patterns, so an integer atomic max is exact). scratch: 8 * D floats
// of shared memory.
template <int D, bool BTHD>
__device__ __forceinline__ void vamax_chunk(const Geo& g, const __nv_bfloat16* __restrict__ v,
                                            float* vamax, int bh, int t0, int t1, float* scratch) {
  constexpr int VPR = D / 8;          // 16-byte vectors per token
  constexpr int RSTEP = 256 / VPR;    // tokens per sweep
  const int tid = threadIdx.x, cv = tid % VPR, tr = tid / VPR;
  float m[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) m[i] = 0.0f;
  const __nv_bfloat16* base = v + tok_off(g, bh, 0) + cv * 8;
  const size_t ts = BTHD ? (size_t)g.H * D : (size_t)D;
  int t = t0 + tr;
  for (; t + 7 * RSTEP < t1; t += 8 * RSTEP) {        // eight loads in flight per thread
    uint4 u[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) u[j] = ld_stream_u4(base + (size_t)(t + j * RSTEP) * ts);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
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
  // lanes of a warp with the same channel vector, then the eight warps
#pragma unroll
  for (int o = VPR; o < 32; o <<= 1) {
#pragma unroll
    for (int i = 0; i < 8; ++i) m[i] = fmaxf(m[i], __shfl_xor_sync(0xffffffffu, m[i], o));
  }
  const int lane = tid & 31, warp = tid >> 5;
  if (lane < VPR) {
#pragma unroll
    for (int i = 0; i < 8; ++i) scratch[warp * D + cv * 8 + i] = m[i];
  }
  __syncthreads();
  if (tid < D) {
    float a = scratch[tid];
#pragma unroll
    for (int k = 1; k < 8; ++k) a = fmaxf(a, scratch[k * D + tid]);
    atomicMax(reinterpret_cast<unsigned int*>(vamax + (size_t)bh * D + tid), __float_as_uint(a));
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

// ---- fused preparation of one (b, h, block) of Q, K (pool + quantise) or V ----
// One CTA stages the window's tokens (bf16, 16-byte copies, padded slots zero) in shared
// memory once, then writes the pooled draft vectors (Q, K), the E4M3 copy and the E2M1 copy
// with its E4M3 group scales in the tile layouts the attention kernel loads directly.
// Shared memory: the staged window X (bs rows of D + 8 bf16), 1 KB of group scales, 128
// floats of reduction scratch, the 128 E4M3 reciprocals, the pooled maxima of the Q/K path.
template <int D>
struct PrepSmem {
  __nv_bfloat16* X;
  uint8_t* sfbuf;
  float* red;
  float* rcp_tab;
};

template <int D, bool BTHD>
__device__ __forceinline__ void stage_window(const Geo& g, const __nv_bfloat16* __restrict__ src,
                                             int bh, int n, __nv_bfloat16* X) {
  constexpr int RS = D + 8;
  constexpr int VPR = D / 8;
  const int tid = threadIdx.x, bs = g.bs;
  const int fpf = g.ny * g.nx;
  const int f = n / fpf, rem = n - f * fpf, by = rem / g.nx, bx = rem - by * g.nx;
  const int y0 = by * g.ph, x0 = bx * g.pw;
  const int hv = min(g.ph, g.Hf - y0), wv = min(g.pw, g.Wf - x0);
  const __nv_bfloat16* sbase = src + tok_off(g, bh, 0);
  const size_t ts = BTHD ? (size_t)g.H * D : (size_t)D;
  // slot s = wy*pw + wx advances by a fixed step per iteration: step the window
  // coordinates instead of dividing every time; every copy of the thread in flight at once
  constexpr int DS = 256 / VPR;
  const int cv = tid % VPR;
  int s0 = tid / VPR;
  int wy = s0 / g.pw, wx = s0 - wy * g.pw;
  const int dy = DS / g.pw, dx = DS - dy * g.pw;
  for (int sl = s0; sl < bs; sl += DS) {
    const bool ok = wy < hv && wx < wv;
    const size_t t = ok ? (size_t)f * g.Hf * g.Wf + (size_t)(y0 + wy) * g.Wf + (x0 + wx) : 0;
    cp_async16(X + sl * RS + cv * 8, sbase + t * ts + cv * 8, ok ? 16u : 0u);
    wx += dx;
    wy += dy;
    if (wx >= g.pw) { wx -= g.pw; ++wy; }
  }
}

// Q (which 0) or K (which 1) block n of head bh from the staged window.
template <int D>
__device__ __forceinline__ void qk_block(const Geo& g, const Ws& w, uint8_t* tiles, int which, int bh, int n,
                                         const PrepSmem<D>& sm) {
  constexpr int RS = D + 8;
  const __nv_bfloat16* X = sm.X;
  uint8_t* sfbuf = sm.sfbuf;
  float* rcp_tab = sm.rcp_tab;
  const int tid = threadIdx.x, bs = g.bs;
  const int fpf = g.ny * g.nx;
  const int f = n / fpf, rem = n - f * fpf, by = rem / g.nx, bx = rem - by * g.nx;
  const int hv = min(g.ph, g.Hf - by * g.ph), wv = min(g.pw, g.Wf - bx * g.pw);
  (void)f;
  const int sfbytes = (int)w.sf_qk;
  // ---- draft pooling and block amax ----
  // Warps [0, NSW): fp32 running sums in slot order (two channels per lane), then an IEEE
  // divide by the number of valid tokens. Warps [NSW, 8): exact maxima and minima as bf16
  // pairs, 16 bytes of channels per lane, the valid slots split into G interleaved groups;
  // the block amax is the largest |max| or |min| (padded zero slots cannot raise it).
  constexpr int NSW = D / 64, CPW = D / 8, SPW = 32 / CPW, NMW = 8 - NSW, G = NMW * SPW;
  float* avg_out = (which == 0 ? w.qavg : w.kavg) + ((size_t)bh * g.N + n) * D;
  float* max_out = (which == 0 ? w.qmax : w.kmax) + ((size_t)bh * g.N + n) * D;
  uint32_t* pmax = reinterpret_cast<uint32_t*>(rcp_tab + 128);   // [NMW][CPW][4]
  float* wam = reinterpret_cast<float*>(pmax + NMW * CPW * 4);    // [NMW]
  const int warp = tid >> 5, lane = tid & 31;
  if (warp < NSW) {
    const int c2 = 2 * (warp * 32 + lane);
    float a0 = 0.0f, a1 = 0.0f;
    for (int wy = 0; wy < hv; ++wy) {
      const __nv_bfloat16* row = X + wy * g.pw * RS + c2;
#pragma unroll 4
      for (int wx = 0; wx < wv; ++wx) acc_bf16x2(*reinterpret_cast<const uint32_t*>(row + wx * RS), a0, a1);
    }
    const float cnt = (float)(hv * wv);
    const float x0 = __fdiv_rn(a0, cnt), x1 = __fdiv_rn(a1, cnt);
    *reinterpret_cast<float2*>(avg_out + c2) = make_float2(x0, x1);
    if (tiles) write_split_pair(tiles, bh, g.N, D, n, 0, c2, x0, x1);
  } else {
    const int mw = warp - NSW, ch = lane % CPW, sg = mw * SPW + lane / CPW;
    uint32_t mx[4], mn[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      mx[i] = 0xFF80FF80u;                                       // -inf pairs
      mn[i] = 0x7F807F80u;                                       // +inf pairs
    }
    bool any = false;
    int wy = sg / g.pw, wx = sg - wy * g.pw;
    const int dy = G / g.pw, dx = G - dy * g.pw;
    for (int sl = sg; sl < bs; sl += G) {
      if (wy < hv && wx < wv) {
        const uint4 u = *reinterpret_cast<const uint4*>(X + sl * RS + ch * 8);
        const uint32_t e[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          mx[i] = bmax2(mx[i], e[i]);
          mn[i] = bmin2(mn[i], e[i]);
        }
        any = true;
      }
      wx += dx;
      wy += dy;
      if (wx >= g.pw) { wx -= g.pw; ++wy; }
    }
    uint32_t a2 = 0u;                                            // |x| maxima as bf16 pairs
    if (any) {
#pragma unroll
      for (int i = 0; i < 4; ++i) a2 = bmax2(a2, bmax2(mx[i] & 0x7FFF7FFFu, mn[i] & 0x7FFF7FFFu));
    }
    float am = fmaxf(__uint_as_float(a2 << 16), __uint_as_float(a2 & 0xFFFF0000u));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, o));
#pragma unroll
    for (int o = CPW; o < 32; o <<= 1) {
#pragma unroll
      for (int i = 0; i < 4; ++i) mx[i] = bmax2(mx[i], __shfl_xor_sync(0xffffffffu, mx[i], o));
    }
    if (lane < CPW) {
#pragma unroll
      for (int i = 0; i < 4; ++i) pmax[(mw * CPW + ch) * 4 + i] = mx[i];
    }
    if (lane == 0) wam[mw] = am;
  }
  __syncthreads();
  if (tid < D / 2) {                                             // channel pair 2 tid, 2 tid + 1
    uint32_t m2 = pmax[tid];
#pragma unroll
    for (int k = 1; k < NMW; ++k) m2 = bmax2(m2, pmax[k * CPW * 4 + tid]);
    const float x0 = __uint_as_float(m2 << 16), x1 = __uint_as_float(m2 & 0xFFFF0000u);
    *reinterpret_cast<float2*>(max_out + 2 * tid) = make_float2(x0, x1);
    if (tiles) write_split_pair(tiles, bh, g.N, D, n, 1, 2 * tid, x0, x1);
  }
  float am = wam[0];
#pragma unroll
  for (int k = 1; k < NMW; ++k) am = fmaxf(am, wam[k]);
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
}

// V block n of head bh from the staged window; the head's channel amax is final.
template <int D>
__device__ __forceinline__ void v_block(const Geo& g, const Ws& w, int bh, int n,
                                        const PrepSmem<D>& sm) {
  constexpr int RS = D + 8;
  const __nv_bfloat16* X = sm.X;
  uint8_t* sfbuf = sm.sfbuf;
  float* red = sm.red;
  const float* rcp_tab = sm.rcp_tab;
  const int tid = threadIdx.x, bs = g.bs;
  const int sfbytes = (int)w.sf_v;
  // ---- V: per-channel outer scale from the amax pre-pass; tiles are channel-major ----
  const float* am = w.vamax + (size_t)bh * D;
  float* vinv = red;                                      // D inverse channel scales
  for (int c = tid; c < D; c += 256) {
    const float a = __ldcg(am + c);
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

template <int D>
__device__ __forceinline__ PrepSmem<D> prep_smem(uint8_t* smem, int bs) {
  PrepSmem<D> sm;
  sm.X = reinterpret_cast<__nv_bfloat16*>(smem);
  sm.sfbuf = smem + (size_t)bs * (D + 8) * 2;              // up to 1 KB of group scales
  sm.red = reinterpret_cast<float*>(sm.sfbuf + 1024);      // reduction scratch / V scales
  sm.rcp_tab = sm.red + 128;                               // 1/value of each E4M3 code
  return sm;
}

// First kernel: one item per CTA, per (b, h) 2N + nc items: amax chunk c at position c*S
// (S = (2N + nc) / nc), the Q blocks then the K blocks in the remaining positions.
template <int D, bool BTHD>
__global__ void __launch_bounds__(256) k_prepare_qk(Geo g, Ws w, const __nv_bfloat16* __restrict__ q,
                                                    const __nv_bfloat16* __restrict__ k,
                                                    const __nv_bfloat16* __restrict__ v,
                                                    uint8_t* qt, uint8_t* kt, int chunk, int nc) {
  extern __shared__ __align__(16) uint8_t smem[];
  const PrepSmem<D> sm = prep_smem<D>(smem, g.bs);
  const int tid = threadIdx.x, N = g.N;
  const int L = 2 * N + nc, S = L / nc;
  const int bh = blockIdx.x / L, r = blockIdx.x - bh * L;
  const int c = r / S;
  if (r - c * S == 0 && c < nc) {
    const int t0 = c * chunk;
    vamax_chunk<D, BTHD>(g, v, w.vamax, bh, t0, min(g.T, t0 + chunk), reinterpret_cast<float*>(smem));
    return;
  }
  const int u = r - min(nc, c + 1);                        // Q/K index: amax items before r skipped
  const int which = u >= N ? 1 : 0, n = u - which * N;
  stage_window<D, BTHD>(g, which == 0 ? q : k, bh, n, sm.X);
  for (int i = tid; i < (int)w.sf_qk / 4; i += 256) reinterpret_cast<uint32_t*>(sm.sfbuf)[i] = 0u;
  if (tid < 128) sm.rcp_tab[tid] = tid > 0 ? __frcp_rn(e4m3_to_f32((uint8_t)tid)) : 0.0f;
  cp_async_wait_all();
  __syncthreads();
  qk_block<D>(g, w, which == 0 ? qt : kt, which, bh, n, sm);
}

// Second kernel: V block blockIdx.x of head blockIdx.y.
template <int D, bool BTHD>
__global__ void __launch_bounds__(256, 4) k_prepare_v(Geo g, Ws w, const __nv_bfloat16* __restrict__ v) {
  extern __shared__ __align__(16) uint8_t smem[];
  const PrepSmem<D> sm = prep_smem<D>(smem, g.bs);
  const int tid = threadIdx.x, bh = blockIdx.y, n = blockIdx.x;
  stage_window<D, BTHD>(g, v, bh, n, sm.X);
  for (int i = tid; i < (int)w.sf_v / 4; i += 256) reinterpret_cast<uint32_t*>(sm.sfbuf)[i] = 0u;
  if (tid < 128) sm.rcp_tab[tid] = tid > 0 ? __frcp_rn(e4m3_to_f32((uint8_t)tid)) : 0.0f;
  cp_async_wait_all();
  __syncthreads();
  v_block<D>(g, w, bh, n, sm);
}

size_t prepare_smem_bytes(const Geo& g) {
  // staged window, group scales, reduction scratch, E4M3 reciprocals, pooled maxima
  return (size_t)g.bs * (g.d + 8) * 2 + 1024 + 4 * 128 + 4 * 128 + 4 * (8 * 16 * 4 + 8);
}

// Tokens per V amax item.
constexpr int kAmaxChunk = 1024;

cudaError_t launch_prepare(const Geo& g, const Ws& w, const void* q, const void* k,
                           const void* v, uint8_t* qt, uint8_t* kt, cudaStream_t st) {
  const int BH = g.B * g.H;
  cudaError_t e = cudaMemsetAsync(w.vamax, 0, sizeof(float) * BH * g.d, st);
  if (e != cudaSuccess) return e;
  e = cudaMemsetAsync(w.err, 0, sizeof(uint32_t), st);
  if (e != cudaSuccess) return e;
  const int nc = (g.T + kAmaxChunk - 1) / kAmaxChunk;
  const size_t smem = prepare_smem_bytes(g);
  const dim3 g1((unsigned)(BH * (2 * g.N + nc))), g2(g.N, BH);
  const auto* qb = static_cast<const __nv_bfloat16*>(q);
  const auto* kb = static_cast<const __nv_bfloat16*>(k);
  const auto* vb = static_cast<const __nv_bfloat16*>(v);
  if (g.d == 128 && !g.bthd) {
    k_prepare_qk<128, false><<<g1, 256, smem, st>>>(g, w, qb, kb, vb, qt, kt, kAmaxChunk, nc);
    k_prepare_v<128, false><<<g2, 256, smem, st>>>(g, w, vb);
  } else if (g.d == 128) {
    k_prepare_qk<128, true><<<g1, 256, smem, st>>>(g, w, qb, kb, vb, qt, kt, kAmaxChunk, nc);
    k_prepare_v<128, true><<<g2, 256, smem, st>>>(g, w, vb);
  } else if (!g.bthd) {
    k_prepare_qk<64, false><<<g1, 256, smem, st>>>(g, w, qb, kb, vb, qt, kt, kAmaxChunk, nc);
    k_prepare_v<64, false><<<g2, 256, smem, st>>>(g, w, vb);
  } else {
    k_prepare_qk<64, true><<<g1, 256, smem, st>>>(g, w, qb, kb, vb, qt, kt, kAmaxChunk, nc);
    k_prepare_v<64, true><<<g2, 256, smem, st>>>(g, w, vb);
  }
  return cudaGetLastError();
}

}  // namespace da2
