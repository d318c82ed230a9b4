// Mixed-precision block-sparse attention (K3).
//
// "DraftAttention2: Fast Video Diffusion with Low-Resolution-Guided Mixed-Precision
// Attention", Abstract: one attention kernel with precision-specific phases that share
// data movement, softmax statistics and output accumulation. "DraftAttention: Fast Video
// Diffusion via Low-Resolution Attention Guidance", Abstract: the output is restored to
// the original token order after the block-sparse attention.
//
// Per (b, h, query block i): the FP8 phase visits list8[i] then the FP4 phase visits
// list4[i], both in ascending block order, with ONE running row max m, ONE running sum l
// and ONE fp32 accumulator. For each visited block: S = (s_q s_k sm_scale) * (q' . k'),
// padded keys masked; m_new = max(m, rowmax S); l = l e^(m-m_new) + sum e^(S-m_new);
// P~ = the block's quantisation of e^(S-m_new) (E4M3 of 448 p, or E2M1 with E4M3 group
// scales over 16 keys of 448 p); acc = acc e^(m-m_new) + P~ V'. Epilogue: O = acc * s_v /
// (448 l), bf16, scattered back to the original token positions.
#include "common.cuh"

namespace da2 {

template <int D>
__device__ void load_qk_tile(float* dst, int ld, const Ws& w, int prec, bool is_q, size_t bhn, int bs) {
  if (prec == 8) {
    const uint8_t* t = (is_q ? w.q8 : w.k8) + bhn * w.tile8_qk;
    for (int u = threadIdx.x; u < bs * D / 16; u += blockDim.x) {
      const int s = u / (D / 16), kc = u - s * (D / 16);
      const uint4 v = *reinterpret_cast<const uint4*>(t + kmajor_off(s, kc * 16, D));
      const uint8_t* b = reinterpret_cast<const uint8_t*>(&v);
#pragma unroll
      for (int e = 0; e < 16; ++e) dst[s * ld + kc * 16 + e] = e4m3_to_f32(b[e]);
    }
  } else {
    const uint8_t* t = (is_q ? w.q4 : w.k4) + bhn * w.tile4_qk;
    const uint8_t* sf = (is_q ? w.sfq4 : w.sfk4) + bhn * w.sf_qk;
    for (int u = threadIdx.x; u < bs * D / 32; u += blockDim.x) {
      const int s = u / (D / 32), kc = u - s * (D / 32);
      const uint4 v = *reinterpret_cast<const uint4*>(t + kmajor_off(s, kc * 16, D / 2));
      const uint8_t* b = reinterpret_cast<const uint8_t*>(&v);
      const float s0 = e4m3_to_f32(sf[sf_off((2 * kc) >> 2, s, (2 * kc) & 3)]);
      const float s1 = e4m3_to_f32(sf[sf_off((2 * kc + 1) >> 2, s, (2 * kc + 1) & 3)]);
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        const float sg = e < 8 ? s0 : s1;
        dst[s * ld + kc * 32 + 2 * e] = sg * e2m1_to_f32(b[e] & 15u);
        dst[s * ld + kc * 32 + 2 * e + 1] = sg * e2m1_to_f32(b[e] >> 4);
      }
    }
  }
}

// V tile of block j into dst[slot][channel]
template <int D>
__device__ void load_v_tile(float* dst, int ld, const Ws& w, int prec, size_t bhn, int bs, int kv4) {
  if (prec == 8) {
    const uint8_t* t = w.v8 + bhn * w.tile8_v;
    for (int u = threadIdx.x; u < D * bs / 16; u += blockDim.x) {
      const int c = u / (bs / 16), sc = u - c * (bs / 16);
      const uint4 v = *reinterpret_cast<const uint4*>(t + kmajor_off(c, sc * 16, bs));
      const uint8_t* b = reinterpret_cast<const uint8_t*>(&v);
#pragma unroll
      for (int e = 0; e < 16; ++e) dst[(sc * 16 + e) * ld + c] = e4m3_to_f32(b[e]);
    }
  } else {
    const uint8_t* t = w.v4 + bhn * w.tile4_v;
    const uint8_t* sf = w.sfv4 + bhn * w.sf_v;
    for (int u = threadIdx.x; u < D * bs / 32; u += blockDim.x) {
      const int c = u / (bs / 32), sc = u - c * (bs / 32);
      const uint4 v = *reinterpret_cast<const uint4*>(t + kmajor_off(c, sc * 16, kv4 / 2));
      const uint8_t* b = reinterpret_cast<const uint8_t*>(&v);
      const float s0 = e4m3_to_f32(sf[sf_off((2 * sc) >> 2, c, (2 * sc) & 3)]);
      const float s1 = e4m3_to_f32(sf[sf_off((2 * sc + 1) >> 2, c, (2 * sc + 1) & 3)]);
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        const float sg = e < 8 ? s0 : s1;
        dst[(sc * 32 + 2 * e) * ld + c] = sg * e2m1_to_f32(b[e] & 15u);
        dst[(sc * 32 + 2 * e + 1) * ld + c] = sg * e2m1_to_f32(b[e] >> 4);
      }
    }
  }
}

template <int D>
__global__ void __launch_bounds__(128) k_attention_cc(Geo g, Ws w, __nv_bfloat16* __restrict__ out) {
  constexpr int LD = D + 1;
  extern __shared__ __align__(16) float ssm[];
  const int bs = g.bs, PL = bs + 1;
  float* Qs = ssm;
  float* KV = Qs + bs * LD;
  float* P = KV + bs * LD;
  const int i = blockIdx.x, bh = blockIdx.y, r = threadIdx.x;
  const int N = g.N, fpf = g.ny * g.nx;
  float o[D];
#pragma unroll
  for (int c = 0; c < D; ++c) o[c] = 0.0f;
  float m = -INFINITY, l = 0.0f;
  const float sqi = w.sq[(size_t)bh * N + i];
  for (int phase = 0; phase < 2; ++phase) {
    const int prec = phase == 0 ? 8 : 4;
    const int cnt = phase == 0 ? g.n8 : g.n4;
    if (cnt == 0) continue;
    const int16_t* lst = (phase == 0 ? w.list8 : w.list4) + ((size_t)bh * N + i) * (phase == 0 ? w.n8s : w.n4s);
    __syncthreads();
    load_qk_tile<D>(Qs, LD, w, prec, true, (size_t)bh * N + i, bs);
    for (int t = 0; t < cnt; ++t) {
      int j = lst[t];
      if (j < 0 || j >= N) {
        if (r == 0) set_error(w.err, kErrBadIndex);
        j = 0;
      }
      __syncthreads();
      load_qk_tile<D>(KV, LD, w, prec, false, (size_t)bh * N + j, bs);
      __syncthreads();
      const float scale = sqi * w.sk[(size_t)bh * N + j] * g.sm_scale;
      const int rem = j % fpf, by = rem / g.nx, bx = rem - by * g.nx;
      const int hv = min(g.ph, g.Hf - by * g.ph), wv = min(g.pw, g.Wf - bx * g.pw);
      if (r < bs) {
        float mx = -INFINITY;
        for (int s = 0; s < bs; ++s) {
          float dot = 0.0f;
#pragma unroll 8
          for (int c = 0; c < D; ++c) dot = fmaf(Qs[r * LD + c], KV[s * LD + c], dot);
          const int wy = s / g.pw, wx = s - wy * g.pw;
          const float S = (wy < hv && wx < wv) ? dot * scale : -INFINITY;
          P[r * PL + s] = S;
          mx = fmaxf(mx, S);
        }
        const float m_new = fmaxf(m, mx);
        const float alpha = (m == -INFINITY) ? 0.0f : expf(m - m_new);
        float lsum = 0.0f;
        for (int s = 0; s < bs; ++s) {
          const float S = P[r * PL + s];
          const float p = (S == -INFINITY) ? 0.0f : expf(S - m_new);
          lsum += p;
          P[r * PL + s] = p * kE4M3Max;
        }
        l = alpha * l + lsum;
        if (prec == 8) {
          for (int s = 0; s < bs; ++s) P[r * PL + s] = e4m3_to_f32(f32_to_e4m3(P[r * PL + s]));
        } else {
          for (int s0 = 0; s0 < bs; s0 += 16) {
            float y[16];
            uint32_t pk[2];
#pragma unroll
            for (int e = 0; e < 16; ++e) y[e] = P[r * PL + s0 + e];
            const float sg = e4m3_to_f32(quant_fp4_group16(y, pk));
#pragma unroll
            for (int e = 0; e < 16; ++e)
              P[r * PL + s0 + e] = sg * e2m1_to_f32((pk[e >> 3] >> (4 * (e & 7))) & 15u);
          }
        }
#pragma unroll
        for (int c = 0; c < D; ++c) o[c] *= alpha;
        m = m_new;
      }
      __syncthreads();
      load_v_tile<D>(KV, LD, w, prec, (size_t)bh * N + j, bs, g.kv4);
      __syncthreads();
      if (r < bs) {
        for (int s = 0; s < bs; ++s) {
          const float ps = P[r * PL + s];
#pragma unroll
          for (int c = 0; c < D; ++c) o[c] = fmaf(ps, KV[s * LD + c], o[c]);
        }
      }
    }
  }
  // epilogue: O = acc * s_v / (448 l), original token order
  if (r < bs) {
    const int f = i / fpf, rem = i - f * fpf, by = rem / g.nx, bx = rem - by * g.nx;
    const int hv = min(g.ph, g.Hf - by * g.ph), wv = min(g.pw, g.Wf - bx * g.pw);
    const int wy = r / g.pw, wx = r - wy * g.pw;
    if (wy < hv && wx < wv) {
      const size_t t = (size_t)f * g.Hf * g.Wf + (size_t)(by * g.ph + wy) * g.Wf + bx * g.pw + wx;
      __nv_bfloat16* dst = out + ((size_t)bh * g.T + t) * D;
      const float inv_l = l > 0.0f ? 1.0f / (l * kE4M3Max) : 0.0f;
      const float* sv = w.sv + (size_t)bh * D;
#pragma unroll
      for (int c = 0; c < D; ++c) dst[c] = __float2bfloat16_rn(o[c] * sv[c] * inv_l);
    }
  }
}

cudaError_t launch_attention(const Geo& g, const Ws& w, void* out, cudaStream_t st) {
  const size_t smem = (size_t)(2 * g.bs * (g.d + 1) + g.bs * (g.bs + 1)) * 4;
  dim3 grid(g.N, g.B * g.H);
  auto* o = static_cast<__nv_bfloat16*>(out);
  cudaError_t e;
  if (g.d == 128) {
    e = cudaFuncSetAttribute(k_attention_cc<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    k_attention_cc<128><<<grid, 128, smem, st>>>(g, w, o);
  } else {
    e = cudaFuncSetAttribute(k_attention_cc<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    k_attention_cc<64><<<grid, 128, smem, st>>>(g, w, o);
  }
  return cudaGetLastError();
}

}  // namespace da2
