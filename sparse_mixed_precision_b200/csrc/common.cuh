// Device helpers shared by the da2 kernels: geometry, tile layouts, E4M3 / E2M1
// conversions (hardware cvt instructions of sm_100a), error word.
#pragma once
#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "../../include/da2.h"

namespace da2 {

constexpr float kE4M3Max = 448.0f;

// Geometry of one call, resolved on the host and passed by value to the kernels.
struct Geo {
  int B, H, d, F, Hf, Wf, ph, pw;
  int ny, nx, N, bs, T, Tp, n8, n4, kv4;
  int nm;     // mixed KV blocks per query block (E4M3 scores, E2M1 P V)
  int n4max;  // FP4 list length per query block (n4 unless the adaptive budget is on)
  float tau;  // adaptive FP4 budget threshold on the draft score (0: off)
  float sm_scale;
  int flags;
  int bthd;   // q, k, v, out token-major [B,T,H,d] instead of [B,H,T,d]
  unsigned long long wait_ns;   // limit of every bounded device wait (%globaltimer ns)
};

// Element offset of token t, channel 0 of head bh = b*H + h in a q/k/v/out tensor.
__host__ __device__ __forceinline__ size_t tok_off(const Geo& g, int bh, size_t t) {
  if (!g.bthd) return ((size_t)bh * g.T + t) * g.d;
  const int b = bh / g.H, h = bh - b * g.H;
  return (((size_t)b * g.T + t) * g.H + h) * g.d;
}
// Elements between consecutive tokens of one head.
__host__ __device__ __forceinline__ size_t tok_stride(const Geo& g) {
  return g.bthd ? (size_t)g.H * g.d : (size_t)g.d;
}

// Workspace base pointers, resolved on the host.
struct Ws {
  uint8_t *q8, *k8, *v8, *q4, *k4, *v4, *sfq4, *sfk4, *sfv4;
  float *sq, *sk, *sv, *vamax, *qavg, *qmax, *kavg, *kmax, *scores;
  uint8_t* tags;
  int16_t *list8, *list4, *listm;
  uint32_t* err;
  size_t tile8_qk, tile4_qk, tile8_v, tile4_v, sf_qk, sf_v;
  int n8s, n4s, nms;
};

// Device error word bits.
enum : uint32_t { kErrWaitTimeout = 1u, kErrBadIndex = 2u };

// ---- tensor-core K-major core-matrix layout (8 rows x 16 bytes per core matrix) ----
// Byte offset of (row r, byte b) in a tile whose rows are `rowbytes` long.
__host__ __device__ __forceinline__ uint32_t kmajor_off(uint32_t r, uint32_t b, uint32_t rowbytes) {
  return (r >> 3) * (rowbytes * 8u) + (b >> 4) * 128u + (r & 7u) * 16u + (b & 15u);
}
// Byte offset of scale j (0..3) of row r (0..127) in k-block kb of a scale-factor tile
// (512-byte atoms: row r%32 owns 16 bytes, holding rows r%32 + 32*i, i = 0..3).
__host__ __device__ __forceinline__ uint32_t sf_off(uint32_t kb, uint32_t r, uint32_t j) {
  return kb * 512u + (r & 31u) * 16u + (r >> 5) * 4u + j;
}

// ---- conversions ----
// Two floats to two E4M3 bytes (lo -> bits 0..7), round to nearest even, saturating.
__device__ __forceinline__ uint16_t f32x2_to_e4m3x2(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}
__device__ __forceinline__ uint8_t f32_to_e4m3(float x) {
  return (uint8_t)(f32x2_to_e4m3x2(x, 0.0f) & 0xFF);
}
// E4M3 byte to float (exact, through the f16x2 conversion).
__device__ __forceinline__ float e4m3_to_f32(uint8_t c) {
  uint32_t h2;
  uint16_t in = c;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(in));
  return __half2float(__ushort_as_half((unsigned short)(h2 & 0xFFFF)));
}
// Eight floats to eight E2M1 codes packed in 32 bits (element i in nibble i).
__device__ __forceinline__ uint32_t f32x8_to_e2m1x8(const float* v) {
  uint32_t out;
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
      "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
      : "=r"(out)
      : "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]), "f"(v[7]));
  return out;
}
__device__ __forceinline__ float e2m1_to_f32(uint32_t code) {
  const float mag = (code & 4u) ? ((code & 2u) ? ((code & 1u) ? 6.0f : 4.0f)
                                               : ((code & 1u) ? 3.0f : 2.0f))
                                : ((code & 2u) ? ((code & 1u) ? 1.5f : 1.0f)
                                               : ((code & 1u) ? 0.5f : 0.0f));
  return (code & 8u) ? -mag : mag;
}

__device__ __forceinline__ void set_error(uint32_t* err, uint32_t bits) {
  if (err) atomicOr(err, bits);
}

}  // namespace da2
