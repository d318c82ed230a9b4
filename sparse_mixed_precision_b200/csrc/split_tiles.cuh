// Layout of the pooled draft vectors as operands of the draft-logit MMAs (kind::tf32): the
// preparation kernel writes them, the draft kernel copies them into shared memory as they
// are.
//
// A tf32 operand keeps 10 of fp32's 23 mantissa bits, so each pooled value x is stored as
// hi = x with its low 13 mantissa bits cleared (exact in tf32) and lo = x - hi (exact in
// fp32); the MMAs sum hi_a hi_b + hi_a lo_b + lo_a hi_b. Per (b, h), 128-row tile of query
// (or key) blocks, map (0 average-pooled, 1 max-pooled) and 16-channel chunk kc there are
// two parts (hi, then lo) of 128 rows x 16 channels, 8 KB each, in the K-major core-matrix
// layout: row r, channel c of the chunk at byte kmajor_off(r, 4 c, 64). Rows past the last
// block of the head are never written and never read into a stored logit.
#pragma once
#include "common.cuh"

namespace da2 {

constexpr int kSplitRows = 128, kSplitKC = 16;
constexpr uint32_t kSplitPart = kSplitRows * kSplitKC * 4;   // one part of one chunk, 8 KB

__host__ __device__ __forceinline__ size_t split_chunk_off(int bh, int rt, int tile, int map, int kc,
                                                            int nkc) {
  return ((((size_t)bh * rt + tile) * 2 + map) * nkc + kc) * 2 * kSplitPart;
}
__host__ __device__ __forceinline__ size_t split_region_bytes(int bh_count, int N, int d) {
  const int rt = (N + kSplitRows - 1) / kSplitRows;
  return (size_t)bh_count * rt * 2 * (d / kSplitKC) * 2 * kSplitPart;
}
__device__ __forceinline__ void split_tf32(float x, float& hi, float& lo) {
  hi = __uint_as_float(__float_as_uint(x) & 0xFFFFE000u);
  lo = x - hi;
}
// Writes the split of channels c, c + 1 (c even) of pooled row n of head bh, map `map`.
__device__ __forceinline__ void write_split_pair(uint8_t* tiles, int bh, int N, int d, int n, int map,
                                                 int c, float x0, float x1) {
  const int rt = (N + kSplitRows - 1) / kSplitRows, nkc = d / kSplitKC;
  uint8_t* chunk = tiles + split_chunk_off(bh, rt, n / kSplitRows, map, c / kSplitKC, nkc);
  const uint32_t off = kmajor_off((uint32_t)(n % kSplitRows), (uint32_t)(c % kSplitKC) * 4u, kSplitKC * 4);
  float h0, l0, h1, l1;
  split_tf32(x0, h0, l0);
  split_tf32(x1, h1, l1);
  *reinterpret_cast<float2*>(chunk + off) = make_float2(h0, h1);
  *reinterpret_cast<float2*>(chunk + kSplitPart + off) = make_float2(l0, l1);
}

}  // namespace da2
