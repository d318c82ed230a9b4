// Debug aids, off unless asked for: guard regions ("canaries") after every workspace region
// (DA2_FLAG_DEBUG_CANARY), and a check of the selection's output contract that DA2_DEBUG
// builds run between the draft selection and the attention.
#include "checks.cuh"

namespace da2 {

// One CTA per guard region: write the guard pattern, or compare against it and set
// kErrCanary in the error word on any difference.
__global__ void k_guards(uint8_t* ws, GuardList gl, int check, uint32_t* err) {
  uint32_t* p = reinterpret_cast<uint32_t*>(ws + gl.off[blockIdx.x]);
  bool bad = false;
  for (int i = threadIdx.x; i < kGuardBytes / 4; i += blockDim.x) {
    if (check) bad |= p[i] != kGuardWord;
    else p[i] = kGuardWord;
  }
  if (__syncthreads_or(bad) && threadIdx.x == 0) atomicOr(err, kErrCanary);
}

// The contract between the draft selection and the attention, one thread per (b, h, query
// block): the FP8, mixed and FP4 lists hold in-range, strictly ascending KV blocks whose tags
// are 2, 3 and 1; the FP4 list is padded with -1 after its last block only; the row has
// exactly n8 FP8 and nm mixed tags and between n4 and n4max FP4 tags, and every tagged block
// is listed. Any violation sets kErrBadIndex.
__global__ void k_check_lists(Geo g, Ws w) {
  const long row = (long)blockIdx.x * blockDim.x + threadIdx.x;
  const int N = g.N;
  if (row >= (long)g.B * g.H * N) return;
  const uint8_t* tags = w.tags + row * N;
  bool ok = true;
  auto check_list = [&](const int16_t* l, int len, int n_valid, uint8_t tag) {
    int prev = -1;
    for (int p = 0; p < len; ++p) {
      const int j = l[p];
      if (p < n_valid) {
        ok &= j > prev && j < N && tags[j] == tag;
        prev = j;
      } else {
        ok &= j == -1;
      }
    }
  };
  int n8 = 0, nm = 0, n4 = 0;
  for (int j = 0; j < N; ++j) {
    const uint8_t t = tags[j];
    n8 += t == 2;
    nm += t == 3;
    n4 += t == 1;
    ok &= t <= 3;
  }
  ok &= n8 == g.n8 && nm == g.nm && n4 >= g.n4 && n4 <= g.n4max;
  if (g.n8 > 0) check_list(w.list8 + row * w.n8s, g.n8, g.n8, 2);
  if (g.nm > 0) check_list(w.listm + row * w.nms, g.nm, g.nm, 3);
  if (g.n4max > 0) check_list(w.list4 + row * w.n4s, g.n4max, n4, 1);
  if (!ok) atomicOr(w.err, kErrBadIndex);
}

cudaError_t launch_guards(uint8_t* ws, const GuardList& gl, bool check, uint32_t* err, cudaStream_t st) {
  if (gl.n <= 0) return cudaSuccess;
  k_guards<<<gl.n, 64, 0, st>>>(ws, gl, check ? 1 : 0, err);
  return cudaGetLastError();
}

cudaError_t launch_check_lists(const Geo& g, const Ws& w, cudaStream_t st) {
  const long rows = (long)g.B * g.H * g.N;
  k_check_lists<<<(unsigned)((rows + 127) / 128), 128, 0, st>>>(g, w);
  return cudaGetLastError();
}

}  // namespace da2
