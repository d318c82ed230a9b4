// Debug aids shared by the C ABI and checks.cu: workspace guard regions and the check of
// the selection's lists and tags.
#pragma once
#include "common.cuh"

namespace da2 {

constexpr int kGuardBytes = 256;               // one guard after every workspace region
constexpr uint32_t kGuardWord = 0xA5A5A5A5u;   // the guard's fill pattern
constexpr uint32_t kErrCanary = 4u;            // error word bit: a guard region was overwritten
constexpr int kMaxGuards = 32;

// Byte offsets of the guard regions of one workspace.
struct GuardList {
  int n;
  unsigned long long off[kMaxGuards];
};

cudaError_t launch_guards(uint8_t* ws, const GuardList& gl, bool check, uint32_t* err, cudaStream_t st);
cudaError_t launch_check_lists(const Geo& g, const Ws& w, cudaStream_t st);

}  // namespace da2
