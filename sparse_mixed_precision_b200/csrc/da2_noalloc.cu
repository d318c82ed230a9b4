// da2_forward_noalloc: the whole hot path without any device allocation by anyone.
//
// Some callers have no way to obtain device memory at the point where they run the
// attention: a plug-in called from a host framework that owns every device byte and
// exposes no allocator to it, or a serving loop that forbids cudaMalloc after start-up
// (it can synchronise the device and can fail under fragmentation). For them this entry
// point keeps its workspace in a fixed device array that is part of the library image.
//
// The array is a file-scope static __device__ object of kScratchBytes (64 MiB). Every GPU
// that loads the library holds it until the process exits. In host code the array's
// name is only a host-side stand-in, so the device address is looked up once per device
// with cudaGetSymbolAddress (with that device current) and handed to the kernels as an
// ordinary pointer.
#include <mutex>

#include "common.cuh"

namespace {

constexpr size_t kScratchBytes = size_t(64) << 20;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_scratch[kScratchBytes];

std::mutex g_mu;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of g_scratch on the current device (looked up on first use per device).
da2_status scratch_address(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return DA2_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return DA2_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_scratch) != cudaSuccess || !p) return DA2_ERR_CUDA;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return DA2_OK;
}

}  // namespace

extern "C" da2_status da2_forward_noalloc(const da2_config* cfg, const void* q, const void* k,
                                          const void* v, void* out, cudaStream_t stream) {
  size_t need = 0;
  const da2_status s = da2_workspace_size(cfg, &need);
  if (s != DA2_OK) return s;
  if (need > kScratchBytes) return DA2_ERR_SCRATCH_TOO_SMALL;
  void* ws = nullptr;
  const da2_status a = scratch_address(&ws);
  if (a != DA2_OK) return a;
  return da2_forward(cfg, q, k, v, out, ws, kScratchBytes, stream);
}
