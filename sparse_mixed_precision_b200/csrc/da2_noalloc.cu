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
// name is only a host-side stand-in, so its device address is looked up with
// cudaGetSymbolAddress, with the caller's device current, and handed to the kernels as an
// ordinary pointer. The lookup is repeated on every call (it is a host-side table lookup):
// an address kept from an earlier call could belong to a context that a device reset has
// since destroyed.
#include "common.cuh"

namespace {

constexpr size_t kScratchBytes = size_t(64) << 20;

static __device__ __align__(256) unsigned char g_scratch[kScratchBytes];

}  // namespace

namespace da2 {

// Device address of the built-in scratch on the current device, and its size.
da2_status noalloc_scratch(void** ptr, size_t* bytes) {
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_scratch) != cudaSuccess || !p) return DA2_ERR_CUDA;
  *ptr = p;
  *bytes = kScratchBytes;
  return DA2_OK;
}

}  // namespace da2

extern "C" da2_status da2_forward_noalloc(const da2_config* cfg, const void* q, const void* k,
                                          const void* v, void* out, cudaStream_t stream) {
  size_t need = 0;
  const da2_status s = da2_workspace_size(cfg, &need);
  if (s != DA2_OK) return s;
  // the exported scores would land in the scratch, where no caller can read them
  if (cfg->flags & DA2_FLAG_EXPORT_SCORES) return DA2_ERR_INVALID_ARG;
  if (need > kScratchBytes) return DA2_ERR_SCRATCH_TOO_SMALL;
  if (!q || !k || !v || !out) return DA2_ERR_INVALID_ARG;
  void* ws = nullptr;
  size_t ws_bytes = 0;
  const da2_status a = da2::noalloc_scratch(&ws, &ws_bytes);
  if (a != DA2_OK) return a;
  return da2_forward(cfg, q, k, v, out, ws, ws_bytes, stream);
}
