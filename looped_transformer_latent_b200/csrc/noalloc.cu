// hla_decode_attn_noalloc: the absorbed latent read for callers that cannot
// allocate device memory.
//
// Who needs it: code that only receives input and output buffers and has no
// way to obtain scratch -- for example a plugin behind a host interface that
// passes tensors but offers no allocator, or a serving engine that reserves
// all device memory for its KV cache up front, where an extra cudaMalloc
// either fails or implicitly synchronises the device in the middle of a
// decode loop.  This entry point takes no workspace argument.  Its scratch is
// one file-scope device array of LLA_NOALLOC_SCRATCH_BYTES, created with the
// library's module on each device that uses it and kept until the process
// exits.  Nothing here calls cudaMalloc, cudaFree or any allocating routine.
//
// The host cannot pass the array's name to a kernel: in host code that name
// is only a stand-in symbol, not a device address.  The device address is
// looked up once per device with cudaGetSymbolAddress, with that device
// current, on the first call made on that device; that first call should
// therefore happen before any stream capture begins.
//
// All calls share the one array and it keeps whatever the last call left in
// it.  The absorbed read writes every scratch word before reading it, so
// nothing has to start at zero.  Two calls whose work overlaps on the GPU
// (different streams, or different host threads without ordering) race on
// the array; order them on one stream or use hla_decode_attn with separate
// workspaces.
#include <mutex>

#include "lla.h"

namespace {

constexpr size_t kScratchBytes = LLA_NOALLOC_SCRATCH_BYTES;
static __device__ __align__(256) unsigned char g_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_setup_mutex;
void* g_scratch_addr[kMaxDevices];  // device address of g_scratch, per device

// Device address of g_scratch on the current device (looked up once).
int scratch_address(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return LLA_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return LLA_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  if (g_scratch_addr[dev] == nullptr) {
    void* addr = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&addr, g_scratch);
    if (e != cudaSuccess || addr == nullptr) return LLA_ERR_CUDA;
    g_scratch_addr[dev] = addr;
  }
  *out = g_scratch_addr[dev];
  return LLA_OK;
}

}  // namespace

extern "C" int hla_decode_attn_noalloc(const hla_decode_params* p, lla_stream stream) {
  if (!p) return LLA_ERR_NULL;
  // Problems whose scratch would not fit are refused before anything runs.
  if (hla_decode_workspace_bytes(p) > kScratchBytes) return LLA_ERR_WORKSPACE;
  void* scratch = nullptr;
  const int st = scratch_address(&scratch);
  if (st != LLA_OK) return st;
  return hla_decode_attn(p, scratch, kScratchBytes, stream);
}
