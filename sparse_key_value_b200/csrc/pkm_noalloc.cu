// pkm_noalloc.cu -- pkm_forward for callers that cannot allocate device
// memory.
//
// Some callers of this library have no way to obtain device memory for the
// forward's scratch: a plain C program that links only libpkm.so and owns no
// allocator, an inference runtime that fixes its memory budget at start-up and
// forbids allocations while serving, or code that must not trigger the
// synchronising cudaMalloc/cudaFree inside a latency-critical loop.  For them
// pkm_forward_noalloc runs the same forward with its scratch in a fixed
// file-scope device array instead of a caller-supplied workspace.
//
// The array is kNoAllocScratchBytes (32 MiB) per device and exists on every
// device that loads the library until the process exits.  Its device address
// is looked up once per device (cudaGetSymbolAddress, with that device
// current) on the first call made on that device.  All calls share the array
// and it keeps the previous call's contents; the forward writes every scratch
// byte it reads before reading it, so nothing needs clearing.  Calls whose
// GPU work overlaps (two streams, or two host threads) race on the array.
#include <mutex>

#include "common.cuh"
#include "kernels.h"

namespace pkm {
namespace {

constexpr size_t kNoAllocScratchBytes = size_t(32) << 20;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

std::mutex g_noalloc_mu;
void* g_noalloc_ptr[64] = {nullptr};

// Device address of the scratch array on the current device (set up once per
// device); nullptr if the lookup failed.
void* noalloc_scratch() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (!g_noalloc_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return nullptr;
    g_noalloc_ptr[dev] = p;
  }
  return g_noalloc_ptr[dev];
}

}  // namespace
}  // namespace pkm

extern "C" pkm_status pkm_forward_noalloc(const pkm_fwd_args* args, pkm_stream_t stream) {
  using namespace pkm;
  // invalid arguments are refused as such before any size is computed from them
  const pkm_status s = check_fwd_args(args);
  if (s != PKM_OK || args->T == 0) return s;
  // the sizes alone decide the scratch need; refuse anything beyond the array
  if (forward_workspace_bytes(args) > kNoAllocScratchBytes) return PKM_ERR_WORKSPACE;
  void* scratch = noalloc_scratch();
  if (!scratch) return PKM_ERR_CUDA;
  return forward_into(args, scratch, kNoAllocScratchBytes, reinterpret_cast<cudaStream_t>(stream));
}
