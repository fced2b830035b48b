// The static device array behind attn_decode_noalloc: decode partials for callers
// that cannot allocate device memory (include/attn.h says who they are).  The entry
// point itself is in api.cu; it validates the request exactly as attn_decode does and
// only then asks for this array.
#include <mutex>

#include "../../include/attn.h"
#include "internal.h"

namespace {

// Shared by every call on a device; held from the module's load until exit.
static __device__ __align__(256) unsigned char g_decode_scratch[ATTN_DECODE_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;

}  // namespace

namespace kvattn {

// Device address of g_decode_scratch on the current device, looked up once per
// device with that device current.  In host code the array's name is only a
// host-side stand-in: passing it to a kernel would read the wrong memory.  The
// address is kept for the life of the process (a context reset invalidates it).
void* noalloc_scratch() {
  static void* ptrs[kMaxDevices] = {};
  static std::mutex mu;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (!ptrs[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_decode_scratch) != cudaSuccess || p == nullptr) return nullptr;
    ptrs[dev] = p;
  }
  return ptrs[dev];
}

}  // namespace kvattn
