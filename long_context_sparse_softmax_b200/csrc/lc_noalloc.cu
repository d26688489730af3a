// Allocation-free variant of the CSA sparse-attention decode call.
//
// The regular decode call (lc_csa_sparse_attn_decode) may split each query's keys across
// CTAs; the partial results of the splits then live in a workspace the caller allocates.
// Some callers cannot allocate device memory at the point of the call: hosts that hand
// every byte of device memory to their own allocator up front and forbid any other
// allocation, and latency-bound serving loops that must never pay for the device-wide
// synchronisation cudaMalloc can imply.  This entry point serves them: its scratch is a
// fixed array compiled into the library, so the call allocates nothing.
//
// The array below is a host-side stand-in in host code, not a device address.  The first
// call on each device, with that device current, asks the runtime for the array's device
// address (cudaGetSymbolAddress) and remembers it; later calls on that device reuse it.
// Make that first call on a device before any stream capture on it.
#include <cstdint>
#include <mutex>

#include "lc_internal.h"

namespace {

constexpr size_t kStaticScratchBytes = 16u << 20;  // 16 MiB on every device that loads the library
constexpr int kMaxDevices = 64;

// Shared by every call on a device and kept until the process exits.
static __device__ __align__(256) uint8_t g_attn_scratch[kStaticScratchBytes];

std::mutex g_mu;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of g_attn_scratch on the current device (looked up once per device).
lc_status scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return LC_ERR_LAUNCH;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_attn_scratch) != cudaSuccess || !p) return LC_ERR_LAUNCH;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return LC_OK;
}

}  // namespace

extern "C" {

size_t lc_csa_sparse_attn_decode_static_capacity(void) { return kStaticScratchBytes; }

lc_status lc_csa_sparse_attn_decode_static(const lc_attn_args* a, void* stream) {
  if (!a) return LC_ERR_ARG;
  // the caller's workspace fields are ignored; the kernel choice (and so the scratch it
  // needs) is made for the 256-byte-aligned array the call will pass
  lc_attn_args b = *a;
  b.workspace = nullptr;
  b.workspace_bytes = 0;
  const size_t need = lc::attn_workspace_bytes(b, true, true);
  if (need > kStaticScratchBytes) return LC_ERR_TOO_LARGE;  // checked before touching the device
  if (need > 0) {
    void* p = nullptr;
    const lc_status s = scratch_address(&p);
    if (s != LC_OK) return s;
    b.workspace = p;
    b.workspace_bytes = kStaticScratchBytes;
  }
  return lc_csa_sparse_attn_decode(&b, stream);
}

}  // extern "C"
