// sbsa_prefill_noalloc: the prefill for callers that cannot allocate device
// memory (see include/sbsa.h).  The temporaries that sbsa_prefill normally
// takes from a caller-supplied workspace (pooled query / key tables, radii
// and, unless the caller passes its own list outputs, the block lists) live
// in a fixed array compiled into the library.
#include <cuda_runtime.h>

#include <cstddef>
#include <cstdint>
#include <mutex>

#include "sbsa.h"

// One copy per GPU that loads the library, held until the process exits.
static __device__ __align__(256) unsigned char g_sbsa_noalloc_scratch[SBSA_NOALLOC_SCRATCH_BYTES];

namespace {

// Device address of the scratch array on the current device.  The name of a
// __device__ array in host code is only a host-side stand-in, so the real
// address is looked up once per device (with that device current) and
// cached; no allocation is involved.
void* scratch_on_current_device() {
  static std::mutex mu;
  static void* cached[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (!cached[dev]) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_sbsa_noalloc_scratch) != cudaSuccess) return nullptr;
    cached[dev] = ptr;
  }
  return cached[dev];
}

}  // namespace

extern "C" int sbsa_prefill_noalloc(const sbsa_params* p, const void* q, const void* k,
                                    const void* v, const void* q_idx, const void* k_idx,
                                    void* o, int32_t* idx_out, int32_t* cnt_out,
                                    uint8_t* flags_out, void* stream) {
  if (!p) return SBSA_ERR_INVALID_ARG;
  // Argument errors take precedence over the size check, as in sbsa_prefill.
  if ((idx_out == nullptr) != (cnt_out == nullptr)) return SBSA_ERR_INVALID_ARG;
  // Worst case: the lists are kept in the scratch too.  When the caller
  // provides idx_out/cnt_out, sbsa_prefill checks the smaller need itself.
  const size_t need = sbsa_prefill_workspace_bytes(p);
  if (need != 0 && idx_out == nullptr && need > (size_t)SBSA_NOALLOC_SCRATCH_BYTES)
    return SBSA_ERR_WORKSPACE;
  void* ws = scratch_on_current_device();
  if (!ws) return SBSA_ERR_CUDA;
  return sbsa_prefill(p, q, k, v, q_idx, k_idx, o, ws, (size_t)SBSA_NOALLOC_SCRATCH_BYTES,
                      idx_out, cnt_out, flags_out, stream);
}
