// Fixed device scratch for metis_residual_quantize_nvfp4_noalloc.
//
// Some callers may not allocate device memory while they run: a step captured
// into a CUDA graph cannot call cudaMalloc, and a framework that owns the
// device memory through its own caching allocator loses track of (and can
// fragment around) memory a library allocates behind it.  For them the
// residual quantizer has a variant whose scratch -- the fp16 hi/lo tiles of
// U diag(S) and V that the tensor cores read, with their per-block scale
// factors -- lives in this file-scope array, reserved once when the library's
// module loads on a device and held until the process exits.
#include <cuda_runtime.h>

#include <mutex>

#include "internal.h"

// 256 bytes per row and column for rows + cols <= 24576 (6 MiB), 1 KiB of block factors
// and a 256-byte tail for the amax word, on every device that loads the library.
static __device__ __align__(256) char g_noalloc_scratch[metis::kNoAllocBytes];

namespace metis {
namespace {
constexpr int kMaxDevices = 64;
char* g_scratch_ptr[kMaxDevices] = {};
std::mutex g_scratch_mutex;
}  // namespace

// Device address of the scratch array on the context's device (which must be
// current).  Looked up once per device; later calls only read the cache.
char* noalloc_scratch(metis_ctx* ctx, metis_status* st) {
  if (ctx->device < 0 || ctx->device >= kMaxDevices) {
    *st = fail(ctx, METIS_ERR_ARG, "device index beyond the scratch table");
    return nullptr;
  }
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  if (!g_scratch_ptr[ctx->device]) {
    void* ptr = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&ptr, g_noalloc_scratch);
    if (e != cudaSuccess || !ptr) {
      *st = check_cuda(ctx, e == cudaSuccess ? cudaErrorInvalidSymbol : e, "cudaGetSymbolAddress(scratch)");
      return nullptr;
    }
    g_scratch_ptr[ctx->device] = static_cast<char*>(ptr);
  }
  *st = METIS_OK;
  return g_scratch_ptr[ctx->device];
}

}  // namespace metis
