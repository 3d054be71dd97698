// cva_chunk_attention_noalloc: the fused chunk call for callers that cannot
// allocate device memory when they call it -- for example a plugin inside a
// host runtime that owns every allocation and hands the plugin only its
// input and output buffers, or a real-time loop that forbids allocation
// after start-up. Instead of a caller-provided workspace it uses one fixed
// scratch array in this file. Under CUDA's lazy module loading (the default)
// the array is reserved on a device when this file's module is first loaded
// there, which is the first call on that device (its cudaGetSymbolAddress);
// from then on it stays reserved until the process exits. That first call can
// therefore fail for lack of device memory, and it should be made during
// start-up, before any stream capture (or load eagerly with
// CUDA_MODULE_LOADING=EAGER, which reserves it when the library's modules load).
#include <stdio.h>

#include <mutex>

#include "kernels.cuh"

namespace {

// Fixed scratch: enough for the 1.3B-shaped 480P chunk (H = 12, D = 128,
// 30 x 52 latent grid, 3 frames per chunk) with any budget up to 1024
// candidate blocks; larger shapes are rejected.
constexpr size_t kNoAllocScratchBytes = 64u << 20;  // 64 MiB
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

// The array's name is only a host-side stand-in; its device address is
// looked up once per device, with that device current, and cached. The
// lookup loads the module (and so reserves the array) on that device.
void* noalloc_scratch_address(int* rc) {
  static std::mutex mu;
  static void* addr[128] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess || dev < 0 || dev >= 128) {
    *rc = cva::report_error(CVA_ELAUNCH, "noalloc: cannot query the current device");
    return nullptr;
  }
  std::lock_guard<std::mutex> lk(mu);
  if (!addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || p == nullptr) {
      char msg[256];
      snprintf(msg, sizeof(msg), "noalloc: cudaGetSymbolAddress of the fixed scratch failed: %s",
               cudaGetErrorString(e));
      *rc = cva::report_error(CVA_ELAUNCH, msg);
      return nullptr;
    }
    addr[dev] = p;
  }
  *rc = CVA_OK;
  return addr[dev];
}

}  // namespace

extern "C" int cva_chunk_attention_noalloc(const void* q, const void* k, const void* v,
                                           const cva_kv_cache* cache, const cva_rope_tables* tables,
                                           int32_t t0, int32_t k_f, int32_t k_b, void* out, float* lse,
                                           cva_stream_t stream) {
  // The arguments are checked first, exactly as cva_chunk_attention checks
  // them (a budget beyond the candidates is CVA_ERANGE, not a size problem);
  // then the scratch this shape and budget need is compared with the array.
  size_t need = 0;
  int rc = cva::check_chunk_call(q, k, v, cache, tables, t0, k_f, k_b, out, &need);
  if (rc) return rc;
  if (need > kNoAllocScratchBytes) {
    char msg[256];
    snprintf(msg, sizeof(msg),
             "noalloc: this shape and budget need %zu bytes of scratch; the fixed scratch holds %zu "
             "(use cva_chunk_attention with a caller workspace)",
             need, kNoAllocScratchBytes);
    return cva::report_error(CVA_ENOMEM, msg);
  }
  void* ws = noalloc_scratch_address(&rc);
  if (!ws) return rc;
  // Nothing in the workspace has to start at zero: every byte the path reads
  // is written earlier in the same call.
  return cva_chunk_attention(q, k, v, cache, tables, t0, k_f, k_b, ws, kNoAllocScratchBytes, out, lse,
                             stream);
}
