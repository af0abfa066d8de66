// thinkv_noalloc.cu -- decode attention with library-owned scratch.
//
// For callers that cannot allocate device memory where they decode (a host
// framework that owns all device memory and gives its plugins no allocator;
// paths that cannot afford cudaMalloc's device-wide synchronisation).  The
// split-K scratch of the decode kernels -- the live-page prefix and the
// per-piece partial outputs and top-k lists -- is one file-scope device array
// of fixed size instead of a caller workspace.  The ThinKV pages have no
// counterpart.
#include <cuda_runtime.h>
#include <mutex>
#include <stdint.h>

#include "thinkv.h"
#include "thinkv_internal.h"

namespace {

constexpr size_t kScratchBytes = THINKV_NOALLOC_SCRATCH_BYTES;

// Every GPU that loads the library holds this array until the process exits.
// In host code the symbol is only a host-side stand-in; the kernel gets the
// device address looked up below.
static __device__ __align__(256) unsigned char g_scratch[kScratchBytes];

std::mutex g_lock;
void* g_ptr[64] = {nullptr};

// Device address of g_scratch on the current device: looked up once per
// device, with that device current (the first call on a device does this).
cudaError_t scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> guard(g_lock);
  if (!g_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_scratch);
    if (e != cudaSuccess) return e;
    g_ptr[dev] = p;
  }
  *out = g_ptr[dev];
  return cudaSuccess;
}

}  // namespace

extern "C" int thinkv_decode_attention_noalloc(const thinkv_cache* C, int32_t n, const int32_t* seq,
                                               const uint16_t* q, uint16_t* out, float* topk_mass,
                                               int32_t topk, float softmax_scale, void* stream) {
  using namespace thinkv;
  if (!cache_ok(C) || n < 1 || n > 16384) return THINKV_ERR_INVALID;
  if (!seq || !q || !out) return THINKV_ERR_INVALID;
  if (topk_mass && (topk < 1 || topk > 64)) return THINKV_ERR_INVALID;
  if (!decode_args_aligned(seq, q, out, topk_mass)) return THINKV_ERR_INVALID;
  const int k = topk_mass ? topk : 0;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return THINKV_ERR_CUDA;
  DecodeLaunch dl;
  if (!plan_decode_launch(C->L, n, k, dev, &dl)) return THINKV_ERR_INVALID;
  if (decode_workspace_bytes(C->L, n, k, dl) > kScratchBytes) return THINKV_ERR_WORKSPACE;
  void* ws = nullptr;
  const cudaError_t e = scratch_address(&ws);
  if (e != cudaSuccess) return cuda_status(e);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  return cuda_status(launch_decode(view_of(C), n, seq, q, out, topk_mass, k, softmax_scale, ws, dl, s));
}
