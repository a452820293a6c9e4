// fvattn_pool_select_noalloc: the pool/select step for callers that cannot
// allocate device memory.
//
// Some callers have no way to obtain a workspace buffer: a plugin running
// inside a host application that owns every device allocation and hands the
// plugin only its input and output tensors, or code on a latency-critical
// path where the device-wide synchronisation of cudaMalloc is not allowed.
// For them this entry point runs the same kernels as fvattn_pool_select with
// its scratch memory (tile tables, pooled Q/K) in one statically sized
// device array that is part of this library.  The caller still provides
// q, k and the block-list buffers.
//
// The array below is a host-side name only: its device address is looked up
// with cudaGetSymbolAddress the first time the entry point runs on each
// device (with that device current) and cached; kernels only ever receive
// that address.
#include <mutex>

#include "fvattn_internal.cuh"

// 32 MiB.  A shape is accepted when its full workspace
// (fvattn_workspace_size) fits: for example the 16x32x32 latent with 12
// heads (13.6 MiB) or the 20x32x52 latent with up to 8 heads (29.0 MiB); the
// 20x32x52 latent with 9 heads (32.6 MiB) or 40 heads (144.2 MiB) is
// rejected.  The first 4 bytes hold the status word that kernels set on a
// device-detected error (fvattn_pool_select_noalloc_status reads it).
static constexpr size_t kNoAllocScratchBytes = size_t(32) << 20;

static __device__ __align__(256) unsigned char g_pool_select_scratch[kNoAllocScratchBytes];

namespace {

constexpr int kMaxDevices = 64;

int scratch_address(void** out) {
  static std::mutex mu;
  static void* addr[kMaxDevices] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return FVATTN_ERR_CUDA;
  std::lock_guard<std::mutex> lock(mu);
  if (!addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_pool_select_scratch) != cudaSuccess || !p) return FVATTN_ERR_CUDA;
    addr[dev] = p;
  }
  *out = addr[dev];
  return FVATTN_OK;
}

}  // namespace

extern "C" int fvattn_pool_select_noalloc(const fvattn_shape* shape, const void* q, const void* k,
                                          const fvattn_rope* rope, float top_p, int32_t k_min,
                                          const fvattn_blocks* out, fvattn_stream_t stream) {
  size_t need = 0;
  const int st = fvattn_workspace_size(shape, rope, &need);
  if (st != FVATTN_OK) return st;
  if (need > kNoAllocScratchBytes) return FVATTN_ERR_WORKSPACE;
  void* scratch = nullptr;
  const int sa = scratch_address(&scratch);
  if (sa != FVATTN_OK) return sa;
  return fvattn_pool_select(shape, q, k, rope, top_p, k_min, out, scratch, kNoAllocScratchBytes, stream);
}

extern "C" int fvattn_pool_select_noalloc_status(fvattn_stream_t stream, int32_t* status) {
  if (!status) return FVATTN_ERR_INVALID_ARG;
  void* scratch = nullptr;
  const int sa = scratch_address(&scratch);
  if (sa != FVATTN_OK) return sa;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(s) != cudaSuccess) return FVATTN_ERR_CUDA;
  int32_t v = 0;
  if (cudaMemcpy(&v, scratch, sizeof(v), cudaMemcpyDeviceToHost) != cudaSuccess) return FVATTN_ERR_CUDA;
  if (cudaMemset(scratch, 0, sizeof(v)) != cudaSuccess) return FVATTN_ERR_CUDA;
  *status = v;
  return FVATTN_OK;
}
