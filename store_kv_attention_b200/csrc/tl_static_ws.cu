// tl_storeh_attn_decode_static_ws: the decode entry point for callers that
// cannot allocate device memory.
//
// Some callers cannot call cudaMalloc at all: code that runs inside a CUDA
// stream-ordered region it does not own, plug-ins hosted by a process whose
// allocator they must not touch, or environments where every device
// allocation is made once, up front, by someone else.  This entry point runs
// the same kernels as tl_storeh_attn_decode, but its scratch (the decode
// workspace) is a fixed array compiled into this library instead of a buffer
// the caller passes in.
//
// The array is a file-scope __device__ variable, so every GPU that loads the
// library holds kStaticScratchBytes of device memory until the process exits.
// In host code its name only stands in for the symbol; the device address is
// looked up with cudaGetSymbolAddress, on the device and context current at the
// call, on every call (a lookup costs far less than the launches it precedes),
// and then passed to the kernels like any other workspace pointer.  Looking it up
// each time keeps the address right after cudaDeviceReset or when another
// context is current.  With CUDA's lazy module loading the array is only
// created by the first lookup on a device, so that first call is where an
// out-of-memory condition shows up (as TL_ERR_CUDA).
#include "tl_internal.cuh"

namespace {

constexpr size_t kStaticScratchBytes = 32u << 20;  // 32 MiB

__device__ __align__(256) unsigned char g_decode_scratch[kStaticScratchBytes];

// Device address of the scratch array in the current context.
cudaError_t scratch_address(void** out) {
  void* p = nullptr;
  cudaError_t e = cudaGetSymbolAddress(&p, g_decode_scratch);
  if (e != cudaSuccess) return e;
  *out = p;
  return cudaSuccess;
}

}  // namespace

extern "C" tl_status tl_storeh_attn_decode_static_ws(const tl_storeh_desc* desc, tl_storeh_cache cache, int32_t iter,
                                                     const int32_t* loops, const int32_t* ctx_len, const void* h_new,
                                                     const void* W_q, const void* W_k, const void* W_v, float* out,
                                                     const float* residual, float threshold, uint8_t* abort_flags,
                                                     int32_t* first_abort_iter, float* norms_out, int32_t n_lanes,
                                                     uint32_t* status_out, tl_stream_t stream) {
  // Size check first, so an oversized request fails before anything touches the device.
  size_t need = 0;
  tl_status st = tl_storeh_workspace_bytes(desc, n_lanes, &need);
  if (st != TL_OK) return st;
  if (need > kStaticScratchBytes) {
    return tl::set_error(TL_ERR_CAPACITY, "decode scratch of %zu bytes exceeds the built-in %zu bytes", need,
                         kStaticScratchBytes);
  }
  void* ws = nullptr;
  cudaError_t e = scratch_address(&ws);
  if (e != cudaSuccess) return tl::set_error(TL_ERR_CUDA, "cudaGetSymbolAddress: %s", cudaGetErrorString(e));
  cudaStream_t cs = (cudaStream_t)stream;
  // The array keeps the previous call's contents; only the status word must start at zero.
  e = cudaMemsetAsync(ws, 0, 256, cs);
  if (e != cudaSuccess) return tl::set_error(TL_ERR_CUDA, "clearing the status word: %s", cudaGetErrorString(e));
  st = tl_storeh_attn_decode(desc, cache, iter, loops, ctx_len, h_new, W_q, W_k, W_v, out, residual, threshold,
                             abort_flags, first_abort_iter, norms_out, ws, kStaticScratchBytes, n_lanes, stream);
  if (st != TL_OK) return st;
  if (status_out) {
    e = cudaMemcpyAsync(status_out, ws, sizeof(uint32_t), cudaMemcpyDeviceToDevice, cs);
    if (e != cudaSuccess) return tl::set_error(TL_ERR_CUDA, "copying the status word: %s", cudaGetErrorString(e));
  }
  return TL_OK;
}
