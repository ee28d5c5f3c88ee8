// noalloc.cu -- a forward entry point for callers that cannot allocate device
// memory.
//
// sigattn_fwd needs a caller-provided workspace (the work list of the ragged
// scheduler and a status word). Some callers have no way to provide one: code
// running where cudaMalloc is forbidden or unavailable (a host with a fixed
// device memory pool owned by someone else, a plugin that may only touch the
// tensors it is handed, a real-time path that must not allocate). For them,
// sigattn_fwd_noalloc uses a fixed scratch array that lives in this library's
// own device image instead.
//
// The array is a file-scope __device__ variable, so every GPU that loads the
// library holds SIGATTN_NOALLOC_SCRATCH_BYTES of it until the process exits.
// In host code its name only stands for the variable: the device address is
// obtained once per device with cudaGetSymbolAddress (with that device
// current) and passed to the kernels.
#include <cstdio>
#include <mutex>

#include "../../include/sigattn.h"
#include "common.cuh"

namespace sigattn {
void set_last_error(const char* msg);
int check_fwd_inputs(const void* q, const void* k, const void* v, const void* o, const int32_t* lengths, int B,
                     int H, int L, int d);
int report_cuda(cudaError_t e);
}

namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[SIGATTN_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mutex;
void* g_noalloc_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device (set up on the
// first call per device). Returns nullptr on failure.
void* scratch_address(cudaError_t* err) {
  int dev = 0;
  *err = cudaGetDevice(&dev);
  if (*err != cudaSuccess) return nullptr;
  if (dev < 0 || dev >= kMaxDevices) {
    *err = cudaErrorInvalidDevice;
    return nullptr;
  }
  std::lock_guard<std::mutex> lock(g_noalloc_mutex);
  if (g_noalloc_ptr[dev] == nullptr) {
    void* p = nullptr;
    *err = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (*err != cudaSuccess) return nullptr;
    g_noalloc_ptr[dev] = p;
  }
  return g_noalloc_ptr[dev];
}

}  // namespace

extern "C" int sigattn_fwd_noalloc(const void* q, const void* k, const void* v, void* o, const int32_t* lengths,
                                   int B, int H, int Lmax, int d, int32_t* status_out, void* stream) {
  // Every argument check comes first, so that a rejected call leaves the
  // shared array and the stream untouched.
  int st = sigattn::check_fwd_inputs(q, k, v, o, lengths, B, H, Lmax, d);
  if (st != SIGATTN_OK) return st;
  if (status_out != nullptr && (reinterpret_cast<uintptr_t>(status_out) & 3u) != 0) return SIGATTN_ERR_INVALID_ARG;
  const size_t need = sigattn_workspace_size(B, H, Lmax, d);
  if (need > static_cast<size_t>(SIGATTN_NOALLOC_SCRATCH_BYTES)) {
    // B * H * ceil(Lmax / 128) work items do not fit the fixed scratch array.
    char msg[160];
    snprintf(msg, sizeof(msg), "sigattn_fwd_noalloc: needs %zu bytes of scratch, the fixed array holds %d", need,
             SIGATTN_NOALLOC_SCRATCH_BYTES);
    sigattn::set_last_error(msg);
    return SIGATTN_ERR_UNSUPPORTED;
  }
  cudaError_t err = cudaSuccess;
  void* scratch = scratch_address(&err);
  if (scratch == nullptr) return sigattn::report_cuda(err);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // The array keeps whatever the previous call left; the status words must
  // start at zero for this call.
  st = sigattn::report_cuda(cudaMemsetAsync(scratch, 0, 2 * sizeof(int32_t), s));
  if (st != SIGATTN_OK) return st;
  st = sigattn_fwd(q, k, v, o, lengths, B, H, Lmax, d, scratch, SIGATTN_NOALLOC_SCRATCH_BYTES, stream);
  if (st != SIGATTN_OK || status_out == nullptr) return st;
  return sigattn::report_cuda(cudaMemcpyAsync(status_out, scratch, sizeof(int32_t), cudaMemcpyDeviceToDevice, s));
}
