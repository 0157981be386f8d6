// fa_static.cu -- fa_decode_run_static: the decode pass for callers that
// cannot allocate device memory.
//
// Some callers cannot call cudaMalloc (or any allocating routine) at the
// point where they run attention: code inside a region that must not touch
// the allocator (an allocator-free inference runtime, a plugin host that owns
// all device memory, a path that must not synchronise the device, which
// cudaMalloc/cudaFree may do).  For them this entry point takes no workspace
// argument: the scratch the kernels need (device-check word, boundary
// records, partial softmax states) lives in a file-scope
// __device__ array of fixed size, which every GPU that loads this library
// holds until the process exits.
#include <cuda_runtime.h>
#include <stdio.h>

#include <mutex>

#include "../../include/fadecode.h"

namespace fa {
size_t plan_zero_prefix_bytes(const fa_plan* plan);
void set_last_error(const char* text);
}

namespace {

// The scratch.  In host code the name below is only a stand-in for the
// device array: its device address is obtained with cudaGetSymbolAddress.
static __device__ __align__(256) unsigned char g_static_scratch[FA_STATIC_WORKSPACE_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_mutex;
void* g_scratch_ptr[kMaxDevices] = {};

fa_status cuda_error(const char* what, cudaError_t e) {
  char text[256];
  snprintf(text, sizeof(text), "%s: %s (%d)", what, cudaGetErrorString(e), static_cast<int>(e));
  fa::set_last_error(text);
  cudaGetLastError();
  return FA_ERR_CUDA;
}

// Device address of the scratch on the current device, looked up once per
// device (the first call on a device does this set-up).  The address is kept
// for the life of the process: after cudaDeviceReset the module may be loaded
// again elsewhere, so the static entry points are not supported after a reset.
fa_status scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_error("cudaGetDevice", e);
  if (dev < 0 || dev >= kMaxDevices) {
    fa::set_last_error("device ordinal beyond the static scratch table");
    return FA_ERR_UNSUPPORTED;
  }
  std::lock_guard<std::mutex> lock(g_mutex);
  if (g_scratch_ptr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_static_scratch);
    if (e != cudaSuccess) return cuda_error("cudaGetSymbolAddress", e);
    if (p == nullptr) {
      fa::set_last_error("cudaGetSymbolAddress returned a null address");
      return FA_ERR_CUDA;
    }
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return FA_OK;
}

}  // namespace

extern "C" fa_status fa_decode_run_static(const fa_plan* plan, const void* q, const void* k,
                                          const void* v, int64_t kv_rows,
                                          const int32_t* page_table, int32_t page_table_stride,
                                          const int32_t* kv_indptr, const float* k_scale,
                                          const float* v_scale, void* out, float* lse,
                                          void* stream) {
  if (plan == nullptr) return FA_ERR_INVALID_ARG;
  fa_plan_info_t info;
  fa_status st = fa_plan_get_info(plan, &info);
  if (st != FA_OK) return st;
  if (info.workspace_bytes > FA_STATIC_WORKSPACE_BYTES) {
    char text[256];
    snprintf(text, sizeof(text), "plan needs %zu bytes of scratch; the static scratch holds %u",
             info.workspace_bytes, static_cast<unsigned>(FA_STATIC_WORKSPACE_BYTES));
    fa::set_last_error(text);
    return FA_ERR_WORKSPACE_TOO_SMALL;
  }
  void* scratch = nullptr;
  st = scratch_address(&scratch);
  if (st != FA_OK) return st;
  // The device-check word must start at zero; the array keeps whatever the
  // previous call (or an aborted one) left there.
  cudaError_t e = cudaMemsetAsync(scratch, 0, fa::plan_zero_prefix_bytes(plan),
                                  static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_error("clearing the static scratch", e);
  return fa_decode_run(plan, q, k, v, kv_rows, page_table, page_table_stride, kv_indptr, k_scale,
                       v_scale, out, lse, scratch, FA_STATIC_WORKSPACE_BYTES, stream);
}

// Size of the scratch header that holds the device-check word (word 0), the
// first failed check (words 1..5) and the first wait that gave up (words
// 8..15); the same 256-byte header as a caller's workspace.
constexpr size_t kHeaderBytes = 256;

extern "C" fa_status fa_decode_status_static(uint32_t* flags, void* stream) {
  if (flags == nullptr) return FA_ERR_INVALID_ARG;
  void* scratch = nullptr;
  fa_status st = scratch_address(&scratch);
  if (st != FA_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint32_t h = 0;
  cudaError_t e = cudaMemcpyAsync(&h, scratch, sizeof(h), cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_error("fa_decode_status_static: read", e);
  *flags = h;
  if (h != 0) {
    e = cudaMemsetAsync(scratch, 0, kHeaderBytes, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return cuda_error("fa_decode_status_static: clear", e);
    return FA_ERR_DEVICE_CHECK;
  }
  return FA_OK;
}
