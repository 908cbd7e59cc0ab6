// An allocation-free form of specopd_tv_overlap_e2e.
//
// Some callers cannot hand the library a workspace: their device memory is
// owned by another allocator they may not bypass, or their hot loop must not
// call cudaMalloc/cudaFree because those calls can stall the whole device.
// For them the scratch of the fused overlap pass lives in a fixed array in
// this file, loaded with the library on every GPU that loads it and kept until
// the process exits.  The caller still passes inputs and outputs.
#include <mutex>

#include "internal.h"

namespace {

constexpr size_t kStaticScratchBytes = SPECOPD_STATIC_SCRATCH_BYTES;
constexpr int kMaxDevices = 64;

__device__ __align__(256) unsigned char g_overlap_scratch[kStaticScratchBytes];

// Device address of g_overlap_scratch, looked up once per device.
std::mutex g_mutex;
void* g_scratch_ptr[kMaxDevices] = {};

int scratch_for_current_device(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return SPECOPD_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mutex);
  if (!g_scratch_ptr[dev]) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_overlap_scratch) != cudaSuccess || !ptr) return SPECOPD_ERR_CUDA;
    g_scratch_ptr[dev] = ptr;
  }
  *out = g_scratch_ptr[dev];
  return SPECOPD_OK;
}

}  // namespace

extern "C" {

int specopd_tv_overlap_e2e_static(const void* draft, const void* teacher, specopd_dtype dtype, int64_t rows,
                                  int64_t V, int64_t ld_draft, int64_t ld_teacher, int64_t num_branches, int W,
                                  double count, float* alpha, float* loss, float* grad_draft, int64_t ld_grad,
                                  int32_t* status, specopd_stream_t stream) {
  // the regular entry point's checks first, so a bad call reports what is wrong with it
  const int c = specopd::check_overlap_e2e_args(draft, teacher, dtype, rows, V, ld_draft, ld_teacher, num_branches,
                                                W, count, alpha, loss, grad_draft, ld_grad, status);
  if (c != SPECOPD_OK) return c;
  if (rows == 0)  // nothing to score: no scratch needed (the loss is set to 0)
    return specopd_tv_overlap_e2e(draft, teacher, dtype, rows, V, ld_draft, ld_teacher, num_branches, W, count,
                                  alpha, loss, grad_draft, ld_grad, nullptr, 0, status, stream);
  if (specopd_overlap_workspace_bytes(rows, V, num_branches) > kStaticScratchBytes) return SPECOPD_ERR_WORKSPACE;
  void* scratch = nullptr;
  const int s = scratch_for_current_device(&scratch);
  if (s != SPECOPD_OK) return s;
  return specopd_tv_overlap_e2e(draft, teacher, dtype, rows, V, ld_draft, ld_teacher, num_branches, W, count,
                                alpha, loss, grad_draft, ld_grad, scratch, kStaticScratchBytes, status, stream);
}

}  // extern "C"
