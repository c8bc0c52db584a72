// Host-side status plumbing shared by every libfl entry point.
#include <stdarg.h>
#include <string.h>

#include "fl_common.cuh"

namespace fl {

static thread_local char g_msg[512] = "";

void set_error(const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_msg, sizeof(g_msg), fmt, ap);
  va_end(ap);
}

fl_status fail(fl_status st, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_msg, sizeof(g_msg), fmt, ap);
  va_end(ap);
  return st;
}

fl_status cuda_fail(cudaError_t e, const char* what) {
  snprintf(g_msg, sizeof(g_msg), "%s: %s", what, cudaGetErrorString(e));
  return FL_ERR_CUDA;
}

int device_sm_count() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  static int cache[64] = {0};
  if (dev >= 0 && dev < 64 && cache[dev] > 0) return cache[dev];
  int n = 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  if (dev >= 0 && dev < 64) cache[dev] = n;
  return n;
}

}  // namespace fl

extern "C" const char* fl_status_string(int status) {
  switch (status) {
    case FL_OK: return "FL_OK";
    case FL_ERR_ARG: return "FL_ERR_ARG";
    case FL_ERR_SHAPE: return "FL_ERR_SHAPE";
    case FL_ERR_UNSUPPORTED: return "FL_ERR_UNSUPPORTED";
    case FL_ERR_ALIGN: return "FL_ERR_ALIGN";
    case FL_ERR_CUDA: return "FL_ERR_CUDA";
    case FL_ERR_WORKSPACE: return "FL_ERR_WORKSPACE";
    default: return "FL_ERR_UNKNOWN";
  }
}

extern "C" const char* fl_last_error(void) { return fl::g_msg; }

extern "C" int fl_version(void) { return 1; }
