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
    case FL_ERR_TIMEOUT: return "FL_ERR_TIMEOUT";
    default: return "FL_ERR_UNKNOWN";
  }
}

extern "C" const char* fl_last_error(void) { return fl::g_msg; }

extern "C" int fl_version(void) { return 1; }

namespace fl {
namespace gemv {
int take_device_error();
}
namespace kq {
int take_device_error();
}
namespace tc {
int take_device_error();
}
int take_gate_error();
}  // namespace fl

extern "C" fl_status fl_device_status(void) {
  using namespace fl;
  FL_CHECK_CUDA(cudaDeviceSynchronize(), "fl_device_status: cudaDeviceSynchronize");
  const int g = gemv::take_device_error(), k = kq::take_device_error(), t = take_gate_error();
  const int c = tc::take_device_error();
  if (g < 0 || k < 0 || t < 0 || c < 0) return fail(FL_ERR_CUDA, "fl_device_status: reading the error words failed");
  if (g == 0 && k == 0 && t == 0 && c == 0) return FL_OK;
  auto what = [](int c) {
    return c == 1 ? "a producer's wait for a free stage" : c == 2 ? "a consumer's wait for a full stage"
         : c == 3 ? "the wait for staged activations" : c == 4 ? "the self-test wait" : "a wait";
  };
  if (g == 5)
    return fail(FL_ERR_ARG, "plane GEMV: a listed block index was out of range; that unit was skipped");
  if (g) return fail(FL_ERR_TIMEOUT, "plane GEMV: %s ran out (code %d); its outputs are not valid", what(g), g);
  if (k) return fail(FL_ERR_TIMEOUT, "K-quant GEMV: %s ran out (code %d); its outputs are not valid", what(k), k);
  if (c) {
    const char* cw = c == 1 ? "the producer's wait for a free stage" : c == 2 ? "the MMA issuer's wait for codes or a free accumulator"
                   : c == 3 ? "a converter's wait for a full stage or a free code buffer" : "an epilogue wait for the MMAs";
    return fail(FL_ERR_TIMEOUT, "tensor-core GEMV: %s ran out (code %d); its outputs are not valid", cw, c);
  }
  return fail(FL_ERR_TIMEOUT, "logit gate: the wait for the cluster's partials ran out; its outputs are NaN");
}
