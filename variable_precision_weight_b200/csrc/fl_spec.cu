// Verified speculation ("Precision on Demand: Escalating Weight Bits at Uncertain Decoding
// Steps in a Small Local Model", abstract: a low-precision draft verified at 8 bits reaches
// the 8-bit model's output, counted in the same weight-byte cost model).
//
// Greedy, over a window of k decode steps: step t's draft token is the argmax of its D4
// logits, its verified token the argmax of its D8 logits, both as the fused gate writes
// them (column 0 of a top-2 row; ties to the lower index). The D8 logits of the whole
// window come from one residual pass at batch k over the drafts' D4 outputs, so the low
// planes are read once per window. The window accepts the longest prefix of steps whose
// tokens agree and emits the verified tokens up to and including the first disagreement:
// emitted = accepted + 1, or k when all agree. One warp compares the k pairs and takes the
// first disagreement from a ballot.
#include "fl_common.cuh"

namespace fl {
namespace spec {

__global__ void __launch_bounds__(32) accept_kernel(const int32_t* __restrict__ draft,
                                                    const int32_t* __restrict__ verified, int k,
                                                    int32_t* __restrict__ result, int32_t* __restrict__ totals) {
  pdl_release();
  pdl_wait();
  const int lane = threadIdx.x;
  const bool miss = lane < k && draft[2 * lane] != verified[2 * lane];
  const unsigned m = __ballot_sync(0xffffffffu, miss);
  const int accepted = m ? __ffs((int)m) - 1 : k;
  const int emitted = accepted < k ? accepted + 1 : k;
  if (lane == 0) {
    result[0] = accepted;
    result[1] = emitted;
    if (totals) {
      atomicAdd(totals, accepted);
      atomicAdd(totals + 1, emitted);
    }
  }
}

}  // namespace spec
}  // namespace fl

extern "C" fl_status fl_spec_accept(const int32_t* draft_top2, const int32_t* verified_top2, int k, int32_t* result,
                                    int32_t* totals, void* stream) {
  using namespace fl;
  const char* what = "fl_spec_accept";
  if (!draft_top2 || !verified_top2 || !result) return fail(FL_ERR_ARG, "%s: NULL pointer argument", what);
  if (k < 1 || k > FL_MAX_BATCH) return fail(FL_ERR_SHAPE, "%s: k=%d (1..%d)", what, k, FL_MAX_BATCH);
  const uintptr_t bad = reinterpret_cast<uintptr_t>(draft_top2) | reinterpret_cast<uintptr_t>(verified_top2) |
                        reinterpret_cast<uintptr_t>(result) | reinterpret_cast<uintptr_t>(totals);
  if (bad & 3u) return fail(FL_ERR_ALIGN, "%s: pointers must be 4-byte aligned", what);
  FL_CHECK_CUDA(launch_pdl(spec::accept_kernel, dim3(1), dim3(32), 0, static_cast<cudaStream_t>(stream), 1,
                           draft_top2, verified_top2, k, result, totals),
                "launch spec_accept");
  return FL_OK;
}
