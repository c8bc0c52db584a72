// The read split across devices: a layer's 64-row blocks partitioned over ranks by the bytes
// their depths read, and the logit gate over a vocabulary that is split with them.
//
// One decode step reads every block of every layer once ("FoQLens" landing page, progress
// table: each block read to its own depth from the one stored copy). Blocks are independent,
// so ranks can each read a contiguous range of every layer's blocks and exchange outputs; the
// work of a block is the bytes its depth reads, 256 G + 2048 G d/2 for G = in / 128 column
// groups, so ranges are balanced by those bytes, not by block count.
//
// The gate ("Precision on Demand", abstract: entropy and top-two margin of the low-precision
// output distribution) needs the whole row of logits. Split over ranks, each rank reduces its
// own share to a partial (max m, S = sum e^(z - m), T = sum (z - m) e^(z - m), the two largest
// values with their global indices); partials merge exactly up to fp32 rounding by rescaling
// S and T to the common maximum. After one exchange of the partials every rank merges the same
// records in the same order, so every rank takes the same escalation decision.
#include <algorithm>

#include "fl_gate_merge.cuh"

namespace fl {

// defined with the whole-row gate kernel: the same cluster reduction, storing the partial
cudaError_t gate_partial_launch(const float* logits, int vocab, int batch, int index_base, GateRec* partial,
                                cudaStream_t st);

namespace shard {

// One warp per row: partials [nparts][batch] merged in part order (lane l takes parts l, l + 32,
// ...), then across lanes; the row's outputs as the gate defines them.
__global__ void __launch_bounds__(32) gate_merge_kernel(const GateRec* __restrict__ parts, int nparts, int batch,
                                                        float tau_h, float tau_m, float* __restrict__ entropy,
                                                        float* __restrict__ margin, int32_t* __restrict__ top2,
                                                        uint8_t* __restrict__ escalate) {
  pdl_release();
  pdl_wait();
  const int row = blockIdx.x, lane = threadIdx.x;
  GateRec r = empty_rec();
  for (int q = lane; q < nparts; q += 32) r = merge2(r, parts[(size_t)q * batch + row]);
  r = warp_merge(r);
  if (lane == 0) gate_outputs(r, tau_h, tau_m, entropy + row, margin + row, top2 + 2 * row, escalate + row);
}

}  // namespace shard
}  // namespace fl

using namespace fl;

static_assert(sizeof(fl_gate_partial) == sizeof(GateRec), "fl_gate_partial mirrors the kernels' partial record");

extern "C" fl_status fl_shard_blocks(const uint8_t* levels, int nblocks, int in, int nranks, int* first_block) {
  const char* what = "fl_shard_blocks";
  if (!first_block || (nblocks > 0 && !levels)) return fail(FL_ERR_ARG, "%s: NULL pointer argument", what);
  if (nblocks < 0 || in <= 0 || in % 128 || nranks < 1)
    return fail(FL_ERR_SHAPE, "%s: nblocks=%d in=%d nranks=%d", what, nblocks, in, nranks);
  const double G = in / 128;
  double total = 0;
  for (int b = 0; b < nblocks; ++b) {
    const int d = std::min((int)levels[b], 4);
    total += d ? 256.0 * G + 2048.0 * G * d : 0.0;
  }
  // rank r starts at the first block whose preceding bytes reach r / nranks of the total
  // (the block is assigned to the range holding its midpoint); ranges are contiguous, may be
  // empty, and cover every block
  first_block[0] = 0;
  double acc = 0;
  int r = 1;
  for (int b = 0; b < nblocks && r < nranks; ++b) {
    const int d = std::min((int)levels[b], 4);
    const double w = d ? 256.0 * G + 2048.0 * G * d : 0.0;
    while (r < nranks && acc + 0.5 * w >= total * r / nranks && (total > 0)) first_block[r++] = b;
    acc += w;
  }
  if (total == 0)  // nothing to read: equal block counts
    for (; r < nranks; ++r) first_block[r] = (int)((long long)nblocks * r / nranks);
  for (; r < nranks; ++r) first_block[r] = nblocks;
  first_block[nranks] = nblocks;
  return FL_OK;
}

extern "C" fl_status fl_logit_gate_partial(const float* logits, int vocab, int batch, int index_base,
                                           fl_gate_partial* partial, void* stream) {
  const char* what = "fl_logit_gate_partial";
  if (!logits || !partial) return fail(FL_ERR_ARG, "%s: NULL pointer argument", what);
  if (batch < 1 || batch > FL_MAX_BATCH) return fail(FL_ERR_SHAPE, "%s: batch=%d (1..16)", what, batch);
  if (vocab < 4 || vocab % 4 || index_base < 0 || (long long)index_base + vocab > (1 << 24))
    return fail(FL_ERR_SHAPE, "%s: vocab=%d index_base=%d (vocab %% 4 == 0, indices below 2^24)", what, vocab,
                index_base);
  if (!aligned16(logits) || !aligned16(partial))
    return fail(FL_ERR_ALIGN, "%s: logits and partial must be 16-byte aligned", what);
  FL_CHECK_CUDA(gate_partial_launch(logits, vocab, batch, index_base, reinterpret_cast<GateRec*>(partial),
                                    static_cast<cudaStream_t>(stream)),
                "launch gate_partial");
  return FL_OK;
}

extern "C" fl_status fl_logit_gate_merge(const fl_gate_partial* partials, int nparts, int batch, float tau_h,
                                         float tau_m, float* entropy, float* margin, int32_t* top2,
                                         uint8_t* escalate, void* stream) {
  const char* what = "fl_logit_gate_merge";
  if (!partials || !entropy || !margin || !top2 || !escalate) return fail(FL_ERR_ARG, "%s: NULL pointer argument", what);
  if (batch < 1 || batch > FL_MAX_BATCH) return fail(FL_ERR_SHAPE, "%s: batch=%d (1..16)", what, batch);
  if (nparts < 1 || nparts > 4096) return fail(FL_ERR_ARG, "%s: nparts=%d (1..4096)", what, nparts);
  if (!aligned16(partials)) return fail(FL_ERR_ALIGN, "%s: partials not 16-byte aligned", what);
  if ((reinterpret_cast<uintptr_t>(entropy) | reinterpret_cast<uintptr_t>(margin) | reinterpret_cast<uintptr_t>(top2)) &
      3u)
    return fail(FL_ERR_ALIGN, "%s: entropy, margin and top2 must be 4-byte aligned", what);
  FL_CHECK_CUDA(launch_pdl(shard::gate_merge_kernel, dim3((unsigned)batch), dim3(32), 0,
                           static_cast<cudaStream_t>(stream), 1, reinterpret_cast<const GateRec*>(partials), nparts,
                           batch, tau_h, tau_m, entropy, margin, top2, escalate),
                "launch gate_merge");
  return FL_OK;
}
