// Plane store packing ("FoQLens" landing page, progress table: the model is
// stored as one stack, a base with refinements, and any depth is read from
// the same copy without repacking).
//
// One thread per (row, 16-column word): it reads 16 int8 codes (one 16-byte
// load), forms u = code + 128, and writes the four plane words of those
// columns, plane k holding p_k = (u >> (6 - 2k)) & 3 of column j at bit
// (8 (j % 4) + 6 - 2k + 2 (j / 4)) mod 32. The thread of word 0 of each
// (row, group) also copies the row's scale into the block's scale area.
// Consecutive threads take consecutive words of a row, so loads and stores
// are coalesced. Bit-exact by construction (integer work only).
#include "fl_common.cuh"

namespace fl {

__global__ void __launch_bounds__(256) pack_planes_kernel(const int8_t* __restrict__ codes,
                                                          const float* __restrict__ scales, int out, int in,
                                                          uint8_t* __restrict__ store) {
  pdl_release();
  pdl_wait();
  const int G = in / 128;
  const long long words = (long long)out * (in / 16);
  for (long long idx = blockIdx.x * (long long)blockDim.x + threadIdx.x; idx < words;
       idx += (long long)gridDim.x * blockDim.x) {
    const int r = (int)(idx / (in / 16));
    const int cw = (int)(idx % (in / 16));  // 16-column word index within the row
    const int g = cw / 8, w = cw % 8;
    const uint4 raw = *reinterpret_cast<const uint4*>(codes + (size_t)r * in + 16 * cw);
    const uint32_t v[4] = {raw.x, raw.y, raw.z, raw.w};
    uint32_t pw[4] = {0, 0, 0, 0};
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      const uint32_t u = ((v[j >> 2] >> (8 * (j & 3))) + 128u) & 0xFFu;
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const uint32_t field = (u >> (6 - 2 * k)) & 3u;
        const int bit = (8 * (j % 4) + 6 - 2 * k + 2 * (j / 4)) & 31;
        pw[k] |= field << bit;
      }
    }
    const int blk = r / 64, rr = r % 64;
    uint8_t* base = store + (size_t)blk * 8448u * G;
#pragma unroll
    for (int k = 0; k < 4; ++k)
      *reinterpret_cast<uint32_t*>(base + 256u * G + 2048u * ((size_t)G * k + g) + 32u * rr + 4u * w) = pw[k];
    if (w == 0) *reinterpret_cast<float*>(base + 4u * (64u * g + rr)) = scales[(size_t)r * G + g];
  }
}

}  // namespace fl

extern "C" size_t fl_plane_store_bytes(int out, int in) {
  if (out <= 0 || in <= 0 || out % 64 || in % 128) return 0;
  return (size_t)(out / 64) * (size_t)(in / 128) * 8448u;
}

extern "C" fl_status fl_pack_planes(const int8_t* codes, const float* scales, int out, int in, uint8_t* store,
                                    void* stream) {
  using namespace fl;
  const char* what = "fl_pack_planes";
  if (!codes || !scales || !store) return fail(FL_ERR_ARG, "%s: NULL pointer argument", what);
  if (out <= 0 || in <= 0 || out % 64 || in % 128)
    return fail(FL_ERR_SHAPE, "%s: out=%d in=%d (need out %% 64 == 0, in %% 128 == 0)", what, out, in);
  if (!aligned16(codes) || !aligned16(store)) return fail(FL_ERR_ALIGN, "%s: codes/store not 16-byte aligned", what);
  if ((reinterpret_cast<uintptr_t>(scales) & 3u) != 0) return fail(FL_ERR_ALIGN, "%s: scales not 4-byte aligned", what);
  const int nsm = device_sm_count();
  if (nsm <= 0) return fail(FL_ERR_CUDA, "%s: no CUDA device", what);
  const long long words = (long long)out * (in / 16);
  long long blocks = (words + 255) / 256;
  if (blocks > (long long)nsm * 16) blocks = (long long)nsm * 16;
  FL_CHECK_CUDA(launch_pdl(pack_planes_kernel, dim3((unsigned)blocks), dim3(256), 0, static_cast<cudaStream_t>(stream),
                           1, codes, scales, out, in, store),
                "launch pack_planes");
  return FL_OK;
}
