// Plane store packing ("FoQLens" landing page, progress table: the model is
// stored as one stack, a base with refinements, and any depth is read from
// the same copy without repacking).
//
// One thread per (row, half of a 128-column group): it reads the half's 64 int8 codes (four
// 16-byte loads), forms u = code + 128 and builds, for each plane k, the four 32-bit words of
// those columns, plane k holding p_k = (u >> (6 - 2k)) & 3 of column j of a 16-column word at
// bit (8 (j % 4) + 6 - 2k + 2 (j / 4)) mod 32; each plane's four words leave in one 16-byte
// store. Threads are ordered half, then row, then group, then block: a warp covers 16 rows of
// one (block, group), so each plane store of the warp fills 512 contiguous bytes and the
// half-0 threads write the 16 rows' scales as 64 contiguous bytes. Bit-exact by construction
// (integer work only).
#include "fl_common.cuh"

namespace fl {

__global__ void __launch_bounds__(256) pack_planes_kernel(const int8_t* __restrict__ codes,
                                                          const float* __restrict__ scales, int out, int in,
                                                          uint8_t* __restrict__ store) {
  pdl_release();
  pdl_wait();
  const int G = in / 128;
  const long long items = (long long)out * G * 2;
  for (long long idx = blockIdx.x * (long long)blockDim.x + threadIdx.x; idx < items;
       idx += (long long)gridDim.x * blockDim.x) {
    const int h = (int)(idx & 1), rr = (int)((idx >> 1) & 63);
    const long long rest = idx >> 7;
    const int g = (int)(rest % G), blk = (int)(rest / G);
    const int r = 64 * blk + rr;
    const uint4* src = reinterpret_cast<const uint4*>(codes + (size_t)r * in + 128 * g + 64 * h);
    uint32_t pw[4][4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const uint4 raw = __ldg(src + q);
      const uint32_t v[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
      for (int k = 0; k < 4; ++k) pw[k][q] = 0u;
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const uint32_t u = ((v[j >> 2] >> (8 * (j & 3))) + 128u) & 0xFFu;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const uint32_t field = (u >> (6 - 2 * k)) & 3u;
          const int bit = (8 * (j % 4) + 6 - 2 * k + 2 * (j / 4)) & 31;
          pw[k][q] |= field << bit;
        }
      }
    }
    uint8_t* base = store + (size_t)blk * 8448u * G;
#pragma unroll
    for (int k = 0; k < 4; ++k)
      *reinterpret_cast<uint4*>(base + 256u * G + 2048u * ((size_t)G * k + g) + 32u * rr + 16u * h) =
          make_uint4(pw[k][0], pw[k][1], pw[k][2], pw[k][3]);
    if (h == 0) *reinterpret_cast<float*>(base + 4u * (64u * g + rr)) = scales[(size_t)r * G + g];
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
  const long long items = (long long)out * (in / 128) * 2;
  long long blocks = (items + 255) / 256;
  if (blocks > (long long)nsm * 16) blocks = (long long)nsm * 16;
  FL_CHECK_CUDA(launch_pdl(pack_planes_kernel, dim3((unsigned)blocks), dim3(256), 0, static_cast<cudaStream_t>(stream),
                           1, codes, scales, out, in, store),
                "launch pack_planes");
  return FL_OK;
}
