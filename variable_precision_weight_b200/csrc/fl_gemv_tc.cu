// Depth GEMV / residual on the fifth-generation tensor cores (tcgen05) for large batches.
//
// What it computes is exactly what fl_gemv.cu computes ("FoQLens" landing page, progress
// table: every block of rows read to its own depth from the one stored copy, here at the
// landing page's own decode batch of 32; "Precision on Demand", abstract: the residual from
// the low planes):
//   depth mode     y[t][r]  = sum_c s[r][c/128] (u_d - 128 + c_d) x[t][c]
//   residual mode  y[t][r] += sum_c s[r][c/128] ((u_b - u_a) + c_b - c_a) x[t][c]
// with the same per-group fixed-point activations (fl_common.cuh: four int8 digits).
//
// How (B200): one persistent CTA per SM, 12 warps.
//  * Unit = (column slice, pair of 64-row blocks) = one M = 128 tile; the two blocks keep their
//    own depths. Each CTA owns a contiguous, cost-balanced range of units.
//  * Two producer threads (one per block of the pair) stream the planes each block's depth
//    needs into a shared-memory ring of four to six stages (as many as the column slices'
//    digits leave room for); a stage holds as many 128-column groups as the deeper block
//    allows, one 1-D bulk copy per plane and block (mbarrier completion).
//  * Warps 4-7 (the four TMEM lane quarters, one row per thread) turn the plane words into u8
//    codes (one AND/OR per plane, one rotate per four columns) and write them straight into
//    tensor memory with tcgen05.st: the A operand of the MMA lives in TMEM (four buffers).
//  * Warp 1 (one lane) issues four tcgen05.mma.kind::i8 (M 128, N = 4 batch rounded up to 16,
//    K 32) per group: A from TMEM, B = the activation digits of the group, resident in shared
//    memory in the no-swizzle K-major core-matrix layout for the CTA's column slices, D int32
//    in TMEM (three buffers), and commits to two mbarriers (codes consumed, sums ready).
//  * The digits are built once per call, for the whole activation, by a small kernel that runs
//    first (programmatic launch) and writes them to the workspace in that layout; each CTA
//    brings its column slices' digits in with bulk copies while the weights start to stream.
//  * Warps 8-15 (two per TMEM lane quarter, each half of the batch rows) read D with
//    tcgen05.ld (one row per thread), join each batch row's two digit pairs, apply the group
//    scale (passed on by the converters through a four-slot ring) and the constant part, and
//    accumulate the row's outputs in registers.
//  * Column slices: partials to the caller's workspace; the last CTA to finish a pair of
//    blocks (acquire-release ticket) adds the slices in order, after its own units, with all
//    twelve warps and 16-byte loads. No CTA waits on another; every wait is bounded; TMEM is
//    freed on every exit path once the CTA's MMAs are complete.
#include <algorithm>

#include "fl_common.cuh"

namespace fl {
namespace tc {

constexpr int kThreads = 512;
constexpr int kMinStages = 4, kMaxStages = 6;  // stages per launch: what the digits leave room for
constexpr int kBlockTile = 2 * 8448;        // one block's share of a stage: two groups at D8 (scales + 4 planes)
constexpr int kStageBytes = 2 * kBlockTile;  // both blocks of a pair
constexpr int kMaxSlots = 4;                 // column slices one CTA may touch
constexpr int kLevelCache = 1024;            // units per CTA
constexpr int kMaxCtas = 1024;
constexpr int kTmemCols = 512;
constexpr int kNA = 4, kND = 3, kNS = 8;     // A (code) buffers, D (sum) buffers, scale-ring slots
constexpr uint32_t kColA = 0, kColD = 128;   // A buffer i at column 32 i, D buffer i at 128 + 128 i
constexpr int kSmemLimit = 232448 - 9216;    // opt-in shared memory per block, less static use
constexpr int kDigitBudget = kSmemLimit - kMinStages * kStageBytes - 1024;
constexpr int kMinBatch = 9;                 // batches from here to FL_MAX_GEMV_BATCH take this path
constexpr int kEpiWarps = 8;                 // warps 8-15

__host__ __device__ constexpr int n_cols(int batch) { return (4 * batch + 15) / 16 * 16; }

// Column slice j of `slices` over G groups: groups [slice_first(j), slice_first(j + 1)), the
// slices as equal as whole groups allow (widths differ by one at most).
__host__ __device__ constexpr int slice_first(int j, int G, int slices) { return (int)((long long)j * G / slices); }

struct Args {
  const uint8_t* store;
  const uint8_t* lv_from;
  const uint8_t* lv_to;
  const uint16_t* x;
  float* y;
  float* partial;     // [slices][npair][batch][128] when slices > 1
  uint32_t* tickets;  // [npair] when slices > 1
  const uint8_t* dig; // workspace: digits [G][N / 8][8 K-cores x 128 B]
  const float4* gct;  // workspace: [G][batch] (2^(16 - sigma), 2^-sigma, 2^-sigma sum v, 0)
  int nblk, npair, G, batch, N, mode, slices, slice_groups;
  int ns;    // stages of the ring (kMinStages .. kMaxStages)
  int ncta;
  int cta_begin[kMaxCtas + 1];  // unit u = slice * npair + pair
};

__device__ int g_error;  // set when a bounded wait runs out (never expected)

struct Slot {
  int j, u0, u1, p0;   // slice, units [u0, u1) of the CTA's range (relative), first pair
  int ng, gfirst;      // groups of the slice, first group of the slice in the row
  uint32_t dig;        // smem: digits [group][N / 8][8 K-cores x 128 B]
  uint32_t gc;         // smem: float4 [ng][batch] = (2^(16 - sigma), 2^-sigma, 2^-sigma sum v, 0)
};

// ---------------------------------------------------------------- tcgen05 wrappers
__device__ __forceinline__ void fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]),
      "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]),
      "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]),
      "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&v)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,"
      "%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]), "=r"(v[8]),
        "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15]), "=r"(v[16]),
        "=r"(v[17]), "=r"(v[18]), "=r"(v[19]), "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]), "=r"(v[24]),
        "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]), "=r"(v[31])
      : "r"(taddr));
}

// Shared-memory matrix descriptor, no swizzle, K-major: 8-row x 16-byte core matrices, the two
// K-adjacent ones of a K = 32 step 128 bytes apart (leading offset), 8-row groups 1024 bytes
// apart (stride offset); descriptor version 1.
__device__ __forceinline__ uint64_t kmajor_desc(uint32_t saddr) {
  return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)(128u >> 4) << 16) | ((uint64_t)(1024u >> 4) << 32) |
         (1ull << 46);
}

// Instruction descriptor of kind::i8: D s32, A u8, B s8, both K-major, N, M = 128.
__host__ __device__ constexpr uint32_t idesc_i8(int n) {
  return (2u << 4) | (0u << 7) | (1u << 10) | ((uint32_t)(n >> 3) << 17) | ((128u >> 4) << 24);
}

__device__ __forceinline__ void mma_i8(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc, bool acc) {
  asm volatile(
      "{ .reg .pred p; setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], [%1], %2, %3, p; }" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"((uint32_t)acc)
      : "memory");
}

__device__ __forceinline__ void mma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ void named_bar(int id, int n) { asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory"); }

__device__ __forceinline__ uint32_t atom_add_acq_rel(uint32_t* p, uint32_t v) {
  uint32_t old;
  asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
  return old;
}

// Mask selecting plane k's fields for column set i (rotl(0x03030303, 6-2k+2i)).
__host__ __device__ constexpr uint32_t plane_mask(int k, int i) {
  return (((6 - 2 * k + 2 * i) & 7) == 0)
             ? 0x03030303u
             : ((0x03030303u << ((6 - 2 * k + 2 * i) & 7)) | (0x03030303u >> (32 - ((6 - 2 * k + 2 * i) & 7))));
}

// The u8 codes of one row for one 128-column group: register 4w + i holds columns 16w + 4i ..
// 16w + 4i + 3 (byte order), i.e. TMEM column 4w + i of the A operand holds K elements
// 4 (4w + i) .. + 3, the natural column order the activation digits use.
template <int K0, int NP>
__device__ __forceinline__ void row_codes(uint32_t rowp, uint32_t pstride, uint32_t (&r)[32]) {
  uint4 W[NP][2];
#pragma unroll
  for (int kk = 0; kk < NP; ++kk) {
    asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(W[kk][0].x), "=r"(W[kk][0].y), "=r"(W[kk][0].z), "=r"(W[kk][0].w)
                 : "r"(rowp + pstride * kk));
    asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(W[kk][1].x), "=r"(W[kk][1].y), "=r"(W[kk][1].z), "=r"(W[kk][1].w)
                 : "r"(rowp + pstride * kk + 16u));
  }
#pragma unroll
  for (int w = 0; w < 8; ++w) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      uint32_t v = 0;
#pragma unroll
      for (int kk = 0; kk < NP; ++kk) {
        const uint4& q = W[kk][w >> 2];
        const uint32_t word = (w & 3) == 0 ? q.x : (w & 3) == 1 ? q.y : (w & 3) == 2 ? q.z : q.w;
        v |= word & plane_mask(K0 + kk, i);
      }
      r[4 * w + i] = (i == 0) ? v : rotr32(v, 2 * i);
    }
  }
}

// rowp: the row's 32 bytes of the first plane read; pstride: bytes between planes in the stage.
__device__ __forceinline__ void codes_dispatch(int k0, int np, uint32_t rowp, uint32_t pstride, uint32_t (&r)[32]) {
  switch (k0 * 8 + np) {
    case 0 * 8 + 1: row_codes<0, 1>(rowp, pstride, r); break;
    case 0 * 8 + 2: row_codes<0, 2>(rowp, pstride, r); break;
    case 0 * 8 + 3: row_codes<0, 3>(rowp, pstride, r); break;
    case 0 * 8 + 4: row_codes<0, 4>(rowp, pstride, r); break;
    case 1 * 8 + 1: row_codes<1, 1>(rowp, pstride, r); break;
    case 1 * 8 + 2: row_codes<1, 2>(rowp, pstride, r); break;
    case 1 * 8 + 3: row_codes<1, 3>(rowp, pstride, r); break;
    case 2 * 8 + 1: row_codes<2, 1>(rowp, pstride, r); break;
    case 2 * 8 + 2: row_codes<2, 2>(rowp, pstride, r); break;
    case 3 * 8 + 1: row_codes<3, 1>(rowp, pstride, r); break;
    default:
#pragma unroll
      for (int j = 0; j < 32; ++j) r[j] = 0u;
  }
}

// c_b - c_a with c_0 = 128: the constant part of the read of planes [k0, k0 + np).
__device__ __forceinline__ float cfac_of(int k0, int np) {
  const int b = 2 * (k0 + np), a = 2 * k0;
  const int cb2 = (1 << (8 - b)) - 1;
  const int ca2 = (a == 0) ? 256 : (1 << (8 - a)) - 1;
  return 0.5f * (float)(cb2 - ca2);
}

// Groups per stage for a pair whose deeper block reads np planes: 7, 3, 2, 2 for 1-4 planes.
__device__ __forceinline__ int stage_groups(int np) { return np == 0 ? 8 : kBlockTile / (256 + 2048 * np); }

// Plane range [k0, k0 + np) read for block b, packed as k0 << 4 | np (0: nothing to read).
__device__ __forceinline__ int plane_range(const Args& a, int b) {
  if (b >= a.nblk) return 0;
  const int lf = min((int)__ldg(a.lv_from + b), 4);
  if (a.mode == 0) return lf;
  const int lt = min((int)__ldg(a.lv_to + b), 4);
  return (lf << 4) | max(0, lt - lf);
}

// The activation digits of one call (fl_common.cuh), in the layout the MMAs read: item = (group
// g, batch row b), one warp per item; digit row n = 4 b + k of group g at
// dig + g N 128 + (n / 8) 1024 + (K column / 16) 128 + (n % 8) 16 + K column % 16.
__global__ void __launch_bounds__(256) tc_digits_kernel(const uint16_t* x, int G, int batch, int N, uint8_t* dig,
                                                         float4* gct) {
  pdl_release();
  pdl_wait();  // x may come from the previous kernel
  const int lane = threadIdx.x & 31;
  const int it = blockIdx.x * 8 + (threadIdx.x >> 5);
  if (it >= G * batch) return;
  const int g = it / batch, b = it % batch;
  const uint2 raw = __ldg(reinterpret_cast<const uint2*>(x + (size_t)b * G * 128 + 128 * g + 4 * lane));
  const float f[4] = {__uint_as_float(raw.x << 16), __uint_as_float(raw.x & 0xFFFF0000u),
                      __uint_as_float(raw.y << 16), __uint_as_float(raw.y & 0xFFFF0000u)};
  uint32_t dw[4];
  int2 part;
  const int sigma = split_digits(f, dw, part);
  uint8_t* gb = dig + (size_t)g * N * 128 + (lane >> 2) * 128 + 4 * (lane & 3);
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int n = 4 * b + k;
    *reinterpret_cast<uint32_t*>(gb + (n >> 3) * 1024 + (n & 7) * 16) = dw[k];
  }
  part.x = __reduce_add_sync(0xffffffffu, part.x);
  part.y = __reduce_add_sync(0xffffffffu, part.y);
  if (lane == 0)
    gct[(size_t)g * batch + b] = make_float4(ldexpf(1.0f, 16 - sigma), ldexpf(1.0f, -sigma),
                                             ldexpf(fmaf(65536.f, (float)part.x, (float)part.y), -sigma), 0.f);
}

enum : int { kBarEpi = 1 };

// NB: batch rows in chunks of 8 (one tcgen05.ld of 32 columns = 8 batch rows x 4 digits); each
// of the two epilogue warps of a lane quarter takes NH = ceil(NB / 2) chunks at most.
template <int NB>
__global__ void __launch_bounds__(kThreads, 1) tc_gemv_kernel(const __grid_constant__ Args a) {
  extern __shared__ __align__(1024) uint8_t smem[];
  __shared__ __align__(8) uint64_t full_bar[kMaxStages], empty_bar[kMaxStages];
  __shared__ __align__(8) uint64_t afull[kNA], afree[kNA], dfull[kND], dfree[kND], sfull[kNS];
  __shared__ __align__(8) uint64_t lv_ready, dig_ready;  // level cache / activation digits built
  __shared__ Slot slots[kMaxSlots];
  __shared__ uint16_t lvc[kLevelCache];
  __shared__ uint16_t won[kLevelCache];  // pairs whose slices this CTA adds up at the end
  __shared__ float scl[kNS][128];        // group scale of each row, ring of eight groups
  __shared__ uint32_t s_tmem;
  __shared__ int s_nslots, s_nwon;

  pdl_release();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int u_begin = a.cta_begin[blockIdx.x], u_end = a.cta_begin[blockIdx.x + 1];
  if (u_begin >= u_end) return;
  const int nunits = u_end - u_begin;

  if (threadIdx.x == 0) {
    for (int s = 0; s < a.ns; ++s) {
      mbar_init(&full_bar[s], 2);  // the two producers' arrivals (and their bytes)
      mbar_init(&empty_bar[s], 4);
    }
    for (int b = 0; b < kNA; ++b) {
      mbar_init(&afull[b], 4);
      mbar_init(&afree[b], 1);
    }
    for (int b = 0; b < kND; ++b) {
      mbar_init(&dfull[b], 1);
      mbar_init(&dfree[b], kEpiWarps);
    }
    for (int b = 0; b < kNS; ++b) mbar_init(&sfull[b], 4);
    mbar_init(&lv_ready, 1);
    mbar_init(&dig_ready, 1);
    fence_mbar_init();
    s_nwon = 0;
    // slot table: the column slices the range touches, digit areas back to back
    const uint32_t base = smem_u32(smem + a.ns * kStageBytes);
    uint32_t off = 0;
    int n = 0;
    for (int u = u_begin; u < u_end && n < kMaxSlots;) {
      const int j = u / a.npair;
      const int ue = min(u_end, (j + 1) * a.npair);
      Slot sl;
      sl.j = j;
      sl.u0 = u - u_begin;
      sl.u1 = ue - u_begin;
      sl.p0 = u - j * a.npair;
      sl.gfirst = slice_first(j, a.G, a.slices);
      sl.ng = slice_first(j + 1, a.G, a.slices) - sl.gfirst;
      sl.dig = base + off;
      off += (uint32_t)(a.N * 128 * sl.ng);
      sl.gc = base + off;
      off += (uint32_t)(16 * a.batch * sl.ng);
      off = (off + 1023u) & ~1023u;
      slots[n++] = sl;
      u = ue;
    }
    s_nslots = n;
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&s_tmem)),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  fence_before();
  __syncthreads();
  fence_after();
  pdl_wait();  // everything above read only the parameters
  const uint32_t tmem = s_tmem;
  const int nsl = s_nslots;

  // ---- prologue. Thread 0 brings the column slices' digits in (bulk copies from the workspace,
  // written by the digit kernel that ran first); warp 0 reads the level bytes into the level
  // cache and then streams weights at once, and the converters start on them as soon as the
  // cache is published. Only the MMA issuer and the epilogue wait for the digits.
  if (warp == 0) {
    if (lane == 0) {
      uint32_t bytes = 0;
      for (int si = 0; si < nsl; ++si) bytes += (uint32_t)(slots[si].ng * (a.N * 128 + 16 * a.batch));
      mbar_expect_tx(&dig_ready, bytes);
      for (int si = 0; si < nsl; ++si) {
        const Slot& sl = slots[si];
        const uint8_t* src = a.dig + (size_t)sl.gfirst * a.N * 128;
        const uint32_t nb = (uint32_t)(sl.ng * a.N * 128);
        for (uint32_t o = 0; o < nb; o += 32768u)
          bulk_g2s(smem + (sl.dig - smem_u32(smem)) + o, src + o, min(32768u, nb - o), &dig_ready);
        bulk_g2s(smem + (sl.gc - smem_u32(smem)), a.gct + (size_t)sl.gfirst * a.batch,
                 (uint32_t)(16 * a.batch * sl.ng), &dig_ready);
      }
    }
    for (int k = lane; k < nunits; k += 32) {
      const int u = u_begin + k, p = u % a.npair;
      lvc[k] = (uint16_t)(plane_range(a, 2 * p) | (plane_range(a, 2 * p + 1) << 8));
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&lv_ready);
  }
  const bool lv_ok = mbar_wait(&lv_ready, 0u);
  if (!lv_ok && lane == 0) atomicExch(&g_error, 5);

  if ((warp == 2 || warp == 3) && lane == 0) {
    // ---------------------------------------------------------------- producers (block bi)
    const int bi = warp - 2;
    int st = 0;  // stages issued
    bool failed = !lv_ok;
    for (int si = 0; si < nsl && !failed; ++si) {
      const Slot& sl = slots[si];
      for (int k = sl.u0; k < sl.u1 && !failed; ++k) {
        const int p = sl.p0 + (k - sl.u0);
        const int pr2 = lvc[k];
        const int pr = (pr2 >> (8 * bi)) & 0xFF, k0 = pr >> 4, np = pr & 15;
        const int tgm = stage_groups(max(pr2 & 15, (pr2 >> 8) & 15));
        const uint8_t* blk = a.store + (size_t)(2 * p + bi) * 8448u * a.G;
        for (int g0 = 0; g0 < sl.ng; g0 += tgm, ++st) {
          const int tg = min(tgm, sl.ng - g0), s = st % a.ns;
          if (st >= a.ns && !mbar_wait(&empty_bar[s], (uint32_t)((st / a.ns - 1) & 1))) {
            atomicExch(&g_error, 1);
            failed = true;
            break;
          }
          mbar_expect_tx(&full_bar[s], np ? (uint32_t)tg * (256u + 2048u * np) : 0u);
          if (np == 0) continue;
          const int gg = sl.gfirst + g0;
          uint8_t* dst = smem + s * kStageBytes + bi * kBlockTile;
          // [tg groups][64 rows] scales, then plane kk as [tg groups][64 rows][32 B]
          bulk_g2s(dst, blk + 256u * gg, 256u * tg, &full_bar[s]);
          for (int kk = 0; kk < np; ++kk)
            bulk_g2s(dst + 256 * tg + 2048 * tg * kk, blk + 256u * a.G + 2048u * ((size_t)a.G * (k0 + kk) + gg),
                     2048u * tg, &full_bar[s]);
        }
      }
    }
    // no copy may still be landing when the CTA exits
    for (int q = max(0, st - a.ns); q < st; ++q)
      if (!mbar_wait(&full_bar[q % a.ns], (uint32_t)((q / a.ns) & 1))) atomicExch(&g_error, 1);
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issue
    if (lane == 0) {
      const uint32_t idesc = idesc_i8(a.N);
      int it = 0;
      bool failed = !lv_ok || !mbar_wait(&dig_ready, 0u);
      if (failed) atomicExch(&g_error, 5);
      for (int si = 0; si < nsl && !failed; ++si) {
        const Slot& sl = slots[si];
        for (int k = sl.u0; k < sl.u1 && !failed; ++k) {
          for (int g = 0; g < sl.ng; ++g, ++it) {
            const int ab = it % kNA, db = it % kND;
            if (!mbar_wait(&afull[ab], (uint32_t)((it / kNA) & 1)) ||
                (it >= kND && !mbar_wait(&dfree[db], (uint32_t)((it / kND - 1) & 1)))) {
              atomicExch(&g_error, 2);
              failed = true;
              break;
            }
            fence_after();
            const uint32_t bt = sl.dig + (uint32_t)(g * a.N * 128);
#pragma unroll
            for (int st = 0; st < 4; ++st)
              mma_i8(tmem + kColD + 128u * db, tmem + kColA + 32u * ab + 8u * st, kmajor_desc(bt + 256u * st), idesc,
                     st > 0);
            mma_commit(&dfull[db]);
            mma_commit(&afree[ab]);
          }
        }
      }
      // the CTA's MMAs are complete before TMEM is freed (a commit tracks every earlier MMA)
      if (it > 0 && !mbar_wait(&afree[(it - 1) % kNA], (uint32_t)(((it - 1) / kNA) & 1))) atomicExch(&g_error, 2);
    }
    __syncwarp();
  } else if (warp >= 4 && warp < 8) {
    // ---------------------------------------------------------------- converters
    const int c = warp - 4, bi = c >> 1, rb = 32 * (c & 1) + lane;
    const uint32_t ta = tmem + ((uint32_t)(32 * c) << 16);
    int it = 0, st = 0;
    bool failed = !__all_sync(0xffffffffu, lv_ok);
    for (int si = 0; si < nsl && !failed; ++si) {
      const Slot& sl = slots[si];
      for (int k = sl.u0; k < sl.u1 && !failed; ++k) {
        const int pr2 = lvc[k];
        const int pr = (pr2 >> (8 * bi)) & 0xFF, k0 = pr >> 4, np = pr & 15;
        const int tgm = stage_groups(max(pr2 & 15, (pr2 >> 8) & 15));
        for (int g0 = 0; g0 < sl.ng && !failed; g0 += tgm, ++st) {
          const int tg = min(tgm, sl.ng - g0), s = st % a.ns;
          if (!__all_sync(0xffffffffu, mbar_wait(&full_bar[s], (uint32_t)((st / a.ns) & 1)))) {
            if (lane == 0) atomicExch(&g_error, 3);
            failed = true;
            break;
          }
          const uint32_t tile = smem_u32(smem + s * kStageBytes + bi * kBlockTile);
          for (int gl = 0; gl < tg; ++gl, ++it) {
            const int ab = it % kNA;
            if (!__all_sync(0xffffffffu, it < kNA || mbar_wait(&afree[ab], (uint32_t)((it / kNA - 1) & 1)))) {
              if (lane == 0) atomicExch(&g_error, 3);
              failed = true;
              break;
            }
            fence_after();
            float sc = 0.f;
            if (np > 0) asm volatile("ld.shared.f32 %0, [%1];" : "=f"(sc) : "r"(tile + 256u * gl + 4u * rb));
            scl[it % kNS][32 * c + lane] = sc;
            uint32_t r[32];
            codes_dispatch(k0, np, tile + 256u * tg + 2048u * gl + 32u * rb, 2048u * tg, r);
            tmem_st32(ta + kColA + 32u * ab, r);
            asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
            fence_before();
            __syncwarp();
            if (lane == 0) {
              mbar_arrive(&sfull[it % kNS]);
              mbar_arrive(&afull[ab]);
            }
          }
          __syncwarp();
          if (lane == 0 && !failed) mbar_arrive(&empty_bar[s]);
        }
      }
    }
    fence_before();
  } else if (warp >= 8) {
    // ---------------------------------------------------------------- epilogue
    constexpr int NH = (NB + 1) / 2;
    const int q = warp & 3, h = (warp - 8) >> 2, bi = q >> 1, rb = 32 * (q & 1) + lane, row = 32 * q + lane;
    const int ch0 = h * NH;  // first batch chunk of this warp
    const uint32_t td = tmem + ((uint32_t)(32 * q) << 16) + kColD;
    float acc[8 * NH];
#pragma unroll
    for (int i = 0; i < 8 * NH; ++i) acc[i] = 0.f;
    int it = 0;
    bool failed = !__all_sync(0xffffffffu, lv_ok && mbar_wait(&dig_ready, 0u));
    if (failed && lane == 0) atomicExch(&g_error, 5);
    const size_t ystride = (size_t)64 * a.nblk;
    for (int si = 0; si < nsl; ++si) {
      const Slot& sl = slots[si];
      for (int k = sl.u0; k < sl.u1; ++k) {
        const int p = sl.p0 + (k - sl.u0);
        const int pr = (lvc[k] >> (8 * bi)) & 0xFF, k0 = pr >> 4, np = pr & 15;
        const int b = 2 * p + bi;
        const bool live = b < a.nblk && np > 0;
        const float cf = cfac_of(k0, np);
        for (int g = 0; g < sl.ng; ++g, ++it) {
          const int db = it % kND;
          if (failed) continue;
          if (!__all_sync(0xffffffffu, mbar_wait(&sfull[it % kNS], (uint32_t)((it / kNS) & 1)) &&
                                           mbar_wait(&dfull[db], (uint32_t)((it / kND) & 1)))) {
            if (lane == 0) atomicExch(&g_error, 4);
            failed = true;
            continue;
          }
          const float sc = live ? scl[it % kNS][row] : 0.f;
          fence_after();
          // every TMEM load of the group first, one wait; the group constants are plain shared
          // loads the compiler can schedule ahead of the arithmetic
          const float4* gcs = reinterpret_cast<const float4*>(smem + (sl.gc - smem_u32(smem))) + g * a.batch;
          uint32_t v[NH][32];
#pragma unroll
          for (int c = 0; c < NH; ++c)
            if (ch0 + c < NB && 8 * (ch0 + c) < a.batch) tmem_ld32(td + 128u * db + 32u * (ch0 + c), v[c]);
          asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
          for (int c = 0; c < NH; ++c) {
            const int ch = ch0 + c;
            if (ch < NB && 8 * ch < a.batch) {
#pragma unroll
              for (int j = 0; j < 8; ++j) {
                const int bb = 8 * ch + j;
                if (bb < a.batch) {
                  // each digit column's sum is below 2^22 in magnitude, so it becomes a float
                  // exactly by the 1.5 * 2^23 bias (integer add, float subtract) on full-rate pipes
                  const float4 gc = gcs[bb];
                  const float f3 = __int_as_float((int)v[c][4 * j] + 0x4B400000) - 12582912.f;
                  const float f2 = __int_as_float((int)v[c][4 * j + 1] + 0x4B400000) - 12582912.f;
                  const float f1 = __int_as_float((int)v[c][4 * j + 2] + 0x4B400000) - 12582912.f;
                  const float f0 = __int_as_float((int)v[c][4 * j + 3] + 0x4B400000) - 12582912.f;
                  const float u = fmaf(f1, 256.f, fmaf(f3, 16777216.f, f2 * 65536.f)) + f0;
                  acc[8 * c + j] = fmaf(sc, fmaf(u, gc.y, cf * gc.z), acc[8 * c + j]);
                }
              }
            }
          }
          fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&dfree[db]);
        }
        // ---- unit done: this thread's row is final (or a slice partial), for its batch rows
        const bool row_ok = b < a.nblk;
        if (a.slices == 1) {
          if (row_ok && !failed) {
#pragma unroll
            for (int i = 0; i < 8 * NH; ++i) {
              const int bb = 8 * ch0 + i;
              if (bb < a.batch) {
                float* yy = a.y + (size_t)bb * ystride + 64 * b + rb;
                if (a.mode == 0)
                  *yy = acc[i];
                else
                  red_add_f32(yy, acc[i]);  // added where y lives: no load on the epilogue's path
              }
            }
          }
        } else {
          float* pp = a.partial + ((size_t)sl.j * a.npair + p) * a.batch * 128 + row;
#pragma unroll
          for (int i = 0; i < 8 * NH; ++i) {
            const int bb = 8 * ch0 + i;
            if (bb < a.batch) pp[(size_t)bb * 128] = acc[i];
          }
          // the barrier orders the eight warps' partial stores before one thread's
          // acquire-release ticket; the last of the slices to arrive adds them up once the
          // CTA's units are done
          named_bar(kBarEpi, 32 * kEpiWarps);
          if (warp == 8 && lane == 0 && atom_add_acq_rel(&a.tickets[p], 1u) == (uint32_t)(a.slices - 1))
            won[s_nwon++] = (uint16_t)p;
        }
#pragma unroll
        for (int i = 0; i < 8 * NH; ++i) acc[i] = 0.f;
      }
    }
    fence_before();
  }

  // ------------------------------------------------------------------ every warp
  __syncthreads();  // every role is done: no copy in flight, every MMA complete, TMEM reads done
  if (warp == 1) {
    fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols) : "memory");
  }
  // Slice sums of the pairs this CTA won, in slice order: item = (pair, batch row, 4 rows), one
  // float4 per slice, eight slices' loads issued before they are added.
  const int nwon = s_nwon;
  for (int wi = 0; wi < nwon; ++wi) {
    const int p = won[wi];
    const float4* base = reinterpret_cast<const float4*>(a.partial + (size_t)p * a.batch * 128);
    const size_t jstride = (size_t)a.npair * a.batch * 32;  // float4 per slice
    for (int item = threadIdx.x; item < a.batch * 32; item += kThreads) {
      const int bb = item >> 5, r4 = item & 31;
      const int b = 2 * p + (r4 >> 4), rb = 4 * (r4 & 15);
      float4 sum = make_float4(0.f, 0.f, 0.f, 0.f);
      for (int j0 = 0; j0 < a.slices; j0 += 8) {
        float4 v[8];
#pragma unroll
        for (int q = 0; q < 8; ++q)
          v[q] = (j0 + q < a.slices) ? __ldcg(base + (size_t)(j0 + q) * jstride + item) : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          sum.x += v[q].x;
          sum.y += v[q].y;
          sum.z += v[q].z;
          sum.w += v[q].w;
        }
      }
      if (b < a.nblk) {  // y is only 4-byte aligned: four scalar stores
        float* yy = a.y + (size_t)bb * 64 * a.nblk + 64 * b + rb;
        if (a.mode == 1) {
          red_add_f32(yy, sum.x);
          red_add_f32(yy + 1, sum.y);
          red_add_f32(yy + 2, sum.z);
          red_add_f32(yy + 3, sum.w);
        } else {
          yy[0] = sum.x;
          yy[1] = sum.y;
          yy[2] = sum.z;
          yy[3] = sum.w;
        }
      }
    }
    __syncthreads();
    if (threadIdx.x == 0) a.tickets[p] = 0u;
  }
}

// ---------------------------------------------------------------- host side

struct Plan {
  int slices, slice_groups, npair, N;
};

static int groups_fit(int batch) {
  const int per = n_cols(batch) * 128 + 16 * batch;
  return std::max(1, (kDigitBudget - 2048) / per);
}

// Column slices: as wide as the digits allow, and narrow enough that the units (slice x block
// pair) number about four per SM, so contiguous ranges balance. The slices are equal to a group
// (slice_first): a short last slice made a CTA of many small units, each paying the unit's fixed
// cost, the launch's slowest (4096 -> 14336 at batch 16: 52.6 us with a two-group last slice,
// 34.0 us with equal ones).
static Plan plan(int nblk, int G, int batch, int nsm) {
  Plan pl;
  pl.npair = (nblk + 1) / 2;
  pl.N = n_cols(batch);
  const int gmax = groups_fit(batch);
  const int s_mem = (G + gmax - 1) / gmax;
  const int s_fill = (4 * nsm + pl.npair - 1) / pl.npair;
  int s = std::max(s_mem, std::min(s_fill, G));
  s = std::min(s, G);
  pl.slice_groups = (G + s - 1) / s;
  pl.slices = (G + pl.slice_groups - 1) / pl.slice_groups;
  return pl;
}

// Workspace: [tickets][slice partials] when the columns are split, then always the digits and
// the group constants the digit kernel writes.
struct WsLayout {
  size_t tickets, partial, dig, gct, total;
};

static WsLayout ws_layout(const Plan& pl, int G, int batch) {
  WsLayout w;
  w.tickets = 0;
  w.partial = pl.slices > 1 ? ((size_t)pl.npair * 4 + 255) / 256 * 256 : 0;
  w.dig = w.partial + (pl.slices > 1 ? (size_t)pl.slices * pl.npair * batch * 128 * 4 : 0);
  w.dig = (w.dig + 255) / 256 * 256;
  w.gct = w.dig + (size_t)G * pl.N * 128;
  w.total = w.gct + (size_t)G * batch * 16;
  return w;
}

// A unit's fixed cost (its end: partial stores, the epilogue's barrier and ticket), in groups.
constexpr double kUnitCost = 1.0;

// Contiguous ranges of units (slice-major), balanced by groups read plus each unit's fixed cost; a range is also cut when
// the digits of the slices it touches would overflow shared memory, at kMaxSlots slices, or at
// the level-cache size; after every cut the rest is spread evenly over the ranges still to make.
static bool partition(Args& a, const Plan& pl, int nsm, size_t* max_dig) {
  const int units = pl.slices * pl.npair;
  const int target = std::max(1, std::min(nsm, units));
  double total = 0;
  for (int j = 0; j < pl.slices; ++j)
    total += (double)pl.npair * (slice_first(j + 1, a.G, pl.slices) - slice_first(j, a.G, pl.slices) + kUnitCost);
  double per = total / target, acc = 0, start = 0;
  int n = 0, nslots = 0, count = 0;
  size_t dig = 0;
  a.cta_begin[0] = 0;
  for (int u = 0; u < units; ++u) {
    const int j = u / pl.npair, p = u % pl.npair;
    const int ng = slice_first(j + 1, a.G, pl.slices) - slice_first(j, a.G, pl.slices);
    const size_t sb = (((size_t)pl.N * 128 * ng + 16 * a.batch * ng) + 1023) / 1024 * 1024;
    bool cut = false;
    if (count > 0) {
      if (n + 1 < target && acc + 0.5 * (ng + kUnitCost) - start > per) cut = true;
      if ((p == 0 || count == 0) && (dig + sb > (size_t)kDigitBudget || nslots == kMaxSlots)) cut = true;
      if (count == kLevelCache) cut = true;
    }
    if (cut) {
      if (n + 1 >= kMaxCtas) return false;
      a.cta_begin[++n] = u;
      *max_dig = std::max(*max_dig, dig);
      dig = 0;
      nslots = 0;
      count = 0;
      start = acc;
      per = (total - acc) / std::max(1, target - n);
    }
    if (p == 0 || count == 0) {
      dig += sb;
      ++nslots;
    }
    acc += ng + kUnitCost;
    ++count;
  }
  a.cta_begin[++n] = units;
  a.ncta = n;
  *max_dig = std::max(*max_dig, dig);
  return true;
}

template <int NB>
static fl_status launch_nb(const Args& a, cudaStream_t st) {
  auto kern = tc_gemv_kernel<NB>;
  FL_CHECK_CUDA(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemLimit),
                "cudaFuncSetAttribute(tc_gemv)");
  FL_CHECK_CUDA(launch_pdl(kern, dim3(a.ncta), dim3(kThreads), (size_t)kSmemLimit, st, 1, a), "launch tc_gemv");
  return FL_OK;
}

}  // namespace tc

// Entry used by the plane GEMV's single-layer calls for batch >= tc::kMinBatch.
bool tc_takes(int batch) { return batch >= tc::kMinBatch; }

size_t tc_workspace_bytes(int out, int in, int batch) {
  const int nsm = device_sm_count();
  if (nsm <= 0) return 0;
  return tc::ws_layout(tc::plan(out / 64, in / 128, batch, nsm), in / 128, batch).total;
}

fl_status tc_single(const fl_plane_weight* w, const uint8_t* lv_from, const uint8_t* lv_to, const uint16_t* x,
                    int batch, float* y, void* ws, size_t ws_bytes, void* stream, int mode, const char* what) {
  const int nsm = device_sm_count();
  if (nsm <= 0) return fail(FL_ERR_CUDA, "%s: no CUDA device", what);
  const int nblk = w->out / 64, G = w->in / 128;
  const tc::Plan pl = tc::plan(nblk, G, batch, nsm);
  const tc::WsLayout wl = tc::ws_layout(pl, G, batch);
  if (!ws || ws_bytes < wl.total)
    return fail(FL_ERR_WORKSPACE, "%s: workspace %zu bytes, need %zu", what, ws ? ws_bytes : (size_t)0, wl.total);
  if (!aligned16(ws)) return fail(FL_ERR_ALIGN, "%s: workspace not 16-byte aligned", what);
  static thread_local tc::Args a;
  a.store = w->store;
  a.lv_from = lv_from;
  a.lv_to = lv_to;
  a.x = x;
  a.y = y;
  a.nblk = nblk;
  a.npair = pl.npair;
  a.G = G;
  a.batch = batch;
  a.N = pl.N;
  a.mode = mode;
  a.slices = pl.slices;
  a.slice_groups = pl.slice_groups;
  uint8_t* wsb = static_cast<uint8_t*>(ws);
  a.tickets = pl.slices > 1 ? reinterpret_cast<uint32_t*>(wsb + wl.tickets) : nullptr;
  a.partial = pl.slices > 1 ? reinterpret_cast<float*>(wsb + wl.partial) : nullptr;
  a.dig = wsb + wl.dig;
  a.gct = reinterpret_cast<const float4*>(wsb + wl.gct);
  size_t max_dig = 0;
  if (!tc::partition(a, pl, nsm, &max_dig)) return fail(FL_ERR_SHAPE, "%s: layer too large for one launch", what);
  a.ns = std::min(tc::kMaxStages, (int)((tc::kSmemLimit - 1024 - max_dig) / tc::kStageBytes));
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  FL_CHECK_CUDA(launch_pdl(tc::tc_digits_kernel, dim3((unsigned)((G * batch + 7) / 8)), dim3(256), 0, st, 1, x, G,
                           batch, pl.N, wsb + wl.dig, reinterpret_cast<float4*>(wsb + wl.gct)),
                "launch tc_digits");
  switch ((batch + 7) / 8) {
    case 1: return tc::launch_nb<1>(a, st);
    case 2: return tc::launch_nb<2>(a, st);
    case 3: return tc::launch_nb<3>(a, st);
    default: return tc::launch_nb<4>(a, st);
  }
}

namespace tc {
// Reads and clears the error word (-1 if that fails).
int take_device_error() {
  int v = 0, z = 0;
  if (cudaMemcpyFromSymbol(&v, g_error, sizeof(int)) != cudaSuccess) return -1;
  if (v != 0 && cudaMemcpyToSymbol(g_error, &z, sizeof(int)) != cudaSuccess) return -1;
  return v;
}
}  // namespace tc

}  // namespace fl
