// K-quant fused dequant GEMV ("v0.3, quantized on disk, quantized in memory":
// native Q4_K and Q6_K kernels that keep the weights compressed and
// dequantize only at block granularity inside the product; per-tensor
// dispatch, unsupported types fail).
//
//   Q4_K:  y[t][r] = sum_sb sum_j ( d sc_j sum_{c in j} q_c x_c  -  dmin mn_j sum_{c in j} x_c )
//   Q6_K:  y[t][r] = sum_sb sum_j   d sc_j sum_{c in j} (q_c - 32) x_c
//
// Same B200 structure as the plane-store GEMV. A unit is one 64-row block times a column
// slice; one persistent CTA per SM takes a contiguous range of units. Four teams, each a
// producer warp (one lane issues copies) and four consumer warps (one per 16-row m-tile),
// walk units t, t + 4, ... of the range through the team's two shared-memory stages. The
// records are stored block-tiled, so a tile (64 rows x 2 Q4_K super-blocks = 18432 B, or
// 64 rows x 1 Q6_K super-block = 13440 B) is one contiguous 1-D bulk copy. Codes become u8
// tensor-core operands with one or two mask/shift operations per four weights (the record
// layouts are built for it); each sub-block is one mma.sync (m16n8k32 for Q4_K's 32-weight
// sub-blocks, m16n8k16 for Q6_K's 16-weight ones) against the activations' four int8 digits
// (fl_common.cuh; two digit pairs per batch row, one MMA column pair each); the sub-block
// scale is applied to the int32 result with an integer multiply-add, each 128-column half of a
// super-block is converted to fp32 once per pair, and a batch row's two pairs meet in one
// shuffle when the unit ends.
#include <algorithm>

#include "fl_common.cuh"

namespace fl {
namespace kq {

constexpr int kTeams = 4;
constexpr int kTeamWarps = 4;
constexpr int kTeamThreads = 32 * kTeamWarps;
constexpr int kConsumerWarps = kTeams * kTeamWarps;
constexpr int kConsumers = 32 * kConsumerWarps;
constexpr int kProducerWarps = kTeams;  // producer warp t feeds team t
constexpr int kThreads = kConsumers + 32 * kProducerWarps;
constexpr int kTeamStages = 2;
constexpr int kStages = kTeams * kTeamStages;
constexpr int kStageBytes = 18432;  // 64 rows x 2 Q4_K records
constexpr int kMaxCtas = 1024;
constexpr int kRed = 8;               // outputs per thread per pass of the slice reduction
constexpr int kMaxSlots = 64;         // distinct (problem, slice) pairs one CTA may touch
constexpr int kSmemLimit = 232448 - 16384;  // opt-in shared memory per block on B200, less static use
constexpr int kDigitBudget = kSmemLimit - kStages * kStageBytes;

__host__ __device__ constexpr int rec_bytes(int type) { return type == FL_GGML_Q4_K ? 144 : 210; }
__host__ __device__ constexpr int tile_sb(int type) { return type == FL_GGML_Q4_K ? 2 : 1; }

struct Problem {
  const uint8_t* blocks;
  const uint16_t* x;
  float* y;
  float* partial;      // [slices][nblocks][batch][64] when slices > 1
  uint32_t* tickets;   // [nblocks] when slices > 1
  int type;            // FL_GGML_Q4_K or FL_GGML_Q6_K
  int nblocks;         // out / 64
  int nsb;             // in / 256
  int slices;
  int slice_sb;        // super-blocks per slice (last slice shorter)
  int unit_begin;      // first global unit index of this problem
};

template <int MAXP>
struct Args {
  int nproblems;
  int batch;
  int ncta;
  int cta_begin[kMaxCtas + 1];
  int cta_slice[kMaxCtas];  // first (problem, slice) pair of the CTA, counted in order, << 7 | pairs touched
  Problem p[MAXP];
};

__device__ int g_error;  // set when a bounded wait runs out (never expected)

// One (problem, column slice) touched by a CTA; see the plane-store GEMV for the scheme.
// Activation digits: rows 4b .. 4b+3 hold digits d3, d2, d1, d0 of batch row b (stride bytes
// per row, Q4_K slots in the permuted order its MMA fragments read), i.e. digit pair p = 2b + r
// is rows 2p, 2p+1; per (padded pair row, 128-column group): iscale = the pair's weight
// (2^(16 - sigma) for r = 0, 2^-sigma for r = 1) and gsum = 8 sums of 16 columns of the pair's
// value (256 d3 + d2, or 256 d1 + d0).
struct __align__(16) Slot {
  int p, j, u0, u1, b0;
  int nblocks, nsb, nsbs, slices, sbfirst;  // nsbs = super-blocks of the slice
  int type, stride, it0, ngroups;           // ngroups = 2 nsbs
  uint32_t digits, iscale, gsum;            // smem addresses
  const uint8_t* blocks;
  const uint16_t* x;
  float* y;
  float* partial;
  uint32_t* tickets;
};

enum : int { kBarTeam0 = 2, kBarX = 6, kBarDigits = 7 };

__device__ __forceinline__ void named_bar(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

__device__ __forceinline__ void bar_arrive(int id, int nthreads) {
  asm volatile("bar.arrive %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

__device__ __forceinline__ float half_bits_to_float(uint32_t h) {
  return __half2float(__ushort_as_half(static_cast<unsigned short>(h & 0xFFFFu)));
}

__device__ __forceinline__ int byte_u(uint32_t w, int j) { return (int)__byte_perm(w, 0u, 0x4440u | (uint32_t)j); }

// Byte j of w, sign-extended. Uses PTX prmt directly: its selector's top bit
// replicates the selected byte's sign, which __byte_perm does not expose.
__device__ __forceinline__ int byte_s(uint32_t w, int j) {
  const uint32_t sj = 8u | (uint32_t)j;
  const uint32_t sel = (uint32_t)j | (sj << 4) | (sj << 8) | (sj << 12);
  uint32_t r;
  asm("prmt.b32 %0, %1, 0, %2;" : "=r"(r) : "r"(w), "r"(sel));
  return (int)r;
}

__device__ __forceinline__ uint32_t lds_u32(uint32_t a) {
  uint32_t v;
  asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(a));
  return v;
}

__device__ __forceinline__ uint32_t lds_u16(uint32_t a) {
  unsigned short v;
  asm volatile("ld.shared.u16 %0, [%1];" : "=h"(v) : "r"(a));
  return v;
}

__device__ __forceinline__ float lds_f32(uint32_t a) {
  float v;
  asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(a));
  return v;
}

__device__ __forceinline__ uint2 lds_v2(uint32_t a) {
  uint2 v;
  asm volatile("ld.shared.v2.u32 {%0,%1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(a));
  return v;
}

__device__ __forceinline__ uint4 lds_v4(uint32_t a) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a));
  return v;
}

__device__ __forceinline__ int4 lds_s4(uint32_t a) {
  int4 v;
  asm volatile("ld.shared.v4.s32 {%0,%1,%2,%3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a));
  return v;
}

__device__ __forceinline__ int slice_nsb(const Problem& P, int j) { return min(P.slice_sb, P.nsb - j * P.slice_sb); }

__device__ __forceinline__ uint32_t atom_add_acq_rel(uint32_t* p, uint32_t v) {
  uint32_t old;
  asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
  return old;
}

// A slot's digit area, pair rows padded to 4 NT. The padded strides spread the rows that
// one warp reads together over distinct shared-memory banks.
//   digits: 4 rows of digit_stride bytes per batch row (d3, d2, d1, d0)
//   iscale: [4 NT][ngroups + 1] floats, area rounded up to 16 bytes
//   gsum:   [4 NT][gsum_row bytes]: per 128-column group 8 int32 sums of 16 columns
__host__ __device__ constexpr int digit_stride(int ngroups) { return 128 * ngroups + 32; }
__host__ __device__ constexpr int iscale_row(int ngroups) { return ngroups + 1; }
__host__ __device__ constexpr int gsum_row(int ngroups) { return 32 * ngroups + 16; }
__host__ __device__ constexpr int iscale_area(int nt, int ngroups) { return (16 * nt * iscale_row(ngroups) + 15) & ~15; }
__host__ __device__ constexpr int slot_area(int batch, int nt, int ngroups) {
  return 4 * batch * digit_stride(ngroups) + iscale_area(nt, ngroups) + 4 * nt * gsum_row(ngroups);
}

// Rows of the 64-row block held by lane row g of warp mt: Q4_K records (144 B) are
// bank-conflict free for consecutive rows; Q6_K records (210 B) are when the eight rows of
// a fragment half are {0, 1, 3, 5} or {7, 2, 4, 6} of an 8-row group plus the same rows 32
// further on.
__device__ __forceinline__ int q6_row(int mt, int h, int g) {
  const int x = g & 3;
  return 8 * mt + (x == 0 ? (h ? 7 : 0) : 2 * x - 1 + h) + 32 * (g >> 2);
}

__device__ __forceinline__ uint2 lds_v2_if(uint32_t a, bool p) {
  uint2 v;
  asm volatile(
      "{ .reg .pred q; setp.ne.u32 q, %3, 0; mov.u32 %0, 0; mov.u32 %1, 0; @q ld.shared.v2.u32 {%0,%1}, [%2]; }"
      : "=r"(v.x), "=r"(v.y)
      : "r"(a), "r"((uint32_t)p));
  return v;
}

__device__ __forceinline__ uint32_t lds_u32_if(uint32_t a, bool p) {
  uint32_t v;
  asm volatile("{ .reg .pred q; setp.ne.u32 q, %2, 0; mov.u32 %0, 0; @q ld.shared.u32 %0, [%1]; }"
               : "=r"(v)
               : "r"(a), "r"((uint32_t)p));
  return v;
}

// ---------------------------------------------------------------- activation digits
// One item = 128 columns of one batch row (see fl_common.cuh for the number format),
// converted by one warp; the Q4_K slots store each word at the place its m16n8k32 B
// fragment reads it.
__device__ __forceinline__ void convert_item(uint2 raw, const Slot& sl, int b, int g, int lane) {
  const float f[4] = {__uint_as_float(raw.x << 16), __uint_as_float(raw.x & 0xFFFF0000u),
                      __uint_as_float(raw.y << 16), __uint_as_float(raw.y & 0xFFFF0000u)};
  uint32_t dw[4];
  int2 part;
  const int sigma = split_digits(f, dw, part);
  const int wpos = (sl.type == FL_GGML_Q4_K) ? (8 * (lane >> 3) + 2 * (lane & 3) + ((lane >> 2) & 1)) : lane;
  const uint32_t dh = sl.digits + (uint32_t)((4 * b) * sl.stride + 128 * g + 4 * wpos);
#pragma unroll
  for (int k = 0; k < 4; ++k)
    asm volatile("st.shared.u32 [%0], %1;" ::"r"(dh + (uint32_t)(k * sl.stride)), "r"(dw[k]) : "memory");
  // sums of 16 columns (4 lanes each), per digit pair
  part.x += __shfl_xor_sync(0xffffffffu, part.x, 1);
  part.x += __shfl_xor_sync(0xffffffffu, part.x, 2);
  part.y += __shfl_xor_sync(0xffffffffu, part.y, 1);
  part.y += __shfl_xor_sync(0xffffffffu, part.y, 2);
  const uint32_t gs0 = sl.gsum + (uint32_t)(2 * b * gsum_row(sl.ngroups) + 32 * g + (lane & ~3));
  if ((lane & 3) == 0) {
    asm volatile("st.shared.s32 [%0], %1;" ::"r"(gs0), "r"(part.x) : "memory");
    asm volatile("st.shared.s32 [%0], %1;" ::"r"(gs0 + (uint32_t)gsum_row(sl.ngroups)), "r"(part.y) : "memory");
  }
  if (lane == 0) {
    const uint32_t is0 = sl.iscale + 4u * (uint32_t)(2 * b * iscale_row(sl.ngroups) + g);
    asm volatile("st.shared.f32 [%0], %1;" ::"r"(is0), "f"(ldexpf(1.0f, 16 - sigma)) : "memory");
    asm volatile("st.shared.f32 [%0], %1;" ::"r"(is0 + 4u * (uint32_t)iscale_row(sl.ngroups)),
                 "f"(ldexpf(1.0f, -sigma))
                 : "memory");
  }
}

// All consumer threads; every thread arrives once on kBarX after its last round of loads is
// issued, which lets the producers start the weight copies behind them.
__device__ __forceinline__ void build_digits(const Slot* slots, int nsl, int batch, int batch_pad, int tid,
                                             int nthreads) {
  const int lane = tid & 31, wid = tid >> 5, nw = nthreads >> 5;
  const Slot& last = slots[nsl - 1];
  const int total = last.it0 + batch * last.ngroups;
  int si = 0;
  for (int round = 0, it0 = wid; round == 0 || it0 < total; ++round, it0 += 4 * nw) {
    uint2 raw[4];
    int sq[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int it = it0 + q * nw;
      sq[q] = -1;
      if (it < total) {
        while (si + 1 < nsl && it >= slots[si + 1].it0) ++si;
        const Slot& sl = slots[si];
        const int local = it - sl.it0, b = local / sl.ngroups, g = local % sl.ngroups;
        raw[q] = __ldg(reinterpret_cast<const uint2*>(sl.x + (size_t)b * sl.nsb * 256 + 256 * sl.sbfirst + 128 * g +
                                                      4 * lane));
        sq[q] = si;
      }
    }
    if (it0 + 4 * nw >= total) bar_arrive(kBarX, kThreads);  // this warp's last round
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      if (sq[q] >= 0) {
        const Slot& sl = slots[sq[q]];
        const int local = it0 + q * nw - sl.it0;
        convert_item(raw[q], sl, local / sl.ngroups, local % sl.ngroups, lane);
      }
    }
  }
  // padded pair rows read zero scales and sums
  for (int i = 0; i < nsl; ++i) {
    const Slot& sl = slots[i];
    const int n = (batch_pad - 2 * batch) * sl.ngroups;
    for (int e = tid; e < 9 * n; e += nthreads) {
      const int b = 2 * batch + (e % n) / sl.ngroups, g = (e % n) % sl.ngroups;
      if (e < n)
        asm volatile("st.shared.f32 [%0], %1;" ::"r"(sl.iscale + 4u * (uint32_t)(b * iscale_row(sl.ngroups) + g)),
                     "f"(0.f)
                     : "memory");
      else
        asm volatile("st.shared.s32 [%0], %1;" ::"r"(sl.gsum + (uint32_t)(b * gsum_row(sl.ngroups) + 32 * g +
                                                                         4 * (e / n - 1))),
                     "r"(0)
                     : "memory");
    }
  }
}

// ---------------------------------------------------------------- Q4_K: half (4 sub-blocks) of one super-block
// rec0 / rec1: records of the lane's two rows; dl: digit rows (+ 8 t, permuted), live: whether
// the lane's digit row is a real batch row (else its B fragment is zero); colg: first
// column of the super-block in the slice; gi: 128-column group of the half in the slice.
template <int NT>
__device__ __forceinline__ void q4k_half(uint32_t rec0, uint32_t rec1, int half, const uint32_t (&dl)[NT],
                                         const bool (&live)[NT], int colg, uint32_t iscale, uint32_t gsum,
                                         int gstride, int gi, int t, float (&acc)[NT][2]) {
  const uint4 h0 = lds_v4(rec0);
  const uint4 h1 = lds_v4(rec1);
  const float d0 = half_bits_to_float(h0.x), dm0 = half_bits_to_float(h0.x >> 16);
  const float d1 = half_bits_to_float(h1.x), dm1 = half_bits_to_float(h1.x >> 16);
  const uint32_t S0 = half ? h0.z : h0.y, S1 = half ? h1.z : h1.y;
  const uint32_t sc0 = S0 & 0x3F3F3F3Fu, sc1 = S1 & 0x3F3F3F3Fu;
  // mn_j bytes: low 2 bits from the top of byte j, high 4 bits from nibble j
  const uint32_t M0 = half ? (h0.w >> 16) : (h0.w & 0xFFFFu), M1 = half ? (h1.w >> 16) : (h1.w & 0xFFFFu);
  const uint32_t mn0 = ((S0 >> 6) & 0x03030303u) | (__byte_perm(M0 & 0x0F0Fu, (M0 >> 4) & 0x0F0Fu, 0x5140u) << 2);
  const uint32_t mn1 = ((S1 >> 6) & 0x03030303u) | (__byte_perm(M1 & 0x0F0Fu, (M1 >> 4) & 0x0F0Fu, 0x5140u) << 2);
  uint32_t q0[4], q1[4];
#pragma unroll
  for (int jj = 0; jj < 4; ++jj) {
    const int j = 4 * half + jj;
    q0[jj] = lds_u32(rec0 + 16u + 16u * j + 4u * t);
    q1[jj] = lds_u32(rec1 + 16u + 16u * j + 4u * t);
  }
  int32_t ai[NT][4];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) ai[nt][0] = ai[nt][1] = ai[nt][2] = ai[nt][3] = 0;
#pragma unroll
  for (int jj = 0; jj < 4; ++jj) {
    const int j = 4 * half + jj;
    const uint32_t a0 = q0[jj] & 0x0F0F0F0Fu, a2 = (q0[jj] >> 4) & 0x0F0F0F0Fu;
    const uint32_t a1 = q1[jj] & 0x0F0F0F0Fu, a3 = (q1[jj] >> 4) & 0x0F0F0F0Fu;
    const int s0 = byte_u(sc0, jj), s1 = byte_u(sc1, jj);
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const uint2 bb = lds_v2_if(dl[nt] + (uint32_t)(colg + 32 * j), live[nt]);
      int32_t C[4] = {0, 0, 0, 0};
      mma_u8s8(C, a0, a1, a2, a3, bb.x, bb.y);
      ai[nt][0] += s0 * C[0];
      ai[nt][1] += s0 * C[1];
      ai[nt][2] += s1 * C[2];
      ai[nt][3] += s1 * C[3];
    }
  }
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    const int pr = 4 * nt + t;  // the lane's digit-pair row
    const float isc = lds_f32(iscale + 4u * (uint32_t)(pr * iscale_row(gstride) + gi));
    // sums over the 32-column sub-blocks from the 16-column sums
    const uint32_t ga = gsum + (uint32_t)(pr * gsum_row(gstride) + 32 * gi);
    const int4 Xa = lds_s4(ga);
    const int4 Xb = lds_s4(ga + 16u);
    const int32_t X0 = Xa.x + Xa.y, X1 = Xa.z + Xa.w, X2 = Xb.x + Xb.y, X3 = Xb.z + Xb.w;
    const int32_t mx0 = byte_u(mn0, 0) * X0 + byte_u(mn0, 1) * X1 + byte_u(mn0, 2) * X2 + byte_u(mn0, 3) * X3;
    const int32_t mx1 = byte_u(mn1, 0) * X0 + byte_u(mn1, 1) * X1 + byte_u(mn1, 2) * X2 + byte_u(mn1, 3) * X3;
    const float v0 = fmaf(256.f, (float)ai[nt][0], (float)ai[nt][1]);
    const float v1 = fmaf(256.f, (float)ai[nt][2], (float)ai[nt][3]);
    acc[nt][0] = fmaf(isc, fmaf(d0, v0, -dm0 * (float)mx0), acc[nt][0]);
    acc[nt][1] = fmaf(isc, fmaf(d1, v1, -dm1 * (float)mx1), acc[nt][1]);
  }
}

// ---------------------------------------------------------------- Q6_K: half (8 sub-blocks of 16) of one super-block
// odd: the rows' parity (their records' layout); dl: digit rows (+ 4 t, natural order).
template <int NT>
__device__ __forceinline__ void q6k_half(uint32_t rec0, uint32_t rec1, int odd0, int odd1, int half,
                                         const uint32_t (&dl)[NT], const bool (&live)[NT], int colg,
                                         uint32_t iscale, uint32_t gsum, int gstride, int gi, int t,
                                         float (&acc)[NT][2]) {
  const uint32_t qa0 = rec0 + (odd0 ? 2u : 0u), qa1 = rec1 + (odd1 ? 2u : 0u);
  const uint32_t sc0p = rec0 + (odd0 ? 194u : 192u), sc1p = rec1 + (odd1 ? 194u : 192u);
  const float d0 = half_bits_to_float(lds_u16(rec0 + (odd0 ? 0u : 208u)));
  const float d1 = half_bits_to_float(lds_u16(rec1 + (odd1 ? 0u : 208u)));
  int32_t ai[NT][4], ao[NT][2];
  int32_t X[NT][8];  // the half's 16-column sums, per batch row
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    ai[nt][0] = ai[nt][1] = ai[nt][2] = ai[nt][3] = ao[nt][0] = ao[nt][1] = 0;
    const uint32_t ga = gsum + (uint32_t)((4 * nt + t) * gsum_row(gstride) + 32 * gi);
    const int4 Xa = lds_s4(ga), Xb = lds_s4(ga + 16u);
    X[nt][0] = Xa.x; X[nt][1] = Xa.y; X[nt][2] = Xa.z; X[nt][3] = Xa.w;
    X[nt][4] = Xb.x; X[nt][5] = Xb.y; X[nt][6] = Xb.z; X[nt][7] = Xb.w;
  }
#pragma unroll
  for (int mm = 0; mm < 2; ++mm) {
    const int m = 2 * half + mm;
    const uint32_t w0 = qa0 + 48u * t + 12u * m;
    const uint32_t w1 = qa1 + 48u * t + 12u * m;
    const uint32_t A0 = lds_u32(w0), B0 = lds_u32(w0 + 4u), C0 = lds_u32(w0 + 8u);
    const uint32_t A1 = lds_u32(w1), B1 = lds_u32(w1 + 4u), C1 = lds_u32(w1 + 8u);
    const uint32_t scw0 = lds_u32(sc0p + 4u * m), scw1 = lds_u32(sc1p + 4u * m);
    uint32_t op0[4], op1[4];
    op0[0] = (A0 & 0x0F0F0F0Fu) | (C0 & 0x30303030u);
    op0[1] = ((A0 >> 4) & 0x0F0F0F0Fu) | ((C0 >> 2) & 0x30303030u);
    op0[2] = (B0 & 0x0F0F0F0Fu) | ((C0 << 4) & 0x30303030u);
    op0[3] = ((B0 >> 4) & 0x0F0F0F0Fu) | ((C0 << 2) & 0x30303030u);
    op1[0] = (A1 & 0x0F0F0F0Fu) | (C1 & 0x30303030u);
    op1[1] = ((A1 >> 4) & 0x0F0F0F0Fu) | ((C1 >> 2) & 0x30303030u);
    op1[2] = (B1 & 0x0F0F0F0Fu) | ((C1 << 4) & 0x30303030u);
    op1[3] = ((B1 >> 4) & 0x0F0F0F0Fu) | ((C1 << 2) & 0x30303030u);
#pragma unroll
    for (int s = 0; s < 4; ++s) {
      const int j = 4 * m + s;  // sub-block of 16 weights
      const int s0 = byte_s(scw0, s), s1 = byte_s(scw1, s);
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        const uint32_t b0 = lds_u32_if(dl[nt] + (uint32_t)(colg + 16 * j), live[nt]);
        int32_t C[4] = {0, 0, 0, 0};
        mma_u8s8_k16(C, op0[s], op1[s], b0);
        ai[nt][0] += s0 * C[0];
        ai[nt][1] += s0 * C[1];
        ai[nt][2] += s1 * C[2];
        ai[nt][3] += s1 * C[3];
        ao[nt][0] += s0 * X[nt][j & 7];
        ao[nt][1] += s1 * X[nt][j & 7];
      }
    }
  }
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    const float isc = lds_f32(iscale + 4u * (uint32_t)((4 * nt + t) * iscale_row(gstride) + gi));
    const float v0 = fmaf(256.f, (float)ai[nt][0], fmaf(-32.f, (float)ao[nt][0], (float)ai[nt][1]));
    const float v1 = fmaf(256.f, (float)ai[nt][2], fmaf(-32.f, (float)ao[nt][1], (float)ai[nt][3]));
    acc[nt][0] = fmaf(isc * d0, v0, acc[nt][0]);
    acc[nt][1] = fmaf(isc * d1, v1, acc[nt][1]);
  }
}

// One tile for one warp (rows row0 / row1 of the 64 per lane): TSB Q4_K super-blocks, the
// tile's first at super-block s0 of the slice.
template <int NT, int TSB>
__device__ __forceinline__ void tile_q4(uint32_t stage, const uint32_t (&dl)[NT], const bool (&live)[NT],
                                        uint32_t iscale, uint32_t gsum, int gstride, int s0, int row0, int row1, int t,
                                        float (&acc)[NT][2]) {
#pragma unroll
  for (int k = 0; k < TSB; ++k) {
    const uint32_t blk = stage + (uint32_t)(64 * 144 * k);
#pragma unroll
    for (int half = 0; half < 2; ++half)
      q4k_half<NT>(blk + 144u * row0, blk + 144u * row1, half, dl, live, 256 * (s0 + k), iscale, gsum, gstride,
                   2 * (s0 + k) + half, t, acc);
  }
}

template <int NT>
__device__ __forceinline__ void tile_q6(uint32_t stage, const uint32_t (&dl)[NT], const bool (&live)[NT],
                                        uint32_t iscale, uint32_t gsum, int gstride, int s0, int row0, int row1, int t,
                                        float (&acc)[NT][2]) {
#pragma unroll
  for (int half = 0; half < 2; ++half)
    q6k_half<NT>(stage + 210u * row0, stage + 210u * row1, row0 & 1, row1 & 1, half, dl, live, 256 * s0, iscale,
                 gsum, gstride, 2 * s0 + half, t, acc);
}

template <int MAXP, int NT>
__global__ void __launch_bounds__(kThreads, 1) kquant_gemv_kernel(const __grid_constant__ Args<MAXP> a) {
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ __align__(8) uint64_t full_bar[kStages], empty_bar[kStages];
  __shared__ Slot slots[kMaxSlots];
  __shared__ int s_ticket[kTeams];
  __shared__ int s_nslots;

  pdl_release();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int u_begin = a.cta_begin[blockIdx.x], u_end = a.cta_begin[blockIdx.x + 1];
  if (u_begin >= u_end) return;
  const int nunits = u_end - u_begin;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], kTeamWarps);
    }
    fence_mbar_init();
  }
  if (warp == 0) {
    // Slot table: lane i fills slot i, the i-th (problem, slice) pair from the CTA's first one
    // (a multi-problem launch has one slice per problem); digit areas laid out back to back.
    const uint32_t base = smem_u32(smem + kStages * kStageBytes);
    const int s0 = a.cta_slice[blockIdx.x] >> 7, nsl_cta = a.cta_slice[blockIdx.x] & 127;
    uint32_t carry = 0;
    int items = 0, n = 0;
    for (int i0 = 0; i0 < nsl_cta; i0 += 32) {
      const int i = i0 + lane;
      const bool live = i < nsl_cta;
      Slot sl;
      uint32_t bytes = 0;
      int nit = 0;
      if (live) {
        const int p = (a.nproblems == 1) ? 0 : s0 + i;
        const int j = (a.nproblems == 1) ? s0 + i : 0;
        const Problem& P = a.p[p];
        const int slice_start = P.unit_begin + j * P.nblocks;
        const int first = max(slice_start, u_begin);
        sl.p = p;
        sl.j = j;
        sl.u0 = first - u_begin;
        sl.u1 = min(u_end, slice_start + P.nblocks) - u_begin;
        sl.b0 = first - slice_start;
        sl.nblocks = P.nblocks;
        sl.nsb = P.nsb;
        sl.nsbs = slice_nsb(P, j);
        sl.slices = P.slices;
        sl.sbfirst = j * P.slice_sb;
        sl.type = P.type;
        sl.ngroups = 2 * sl.nsbs;
        sl.stride = digit_stride(sl.ngroups);
        sl.blocks = P.blocks;
        sl.x = P.x;
        sl.y = P.y;
        sl.partial = P.partial;
        sl.tickets = P.tickets;
        bytes = (uint32_t)slot_area(a.batch, NT, sl.ngroups);
        nit = a.batch * sl.ngroups;
      }
      uint32_t incl = bytes;
      int iincl = nit;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t v = __shfl_up_sync(0xffffffffu, incl, o);
        const int w = __shfl_up_sync(0xffffffffu, iincl, o);
        if (lane >= o) {
          incl += v;
          iincl += w;
        }
      }
      if (live) {
        sl.digits = base + carry + incl - bytes;
        sl.iscale = sl.digits + (uint32_t)(4 * a.batch * sl.stride);
        sl.gsum = sl.iscale + (uint32_t)iscale_area(NT, sl.ngroups);
        sl.it0 = items + iincl - nit;
        slots[i] = sl;
      }
      carry += __shfl_sync(0xffffffffu, incl, 31);
      items += __shfl_sync(0xffffffffu, iincl, 31);
      n += __popc(__ballot_sync(0xffffffffu, live));
    }
    if (lane == 0) s_nslots = n;
  }
  __syncthreads();
  pdl_wait();  // everything above read only the parameters

  // Team t (producer warp t and consumer warps 4t..4t+3) walks units t, t + kTeams, ... of the
  // range; both sides derive the same tile sequence from the slot table, so the only hand-offs
  // are the full / empty barriers of the team's two stages. The producers start copying once
  // every consumer has issued its activation reads (kBarX), so those small reads do not queue
  // behind the weight stream.
  const int nsl = s_nslots;
  if (warp >= kConsumerWarps) {
    // ---------------------------------------------------------------- producer warps
    named_bar(kBarX, kThreads);
    if (lane != 0) return;
    const int team = warp - kConsumerWarps;
    int issued = 0, si = 0;
    for (int k = team; k < nunits; k += kTeams) {
      while (si + 1 < nsl && k >= slots[si].u1) ++si;
      const Slot& sl = slots[si];
      const int b = sl.b0 + (k - sl.u0);
      const int rec = rec_bytes(sl.type), tsbm = tile_sb(sl.type);
      const uint8_t* src = sl.blocks + ((size_t)b * sl.nsb + sl.sbfirst) * 64u * rec;
      for (int s0 = 0; s0 < sl.nsbs; s0 += tsbm) {
        const int tsb = min(tsbm, sl.nsbs - s0);
        const int s = kTeamStages * team + (issued % kTeamStages);
        if (issued >= kTeamStages &&
            !mbar_wait(&empty_bar[s], (uint32_t)((issued / kTeamStages - 1) & 1))) {
          atomicExch(&g_error, 1);
          return;
        }
        const uint32_t bytes = (uint32_t)(tsb * 64 * rec);
        mbar_expect_tx(&full_bar[s], bytes);
        bulk_g2s(smem + s * kStageBytes, src + (size_t)s0 * 64u * rec, bytes, &full_bar[s]);
        ++issued;
      }
    }
    return;
  }

  // ------------------------------------------------------------------ consumer warps
  // 1. activation digits of every (problem, slice) the range touches
  build_digits(slots, nsl, a.batch, 4 * NT, threadIdx.x, kConsumers);
  named_bar(kBarDigits, kConsumers);

  // 2. team loop
  const int team = warp / kTeamWarps, mt = warp % kTeamWarps;
  const int tt = threadIdx.x % kTeamThreads;
  const int g = lane >> 2, t = lane & 3;
  const uint32_t smem_base = smem_u32(smem);
  uint32_t dl[NT];
  bool live[NT];
  int row0 = 0, row1 = 0;
  int cur_slot = -1, si = 0, used = 0;
  // failed: a wait of this warp ran out. From then on the warp skips its waits and its math but
  // still takes every team barrier below, so no named barrier is left short of a participant;
  // the outputs are not valid and the error word says so.
  bool failed = false;
  for (int k = team; k < nunits; k += kTeams) {
    while (si + 1 < nsl && k >= slots[si].u1) ++si;
    const Slot& sl = slots[si];
    const int b = sl.b0 + (k - sl.u0);
    const bool q4 = sl.type == FL_GGML_Q4_K;
    if (si != cur_slot) {
      cur_slot = si;
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        const int row = 8 * nt + g;  // digit row (4 per batch row) this lane's B fragment reads
        live[nt] = row < 4 * a.batch;
        dl[nt] = sl.digits + (uint32_t)(min(row, 4 * a.batch - 1) * sl.stride) + (q4 ? 8u * t : 4u * t);
      }
      row0 = q4 ? 16 * mt + g : q6_row(mt, 0, g);
      row1 = q4 ? 16 * mt + g + 8 : q6_row(mt, 1, g);
    }
    const uint32_t iscale = sl.iscale, gsum = sl.gsum;
    const int gstride = sl.ngroups;
    float acc[NT][2];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) acc[nt][0] = acc[nt][1] = 0.f;
    const int tsbm = q4 ? 2 : 1;
    for (int s0 = 0; s0 < sl.nsbs; s0 += tsbm) {
      const int s = kTeamStages * team + (used % kTeamStages);
      ++used;
      if (failed) continue;
      if (!__all_sync(0xffffffffu, mbar_wait(&full_bar[s], (uint32_t)(((used - 1) / kTeamStages) & 1)))) {
        if (lane == 0) atomicExch(&g_error, 2);
        failed = true;
        continue;
      }
      const uint32_t stage = smem_base + s * kStageBytes;
      if (!q4)
        tile_q6<NT>(stage, dl, live, iscale, gsum, gstride, s0, row0, row1, t, acc);
      else if (s0 + 2 <= sl.nsbs)
        tile_q4<NT, 2>(stage, dl, live, iscale, gsum, gstride, s0, row0, row1, t, acc);
      else
        tile_q4<NT, 1>(stage, dl, live, iscale, gsum, gstride, s0, row0, row1, t, acc);
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty_bar[s]);
    }

    // ---- unit done: this warp's 16 rows are final (or a slice partial). Lane t holds digit
    // pair t & 1 of batch row 2 nt + t / 2; the pairs' sums meet in one shuffle and the even
    // lane writes.
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      acc[nt][0] += __shfl_xor_sync(0xffffffffu, acc[nt][0], 1);
      acc[nt][1] += __shfl_xor_sync(0xffffffffu, acc[nt][1], 1);
    }
    const size_t ystride = (size_t)64 * sl.nblocks;
    if (sl.slices == 1) {
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        const int bb = 2 * nt + (t >> 1);
        if ((t & 1) == 0 && bb < a.batch) {
          float* yb = sl.y + (size_t)bb * ystride + 64 * b;
          yb[row0] = acc[nt][0];
          yb[row1] = acc[nt][1];
        }
      }
    } else {
      // partial for this slice; the last team to finish the block adds the slices in order
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        const int bb = 2 * nt + (t >> 1);
        if ((t & 1) == 0 && bb < a.batch) {
          float* pp = sl.partial + (((size_t)sl.j * sl.nblocks + b) * a.batch + bb) * 64;
          pp[row0] = acc[nt][0];
          pp[row1] = acc[nt][1];
        }
      }
      // The barrier orders the team's partial stores before thread 0's acquire-release ticket
      // (release is cumulative); the last team's reads follow the ticket's acquire.
      named_bar(kBarTeam0 + team, kTeamThreads);
      if (tt == 0) s_ticket[team] = (int)atom_add_acq_rel(&sl.tickets[b], 1u);
      named_bar(kBarTeam0 + team, kTeamThreads);
      if (s_ticket[team] == sl.slices - 1) {
        if (a.batch * 64 <= kTeamThreads) {  // one output per thread at most
          const int e = tt;
          if (e < a.batch * 64) {
            float sum = 0.f;
#pragma unroll 4
            for (int jj = 0; jj < sl.slices; ++jj)
              sum += __ldcg(sl.partial + (((size_t)jj * sl.nblocks + b) * a.batch + e / 64) * 64 + e % 64);
            sl.y[(size_t)(e / 64) * ystride + 64 * b + e % 64] = sum;
          }
        } else
        // each thread's outputs (up to kRed) and slices: every load is issued before the sums
        for (int e0 = tt; e0 < a.batch * 64; e0 += kRed * kTeamThreads) {
          float sum[kRed];
#pragma unroll
          for (int q = 0; q < kRed; ++q) sum[q] = 0.f;
          for (int jj = 0; jj < sl.slices; ++jj) {
            float v[kRed];
#pragma unroll
            for (int q = 0; q < kRed; ++q) {
              const int e = e0 + q * kTeamThreads;
              v[q] = (e < a.batch * 64)
                         ? __ldcg(sl.partial + (((size_t)jj * sl.nblocks + b) * a.batch + e / 64) * 64 + e % 64)
                         : 0.f;
            }
#pragma unroll
            for (int q = 0; q < kRed; ++q) sum[q] += v[q];
          }
#pragma unroll
          for (int q = 0; q < kRed; ++q) {
            const int e = e0 + q * kTeamThreads;
            if (e < a.batch * 64) sl.y[(size_t)(e / 64) * ystride + 64 * b + e % 64] = sum[q];
          }
        }
        if (tt == 0) sl.tickets[b] = 0u;
      }
      named_bar(kBarTeam0 + team, kTeamThreads);
    }
  }
}

// ---------------------------------------------------------------- host side

struct Plan {
  int slices, slice_sb;
};

// Shared memory of one slot's activation digits, scales and 16-column sums.
// N-tiles of the products: two digit pairs per batch row, four pairs per 8-column N-tile.
__host__ __device__ constexpr int ntiles(int batch) { return (batch + 1) / 2; }

static size_t slot_bytes(int batch, int nsbs) { return (size_t)slot_area(batch, ntiles(batch), 2 * nsbs); }

// Widest column slice (in super-blocks) whose digits fit in one slot.
static int max_sb_fit(int batch) {
  int s = 1;
  while (slot_bytes(batch, s + 1) <= (size_t)kDigitBudget) ++s;
  return s;
}

// Column split for a single tensor: enough units to fill the GPU, slices of whole
// super-blocks, and a slice narrow enough for the activation digits to fit in smem.
static Plan plan_single(int nblocks, int nsb, int batch, int nsm) {
  Plan pl;
  const int max_sb = max_sb_fit(batch);
  const int s_mem = (nsb + max_sb - 1) / max_sb;
  const int s_fill = (2 * nsm + nblocks - 1) / nblocks;
  int s = std::max(s_mem, std::min(s_fill, std::max(1, nsb / 4)));
  s = std::min(s, nsb);
  pl.slice_sb = (nsb + s - 1) / s;
  pl.slices = (nsb + pl.slice_sb - 1) / pl.slice_sb;
  return pl;
}

static size_t workspace_for(const Plan& pl, int nblocks, int batch) {
  if (pl.slices <= 1) return 0;
  const size_t tickets = ((size_t)nblocks * 4 + 255) / 256 * 256;
  return tickets + (size_t)pl.slices * nblocks * batch * 64 * 4;
}

// Contiguous byte-balanced unit ranges, one per CTA. A range is also closed early when the
// digits of its distinct (problem, slice) pairs would overflow shared memory or at kMaxSlots
// pairs; after every cut the cost still to place is spread evenly over the ranges still to
// make, so an early cut does not leave a later range oversized. Cuts can still make more
// ranges than SMs (a second, partial wave) when memory forces more than that.
template <int MAXP>
static bool partition(Args<MAXP>& a, int nsm) {
  double total = 0;
  for (int i = 0; i < a.nproblems; ++i) total += (double)a.p[i].nblocks * a.p[i].nsb * rec_bytes(a.p[i].type);
  const Problem& L = a.p[a.nproblems - 1];
  const int units = L.unit_begin + L.nblocks * L.slices;
  const int target = std::max(1, std::min(nsm, units));
  double per_cta = total / target;
  double start = 0;  // cumulative cost where the current range began
  int n = 0;
  a.cta_begin[0] = 0;
  a.cta_slice[0] = 0;
  double acc = 0;
  size_t dig = 0;
  int nslots = 0, count = 0;
  for (int i = 0; i < a.nproblems; ++i) {
    const Problem& P = a.p[i];
    for (int j = 0; j < P.slices; ++j) {
      const int ns = std::min(P.slice_sb, P.nsb - j * P.slice_sb);
      const size_t sb = slot_bytes(a.batch, ns);
      const double cost = (double)ns * rec_bytes(P.type);
      for (int b = 0; b < P.nblocks; ++b) {
        const int u = P.unit_begin + j * P.nblocks + b;
        bool cut = false;
        if (count > 0) {
          if (n + 1 < target && acc + 0.5 * cost - start > per_cta) cut = true;
          if (b == 0 && (dig + sb > (size_t)kDigitBudget || nslots == kMaxSlots)) cut = true;
        }
        if (cut) {
          if (n + 1 >= kMaxCtas) return false;
          a.cta_slice[n] |= nslots;
          a.cta_begin[++n] = u;
          a.cta_slice[n] = ((a.nproblems == 1) ? j : i) << 7;
          dig = 0;
          nslots = 0;
          count = 0;
          start = acc;
          per_cta = (total - acc) / std::max(1, target - n);
        }
        if (b == 0 || count == 0) {
          dig += sb;
          ++nslots;
        }
        acc += cost;
        ++count;
      }
    }
  }
  a.cta_slice[n] |= nslots;
  a.cta_begin[++n] = units;
  a.ncta = n;
  return true;
}

template <int MAXP, int NT>
static fl_status launch(const Args<MAXP>& a, cudaStream_t st) {
  const size_t smem = (size_t)kSmemLimit;
  auto kern = kquant_gemv_kernel<MAXP, NT>;
  FL_CHECK_CUDA(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem),
                "cudaFuncSetAttribute(kquant_gemv)");
  FL_CHECK_CUDA(launch_pdl(kern, dim3(a.ncta), dim3(kThreads), smem, st, 1, a), "launch kquant_gemv");
  return FL_OK;
}

template <int MAXP>
static fl_status launch_nt(const Args<MAXP>& a, cudaStream_t st) {
  switch (ntiles(a.batch)) {
    case 1: return launch<MAXP, 1>(a, st);
    case 2: return launch<MAXP, 2>(a, st);
    case 3: return launch<MAXP, 3>(a, st);
    case 4: return launch<MAXP, 4>(a, st);
    case 5: return launch<MAXP, 5>(a, st);
    case 6: return launch<MAXP, 6>(a, st);
    case 7: return launch<MAXP, 7>(a, st);
    default: return launch<MAXP, 8>(a, st);
  }
}

static fl_status check_tensor(const void* blocks, int type, int out, int in, const char* what, int idx) {
  if (type != FL_GGML_Q4_K && type != FL_GGML_Q6_K)
    return fail(FL_ERR_UNSUPPORTED, "%s: tensor %d has GGUF type %d; the fast path implements Q4_K (12) and Q6_K (14)",
                what, idx, type);
  if (!blocks) return fail(FL_ERR_ARG, "%s: tensor %d blocks pointer is NULL", what, idx);
  if (out <= 0 || out % 64 || in <= 0 || in % 256)
    return fail(FL_ERR_SHAPE, "%s: tensor %d out=%d in=%d (out %% 64 == 0, in %% 256 == 0)", what, idx, out, in);
  if (!aligned16(blocks)) return fail(FL_ERR_ALIGN, "%s: tensor %d blocks not 16-byte aligned", what, idx);
  return FL_OK;
}

}  // namespace kq
}  // namespace fl

namespace fl {
namespace kq {

// Reads and clears the error word (-1 if that fails).
int take_device_error() {
  int v = 0, z = 0;
  if (cudaMemcpyFromSymbol(&v, g_error, sizeof(int)) != cudaSuccess) return -1;
  if (v != 0 && cudaMemcpyToSymbol(g_error, &z, sizeof(int)) != cudaSuccess) return -1;
  return v;
}

}  // namespace kq
}  // namespace fl

using namespace fl;

extern "C" size_t fl_kquant_bytes(int ggml_type, int out, int in) {
  if (out <= 0 || in <= 0 || in % 256) return 0;
  if (ggml_type == FL_GGML_Q4_K) return (size_t)out * (in / 256) * 144u;
  if (ggml_type == FL_GGML_Q6_K) return (size_t)out * (in / 256) * 210u;
  return 0;
}

extern "C" size_t fl_kquant_workspace_bytes(int ggml_type, int out, int in, int batch) {
  if (ggml_type != FL_GGML_Q4_K && ggml_type != FL_GGML_Q6_K) return 0;
  if (out <= 0 || out % 64 || in <= 0 || in % 256 || batch < 1 || batch > FL_MAX_BATCH) return 0;
  const int nsm = device_sm_count();
  if (nsm <= 0) return 0;
  kq::Plan pl = kq::plan_single(out / 64, in / 256, batch, nsm);
  return kq::workspace_for(pl, out / 64, batch);
}

extern "C" fl_status fl_gemv_kquant(const void* blocks, int ggml_type, int out, int in, const uint16_t* x, int batch,
                                    float* y, void* workspace, size_t workspace_bytes, void* stream) {
  const char* what = "fl_gemv_kquant";
  fl_status st = kq::check_tensor(blocks, ggml_type, out, in, what, 0);
  if (st != FL_OK) return st;
  if (!x || !y) return fail(FL_ERR_ARG, "%s: NULL x/y", what);
  if (reinterpret_cast<uintptr_t>(y) & 3u) return fail(FL_ERR_ALIGN, "%s: y not 4-byte aligned", what);
  if (batch < 1 || batch > FL_MAX_BATCH) return fail(FL_ERR_SHAPE, "%s: batch=%d (1..16)", what, batch);
  if (!aligned16(x)) return fail(FL_ERR_ALIGN, "%s: x not 16-byte aligned", what);
  const int nsm = device_sm_count();
  if (nsm <= 0) return fail(FL_ERR_CUDA, "%s: no CUDA device", what);
  const int nblocks = out / 64, nsb = in / 256;
  kq::Plan pl = kq::plan_single(nblocks, nsb, batch, nsm);
  const size_t need = kq::workspace_for(pl, nblocks, batch);
  if (need > 0 && (!workspace || workspace_bytes < need))
    return fail(FL_ERR_WORKSPACE, "%s: workspace %zu bytes, need %zu", what, workspace ? workspace_bytes : (size_t)0,
                need);
  if (need > 0 && !aligned16(workspace)) return fail(FL_ERR_ALIGN, "%s: workspace not 16-byte aligned", what);
  static thread_local kq::Args<1> a;
  a.nproblems = 1;
  a.batch = batch;
  kq::Problem& P = a.p[0];
  P.blocks = static_cast<const uint8_t*>(blocks);
  P.x = x;
  P.y = y;
  P.type = ggml_type;
  P.nblocks = nblocks;
  P.nsb = nsb;
  P.slices = pl.slices;
  P.slice_sb = pl.slice_sb;
  P.unit_begin = 0;
  if (pl.slices > 1) {
    const size_t tick = ((size_t)nblocks * 4 + 255) / 256 * 256;
    P.tickets = static_cast<uint32_t*>(workspace);
    P.partial = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + tick);
  } else {
    P.tickets = nullptr;
    P.partial = nullptr;
  }
  if (!kq::partition(a, nsm)) return fail(FL_ERR_SHAPE, "%s: tensor too large for one launch", what);
  return kq::launch_nt(a, static_cast<cudaStream_t>(stream));
}

extern "C" fl_status fl_gemv_kquant_batched(const fl_kquant_problem* problems, int n, int batch, void* stream) {
  const char* what = "fl_gemv_kquant_batched";
  if (!problems) return fail(FL_ERR_ARG, "%s: problems is NULL", what);
  if (n < 1 || n > FL_MAX_PROBLEMS) return fail(FL_ERR_ARG, "%s: n=%d (1..%d)", what, n, FL_MAX_PROBLEMS);
  if (batch < 1 || batch > FL_MAX_BATCH) return fail(FL_ERR_SHAPE, "%s: batch=%d (1..16)", what, batch);
  static thread_local kq::Args<FL_MAX_PROBLEMS> a;
  a.nproblems = n;
  a.batch = batch;
  int unit = 0;
  for (int i = 0; i < n; ++i) {
    const fl_kquant_problem& q = problems[i];
    fl_status st = kq::check_tensor(q.blocks, q.ggml_type, q.out, q.in, what, i);
    if (st != FL_OK) return st;
    if (!q.x || !q.y) return fail(FL_ERR_ARG, "%s: tensor %d NULL x/y", what, i);
    if (reinterpret_cast<uintptr_t>(q.y) & 3u) return fail(FL_ERR_ALIGN, "%s: tensor %d y not 4-byte aligned", what, i);
    if (!aligned16(q.x)) return fail(FL_ERR_ALIGN, "%s: tensor %d x not 16-byte aligned", what, i);
    const int nsb = q.in / 256;
    if (nsb > kq::max_sb_fit(batch))
      return fail(FL_ERR_SHAPE, "%s: tensor %d in=%d too wide for batch %d in one launch (in <= %d)", what, i, q.in,
                  batch, 256 * kq::max_sb_fit(batch));
    kq::Problem& P = a.p[i];
    P.blocks = static_cast<const uint8_t*>(q.blocks);
    P.x = q.x;
    P.y = q.y;
    P.partial = nullptr;
    P.tickets = nullptr;
    P.type = q.ggml_type;
    P.nblocks = q.out / 64;
    P.nsb = nsb;
    P.slices = 1;
    P.slice_sb = nsb;
    P.unit_begin = unit;
    unit += P.nblocks;
  }
  const int nsm = device_sm_count();
  if (nsm <= 0) return fail(FL_ERR_CUDA, "%s: no CUDA device", what);
  if (!kq::partition(a, nsm)) return fail(FL_ERR_SHAPE, "%s: tensors too large for one launch", what);
  return kq::launch_nt(a, static_cast<cudaStream_t>(stream));
}
