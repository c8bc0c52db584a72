// In-pass level decision ("FoQLens" landing page, FoQZones mechanism: the layer decides
// for itself from what has just entered it; score, reduced score, a ladder of thresholds
// lambda 16^j capped at kappa, or the top share f of the layer by reduced score).
//
// The score is the draft variant: a layer read at the base level gamma shows which of its
// 64-row blocks carry the step. For block c of a layer with `in` columns:
//   s_c = ||y_c||^2 * D_c^2   (y_c: the block's base-level outputs, every batch row)
//   D_c^2 = mean over the block's rows and 128-column groups of (scale * 2^(8 - 2 gamma))^2
//   r_c = s_c * D_c^2 / (64 in)
//   ladder: level = gamma + #{ j >= 1 : r_c >= lambda 16^j }, at most kappa
//   share:  the floor(f * nblocks) blocks with the largest r_c (equal r_c: lower index
//           first) rise to kappa, the rest stay at gamma.
// The decided levels feed the residual pass (from gamma to the decided level), so a layer
// is read once at the base and only its lifted blocks' low planes are read again.
//
// Kernels. score_kernel: one warp per block, every block of every problem in one grid; the
// warp streams the block's 64 G scales (the head of the block in the plane store) and its
// 64 outputs per batch row, reduces both in a fixed shuffle order, and writes the reduced
// score (and, for the ladder, the level). share_kernel (share rule only): one CTA per
// problem picks the floor(f n) largest keys (score bits, then the complemented index, so
// equal scores rank the lower index first). A layer of up to 256 blocks is ranked by one
// warp (every key against every other, no barrier); a larger one by an 8-bit radix select
// over the 64-bit keys with per-warp shared-memory histograms, its scores staged in shared
// memory up to 7,680 blocks. It then writes every block's level and, when asked, the lifted
// blocks' indices in ascending order (a block-wide scan per 512 blocks).
// score_select_kernel (share rule with caller counters, one launch): CTAs score contiguous
// chunks of blocks and count them per layer; the CTA that completes a layer's count runs the
// same selection with its 256 threads. On the 197-layer decode step it measured slower than
// the two launches (16.4 against 11.4 us): the head layer's selection then starts only after
// the last chunk is scored and runs on half the threads.
#include <math.h>

#include "fl_common.cuh"

namespace fl {
namespace decide {

constexpr int kWarps = 8;          // blocks per CTA of the score kernel
constexpr int kShareThreads = 512;

struct Problem {
  const uint8_t* store;
  const float* y;
  uint8_t* levels;
  float* score;
  int32_t* lifted;                 // share rule: ascending indices of the lifted blocks (or NULL)
  int out;
  int G;
  int block_begin;                 // first global block index of this problem
  int n_up;                        // share rule: blocks that rise
};

template <int MAXP>
struct Args {
  Problem p[MAXP];
  int nproblems;
  int nblocks;                     // total over the problems
  int batch;
  int rule;
  int gamma;
  int kappa;
  float lambda;
  float step2;                     // (2^(8 - 2 gamma))^2
  int32_t* counters;               // share rule in one launch: blocks scored per problem (or NULL)
  int chunk;                       // blocks per CTA of the one-launch variant
};

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

constexpr int kWarpRank = 256;     // layers up to this many blocks: one warp ranks the keys
constexpr int kSmemScores = 7680;   // a layer's scores staged in shared memory up to this many blocks (30 KB)

// key of block i: larger score first, then the lower index (scores are >= 0, so their bit
// patterns order like their values). Scores may have been written by other CTAs of the same
// launch: they are read at L2 (`ld.global.cg`), never from a CTA's own L1.
__device__ __forceinline__ uint64_t share_key(const float* score, int i) {
  return ((uint64_t)__float_as_uint(__ldcg(score + i)) << 32) | (uint32_t)(0xFFFFFFFFu - (uint32_t)i);
}
__device__ __forceinline__ uint64_t share_key_smem(const float* score, int i) {
  return ((uint64_t)__float_as_uint(score[i]) << 32) | (uint32_t)(0xFFFFFFFFu - (uint32_t)i);
}

template <int T>
struct ShareSmem {
  uint32_t hist[T / 32][256];  // one histogram per warp: positive scores share their top bits,
                               // so one shared bin would serialise
  uint64_t prefix;
  uint32_t left, tied;
  int warp_up[T / 32];
};

// The share rule for problem P by all T threads of a CTA: the floor(f n) largest keys rise to
// kappa. s_score: dynamic shared memory for up to kSmemScores staged scores.
template <int T>
__device__ void select_share(const Problem& P, int gamma, int kappa, float* s_score, ShareSmem<T>& sm, int tid) {
  constexpr int W = T / 32;
  const int nb = P.out / 64;
  const float* score = P.score;
  if (nb <= kWarpRank) {
    // small layer: one warp ranks every key against all others (keys are distinct, so a key
    // rises iff fewer than n_up keys exceed it); no block-wide barrier
    if (tid >= 32) return;
    uint64_t key[kWarpRank / 32];
#pragma unroll
    for (int m = 0; m < kWarpRank / 32; ++m) {
      const int i = 32 * m + tid;
      key[m] = i < nb ? share_key(score, i) : 0ull;
    }
    int above[kWarpRank / 32] = {};
#pragma unroll
    for (int m2 = 0; m2 < kWarpRank / 32; ++m2) {
      if (32 * m2 >= nb) break;
      for (int src = 0; src < 32; ++src) {
        const uint64_t kj = __shfl_sync(0xffffffffu, key[m2], src);
        if (32 * m2 + src < nb) {
#pragma unroll
          for (int m = 0; m < kWarpRank / 32; ++m) above[m] += kj > key[m];
        }
      }
    }
    int base = 0;
#pragma unroll
    for (int m = 0; m < kWarpRank / 32; ++m) {
      const int i = 32 * m + tid;
      const bool up = i < nb && above[m] < P.n_up;
      if (i < nb) P.levels[i] = (uint8_t)(up ? kappa : gamma);
      const unsigned bal = __ballot_sync(0xffffffffu, up);
      if (up && P.lifted) P.lifted[base + __popc(bal & ((1u << tid) - 1u))] = i;
      base += __popc(bal);
    }
    return;
  }
  const bool staged = nb <= kSmemScores;
  if (staged) {
    for (int i = tid; i < nb; i += T) s_score[i] = __ldcg(score + i);
    __syncthreads();
  }
  auto key_of = [&](int i) { return staged ? share_key_smem(s_score, i) : share_key(score, i); };
  uint64_t kth = 0;                         // with 0 < n_up < nb: the keys >= kth rise
  if (P.n_up > 0 && P.n_up < nb) {
    if (tid == 0) {
      sm.prefix = 0;
      sm.left = (uint32_t)P.n_up;
    }
    // radix select of the n_up-th largest key, 8 bits a pass from the top; the four passes
    // over the score bits settle it unless the cut falls inside a group of equal scores,
    // which the four passes over the index bits then split lower index first
    for (int pass = 0; pass < 8; ++pass) {
      const int shift = 56 - 8 * pass;
      for (int d = tid; d < W * 256; d += T) (&sm.hist[0][0])[d] = 0;
      __syncthreads();
      const uint64_t prefix = sm.prefix;
      const uint64_t mask = pass == 0 ? 0ull : (~0ull << (shift + 8));
      uint32_t* const my = sm.hist[tid >> 5];
      for (int i = tid; i < nb; i += T) {
        const uint64_t k = key_of(i);
        if ((k & mask) == prefix) atomicAdd(&my[(k >> shift) & 255u], 1u);
      }
      __syncthreads();
      for (int d = tid; d < 256; d += T) {
        uint32_t sum = 0;
#pragma unroll
        for (int w = 0; w < W; ++w) sum += sm.hist[w][d];
        sm.hist[0][d] = sum;
      }
      __syncthreads();
      if (tid < 32) {
        // lane l owns digits 255 - 8 l down to 248 - 8 l; find the digit where the count of
        // larger keys first reaches left
        uint32_t cnt[8], tot = 0;
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          cnt[k] = sm.hist[0][255 - 8 * tid - k];
          tot += cnt[k];
        }
        uint32_t before = tot;              // inclusive scan over lanes, then exclusive
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const uint32_t v = __shfl_up_sync(0xffffffffu, before, o);
          if (tid >= o) before += v;
        }
        before -= tot;
        const uint32_t left = sm.left;
        const bool mine = before < left && left <= before + tot;
        if (mine) {
          uint32_t acc = before;
          int k = 0;
          while (acc + cnt[k] < left) acc += cnt[k++];
          const uint32_t digit = 255u - 8u * tid - (uint32_t)k;
          sm.prefix = prefix | ((uint64_t)digit << shift);
          sm.left = left - acc;
          sm.tied = cnt[k];
        }
      }
      __syncthreads();
      if (pass == 3 && sm.left == sm.tied) break;   // every key with the cut's score rises
    }
    kth = sm.prefix;
  }
  // levels, and the lifted indices in ascending order (a block-wide scan per T blocks)
  int base = 0;
  for (int i0 = 0; i0 < nb; i0 += T) {
    const int i = i0 + tid;
    const bool up = i < nb && (P.n_up >= nb || (P.n_up > 0 && key_of(i) >= kth));
    if (i < nb) P.levels[i] = (uint8_t)(up ? kappa : gamma);
    if (P.lifted == nullptr) continue;
    const unsigned bal = __ballot_sync(0xffffffffu, up);
    if ((tid & 31) == 0) sm.warp_up[tid >> 5] = __popc(bal);
    __syncthreads();
    int before = base, total = 0;
    for (int w = 0; w < W; ++w) {
      const int c = sm.warp_up[w];
      if (w < (tid >> 5)) before += c;
      total += c;
    }
    if (up) P.lifted[before + __popc(bal & ((1u << (tid & 31)) - 1u))] = i;
    base += total;
    __syncthreads();
  }
}

// The score of every block (one warp per block) and, for the ladder, its level. The fused
// variant (share rule, one launch): each CTA scores a contiguous chunk of a.chunk blocks, adds
// them to the counters of the layers they belong to, and the CTA whose addition completes a
// layer selects that layer's share at once (select_share with the CTA's 256 threads), then
// clears the counter.
constexpr int kMaxChunk = 64;   // blocks per CTA of the fused variant

// The problem holding global block gb: the last one whose block_begin <= gb.
template <int MAXP>
__device__ __forceinline__ int problem_of(const Args<MAXP>& a, int gb) {
  int lo = 0, hi = a.nproblems - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (a.p[mid].block_begin <= gb) lo = mid;
    else hi = mid - 1;
  }
  return lo;
}

template <int MAXP>
__device__ __forceinline__ void score_block(const Args<MAXP>& a, int gb, int lo, int lane) {
  const Problem& P = a.p[lo];
  const int c = gb - P.block_begin;
  // squared outputs of the block's 64 rows, every batch row, and squared scales of the
  // block ([G][64] fp32 at the head of its 8448 G bytes); loads issued four at a time
  float yy = 0.f, ss = 0.f;
  for (int t0 = 0; t0 < a.batch; t0 += 4) {
    float2 v[4];
#pragma unroll
    for (int u = 0; u < 4; ++u)
      v[u] = t0 + u < a.batch ? *reinterpret_cast<const float2*>(P.y + (size_t)(t0 + u) * P.out + 64 * c + 2 * lane)
                              : make_float2(0.f, 0.f);
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      yy = fmaf(v[u].x, v[u].x, yy);
      yy = fmaf(v[u].y, v[u].y, yy);
    }
  }
  const float4* s4 = reinterpret_cast<const float4*>(P.store + (size_t)c * 8448u * P.G);
  const int n4 = 16 * P.G;
  for (int i0 = 0; i0 < n4; i0 += 128) {
    float4 v[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int i = i0 + 32 * u + lane;
      v[u] = i < n4 ? __ldg(s4 + i) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      ss = fmaf(v[u].x, v[u].x, ss);
      ss = fmaf(v[u].y, v[u].y, ss);
      ss = fmaf(v[u].z, v[u].z, ss);
      ss = fmaf(v[u].w, v[u].w, ss);
    }
  }
  ss = warp_sum(ss);
  yy = warp_sum(yy);
  if (lane != 0) return;
  const float d2 = ss * a.step2 / (float)(64 * P.G);
  const float red = (yy * d2) * d2 / (float)(8192 * P.G);     // w_c = 64 * in = 8192 G
  if (P.score) P.score[c] = red;
  if (a.rule == 0) {
    int lev = a.gamma;
    float thr = a.lambda;
    for (int j = 1; j <= a.kappa - a.gamma; ++j) {
      thr *= 16.f;
      if (red >= thr) ++lev;
    }
    P.levels[c] = (uint8_t)lev;
  }
  if (a.counters) __threadfence();  // the score, device-wide, before the CTA's count
}

template <int MAXP>
__global__ void __launch_bounds__(32 * kWarps) score_kernel(const __grid_constant__ Args<MAXP> a) {
  pdl_release();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gb = blockIdx.x * kWarps + warp;
  if (gb >= a.nblocks) return;
  const int lo = problem_of(a, gb);  // parameters only: before the wait
  pdl_wait();
  score_block(a, gb, lo, lane);
}

template <int MAXP>
__global__ void __launch_bounds__(32 * kWarps) score_select_kernel(const __grid_constant__ Args<MAXP> a) {
  extern __shared__ float s_score[];             // the selected layer's staged scores
  __shared__ ShareSmem<32 * kWarps> sm;
  __shared__ int s_last[kMaxChunk];              // layers whose counts this CTA completed
  __shared__ int s_nlast;
  pdl_release();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int c0 = blockIdx.x * a.chunk, c1 = min(c0 + a.chunk, a.nblocks);
  pdl_wait();
  for (int gb = c0 + warp; gb < c1; gb += kWarps) score_block(a, gb, problem_of(a, gb), lane);
  __syncthreads();
  if (threadIdx.x == 0) {
    // the layers overlapping [c0, c1), from the one holding block c0
    const int lo = problem_of(a, c0);
    int n = 0;
    for (int p = lo; p < a.nproblems && a.p[p].block_begin < c1; ++p) {
      const int pb = a.p[p].block_begin, nb = a.p[p].out / 64;
      const int cnt = min(c1, pb + nb) - max(c0, pb);
      if (cnt > 0 && atomicAdd(&a.counters[p], cnt) + cnt == nb) s_last[n++] = p;
    }
    if (n) __threadfence();  // the other CTAs' scores are read after their counts
    s_nlast = n;
  }
  __syncthreads();
  for (int k = 0; k < s_nlast; ++k) {
    const int p = s_last[k];
    select_share<32 * kWarps>(a.p[p], a.gamma, a.kappa, s_score, sm, threadIdx.x);
    __syncthreads();
    if (threadIdx.x == 0) a.counters[p] = 0;
  }
}

template <int MAXP>
__global__ void __launch_bounds__(kShareThreads) share_kernel(const __grid_constant__ Args<MAXP> a) {
  extern __shared__ float s_score[];
  __shared__ ShareSmem<kShareThreads> sm;
  pdl_release();
  const Problem& P = a.p[blockIdx.x];
  pdl_wait();
  select_share<kShareThreads>(P, a.gamma, a.kappa, s_score, sm, threadIdx.x);
}

}  // namespace decide
}  // namespace fl

extern "C" fl_status fl_level_decide(const fl_decide_problem* problems, int n, int batch,
                                     const fl_decide_params* params, void* stream) {
  using namespace fl;
  using namespace fl::decide;
  const char* what = "fl_level_decide";
  if (!problems || !params) return fail(FL_ERR_ARG, "%s: NULL problems or params", what);
  if (n < 1 || n > FL_MAX_PROBLEMS) return fail(FL_ERR_ARG, "%s: n=%d (1..%d)", what, n, FL_MAX_PROBLEMS);
  if (batch < 1 || batch > FL_MAX_BATCH) return fail(FL_ERR_SHAPE, "%s: batch=%d (1..16)", what, batch);
  const fl_decide_params& q = *params;
  if (q.rule != FL_DECIDE_LADDER && q.rule != FL_DECIDE_SHARE)
    return fail(FL_ERR_ARG, "%s: rule=%d (0 ladder, 1 share)", what, q.rule);
  if (q.gamma < 1 || q.kappa < q.gamma || q.kappa > 4)
    return fail(FL_ERR_ARG, "%s: gamma=%d kappa=%d (1 <= gamma <= kappa <= 4)", what, q.gamma, q.kappa);
  if (q.rule == FL_DECIDE_LADDER && !(q.lambda >= 0.f && q.lambda <= 3.0e38f))
    return fail(FL_ERR_ARG, "%s: lambda=%g (finite, >= 0)", what, (double)q.lambda);
  if (q.rule == FL_DECIDE_SHARE && !(q.f >= 0.f && q.f <= 1.f))
    return fail(FL_ERR_ARG, "%s: f=%g (0..1)", what, (double)q.f);
  static thread_local Args<FL_MAX_PROBLEMS> a;
  a.nproblems = n;
  a.batch = batch;
  a.rule = q.rule;
  a.gamma = q.gamma;
  a.kappa = q.kappa;
  a.lambda = q.lambda;
  a.counters = q.rule == FL_DECIDE_SHARE ? q.counters : nullptr;
  if (reinterpret_cast<uintptr_t>(q.counters) & 3u) return fail(FL_ERR_ALIGN, "%s: counters not 4-byte aligned", what);
  const float step = (float)(1 << (8 - 2 * q.gamma));
  a.step2 = step * step;
  long blocks = 0;
  for (int i = 0; i < n; ++i) {
    const fl_decide_problem& p = problems[i];
    if (!p.w.store || !p.y || !p.levels) return fail(FL_ERR_ARG, "%s: problem %d has a NULL pointer", what, i);
    if (q.rule == FL_DECIDE_SHARE && !p.score)
      return fail(FL_ERR_ARG, "%s: problem %d: the share rule needs the score array", what, i);
    if (p.w.out <= 0 || p.w.in <= 0 || p.w.out % 64 || p.w.in % 128)
      return fail(FL_ERR_SHAPE, "%s: problem %d shape %dx%d (out %% 64 == 0, in %% 128 == 0)", what, i, p.w.out,
                  p.w.in);
    if (!aligned16(p.w.store)) return fail(FL_ERR_ALIGN, "%s: problem %d store not 16-byte aligned", what, i);
    if (reinterpret_cast<uintptr_t>(p.y) & 7u)
      return fail(FL_ERR_ALIGN, "%s: problem %d y not 8-byte aligned", what, i);
    if (p.score && (reinterpret_cast<uintptr_t>(p.score) & 3u))
      return fail(FL_ERR_ALIGN, "%s: problem %d score not 4-byte aligned", what, i);
    if (p.lifted && (reinterpret_cast<uintptr_t>(p.lifted) & 3u))
      return fail(FL_ERR_ALIGN, "%s: problem %d lifted not 4-byte aligned", what, i);
    Problem& P = a.p[i];
    P.store = p.w.store;
    P.y = p.y;
    P.levels = p.levels;
    P.score = p.score;
    P.lifted = q.rule == FL_DECIDE_SHARE ? p.lifted : nullptr;
    P.out = p.w.out;
    P.G = p.w.in / 128;
    P.block_begin = (int)blocks;
    const int nb = p.w.out / 64;
    P.n_up = (int)floor((double)q.f * (double)nb);      // the share's block count, decided on the host
    if (P.n_up > nb) P.n_up = nb;
    blocks += nb;
    if (blocks > (1l << 30)) return fail(FL_ERR_SHAPE, "%s: too many blocks", what);
  }
  a.nblocks = (int)blocks;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const unsigned grid = (unsigned)((blocks + kWarps - 1) / kWarps);
  int max_nb = 0;
  for (int i = 0; i < n; ++i) max_nb = max_nb > problems[i].w.out / 64 ? max_nb : problems[i].w.out / 64;
  const size_t stage = sizeof(float) * (size_t)(max_nb < kSmemScores ? max_nb : kSmemScores);
  if (a.counters) {  // share rule, one launch: the last CTA to score a layer selects it
    // chunks of whole warps' blocks, about four CTAs per SM (one wave at this kernel's registers)
    const int nsm = device_sm_count();
    if (nsm <= 0) return fail(FL_ERR_CUDA, "%s: no CUDA device", what);
    long per = (blocks + 4L * nsm - 1) / (4L * nsm);
    per = (per + kWarps - 1) / kWarps * kWarps;
    a.chunk = (int)(per < kWarps ? kWarps : per > kMaxChunk ? kMaxChunk : per);
    const unsigned fgrid = (unsigned)((blocks + a.chunk - 1) / a.chunk);
    FL_CHECK_CUDA(launch_pdl(score_select_kernel<FL_MAX_PROBLEMS>, dim3(fgrid), dim3(32 * kWarps), stage, st, 1, a),
                  "launch level_decide score+select");
    return FL_OK;
  }
  FL_CHECK_CUDA(launch_pdl(score_kernel<FL_MAX_PROBLEMS>, dim3(grid), dim3(32 * kWarps), 0, st, 1, a),
                "launch level_decide score");
  if (q.rule == FL_DECIDE_SHARE)
    FL_CHECK_CUDA(launch_pdl(share_kernel<FL_MAX_PROBLEMS>, dim3((unsigned)n), dim3(kShareThreads), stage, st, 1, a),
                  "launch level_decide share");
  return FL_OK;
}
