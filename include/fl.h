/*
 * fl.h -- C ABI of the variable-precision weight read path (libfl.so, sm_100a).
 *
 * A linear layer's weights are stored once as 8-bit codes split into four
 * 2-bit planes; every 64-output-row block is read at its own depth
 * (ZERO, D2, D4, D6, D8) straight from that one copy, a D4 pass can be
 * escalated to D8 by adding the low planes, an entropy / top-two-margin gate
 * over the logits decides which steps escalate, and GGUF-style Q4_K / Q6_K
 * super-blocks are dequantized inside the product.
 *
 * Sources (page title, section):
 *   [FoQLens]  "FoQLens" landing page: progress table ("a format of our own":
 *              2, 4, 6 or 8 bits read from one copy without repacking; "the
 *              card reads a layout inside the pass": each block of rows read
 *              to its own depth) and the FoQZones mechanism.
 *   [Lens]     "Precision where the question is, not everywhere", section
 *              "The mechanism", rules 1-7, ladder ZERO < D2 < D4 < D6 < D8.
 *   [PoD]      "Precision on Demand: Escalating Weight Bits at Uncertain
 *              Decoding Steps in a Small Local Model", abstract.
 *   [Ember]    "v0.3, quantized on disk, quantized in memory": GGUF K-quant
 *              layouts, per-tensor dispatch with no silent fallback,
 *              validated construction, dequantize only at block granularity
 *              inside the matmul.
 *
 * Conventions for every call:
 *   - Pointers named as device pointers must point to device memory of the
 *     current CUDA device; the caller owns all buffers. The library never
 *     allocates device or host memory.
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy
 *     default stream). Argument, shape and alignment errors are detected on
 *     the host before anything is launched and are returned synchronously;
 *     a failed launch returns FL_ERR_CUDA. Nothing falls back to another
 *     path: unsupported inputs fail.
 *   - fl_last_error() returns a message describing the most recent failure
 *     on the calling thread.
 *   - bf16 activations are passed as their 16-bit patterns (uint16_t).
 *   - Batch (tokens per call) is 1..16 (1..32 for fl_gemv_depth and
 *     fl_gemv_residual); activations are row-major
 *     [batch][in], outputs row-major [batch][out] fp32.
 */
#ifndef FL_H_
#define FL_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define FL_API __attribute__((visibility("default")))
#else
#define FL_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  FL_OK = 0,
  FL_ERR_ARG = -1,          /* null pointer, bad count, bad parameter value    */
  FL_ERR_SHAPE = -2,        /* out/in/batch/vocab outside what the call takes  */
  FL_ERR_UNSUPPORTED = -3,  /* a weight type the fast path does not implement  */
  FL_ERR_ALIGN = -4,        /* a pointer is not aligned as the call requires   */
  FL_ERR_CUDA = -5,         /* a CUDA runtime call or launch failed            */
  FL_ERR_WORKSPACE = -6,    /* workspace missing or smaller than required      */
  FL_ERR_TIMEOUT = -7       /* a kernel's bounded wait ran out (fl_device_status) */
} fl_status;

#define FL_MAX_BATCH 16
/* Single-layer depth / residual calls (fl_gemv_depth, fl_gemv_residual) take batches up to
 * this; from batch 9 they run on the fifth-generation tensor cores (tcgen05, TMEM). */
#define FL_MAX_GEMV_BATCH 32
#define FL_MAX_STOPS 16
#define FL_MAX_PROBLEMS 256

/* GGUF tensor type ids of the two K-quant formats on the fast path ([Ember],
 * GGUF layouts: Q2_K = 10 ... Q6_K = 14). */
#define FL_GGML_Q4_K 12
#define FL_GGML_Q6_K 14

FL_API const char* fl_status_string(int status);

/* Device-side failure detection. Every wait inside a kernel (a stage barrier, the gate's
 * cluster hand-off) is bounded by a deadline of 1 s on the GPU's global timer; when one
 * runs out the kernel records an error word and returns instead of hanging, and its
 * outputs are not valid. Device data the host cannot
 * check (the block lists of fl_gemv_batched_listed) is checked in the kernel the same way.
 * The launching call cannot see either (it returned before the kernel ran), so this call
 * waits for the device, reads and clears every kernel's error word, and returns
 * FL_ERR_TIMEOUT for a wait that ran out, FL_ERR_ARG for a bad list entry (with
 * fl_last_error naming the kernel and the cause), or FL_OK. */
FL_API fl_status fl_device_status(void);

/* Self-test of the failure path above: one thread waits, with a deadline of 1 ms, on a
 * barrier that nothing completes, and records the time-out like a real wait would. The
 * next fl_device_status returns FL_ERR_TIMEOUT. */
FL_API fl_status fl_selftest_wait_timeout(void* stream);
FL_API const char* fl_last_error(void);
FL_API int fl_version(void);

/* ========================================================================= */
/* Plane store ([FoQLens] progress table, "a format of our own": one stored   */
/* stack, a base with refinements, any depth read from the same copy).       */
/*                                                                           */
/* Layout (this library's own): per block b of 64 rows, 8448 * G bytes with  */
/* G = in / 128 column groups:                                               */
/*   [0, 256 G)                         fp32 scale of (group g, row r) at    */
/*                                      byte 4 (64 g + r)                    */
/*   256 G + 2048 (G k + g) + 32 r      32 bytes of plane k (0 = top bits)   */
/*                                      for group g, row r                   */
/* A block read at depth d is the contiguous prefix of 256 G + 1024 G d      */
/* bytes. Inside the 32 bytes of (k, g, r) the 128 columns are four          */
/* little-endian 32-bit words of 16 columns; column j of word w holds        */
/* p_k = (u >> (6 - 2k)) & 3 of u = code + 128 at bit                        */
/* (8 (j % 4) + 6 - 2 k + 2 (j / 4)) mod 32.                                 */
/* ========================================================================= */

/* Bytes of the plane store of an out x in layer (out % 64 == 0, in % 128 == 0);
 * 0 for an invalid shape. */
FL_API size_t fl_plane_store_bytes(int out, int in);

/* Pack int8 codes and their scales into the plane store.
 *   codes  device, int8 [out][in] row-major, values in [-128, 127]
 *   scales device, fp32 [out][in / 128] row-major (one scale per row per
 *          128-column group)
 *   store  device, fl_plane_store_bytes(out, in) bytes, 16-byte aligned;
 *          fully overwritten.
 * out % 64 == 0 and in % 128 == 0, else FL_ERR_SHAPE. Bit-exact. */
FL_API fl_status fl_pack_planes(const int8_t* codes, const float* scales, int out, int in, uint8_t* store, void* stream);

/* A packed layer: device pointer to its plane store and its shape. */
typedef struct {
  const uint8_t* store;
  int out;
  int in;
} fl_plane_weight;

/* ========================================================================= */
/* Level map ([Lens] "The mechanism", rules 1-6).                            */
/*   R_i = r_i f / (1 - f);  kappa = gamma + floor(g (m - gamma));           */
/*   rho_i = |xy_b - c_i| / R_i;  L_i = max(0, 1 - rho_i / s_last);          */
/*   L = min(1, sum_i L_i) (combine 0) or max_i L_i (combine 1);             */
/*   rho* = s_last (1 - L); level = the ring rho* falls into, where ring j   */
/*   covers [s_(j+1), s_j) with s_(kappa+1) = 0; outside every lens: gamma.  */
/* Distance is Euclidean in the plane. R = 0 gives rho = 0 on a centre and   */
/* +inf elsewhere. kappa == gamma (no rings) puts every block at gamma.      */
/* Every operation is an IEEE-rounded fp32 operation in the order above      */
/* (no fused multiply-add), so levels are reproducible bit for bit.          */
/* ========================================================================= */
typedef struct {
  float f;                     /* focus area, 0 <= f < 1                     */
  float g;                     /* focus strength, 0 <= g <= 1                */
  int gamma;                   /* glass level, 0 <= gamma <= m               */
  int m;                       /* top ladder index, 1 <= m <= 15             */
  int nstops;                  /* must equal kappa - gamma                   */
  float stops[FL_MAX_STOPS];   /* s_kappa < ... < s_(gamma+1), ascending, > 0 */
  int combine;                 /* 0 = sum clamped to 1, 1 = max              */
} fl_lens_params;

/* xy      device, fp32 [nblocks][2] block coordinates
 * centers device, fp32 [nlenses][2]; radii device, fp32 [nlenses] (r_i >= 0)
 * levels  device, uint8 [nblocks] (output, level index 0..m)
 * (xy, centers, radii and counts 4-byte aligned)
 * counts  device, uint32 [m + 1] or NULL: per-level block counts are ADDED
 *         to it (the caller zeroes it first).
 * nblocks >= 0, 0 <= nlenses <= 64. */
FL_API fl_status fl_level_map(const float* xy, int nblocks, const float* centers, const float* radii, int nlenses,
                       const fl_lens_params* params, uint8_t* levels, uint32_t* counts, void* stream);

/* ========================================================================= */
/* Depth GEMV / skinny GEMM ([FoQLens] "the card reads a layout inside the   */
/* pass"; [PoD] top bits of 8-bit weights).                                  */
/*   y[t][r] = sum_c w_d[r][c] x[t][c],  d = 2 * levels[r / 64],             */
/*   w_d = s[r][c / 128] (u_d - 128 + c_d), u_d = u with its low 8 - d bits  */
/*   cleared, c_d = (2^(8-d) - 1) / 2; a ZERO block gives y = 0.             */
/* Arithmetic: codes enter an int8 tensor-core product exactly; x enters as  */
/* a 31-bit fixed-point value per 128-column group (four int8 digits): every */
/* element at least 2^-22 of the group's largest |x| is exact (bf16 has 8    */
/* significant bits), a smaller one is off by at most 2^-30 of that largest  */
/* |x|; products accumulate exactly in int32 per group and in fp32 across    */
/* groups. The K-quant GEMV below uses the same activation form.             */
/*                                                                           */
/* levels   device, uint8 [out / 64], values 0..4 (0 ZERO .. 4 D8); values   */
/*          above 4 are read as 4.                                           */
/* x        device, bf16 [batch][in], 16-byte aligned; batch 1..32 (batch 9  */
/*          and up run on the tcgen05 tensor cores: u8 codes in TMEM, digits  */
/*          in shared memory, int32 accumulators in TMEM)                     */
/* y        device, fp32 [batch][out], 4-byte aligned; overwritten           */
/* workspace device scratch for splitting a layer's columns across CTAs:     */
/*          at least fl_gemv_workspace_bytes(out, in, batch) bytes, 16-byte  */
/*          aligned, ZERO-FILLED before its first use; every successful call */
/*          leaves it zero-filled again. Calls that share a workspace must   */
/*          not overlap on the GPU. May be NULL when the size is 0.          */
/* ========================================================================= */
FL_API size_t fl_gemv_workspace_bytes(int out, int in, int batch);

FL_API fl_status fl_gemv_depth(const fl_plane_weight* w, const uint8_t* levels, const uint16_t* x, int batch, float* y,
                        void* workspace, size_t workspace_bytes, void* stream);

/* Depth GEMV without a caller workspace. No counterpart in the pages: an
 * operational variant of fl_gemv_depth for callers that cannot hand over a
 * device buffer, e.g. a plugin host that passes only the operation's own
 * tensors, or a runtime that reserves all device memory up front (an extra
 * cudaMalloc would fail there, and it may synchronize the device inside the
 * decode loop). The column-split scratch lives in a fixed array of
 * FL_GEMV_STATIC_SCRATCH_BYTES inside the library's device image, so this
 * call allocates nothing.
 *   - Same arguments and arithmetic as fl_gemv_depth, minus the workspace;
 *     batch 1..16, always on the int8 mma.sync kernel (fl_gemv_depth moves
 *     batches 9 and up to the tcgen05 kernel, whose split is sized apart).
 *   - Shapes whose split needs more scratch than the array holds return
 *     FL_ERR_WORKSPACE (for batch 1..8 that is when
 *     fl_gemv_workspace_bytes(out, in, batch) > FL_GEMV_STATIC_SCRATCH_BYTES);
 *     use fl_gemv_depth for them.
 *   - The first call on a device looks up the array's device address (with
 *     that device current); make that first call before any stream capture.
 *     The address is kept for the life of the process, per device ordinal: it
 *     does not survive cudaDeviceReset or a switch to another context on the
 *     same device (the library's device image is loaded anew there), so do
 *     not call this entry point after either.
 *   - Every host-side check runs before anything is enqueued, so a rejected
 *     call leaves the array untouched.
 *   - Every call on a device shares the one array, which keeps the previous
 *     call's contents; each call clears the part that must start at zero on
 *     its stream before the launch. Calls that overlap on the GPU (two
 *     streams, or two host threads) race on the array: serialize them. */
#define FL_GEMV_STATIC_SCRATCH_BYTES (4u << 20)
FL_API fl_status fl_gemv_depth_static(const fl_plane_weight* w, const uint8_t* levels, const uint16_t* x, int batch,
                               float* y, void* stream);

/* Escalation residual ([PoD]: redo a step at 8 bits, written as an addition
 * to the low pass):  y[t][r] += sum_c (w_b - w_a)[r][c] x[t][c]  with
 * a = 2 from_levels[blk], b = 2 to_levels[blk], w_0 = 0. Reads only planes
 * a/2 .. b/2 - 1. The levels live on the device, so the host cannot check
 * them: a block whose to-level is not above its from-level adds nothing.
 * Same arguments as fl_gemv_depth. */
FL_API fl_status fl_gemv_residual(const fl_plane_weight* w, const uint8_t* from_levels, const uint8_t* to_levels,
                           const uint16_t* x, int batch, float* y, void* workspace, size_t workspace_bytes,
                           void* stream);

/* Several independent layers in one launch (a decode step's GEMVs).
 * mode 0: depth GEMV (y =), levels = the depth map, to_levels unused.
 * mode 1: residual (y +=), levels = from-levels, to_levels = to-levels.
 * Problems are not split across CTAs, so no workspace is used. 1 <= n <=
 * FL_MAX_PROBLEMS; all problems share `batch`. */
typedef struct {
  fl_plane_weight w;
  const uint8_t* levels;
  const uint8_t* to_levels;
  const uint16_t* x;
  float* y;
} fl_gemv_problem;

FL_API fl_status fl_gemv_batched(const fl_gemv_problem* problems, int n, int batch, int mode, void* stream);

/* fl_gemv_batched over listed blocks only: problem i reads and writes the blocks
 * lists[i][0 .. counts[i]) (device int32 block indices, distinct, each < out / 64; any
 * order) and leaves every other output row as it was. The launch is partitioned over
 * the listed blocks alone, so a sparse set (the blocks an in-pass decision lifted, for
 * a mode 1 residual) is spread evenly over the SMs. lists: host array of n device
 * pointers; counts: host array of n values in 0 .. out / 64 (a problem with count 0
 * is skipped; all zero: nothing is launched). No gate; otherwise as fl_gemv_batched.
 * The lists are device data, so the kernel checks them: an index outside 0 .. out/64 - 1
 * is skipped and the next fl_device_status() returns FL_ERR_ARG. */
FL_API fl_status fl_gemv_batched_listed(const fl_gemv_problem* problems, const int32_t* const* lists,
                                        const int* counts, int n, int batch, int mode, void* stream);

/* fl_gemv_batched with the logit gate fused in ([PoD] abstract: the gate reads the
 * distribution the low-precision step produced). Problem `problem`'s outputs y[t][0..out)
 * are the logits of batch row t; as its blocks are produced, each CTA folds them into
 * entropy / top-2 partials, and the last CTA to finish merges them and writes
 * entropy / margin / top2 / escalate exactly as fl_logit_gate defines them (equal up to
 * fp32 summation order). In mode 1 the gate reads the updated y. y is written as by
 * fl_gemv_batched. No counterpart of the separate launch is needed.
 * entropy, margin  device, fp32 [batch]      top2  device, int32 [batch][2] (all 4-byte aligned)
 * escalate         device, uint8 [batch]
 * workspace        device, >= fl_gemv_gate_workspace_bytes(batch) bytes, 16-byte
 *                  aligned, ZERO-FILLED before first use; every completed launch leaves
 *                  its counter at zero. Launches sharing a workspace must not overlap. */
typedef struct {
  int problem;
  float tau_h;
  float tau_m;
  float* entropy;
  float* margin;
  int32_t* top2;
  uint8_t* escalate;
  void* workspace;
  size_t workspace_bytes;
} fl_gate_spec;

FL_API size_t fl_gemv_gate_workspace_bytes(int batch);

FL_API fl_status fl_gemv_batched_gate(const fl_gemv_problem* problems, int n, int batch, int mode,
                               const fl_gate_spec* gate, void* stream);

/* Device-side conditional escalation ([PoD] abstract: redo only the uncertain steps, here
 * decided on the device, with no read-back to the host): fl_gemv_batched_gate that runs
 * only if the byte at run_if (device, typically the escalate flag a preceding gated pass
 * wrote) is non-zero, and otherwise returns at once, leaving y and the gate outputs as
 * they were. runs: device uint32 (4-byte aligned) or NULL; each pass that ran adds 1 to it. */
FL_API fl_status fl_gemv_batched_gate_if(const fl_gemv_problem* problems, int n, int batch, int mode,
                                  const fl_gate_spec* gate, const uint8_t* run_if, uint32_t* runs,
                                  void* stream);

/* ========================================================================= */
/* In-pass level decision ([FoQLens] FoQZones mechanism: the layer decides   */
/* for itself from what entered it; the draft score, the reduced score, the  */
/* ladder lambda 16^j capped at kappa, or the top share f).                   */
/* For block c (64 rows) of a layer read at the base level gamma:            */
/*   s_c = ||y_c||^2 D_c^2, y_c the block's base-level outputs over its 64    */
/*         rows and every batch row;                                          */
/*   D_c^2 = mean over the block's rows and 128-column groups of              */
/*         (scale 2^(8 - 2 gamma))^2, the squared base quantization step;     */
/*   r_c = s_c D_c^2 / (64 in)  (the reduced score; w_c = 64 in weights);     */
/*   FL_DECIDE_LADDER: level = gamma + #{ j >= 1 : r_c >= lambda 16^j },      */
/*         at most kappa;                                                     */
/*   FL_DECIDE_SHARE: the floor(f * out / 64) blocks of largest r_c (equal    */
/*         r_c: lower block index first) get kappa, the others gamma.         */
/* The levels then drive the residual pass from gamma (fl_gemv_residual or    */
/* fl_gemv_batched mode 1 with to_levels = these levels), so only the lifted  */
/* blocks' low planes are read a second time. fp32 arithmetic: a decision can */
/* differ from an exact one only when r_c lies within fp32 rounding of a      */
/* threshold (or of another block's score, for the share rule).               */
/*                                                                           */
/* Per problem (one layer; all share `batch`, 1 <= n <= FL_MAX_PROBLEMS):     */
/*   w       the layer's plane store (its scales are read), 16-byte aligned   */
/*   y       device fp32 [batch][out], 8-byte aligned: the base-level outputs */
/*   levels  device uint8 [out / 64], written                                 */
/*   score   device fp32 [out / 64], written with r_c; may be NULL for the   */
/*           ladder rule, required for the share rule                         */
/*   lifted  device int32 [out / 64] or NULL; share rule only: its first      */
/*           floor(f * out / 64) entries receive the lifted blocks' indices   */
/*           in ascending order (the block list of fl_gemv_batched_listed)    */
/* params: 1 <= gamma <= kappa <= 4; ladder: lambda finite, >= 0; share:     */
/* 0 <= f <= 1. One launch (ladder, or share with counters) or two (share),   */
/* asynchronous on stream.                                                    */
/* ========================================================================= */
#define FL_DECIDE_LADDER 0
#define FL_DECIDE_SHARE 1

typedef struct {
  fl_plane_weight w;
  const float* y;
  uint8_t* levels;
  float* score;
  int32_t* lifted;
} fl_decide_problem;

/* counters (share rule; may be NULL): device int32 [n], 4-byte aligned, ZERO-FILLED before
 * first use and left zero by every completed call. With counters the share rule takes one
 * launch: each CTA adds the blocks it scored to its layers' counters, and the CTA whose addition
 * completes a layer selects that layer's share at once. Without them (and for the ladder) the
 * selection is a second launch. Calls sharing counters must not overlap. */
typedef struct {
  int rule;
  int gamma;
  int kappa;
  float lambda;
  float f;
  int32_t* counters;
} fl_decide_params;

FL_API fl_status fl_level_decide(const fl_decide_problem* problems, int n, int batch, const fl_decide_params* params,
                                 void* stream);

/* ========================================================================= */
/* Uncertainty gate ([PoD]: redo at 8 bits when the low-precision output     */
/* distribution looks uncertain: entropy above a threshold or a small        */
/* top-two margin).  Per row t of logits z:                                  */
/*   m = max z, S = sum e^(z - m), T = sum (z - m) e^(z - m),                */
/*   entropy = ln S - T / S (nats),  i1, i2 = indices of the two largest     */
/*   logits (ties to the lower index), margin = p1 - p2 = (1 - e^(z_i2-m))/S,*/
/*   escalate = (entropy > tau_h) || (margin < tau_m).                       */
/* logits device fp32 [batch][vocab], 16-byte aligned, vocab % 4 == 0,      */
/* 4 <= vocab <= 2^24; outputs device (4-byte aligned): entropy, margin fp32      */
/* [batch], top2 int32                                                        */
/* [batch][2], escalate uint8 [batch]. fp32 arithmetic.                      */
/* ========================================================================= */
FL_API fl_status fl_logit_gate(const float* logits, int vocab, int batch, float tau_h, float tau_m, float* entropy,
                        float* margin, int32_t* top2, uint8_t* escalate, void* stream);

/* ========================================================================= */
/* The read split over devices. Blocks are independent, so ranks can each    */
/* read a contiguous range of every layer's 64-row blocks (the same          */
/* fl_gemv_* calls on the range: plane store + first * 8448 * (in / 128),    */
/* out = 64 * count, levels + first) and exchange their outputs; the gate    */
/* then needs the whole row of logits, which the ranks hold in pieces, so   */
/* each rank reduces its piece to a partial and every rank merges all the   */
/* partials the same way ([PoD] abstract: the gate reads the low-precision  */
/* output distribution; [FoQLens] progress table: each block read to its    */
/* own depth).                                                               */
/* ========================================================================= */

/* Contiguous block ranges for nranks ranks, balanced by the bytes each block's depth reads
 * (256 G + 2048 G d / 2 at depth d, G = in / 128; ZERO blocks read nothing): rank r reads
 * blocks [first_block[r], first_block[r + 1]), first_block[0] = 0, first_block[nranks] =
 * nblocks; a block goes to the range that holds the midpoint of its bytes, so ranges differ
 * by at most one block's bytes. Ranges may be empty (nranks > nblocks). A layer that reads
 * nothing is split by block count. Host only: levels is a HOST array of nblocks level bytes
 * (values above 4 read as 4), first_block a HOST array of nranks + 1 ints. */
FL_API fl_status fl_shard_blocks(const uint8_t* levels, int nblocks, int in, int nranks, int* first_block);

/* A rank's partial of the gate over its piece of the logits: per row, m = max z,
 * s = sum e^(z - m), t = sum (z - m) e^(z - m), the largest and second largest value (v2)
 * with their GLOBAL indices i1, i2 (piece index + index_base; ties to the lower index).
 * 32 bytes, the same record the fused gate merges. */
typedef struct {
  float m, s, t, v2;
  int32_t i1, i2, pad0, pad1;
} fl_gate_partial;

/* logits  device fp32 [batch][vocab] (this rank's piece of each row), 16-byte aligned,
 *         vocab % 4 == 0; index_base + vocab <= 2^24
 * partial device fl_gate_partial [batch], 16-byte aligned, written. One launch: a cluster of
 *         8 or 16 CTAs per row, the reduction fl_logit_gate runs. If the cluster's wait for its
 *         CTAs' partials runs out (1 s) the record's s is NaN, so the merged entropy and margin
 *         are NaN, and fl_device_status reports the wait. */
FL_API fl_status fl_logit_gate_partial(const float* logits, int vocab, int batch, int index_base,
                                       fl_gate_partial* partial, void* stream);

/* The batched pass with the gate fused (fl_gemv_batched_gate, and fl_gemv_batched_gate_if when
 * run_if is not NULL) that writes, instead of the gate's outputs, the merged partial of the
 * gate problem's logits per batch row to partial [batch] (device, 16-byte aligned), indices
 * offset by index_base (index_base + out <= 2^24): a rank's piece of a vocabulary split over
 * devices, reduced in the launch that computes it. The gate spec's thresholds and output
 * pointers are not used (they may be NULL); its problem and workspace are. runs as
 * fl_gemv_batched_gate_if. */
FL_API fl_status fl_gemv_batched_gate_partial(const fl_gemv_problem* problems, int n, int batch, int mode,
                                              const fl_gate_spec* gate, const uint8_t* run_if, uint32_t* runs,
                                              int index_base, fl_gate_partial* partial, void* stream);

/* Merge nparts partials per row, partials laid out [nparts][batch] (the gathered pieces in
 * rank order), in one fixed order (lane l of a warp takes parts l, l + 32, ..., then the lanes
 * merge in a fixed tree), and write entropy / margin / top2 / escalate exactly as fl_logit_gate
 * defines them for the whole row (equal up to fp32 summation order; top2 ties go to the lower
 * global index). Every rank that merges the same partials computes the same outputs. Output pointers as fl_logit_gate;
 * partials device, 16-byte aligned; 1 <= nparts <= 4096. One launch. */
FL_API fl_status fl_logit_gate_merge(const fl_gate_partial* partials, int nparts, int batch, float tau_h, float tau_m,
                                     float* entropy, float* margin, int32_t* top2, uint8_t* escalate, void* stream);

/* ========================================================================= */
/* Verified speculation ([PoD] abstract: a low-precision draft verified at   */
/* 8 bits gives the 8-bit model's output at a comparable weight-byte cost).  */
/* Greedy, over a window of k steps (1 <= k <= FL_MAX_BATCH):                */
/*   draft token t    = draft_top2[t][0], the argmax of step t's D4 logits    */
/*                      (the top2 row a gated D4 pass writes);                */
/*   verified token t = verified_top2[t][0], the argmax of step t's D8 logits */
/*                      (the top2 rows of one gated residual pass at batch k  */
/*                      over the window's D4 outputs);                        */
/*   accepted = the length of the longest prefix where the two agree;        */
/*   emitted  = accepted + 1 if accepted < k, else k: the verified tokens of  */
/*              steps 0 .. emitted - 1, the 8-bit model's own greedy choice.  */
/* draft_top2, verified_top2  device int32 [k][2]                             */
/* result  device int32 [2] = {accepted, emitted}, written                    */
/* totals  device int32 [2] or NULL: accepted and emitted are ADDED to it     */
/* One launch, asynchronous on stream.                                        */
/* ========================================================================= */
FL_API fl_status fl_spec_accept(const int32_t* draft_top2, const int32_t* verified_top2, int k, int32_t* result,
                                int32_t* totals, void* stream);

/* ========================================================================= */
/* K-quant GEMV ([Ember]: Q4_K / Q6_K native kernels, dequantize only at     */
/* block granularity inside the product, per-tensor dispatch, unsupported    */
/* types fail). Records of 256 weights stored block-tiled: 64-row blocks,   */
/* then super-blocks, then the block's 64 rows, i.e. record number           */
/* ((r / 64) * (in / 256) + sb) * 64 + r % 64 holds row r, super-block sb,   */
/* so 64 rows x k super-blocks is one contiguous range. The value rules are  */
/* GGUF's; the byte layout is this library's own with the GGUF byte counts:  */
/*   Q4_K 144 B, sub-blocks j of 32: [0,2) d fp16, [2,4) dmin fp16,          */
/*        byte 4 + j = sc_j | (mn_j & 3) << 6, nibble j of the word at 12 =   */
/*        mn_j >> 2, byte 16 + 16 j + b = q[32 j + b] | q[32 j + 16 + b] << 4;*/
/*        w = d sc_j q - dmin mn_j.                                          */
/*   Q6_K 210 B, sub-blocks j of 16, q in 0..63: a record of an even row is */
/*        [q area 192][sc_j int8 x16][d fp16], of an odd row                 */
/*        [d fp16][q area 192][sc_j int8 x16]; q area: chunk t (48 B) x      */
/*        group m (12 B = words A, B, C), W(j, L) = 16 j + 4 t + L:          */
/*        A byte L = lo4 q[W(4m,L)] | lo4 q[W(4m+1,L)] << 4,                 */
/*        B byte L = lo4 q[W(4m+2,L)] | lo4 q[W(4m+3,L)] << 4,               */
/*        C byte L = hi2 q[W(4m+2,L)] | hi2 q[W(4m+3,L)] << 2                */
/*                 | hi2 q[W(4m,L)] << 4 | hi2 q[W(4m+1,L)] << 6;            */
/*        w = d sc_j (q - 32).                                               */
/* blocks: device, 16-byte aligned; out % 64 == 0, in % 256 == 0.           */
/* ggml_type other than FL_GGML_Q4_K / FL_GGML_Q6_K -> FL_ERR_UNSUPPORTED.    */
/* Same x / y / workspace rules as fl_gemv_depth.                            */
/* ========================================================================= */
FL_API size_t fl_kquant_bytes(int ggml_type, int out, int in);
FL_API size_t fl_kquant_workspace_bytes(int ggml_type, int out, int in, int batch);

FL_API fl_status fl_gemv_kquant(const void* blocks, int ggml_type, int out, int in, const uint16_t* x, int batch, float* y,
                         void* workspace, size_t workspace_bytes, void* stream);

typedef struct {
  const void* blocks;
  int ggml_type;
  int out;
  int in;
  const uint16_t* x;
  float* y;
} fl_kquant_problem;

/* Several K-quant tensors in one launch (a decode step); no workspace. */
FL_API fl_status fl_gemv_kquant_batched(const fl_kquant_problem* problems, int n, int batch, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* FL_H_ */
