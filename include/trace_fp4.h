/*
 * trace_fp4.h -- C ABI of the B200 (sm_100a) TRACE rollout-guided NVFP4
 * rounding library (libtrace_fp4.so).
 *
 * The method is the one the rcap.io post "TRACE: Rollout-Guided
 * Quantization-Aware Training for FP4" (2026-10-06) describes: during the
 * rollout, every quantisation site records a compact cache (one mantissa bit
 * per element plus the scale metadata; section "compact cache" and the
 * capture half of the pseudocode listing); during the QAT forward on the
 * paired training activation, each element is rounded to whichever of its
 * two neighbouring FP4 codewords agrees with the rollout (section
 * "rollout-guided rounding" and the QAT-forward half of the listing), and the
 * straight-through estimator passes the gradient back.
 *
 * Number format (NVFP4, as the post's rollout uses it):
 *   - x is bf16, row-major [rows, cols], cols a multiple of 32;
 *   - one fp32 global scale per group: s_g = amax / (6*448), or 1 if amax = 0;
 *   - one E4M3 block scale per 16 consecutive elements of a row:
 *     s_b = E4M3(bmax / (6*s_g)), round to nearest even, saturating at 448;
 *   - z = x / (s_g*s_b) (a zero denominator gives z = +-0), clipped to [-6,6],
 *     on the E2M1 grid {0, .5, 1, 1.5, 2, 3, 4, 6}; code = sign<<3 | magnitude
 *     code 0..7; the mantissa bit of a code is its lowest bit.
 *
 * Layouts (N = rows*cols, element i = row*cols + col):
 *   codes   : uint8[N/2]; byte k holds element 2k in its low nibble and
 *             element 2k+1 in its high nibble.
 *   mbits   : uint32[N/32]; element i is bit (i & 31) of word (i >> 5).
 *   scales  : uint8[rows, cols/16] E4M3 bytes, row-major (the _ex calls
 *             further down also read and write the 128 x 4 tiled layout of a
 *             block-scaled GEMM).
 *   gscale  : float[G], one per group.
 *   ste_mask: uint32[N/32], same packing as mbits; bit set where |z| <= 6
 *             (z before clipping).
 *   Groups: G >= 1 contiguous row ranges (e.g. the experts of a MoE layer),
 *   given as int64 device offsets [G+1] with offsets[0] = 0,
 *   offsets[G] = rows, non-decreasing (empty groups allowed).  NULL offsets
 *   mean G == 1.
 *
 * Ownership and execution: every pointer except `stream` is a DEVICE
 * pointer owned by the caller; the library never allocates, frees or
 * synchronises.  All calls are asynchronous on `stream` (a cudaStream_t
 * passed as void*, NULL = the legacy default stream).  The library holds no
 * mutable global state apart from a per-device cache of the SM count (and
 * the static scratch of trace_capture_static_ws, see there), so it may be
 * called from several host threads.  Every call that takes its scratch
 * memory from the caller is capturable into a CUDA graph.
 *
 * Contents, in order: status and version; workspace and record-size queries;
 * the NVFP4 path (capture, 1-bit guided and full-information guided
 * forwards); the mismatch diagnostic; the MXFP4 (W4A4) and W4A8 variants;
 * the tiled scale layout (_ex calls); capture's two passes for sharded or
 * streamed tensors; the straight-through backward and the round-to-nearest
 * comparator; the E4M3 self-test and the copy yardstick; capture without a
 * workspace.
 *
 * Errors: arguments are checked on the host before anything is enqueued; a
 * failed check returns its code and enqueues nothing.  A launch failure
 * returns TRACE_ERR_CUDA.  Device-side preconditions that the host cannot
 * see are stated per call; breaking them gives unspecified results (never an
 * out-of-bounds access in this library's kernels, apart from reading the
 * offsets array itself, which must hold G+1 entries).
 *   - inputs are finite bf16 (no NaN or infinity);
 *   - scale bytes passed to the forward kernels are non-negative finite E4M3
 *     (0x00..0x7E) and global scales finite and positive, as capture writes;
 *   - the group offsets satisfy the rules above.
 * Limits: N/16 < 2^32 - 512 (N < 2^36 elements per call).  With rows == 0
 * (numel == 0) the data pointers may be NULL.
 */
#ifndef TRACE_FP4_H
#define TRACE_FP4_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  TRACE_OK = 0,
  TRACE_ERR_NULL = 1,      /* a required pointer is NULL */
  TRACE_ERR_SHAPE = 2,     /* rows < 0, cols <= 0, cols % 32, G < 1, size limit */
  TRACE_ERR_ALIGN = 3,     /* a pointer is not aligned as the call requires */
  TRACE_ERR_WORKSPACE = 4, /* workspace smaller than the query returned */
  TRACE_ERR_CUDA = 5,      /* a CUDA runtime call or launch failed */
  TRACE_ERR_TIMEOUT = 6    /* a capture gave up waiting at its grid barrier
                              (reported by trace_capture_status) */
} trace_status;

/* Human-readable name of a status code (static string, never NULL). */
const char* trace_strerror(int status);

/* ABI version of this header (bumped on any incompatible change). */
#define TRACE_ABI_VERSION 2
int trace_abi_version(void);

/* Bytes of device workspace that trace_capture needs for G groups: four
 * words of grid-barrier state, then the per-group amax accumulators (4 bytes
 * each), rounded up to 256.  Returns 0 when the shape is invalid. */
size_t trace_capture_workspace_bytes(int64_t rows, int64_t cols,
                                     int32_t num_groups);

/* Layout of one site's compact-cache record: the mantissa bits, block
 * scales and global scales of a capture in ONE contiguous buffer, so that a
 * cache tier moves a site with a single copy each way (the post's "cache
 * tier that holds" the per-site records, stack-and-caveats list).  Host
 * function; touches no device.
 *   Returns the record's size in bytes (a multiple of 16), or 0 for an
 *   invalid shape (the rules of trace_capture).  Writes the byte offsets of
 *   mbits (uint32[N/32]), scales (uint8[N/16]) and gscale (float[G]) inside
 *   the record to the non-NULL out-pointers; each offset is a multiple of 16,
 *   so a record whose base is 16-byte aligned satisfies every alignment the
 *   calls below ask of these arrays.  Size: N/8 + N/16 + 4G bytes plus at
 *   most 45 bytes of padding, i.e. 1.5 bits per element. */
size_t trace_cache_record_bytes(int64_t rows, int64_t cols, int32_t num_groups,
                                size_t* mbits_offset, size_t* scales_offset,
                                size_t* gscale_offset);

/* Rollout capture: fp4_quantize(x_rollout) plus low_bits(q_roll, 1) and the
 * scales (the capture half of the post's pseudocode listing; the compact
 * cache is mbits + scales + gscale, 1.5 bits per element).
 *   x       : bf16 [rows, cols], 32-byte aligned.
 *   codes   : out, uint8[N/2], 16-byte aligned (the full NVFP4 codes, for the
 *             rollout's own FP4 GEMM).
 *   mbits   : out, uint32[N/32], 16-byte aligned.
 *   scales  : out, uint8[N/16], 16-byte aligned.
 *   gscale  : out, float[G], 4-byte aligned.
 *   workspace: device scratch of at least trace_capture_workspace_bytes()
 *             bytes, 256-byte aligned, holding zeros before its first use
 *             (e.g. cudaMemsetAsync once, when it is allocated); every call
 *             leaves it ready for the next, so a workspace can serve any
 *             number of calls one after another (not two calls that may run
 *             at the same time).  Words: [0] an arrival count and [4, 4+G)
 *             the accumulators, both zero again after every call; [1] counts
 *             calls; [2] is set to nonzero if a CTA ever gave up waiting at
 *             the grid barrier (about two seconds; with the cooperative launch
 *             every CTA is resident, so it is not expected), in which case
 *             that call's outputs are not valid; [3] is unused.
 * One cooperative launch (every CTA resident at once, a few per SM): each
 * CTA max-accumulates the amax of its tiles into the workspace, the CTAs
 * meet at a grid barrier whose last arriving CTA writes gscale and zeroes
 * the accumulators, and each CTA then quantises its own tiles, last read
 * first (from L2 where the tensor fits there). */
int trace_capture(const uint16_t* x, int64_t rows, int64_t cols,
                  int32_t num_groups, const int64_t* group_row_offsets,
                  uint8_t* codes, uint32_t* mbits, uint8_t* scales,
                  float* gscale, void* workspace, size_t workspace_bytes,
                  void* stream);

/* Whether a capture that used `workspace` gave up waiting at its grid
 * barrier: the one device-side wait of the path.  Capture is asynchronous,
 * so it cannot return this itself; this call waits for the work queued on
 * `stream` to finish, reads the workspace's error word (word 2), clears it
 * and returns TRACE_ERR_TIMEOUT if it was set (the outputs of the capture(s)
 * since the last check are then not valid), else TRACE_OK.  workspace:
 * device, as given to trace_capture, 4-byte aligned; NULL returns
 * TRACE_ERR_NULL.  Not for use during stream capture (it synchronises). */
int trace_capture_status(void* workspace, void* stream);

/* Guided QAT fake-quant forward (the QAT-forward half of the listing):
 * z = clip(x_train / (s_g*s_b), -6, 6) with the ROLLOUT's scales; of the two
 * codewords bracketing z (one, if z is a codeword) take the one whose
 * mantissa bit equals the cached bit; out = bf16((q* * s_b) * s_g) with the
 * sign of z (fp32 product, round to nearest even into bf16); ste_mask bit =
 * |z| <= 6.
 *   x_train : bf16 [rows, cols], 32-byte aligned.
 *   mbits, scales, gscale: the rollout's compact cache (capture's outputs).
 *   out     : out, bf16 [rows, cols], 32-byte aligned; may alias x_train.
 *   ste_mask: out, uint32[N/32], 16-byte aligned. */
int trace_guided_fq_fwd(const uint16_t* x_train, int64_t rows, int64_t cols,
                        int32_t num_groups, const int64_t* group_row_offsets,
                        const uint32_t* mbits, const uint8_t* scales,
                        const float* gscale, uint16_t* out, uint32_t* ste_mask,
                        void* stream);

/* Full-information guided fake-quant forward: the upper bound the post's
 * ablation compares the 1-bit cache against ("keeping only 1 mantissa bit ...
 * is close to full-information guidance", results list).  The cache keeps
 * the rollout's whole 4-bit code, and q* is the listing's argmin taken with
 * the exact rollout codeword: of the two codewords bracketing z (one if z is
 * a codeword), the one nearest q_roll.  This makes the per-site guarantee of
 * the rollout-guided-rounding paragraph exact: |q* - q_roll| <=
 * |RTN(z) - q_roll| everywhere.  As trace_guided_fq_fwd, except:
 *   codes: the rollout's packed 4-bit codes (capture's `codes` output),
 *          uint8[N/2], 16-byte aligned (read 0.5 byte per element instead of
 *          0.125 for the bits). */
int trace_full_guided_fq_fwd(const uint16_t* x_train, int64_t rows,
                             int64_t cols, int32_t num_groups,
                             const int64_t* group_row_offsets,
                             const uint8_t* codes, const uint8_t* scales,
                             const float* gscale, uint16_t* out,
                             uint32_t* ste_mask, void* stream);

/* Mismatch diagnostic: how far the training side's FP4 codes land from the
 * rollout's (the compact-cache paragraph reports that nearly all sites where
 * the two sides disagree differ by one adjacent codebook entry).  For every
 * element, z is formed from x_train with the ROLLOUT's scales, and three
 * codes are taken: round to nearest (as trace_rtn_fq_fwd), 1-bit guided (as
 * trace_guided_fq_fwd, with the mantissa bit of the rollout's code) and
 * full-information guided (as trace_full_guided_fq_fwd).  Each code's
 * distance to the rollout's code q_roll is counted on the signed E2M1 ladder
 * -6, -4, ..., -0.5, 0, 0.5, ..., 6 (15 points; +0 and -0 are one point), so
 * distances are 0..14:
 *   hist[k*15 + d] += number of elements whose rule-k code lies d ladder
 *   steps from q_roll; k = 0 round to nearest, 1 1-bit guided, 2 full.
 * The counts are ADDED to hist (zero it first; summing several sites into
 * one histogram is allowed).  Row k = 2, bin 0 counts the sites where q_roll
 * is in the bracket of z_train; all other sites have q_roll outside it.
 *   x_train : bf16 [rows, cols], 32-byte aligned.
 *   codes, scales, gscale: the rollout's capture outputs (codes uint8[N/2],
 *             16-byte aligned).
 *   hist    : in/out, uint64[45], 8-byte aligned; NULL is an error even when
 *             rows == 0 (then nothing is added). */
int trace_mismatch_histogram(const uint16_t* x_train, int64_t rows,
                             int64_t cols, int32_t num_groups,
                             const int64_t* group_row_offsets,
                             const uint8_t* codes, const uint8_t* scales,
                             const float* gscale, uint64_t* hist,
                             void* stream);
/* The same diagnostic for the MXFP4 variant: z from the rollout's E8M0
 * scales (uint8[rows, cols/32], row-major, no alignment requirement); codes
 * as trace_mx_capture writes them; no groups. */
int trace_mx_mismatch_histogram(const uint16_t* x_train, int64_t rows,
                                int64_t cols, const uint8_t* codes,
                                const uint8_t* scales, uint64_t* hist,
                                void* stream);

/* ---- MXFP4 variant ------------------------------------------------------
 * The post's results list reports that the method carries over to MXFP4.
 * The pages give no MX arithmetic beyond power-of-two scales, so the format
 * is the OCP Microscaling one: 32-element blocks along a row, one E8M0 scale
 * byte b per block, X = 2^(b-127), chosen as 2^(floor(log2 max|x|) - 2)
 * (2 is the exponent of E2M1's largest value 6) and clamped at 2^-127 (an
 * all-zero block gets b = 0); no global scale, no groups.  z = x / X, and
 * the rest -- clip, E2M1 rounding, cached bit, STE mask (|z| <= 6),
 * out = bf16(q* * X) -- is as in the NVFP4 calls above.
 *   scales: uint8[rows, cols/32] E8M0 bytes, row-major, no alignment
 *           requirement.  Capture writes 0..252 (a bf16 maximum stays below
 *           2^128); bytes passed to the forwards must be 0..252 too, since
 *           6 * 2^126 and above overflow the bf16 output.
 *   codes, mbits, ste_mask: layouts as above; x/out 32-byte aligned, codes
 *   16-byte, mbits and ste_mask 4-byte aligned.  trace_fq_bwd serves both
 *   formats.  The compact MX cache is mbits + scales: 1.25 bits/element. */
int trace_mx_capture(const uint16_t* x, int64_t rows, int64_t cols,
                     uint8_t* codes, uint32_t* mbits, uint8_t* scales,
                     void* stream);
int trace_mx_guided_fq_fwd(const uint16_t* x_train, int64_t rows, int64_t cols,
                           const uint32_t* mbits, const uint8_t* scales,
                           uint16_t* out, uint32_t* ste_mask, void* stream);
int trace_mx_full_guided_fq_fwd(const uint16_t* x_train, int64_t rows,
                                int64_t cols, const uint8_t* codes,
                                const uint8_t* scales, uint16_t* out,
                                uint32_t* ste_mask, void* stream);
int trace_mx_rtn_fq_fwd(const uint16_t* x, int64_t rows, int64_t cols,
                        const uint8_t* scales, uint16_t* out,
                        uint32_t* ste_mask, void* stream);

/* ---- W4A8: TRACE on FP8 (E4M3) activations with MX scales --------------
 * The results list names the W4A8 setting beside MXFP4.  With 8-bit
 * activations the elements are E4M3 in 32-element blocks with an E8M0 scale
 * X = 2^e, e = floor(log2 max|x|) - 8 (448 = 1.75 * 2^8 is E4M3's largest
 * value), clamped at -127 (-127 for an all-zero block); z = x / X, clipped
 * to [-448, 448]; round to nearest E4M3 with ties to the even mantissa; the
 * cached bit is the lowest bit of the magnitude code; the guided choice is
 * the bracket member (on the E4M3 grid, subnormals included) whose lowest
 * bit equals it; the STE mask is |z| <= 448; out = bf16(q* * X).
 *   codes : uint8[N], one E4M3 byte per element (sign in bit 7), 32-byte
 *           aligned.
 *   mbits : uint32[N/32] (element i = bit i&31 of word i>>5), 4-byte aligned.
 *   scales: uint8[rows, cols/32] E8M0 bytes, no alignment requirement.
 *           Capture writes 0..246 (a bf16 maximum stays below 2^128); the
 *           forwards need 0..246 as well (448 * 2^120 would overflow).
 *   x / out 32-byte aligned, ste_mask 4-byte aligned.  trace_fq_bwd serves
 *   this format too.  The compact cache is mbits + scales: 1.25 bits per
 *   element against 8.25 for the full FP8 codes. */
int trace_mx8_capture(const uint16_t* x, int64_t rows, int64_t cols,
                      uint8_t* codes, uint32_t* mbits, uint8_t* scales,
                      void* stream);
int trace_mx8_guided_fq_fwd(const uint16_t* x_train, int64_t rows,
                            int64_t cols, const uint32_t* mbits,
                            const uint8_t* scales, uint16_t* out,
                            uint32_t* ste_mask, void* stream);
int trace_mx8_full_guided_fq_fwd(const uint16_t* x_train, int64_t rows,
                                 int64_t cols, const uint8_t* codes,
                                 const uint8_t* scales, uint16_t* out,
                                 uint32_t* ste_mask, void* stream);
int trace_mx8_rtn_fq_fwd(const uint16_t* x, int64_t rows, int64_t cols,
                         const uint8_t* scales, uint16_t* out,
                         uint32_t* ste_mask, void* stream);

/* ---- Block-scale layout of a block-scaled FP4 GEMM ------------------------
 * The abstract on the thelatestinai.com TRACE page credits NVFP4 with FP4
 * GEMMs that run W4A4 natively.  The rollout's own FP4 GEMM (a tcgen05
 * block-scaled MMA) reads the block scales in a tiled layout rather than
 * row-major; these entry points let capture write them in that layout
 * directly (no separate reformatting pass over the scales) and let the
 * forwards read it.  Layout TRACE_SCALES_TILED_128x4: the [rows, scols]
 * scale matrix (scols = cols/16 E4M3 scales, or cols/32 E8M0 scales for
 * MXFP4) is cut into 128-row x 4-column tiles of 512 bytes, stored in
 * row-major tile order; inside a tile the scale of row r and column c is at
 * byte 16*(r % 32) + 4*(r / 32) + c.  Rows are padded to a multiple of 128
 * and scale columns to a multiple of 4; the kernels never write or read the
 * padding (zero it once if the GEMM reads it).
 *   rule: TRACE_RULE_RTN (trace_rtn_fq_fwd), TRACE_RULE_GUIDED
 *         (trace_guided_fq_fwd: mbits), TRACE_RULE_FULL
 *         (trace_full_guided_fq_fwd: codes); the pointer the rule does not
 *         read may be NULL.
 *   Everything else as the calls without _ex (which are scale_layout =
 *   TRACE_SCALES_ROW_MAJOR).  An unknown layout or rule returns
 *   TRACE_ERR_SHAPE.  The mismatch histogram and the cache record take
 *   row-major scales only. */
typedef enum { TRACE_SCALES_ROW_MAJOR = 0, TRACE_SCALES_TILED_128x4 = 1 } trace_scale_layout;
typedef enum { TRACE_RULE_RTN = 0, TRACE_RULE_GUIDED = 1, TRACE_RULE_FULL = 2 } trace_rule;

/* Bytes of the scale array for block_size 16 (NVFP4) or 32 (MXFP4) in a
 * layout (padding included); 0 for an invalid argument.  Host only. */
size_t trace_scale_bytes(int64_t rows, int64_t cols, int32_t block_size,
                         int32_t scale_layout);
int trace_capture_ex(const uint16_t* x, int64_t rows, int64_t cols,
                     int32_t num_groups, const int64_t* group_row_offsets,
                     uint8_t* codes, uint32_t* mbits, uint8_t* scales,
                     float* gscale, void* workspace, size_t workspace_bytes,
                     int32_t scale_layout, void* stream);
int trace_fq_fwd_ex(int32_t rule, const uint16_t* x_train, int64_t rows,
                    int64_t cols, int32_t num_groups,
                    const int64_t* group_row_offsets, const uint32_t* mbits,
                    const uint8_t* codes, const uint8_t* scales,
                    const float* gscale, uint16_t* out, uint32_t* ste_mask,
                    int32_t scale_layout, void* stream);
int trace_mx_capture_ex(const uint16_t* x, int64_t rows, int64_t cols,
                        uint8_t* codes, uint32_t* mbits, uint8_t* scales,
                        int32_t scale_layout, void* stream);
int trace_mx_fq_fwd_ex(int32_t rule, const uint16_t* x_train, int64_t rows,
                       int64_t cols, const uint32_t* mbits,
                       const uint8_t* codes, const uint8_t* scales,
                       uint16_t* out, uint32_t* ste_mask, int32_t scale_layout,
                       void* stream);
/* The same for the W4A8 calls (E8M0 scales of 32-element blocks, the layout a
 * block-scaled FP8 GEMM reads too). */
int trace_mx8_capture_ex(const uint16_t* x, int64_t rows, int64_t cols,
                         uint8_t* codes, uint32_t* mbits, uint8_t* scales,
                         int32_t scale_layout, void* stream);
int trace_mx8_fq_fwd_ex(int32_t rule, const uint16_t* x_train, int64_t rows,
                        int64_t cols, const uint32_t* mbits,
                        const uint8_t* codes, const uint8_t* scales,
                        uint16_t* out, uint32_t* ste_mask, int32_t scale_layout,
                        void* stream);

/* ---- Capture of a row-sharded tensor -------------------------------------
 * When one tensor's rows are spread over several GPUs, its global scale
 * needs the maximum over every shard.  Capture's two passes are then called
 * separately around an all-reduce(MAX) of the G accumulators (4 bytes per
 * group; as uint32 the bf16 bit patterns of non-negative values order like
 * the values, so an integer MAX reduction is exact):
 *   trace_capture_amax: zeroes amax[G] and writes max|x| per group over
 *     this shard's rows (bf16 bits in uint32; a group with no rows here
 *     stays 0).  amax: device uint32[G], 4-byte aligned.
 *   trace_capture_with_amax: the quantisation pass of trace_capture with
 *     the given (reduced) amax: gscale[g] = amax/2688 or 1, scales, codes,
 *     mbits.  scale_layout as trace_capture_ex.
 *   trace_capture_amax_accumulate: as trace_capture_amax without the
 *     zeroing: max-accumulates this part's maxima into amax, so a tensor that
 *     arrives in row chunks (e.g. copied from the host chunk by chunk) gets
 *     its whole-tensor amax from one trace_capture_amax on the first chunk
 *     and this call on the others.
 * On one GPU, trace_capture_amax followed by trace_capture_with_amax equals
 * trace_capture.  Group offsets are this shard's, over its own rows. */
int trace_capture_amax(const uint16_t* x, int64_t rows, int64_t cols,
                       int32_t num_groups, const int64_t* group_row_offsets,
                       uint32_t* amax, void* stream);
int trace_capture_amax_accumulate(const uint16_t* x, int64_t rows,
                                  int64_t cols, int32_t num_groups,
                                  const int64_t* group_row_offsets,
                                  uint32_t* amax, void* stream);
int trace_capture_with_amax(const uint16_t* x, int64_t rows, int64_t cols,
                            int32_t num_groups,
                            const int64_t* group_row_offsets,
                            const uint32_t* amax, uint8_t* codes,
                            uint32_t* mbits, uint8_t* scales, float* gscale,
                            int32_t scale_layout, void* stream);

/* Masked straight-through-estimator backward: the gradient half of the
 * listing's straight_through_estimator(x_train, s * q_star) (QAT-forward half
 * of the post's pseudocode listing), which passes the upstream gradient
 * through the fake-quant unchanged; masked where the forward clipped:
 * grad_in[i] = mask bit i ? grad_out[i] : +0.0 (bit copy).
 *   grad_out, grad_in: bf16 [numel], 32-byte aligned; may alias.
 *   ste_mask: uint32[numel/32], 16-byte aligned.  numel % 32 == 0. */
int trace_fq_bwd(const uint16_t* grad_out, const uint32_t* ste_mask,
                 int64_t numel, uint16_t* grad_in, void* stream);

/* Plain round-to-nearest fake-quant with given scales (the vanilla QAT
 * comparator the post measures TRACE against): as trace_guided_fq_fwd with
 * q* replaced by round-to-nearest (ties to the even code).  Vanilla QAT
 * with the training side's own scales is trace_capture(x) followed by this
 * call with the scales it wrote. */
int trace_rtn_fq_fwd(const uint16_t* x, int64_t rows, int64_t cols,
                     int32_t num_groups, const int64_t* group_row_offsets,
                     const uint8_t* scales, const float* gscale, uint16_t* out,
                     uint32_t* ste_mask, void* stream);

/* Self-test, not a step of the method: the E4M3 rounding that capture applies
 * to t = bmax / (6 s_g) (round to nearest even, saturating at 448), run on the
 * fp32 values whose bit patterns are first_bits .. first_bits + count - 1,
 * written to out[count] (device, no alignment requirement).  The range must
 * hold positive finite values only (below 0x7F800000), else TRACE_ERR_SHAPE.
 * It lets a test compare the device conversion with a reference on every
 * positive finite fp32. */
int trace_selftest_e4m3_sweep(uint32_t first_bits, uint32_t count, uint8_t* out,
                              void* stream);

/* Check a group-offset array on the device (the calls above take its
 * contents as a precondition they cannot check on the host): writes to
 * *flag (device uint32, 4-byte aligned) 0 when offsets[0] == 0,
 * offsets[G] == rows and the entries never decrease, else 1 + the index of
 * the first offending entry.  offsets: int64[G+1], 8-byte aligned.  Read the
 * flag after the stream reaches it. */
int trace_validate_offsets(const int64_t* group_row_offsets, int32_t num_groups,
                           int64_t rows, uint32_t* flag, void* stream);

/* Plain bf16 copy (dst = src) with the same load/store path as the kernels
 * above: the measured-bandwidth yardstick for the roofline.  Not part of the
 * method.  32-byte aligned, numel % 16 == 0, no overlap. */
int trace_copy_bf16(const uint16_t* src, uint16_t* dst, int64_t numel,
                    void* stream);

/* The same copy with the reads staged through shared memory by the bulk-copy
 * engine (cp.async.bulk global -> shared, an mbarrier per stage, four 16 KiB
 * tiles in flight per CTA, two CTAs per SM), each thread then storing its
 * part from registers: the yardstick of a TMA-staged pipeline, measured
 * beside the plain copy.  Not part of the method.  err: device uint32,
 * 4-byte aligned, set to 1 if a CTA gave up waiting for a stage (a bounded
 * wait; never expected) and left alone otherwise -- the caller zeroes it and
 * reads it after the stream reaches the copy.  Same shape and alignment rules
 * as trace_copy_bf16. */
int trace_copy_bf16_staged(const uint16_t* src, uint16_t* dst, int64_t numel,
                           uint32_t* err, void* stream);

/* Rollout capture for callers that cannot provide a workspace.  The paper
 * has no counterpart: this is a calling convention, not a step of the method.
 * Who needs it: a caller that may not allocate device memory when it calls
 * the library -- e.g. a host program whose device memory is fixed at
 * start-up, or a binding that can only pass along the buffers it was given.
 * Instead of a `workspace` argument, the amax accumulators live in a static
 * array inside the library: TRACE_STATIC_MAX_GROUPS + 64 uint32 (16.25 KiB:
 * the accumulators, the barrier's state and padding) per GPU that loads the
 * library, kept until the process exits.
 *   Arguments and outputs are those of trace_capture without `workspace`.
 *   num_groups > TRACE_STATIC_MAX_GROUPS: returns TRACE_ERR_WORKSPACE and
 *   enqueues nothing.
 *   The first call on each device looks up the array's device address
 *   (cudaGetSymbolAddress, with that device current); make that first call
 *   before any stream capture.  Every later call made outside stream capture
 *   looks the address up again, because cudaDeviceReset unloads the module
 *   and the array may come back at another address: after a reset, make the
 *   first call outside stream capture too.  Nothing here calls cudaMalloc or
 *   cudaFree.
 *   Every call on a device shares the one array (its contents are zeroed at
 *   the start of each call): two calls that may run at the same time on the
 *   GPU -- e.g. on streams with no ordering between them -- race on it and
 *   give wrong results; order them (one stream, or events). */
#define TRACE_STATIC_MAX_GROUPS 4096
int trace_capture_static_ws(const uint16_t* x, int64_t rows, int64_t cols,
                            int32_t num_groups,
                            const int64_t* group_row_offsets, uint8_t* codes,
                            uint32_t* mbits, uint8_t* scales, float* gscale,
                            void* stream);

#ifdef __cplusplus
}
#endif

#endif /* TRACE_FP4_H */
