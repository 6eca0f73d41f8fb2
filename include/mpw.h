/*
 * mpw.h -- packed INT-b weight rows and the fused dequantize-linear layer on
 * B200 (sm_100a).  C ABI of libmpw.so.
 *
 * What it computes (page title, section):
 *   - Quantization tutorial (aiknowledge.cn, "量化"), "How quantization works":
 *     symmetric quantization, scale = max|w| / max_int, q = round(w / scale),
 *     reconstruction q * scale, one scale per output channel.
 *   - Same page, "Step 1: symmetric quantization": max_int = 2^(b-1) - 1,
 *     round half to even, a zero channel takes the scale 1 / max_int.
 *   - DynaQuant (zingnex forum thread), "Step 3: apply the recipe": one bit
 *     width per weight matrix; "Custom kernel architecture": packed N-bit
 *     weights are read from memory, expanded in registers to a tensor-core
 *     format and multiplied; "Status": bit pack / unpack tools.
 *
 * Conventions shared by every entry point
 *   - W is [N, K] row-major: N output features (rows), K input features.
 *     One fp32 scale per row: s_n = fl32(max_k |w_nk| / Q), Q = 2^(b-1) - 1,
 *     an IEEE division; a zero row takes s_n = fl32(1 / Q).
 *   - Codes q = clamp(rint_half_even(fl32(w / s_n)), -Q, Q), IEEE division.
 *   - Packed format ("canonical"): row n occupies mpw_packed_row_bytes(K, b)
 *     bytes starting at packed + n * row_bytes.  Code k of the row is stored
 *     as b-bit two's complement in bits [k*b, k*b + b) of the row read as a
 *     little-endian integer (LSB-first along K).  The row is padded with zero
 *     bits to 16 * ceil(K*b / 128) bytes.
 *   - bits must be in 4..15, N >= 1, K >= 1.
 *   - Activations x and outputs y are bfloat16, passed as raw uint16_t bit
 *     patterns, row-major [M, K] and [M, N].
 *   - All pointers named "device" are device memory owned by the caller; the
 *     library never allocates, frees or retains caller memory.
 *   - Every call is asynchronous on `stream` (NULL = legacy default stream)
 *     and returns its status synchronously.  On an argument error nothing is
 *     launched.  No C++ exception crosses this boundary.  Entry points marked
 *     "host only" (mpw_allocate_*, mpw_recipe_plan, mpw_file_*) do no
 *     device work, take host memory and run to completion before returning.
 *   - Alignment: `packed` must be 16-byte aligned.  Everything else needs
 *     only its natural alignment, except where an entry point says otherwise.
 *   - A second, kernel-private ordering of the same bits ("paired halves",
 *     mpw_layout below) is read fastest by the decode kernels; mpw_repack
 *     converts between the two and the *_ex / mpw_linear.layout entry points
 *     take either.
 */
#ifndef MPW_H_
#define MPW_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MPW_API __attribute__((visibility("default")))
#else
#define MPW_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

struct CUstream_st;
typedef struct CUstream_st* mpw_stream_t; /* a cudaStream_t */

typedef enum mpw_status {
  MPW_OK = 0,
  MPW_E_INVALID_ARG = 1,      /* null pointer, non-positive size, bad count */
  MPW_E_UNSUPPORTED_BITS = 2, /* bits outside 4..15 */
  MPW_E_MISALIGNED = 3,       /* pointer alignment rule above violated */
  MPW_E_CUDA = 4,             /* a CUDA runtime call or launch failed */
  MPW_E_NONFINITE = 5,        /* reserved: reported through the flag word */
  MPW_E_TIMEOUT = 6,          /* a device-side wait gave up (see mpw_device_error) */
  MPW_E_SCRATCH_LIMIT = 7,    /* mpw_qlinear_noalloc: the call needs more than its fixed scratch */
  MPW_E_IO = 8,               /* mpw_file_*: the file cannot be opened, read or written */
  MPW_E_FORMAT = 9,           /* mpw_file_*: not a valid container, truncated, or a checksum differs */
  MPW_E_UNSUPPORTED = 10      /* mpw_pass_create: a linear or M the planned pass does not take */
} mpw_status;

/* Static English text for a status code; never NULL. */
MPW_API const char* mpw_status_str(int status);

/* Library version, major * 10000 + minor * 100 + patch. */
MPW_API int mpw_version(void);

/* Bytes of one packed row: 16 * ceil(K * bits / 128).  Returns 0 if bits is
 * outside 4..15 or K < 1. */
MPW_API size_t mpw_packed_row_bytes(int64_t K, int bits);

/*
 * mpw_quantize_pack -- per-row symmetric quantization and canonical packing.
 *   W        device, fp32 [N, K] row-major, finite values (precondition).
 *   packed   device, uint8 [N, mpw_packed_row_bytes(K, bits)], 16-B aligned;
 *            every byte, padding included, is written.
 *   scales   device, fp32 [N]; receives s_n.
 *   nonfinite_flag  device int32 or NULL.  If not NULL and some w is not
 *            finite, 1 is stored there (the caller clears it beforehand and
 *            reads it after synchronising); codes of such rows are undefined.
 * Pages: tutorial "How quantization works", "Step 1"; DynaQuant "Step 3".
 */
MPW_API mpw_status mpw_quantize_pack(const float* W, int64_t N, int64_t K, int bits,
                             uint8_t* packed, float* scales,
                             int32_t* nonfinite_flag, mpw_stream_t stream);

/*
 * mpw_unpack -- canonical packed rows back to sign-extended codes.
 *   packed   device, uint8 [N, row_bytes], 16-B aligned.
 *   codes    device, int16 [N, K] row-major.
 * Pages: DynaQuant "Status" (bit pack / unpack tools).
 */
MPW_API mpw_status mpw_unpack(const uint8_t* packed, int64_t N, int64_t K, int bits,
                      int16_t* codes, mpw_stream_t stream);

/*
 * mpw_dequantize -- reconstruction w_hat = fl32(q * s_n), fp32 [N, K].
 * Pages: tutorial "How quantization works" (reconstructed = quantized * scale).
 */
MPW_API mpw_status mpw_dequantize(const uint8_t* packed, const float* scales,
                          int64_t N, int64_t K, int bits, float* W_hat,
                          mpw_stream_t stream);

/*
 * mpw_qlinear -- fused dequantize-linear y = x @ (q * s)^T.
 *   x        device, bf16 [M, K] row-major.
 *   packed, scales  as produced by mpw_quantize_pack for W [N, K].
 *   y        device, bf16 [M, N] row-major; y[m, n] is
 *            bf16_rn(s_n * sum_k x[m, k] * q[n, k]) with an fp32 accumulator.
 *   M >= 1.  M <= 32 runs a decode kernel (packed rows streamed once,
 *   unpacked in registers, mma.sync or tcgen05 tensor cores); larger M runs
 *   the prefill GEMM on tcgen05 tensor cores with the accumulator in tensor
 *   memory.  Every code reaches the tensor cores as exact bf16 values: whole
 *   when it has at most 9 bits, else split as lo7 + 128 * hi (lo7 = q & 127,
 *   hi = q >> 7, arithmetic) in the GEMM and on paired rows, and into 7-bit
 *   fields in the canonical-row decode kernels; each term is exact in bf16,
 *   so no code is ever rounded.
 * Pages: DynaQuant "Custom kernel architecture" (packed N-bit -> registers ->
 * tensor core; 9-15 bit codes on BF16 tensor cores).
 */
MPW_API mpw_status mpw_qlinear(const uint16_t* x, const uint8_t* packed,
                       const float* scales, int bits, int64_t M, int64_t N,
                       int64_t K, uint16_t* y, mpw_stream_t stream);

/* Kernel choice for mpw_qlinear_path. */
typedef enum mpw_path {
  MPW_PATH_AUTO = 0, /* what mpw_qlinear does */
  MPW_PATH_GEMV = 1, /* decode kernel for any M (re-streams W per 32 rows of x) */
  MPW_PATH_GEMM = 2  /* tensor-core prefill kernel for any M */
} mpw_path;

/* mpw_qlinear with an explicit kernel choice; same arguments and results. */
MPW_API mpw_status mpw_qlinear_path(const uint16_t* x, const uint8_t* packed,
                            const float* scales, int bits, int64_t M,
                            int64_t N, int64_t K, uint16_t* y, int path,
                            mpw_stream_t stream);

/* Packed layouts. */
typedef enum mpw_layout {
  MPW_LAYOUT_CANONICAL = 0, /* the format above; what mpw_quantize_pack writes */
  MPW_LAYOUT_PAIRED = 1     /* paired halves; needs K % 32 == 0 */
} mpw_layout;

/*
 * mpw_repack -- re-orders packed rows from layout_in to layout_out.
 *   Paired halves: each row is cut into groups of 32 codes; in group g the
 *   even codes (32g + 2i, i = 0..15) form one stream and the odd codes
 *   (32g + 2i + 1) another, code i of a stream in bits [i*b, i*b + b) of it
 *   (two's complement, LSB first).  Little-endian 32-bit word g*b + h of the
 *   row holds 16-bit half-word h of the even stream in its low half and
 *   half-word h of the odd stream in its high half; padding stays zero.  The
 *   row stride is the canonical one and the layout holds the same bits,
 *   re-ordered, so a decode kernel can turn the two codes of a pair into one
 *   bf16x2 operand with a shift and a bit operation.  No page defines this
 *   layout; it is storage for this library's decode kernels.
 *   in, out   device, uint8 [N, mpw_packed_row_bytes(K, bits)], 16-B
 *             aligned; out == in is allowed (in place), other overlap is not.
 *   layout_in != layout_out, both MPW_LAYOUT_*; K % 32 == 0.
 */
MPW_API mpw_status mpw_repack(const uint8_t* in, int64_t N, int64_t K, int bits, int layout_in,
                              int layout_out, uint8_t* out, mpw_stream_t stream);

/*
 * mpw_qlinear_ex -- mpw_qlinear_path for packed rows in either layout.
 *   With MPW_LAYOUT_PAIRED: K % 32 == 0 (else MPW_E_INVALID_ARG) and x
 *   16-byte aligned (else MPW_E_MISALIGNED).  Results are identical to the
 *   canonical call on the same codes up to the fp32 summation order.
 */
MPW_API mpw_status mpw_qlinear_ex(const uint16_t* x, const uint8_t* packed, const float* scales,
                                  int bits, int layout, int64_t M, int64_t N, int64_t K,
                                  uint16_t* y, int path, mpw_stream_t stream);

/*
 * Group-wise scales (quantization tutorial, exercises, item 1: one scale per
 * 128 weights instead of one per output channel; group sizes 32, 64, 128 and
 * 256 compared).  Groups are `group` consecutive weights of a row along K,
 * the last one shorter when group does not divide K; each group is quantized
 * with the per-row formula above applied to the group (s_nj = fl32(max |w| /
 * Q) over group j, a zero group takes fl32(1 / Q)).  The codes are stored in
 * the canonical packed format (mpw_unpack reads them; mpw_repack re-orders
 * them), the scales as fp32 [N, ceil(K / group)] row-major.
 *
 * mpw_quantize_pack_groups -- group-wise quantization and canonical packing.
 *   group    a power of two in 32..1024 (else MPW_E_INVALID_ARG).
 *   W, packed, nonfinite_flag  as for mpw_quantize_pack.
 *   scales   device, fp32 [N, ceil(K / group)].
 */
MPW_API mpw_status mpw_quantize_pack_groups(const float* W, int64_t N, int64_t K, int bits, int64_t group,
                                            uint8_t* packed, float* scales, int32_t* nonfinite_flag,
                                            mpw_stream_t stream);

/*
 * mpw_qlinear_groups -- y = x @ (q * s_group)^T for group-scaled rows:
 *   y[m, n] = bf16_rn(sum_j s_nj * sum_{k in group j} x[m, k] q[n, k]), each
 *   group's sum in fp32, scaled in fp32 and added to an fp32 accumulator.
 *   group    a power of two in 128..1024 (a group then holds whole 128-code
 *            chunks of the decode kernel); smaller groups: MPW_E_INVALID_ARG.
 *   layout   MPW_LAYOUT_* of `packed`.
 *   M >= 1, run as the decode kernel in passes of 32 tokens; K % 8 == 0
 *   (K % 32 == 0 for paired rows); x 16-byte aligned (else MPW_E_MISALIGNED).
 *   flags    0, MPW_QLINEAR_X_READY or MPW_QLINEAR_X_READY |
 *            MPW_QLINEAR_Y_UNSHARED, with the meaning they have for
 *            mpw_qlinear_flags (defined below).
 */
MPW_API mpw_status mpw_qlinear_groups(const uint16_t* x, const uint8_t* packed, const float* scales, int bits,
                                      int64_t group, int layout, int64_t M, int64_t N, int64_t K, uint16_t* y,
                                      unsigned flags, mpw_stream_t stream);

/*
 * Workspace of the decode kernels.  For M <= 32 the fastest decode kernel
 * splits the (16-row tile, 128-code chunk) units of W evenly over a
 * persistent grid; a tile shared by two or more CTAs is combined through a
 * small caller-provided workspace (partial sums and one counter per tile).
 *   - device memory, 16-byte aligned, at least the size returned below;
 *   - zero-filled by the caller once before its first use; every call that
 *     completes leaves it ready for the next one (its counters back at zero);
 *     after a call that reported MPW_E_TIMEOUT it must be zero-filled again;
 *   - calls that share one workspace must not run at the same time (calls on
 *     one stream never do).
 * mpw_qlinear_workspace_bytes returns the bytes a call with these arguments
 * needs (0 when it uses no workspace).  A NULL workspace selects the
 * per-tile decode kernel, which needs none; a non-NULL workspace smaller
 * than required is an argument error.
 */
MPW_API size_t mpw_qlinear_workspace_bytes(int bits, int layout, int64_t M, int64_t N, int64_t K);

/* mpw_qlinear_ex with a decode workspace (see above); same results. */
MPW_API mpw_status mpw_qlinear_ws(const uint16_t* x, const uint8_t* packed, const float* scales,
                                  int bits, int layout, int64_t M, int64_t N, int64_t K,
                                  uint16_t* y, int path, void* workspace, size_t workspace_bytes,
                                  mpw_stream_t stream);

/*
 * mpw_qlinear_flags -- mpw_qlinear_ex with flags (0, MPW_QLINEAR_X_READY or
 * MPW_QLINEAR_X_READY | MPW_QLINEAR_Y_UNSHARED; other bits are
 * MPW_E_INVALID_ARG).
 *   MPW_QLINEAR_X_READY: the caller states that x was written before the
 *   launch that precedes the current run of flagged calls on `stream` (the
 *   consecutive calls made with this flag, this one included): neither a
 *   call of the run nor the launch just before it wrote x.  Typical uses: q
 *   called without the flag, then k and v with it, all three reading a hidden
 *   state written earlier; a set of matrices applied to one x that was
 *   complete before the set began.  A flagged decode kernel lets the next
 *   kernel start at once and loads x together with its weights without
 *   waiting for its predecessor, so consecutive flagged calls overlap in
 *   full; only its write of y waits for the preceding launch, so results
 *   land in call order.  The statement suffices because this library's
 *   unflagged decode kernels let their successor start only after they have
 *   themselves waited for their predecessor; the launch before the run must
 *   be one of this library's kernels, a copy, or a kernel launched without
 *   programmatic dependent launch.  A false statement is a data race (stale
 *   x), not an error code.  Results are those of mpw_qlinear_ex.
 */
#define MPW_QLINEAR_X_READY 1u
/*
 *   MPW_QLINEAR_Y_UNSHARED (only with MPW_QLINEAR_X_READY, else
 *   MPW_E_INVALID_ARG): the caller also states that no other call of the run
 *   and not the launch just before it reads or writes y (q, k and v writing
 *   three different buffers; distinct outputs for a set of matrices).  The
 *   kernel then writes y without waiting for its predecessor; one of its
 *   blocks still waits, so kernels complete in launch order and an unflagged
 *   call after the run sees every output of it.  A false statement is a data
 *   race, not an error code.
 */
#define MPW_QLINEAR_Y_UNSHARED 2u
MPW_API mpw_status mpw_qlinear_flags(const uint16_t* x, const uint8_t* packed, const float* scales,
                                     int bits, int layout, int64_t M, int64_t N, int64_t K,
                                     uint16_t* y, int path, unsigned flags, mpw_stream_t stream);

/*
 * One linear of a recipe stack (DynaQuant "Step 3": every matrix carries its
 * own bit width).  Activations move between caller-owned "slots".
 *   packed, scales, N, K, bits  the quantized matrix (device pointers).
 *   in_slot   index of the slot holding x [M, K] (bf16).
 *   out_slot  index of the slot receiving y [M, N] (bf16).
 *   norm_input  if nonzero, the linear reads the RMS-normalised input:
 *             y[m, n] = bf16(s_n * r_m * sum_k x[m, k] q[n, k]) with
 *             r_m = 1 / sqrt(mean_k x[m, k]^2 + 1e-6), evaluated in fp32 (the
 *             normalisation is a per-token scale of the product; x itself is
 *             not modified).
 *   layout    MPW_LAYOUT_* of `packed` (paired: K % 32 == 0 and the slots
 *             16-byte aligned).
 *   reserved  must be 0.
 */
typedef struct mpw_linear {
  const uint8_t* packed;
  const float* scales;
  int64_t N;
  int64_t K;
  int32_t bits;
  int32_t in_slot;
  int32_t out_slot;
  int32_t norm_input;
  int32_t layout;
  int32_t reserved;
} mpw_linear;

/*
 * mpw_recipe_run -- apply a per-matrix bit-width recipe to a stack of linears:
 * launches `count` qlinear kernels in order on `stream` (capturable in a CUDA
 * graph).  A linear whose input bytes were written neither by the linear
 * before the current run of such linears nor by one inside it (k and v after
 * q; up after gate) is launched with MPW_QLINEAR_X_READY, so that it runs
 * alongside its predecessors, and also with MPW_QLINEAR_Y_UNSHARED when its
 * output bytes are neither read nor written by that run and linear; the
 * first linear is never flagged.  slots[i] are device bf16 buffers; each must hold M * (largest N or
 * K that touches it) elements.  M must be in 1..32 (the decode pass).
 * A linear whose in_slot equals its out_slot is rejected.
 */
MPW_API mpw_status mpw_recipe_run(const mpw_linear* layers, int64_t count,
                          uint16_t* const* slots, int64_t num_slots, int64_t M,
                          mpw_stream_t stream);

/*
 * mpw_recipe_plan -- the flags mpw_recipe_run launches each linear with
 * (0, MPW_QLINEAR_X_READY, or MPW_QLINEAR_X_READY | MPW_QLINEAR_Y_UNSHARED),
 * written to flags[count] (host memory), from the same arguments (validated
 * alike; slot pointers are compared, never dereferenced).  Host only.
 */
MPW_API mpw_status mpw_recipe_plan(const mpw_linear* layers, int64_t count, uint16_t* const* slots,
                                   int64_t num_slots, int64_t M, uint32_t* flags);

/* Workspace bytes for mpw_recipe_run_ws over these layers (the largest any
 * one of them needs). */
MPW_API size_t mpw_recipe_workspace_bytes(const mpw_linear* layers, int64_t count, int64_t M);

/* mpw_recipe_run with a decode workspace (see mpw_qlinear_workspace_bytes);
 * the linears that use it run one after another and share it. */
MPW_API mpw_status mpw_recipe_run_ws(const mpw_linear* layers, int64_t count,
                                     uint16_t* const* slots, int64_t num_slots, int64_t M,
                                     void* workspace, size_t workspace_bytes, mpw_stream_t stream);

/*
 * mpw_pass_create / mpw_pass_run / mpw_pass_info / mpw_pass_destroy -- the
 * same decode pass as mpw_recipe_run, planned once and run as ONE persistent
 * kernel per call.
 * Pages: DynaQuant "Step 3" (a stack of linears, each at its own bit width)
 * and "Custom kernel architecture" (in decode the packed bytes streamed are
 * the cost).  Launched one kernel per linear, a linear that depends on its
 * predecessor starts on a nearly idle GPU; the planned pass keeps every SM
 * streaming weights across linears (work items of 16 rows and a run of K;
 * each linear waits, on the device, only for the earlier linears that write
 * what it reads or read or write what it writes).
 *   mpw_pass_create  arguments as mpw_recipe_run (validated alike).  Takes
 *            M == 1, every linear in MPW_LAYOUT_PAIRED with bits 4..8 and
 *            K % 128 == 0 (else MPW_E_UNSUPPORTED: use mpw_recipe_run), and
 *            no linear whose input and output bytes overlap
 *            (MPW_E_INVALID_ARG).  Allocates device memory for the plan
 *            (descriptors, TMA tensor maps, dependency lists, counters and
 *            partial sums: about 128 B per split 16-row tile) and returns it in
 *            *pass.  The plan records the slot and matrix pointers: they must
 *            stay valid, and the slots keep their sizes, while it is used.
 *            Synchronous (host to device copies); not capturable.
 *   mpw_pass_run  zeroes the plan's counters and launches the kernel on
 *            `stream` (capturable in a CUDA graph).  One run at a time per
 *            plan.  Results equal mpw_recipe_run's within the decode
 *            tolerance (linears split along K add their parts' fp32 sums in a
 *            fixed order; not bit-identical to the per-linear kernels).
 *            A device-side wait that gives up sets the error word (kernel 6,
 *            place 11 for the wait on other linears, see mpw_device_error).
 *   mpw_pass_info  info[0..3] = grid size (CTAs), ring stages per CTA, work
 *            items, dynamic shared memory bytes per CTA.
 *   mpw_pass_destroy  frees the plan (after its last run has completed);
 *            NULL is a no-op.
 */
typedef struct mpw_pass mpw_pass;
/* mpw_pass_dependencies -- host only: the earlier linears each linear of the
 * planned pass waits for (those that write bytes it reads, or read or write
 * bytes it writes, minus those another listed one waits for, transitively):
 * linear i waits for deps[offsets[i] .. offsets[i+1]).  offsets has count + 1
 * entries and is always filled on success of the validation; deps must hold
 * offsets[count] entries (else MPW_E_INVALID_ARG, with offsets filled).
 * Arguments and errors as mpw_pass_create; slot pointers are compared, never
 * dereferenced. */
MPW_API mpw_status mpw_pass_dependencies(const mpw_linear* layers, int64_t count, uint16_t* const* slots,
                                         int64_t num_slots, int64_t M, int32_t* offsets, int32_t* deps,
                                         int64_t deps_capacity);
MPW_API mpw_status mpw_pass_create(const mpw_linear* layers, int64_t count, uint16_t* const* slots,
                                   int64_t num_slots, int64_t M, mpw_pass** pass);
MPW_API mpw_status mpw_pass_run(const mpw_pass* pass, mpw_stream_t stream);
MPW_API mpw_status mpw_pass_info(const mpw_pass* pass, int64_t* info);
MPW_API void mpw_pass_destroy(mpw_pass* pass);

/*
 * mpw_allocate_bits -- per-matrix bit widths under a byte budget.
 * Pages: DynaQuant "Step 2: bit allocation" (water filling over a max-heap of
 * marginal bit upgrades: each step raises one matrix to its next level, by
 * quality gain per byte of cost; hardware-native {4, 8, 16} or full 4..16).
 * The gain and the cost are this library's readings: the loss of a matrix at
 * b bits is sens / (2^(b-1) - 1)^2 (zero at 16 bits, the unquantized bf16
 * matrix), its cost the bytes it is stored in here (N * mpw_packed_row_bytes
 * + 4 * N for the scales; 2 * N * K at 16 bits).  Every matrix starts at 4
 * bits; upgrades are taken by gain / extra bytes (fp64), ties to the lower
 * index, and one that no longer fits is dropped while the others go on.
 *   sens    host, double [count]: per-matrix sensitivity, finite and >= 0.
 *   N, K    host, int64 [count]: output rows and inputs of each matrix, in
 *           1 .. 2^31 - 1.
 *   budget  bytes for all matrices together.
 *   mode    MPW_ALLOC_NATIVE or MPW_ALLOC_FULL.
 *   bits    host, int32 [count], written: 4..16 (16 = keep bf16).
 *   total   host, nullable: receives the bytes of the allocation.
 * Runs on the host (no device work, no stream).  Null pointers, count outside
 * 1 .. 2^24, a bad mode or size, a negative or non-finite sensitivity, or a
 * budget below the cost of 4 bits everywhere: MPW_E_INVALID_ARG, nothing
 * written.
 */
typedef enum mpw_alloc_mode {
  MPW_ALLOC_NATIVE = 0, /* {4, 8, 16} */
  MPW_ALLOC_FULL = 1    /* {4, 5, ..., 16} */
} mpw_alloc_mode;
MPW_API mpw_status mpw_allocate_bits(const double* sens, const int64_t* N, const int64_t* K, int64_t count,
                                     uint64_t budget, int mode, int32_t* bits, uint64_t* total);

/*
 * mpw_allocate_frontier -- the trade-off curve the water filling walks
 * (DynaQuant "Step 2": a Pareto-front allocator): the bytes and the total
 * loss (sum of sens / (2^(b-1) - 1)^2, as for mpw_allocate_bits) after each
 * upgrade of the filling without a budget, from 4 bits everywhere to bf16
 * everywhere; each point is the allocation mpw_allocate_bits returns for
 * that many bytes.  The total loss is updated by subtracting each
 * upgrade's gain, in fp64, in that order.
 *   sens, N, K, count, mode  as for mpw_allocate_bits.
 *   bytes, loss  host, [max_points]: the first min(points, max_points)
 *           points (may be NULL when max_points is 0).
 *   n_points  receives the number of points (count * levels-above-4 + 1).
 * Host only.  Errors as for mpw_allocate_bits (there is no budget).
 */
MPW_API mpw_status mpw_allocate_frontier(const double* sens, const int64_t* N, const int64_t* K, int64_t count,
                                         int mode, uint64_t* bytes, double* loss, int64_t max_points,
                                         int64_t* n_points);

/*
 * Packed-weight files (host only).
 * Pages: DynaQuant "Status" (a packed weight format for disk storage is in
 * progress); the format itself is this library's:
 *   header, 32 bytes: "MPWPACK\0", u32 version (1), u32 count, u64 index
 *     offset (32), u64 data offset;
 *   index, 64 bytes per matrix: u64 N, u64 K, u32 bits, u32 layout, u64
 *     packed offset, u64 packed bytes (N * mpw_packed_row_bytes(K, bits)),
 *     u64 scales offset, u32 CRC-32 of the packed bytes, u32 CRC-32 of the
 *     scales, u64 reserved (0);
 *   data: each matrix's packed rows, then its fp32 scales, each at a multiple
 *     of 64 bytes (zero fill).
 * Little-endian throughout; CRC-32 of IEEE 802.3 (as zlib's crc32).
 * Errors: MPW_E_INVALID_ARG (null pointer, bad count or index, bad shape or
 * layout), MPW_E_UNSUPPORTED_BITS, MPW_E_IO (open / read / write failed),
 * MPW_E_FORMAT (not a container of this version, an index entry out of the
 * file, a checksum that differs).
 */
typedef struct mpw_file_matrix {
  int64_t N;
  int64_t K;
  int32_t bits;
  int32_t layout;          /* MPW_LAYOUT_* of the rows, as stored */
  const uint8_t* packed;   /* host, N * mpw_packed_row_bytes(K, bits) bytes */
  const float* scales;     /* host, N */
} mpw_file_matrix;

/* Writes `count` matrices (host buffers) to `path`, replacing the file. */
MPW_API mpw_status mpw_file_write(const char* path, const mpw_file_matrix* matrices, int64_t count);
/* Number of matrices in the file. */
MPW_API mpw_status mpw_file_count(const char* path, int64_t* count);
/* Shape, bit width and layout of matrix `index`. */
MPW_API mpw_status mpw_file_info(const char* path, int64_t index, int64_t* N, int64_t* K, int32_t* bits,
                                 int32_t* layout);
/* Reads matrix `index` into host buffers of the sizes mpw_file_info implies
 * and checks both checksums (MPW_E_FORMAT if either differs; the buffers may
 * then hold the bytes read). */
MPW_API mpw_status mpw_file_read(const char* path, int64_t index, uint8_t* packed, float* scales);

/*
 * mpw_qlinear_noalloc -- the decode linear (M <= 32) on the stream-K kernel,
 * with its workspace taken from a fixed array inside the library instead of
 * from the caller, so that the call allocates no memory of any kind.
 *
 * No page describes this: it has no counterpart in the paper.  It exists for
 * callers that must not allocate device memory at all -- code embedded in a
 * host program that owns every allocation, work recorded where allocation
 * calls are not allowed, or loops with a strict no-allocation rule -- and
 * that therefore cannot provide the workspace mpw_qlinear_ws needs.
 *   - The array holds MPW_NOALLOC_SCRATCH_BYTES (4 MiB) on every device that
 *     loads the library, for the life of the process.  A call whose
 *     workspace would exceed it returns MPW_E_SCRATCH_LIMIT and launches
 *     nothing; mpw_qlinear_workspace_bytes tells the size in advance.
 *     The 27B-class gate/up matrices (17408 x 5120) at M = 32 already need
 *     more and are refused; at M <= 8 they fit.
 *   - The first call on a device looks up the array's device address (once
 *     per device, with that device current); make that first call before any
 *     stream capture.  The address is kept for the life of the process, so
 *     after cudaDeviceReset this entry point must not be called again in
 *     that process.
 *   - Every call shares the array.  Each call clears the per-tile counters
 *     it uses (a memset on `stream`) before its kernel; the partial sums need
 *     no clearing.  Calls that overlap on the GPU (on different streams, or
 *     in different host threads) race on the array and give wrong results.
 *   - Arguments as mpw_qlinear_ex, with M in 1..32, K % 8 == 0 and x 16-byte
 *     aligned (MPW_E_INVALID_ARG / MPW_E_MISALIGNED otherwise).
 */
#define MPW_NOALLOC_SCRATCH_BYTES ((size_t)4 << 20)
MPW_API mpw_status mpw_qlinear_noalloc(const uint16_t* x, const uint8_t* packed, const float* scales,
                                       int bits, int layout, int64_t M, int64_t N, int64_t K,
                                       uint16_t* y, mpw_stream_t stream);

/*
 * FP8 (E4M3) prefill for codes of 4 or 5 bits.
 * Pages: DynaQuant "Custom kernel architecture" (5-7-bit codes expanded to
 * FP8 E4M3 and multiplied on FP8 tensor cores).  E4M3 holds integers exactly
 * up to 16, so codes of b <= 5 (|q| <= 15) are exact; wider codes are
 * refused (MPW_E_UNSUPPORTED_BITS).  The product needs x in E4M3 as well;
 * this library's reading is the tutorial's symmetric per-channel formula per
 * token, with E4M3's largest value 448 as max_int:
 *   sx_m = fl32(max_k |x_mk| / 448) (a zero token: fl32(1 / 448)),
 *   xq_mk = E4M3 of fl32(x_mk / sx_m), round to nearest even, saturating,
 *   y_mn = bf16_rn(s_n * sx_m * sum_k xq_mk q_nk), fp32 accumulation.
 * The result differs from mpw_qlinear's by the rounding of x to E4M3 (at most
 * half an E4M3 step per element, 2^-4 relative); it is exact otherwise.
 *
 * mpw_quantize_x_fp8 -- x bf16 [M, K] -> xq E4M3 bytes [M, K] and sx fp32 [M].
 *   K % 16 == 0; x and xq 16-byte aligned.
 */
MPW_API mpw_status mpw_quantize_x_fp8(const uint16_t* x, int64_t M, int64_t K, uint8_t* xq, float* sx,
                                      mpw_stream_t stream);

/*
 * mpw_qlinear_fp8 -- y = sx * (xq @ q^T) * s on tcgen05 FP8 tensor cores
 * (kind::f8f6f4), for any M (tiles of 256 tokens; M <= 16,776,960).
 *   xq, sx   from mpw_quantize_x_fp8 (several linears may share them).
 *   packed, scales  as produced by mpw_quantize_pack, bits 4 or 5, in
 *            `layout` (MPW_LAYOUT_*; paired needs K % 32 == 0).
 *   y        device, bf16 [M, N].  K % 16 == 0; xq and packed 16-byte aligned.
 */
MPW_API mpw_status mpw_qlinear_fp8(const uint8_t* xq, const float* sx, const uint8_t* packed, const float* scales,
                                   int bits, int layout, int64_t M, int64_t N, int64_t K, uint16_t* y,
                                   mpw_stream_t stream);

/*
 * mpw_gather_shards -- re-orders the gathered outputs of an output-row
 * (N) sharded linear into y.  No page describes tensor parallelism; the
 * partition is this library's: rank r of `world` owns weight rows
 * r * Nl .. r * Nl + Nl - 1 (zero rows past N) and computes y_r [M, Nl] for
 * the replicated x; an all-gather of the y_r (NCCL, by the caller) leaves
 * blocks [world, M, Nl] rank after rank.
 *   blocks  device, bf16 [world, M, Nl].
 *   y       device, bf16 [M, N]: y[m, n] = blocks[n / Nl, m, n % Nl].
 *   N <= world * Nl.  For M = 1 the blocks already are y (the first N
 *   values) and no call is needed.
 */
MPW_API mpw_status mpw_gather_shards(const uint16_t* blocks, int64_t world, int64_t M, int64_t Nl, int64_t N,
                                     uint16_t* y, mpw_stream_t stream);

/*
 * mpw_device_error -- synchronises the current device, returns in *code the
 * library's device-side error word and clears it.  Returns MPW_E_TIMEOUT
 * when the word was set, MPW_OK otherwise.
 *   0      no wait gave up since the word was last read.
 *   other  the first bounded wait (2 s of waiting) inside a TMA / tensor-core
 *          kernel that gave up, as 100 * kernel + place: kernel 1 = per-tile
 *          decode, 2 = tensor-memory decode, 3 = prefill GEMM, 4 = stream-K
 *          decode, 5 = FP8 prefill GEMM, 6 = planned decode pass (mpw_pass_run);
 *          place 1 = x producer waiting for a free stage, 2 = x
 *          producer waiting for its last copies, 3 / 4 = the same for the
 *          weight (or combined) producer, 5 = consumer or MMA issuer waiting
 *          for a loaded stage, 6 = MMA issuer waiting for converted weights,
 *          7 = converter waiting for a loaded weight stage, 8 = converter
 *          waiting for a free tensor-memory stage, 9 = epilogue waiting for
 *          the accumulator, 10 = sums of squares waiting for a loaded x stage,
 *          11 = a pass item waiting for the linears it depends on.  In the
 *          planned pass the other waits give up soon after the first one
 *          did (without codes of their own).
 *          The outputs of the call that gave up, and of calls that depend
 *          on them, are undefined.
 */
MPW_API mpw_status mpw_device_error(int32_t* code);

#ifdef __cplusplus
}
#endif

#endif /* MPW_H_ */
