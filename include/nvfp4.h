/*
 * nvfp4.h -- C ABI of the NVFP4 W4A4 linear layer for B200 (sm_100a).
 *
 * The layer is the one every linear layer of the hybrid Gated DeltaNet /
 * attention model becomes in the paper "Why Gated DeltaNet Survives 4-Bit
 * Quantization: NVFP4 W4A4 for the Recurrent Half of a Hybrid 27B LLM":
 * 4-bit weights and 4-bit activations in NVFP4 (nefut abstract, "Minima:
 * NVFP4 W4A4, quantizing all 496 linear layers"), 16-element block scaling
 * (bayesiansapien wiki, "The four-part mechanism study", part 1), fused
 * multi-module projections whose per-module global scales are applied
 * separately (wiki, "Two practical repairs"; aimodeling, "What engineers
 * should actually take away"), optionally followed by the GDN gate
 * nonlinearities (wiki, mechanism study part 2).
 *
 * Number format (the pages give none; these are the readings the library
 * implements):
 *   codes   E2M1, 4 bits, magnitudes {0,.5,1,1.5,2,3,4,6}, bit 3 = sign.
 *           Packed two per byte along K: element 2i in the LOW nibble.
 *   scales  unsigned E4M3 (bias 7, max 448), one per 16 consecutive K elements.
 *   gs      FP32 global scale per tensor (per module for fused weights),
 *           gs = fp32(amax) / fp32(2688).
 *   quantize: s = E4M3_RNE_satfinite(fp32(amax16 / fp32(6 gs)));
 *             q = E2M1_RNE_satfinite(fp32(x * fp32(1 / fp32(s_dec gs)))),
 *             all codes 0 when s_dec == 0.
 *
 * Memory layouts (all buffers are owned by the caller; the library never
 * allocates memory and never frees it):
 *   bf16 inputs   row-major [rows, ld], ld >= K elements, ld % 8 == 0,
 *                 base 16-byte aligned.
 *   codes         dense row-major uint8 [rows, K/2] (row stride K/2 bytes),
 *                 nvfp4_codes_bytes(rows, K) bytes, base 16-byte aligned.
 *   scales        "128x4 atom" layout consumed by tcgen05 block-scaled MMA:
 *                 the byte of logical scale S[r, j] (row r, block j = k/16)
 *                 sits at
 *                   ((r/128) * (K/64) + j/4) * 512 + (r%32) * 16
 *                     + ((r/32)%4) * 4 + j%4
 *                 Rows are padded to a multiple of 128; padding bytes are
 *                 written as 0 by the quantisers.  nvfp4_scale_bytes(rows, K)
 *                 bytes, base 16-byte aligned.
 *   outputs y     row-major [M, ldy], ldy >= N, bf16 (ldy % 8 == 0) or fp32
 *                 (ldy % 4 == 0), base 16-byte aligned.
 *
 * Shapes: K % 64 == 0 and K >= 64; N % 16 == 0; M >= 0 (M == 0 is a no-op).
 *
 * Errors: every call returns an nvfp4_status and never throws.  Arguments
 * are validated on the host before anything is launched; validation
 * failures return INVALID_ARG / ALIGNMENT / UNSUPPORTED_SHAPE without
 * touching the GPU.  Launch failures return NVFP4_ERR_CUDA.  Kernels never
 * trap: every wait inside a kernel is bounded in time, and a wait that runs
 * out records a device error word and makes the kernel return;
 * nvfp4_last_device_error() reads (and clears) it.  NaN/Inf inputs are
 * outside the contract (results undefined, no fault).
 *
 * Streams: `stream` is a cudaStream_t (NULL = legacy default stream).  All
 * calls are asynchronous on that stream except nvfp4_quantize_weight() and
 * nvfp4_last_device_error(), which synchronise it.
 *
 * Per-device state: the library caches, per device, its capability checks,
 * kernel attributes, occupancy figures and TMA descriptors (keyed by
 * pointer and shape).  They stay valid for the life of the device's primary
 * context; after cudaDeviceReset the library must not be called on that
 * device again in the same process.
 */
#ifndef NVFP4_H_
#define NVFP4_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#pragma GCC visibility push(default)
#endif

typedef struct CUstream_st* nvfp4_stream_t; /* same type as cudaStream_t */

typedef enum {
  NVFP4_OK = 0,
  NVFP4_ERR_INVALID_ARG = -1,        /* null pointer, bad enum, bad segment table, bad scale */
  NVFP4_ERR_ALIGNMENT = -2,          /* pointer or leading dimension not 16-byte aligned */
  NVFP4_ERR_UNSUPPORTED_SHAPE = -3,  /* K % 64, N % 16, ld < K, ... */
  NVFP4_ERR_CUDA = -4,               /* a CUDA runtime/driver call failed */
  NVFP4_ERR_TIMEOUT = -5,            /* a bounded in-kernel wait ran out */
  NVFP4_ERR_UNSUPPORTED_DEVICE = -6  /* current device is not compute capability 10.0 */
} nvfp4_status;

typedef enum {
  NVFP4_OP_NONE = 0,      /* y = alpha * acc */
  NVFP4_OP_SIGMOID = 1,   /* beta = 1 / (1 + exp(-alpha * acc)) */
  NVFP4_OP_GDN_DECAY = 2  /* g = -exp(A_log[h]) * softplus(alpha * acc + dt_bias[h]) */
} nvfp4_op;

typedef enum {
  NVFP4_OUT_BF16 = 0,     /* round to nearest even */
  NVFP4_OUT_FP32 = 1      /* the fp32 epilogue value before bf16 rounding (test mode) */
} nvfp4_out_dtype;

/* One module of a fused projection: columns [n_offset, next n_offset) of y.
 * alpha = fp32(a_gs * w_gs) is applied to that module's columns only -- the
 * global-scale mismatch repair.  For NVFP4_OP_GDN_DECAY, a_log and dt_bias
 * are DEVICE pointers to `width` floats each (h = column - n_offset);
 * otherwise they are ignored. */
typedef struct {
  int64_t n_offset;
  float w_gs;
  float a_gs;
  int32_t op;
  const float* a_log;
  const float* dt_bias;
} nvfp4_segment;

#define NVFP4_MAX_SEGMENTS 32

/* Byte sizes of the code and scale buffers for `rows` x K elements. */
size_t nvfp4_codes_bytes(int64_t rows, int64_t K);
size_t nvfp4_scale_bytes(int64_t rows, int64_t K);   /* ceil(rows/128)*128 * K/16 */

/* gs = fp32(amax) / fp32(2688) (reading of the calibrated FP32 per-tensor
 * global scale; host arithmetic, IEEE division).  amax == 0 gives 1: an
 * all-zero tensor quantises to zero codes and scales under any positive gs. */
float nvfp4_global_scale(float amax);

/* amax_dev[0] = max |x| over x[0:R, 0:K] (bf16, row stride ldx elements).
 * amax_dev: caller-owned DEVICE float (the result, overwritten).  Used for
 * static activation calibration (calibration-only PTQ: aimodeling "Where the
 * taboo came from") and for weight global scales. */
nvfp4_status nvfp4_amax(const void* x_bf16, int64_t R, int64_t K, int64_t ldx,
                        float* amax_dev, nvfp4_stream_t stream);

/* Activation quantisation (step a1): bf16 x [M, K] -> codes [M, K/2] and
 * scales (atom layout, padding rows zeroed) under the static global scale
 * a_gs > 0.  The operation is the NVFP4 16-element block scaling of the
 * activations (bayesiansapien wiki, "The four-part mechanism study", part 1;
 * nefut abstract: all linear layers W4A4) under a calibrated static scale
 * (aimodeling, "Where the taboo came from": calibration-only PTQ).  All
 * pointers are caller-owned device memory; x is read, codes and scales are
 * overwritten.  Arguments are checked before any launch (INVALID_ARG,
 * ALIGNMENT, UNSUPPORTED_SHAPE); the kernel is queued on `stream`. */
nvfp4_status nvfp4_quantize_act(const void* x_bf16, int64_t M, int64_t K, int64_t ldx,
                                float a_gs, void* codes, void* scales,
                                nvfp4_stream_t stream);

/* Weight quantisation (step a2, offline; the W4 half of W4A4, nefut
 * abstract, with one global scale per module as the fused-projection repair
 * needs: bayesiansapien wiki, "Two practical repairs").  W [N, K] bf16 is
 * split into modules at seg_offsets (HOST array of nseg ascending row offsets, first 0,
 * each a multiple of 16; NULL with nseg == 1 means one module).  Each module
 * gets its own w_gs = amax(module)/2688, written to w_gs_out (HOST array of
 * nseg floats), and is quantised with it into the shared codes / scales
 * buffers (padding rows zeroed).  `workspace` is caller-owned DEVICE scratch
 * of nvfp4_quantize_weight_workspace_bytes(nseg) bytes (the per-module amax
 * reduction); its contents on entry do not matter.  Synchronises `stream`
 * and returns once the codes and scales are written. */
size_t nvfp4_quantize_weight_workspace_bytes(int32_t nseg);
nvfp4_status nvfp4_quantize_weight(const void* w_bf16, int64_t N, int64_t K, int64_t ldw,
                                   const int64_t* seg_offsets, int32_t nseg,
                                   float* w_gs_out, void* codes, void* scales,
                                   void* workspace, nvfp4_stream_t stream);

/* Weight quantisation that allocates nothing and takes no workspace.
 * The paper has no counterpart; this is a library convenience.
 * Some callers cannot call cudaMalloc at all: a serving runtime or plugin
 * host that owns every byte of device memory through its own arena and hands
 * an operator only its input and output buffers, or an embedded caller whose
 * device-memory budget is fixed when it starts.  Such callers cannot create
 * the workspace nvfp4_quantize_weight needs.  This entry point computes the
 * same result (same codes, scales and w_gs) with its per-module amax scratch
 * in a fixed array inside the library: NVFP4_NOALLOC_MAX_SEGMENTS floats
 * (128 bytes), which every GPU that loads the library keeps until the
 * process exits.  nseg above NVFP4_NOALLOC_MAX_SEGMENTS is rejected with
 * NVFP4_ERR_INVALID_ARG before anything runs.  The first call on a device
 * looks up the array's device address (cudaGetSymbolAddress) with that
 * device current; make that first call before any stream capture.  All
 * calls share the one array per device: the accumulators are cleared on
 * `stream` at the start of every call, and calls whose work overlaps on the
 * GPU (e.g. on different streams) race on it.  The looked-up address is kept
 * for the life of the process: after cudaDeviceReset (or any teardown of the
 * device's primary context) it no longer names the array, so the library
 * must not be called on that device again.  Arguments, layouts and the
 * synchronisation of `stream` are those of nvfp4_quantize_weight. */
#define NVFP4_NOALLOC_MAX_SEGMENTS 32
nvfp4_status nvfp4_quantize_weight_noalloc(const void* w_bf16, int64_t N, int64_t K, int64_t ldw,
                                           const int64_t* seg_offsets, int32_t nseg,
                                           float* w_gs_out, void* codes, void* scales,
                                           nvfp4_stream_t stream);
/* The module limit of nvfp4_quantize_weight_noalloc as compiled into the
 * library (NVFP4_NOALLOC_MAX_SEGMENTS), for callers that bind the library
 * without this header. */
int32_t nvfp4_noalloc_max_segments(void);

/* Block-scaled FP4 x FP4 GEMM (step a3) with a single module (step a4 with
 * op NONE): y[m, n] = fp32(a_gs * w_gs) * sum_k e2m1(qa[m,k]) sa[m,k/16]
 * e2m1(qw[n,k]) sw[n,k/16], accumulated in fp32 — the product of the
 * dequantised operands (nefut abstract: W4A4 linear layers).  a_* describe
 * the quantised activations [M, K], w_* the quantised weights [N, K] (both
 * K-major, y = x W^T), y is bf16 (or fp32) [M, N] with row stride ldy.
 * Caller-owned device pointers; y is overwritten, nothing else is written.
 * Errors as for nvfp4_fused_linear. */
nvfp4_status nvfp4_linear(const void* a_codes, const void* a_scales, float a_gs,
                          const void* w_codes, const void* w_scales, float w_gs,
                          int64_t M, int64_t N, int64_t K,
                          void* y, int64_t ldy, nvfp4_out_dtype out_dtype,
                          nvfp4_stream_t stream);

/* Fused multi-module projection (steps a3 + a4): one GEMM over the
 * concatenated weight [N, K]; the epilogue applies each module's own alpha =
 * fp32(a_gs * w_gs) — the repair of the global-scale mismatch of fused
 * kernels (bayesiansapien wiki, "Two practical repairs"; aimodeling, "What
 * engineers should actually take away") — and its op: none, beta =
 * sigmoid(y), or g = -exp(A_log[h]) * softplus(y + dt_bias[h]) with h the
 * column within the module (the GDN gates: wiki, mechanism study part 2).
 * segs: HOST array of nseg (1..NVFP4_MAX_SEGMENTS) entries, n_offset
 * strictly ascending, first 0, each a multiple of 16 and < N; copied during
 * the call; a_log / dt_bias are device arrays of the module's width (decay
 * modules only).  For M <= 64 the small-M weight-streaming kernel is used
 * (step a5), otherwise the persistent tensor-core kernel.  Requires K % 64
 * == 0, N % 16 == 0, 16-byte aligned pointers, ldy >= N (a multiple of 8
 * bf16 / 4 fp32 elements); violations return before any launch.  The
 * kernel is queued on `stream`; a bounded in-kernel wait that runs out is
 * reported by nvfp4_last_device_error. */
nvfp4_status nvfp4_fused_linear(const void* a_codes, const void* a_scales,
                                const void* w_codes, const void* w_scales,
                                int64_t M, int64_t N, int64_t K,
                                const nvfp4_segment* segs, int32_t nseg,
                                void* y, int64_t ldy, nvfp4_out_dtype out_dtype,
                                nvfp4_stream_t stream);

/* Workspace of nvfp4_fused_linear_ws: NVFP4_GEMM_WS_COUNTER_BYTES of flags
 * followed by 256 KB fp32 partial tiles, one per CTA pair of the launch. */
#define NVFP4_GEMM_WS_COUNTER_BYTES 4096
#define NVFP4_GEMM_WS_MAX_UNITS 128

/* Bytes of a workspace large enough for any launch of
 * nvfp4_fused_linear_ws (NVFP4_GEMM_WS_COUNTER_BYTES + 128 partial tiles,
 * about 32 MB; a B200 runs 74 CTA pairs).  Any device. */
size_t nvfp4_gemm_workspace_bytes(void);

/* nvfp4_fused_linear with a caller-owned device workspace that lets the
 * CTA-pair kernel balance its last, partial wave of tiles (a stream-K
 * tail): when the 256 x 256 tiles are not a multiple of the pairs, the last
 * (pairs + remainder) tiles are cut into equal ranges of k-tiles, one per
 * pair, after the pairs' whole tiles.  A tile shared by two pairs is
 * finished by the pair that runs its first k-tiles: the other pair
 * publishes its fp32 partial tile in the workspace, and the sum is always
 * formed as (first k-tiles) + (last k-tiles), so results do not depend on
 * timing.  They differ from nvfp4_fused_linear's by fp32 rounding only.
 * workspace: 16-byte aligned; its first NVFP4_GEMM_WS_COUNTER_BYTES must be
 * zero before its first use (every call that completes without an error
 * leaves them zero; after a bounded wait ran out, clear them again); it
 * must not be in use by another call that may run at the same time.
 * workspace_bytes below NVFP4_GEMM_WS_COUNTER_BYTES + (pairs) x 256 KB, or
 * a NULL workspace, runs every tile whole, exactly like
 * nvfp4_fused_linear.  Other arguments, layouts and errors as for
 * nvfp4_fused_linear; an unaligned workspace returns NVFP4_ERR_ALIGNMENT. */
nvfp4_status nvfp4_fused_linear_ws(const void* a_codes, const void* a_scales,
                                   const void* w_codes, const void* w_scales,
                                   int64_t M, int64_t N, int64_t K,
                                   const nvfp4_segment* segs, int32_t nseg,
                                   void* y, int64_t ldy, nvfp4_out_dtype out_dtype,
                                   void* workspace, size_t workspace_bytes,
                                   nvfp4_stream_t stream);

/* The MLP pair's first half in one kernel (gate_up GEMM, SiLU(gate) * up
 * and the NVFP4 quantisation of the product that the down projection
 * consumes; the all-linear-layers W4A4 recipe: nefut abstract).  The weight
 * [2H, K] holds the gate module's H rows, then the up module's H rows, each
 * quantised with its own global scale (w_gs_gate, w_gs_up).  For every
 * activation row m and h < H:
 *   g = bf16(fp32(a_gs * w_gs_gate) * acc_gate[m, h]),
 *   u = bf16(fp32(a_gs * w_gs_up) * acc_up[m, h]),
 *   h = bf16(g / (1 + exp(-g)) * u)        (fp32 steps, as nvfp4_silu_mul),
 * and h [M, H] is quantised under the static global scale h_gs exactly as
 * nvfp4_quantize_act quantises it: h_codes [M, H/2], h_scales
 * nvfp4_scale_bytes(M, H) bytes in the atom layout (padding rows zero).
 * The result equals nvfp4_fused_linear (bf16 out, segments gate | up) ->
 * nvfp4_silu_mul -> nvfp4_quantize_act bit for bit, without the bf16
 * [M, 2H] and [M, H] intermediates.  Requires H % 128 == 0, K % 64 == 0,
 * 16-byte aligned caller-owned device pointers, finite positive scales;
 * violations return before any launch.  Queued on `stream`. */
nvfp4_status nvfp4_gate_up_silu_quantize(const void* a_codes, const void* a_scales,
                                          const void* w_codes, const void* w_scales,
                                          int64_t M, int64_t H, int64_t K,
                                          float a_gs, float w_gs_gate, float w_gs_up,
                                          float h_gs, void* h_codes, void* h_scales,
                                          nvfp4_stream_t stream);

/* MLP glue between the two projections of the MLP pair (not an NVFP4 step):
 * h[m, j] = bf16(silu(gu[m, j]) * gu[m, H + j]) for j < H, computed in fp32.
 * gu: bf16 [M, ld_in] with ld_in >= 2H; h: bf16 [M, ld_out], ld_out >= H.
 * H % 8 == 0. */
nvfp4_status nvfp4_silu_mul(const void* gu_bf16, int64_t M, int64_t H, int64_t ld_in,
                            void* h_bf16, int64_t ld_out, nvfp4_stream_t stream);

/* FP8 KV cache: the pages' other shipped recipe, calibrated per-tensor FP8
 * E4M3 KV-cache scales ("quantize everything, ship KV scales": nefut
 * abstract; aimodeling, "What engineers should actually take away").
 * nvfp4_kv_scale: fp32(amax) / 448 of a calibration batch (1 when amax <= 0;
 * amax from nvfp4_amax).  nvfp4_kv_quantize_fp8: out[i] = sign(x[i]) |
 * E4M3_RNE_satfinite(|fp32(x[i] * fp32(1 / scale))|) for n bf16 values x
 * (device, 16-byte aligned; n % 8 == 0) into n bytes of out (device,
 * 16-byte aligned); values past the calibrated range saturate at +-448 and
 * zeros keep their sign.  Caller-owned buffers; violations return before any
 * launch; queued on `stream`. */
float nvfp4_kv_scale(float amax);
nvfp4_status nvfp4_kv_quantize_fp8(const void* x_bf16, int64_t n, float scale, void* out_e4m3,
                                   nvfp4_stream_t stream);

/* Gated DeltaNet state recurrence over T tokens of one sequence (the step
 * after the GDN in-projection; the pages' third mechanism: each write
 * overwrites the state along its key direction -- bayesiansapien wiki, "The
 * four-part mechanism study", part 3; the formula is the published gated
 * delta rule):  S_t = exp(g_t) S_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t
 * k_t^T,  o_t = S_t q_t, per value head.  Device fp32 arrays, token-major:
 * q, k [T, Hv/group, 128] (k rows of unit length), v and o [T, Hv, 128],
 * g (log decay, <= 0) and beta [T, Hv], state [Hv, 128 (value), 128 (key)]
 * holding the initial state on entry and the final state on return.  Value
 * head h reads key head h / group.  head_dim must be 128; pointers 16-byte
 * aligned.  Computed chunk by chunk (64 tokens) in fp32.  Queued on
 * `stream`. */
nvfp4_status nvfp4_gdn_recurrence(const float* q, const float* k, const float* v,
                                  const float* g, const float* beta, int64_t T, int32_t Hv,
                                  int32_t group, int32_t head_dim, float* o, float* state,
                                  nvfp4_stream_t stream);

/* Human-readable status. */
const char* nvfp4_status_string(nvfp4_status status);

/* Synchronises `stream`, then reads and clears the device error word that
 * bounded in-kernel waits set when they run out.  Returns NVFP4_OK or
 * NVFP4_ERR_TIMEOUT (info, if non-NULL, receives the raw word: bits 63..48
 * site code, 47..32 role, 31..0 block index), or NVFP4_ERR_CUDA. */
nvfp4_status nvfp4_last_device_error(nvfp4_stream_t stream, uint64_t* info);

/* Kernel-path selection for tests: 0 = automatic (M <= 64 -> small-M
 * kernel, 64 < M <= 128 -> one-CTA tensor-core kernel, M > 128 -> CTA-pair
 * tensor-core kernel), 1 = always the one-CTA tensor-core kernel (128 x 256
 * tiles), 2 = always the small-M kernel (requires M <= 64), 3 = always the
 * CTA-pair tensor-core kernel (256 x 256 tiles on clusters of two CTAs),
 * 4 = the CTA-pair kernel with its tiles walked N fastest (the order chosen
 * automatically when the activation codes exceed 64 MB and the weight codes
 * are smaller).  Process-wide. */
nvfp4_status nvfp4_set_gemm_path(int32_t path);

/* Launch overlap (process-wide, off by default; on = 1, off = 0): the
 * activation quantiser and every GEMM (nvfp4_linear, nvfp4_fused_linear,
 * nvfp4_fused_linear_ws, nvfp4_gate_up_silu_quantize) are launched with
 * programmatic stream serialization, so that each may start while the
 * kernel ahead of it on the stream is still running: its setup and the
 * first stages of its weight stream overlap that kernel's tail (the decode
 * loop of consecutive layers; the last partial wave of a large GEMM).  The
 * quantiser waits for the kernel ahead before it reads x or writes codes
 * and scales.  A GEMM waits for it before it reads the activation codes or
 * any scales and before it writes y (h) or its workspace, but streams the
 * weight codes from its start (the small-M GEMM also the weight scales):
 * with overlap on, the kernel launched just ahead of a GEMM on the same
 * stream must not write that GEMM's weight codes or scales (weights
 * quantised offline, or any other kernel in between, satisfy this).
 * Results are identical with overlap on or off. */
nvfp4_status nvfp4_set_launch_overlap(int32_t on);

/* Time limit of every bounded in-kernel wait, in nanoseconds (default 2e9;
 * also read once from the environment variable NVFP4_SPIN_LIMIT_NS). */
nvfp4_status nvfp4_set_wait_limit_ns(uint64_t limit_ns);

/* ---- test entry points (conversion checks; not part of the layer) ------ */

/* out[i] = E2M1 code of in[i] (fp32 -> E2M1, RNE, satfinite), with the same
 * device conversion the activation quantiser uses.  Device pointers. */
nvfp4_status nvfp4_test_e2m1(const float* in, uint8_t* out, int64_t n, nvfp4_stream_t stream);
/* out[i] = unsigned E4M3 code of in[i] >= 0 (RNE, satfinite), the quantiser's
 * block-scale conversion.  Device pointers. */
nvfp4_status nvfp4_test_e4m3(const float* in, uint8_t* out, int64_t n, nvfp4_stream_t stream);
/* Launches one CTA that waits on an mbarrier nobody arrives on, with the
 * wait limit set to limit_ns; returns what nvfp4_last_device_error reports
 * (NVFP4_ERR_TIMEOUT when the bound works).  Synchronises `stream`. */
nvfp4_status nvfp4_test_wait_timeout(uint64_t limit_ns, nvfp4_stream_t stream);

#if defined(__GNUC__)
#pragma GCC visibility pop
#endif

#ifdef __cplusplus
}
#endif

#endif /* NVFP4_H_ */
