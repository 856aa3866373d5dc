/*
 * moeq.h -- C ABI of libmoeq.so: the forward pass of one affine-quantised
 * mixture-of-experts FFN layer on an NVIDIA B200 (sm_100a).
 *
 * Weight format (sources: "danveloper/flash-moe" issue thread, the
 * mixed-precision comment; "flash-moe-inference", the matvec_4bit_fma
 * listing; "markbaseengine/MOE_FIX_SUCCESS_EXPERT_WORKS.md", "Why This
 * Worked"):
 *   - a matrix of out_dim rows by in_dim inputs holds unsigned b-bit codes
 *     q, b in {2, 4, 8}, packed 32/b per uint32 word, row-major
 *     ([out_dim][in_dim*b/32] words); value j of a word sits in bits
 *     [j*b, (j+1)*b) (low bits first);
 *   - b in {3, 5, 6} (the mlx issue page's table runs an affine 5-bit
 *     model): each row is one little-endian bit stream of u32 words, value
 *     i at bits [i*b, (i+1)*b), so a value may straddle two words -- the
 *     same rule, extended to widths that do not divide 32; decode path
 *     only;
 *   - each row is cut into groups of group_size consecutive inputs
 *     (64 on the pages; 32 and 128 are also accepted) and each group has
 *     one bf16 scale and one bf16 bias, [out_dim][in_dim/group_size] each;
 *   - the weight is w = q * scale + bias (affine mode);
 *   - bit widths are per tensor, so an 8-bit router sits beside 4-bit
 *     experts.
 * A bank of E experts stores matrix e at w + e*expert_stride_w (words)
 * and scales/biases + e*expert_stride_sb (entries); strides of 0 mean a
 * single matrix.
 *
 * Conventions for every entry point:
 *   - all tensor pointers are DEVICE pointers owned by the caller; the
 *     library never allocates or frees them; descriptor structs may live
 *     in host memory and are read during the call only;
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream); every call is asynchronous on it and does no host
 *     synchronisation and no device allocation;
 *   - arguments are checked on the host before anything is launched; a
 *     failed check returns an error code and launches nothing;
 *   - problems only the device can see (a bounded wait that ran out, an
 *     operand outside the fp16 range of the prefill tiles) set a device
 *     status word, read and cleared by moeq_device_status;
 *   - bf16 values travel as their 16-bit patterns (uint16_t);
 *   - row offsets are 64-bit; no index arithmetic is narrowed to 16 bits.
 */
#ifndef MOEQ_H
#define MOEQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MOEQ_OK = 0,
  MOEQ_ERR_INVALID_ARG = 1,  /* null pointer, size <= 0, K > E, index out of range ... */
  MOEQ_ERR_UNSUPPORTED = 2,  /* bits not in {2,3,4,5,6,8} (prefill: {2,4,8}), group size not in
                                {32,64,128}, sizes beyond limits */
  MOEQ_ERR_ALIGNMENT = 3,    /* pointer not 16-byte aligned, in_dim not a multiple of group_size */
  MOEQ_ERR_WORKSPACE = 4,    /* workspace missing or smaller than moeq_workspace_bytes */
  MOEQ_ERR_CUDA = 5,         /* a CUDA runtime call failed */
  MOEQ_ERR_TIMEOUT = 6,      /* device status: a bounded device-side wait ran out */
  MOEQ_ERR_RANGE = 7         /* device status: a prefill operand exceeded the fp16 range */
} moeq_status;

typedef enum {
  MOEQ_MODE_AUTO = 0,    /* decode while M*K <= 96 (and M <= 64), prefill beyond
                            (decode up to M = 64 for layers prefill cannot take) */
  MOEQ_MODE_DECODE = 1,  /* HBM-bound split-K quantised matvec path */
  MOEQ_MODE_PREFILL = 2  /* sort-by-expert gather-QMM on tcgen05 tensor cores */
} moeq_mode;

/* Code formats of a tensor. */
typedef enum {
  /* w = q * scale + bias per group, bf16 scale and bias ("danveloper/
   * flash-moe" thread and "flash-moe-inference": the affine format) */
  MOEQ_FMT_AFFINE = 0,
  /* MX FP4 (the mlx issue page's mode="mxfp4", bits 4, group_size 32):
   * each 4-bit code is an E2M1 value (bit 3 sign, bits 2..1 exponent, bit 0
   * mantissa: 0, 0.5, 1, 1.5, 2, 3, 4, 6, signed) and each group of 32
   * shares one E8M0 scale byte e, w = e2m1(q) * 2^(e - 127).  scales points
   * at the uint8 exponents (same shape and strides as the affine scales,
   * one byte per entry); biases is unused. */
  MOEQ_FMT_MXFP4 = 1
} moeq_format;

/* One packed tensor or bank of tensors (device memory). */
typedef struct {
  const uint32_t* w;        /* codes, [E][out_dim][in_dim*bits/32] */
  const uint16_t* scales;   /* bf16 bits, [E][out_dim][in_dim/group_size] (MXFP4: uint8) */
  const uint16_t* biases;   /* bf16 bits, same shape as scales (MXFP4: unused) */
  int32_t out_dim;
  int32_t in_dim;
  int32_t bits;             /* 2, 4 or 8; 3, 5 or 6 (decode only): each row one little-endian
                               bit stream, value i at bits [i*b, (i+1)*b), values may
                               straddle words, rows of whole 16-byte runs; MXFP4: 4 */
  int32_t group_size;       /* values per group along in_dim: 64 (or 32, 128; MXFP4: 32) */
  int64_t expert_stride_w;  /* words from one expert's matrix to the next (0: single matrix) */
  int64_t expert_stride_sb; /* scale/bias entries from one expert to the next */
  int32_t format;           /* moeq_format (0, the affine format, when zero-initialised) */
} moeq_qtensor;

/*
 * One layer ("markbaseengine/MOE_ROUTER_WORKS_BREAKTHROUGH.md", "Forward
 * Pass Sequence"; "flash-moe-inference", per-layer pipeline):
 *   router [E][H]; gate, up [E][I][H]; down [E][H][I];
 *   optional shared expert: sh_gate, sh_up [I_sh][H], sh_down [H][I_sh],
 *   and its sigmoid gate sh_expert_gate [1][H] ("danveloper/flash-moe"
 *   thread: mlp.shared_expert_gate, 8-bit).
 */
typedef struct {
  moeq_qtensor router;
  moeq_qtensor gate;
  moeq_qtensor up;
  moeq_qtensor down;
  int32_t has_shared;       /* 0 or 1 */
  moeq_qtensor sh_gate;
  moeq_qtensor sh_up;
  moeq_qtensor sh_down;
  moeq_qtensor sh_expert_gate;
  int32_t hidden;           /* H */
  int32_t inter;            /* I */
  int32_t n_experts;        /* E */
  int32_t top_k;            /* K, 1 <= K <= min(E, 32) */
  int32_t renorm;           /* 1: routed weights renormalised to sum 1 over the K chosen */
  float router_scale;       /* logits are multiplied by this before the softmax (default 1) */
} moeq_layer;

/*
 * Unpack and dequantise matrix `expert` of `t` (source: "flash-moe-inference",
 * dequantised value nibble*scale + bias).
 *   q_out: nullable, uint8 [out_dim][in_dim], the codes;
 *   w_out: nullable, fp32 [out_dim][in_dim], fmaf(q, scale, bias) -- one
 *          correctly rounded fp32 operation, so the result is exact to the bit.
 * Errors: INVALID_ARG (t NULL, both outputs NULL, expert < 0), UNSUPPORTED,
 * ALIGNMENT, CUDA.
 */
moeq_status moeq_dequant(const moeq_qtensor* t, int32_t expert, uint8_t* q_out, float* w_out,
                         void* stream);

/*
 * y[m][r] = sum_g ( s[r,g] * sum_{c in g} q[r,c] x[m][c]  +  b[r,g] * sum_{c in g} x[m][c] )
 * for m < M tokens: the group form of the fma(q, scale*x, bias*x) factoring
 * ("flash-moe-inference", matvec_4bit_fma listing), accumulated in fp32.
 *   x: bf16 [M][in_dim], 16-byte aligned rows; y: fp32 [M][out_dim].
 * 1 <= M <= 64.  Errors: INVALID_ARG, UNSUPPORTED, ALIGNMENT, CUDA.
 */
moeq_status moeq_qmv(const moeq_qtensor* t, int32_t expert, const uint16_t* x, int32_t M, float* y,
                     void* stream);

/*
 * Routing ("markbaseengine/MOE_ROUTER_WORKS_BREAKTHROUGH.md", Forward Pass
 * Sequence steps 3-4; "flash-moe-inference", softmax + topK):
 *   p = softmax(router_scale * logits[m]); the K largest p (ties to the
 *   lower expert index) in order of p descending; w = p_k / sum of the K
 *   chosen p when renorm, else p_k.
 *   logits: fp32 [M][E]; idx: int32 [M][K]; w: fp32 [M][K].
 * 1 <= K <= min(E, 32); E <= 4096; M >= 0 (M = 0 launches nothing).
 * Errors: INVALID_ARG, UNSUPPORTED, CUDA.
 */
moeq_status moeq_route_topk(const float* logits, int32_t M, int32_t E, int32_t K, int32_t renorm,
                            float router_scale, int32_t* idx, float* w, void* stream);

/*
 * Experts and combine with the routing given ("flash-moe-inference",
 * swiglu and moe_combine_residual listings; "markbaseengine/MOE_FIX_SUCCESS_
 * EXPERT_WORKS.md", fused gate/up):
 *   y[m] = sum_k w[m][k] * Wd_e (silu(Wg_e x_m) * (Wu_e x_m)),  e = idx[m][k]
 *          + sigmoid(Wsg x_m) * SharedExpert(x_m)        (if has_shared)
 *          + residual[m]                                  (if residual != NULL)
 * summed over k in order 0..K-1.
 *   x: bf16 [M][H]; idx int32 [M][K] (each in [0,E)); w fp32 [M][K];
 *   residual: nullable fp32 [M][H]; y: fp32 [M][H].
 *   ws: device workspace of at least moeq_workspace_bytes(L, M, mode) bytes,
 *   256-byte aligned, owned by the caller, contents ignored on entry.
 * mode: DECODE requires M <= 64 and rows of at most 4096 bytes of codes.
 * PREFILL requires group sizes of 32, 64 or 128 (32 only for 4- and 8-bit
 * codes), one group size for gate and up and one for the shared expert's
 * gate and up, H, I (and the shared expert's I) multiples of 128 and of
 * 2 * group_size for the tensors that reduce over them, 4-byte aligned
 * scale/bias arrays, and
 * values that fit the fp16 tensor-core operands (|x|, |bias| and
 * |bias + (2^b-1)*scale| at most 65504, every scale exactly representable
 * as fp16: all bf16 scales of magnitude 2^-17 to 65504 are, and smaller
 * ones whose lowest significant bit is at least 2^-24; the SwiGLU outputs
 * and per-expert down rows at most 65504); outside that range the device
 * status reports MOEQ_ERR_RANGE and the outputs are not valid.  The decode
 * path has none of these limits.  The
 * prefill path computes every output row from its own token with the same
 * kernels for any M, so splitting the tokens into chunks gives
 * bit-identical results.  Only PREFILL mode has that property: AUTO picks
 * the path per call from that call's M (decode while M*K <= 96), so a
 * chunked sequence run in AUTO mode whose last chunk is that small gets
 * that chunk from the decode path, whose arithmetic differs (the results
 * agree within the layer tolerance, not bit for bit).  Pass PREFILL for
 * every chunk to keep chunked and one-shot results bit-identical.
 * idx is not read on the host; an index outside [0,E) found on the device
 * sets MOEQ_ERR_INVALID_ARG in the device status word and expert 0 is used
 * in its place.
 * Errors: INVALID_ARG, UNSUPPORTED, ALIGNMENT, WORKSPACE, CUDA.
 */
moeq_status moeq_expert_ffn(const moeq_layer* L, const uint16_t* x, int32_t M, const int32_t* idx,
                            const float* w, const float* residual, float* y, void* ws,
                            size_t ws_bytes, int32_t mode, void* stream);

/*
 * The whole layer: router qmv -> route_topk -> expert_ffn, on the device,
 * with no host round trip.  idx_out/w_out: nullable, receive the routing.
 * Same buffers, workspace and errors as moeq_expert_ffn.
 * Single-token decode (M = 1, here and in moeq_expert_ffn) runs as three
 * lean launches when the layer's formats allow it:
 *   - 2-, 4- or 8-bit affine experts, with a shared expert of the same
 *     width or a 4-bit one beside 2-bit experts;
 *   - an 8-bit router with at most 512 experts, top_k <= 16;
 *   - each CTA's row blocks fitting in shared memory.
 * The launches are the router rows, then top-K with gate/up + SwiGLU, then
 * down + combine.  Other layers and M > 1 use the general decode launches.
 * Both agree with the oracle within the layer tolerance; each is
 * deterministic.
 * The environment variable MOEQ_SINGLE_DECODE=0 (read on every call)
 * selects the general launches for M = 1.  MOEQ_FUSED_DECODE=1 runs a layer
 * whose tensors all use group_size 64 with rows of whole 8-group runs as one
 * persistent launch instead.  That launch gives the same results within the
 * layer tolerance and needs every CTA of its grid resident at once, one per
 * SM.
 */
moeq_status moeq_layer_forward(const moeq_layer* L, const uint16_t* x, int32_t M, float* y,
                               const float* residual, int32_t* idx_out, float* w_out, void* ws,
                               size_t ws_bytes, int32_t mode, void* stream);

/*
 * moeq_layer_forward followed by the step the pages run after the combine,
 * the RMS norm of the combined output ("flash-moe-inference", per-layer
 * pipeline "CMD3: expert forward + combine + norm"; Key Metal kernels
 * rms_norm_pass1 / rms_norm_pass2):
 *   y[m]         as moeq_layer_forward (fp32 [M][H], the residual stream)
 *   y_norm[m][j] = bf16( y[m][j] / sqrt((1/H) sum_i y[m][i]^2 + eps) * gamma[j] )
 *                  (round to nearest even), the next layer's bf16 input.
 *   gamma: bf16 [H] (device, 16-byte aligned); y_norm: bf16 [M][H] (device,
 *   16-byte aligned, written whole); eps > 0 and finite.  The sum of
 *   squares is an fp32 sum in a fixed order, so results are deterministic;
 *   in PREFILL mode the norm runs inside the combine (one pass over the
 *   rows) and chunked calls stay bit-identical; in DECODE mode one row-norm
 *   launch follows the combine.
 * Same workspace as moeq_layer_forward.  Errors: those of
 * moeq_layer_forward; INVALID_ARG for a null gamma or y_norm or a bad eps,
 * ALIGNMENT for a misaligned gamma or y_norm.
 */
moeq_status moeq_layer_forward_norm(const moeq_layer* L, const uint16_t* x, int32_t M, float* y,
                                    const float* residual, const uint16_t* gamma, float eps,
                                    uint16_t* y_norm, int32_t* idx_out, float* w_out, void* ws,
                                    size_t ws_bytes, int32_t mode, void* stream);

/*
 * Expert streaming from host memory with an HBM expert cache
 * ("flash-moe-inference", per-layer pipeline "I/O: parallel pread K=4
 * experts" and the parallel expert loading listing: the routed experts live
 * in slower storage, the K a token selects are read in parallel, the
 * operating system's page cache keeps recent ones, LRU).  Here the slower
 * tier is host memory and the cache holds `slots` experts in HBM, least
 * recently used out first.  For layers whose expert banks do not fit the
 * GPU's memory.
 *
 * moeq_cache_create: L as moeq_layer_forward, except that gate, up and down
 *   (all E experts) are in HOST memory (page-locked, e.g. cudaHostAlloc, so
 *   that the copies run asynchronously); the router and the shared expert
 *   are in device memory.  slots in [K, E]; max_tokens in [1, 64] with
 *   max_tokens * K <= slots (one step's experts always fit).  Allocates the
 *   slot banks and step buffers in device memory (call with the device
 *   current).  Errors: INVALID_ARG, UNSUPPORTED (shapes outside the decode
 *   path), CUDA (allocation).
 * moeq_cache_forward: one decode step of M <= max_tokens tokens on `stream`:
 *   router qmv and top-K on the device, the selection read back to the host
 *   (synchronises `stream`), each selected expert not in a slot copied into
 *   an empty slot or the least recently used slot the step does not use,
 *   then moeq_expert_ffn on the slots.  Outputs as moeq_layer_forward
 *   (decode path).  ws: device workspace of moeq_cache_workspace_bytes(c, M)
 *   bytes.  One stream per cache; not thread-safe.
 * moeq_cache_stats: distinct experts found in a slot (hits) and copied in
 *   (misses) over all steps, and the bytes copied from host memory.
 */
typedef struct moeq_expert_cache moeq_expert_cache;
moeq_status moeq_cache_create(const moeq_layer* L, int32_t slots, int32_t max_tokens,
                              moeq_expert_cache** out);
size_t moeq_cache_workspace_bytes(const moeq_expert_cache* c, int32_t M);
moeq_status moeq_cache_forward(moeq_expert_cache* c, const uint16_t* x, int32_t M, float* y,
                               const float* residual, int32_t* idx_out, float* w_out, void* ws,
                               size_t ws_bytes, void* stream);
moeq_status moeq_cache_stats(const moeq_expert_cache* c, uint64_t* hits, uint64_t* misses,
                             uint64_t* bytes_copied);
void moeq_cache_destroy(moeq_expert_cache* c);

/* Workspace bytes moeq_expert_ffn / moeq_layer_forward need for M tokens
 * in `mode` (0 if the arguments are invalid). */
size_t moeq_workspace_bytes(const moeq_layer* L, int32_t M, int32_t mode);

/*
 * moeq_layer_forward in DECODE mode with the workspace taken from a fixed
 * device array inside this library instead of from the caller.  The paper
 * has no counterpart: the method's pages do not discuss where intermediate
 * buffers live.  This entry point allocates no device or host memory; it is
 * for callers that cannot pass a workspace, because they have no device
 * allocator at the call site or must not allocate while serving (an
 * allocation can synchronise the device; a pool sized at start-up may not
 * grow).
 *   Arguments, layouts and device-side errors are those of
 *   moeq_layer_forward with mode DECODE (M <= 64); its argument checks
 *   (layer, M, x, y, residual) run first and fail with the same status.
 *   Capacity: moeq_static_workspace_capacity() bytes (8 MiB) per device,
 *   which covers for example H 4096, I 1024, E 512, K 4 with a shared
 *   expert up to M 64.  When moeq_workspace_bytes(L, M, DECODE) exceeds it
 *   the call launches nothing and returns MOEQ_ERR_WORKSPACE.
 *   Set-up: the first call on each device (with that device current) looks
 *   up the array's device address; make that first call before any stream
 *   capture begins.  A failed lookup returns MOEQ_ERR_CUDA.
 *   Sharing: all calls on a device use the same array.  Nothing in it has to
 *   start at zero, but calls whose work overlaps in time on one device (on
 *   different streams, or from host threads without ordering between them)
 *   race on it; order such calls (one stream, or events) yourself.
 * Errors: those of moeq_layer_forward, and WORKSPACE / CUDA as above.
 */
moeq_status moeq_layer_forward_static(const moeq_layer* L, const uint16_t* x, int32_t M,
                                      float* y, const float* residual, int32_t* idx_out,
                                      float* w_out, void* stream);

/* Bytes of the fixed per-device workspace of moeq_layer_forward_static. */
size_t moeq_static_workspace_capacity(void);

/* Reads and clears the device status word of the current device (synchronises
 * `stream`).  *status_out receives MOEQ_OK or the first device error seen. */
moeq_status moeq_device_status(void* stream, int32_t* status_out);

/*
 * Failure-path self test (the pages have no counterpart).  Launches one CTA
 * on `stream` whose two bounded waits, the kinds every kernel of this
 * library uses, run out: warp 0 waits on an mbarrier phase that never
 * completes, warp 1 polls a device flag that nothing sets.  Each gives up
 * after about two seconds, sets MOEQ_ERR_TIMEOUT in the device status word
 * and returns, so the context stays usable (read the word with
 * moeq_device_status).  Asynchronous; returns CUDA if the launch fails.
 */
moeq_status moeq_selftest_wait_timeout(void* stream);

/*
 * Diagnostics for benchmarks.
 *
 * moeq_set_profile_events: when `start` and `stop` are cudaEvent_t handles
 * (passed as void*), every later moeq_layer_forward / moeq_expert_ffn call
 * made from the same host thread records `start` on its stream right before
 * its main weight-streaming kernel (decode: the gate/up GEMV; prefill: the
 * gate/up gather-QMM) and `stop` right after it, so cudaEventElapsedTime
 * gives that kernel's duration.  Recording also works while the stream is
 * being captured into a CUDA graph.  NULL, NULL turns it off.  The caller
 * owns the events.  Returns INVALID_ARG if exactly one of them is NULL.
 *
 * moeq_launch_count: number of kernels this library has launched (or added
 * to a graph being captured) from any thread since it was loaded.
 */
moeq_status moeq_set_profile_events(void* start, void* stop);
uint64_t moeq_launch_count(void);

/* Text of a status code (static storage). */
const char* moeq_status_str(int32_t status);

/* Library version string (static storage). */
const char* moeq_version(void);

#ifdef __cplusplus
}
#endif

#endif /* MOEQ_H */
