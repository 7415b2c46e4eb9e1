/*
 * lsq.h - C ABI of the streamed NF4-LoRA training path on one B200 (sm_100a).
 *
 * The method: the frozen base of a Llama/Qwen decoder stack is quantised once,
 * offline, to blockwise NF4 and kept in page-locked host RAM; during training
 * each decoder layer's quantised bytes are copied into a small pool of HBM
 * slots on a copy stream while the previous layer computes, forward
 * 0 -> L-1 and, under gradient checkpointing, backward L-1 -> 0; only the LoRA
 * adapters train.  Sources: "Soup" README snapshot (headline + "Citing Soup");
 * soup-cli 0.72.0 -> 0.72.2 diff, CHANGELOG [0.72.2] and
 * docs/performance-and-quantization.md "Layer Streaming" / "NF4 streaming";
 * themenonlab blog "The trick: layer streaming"; aiany.app listing "How It
 * Works".  The pages fix no kernel; formats that they leave open are stated
 * below as readings.
 *
 * Conventions for every call:
 *  - The caller owns every buffer.  Device pointers are CUDA device memory of
 *    the current device; "host pinned" means page-locked host memory
 *    (cudaHostAlloc / cudaHostRegister).  The library allocates no device
 *    memory on any call below; scratch is passed in as `workspace`.
 *  - A workspace (and a rank state) serves one call at a time: calls that
 *    share one must be ordered on the GPU (the same stream, or events).  The
 *    caller orders its own buffers the same way: memory a call reads or
 *    writes must not be in use by work on another stream that the call's
 *    stream does not wait for.
 *  - bf16 means IEEE bfloat16 (2 bytes); all matrices are row-major, dense,
 *    with the stated leading dimension equal to the row length.
 *  - Calls are asynchronous: they validate, enqueue on the given stream and
 *    return.  A NULL stream means the legacy default stream.
 *  - Errors are returned, never thrown, and nothing is enqueued when a call
 *    returns non-OK.  lsq_last_error() gives a message for the calling thread.
 *    Kernels never trap: a bounded device-side wait that expires records
 *    LSQ_ETIMEOUT in a device status word read by lsq_device_status().
 */
#ifndef LSQ_H_
#define LSQ_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* lsq_cuda_stream; /* a cudaStream_t */

typedef enum lsq_status {
  LSQ_OK = 0,
  LSQ_EINVAL = 1,       /* bad argument: size, alignment, NULL pointer */
  LSQ_ENOTPINNED = 2,   /* a host source is not page-locked */
  LSQ_ECUDA = 3,        /* a CUDA runtime call failed (message in lsq_last_error) */
  LSQ_ETIMEOUT = 4,     /* a bounded device wait expired */
  LSQ_ESTATE = 5,       /* call out of order (stream scheduler) */
  LSQ_EUNSUPPORTED = 6, /* device is not sm_100 or a limit of this build */
  LSQ_ECALLBACK = 7     /* a caller-supplied callback reported failure */
} lsq_status;

/* Static message for a status code. */
const char* lsq_status_str(lsq_status s);
/* Message of the last non-OK status returned on this host thread ("" if none). */
const char* lsq_last_error(void);
/* ABI version: 100 * major + minor. */
int lsq_version(void);
/* Reads and clears the device status word of the current device (a
 * synchronous cudaMemcpy): *status = LSQ_OK or the first device-side error
 * since the last read, *where = the site code of that error. */
lsq_status lsq_device_status(int32_t* status, int32_t* where);
/* Enqueues on `stream` one thread that waits until the device word *flag
 * (8-byte aligned) equals value, read with acquire semantics at GPU scope, and
 * gives up after limit_ns nanoseconds (1 .. 1e10) of the global timer,
 * recording LSQ_ETIMEOUT at site 901 in the device status word; work after it
 * on the stream then runs normally.  The same bounded wait guards the fused
 * GEMM's stream-K partials; exposed for stream-ordered signalling and to test
 * the timeout path without faulting the device. */
lsq_status lsq_wait_flag(const uint64_t* flag, uint64_t value, int64_t limit_ns, lsq_cuda_stream stream);

/* ------------------------------------------------------------------------
 * NF4 blockwise format.
 *
 * Pages: the streamed base is "quantised once, offline, one tensor at a
 * time" to NF4 (soup-cli diff, docs "NF4 streaming (quantization: 4bit)";
 * CHANGELOG [0.72.2]).  Readings (the pages give no format): the 16-level
 * NormalFloat codebook of QLoRA (8 positive and 7 negative normal quantiles,
 * an exact 0, scaled to [-1, 1]); block = 64 consecutive elements of a
 * row-major [n_out, k_in] weight (k_in % 64 == 0); one fp32 absmax per block,
 * stored row-major [n_out][k_in/64]; code = nearest level to w/absmax (fp32
 * division, ties to the lower level, all-zero block -> absmax 0, codes 7);
 * two codes per byte, first element in the high nibble; dequantised value
 * bf16_rn(fp32(level) * absmax).
 * ---------------------------------------------------------------------- */
typedef struct lsq_nf4_weight {
  const uint8_t* codes; /* device, n_out*k_in/2 bytes, 16-byte aligned */
  const float* absmax;  /* device, n_out*(k_in/64) fp32, 4-byte aligned */
  int64_t n_out;        /* rows (output features), >= 1, multiple of 8 */
  int64_t k_in;         /* columns (input features), multiple of 64 */
} lsq_nf4_weight;

/* Copies the library's 16 NF4 levels (ascending fp32) into host array out. */
lsq_status lsq_nf4_codebook(float out[16]);

/* Quantise a bf16 weight (device, [n_out, k_in] row-major) into codes
 * (device, n_out*k_in/2 bytes) and absmax (device, n_out*k_in/64 fp32).
 * Definition: "NF4 blockwise format" above.  Bit-exact with a CPU
 * implementation of that definition.  EINVAL on k_in % 64 or NULLs. */
lsq_status lsq_nf4_quantize(const void* w_bf16, int64_t n_out, int64_t k_in, uint8_t* codes, float* absmax,
                            lsq_cuda_stream stream);

/* Dequantise into a bf16 [n_out, k_in] device buffer (the exact values the
 * fused kernels feed to the tensor cores); for tests and diagnostics. */
lsq_status lsq_nf4_dequantize(const lsq_nf4_weight* w, void* w_bf16, lsq_cuda_stream stream);

/* ------------------------------------------------------------------------
 * Double-quantised absmax (8-bit second level).
 *
 * Pages: the 8B base store is 3.60 GB and each layer buffer 113 MB ("Soup"
 * README, layer-streaming figure and its benchmark table) - the size of 4-bit
 * codes plus about one byte, not four, per 64-weight block.  Construction:
 * QLoRA's double quantization (Dettmers et al. 2023, sec. 3: the absmax
 * constants quantised again to 8-bit floats in blocks of 256, after
 * centring).  Readings: the 8-bit float is E4M3 (bias 7, 3 mantissa bits,
 * largest finite 448); per block of 256 consecutive absmax values of one
 * tensor (the last block may be shorter), lo / hi = its smallest / largest
 * value, centre = fp32(fp32(hi + lo) * 0.5), half = fp32(fp32(hi - lo) * 0.5),
 * scale = fp32(half / 448); code = E4M3 nearest to fp32(fp32(a - centre) /
 * scale), ties to even, saturating at +-448, zero stored as +0; scale 0
 * stores code 0.  Expansion: a' = fp32(fp32(e4m3(code) * scale) + centre).
 *
 * lsq_absmax_double_quantize: absmax fp32 [nb] -> codes u8 [nb] and params
 *   fp32 [ceil(nb/256)][2] = (centre, scale).  Device pointers; absmax 4-byte,
 *   params 8-byte aligned.  Bit-exact with a CPU implementation of the
 *   definition.  EINVAL on NULLs, nb < 1 or alignment.
 * lsq_absmax_expand: codes + params -> absmax fp32 [nb] (the values the fused
 *   GEMMs then read).  Same pointer rules.
 * The streaming scheduler runs the expansion itself after each upload when
 * given the record's layout (lsq_stream_set_absmax_expand).
 * ---------------------------------------------------------------------- */
lsq_status lsq_absmax_double_quantize(const float* absmax, int64_t nb, uint8_t* codes, float* params,
                                      lsq_cuda_stream stream);
lsq_status lsq_absmax_expand(const uint8_t* codes, const float* params, int64_t nb, float* absmax,
                             lsq_cuda_stream stream);

/* ------------------------------------------------------------------------
 * Fused NF4-dequant GEMM with LoRA, forward.
 *
 * Y = residual + X deq(W)^T + s (X A^T) B^T,   U = X A^T
 * The frozen-base linear with a LoRA adapter that layer streaming trains
 * (themenonlab blog, "The trick: layer streaming": the adapter is the only
 * trained part; soup-cli diff docs "Layer Streaming", lora.r / lora.alpha).
 * s = alpha / r.  The dequantised tile never reaches HBM: pairs of SMs decode
 * NF4 into shared memory and multiply on the tensor cores (tcgen05 with
 * cta_group::2, fp32 accumulation in TMEM).  U is computed first by a split-K
 * tensor-core kernel (kept in fp32 in u_out, and as s*U in bf16 in the
 * workspace); (s U) B^T then runs as one more contraction block of the main
 * GEMM, so Y is rounded to bf16 once.  Workspace bytes beyond the rank-r part
 * (lsq_nf4_lora_fwd_workspace_size includes them) let the GEMM share out its
 * last rounds of tiles (stream-K); results stay deterministic.
 *  x        device bf16 [M, k_in], 16-byte aligned
 *  A        device bf16 [r, k_in]   (LoRA down), NULL with r = 0 disables LoRA
 *  B        device bf16 [n_out, r]  (LoRA up)
 *  residual device bf16 [M, n_out] or NULL; may alias y
 *  y        device bf16 [M, n_out]
 *  u_out    device fp32 [M, r] or NULL (kept for the backward)
 *  workspace  device scratch of lsq_nf4_lora_fwd_workspace_size() bytes,
 *             256-byte aligned (may be NULL when r = 0); contents undefined
 *             after the call.  LSQ_EINVAL if missing or too small.
 * Limits: 1 <= M, 0 <= r <= 64.  Deterministic (no atomics, fixed order). */
size_t lsq_nf4_lora_fwd_workspace_size(int32_t nseg, int64_t M, int64_t k_in, const int64_t* n_out, int32_t r);
lsq_status lsq_nf4_lora_fwd(const lsq_nf4_weight* W, const void* x, int64_t M, const void* A, const void* B,
                            int32_t r, float s, const void* residual, void* y, float* u_out, void* workspace,
                            size_t workspace_bytes, lsq_cuda_stream stream);

/* Up to three linears that read the same x in one launch (q/k/v, gate/up);
 * segment i uses W[i], A[i], B[i], residual[i], y[i], u_out[i] exactly as
 * lsq_nf4_lora_fwd.  All W[i].k_in equal; r and s shared; the workspace size
 * is lsq_nf4_lora_fwd_workspace_size(nseg, ...) over the n_out of every segment. */
lsq_status lsq_nf4_lora_fwd_multi(int32_t nseg, const lsq_nf4_weight* W, const void* x, int64_t M,
                                  const void* const* A, const void* const* B, int32_t r, float s,
                                  const void* const* residual, void* const* y, float* const* u_out,
                                  void* workspace, size_t workspace_bytes, lsq_cuda_stream stream);

/* ------------------------------------------------------------------------
 * Backward of the fused linear (frozen W: no weight gradient).
 *
 * G = dY B;  dX = dY deq(W) + s G A;  dB (+)= s dY^T U;  dA (+)= s G^T X.
 * The gradients whose presence at the first layer the pages test (soup-cli
 * diff, CHANGELOG [0.72.2], "Correctness").  G comes from a split-K
 * tensor-core kernel; dX runs on SM pairs against the dequantised tile in
 * MN-major layout with (s G) A as one extra contraction block; dA and dB are
 * deterministic two-stage reductions over M (no atomics).
 *  x    device bf16 [M, k_in]   forward input
 *  dy   device bf16 [M, n_out]  upstream gradient
 *  u    device fp32 [M, r]      U from the forward
 *  dx   device bf16 [M, k_in] or NULL
 *  dA   device fp32 [r, k_in];  dB device fp32 [n_out, r]
 *  accumulate  0: overwrite dA/dB, 1: add into them
 *  workspace   device scratch of lsq_nf4_lora_bwd_workspace_size() bytes,
 *              256-byte aligned; contents undefined after the call.
 * With dx and r > 0 the dA / dB kernels run on a stream the library keeps
 * per host thread and device, concurrently with the dX GEMM, ordered by
 * events: everything enqueued on `stream` after the call sees dA and dB
 * (also under stream capture, which records the fork and join). */
size_t lsq_nf4_lora_bwd_workspace_size(int32_t nseg, int64_t M, int64_t k_in, const int64_t* n_out, int32_t r);
lsq_status lsq_nf4_lora_bwd(const lsq_nf4_weight* W, const void* x, const void* dy, int64_t M, const void* A,
                            const void* B, int32_t r, float s, const float* u, void* dx, float* dA, float* dB,
                            int32_t accumulate, void* workspace, size_t workspace_bytes,
                            lsq_cuda_stream stream);

/* Up to three linears that read the same x: dx = sum_i (dy[i] W[i] + s G[i] A[i]),
 * per-segment dA[i], dB[i].  dx may be NULL (gradients of the adapters only). */
lsq_status lsq_nf4_lora_bwd_multi(int32_t nseg, const lsq_nf4_weight* W, const void* x, const void* const* dy,
                                  int64_t M, const void* const* A, const void* const* B, int32_t r, float s,
                                  const float* const* u, void* dx, float* const* dA, float* const* dB,
                                  int32_t accumulate, void* workspace, size_t workspace_bytes,
                                  lsq_cuda_stream stream);

/* ------------------------------------------------------------------------
 * The fused linear with its rank-r operands kept between passes.
 *
 * Under gradient checkpointing each layer's forward runs twice, with the
 * same x, A and B (the pages' trainer recomputes the layer in the backward,
 * soup-cli docs "Layer Streaming"; the adapters change only at the optimizer
 * step).  The rank state of one call keeps what both passes and the backward
 * need from the rank-r side: s*U of each segment [M, 64] bf16 (zero-padded),
 * B of each segment padded to [n_out, 64], B^T [round16(r), n_out] and the
 * A^T of all segments side by side [k_in, 64].
 * lsq_nf4_lora_state_size: bytes of one call's state.
 * lsq_nf4_lora_fwd_multi_ex: as lsq_nf4_lora_fwd_multi, with
 *   state        device, 256-byte aligned, lsq_nf4_lora_state_size() bytes
 *                (may be NULL when r = 0)
 *   state_ready  0: compute the rank-r side (U into u_out, s*U, the padded
 *                and transposed operands into state); 1: the state already
 *                holds them from an earlier call with the same x, A, B, s and
 *                shapes (the recompute): only the main GEMM runs, and u_out
 *                is not written.  Y is bit-identical either way.
 *   workspace    optional scratch (NULL, or lsq_nf4_lora_fwd_workspace_size
 *                bytes, 256-byte aligned) that lets the GEMM balance its last
 *                rounds (stream-K)
 * lsq_nf4_lora_bwd_multi_ex: as lsq_nf4_lora_bwd_multi, reading s*U, B^T and
 *   A^T from that state instead of rebuilding them (u may then be NULL);
 *   results bit-identical to lsq_nf4_lora_bwd_multi. */
size_t lsq_nf4_lora_state_size(int32_t nseg, int64_t M, int64_t k_in, const int64_t* n_out, int32_t r);
lsq_status lsq_nf4_lora_fwd_multi_ex(int32_t nseg, const lsq_nf4_weight* W, const void* x, int64_t M,
                                     const void* const* A, const void* const* B, int32_t r, float s,
                                     const void* const* residual, void* const* y, float* const* u_out,
                                     void* state, int32_t state_ready, void* workspace, size_t workspace_bytes,
                                     lsq_cuda_stream stream);
lsq_status lsq_nf4_lora_bwd_multi_ex(int32_t nseg, const lsq_nf4_weight* W, const void* x, const void* const* dy,
                                     int64_t M, const void* const* A, const void* const* B, int32_t r, float s,
                                     const float* const* u, const void* state, void* dx, float* const* dA,
                                     float* const* dB, int32_t accumulate, void* workspace,
                                     size_t workspace_bytes, lsq_cuda_stream stream);

/* Rotate-half RoPE of some segments' outputs, applied in the fused GEMM's
 * epilogue (the decoder layer rotates q and k right after their projections;
 * Llama / Qwen stacks, soup-cli diff, docs "Layer Streaming", "Honest scope"):
 * rows of y are (sequence, position) with position = row % seq, heads of hd
 * columns; column i < hd/2 of a head pairs with column i + hd/2 and the pair
 * is rotated by the angle position * theta^(-2i/hd), in fp32 on the
 * accumulator, before the one bf16 rounding of the output.
 *  table:    lsq_rope_table's output for this seq and hd (device, 16-byte
 *            aligned); the epilogue takes the frequencies after the pairs and
 *            forms each angle as position x frequency in fp32, its cosine and
 *            sine with a two-part reduction by 2 pi and the special-function
 *            unit (error about 1e-6 of the rotated value, against 2^-8 for the
 *            bf16 rounding after it)
 *  seq, hd:  positions per sequence (M a multiple of seq); head dim 64, 128
 *            or 256
 *  segments: bit i set = rotate segment i (n_out a multiple of hd, no
 *            residual) */
typedef struct lsq_rope_spec {
  const float* table;
  int32_t seq, hd;
  int32_t segments;
} lsq_rope_spec;
/* cos and sin of position * theta^(-2i/hd) for positions 0..seq-1 and
 * i = 0..hd/2-1, computed in double and rounded to fp32 (the angles lsq_rope
 * uses), written as (cos, sin) pairs [seq][hd/2][2], followed by the hd/2
 * frequencies theta^(-2i/hd) in fp32: lsq_rope_table_size(seq, hd) bytes of
 * device memory.  hd even and <= 1024, theta > 1, seq >= 1, else EINVAL. */
size_t lsq_rope_table_size(int64_t seq, int64_t hd);
lsq_status lsq_rope_table(float theta, int64_t seq, int64_t hd, float* table, lsq_cuda_stream stream);
/* lsq_nf4_lora_fwd_multi_ex with the RoPE of the segments `rope` marks
 * (NULL or no bits: exactly lsq_nf4_lora_fwd_multi_ex); with state NULL,
 * lsq_nf4_lora_fwd_multi (the rank-r operands rebuilt in the workspace of
 * lsq_nf4_lora_fwd_workspace_size bytes) with that RoPE.  EINVAL for a bad
 * spec, before anything is enqueued. */
lsq_status lsq_nf4_lora_fwd_multi_ex2(int32_t nseg, const lsq_nf4_weight* W, const void* x, int64_t M,
                                      const void* const* A, const void* const* B, int32_t r, float s,
                                      const void* const* residual, void* const* y, float* const* u_out,
                                      void* state, int32_t state_ready, const lsq_rope_spec* rope,
                                      void* workspace, size_t workspace_bytes, lsq_cuda_stream stream);

/* Backward of one fused linear for callers that cannot allocate device
 * memory.  The paper has no counterpart (its trainer allocates through
 * PyTorch); this entry point exists for code that runs where a cudaMalloc is
 * unavailable or unsafe: inside a host framework that owns the whole device
 * pool and exposes no allocator, or in a process held to a hard memory cap
 * where an extra allocation mid-step could fail.
 * Same arguments and results as lsq_nf4_lora_bwd without the workspace: the
 * scratch (G, the padded LoRA operands, the partial sums and the dX GEMM's
 * stream-K partials) is one fixed array of
 * lsq_nf4_lora_bwd_noalloc_max_scratch() bytes (64 MiB) in the device memory
 * of every GPU that loads the library, held until the process exits.  Up to
 * the sizes of any one linear of the 8B shape at 2048 tokens and r = 16 the
 * call takes the plan lsq_nf4_lora_bwd takes with a workspace of
 * lsq_nf4_lora_bwd_workspace_size() bytes, bit for bit the same results;
 * beyond that, where the array has no room left for the stream-K partials,
 * the dX GEMM runs whole tiles and its fp32 sums may differ in the last bits.
 * A size whose scratch exceeds the array is rejected with LSQ_EINVAL before
 * anything is enqueued.  The first call on a device looks up the array's
 * device address (cudaGetSymbolAddress) with that device current, and the
 * first call on a host thread creates the library's per-thread side stream
 * and events and queries device attributes.  Every call shares the array
 * and leaves its last contents there; nothing in it needs to start at zero
 * (each call writes all the scratch it reads, and stream-K flags carry a
 * per-launch value).  Calls that overlap on the GPU (other streams or host
 * threads) race on the array: the caller must serialise them. */
size_t lsq_nf4_lora_bwd_noalloc_max_scratch(void);
lsq_status lsq_nf4_lora_bwd_noalloc(const lsq_nf4_weight* W, const void* x, const void* dy, int64_t M,
                                    const void* A, const void* B, int32_t r, float s, const float* u, void* dx,
                                    float* dA, float* dB, int32_t accumulate, lsq_cuda_stream stream);

/* ------------------------------------------------------------------------
 * Dense bf16 GEMM for the lm_head, which the pages keep on the GPU and
 * unquantised (soup-cli diff, docs "NF4 streaming").  tcgen05, fp32 accumulation.
 *  trans_b = 0:  out[M,N] = a[M,K] b[N,K]^T   (logits = h E^T)
 *  trans_b = 1:  out[M,N] = a[M,K] b[K,N]     (dh = dlogits E)
 *  out_f32 = 1: fp32 output, else bf16.  K % 8 == 0, N % 8 == 0. */
lsq_status lsq_dense_gemm(const void* a, const void* b, void* out, int64_t M, int64_t N, int64_t K,
                          int32_t trans_b, int32_t out_f32, lsq_cuda_stream stream);
/* The same GEMM on column blocks of wider row-major tensors, with a split
 * contraction: the lm_head streamed in vocabulary chunks (the pages plan the
 * untied embed_tokens and lm_head as streamed large layers, soup-cli diff,
 * docs "Layer Streaming", "NF4 streaming").
 *  a: rows of lda elements (lda >= K); out (and acc_in): rows of ldo elements
 *  (ldo >= N); lda, ldo multiples of 8.
 *  acc_in: NULL, or the fp32 accumulator [M, N] (row stride ldo, may alias an
 *  fp32 out) that earlier calls over the preceding K range left: the call
 *  continues the contraction from it.  With K ranges cut at multiples of 64 a
 *  chain of calls gives bit for bit what one call over the whole K gives
 *  (the accumulator enters the tensor memory exactly as it left it).
 * Other rules as lsq_dense_gemm; EINVAL before anything is enqueued. */
lsq_status lsq_dense_gemm_ex(const void* a, int64_t lda, const void* b, void* out, int64_t ldo, const float* acc_in,
                             int64_t M, int64_t N, int64_t K, int32_t trans_b, int32_t out_f32,
                             lsq_cuda_stream stream);

/* ------------------------------------------------------------------------
 * Decoder-layer kernels around the linears (Llama / Qwen, "Llama / Qwen
 * only", soup-cli diff docs "Layer Streaming", "Honest scope").  Activations
 * bf16, reductions fp32.  Row-major [rows, d] unless stated.
 * ---------------------------------------------------------------------- */
/* Shape and alignment rules of this section: device pointers; d (feature
 * count) and n (element count) multiples of 8 with bf16 operands 16-byte
 * aligned; anything else is EINVAL, with nothing enqueued. */
/* y = x / sqrt(mean(x^2) + eps) * g;  rstd[row] = 1/sqrt(mean(x^2)+eps) (fp32, may be NULL). */
lsq_status lsq_rmsnorm_fwd(const void* x, const void* g, void* y, float* rstd, int64_t rows, int64_t d, float eps,
                           lsq_cuda_stream stream);
/* dres_out = dres_in + d/dx of the norm given dy (g frozen); dres_in may be
 * NULL (treated as 0) or alias dres_out. */
lsq_status lsq_rmsnorm_bwd(const void* dy, const void* x, const void* g, const float* rstd, const void* dres_in,
                           void* dres_out, int64_t rows, int64_t d, lsq_cuda_stream stream);
/* In-place rotate-half RoPE on x viewed as [batch, seq, heads, hd] at
 * positions 0..seq-1; inverse = 1 applies the transpose (backward).  Angles
 * pos * theta^(-2i/hd) in double, rotation in fp32.  hd even and <= 1024,
 * theta > 1, else EINVAL; x 2-byte aligned (16-byte loads where hd % 16 == 0
 * and x is 16-byte aligned). */
lsq_status lsq_rope(void* x, int64_t batch, int64_t seq, int64_t heads, int64_t hd, float theta, int32_t inverse,
                    lsq_cuda_stream stream);
/* Causal GQA attention: q [B,S,Hq,hd], k,v [B,S,Hkv,hd] -> o [B,S,Hq,hd],
 * lse [B,Hq,S] fp32 (log-sum-exp of the scaled scores).  Scale 1/sqrt(hd).
 * Query head h reads kv head h / (Hq / Hkv).  hd 64 or 128 (else
 * EUNSUPPORTED); Hq % Hkv == 0, S <= 2^20, B*S*Hq <= 2^31 and every bf16
 * pointer 16-byte aligned (else EINVAL).  hd 128 with S <= 512 runs on the
 * tensor cores (tcgen05), other shapes on mma.sync kernels; both exact
 * softmax, no atomics. */
lsq_status lsq_attention_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int64_t batch,
                             int64_t seq, int64_t hq, int64_t hkv, int64_t hd, lsq_cuda_stream stream);
/* Gradients dq, dk, dv (bf16, same layouts) from do, given the forward's o
 * and lse; deterministic (each output written by one CTA, fixed summation
 * order).  Same limits as the forward; workspace:
 * lsq_attention_bwd_workspace_size() bytes, 16-byte aligned (per-row
 * statistics: D = rowsum(do * o) and, for head dim 128 up to 512 positions,
 * the log-sum-exp beside it); a smaller or misaligned workspace is EINVAL. */
size_t lsq_attention_bwd_workspace_size(int64_t batch, int64_t seq, int64_t hq);
lsq_status lsq_attention_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse,
                             const void* d_o, void* dq, void* dk, void* dv, int64_t batch, int64_t seq, int64_t hq,
                             int64_t hkv, int64_t hd, void* workspace, size_t workspace_bytes,
                             lsq_cuda_stream stream);
/* lsq_attention_bwd for q and k that the forward rotated with RoPE (the
 * q / k projections of lsq_nf4_lora_fwd_multi_ex2): with rope_table (from
 * lsq_rope_table for this seq and hd; NULL = plain lsq_attention_bwd), dq and
 * dk come out as the gradients of the unrotated q and k - the transpose of the
 * rotation applied to the fp32 gradient before its one bf16 rounding, with
 * the angles formed as in lsq_nf4_lora_fwd_multi_ex2 (head dim 128 up to 512
 * positions; other shapes rotate the bf16 gradients with the table's pairs
 * in a pass after the backward kernels).  rope_table 16-byte aligned. */
lsq_status lsq_attention_bwd_ex(const void* q, const void* k, const void* v, const void* o, const float* lse,
                                const void* d_o, void* dq, void* dk, void* dv, int64_t batch, int64_t seq, int64_t hq,
                                int64_t hkv, int64_t hd, const float* rope_table, void* workspace,
                                size_t workspace_bytes, lsq_cuda_stream stream);
/* m = silu(g) * u over n elements. */
lsq_status lsq_swiglu_fwd(const void* g, const void* u, void* m, int64_t n, lsq_cuda_stream stream);
/* dg, du from dm (dg/du may alias g/u: in-place). */
lsq_status lsq_swiglu_bwd(const void* dm, const void* g, const void* u, void* dg, void* du, int64_t n,
                          lsq_cuda_stream stream);
/* h[i, :] = table[ids[i], :], ids int32 device [rows]; table bf16 [vocab, d]
 * (device memory, or page-locked host memory mapped into the device address
 * space: the gather then reads the rows over the host link).  An id outside
 * [0, vocab) gives a zero row and records EINVAL in the device status word
 * (lsq_device_status). */
lsq_status lsq_embed_gather(const int32_t* ids, const void* table, void* h, int64_t rows, int64_t d,
                            int64_t vocab, lsq_cuda_stream stream);
/* Causal-LM cross entropy over logits fp32 [batch*seq, V]: target of row
 * (b, t) is ids[b, t+1] for t < seq-1; the last row of each sequence is
 * ignored.  loss (device fp32 scalar) = mean NLL over batch*(seq-1) rows;
 * dlogits bf16 [batch*seq, V] = (softmax - onehot) / (batch*(seq-1)), zero
 * on ignored rows.  workspace: lsq_xent_workspace_size() bytes. */
size_t lsq_xent_workspace_size(int64_t rows);
lsq_status lsq_xent_fwd_bwd(const float* logits, const int32_t* ids, int64_t batch, int64_t seq, int64_t V,
                            float* loss, void* dlogits, void* workspace, size_t workspace_bytes,
                            lsq_cuda_stream stream);
/* ------------------------------------------------------------------------
 * Preference loss (DPO) on the streamed base.  The pages serve preference
 * losses from the same streamed base, taking the base with the adapters
 * switched off as the reference model (aiany.app listing, "How It Works
 * (concise)"; soup-cli docs "Layer Streaming", preference losses v0.72.4).
 * They give no formula: the reading is DPO (Rafailov et al. 2023, eq. 7)
 * over pairs of sequences, chosen = row 2i, rejected = row 2i+1 of the batch,
 * with whole-sequence summed next-token log-probabilities.
 *
 * lsq_seq_logprob: seq_logp[b] = sum over t < seq-1 of log softmax(logits[b, t])[ids[b, t+1]];
 *   logits fp32 [batch*seq, V], ids int32 [batch*seq] (device); row_lse fp32
 *   [batch*seq] receives each row's log-sum-exp (for the backward); seq_logp
 *   fp32 [batch]; workspace lsq_seq_logprob_workspace_size(batch*seq) bytes.
 *   Fixed-order reductions (deterministic).
 * lsq_dpo_loss: z_i = beta ((pi[2i] - ref[2i]) - (pi[2i+1] - ref[2i+1])),
 *   loss (device fp32 scalar) = mean_i log(1 + exp(-z_i)); dseq fp32 [2 npairs]
 *   = d loss / d pi.  All pointers device memory.
 * lsq_seq_logprob_bwd: dlogits bf16 [batch*seq, V] = dseq[b] * (onehot(ids[b, t+1])
 *   - softmax(logits[b, t])), zero on each sequence's last row (the gradient of
 *   the loss through seq_logp). */
size_t lsq_seq_logprob_workspace_size(int64_t rows);
lsq_status lsq_seq_logprob(const float* logits, const int32_t* ids, int64_t batch, int64_t seq, int64_t V,
                           float* row_lse, float* seq_logp, void* workspace, size_t workspace_bytes,
                           lsq_cuda_stream stream);
lsq_status lsq_dpo_loss(const float* policy_logp, const float* ref_logp, int32_t npairs, float beta, float* loss,
                        float* dseq, lsq_cuda_stream stream);
lsq_status lsq_seq_logprob_bwd(const float* logits, const int32_t* ids, int64_t batch, int64_t seq, int64_t V,
                               const float* row_lse, const float* dseq, void* dlogits, lsq_cuda_stream stream);

/* AdamW on n fp32 masters p with grads g and moments m, v (all device fp32);
 * writes the bf16 operand copies p_bf16 (device, may be NULL).  step >= 1. */
lsq_status lsq_adamw_step(float* p, const float* g, float* m, float* v, void* p_bf16, int64_t n, int32_t step,
                          float lr, float beta1, float beta2, float eps, float weight_decay,
                          lsq_cuda_stream stream);
/* The bf16 operand copies p_bf16 of n fp32 masters p (device pointers), each
 * rounded to nearest even: the operand refresh that closes lsq_adamw_step,
 * alone, for the operands' first fill before any step.  fp32 masters with
 * bf16 operand copies are this library's reading of the optimizer step (the
 * pages name only PagedAdamW8bit, CHANGELOG [0.72.2] benchmark setup).
 * n >= 1, else EINVAL. */
lsq_status lsq_lora_refresh_bf16(const float* p, void* p_bf16, int64_t n, lsq_cuda_stream stream);

/* ------------------------------------------------------------------------
 * Layer streaming scheduler.
 *
 * The frozen base sits in host RAM and reaches the GPU one decoder layer at a
 * time through a pair of buffers allocated up front (soup-cli diff, CHANGELOG
 * [0.72.0]); `stream_buffers` 2..8, default 2 (docs "Layer Streaming");
 * page-locked RAM is what lets the copy overlap compute (docs "NF4
 * streaming", point 2); backward under gradient checkpointing re-streams the
 * layers in reverse.  The scheduler owns only CUDA events and bookkeeping;
 * the caller owns the slots (device), the records (host pinned) and both
 * streams.  Every layer record has the same size.
 * ---------------------------------------------------------------------- */
typedef struct lsq_stream lsq_stream;

/* Sharded upload (several GPUs, one process each, training data-parallel on
 * the same frozen base): rank r of W holds only bytes [r S, (r + 1) S) of
 * every record (S = record_bytes / W) in its page-locked store and copies
 * only those into the slot, at the same offset; the gather callback then
 * completes the slot from the other ranks (an all-gather over NVLink),
 * enqueued on `copy` after this rank's copy and before the upload's event.
 * Each GPU's host link carries 1/W of the bytes, and the node pins the store
 * once instead of once per rank.  The callback must return 0 on success; the
 * scheduler calls it for every upload, in the policy's order, which is the
 * same on every rank given the same sequence of steps. */
typedef int32_t (*lsq_gather_fn)(void* user, int32_t layer, int32_t slot, void* slot_ptr, size_t record_bytes,
                                 lsq_cuda_stream copy);

typedef struct lsq_stream_cfg {
  int32_t n_layers;                  /* >= 1 */
  int32_t n_slots;                   /* 2..8 (or n_layers for a resident run) */
  size_t record_bytes;               /* bytes per layer record, > 0, a multiple of 256 x max(1, shard_world) */
  void* const* slots;                /* n_slots device pointers, 256-byte aligned, >= record_bytes each */
  const void* const* host_records;   /* n_layers host pointers, page-locked; with sharding each points
                                        at this rank's record_bytes / shard_world bytes; NULL with disk_path */
  int32_t shard_rank;                /* sharded upload: this rank, 0 <= shard_rank < shard_world */
  int32_t shard_world;               /* ranks sharing each record; record_bytes % (256 shard_world) == 0 */
  lsq_gather_fn gather;              /* NULL: no sharding (shard_rank 0, shard_world 0 or 1) */
  void* gather_user;                 /* passed to gather */
  /* Disk tier (host_records NULL): the parts are read from the file at
   * disk_path, which holds n_layers parts of record_bytes / max(1, shard_world)
   * bytes back to back (this rank's parts), by disk_threads host threads into
   * n_staging page-locked staging buffers of one part each, in upload order;
   * the copy stream waits for each part (host function, bounded) before its
   * copy.  A failed read or a wait that runs out makes the next scheduler call
   * return EINVAL / ETIMEOUT. */
  const char* disk_path;             /* NULL: records come from host_records */
  void* const* staging;              /* n_staging host pointers, page-locked */
  int32_t n_staging;                 /* 2..8 */
  int32_t disk_threads;              /* 1..16 reader threads (each reads one slice of every part) */
} lsq_stream_cfg;

/* Creates the scheduler; ENOTPINNED if any record is not page-locked (the
 * pages fall back to pageable memory silently; here it is an error).  Upload
 * calls that run the gather callback return ECALLBACK if it fails (the slot
 * is then incomplete: destroy the scheduler).  The first upload into each slot
 * is ordered after all work queued on the compute stream when the scheduler
 * is created (a caching allocator may hand out slot memory whose previous
 * owner's kernels are still queued there). */
lsq_status lsq_stream_create(const lsq_stream_cfg* cfg, lsq_cuda_stream compute, lsq_cuda_stream copy,
                             lsq_stream** out);
/* Enqueue on the copy stream: wait until the compute stream is done with the
 * slot's previous occupant, copy layer's record into the slot, record the
 * layer's upload event.  ESTATE if the slot holds the layer in current use. */
lsq_status lsq_layer_upload_async(lsq_stream* st, int32_t layer, int32_t slot);
/* One double-quantised absmax array of a layer record: byte offsets from the
 * slot's start of its codes (u8 [nb]) and params (fp32 pairs, 8-byte
 * aligned), both inside the record, and of the fp32 [nb] output, which lies
 * past the record's end and within the slot (4-byte aligned). */
typedef struct lsq_absmax_dq_item {
  uint64_t codes_off;
  uint64_t params_off;
  uint64_t out_off;
  int64_t nb;
} lsq_absmax_dq_item;
/* Records carry double-quantised absmax: after every upload the scheduler
 * expands the n_items (0..8; 0 switches it off) arrays into fp32 inside the
 * slot, on the copy stream, before the upload's event - compute sees the
 * layer only once its fp32 absmax is in place.  slot_bytes: the size of every
 * slot (the caller's allocations; >= the largest out_off + 4 nb).  Call before
 * the first upload (ESTATE otherwise); EINVAL on bounds, alignment or
 * overlapping outputs. */
lsq_status lsq_stream_set_absmax_expand(lsq_stream* st, const lsq_absmax_dq_item* items, int32_t n_items,
                                        size_t slot_bytes);
/* Begin compute on `layer`, walking in `direction` (+1 forward, -1
 * backward): release the previously stepped layer's slot after the compute
 * work enqueued so far; upload `layer` if no slot holds it; make the compute
 * stream wait for its upload; prefetch layer + direction into the least
 * recently used other slots (up to n_slots - 1 layers ahead, never evicting
 * the layer in use or one already inside that window).  *slot_ptr = device
 * address of the record. */
lsq_status lsq_stream_step(lsq_stream* st, int32_t layer, int32_t direction, void** slot_ptr);
/* The scheduler's slot policy without CUDA (for tests and planning): runs the
 * same decisions lsq_stream_step makes for the n_steps (layers[i],
 * directions[i]) calls and writes each action as three int32 (kind, layer,
 * slot) into `actions` (host, 3 * max_actions ints): kind 1 = release the
 * slot once the compute enqueued so far is done, 2 = upload the layer into
 * the slot (after that release), 3 = compute waits for the layer's upload.
 * *n_actions = the number written; EINVAL if more than max_actions. */
lsq_status lsq_stream_simulate(int32_t n_layers, int32_t n_slots, int32_t n_steps, const int32_t* layers,
                               const int32_t* directions, int32_t* actions, int32_t max_actions,
                               int32_t* n_actions);
/* Counters since create: uploads issued, bytes copied, uploads skipped
 * because the layer was still resident. */
lsq_status lsq_stream_stats(const lsq_stream* st, int64_t* uploads, int64_t* bytes, int64_t* reused);
/* Device time (ms) of the last completed upload of `layer` (event pair on the
 * copy stream); synchronises on that upload. */
lsq_status lsq_stream_upload_ms(lsq_stream* st, int32_t layer, float* ms);
/* Exposed-copy timing (the measure of copy time that compute could not hide):
 * with capacity > 0, each compute-stream wait on an upload that
 * lsq_stream_step enqueues is bracketed by two timing events recorded on the
 * compute stream, before and after the wait, so the time between them is how
 * long compute stood still for that layer's copy (the pages judge streaming by
 * how long compute waits on copies, README "Citing Soup", measured share of
 * the step).  Up to `capacity` waits are kept between two lsq_stream_wait_ms
 * calls; later ones are counted as dropped.  capacity 0 turns it off.  Waits
 * for the compute stream before it replaces the events.  capacity 0..2^20. */
lsq_status lsq_stream_time_waits(lsq_stream* st, int32_t capacity);
/* The summed time (ms) of the kept waits since the previous call, split by
 * the walking direction of the step that enqueued them (+1: fwd_ms, -1:
 * bwd_ms), their number and the number dropped; waits for those events and
 * starts a new count.  ESTATE when timing is off. */
lsq_status lsq_stream_wait_ms(lsq_stream* st, float* fwd_ms, float* bwd_ms, int32_t* n_waits, int32_t* n_dropped);
/* Forget all residency (next step re-uploads); waits for pending copies.
 * ESTATE while a capture is open. */
lsq_status lsq_stream_reset(lsq_stream* st);
/* Recording one training step as a CUDA graph (stream capture), so that a
 * step's several hundred kernels are launched from device memory: eager
 * launches fetch their commands over the host link, which the layer copies
 * keep busy, and measured on B200 they slow down by up to half under that
 * load, while graph launches do not.
 *
 * lsq_stream_capture_begin, called after the caller began a capture on the
 * compute stream (cudaStreamBeginCapture), brings the copy stream into that
 * capture; lsq_stream_step then records its uploads, releases and waits into
 * the graph instead of running them, and lsq_stream_capture_end, called
 * before the capture ends, joins the copy stream back.  Inside the capture,
 * a wait on a release or an upload recorded before it is left out: the graph
 * starts after the compute stream's earlier work, and the caller makes the
 * compute stream wait for the copy stream's earlier work before each launch
 * of the graph.
 *
 * The captured step has not run: the policy's host state has advanced as if
 * it had, so launch the graph once before any other use of the scheduler.
 * Replaying it is only right when the step leaves the slot map (the layer
 * each slot holds, their LRU order, the current layer) as it found it, which
 * holds from the second step of a fixed 0 -> L-1 -> 0 walk on; capture_end
 * checks this and returns ESTATE otherwise.  Events recorded in the capture
 * are recorded again on the compute stream at the next eager use of the
 * scheduler (lsq_stream_upload_ms then returns ESTATE for those layers until
 * an eager step uploads them again).  Counters (lsq_stream_stats) advance at
 * capture, not at replay.
 *
 * capture_begin: EINVAL with the disk tier, sharded uploads or wait timing
 * on (they do host work in each step); ESTATE if the compute stream is not
 * capturing or a capture is open.  capture_end: ESTATE if none is open or
 * the slot map changed. */
lsq_status lsq_stream_capture_begin(lsq_stream* st);
lsq_status lsq_stream_capture_end(lsq_stream* st);
lsq_status lsq_stream_destroy(lsq_stream* st);

#ifdef __cplusplus
}
#endif
#endif /* LSQ_H_ */
