/*
 * jattn -- joint (text + image + reference) DiT attention forward for NVIDIA
 * B200 (sm_100a), BF16 and FP8 paths.
 *
 * The operation ("Speed Up Image Generation with FLUX 3 Image Klein on NVIDIA
 * Blackwell GPUs"):
 *   - section "FLUX 3 inference with TensorRT LLM VisualGen": the text, noisy
 *     target-image and optional reference-image token streams are combined
 *     through joint attention, i.e. one attention over their concatenation;
 *   - section "GEMM kernel optimization": rotary position embeddings (RoPE)
 *     are applied to the query and key projections;
 *   - section "Quantized and sparse attention": dense BF16 attention and FP8
 *     attention with FP8 query/key and FP8 value (qk_dtype / v_dtype fp8).
 * Readings where the page is silent: joint order txt | img | ref with no mask;
 * 2D axial RoPE over (t, row, col) with per-axis channel spans split[3]
 * (in that order), interleaved pairs (2p, 2p+1) inside a span of n channels
 * rotated by pos_axis * theta^(-2p/n); softmax scale 1/sqrt(d); FP8 = e4m3
 * with one fp32 scale per (batch, head, 128-token block).
 *
 * Conventions for every entry point:
 *   - All tensor pointers are DEVICE pointers, 16-byte aligned, row-major and
 *     contiguous in the layout stated.  The caller allocates and owns every
 *     buffer; the library allocates nothing and keeps no pointer after the
 *     call returns.
 *   - Work is enqueued on `stream` (a cudaStream_t; NULL = legacy default
 *     stream) and the call returns without synchronising.  The host does no
 *     device synchronisation and no allocation, so the calls can be captured
 *     into a CUDA graph.
 *   - Argument errors are reported synchronously, before anything is
 *     launched: JATTN_ERR_INVALID_ARG (null or inconsistent arguments),
 *     JATTN_ERR_UNSUPPORTED (d not 64 or 128, dtype not allowed here),
 *     JATTN_ERR_ALIGNMENT (a pointer not 16-byte aligned).  A failed launch
 *     returns JATTN_ERR_CUDA.
 *   - Errors found on the device (a pipeline wait that ran out of time, a
 *     value out of the 16-bit output range) are recorded in a per-device
 *     status word; read it with jattn_last_device_status() (or
 *     jattn_device_status(), which can also clear it).  No kernel traps.
 *   - No C++ exception crosses this interface.
 */
#ifndef JATTN_H_
#define JATTN_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  JATTN_OK = 0,
  JATTN_ERR_INVALID_ARG = 1,
  JATTN_ERR_UNSUPPORTED = 2,
  JATTN_ERR_ALIGNMENT = 3,
  JATTN_ERR_CUDA = 4,
  JATTN_ERR_TIMEOUT = 5, /* a kernel gave up waiting; see jattn_device_status */
  JATTN_ERR_RANGE = 6,   /* a value exceeded the 16-bit output range (saturated) */
  JATTN_ERR_INTERNAL = 7 /* a kernel's internal consistency check failed */
} jattn_status;

/* Bits of the device status word. */
#define JATTN_DEV_TIMEOUT 1u
#define JATTN_DEV_RANGE 2u
#define JATTN_DEV_CHECK 4u

typedef enum { JATTN_BF16 = 0, JATTN_FP16 = 1, JATTN_E4M3 = 2 } jattn_dtype;

/* Problem shape.  S = S_txt + S_img + S_ref in [1, 2^24], each part >= 0;
 * B, H >= 1 with B * H <= 65535 and ceil(S / 256) * B * H < 2^31; d in
 * {64, 128} (JATTN_ERR_UNSUPPORTED otherwise, JATTN_ERR_INVALID_ARG for the
 * other limits). */
typedef struct {
  int32_t B, H, S_txt, S_img, S_ref, d;
} jattn_shape;

/* Tokens per FP8 scale block (and per attention tile). */
#define JATTN_BLOCK 128

/*
 * Joint-sequence assembly + 2D axial RoPE on Q and K (+ optional per-block
 * e4m3 quantisation), one pass over the inputs.
 *
 *   qkv_txt, qkv_img, qkv_ref : bf16 [B, S_part, 3, H, d] (index 0 = Q,
 *       1 = K, 2 = V) -- the output of each stream's QKV projection.  A part
 *       with S_part == 0 may be NULL.
 *   pos    : int32 [S, 3], (t, row, col) of every joint token in the order
 *            txt | img | ref, shared by all batch entries.
 *   theta  : RoPE base (> 0), e.g. 10000.
 *   split  : host array of 3 even, non-negative channel counts for the t, row
 *            and col axes, summing to d.
 *   out_dtype:
 *     JATTN_FP16 / JATTN_BF16 : q, k, v are [B, H, S, d] in that type; q and
 *        k rotated, v converted.  scales is ignored (may be NULL).  FP16
 *        values beyond +-65504 are saturated and JATTN_DEV_RANGE is recorded.
 *     JATTN_E4M3 : q, k, v are e4m3 [B, H, S, d]; scales is fp32
 *        [3][B][H][ceil(S/128)] (Q, K, V), scale = amax/448 of the block's
 *        fp32 values (1 for an all-zero block), code = RNE-satfinite
 *        e4m3(x * (448/amax)).
 */
jattn_status jattn_rope_qkv(const jattn_shape* shape, const void* qkv_txt, const void* qkv_img,
                            const void* qkv_ref, const int32_t* pos, float theta,
                            const int32_t split[3], jattn_dtype out_dtype, void* q, void* k,
                            void* v, float* scales, void* stream);

/*
 * As jattn_rope_qkv, with query/key normalisation fused in front of the
 * rotation ("Speed Up Image Generation with FLUX 3 Image Klein on NVIDIA
 * Blackwell GPUs", section "GEMM kernel optimization": the fused QKV
 * projection applies query/key normalisation and RoPE).  The page does not
 * spell the normalisation out; it is taken as RMSNorm over the d channels of
 * one (token, head), before the rotation:
 *   x -> w[stream][Q or K][c] * x_c / sqrt(mean_c(x_c^2) + eps)
 * computed in fp32 (sum of squares, then a correctly rounded 1/sqrt).
 *   norm_w : device fp32 [3][2][d]: stream (0 = txt, 1 = img, 2 = ref), then
 *            0 = Q, 1 = K.  Pass the same values twice to share weights
 *            between streams.  Must not be NULL; 16-byte aligned.
 *   eps    : > 0 and finite (1e-6 in the FLUX family); else
 *            JATTN_ERR_INVALID_ARG.
 * V is not normalised.  All other arguments, layouts and errors as
 * jattn_rope_qkv; with out_dtype JATTN_E4M3 the block scales are those of
 * the normalised, rotated values.
 */
jattn_status jattn_rope_qkv_norm(const jattn_shape* shape, const void* qkv_txt, const void* qkv_img,
                                 const void* qkv_ref, const int32_t* pos, float theta,
                                 const int32_t split[3], const float* norm_w, float eps,
                                 jattn_dtype out_dtype, void* q, void* k, void* v, float* scales,
                                 void* stream);

/*
 * Per-block e4m3 quantisation of one laid-out 16-bit tensor.
 *   x      : in_dtype (JATTN_BF16 or JATTN_FP16) [B, H, S, d]
 *   x8     : e4m3 [B, H, S, d]
 *   scales : fp32 [B][H][ceil(S/128)], same arithmetic as jattn_rope_qkv.
 * Only shape->B, H, d and S = S_txt + S_img + S_ref are used.
 */
jattn_status jattn_quant_fp8(const jattn_shape* shape, jattn_dtype in_dtype, const void* x,
                             void* x8, float* scales, void* stream);

/*
 * Attention forward, 16-bit operands: O = softmax(Q K^T * softmax_scale) V
 * over the whole joint sequence (no mask), FP32 accumulation in tensor
 * memory, online softmax.
 *   q, k, v : in_dtype (JATTN_FP16 or JATTN_BF16) [B, H, S, d], as written by
 *             jattn_rope_qkv.
 *   o       : bf16 [B, S, H, d] (token-major, ready for the output
 *             projection).  16-byte alignment is required; a 32-byte
 *             aligned o is written with 256-bit stores (fewer store requests,
 *             same bits).
 *   lse     : fp32 [B, H, S] natural-log sum-exp of the scaled logits, or NULL.
 *   softmax_scale <= 0 selects 1/sqrt(d).
 */
jattn_status jattn_fwd_bf16(const jattn_shape* shape, jattn_dtype in_dtype, const void* q,
                            const void* k, const void* v, void* o, float* lse,
                            float softmax_scale, void* stream);

/*
 * Attention forward, e4m3 operands with per-(b, h, 128-token block) scales:
 * logits = (q8 . k8) * s_q * s_k, probabilities rounded to e4m3 for the P.V
 * product, V dequantised by s_v.
 *   q8, k8, v8 : e4m3 [B, H, S, d] (jattn_rope_qkv with JATTN_E4M3)
 *   scales     : fp32 [3][B][H][ceil(S/128)]
 *   o, lse, softmax_scale : as jattn_fwd_bf16.
 */
jattn_status jattn_fwd_fp8(const jattn_shape* shape, const void* q8, const void* k8,
                           const void* v8, const float* scales, void* o, float* lse,
                           float softmax_scale, void* stream);

/*
 * High-precision 16-bit path: the BF16 path of jattn_rope_qkv(_norm) +
 * jattn_fwd_bf16, computed so that it stays within the BF16 path's error
 * bars (rel-L2 5e-3, max-abs 2e-2 against the exact result) also when a few
 * channels of a head carry activation outliers, and with no saturation.
 * ("Speed Up Image Generation with FLUX 3 Image Klein on NVIDIA Blackwell
 * GPUs", section "Quantized and sparse attention": dense BF16 attention is
 * the accuracy reference of the quantised variants.)  Two differences from
 * the plain fp16-operand path:
 *   - range: every (Q|K|V, batch, head, 128-token block) tile is stored as
 *     fp16(x * 2^-e), e >= 0 the smallest exponent that keeps the tile
 *     within +-65504 (0 for all ordinary inputs); the scales 2^e are folded
 *     into the softmax exactly like the e4m3 block scales;
 *   - precision: fp16 rounding of the rotated Q / K costs each logit an
 *     error proportional to |q_pair| |k_pair| summed over channel pairs; per
 *     (batch, head) the 4 pairs with the largest max|q_pair| * max|k_pair|
 *     (ties to the lower pair) get their rounding residual back: correction
 *     rows qc = [hi | lo] and kc = [lo | hi] of those 8 channels (hi the
 *     stored fp16 value, lo = fp16(x - hi)) add hi_q lo_k + lo_q hi_k to
 *     every logit through one more 16-deep MMA.
 *
 * jattn_rope_qkv_hp: the prologue (assembly, optional query/key RMSNorm as
 * jattn_rope_qkv_norm -- norm_w may be NULL for none --, RoPE) and the
 * correction rows, three launches on `stream`.
 *   qkv_*, pos, theta, split, norm_w, eps : as jattn_rope_qkv_norm.
 *   q, k, v    : fp16 [B, H, S, d], the scaled values fp16(x * 2^-e).
 *   scales     : fp32 [3][B][H][ceil(S/128)], the powers of two 2^e (Q, K, V).
 *   qc, kc     : fp16 [B, H, S, 16], the correction rows.
 *   workspace  : device scratch of at least jattn_rope_qkv_hp_workspace(shape)
 *                bytes, 256-byte aligned, owned by the caller (per-block
 *                pair statistics, the selection, RMSNorm row factors).
 * jattn_fwd_bf16_hp: the forward on those operands; o, lse, softmax_scale as
 * jattn_fwd_bf16.
 * Errors: as jattn_rope_qkv / jattn_fwd_bf16; JATTN_ERR_INVALID_ARG for a
 * NULL scales, qc, kc or workspace, or a workspace that is too small;
 * JATTN_ERR_ALIGNMENT for a workspace not 256-byte aligned.
 */
size_t jattn_rope_qkv_hp_workspace(const jattn_shape* shape);   /* 0 on invalid arguments */
jattn_status jattn_rope_qkv_hp(const jattn_shape* shape, const void* qkv_txt, const void* qkv_img,
                               const void* qkv_ref, const int32_t* pos, float theta,
                               const int32_t split[3], const float* norm_w, float eps, void* q, void* k,
                               void* v, float* scales, void* qc, void* kc, void* workspace,
                               size_t workspace_bytes, void* stream);
jattn_status jattn_fwd_bf16_hp(const jattn_shape* shape, const void* q, const void* k, const void* v,
                               const float* scales, const void* qc, const void* kc, void* o, float* lse,
                               float softmax_scale, void* stream);

/*
 * Block-sparse attention forward, 16-bit operands ("Speed Up Image Generation
 * with FLUX 3 Image Klein on NVIDIA Blackwell GPUs", sections "Quantized and
 * sparse attention" and "Optimized single-GPU deployment": Sol-Attention, a
 * block-sparse attention whose sparsity tau controls -- higher tau drops
 * more blocks -- run dense until a noise-level cutoff, which is the caller's
 * choice of tau = 0 for those steps).  The page names no selection rule;
 * this library reads it as:
 *   - queries in blocks of 256 joint tokens, keys in blocks of 128 (the last
 *     block of each may be shorter), each block represented by the mean of
 *     its rotated rows;
 *   - the estimated attention share of key block J for query block I is the
 *     softmax over J of qbar_I . kbar_J * softmax_scale;
 *   - J is kept iff its share >= tau / n_kb (n_kb = ceil(S/128): tau times a
 *     uniform share), and the largest share is always kept (ties to the
 *     lower J); tau = 0 keeps everything (the dense result);
 *   - every query row attends, with an exact softmax, to the keys of its
 *     block's kept key blocks only.
 * Three launches on `stream`: block means, selection, the forward walking
 * the kept key tiles.
 *   q, k, v, in_dtype, o, lse, softmax_scale : as jattn_fwd_bf16.
 *   tau        : >= 0 and finite, else JATTN_ERR_INVALID_ARG.
 *   workspace  : device scratch of at least
 *                jattn_fwd_block_sparse_workspace(shape) bytes, 256-byte
 *                aligned, owned by the caller.
 *   kv_list    : NULL, or int32 [B][H][ceil(S/256)][ceil(S/128)]: row (b, h,
 *                I) receives the kept key blocks of query block I in
 *                ascending order (the entries past its count are undefined);
 *   kv_count   : NULL, or int32 [B][H][ceil(S/256)]: how many.
 * Errors: as jattn_fwd_bf16; JATTN_ERR_INVALID_ARG for a NULL or too small
 * workspace; JATTN_ERR_ALIGNMENT for a workspace not 256-byte aligned.
 */
size_t jattn_fwd_block_sparse_workspace(const jattn_shape* shape);   /* 0 on invalid arguments */
jattn_status jattn_fwd_block_sparse(const jattn_shape* shape, jattn_dtype in_dtype, const void* q, const void* k,
                                    const void* v, float tau, void* workspace, size_t workspace_bytes, void* o,
                                    float* lse, int32_t* kv_list, int32_t* kv_count, float softmax_scale,
                                    void* stream);

/*
 * FP8 attention with token repair ("Speed Up Image Generation with FLUX 3
 * Image Klein on NVIDIA Blackwell GPUs", section "Quantized and sparse
 * attention": a repair budget rho -- 0.005 in the tested configuration --
 * selects the fraction of tokens with the highest quantisation error for a
 * residual correction).  The page names neither the error measure nor the
 * correction; this library reads them as:
 *   - per (batch, head), n = min(S, ceil(rho * S - 1e-3)) tokens (rho as
 *     passed, a float; see jattn_repair_count) are repaired;
 *   - a token's quantisation error is the e4m3 error bound of its key and
 *     value rows, which grows with their magnitude: the n largest
 *     |k_j|^2 + |v_j|^2 (fp32, rotated / normalised key before quantisation)
 *     are taken, ties to the lower token index;
 *   - a repaired token enters the attention with its exact key and value and
 *     the logit of the 16-bit (fp16) query and key; every other token with
 *     the e4m3 operands.  One softmax over all S keys.
 * The whole path in one call, on `stream`:
 *   prologue (as jattn_rope_qkv_norm / jattn_rope_qkv with JATTN_E4M3, plus
 *   fp16 Q and the scores) -> selection -> exact fp16 keys / values of the
 *   selected tokens -> fp16 attention over the selected keys (a partial o
 *   and log-sum-exp) -> FP8 attention over the other keys, merged into that
 *   partial result through the two partial log-sum-exps.
 *   qkv_*, pos, theta, split : as jattn_rope_qkv.
 *   norm_w, eps : query/key RMSNorm as jattn_rope_qkv_norm, or norm_w = NULL.
 *   rho        : 0 <= rho <= 1 (0: plain FP8 path, nothing repaired).
 *   workspace  : device scratch of at least
 *                jattn_fwd_fp8_repair_workspace(shape, rho) bytes, 256-byte
 *                aligned, owned by the caller; contents undefined afterwards.
 *   o, lse, softmax_scale : as jattn_fwd_fp8.
 *   repaired   : NULL, or int32 [B][H][n]: the repaired token indices (in
 *                index order) are written there.
 * Errors: as jattn_rope_qkv and jattn_fwd_fp8; JATTN_ERR_INVALID_ARG for rho
 * outside [0, 1], a NULL or too small workspace; JATTN_ERR_ALIGNMENT for a
 * workspace not 256-byte aligned.
 */
int32_t jattn_repair_count(const jattn_shape* shape, float rho);   /* n; -1 on invalid arguments */
size_t jattn_fwd_fp8_repair_workspace(const jattn_shape* shape, float rho);   /* 0 on invalid arguments */
jattn_status jattn_fwd_fp8_repair(const jattn_shape* shape, const void* qkv_txt, const void* qkv_img,
                                  const void* qkv_ref, const int32_t* pos, float theta,
                                  const int32_t split[3], const float* norm_w, float eps, float rho,
                                  void* workspace, size_t workspace_bytes, void* o, float* lse,
                                  int32_t* repaired, float softmax_scale, void* stream);

/*
 * jattn_fwd_fp8_repair for callers that cannot allocate device memory.  (No
 * counterpart on the page: this is an interface for integrators.)  Some
 * callers may not call cudaMalloc at all: a plug-in whose host framework owns
 * every device allocation, code running inside a stream capture whose memory
 * policy forbids allocation, or a latency-bound loop that must not block on
 * the allocator.  They pass inputs and outputs as usual; the scratch the path
 * needs is a file-scope device array of JATTN_NOALLOC_SCRATCH_BYTES inside
 * the library.
 *   Memory: with the CUDA runtime's default lazy module loading the array is
 *   reserved on a device when a process first calls this function there;
 *   with CUDA_MODULE_LOADING=EAGER every process that loads the library
 *   reserves it on each device when its context is created.  The device holds
 *   it until the process exits.  The path itself allocates nothing.
 *   Set-up: the array's device address is looked up on the first call on a
 *   device (make that call before any stream capture) and looked up again if
 *   the device's context changed (after a cudaDeviceReset).
 *   Arguments: as jattn_fwd_fp8_repair without workspace / workspace_bytes.
 *   Errors: as jattn_fwd_fp8_repair; JATTN_ERR_UNSUPPORTED when
 *   jattn_fwd_fp8_repair_workspace(shape, rho) exceeds the array (checked
 *   before anything is launched), JATTN_ERR_CUDA if the array's address
 *   cannot be looked up.
 *   Calls on one device share the array and overwrite what the last call
 *   left there: calls that overlap on the GPU race (use one stream per
 *   device, or serialise them).
 */
#define JATTN_NOALLOC_SCRATCH_BYTES ((size_t)640 << 20)
jattn_status jattn_fwd_fp8_repair_noalloc(const jattn_shape* shape, const void* qkv_txt, const void* qkv_img,
                                          const void* qkv_ref, const int32_t* pos, float theta,
                                          const int32_t split[3], const float* norm_w, float eps, float rho,
                                          void* o, float* lse, int32_t* repaired, float softmax_scale,
                                          void* stream);

/*
 * The whole path on HOST buffers, for callers whose inputs and outputs live
 * in host memory: copies in, then per chunk the high-precision 16-bit pair
 * jattn_rope_qkv_hp + jattn_fwd_bf16_hp (path JATTN_FP16), jattn_rope_qkv +
 * jattn_fwd_bf16 with bf16 operands (path JATTN_BF16) or jattn_rope_qkv +
 * jattn_fwd_fp8 (path JATTN_E4M3), copy of O out.  The work is pipelined
 * over (batch entry, head group) chunks: the copies of one chunk overlap the
 * kernels of another, on two copy streams the library creates once per host
 * thread and device.  The call is
 * ordered like one operation on `stream`: it starts after the work already
 * enqueued there, and `stream` completes only after O is in host memory.
 *   qkv_*, pos : HOST pointers, layouts as jattn_rope_qkv.  Page-locked
 *                (pinned) memory lets the copies overlap the kernels;
 *                pageable memory works but serialises them.
 *   o          : HOST pointer, bf16 [B, S, H, d].
 *   workspace  : DEVICE scratch of jattn_joint_attention_host_workspace()
 *                bytes, 256-byte aligned, owned by the caller.
 * Errors: as the device entry points, checked before anything is enqueued;
 * JATTN_ERR_INVALID_ARG for a NULL or too small workspace.
 */
size_t jattn_joint_attention_host_workspace(const jattn_shape* shape, jattn_dtype path);   /* 0 if invalid */
jattn_status jattn_joint_attention_host(const jattn_shape* shape, const void* qkv_txt, const void* qkv_img,
                                        const void* qkv_ref, const int32_t* pos, float theta,
                                        const int32_t split[3], jattn_dtype path, void* o, float softmax_scale,
                                        void* workspace, size_t workspace_bytes, void* stream);

/*
 * The boundary's status query: wait for the work enqueued on `stream` so far,
 * then return what the current device's status word records (JATTN_OK,
 * JATTN_ERR_INTERNAL, JATTN_ERR_TIMEOUT or JATTN_ERR_RANGE, in that order of
 * precedence) without clearing it.  JATTN_ERR_CUDA if the stream or the word
 * cannot be read.  The word is per device: kernels of every stream and thread
 * on the device record into it.
 */
jattn_status jattn_last_device_status(void* stream);

/*
 * Synchronise `stream`, read the current device's status word and return
 * JATTN_OK, JATTN_ERR_INTERNAL, JATTN_ERR_TIMEOUT or JATTN_ERR_RANGE (in
 * that order of precedence).  The raw
 * bits go to *bits if bits is non-NULL.  clear != 0 resets the word.
 */
jattn_status jattn_device_status(void* stream, int clear, uint32_t* bits);

/*
 * Self-test of the bounded waits: one CTA waits on an mbarrier that nothing
 * arrives on, with a limit of `limit_ms` milliseconds, then records
 * JATTN_DEV_TIMEOUT and returns.  Used by the failure-detection tests.
 */
jattn_status jattn_selftest_wait_timeout(int32_t limit_ms, void* stream);

/* Static description of a status code. */
const char* jattn_status_string(jattn_status s);

/* Library version, "major.minor.patch". */
const char* jattn_version(void);

#ifdef __cplusplus
}
#endif

#endif /* JATTN_H_ */
